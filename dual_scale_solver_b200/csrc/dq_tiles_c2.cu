// Tile kernels for one format set: E2M1 codes, E8M0 group scales, E8M0 outer scales (MXFP4).
#include "dq_launch.h"

namespace dq {
cudaError_t launch_tile_c2(const TileLaunch &L) { return launch_tile_combo<CODES_E2M1, SC_E8M0, SC_E8M0>(L); }
}  // namespace dq
