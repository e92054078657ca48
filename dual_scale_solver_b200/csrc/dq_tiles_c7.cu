// Tile kernels for one format set: E4M3 element codes (MXFP8), E8M0 group scales, E8M0 outer scales.
#include "dq_launch.h"

namespace dq {
cudaError_t launch_tile_c7(const TileLaunch &L) { return launch_tile_combo<CODES_E4M3, SC_E8M0, SC_E8M0>(L); }
}  // namespace dq
