// Tile kernels for one format set: E3M2 element codes (MXFP6), E8M0 group scales, E8M0 outer scales.
#include "dq_launch.h"

namespace dq {
cudaError_t launch_tile_c10(const TileLaunch &L) { return launch_tile_combo<CODES_E3M2, SC_E8M0, SC_E8M0>(L); }
}  // namespace dq
