// Tile kernels for one format set: E2M1 codes, E4M3 group scales, BF16 outer scales (NVFP4).
#include "dq_launch.h"

namespace dq {
cudaError_t launch_tile_c3(const TileLaunch &L) { return launch_tile_combo<CODES_E2M1, SC_E4M3, SC_BF16>(L); }
}  // namespace dq
