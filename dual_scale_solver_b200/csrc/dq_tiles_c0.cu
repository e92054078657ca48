// Tile kernels for one format set: INT4 codes, BF16 group scales, BF16 outer scales.
#include "dq_launch.h"

namespace dq {
cudaError_t launch_tile_c0(const TileLaunch &L) { return launch_tile_combo<CODES_INT4, SC_BF16, SC_BF16>(L); }
}  // namespace dq
