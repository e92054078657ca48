// Tile kernels for one format set: INT4 codes, E8M0 group scales, BF16 outer scales.
#include "dq_launch.h"

namespace dq {
cudaError_t launch_tile_c4(const TileLaunch &L) { return launch_tile_combo<CODES_INT4, SC_E8M0, SC_BF16>(L); }
}  // namespace dq
