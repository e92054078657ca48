// dq_launch.h — host-side launch entry points of the per-format kernel
// translation units (one unit per (codes, group scale, outer scale) set, so
// that they compile in parallel).
#pragma once

#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <utility>

#include "dq_device.cuh"

namespace dq {

// Tile geometry of one matrix: wc warp columns of 256 bf16 (128 float32)
// columns per CTA, ncb column blocks, tr[mode slot] rows per tile and the
// tile counts; it fixes each tile kernel's traffic (the column partials are
// one float2 per column per row block of the column statistics).
struct Geom {
    int wc, ncb;
    int tr[3];
    int64_t ntiles[3];
    int64_t nrb_col;
};

// tall: a batch with many tiles (kTallTiles at the default geometry) gives
// every matrix at least 64 rows per warp: short matrices then take fewer,
// longer tiles (a tile's set-up and drain cost about as much as 16 of its
// rows), while alone they keep about 16 row blocks to spread over the GPU.
constexpr int64_t kTallTiles = 8 * 2 * 148;      // 8 waves of the column pass (2 CTAs per SM)
inline Geom geometry(int64_t rows, int64_t cols, bool f32, bool tall = false) {
    Geom g{};
    const int epc = f32 ? 4 : 8, seg = 32 * epc;
    const int64_t nseg = (cols + seg - 1) / seg;
    // warps across columns: of 8, 4, 2 and 1 the one whose column blocks
    // (wc warp segments each) cover a row with the fewest segments, since a
    // warp segment past the last column computes on zeros; ties go to the
    // wider block (8 for 4096 columns; 1 for 576, in three column blocks,
    // and 2 for 1536, where a power of two at least the segment count would
    // leave a quarter or more of the lanes idle)
    int wc = 8;
    int64_t best = (nseg + 7) / 8 * 8;
    for (int w = 4; w >= 1; w >>= 1) {
        const int64_t segs = (nseg + w - 1) / w * w;
        if (segs < best) { best = segs; wc = w; }
    }
    g.wc = wc;
    g.ncb = (int)((nseg + wc - 1) / wc);
    const int wr = kWarps / wc;
    // rows per warp: 256 for column statistics (fewer partial sums), 128 for
    // the other modes (tile set-up spread over the rows), both reduced for
    // short matrices so that they still make about 16 row blocks (at least
    // 16 rows, or 64 in a tall batch)
    int rpw_long = tall ? 64 : 16;
    while (rpw_long < 128 && 2 * rpw_long <= rows / (wr * 16)) rpw_long *= 2;
    int rpw_col = rpw_long;
    while (rpw_col < 256 && 2 * rpw_col <= rows / (wr * 16)) rpw_col *= 2;
    const int rpw[3] = {rpw_long, rpw_col, rpw_long};
    for (int m = 0; m < 3; ++m) {
        g.tr[m] = rpw[m] * wr;
        const int64_t nrb = (rows + g.tr[m] - 1) / g.tr[m];
        g.ntiles[m] = (rows > 0 && cols > 0) ? nrb * g.ncb : 0;
    }
    g.nrb_col = (rows + g.tr[1] - 1) / g.tr[1];
    return g;
}

struct TileLaunch {
    Table tab;
    int64_t grid;       // CTAs launched (tiles are visited grid-stride)
    int64_t tiles;      // number of tiles
    int mode;           // MODE_*
    int slot;           // tile table slot: 0 ROW, 1 COL, 2 PACK/ACT
    int f32;            // 1: float32 input, 0: bfloat16
    int G;              // 16, 32, 64
    int want_res;       // 1: accumulate the residual (an MSE output is wanted)
    unsigned int *flags;  // fused-path flags of the iteration (or NULL)
    int gate;           // 0 always run; 1 run if flags[0]; 2 run if flags[0] | flags[1]
    cudaStream_t stream;
};

// Format sets with compiled kernels.
enum Combo {
    COMBO_INT4_BF16_BF16 = 0,   // INT4, BF16 group, BF16 outer     ("int4_bf16")
    COMBO_INT4_E8M0_E8M0 = 1,   // INT4, E8M0 group, E8M0 outer     ("mxint4")
    COMBO_E2M1_E8M0_E8M0 = 2,   // E2M1, E8M0 group, E8M0 outer     ("mxfp4")
    COMBO_E2M1_E4M3_BF16 = 3,   // E2M1, E4M3 group, BF16 outer     ("nvfp4")
    COMBO_INT4_E8M0_BF16 = 4,   // INT4, E8M0 group, BF16 outer
    COMBO_E2M1_E8M0_BF16 = 5,   // E2M1, E8M0 group, BF16 outer
    COMBO_INT8_E8M0_E8M0 = 6,   // INT8, E8M0, E8M0                 ("mxint8")
    COMBO_E4M3_E8M0_E8M0 = 7,   // E4M3 elements, E8M0, E8M0        ("mxfp8_e4m3")
    COMBO_E5M2_E8M0_E8M0 = 8,   // E5M2 elements, E8M0, E8M0        ("mxfp8_e5m2")
    COMBO_E2M3_E8M0_E8M0 = 9,   // E2M3 elements, E8M0, E8M0        ("mxfp6_e2m3")
    COMBO_E3M2_E8M0_E8M0 = 10,  // E3M2 elements, E8M0, E8M0        ("mxfp6_e3m2")
    COMBO_COUNT = 11
};

// Launch with programmatic stream serialization: the kernel may start while
// the previous kernel of the stream finishes; every kernel of the library
// begins with grid_dependency_begin(), which keeps the stream's order of
// memory accesses.
template <typename... P, typename... A>
cudaError_t launch_k(void (*kern)(P...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                     A &&...args) {
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<A>(args)...);
}

// Two-level absmax quantization (dq_twolevel.cu).
struct TwoLevelLaunch {
    const void *X;
    int64_t rows, cols, nblk;
    int dual_block;         // 256, 512 or 1024
    int f32;                // 1: float32 input, 0: bfloat16
    uint8_t *codes;         // [rows, cols/2] E2M1
    uint8_t *iscales;       // [rows, cols/32] E8M0
    float *oscales;         // [rows, nblk]
    float *qdq;             // [rows, cols] or NULL
    unsigned int *status;
    cudaStream_t stream;
};
cudaError_t launch_two_level(const TwoLevelLaunch &L);

// Block-scaled W4A4 GEMM (dq_gemm.cu): out[M, N] = a_n ts * Qx[M, K] . Qw[N, K]^T.
struct GemmLaunch {
    const uint8_t *codes_x, *scales_x;   // [M, K/2] E2M1, M*K/G group scales in scale tiles
    const uint8_t *codes_w, *scales_w;   // [N, K/2] E2M1, N*K/G group scales in scale tiles
    const float *a;                      // [N]
    const float *ts;                     // the weights' tensor scale (1 float) or NULL (1)
    float *out;                          // [M, N]
    int64_t M, N, K;                     // multiples of 128, 128, 256
    int nv;                              // 1: NVFP4 (E4M3 scales, G16); 0: MXFP4 (E8M0, G32)
    unsigned int *status;
    int stall;                           // test support: skip the loads of the first K tile
    cudaStream_t stream;
};
cudaError_t launch_w4a4_gemm(const GemmLaunch &L);
// Row-major group scales [rows, K/G] -> the GEMM's scale tiles (rows a
// multiple of 128, K of 4 G).
cudaError_t launch_scale_tiles(const uint8_t *scales, int64_t rows, int64_t K, int G, uint8_t *tiles,
                               cudaStream_t stream);

cudaError_t launch_tile_c0(const TileLaunch &L);
cudaError_t launch_tile_c1(const TileLaunch &L);
cudaError_t launch_tile_c2(const TileLaunch &L);
cudaError_t launch_tile_c3(const TileLaunch &L);
cudaError_t launch_tile_c4(const TileLaunch &L);
cudaError_t launch_tile_c5(const TileLaunch &L);
cudaError_t launch_tile_c6(const TileLaunch &L);
cudaError_t launch_tile_c7(const TileLaunch &L);
cudaError_t launch_tile_c8(const TileLaunch &L);
cudaError_t launch_tile_c9(const TileLaunch &L);
cudaError_t launch_tile_c10(const TileLaunch &L);

// Raise a kernel's dynamic shared-memory limit on the current device, once
// per device and kernel (`done`: one flag per device, owned by the caller's
// instantiation).  Host threads racing on the first call both make the same
// idempotent attribute call.
template <typename K>
cudaError_t smem_opt_in(K kern, size_t bytes, std::atomic<bool> (&done)[64]) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!done[dev].load(std::memory_order_acquire)) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
        if (e != cudaSuccess) return e;
        done[dev].store(true, std::memory_order_release);
    }
    return cudaSuccess;
}

// One tile-kernel launch; the shared memory is dynamic (the row-statistics
// layout needs more than the 48 KB default, opted in once per device).
template <int CODES, int GS, int OS, int MODE, typename TIn, int G>
cudaError_t launch_tile_one(const TileLaunch &L) {
    constexpr size_t bytes = sizeof(TileSmem<MODE, Chunk<TIn>::EPC>);
    auto kern = tile_kernel<CODES, GS, OS, MODE, TIn, G>;
    if (bytes > 48 * 1024) {
        static std::atomic<bool> done[64];
        cudaError_t e = smem_opt_in(kern, bytes, done);
        if (e != cudaSuccess) return e;
    }
    return launch_k(kern, dim3((unsigned)L.grid), dim3(kThreads), bytes, L.stream, L.tab, L.slot,
                    L.want_res, L.tiles, L.flags, L.gate);
}

// Dispatch over mode, dtype and G for one format set (used by each unit).
template <int CODES, int GS, int OS>
cudaError_t launch_tile_combo(const TileLaunch &L) {
    if (L.grid <= 0 || L.tiles <= 0) return cudaSuccess;
#define DQ_TILE(MODE, TIN, GG) return launch_tile_one<CODES, GS, OS, MODE, TIN, GG>(L)
#define DQ_BY_G(MODE, TIN)                          \
    switch (L.G) {                                  \
        case 16: DQ_TILE(MODE, TIN, 16);            \
        case 32: DQ_TILE(MODE, TIN, 32);            \
        case 64: DQ_TILE(MODE, TIN, 64);            \
        default: return cudaErrorInvalidValue;      \
    }
#define DQ_BY_T(MODE)                                      \
    if (L.f32) { DQ_BY_G(MODE, float) } else { DQ_BY_G(MODE, Bf16Tag) }
    switch (L.mode) {
        case MODE_ROW: DQ_BY_T(MODE_ROW);
        case MODE_COL: DQ_BY_T(MODE_COL);
        case MODE_FUSED:
            if constexpr (GS == SC_E8M0 && OS == SC_E8M0) { DQ_BY_T(MODE_FUSED); }
            return cudaErrorInvalidValue;
        case MODE_ROW_W2:
            if constexpr (CodeTraits<CODES>::kBits == 4) { DQ_BY_T(MODE_ROW_W2); }
            return cudaErrorInvalidValue;
        case MODE_FUSED_W2:
            if constexpr (GS == SC_E8M0 && OS == SC_E8M0 && CodeTraits<CODES>::kBits == 4) {
                DQ_BY_T(MODE_FUSED_W2);
            }
            return cudaErrorInvalidValue;
        case MODE_PACK: DQ_BY_T(MODE_PACK);
        case MODE_ACT:
            if (L.f32) return cudaErrorInvalidValue;
            DQ_BY_G(MODE_ACT, Bf16Tag);
        default: return cudaErrorInvalidValue;
    }
#undef DQ_BY_T
#undef DQ_BY_G
#undef DQ_TILE
}

}  // namespace dq
