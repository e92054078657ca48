// dq_gemm.cu — block-scaled W4A4 GEMM on the 5th-generation tensor cores:
// the inference step that consumes the solver's output (eq. (1) of the daiwk
// note: X W^T ~= (X D_b) Qhat^T D_a; trove summary, "How to use it": beta is
// applied in the activation-quantization kernel, the weights are stored with
// their codes and scales).
//
//   out[m, n] = a_n * sum_k  Qx[m, k] * Qw[n, k]
//
// Qx = the E2M1 codes and group scales of Q(X D_b) (dq_act_rescale_quant),
// Qw = the E2M1 codes and group scales of Q(W / (a b^T)) (the solve), a = the
// outer row scales of W.  Both operands are K-major E2M1, two codes per byte,
// with one group scale per G elements of K: MXFP4, an E8M0 scale per 32
// (kind::mxf4, block32); NVFP4, an E4M3 scale per 16 (kind::mxf4nvf4,
// block16) and the weights' tensor scale ts (a power of two) applied with
// a_n in the epilogue (news article, "适配 MXFP4 与 NVFP4 块结构").  The
// scales come in scale tiles, the layout the tensor core reads
// (scale_tiles_kernel below): per 128-row block and 4 G elements of K one
// 512-byte chunk holding the scale k (0..3) of row r at byte (r % 32) * 16 +
// (r / 32) * 4 + k.
//
// A persistent CTA per SM walks 128 x BN tiles of `out` (BN = 256, or 128
// when N is not a multiple of 256) with tcgen05.mma kind::mxf4 (M = 128,
// N = BN, K = 64 per instruction, block scales of 32 from TMEM),
// accumulating in float32 in TMEM.  K advances in tiles of 256 elements (128
// bytes per row) through a 4-stage shared-memory ring that runs on across
// output tiles:
//   warp 0     producer: TMA loads of the A and B tiles (128-byte swizzle;
//              every CTA loads its own) and bulk copies of their scale tiles;
//   warp 1     TMEM allocation; lane 0 issues tcgen05.cp (scales to TMEM),
//              the MMAs and the tcgen05.commit arrivals;
//   warps 2-9  epilogue: TMEM -> registers (tcgen05.ld; TMEM is handed back
//              before the stores) -> shared memory -> row-contiguous float32
//              stores, times a_n.
// Every wait on an mbarrier is bounded: a wait that runs out raises a device
// status bit, the CTA stops issuing work, waits (bounded) for its copies in
// flight, frees its TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "dq_launch.h"

namespace dq {

namespace {

constexpr int kBM = 128;
constexpr int kSfChunk = 512;                  // 128 rows x 4 scales
constexpr int kThreadsGemm = 320;               // 10 warps: producer, MMA, 8 epilogue
constexpr uint64_t kWaitLimitNs = 1000000000ull;   // a wait gives up after 1 s

// BN = 128 or 256 output columns per CTA; BK = 128 or 256 K elements per
// stage (64- or 128-byte rows, 64- or 128-byte swizzle); NV: NVFP4 (scale
// chunks of 64 elements of K) rather than MXFP4 (128).
template <int BN, int BK, bool NV>
struct __align__(1024) GemmSmem {
    // 128-column tiles run two CTAs per SM (one's epilogue overlaps the
    // other's MMAs); the ring depth fills the shared memory
    static constexpr int kCtasPerSm = BN == 128 ? 2 : 1;
    static constexpr int NB = BN / 128;                        // 128-row blocks of B
    static constexpr int KC = BK / (NV ? 64 : 128);            // 4-scale chunks per row and stage
    static constexpr int kRowBytes = BK / 2;
    static constexpr int kTileBytesA = kBM * kRowBytes;
    static constexpr int kTileBytesB = BN * kRowBytes;
    static constexpr int kStageBytes = kTileBytesA + kTileBytesB + (1 + NB) * KC * kSfChunk;
    // epilogue staging: per epilogue warp 32 rows x EC float32 columns,
    // 16-byte chunks swizzled so that a row-per-lane write and a
    // row-contiguous read are both free of bank conflicts
    static constexpr int EC = BN == 128 ? 8 : 16;
    static constexpr int kStgBytes = 8 * 32 * EC * 4;
    static constexpr int kStages =
        ((kCtasPerSm == 2 ? 112 * 1024 : 226 * 1024) - kStgBytes - 1024) / kStageBytes;
    static constexpr uint32_t kStageTx = kStageBytes;      // bytes that land per stage
    // TMEM: accumulator BN columns, then two slots of scales, each A's (KC
    // chunks x 4 columns) then B's (KC k-chunks x NB row blocks x 4 columns)
    static constexpr uint32_t kTmemCols = BN == 128 ? 256 : 512;
    uint8_t a[kStages][kTileBytesA];
    uint8_t b[kStages][kTileBytesB];
    uint8_t sfa[kStages][KC * kSfChunk];            // [k-chunk][512]
    uint8_t sfb[kStages][NB * KC * kSfChunk];       // [row block][k-chunk][512]
    float4 stg[8][32 * EC / 4];
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t acc_full;      // MMA -> epilogue: the tile's accumulator is complete
    uint64_t acc_empty;     // epilogue -> MMA: the accumulator has been read out
    uint32_t tmem_base;
    int abort;
};

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t *b, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(smem_u32(b)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *b, uint32_t tx) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
                 :: "r"(smem_u32(b)), "r"(tx) : "memory");
}

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ bool mbar_test(uint32_t addr, uint32_t parity) {
    uint32_t done;
    asm volatile("{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; "
                 "selp.u32 %0, 1, 0, p; }"
                 : "=r"(done) : "r"(addr), "r"(parity) : "memory");
    return done != 0;
}

// Bounded wait for the phase with the given parity to complete.  Returns
// false if another thread of the CTA gave up, or (raising the status bit and
// the CTA's abort flag) if this wait ran past its time limit.
__device__ __forceinline__ bool mbar_wait(uint64_t *b, uint32_t parity, volatile int *abort,
                                          unsigned int *status) {
    const uint32_t addr = smem_u32(b);
    if (mbar_test(addr, parity)) return true;
    const uint64_t t0 = global_ns();
    while (true) {
        if (mbar_test(addr, parity)) return true;
        if (*abort) return false;
        if (global_ns() - t0 > kWaitLimitNs) break;
    }
    *abort = 1;
    atomicOr(status, STATUS_TIMEOUT);
    return false;
}

// Untiled bulk copy global -> this CTA's shared memory, completion counted in
// bytes on the mbarrier; both addresses 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        :: "r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y,
                                            uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];"
        :: "r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y),
           "r"(smem_u32(bar))
        : "memory");
}

// UMMA shared-memory descriptor, K-major, ROWB-byte swizzle (128 or 64):
// rows of ROWB bytes, 8-row atoms 8 * ROWB bytes apart (stride byte
// offset), version 1; layout type 2 = 128-byte swizzle, 4 = 64-byte.
template <int ROWB>
__device__ __forceinline__ uint64_t desc_swz(uint32_t saddr) {
    constexpr uint64_t kLayout = ROWB == 128 ? 2ull : 4ull;
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | (1ull << 16) | ((uint64_t)(8 * ROWB / 16) << 32) |
           (1ull << 46) | (kLayout << 61);
}

// Descriptor of one 512-byte scale chunk for tcgen05.cp 32x128b: 32 rows of
// 16 bytes, 8-row groups 128 bytes apart, no swizzle.
__device__ __forceinline__ uint64_t desc_sf(uint32_t saddr) {
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | (1ull << 16) | (8ull << 32) | (1ull << 46);
}

// Instruction descriptor of the block-scaled E2M1 kinds: A and B E2M1
// (format 1, K-major), M = BM (128, or 256 for a CTA pair), N = BN, the
// scale type (bit 23: 1 = UE8M0 for MXFP4, 0 = UE4M3 for NVFP4) and the
// scale-factor byte ids of A and B.
template <int BM, int BN, bool NV>
__device__ __forceinline__ uint32_t idesc_mxf4_m(uint32_t sfa_id, uint32_t sfb_id) {
    return (sfb_id << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
           ((NV ? 0u : 1u) << 23) | ((uint32_t)(BM >> 4) << 24) | (sfa_id << 29);
}
template <int BN, bool NV>
__device__ __forceinline__ uint32_t idesc_mxf4(uint32_t sfa_id, uint32_t sfb_id) {
    return idesc_mxf4_m<kBM, BN, NV>(sfa_id, sfb_id);
}

// Output tile t -> (m0, n0).  Tiles go in bands of up to kBandTiles tile
// columns: within a band every row of tiles is visited before the next band,
// so the CTAs running together share the band's B tiles (which stay in L2)
// and each A tile is read once per band.  8 columns: the 74 CTA pairs (or
// 148 CTAs on 128 x 256 tiles) running together then cover a roughly square
// block of the output, which needs the fewest distinct A and B tiles.
constexpr int kBandTiles = 8;
__device__ __forceinline__ void tile_coords(int t, int m_tiles, int n_tiles, int bm, int bn,
                                            int &m0, int &n0) {
    const int band = t / (m_tiles * kBandTiles);
    const int nb0 = band * kBandTiles;
    const int width = min(kBandTiles, n_tiles - nb0);
    const int r = t - band * (m_tiles * kBandTiles);
    m0 = (r / width) * bm;
    n0 = (nb0 + r % width) * bn;
}

// One MMA of K = 64: MXFP4 takes 2 E8M0 scales per row (bytes id, id + 1
// of the scale column), NVFP4 4 E4M3 scales (the whole column, id 0).
template <bool NV>
__device__ __forceinline__ void mma_mxf4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                         uint32_t accumulate) {
    if constexpr (NV)
        asm volatile(
            "{ .reg .pred p; setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p; }"
            :: "r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem),
               "r"(sfb_tmem)
            : "memory");
    else
        asm volatile(
            "{ .reg .pred p; setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p; }"
            :: "r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem),
               "r"(sfb_tmem)
            : "memory");
}

__device__ __forceinline__ void tmem_cp_sf(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" :: "r"(taddr), "l"(sdesc)
                 : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 :: "r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// 32 consecutive 32-bit columns of this thread's TMEM lane; the registers
// are valid after tmem_wait_ld on them.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}

// Waits for this thread's TMEM loads; passing the registers through makes
// every later use of them depend on the wait.
__device__ __forceinline__ void tmem_wait_ld(uint32_t (&r)[32]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;" : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31]) :: "memory");
}

// Bounded wait used while draining at exit (no abort check).
__device__ __forceinline__ void mbar_drain(uint64_t *b, uint32_t parity) {
    const uint32_t addr = smem_u32(b);
    const uint64_t t0 = global_ns();
    while (!mbar_test(addr, parity) && global_ns() - t0 <= kWaitLimitNs) {
    }
}

template <int BN, int BK, bool NV>
__global__ void __launch_bounds__(kThreadsGemm, GemmSmem<BN, BK, NV>::kCtasPerSm)
w4a4_gemm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                 const uint8_t *sf_a, const uint8_t *sf_b, const float *a_row, const float *ts_w,
                 float *out, int M, int N, int K, unsigned int *status, int stall) {
    using Smem = GemmSmem<BN, BK, NV>;
    constexpr int kStages = Smem::kStages;
    constexpr int KC = Smem::KC;
    constexpr int NB = Smem::NB;
    grid_dependency_begin();
    extern __shared__ uint8_t gemm_smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>(
        (reinterpret_cast<uintptr_t>(gemm_smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KT = K / BK;
    const int n_tiles = N / BN, m_tiles = M / kBM;
    const int tiles = m_tiles * n_tiles;
    volatile int *abort = &sm.abort;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm.full[s], 1);              // the producer's arrival (+ the stage's bytes)
            mbar_init(&sm.empty[s], 1);
        }
        mbar_init(&sm.acc_full, 1);
        mbar_init(&sm.acc_empty, 8);                // one arrival per epilogue warp
        sm.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     :: "r"(smem_u32(&sm.tmem_base)), "r"(Smem::kTmemCols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;             // accumulator: columns [0, BN)
    // scales of even / odd K tiles in two slots, so that copying the next
    // tile's scales never waits for the MMAs still reading the current ones
    constexpr uint32_t kSfSlot = 4 * KC * (1 + NB);
    const uint32_t sfa_t0 = tmem + BN, sfb_t0 = tmem + BN + 4 * KC;

    // The CTA walks the output tiles t = blockIdx.x, + gridDim.x, ... in the
    // band order of tile_coords.
    int issued = 0;                                 // K tiles the producer issued (warp 0)
    if (warp == 0) {
        // ---- producer (lane 0): per K tile, TMA loads of the two code tiles
        // and bulk copies of their scale tiles (KC consecutive 512-byte
        // chunks per 128-row block), all counted in bytes on the stage's
        // barrier.  The ring runs on across tiles (g counts K tiles of all
        // the CTA's output tiles), so the next tile's operands arrive during
        // the current tile's last MMAs and epilogue. ----
        int g = 0;
        bool stop = false;
        const int64_t kblocks = K / (NV ? 64 : 128);  // scale chunks per 128-row block
        for (int t = blockIdx.x; t < tiles && !stop; t += gridDim.x) {
            int m0, n0;
            tile_coords(t, m_tiles, n_tiles, kBM, BN, m0, n0);
            for (int kt = 0; kt < KT; ++kt, ++g) {
                const int s = g % kStages;
                if (g >= kStages) {
                    int ok = 1;
                    if (lane == 0) ok = mbar_wait(&sm.empty[s], ((g / kStages) - 1) & 1, abort, status);
                    if (!__shfl_sync(0xffffffffu, ok, 0)) { stop = true; break; }
                }
                // (test support: `stall` leaves the first K tile unloaded, so the
                // MMA thread's bounded wait for it runs out)
                if (lane == 0 && !(stall && g == 0)) {
                    mbar_arrive_expect_tx(&sm.full[s], Smem::kStageTx);
                    tma_load_2d(sm.a[s], &map_a, kt * (BK / 2), m0, &sm.full[s]);
                    tma_load_2d(sm.b[s], &map_b, kt * (BK / 2), n0, &sm.full[s]);
                    bulk_load(sm.sfa[s], sf_a + ((m0 / 128) * kblocks + (int64_t)kt * KC) * kSfChunk,
                              KC * kSfChunk, &sm.full[s]);
#pragma unroll
                    for (int nb = 0; nb < NB; ++nb)
                        bulk_load(sm.sfb[s] + nb * KC * kSfChunk,
                                  sf_b + ((n0 / 128 + nb) * kblocks + (int64_t)kt * KC) * kSfChunk,
                                  KC * kSfChunk, &sm.full[s]);
                }
            }
        }
        issued = g;
    } else if (warp == 1) {
        // ---- MMA issuer ----
        if (lane == 0) {
            int g = 0, j = 0;
            bool stop = false;
            for (int t = blockIdx.x; t < tiles && !stop; t += gridDim.x, ++j) {
                // the epilogue has read out the previous tile's accumulator
                if (j > 0 && !mbar_wait(&sm.acc_empty, (j - 1) & 1, abort, status)) break;
                tc_fence_after();
                for (int kt = 0; kt < KT; ++kt, ++g) {
                    const int s = g % kStages;
                    if (!mbar_wait(&sm.full[s], (g / kStages) & 1, abort, status)) { stop = true; break; }
                    tc_fence_after();
                    const uint32_t sfa_t = sfa_t0 + (g & 1) * kSfSlot, sfb_t = sfb_t0 + (g & 1) * kSfSlot;
#pragma unroll
                    for (int kc = 0; kc < KC; ++kc)
                        tmem_cp_sf(sfa_t + 4 * kc, desc_sf(smem_u32(&sm.sfa[s][kc * kSfChunk])));
#pragma unroll
                    for (int q = 0; q < KC * NB; ++q)     // TMEM: [k-chunk][row block]
                        tmem_cp_sf(sfb_t + 4 * q,
                                   desc_sf(smem_u32(&sm.sfb[s][((q % NB) * KC + q / NB) * kSfChunk])));
                    const uint32_t a0 = smem_u32(sm.a[s]), b0 = smem_u32(sm.b[s]);
#pragma unroll
                    for (int kb = 0; kb < BK / 64; ++kb) {
                        // K = 64 per instruction: 32 bytes of each row.
                        // MXFP4: scale blocks 2kb, 2kb+1 = k-chunk kb/2, bytes
                        // 2(kb%2), 2(kb%2)+1 of the word; NVFP4: scale blocks
                        // 4kb .. 4kb+3 = k-chunk kb, the whole word.  B's
                        // scales of a k-chunk span NB x 4 columns
                        const uint32_t c = NV ? kb : kb >> 1, id = NV ? 0 : (kb & 1) * 2;
                        mma_mxf4<NV>(tmem, desc_swz<BK / 2>(a0 + kb * 32), desc_swz<BK / 2>(b0 + kb * 32),
                                     idesc_mxf4<BN, NV>(id, id), sfa_t + 4 * c, sfb_t + 4 * NB * c,
                                     (kt | kb) != 0);
                    }
                    umma_commit(&sm.empty[s]);      // frees the stage once these MMAs are done
                }
                umma_commit(&sm.acc_full);          // also after an abort: the epilogue waits on it
            }
        }
        __syncwarp();
    } else {
        // ---- epilogue: warps 2-9; a warp reads TMEM lane quadrant warp % 4
        // (rows quad*32 .. +31 of the tile) and column half (warp - 2) / 4.
        // It loads its whole share (BN/2 columns) into registers and hands
        // TMEM back to the MMA warp at once, so the next tile's MMAs run
        // while it stores: registers (lane = row) -> its staging block in
        // shared memory (EC columns at a time) -> global memory with each
        // store instruction covering whole row segments (CPR lanes per
        // row), times a_n. ----
        constexpr int EC = Smem::EC;
        constexpr int CPR = EC / 4;                  // 16-byte chunks per staged row
        constexpr int RPP = 32 / CPR;                // rows per store instruction
        constexpr int HALF = BN / 2;                 // columns per warp
        const int quad = warp & 3, ew = warp - 2;
        const int cbase = (ew >> 2) * HALF;
        float4 *stg = sm.stg[ew];
        // chunk c of row r sits at chunk c ^ sw(r) of the row: 8 consecutive
        // rows then cover all eight 16-byte bank groups
        auto sw = [](int r) { return (r / (8 / CPR)) % CPR; };
        const int rr = lane / CPR, cc = lane % CPR;  // this lane's row / chunk in the store pass
        const float ts = ts_w ? __ldg(ts_w) : 1.0f;  // the weights' tensor scale
        int j = 0;
        for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++j) {
            int m0, n0;
            tile_coords(t, m_tiles, n_tiles, kBM, BN, m0, n0);
            int ok = 1;
            if (lane == 0) ok = mbar_wait(&sm.acc_full, j & 1, abort, status) && !*abort;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            tc_fence_after();
            uint32_t v[HALF / 32][32];
            const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)cbase;
#pragma unroll
            for (int i = 0; i < HALF / 32; ++i) tmem_ld32(taddr + 32 * i, v[i]);
#pragma unroll
            for (int i = 0; i < HALF / 32; ++i) tmem_wait_ld(v[i]);
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];"
                             :: "r"(smem_u32(&sm.acc_empty)) : "memory");
            float *const orow = out + (int64_t)(m0 + quad * 32) * N + n0 + cbase;
#pragma unroll
            for (int h = 0; h < HALF / EC; ++h) {
#pragma unroll
                for (int c = 0; c < CPR; ++c) {
                    const int e = h * EC + 4 * c;
                    stg[lane * CPR + (c ^ sw(lane))] = make_float4(
                        __uint_as_float(v[e / 32][e % 32]), __uint_as_float(v[e / 32][e % 32 + 1]),
                        __uint_as_float(v[e / 32][e % 32 + 2]), __uint_as_float(v[e / 32][e % 32 + 3]));
                }
                __syncwarp();
                const int col = h * EC + 4 * cc;
                float4 sc = __ldg(reinterpret_cast<const float4 *>(a_row + n0 + cbase + col));
                sc = make_float4(sc.x * ts, sc.y * ts, sc.z * ts, sc.w * ts);   // exact: ts = 2^k
#pragma unroll
                for (int p = 0; p < CPR; ++p) {
                    const int r = p * RPP + rr;
                    const float4 x = stg[r * CPR + (cc ^ sw(r))];
                    *reinterpret_cast<float4 *>(orow + (int64_t)r * N + col) =
                        make_float4(x.x * sc.x, x.y * sc.y, x.z * sc.z, x.w * sc.w);
                }
                __syncwarp();
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    // after an abort (known to every thread by now), let the copies already
    // issued land before the CTA frees its resources and exits
    if (warp == 0 && lane == 0 && *abort) {
        for (int k = max(0, issued - kStages); k < issued; ++k)
            mbar_drain(&sm.full[k % kStages], (k / kStages) & 1);
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;"
                     :: "r"(tmem), "r"(Smem::kTmemCols) : "memory");
    }
}

// ---------------------------------------------------------------------------
// CTA-pair variant (M and N multiples of 256): a cluster of two CTAs on two
// SMs computes a 256 x 256 tile with tcgen05.mma.cta_group::2 (M = 256, N =
// 256): CTA rank r holds rows 128r..128r+127 of the A tile and rows
// 128r..128r+127 of the B tile (its half of N) in its shared memory, the
// A scales of its own rows and the B scales of all 256 rows; its TMEM holds
// its 128 accumulator rows x 256 columns.  Per SM that is 32 KB of codes per
// K tile of 256 instead of 48 KB, so the ring is 6 stages deep.
//   both CTAs   warp 0 lane 0 loads its halves by TMA (.cta_group::2: the
//               completion is counted on the barrier of CTA 0);
//               warps 2-9 drain their own accumulator rows (as above) and
//               release the accumulator on CTA 0's barrier;
//               warp 1 allocates / frees TMEM (cta_group::2, both CTAs).
//   CTA 0       warp 1 lane 0 waits for both halves of a stage, copies the
//               scales to both TMEMs (tcgen05.cp.cta_group::2), issues the
//               MMAs, and commits to the barriers of both CTAs.
// ---------------------------------------------------------------------------
template <int BK, bool NV>
struct __align__(1024) GemmPairSmem {
    static constexpr int KC = BK / (NV ? 64 : 128);
    static constexpr int kRowBytes = BK / 2;
    static constexpr int kTileBytes = 128 * kRowBytes;                 // A or B half, per CTA
    static constexpr int kStageBytes = 2 * kTileBytes + 3 * KC * kSfChunk;
    static constexpr int EC = 8;
    static constexpr int kStgBytes = 8 * 32 * EC * 4;
    static constexpr int kStages = (226 * 1024 - kStgBytes - 1024) / kStageBytes;
    static constexpr uint32_t kPairTx = 2 * kStageBytes;              // both CTAs' bytes
    static constexpr uint32_t kTmemCols = 512;
    uint8_t a[kStages][kTileBytes];
    uint8_t b[kStages][kTileBytes];
    uint8_t sfa[kStages][KC * kSfChunk];            // [k-chunk][512], own rows
    uint8_t sfb[kStages][2 * KC * kSfChunk];        // [row block][k-chunk][512], all 256 rows
    float4 stg[8][32 * EC / 4];
    uint64_t full[kStages];     // CTA 0: both CTAs' bytes of the stage have landed
    uint64_t empty[kStages];    // the MMAs reading the stage are done (each CTA)
    uint64_t acc_full;          // the tile's accumulator is complete (each CTA)
    uint64_t acc_empty;         // CTA 0: both CTAs' epilogues have read it out
    uint32_t tmem_base;
    int abort;
};

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Shared-memory address of the same variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t cluster_addr(const void *p, uint32_t rank) {
    uint32_t a;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(smem_u32(p)), "r"(rank));
    return a;
}

__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
                 "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// TMA load into this CTA's shared memory (and no other CTA's) whose
// completion is counted on an mbarrier of either CTA of the pair (bar:
// shared::cluster address).
__device__ __forceinline__ void tma_load_2d_pair(void *dst, const CUtensorMap *map, int x, int y,
                                                 uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];"
        :: "r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

template <bool NV>
__device__ __forceinline__ void mma_mxf4_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                              uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                              uint32_t accumulate) {
    if constexpr (NV)
        asm volatile(
            "{ .reg .pred p; setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p; }"
            :: "r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem),
               "r"(sfb_tmem)
            : "memory");
    else
        asm volatile(
            "{ .reg .pred p; setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p; }"
            :: "r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem),
               "r"(sfb_tmem)
            : "memory");
}

__device__ __forceinline__ void tmem_cp_sf_pair(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" :: "r"(taddr), "l"(sdesc)
                 : "memory");
}

// Arrive on the mbarrier at this offset in both CTAs of the pair once the
// tcgen05 operations issued so far by this thread are complete.
__device__ __forceinline__ void umma_commit_pair(uint64_t *bar) {
    asm volatile(
        "{ .reg .b16 m; mov.b16 m, 3;\n\t"
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%0], m; }"
        :: "r"(smem_u32(bar)) : "memory");
}

template <int BK, bool NV>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreadsGemm, 1)
w4a4_gemm_pair_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                      const __grid_constant__ CUtensorMap map_sfa,
                      const __grid_constant__ CUtensorMap map_sfb, const float *a_row,
                      const float *ts_w, float *out, int M, int N, int K, unsigned int *status,
                      int stall) {
    using Smem = GemmPairSmem<BK, NV>;
    constexpr int kStages = Smem::kStages;
    constexpr int KC = Smem::KC;
    constexpr int BN = 256;
    grid_dependency_begin();
    extern __shared__ uint8_t gemm_smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>(
        (reinterpret_cast<uintptr_t>(gemm_smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const bool leader = rank == 0;
    const int KT = K / BK;
    const int n_tiles = N / BN, m_tiles = M / 256;
    const int tiles = m_tiles * n_tiles;
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    const int64_t kblocks = K / (NV ? 64 : 128);    // scale chunks per 128-row block
    volatile int *abort = &sm.abort;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm.full[s], 1);              // CTA 0's producer (+ both CTAs' bytes)
            mbar_init(&sm.empty[s], 1);             // CTA 0's commit
        }
        mbar_init(&sm.acc_full, 1);                 // CTA 0's commit
        mbar_init(&sm.acc_empty, 16);               // 8 epilogue warps per CTA
        sm.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
                     :: "r"(smem_u32(&sm.tmem_base)), "r"(Smem::kTmemCols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    cluster_sync_all();                             // barriers and TMEM ready in both CTAs
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;             // accumulator: columns [0, 256)
    constexpr uint32_t kSfSlot = 4 * KC * 3;        // two scale slots, as above
    const uint32_t sfa_t0 = tmem + BN, sfb_t0 = tmem + BN + 4 * KC;

    int issued = 0;                                 // K tiles the producer issued (warp 0)
    if (warp == 0) {
        if (lane == 0) {
            // ---- producer: this CTA's halves of every K tile ----
            const uint32_t full0 = cluster_addr(&sm.full[0], 0);
            int g = 0;
            bool stop = false;
            for (int t = pair; t < tiles && !stop; t += npairs) {
                int m0, n0;
                tile_coords(t, m_tiles, n_tiles, 256, BN, m0, n0);
                const int ma = m0 + 128 * (int)rank, nb0 = n0 + 128 * (int)rank;
                for (int kt = 0; kt < KT; ++kt, ++g) {
                    const int s = g % kStages;
                    if (g >= kStages && !mbar_wait(&sm.empty[s], ((g / kStages) - 1) & 1, abort, status)) {
                        stop = true;
                        break;
                    }
                    if (stall && g == 0) continue;       // test support, as above
                    const uint32_t bar = full0 + (uint32_t)(s * sizeof(uint64_t));
                    if (leader) mbar_arrive_expect_tx(&sm.full[s], Smem::kPairTx);
                    tma_load_2d_pair(sm.a[s], &map_a, kt * (BK / 2), ma, bar);
                    tma_load_2d_pair(sm.b[s], &map_b, kt * (BK / 2), nb0, bar);
                    tma_load_2d_pair(sm.sfa[s], &map_sfa, 0, (int)((ma / 128) * kblocks + kt * KC), bar);
#pragma unroll
                    for (int nb = 0; nb < 2; ++nb)
                        tma_load_2d_pair(sm.sfb[s] + nb * KC * kSfChunk, &map_sfb, 0,
                                         (int)((n0 / 128 + nb) * kblocks + kt * KC), bar);
                }
            }
            issued = g;
        }
        __syncwarp();
    } else if (warp == 1) {
        if (leader && lane == 0) {
            // ---- MMA issuer (CTA 0) ----
            int g = 0, j = 0;
            bool stop = false;
            for (int t = pair; t < tiles && !stop; t += npairs, ++j) {
                // both CTAs' epilogues have read out the previous accumulator
                if (j > 0 && !mbar_wait(&sm.acc_empty, (j - 1) & 1, abort, status)) break;
                tc_fence_after();
                for (int kt = 0; kt < KT; ++kt, ++g) {
                    const int s = g % kStages;
                    if (!mbar_wait(&sm.full[s], (g / kStages) & 1, abort, status)) { stop = true; break; }
                    tc_fence_after();
                    const uint32_t sfa_t = sfa_t0 + (g & 1) * kSfSlot, sfb_t = sfb_t0 + (g & 1) * kSfSlot;
#pragma unroll
                    for (int kc = 0; kc < KC; ++kc)
                        tmem_cp_sf_pair(sfa_t + 4 * kc, desc_sf(smem_u32(&sm.sfa[s][kc * kSfChunk])));
#pragma unroll
                    for (int q = 0; q < 2 * KC; ++q)      // TMEM: [k-chunk][row block]
                        tmem_cp_sf_pair(sfb_t + 4 * q,
                                        desc_sf(smem_u32(&sm.sfb[s][((q % 2) * KC + q / 2) * kSfChunk])));
                    const uint32_t a0 = smem_u32(sm.a[s]), b0 = smem_u32(sm.b[s]);
#pragma unroll
                    for (int kb = 0; kb < BK / 64; ++kb) {
                        const uint32_t c = NV ? kb : kb >> 1, id = NV ? 0 : (kb & 1) * 2;
                        mma_mxf4_pair<NV>(tmem, desc_swz<BK / 2>(a0 + kb * 32), desc_swz<BK / 2>(b0 + kb * 32),
                                          idesc_mxf4_m<256, BN, NV>(id, id), sfa_t + 4 * c, sfb_t + 8 * c,
                                          (kt | kb) != 0);
                    }
                    umma_commit_pair(&sm.empty[s]);  // frees the stage in both CTAs
                }
                umma_commit_pair(&sm.acc_full);      // also after an abort: the epilogues wait on it
            }
        }
        __syncwarp();
    } else {
        // ---- epilogue (both CTAs): rows m0 + 128 rank + quad*32 + lane ----
        constexpr int EC = Smem::EC;
        constexpr int CPR = EC / 4;
        constexpr int RPP = 32 / CPR;
        constexpr int HALF = BN / 2;
        const int quad = warp & 3, ew = warp - 2;
        const int cbase = (ew >> 2) * HALF;
        float4 *stg = sm.stg[ew];
        auto sw = [](int r) { return (r / (8 / CPR)) % CPR; };
        const int rr = lane / CPR, cc = lane % CPR;
        const uint32_t acc_empty0 = cluster_addr(&sm.acc_empty, 0);
        const float ts = ts_w ? __ldg(ts_w) : 1.0f;  // the weights' tensor scale
        int j = 0;
        for (int t = pair; t < tiles; t += npairs, ++j) {
            int m0, n0;
            tile_coords(t, m_tiles, n_tiles, 256, BN, m0, n0);
            int ok = 1;
            if (lane == 0) ok = mbar_wait(&sm.acc_full, j & 1, abort, status) && !*abort;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            tc_fence_after();
            uint32_t v[HALF / 32][32];
            const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)cbase;
#pragma unroll
            for (int i = 0; i < HALF / 32; ++i) tmem_ld32(taddr + 32 * i, v[i]);
#pragma unroll
            for (int i = 0; i < HALF / 32; ++i) tmem_wait_ld(v[i]);
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];"
                             :: "r"(acc_empty0) : "memory");
            float *const orow = out + (int64_t)(m0 + 128 * (int)rank + quad * 32) * N + n0 + cbase;
#pragma unroll
            for (int h = 0; h < HALF / EC; ++h) {
#pragma unroll
                for (int c = 0; c < CPR; ++c) {
                    const int e = h * EC + 4 * c;
                    stg[lane * CPR + (c ^ sw(lane))] = make_float4(
                        __uint_as_float(v[e / 32][e % 32]), __uint_as_float(v[e / 32][e % 32 + 1]),
                        __uint_as_float(v[e / 32][e % 32 + 2]), __uint_as_float(v[e / 32][e % 32 + 3]));
                }
                __syncwarp();
                const int col = h * EC + 4 * cc;
                float4 sc = __ldg(reinterpret_cast<const float4 *>(a_row + n0 + cbase + col));
                sc = make_float4(sc.x * ts, sc.y * ts, sc.z * ts, sc.w * ts);   // exact: ts = 2^k
#pragma unroll
                for (int p = 0; p < CPR; ++p) {
                    const int r = p * RPP + rr;
                    const float4 x = stg[r * CPR + (cc ^ sw(r))];
                    *reinterpret_cast<float4 *>(orow + (int64_t)r * N + col) =
                        make_float4(x.x * sc.x, x.y * sc.y, x.z * sc.z, x.w * sc.w);
                }
                __syncwarp();
            }
        }
    }
    // every MMA of the pair has completed (each CTA's epilogue saw the last
    // commit, or gave up): no CTA leaves while its partner may still signal
    // its barriers or read its TMEM
    tc_fence_before();
    __syncthreads();
    // after an abort (known to every thread of this CTA by now), let the
    // copies already issued land: CTA 0's barriers count both CTAs' bytes;
    // CTA 1 only waits a little, its partner drains before the cluster
    // barrier below
    if (warp == 0 && lane == 0 && *abort) {
        if (leader) {
            for (int k = max(0, issued - kStages); k < issued; ++k)
                mbar_drain(&sm.full[k % kStages], (k / kStages) & 1);
        } else {
            const uint64_t t0 = global_ns();
            while (global_ns() - t0 < 2000000ull) {
            }
        }
    }
    __syncthreads();
    cluster_sync_all();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;"
                     :: "r"(tmem), "r"(Smem::kTmemCols) : "memory");
    }
}

// Row-major group scales [rows, K/G] -> scale tiles: one thread per 4-byte
// word (the 4 scales of one row in one 4G-element K block); word w of chunk
// (rb, kc) holds row rb*128 + (w % 4)*32 + w/4, so the writes are coalesced.
__global__ void __launch_bounds__(256)
scale_tiles_kernel(const uint8_t *scales, int64_t words, int64_t kblocks, uint8_t *tiles) {
    grid_dependency_begin();
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < words;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t chunk = i >> 7;
        const int w = (int)(i & 127);
        const int64_t rb = chunk / kblocks, kc = chunk % kblocks;
        const int64_t r = rb * 128 + (w & 3) * 32 + (w >> 2);
        const uint32_t v = __ldg(reinterpret_cast<const uint32_t *>(scales + r * (kblocks * 4) + kc * 4));
        reinterpret_cast<uint32_t *>(tiles)[i] = v;
    }
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// 2-D map over a [rows, K/2]-byte code matrix: boxes of box_rows x row_bytes,
// swizzled by row_bytes (128 or 64).
bool code_map(CUtensorMap *m, const uint8_t *codes, int64_t rows, int64_t K, int box_rows,
              int row_bytes) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)(K / 2), (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)(K / 2)};
    const cuuint32_t box[2] = {(cuuint32_t)row_bytes, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUtensorMapSwizzle swz = row_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(codes), dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D map over scale tiles as rows of one 512-byte chunk (256 x 16-bit
// elements): boxes of KC consecutive chunks, no swizzle; kblocks chunks per
// 128-row block.
bool scale_tile_map(CUtensorMap *m, const uint8_t *tiles, int64_t rows, int64_t kblocks, int kc) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[2] = {256, (cuuint64_t)(rows / 128 * kblocks)};
    const cuuint64_t strides[1] = {512};
    const cuuint32_t box[2] = {256, (cuuint32_t)kc};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<uint8_t *>(tiles), dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BK, bool NV>
cudaError_t launch_pair(const GemmLaunch &L) {
    using Smem = GemmPairSmem<BK, NV>;
    static_assert(sizeof(Smem) + 1024 <= 232448, "shared memory of the GEMM CTA");
    CUtensorMap ma, mb, msa, msb;
    const int64_t kblocks = L.K / (NV ? 64 : 128);
    if (!code_map(&ma, L.codes_x, L.M, L.K, 128, BK / 2) || !code_map(&mb, L.codes_w, L.N, L.K, 128, BK / 2) ||
        !scale_tile_map(&msa, L.scales_x, L.M, kblocks, Smem::KC) ||
        !scale_tile_map(&msb, L.scales_w, L.N, kblocks, Smem::KC))
        return cudaErrorInvalidValue;
    const size_t smem = sizeof(Smem) + 1024;
    static std::atomic<bool> done[64];
    cudaError_t e = smem_opt_in(w4a4_gemm_pair_kernel<BK, NV>, smem, done);
    if (e != cudaSuccess) return e;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
    // persistent: one CTA pair per two SMs, or fewer tiles
    int sms = 148;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) sms = 148;
    const int64_t tiles = (L.M / 256) * (L.N / 256);
    const unsigned grid = 2u * (unsigned)std::min<int64_t>(tiles, sms / 2);
    return launch_k(w4a4_gemm_pair_kernel<BK, NV>, dim3(grid), dim3(kThreadsGemm), smem, L.stream, ma,
                    mb, msa, msb, L.a, L.ts, L.out, (int)L.M, (int)L.N, (int)L.K, L.status, L.stall);
}

template <int BN, int BK, bool NV>
cudaError_t launch_bn(const GemmLaunch &L) {
    using Smem = GemmSmem<BN, BK, NV>;
    static_assert(sizeof(Smem) + 1024 <= (Smem::kCtasPerSm == 2 ? 115712 : 232448),
                  "shared memory of the GEMM CTA");
    CUtensorMap ma, mb;
    if (!code_map(&ma, L.codes_x, L.M, L.K, kBM, BK / 2) || !code_map(&mb, L.codes_w, L.N, L.K, BN, BK / 2))
        return cudaErrorInvalidValue;
    const size_t smem = sizeof(Smem) + 1024;
    static std::atomic<bool> done[64];
    cudaError_t e = smem_opt_in(w4a4_gemm_kernel<BN, BK, NV>, smem, done);
    if (e != cudaSuccess) return e;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
    // persistent: kCtasPerSm CTAs per SM, or fewer tiles
    int sms = 148;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) sms = 148;
    const int64_t tiles = (L.M / kBM) * (L.N / BN);
    const unsigned grid = (unsigned)std::min<int64_t>(tiles, (int64_t)sms * Smem::kCtasPerSm);
    return launch_k(w4a4_gemm_kernel<BN, BK, NV>, dim3(grid), dim3(kThreadsGemm), smem, L.stream, ma,
                    mb, L.scales_x, L.scales_w, L.a, L.ts, L.out, (int)L.M, (int)L.N, (int)L.K,
                    L.status, L.stall);
}

}  // namespace

constexpr int kGemmBK = 256;

// A CTA pair per 256 x 256 tile when M and N allow it; else one CTA per
// 128 x 256 tile when N allows it (A tiles reused twice as often), else
// 128 x 128.
cudaError_t launch_scale_tiles(const uint8_t *scales, int64_t rows, int64_t K, int G, uint8_t *tiles,
                               cudaStream_t stream) {
    const int64_t words = rows * K / (4 * G);
    if (words == 0) return cudaSuccess;
    const int64_t blocks = std::min<int64_t>((words + 255) / 256, 148 * 16);
    return launch_k(scale_tiles_kernel, dim3((unsigned)blocks), dim3(256), 0, stream, scales, words,
                    K / (4 * G), tiles);
}

template <bool NV>
cudaError_t launch_w4a4_gemm_fmt(const GemmLaunch &L) {
    if (L.M % 256 == 0 && L.N % 256 == 0) return launch_pair<kGemmBK, NV>(L);
    return (L.N % 256 == 0) ? launch_bn<256, kGemmBK, NV>(L) : launch_bn<128, kGemmBK, NV>(L);
}

cudaError_t launch_w4a4_gemm(const GemmLaunch &L) {
    if (L.M == 0 || L.N == 0) return cudaSuccess;
    return L.nv ? launch_w4a4_gemm_fmt<true>(L) : launch_w4a4_gemm_fmt<false>(L);
}

}  // namespace dq
