// dq_twolevel.cu — two-level absmax quantization (msmodelslim.readthedocs.io,
// DualScale page, "算法原理" 1(a)-(c), 2(a)-(b)): per row and block of D
// columns an outer float32 scale S = max|X_block| / 6 (the largest normal
// E2M1 value), the block divided by S, quantized with MXFP4 (E2M1 codes,
// E8M0 group scale per 32 columns, rounded up as in Q), and the
// reconstruction (c * s) * S.
//
// One warp per (row, block): a lane owns EPL = D / 32 consecutive columns,
// so the block max is a 5-step shuffle butterfly and an inner group of 32
// columns spans 32 / EPL lanes.  S and X / S are IEEE float32 divisions
// (correctly rounded); the E8M0 scale and the codes of X / S are exact
// decisions (powers of two).
#include <cuda_runtime.h>

#include "dq_launch.h"

namespace dq {

namespace {

template <typename TIn, int EPL>
__device__ __forceinline__ void load_lane(const void *X, int64_t off, float (&x)[EPL]) {
    if constexpr (sizeof(TIn) == 2) {
        const uint4 *p = reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(X) + off);
#pragma unroll
        for (int k = 0; k < EPL / 8; ++k) {
            const uint4 v = __ldg(p + k);
            const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                x[8 * k + 2 * j] = __uint_as_float(u[j] << 16);
                x[8 * k + 2 * j + 1] = __uint_as_float(u[j] & 0xFFFF0000u);
            }
        }
    } else {
        const float4 *p = reinterpret_cast<const float4 *>(static_cast<const float *>(X) + off);
#pragma unroll
        for (int k = 0; k < EPL / 4; ++k) {
            const float4 v = __ldg(p + k);
            x[4 * k] = v.x;
            x[4 * k + 1] = v.y;
            x[4 * k + 2] = v.z;
            x[4 * k + 3] = v.w;
        }
    }
}

// TIn: uint16_t (bf16 bits) or float.
template <typename TIn, int EPL>
__global__ void __launch_bounds__(256)
two_level_kernel(const void *X, int64_t rows, int64_t cols, int64_t nblk, uint8_t *codes,
                 uint8_t *iscales, float *oscales, float *qdq, unsigned int *status) {
    grid_dependency_begin();
    constexpr int D = 32 * EPL;
    constexpr int LPG = 32 / EPL;                    // lanes per inner group of 32 columns
    const int lane = threadIdx.x & 31;
    const int64_t units = rows * nblk;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t u = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; u < units;
         u += nwarps) {
        const int64_t r = u / nblk, kb = u % nblk;
        const int64_t c0 = kb * D + (int64_t)lane * EPL;
        // cols is a multiple of 32 and EPL divides 32: a lane's columns are
        // all inside or all past the end
        const bool ok = c0 < cols;
        float x[EPL];
        if (ok) {
            load_lane<TIn, EPL>(X, r * cols + c0, x);
        } else {
#pragma unroll
            for (int j = 0; j < EPL; ++j) x[j] = 0.0f;
        }
        // outer scale: block max / 6 (float32 division), 1 for a zero block
        float m = 0.0f;
#pragma unroll
        for (int j = 0; j < EPL; ++j) m = max_nan(m, fabsf(x[j]));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = max_nan(m, __shfl_xor_sync(0xffffffffu, m, o));
        const bool finite = (__float_as_uint(m) & 0x7F800000u) != 0x7F800000u;
        if (!finite && lane == 0) atomicOr(status, STATUS_NONFINITE);
        const float S = (m > 0.0f && finite) ? __fdiv_rn(m, 6.0f) : 1.0f;
        float y[EPL];
#pragma unroll
        for (int j = 0; j < EPL; ++j) y[j] = __fdiv_rn(x[j], S);
        // inner E8M0 scale of each group of 32: smallest 2^e with 6 * 2^e >= g
        float g = 0.0f;
#pragma unroll
        for (int j = 0; j < EPL; ++j) g = max_nan(g, fabsf(y[j]));
#pragma unroll
        for (int o = 1; o < LPG; o <<= 1) g = max_nan(g, __shfl_xor_sync(0xffffffffu, g, o));
        const uint32_t gb = __float_as_uint(g);
        constexpr uint32_t MT = CodeTraits<CODES_E2M1>::kMT;
        constexpr int QE = CodeTraits<CODES_E2M1>::kQE;
        float s = __uint_as_float(
            (uint32_t)max((int)((gb + (0x7FFFFFu - MT)) & 0x7F800000u) - (QE << 23), 1 << 23));
        if (!(g > 0.0f)) s = 1.0f;                   // all-zero group: stored scale 1
        const float rs = recip_pow2(s);
        // codes (E2M1, nearest even) and the reconstruction (c * s) * S
        uint32_t cw[EPL / 8] = {};
        float out[EPL];
#pragma unroll
        for (int j = 0; j < EPL; j += 2) {
            uint32_t byte;
            const float2 c = e2m1_round2_byte(y[j] * rs, y[j + 1] * rs, byte);
            cw[j / 8] |= byte << (8 * ((j / 2) % 4));
            out[j] = (c.x * s) * S;
            out[j + 1] = (c.y * s) * S;
        }
        if (ok) {
            uint8_t *cp = codes + (r * cols + c0) / 2;
            if constexpr (EPL == 8) {
                *reinterpret_cast<uint32_t *>(cp) = cw[0];
            } else if constexpr (EPL == 16) {
                *reinterpret_cast<uint2 *>(cp) = make_uint2(cw[0], cw[1]);
            } else {
                *reinterpret_cast<uint4 *>(cp) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
            }
            if (lane % LPG == 0)
                iscales[r * (cols / 32) + c0 / 32] = (uint8_t)((__float_as_uint(s) >> 23) & 0xFF);
            if (qdq != nullptr) {
                float4 *q4 = reinterpret_cast<float4 *>(qdq + r * cols + c0);
#pragma unroll
                for (int k = 0; k < EPL / 4; ++k)
                    q4[k] = make_float4(out[4 * k], out[4 * k + 1], out[4 * k + 2], out[4 * k + 3]);
            }
        }
        if (lane == 0) oscales[r * nblk + kb] = S;
    }
}

template <typename TIn>
cudaError_t launch_typed(const TwoLevelLaunch &L) {
    const int64_t units = L.rows * L.nblk;
    if (units == 0) return cudaSuccess;
    const int64_t blocks = std::min<int64_t>((units + 7) / 8, 148 * 8);
    const dim3 grid((unsigned)blocks), block(256);
    switch (L.dual_block) {
        case 256:
            return launch_k(two_level_kernel<TIn, 8>, grid, block, 0, L.stream, L.X, L.rows, L.cols,
                            L.nblk, L.codes, L.iscales, L.oscales, L.qdq, L.status);
        case 512:
            return launch_k(two_level_kernel<TIn, 16>, grid, block, 0, L.stream, L.X, L.rows,
                            L.cols, L.nblk, L.codes, L.iscales, L.oscales, L.qdq, L.status);
        case 1024:
            return launch_k(two_level_kernel<TIn, 32>, grid, block, 0, L.stream, L.X, L.rows,
                            L.cols, L.nblk, L.codes, L.iscales, L.oscales, L.qdq, L.status);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_two_level(const TwoLevelLaunch &L) {
    return L.f32 ? launch_typed<float>(L) : launch_typed<uint16_t>(L);
}

}  // namespace dq
