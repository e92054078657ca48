// dq_device.cuh — device side of the dual-scale solver: format units, the
// streaming tile kernel (row statistics, column statistics, pack, activation)
// and the small finalize kernels.
//
// Method: DualQuant, daiwk.github.io reproduction note, section "核心公式":
// eq. (1) W ~= D_a Q(D_a^-1 W D_b^-1) D_b, eq. (2) the closed-form row and
// column updates, and the order stated under eq. (2) (row update, re-quantize,
// column update, re-quantize; zero-code slice -> scale 1; projected inverse
// scales).  Formats: same note, "本地复现" (INT4 [-8,7] with BF16 or E8M0
// scales, exponent in [-126,126]); news.yiqijian.com article (MXFP4: E2M1 in
// blocks of 32 with an E8M0 scale; NVFP4: E2M1 in blocks of 16 with an E4M3
// scale).
//
// Exactness.  Every rounding decision (group scale, code) equals the decision
// on the exact real value W_ij / (a_i b_j s ts).  The fast path computes it in
// float32; when the float32 value lies within a few ulps of a decision
// boundary the kernel settles the decision with an fma whose sign is exact
// (the products a_i*b_j*s are exact in float32 for the formats here: at most
// 8+8+8 significant bits).  Power-of-two scalings are exact and skip the check.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace dq {

enum { CODES_INT4 = 0, CODES_E2M1 = 1, CODES_INT8 = 2, CODES_E4M3 = 3, CODES_E5M2 = 4,
       CODES_E2M3 = 5, CODES_E3M2 = 6 };
enum { SC_BF16 = 0, SC_E8M0 = 1, SC_E4M3 = 2 };
// MODE_FUSED_W2 / MODE_ROW_W2: MODE_FUSED / MODE_ROW that also sum each
// row's squares (the first iteration of a solve with 4-bit codes, and the
// row step entry point; see the tile kernel)
enum { MODE_ROW = 0, MODE_COL = 1, MODE_PACK = 2, MODE_ACT = 3, MODE_FUSED = 4, MODE_FUSED_W2 = 5,
       MODE_ROW_W2 = 6 };
enum { STATUS_NONFINITE = 1u, STATUS_RANGE = 2u, STATUS_TIMEOUT = 4u };

constexpr int kWarps = 8;            // warps per CTA of the tile kernel
constexpr int kThreads = 32 * kWarps;
constexpr int kRowsPerWarp[7] = {128, 256, 128, 128, 256, 256, 128};   // per mode (at most)
constexpr int kRowFinRows = 256;     // rows per block of the row finalize
constexpr int kRing = 4;             // cp.async ring slots per lane (rows in flight + 1)
constexpr float kBf16Max = 3.38953138925153547590470800371487866880e+38f;  // (2-2^-7)*2^127
constexpr float kMinNormal = 1.17549435082228750796873653722224568e-38f;    // 2^-126

// Element grid of each code type.  qmax = the largest code magnitude =
// (1 + kMT / 2^23) * 2^kQE; kBits stored bits per code.  INT4 and E2M1 are
// the pages' codebooks; INT8, E4M3, E5M2 (MXFP8), E2M3 and E3M2 (MXFP6) are
// the other element formats of the MX family (OCP Microscaling definition).
template <int CODES> struct CodeTraits;
template <> struct CodeTraits<CODES_INT4> {
    static constexpr float kQmax = 7.0f;   static constexpr int kQE = 2;  static constexpr uint32_t kMT = 0x600000u; static constexpr int kBits = 4; };
template <> struct CodeTraits<CODES_E2M1> {
    static constexpr float kQmax = 6.0f;   static constexpr int kQE = 2;  static constexpr uint32_t kMT = 0x400000u; static constexpr int kBits = 4; };
template <> struct CodeTraits<CODES_INT8> {
    static constexpr float kQmax = 127.0f; static constexpr int kQE = 6;  static constexpr uint32_t kMT = 0x7E0000u; static constexpr int kBits = 8; };
template <> struct CodeTraits<CODES_E4M3> {
    static constexpr float kQmax = 448.0f; static constexpr int kQE = 8;  static constexpr uint32_t kMT = 0x600000u; static constexpr int kBits = 8; };
template <> struct CodeTraits<CODES_E5M2> {
    static constexpr float kQmax = 57344.0f; static constexpr int kQE = 15; static constexpr uint32_t kMT = 0x600000u; static constexpr int kBits = 8; };
template <> struct CodeTraits<CODES_E2M3> {
    static constexpr float kQmax = 7.5f;   static constexpr int kQE = 2;  static constexpr uint32_t kMT = 0x700000u; static constexpr int kBits = 6; };
template <> struct CodeTraits<CODES_E3M2> {
    static constexpr float kQmax = 28.0f;  static constexpr int kQE = 4;  static constexpr uint32_t kMT = 0x600000u; static constexpr int kBits = 6; };

// Programmatic dependent launch.  The library launches its kernels with
// programmatic stream serialization, so a kernel may start while the one
// before it on the stream is finishing.  Every kernel therefore first waits
// for the grids it depends on to complete (their writes are then visible),
// before it reads or writes global memory, and then lets the next kernel of
// the stream launch early (its blocks wait in the same way).
__device__ __forceinline__ void grid_dependency_begin() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// One matrix of a launch.  Tiles of mode m of this matrix are the global
// tiles [tile0[m], tile0[m] + ntiles[m]); a tile is tr[m] rows by
// wc * 32 * EPC columns (EPC = 16 bytes of input per lane).
struct MatDesc {
    const void *W;
    int64_t rows, cols;
    const float *a;          // state a (NULL: ones)
    const float *b;          // state b (NULL: ones)
    float *a_out, *b_out;    // finalize outputs
    float *a_pre, *b_pre;    // unprojected ratios (may be NULL)
    uint8_t *codes;
    void *gscales;
    const float *ts_ptr;     // tensor scale (device) or NULL: use ts_val
    float ts_val;
    int32_t wc;              // warps across columns (1, 2, 4, 8)
    int32_t ncb;             // column blocks
    int32_t tr[3];           // rows per tile: ROW, COL, PACK/ACT
    int64_t tile0[3];
    int64_t ntiles[3];
    int64_t row0, col0;      // global row / column offsets (finalize kernels)
    int64_t cunit0;          // global offset of its work units (column finalize)
    int64_t rchunk0;         // global offset of its 256-row chunks (row finalize)
    float2 *rowpart;         // [rows][ncb]  (num, den)
    float *rowsq;            // [rows][ncb]  sum of W^2 (MODE_FUSED_W2)
    double *w2row;           // [rows]  sum of W^2 per row (4-bit MX one-pass path)
    double *mse_part;        // [ceil(rows / 256)]  squared error of each 256-row chunk (same)
    float2 *colpart;         // [nrb_col][cols]  (P, E)
    double *res_row;         // [ntiles ROW]  residual partials (also PACK)
    double *res_col;         // [ntiles COL]
    unsigned int *amax;      // 1 word (tensor-scale pass)
    float *ts_out;           // tensor scale output
    const float *a0, *b0;    // initial state (init kernel)
    double *mse_trace, *mse_half;
};

struct Table {
    const MatDesc *dev;      // n entries in device memory, or NULL when n == 1
    MatDesc one;             // the single entry when dev == NULL
    int n;
    unsigned int *status;    // device flag word (STATUS_*)
    __device__ __forceinline__ const MatDesc &get(int i) const { return dev ? dev[i] : one; }
};

// Index of the matrix owning global item `t` (tiles, rows or columns), given
// a monotone per-matrix start offset.
template <class F>
__device__ __forceinline__ int find_owner(const Table &tab, int64_t t, F start) {
    if (tab.dev == nullptr) return 0;
    int lo = 0, hi = tab.n - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (start(tab.dev[mid]) <= t) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// ------------------------------------------------------------------------- //
// small float helpers
// ------------------------------------------------------------------------- //

__device__ __forceinline__ float pow2f(int e) {            // 2^e, e in [-126, 127]
    return __uint_as_float((uint32_t)(e + 127) << 23);
}
__device__ __forceinline__ int ilog2f(float x) {            // floor(log2 x), x normal > 0
    return (int)((__float_as_uint(x) >> 23) & 0xFF) - 127;
}
__device__ __forceinline__ float max_nan(float a, float b) {
    float r;
    asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ uint32_t cvt_e2m1x2(float hi, float lo) {
    uint16_t r;
    asm("{ .reg .b8 t; cvt.rn.satfinite.e2m1x2.f32 t, %1, %2; cvt.u16.u8 %0, t; }"
        : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}
__device__ __forceinline__ float2 e2m1x2_to_f32(uint32_t byte) {  // .x = low nibble
    uint32_t h2;
    uint16_t b16 = (uint16_t)byte;
    asm("{ .reg .b8 t; cvt.u8.u16 t, %1; cvt.rn.f16x2.e2m1x2 %0, t; }" : "=r"(h2) : "h"(b16));
    float lo, hi;
    asm("{ .reg .f16 l, h; mov.b32 {l, h}, %2; cvt.f32.f16 %0, l; cvt.f32.f16 %1, h; }"
        : "=f"(lo), "=f"(hi) : "r"(h2));
    return make_float2(lo, hi);
}
// Round a pair to E2M1 (nearest even, saturating) and return the code values
// as float32 (.x from lo, .y from hi), optionally with the code byte.
__device__ __forceinline__ float2 e2m1_round2(float lo, float hi) {
    float a, b;
    asm("{ .reg .b8 t; .reg .b32 p; .reg .f16 l, h;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t, %3, %2;\n\t"
        "cvt.rn.f16x2.e2m1x2 p, t;\n\t"
        "mov.b32 {l, h}, p;\n\t"
        "cvt.f32.f16 %0, l;\n\t"
        "cvt.f32.f16 %1, h; }"
        : "=f"(a), "=f"(b) : "f"(lo), "f"(hi));
    return make_float2(a, b);
}
__device__ __forceinline__ float2 e2m1_round2_byte(float lo, float hi, uint32_t &byte) {
    float a, b;
    asm("{ .reg .b8 t; .reg .b32 p; .reg .f16 l, h;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t, %4, %3;\n\t"
        "cvt.u32.u8 %2, t;\n\t"
        "cvt.rn.f16x2.e2m1x2 p, t;\n\t"
        "mov.b32 {l, h}, p;\n\t"
        "cvt.f32.f16 %0, l;\n\t"
        "cvt.f32.f16 %1, h; }"
        : "=f"(a), "=f"(b), "=r"(byte) : "f"(lo), "f"(hi));
    return make_float2(a, b);
}

// Round a pair to an MX float element format (nearest even, saturating at
// the largest finite value) and return the values as float32 (.x from lo);
// `pair` receives the two codes, lo's in bits 0-7 and hi's in bits 8-15 (a
// 6-bit code sits in the low bits of its byte).
template <int CODES>
__device__ __forceinline__ float2 fp_elem_round2(float lo, float hi, uint32_t &pair) {
    uint16_t b;
    uint32_t h2;
    if constexpr (CODES == CODES_E4M3) {
        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(b) : "f"(hi), "f"(lo));
        asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(b));
    } else if constexpr (CODES == CODES_E5M2) {
        asm("cvt.rn.satfinite.e5m2x2.f32 %0, %1, %2;" : "=h"(b) : "f"(hi), "f"(lo));
        asm("cvt.rn.f16x2.e5m2x2 %0, %1;" : "=r"(h2) : "h"(b));
    } else if constexpr (CODES == CODES_E2M3) {
        asm("cvt.rn.satfinite.e2m3x2.f32 %0, %1, %2;" : "=h"(b) : "f"(hi), "f"(lo));
        asm("cvt.rn.f16x2.e2m3x2 %0, %1;" : "=r"(h2) : "h"(b));
    } else {
        static_assert(CODES == CODES_E3M2, "float element formats only");
        asm("cvt.rn.satfinite.e3m2x2.f32 %0, %1, %2;" : "=h"(b) : "f"(hi), "f"(lo));
        asm("cvt.rn.f16x2.e3m2x2 %0, %1;" : "=r"(h2) : "h"(b));
    }
    pair = b;
    float x, y;
    asm("{ .reg .f16 l, h; mov.b32 {l, h}, %2; cvt.f32.f16 %0, l; cvt.f32.f16 %1, h; }"
        : "=f"(x), "=f"(y) : "r"(h2));
    return make_float2(x, y);
}

// Pack NP code pairs (8-bit codes in bits 0-7 and 8-15) into the stored
// code words: 8-bit codes one per byte; 6-bit codes four per 24-bit
// little-endian word (the first in the low bits), 3 bytes per 4 codes.
template <int BITS, int NP>
__device__ __forceinline__ void pack_code_pairs(const uint32_t (&pair)[NP], uint32_t (&cw)[2]) {
    if constexpr (BITS == 8) {
#pragma unroll
        for (int k = 0; k < NP; ++k) cw[k >> 1] |= pair[k] << (16 * (k & 1));
    } else {
        static_assert(BITS == 6 && (NP == 2 || NP == 4), "6-bit codes come in quads");
        uint32_t wq[NP / 2];
#pragma unroll
        for (int k = 0; k < NP / 2; ++k) {
            const uint32_t p0 = pair[2 * k], p1 = pair[2 * k + 1];
            wq[k] = (p0 & 0x3Fu) | (((p0 >> 8) & 0x3Fu) << 6) | ((p1 & 0x3Fu) << 12) |
                    (((p1 >> 8) & 0x3Fu) << 18);
        }
        if constexpr (NP == 4) {
            cw[0] = wq[0] | (wq[1] << 24);
            cw[1] = wq[1] >> 8;
        } else {
            cw[0] = wq[0];
        }
    }
}
__device__ __forceinline__ uint32_t e4m3_bits(float x) {    // x exactly representable
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(x));
    return r & 0xFF;
}

// 1/x for a normal power of two x (exact)
__device__ __forceinline__ float recip_pow2(float x) {
    return __uint_as_float(0x7F000000u - __float_as_uint(x));
}
// 1/x within about one ulp (only feeds estimates that are checked against
// exact boundaries)
__device__ __forceinline__ float recip_approx(float x) {
    float r;
    asm("rcp.approx.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

template <int LPG>
__device__ __forceinline__ float grp_max(float v) {
#pragma unroll
    for (int o = 1; o < LPG; o <<= 1) v = max_nan(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
template <int LPG>
__device__ __forceinline__ int grp_or(int v) {
#pragma unroll
    for (int o = 1; o < LPG; o <<= 1) v |= __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// ------------------------------------------------------------------------- //
// Group-scale projection P_grp(m / (qmax ts)) with a boundary description
// ------------------------------------------------------------------------- //

struct ScaleChoice {
    float s;          // fast-path choice
    float s_lo, s_hi; // the two candidates around the nearby boundary
    float s_tie;      // the choice when the exact value sits on the boundary
    float thr;        // group max m at the boundary (exact float)
    bool near;        // fast path within tolerance of the boundary
};

// m > 0 finite.  qts = qmax*ts (exact), rqts ~ 1/qts.
template <int GS, int CODES>
__device__ __forceinline__ ScaleChoice project_group(float m, float qts, float rqts, float inv_ts) {
    ScaleChoice c;
    c.near = false;
    c.thr = 0.f;
    if (GS == SC_E8M0) {
        // smallest 2^e with qmax * 2^e >= m/ts, e in [-126, 126]
        float mm = m * inv_ts;                         // exact (power of two)
        int e;
        if (mm < kMinNormal) {
            e = -126;
            c.s_lo = c.s_hi = c.s_tie = c.s = pow2f(e);
            return c;
        }
        uint32_t u = __float_as_uint(mm);
        int k = ilog2f(mm);
        uint32_t mant = u & 0x7FFFFFu;
        constexpr uint32_t MT = CodeTraits<CODES>::kMT;
        constexpr int QE = CodeTraits<CODES>::kQE;
        e = k - QE + (mant > MT ? 1 : 0);
        int elo = min(max(k - QE, -126), 126), ehi = min(max(k - QE + 1, -126), 126);
        e = min(max(e, -126), 126);
        c.s = pow2f(e);
        c.s_lo = pow2f(elo);
        c.s_hi = pow2f(ehi);
        c.s_tie = c.s_lo;                              // m == qmax*2^(k-QE): ceil is exact
        int d = (int)mant - (int)MT;
        c.near = (d < 16 && d > -16);
        c.thr = __uint_as_float((u & 0xFF800000u) | MT) * (1.0f / inv_ts);  // Q*2^k*ts
        return c;
    } else if (GS == SC_BF16) {
        float g = m * rqts;
        if (g < kMinNormal) { c.s = c.s_lo = c.s_hi = c.s_tie = kMinNormal; return c; }
        if (g >= kBf16Max) { c.s = c.s_lo = c.s_hi = c.s_tie = kBf16Max; return c; }
        uint32_t u = __float_as_uint(g);
        uint32_t lo = u & 0xFFFF0000u, low = u & 0xFFFFu;
        float flo = __uint_as_float(lo);
        float fhi = fminf(__uint_as_float(lo + 0x10000u), kBf16Max);
        bool odd = (lo & 0x10000u) != 0;
        c.s_lo = flo;
        c.s_hi = fhi;
        c.s_tie = odd ? fhi : flo;
        c.s = (low > 0x8000u || (low == 0x8000u && odd)) ? fhi : flo;
        int d = (int)low - 0x8000;
        c.near = (d < 16 && d > -16);
        c.thr = __uint_as_float(lo | 0x8000u) * qts;   // 9 bits x qmax*ts: exact
        return c;
    } else {  // E4M3, round to nearest even, saturating at 448, 0 -> 2^-9
        float g = m * rqts;
        if (g >= 448.0f) { c.s = c.s_lo = c.s_hi = c.s_tie = 448.0f; return c; }
        int E = (g < 0.015625f) ? -6 : ilog2f(g);      // 2^-6: smallest normal
        float quant = pow2f(E - 3);
        float t = g * pow2f(3 - E);                    // exact
        float fl = floorf(t);
        float frac = t - fl;
        float slo = fl * quant, shi = (fl + 1.0f) * quant;
        if (slo == 0.0f) slo = 0.001953125f;           // 2^-9
        shi = fminf(shi, 448.0f);
        c.s_lo = slo;
        c.s_hi = shi;
        bool odd = (((int)fl) & 1) != 0;
        c.s_tie = odd ? shi : slo;
        c.s = (frac > 0.5f || (frac == 0.5f && odd)) ? shi : slo;
        c.near = fabsf(frac - 0.5f) <= t * 1.9073486e-06f;   // t * 2^-19
        c.thr = (fl + 0.5f) * quant * qts;
        return c;
    }
}

// The fast-path choice of project_group alone: the same scale s and the
// same `near` flag, without the boundary description (which project_group
// computes when a group does sit near its boundary).
template <int GS, int CODES>
__device__ __forceinline__ float project_group_fast(float m, float rqts, float inv_ts, bool &near) {
    near = false;
    if (GS == SC_E8M0) {
        const float mm = m * inv_ts;                   // exact (power of two)
        if (mm < kMinNormal) return pow2f(-126);
        const uint32_t u = __float_as_uint(mm);
        constexpr uint32_t MT = CodeTraits<CODES>::kMT;
        constexpr int QE = CodeTraits<CODES>::kQE;
        const int mant = (int)(u & 0x7FFFFFu);
        const int e = ilog2f(mm) - QE + (mant > (int)MT ? 1 : 0);
        const int d = mant - (int)MT;
        near = d < 16 && d > -16;
        return pow2f(min(max(e, -126), 126));
    } else if (GS == SC_BF16) {
        const float g = m * rqts;
        if (g < kMinNormal) return kMinNormal;
        if (g >= kBf16Max) return kBf16Max;
        // round to nearest even at the bfloat16 position (g < kBf16Max, so
        // the rounded value stays finite and at most kBf16Max)
        const uint32_t u = __float_as_uint(g);
        const int d = (int)(u & 0xFFFFu) - 0x8000;
        near = d < 16 && d > -16;
        return __uint_as_float((u + 0x7FFFu + ((u >> 16) & 1u)) & 0xFFFF0000u);
    } else {  // E4M3, round to nearest even, saturating at 448, 0 -> 2^-9
        const float g = m * rqts;
        if (g >= 448.0f) return 448.0f;
        const int E = (g < 0.015625f) ? -6 : ilog2f(g);
        const float t = g * pow2f(3 - E);              // exact
        const float frac = t - floorf(t);
        near = fabsf(frac - 0.5f) <= t * 1.9073486e-06f;
        const float s = rintf(t) * pow2f(E - 3);       // ties to even, as project_group
        return s == 0.0f ? 0.001953125f : fminf(s, 448.0f);
    }
}

// ------------------------------------------------------------------------- //
// Packed float32x2 helpers (sm_100 FFMA2 / FMUL2)
// ------------------------------------------------------------------------- //

typedef float2 f2;
__device__ __forceinline__ f2 mul2(f2 a, f2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ f2 fma2(f2 a, f2 b, f2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ f2 bcast(float v) { return make_float2(v, v); }
__device__ __forceinline__ f2 neg2(f2 v) { return make_float2(-v.x, -v.y); }
__device__ __forceinline__ float max3_nan(float a, float b, float c) {
    float r;
    asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// ------------------------------------------------------------------------- //
// Quantization of one lane's chunk: NP pairs of consecutive elements of a row
// ------------------------------------------------------------------------- //

template <int CODES, int GS, int OS, bool ACT, int NP, int LPG>
struct Quant {
    // a second-level tensor scale exists only with E4M3 group scales (NVFP4)
    static constexpr bool kHasTs = GS == SC_E4M3;
    // exact fast path: all scalings are powers of two
    static constexpr bool kExactQ = ACT ? (GS == SC_E8M0) : (GS == SC_E8M0 && OS == SC_E8M0);
    // exact group max (the inner scaling by b, and by a, is exact)
    static constexpr bool kExactM = ACT ? true : (OS == SC_E8M0);
    static constexpr float kQmax = CodeTraits<CODES>::kQmax;
    static constexpr int kBits = CodeTraits<CODES>::kBits;

    // Bits of the E8M0 group scale of an exact, finite group max with bits
    // mb: the smallest 2^e with qmax 2^e >= m, e = E(m) - E(qmax), plus 1
    // when m's significand exceeds qmax's (the carry of the addition adds it
    // to the exponent field); at least 2^-126 (also for subnormal and zero
    // m).  Non-decreasing in mb over finite values.
    __device__ __forceinline__ static uint32_t e8m0_scale_bits(uint32_t mb) {
        constexpr uint32_t MT = CodeTraits<CODES>::kMT;
        constexpr int QE = CodeTraits<CODES>::kQE;
        return (uint32_t)max((int)((mb + (0x7FFFFFu - MT)) & 0x7F800000u) - (QE << 23), 1 << 23);
    }

    // In: w (input values), z = inner-scaled values before the row factor
    // (w/b_j for weights, x*b_j for activations), a and ia = 1/a (1 for ACT),
    // bj (b_j; read on the exact path only), ts and 1/ts (E4M3 only).
    // Out: c (code values), s (stored group scale), s_eff = s*ts, cw (the
    // chunk's stored codes, element 0 lowest, kBits each -- 4-bit codes two
    // per byte, 8-bit codes one per byte, 6-bit codes four per 3 bytes; only
    // when NIB), nonzero (the group max is positive and finite), mbits (the
    // bits of the group max).  UNIT_A: the row factor is 1 (a = ia = 1).
    template <bool NIB, bool UNIT_A = false>
    __device__ __forceinline__ static void run(const f2 (&w)[NP], const f2 (&z)[NP], float a,
                                               float ia, const f2 (&bj)[NP], float ts,
                                               float inv_ts, unsigned int *status, f2 (&c)[NP],
                                               float &s, float &s_eff, uint32_t (&cw)[2],
                                               bool &nonzero, uint32_t &mbits) {
        float mz = 0.0f;
#pragma unroll
        for (int k = 0; k < NP; ++k) mz = max3_nan(mz, fabsf(z[k].x), fabsf(z[k].y));
        mz = grp_max<LPG>(mz);
        const float m = ACT ? mz : mz * ia;
        const uint32_t mb = __float_as_uint(m);
        mbits = mb;
        const bool finite = (mb & 0x7F800000u) != 0x7F800000u;
        // row and column statistics carry a NaN/Inf into their sums, which the
        // finalize kernels flag; the other modes flag it here
        if (NIB && !finite) atomicOr(status, STATUS_NONFINITE);
        const bool pos = finite && m > 0.0f;
        nonzero = pos;
        if (GS == SC_E8M0 && kExactM) {
            // (e <= 126 holds for finite m)
            s = __uint_as_float(e8m0_scale_bits(mb));
            // an all-zero group (also the zero chunks of lanes past the last
            // column) takes scale 1: its stored scale, and, with a row factor,
            // the scale its codes are formed with -- with s at the 2^-126
            // floor, 1 / (a s) would overflow for a <= 1/4 and turn the zeros
            // into NaN (without a row factor 1/s = 2^126 stays finite and the
            // zeros stay zeros)
            if ((NIB || !(ACT || UNIT_A)) && !pos) s = 1.0f;
        } else {
            // every lane takes part in the warp vote and group shuffles below,
            // whatever its group holds (all-zero and out-of-range groups too)
            const float qts = kHasTs ? kQmax * ts : kQmax;
            const float rqts = kHasTs ? 1.0f / qts : 1.0f / kQmax;
            bool near;
            s = project_group_fast<GS, CODES>(pos ? m : 1.0f, rqts, kHasTs ? inv_ts : 1.0f, near);
            const bool resolve = pos && near;
            if (__any_sync(0xffffffffu, resolve)) {
                // exact comparison of the true group max with sc.thr
                const ScaleChoice sc = project_group<GS, CODES>(pos ? m : 1.0f, qts, rqts,
                                                                kHasTs ? inv_ts : 1.0f);
                int gt = 0, eq = 0;
                if (resolve) {
                    if (kExactM) {
                        const float d = m - sc.thr;              // both exact: sign exact
                        gt = d > 0.0f;
                        eq = d == 0.0f;
                    } else {
#pragma unroll
                        for (int k = 0; k < NP; ++k) {
                            const float d0 = fmaf(-sc.thr, a * bj[k].x, fabsf(w[k].x));
                            const float d1 = fmaf(-sc.thr, a * bj[k].y, fabsf(w[k].y));
                            gt |= (d0 > 0.0f) | (d1 > 0.0f);
                            eq |= (d0 == 0.0f) | (d1 == 0.0f);
                        }
                    }
                }
                if (!kExactM) {
                    gt = grp_or<LPG>(gt);
                    eq = grp_or<LPG>(eq);
                }
                if (resolve) s = gt ? sc.s_hi : (eq ? sc.s_tie : sc.s_lo);
            }
            if (!pos) s = 1.0f;
        }
        s_eff = kHasTs ? s * ts : s;
        const float r = (GS == SC_E8M0) ? (ACT ? recip_pow2(s_eff) : ia * recip_pow2(s_eff))
                                        : (ACT ? recip_approx(s_eff) : ia * recip_approx(s_eff));
        f2 q[NP];
#pragma unroll
        for (int k = 0; k < NP; ++k) q[k] = mul2(z[k], bcast(r));
        cw[0] = 0;
        cw[1] = 0;
        if constexpr (CODES == CODES_INT4 || CODES == CODES_INT8) {
            // round half to even; |q| <= qmax (E8M0 round-up) or < qmax + 0.5
            // (BF16 nearest, INT4 only) so the codebook clamp never binds.
            // Adding and subtracting 1.5 * 2^23 rounds any |q| < 2^22 to the
            // nearest integer, ties to even (the sum lies in [2^23, 2^24),
            // where the spacing is 1; the subtraction is exact), on the FMA
            // pipe; a negative q that rounds to zero gives +0, which encodes
            // as the same integer code.
            constexpr float kRound = 12582912.0f;   // 1.5 * 2^23
#pragma unroll
            for (int k = 0; k < NP; ++k)
                c[k] = __fadd2_rn(__fadd2_rn(q[k], bcast(kRound)), bcast(-kRound));
            if (!kExactQ) {
                // largest distance of q from its rounded value: near 0.5 only
                // when some element sits within 2^-16 of a half-integer
                float dmax = 0.0f;
#pragma unroll
                for (int k = 0; k < NP; ++k) {
                    const f2 d = __fadd2_rn(q[k], neg2(c[k]));
                    dmax = max3_nan(dmax, fabsf(d.x), fabsf(d.y));
                }
                // (rare: a warp-uniform branch, so that the fix-up below is
                // not issued for every chunk)
                if (__any_sync(0xffffffffu, dmax > 0.5f - 1.52587890625e-05f)) {
#pragma unroll
                    for (int k = 0; k < NP; ++k)
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const float qq = h ? q[k].y : q[k].x;
                            const float cc = h ? c[k].y : c[k].x;
                            if (fabsf(qq - cc) > 0.5f - 1.52587890625e-05f) {
                                const float aq = fabsf(qq), lo = floorf(aq), mid = lo + 0.5f;
                                const float ww = h ? w[k].y : w[k].x, zz = h ? z[k].y : z[k].x;
                                const float bb = h ? bj[k].y : bj[k].x;
                                const float d = ACT ? fmaf(-mid, s_eff, fabsf(zz))
                                                    : fmaf(-mid, (a * bb) * s_eff, fabsf(ww));
                                const float mag = d > 0.0f ? lo + 1.0f
                                                : (d < 0.0f ? lo : ((((int)lo) & 1) ? lo + 1.0f : lo));
                                const float v = copysignf(mag, qq);
                                if (h) c[k].y = v; else c[k].x = v;
                            }
                        }
                }
            }
            if (NIB) {
                if constexpr (kBits == 4) {
#pragma unroll
                    for (int k = 0; k < NP; ++k)
                        cw[0] |= ((((uint32_t)(int)c[k].x) & 0xFu) |
                                  ((((uint32_t)(int)c[k].y) & 0xFu) << 4)) << (8 * k);
                } else {
                    uint32_t pair[NP];
#pragma unroll
                    for (int k = 0; k < NP; ++k)
                        pair[k] = (((uint32_t)(int)c[k].x) & 0xFFu) |
                                  ((((uint32_t)(int)c[k].y) & 0xFFu) << 8);
                    pack_code_pairs<kBits, NP>(pair, cw);
                }
            }
        } else if constexpr (CODES == CODES_E2M1) {
            if (kExactQ && !NIB) {
#pragma unroll
                for (int k = 0; k < NP; ++k) c[k] = e2m1_round2(q[k].x, q[k].y);
            } else {
                uint32_t byte[NP];
#pragma unroll
                for (int k = 0; k < NP; ++k) c[k] = e2m1_round2_byte(q[k].x, q[k].y, byte[k]);
                if (!kExactQ) {
                    // a code is near a decision boundary when q scaled by
                    // 1 +- 2^-17 rounds to two different codes; such codes
                    // (rare) are settled exactly behind one warp-uniform branch
                    const f2 up = bcast(1.0f + 7.62939453125e-06f), dn = bcast(1.0f - 7.62939453125e-06f);
                    uint32_t bh[NP], bl[NP];
                    bool any_near = false;
#pragma unroll
                    for (int k = 0; k < NP; ++k) {
                        const f2 qh = mul2(q[k], up), ql = mul2(q[k], dn);
                        bh[k] = cvt_e2m1x2(qh.y, qh.x);
                        bl[k] = cvt_e2m1x2(ql.y, ql.x);
                        any_near |= bh[k] != bl[k];
                    }
                    if (__any_sync(0xffffffffu, any_near)) {
#pragma unroll
                    for (int k = 0; k < NP; ++k) {
                        if (bh[k] != bl[k]) {
#pragma unroll
                            for (int h = 0; h < 2; ++h) {
                                const uint32_t nh = (bh[k] >> (4 * h)) & 0xF, nl = (bl[k] >> (4 * h)) & 0xF;
                                if (nh != nl) {
                                    const float2 vh = e2m1x2_to_f32(nh), vl = e2m1x2_to_f32(nl);
                                    const float mh = fabsf(vh.x), ml = fabsf(vl.x);
                                    const float mid = 0.5f * (mh + ml);
                                    const float ww = h ? w[k].y : w[k].x, zz = h ? z[k].y : z[k].x;
                                    const float bb = h ? bj[k].y : bj[k].x, qq = h ? q[k].y : q[k].x;
                                    const float d = ACT ? fmaf(-mid, s_eff, fabsf(zz))
                                                        : fmaf(-mid, (a * bb) * s_eff, fabsf(ww));
                                    // the even code of the two neighbours has mantissa bit 0
                                    const float even = ((nh & 1u) == 0) ? mh : ml;
                                    const float mag = d > 0.0f ? mh : (d < 0.0f ? ml : even);
                                    const float v = copysignf(mag, qq);
                                    const uint32_t nn = cvt_e2m1x2(0.0f, v) & 0xF;
                                    byte[k] = (byte[k] & ~(0xFu << (4 * h))) | (nn << (4 * h));
                                    if (h) c[k].y = v; else c[k].x = v;
                                }
                            }
                        }
                    }
                    }
                }
                if (NIB) {
#pragma unroll
                    for (int k = 0; k < NP; ++k) cw[0] |= byte[k] << (8 * k);
                }
            }
        } else {
            // MX float elements (E4M3, E5M2, E2M3, E3M2): with power-of-two
            // scales q is exact, so the hardware conversion decides each code
            static_assert(kExactQ, "float element codes need power-of-two scales");
            uint32_t pair[NP];
#pragma unroll
            for (int k = 0; k < NP; ++k) c[k] = fp_elem_round2<CODES>(q[k].x, q[k].y, pair[k]);
            if constexpr (NIB) pack_code_pairs<kBits, NP>(pair, cw);
        }
    }
};

// ------------------------------------------------------------------------- //
// Loading one lane's chunk (16 bytes)
// ------------------------------------------------------------------------- //

template <typename TIn> struct Chunk;
template <> struct Chunk<float> {
    static constexpr int EPC = 4;
    uint4 raw;
    __device__ __forceinline__ void load(const void *p) {
        raw = __ldg(reinterpret_cast<const uint4 *>(p));
    }
    __device__ __forceinline__ void zero() { raw = make_uint4(0, 0, 0, 0); }
    __device__ __forceinline__ void unpack(float (&w)[4]) const {
        w[0] = __uint_as_float(raw.x); w[1] = __uint_as_float(raw.y);
        w[2] = __uint_as_float(raw.z); w[3] = __uint_as_float(raw.w);
    }
    __device__ __forceinline__ void unpack2(f2 (&w)[2]) const {
        w[0] = make_float2(__uint_as_float(raw.x), __uint_as_float(raw.y));
        w[1] = make_float2(__uint_as_float(raw.z), __uint_as_float(raw.w));
    }
};
struct Bf16Tag {};
template <> struct Chunk<Bf16Tag> {
    static constexpr int EPC = 8;
    uint4 raw;
    __device__ __forceinline__ void load(const void *p) {
        raw = __ldg(reinterpret_cast<const uint4 *>(p));
    }
    __device__ __forceinline__ void zero() { raw = make_uint4(0, 0, 0, 0); }
    __device__ __forceinline__ void unpack(float (&w)[8]) const {
        const uint32_t v[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            w[2 * k] = __uint_as_float(v[k] << 16);
            w[2 * k + 1] = __uint_as_float(v[k] & 0xFFFF0000u);
        }
    }
    __device__ __forceinline__ void unpack2(f2 (&w)[4]) const {
        const uint32_t v[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int k = 0; k < 4; ++k)
            w[k] = make_float2(__uint_as_float(v[k] << 16), __uint_as_float(v[k] & 0xFFFF0000u));
    }
};

__device__ __forceinline__ float tensor_scale_of(const MatDesc &md) {
    return md.ts_ptr ? *md.ts_ptr : md.ts_val;
}

// Projection of an outer inverse scale onto its set (nearest value).
template <int OS>
__device__ __forceinline__ float project_outer(float x, bool &clamped) {
    clamped = false;
    if (OS == SC_E8M0) {
        // nearest power of two, midpoint 1.5*2^k, tie up; exponent in [-126, 126]
        if (x < kMinNormal) { clamped = true; return kMinNormal; }
        uint32_t u = __float_as_uint(x);
        int k = ilog2f(x) + (((u & 0x7FFFFFu) >= 0x400000u) ? 1 : 0);
        if (k > 126) { clamped = true; k = 126; }
        if (k < -126) { clamped = true; k = -126; }
        return pow2f(k);
    } else {
        // bfloat16 round to nearest even, clamped to [2^-126, max]
        if (!(x < kBf16Max)) { clamped = true; return kBf16Max; }
        uint32_t u = __float_as_uint(x);
        uint32_t r = (u + 0x7FFFu + ((u >> 16) & 1u)) & 0xFFFF0000u;
        float v = __uint_as_float(r);
        if (v < kMinNormal) { clamped = true; v = kMinNormal; }
        if (!(v <= kBf16Max)) { clamped = true; v = kBf16Max; }
        return v;
    }
}

// ------------------------------------------------------------------------- //
// The streaming tile kernel
// ------------------------------------------------------------------------- //
//
// CTA = 8 warps = wr x wc (wc warps across columns).  Warp (r, c) handles the
// tile's rows r, r + wr, r + 2 wr, ... of column segment c (32 lanes x EPC
// columns).  Each lane keeps b_j and 1/b_j of its EPC columns in registers
// for the whole tile; arithmetic runs on float32 pairs (FFMA2/FMUL2).
//   ROW : per row, sum_j W_ij R_ij and sum_j R_ij^2 (R = Qhat D_b) over the
//         tile's columns -> rowpart[row][cb]; residual of the state -> res_row
//         (wider than 4-bit codes; for 4-bit codes the row finalize forms
//         it from the row sums)
//   COL : per column, sum_i W_ij S_ij and sum_i S_ij^2 (S = D_a Qhat) over the
//         tile's rows -> colpart[rb][col]; residual -> res_col
//   FUSED (power-of-two scales): ROW and COL from one quantization
//   ROW_W2, FUSED_W2 (4-bit codes): also sum_j W_ij^2 per row -> rowsq[row][cb]
//   PACK: codes and group scales of Q(W / (a b)); residual -> res_row
//   ACT : codes and group scales of Q(X * b)
// Tiles have up to kRowsPerWarp[mode] rows per warp (the host picks fewer for
// short matrices).  `want_res` = 0 skips the residual (its MSE output was
// not requested).
// Shared memory of one tile CTA, by mode.
template <int MODE, int EPC>
struct TileSmem {
    static constexpr int RPW = kRowsPerWarp[MODE];
    static constexpr bool kFused = MODE == MODE_FUSED || MODE == MODE_FUSED_W2;
    static constexpr bool kRowM = MODE == MODE_ROW || MODE == MODE_ROW_W2;
    static constexpr bool kW2 = MODE == MODE_FUSED_W2 || MODE == MODE_ROW_W2;
    // ROW, FUSED: per (warp, row of a batch of 8, lane) partial (num, den),
    // reduced every 8 rows.  Row stride padded by one entry.
    static constexpr int kRed = (kRowM || kFused) ? kWarps * 8 * 33 : 1;
    // ROW, FUSED: per (row, warp) totals
    static constexpr int kRtot = (kRowM || kFused) ? RPW * kWarps : 1;
    // COL, FUSED: per (warp-row, column) partials
    static constexpr int kPart = (MODE == MODE_COL || kFused) ? kWarps * 32 * EPC : 1;
    float2 red[kRed];
    float2 rtot[kRtot];
    float2 part[kPart];
    // FUSED_W2: the same two stages for the sums of squares
    float red2[kW2 ? kRed : 1];
    float rtot2[kW2 ? kRtot : 1];
    double res[kWarps];
    uint4 ring[kWarps][kRing][32];
};

// Column statistics keep 2 x EPC accumulators per lane: those modes run 2
// CTAs per SM (up to 128 registers), the others 3.
template <int MODE> struct TileOcc {
    static constexpr int kMinBlocks = (MODE == MODE_COL || MODE == MODE_FUSED || MODE == MODE_FUSED_W2) ? 2 : 3;   // (ROW_W2: 3)
};

template <int CODES, int GS, int OS, int MODE, typename TIn, int G>
__global__ void __launch_bounds__(kThreads, TileOcc<MODE>::kMinBlocks)
tile_kernel(const __grid_constant__ Table tab, int mode_slot, int want_res, int64_t total_tiles,
            unsigned int *flags, int gate) {
    grid_dependency_begin();
    using CK = Chunk<TIn>;
    constexpr int EPC = CK::EPC;
    constexpr int NP = EPC / 2;
    constexpr int SEG = 32 * EPC;
    constexpr int LPG = G / EPC;
    constexpr bool ACT = MODE == MODE_ACT;
    constexpr bool NIB = MODE == MODE_PACK || MODE == MODE_ACT;
    constexpr bool FUSED = MODE == MODE_FUSED || MODE == MODE_FUSED_W2;
    constexpr bool ROWM = MODE == MODE_ROW || MODE == MODE_ROW_W2;
    constexpr bool W2 = MODE == MODE_FUSED_W2 || MODE == MODE_ROW_W2;
    // 4-bit codes: the squared error of the state is taken per row from its
    // row sums (the row finalize), not summed by the passes with row sums
    constexpr bool kRowMse = (FUSED || ROWM) && CodeTraits<CODES>::kBits == 4;
    static_assert(!W2 || kRowMse, "row sums of squares serve the 4-bit codes");
    constexpr bool ROWSTAT = ROWM || FUSED;
    constexpr bool COLSTAT = MODE == MODE_COL || FUSED;
    using Q = Quant<CODES, GS, OS, ACT, NP, LPG>;
    static_assert(!FUSED || (GS == SC_E8M0 && OS == SC_E8M0), "fused statistics need power-of-two scales");
    constexpr int ESZ = 16 / EPC;                    // bytes per element

    extern __shared__ __align__(16) unsigned char tile_smem[];
    TileSmem<MODE, EPC> &sm = *reinterpret_cast<TileSmem<MODE, EPC> *>(tile_smem);

    // gated launches (the literal fallback of a fused iteration) run only when
    // an earlier kernel of the iteration raised the flag
    if (gate == 1 && flags[0] == 0) return;
    if (gate == 2 && (flags[0] | flags[1]) == 0) return;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool res_on = !ACT && !kRowMse && want_res != 0;

    for (int64_t t = blockIdx.x; t < total_tiles; t += gridDim.x) {
    const int mi = find_owner(tab, t, [mode_slot](const MatDesc &d) { return d.tile0[mode_slot]; });
    const MatDesc &md = tab.get(mi);
    const int64_t lt = t - md.tile0[mode_slot];
    if (lt >= md.ntiles[mode_slot]) continue;        // (uniform per CTA)
    const int wc = md.wc, wr = kWarps / wc;
    // tile rows: up to RPW per warp (fewer for short matrices, so that they
    // still spread over many CTAs)
    const int tr = md.tr[mode_slot];
    const int rpw = tr / wr;
    const int64_t rb = lt / md.ncb, cb = lt % md.ncb;
    const int my_c = warp % wc, my_r = warp / wc;
    const int64_t cols = md.cols, rows = md.rows;
    const int64_t col = (cb * wc + my_c) * (int64_t)SEG + lane * EPC;
    const bool col_ok = col < cols;
    const int64_t row_first = rb * tr;
    const int64_t row0 = row_first + my_r;           // this warp's first row
    // rows of this tile that this warp handles (k = 0 .. nk-1 -> row0 + k*wr)
    const int nk = (int)max((int64_t)0, min((int64_t)rpw, (rows - row0 + wr - 1) / wr));

    // per-lane column data, as pairs: b_j and the inner factor (1/b_j, or b_j for ACT)
    f2 bj[NP], cm[NP];
#pragma unroll
    for (int k = 0; k < NP; ++k) {
        float b0 = 1.0f, b1 = 1.0f;
        if (md.b != nullptr && col_ok) {
            b0 = __ldg(md.b + col + 2 * k);
            b1 = __ldg(md.b + col + 2 * k + 1);
        }
        bj[k] = make_float2(b0, b1);
        if (ACT) cm[k] = bj[k];
        else if (OS == SC_E8M0) cm[k] = make_float2(recip_pow2(b0), recip_pow2(b1));
        else cm[k] = make_float2(recip_approx(b0), recip_approx(b1));
    }
    // row factors a_i are read per row (one cached load per lane)
    const float *const pa = ACT ? nullptr : md.a;

    const float ts = (GS == SC_E4M3 && !ACT) ? tensor_scale_of(md) : 1.0f;
    const float inv_ts = 1.0f / ts;                 // ts is a power of two

    f2 acc_p[NP], acc_e[NP];                         // column accumulators
#pragma unroll
    for (int k = 0; k < NP; ++k) { acc_p[k] = bcast(0.0f); acc_e[k] = bcast(0.0f); }
    f2 res2 = bcast(0.0f);
    // FUSED: smallest (bits - 1, unsigned: zero groups drop out) and largest
    // bits of the lane's group maxima, for the exponent margin check
    uint32_t m_lo = 0xFFFFFFFFu, m_hi = 0u;

    // Each lane streams its own 16-byte chunk of the warp's rows through a
    // private ring of kRing shared-memory slots with cp.async (one commit
    // group per row, kRing - 1 rows in flight); only the lane that copied a
    // slot reads it, so no barrier is needed.  Lanes past the last column
    // never copy: their slots hold zeros.
    if (!col_ok) {
#pragma unroll
        for (int q = 0; q < kRing; ++q) sm.ring[warp][q][lane] = make_uint4(0, 0, 0, 0);
    }
    const int64_t row_step = (int64_t)wr * cols * ESZ;
    const char *src = reinterpret_cast<const char *>(md.W) + (row0 * cols + col) * ESZ;
    const uint32_t ring0 = (uint32_t)__cvta_generic_to_shared(&sm.ring[warp][0][lane]);
    // copy of row k into slot k % kRing (k < nk; lanes past the last column never copy)
    auto issue = [&](int k, int slot) {
        if (k < nk && col_ok) {
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;"
                         :: "r"(ring0 + (uint32_t)(slot * 32 * 16)),
                            "l"(src + (int64_t)k * row_step) : "memory");
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
#pragma unroll
    for (int k = 0; k < kRing - 1; ++k) issue(k, k);

    // One row of the warp: row k, in ring slot u % kRing (u is a constant
    // where the loops below unroll); batch_end closes a batch of 8 rows of
    // the row statistics.
    auto one_row = [&](const int k, const int u, const bool batch_end) {
        issue(k + kRing - 1, (u + kRing - 1) % kRing);
        asm volatile("cp.async.wait_group %0;" :: "n"(kRing - 1) : "memory");
        CK ck;
        ck.raw = sm.ring[warp][u % kRing][lane];
        float a = 1.0f, ia = 1.0f;
        if (!ACT && !FUSED && pa != nullptr) {
            a = __ldg(pa + row0 + (int64_t)k * wr);
            ia = (OS == SC_E8M0) ? recip_pow2(a) : recip_approx(a);
        }
        f2 w[NP], z[NP], c[NP];
        ck.unpack2(w);
#pragma unroll
        for (int j = 0; j < NP; ++j) z[j] = mul2(w[j], cm[j]);
        float s, s_eff;
        uint32_t cw[2], mbits;
        bool nonzero;
        if (FUSED) {
            // Q(W / b): with power-of-two scales D_a Q(W / (a b)) equals it
            // exactly, for the row's a before and after its update, as long
            // as no group exponent of either reaches the E8M0 bounds: here
            // |e(s)| <= 100 for every non-zero group (checked after the
            // tile's rows on the extremes of the group maxima); the row
            // finalize keeps |e(a)| <= 20 (old) and <= 26 (new)
            Q::template run<NIB, true>(w, z, 1.0f, 1.0f, bj, ts, inv_ts, tab.status, c, s, s_eff,
                                       cw, nonzero, mbits);
            m_lo = min(m_lo, mbits - 1u);
            m_hi = max(m_hi, mbits);
        } else {
            Q::template run<NIB>(w, z, a, ia, bj, ts, inv_ts, tab.status, c, s, s_eff, cw,
                                 nonzero, mbits);
        }
        // FUSED: S = Qhat s (a = 1), shared by both statistics
        f2 v[NP];
        if (FUSED) {
#pragma unroll
            for (int j = 0; j < NP; ++j) v[j] = mul2(c[j], bcast(s_eff));
        }
        if (ROWSTAT) {
            // the row statistics of the literal row step: R = Qhat D_b with
            // Qhat = Q(W / (a b)); FUSED writes them for a = 1 and the row
            // finalize scales the sums by 1/a and 1/a^2 (exact: a is a power
            // of two), which gives the literal bits
            // (FUSED takes the group scale into R first: R = (Qhat s) b_j.
            // Scaling by a power of two commutes with rounding, so the
            // sums and the share are the same bits as the literal form's
            // while every value stays in float32's normal range.)
            const float s_row = s_eff;
            f2 gn = bcast(0.0f), gd = bcast(0.0f);
            const f2 nas = bcast(FUSED ? -1.0f : -(a * s_eff));
#pragma unroll
            for (int j = 0; j < NP; ++j) {
                const f2 uq = FUSED ? mul2(v[j], bj[j]) : mul2(c[j], bj[j]);
                gn = fma2(w[j], uq, gn);
                gd = fma2(uq, uq, gd);
                if (res_on) {
                    const f2 d = fma2(nas, uq, w[j]);
                    res2 = fma2(d, d, res2);
                }
            }
            const float2 share =
                FUSED ? make_float2(gn.x + gn.y, gd.x + gd.y)
                      : make_float2((gn.x + gn.y) * s_row, (gd.x + gd.y) * (s_row * s_row));
            // batches of 8 rows: lane 4r + q adds the 8 shares of quarter q
            // of the batch's row r as a fixed tree, then the quarters are
            // added ((q0 + q1) + (q2 + q3), by two shuffle levels) -- one
            // fixed order, the same in every mode with row statistics
            sm.red[(warp * 8 + (k & 7)) * 33 + lane] = share;
            if (W2) {
                // sum of squares of the row, in the order of the sums above
                // (for a row that Q reproduces exactly, R = W and the three
                // sums are the same bits)
                f2 gq = bcast(0.0f);
#pragma unroll
                for (int j = 0; j < NP; ++j) gq = fma2(w[j], w[j], gq);
                sm.red2[(warp * 8 + (k & 7)) * 33 + lane] = gq.x + gq.y;
            }
            if (batch_end) {
                __syncwarp();
                const int rr = lane >> 2, qq = lane & 3;
                const float2 *p = &sm.red[(warp * 8 + rr) * 33 + 8 * qq];
                const f2 s01 = __fadd2_rn(p[0], p[1]), s23 = __fadd2_rn(p[2], p[3]);
                const f2 s45 = __fadd2_rn(p[4], p[5]), s67 = __fadd2_rn(p[6], p[7]);
                f2 acc = __fadd2_rn(__fadd2_rn(s01, s23), __fadd2_rn(s45, s67));
                acc.x += __shfl_xor_sync(0xffffffffu, acc.x, 1);
                acc.y += __shfl_xor_sync(0xffffffffu, acc.y, 1);
                acc.x += __shfl_xor_sync(0xffffffffu, acc.x, 2);
                acc.y += __shfl_xor_sync(0xffffffffu, acc.y, 2);
                const int kk = (k & ~7) + rr;
                if (qq == 0 && kk <= k) sm.rtot[kk * kWarps + warp] = acc;
                if (W2) {
                    const float *q2 = &sm.red2[(warp * 8 + rr) * 33 + 8 * qq];
                    const float t01 = q2[0] + q2[1], t23 = q2[2] + q2[3];
                    const float t45 = q2[4] + q2[5], t67 = q2[6] + q2[7];
                    float sq = (t01 + t23) + (t45 + t67);
                    sq += __shfl_xor_sync(0xffffffffu, sq, 1);
                    sq += __shfl_xor_sync(0xffffffffu, sq, 2);
                    if (qq == 0 && kk <= k) sm.rtot2[kk * kWarps + warp] = sq;
                }
                __syncwarp();
            }
        }
        if (COLSTAT) {
            // the column statistics of the literal column step: S = D_a Qhat
            const f2 as = bcast(a * s_eff);
#pragma unroll
            for (int j = 0; j < NP; ++j) {
                const f2 sv = FUSED ? v[j] : mul2(c[j], as);
                acc_p[j] = fma2(w[j], sv, acc_p[j]);
                acc_e[j] = fma2(sv, sv, acc_e[j]);
                if (!FUSED && res_on) {
                    const f2 d = fma2(sv, bj[j], neg2(w[j]));
                    res2 = fma2(d, d, res2);
                }
            }
        }
        if (NIB) {
            const int64_t r = row0 + (int64_t)k * wr;
            if (MODE == MODE_PACK && res_on) {
                const f2 nas = bcast(-(a * s_eff));
#pragma unroll
                for (int j = 0; j < NP; ++j) {
                    const f2 d = fma2(nas, mul2(c[j], bj[j]), w[j]);
                    res2 = fma2(d, d, res2);
                }
            }
            if (col_ok) {
                // codes: cols * BITS / 8 bytes per row; this lane's EPC codes
                // start at byte col * BITS / 8 (aligned to their size: 4 or
                // 8 bytes for 4- and 8-bit codes, 2 bytes for 6-bit codes
                // in bf16 chunks, 1 byte in float32 chunks)
                constexpr int BITS = CodeTraits<CODES>::kBits;
                uint8_t *cp = md.codes + r * (cols * BITS / 8) + col * BITS / 8;
                if (BITS == 4) {
                    if (EPC == 8) *reinterpret_cast<uint32_t *>(cp) = cw[0];
                    else *reinterpret_cast<uint16_t *>(cp) = (uint16_t)cw[0];
                } else if (BITS == 8) {
                    if (EPC == 8) *reinterpret_cast<uint2 *>(cp) = make_uint2(cw[0], cw[1]);
                    else *reinterpret_cast<uint32_t *>(cp) = cw[0];
                } else if (EPC == 8) {                      // 6-bit codes: 6 bytes
                    uint16_t *cp2 = reinterpret_cast<uint16_t *>(cp);
                    cp2[0] = (uint16_t)cw[0];
                    cp2[1] = (uint16_t)(cw[0] >> 16);
                    cp2[2] = (uint16_t)cw[1];
                } else {                                    // 6-bit codes: 3 bytes
                    cp[0] = (uint8_t)cw[0];
                    cp[1] = (uint8_t)(cw[0] >> 8);
                    cp[2] = (uint8_t)(cw[0] >> 16);
                }
                if ((lane % LPG) == 0) {
                    const int64_t gi = r * (cols / G) + col / G;
                    if (GS == SC_BF16)
                        reinterpret_cast<uint16_t *>(md.gscales)[gi] = (uint16_t)(__float_as_uint(s) >> 16);
                    else if (GS == SC_E8M0)
                        reinterpret_cast<uint8_t *>(md.gscales)[gi] = (uint8_t)((__float_as_uint(s) >> 23) & 0xFF);
                    else
                        reinterpret_cast<uint8_t *>(md.gscales)[gi] = (uint8_t)e4m3_bits(s);
                }
            }
        }
    };
    // full groups of GRP rows as straight-line code (8 in the fused mode; 4
    // in the others, which run 3 CTAs per SM and have fewer registers), then
    // the tail; a batch of the row statistics ends every 8 rows
    constexpr int GRP = FUSED ? 8 : 4;
    int k0 = 0;
#pragma unroll 1
    for (; k0 + GRP <= nk; k0 += GRP) {
        // FUSED: k0 is a multiple of 8 and row k0 + 7 exists, so the group's
        // last row closes the batch and no other row does (a compile-time
        // fact; the other modes keep the run-time test, which the compiler
        // schedules with fewer registers live across rows)
#pragma unroll
        for (int u = 0; u < GRP; ++u)
            one_row(k0 + u, u, FUSED ? u == GRP - 1 : (((k0 + u) & 7) == 7 || k0 + u == nk - 1));
    }
#pragma unroll
    for (int u = 0; u < GRP - 1; ++u) {
        if (k0 + u >= nk) break;                     // warp-uniform
        one_row(k0 + u, u, k0 + u == nk - 1 || ((k0 + u) & 7) == 7);
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    if (FUSED && m_lo != 0xFFFFFFFFu) {
        // some group max is non-zero: its scale must be 2^e with |e| <= 100
        // (exponent field in [27, 227]); the scale bits grow with the max,
        // so the extremes decide; a non-finite max also takes the literal
        // passes (which carry it into the sums as well)
        const uint32_t lo = Q::e8m0_scale_bits(m_lo + 1u), hi = Q::e8m0_scale_bits(m_hi);
        if (lo < (27u << 23) || hi > (227u << 23) || m_hi >= 0x7F800000u) atomicOr(&flags[0], 1u);
    }

    // ---- tile epilogue ----
    if (ROWSTAT) {
        __syncthreads();
        // rows of the tile: local row k*wr + r is warp-row r's k-th row
        for (int lr = threadIdx.x; lr < tr; lr += kThreads) {
            const int k = lr / wr, r = lr % wr;
            const int64_t row = row_first + r + (int64_t)k * wr;
            if (row < rows) {
                float num = 0.0f, den = 0.0f;
                for (int c2 = 0; c2 < wc; ++c2) {          // fixed order over segments
                    float2 p = sm.rtot[k * kWarps + r * wc + c2];
                    num += p.x;
                    den += p.y;
                }
                md.rowpart[row * md.ncb + cb] = make_float2(num, den);
                if (W2) {
                    float sq = 0.0f;
                    for (int c2 = 0; c2 < wc; ++c2) sq += sm.rtot2[k * kWarps + r * wc + c2];
                    md.rowsq[row * md.ncb + cb] = sq;
                }
            }
        }
    }
    if (COLSTAT) {
        if (wr == 1) {
            if (col_ok) {
                float2 *dst = md.colpart + rb * cols + col;
#pragma unroll
                for (int k = 0; k < NP; ++k) {
                    dst[2 * k] = make_float2(acc_p[k].x, acc_e[k].x);
                    dst[2 * k + 1] = make_float2(acc_p[k].y, acc_e[k].y);
                }
            }
        } else {
            // reduce over the wr warp-rows of each segment in fixed order
            const int seg_cols = wc * SEG;
#pragma unroll
            for (int k = 0; k < NP; ++k) {
                const int base = my_r * seg_cols + my_c * SEG + lane * EPC + 2 * k;
                sm.part[base] = make_float2(acc_p[k].x, acc_e[k].x);
                sm.part[base + 1] = make_float2(acc_p[k].y, acc_e[k].y);
            }
            __syncthreads();
            for (int cc = threadIdx.x; cc < seg_cols; cc += kThreads) {
                const int64_t gc = cb * seg_cols + cc;
                if (gc < cols) {
                    float p = 0.0f, e = 0.0f;
                    for (int r = 0; r < wr; ++r) {
                        float2 v = sm.part[r * seg_cols + cc];
                        p += v.x;
                        e += v.y;
                    }
                    md.colpart[rb * cols + gc] = make_float2(p, e);
                }
            }
        }
    }
    if (!ACT && res_on) {
        double rd = (double)res2.x + (double)res2.y;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) rd += __shfl_xor_sync(0xffffffffu, rd, o);
        if (lane == 0) sm.res[warp] = rd;
        __syncthreads();
        double *slot = (MODE == MODE_COL) ? md.res_col : md.res_row;
        if (threadIdx.x == 0 && slot != nullptr) {
            double tot = 0.0;
            for (int k = 0; k < kWarps; ++k) tot += sm.res[k];
            slot[lt] = tot;
        }
    }
    __syncthreads();                                 // shared memory reused by the next tile
    }
}

// ------------------------------------------------------------------------- //
// Finalize kernels
// ------------------------------------------------------------------------- //

// a_i <- Pi(sum num / sum den) over the row's column blocks (fixed order).
// With `flags` (an iteration of the one-pass MX path): unless flags[0] says
// the literal row pass ran, the sums were taken for a = 1 and are scaled by
// 1/a_old and 1/a_old^2 here; a new scale with |e(a)| > 26 raises flags[1]
// (the column step is redone literally) and one with |e(a)| > 20 raises the
// next iteration's flags[0] (its row step is done literally).
// row_mse (the formats with 4-bit codes): the squared error of each row of
// the state, sum_j (W_ij - a_i R_ij)^2 = sum W^2 - 2 a sum W R + a^2 sum
// R^2 from its row sums (the one-pass sums are for a = 1), summed over the
// block's rows in a fixed order -> mse_part[chunk]; row_mse = 2 first sums
// the row's squares from the pass's (rowsq -> w2row), 1 reads them.
// A block handles one 256-row chunk of one matrix at a time (chunks of all
// matrices in order, grid-stride).
template <int OS>
__global__ void __launch_bounds__(kRowFinRows)
row_finalize_kernel(const __grid_constant__ Table tab, int64_t total_chunks, unsigned int *flags,
                    unsigned int *next_flags, int row_mse) {
    grid_dependency_begin();
    __shared__ double wsum[kRowFinRows / 32];
    const bool scale_old = flags != nullptr && flags[0] == 0;
    for (int64_t ch = blockIdx.x; ch < total_chunks; ch += gridDim.x) {
        const int mi = find_owner(tab, ch, [](const MatDesc &d) { return d.rchunk0; });
        const MatDesc &md = tab.get(mi);
        const int64_t r = (ch - md.rchunk0) * kRowFinRows + threadIdx.x;
        double err = 0.0;
        if (r < md.rows) {
            // (the row's old scale and stored sum of squares are loaded ahead
            // of its partial sums)
            const float a_old = ((scale_old || row_mse) && md.a) ? md.a[r] : 1.0f;
            const double w2_old = row_mse == 1 ? md.w2row[r] : 0.0;
            double num = 0.0, den = 0.0;
            const float2 *p = md.rowpart + r * md.ncb;
            // the row's column blocks in order; loads issued a batch ahead of
            // the sums (the order of the sums is unchanged)
            for (int k0 = 0; k0 < md.ncb; k0 += 8) {
                float2 v[8];
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    if (k0 + u < md.ncb) v[u] = __ldg(p + k0 + u);
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    if (k0 + u < md.ncb) { num += v[u].x; den += v[u].y; }
            }
            if (row_mse) {
                double w2 = 0.0;
                if (row_mse == 2) {
                    // the same order as num: for a row that Q reproduces
                    // exactly the three sums are equal and its error is 0
                    const float *q = md.rowsq + r * md.ncb;
                    for (int k = 0; k < md.ncb; ++k) w2 += __ldg(q + k);
                    md.w2row[r] = w2;
                } else {
                    w2 = w2_old;
                }
                // the one-pass sums are for a = 1 (R = D_a Qhat D_b); the
                // literal ones for R = Qhat D_b, whose state is a R
                if (scale_old) {
                    err = (w2 - 2.0 * num) + den;
                } else {
                    const double as = (double)a_old;
                    err = (w2 - 2.0 * as * num) + (as * as) * den;
                }
            }
            if (scale_old) {
                const double ia = (double)recip_pow2(a_old);
                num *= ia;
                den *= ia * ia;
            }
            float a = 1.0f, pre = __int_as_float(0x7fc00000);
            if (den > 0.0) {
                pre = (float)(num / den);
                bool cl;
                a = project_outer<OS>(pre, cl);
                if (cl) atomicOr(tab.status, STATUS_RANGE);
            }
            if (!isfinite(num) || !isfinite(den)) atomicOr(tab.status, STATUS_NONFINITE);
            if (flags != nullptr) {
                const int ea = (int)((__float_as_uint(a) >> 23) & 0xFF) - 127;
                if (ea > 26 || ea < -26) atomicOr(&flags[1], 1u);
                if (ea > 20 || ea < -20) atomicOr(&next_flags[0], 1u);
            }
            md.a_out[r] = a;
            if (md.a_pre) md.a_pre[r] = pre;
        }
        if (row_mse) {                                    // (uniform per block)
            // the chunk's errors in a fixed order: lanes, then warps
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) err += __shfl_xor_sync(0xffffffffu, err, o);
            if ((threadIdx.x & 31) == 0) wsum[threadIdx.x >> 5] = err;
            __syncthreads();
            if (threadIdx.x == 0) {
                double t = 0.0;
                for (int w = 0; w < kRowFinRows / 32; ++w) t += wsum[w];
                md.mse_part[ch - md.rchunk0] = t;
            }
            __syncthreads();
        }
    }
}

// ------------------------------------------------------------------------- //
// MSE reductions (one warp per (matrix, which); 8 per block of 256 threads)
// ------------------------------------------------------------------------- //

// Sum n residual slots in a fixed order (lane l: slots l, l + 32, ... in
// order; then the lanes by a fixed butterfly) and store sum / (rows * cols).
// Called by a whole warp.
__device__ __forceinline__ void mse_reduce_warp(const double *src, int64_t n, double *dst,
                                                const MatDesc &md) {
    const int lane = threadIdx.x & 31;
    double acc = 0.0;
    for (int64_t k = lane; k < n; k += 32) acc += src[k];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) {
        const double cnt = (double)md.rows * (double)md.cols;
        // (a sum of row errors taken from row sums can round below 0 only
        // when the error is 0 up to rounding; a NaN passes)
        const double tot = acc < 0.0 ? 0.0 : acc;
        *dst = cnt > 0 ? tot / cnt : 0.0;
    }
}

// Item blk = 2 mi + which of the MSE of the literal passes: which = 0:
// res_row[ntiles[row_slot]] (or, with row_slot = kSlotRows, the row
// finalize's per-chunk errors mse_part) -> mse_trace[idx_trace] (or
// out_row[mi]); which = 1: res_col[ntiles[COL]] -> mse_half[idx_half] (or
// out_col[mi]).  Called by a whole warp.
constexpr int kSlotRows = 3;
__device__ __forceinline__ void mse_literal_item(const Table &tab, int blk, int row_slot,
                                                 int idx_trace, int idx_half, double *out_row,
                                                 double *out_col) {
    const int mi = blk >> 1, which = blk & 1;
    const MatDesc &md = tab.get(mi);
    double *dst;
    const double *src;
    int64_t n;
    if (which == 0) {
        dst = out_row ? out_row + mi : (md.mse_trace && idx_trace >= 0 ? md.mse_trace + idx_trace : nullptr);
        src = row_slot == kSlotRows ? md.mse_part : md.res_row;
        n = row_slot == kSlotRows ? (md.rows + kRowFinRows - 1) / kRowFinRows
                                  : ((row_slot >= 0) ? md.ntiles[row_slot] : 0);
    } else {
        dst = out_col ? out_col + mi : (md.mse_half && idx_half >= 0 ? md.mse_half + idx_half : nullptr);
        src = md.res_col;
        n = md.ntiles[MODE_COL];
    }
    if (dst == nullptr || (which == 0 && row_slot < 0)) return;   // (uniform per warp)
    mse_reduce_warp(src, n, dst, md);
}

// Item blk of the MSE of an iteration of the fused path: the residual of
// its state comes from the fused tiles (res_row, column-tile geometry; or,
// with rows_mse, the row finalize's per-chunk errors mse_part) unless the row
// step was redone literally (res_row, row-tile geometry); the half-step
// residual equals it (power-of-two row scales leave D_a Qhat unchanged)
// unless the column step was redone literally (res_col).  Item 0 also
// clears the flag slot the next iteration's row finalize may raise after
// the one after it.  Called by a whole warp.
__device__ __forceinline__ void mse_fused_item(const Table &tab, int blk,
                                               const unsigned int *flags,
                                               unsigned int *next_flags, int idx,
                                               bool rows_mse) {
    if (blk == 0 && (threadIdx.x & 31) == 0) { next_flags[0] = 0u; next_flags[1] = 0u; }
    const int mi = blk >> 1, which = blk & 1;
    const MatDesc &md = tab.get(mi);
    const bool lit_row = flags[0] != 0, lit_col = (flags[0] | flags[1]) != 0;
    double *dst;
    const double *src;
    int64_t n;
    // the one-pass residual of the state
    const double *src1 = rows_mse ? md.mse_part : md.res_row;
    const int64_t n1 = rows_mse ? (md.rows + kRowFinRows - 1) / kRowFinRows : md.ntiles[MODE_COL];
    if (which == 0) {
        // (with rows_mse a literal row step's error comes from its row sums too)
        dst = md.mse_trace ? md.mse_trace + idx : nullptr;
        src = (lit_row && !rows_mse) ? md.res_row : src1;
        n = (lit_row && !rows_mse) ? md.ntiles[MODE_ROW] : n1;
    } else {
        dst = md.mse_half ? md.mse_half + idx : nullptr;
        src = lit_col ? md.res_col : src1;
        n = lit_col ? md.ntiles[MODE_COL] : n1;
    }
    if (dst == nullptr) return;                                   // (uniform per warp)
    mse_reduce_warp(src, n, dst, md);
}

// b_j <- Pi(sum P / sum E) over the column's row blocks, summed in double
// in a fixed order that depends only on the matrix's shape: the column's row
// blocks are split into 8 slices (slice s: row blocks s, s+8, ... added in
// order), and the slices are added in order.  A matrix whose column pass has
// more than 8 row blocks takes a block per 128 consecutive columns (a lane
// reads the partials of four adjacent columns as two 16-byte loads), a warp
// per slice; a shorter one a warp per 32 columns, a lane per column holding
// all of its row blocks in registers and forming the same sums in the same
// order (a block: 256 columns).  Work units (a block's columns) of all
// matrices in order.  (Columns come in multiples of 16: a lane's four are
// all in or all out.)
constexpr int kColFinCols = 128, kColFinSlices = 8;
constexpr int kColFinThreads = 32 * kColFinSlices;
constexpr int kColFinWarpRb = kColFinSlices;       // most row blocks of the lane-per-column form
__host__ __device__ __forceinline__ int64_t col_units(int64_t rows_blocks, int64_t cols) {
    return rows_blocks > kColFinWarpRb ? (cols + kColFinCols - 1) / kColFinCols
                                       : (cols + 32 * kColFinSlices - 1) / (32 * kColFinSlices);
}
// Column cc's projection from its total sums.
template <int OS>
__device__ __forceinline__ void col_finish(const Table &tab, const MatDesc &md, int64_t cc,
                                           double pt, double et) {
    float b = 1.0f, pre = __int_as_float(0x7fc00000);
    if (et > 0.0) {
        pre = (float)(pt / et);
        bool cl;
        b = project_outer<OS>(pre, cl);
        if (cl) atomicOr(tab.status, STATUS_RANGE);
    }
    if (!isfinite(pt) || !isfinite(et)) atomicOr(tab.status, STATUS_NONFINITE);
    md.b_out[cc] = b;
    if (md.b_pre) md.b_pre[cc] = pre;
}
// The lane-per-column form (a matrix with at most 8 row blocks in its
// column pass, so that every slice holds at most one): lane l of warp w
// takes column 256 (unit - cunit0) + 32 w + l and adds its row blocks in
// order -- the sums of the block form, since its running sums are never -0.
template <int OS>
__device__ __forceinline__ void col_lane_unit(const Table &tab, const MatDesc &md, int64_t unit,
                                              int64_t nrb) {
    const int64_t c = (unit - md.cunit0) * (32 * kColFinSlices) + (threadIdx.x & ~31) +
                      (threadIdx.x & 31);
    if (c >= md.cols) return;
    const float2 *src = md.colpart + c;
    float2 v[kColFinSlices];
#pragma unroll
    for (int k = 0; k < kColFinSlices; ++k)
        if (k < nrb) v[k] = __ldg(src + k * md.cols);
    double pt = 0.0, et = 0.0;
#pragma unroll
    for (int k = 0; k < kColFinSlices; ++k)
        if (k < nrb) { pt += v[k].x; et += v[k].y; }
    col_finish<OS>(tab, md, c, pt, et);
}

// With mse_mode != 0 the last ceil(2n / 8) blocks of the grid finish the
// iteration's MSE instead, a warp per item (1: mse_fused_item with flags /
// next_flags; 3: the same with the per-row errors of the row finalize; 2:
// mse_literal_item of the row and column passes; 4: the same with the
// per-row errors), saving a launch.
enum { MSE_NONE = 0, MSE_FUSED = 1, MSE_LITERAL = 2, MSE_FUSED_ROWS = 3, MSE_LITERAL_ROWS = 4 };
template <int OS>
__global__ void __launch_bounds__(kColFinThreads, 3)
col_finalize_kernel(const __grid_constant__ Table tab, int64_t total_units, int mse_mode,
                    const unsigned int *flags, unsigned int *next_flags, int idx) {
    grid_dependency_begin();
    const int nmse = mse_mode != MSE_NONE ? (2 * tab.n + kColFinSlices - 1) / kColFinSlices : 0;
    const int gunits = (int)gridDim.x - nmse;           // blocks of the column update
    if ((int)blockIdx.x >= gunits) {
        const int blk = ((int)blockIdx.x - gunits) * kColFinSlices + (int)(threadIdx.x >> 5);
        if (blk >= 2 * tab.n) return;                   // (uniform per warp)
        if (mse_mode == MSE_FUSED || mse_mode == MSE_FUSED_ROWS)
            mse_fused_item(tab, blk, flags, next_flags, idx, mse_mode == MSE_FUSED_ROWS);
        else mse_literal_item(tab, blk, mse_mode == MSE_LITERAL_ROWS ? kSlotRows : MODE_ROW, idx, idx,
                              nullptr, nullptr);
        return;
    }
    __shared__ double sp[kColFinSlices][kColFinCols], se[kColFinSlices][kColFinCols];
    const int lane = threadIdx.x & 31, sl = threadIdx.x >> 5;
    for (int64_t unit = blockIdx.x; unit < total_units; unit += gunits) {
        const int mi = find_owner(tab, unit, [](const MatDesc &d) { return d.cunit0; });
        const MatDesc &md = tab.get(mi);
        const int64_t nrb = md.ntiles[MODE_COL] / max(md.ncb, 1);
        const int64_t stride = md.cols / 2;                  // float4 per row block
        if (nrb <= kColFinWarpRb) {                          // (uniform per block)
            col_lane_unit<OS>(tab, md, unit, nrb);
            continue;
        }
        const int64_t c0 = (unit - md.cunit0) * kColFinCols;
        const int64_t c = c0 + 4 * lane;
        const bool ok = c < md.cols;
        double p0 = 0.0, e0 = 0.0, p1 = 0.0, e1 = 0.0, p2 = 0.0, e2 = 0.0, p3 = 0.0, e3 = 0.0;
        if (ok) {
            const float4 *src = reinterpret_cast<const float4 *>(md.colpart + c);
            // this slice's row blocks in order; the loads of 2 of them are
            // issued ahead of their sums (the order of the sums is unchanged)
            for (int64_t k0 = sl; k0 < nrb; k0 += 2 * kColFinSlices) {
                float4 v[2], w[2];
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int64_t k = k0 + (int64_t)u * kColFinSlices;
                    if (k < nrb) {
                        v[u] = __ldg(src + k * stride);
                        w[u] = __ldg(src + k * stride + 1);
                    }
                }
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    if (k0 + (int64_t)u * kColFinSlices < nrb) {
                        p0 += v[u].x;
                        e0 += v[u].y;
                        p1 += v[u].z;
                        e1 += v[u].w;
                        p2 += w[u].x;
                        e2 += w[u].y;
                        p3 += w[u].z;
                        e3 += w[u].w;
                    }
                }
            }
        }
        sp[sl][4 * lane] = p0;
        se[sl][4 * lane] = e0;
        sp[sl][4 * lane + 1] = p1;
        se[sl][4 * lane + 1] = e1;
        sp[sl][4 * lane + 2] = p2;
        se[sl][4 * lane + 2] = e2;
        sp[sl][4 * lane + 3] = p3;
        se[sl][4 * lane + 3] = e3;
        __syncthreads();
        const int cl = threadIdx.x;
        if (cl < kColFinCols && c0 + cl < md.cols) {
            double pt = 0.0, et = 0.0;
            for (int q = 0; q < kColFinSlices; ++q) { pt += sp[q][cl]; et += se[q][cl]; }
            col_finish<OS>(tab, md, c0 + cl, pt, et);
        }
        __syncthreads();
    }
}

#ifdef DQ_DEFINE_HOST_KERNELS
// Non-template kernels: defined in exactly one translation unit.

__global__ void mse_finalize_kernel(const __grid_constant__ Table tab, int row_slot, int idx_trace, int idx_half,
                                    double *out_row, double *out_col) {
    grid_dependency_begin();
    const int blk = (int)blockIdx.x * 8 + (int)(threadIdx.x >> 5);
    if (blk >= 2 * tab.n) return;                       // (uniform per warp)
    mse_literal_item(tab, blk, row_slot, idx_trace, idx_half, out_row, out_col);
}

// Initial state: a <- a0 or 1, b <- b0 or 1 (rows then columns, all matrices).
// With `flags` (one-pass MX path): an initial |e(a)| > 20 makes iteration 0
// take its row step literally.
__global__ void init_state_kernel(const __grid_constant__ Table tab, int64_t total_rows,
                                  int64_t total_cols, unsigned int *flags) {
    grid_dependency_begin();
    for (int64_t g = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; g < total_rows + total_cols;
         g += (int64_t)gridDim.x * blockDim.x) {
        if (g < total_rows) {
            const int mi = find_owner(tab, g, [](const MatDesc &d) { return d.row0; });
            const MatDesc &md = tab.get(mi);
            const int64_t r = g - md.row0;
            const float a = md.a0 ? md.a0[r] : 1.0f;
            md.a_out[r] = a;
            if (flags != nullptr) {
                const int ea = (int)((__float_as_uint(a) >> 23) & 0xFF) - 127;
                if (ea > 20 || ea < -20) atomicOr(&flags[0], 1u);
            }
        } else {
            const int64_t gc = g - total_rows;
            const int mi = find_owner(tab, gc, [](const MatDesc &d) { return d.col0; });
            const MatDesc &md = tab.get(mi);
            const int64_t c = gc - md.col0;
            md.b_out[c] = md.b0 ? md.b0[c] : 1.0f;
        }
    }
}

#endif  // DQ_DEFINE_HOST_KERNELS

// amax over each matrix (tiles of the PACK geometry), for the tensor scale.
template <typename TIn>
__global__ void __launch_bounds__(kThreads) amax_kernel(const __grid_constant__ Table tab) {
    grid_dependency_begin();
    constexpr int EPC = Chunk<TIn>::EPC;
    const int64_t t = blockIdx.x;
    const int mi = find_owner(tab, t, [](const MatDesc &d) { return d.tile0[MODE_PACK]; });
    const MatDesc &md = tab.get(mi);
    const int64_t lt = t - md.tile0[MODE_PACK];
    if (lt >= md.ntiles[MODE_PACK]) return;
    // the tile's rows as a flat range of 16-byte chunks
    // tile (rb, cb): the cb == 0 tiles scan their whole row block
    const int64_t cpr = md.cols / EPC;
    const int64_t tr = md.tr[MODE_PACK];
    const int64_t rb = lt / md.ncb, cb = lt % md.ncb;
    float m = 0.0f;
    if (cb == 0) {
        const int64_t r0 = rb * tr, r1 = min(md.rows, r0 + tr);
        const uint4 *base = reinterpret_cast<const uint4 *>(md.W);
        for (int64_t k = r0 * cpr + threadIdx.x; k < r1 * cpr; k += kThreads) {
            Chunk<TIn> ck;
            ck.raw = __ldg(base + k);
            float w[EPC];
            ck.unpack(w);
#pragma unroll
            for (int j = 0; j < EPC; ++j) m = max_nan(m, fabsf(w[j]));
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max_nan(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0 && cb == 0) {
        if (!isfinite(m)) atomicOr(tab.status, STATUS_NONFINITE);
        else atomicMax(md.amax, __float_as_uint(m));   // non-negative floats order as uints
    }
}

#ifdef DQ_DEFINE_HOST_KERNELS
// ts = 2^ceil(log2(amax / (448 qmax))), exponent in [-126, 126]; 1 if amax == 0.
__global__ void tensor_scale_kernel(const __grid_constant__ Table tab, float qmax, int enabled) {
    grid_dependency_begin();
    const int mi = blockIdx.x * blockDim.x + threadIdx.x;
    if (mi >= tab.n) return;
    const MatDesc &md = tab.get(mi);
    float ts = 1.0f;
    if (enabled) {
        float amax = __uint_as_float(*md.amax);
        if (amax > 0.0f) {
            // 448*qmax = C * 2^11 with C = 1.3125 (qmax 6) or 1.53125 (qmax 7)
            const uint32_t CT = (qmax == 6.0f) ? 0x280000u : 0x440000u;
            int e;
            if (amax < kMinNormal) e = -126;
            else {
                int k = ilog2f(amax);
                e = ((__float_as_uint(amax) & 0x7FFFFFu) <= CT) ? k - 11 : k - 10;
            }
            e = min(max(e, -126), 126);
            ts = pow2f(e);
        }
    }
    *md.ts_out = ts;
}

#endif  // DQ_DEFINE_HOST_KERNELS

}  // namespace dq
