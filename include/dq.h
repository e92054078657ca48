/*
 * dq.h — C ABI of the B200 dual-scale weight quantization library.
 *
 * The library solves the DualQuant dual-scale model of a weight matrix
 * (DualQuant reproduction note, daiwk.github.io, section "核心公式", eq. (1)):
 *
 *     W  ~=  D_a · Q( D_a^-1 · W · D_b^-1 ) · D_b
 *
 * with one outer inverse scale a_i per row and b_j per column, and Q a group
 * quantizer on a fixed grid whose group scales lie in the format's scale set.
 * It runs the block coordinate descent of eq. (2) of the same section: with
 * the codes fixed, a_i <- Pi(sum_j W_ij R_ij / sum_j R_ij^2) with R = Qhat D_b,
 * re-quantize, then b_j <- Pi(sum_i W_ij S_ij / sum_i S_ij^2) with S = D_a Qhat,
 * re-quantize; a slice with all-zero codes keeps scale 1.  The activation side
 * (second half of eq. (1)) multiplies X by b per input channel and quantizes.
 *
 * Conventions for every entry point:
 *  - W and X are row-major [rows, cols] (out-features x in-features; groups of
 *    G consecutive columns share a group scale).
 *  - Pointers are DEVICE pointers unless marked (host).  The caller owns every
 *    buffer; the library allocates no device memory.
 *  - Calls are asynchronous and ordered on `stream` (a cudaStream_t; NULL is
 *    the legacy default stream).  Argument errors are reported synchronously
 *    through the return value and launch nothing.  Input data errors found on
 *    the device (non-finite values, scale-range clamps) set flags that
 *    dq_last_device_status() reports; kernels never trap.
 *  - Shapes: cols % G == 0, G in {16, 32, 64}; rows >= 0 (rows == 0 or
 *    cols == 0 is a valid empty call).  W, X, codes and gscales must be
 *    16-byte aligned (base pointers), a/b/scale vectors 4-byte aligned.
 *  - Codes: two 4-bit codes per byte, the even column in the low nibble.
 *    INT4 is two's complement in [-8, 7]; E2M1 is the nibble s|ee|m.
 *    Row i of the codes starts at byte i * cols / 2.
 *  - Group scales: [rows, cols / G] row-major; BF16 as its uint16 bit
 *    pattern, E8M0 as a biased exponent byte (127 + e), E4M3 as its byte
 *    (OCP FP8 E4M3 "fn").  A group whose values are all zero stores 1.0.
 *  - a, b: float32 values that lie exactly in the outer scale set.
 *  - MSE values are sum (W - D_a Qhat D_b)^2 / (rows * cols), in double.
 */
#ifndef DQ_H
#define DQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define DQ_API __attribute__((visibility("default")))
#else
#define DQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *dq_stream; /* cudaStream_t */

typedef enum dq_status {
    DQ_OK = 0,
    DQ_ERR_ARG = -1,            /* null pointer, bad enum, T < 0, n < 0 */
    DQ_ERR_SHAPE = -2,          /* cols % G != 0, negative size */
    DQ_ERR_FORMAT = -3,         /* unknown preset or unsupported combination */
    DQ_ERR_NONFINITE = -4,      /* (device flag) NaN or Inf in W or X, or W/(a b)
                                   beyond the float32 range */
    DQ_ERR_RANGE = -5,          /* (device flag) an outer scale hit the set's bound */
    DQ_ERR_CUDA = -6,           /* a CUDA runtime call failed */
    DQ_ERR_WORKSPACE = -7,      /* workspace null or smaller than dq_workspace_size */
    DQ_ERR_NOT_IMPLEMENTED = -8,
    DQ_ERR_ALIGN = -9,          /* a pointer misses its alignment */
    DQ_ERR_SCRATCH = -10,       /* matrix needs more than the built-in scratch buffer */
    DQ_ERR_TIMEOUT = -11        /* (device flag) a bounded wait in a kernel ran out */
} dq_status;

/* Code (element) types: the pages' INT4 and E2M1 codebooks, and the other
 * element formats of the MX family the pages claim (OCP Microscaling
 * definition): INT8 (MXINT8), E4M3 and E5M2 (MXFP8), E2M3 and E3M2 (MXFP6).
 * qmax = 7, 6, 127, 448, 57344, 7.5, 28.  The last five need E8M0 group and
 * outer scales. */
enum { DQ_CODES_INT4 = 0, DQ_CODES_E2M1 = 1, DQ_CODES_INT8 = 2, DQ_CODES_E4M3 = 3,
       DQ_CODES_E5M2 = 4, DQ_CODES_E2M3 = 5, DQ_CODES_E3M2 = 6 };
enum { DQ_SCALE_BF16 = 0, DQ_SCALE_E8M0 = 1, DQ_SCALE_E4M3 = 2 };
enum { DQ_DT_F32 = 0, DQ_DT_BF16 = 1 };

/* Format descriptor.  Scale sets (DualQuant pages: daiwk note "本地复现";
 * news.yiqijian.com article, MXFP4/NVFP4 block structure):
 *   BF16  — bfloat16 values; as an outer or group scale clamped to the
 *           normal range [2^-126, max].
 *   E8M0  — powers of two 2^e, e in [-126, 126].
 *   E4M3  — OCP FP8 E4M3 values (group scale only), saturating at 448.
 * Group scales are the projection of (group absmax / qmax) onto the set:
 * BF16 and E4M3 round to nearest even, E8M0 rounds up (the smallest power of
 * two that keeps every code in range).  Outer scales a, b are the nearest
 * value of their set (E8M0: an exact tie goes up).
 * tensor_scale_auto = 1 gives weights a second-level scale
 * ts = 2^ceil(log2(amax(W) / (448 * qmax))) (NVFP4); otherwise ts = 1. */
typedef struct dq_format {
    int32_t codes;             /* DQ_CODES_* */
    int32_t group;             /* G in {16, 32, 64} */
    int32_t group_scale;       /* DQ_SCALE_* */
    int32_t outer_scale;       /* DQ_SCALE_BF16 or DQ_SCALE_E8M0 */
    int32_t tensor_scale_auto; /* 0 or 1 */
} dq_format;

/* One matrix of a batched solve.  All pointers are device pointers. */
typedef struct dq_matrix {
    const void *W;             /* [rows, cols] of the call's dtype */
    int64_t rows, cols;
    const float *a0, *b0;      /* initial a [rows], b [cols]; NULL = all ones */
    uint8_t *codes;            /* out: dq_code_bytes(fmt, rows, cols) bytes of codes */
    void *gscales;             /* out: [rows, cols/G] group scales */
    float *a, *b;              /* out: final outer inverse scales */
    float *tensor_scale;       /* out: 1 float, the ts used (1.0 unless auto) */
    double *mse_trace;         /* out: T+1 doubles ([0] initial state), or NULL */
    double *mse_half;          /* out: T doubles (after each row step), or NULL */
} dq_matrix;

/* Library version string (static storage). */
DQ_API const char *dq_version(void);

/* Text of a status code (static storage). */
DQ_API const char *dq_strerror(dq_status s);

/* Fill `out` (host) with a named preset: "int4_bf16" (INT4 codes, BF16 group
 * and outer scales, default G 64), "mxint4" (INT4, E8M0, E8M0, G 32),
 * "mxfp4" (E2M1, E8M0, E8M0, G 32), "nvfp4" (E2M1, E4M3 group, BF16 outer,
 * G 16, tensor_scale_auto); the rest of the MX family, all E8M0/E8M0 and
 * G 32: "mxint8", "mxfp8_e4m3", "mxfp8_e5m2", "mxfp6_e2m3", "mxfp6_e3m2";
 * the MX block formats with BF16 outer scales (E8M0 group scales, G 32):
 * "mxint4_bf16outer", "mxfp4_bf16outer".  group == 0 keeps the preset's G.  Presets follow the formats of Table 1 of
 * the daiwk note, the news article's MXFP4/NVFP4 description and its claim of
 * the whole MX family.  Errors: DQ_ERR_ARG (null), DQ_ERR_FORMAT (unknown
 * name or G). */
DQ_API dq_status dq_format_preset(const char *name, int32_t group, dq_format *out);

/* Size in bytes of the codes of a rows x cols matrix in format `fmt`: rows
 * rows of cols * bits / 8 bytes each.  Layout of a row: 4-bit codes two per
 * byte, the even column in the low nibble (INT4 two's complement, E2M1
 * s|ee|m); 8-bit codes one per byte (INT8 two's complement, E4M3 s|eeee|mmm,
 * E5M2 s|eeeee|mm); 6-bit codes (E2M3 s|ee|mmm, E3M2 s|eee|mm) four per 3
 * bytes as one little-endian 24-bit word, the first column in the low bits.
 * Returns -1 for an invalid format or shape (cols % G != 0). */
DQ_API int64_t dq_code_bytes(const dq_format *fmt, int64_t rows, int64_t cols);

/* Bytes of device workspace a solve or a single update of the listed
 * matrices needs (host arrays rows[n], cols[n]; result in *bytes, host).
 * Workspace holds per-tile partial sums; it needs no initialisation and no
 * alignment beyond 256 bytes.  Errors: DQ_ERR_ARG, DQ_ERR_SHAPE, DQ_ERR_FORMAT. */
DQ_API dq_status dq_workspace_size(int32_t n, const int64_t *rows, const int64_t *cols,
                            const dq_format *fmt, size_t *bytes);

/* Q(X ⊘ (a bᵀ)): the black-box group quantizer (daiwk note, "原始论文总结")
 * applied to X / (a_i b_j) with second-level scale `tensor_scale` (host value,
 * a power of two; it must be 1.0 unless the group scales are E4M3).  a (rows) and b (cols) may be
 * NULL (all ones).  Writes the codes (dq_code_bytes layout) and group scales.
 * No workspace. */
DQ_API dq_status dq_quantize(const void *X, int32_t dtype, int64_t rows, int64_t cols,
                      const dq_format *fmt, const float *a, const float *b,
                      float tensor_scale, uint8_t *codes, void *gscales,
                      dq_stream stream);

/* out_ij = a_i * c_ij * s_g * ts * b_j (float32), the reconstruction
 * D_a Qhat D_b of eq. (1).  a or b may be NULL (ones). */
DQ_API dq_status dq_dequantize(const uint8_t *codes, const void *gscales, int64_t rows,
                        int64_t cols, const dq_format *fmt, float tensor_scale,
                        const float *a, const float *b, float *out, dq_stream stream);

/* Full DualQuant solve of one matrix: initialise (a0, b0 or ones), then T
 * iterations of {row update, re-quantize, column update, re-quantize}
 * (eq. (2) and the order stated under it), then write the codes and group
 * scales of Q(W ⊘ (a bᵀ)) for the final a, b.  tensor_scale (1 float) receives
 * the ts used.  mse_trace (T+1) and mse_half (T) may be NULL; entry t is
 * mean((W - D_a Qhat D_b)^2) of the state before iteration t's row step
 * (mse_half: before its column step), the last entry that of the final
 * state.  The last entry is summed as (W - R)^2; for the formats with 4-bit
 * codes (INT4, E2M1) the others are taken per row as sum W^2 - 2 a sum W R
 * + a^2 sum R^2 from float32 row sums (correct to about 1e-5 relative; for
 * MXFP4 and MXINT4, whose sums are taken for a = 1, exactly 0 for rows that
 * Q reproduces); mse_half entries of the literal formats sum (W - R)^2.  `workspace` must hold dq_workspace_size bytes for this one
 * matrix. */
DQ_API dq_status dq_solve_dual_scale(const void *W, int32_t dtype, int64_t rows, int64_t cols,
                              const dq_format *fmt, int32_t T, const float *a0,
                              const float *b0, uint8_t *codes, void *gscales, float *a,
                              float *b, float *tensor_scale, double *mse_trace,
                              double *mse_half, void *workspace, size_t ws_bytes,
                              dq_stream stream);

/* The same solve for n independent matrices (host array mats[n]) sharing one
 * format, dtype and T, in one launch sequence (every kernel covers all
 * matrices).  Workspace: dq_workspace_size over all n shapes.  The work table
 * (one entry per matrix) is built in a host buffer the library keeps per
 * thread and copied into the workspace with one cudaMemcpyAsync; the call
 * returns once the table is staged, so `mats` may be reused at once. */
DQ_API dq_status dq_solve_dual_scale_batched(int32_t n, const dq_matrix *mats, int32_t dtype,
                                      const dq_format *fmt, int32_t T, void *workspace,
                                      size_t ws_bytes, dq_stream stream);

/* The batched solve as a CUDA graph, for repeated solves of the same shapes
 * (the launch sequence of dq_solve_dual_scale_batched, about 6 kernels per
 * iteration, captured once and replayed with one launch; the solve is
 * launch-bound on small matrices).  Arguments as dq_solve_dual_scale_batched;
 * they are checked when the graph is made, and every device pointer in
 * `mats` and the workspace is baked into the graph: they must stay
 * allocated, and keep their shapes, until dq_graph_destroy.  Each replay
 * reads W (and a0, b0) as they are at that time and writes every output
 * again, so new weights of the same shapes take a replay, not a new graph.
 * The graph owns a pinned host copy of the work table, uploaded by every
 * replay (a caller may use the workspace for other calls between replays).
 * Kernel timing (dq_kernel_timing) does not apply to graph launches.
 * Errors: DQ_ERR_ARG (out NULL, n == 0), DQ_ERR_CUDA (capture or
 * instantiation failed), and the argument codes of dq_solve_dual_scale_batched
 * (checked before any CUDA call); *out is NULL then. */
typedef struct dq_graph_s *dq_graph;
DQ_API dq_status dq_graph_solve_batched(int32_t n, const dq_matrix *mats, int32_t dtype,
                                        const dq_format *fmt, int32_t T, void *workspace,
                                        size_t ws_bytes, dq_graph *out);
/* One replay on `stream` (the device the graph was made on must be current:
 * DQ_ERR_ARG otherwise, and for a NULL graph).  Replays on one stream run in
 * order; replays of one graph on different streams must not overlap, since
 * they share the workspace. */
DQ_API dq_status dq_graph_launch(dq_graph g, dq_stream stream);
/* Kernels one replay launches (0 for NULL). */
DQ_API int64_t dq_graph_launches(dq_graph g);
/* Frees the graph (NULL: no-op).  The call waits for the graph's last
 * replay to finish (only that: other work on the device is not waited
 * for), then frees the graph and its pinned table. */
DQ_API dq_status dq_graph_destroy(dq_graph g);

/* One row half-step of eq. (2) from the state (a_in, b_in):
 * a_out_i = Pi_Fa(<W_i, R_i> / <R_i, R_i>), R = Q(W ⊘ a_in b_inᵀ) D_b, zero
 * slice -> 1.  a_pre (rows, may be NULL) receives the unprojected ratio
 * (NaN on zero slices); mse_in (1 double, may be NULL) the MSE of the input
 * state (for 4-bit codes formed per row from the row sums, as in the
 * solves; see dq_solve_dual_scale).  a_out may alias a_in. */
DQ_API dq_status dq_row_update(const void *W, int32_t dtype, int64_t rows, int64_t cols,
                        const dq_format *fmt, float tensor_scale, const float *a_in,
                        const float *b_in, float *a_out, float *a_pre, double *mse_in,
                        void *workspace, size_t ws_bytes, dq_stream stream);

/* One column half-step of eq. (2) from the state (a_in, b_in):
 * b_out_j = Pi_Fb(<W_:j, S_:j> / <S_:j, S_:j>), S = D_a Q(W ⊘ a_in b_inᵀ).
 * b_pre (cols, may be NULL): unprojected ratio; mse_in: MSE of the input
 * state.  b_out may alias b_in. */
DQ_API dq_status dq_col_update(const void *W, int32_t dtype, int64_t rows, int64_t cols,
                        const dq_format *fmt, float tensor_scale, const float *a_in,
                        const float *b_in, float *b_out, float *b_pre, double *mse_in,
                        void *workspace, size_t ws_bytes, dq_stream stream);

/* The column half-step split for a matrix whose rows are sharded (over
 * GPUs, say): the column statistics of eq. (2) are sums over all rows, so
 * each shard contributes partial sums and one fixed-order sum of all
 * shards' partials gives the update.  No counterpart in the pages (the
 * multi-GPU split of the closed form).
 * dq_col_row_block: the number of rows per row block of the column
 *   statistics of a rows x cols matrix (dtype DQ_DT_BF16 or DQ_DT_F32), as
 *   dq_col_update and the solves use it; -1 on bad arguments.
 * dq_col_partials: for the shard W [rows, cols] (its own rows, with their
 *   row scales a [rows] and the matrix's b [cols]; tensor_scale as in
 *   dq_col_update), the partial sums (sum_i W_ij S_ij, sum_i S_ij^2),
 *   S = D_a Q(W ⊘ a bᵀ), over each block of `row_block` consecutive shard
 *   rows: `partials` receives ceil(rows / row_block) x cols float pairs
 *   (P, E), row block major, 16-byte aligned, caller-owned.  row_block is
 *   the whole matrix's dq_col_row_block (a shard's own is never larger;
 *   a smaller one is refused with DQ_ERR_SHAPE).  mse_in (1 double, may be
 *   NULL) receives the shard's MSE sum / (rows cols) at the input state.
 *   workspace as dq_col_update.
 * dq_col_finalize: b_out_j = Pi_Fb(sum_k P[k][j] / sum_k E[k][j]) (zero
 *   slice -> 1) over row_blocks slabs of cols float pairs (row block
 *   major; cols a multiple of fmt's group size, as for the solves, else
 *   DQ_ERR_SHAPE), summed in the fixed order of the solves' column update;
 *   b_pre (may be NULL) the unprojected ratios.
 * With shards whose first rows are multiples of row_block, the shards'
 * partials concatenated in row order are the whole matrix's, so
 * dq_col_finalize gives dq_col_update's b bit for bit. */
DQ_API int64_t dq_col_row_block(int64_t rows, int64_t cols, int32_t dtype);
DQ_API dq_status dq_col_partials(const void *W, int32_t dtype, int64_t rows, int64_t cols,
                                 const dq_format *fmt, float tensor_scale, const float *a,
                                 const float *b, int64_t row_block, float *partials,
                                 double *mse_in, void *workspace, size_t ws_bytes,
                                 dq_stream stream);
DQ_API dq_status dq_col_finalize(const float *partials, int64_t row_blocks, int64_t cols,
                                 const dq_format *fmt, float *b_out, float *b_pre,
                                 dq_stream stream);

/* Activation side of eq. (1): Q(X D_b) with ts = 1 — each input channel j is
 * multiplied by b_j, then quantized in groups of G along K (the trove summary,
 * "How to use it": beta is applied inside the activation-quantization kernel).
 * X is bf16 [tokens, K]; b float [K].  Writes the codes (dq_code_bytes(fmt,
 * tokens, K) bytes) and group scales [tokens, K/G].  No workspace. */
DQ_API dq_status dq_act_rescale_quant(const void *X, int64_t tokens, int64_t K, const float *b,
                               const dq_format *fmt, uint8_t *codes, void *gscales,
                               dq_stream stream);

/* Two-level absmax quantization (msmodelslim.readthedocs.io, DualScale page,
 * "算法原理" 1(a)-(c) and 2(a)-(b)) — a second, non-iterative method.  Per
 * row and block of `dual_block` consecutive columns (256, 512 or 1024; the
 * last block may be shorter): outer scale S = max|X_block| / 6 (6 = the
 * largest normal E2M1 value; float32 division; S = 1 for an all-zero
 * block), then the inner format (`inner` must be MXFP4: E2M1 codes, E8M0
 * group scales, G = 32) quantizes X / S (float32 division) exactly as
 * dq_quantize does, and the reconstruction is qdq = (c * s) * S (float32).
 * X: [rows, cols] of `dtype`, cols a multiple of 32.  Outputs (device,
 * caller-owned): codes [rows, cols/2] (dq_code_bytes layout), inner_scales
 * [rows, cols/32] E8M0 bytes, outer_scales [rows, ceil(cols/dual_block)]
 * float32, qdq [rows, cols] float32 or NULL (not written).  16-byte aligned
 * X, codes, inner_scales and qdq.  Errors: DQ_ERR_FORMAT (inner not MXFP4),
 * DQ_ERR_ARG (block size, dtype, null pointer), DQ_ERR_SHAPE, DQ_ERR_ALIGN;
 * a non-finite input raises the device flag. */
DQ_API dq_status dq_two_level_quant(const void *X, int32_t dtype, int64_t rows, int64_t cols,
                                    int32_t dual_block, const dq_format *inner, uint8_t *codes,
                                    void *inner_scales, float *outer_scales, float *qdq,
                                    dq_stream stream);

/* Scale tiles: the layout in which dq_w4a4_gemm takes group scales (E8M0
 * per 32 elements for MXFP4, E4M3 per 16 for NVFP4), the one the tensor core
 * reads them in.  For every block of 128 rows and every 4 G elements of K (4
 * scales per row) one 512-byte chunk, chunks ordered [row block][K block];
 * inside a chunk the scale k (0..3) of row r (0..127 within the block) sits
 * at byte (r % 32) * 16 + (r / 32) * 4 + k.  rows * K / G bytes in all, like
 * the row-major array.
 * dq_scale_tiles rewrites row-major scales [rows, K/G] (the layout written
 * by dq_solve_dual_scale, dq_quantize and dq_act_rescale_quant) into scale
 * tiles: G = 16 or 32, rows a multiple of 128 and K of 4 G, both pointers
 * 16-byte aligned, device, caller-owned, not overlapping.  Errors:
 * DQ_ERR_SHAPE, DQ_ERR_ARG (also for another G), DQ_ERR_ALIGN.  (No
 * counterpart in the method: a data layout.) */
DQ_API dq_status dq_scale_tiles(const void *scales, int64_t rows, int64_t K, int32_t group,
                                uint8_t *tiles, dq_stream stream);

/* Block-scaled W4A4 GEMM on the tensor cores, the inference step of eq. (1)
 * (daiwk note, "核心公式": X W^T ~= (X D_b) Qhat^T D_a; trove summary, "How to
 * use it"):  out[m, n] = a_n * ts * sum_k Qx[m, k] * Qw[n, k], float32,
 * where Qx is given by codes_x [M, K/2] and scales_x (M * K/G bytes, scale
 * tiles of the dq_act_rescale_quant scales) and Qw by codes_w [N, K/2] and
 * scales_w (N * K/G bytes, scale tiles of the solve's group scales), a [N]
 * the outer row scales of W and ts the weights' tensor scale (device, one
 * float as the solve wrote it; NULL reads as 1).  `fmt` is MXFP4 (E2M1
 * codes, E8M0 group scales, G = 32) or NVFP4 (E2M1 codes, E4M3 group scales,
 * G = 16; news article, "适配 MXFP4 与 NVFP4 块结构"); the activations are
 * quantized with tensor scale 1.  M and N multiples of 128, K a multiple of
 * 256; every pointer 16-byte aligned (tensor_scale 4-byte); out [M, N]
 * row-major, caller-owned.  The products are accumulated in float32.
 * Errors: DQ_ERR_FORMAT, DQ_ERR_SHAPE, DQ_ERR_ARG, DQ_ERR_ALIGN; a stalled
 * pipeline (a bounded wait that ran out) raises the device flag read by
 * dq_last_device_status as DQ_ERR_TIMEOUT. */
DQ_API dq_status dq_w4a4_gemm(const uint8_t *codes_x, const void *scales_x, const uint8_t *codes_w,
                              const void *scales_w, const float *a, const float *tensor_scale,
                              int64_t M, int64_t N, int64_t K, const dq_format *fmt, float *out,
                              dq_stream stream);

/* Test support for the failure path (no counterpart in the method): the
 * next dq_w4a4_gemm call on any thread has its producer skip the loads of
 * its first K tile, so the MMA thread's bounded wait for that tile runs out
 * (after about 1 s); every CTA then stops issuing work, waits (bounded) for
 * its copies in flight, frees its TMEM and returns, and the device flag reads
 * DQ_ERR_TIMEOUT.  The output of that call is undefined.  Nothing faults or
 * hangs; later calls run normally. */
DQ_API dq_status dq_test_stall_next_gemm(void);

/* Synchronise `stream`, read and clear the device flags raised by earlier
 * calls on this device: DQ_ERR_NONFINITE if an input held NaN/Inf (or
 * scaling it by the outer scales left the float32 range),
 * DQ_ERR_RANGE if an outer scale was clamped at its set's bound, DQ_OK
 * otherwise (NONFINITE wins when both are set).  The flags are one word per
 * device shared by all streams. */
DQ_API dq_status dq_last_device_status(dq_stream stream);

/* Variant of dq_solve_dual_scale for callers that cannot allocate device
 * memory: code that runs inside another framework's memory pool or under a
 * strict memory budget, plug-ins that may not call cudaMalloc, or C hosts
 * without a device allocator at hand.  It takes no workspace argument; its
 * per-tile partial sums live in one scratch buffer of DQ_NOALLOC_SCRATCH_BYTES
 * (32 MiB) built into the library, which every GPU that loads the library
 * holds until the process exits.  The paper has no counterpart of this call.
 *  - The first call on a device looks up the buffer's device address with
 *    that device current (cudaGetSymbolAddress); make that first call before
 *    any stream capture.
 *  - A matrix whose scratch need exceeds the buffer is refused with
 *    DQ_ERR_SCRATCH (dq_workspace_size gives the need: 8192 x 28672 bf16
 *    fits, for example).
 *  - Every call shares the one buffer per device: calls that overlap on the
 *    GPU (on different streams, or from several host threads) race and give
 *    wrong results; serialise them.  The buffer keeps the last call's
 *    contents; the call clears what it needs to start at zero.
 *  - Allocates nothing (no cudaMalloc, cudaFree or allocating library call).
 *  - Runs the launch sequence of dq_solve_dual_scale (the MX formats take
 *    the one-pass iteration), so its results equal that call's bit for bit.
 * Arguments, outputs and errors as dq_solve_dual_scale. */
#define DQ_NOALLOC_SCRATCH_BYTES (32u << 20)
DQ_API dq_status dq_solve_dual_scale_noalloc(const void *W, int32_t dtype, int64_t rows,
                                             int64_t cols, const dq_format *fmt, int32_t T,
                                             const float *a0, const float *b0, uint8_t *codes,
                                             void *gscales, float *a, float *b,
                                             float *tensor_scale, double *mse_trace,
                                             double *mse_half, dq_stream stream);

/* The batched solve for matrices whose inputs and outputs live in host
 * memory, with the transfers overlapped with the solves (no counterpart in
 * the pages: the way to feed the solver from the host).  host[i] and dev[i]
 * describe matrix i twice, with equal rows and cols:
 *  - host[i].W (and a0 / b0 when not NULL) are read from host memory; the
 *    outputs whose host[i] pointer is not NULL (codes, gscales, a, b,
 *    tensor_scale, mse_trace, mse_half) are written to host memory;
 *  - dev[i] holds device buffers of the same sizes, caller-owned: W (and
 *    a0 / b0 when host[i] has them) receive the copies of the inputs, the
 *    outputs are written there as by dq_solve_dual_scale and stay there.
 * The matrices are taken in order in groups of consecutive matrices (about
 * 1/8 of all the input bytes per group, at least 32 MiB, and no more than
 * `workspace` can hold as one batched solve; it must hold at least
 * dq_workspace_size for the largest single matrix, and dq_workspace_size
 * over all n shapes always lets the groups form fully).  For each group:
 * its inputs are copied on stream `h2d`, it is solved on `compute` as one
 * batched solve once they have landed, and the requested outputs are copied
 * back on `d2h` once that solve is done; so group g+1 crosses the bus while
 * group g is solved and group g-1's results return.  The call only enqueues: the host outputs
 * are valid once the work queued on `d2h` has completed.  Host memory must
 * be page-locked (cudaHostAlloc / cudaHostRegister) for the copies to
 * overlap; pageable memory works but serialises.  Each call first orders
 * `h2d` after the work already queued on `compute` and `compute` after the
 * work already queued on `d2h`, so consecutive calls may reuse the same
 * buffers.  Calls are serialised inside the library (one set of internal
 * events per device).  One cudaMemcpyAsync per buffer.  Results equal
 * dq_solve_dual_scale on each matrix, whatever the grouping.  Errors: as dq_solve_dual_scale_batched,
 * plus DQ_ERR_SHAPE when host[i] and dev[i] disagree and DQ_ERR_ARG when a
 * host input or requested output has no device counterpart; on an error the
 * work already queued stays queued. */
DQ_API dq_status dq_solve_dual_scale_batched_host(int32_t n, const dq_matrix *host,
                                                  const dq_matrix *dev, int32_t dtype,
                                                  const dq_format *fmt, int32_t T,
                                                  void *workspace, size_t ws_bytes,
                                                  dq_stream compute, dq_stream h2d,
                                                  dq_stream d2h);

/* Measurement support (no counterpart in the method).  dq_kernel_timing(kinds)
 * makes the tile-kernel launches of the kinds whose bit is set in `kinds`
 * (bit k for kind k: 0 row statistics, 1 column statistics, 2 pack,
 * 3 activation, 4 row and column statistics in one pass; 0 turns timing off)
 * record a CUDA event pair on their own stream; dq_kernel_time synchronises
 * those events and returns (and clears) the summed milliseconds and the
 * launch count of one kind.  Each event pair separates its launch from the
 * kernels around it on the stream, so time only the kinds of interest.
 * dq_launch_count returns the number of kernels this library has launched in
 * the process so far (all kinds, including finalize kernels). */
DQ_API dq_status dq_kernel_timing(int32_t kinds);
DQ_API dq_status dq_kernel_time(int32_t kind, double *ms, int64_t *launches);
DQ_API int64_t dq_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* DQ_H */
