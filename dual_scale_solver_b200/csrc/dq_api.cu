// dq_api.cu — the C ABI declared in include/dq.h: argument checks, tile
// geometry, workspace layout, and the launch sequences of the solver.
//
// Launch sequence of a solve (DualQuant, daiwk.github.io reproduction note,
// "核心公式" eq. (2) and the order stated under it; trove summary, flowchart
// of "How it works"):
//   [amax + tensor scale]  init a, b
//   for t in 1..T:
//     ROW tiles   -> per-row partial sums of <W,R>, <R,R>; residual of state t-1
//     row finalize: a <- Pi(sum/sum), zero slice -> 1
//     COL tiles   -> per-column partial sums of <W,S>, <S,S> with the new a
//     col finalize: b <- Pi(sum/sum), zero slice -> 1
//     mse finalize: mse_trace[t-1], mse_half[t-1]
//   PACK tiles -> codes, group scales, residual; mse finalize -> mse_trace[T]
// The re-quantization after each update is not a separate pass: every tile
// pass quantizes W with the current (a, b) on the fly.
#include <cuda_runtime.h>

#include <cstdio>
#include <cstring>
#include <algorithm>
#include <atomic>
#include <mutex>
#include <new>
#include <vector>

#include "../../include/dq.h"
#define DQ_DEFINE_HOST_KERNELS
#include "dq_launch.h"

using namespace dq;

namespace {

__device__ unsigned int g_dq_status_word;

constexpr int kMaxDevices = 64;
unsigned int *g_status_ptr[kMaxDevices];
std::once_flag g_status_once[kMaxDevices];

// Device address of the status word on the current device (looked up once
// per device with that device current).
unsigned int *status_ptr() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::call_once(g_status_once[dev], [dev]() {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_dq_status_word) == cudaSuccess)
            g_status_ptr[dev] = static_cast<unsigned int *>(p);
    });
    return g_status_ptr[dev];
}

// ---- measurement support: launch counter and optional per-kind event timing
std::atomic<int64_t> g_launches{0};
std::mutex g_timing_mu;
unsigned int g_timing_kinds = 0;   // bit k: time tile launches of kind k
struct TimedLaunch { cudaEvent_t beg, end; int kind; };
std::vector<TimedLaunch> g_timed;       // recorded, not yet read
std::vector<cudaEvent_t> g_event_pool;  // free events

cudaEvent_t take_event() {
    if (!g_event_pool.empty()) {
        cudaEvent_t e = g_event_pool.back();
        g_event_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}

// Graph capture on this thread (dq_graph_solve_batched): launches are
// counted into the graph, not the global counter, tile launches take no
// timing events, and the work table is copied from the graph's pinned copy.
thread_local bool t_capturing = false;
thread_local int64_t t_captured_launches = 0;
thread_local void *t_pinned_table = nullptr;

void count_launches(int k) {
    if (t_capturing) t_captured_launches += k;
    else g_launches.fetch_add(k, std::memory_order_relaxed);
}

struct FmtInfo {
    int combo;
    int G;
    float qmax;
    int bits;       // stored bits per code
};

dq_status check_format(const dq_format *f, FmtInfo *out) {
    if (!f) return DQ_ERR_ARG;
    if (f->group != 16 && f->group != 32 && f->group != 64) return DQ_ERR_FORMAT;
    if (f->tensor_scale_auto != 0 && f->tensor_scale_auto != 1) return DQ_ERR_FORMAT;
    if (f->tensor_scale_auto && f->group_scale != DQ_SCALE_E4M3) return DQ_ERR_FORMAT;
    int combo = -1;
    const int c = f->codes, g = f->group_scale, o = f->outer_scale;
    if (c == DQ_CODES_INT4 && g == DQ_SCALE_BF16 && o == DQ_SCALE_BF16) combo = COMBO_INT4_BF16_BF16;
    if (c == DQ_CODES_INT4 && g == DQ_SCALE_E8M0 && o == DQ_SCALE_E8M0) combo = COMBO_INT4_E8M0_E8M0;
    if (c == DQ_CODES_E2M1 && g == DQ_SCALE_E8M0 && o == DQ_SCALE_E8M0) combo = COMBO_E2M1_E8M0_E8M0;
    if (c == DQ_CODES_E2M1 && g == DQ_SCALE_E4M3 && o == DQ_SCALE_BF16) combo = COMBO_E2M1_E4M3_BF16;
    if (c == DQ_CODES_INT4 && g == DQ_SCALE_E8M0 && o == DQ_SCALE_BF16) combo = COMBO_INT4_E8M0_BF16;
    if (c == DQ_CODES_E2M1 && g == DQ_SCALE_E8M0 && o == DQ_SCALE_BF16) combo = COMBO_E2M1_E8M0_BF16;
    // the other MX element formats: E8M0 group and outer scales only
    const bool mx = g == DQ_SCALE_E8M0 && o == DQ_SCALE_E8M0;
    if (mx && c == DQ_CODES_INT8) combo = COMBO_INT8_E8M0_E8M0;
    if (mx && c == DQ_CODES_E4M3) combo = COMBO_E4M3_E8M0_E8M0;
    if (mx && c == DQ_CODES_E5M2) combo = COMBO_E5M2_E8M0_E8M0;
    if (mx && c == DQ_CODES_E2M3) combo = COMBO_E2M3_E8M0_E8M0;
    if (mx && c == DQ_CODES_E3M2) combo = COMBO_E3M2_E8M0_E8M0;
    if (combo < 0) return DQ_ERR_FORMAT;
    if (out) {
        static const float qmax[7] = {7.0f, 6.0f, 127.0f, 448.0f, 57344.0f, 7.5f, 28.0f};
        static const int bits[7] = {4, 4, 8, 8, 8, 6, 6};
        out->combo = combo;
        out->G = f->group;
        out->qmax = qmax[c];
        out->bits = bits[c];
    }
    return DQ_OK;
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Tile geometry of one matrix (see the tile kernel's description).
// Workspace bytes of one matrix (each region 256-byte aligned).
size_t matrix_ws(int64_t rows, int64_t cols, bool f32) {
    const Geom g = geometry(rows, cols, f32);
    size_t b = 0;
    b += round_up((size_t)rows * g.ncb * sizeof(float2), 256);               // rowpart
    b += round_up((size_t)rows * g.ncb * sizeof(float), 256);                // rowsq
    b += round_up((size_t)rows * sizeof(double), 256);                       // w2row
    b += round_up((size_t)((rows + kRowFinRows - 1) / kRowFinRows) * 8, 256); // mse_part
    b += round_up((size_t)g.nrb_col * cols * sizeof(float2), 256);           // colpart
    b += round_up((size_t)std::max(g.ntiles[0], g.ntiles[2]) * 8, 256);      // res_row
    b += round_up((size_t)g.ntiles[1] * 8, 256);                             // res_col
    b += 256;                                                                // amax
    return b;
}

size_t table_ws(int n) { return n > 1 ? round_up((size_t)n * sizeof(MatDesc), 256) : 0; }

struct Carve {
    char *p;
    char *end;
    template <class T> T *take(size_t bytes) {
        T *r = reinterpret_cast<T *>(p);
        p += round_up(bytes, 256);
        return r;
    }
};

// Fill geometry and workspace pointers of one descriptor.
void place(MatDesc &d, bool f32, Carve &cv, int64_t tile_base[3], int64_t &row_base,
           int64_t &col_base, int64_t &unit_base, int64_t &chunk_base, bool tall = false) {
    const Geom g = geometry(d.rows, d.cols, f32, tall);
    d.wc = g.wc;
    d.ncb = g.ncb;
    for (int m = 0; m < 3; ++m) {
        d.tr[m] = g.tr[m];
        d.ntiles[m] = g.ntiles[m];
        d.tile0[m] = tile_base[m];
        tile_base[m] += g.ntiles[m];
    }
    d.row0 = row_base;
    d.col0 = col_base;
    // (work units of the column finalize before this matrix)
    d.cunit0 = unit_base;
    unit_base += col_units(g.nrb_col, d.cols);
    // (256-row chunks of the row finalize, likewise)
    d.rchunk0 = chunk_base;
    chunk_base += (d.rows + kRowFinRows - 1) / kRowFinRows;
    row_base += d.rows;
    col_base += d.cols;
    if (cv.p) {
        d.rowpart = cv.take<float2>((size_t)d.rows * g.ncb * sizeof(float2));
        d.rowsq = cv.take<float>((size_t)d.rows * g.ncb * sizeof(float));
        d.w2row = cv.take<double>((size_t)d.rows * sizeof(double));
        d.mse_part = cv.take<double>((size_t)((d.rows + kRowFinRows - 1) / kRowFinRows) * sizeof(double));
        d.colpart = cv.take<float2>((size_t)g.nrb_col * d.cols * sizeof(float2));
        d.res_row = cv.take<double>((size_t)std::max(g.ntiles[0], g.ntiles[2]) * 8);
        d.res_col = cv.take<double>((size_t)g.ntiles[1] * 8);
        d.amax = cv.take<unsigned int>(256);
    }
}

cudaError_t launch_tiles(int combo, const TileLaunch &L) {
    switch (combo) {
        case 0: return launch_tile_c0(L);
        case 1: return launch_tile_c1(L);
        case 2: return launch_tile_c2(L);
        case 3: return launch_tile_c3(L);
        case 4: return launch_tile_c4(L);
        case 5: return launch_tile_c5(L);
        case 6: return launch_tile_c6(L);
        case 7: return launch_tile_c7(L);
        case 8: return launch_tile_c8(L);
        case 9: return launch_tile_c9(L);
        case 10: return launch_tile_c10(L);
    }
    return cudaErrorInvalidValue;
}

// format sets whose group and outer scales are both E8M0 (the MX family)
bool all_e8m0(int combo) {
    return combo == COMBO_INT4_E8M0_E8M0 || combo == COMBO_E2M1_E8M0_E8M0 ||
           combo >= COMBO_INT8_E8M0_E8M0;
}

int outer_of(int combo) { return all_e8m0(combo) ? SC_E8M0 : SC_BF16; }

unsigned grid_for(int64_t n, int block) {
    int64_t g = (n + block - 1) / block;
    if (g > 148 * 32) g = 148 * 32;
    return (unsigned)(g < 1 ? 1 : g);
}

#define DQ_CUDA(x)                                      \
    do {                                                \
        cudaError_t e_ = (x);                           \
        if (e_ != cudaSuccess) return DQ_ERR_CUDA;      \
    } while (0)

struct Launcher {
    Table tab;
    const MatDesc *host_table = nullptr;   // host copy of tab.dev's entries
    int combo, G;
    bool f32;
    float qmax;
    int64_t tiles[3] = {0, 0, 0};
    int64_t total_rows = 0, total_cols = 0;
    cudaStream_t st;
    // the iterations take each row's squared error from its row sums (4-bit
    // codes; set when an MSE output is wanted)
    bool row_mse = false;

    // One tile pass.  A gated pass (the literal fallback of a fused
    // iteration) launches a small grid that visits the tiles grid-stride and
    // returns at once unless its flag is up.
    dq_status tiles_pass(int mode, bool want_res, unsigned int *flags = nullptr, int gate = 0) {
        TileLaunch L;
        L.tab = tab;
        L.mode = mode;
        L.slot = (mode == MODE_ACT) ? 2
                 : ((mode == MODE_FUSED || mode == MODE_FUSED_W2) ? 1 : (mode == MODE_ROW_W2 ? 0 : mode));
        L.tiles = tiles[L.slot];
        L.grid = gate ? std::min<int64_t>(L.tiles, 148) : L.tiles;
        L.f32 = f32 ? 1 : 0;
        L.G = G;
        L.want_res = want_res ? 1 : 0;
        L.flags = flags;
        L.gate = gate;
        L.stream = st;
        if (L.grid <= 0) return DQ_OK;
        cudaEvent_t beg = nullptr, end = nullptr;
        // (the variants that also sum each row's squares are timed as their kind)
        const int kind = mode == MODE_FUSED_W2 ? MODE_FUSED : (mode == MODE_ROW_W2 ? MODE_ROW : mode);
        {
            std::lock_guard<std::mutex> lk(g_timing_mu);
            if (!t_capturing && (g_timing_kinds & (1u << kind))) { beg = take_event(); end = take_event(); }
        }
        if (beg && end) DQ_CUDA(cudaEventRecord(beg, st));
        DQ_CUDA(launch_tiles(combo, L));
        count_launches(1);
        if (beg && end) {
            DQ_CUDA(cudaEventRecord(end, st));
            std::lock_guard<std::mutex> lk(g_timing_mu);
            g_timed.push_back({beg, end, kind});
        }
        return DQ_OK;
    }
    dq_status row_finalize(unsigned int *flags = nullptr, unsigned int *next_flags = nullptr,
                           int rmse = 0) {
        if (total_rows == 0) return DQ_OK;
        // one block per 256-row chunk (chunks of all matrices, in order)
        int64_t chunks = 0;
        for (int i = 0; i < tab.n; ++i) {
            const MatDesc &d = tab.dev ? host_table[i] : tab.one;
            chunks += (d.rows + kRowFinRows - 1) / kRowFinRows;
        }
        const dim3 grid((unsigned)std::max<int64_t>(1, std::min<int64_t>(chunks, 148 * 32)));
        if (outer_of(combo) == SC_E8M0)
            DQ_CUDA(launch_k(row_finalize_kernel<SC_E8M0>, grid, dim3(kRowFinRows), 0, st, tab,
                             chunks, flags, next_flags, rmse));
        else
            DQ_CUDA(launch_k(row_finalize_kernel<SC_BF16>, grid, dim3(kRowFinRows), 0, st, tab,
                             chunks, flags, next_flags, rmse));
        count_launches(1);
        return DQ_OK;
    }
    // The column update of every matrix; with mse_mode the same launch also
    // finishes the iteration's MSE (MSE_FUSED: flags / clear of the one-pass
    // iteration; MSE_LITERAL: the row and column passes' residuals), entry idx.
    dq_status col_finalize(int mse_mode = MSE_NONE, unsigned int *flags = nullptr,
                           unsigned int *clear = nullptr, int idx = 0) {
        if (total_cols == 0 && mse_mode == MSE_NONE) return DQ_OK;
        // one block per work unit (units of all matrices, in order)
        int64_t units = 0;
        for (int i = 0; i < tab.n; ++i) {
            const MatDesc &d = tab.dev ? host_table[i] : tab.one;
            units += col_units(d.ntiles[MODE_COL] / std::max(d.ncb, 1), d.cols);
        }
        const int64_t gcols = total_cols == 0 ? 0 : std::max<int64_t>(1, std::min<int64_t>(units, 148 * 16));
        const unsigned grid = (unsigned)(gcols + (mse_mode != MSE_NONE ? (2 * tab.n + 7) / 8 : 0));
        const int threads = kColFinThreads;
        if (outer_of(combo) == SC_E8M0)
            DQ_CUDA(launch_k(col_finalize_kernel<SC_E8M0>, dim3(grid), dim3(threads), 0, st, tab,
                             units, mse_mode, flags, clear, idx));
        else
            DQ_CUDA(launch_k(col_finalize_kernel<SC_BF16>, dim3(grid), dim3(threads), 0, st, tab,
                             units, mse_mode, flags, clear, idx));
        count_launches(1);
        return DQ_OK;
    }
    dq_status mse(int row_slot, int idx_trace, int idx_half, double *out_row, double *out_col) {
        // a warp per (matrix, which), 8 per block
        DQ_CUDA(launch_k(mse_finalize_kernel, dim3((2 * tab.n + 7) / 8), dim3(256), 0, st, tab, row_slot,
                         idx_trace, idx_half, out_row, out_col));
        count_launches(1);
        return DQ_OK;
    }

    // One BCD iteration: row statistics, row update, column statistics,
    // column update, MSE.  With power-of-two outer and group scales (MX
    // formats) both statistics come from one pass over W (`fused`); the
    // literal passes stand by behind the iteration's flags.
    dq_status iteration(int t, bool fused, unsigned int *flag_slots, bool want_trace,
                        bool want_half) {
        dq_status s;
        // iteration t uses flag slot t % 3; its row finalize may raise the
        // next slot, its MSE kernel clears the slot after that
        unsigned int *flags = flag_slots + 2 * (t % 3);
        unsigned int *next = flag_slots + 2 * ((t + 1) % 3);
        unsigned int *clear = flag_slots + 2 * ((t + 2) % 3);
        if (!fused) {
            // with row_mse the first iteration's row pass also sums the rows' squares
            const int rmode = (row_mse && t == 0) ? MODE_ROW_W2 : MODE_ROW;
            if ((s = tiles_pass(rmode, want_trace)) != DQ_OK) return s;
            if ((s = row_finalize(nullptr, nullptr, row_mse ? (t == 0 ? 2 : 1) : 0)) != DQ_OK) return s;
            if ((s = tiles_pass(MODE_COL, want_half)) != DQ_OK) return s;
            return col_finalize(row_mse ? MSE_LITERAL_ROWS : MSE_LITERAL, nullptr, nullptr, t);
        }
        // with row_mse the first iteration's pass also sums the rows' squares
        const int fmode = (row_mse && t == 0) ? MODE_FUSED_W2 : MODE_FUSED;
        if ((s = tiles_pass(fmode, want_trace || want_half, flags, 0)) != DQ_OK) return s;
        if ((s = tiles_pass(MODE_ROW, want_trace, flags, 1)) != DQ_OK) return s;
        if ((s = row_finalize(flags, next, row_mse ? (t == 0 ? 2 : 1) : 0)) != DQ_OK) return s;
        if ((s = tiles_pass(MODE_COL, want_half, flags, 2)) != DQ_OK) return s;
        return col_finalize(row_mse ? MSE_FUSED_ROWS : MSE_FUSED, flags, clear, t);
    }
};

// MX formats: power-of-two outer and group scales
bool fused_ok(int combo) { return all_e8m0(combo); }
// Formats with 4-bit codes: their iterations take the squared error of the
// state per row from the row sums (about 1% of sum W^2 for 4-bit codes, so
// the float32 row sums leave it correct to about 1e-5 relative; wider
// codes, whose error is a far smaller share of sum W^2, sum (W - R)^2
// directly)
bool row_mse_ok(int combo) { return combo <= COMBO_E2M1_E8M0_BF16; }

thread_local std::vector<MatDesc> t_table;
thread_local std::vector<int> t_order;

// Host-side checks of a batched solve's arguments (no CUDA call).
dq_status check_batch(int32_t n, const dq_matrix *mats, int32_t dtype, const dq_format *fmt,
                      int32_t T, void *workspace, size_t ws_bytes, FmtInfo *fi_out) {
    if (n < 0 || T < 0 || !mats) return DQ_ERR_ARG;
    if (dtype != DQ_DT_F32 && dtype != DQ_DT_BF16) return DQ_ERR_ARG;
    FmtInfo fi;
    dq_status s = check_format(fmt, &fi);
    if (s != DQ_OK) return s;
    if (fi_out) *fi_out = fi;
    if (n == 0) return DQ_OK;
    const bool f32 = dtype == DQ_DT_F32;
    size_t need = table_ws(n) + 256;
    for (int i = 0; i < n; ++i) {
        const dq_matrix &m = mats[i];
        if (m.rows < 0 || m.cols < 0) return DQ_ERR_SHAPE;
        if (m.cols % fi.G) return DQ_ERR_SHAPE;
        const bool empty = m.rows == 0 || m.cols == 0;
        if (!empty && (!m.W || !m.codes || !m.gscales)) return DQ_ERR_ARG;
        if ((m.rows > 0 && !m.a) || (m.cols > 0 && !m.b) || !m.tensor_scale) return DQ_ERR_ARG;
        if (!aligned(m.W, 16) || !aligned(m.codes, 16) || !aligned(m.gscales, 16)) return DQ_ERR_ALIGN;
        if (!aligned(m.a, 4) || !aligned(m.b, 4) || !aligned(m.tensor_scale, 4)) return DQ_ERR_ALIGN;
        if (!aligned(m.a0, 4) || !aligned(m.b0, 4)) return DQ_ERR_ALIGN;
        if (!aligned(m.mse_trace, 8) || !aligned(m.mse_half, 8)) return DQ_ERR_ALIGN;
        need += matrix_ws(m.rows, m.cols, f32);
    }
    if (!workspace || ws_bytes < need) return DQ_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return DQ_ERR_ALIGN;
    return DQ_OK;
}

// Whether a batch is tall (see geometry): its column passes make at least
// kTallTiles tiles at the default geometry.
bool tall_batch(int32_t n, const dq_matrix *mats, bool f32) {
    int64_t tiles = 0;
    for (int i = 0; i < n; ++i) tiles += geometry(mats[i].rows, mats[i].cols, f32).ntiles[1];
    return tiles >= kTallTiles;
}
// The same choice for one matrix alone (the single-matrix entry points take
// it, so that their sums are those of dq_solve_dual_scale).
bool tall_single(int64_t rows, int64_t cols, bool f32) {
    return geometry(rows, cols, f32).ntiles[1] >= kTallTiles;
}

// tall_hint: -1 decides from this batch; 0 or 1 as given (a call that solves
// a batch in parts passes the whole batch's choice, so that every part has
// the geometry, and the sums, of the whole).
dq_status solve_impl(int32_t n, const dq_matrix *mats, int32_t dtype, const dq_format *fmt,
                     int32_t T, void *workspace, size_t ws_bytes, cudaStream_t st,
                     int tall_hint = -1) {
    FmtInfo fi;
    dq_status s = check_batch(n, mats, dtype, fmt, T, workspace, ws_bytes, &fi);
    if (s != DQ_OK || n == 0) return s;
    const bool f32 = dtype == DQ_DT_F32;
    const bool tall = tall_hint < 0 ? tall_batch(n, mats, f32) : tall_hint != 0;

    unsigned int *status = status_ptr();
    if (!status) return DQ_ERR_CUDA;

    Carve cv{static_cast<char *>(workspace), static_cast<char *>(workspace) + ws_bytes};
    MatDesc *dev_table = n > 1 ? cv.take<MatDesc>((size_t)n * sizeof(MatDesc)) : nullptr;
    unsigned int *flags = cv.take<unsigned int>(256);     // fused-path flags: 3 slots x 2 words
    // The work table lists the matrices by decreasing tile height (stable):
    // CTAs are dispatched in tile order, so the short tiles of short matrices
    // fill the last wave instead of leaving SMs idle behind full-size tiles.
    // Each matrix's tiles and sums depend on its own shape (and the batch's
    // tall choice) alone, so the order changes no result.
    t_order.resize(n);
    for (int i = 0; i < n; ++i) t_order[i] = i;
    std::stable_sort(t_order.begin(), t_order.end(), [&](int x, int y) {
        return geometry(mats[x].rows, mats[x].cols, f32, tall).tr[1] >
               geometry(mats[y].rows, mats[y].cols, f32, tall).tr[1];
    });
    t_table.assign(n, MatDesc{});
    int64_t tile_base[3] = {0, 0, 0}, row_base = 0, col_base = 0, unit_base = 0, chunk_base = 0;
    for (int i = 0; i < n; ++i) {
        const dq_matrix &m = mats[t_order[i]];
        MatDesc &d = t_table[i];
        d.W = m.W;
        d.rows = m.rows;
        d.cols = m.cols;
        d.a = m.a;
        d.b = m.b;
        d.a_out = m.a;
        d.b_out = m.b;
        d.codes = m.codes;
        d.gscales = m.gscales;
        d.ts_ptr = m.tensor_scale;
        d.ts_out = m.tensor_scale;
        d.ts_val = 1.0f;
        d.a0 = m.a0;
        d.b0 = m.b0;
        d.mse_trace = m.mse_trace;
        d.mse_half = m.mse_half;
        place(d, f32, cv, tile_base, row_base, col_base, unit_base, chunk_base, tall);
    }
    Launcher L;
    L.tab.dev = dev_table;
    L.host_table = t_table.data();
    L.tab.n = n;
    L.tab.status = status;
    if (n == 1) L.tab.one = t_table[0];
    L.combo = fi.combo;
    L.G = fi.G;
    L.f32 = f32;
    L.qmax = fi.qmax;
    for (int m = 0; m < 3; ++m) L.tiles[m] = tile_base[m];
    L.total_rows = row_base;
    L.total_cols = col_base;
    L.st = st;
    if (dev_table) {
        // (inside a graph capture the copy reads the graph's pinned table,
        // which every replay uploads again)
        const void *src = t_table.data();
        if (t_pinned_table) {
            std::memcpy(t_pinned_table, t_table.data(), (size_t)n * sizeof(MatDesc));
            src = t_pinned_table;
        }
        DQ_CUDA(cudaMemcpyAsync(dev_table, src, (size_t)n * sizeof(MatDesc),
                                cudaMemcpyHostToDevice, st));
    }

    // tensor scale (NVFP4 weights: from amax of W; otherwise 1)
    if (fmt->tensor_scale_auto) {
        for (int i = 0; i < n; ++i)
            DQ_CUDA(cudaMemsetAsync(t_table[i].amax, 0, sizeof(unsigned int), st));
        if (L.tiles[2] > 0) {
            if (f32) DQ_CUDA(launch_k(amax_kernel<float>, dim3((unsigned)L.tiles[2]),
                                      dim3(kThreads), 0, st, L.tab));
            else DQ_CUDA(launch_k(amax_kernel<Bf16Tag>, dim3((unsigned)L.tiles[2]), dim3(kThreads),
                                  0, st, L.tab));
            count_launches(1);
        }
    }
    DQ_CUDA(launch_k(tensor_scale_kernel, dim3((n + 127) / 128), dim3(128), 0, st, L.tab, fi.qmax,
                     fmt->tensor_scale_auto));
    count_launches(1);
    const bool fused = fused_ok(fi.combo) && T > 0;
    if (fused) DQ_CUDA(cudaMemsetAsync(flags, 0, 6 * sizeof(unsigned int), st));
    if (row_base + col_base > 0) {
        DQ_CUDA(launch_k(init_state_kernel, dim3(grid_for(row_base + col_base, 256)), dim3(256), 0,
                         st, L.tab, row_base, col_base, fused ? flags : nullptr));
        count_launches(1);
    }
    bool want_trace = false, want_half = false;
    for (int i = 0; i < n; ++i) {
        want_trace |= mats[i].mse_trace != nullptr;
        want_half |= mats[i].mse_half != nullptr;
    }
    L.row_mse = T > 0 && row_mse_ok(fi.combo) && (want_trace || want_half);
    for (int t = 0; t < T; ++t)
        if ((s = L.iteration(t, fused, flags, want_trace, want_half)) != DQ_OK) return s;
    if ((s = L.tiles_pass(MODE_PACK, want_trace)) != DQ_OK) return s;
    if ((s = L.mse(2, T, -1, nullptr, nullptr)) != DQ_OK) return s;
    return DQ_OK;
}

// Single-matrix descriptor for the no-workspace / step entry points.
dq_status single(const void *W, int32_t dtype, int64_t rows, int64_t cols, const dq_format *fmt,
                 FmtInfo *fi, MatDesc &d) {
    if (dtype != DQ_DT_F32 && dtype != DQ_DT_BF16) return DQ_ERR_ARG;
    dq_status s = check_format(fmt, fi);
    if (s != DQ_OK) return s;
    if (rows < 0 || cols < 0) return DQ_ERR_SHAPE;
    if (cols % fi->G) return DQ_ERR_SHAPE;
    if (rows > 0 && cols > 0 && !W) return DQ_ERR_ARG;
    if (!aligned(W, 16)) return DQ_ERR_ALIGN;
    d = MatDesc{};
    d.W = W;
    d.rows = rows;
    d.cols = cols;
    d.ts_val = 1.0f;
    return DQ_OK;
}

dq_status step_impl(bool row_step, const void *W, int32_t dtype, int64_t rows, int64_t cols,
                    const dq_format *fmt, float ts, const float *a_in, const float *b_in,
                    float *out, float *pre, double *mse_in, void *workspace, size_t ws_bytes,
                    cudaStream_t st) {
    FmtInfo fi;
    MatDesc d;
    dq_status s = single(W, dtype, rows, cols, fmt, &fi, d);
    if (s != DQ_OK) return s;
    if (!a_in || !b_in || !out) return DQ_ERR_ARG;
    if (!(ts > 0.0f)) return DQ_ERR_ARG;
    if (fmt->group_scale != DQ_SCALE_E4M3 && ts != 1.0f) return DQ_ERR_ARG;
    if (!aligned(a_in, 4) || !aligned(b_in, 4) || !aligned(out, 4) || !aligned(pre, 4) ||
        !aligned(mse_in, 8))
        return DQ_ERR_ALIGN;
    const bool f32 = dtype == DQ_DT_F32;
    if (!workspace || ws_bytes < matrix_ws(rows, cols, f32)) return DQ_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return DQ_ERR_ALIGN;
    unsigned int *status = status_ptr();
    if (!status) return DQ_ERR_CUDA;
    d.a = a_in;
    d.b = b_in;
    d.ts_val = ts;
    if (row_step) { d.a_out = out; d.a_pre = pre; }
    else { d.b_out = out; d.b_pre = pre; }
    Carve cv{static_cast<char *>(workspace), static_cast<char *>(workspace) + ws_bytes};
    int64_t tb[3] = {0, 0, 0}, rb = 0, cb = 0, sb = 0, hb = 0;
    place(d, f32, cv, tb, rb, cb, sb, hb, tall_single(d.rows, d.cols, f32));
    Launcher L;
    L.tab.dev = nullptr;
    L.tab.one = d;
    L.tab.n = 1;
    L.tab.status = status;
    L.combo = fi.combo;
    L.G = fi.G;
    L.f32 = f32;
    L.qmax = fi.qmax;
    for (int m = 0; m < 3; ++m) L.tiles[m] = tb[m];
    L.total_rows = rb;
    L.total_cols = cb;
    L.st = st;
    if (row_step) {
        // 4-bit codes: the state's squared error from the row sums, with the
        // rows' squares summed by the same pass
        const bool rows = mse_in != nullptr && row_mse_ok(fi.combo);
        if ((s = L.tiles_pass(rows ? MODE_ROW_W2 : MODE_ROW, mse_in != nullptr)) != DQ_OK) return s;
        if ((s = L.row_finalize(nullptr, nullptr, rows ? 2 : 0)) != DQ_OK) return s;
        if (mse_in) return L.mse(rows ? kSlotRows : MODE_ROW, -1, -1, mse_in, nullptr);
    } else {
        if ((s = L.tiles_pass(MODE_COL, mse_in != nullptr)) != DQ_OK) return s;
        if ((s = L.col_finalize()) != DQ_OK) return s;
        if (mse_in) return L.mse(-1, -1, -1, nullptr, mse_in);
    }
    return DQ_OK;
}

// Column statistics of a row shard with the whole matrix's row blocks
// (dq_col_partials): the column pass of one matrix whose row blocks have
// `row_block` rows, writing its partial sums to the caller's slab.
dq_status col_partials_impl(const void *W, int32_t dtype, int64_t rows, int64_t cols,
                            const dq_format *fmt, float ts, const float *a, const float *b,
                            int64_t row_block, float *partials, double *mse, void *workspace,
                            size_t ws_bytes, cudaStream_t st) {
    FmtInfo fi;
    MatDesc d;
    dq_status s = single(W, dtype, rows, cols, fmt, &fi, d);
    if (s != DQ_OK) return s;
    if (!a || !b || !partials) return DQ_ERR_ARG;
    if (!(ts > 0.0f)) return DQ_ERR_ARG;
    if (fmt->group_scale != DQ_SCALE_E4M3 && ts != 1.0f) return DQ_ERR_ARG;
    if (!aligned(a, 4) || !aligned(b, 4) || !aligned(partials, 16) || !aligned(mse, 8))
        return DQ_ERR_ALIGN;
    const bool f32 = dtype == DQ_DT_F32;
    const Geom g = geometry(rows, cols, f32);
    const int wr = kWarps / g.wc;
    // (the residual slots in the workspace are sized for the shard's own row
    // blocks: a row block below the shard's own is refused; the row block
    // of a matrix never decreases with its rows, so a shard of it passes)
    if (row_block <= 0 || row_block % wr || row_block / wr > kRowsPerWarp[MODE_COL] ||
        row_block < g.tr[1])
        return DQ_ERR_SHAPE;
    if (!workspace || ws_bytes < matrix_ws(rows, cols, f32)) return DQ_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return DQ_ERR_ALIGN;
    if (rows == 0 || cols == 0) return DQ_OK;
    unsigned int *status = status_ptr();
    if (!status) return DQ_ERR_CUDA;
    d.a = a;
    d.b = b;
    d.ts_val = ts;
    Carve cv{static_cast<char *>(workspace), static_cast<char *>(workspace) + ws_bytes};
    int64_t tb[3] = {0, 0, 0}, rb = 0, cb = 0, sb = 0, hb = 0;
    place(d, f32, cv, tb, rb, cb, sb, hb);
    // the column pass with the whole matrix's row blocks, into the caller's slab
    d.tr[1] = (int32_t)row_block;
    d.ntiles[1] = (rows + row_block - 1) / row_block * d.ncb;
    d.colpart = reinterpret_cast<float2 *>(partials);
    Launcher L;
    L.tab.dev = nullptr;
    L.tab.one = d;
    L.tab.n = 1;
    L.tab.status = status;
    L.combo = fi.combo;
    L.G = fi.G;
    L.f32 = f32;
    L.qmax = fi.qmax;
    L.tiles[0] = d.ntiles[0];
    L.tiles[1] = d.ntiles[1];
    L.tiles[2] = d.ntiles[2];
    L.total_rows = rb;
    L.total_cols = cb;
    L.st = st;
    if ((s = L.tiles_pass(MODE_COL, mse != nullptr)) != DQ_OK) return s;
    if (mse) return L.mse(-1, -1, -1, nullptr, mse);
    return DQ_OK;
}

// Value of the stored code of element (r, c) (layouts as the tile kernel
// writes them: 4-bit codes two per byte, 8-bit one per byte, 6-bit four per
// 3 bytes).  Float element formats decode from their bit fields.
__device__ float code_value(const uint8_t *codes, int64_t r, int64_t c, int64_t cols, int kind) {
    if (kind == DQ_CODES_INT4 || kind == DQ_CODES_E2M1) {
        const uint8_t byte = codes[r * (cols / 2) + c / 2];
        const uint32_t nib = (c & 1) ? (byte >> 4) : (byte & 0xF);
        if (kind == DQ_CODES_INT4) return (float)((int)(nib ^ 8u) - 8);
        const float mag[8] = {0.f, 0.5f, 1.f, 1.5f, 2.f, 3.f, 4.f, 6.f};
        return (nib & 8u) ? -mag[nib & 7u] : mag[nib & 7u];
    }
    if (kind == DQ_CODES_INT8) return (float)(int8_t)codes[r * cols + c];
    uint32_t u;
    int eb, mb, bias;
    if (kind == DQ_CODES_E4M3 || kind == DQ_CODES_E5M2) {
        u = codes[r * cols + c];
        eb = kind == DQ_CODES_E4M3 ? 4 : 5;
    } else {
        const uint8_t *q = codes + r * (cols / 4 * 3) + (c / 4) * 3;
        const uint32_t w = q[0] | ((uint32_t)q[1] << 8) | ((uint32_t)q[2] << 16);
        u = (w >> (6 * (c % 4))) & 0x3Fu;
        eb = kind == DQ_CODES_E2M3 ? 2 : 3;
    }
    mb = (kind == DQ_CODES_E4M3 || kind == DQ_CODES_E2M3) ? 3 : 2;
    bias = (1 << (eb - 1)) - 1;
    const uint32_t e = (u >> mb) & ((1u << eb) - 1), m = u & ((1u << mb) - 1);
    const float v = e == 0 ? ldexpf((float)m, 1 - bias - mb)
                           : ldexpf((float)((1u << mb) + m), (int)e - bias - mb);
    return (u >> (eb + mb)) & 1u ? -v : v;
}

// out_ij = a_i * c_ij * s_g * ts * b_j
__global__ void dequant_kernel(const uint8_t *codes, const void *gs, int64_t rows, int64_t cols,
                               int G, int codes_kind, int gs_kind, float ts, const float *a,
                               const float *b, float *out) {
    grid_dependency_begin();
    const int64_t n = rows * cols;
    for (int64_t k = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; k < n;
         k += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = k / cols, c = k % cols;
        const float cv = code_value(codes, r, c, cols, codes_kind);
        const int64_t gi = r * (cols / G) + c / G;
        float s;
        if (gs_kind == DQ_SCALE_BF16) {
            s = __uint_as_float((uint32_t)reinterpret_cast<const uint16_t *>(gs)[gi] << 16);
        } else if (gs_kind == DQ_SCALE_E8M0) {
            s = __uint_as_float((uint32_t)reinterpret_cast<const uint8_t *>(gs)[gi] << 23);
        } else {
            const uint32_t e = reinterpret_cast<const uint8_t *>(gs)[gi];
            const uint32_t ex = (e >> 3) & 15u, m = e & 7u;
            s = ex == 0 ? (float)m * 0.001953125f : __uint_as_float(((ex + 120u) << 23) | (m << 20));
            if (e & 128u) s = -s;
        }
        const float av = a ? a[r] : 1.0f, bv = b ? b[c] : 1.0f;
        out[k] = av * (cv * (s * ts)) * bv;
    }
}

}  // namespace

extern "C" {

const char *dq_version(void) { return "dq 0.1.0 (sm_100a)"; }

const char *dq_strerror(dq_status s) {
    switch (s) {
        case DQ_OK: return "ok";
        case DQ_ERR_ARG: return "invalid argument";
        case DQ_ERR_SHAPE: return "invalid shape (cols must be a multiple of the group size)";
        case DQ_ERR_FORMAT: return "unsupported format";
        case DQ_ERR_NONFINITE: return "non-finite value in the input";
        case DQ_ERR_RANGE: return "an outer scale was clamped at its set's bound";
        case DQ_ERR_CUDA: return "CUDA runtime error";
        case DQ_ERR_WORKSPACE: return "workspace missing or too small";
        case DQ_ERR_NOT_IMPLEMENTED: return "not implemented";
        case DQ_ERR_ALIGN: return "pointer alignment";
        case DQ_ERR_SCRATCH:
            return "matrix needs more scratch than the built-in 32 MiB buffer of "
                   "dq_solve_dual_scale_noalloc holds";
        case DQ_ERR_TIMEOUT: return "a kernel's bounded wait ran out (stalled pipeline)";
    }
    return "unknown status";
}

dq_status dq_format_preset(const char *name, int32_t group, dq_format *out) {
    if (!name || !out) return DQ_ERR_ARG;
    dq_format f{};
    if (!strcmp(name, "int4_bf16")) f = {DQ_CODES_INT4, 64, DQ_SCALE_BF16, DQ_SCALE_BF16, 0};
    else if (!strcmp(name, "mxint4")) f = {DQ_CODES_INT4, 32, DQ_SCALE_E8M0, DQ_SCALE_E8M0, 0};
    else if (!strcmp(name, "mxfp4")) f = {DQ_CODES_E2M1, 32, DQ_SCALE_E8M0, DQ_SCALE_E8M0, 0};
    else if (!strcmp(name, "nvfp4")) f = {DQ_CODES_E2M1, 16, DQ_SCALE_E4M3, DQ_SCALE_BF16, 1};
    else if (!strcmp(name, "mxint8")) f = {DQ_CODES_INT8, 32, DQ_SCALE_E8M0, DQ_SCALE_E8M0, 0};
    else if (!strcmp(name, "mxfp8_e4m3")) f = {DQ_CODES_E4M3, 32, DQ_SCALE_E8M0, DQ_SCALE_E8M0, 0};
    else if (!strcmp(name, "mxfp8_e5m2")) f = {DQ_CODES_E5M2, 32, DQ_SCALE_E8M0, DQ_SCALE_E8M0, 0};
    else if (!strcmp(name, "mxfp6_e2m3")) f = {DQ_CODES_E2M3, 32, DQ_SCALE_E8M0, DQ_SCALE_E8M0, 0};
    else if (!strcmp(name, "mxfp6_e3m2")) f = {DQ_CODES_E3M2, 32, DQ_SCALE_E8M0, DQ_SCALE_E8M0, 0};
    else if (!strcmp(name, "mxint4_bf16outer")) f = {DQ_CODES_INT4, 32, DQ_SCALE_E8M0, DQ_SCALE_BF16, 0};
    else if (!strcmp(name, "mxfp4_bf16outer")) f = {DQ_CODES_E2M1, 32, DQ_SCALE_E8M0, DQ_SCALE_BF16, 0};
    else return DQ_ERR_FORMAT;
    if (group != 0) f.group = group;
    dq_status s = check_format(&f, nullptr);
    if (s != DQ_OK) return s;
    *out = f;
    return DQ_OK;
}

int64_t dq_code_bytes(const dq_format *fmt, int64_t rows, int64_t cols) {
    FmtInfo fi;
    if (check_format(fmt, &fi) != DQ_OK) return -1;
    if (rows < 0 || cols < 0 || cols % fi.G) return -1;
    return rows * (cols * fi.bits / 8);
}

dq_status dq_workspace_size(int32_t n, const int64_t *rows, const int64_t *cols,
                            const dq_format *fmt, size_t *bytes) {
    if (n < 0 || !bytes || (n > 0 && (!rows || !cols))) return DQ_ERR_ARG;
    FmtInfo fi;
    dq_status s = check_format(fmt, &fi);
    if (s != DQ_OK) return s;
    size_t b = table_ws(n);
    for (int i = 0; i < n; ++i) {
        if (rows[i] < 0 || cols[i] < 0 || cols[i] % fi.G) return DQ_ERR_SHAPE;
        // the larger of the bf16 and float32 layouts, so one size serves both
        b += std::max(matrix_ws(rows[i], cols[i], false), matrix_ws(rows[i], cols[i], true));
    }
    *bytes = b + 512;
    return DQ_OK;
}

dq_status dq_quantize(const void *X, int32_t dtype, int64_t rows, int64_t cols,
                      const dq_format *fmt, const float *a, const float *b, float tensor_scale,
                      uint8_t *codes, void *gscales, dq_stream stream) {
    FmtInfo fi;
    MatDesc d;
    dq_status s = single(X, dtype, rows, cols, fmt, &fi, d);
    if (s != DQ_OK) return s;
    if (rows == 0 || cols == 0) return DQ_OK;
    if (!codes || !gscales) return DQ_ERR_ARG;
    if (!(tensor_scale > 0.0f)) return DQ_ERR_ARG;
    if (fmt->group_scale != DQ_SCALE_E4M3 && tensor_scale != 1.0f) return DQ_ERR_ARG;
    if (!aligned(codes, 16) || !aligned(gscales, 16) || !aligned(a, 4) || !aligned(b, 4))
        return DQ_ERR_ALIGN;
    unsigned int *status = status_ptr();
    if (!status) return DQ_ERR_CUDA;
    const bool f32 = dtype == DQ_DT_F32;
    d.a = a;
    d.b = b;
    d.codes = codes;
    d.gscales = gscales;
    d.ts_val = tensor_scale;
    Carve none{nullptr, nullptr};
    int64_t tb[3] = {0, 0, 0}, rb = 0, cb = 0, sb = 0, hb = 0;
    place(d, f32, none, tb, rb, cb, sb, hb);
    Launcher L;
    L.tab.dev = nullptr;
    L.tab.one = d;
    L.tab.n = 1;
    L.tab.status = status;
    L.combo = fi.combo;
    L.G = fi.G;
    L.f32 = f32;
    L.qmax = fi.qmax;
    for (int m = 0; m < 3; ++m) L.tiles[m] = tb[m];
    L.st = reinterpret_cast<cudaStream_t>(stream);
    return L.tiles_pass(MODE_PACK, false);
}

dq_status dq_act_rescale_quant(const void *X, int64_t tokens, int64_t K, const float *b,
                               const dq_format *fmt, uint8_t *codes, void *gscales,
                               dq_stream stream) {
    FmtInfo fi;
    MatDesc d;
    dq_status s = single(X, DQ_DT_BF16, tokens, K, fmt, &fi, d);
    if (s != DQ_OK) return s;
    if (tokens == 0 || K == 0) return DQ_OK;
    if (!codes || !gscales || !b) return DQ_ERR_ARG;
    if (!aligned(codes, 16) || !aligned(gscales, 16) || !aligned(b, 4)) return DQ_ERR_ALIGN;
    unsigned int *status = status_ptr();
    if (!status) return DQ_ERR_CUDA;
    d.b = b;
    d.codes = codes;
    d.gscales = gscales;
    Carve none{nullptr, nullptr};
    int64_t tb[3] = {0, 0, 0}, rb = 0, cb = 0, sb = 0, hb = 0;
    place(d, false, none, tb, rb, cb, sb, hb);
    Launcher L;
    L.tab.dev = nullptr;
    L.tab.one = d;
    L.tab.n = 1;
    L.tab.status = status;
    L.combo = fi.combo;
    L.G = fi.G;
    L.f32 = false;
    L.qmax = fi.qmax;
    for (int m = 0; m < 3; ++m) L.tiles[m] = tb[m];
    L.st = reinterpret_cast<cudaStream_t>(stream);
    return L.tiles_pass(MODE_ACT, false);
}

dq_status dq_two_level_quant(const void *X, int32_t dtype, int64_t rows, int64_t cols,
                             int32_t dual_block, const dq_format *inner, uint8_t *codes,
                             void *inner_scales, float *outer_scales, float *qdq,
                             dq_stream stream) {
    if (!inner) return DQ_ERR_ARG;
    if (inner->codes != DQ_CODES_E2M1 || inner->group != 32 || inner->group_scale != DQ_SCALE_E8M0 ||
        inner->tensor_scale_auto != 0)
        return DQ_ERR_FORMAT;
    if (dual_block != 256 && dual_block != 512 && dual_block != 1024) return DQ_ERR_ARG;
    if (dtype != DQ_DT_F32 && dtype != DQ_DT_BF16) return DQ_ERR_ARG;
    if (rows < 0 || cols < 0 || cols % 32) return DQ_ERR_SHAPE;
    if (rows == 0 || cols == 0) return DQ_OK;
    if (!X || !codes || !inner_scales || !outer_scales) return DQ_ERR_ARG;
    if (!aligned(X, 16) || !aligned(codes, 16) || !aligned(inner_scales, 16) ||
        !aligned(outer_scales, 4) || !aligned(qdq, 16))
        return DQ_ERR_ALIGN;
    unsigned int *status = status_ptr();
    if (!status) return DQ_ERR_CUDA;
    TwoLevelLaunch L;
    L.X = X;
    L.rows = rows;
    L.cols = cols;
    L.nblk = (cols + dual_block - 1) / dual_block;
    L.dual_block = dual_block;
    L.f32 = dtype == DQ_DT_F32;
    L.codes = codes;
    L.iscales = static_cast<uint8_t *>(inner_scales);
    L.oscales = outer_scales;
    L.qdq = qdq;
    L.status = status;
    L.stream = reinterpret_cast<cudaStream_t>(stream);
    DQ_CUDA(launch_two_level(L));
    count_launches(1);
    return DQ_OK;
}

namespace {
std::atomic<int> g_stall_next_gemm{0};
}  // namespace

dq_status dq_test_stall_next_gemm(void) {
    g_stall_next_gemm.store(1);
    return DQ_OK;
}

dq_status dq_w4a4_gemm(const uint8_t *codes_x, const void *scales_x, const uint8_t *codes_w,
                       const void *scales_w, const float *a, const float *tensor_scale, int64_t M,
                       int64_t N, int64_t K, const dq_format *fmt, float *out, dq_stream stream) {
    if (!fmt) return DQ_ERR_ARG;
    const bool mx = fmt->codes == DQ_CODES_E2M1 && fmt->group == 32 &&
                    fmt->group_scale == DQ_SCALE_E8M0 && fmt->tensor_scale_auto == 0;
    const bool nv = fmt->codes == DQ_CODES_E2M1 && fmt->group == 16 &&
                    fmt->group_scale == DQ_SCALE_E4M3;
    if (!mx && !nv) return DQ_ERR_FORMAT;
    if (M < 0 || N < 0 || K < 0 || M % 128 || N % 128 || K % 256) return DQ_ERR_SHAPE;
    if (M == 0 || N == 0) return DQ_OK;
    if (K == 0) return DQ_ERR_SHAPE;
    if (!codes_x || !scales_x || !codes_w || !scales_w || !a || !out) return DQ_ERR_ARG;
    if (!aligned(codes_x, 16) || !aligned(scales_x, 16) || !aligned(codes_w, 16) ||
        !aligned(scales_w, 16) || !aligned(a, 16) || !aligned(out, 16) || !aligned(tensor_scale, 4))
        return DQ_ERR_ALIGN;
    unsigned int *status = status_ptr();
    if (!status) return DQ_ERR_CUDA;
    GemmLaunch L;
    L.codes_x = codes_x;
    L.scales_x = static_cast<const uint8_t *>(scales_x);
    L.codes_w = codes_w;
    L.scales_w = static_cast<const uint8_t *>(scales_w);
    L.a = a;
    L.ts = tensor_scale;
    L.out = out;
    L.M = M;
    L.N = N;
    L.K = K;
    L.nv = nv ? 1 : 0;
    L.status = status;
    L.stall = g_stall_next_gemm.exchange(0);
    L.stream = reinterpret_cast<cudaStream_t>(stream);
    DQ_CUDA(launch_w4a4_gemm(L));
    count_launches(1);
    return DQ_OK;
}

dq_status dq_scale_tiles(const void *scales, int64_t rows, int64_t K, int32_t group,
                         uint8_t *tiles, dq_stream stream) {
    if (group != 16 && group != 32) return DQ_ERR_ARG;
    if (rows < 0 || K < 0 || rows % 128 || K % (4 * group)) return DQ_ERR_SHAPE;
    if (rows == 0 || K == 0) return DQ_OK;
    if (!scales || !tiles) return DQ_ERR_ARG;
    if (!aligned(scales, 16) || !aligned(tiles, 16)) return DQ_ERR_ALIGN;
    DQ_CUDA(launch_scale_tiles(static_cast<const uint8_t *>(scales), rows, K, group, tiles,
                               reinterpret_cast<cudaStream_t>(stream)));
    count_launches(1);
    return DQ_OK;
}

dq_status dq_dequantize(const uint8_t *codes, const void *gscales, int64_t rows, int64_t cols,
                        const dq_format *fmt, float tensor_scale, const float *a, const float *b,
                        float *out, dq_stream stream) {
    FmtInfo fi;
    dq_status s = check_format(fmt, &fi);
    if (s != DQ_OK) return s;
    if (rows < 0 || cols < 0 || cols % fi.G) return DQ_ERR_SHAPE;
    if (rows == 0 || cols == 0) return DQ_OK;
    if (!codes || !gscales || !out) return DQ_ERR_ARG;
    const int64_t n = rows * cols;
    DQ_CUDA(launch_k(dequant_kernel, dim3(grid_for(n, 256)), dim3(256), 0,
                     reinterpret_cast<cudaStream_t>(stream), codes, gscales, rows, cols, fi.G,
                     fmt->codes, fmt->group_scale, tensor_scale, a, b, out));
    count_launches(1);
    return DQ_OK;
}

dq_status dq_solve_dual_scale(const void *W, int32_t dtype, int64_t rows, int64_t cols,
                              const dq_format *fmt, int32_t T, const float *a0, const float *b0,
                              uint8_t *codes, void *gscales, float *a, float *b,
                              float *tensor_scale, double *mse_trace, double *mse_half,
                              void *workspace, size_t ws_bytes, dq_stream stream) {
    dq_matrix m;
    m.W = W;
    m.rows = rows;
    m.cols = cols;
    m.a0 = a0;
    m.b0 = b0;
    m.codes = codes;
    m.gscales = gscales;
    m.a = a;
    m.b = b;
    m.tensor_scale = tensor_scale;
    m.mse_trace = mse_trace;
    m.mse_half = mse_half;
    return solve_impl(1, &m, dtype, fmt, T, workspace, ws_bytes,
                      reinterpret_cast<cudaStream_t>(stream));
}

dq_status dq_solve_dual_scale_batched(int32_t n, const dq_matrix *mats, int32_t dtype,
                                      const dq_format *fmt, int32_t T, void *workspace,
                                      size_t ws_bytes, dq_stream stream) {
    return solve_impl(n, mats, dtype, fmt, T, workspace, ws_bytes,
                      reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"

struct dq_graph_s {
    cudaGraph_t graph = nullptr;
    cudaGraphExec_t exec = nullptr;
    void *pinned = nullptr;      // host copy of the work table (n > 1)
    cudaEvent_t done = nullptr;  // recorded after every replay
    int64_t launches = 0;        // kernels per replay
    int device = -1;
};

namespace {
// An executable graph still in flight is freed when it completes; the
// pinned table it may still be reading is freed once the last replay has
// finished (the replays of one executable graph run in launch order, so
// the event recorded after the last one covers them all).
void graph_free(dq_graph g) {
    if (!g) return;
    if (g->done) cudaEventSynchronize(g->done);
    if (g->exec) cudaGraphExecDestroy(g->exec);
    if (g->graph) cudaGraphDestroy(g->graph);
    if (g->done) cudaEventDestroy(g->done);
    if (g->pinned) cudaFreeHost(g->pinned);
    delete g;
}
}  // namespace

extern "C" {

dq_status dq_graph_solve_batched(int32_t n, const dq_matrix *mats, int32_t dtype,
                                 const dq_format *fmt, int32_t T, void *workspace,
                                 size_t ws_bytes, dq_graph *out) {
    if (!out) return DQ_ERR_ARG;
    *out = nullptr;
    if (n == 0 || t_capturing) return DQ_ERR_ARG;      // empty batch; nested capture
    dq_status s = check_batch(n, mats, dtype, fmt, T, workspace, ws_bytes, nullptr);
    if (s != DQ_OK) return s;
    dq_graph g = new (std::nothrow) dq_graph_s;
    if (!g) return DQ_ERR_CUDA;
    if (cudaGetDevice(&g->device) != cudaSuccess) { graph_free(g); return DQ_ERR_CUDA; }
    if (cudaEventCreateWithFlags(&g->done, cudaEventDisableTiming) != cudaSuccess) {
        g->done = nullptr;
        graph_free(g);
        return DQ_ERR_CUDA;
    }
    if (n > 1 && cudaMallocHost(&g->pinned, (size_t)n * sizeof(MatDesc)) != cudaSuccess) {
        g->pinned = nullptr;
        graph_free(g);
        return DQ_ERR_CUDA;
    }
    cudaStream_t cs = nullptr;
    if (cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking) != cudaSuccess) { graph_free(g); return DQ_ERR_CUDA; }
    if (cudaStreamBeginCapture(cs, cudaStreamCaptureModeRelaxed) != cudaSuccess) {
        cudaStreamDestroy(cs);
        graph_free(g);
        return DQ_ERR_CUDA;
    }
    t_capturing = true;
    t_captured_launches = 0;
    t_pinned_table = g->pinned;
    s = solve_impl(n, mats, dtype, fmt, T, workspace, ws_bytes, cs);
    t_capturing = false;
    t_pinned_table = nullptr;
    g->launches = t_captured_launches;
    const cudaError_t e = cudaStreamEndCapture(cs, &g->graph);
    cudaStreamDestroy(cs);
    if (s == DQ_OK && e != cudaSuccess) s = DQ_ERR_CUDA;
    if (s == DQ_OK && cudaGraphInstantiate(&g->exec, g->graph, 0) != cudaSuccess) {
        g->exec = nullptr;
        s = DQ_ERR_CUDA;
    }
    if (s != DQ_OK) {
        graph_free(g);
        return s;
    }
    *out = g;
    return DQ_OK;
}

dq_status dq_graph_launch(dq_graph g, dq_stream stream) {
    if (!g || !g->exec) return DQ_ERR_ARG;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return DQ_ERR_CUDA;
    if (dev != g->device) return DQ_ERR_ARG;
    DQ_CUDA(cudaGraphLaunch(g->exec, reinterpret_cast<cudaStream_t>(stream)));
    DQ_CUDA(cudaEventRecord(g->done, reinterpret_cast<cudaStream_t>(stream)));
    g_launches.fetch_add(g->launches, std::memory_order_relaxed);
    return DQ_OK;
}

int64_t dq_graph_launches(dq_graph g) { return g ? g->launches : 0; }

dq_status dq_graph_destroy(dq_graph g) {
    graph_free(g);
    return DQ_OK;
}

namespace {

// Events of the host-streamed solve (created once, reused; calls serialised).
std::mutex g_host_mu;
std::vector<cudaEvent_t> g_host_events[kMaxDevices];

dq_status host_events(int dev, size_t k, cudaEvent_t **out) {
    std::vector<cudaEvent_t> &v = g_host_events[dev];
    while (v.size() < k) {
        cudaEvent_t e = nullptr;
        if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return DQ_ERR_CUDA;
        v.push_back(e);
    }
    *out = v.data();
    return DQ_OK;
}

dq_status copy_async(void *dst, const void *src, size_t bytes, cudaMemcpyKind kind,
                     cudaStream_t st) {
    if (bytes == 0 || dst == nullptr) return DQ_OK;
    if (src == nullptr) return DQ_ERR_ARG;
    DQ_CUDA(cudaMemcpyAsync(dst, src, bytes, kind, st));
    return DQ_OK;
}

}  // namespace

dq_status dq_solve_dual_scale_batched_host(int32_t n, const dq_matrix *host, const dq_matrix *dev,
                                           int32_t dtype, const dq_format *fmt, int32_t T,
                                           void *workspace, size_t ws_bytes, dq_stream compute,
                                           dq_stream h2d, dq_stream d2h) {
    if (n < 0 || T < 0 || (n > 0 && (!host || !dev))) return DQ_ERR_ARG;
    if (dtype != DQ_DT_F32 && dtype != DQ_DT_BF16) return DQ_ERR_ARG;
    FmtInfo fi;
    dq_status s = check_format(fmt, &fi);
    if (s != DQ_OK) return s;
    if (n == 0) return DQ_OK;
    const size_t esz = dtype == DQ_DT_F32 ? 4 : 2;
    const size_t gsz = fmt->group_scale == DQ_SCALE_BF16 ? 2 : 1;
    for (int i = 0; i < n; ++i) {
        const dq_matrix &h = host[i], &d = dev[i];
        if (h.rows != d.rows || h.cols != d.cols) return DQ_ERR_SHAPE;
        if (h.rows < 0 || h.cols < 0 || h.cols % fi.G) return DQ_ERR_SHAPE;
        if (h.rows > 0 && h.cols > 0 && (!h.W || !d.W)) return DQ_ERR_ARG;
        if ((h.a0 && !d.a0) || (h.b0 && !d.b0)) return DQ_ERR_ARG;
        if ((h.mse_trace && !d.mse_trace) || (h.mse_half && !d.mse_half)) return DQ_ERR_ARG;
    }
    // Consecutive matrices are solved together, as one batched solve, up to
    // about 1/8 of all the input bytes per group (at least 32 MiB) and as far
    // as the workspace allows: enough groups for the copies to overlap, large
    // enough groups that many small matrices still fill the GPU.
    const bool f32 = dtype == DQ_DT_F32;
    size_t total_in = 0;
    for (int i = 0; i < n; ++i) total_in += (size_t)host[i].rows * (size_t)host[i].cols * esz;
    // every group takes the whole batch's geometry (the device batched
    // solve's sums)
    const int tall = tall_batch(n, host, f32) ? 1 : 0;
    const size_t target = std::max(total_in / 8, (size_t)32 << 20);
    int devno = 0;
    if (cudaGetDevice(&devno) != cudaSuccess || devno < 0 || devno >= kMaxDevices) return DQ_ERR_CUDA;
    const cudaStream_t sc = reinterpret_cast<cudaStream_t>(compute);
    const cudaStream_t sh = reinterpret_cast<cudaStream_t>(h2d);
    const cudaStream_t sd = reinterpret_cast<cudaStream_t>(d2h);
    std::lock_guard<std::mutex> lk(g_host_mu);
    cudaEvent_t *ev = nullptr;
    if ((s = host_events(devno, 2 + 2 * (size_t)n, &ev)) != DQ_OK) return s;
    std::vector<dq_matrix> dm(dev, dev + n);
    for (int i = 0; i < n; ++i) {
        if (!host[i].a0) dm[i].a0 = nullptr;
        if (!host[i].b0) dm[i].b0 = nullptr;
    }
    // an earlier call may still be solving from the staging buffers (h2d
    // must not overwrite them yet) or copying out its results (compute must
    // not overwrite those yet)
    DQ_CUDA(cudaEventRecord(ev[0], sc));
    DQ_CUDA(cudaStreamWaitEvent(sh, ev[0], 0));
    DQ_CUDA(cudaEventRecord(ev[1], sd));
    DQ_CUDA(cudaStreamWaitEvent(sc, ev[1], 0));
    int g = 0;
    for (int i = 0; i < n; ++g) {
        // the group: matrices i .. j-1
        int j = i;
        size_t in_bytes = 0, mat_ws = 0;           // the group's inputs and per-matrix workspace
        while (j < n) {
            const size_t ws_j = mat_ws + matrix_ws(host[j].rows, host[j].cols, f32);
            const size_t need_j = 256 + table_ws(j - i + 1) + ws_j;   // as solve_impl needs
            if (j > i && (in_bytes >= target || need_j > ws_bytes)) break;
            if (need_j > ws_bytes) return DQ_ERR_WORKSPACE;        // not even matrix i alone
            mat_ws = ws_j;
            in_bytes += (size_t)host[j].rows * (size_t)host[j].cols * esz;
            ++j;
        }
        cudaEvent_t in = ev[2 + 2 * g], out = ev[3 + 2 * g];
        // in: W (and the initial scales) of the group's matrices
        for (int k = i; k < j; ++k) {
            const dq_matrix &h = host[k], &d = dev[k];
            const size_t rows = (size_t)h.rows, cols = (size_t)h.cols;
            if ((s = copy_async(const_cast<void *>(d.W), h.W, rows * cols * esz, cudaMemcpyHostToDevice, sh)) != DQ_OK) return s;
            if (h.a0 && (s = copy_async(const_cast<float *>(d.a0), h.a0, rows * 4, cudaMemcpyHostToDevice, sh)) != DQ_OK) return s;
            if (h.b0 && (s = copy_async(const_cast<float *>(d.b0), h.b0, cols * 4, cudaMemcpyHostToDevice, sh)) != DQ_OK) return s;
        }
        DQ_CUDA(cudaEventRecord(in, sh));
        // solve them on the compute stream once their inputs have landed
        DQ_CUDA(cudaStreamWaitEvent(sc, in, 0));
        if ((s = solve_impl(j - i, dm.data() + i, dtype, fmt, T, workspace, ws_bytes, sc, tall)) != DQ_OK) return s;
        DQ_CUDA(cudaEventRecord(out, sc));
        // out: the results the caller asked for in host memory
        DQ_CUDA(cudaStreamWaitEvent(sd, out, 0));
        for (int k = i; k < j; ++k) {
            const dq_matrix &h = host[k], &d = dev[k];
            const size_t rows = (size_t)h.rows, cols = (size_t)h.cols;
            const size_t code_bytes = rows * (cols * (size_t)fi.bits / 8);
            const size_t gs_bytes = rows * (cols / (size_t)fi.G) * gsz;
            if ((s = copy_async(h.codes, d.codes, code_bytes, cudaMemcpyDeviceToHost, sd)) != DQ_OK ||
                (s = copy_async(h.gscales, d.gscales, gs_bytes, cudaMemcpyDeviceToHost, sd)) != DQ_OK ||
                (s = copy_async(h.a, d.a, rows * 4, cudaMemcpyDeviceToHost, sd)) != DQ_OK ||
                (s = copy_async(h.b, d.b, cols * 4, cudaMemcpyDeviceToHost, sd)) != DQ_OK ||
                (s = copy_async(h.tensor_scale, d.tensor_scale, 4, cudaMemcpyDeviceToHost, sd)) != DQ_OK ||
                (s = copy_async(h.mse_trace, d.mse_trace, ((size_t)T + 1) * 8, cudaMemcpyDeviceToHost, sd)) != DQ_OK ||
                (s = copy_async(h.mse_half, d.mse_half, (size_t)T * 8, cudaMemcpyDeviceToHost, sd)) != DQ_OK)
                return s;
        }
        i = j;
    }
    return DQ_OK;
}

dq_status dq_row_update(const void *W, int32_t dtype, int64_t rows, int64_t cols,
                        const dq_format *fmt, float tensor_scale, const float *a_in,
                        const float *b_in, float *a_out, float *a_pre, double *mse_in,
                        void *workspace, size_t ws_bytes, dq_stream stream) {
    return step_impl(true, W, dtype, rows, cols, fmt, tensor_scale, a_in, b_in, a_out, a_pre,
                     mse_in, workspace, ws_bytes, reinterpret_cast<cudaStream_t>(stream));
}

dq_status dq_col_update(const void *W, int32_t dtype, int64_t rows, int64_t cols,
                        const dq_format *fmt, float tensor_scale, const float *a_in,
                        const float *b_in, float *b_out, float *b_pre, double *mse_in,
                        void *workspace, size_t ws_bytes, dq_stream stream) {
    return step_impl(false, W, dtype, rows, cols, fmt, tensor_scale, a_in, b_in, b_out, b_pre,
                     mse_in, workspace, ws_bytes, reinterpret_cast<cudaStream_t>(stream));
}

int64_t dq_col_row_block(int64_t rows, int64_t cols, int32_t dtype) {
    if (rows < 0 || cols < 0 || (dtype != DQ_DT_F32 && dtype != DQ_DT_BF16)) return -1;
    const bool f32 = dtype == DQ_DT_F32;
    return geometry(rows, cols, f32, tall_single(rows, cols, f32)).tr[1];
}

dq_status dq_col_partials(const void *W, int32_t dtype, int64_t rows, int64_t cols,
                          const dq_format *fmt, float tensor_scale, const float *a, const float *b,
                          int64_t row_block, float *partials, double *mse_in, void *workspace,
                          size_t ws_bytes, dq_stream stream) {
    return col_partials_impl(W, dtype, rows, cols, fmt, tensor_scale, a, b, row_block, partials,
                             mse_in, workspace, ws_bytes, reinterpret_cast<cudaStream_t>(stream));
}

dq_status dq_col_finalize(const float *partials, int64_t row_blocks, int64_t cols,
                          const dq_format *fmt, float *b_out, float *b_pre, dq_stream stream) {
    FmtInfo fi;
    dq_status s = check_format(fmt, &fi);
    if (s != DQ_OK) return s;
    if (row_blocks < 0 || cols < 0 || cols % fi.G) return DQ_ERR_SHAPE;   // (as the solves)
    if (cols == 0) return DQ_OK;
    if (!b_out || (row_blocks > 0 && !partials)) return DQ_ERR_ARG;
    if (!aligned(partials, 16) || !aligned(b_out, 4) || !aligned(b_pre, 4)) return DQ_ERR_ALIGN;
    unsigned int *status = status_ptr();
    if (!status) return DQ_ERR_CUDA;
    MatDesc d{};
    d.cols = cols;
    d.ncb = 1;
    d.ntiles[1] = row_blocks;
    d.colpart = reinterpret_cast<float2 *>(const_cast<float *>(partials));
    d.b_out = b_out;
    d.b_pre = b_pre;
    Launcher L;
    L.tab.dev = nullptr;
    L.tab.one = d;
    L.tab.n = 1;
    L.tab.status = status;
    L.combo = fi.combo;
    L.G = fi.G;
    L.total_cols = cols;
    L.st = reinterpret_cast<cudaStream_t>(stream);
    return L.col_finalize();
}

dq_status dq_last_device_status(dq_stream stream) {
    unsigned int *p = status_ptr();
    if (!p) return DQ_ERR_CUDA;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    DQ_CUDA(cudaStreamSynchronize(st));
    unsigned int v = 0;
    DQ_CUDA(cudaMemcpy(&v, p, sizeof(v), cudaMemcpyDeviceToHost));
    const unsigned int zero = 0;
    DQ_CUDA(cudaMemcpy(p, &zero, sizeof(zero), cudaMemcpyHostToDevice));
    if (v & STATUS_TIMEOUT) return DQ_ERR_TIMEOUT;  // a kernel's bounded wait ran out
    if (v & STATUS_NONFINITE) return DQ_ERR_NONFINITE;
    if (v & STATUS_RANGE) return DQ_ERR_RANGE;
    return DQ_OK;
}

dq_status dq_kernel_timing(int32_t kinds) {
    std::lock_guard<std::mutex> lk(g_timing_mu);
    g_timing_kinds = (unsigned int)kinds & 0x1Fu;
    return DQ_OK;
}

dq_status dq_kernel_time(int32_t kind, double *ms, int64_t *launches) {
    if (!ms || !launches || kind < 0 || kind > 4) return DQ_ERR_ARG;
    std::lock_guard<std::mutex> lk(g_timing_mu);
    double tot = 0.0;
    int64_t cnt = 0;
    std::vector<TimedLaunch> keep;
    for (const TimedLaunch &t : g_timed) {
        if (t.kind != kind) { keep.push_back(t); continue; }
        float m = 0.0f;
        DQ_CUDA(cudaEventSynchronize(t.end));
        DQ_CUDA(cudaEventElapsedTime(&m, t.beg, t.end));
        tot += m;
        ++cnt;
        g_event_pool.push_back(t.beg);
        g_event_pool.push_back(t.end);
    }
    g_timed.swap(keep);
    *ms = tot;
    *launches = cnt;
    return DQ_OK;
}

int64_t dq_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

}  // extern "C"

// ------------------------------------------------------------------------- //
// Solve without any allocation: scratch in a built-in device buffer
// ------------------------------------------------------------------------- //
//
// For callers that cannot allocate device memory.  The per-tile partial sums
// that dq_solve_dual_scale keeps in the caller's workspace live here in one
// static buffer per device (held for the life of the process).  In host code
// the array's name is only a host-side stand-in: its device address comes
// from cudaGetSymbolAddress, looked up once per device with that device
// current (the first call on a device does this, so it should come before
// any stream capture).  Calls that overlap on the GPU share the buffer and
// race.  The regions that must start at zero (the flag words of the
// one-pass MX iteration and the amax word of the tensor-scale pass) are
// cleared by the solve sequence itself.

namespace {

static __device__ __align__(256) unsigned char g_dq_noalloc_scratch[DQ_NOALLOC_SCRATCH_BYTES];

unsigned char *g_scratch_ptr[kMaxDevices];
cudaError_t g_scratch_err[kMaxDevices];
std::once_flag g_scratch_once[kMaxDevices];

// Device address of the scratch buffer on the current device, or NULL.
unsigned char *noalloc_scratch() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::call_once(g_scratch_once[dev], [dev]() {
        void *p = nullptr;
        g_scratch_err[dev] = cudaGetSymbolAddress(&p, g_dq_noalloc_scratch);
        g_scratch_ptr[dev] = (g_scratch_err[dev] == cudaSuccess)
                                 ? static_cast<unsigned char *>(p) : nullptr;
    });
    return g_scratch_ptr[dev];
}

}  // namespace

extern "C" dq_status dq_solve_dual_scale_noalloc(const void *W, int32_t dtype, int64_t rows,
                                                 int64_t cols, const dq_format *fmt, int32_t T,
                                                 const float *a0, const float *b0,
                                                 uint8_t *codes, void *gscales, float *a,
                                                 float *b, float *tensor_scale,
                                                 double *mse_trace, double *mse_half,
                                                 dq_stream stream) {
    if (T < 0) return DQ_ERR_ARG;
    if (dtype != DQ_DT_F32 && dtype != DQ_DT_BF16) return DQ_ERR_ARG;
    FmtInfo fi;
    dq_status s = check_format(fmt, &fi);
    if (s != DQ_OK) return s;
    if (rows < 0 || cols < 0 || cols % fi.G) return DQ_ERR_SHAPE;
    const bool f32 = dtype == DQ_DT_F32;
    const bool empty = rows == 0 || cols == 0;
    if (!empty && (!W || !codes || !gscales)) return DQ_ERR_ARG;
    if ((rows > 0 && !a) || (cols > 0 && !b) || !tensor_scale) return DQ_ERR_ARG;
    if (!aligned(W, 16) || !aligned(codes, 16) || !aligned(gscales, 16)) return DQ_ERR_ALIGN;
    if (!aligned(a, 4) || !aligned(b, 4) || !aligned(tensor_scale, 4)) return DQ_ERR_ALIGN;
    if (!aligned(a0, 4) || !aligned(b0, 4)) return DQ_ERR_ALIGN;
    if (!aligned(mse_trace, 8) || !aligned(mse_half, 8)) return DQ_ERR_ALIGN;
    const size_t need = 256 + matrix_ws(rows, cols, f32);        // flag words + partial sums
    if (need > (size_t)DQ_NOALLOC_SCRATCH_BYTES) return DQ_ERR_SCRATCH;
    unsigned char *scratch = noalloc_scratch();
    if (!scratch) return DQ_ERR_CUDA;
    unsigned int *status = status_ptr();
    if (!status) return DQ_ERR_CUDA;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);

    // descriptor of the one matrix, on the stack (no table copy)
    MatDesc d{};
    d.W = W;
    d.rows = rows;
    d.cols = cols;
    d.a = a;
    d.b = b;
    d.a_out = a;
    d.b_out = b;
    d.codes = codes;
    d.gscales = gscales;
    d.ts_ptr = tensor_scale;
    d.ts_out = tensor_scale;
    d.ts_val = 1.0f;
    d.a0 = a0;
    d.b0 = b0;
    d.mse_trace = mse_trace;
    d.mse_half = mse_half;
    Carve cv{reinterpret_cast<char *>(scratch),
             reinterpret_cast<char *>(scratch) + DQ_NOALLOC_SCRATCH_BYTES};
    unsigned int *flags = cv.take<unsigned int>(256);     // one-pass MX flags: 3 slots x 2 words
    int64_t tb[3] = {0, 0, 0}, rb = 0, cb = 0, sb = 0, hb = 0;
    place(d, f32, cv, tb, rb, cb, sb, hb, tall_single(d.rows, d.cols, f32));
    Launcher L;
    L.tab.dev = nullptr;
    L.tab.one = d;
    L.tab.n = 1;
    L.tab.status = status;
    L.combo = fi.combo;
    L.G = fi.G;
    L.f32 = f32;
    L.qmax = fi.qmax;
    for (int m = 0; m < 3; ++m) L.tiles[m] = tb[m];
    L.total_rows = rb;
    L.total_cols = cb;
    L.st = st;

    // the launch sequence of dq_solve_dual_scale for one matrix (the MX
    // formats take the one-pass iteration)
    if (fmt->tensor_scale_auto) {
        DQ_CUDA(cudaMemsetAsync(d.amax, 0, sizeof(unsigned int), st));   // starts at zero
        if (L.tiles[2] > 0) {
            if (f32) DQ_CUDA(launch_k(amax_kernel<float>, dim3((unsigned)L.tiles[2]),
                                      dim3(kThreads), 0, st, L.tab));
            else DQ_CUDA(launch_k(amax_kernel<Bf16Tag>, dim3((unsigned)L.tiles[2]), dim3(kThreads),
                                  0, st, L.tab));
            count_launches(1);
        }
    }
    DQ_CUDA(launch_k(tensor_scale_kernel, dim3(1), dim3(128), 0, st, L.tab, fi.qmax,
                     fmt->tensor_scale_auto));
    count_launches(1);
    const bool fused = fused_ok(fi.combo) && T > 0;
    if (fused) DQ_CUDA(cudaMemsetAsync(flags, 0, 6 * sizeof(unsigned int), st));   // start at zero
    if (rb + cb > 0) {
        DQ_CUDA(launch_k(init_state_kernel, dim3(grid_for(rb + cb, 256)), dim3(256), 0, st, L.tab,
                         rb, cb, fused ? flags : nullptr));
        count_launches(1);
    }
    L.row_mse = T > 0 && row_mse_ok(fi.combo) && (mse_trace != nullptr || mse_half != nullptr);
    for (int t = 0; t < T; ++t)
        if ((s = L.iteration(t, fused, flags, mse_trace != nullptr, mse_half != nullptr)) != DQ_OK)
            return s;
    if ((s = L.tiles_pass(MODE_PACK, mse_trace != nullptr)) != DQ_OK) return s;
    return L.mse(2, T, -1, nullptr, nullptr);
}
