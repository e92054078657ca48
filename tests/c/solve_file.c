/* Test program (C99): one DualQuant solve driven from C through the library's
 * C ABI, with device memory from the CUDA runtime.
 *   solve_file <W.bin: bf16 bits, rows x cols> <rows> <cols> <T> <preset> <G> <out.bin>
 * writes to out.bin: status (int32), tensor_scale (float32), a (rows float32),
 * b (cols float32), mse_trace (T+1 float64), codes (dq_code_bytes bytes) and
 * group scales (rows x cols/G elements of the preset's scale type). */
#include <stdio.h>
#include <stdlib.h>

#include <cuda_runtime.h>

#include "dq.h"

#define CK(x)                                                           \
    do {                                                                \
        if ((x) != cudaSuccess) {                                       \
            fprintf(stderr, "CUDA error at %s:%d\n", __FILE__, __LINE__); \
            return 2;                                                   \
        }                                                               \
    } while (0)

int main(int argc, char **argv) {
    if (argc != 8) {
        fprintf(stderr, "usage: solve_file W.bin rows cols T preset G out.bin\n");
        return 2;
    }
    const int64_t rows = atoll(argv[2]), cols = atoll(argv[3]);
    const int32_t T = atoi(argv[4]), G = atoi(argv[6]);
    dq_format f;
    if (dq_format_preset(argv[5], G, &f) != DQ_OK) return 3;
    const size_t w_bytes = (size_t)(rows * cols) * 2;
    const int64_t code_bytes = dq_code_bytes(&f, rows, cols);
    const size_t gs_elem = f.group_scale == DQ_SCALE_BF16 ? 2 : 1;
    const size_t gs_bytes = (size_t)(rows * (cols / G)) * gs_elem;
    size_t ws_bytes = 0;
    if (code_bytes < 0 || dq_workspace_size(1, &rows, &cols, &f, &ws_bytes) != DQ_OK) return 3;

    unsigned char *hw = (unsigned char *)malloc(w_bytes);
    FILE *in = fopen(argv[1], "rb");
    if (!hw || !in || fread(hw, 1, w_bytes, in) != w_bytes) return 4;
    fclose(in);

    void *dW, *dcodes, *dgs, *dws;
    float *da, *db, *dts;
    double *dmse;
    CK(cudaMalloc(&dW, w_bytes));
    CK(cudaMalloc(&dcodes, (size_t)code_bytes));
    CK(cudaMalloc(&dgs, gs_bytes));
    CK(cudaMalloc((void **)&da, (size_t)rows * 4));
    CK(cudaMalloc((void **)&db, (size_t)cols * 4));
    CK(cudaMalloc((void **)&dts, 4));
    CK(cudaMalloc((void **)&dmse, (size_t)(T + 1) * 8));
    CK(cudaMalloc(&dws, ws_bytes));
    CK(cudaMemcpy(dW, hw, w_bytes, cudaMemcpyHostToDevice));

    int32_t st = dq_solve_dual_scale(dW, DQ_DT_BF16, rows, cols, &f, T, NULL, NULL, dcodes, dgs,
                                     da, db, dts, dmse, NULL, dws, ws_bytes, NULL);
    if (st == DQ_OK) st = dq_last_device_status(NULL);

    float *ha = (float *)malloc((size_t)rows * 4), *hb = (float *)malloc((size_t)cols * 4), ts = 0.0f;
    double *hm = (double *)malloc((size_t)(T + 1) * 8);
    unsigned char *hc = (unsigned char *)malloc((size_t)code_bytes), *hg = (unsigned char *)malloc(gs_bytes);
    if (!ha || !hb || !hm || !hc || !hg) return 4;
    CK(cudaMemcpy(ha, da, (size_t)rows * 4, cudaMemcpyDeviceToHost));
    CK(cudaMemcpy(hb, db, (size_t)cols * 4, cudaMemcpyDeviceToHost));
    CK(cudaMemcpy(&ts, dts, 4, cudaMemcpyDeviceToHost));
    CK(cudaMemcpy(hm, dmse, (size_t)(T + 1) * 8, cudaMemcpyDeviceToHost));
    CK(cudaMemcpy(hc, dcodes, (size_t)code_bytes, cudaMemcpyDeviceToHost));
    CK(cudaMemcpy(hg, dgs, gs_bytes, cudaMemcpyDeviceToHost));

    FILE *out = fopen(argv[7], "wb");
    if (!out) return 4;
    fwrite(&st, 4, 1, out);
    fwrite(&ts, 4, 1, out);
    fwrite(ha, 4, (size_t)rows, out);
    fwrite(hb, 4, (size_t)cols, out);
    fwrite(hm, 8, (size_t)(T + 1), out);
    fwrite(hc, 1, (size_t)code_bytes, out);
    fwrite(hg, 1, gs_bytes, out);
    fclose(out);
    printf("status %d mse %g -> %g\n", st, hm[0], hm[T]);
    return st == DQ_OK ? 0 : 1;
}
