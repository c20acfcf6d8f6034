/* A plain C caller of libuw (include/uw.h) on the GPU, with no Python in the
 * loop: encode a synthetic BF16 matrix on the host, copy the blob to device
 * memory the caller allocates, bind it, decode it back to BF16 (must equal
 * the input bit for bit), and run the fused matmul with a stream-K plan
 * against the same kernel on the plain BF16 weights (must be bit-identical).
 * Exit status 0 on success; a message on stderr otherwise. */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime_api.h>

#include "uw.h"

#define N 256
#define K 1024
#define M 3

static uint32_t rng_state = 12345u;
static uint32_t next_u32(void) {          /* xorshift32 */
    rng_state ^= rng_state << 13;
    rng_state ^= rng_state >> 17;
    rng_state ^= rng_state << 5;
    return rng_state;
}

/* a BF16 pattern with a small exponent spread (plus a rare large one) */
static uint16_t weight_bits(void) {
    const uint32_t r = next_u32();
    const uint32_t sign = r & 1u, mant = (r >> 1) & 0x7Fu;
    uint32_t exp = 118u + ((r >> 8) % 5u);             /* a handful of common exponents */
    if (((r >> 16) & 1023u) == 0u) exp = 127u;         /* about one weight in 1024: an outlier */
    return (uint16_t)(sign << 15 | exp << 7 | mant);
}

#define CHECK_CUDA(x) do { cudaError_t e_ = (x); if (e_ != cudaSuccess) { \
    fprintf(stderr, "%s: %s\n", #x, cudaGetErrorString(e_)); return 2; } } while (0)
#define CHECK_UW(x) do { uw_status s_ = (x); if (s_ != UW_OK) { \
    fprintf(stderr, "%s: %s\n", #x, uw_status_str(s_)); return 3; } } while (0)

int main(void) {
    static uint16_t w[N * K], wd[N * K], x[M * K];
    static float y_fused[M * N], y_plain[M * N];
    for (int i = 0; i < N * K; i++) w[i] = weight_bits();
    for (int i = 0; i < M * K; i++) x[i] = (uint16_t)(((next_u32() & 1u) << 15) | (126u << 7) | (next_u32() & 0x7Fu));

    uw_blob *blob = NULL;
    CHECK_UW(uw_encode(w, N, K, UW_EMIT_HUFFMAN | UW_EMIT_PALETTE, &blob));
    size_t bytes = 0;
    const void *host = uw_blob_data(blob, &bytes);

    void *d_blob = NULL, *d_w = NULL, *d_x = NULL, *d_y = NULL, *d_ws = NULL;
    uint32_t *d_status = NULL;
    CHECK_CUDA(cudaMalloc(&d_blob, bytes));
    CHECK_CUDA(cudaMalloc((void **)&d_status, 4));
    CHECK_CUDA(cudaMalloc(&d_w, sizeof w));
    CHECK_CUDA(cudaMalloc(&d_x, sizeof x));
    CHECK_CUDA(cudaMalloc(&d_y, sizeof y_fused));
    CHECK_CUDA(cudaMemcpy(d_blob, host, bytes, cudaMemcpyHostToDevice));
    CHECK_CUDA(cudaMemcpy(d_w, w, sizeof w, cudaMemcpyHostToDevice));
    CHECK_CUDA(cudaMemcpy(d_x, x, sizeof x, cudaMemcpyHostToDevice));
    CHECK_CUDA(cudaMemset(d_status, 0, 4));

    uw_dmat mat;
    CHECK_UW(uw_matrix_bind(host, bytes, d_blob, d_status, 1, &mat));

    /* decode back to BF16: the caller's buffer, the legacy default stream */
    uint16_t *d_dec = NULL;
    CHECK_CUDA(cudaMalloc((void **)&d_dec, sizeof wd));
    CHECK_UW(uw_decode_to_bf16(&mat, d_dec, NULL));
    CHECK_UW(uw_device_status(&mat, NULL));
    CHECK_CUDA(cudaMemcpy(wd, d_dec, sizeof wd, cudaMemcpyDeviceToHost));
    if (memcmp(w, wd, sizeof w) != 0) {
        fprintf(stderr, "decode is not bit-exact\n");
        return 4;
    }

    /* fused matmul (stream-K plan) against the same kernel on BF16 weights */
    uw_plan plan;
    memset(&plan, 0, sizeof plan);
    plan.pipeline = UW_PIPE_DIRECT_PALETTE;
    plan.kernel = UW_KERNEL_TC_SK;
    plan.bn = 16;
    plan.split_k = 1;
    size_t ws_bytes = 0;
    CHECK_UW(uw_workspace_size(M, N, K, &plan, &ws_bytes));
    CHECK_CUDA(cudaMalloc(&d_ws, ws_bytes));
    CHECK_CUDA(cudaMemset(d_ws, 0, ws_bytes));      /* stream-K tile counters start at zero */
    CHECK_UW(uw_fused_matmul((const uint16_t *)d_x, M, &mat, NULL, (float *)d_y, &plan, d_ws, ws_bytes, NULL));
    CHECK_UW(uw_device_status(&mat, NULL));
    CHECK_CUDA(cudaMemcpy(y_fused, d_y, sizeof y_fused, cudaMemcpyDeviceToHost));
    CHECK_UW(uw_matmul_bf16((const uint16_t *)d_x, M, (const uint16_t *)d_w, N, K, (float *)d_y, &plan, d_ws,
                            ws_bytes, d_status, NULL));
    CHECK_UW(uw_device_status(&mat, NULL));
    CHECK_CUDA(cudaMemcpy(y_plain, d_y, sizeof y_plain, cudaMemcpyDeviceToHost));
    if (memcmp(y_fused, y_plain, sizeof y_fused) != 0) {
        fprintf(stderr, "fused matmul differs from the plain kernel\n");
        return 5;
    }
    double s = 0.0;
    for (int i = 0; i < M * N; i++) s += y_fused[i];
    printf("c caller ok: decode bit-exact, fused == plain over %d outputs (sum %.6g)\n", M * N, s);

    cudaFree(d_ws);
    cudaFree(d_dec);
    cudaFree(d_y);
    cudaFree(d_x);
    cudaFree(d_w);
    cudaFree(d_status);
    cudaFree(d_blob);
    uw_blob_free(blob);
    return 0;
}
