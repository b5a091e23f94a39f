/*
 * A plain-C client of libtlg: no Python, no torch, only the C interface in
 * include/tlg.h and the CUDA runtime.  Used by tests/test_c_client.py.
 *
 *   c_abi_client <in.bin> <out.bin>
 *
 * in.bin : int64 M, N, K, then M*K fp16 bits of A (row-major), K*N of B, N of
 *          the bias, M*N of a residual R.
 * out.bin: M*N fp16 bits of tlg_gemm_bias_relu_f16(A, B, bias), then M*N fp16
 *          bits of tlg_gemm_fused(A, B, bias, GELU, residual R, in place: R is
 *          copied into C and passed as C's own residual).
 * Exit status 0 on success; otherwise a message on stderr naming the failed
 * call and its status string.
 */
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>

#include "tlg.h"

static int fail(const char *what, const char *why)
{
    fprintf(stderr, "c_abi_client: %s: %s\n", what, why);
    return 1;
}

#define CUDA_OK(call)                                                   \
    do {                                                                \
        cudaError_t e_ = (call);                                        \
        if (e_ != cudaSuccess) return fail(#call, cudaGetErrorString(e_)); \
    } while (0)

#define TLG_OK_OR_FAIL(call)                                            \
    do {                                                                \
        tlg_status s_ = (call);                                         \
        if (s_ != TLG_OK) return fail(#call, tlg_status_string(s_));    \
    } while (0)

int main(int argc, char **argv)
{
    if (argc != 3) return fail("usage", "c_abi_client <in.bin> <out.bin>");
    FILE *f = fopen(argv[1], "rb");
    if (!f) return fail("fopen", argv[1]);
    int64_t dims[3];
    if (fread(dims, sizeof(int64_t), 3, f) != 3) return fail("fread", "header");
    const int64_t M = dims[0], N = dims[1], K = dims[2];
    if (M <= 0 || N <= 0 || K <= 0 || M > 65536 || N > 65536 || K > 65536)
        return fail("header", "sizes out of range for this client");
    const size_t nA = (size_t)(M * K), nB = (size_t)(K * N), nC = (size_t)(M * N);
    uint16_t *h = (uint16_t *)malloc((nA + nB + (size_t)N + 3 * nC) * sizeof(uint16_t));
    if (!h) return fail("malloc", "host buffers");
    uint16_t *hA = h, *hB = hA + nA, *hbias = hB + nB, *hR = hbias + N, *hC1 = hR + nC,
             *hC2 = hC1 + nC;
    if (fread(hA, 2, nA + nB + (size_t)N + nC, f) != nA + nB + (size_t)N + nC)
        return fail("fread", "payload");
    fclose(f);

    void *dA, *dB, *dbias, *dC1, *dC2;
    CUDA_OK(cudaMalloc(&dA, nA * 2));
    CUDA_OK(cudaMalloc(&dB, nB * 2));
    CUDA_OK(cudaMalloc(&dbias, (size_t)N * 2));
    CUDA_OK(cudaMalloc(&dC1, nC * 2));
    CUDA_OK(cudaMalloc(&dC2, nC * 2));
    cudaStream_t s;
    CUDA_OK(cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking));
    CUDA_OK(cudaMemcpyAsync(dA, hA, nA * 2, cudaMemcpyHostToDevice, s));
    CUDA_OK(cudaMemcpyAsync(dB, hB, nB * 2, cudaMemcpyHostToDevice, s));
    CUDA_OK(cudaMemcpyAsync(dbias, hbias, (size_t)N * 2, cudaMemcpyHostToDevice, s));
    CUDA_OK(cudaMemcpyAsync(dC2, hR, nC * 2, cudaMemcpyHostToDevice, s));

    /* 1. the section 4.2 call: C1 = fp16(max(A.B + bias, 0)) */
    TLG_OK_OR_FAIL(tlg_gemm_bias_relu_f16(M, N, K, dA, K, dB, N, dbias, dC1, N, s));

    /* 2. the general fused epilogue, in place: C2 = fp16(gelu(A.B + bias) + C2) */
    tlg_fused_epilogue epi;
    epi.bias = dbias;
    epi.activation = TLG_ACT_GELU;
    epi.residual = dC2;
    epi.ldr = N;
    TLG_OK_OR_FAIL(tlg_gemm_fused(M, N, K, TLG_OP_N, dA, K, TLG_OP_N, dB, N, &epi, dC2, N,
                                  TLG_OUT_F16, NULL, NULL, 0, s));

    CUDA_OK(cudaMemcpyAsync(hC1, dC1, nC * 2, cudaMemcpyDeviceToHost, s));
    CUDA_OK(cudaMemcpyAsync(hC2, dC2, nC * 2, cudaMemcpyDeviceToHost, s));
    CUDA_OK(cudaStreamSynchronize(s));
    uint32_t code = 0;
    TLG_OK_OR_FAIL(tlg_device_error(1, &code));

    f = fopen(argv[2], "wb");
    if (!f) return fail("fopen", argv[2]);
    if (fwrite(hC1, 2, 2 * nC, f) != 2 * nC) return fail("fwrite", argv[2]);
    fclose(f);
    cudaFree(dA);
    cudaFree(dB);
    cudaFree(dbias);
    cudaFree(dC1);
    cudaFree(dC2);
    cudaStreamDestroy(s);
    free(h);
    return 0;
}
