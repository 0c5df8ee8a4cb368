/*
 * bakron_internal.h -- test hooks of libbakron.so. Not part of the solver's interface: they
 * expose building blocks so that the test suite can check them in isolation. Same
 * conventions as bakron.h (device pointers, row-major, caller-owned workspace, asynchronous on
 * `stream`, device errors in *dev_status).
 */
#ifndef BAKRON_INTERNAL_H_
#define BAKRON_INTERNAL_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* C = A B^T with the 3xTF32 tensor-core engine. A is M x K (row stride lda), B is N x K
 * (row stride ldb), C is M x N (row stride ldc); fp32. */
size_t bakron_internal_gemm3x_workspace_bytes(int M, int N, int K);
int bakron_internal_gemm3x(const float* A, int M, int K, int lda, const float* B, int N, int ldb,
                           float* C, int ldc, void* ws, size_t ws_bytes, int* dev_status,
                           void* stream);

/* The first, CUDA-core version of bakron_proxy_loss (same contract), kept as a cross-check of
 * the tensor-core version. */
size_t bakron_internal_proxy_loss_simt_workspace_bytes(int m, int n);
int bakron_internal_proxy_loss_simt(const float* dW, int m, int n, const float* H_O,
                                    const float* H_I, double* loss, void* ws, size_t ws_bytes,
                                    void* stream);

/* Writes the order-28 Hadamard matrix the transform of bakron_rht uses (row-major, 784 HOST
 * bytes of +1 / -1). Host only; no device work. */
void bakron_internal_hadamard28(signed char* out);

#ifdef __cplusplus
}
#endif

#endif /* BAKRON_INTERNAL_H_ */
