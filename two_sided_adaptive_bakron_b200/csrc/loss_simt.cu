// loss.cu -- bakron_proxy_loss: tr(H_O dW H_I dW^T) = vec(dW)^T (H_O (x) H_I) vec(dW).
//
// YAQA article (news.43b.com.cn/a/479517.html), section 4: the layer proxy error
// dW (H_O (x) H_I) dW^T bounded there by tr(D_I) tr(D_O) sigma^2; section 2: the second-order
// objective (its factor 1/2 is not applied here).
//
// Evaluated as  sum_ij (H_O dW)_ij (dW H_I)_ij :
//   Y = dW H_I                 (GEMM, stored to the workspace)
//   Z = H_O dW, tile by tile    (GEMM whose epilogue forms the fp64 partial sum of Z o Y)
//   loss = sum of the per-tile partials, in a fixed order (bitwise reproducible).
#include "common.cuh"

namespace bakron {
namespace {

constexpr int BM = 64, BN = 64, BK = 16, NTH = 256;

// acc(64x64 tile at m0,n0) = A[M x K] B[K x N], both row-major; 256 threads, 4x4 per thread.
__device__ __forceinline__ void gemm_tile(float (&acc)[4][4], const float* __restrict__ A,
                                          int lda, const float* __restrict__ B, int ldb, int M,
                                          int N, int K, int m0, int n0,
                                          float (*sA)[BM + 4], float (*sB)[BN + 4]) {
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    for (int k0 = 0; k0 < K; k0 += BK) {
#pragma unroll
        for (int q = 0; q < (BM * BK) / NTH; ++q) {
            const int e = threadIdx.x + q * NTH, r = e / BK, c = e % BK;
            sA[c][r] = (m0 + r < M && k0 + c < K) ? __ldg(&A[(size_t)(m0 + r) * lda + k0 + c])
                                                  : 0.f;
        }
#pragma unroll
        for (int q = 0; q < (BK * BN) / NTH; ++q) {
            const int e = threadIdx.x + q * NTH, r = e / BN, c = e % BN;
            sB[r][c] = (k0 + r < K && n0 + c < N) ? __ldg(&B[(size_t)(k0 + r) * ldb + n0 + c])
                                                  : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < BK; ++kk) {
            float a[4], b[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) { a[q] = sA[kk][ty * 4 + q]; b[q] = sB[kk][tx * 4 + q]; }
#pragma unroll
            for (int p = 0; p < 4; ++p)
#pragma unroll
                for (int q = 0; q < 4; ++q) acc[p][q] = fmaf(a[p], b[q], acc[p][q]);
        }
        __syncthreads();
    }
}

__global__ void __launch_bounds__(NTH) y_kernel(const float* __restrict__ dW,
                                                const float* __restrict__ HI,
                                                float* __restrict__ Y, int m, int n) {
    __shared__ float sA[BK][BM + 4];
    __shared__ float sB[BK][BN + 4];
    const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
    float acc[4][4] = {};
    gemm_tile(acc, dW, n, HI, n, m, n, n, m0, n0, sA, sB);
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
#pragma unroll
    for (int p = 0; p < 4; ++p)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int i = m0 + ty * 4 + p, j = n0 + tx * 4 + q;
            if (i < m && j < n) Y[(size_t)i * n + j] = acc[p][q];
        }
}

__global__ void __launch_bounds__(NTH) zdot_kernel(const float* __restrict__ HO,
                                                   const float* __restrict__ dW,
                                                   const float* __restrict__ Y,
                                                   double* __restrict__ partial, int m, int n) {
    __shared__ float sA[BK][BM + 4];
    __shared__ float sB[BK][BN + 4];
    __shared__ double red[NTH / 32];
    const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
    float acc[4][4] = {};
    gemm_tile(acc, HO, m, dW, n, m, n, m, m0, n0, sA, sB);
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    double s = 0.0;
#pragma unroll
    for (int p = 0; p < 4; ++p)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int i = m0 + ty * 4 + p, j = n0 + tx * 4 + q;
            if (i < m && j < n) s += (double)acc[p][q] * (double)Y[(size_t)i * n + j];
        }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_down_sync(0xffffffffu, s, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
    __syncthreads();
    if (threadIdx.x == 0) {
        double t = 0.0;
        for (int w = 0; w < NTH / 32; ++w) t += red[w];
        partial[(size_t)blockIdx.y * gridDim.x + blockIdx.x] = t;
    }
}

__global__ void final_sum_kernel(const double* __restrict__ partial, size_t count,
                                 double* __restrict__ loss) {
    __shared__ double red[1024];
    double s = 0.0;
    for (size_t e = threadIdx.x; e < count; e += blockDim.x) s += partial[e];
    red[threadIdx.x] = s;
    __syncthreads();
    for (int w = blockDim.x / 2; w > 0; w >>= 1) {
        if ((int)threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x == 0) *loss = red[0];
}

}  // namespace
}  // namespace bakron

using namespace bakron;

extern "C" size_t bakron_internal_proxy_loss_simt_workspace_bytes(int m, int n) {
    if (m < 1 || n < 1) return 0;
    WsSizer z;
    z.take<float>((size_t)m * n);
    z.take<double>((size_t)((m + BM - 1) / BM) * ((n + BN - 1) / BN));
    return z.bytes();
}

extern "C" int bakron_internal_proxy_loss_simt(const float* dW, int m, int n, const float* H_O,
                                 const float* H_I, double* loss, void* ws, size_t ws_bytes,
                                 void* stream) {
    if (m < 1 || n < 1 || !dW || !H_O || !H_I || !loss) return BAKRON_ERR_INVALID_ARG;
    if (!ws_ok(ws, ws_bytes, bakron_internal_proxy_loss_simt_workspace_bytes(m, n))) return BAKRON_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    WsCarver c(ws);
    float* Y = c.take<float>((size_t)m * n);
    const dim3 grid((n + BN - 1) / BN, (m + BM - 1) / BM);
    double* partial = c.take<double>((size_t)grid.x * grid.y);
    y_kernel<<<grid, NTH, 0, st>>>(dW, H_I, Y, m, n);
    zdot_kernel<<<grid, NTH, 0, st>>>(H_O, dW, Y, partial, m, n);
    final_sum_kernel<<<1, 1024, 0, st>>>(partial, (size_t)grid.x * grid.y, loss);
    count_launches(3);
    return cuda_err(cudaGetLastError());
}
