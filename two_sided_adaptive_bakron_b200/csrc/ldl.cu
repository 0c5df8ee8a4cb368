// ldl.cu -- bakron_ldl: H = (I + L) D (I + L)^T, L strictly upper triangular.
//
// YAQA article (news.43b.com.cn/a/479517.html), section 4: L_O, L_I of the rounding rule come
// from the LDL decomposition H = (L + I) D (L + I)^T of each damped Kronecker factor; the rule
// of the same section makes L strictly upper (a U D U^T factorisation, i.e. LDL^T of H with its
// index order reversed).
//
// Blocked right-looking algorithm, last block of indices first. With the index set split into
// A (still pending, lower indices), B (the current block) and C (done), and H' the Schur
// complement left by C:
//   H'_BB = U_BB D_B U_BB^T               (unblocked, one warp, fp64)
//   U_AB  = H'_AB U_BB^{-T} D_B^{-1}        (one thread per row of A, back substitution)
//   H'_AA -= (U_AB D_B) U_AB^T             (upper triangle only)
// The factor is built in place in the output buffer L, which first receives a copy of the
// upper triangle of H; the entries on and below the diagonal are cleared at the end.
#include <algorithm>

#include "common.cuh"

namespace bakron {
namespace {

constexpr int NB = 32;  // block of indices per step

__global__ void copy_upper_kernel(const float* __restrict__ H, float* __restrict__ L, int n) {
    const size_t total = (size_t)n * n;
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < total;
         e += (size_t)gridDim.x * blockDim.x) {
        const int i = (int)(e / n), j = (int)(e % n);
        L[e] = (j >= i) ? H[e] : 0.f;
    }
}

__global__ void clear_lower_kernel(float* __restrict__ L, int n) {
    const size_t total = (size_t)n * n;
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < total;
         e += (size_t)gridDim.x * blockDim.x) {
        const int i = (int)(e / n), j = (int)(e % n);
        if (j <= i) L[e] = 0.f;
    }
}

// Unblocked U D U^T of the b x b diagonal block [k0, k0+b), one warp, fp64; lane i owns row i.
__global__ void diag_block_kernel(float* __restrict__ L, float* __restrict__ D, int n, int k0,
                                  int b, int* status) {
    __shared__ double h[NB][NB + 1];
    const int lane = threadIdx.x;
    for (int c = 0; c < NB; ++c)
        h[lane][c] = (lane < b && c < b && c >= lane) ? (double)L[(size_t)(k0 + lane) * n + k0 + c]
                                                      : 0.0;
    __syncwarp();
    for (int j = b - 1; j >= 0; --j) {
        double d = h[j][j];
        if (!(d > 0.0) || !isfinite(d)) {
            if (lane == 0) set_status(status, BAKRON_ERR_NOT_PD);
            d = 1.0;
        }
        double u = 0.0;
        if (lane < j) u = h[lane][j] / d;
        __syncwarp();
        if (lane < j) h[lane][j] = u;   // column j of U (strictly upper part)
        if (lane == 0) D[k0 + j] = (float)d;
        __syncwarp();
        // rank-1 downdate of the leading (j x j) block, upper triangle
        if (lane < j) {
            for (int l = lane; l < j; ++l) h[lane][l] -= u * d * h[l][j];
        }
        __syncwarp();
    }
    for (int c = 0; c < NB; ++c)
        if (lane < b && c < b && c > lane) L[(size_t)(k0 + lane) * n + k0 + c] = (float)h[lane][c];
}

// Rows i < k0: y U_BB^T = H'_{iB} (back substitution), U_{iB} = y / D_B; y kept for the update.
__global__ void panel_kernel(float* __restrict__ L, const float* __restrict__ D,
                             float* __restrict__ Y, int n, int k0, int b) {
    __shared__ float u[NB][NB + 1];
    __shared__ float dinv[NB];
    for (int e = threadIdx.x; e < NB * NB; e += blockDim.x) {
        const int r = e / NB, c = e % NB;
        u[r][c] = (r < b && c < b && c > r) ? L[(size_t)(k0 + r) * n + k0 + c] : 0.f;
    }
    if (threadIdx.x < NB) dinv[threadIdx.x] = (threadIdx.x < b) ? 1.f / D[k0 + threadIdx.x] : 0.f;
    __syncthreads();
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= k0) return;
    float y[NB];
#pragma unroll
    for (int c = 0; c < NB; ++c) y[c] = (c < b) ? L[(size_t)i * n + k0 + c] : 0.f;
#pragma unroll
    for (int jj = NB - 1; jj >= 0; --jj) {
        float acc = y[jj];
#pragma unroll
        for (int l = jj + 1; l < NB; ++l) acc = fmaf(-u[jj][l], y[l], acc);
        y[jj] = acc;
    }
#pragma unroll
    for (int c = 0; c < NB; ++c) {
        if (c < b) {
            Y[(size_t)i * NB + c] = y[c];
            L[(size_t)i * n + k0 + c] = y[c] * dinv[c];
        }
    }
}

// H'_AA -= Y U_AB^T on the upper triangle of [0, k0)^2; 64 x 64 output tiles, K = NB.
__global__ void __launch_bounds__(256) syrk_update_kernel(float* __restrict__ L,
                                                         const float* __restrict__ Y, int n,
                                                         int k0, int T) {
    // blockIdx.x -> (ti, tj), ti <= tj < T
    int rem = blockIdx.x, ti = 0;
    while (rem >= T - ti) { rem -= T - ti; ++ti; }
    const int tj = ti + rem;
    __shared__ float sY[NB][64 + 4];
    __shared__ float sP[NB][64 + 4];
    const int i0 = ti * 64, j0 = tj * 64;
    for (int e = threadIdx.x; e < 64 * NB; e += 256) {
        const int r = e / NB, c = e % NB;
        sY[c][r] = (i0 + r < k0) ? Y[(size_t)(i0 + r) * NB + c] : 0.f;
        sP[c][r] = (j0 + r < k0) ? L[(size_t)(j0 + r) * n + k0 + c] : 0.f;
    }
    __syncthreads();
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    float acc[4][4] = {};
#pragma unroll 8
    for (int k = 0; k < NB; ++k) {
        float a[4], bb[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) { a[q] = sY[k][ty * 4 + q]; bb[q] = sP[k][tx * 4 + q]; }
#pragma unroll
        for (int p = 0; p < 4; ++p)
#pragma unroll
            for (int q = 0; q < 4; ++q) acc[p][q] = fmaf(a[p], bb[q], acc[p][q]);
    }
#pragma unroll
    for (int p = 0; p < 4; ++p)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int i = i0 + ty * 4 + p, j = j0 + tx * 4 + q;
            if (i < k0 && j < k0 && j >= i) L[(size_t)i * n + j] -= acc[p][q];
        }
}

}  // namespace
}  // namespace bakron

using namespace bakron;

extern "C" size_t bakron_ldl_workspace_bytes(int n) {
    if (n < 1) return 0;
    WsSizer z;
    z.take<float>((size_t)n * NB);  // Y = U_AB D_B panel
    return z.bytes();
}

extern "C" int bakron_ldl(const float* H, int n, float* L, float* D, void* ws, size_t ws_bytes,
                          int* dev_status, void* stream) {
    if (n < 1 || n > 65536 || !H || !L || !D || !dev_status) return BAKRON_ERR_INVALID_ARG;
    if (!ws_ok(ws, ws_bytes, bakron_ldl_workspace_bytes(n))) return BAKRON_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    WsCarver c(ws);
    float* Y = c.take<float>((size_t)n * NB);
    const int eb = 1184;  // elementwise grid
    copy_upper_kernel<<<eb, 256, 0, st>>>(H, L, n);
    for (int k1 = n; k1 > 0; k1 -= NB) {
        const int k0 = std::max(0, k1 - NB), b = k1 - k0;
        diag_block_kernel<<<1, 32, 0, st>>>(L, D, n, k0, b, dev_status);
        if (k0 > 0) {
            panel_kernel<<<(k0 + 127) / 128, 128, 0, st>>>(L, D, Y, n, k0, b);
            const int T = (k0 + 63) / 64;
            syrk_update_kernel<<<T * (T + 1) / 2, 256, 0, st>>>(L, Y, n, k0, T);
        }
    }
    clear_lower_kernel<<<eb, 256, 0, st>>>(L, n);
    const long long nblk = (n + NB - 1) / NB;
    count_launches(2 + 3 * nblk - 2);
    return cuda_err(cudaGetLastError());
}
