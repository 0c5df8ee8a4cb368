// hessian.cu -- the damped Kronecker factors: bakron_damped_gram and bakron_sketch_b.
//
// YAQA article (news.43b.com.cn/a/479517.html), section 3: the factors of the Kronecker
// approximation H ~ H_O (x) H_I are second moments. H_1 = E[x^T x] over the input rows x is the
// one-sided factor (and Sketch A's starting point); Sketch B, one power-iteration round from
// H_O = H_I = I, gives (H_I)_1 = E_s[G_s^T G_s] / m and (H_O)_1 = E_s[G_s G_s^T] / n over the
// per-sequence weight gradients G_s (m x n). Every factor gets the relative damping of the
// solver's inputs: H + damp * mean(diag(H)) * I.
//
// Each factor is H = P P^T / K for a K-major operand P (d rows = features, K columns =
// samples), built as hi/lo tf32 planes:
//   E[x^T x]:           P = X^T                        (d = n, K = N)
//   Sketch B, H_I:      P = [G_1; ...; G_S]^T          (d = n, K = S m)
//   Sketch B, H_O:      P = [G_1, G_2, ..., G_S]       (d = m, K = S n)
// The product runs on the 3xTF32 tcgen05 GEMM engine over the upper block triangle only
// (d (d + 1) K / 2 multiply-adds) in chunks of kChunkK samples: the tensor core's fp32
// accumulator is restarted every chunk and the chunk sums are added in round-to-nearest fp32,
// so the accumulation error stays at one chunk's level instead of growing with K. Then the diagonal is summed in fp64 in a fixed order and one
// kernel transposes the upper triangle into the lower one through shared memory while adding
// damp * mean(diag) to the diagonal, so H is exactly symmetric.
#include <algorithm>

#include "tcgemm_host.cuh"

namespace bakron {
namespace {

constexpr int BN = 128;   // square tiles (BM == BN) for the upper block triangle
constexpr int STAGES = 3;
constexpr int kChunkKb = 8;                 // k-blocks per accumulator chunk
constexpr int kChunkK = kChunkKb * tc::BK;  // = 256 samples
constexpr int kMaxSplitRows = 65535 * 32;   // the transposed plane split's grid limit

// out[0] = sum_i H[i][i], one block, fixed order.
__global__ void diag_sum_kernel(const float* __restrict__ H, int d, double* __restrict__ out) {
    __shared__ double red[1024];
    double s = 0.0;
    for (int i = threadIdx.x; i < d; i += blockDim.x) s += (double)H[(size_t)i * d + i];
    red[threadIdx.x] = s;
    __syncthreads();
    for (int w = blockDim.x / 2; w > 0; w >>= 1) {
        if ((int)threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x == 0) out[0] = red[0];
}

// Block (x, y) owns the 32 x 32 target tile at tile row y, tile column x, on or below the
// diagonal (x <= y): it reads the upper source tile (x, y), and writes H[r][c] = H[c][r] for
// r > c and H[i][i] + damp * mean(diag) on the diagonal. Only diagonal blocks read what they
// write, and they read it all before the barrier.
__global__ void mirror_damp_kernel(float* __restrict__ H, int d,
                                   const double* __restrict__ diag_sum, float damp) {
    const int ty = blockIdx.y, tx = blockIdx.x;
    if (tx > ty) return;
    __shared__ float t[32][33];
    const int x = threadIdx.x;
    for (int y = threadIdx.y; y < 32; y += 8) {
        const int r = tx * 32 + y, c = ty * 32 + x;
        t[y][x] = (r < d && c < d && c >= r) ? H[(size_t)r * d + c] : 0.f;
    }
    __syncthreads();
    const double add = (double)damp * (*diag_sum / (double)d);
    for (int y = threadIdx.y; y < 32; y += 8) {
        const int r = ty * 32 + y, c = tx * 32 + x;   // = source (c, r) = t[x][y]
        if (r < d && c < d && r >= c) {
            const float v = t[x][y];
            H[(size_t)r * d + c] = (r == c) ? (float)((double)v + add) : v;
        }
    }
}

// H = P P^T / K + damp * mean(diag) * I from the planes of P (d x K, row stride ldk).
int gram_from_planes(float* p_hi, float* p_lo, int d, int K, int ldk, float damp, float* H,
                     double* dsum, int* dev_status, cudaStream_t st) {
    int e;
    CUtensorMap mh, ml;
    if ((e = tc::make_kmajor_map(&mh, p_hi, d, K, ldk, tc::BM))) return e;
    if ((e = tc::make_kmajor_map(&ml, p_lo, d, K, ldk, tc::BM))) return e;
    tc::ProblemList pl(BN);
    pl.add(0, 0, 0, 0, d, d, K, 0, 0, 1.f / (float)K, /*upper_only=*/1);
    tc::EpiStore epi{H, d, /*accumulate=*/0, /*upper=*/1};
    if ((e = tc::launch_gemm3x<BN, STAGES, kChunkKb>(mh, ml, mh, ml, pl, epi, dev_status, st)))
        return e;
    diag_sum_kernel<<<1, 1024, 0, st>>>(H, d, dsum);
    const int nt = (d + 31) / 32;
    mirror_damp_kernel<<<dim3(nt, nt), dim3(32, 8), 0, st>>>(H, d, dsum, damp);
    count_launches(2);
    return cuda_err(cudaGetLastError());
}

size_t planes_bytes(int d, int K) { return 2 * (size_t)d * tc::plane_ld(K) * sizeof(float); }

bool damp_ok(float damp) { return damp >= 0.f && damp < 3.0e38f; }

}  // namespace
}  // namespace bakron

using namespace bakron;

extern "C" size_t bakron_damped_gram_workspace_bytes(int N, int d) {
    if (N < 1 || d < 1) return 0;
    WsSizer z;
    z.take<char>(planes_bytes(d, N));
    z.take<double>(32);
    return z.bytes();
}

extern "C" int bakron_damped_gram(const float* X, int N, int d, float damp, float* H, void* ws,
                                  size_t ws_bytes, int* dev_status, void* stream) {
    if (N < 1 || d < 1 || d > 65536 || N > kMaxSplitRows || !damp_ok(damp) || !X || !H ||
        !dev_status)
        return BAKRON_ERR_INVALID_ARG;
    if (!ws_ok(ws, ws_bytes, bakron_damped_gram_workspace_bytes(N, d)))
        return BAKRON_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int ldk = tc::plane_ld(N);
    WsCarver c(ws);
    float* p = c.take<float>(planes_bytes(d, N) / sizeof(float));
    double* dsum = c.take<double>(32);
    float* p_hi = p;
    float* p_lo = p + (size_t)d * ldk;
    tc::split_planes(X, N, d, d, p_hi, p_lo, ldk, /*transpose=*/1, st);   // P = X^T
    return gram_from_planes(p_hi, p_lo, d, N, ldk, damp, H, dsum, dev_status, st);
}

extern "C" size_t bakron_sketch_b_workspace_bytes(int S, int m, int n) {
    if (S < 1 || m < 1 || n < 1) return 0;
    WsSizer z;
    z.take<char>(std::max(planes_bytes(n, S * m), planes_bytes(m, S * n)));
    z.take<double>(32);
    return z.bytes();
}

extern "C" int bakron_sketch_b(const float* G, int S, int m, int n, float damp, float* H_O,
                               float* H_I, void* ws, size_t ws_bytes, int* dev_status,
                               void* stream) {
    if (S < 1 || m < 1 || n < 1 || m > 65536 || n > 65536 || (long long)S * m > kMaxSplitRows ||
        (long long)S * n > (1LL << 30) || !damp_ok(damp) || !G || !H_O || !H_I || !dev_status)
        return BAKRON_ERR_INVALID_ARG;
    if (!ws_ok(ws, ws_bytes, bakron_sketch_b_workspace_bytes(S, m, n)))
        return BAKRON_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    WsCarver c(ws);
    float* p = c.take<float>(std::max(planes_bytes(n, S * m), planes_bytes(m, S * n)) /
                             sizeof(float));
    double* dsum = c.take<double>(32);
    int e;
    // H_I: P = (the S m x n stack of the G_s)^T, K = S m
    {
        const int K = S * m, ldk = tc::plane_ld(K);
        float* p_hi = p;
        float* p_lo = p + (size_t)n * ldk;
        tc::split_planes(G, K, n, n, p_hi, p_lo, ldk, /*transpose=*/1, st);
        if ((e = gram_from_planes(p_hi, p_lo, n, K, ldk, damp, H_I, dsum, dev_status, st)))
            return e;
    }
    // H_O: P = [G_1, ..., G_S] (m x S n), K = S n; the planes are reused in stream order
    {
        const int K = S * n, ldk = tc::plane_ld(K);
        float* p_hi = p;
        float* p_lo = p + (size_t)m * ldk;
        for (int s = 0; s < S; ++s)
            tc::split_planes(G + (size_t)s * m * n, m, n, n, p_hi + (size_t)s * n,
                             p_lo + (size_t)s * n, ldk, /*transpose=*/0, st);
        if ((e = gram_from_planes(p_hi, p_lo, m, K, ldk, damp, H_O, dsum + 1, dev_status, st)))
            return e;
    }
    return BAKRON_OK;
}
