// ldl.cu -- bakron_ldl: H = (I + L) D (I + L)^T, L strictly upper triangular.
//
// YAQA article (news.43b.com.cn/a/479517.html), section 4: L_O, L_I of the rounding rule come
// from the LDL decomposition H = (L + I) D (L + I)^T of each damped Kronecker factor; the rule
// of the same section makes L strictly upper (a U D U^T factorisation, i.e. LDL^T of H with its
// index order reversed).
//
// Two-level blocked right-looking algorithm, last indices first, built in place in the output
// L (which first receives the upper triangle of H). With U = I + L, pending indices A, the
// current block B and H' the Schur complement left by the indices after B:
//   H'_BB = U_BB D_B U_BB^T                  one CTA per 128-index block (fp64 in shared
//                                             memory), which also forms U_BB^{-1};
//   X     = H'_AB U_BB^{-T},  U_AB = X D_B^{-1} 3xTF32 tensor-core GEMM (K = 128) whose
//                                             epilogue writes U_AB into L and the hi/lo planes
//                                             of X and U_AB;
//   H'_AA -= X U_AB^T                        split in two: columns inside the current 512-index
//                                             outer block right away (K = 128), the rest once
//                                             per outer block (K = 512, upper block triangle),
//                                             so the trailing matrix is streamed n/512 times.
#include <algorithm>

#include "tcgemm_host.cuh"

namespace bakron {
namespace {

constexpr int NBI = 128;   // inner block: diagonal factorisation in one CTA
constexpr int NBO = 512;   // outer block: K of the trailing update
constexpr int BN = 128;
constexpr int STAGES = 3;
constexpr int DIAG_THREADS = 512;

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

constexpr int SUB = 32;                                   // sub-block of the diagonal block
constexpr int NSUB = NBI / SUB;
constexpr size_t kSOff = 0;                               // S: [NBI][NBI+1] fp64
constexpr size_t kXOff = kSOff + (size_t)NBI * (NBI + 1); // X: [NBI-SUB][SUB+1] fp64
constexpr size_t kTOff = kXOff + (size_t)(NBI - SUB) * (SUB + 1);  // T: [NSUB-1][SUB][SUB+1]
constexpr size_t kDiagSmem =
    (kTOff + (size_t)(NSUB - 1) * SUB * (SUB + 1) + NBI) * sizeof(double);

// U D U^T of the b x b diagonal block at [k0, k0 + b) (b <= 128) in fp64 shared memory;
// writes U's strictly upper part into L, the pivots into D, and U^{-1} (unit upper, zero
// padded to 128 x 128) as hi/lo planes with row stride 128.
//
// Indices >= b are padded with the identity (pivot 1, no coupling), so the block is always
// 128 wide. It is processed in 32-index sub-blocks, last first:
//  (1) one warp factors the 32 x 32 diagonal sub-block by rank-1 steps and accumulates its
//      inverse alongside: column j of U is u_j + e_j and U = G_31 ... G_1 with
//      G_j = I + u_j e_j^T, so U^{-1} = G_1^{-1} ... G_31^{-1}, G_j^{-1} = I - u_j e_j^T;
//  (2) all threads: X = H'[rows above, sub-block] W_JJ^T and U = X D^{-1} for the rows above;
//  (3) all threads: H'[rows above]^2 -= X U^T on the upper triangle.
// The inverse's off-diagonal blocks follow by block back substitution,
// W_IJ = -W_II sum_{I<K<=J} U_IK W_KJ. S keeps U in its strict upper triangle and W^T in its
// strict lower triangle (both unit diagonals implicit).
__global__ void __launch_bounds__(DIAG_THREADS) diag_block_kernel(float* __restrict__ L, int n,
                                                                int k0, int b,
                                                                float* __restrict__ D,
                                                                float* __restrict__ inv_hi,
                                                                float* __restrict__ inv_lo,
                                                                int* status) {
    extern __shared__ double dsm[];
    double(*S)[NBI + 1] = reinterpret_cast<double(*)[NBI + 1]>(dsm + kSOff);
    double(*X)[SUB + 1] = reinterpret_cast<double(*)[SUB + 1]>(dsm + kXOff);
    double(*T)[SUB][SUB + 1] = reinterpret_cast<double(*)[SUB][SUB + 1]>(dsm + kTOff);
    double* sD = dsm + kTOff + (size_t)(NSUB - 1) * SUB * (SUB + 1);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    for (int e = tid; e < NBI * NBI; e += DIAG_THREADS) {
        const int r = e / NBI, c = e % NBI;
        double v = 0.0;
        if (r < b && c < b) v = (c >= r) ? (double)L[(size_t)(k0 + r) * n + k0 + c] : 0.0;
        else if (r == c) v = 1.0;
        S[r][c] = v;
    }
    __syncthreads();
    for (int J = NSUB - 1; J >= 0; --J) {
        const int j0 = J * SUB;
        // (1) the diagonal sub-block, one warp
        if (warp == 0) {
            // lane = row r of the sub-block; the pivot column and the W row are read into
            // registers first (broadcast loads), then every update has a static offset
            double* Srow = &S[j0 + lane][j0];          // S[r][j0 + l]
            for (int jj = SUB - 1; jj >= 0; --jj) {
                const int j = j0 + jj;
                double d = S[j][j];
                const bool bad = !(d > 0.0) || !isfinite(d);
                if (bad) d = 1.0;
                if (lane == 0) {
                    sD[j] = d;
                    if (j < b) {
                        if (bad) set_status(status, BAKRON_ERR_NOT_PD);
                        D[k0 + j] = (float)d;
                    }
                }
                const double u = (lane < jj) ? S[j0 + lane][j] / d : 0.0;
                __syncwarp();
                if (lane < jj) S[j0 + lane][j] = u;
                const double ud = u * d;
                const bool act = lane < jj;
                // S[r][l] -= u_r d u_l for r <= l < j (u_l by shuffle: no shared-memory alias)
#pragma unroll
                for (int l = 0; l < SUB; ++l) {
                    const double ul = __shfl_sync(0xffffffffu, u, l);
                    if (act && l >= lane && l < jj) Srow[l] -= ud * ul;
                }
                // W[r][c] -= u_r W[j][c] for c > j, stored at S[j0+c][j0+r]; W[r][j] = -u_r.
                // W[j][c] = S[j0+c][j] is read 8 columns at a time before the 8 updates.
                if (act) S[j][j0 + lane] = -u;
#pragma unroll
                for (int c0 = 0; c0 < SUB; c0 += 8) {
                    double wrow[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q) wrow[q] = (c0 + q > jj) ? S[j0 + c0 + q][j] : 0.0;
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        if (act && c0 + q > jj) S[j0 + c0 + q][j0 + lane] -= u * wrow[q];
                }
                __syncwarp();
            }
        }
        __syncthreads();
        if (J == 0) break;
        // (2) X[r][c] = sum_{t >= c} H'[r][j0+t] W_JJ[c][t], rows r < j0 (4x4 register tiles)
        for (int e = tid; e < (j0 / 4) * (SUB / 4); e += DIAG_THREADS) {
            const int r0 = (e / (SUB / 4)) * 4, c0 = (e % (SUB / 4)) * 4;
            double acc[4][4] = {};
            for (int t = 0; t < SUB; ++t) {
                double h[4], w[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) h[i] = S[r0 + i][j0 + t];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int c = c0 + q;
                    w[q] = (t > c) ? S[j0 + t][j0 + c] : (t == c ? 1.0 : 0.0);
                }
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int q = 0; q < 4; ++q) acc[i][q] += h[i] * w[q];
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int q = 0; q < 4; ++q) X[r0 + i][c0 + q] = acc[i][q];
        }
        __syncthreads();
        for (int e = tid; e < j0 * SUB; e += DIAG_THREADS) {
            const int r = e / SUB, c = e % SUB;
            S[r][j0 + c] = X[r][c] / sD[j0 + c];
        }
        __syncthreads();
        // (3) H'[r][l] -= sum_c X[r][c] U[l][c], r <= l < j0, 4x4 tiles on the upper triangle
        {
            const int n4 = j0 / 4;
            for (int e = tid; e < n4 * (n4 + 1) / 2; e += DIAG_THREADS) {
                int R = 0, rem = e, rowlen = n4;
                while (rem >= rowlen) { rem -= rowlen; ++R; --rowlen; }
                const int Lt = R + rem, r0 = R * 4, l0 = Lt * 4;
                double acc[4][4] = {};
                for (int c = 0; c < SUB; ++c) {
                    double x[4], u[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) x[i] = X[r0 + i][c];
#pragma unroll
                    for (int q = 0; q < 4; ++q) u[q] = S[l0 + q][j0 + c];
#pragma unroll
                    for (int i = 0; i < 4; ++i)
#pragma unroll
                        for (int q = 0; q < 4; ++q) acc[i][q] += x[i] * u[q];
                }
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        if (l0 + q >= r0 + i) S[r0 + i][l0 + q] -= acc[i][q];
            }
        }
        __syncthreads();
    }
    // off-diagonal blocks of W = U^{-1}, by distance J - I = 1 .. NSUB-1 (4x4 register tiles)
    for (int dist = 1; dist < NSUB; ++dist) {
        const int npairs = NSUB - dist;
        // T_I = sum_{K=I+1..J} U_IK W_KJ
        for (int e = tid; e < npairs * (SUB / 4) * (SUB / 4); e += DIAG_THREADS) {
            const int I = e / ((SUB / 4) * (SUB / 4));
            const int t0 = ((e / (SUB / 4)) % (SUB / 4)) * 4, c0 = (e % (SUB / 4)) * 4;
            const int Jb = I + dist, i0 = I * SUB, jb0 = Jb * SUB;
            double acc[4][4] = {};
            for (int K = I + 1; K <= Jb; ++K) {
                const int kk0 = K * SUB;
                for (int sx = 0; sx < SUB; ++sx) {
                    double uu[4], w[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) uu[i] = S[i0 + t0 + i][kk0 + sx];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int c = c0 + q;   // W_KJ[sx][c]
                        w[q] = (K < Jb) ? S[jb0 + c][kk0 + sx]
                                        : ((c > sx) ? S[jb0 + c][jb0 + sx] : (c == sx ? 1.0 : 0.0));
                    }
#pragma unroll
                    for (int i = 0; i < 4; ++i)
#pragma unroll
                        for (int q = 0; q < 4; ++q) acc[i][q] += uu[i] * w[q];
                }
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int q = 0; q < 4; ++q) T[I][t0 + i][c0 + q] = acc[i][q];
        }
        __syncthreads();
        // W_IJ[a][c] = -sum_{t >= a} W_II[a][t] T[t][c], stored as S[J0+c][I0+a]
        for (int e = tid; e < npairs * (SUB / 4) * (SUB / 4); e += DIAG_THREADS) {
            const int I = e / ((SUB / 4) * (SUB / 4));
            const int a0 = ((e / (SUB / 4)) % (SUB / 4)) * 4, c0 = (e % (SUB / 4)) * 4;
            const int Jb = I + dist, i0 = I * SUB, jb0 = Jb * SUB;
            double acc[4][4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int q = 0; q < 4; ++q) acc[i][q] = T[I][a0 + i][c0 + q];
            for (int t = a0 + 1; t < SUB; ++t) {
                double wi[4], tt[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) wi[i] = (t > a0 + i) ? S[i0 + t][i0 + a0 + i] : 0.0;
#pragma unroll
                for (int q = 0; q < 4; ++q) tt[q] = T[I][t][c0 + q];
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int q = 0; q < 4; ++q) acc[i][q] += wi[i] * tt[q];
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int q = 0; q < 4; ++q) S[jb0 + c0 + q][i0 + a0 + i] = -acc[i][q];
        }
        __syncthreads();
    }
    for (int e = tid; e < NBI * NBI; e += DIAG_THREADS) {
        const int r = e / NBI, c = e % NBI;
        if (r < b && c < b && c > r) L[(size_t)(k0 + r) * n + k0 + c] = (float)S[r][c];
        // U^{-1}[r][c] (zero padded beyond b), hi/lo planes
        const float x = (r < b && c < b) ? (c > r ? (float)S[c][r] : (c == r ? 1.f : 0.f)) : 0.f;
        const float h = sm100::tf32_hi(x);
        inv_hi[e] = h;
        inv_lo[e] = x - h;
    }
}

// Panel epilogue: x = (H'_AB U_BB^{-T})[i][c]; U_AB = x / D_c goes to L; x and U_AB also go
// to the hi/lo planes used by the trailing updates (column offset c_off in the outer block).
struct EpiPanel {
    float* L;
    int n;
    const float* D;
    int kb0;
    float* xh;
    float* xl;
    float* uh;
    float* ul;
    int ldx;
    int c_off;
    __device__ void chunk(const tc::Problem& P, int row0, int c, int, int, const float* v) {
        if (c >= P.N) return;
        const float dc = D[kb0 + c];
#pragma unroll 8
        for (int rr = 0; rr < 32; ++rr) {
            const int row = row0 + rr;
            if (row >= P.M) break;
            const float x = v[rr * 33];
            const float u = __fdiv_rn(x, dc);
            L[(size_t)row * n + kb0 + c] = u;
            const size_t o = (size_t)row * ldx + c_off + c;
            const float xh_ = sm100::tf32_hi(x), uh_ = sm100::tf32_hi(u);
            xh[o] = xh_;
            xl[o] = x - xh_;
            uh[o] = uh_;
            ul[o] = u - uh_;
        }
    }
    __device__ void finish(const tc::Problem&, int) {}
};

struct LdlWs {
    float *inv_hi, *inv_lo, *p_hi, *p_lo, *x_hi, *x_lo, *u_hi, *u_lo;
};

template <class F>
void ldl_ws_layout(int n, F&& take) {
    take((size_t)NBI * NBI);        // inv_hi
    take((size_t)NBI * NBI);        // inv_lo
    take((size_t)n * NBI);          // p_hi  (panel of H')
    take((size_t)n * NBI);          // p_lo
    take((size_t)n * NBO);          // x_hi  (X of the outer block)
    take((size_t)n * NBO);          // x_lo
    take((size_t)n * NBO);          // u_hi  (U_AB of the outer block)
    take((size_t)n * NBO);          // u_lo
}

}  // namespace
}  // namespace bakron

using namespace bakron;

extern "C" size_t bakron_ldl_workspace_bytes(int n) {
    if (n < 1) return 0;
    WsSizer z;
    ldl_ws_layout(n, [&](size_t k) { z.take<float>(k); });
    return z.bytes();
}

extern "C" int bakron_ldl(const float* H, int n, float* L, float* D, void* ws, size_t ws_bytes,
                          int* dev_status, void* stream) {
    if (n < 1 || n > 65536 || !H || !L || !D || !dev_status) return BAKRON_ERR_INVALID_ARG;
    if (!ws_ok(ws, ws_bytes, bakron_ldl_workspace_bytes(n))) return BAKRON_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    WsCarver c(ws);
    float* bufs[8];
    int bi = 0;
    ldl_ws_layout(n, [&](size_t k) { bufs[bi++] = c.take<float>(k); });
    LdlWs w{bufs[0], bufs[1], bufs[2], bufs[3], bufs[4], bufs[5], bufs[6], bufs[7]};

    static bool diag_configured = false;
    if (!diag_configured) {
        if (cudaFuncSetAttribute(diag_block_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kDiagSmem) != cudaSuccess)
            return BAKRON_ERR_CUDA;
        diag_configured = true;
    }
    int e;
    // Tensor maps over the outer-block planes (fixed for the whole call).
    CUtensorMap m_xh, m_xl, m_uh, m_ul;
    if ((e = tc::make_kmajor_map(&m_xh, w.x_hi, n, NBO, NBO, tc::BM))) return e;
    if ((e = tc::make_kmajor_map(&m_xl, w.x_lo, n, NBO, NBO, tc::BM))) return e;
    if ((e = tc::make_kmajor_map(&m_uh, w.u_hi, n, NBO, NBO, BN))) return e;
    if ((e = tc::make_kmajor_map(&m_ul, w.u_lo, n, NBO, NBO, BN))) return e;

    const int eb = 1184;
    copy_upper_kernel<<<eb, 256, 0, st>>>(H, L, n);
    count_launches(1);
    for (int ko1 = n; ko1 > 0; ko1 -= NBO) {
        const int ko0 = std::max(0, ko1 - NBO);
        for (int t = 0, kb1 = ko1; kb1 > ko0; ++t, kb1 -= NBI) {
            // plane columns of this inner block, counted from the end of the outer block so
            // that they stay 128-aligned even when the outer block is a partial one
            const int kb0 = std::max(ko0, kb1 - NBI), b = kb1 - kb0, c_off = NBO - NBI * (t + 1);
            diag_block_kernel<<<1, DIAG_THREADS, kDiagSmem, st>>>(L, n, kb0, b, D, w.inv_hi,
                                                                  w.inv_lo, dev_status);
            count_launches(1);
            if (kb0 == 0) continue;
            // panel: X = H'[0:kb0, B] U_BB^{-T}
            tc::split_planes(L + kb0, kb0, b, n, w.p_hi, w.p_lo, NBI, 0, st);
            CUtensorMap m_ph, m_pl, m_ih, m_il;
            if ((e = tc::make_kmajor_map(&m_ph, w.p_hi, kb0, b, NBI, tc::BM))) return e;
            if ((e = tc::make_kmajor_map(&m_pl, w.p_lo, kb0, b, NBI, tc::BM))) return e;
            if ((e = tc::make_kmajor_map(&m_ih, w.inv_hi, NBI, b, NBI, BN))) return e;
            if ((e = tc::make_kmajor_map(&m_il, w.inv_lo, NBI, b, NBI, BN))) return e;
            tc::ProblemList pl(BN);
            pl.add(0, 0, 0, 0, kb0, b, b, 0, 0);
            EpiPanel ep{L, n, D, kb0, w.x_hi, w.x_lo, w.u_hi, w.u_lo, NBO, c_off};
            if ((e = tc::launch_gemm3x<BN, STAGES>(m_ph, m_pl, m_ih, m_il, pl, ep, dev_status, st)))
                return e;
            // columns of the outer block still pending: H'[0:kb0, ko0:kb0] -= X U_AB^T
            if (kb0 > ko0) {
                tc::ProblemList wl(BN);
                wl.add(0, c_off, ko0, c_off, kb0, kb0 - ko0, b, 0, ko0, -1.f);
                tc::EpiStore es{L, n, 1, 1};
                if ((e = tc::launch_gemm3x<BN, STAGES>(m_xh, m_xl, m_uh, m_ul, wl, es, dev_status,
                                                       st)))
                    return e;
            }
        }
        // the rest of the trailing matrix, once per outer block: upper block triangle
        if (ko0 > 0) {
            tc::ProblemList tl(BN);
            tl.add(0, 0, 0, 0, ko0, ko0, ko1 - ko0, 0, 0, -1.f, /*upper_only=*/1);
            tc::EpiStore es{L, n, 1, 1};
            if ((e = tc::launch_gemm3x<BN, STAGES>(m_xh, m_xl, m_uh, m_ul, tl, es, dev_status, st)))
                return e;
        }
    }
    clear_lower_kernel<<<eb, 256, 0, st>>>(L, n);
    count_launches(1);
    return cuda_err(cudaGetLastError());
}
