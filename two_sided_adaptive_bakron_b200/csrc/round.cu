// round.cu -- bakron_round: the BaKron solve of the two-sided adaptive rounding rule.
//
// What is computed (YAQA article, news.43b.com.cn/a/479517.html, section 4, rounding rule):
//   pre_ij = W*_ij + a_i^T E[:i,:j] b_j + a_i^T E[:i,j] + E[i,:j] b_j,  E = W* - W,
//   W_ij   = s_i * clamp(rint(pre_ij / s_i)).
// Entry (i,j) reads only entries (k,l) with k <= i, l <= j, so every anti-diagonal i+j = const
// is independent (BaKron page, abstract: O(m+n) sequential steps).
//
// Reformulation used here. With U = (I + L_O)^T E (column-causal) the rule reads
//   pre_ij = W*_ij + T_ij + R_ij,   T_ij = sum_{k<i} L_O[k,i] E_kj,   U_ij = T_ij + E_ij,
//                                   R_ij = sum_{l<j} U_il L_I[l,j],
// i.e. a vertical sum over E (from rows above) and a horizontal sum over U (from columns to
// the left); the bilinear term a_i^T E[:i,:j] b_j is carried by U.
//
// Structure (one persistent cooperative launch):
//  * The matrix is cut into 32x32 leaves. Leaf (I,J) depends on leaves (I',J) with I' < I
//    (through E) and (I,J') with J' < J (through U).
//  * Blocks take leaves in anti-diagonal order, round robin. Leaves of earlier diagonals have
//    smaller indices, every block walks its leaves in increasing index order and all blocks
//    are co-resident (cooperative launch), so the dependency waits cannot form a cycle.
//  * For its leaf a block first gathers the contributions of all earlier leaves (T from the
//    leaves above, R from the leaves to the left), waiting on each source leaf's ready flag
//    with a bounded spin. Then one warp runs the in-leaf anti-diagonal wavefront (63 steps):
//    lane j owns column j; values are indexed by step ("slot" t = r + j) so that every register
//    index is a compile-time constant; the vertical in-leaf updates stay in the lane, the
//    horizontal ones travel by warp shuffles. Finally the block publishes E and U of the leaf
//    and raises the leaf's flag (release), which readers acquire.
//  * E and U are read with ld.global.cg (L2, never a possibly stale L1 line).
#include <algorithm>

#include "common.cuh"

namespace bakron {
namespace {

constexpr int LB = 32;          // leaf edge
constexpr int NSLOT = 2 * LB - 1;
constexpr int NTH = 128;        // threads per block

struct RoundArgs {
    const float* Ws;
    const float* LO;
    const float* LI;
    const float* sc;
    int m, n, Mt, Nt;
    float qlo, qhi;
    int8_t* codes;
    float* Wq;
    float* E;
    float* U;
    int* flags;
    int* abort_word;
    int* status;
    uint64_t limit_ns;
    long long total;
};

__device__ __forceinline__ int diag_count(int D, int Mt, int Nt) {
    return min(D, Mt - 1) - max(0, D - Nt + 1) + 1;
}

// The in-leaf wavefront, run by one warp. Inputs live in shared memory with row stride LB:
// element (r, c) of a leaf sits at r*LB + c, so both an anti-diagonal (distinct c) and a row
// (distinct c) hit 32 distinct banks.
__device__ __forceinline__ void solve_leaf(int lane, int rows, int cols, float qlo, float qhi,
                                           const float* sW, const float* sT, const float* sR,
                                           const float* sLO, const float* sLI, const float* sS,
                                           int8_t* oC, float* oW, float* oE, float* oU,
                                           int* status) {
    const int j = lane;
    const bool colok = j < cols;
    float aT[NSLOT], aR[NSLOT];
#pragma unroll
    for (int t = 0; t < NSLOT; ++t) {
        const int r = t - j;
        const bool ok = (r >= 0) && (r < LB);
        const int rr = ok ? r : 0;
        aT[t] = ok ? sT[rr * LB + j] : 0.f;
        aR[t] = ok ? sR[rr * LB + j] : 0.f;
    }
    bool bad = false;
#pragma unroll
    for (int s = 0; s < NSLOT; ++s) {
        const int r = s - j;
        const bool inleaf = (r >= 0) && (r < LB);
        const int rr = inleaf ? r : 0;
        const bool act = inleaf && (r < rows) && colok;
        float e = 0.f, u = 0.f;
        if (act) {
            const float w_star = sW[rr * LB + j];
            const float pre = w_star + aT[s] + aR[s];
            const float sr = sS[rr];
            float q = 0.f;
            if (sr > 0.f) {
                q = rintf(__fdiv_rn(pre, sr));
                q = fminf(fmaxf(q, qlo), qhi);
            }
            bad |= !isfinite(pre);
            const float w = sr * q;
            e = w_star - w;
            u = aT[s] + e;
            oC[rr * LB + j] = (int8_t)q;
            oW[rr * LB + j] = w;
            oE[rr * LB + j] = e;
            oU[rr * LB + j] = u;
        }
        // vertical: E_rj feeds rows r+d of the same column (slot s+d of this lane)
#pragma unroll
        for (int d = 1; d < LB; ++d) {
            if (s + d < NSLOT) aT[s + d] = fmaf(sLO[d * LB + rr], e, aT[s + d]);
        }
        // horizontal: U_rj feeds columns j+d of the same row (slot s+d of lane j+d)
#pragma unroll
        for (int d = 1; d < LB; ++d) {
            if (s + d < NSLOT) {
                const float v = __shfl_up_sync(0xffffffffu, u, d);
                if (j >= d) aR[s + d] = fmaf(v, sLI[d * LB + (j - d)], aR[s + d]);
            }
        }
    }
    if (bad) set_status(status, BAKRON_ERR_NONFINITE);
}

__global__ void __launch_bounds__(NTH) round_leaves_kernel(RoundArgs a) {
    __shared__ float sA[LB][LB + 1];
    __shared__ float sB[LB][LB + 1];
    __shared__ float sT[LB * LB], sR[LB * LB], sW[LB * LB], sLO[LB * LB], sLI[LB * LB];
    __shared__ float oW[LB * LB], oE[LB * LB], oU[LB * LB];
    __shared__ int8_t oC[LB * LB];
    __shared__ float sS[LB];
    __shared__ int s_stop;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int m = a.m, n = a.n;
    int Dg = 0;
    long long base = 0;

    for (long long g = blockIdx.x; g < a.total; g += gridDim.x) {
        while (true) {
            const int c = diag_count(Dg, a.Mt, a.Nt);
            if (g < base + c) break;
            base += c;
            ++Dg;
        }
        const int I = max(0, Dg - (a.Nt - 1)) + (int)(g - base);
        const int J = Dg - I;
        const int i0 = I * LB, j0 = J * LB;
        const int rows = min(LB, m - i0), cols = min(LB, n - j0);

        float accT[8], accR[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) accT[t] = accR[t] = 0.f;

        // ---- vertical contributions of the leaves above: T += L_O[K-rows, leaf rows]^T E
        for (int Kp = 0; Kp < I; ++Kp) {
            if (tid == 0)
                s_stop = wait_flag(&a.flags[(size_t)Kp * a.Nt + J], a.abort_word, a.status,
                                   a.limit_ns) ? 0 : 1;
            __syncthreads();
            if (s_stop) return;
#pragma unroll
            for (int q = 0; q < (LB * LB) / NTH; ++q) {
                const int e = tid + q * NTH, kk = e >> 5, c = e & 31;
                const size_t k = (size_t)Kp * LB + kk;
                sA[kk][c] = (c < rows) ? __ldg(&a.LO[k * m + i0 + c]) : 0.f;
                sB[kk][c] = (c < cols) ? __ldcg(&a.E[k * n + j0 + c]) : 0.f;
            }
            __syncthreads();
#pragma unroll 8
            for (int kk = 0; kk < LB; ++kk) {
                const float b = sB[kk][lane];
#pragma unroll
                for (int t = 0; t < 8; ++t) accT[t] = fmaf(sA[kk][warp * 8 + t], b, accT[t]);
            }
            __syncthreads();
        }
        // ---- horizontal contributions of the leaves to the left: R += U[leaf rows, L-cols] L_I
        for (int Lp = 0; Lp < J; ++Lp) {
            if (tid == 0)
                s_stop = wait_flag(&a.flags[(size_t)I * a.Nt + Lp], a.abort_word, a.status,
                                   a.limit_ns) ? 0 : 1;
            __syncthreads();
            if (s_stop) return;
#pragma unroll
            for (int q = 0; q < (LB * LB) / NTH; ++q) {
                const int e = tid + q * NTH, rr = e >> 5, c = e & 31;
                const size_t l = (size_t)Lp * LB;
                sA[rr][c] = (rr < rows) ? __ldcg(&a.U[(size_t)(i0 + rr) * n + l + c]) : 0.f;
                sB[rr][c] = (c < cols) ? __ldg(&a.LI[(l + rr) * n + j0 + c]) : 0.f;
            }
            __syncthreads();
#pragma unroll 8
            for (int ll = 0; ll < LB; ++ll) {
                const float b = sB[ll][lane];
#pragma unroll
                for (int t = 0; t < 8; ++t) accR[t] = fmaf(sA[warp * 8 + t][ll], b, accR[t]);
            }
            __syncthreads();
        }

        // ---- stage the leaf
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            sT[(warp * 8 + t) * LB + lane] = accT[t];
            sR[(warp * 8 + t) * LB + lane] = accR[t];
        }
#pragma unroll
        for (int q = 0; q < (LB * LB) / NTH; ++q) {
            const int e = tid + q * NTH, r = e >> 5, c = e & 31;
            sW[e] = (r < rows && c < cols) ? __ldg(&a.Ws[(size_t)(i0 + r) * n + j0 + c]) : 0.f;
            // skewed diagonal blocks: sLO[d][r] = L_O[i0+r][i0+r+d], sLI[d][c] = L_I[j0+c][j0+c+d]
            const int d = r, x = c;
            sLO[e] = (d >= 1 && x + d < rows)
                         ? __ldg(&a.LO[(size_t)(i0 + x) * m + i0 + x + d]) : 0.f;
            sLI[e] = (d >= 1 && x + d < cols)
                         ? __ldg(&a.LI[(size_t)(j0 + x) * n + j0 + x + d]) : 0.f;
        }
        if (tid < LB) sS[tid] = (tid < rows) ? __ldg(&a.sc[i0 + tid]) : 0.f;
        __syncthreads();

        if (warp == 0)
            solve_leaf(lane, rows, cols, a.qlo, a.qhi, sW, sT, sR, sLO, sLI, sS, oC, oW, oE, oU,
                       a.status);
        __syncthreads();

        // ---- publish
#pragma unroll
        for (int q = 0; q < (LB * LB) / NTH; ++q) {
            const int e = tid + q * NTH, r = e >> 5, c = e & 31;
            if (r < rows && c < cols) {
                const size_t o = (size_t)(i0 + r) * n + j0 + c;
                a.codes[o] = oC[e];
                a.Wq[o] = oW[e];
                __stcg(&a.E[o], oE[e]);
                __stcg(&a.U[o], oU[e]);
            }
        }
        __threadfence();
        __syncthreads();
        if (tid == 0) st_release_gpu(&a.flags[(size_t)I * a.Nt + J], 1);
    }
}

struct Layout {
    int Mt, Nt;
    size_t mn;
};

Layout layout(int m, int n) {
    Layout L;
    L.Mt = (m + LB - 1) / LB;
    L.Nt = (n + LB - 1) / LB;
    L.mn = (size_t)m * n;
    return L;
}

}  // namespace
}  // namespace bakron

using namespace bakron;

extern "C" size_t bakron_round_workspace_bytes(int m, int n) {
    if (m < 1 || n < 1) return 0;
    const Layout L = layout(m, n);
    WsSizer z;
    z.take<float>(L.mn);                      // E
    z.take<float>(L.mn);                      // U
    z.take<int>((size_t)L.Mt * L.Nt + 64);    // leaf flags + abort word
    return z.bytes();
}

extern "C" int bakron_round(const float* Wstar, int m, int n, const float* L_O, const float* L_I,
                            const float* scales, int bits, int8_t* codes, float* W, void* ws,
                            size_t ws_bytes, int* dev_status, void* stream) {
    if (m < 1 || n < 1 || (long long)m * n >= (1LL << 31) || bits < 2 || bits > 8 ||
        !Wstar || !L_O || !L_I || !scales || !codes || !W || !dev_status)
        return BAKRON_ERR_INVALID_ARG;
    if (!ws_ok(ws, ws_bytes, bakron_round_workspace_bytes(m, n))) return BAKRON_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const Layout L = layout(m, n);
    WsCarver c(ws);
    RoundArgs a;
    a.E = c.take<float>(L.mn);
    a.U = c.take<float>(L.mn);
    a.flags = c.take<int>((size_t)L.Mt * L.Nt + 64);
    a.abort_word = a.flags + (size_t)L.Mt * L.Nt;
    int e = cuda_err(cudaMemsetAsync(a.flags, 0, ((size_t)L.Mt * L.Nt + 64) * sizeof(int), st));
    if (e) return e;
    a.Ws = Wstar; a.LO = L_O; a.LI = L_I; a.sc = scales;
    a.m = m; a.n = n; a.Mt = L.Mt; a.Nt = L.Nt;
    a.qlo = (float)(-(1 << (bits - 1)));
    a.qhi = (float)((1 << (bits - 1)) - 1);
    a.codes = codes; a.Wq = W;
    a.status = dev_status;
    a.limit_ns = spin_limit_ns();
    a.total = (long long)L.Mt * L.Nt;

    int dev = 0, nsm = 0, per_sm = 0;
    if ((e = cuda_err(cudaGetDevice(&dev)))) return e;
    if ((e = cuda_err(cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev)))) return e;
    if ((e = cuda_err(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, round_leaves_kernel,
                                                                    NTH, 0))))
        return e;
    if (per_sm < 1) return BAKRON_ERR_CUDA;
    const long long grid = std::min<long long>(a.total, (long long)per_sm * nsm);
    void* params[] = {&a};
    count_launches(1);
    return cuda_err(cudaLaunchCooperativeKernel((const void*)round_leaves_kernel, dim3((unsigned)grid),
                                                dim3(NTH), params, 0, st));
}
