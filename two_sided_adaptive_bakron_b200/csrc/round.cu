// round.cu -- bakron_round: the BaKron solve of the two-sided adaptive rounding rule.
//
// What is computed (YAQA article, news.43b.com.cn/a/479517.html, section 4, rounding rule):
//   pre_ij = W*_ij + a_i^T E[:i,:j] b_j + a_i^T E[:i,j] + E[i,:j] b_j,  E = W* - W,
//   W_ij   = s_i * clamp(rint(pre_ij / s_i)).
// Entry (i,j) reads only entries (k,l) with k <= i, l <= j, so every anti-diagonal i+j = const
// is independent (BaKron page, abstract: O(m+n) sequential steps, anti-diagonal parallelism
// combined with a divide-and-conquer construction that brings the work to O(mn(m+n))).
//
// Reformulation. With U = (I + L_O)^T E (column-causal) the rule reads
//   pre_ij = W*_ij + T_ij + R_ij,   T_ij = sum_{k<i} L_O[k,i] E_kj,   U_ij = T_ij + E_ij,
//                                   R_ij = sum_{l<j} U_il L_I[l,j],
// a vertical sum over E (rows above) and a horizontal sum over U (columns to the left); the
// bilinear term a_i^T E[:i,:j] b_j is carried by U.
//
// Structure. The matrix is cut into 256 x 256 super-blocks, processed one super-block
// anti-diagonal ("phase") at a time; the blocks of a phase are independent of each other.
//  * Leaf launch (persistent, cooperative, one CTA per SM): every block of the phase is cut
//    into 32 x 32 leaves, taken in anti-diagonal order across all blocks of the phase, round
//    robin over the CTAs. In each CTA four loader warps stage a leaf: the far sums T_far,
//    R_far (everything outside its block, already accumulated) plus the contributions of the
//    leaves above / to the left inside its block (CUDA-core dot products, after a bounded wait
//    on each source leaf's ready flag). A fifth, solver warp runs the in-leaf wavefront of the
//    previous leaf meanwhile (two staging buffers, mbarrier handoff) and publishes it: codes,
//    W, E (row-major), E^T and U as hi/lo planes, then the leaf's release flag.
//  * Push launches (3xTF32 tcgen05 GEMMs, one grouped launch per direction): every block of
//    the phase pushes its E into T_far of all rows below it and its U into R_far of all
//    columns to its right (K = 256), i.e. the divide-and-conquer off-diagonal updates as dense
//    block products.
#include <algorithm>

#include "round_leaf.cuh"
#include "tcgemm_host.cuh"

namespace bakron {
namespace {

using leaf::LB;
constexpr int SB = 256;         // super-block edge
constexpr int LPB = SB / LB;    // leaves per super-block edge
constexpr int BN = 128;
constexpr int STAGES = 3;

struct PhaseArgs {
    const float* Ws;
    const float* LO;
    const float* LI;
    const float* sc;
    const float* Tf;
    const float* Rf;
    int m, n, Nt;
    int delta, p_lo, p_hi, maxd;
    float qlo, qhi;
    int8_t* codes;
    float* Wq;
    float* E;
    float* et_hi;
    float* et_lo;
    int ldm;
    float* u_hi;
    float* u_lo;
    int ldn;
    int* flags;
    int* abort_word;
    int* status;
    uint64_t limit_ns;
    int total;
};

__device__ __forceinline__ int leaves_of(int extent, int blk) {
    const int e = min(SB, extent - blk * SB);
    return (e + LB - 1) / LB;
}

// number of leaves (a, c) with a + c = d in a block of lm x ln leaves
__device__ __forceinline__ int diag_len(int d, int lm, int ln) {
    const int lo = max(0, d - ln + 1), hi = min(d, lm - 1);
    return hi >= lo ? hi - lo + 1 : 0;
}

constexpr int NLOAD = 128;       // loader threads (warps 0-3)
constexpr int NTHW = NLOAD + 32; // + the solver warp (warp 4)
using leaf::LS;
using leaf::LeafBuf;
using leaf::solve_leaf;

struct LeafSmem {
    LeafBuf buf[2];
    float sA[LB][LB + 1];        // pull staging
    float sB[LB][LB + 1];
    uint64_t full[2], empty[2];
    int stop;
};

__device__ __forceinline__ void loader_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(NLOAD) : "memory");
}

// Walks the phase's tasks: (local anti-diagonal d, block row P) in order, counting leaves.
struct TaskWalker {
    int d, P;
    long long base;
    __device__ void init(int p_lo) { d = 0; P = p_lo; base = 0; }
    __device__ void find(const PhaseArgs& a, int g, int& I, int& J) {
        int ln;
        while (true) {
            const int Q = a.delta - P;
            const int lm = leaves_of(a.m, P);
            ln = leaves_of(a.n, Q);
            const int cnt = diag_len(d, lm, ln);
            if (g < base + cnt) break;
            base += cnt;
            if (++P > a.p_hi) { P = a.p_lo; ++d; }
        }
        const int la = max(0, d - ln + 1) + (int)(g - base);
        I = P * LPB + la;
        J = (a.delta - P) * LPB + (d - la);
    }
};

// Codes, W and the E^T planes of the leaf solved from B (its E and U went out with its flag);
// run by the 128 loader threads before they stage a new leaf into B.
__device__ __forceinline__ void publish_rest(const PhaseArgs& a, const LeafBuf& B, int tid) {
    const int I = B.meta[0], J = B.meta[1], rows = B.meta[2], cols = B.meta[3];
    const int i0 = I * LB, j0 = J * LB;
#pragma unroll
    for (int q = 0; q < (LB * LB) / NLOAD; ++q) {
        const int e = tid + q * NLOAD, r = e >> 5, c = e & 31;
        if (r < rows && c < cols) {
            const size_t o = (size_t)(i0 + r) * a.n + j0 + c;
            a.codes[o] = B.oC[r * LB + c];
            a.Wq[o] = B.oW[r * LB + c];
        }
        // E^T: element (c, r) of the transposed planes, lane = row for coalescing
        if (c < rows && r < cols) {
            const float x = B.oEt[r * LB + c], xh = sm100::tf32_hi(x);
            const size_t ot = (size_t)(j0 + r) * a.ldm + i0 + c;
            a.et_hi[ot] = xh;
            a.et_lo[ot] = x - xh;
        }
    }
}

// Warps 0-3 stage leaf k into buffer k&1 (W*, the diagonal blocks of L_O and L_I, then the far
// sums plus the in-block contributions of the leaves above / left, each after a bounded wait
// on that leaf's ready flag) while warp 4 solves leaf k-1 from the other buffer and publishes
// what other leaves read (E, U) followed by its release flag; before restaging a buffer the
// loaders publish the rest of the leaf solved from it (codes, W, E^T planes). The solver warp never runs the staging code and the loaders never run the
// solver, so each keeps its own instruction stream.
__global__ void __launch_bounds__(NTHW, 1) phase_leaves_kernel(PhaseArgs a) {
    extern __shared__ __align__(16) uint8_t leaf_smem_raw[];
    LeafSmem& sm = *reinterpret_cast<LeafSmem*>(leaf_smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int m = a.m, n = a.n;
    if (tid == 0) {
        for (int b = 0; b < 2; ++b) {
            sm100::mbar_init(&sm.full[b], 1);
            sm100::mbar_init(&sm.empty[b], 1);
        }
        sm.stop = 0;
        sm100::fence_mbar_init();
    }
    __syncthreads();
    TaskWalker wk;
    wk.init(a.p_lo);

    if (warp < 4) {
        // ------------------------------------------------------------ loaders
        int k = 0;
        for (int g = blockIdx.x; g < a.total; g += gridDim.x, ++k) {
            const int b = k & 1;
            LeafBuf& B = sm.buf[b];
            if (k >= 2) {
                if (tid == 0 && !sm100::mbar_wait(&sm.empty[b], ((k >> 1) - 1) & 1, a.status,
                                                  a.limit_ns)) {
                    atomicExch(a.abort_word, 1);
                    sm.stop = 1;
                }
                loader_sync();
                if (*(volatile int*)&sm.stop) break;
                publish_rest(a, B, tid);   // leaf k - 2, solved from this buffer
                loader_sync();             // its meta is read before it is overwritten
            }
            int I, J;
            wk.find(a, g, I, J);
            const int P = wk.P, Q = a.delta - P;
            const int la = I - P * LPB, lc = J - Q * LPB;
            const int i0 = I * LB, j0 = J * LB;
            const int rows = min(LB, m - i0), cols = min(LB, n - j0);
            float accT[8], accR[8];
#pragma unroll
            for (int t = 0; t < 8; ++t) {
                const int r = warp * 8 + t;
                const bool ok = r < rows && lane < cols;
                const size_t o = (size_t)(i0 + r) * n + j0 + lane;
                accT[t] = ok ? __ldcg(&a.Tf[o]) : 0.f;
                accR[t] = ok ? __ldcg(&a.Rf[o]) : 0.f;
            }
            // what does not depend on other leaves first: W*, the diagonal blocks of L_O and
            // L_I, the scales (sA / sB are free again after the skew below)
#pragma unroll
            for (int q = 0; q < (LB * LB) / NLOAD; ++q) {
                const int e = tid + q * NLOAD, r = e >> 5, c = e & 31;
                B.W[e] = (r < rows && c < cols) ? __ldg(&a.Ws[(size_t)(i0 + r) * n + j0 + c]) : 0.f;
                sm.sA[r][c] = (r < rows && c < rows) ? __ldg(&a.LO[(size_t)(i0 + r) * m + i0 + c]) : 0.f;
                sm.sB[r][c] = (r < cols && c < cols) ? __ldg(&a.LI[(size_t)(j0 + r) * n + j0 + c]) : 0.f;
            }
            if (tid < LB) {
                const float sv = (tid < rows) ? __ldg(&a.sc[i0 + tid]) : 0.f;
                B.S[tid] = sv;
                B.S[LB + tid] = sv > 0.f ? __frcp_rn(sv) : 0.f;
            }
            if (tid == 0) { B.meta[0] = I; B.meta[1] = J; B.meta[2] = rows; B.meta[3] = cols; }
            loader_sync();
            for (int e = tid; e < LB * LS; e += NLOAD) {
                const int x = e / LS, dd = e % LS;
                B.LOr[e] = (dd >= 1 && dd < LB && x + dd < LB) ? sm.sA[x][x + dd] : 0.f;
                B.LIc[e] = (dd >= 1 && dd < LB && x - dd >= 0) ? sm.sB[x - dd][x] : 0.f;
            }
            loader_sync();
            bool stop = false;
            // In-block sources: the leaves above (vertical, via E) and to the left (horizontal,
            // via U). The two most recent ones, (la-1, lc) and (la, lc-1), finish last, so every
            // older source is pulled first and those two close the list.
            const int nv = max(la - 1, 0), nh = max(lc - 1, 0);
            const int nsrc = la + lc;
            for (int idx = 0; idx < nsrc && !stop; ++idx) {
                bool vert;
                int src;
                if (idx < nv) { vert = true; src = idx; }
                else if (idx < nv + nh) { vert = false; src = idx - nv; }
                else if (idx == nv + nh && la > 0) { vert = true; src = la - 1; }
                else { vert = false; src = lc - 1; }
                const int Is = vert ? P * LPB + src : I, Js = vert ? J : Q * LPB + src;
                if (tid == 0)
                    sm.stop = wait_flag(&a.flags[(size_t)Is * a.Nt + Js], a.abort_word, a.status,
                                        a.limit_ns) ? 0 : 1;
                loader_sync();
                if (*(volatile int*)&sm.stop) { stop = true; break; }
                if (vert) {
#pragma unroll
                    for (int q = 0; q < (LB * LB) / NLOAD; ++q) {
                        const int e = tid + q * NLOAD, kk = e >> 5, c = e & 31;
                        const size_t kr = (size_t)Is * LB + kk;
                        sm.sA[kk][c] = (c < rows) ? __ldg(&a.LO[kr * m + i0 + c]) : 0.f;
                        sm.sB[kk][c] = (c < cols) ? __ldcg(&a.E[kr * n + j0 + c]) : 0.f;
                    }
                    loader_sync();
#pragma unroll 8
                    for (int kk = 0; kk < LB; ++kk) {
                        const float bv = sm.sB[kk][lane];
#pragma unroll
                        for (int t = 0; t < 8; ++t)
                            accT[t] = fmaf(sm.sA[kk][warp * 8 + t], bv, accT[t]);
                    }
                } else {
#pragma unroll
                    for (int q = 0; q < (LB * LB) / NLOAD; ++q) {
                        const int e = tid + q * NLOAD, rr = e >> 5, c = e & 31;
                        const size_t l = (size_t)Js * LB;
                        const size_t o = (size_t)(i0 + rr) * a.ldn + l + c;
                        sm.sA[rr][c] = (rr < rows) ? (__ldcg(&a.u_hi[o]) + __ldcg(&a.u_lo[o])) : 0.f;
                        sm.sB[rr][c] = (c < cols) ? __ldg(&a.LI[(l + rr) * n + j0 + c]) : 0.f;
                    }
                    loader_sync();
#pragma unroll 8
                    for (int ll = 0; ll < LB; ++ll) {
                        const float bv = sm.sB[ll][lane];
#pragma unroll
                        for (int t = 0; t < 8; ++t)
                            accR[t] = fmaf(sm.sA[warp * 8 + t][ll], bv, accR[t]);
                    }
                }
                loader_sync();
            }
            if (stop) break;
            // the far and in-block sums
#pragma unroll
            for (int t = 0; t < 8; ++t) {
                B.T[(warp * 8 + t) * LB + lane] = accT[t];
                B.R[(warp * 8 + t) * LB + lane] = accR[t];
            }
            loader_sync();
            if (tid == 0) {
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(sm100::smem_u32(&sm.full[b])) : "memory");
            }
        }
        if (tid == 0) {
            // loaders ended early: let the solver warp see it
            if (*(volatile int*)&sm.stop) atomicExch(a.abort_word, 1);
        }
        // the last (up to) two leaves: wait until they are solved, then publish the rest
        if (!*(volatile int*)&sm.stop) {
            for (int kk = (k >= 2 ? k - 2 : 0); kk < k; ++kk) {
                const int b = kk & 1;
                if (tid == 0 && !sm100::mbar_wait(&sm.empty[b], (kk >> 1) & 1, a.status,
                                                  a.limit_ns)) {
                    atomicExch(a.abort_word, 1);
                    sm.stop = 1;
                }
                loader_sync();
                if (*(volatile int*)&sm.stop) break;
                publish_rest(a, sm.buf[b], tid);
            }
        }
    } else {
        // ------------------------------------------------------------ solver warp
        int k = 0;
        for (int g = blockIdx.x; g < a.total; g += gridDim.x, ++k) {
            const int b = k & 1;
            LeafBuf& B = sm.buf[b];
            bool ok = true;
            if (lane == 0) ok = sm100::mbar_wait(&sm.full[b], (k >> 1) & 1, a.status, a.limit_ns);
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!ok || ld_acquire_gpu(a.abort_word) != 0) {
                if (lane == 0) atomicExch(a.abort_word, 1);
                break;
            }
            const int I = B.meta[0], J = B.meta[1], rows = B.meta[2], cols = B.meta[3];
            const int i0 = I * LB, j0 = J * LB;
            solve_leaf(lane, rows, cols, a.qlo, a.qhi, B, a.status);
            __syncwarp();
            // publish what other leaves read (E for the vertical pulls, U for the horizontal
            // ones), then the flag; codes, W and the E^T planes follow from the loader warps
            if (lane < cols) {
                for (int r = 0; r < rows; ++r) {
                    const size_t o = (size_t)(i0 + r) * n + j0 + lane;
                    __stcg(&a.E[o], B.oE[r * LB + lane]);
                    const float u = B.oU[r * LB + lane], uh = sm100::tf32_hi(u);
                    const size_t ou = (size_t)(i0 + r) * a.ldn + j0 + lane;
                    __stcg(&a.u_hi[ou], uh);
                    __stcg(&a.u_lo[ou], u - uh);
                }
            }
            __threadfence();
            __syncwarp();
            if (lane == 0) {
                st_release_gpu(&a.flags[(size_t)I * a.Nt + J], 1);
                asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(sm100::smem_u32(&sm.empty[b])) : "memory");
            }
        }
    }
}

struct Layout {
    int Mt, Nt, MS, NS, ldm, ldn;
    size_t mn;
};

Layout layout(int m, int n) {
    Layout L;
    L.Mt = (m + LB - 1) / LB;
    L.Nt = (n + LB - 1) / LB;
    L.MS = (m + SB - 1) / SB;
    L.NS = (n + SB - 1) / SB;
    L.ldm = tc::plane_ld(m);
    L.ldn = tc::plane_ld(n);
    L.mn = (size_t)m * n;
    return L;
}

template <class F>
void round_ws_layout(const Layout& L, int m, int n, F&& take) {
    take((size_t)L.mn * 4);                         // E (row-major, first: see bakron.h)
    take((size_t)m * L.ldm * 4); take((size_t)m * L.ldm * 4);   // L_O^T planes
    take((size_t)n * L.ldn * 4); take((size_t)n * L.ldn * 4);   // L_I^T planes
    take((size_t)n * L.ldm * 4); take((size_t)n * L.ldm * 4);   // E^T planes
    take((size_t)m * L.ldn * 4); take((size_t)m * L.ldn * 4);   // U planes
    take((size_t)L.mn * 4);                         // T_far
    take((size_t)L.mn * 4);                         // R_far
    take(((size_t)L.Mt * L.Nt + 64) * 4);           // leaf flags + abort word
}

int leaf_grid(int tasks) {
    static int cached = 0;
    if (!cached) {
        int dev = 0, nsm = 0, per_sm = 0;
        if (cudaGetDevice(&dev) != cudaSuccess) return -1;
        if (cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return -1;
        if (cudaFuncSetAttribute(phase_leaves_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)sizeof(LeafSmem)) != cudaSuccess)
            return -1;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, phase_leaves_kernel, NTHW,
                                                          sizeof(LeafSmem)) != cudaSuccess)
            return -1;
        if (per_sm < 1) return -1;
        cached = per_sm * nsm;
    }
    return std::min(tasks, cached);
}

}  // namespace
}  // namespace bakron

using namespace bakron;

extern "C" size_t bakron_round_workspace_bytes(int m, int n) {
    if (m < 1 || n < 1) return 0;
    const Layout L = layout(m, n);
    WsSizer z;
    round_ws_layout(L, m, n, [&](size_t bytes) { z.take<char>(bytes); });
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
    char* p[12];
    int k = 0;
    round_ws_layout(L, m, n, [&](size_t bytes) { p[k++] = c.take<char>(bytes); });
    float* E = (float*)p[0];
    float *lot_hi = (float*)p[1], *lot_lo = (float*)p[2];
    float *lit_hi = (float*)p[3], *lit_lo = (float*)p[4];
    float *et_hi = (float*)p[5], *et_lo = (float*)p[6];
    float *u_hi = (float*)p[7], *u_lo = (float*)p[8];
    float *Tf = (float*)p[9], *Rf = (float*)p[10];
    int* flags = (int*)p[11];
    int e;
    if ((e = cuda_err(cudaMemsetAsync(flags, 0, ((size_t)L.Mt * L.Nt + 64) * 4, st)))) return e;
    if ((e = cuda_err(cudaMemsetAsync(Tf, 0, L.mn * 4, st)))) return e;
    if ((e = cuda_err(cudaMemsetAsync(Rf, 0, L.mn * 4, st)))) return e;
    // static operands of the pushes: L_O^T and L_I^T as hi/lo planes
    tc::split_planes(L_O, m, m, m, lot_hi, lot_lo, L.ldm, 1, st);
    tc::split_planes(L_I, n, n, n, lit_hi, lit_lo, L.ldn, 1, st);

    CUtensorMap m_loth, m_lotl, m_eth, m_etl, m_uh, m_ul, m_lith, m_litl;
    if ((e = tc::make_kmajor_map(&m_loth, lot_hi, m, m, L.ldm, tc::BM))) return e;
    if ((e = tc::make_kmajor_map(&m_lotl, lot_lo, m, m, L.ldm, tc::BM))) return e;
    if ((e = tc::make_kmajor_map(&m_eth, et_hi, n, m, L.ldm, BN))) return e;
    if ((e = tc::make_kmajor_map(&m_etl, et_lo, n, m, L.ldm, BN))) return e;
    if ((e = tc::make_kmajor_map(&m_uh, u_hi, m, n, L.ldn, tc::BM))) return e;
    if ((e = tc::make_kmajor_map(&m_ul, u_lo, m, n, L.ldn, tc::BM))) return e;
    if ((e = tc::make_kmajor_map(&m_lith, lit_hi, n, n, L.ldn, BN))) return e;
    if ((e = tc::make_kmajor_map(&m_litl, lit_lo, n, n, L.ldn, BN))) return e;

    PhaseArgs a;
    a.Ws = Wstar; a.LO = L_O; a.LI = L_I; a.sc = scales; a.Tf = Tf; a.Rf = Rf;
    a.m = m; a.n = n; a.Nt = L.Nt;
    a.qlo = (float)(-(1 << (bits - 1)));
    a.qhi = (float)((1 << (bits - 1)) - 1);
    a.codes = codes; a.Wq = W; a.E = E;
    a.et_hi = et_hi; a.et_lo = et_lo; a.ldm = L.ldm;
    a.u_hi = u_hi; a.u_lo = u_lo; a.ldn = L.ldn;
    a.flags = flags;
    a.abort_word = flags + (size_t)L.Mt * L.Nt;
    a.status = dev_status;
    a.limit_ns = spin_limit_ns();

    for (int delta = 0; delta < L.MS + L.NS - 1; ++delta) {
        const int p_lo = std::max(0, delta - (L.NS - 1)), p_hi = std::min(delta, L.MS - 1);
        int total = 0, maxd = 0;
        for (int P = p_lo; P <= p_hi; ++P) {
            const int lm = (std::min(SB, m - P * SB) + LB - 1) / LB;
            const int ln = (std::min(SB, n - (delta - P) * SB) + LB - 1) / LB;
            total += lm * ln;
            maxd = std::max(maxd, lm + ln - 2);
        }
        a.delta = delta; a.p_lo = p_lo; a.p_hi = p_hi; a.maxd = maxd; a.total = total;
        const int grid = leaf_grid(total);
        if (grid < 1) return BAKRON_ERR_CUDA;
        void* params[] = {&a};
        count_launches(1);
        if ((e = cuda_err(cudaLaunchCooperativeKernel((const void*)phase_leaves_kernel,
                                                      dim3(grid), dim3(NTHW), params,
                                                      sizeof(LeafSmem), st))))
            return e;

        // pushes of the phase's blocks: E down into T_far, U right into R_far
        tc::ProblemList pv(BN), ph(BN);
        auto flush_v = [&]() -> int {
            tc::EpiStore epi{Tf, n, 1, 0};
            int r = tc::launch_gemm3x<BN, STAGES>(m_loth, m_lotl, m_eth, m_etl, pv, epi,
                                                   dev_status, st);
            pv = tc::ProblemList(BN);
            return r;
        };
        auto flush_h = [&]() -> int {
            tc::EpiStore epi{Rf, n, 1, 0};
            int r = tc::launch_gemm3x<BN, STAGES>(m_uh, m_ul, m_lith, m_litl, ph, epi,
                                                   dev_status, st);
            ph = tc::ProblemList(BN);
            return r;
        };
        for (int P = p_lo; P <= p_hi; ++P) {
            const int Q = delta - P;
            const int r0 = P * SB, c0 = Q * SB;
            const int br = std::min(SB, m - r0), bc = std::min(SB, n - c0);
            if (r0 + br < m) {
                if (!pv.add(r0 + br, r0, c0, r0, m - (r0 + br), bc, br, r0 + br, c0)) {
                    if ((e = flush_v())) return e;
                    pv.add(r0 + br, r0, c0, r0, m - (r0 + br), bc, br, r0 + br, c0);
                }
            }
            if (c0 + bc < n) {
                if (!ph.add(r0, c0, c0 + bc, c0, br, n - (c0 + bc), bc, r0, c0 + bc)) {
                    if ((e = flush_h())) return e;
                    ph.add(r0, c0, c0 + bc, c0, br, n - (c0 + bc), bc, r0, c0 + bc);
                }
            }
        }
        if (!pv.empty() && (e = flush_v())) return e;
        if (!ph.empty() && (e = flush_h())) return e;
    }
    return cuda_err(cudaGetLastError());
}
