// round.cu -- bakron_round: the BaKron solve of the two-sided adaptive rounding rule.
//
// What is computed (YAQA article, news.43b.com.cn/a/479517.html, section 4, rounding rule):
//   pre_ij = W*_ij + a_i^T E[:i,:j] b_j + a_i^T E[:i,j] + E[i,:j] b_j,  E = W* - W,
//   W_ij   = s_i * clamp(rint(pre_ij / s_i))
// (or stochastic rounding, or a per-group grid step and a scalar codebook: round_leaf.cuh).
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
// Structure: one persistent cooperative launch over the whole matrix, cut into 32 x 32 leaves
// and 256 x 256 super-blocks, with two kinds of CTAs.
//  * Leaf CTAs take the leaves in anti-diagonal order (round robin over two groups per CTA,
//    each with two loader warps, a solver warp and its helper warp). A leaf's sums come in two
//    parts. The near field, the leaves above / to the left inside its own super-block and the
//    adjacent one, is pulled by the loaders (one warp per direction, 32 x 32 x 32 products on
//    the tensor cores from boxes brought in by TMA) after a bounded wait on each source leaf's
//    flag; the source to the left is usually the group's previous leaf, read from shared
//    memory. The far field, everything at least two super-blocks away, is read from T_far /
//    R_far once the leaf's 128 x 128 tile counters say that every far source has been added.
//    The solver and helper warps run the in-leaf wavefront (round_leaf.cuh); the solver then
//    publishes E and U^T and releases the leaf's flag, the helper publishes the U and E^T
//    planes and counts the leaf into its super-block, and the loaders copy out codes and W.
//  * GEMM CTAs run the far-field pushes as 3xTF32 tcgen05 tile tasks (128 x 128): E of the
//    super-blocks (A', C) into T_far of a target (A, C) with A >= A' + 2, and U of (A, C')
//    into R_far of (A, C) with C >= C' + 2, i.e. the divide-and-conquer off-diagonal products
//    as dense block products. A target takes its sources in batches by distance, {2}, {3},
//    {4, 5}, {6 .. 9}, {10 .. 17}, ... (consecutive super-blocks, so one batch is one product
//    over their joint K range): the nearest source, which is needed soonest, alone, the older
//    ones in ever longer products, so a target with c sources takes about log2(c) additions of
//    its tile instead of c. Tasks are ordered by their newest source super-block in the order
//    the sources finish (anti-diagonal, then row), nearest targets first, and handed out one at
//    a time from a global counter, so a free CTA always takes the oldest task nobody has taken;
//    each output tile takes its batches oldest first (a per-tile counter), so sums are
//    deterministic.
// Every task depends only on tasks that come earlier in one global order (leaves by
// anti-diagonal, the pushes of a super-block right after its last leaf and before the first
// leaf two super-blocks on), so the persistent CTAs always make progress; every wait is
// bounded and ends the launch through a shared abort word when it expires.
#include <algorithm>
#include <cstddef>
#include <cstring>
#include <limits>

#include "philox.cuh"
#include "round_leaf.cuh"
#include "tcgemm_host.cuh"

namespace bakron {
namespace {

using leaf::LB;
using leaf::LeafBuf;
using leaf::LS;
using leaf::LeafXchg;
using leaf::QKind;
using leaf::kMaxCodebook;
using leaf::solve_leaf_chain;
using leaf::solve_leaf_pushes;
using leaf::swz;

constexpr int SB = 256;              // super-block edge
constexpr int LPB = SB / LB;         // leaves per super-block edge
constexpr int TB = tc::BM;           // push tile edge (128)
constexpr int BN = 128;
constexpr int STAGES = 3;
constexpr int NTH = 256;             // 8 warps; each role uses 6 of them (see leaf_role, gemm_role)
constexpr int NLOAD = 64;            // loader threads of one leaf group
constexpr int kMaxLeafCtas = 96;
static_assert(TB % LB == 0 && SB % TB == 0, "tile nesting");

struct FusedArgs {
    const float* Ws;
    const float* LO;
    const float* LI;
    const float* sc;
    int m, n;
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
    float* Tf;
    float* Rf;
    float* Ut;           // U^T in full precision (n x ldm), read by the horizontal pulls
    int box_loads;       // 1: the leaf loaders read through the LeafMaps box maps
    int* flags;          // [Mt * Nt] leaf solved (E and U published)
    int* sb_done;        // [MS * NS] leaves of the super-block with E^T published
    int* cntT;           // [TM * TN] far sources added into the T_far tile
    int* cntR;           // [TM * TN] far sources added into the R_far tile
    int* abort_word;
    int* task_next;      // next push task to hand out (GEMM CTAs take tasks from it)
    int* status;
    const int* task_pre; // [nsb + 1] first push task of each source super-block (in order)
    const int2* task_sb; // [nsb] (A, C) of the source super-blocks, anti-diagonal order
    int nsb;
    int Mt, Nt, MS, NS, TN;
    int leaf_ctas;
    uint64_t limit_ns;
    int stoch;           // 1: stochastic Q with the variates of `seed`
    unsigned long long seed;
    int n_groups;        // grid steps per row (scales is m x n_groups)
    int group_size;      // columns per grid step: a multiple of the leaf width, or n
    int ncb;             // codebook entries (0: the integer grid)
    float cb[kMaxCodebook];       // the sorted codebook, last entry repeated
    float cbmid[kMaxCodebook];    // fl32((c_k + c_{k+1}) / 2), +inf past the last threshold
};

// 32 x 32 fp32 box maps (no swizzle) of the matrices a leaf reads; only valid when m and n are
// multiples of 4 (16-byte row strides), otherwise the loaders use plain loads.
struct LeafMaps {
    CUtensorMap lo;   // L_O (m x m), 128-byte swizzle (near-field operands)
    CUtensorMap li;   // L_I (n x n), 128-byte swizzle
    CUtensorMap lod;  // L_O, no swizzle (the leaf's diagonal block)
    CUtensorMap lid;  // L_I, no swizzle
    CUtensorMap e;    // E (m x n)
    CUtensorMap ut;   // U^T (n x m, row stride ldm)
    CUtensorMap ws;   // W* (m x n)
    CUtensorMap tf;   // T_far (m x n)
    CUtensorMap rf;   // R_far (m x n)
};

constexpr int NRING = 4;             // sources in flight per leaf group (box-load path)
constexpr int kBox = LB * LB;        // floats of one 32 x 32 box

struct alignas(1024) LeafGroupSmem {
    // box-load path: NRING stages of two boxes (swizzled copies: 1024-byte aligned); plain
    // path: sA, sB in stage 0
    float ring[NRING][2][kBox];
    LeafBuf buf[2];
    uint64_t rfull[NRING];       // box loads of a ring stage landed
    uint64_t sbar;               // W* and the diagonal blocks landed
    uint64_t tbar;               // T_far and R_far landed
    uint64_t full[2], empty[2];
    uint64_t solved[2];          // the solver is done with the leaf's wavefront (outputs in B)
    LeafXchg xch;                // solver / helper exchange
    int go;                      // solver -> helper: this leaf is on
    int stop;
};
struct LeafCtaSmem {
    LeafGroupSmem g[2];
    float qcb[kMaxCodebook];     // the codebook (read with a per-lane index)
};
static_assert(sizeof(LeafGroupSmem) % 1024 == 0 && offsetof(LeafGroupSmem, buf) % 128 == 0 &&
                  offsetof(LeafGroupSmem, ring) % 1024 == 0 && (kBox * 4) % 1024 == 0,
              "leaf group layout: 16-byte staging rows, 128-byte box destinations, 1024-byte "
              "swizzled box destinations");

constexpr size_t kGemmSmem = tc::gemm_smem_bytes<BN, STAGES>();
constexpr size_t kLeafSmem = sizeof(LeafCtaSmem) + 1024;  // + alignment slack
constexpr size_t kSmem = kLeafSmem > kGemmSmem ? kLeafSmem : kGemmSmem;
static_assert(kSmem <= 227 * 1024, "shared memory above the per-CTA limit");
static_assert(kGemmSmem + 256 <= kSmem, "room for the push CTAs' task ring after the barriers");

__device__ __forceinline__ int leaves_in(int extent_leaves, int blk) {
    return min(LPB, extent_leaves - blk * LPB);
}

// Batch j of a target's far sources: the super-blocks at distances bd_min(j) .. bd_max(j)
// (2, 3, 4-5, 6-9, 10-17, ...). A target at index X along the push direction has its sources at
// distances 2 .. X, in n_batches(X) batches; a source at index Xs is the newest source of
// batch j of the target Xs + bd_min(j), for the n_ready(Xs, NX) such targets inside the matrix.
__host__ __device__ constexpr int bd_min(int j) { return j < 2 ? 2 + j : (1 << (j - 1)) + 2; }
__host__ __device__ constexpr int bd_max(int j) { return j < 2 ? 2 + j : (1 << j) + 1; }
__host__ __device__ inline int n_batches(int X) {
    int j = 0;
    while (bd_min(j) <= X) ++j;
    return j;
}
__host__ __device__ inline int n_ready(int Xs, int NX) {
    int j = 0;
    while (Xs + bd_min(j) < NX) ++j;
    return j;
}

// Walks the leaves in anti-diagonal order (d = I + J, then I); g must not decrease.
struct LeafWalker {
    int d;
    long long base;
    __device__ void init() { d = 0; base = 0; }
    __device__ void find(int Mt, int Nt, long long g, int& I, int& J) {
        while (true) {
            const int lo = max(0, d - Nt + 1), hi = min(d, Mt - 1);
            const int cnt = hi - lo + 1;
            if (g < base + cnt) {
                I = lo + (int)(g - base);
                J = d - I;
                return;
            }
            base += cnt;
            ++d;
        }
    }
};

__device__ __forceinline__ void group_sync(int g) {
    asm volatile("bar.sync %0, %1;" ::"r"(1 + g), "n"(NLOAD) : "memory");
}

// Codes and W of the leaf solved from B (W = s_r q, or s_r c_q with a codebook, formed as in
// the solver); run by the group's loader threads before they restage B.
__device__ __forceinline__ void publish_rest(const FusedArgs& a, const LeafBuf& B, int lt,
                                             const float* qcb) {
    const int I = B.meta[0], J = B.meta[1], rows = B.meta[2], cols = B.meta[3];
    const int i0 = I * LB, j0 = J * LB;
#pragma unroll 4
    for (int q = 0; q < (LB * LB) / NLOAD; ++q) {
        const int e = lt + q * NLOAD, r = e >> 5, c = e & 31;
        if (r < rows && c < cols) {
            const size_t o = (size_t)(i0 + r) * a.n + j0 + c;
            const int q = B.oC[r * LB + c];
            a.codes[o] = (int8_t)q;
            a.Wq[o] = B.S[r] * (a.ncb > 0 ? qcb[q] : (float)q);
        }
    }
}

// One source's contribution D[m][n] += sum_k X[k][m] Y[k][n] (X, Y: 32 x 32 tiles in the
// swizzled layout swz) on the tensor cores, 3xTF32 as in the GEMM engine (hi = tf32
// truncation, lo = x - hi, hi*hi + hi*lo + lo*hi). Warp w of the group holds rows
// 16w .. 16w + 15, all 32 columns: acc[nt] is the m16n8 accumulator of columns 8nt .. 8nt + 7
// (element q at row 16w + g + 8 (q >> 1), column 8nt + 2t + (q & 1), g = lane / 4,
// t = lane % 4). Within each group of 8 k the fragment's k = t is taken from tile row 2t and
// k = t + 4 from row 2t + 1 (the same permutation for X and Y leaves the sum unchanged), so
// that every fragment load of the swizzled tiles hits 32 distinct banks.
__device__ __forceinline__ void product_mma(const float* X, const float* Y, int w, int lane,
                                            float (&acc)[4][4]) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int k0 = 0; k0 < LB; k0 += 8) {
        const int ka = k0 + 2 * t, kb = ka + 1;
        const float a[4] = {X[swz(ka, 16 * w + g)], X[swz(ka, 16 * w + g + 8)],
                            X[swz(kb, 16 * w + g)], X[swz(kb, 16 * w + g + 8)]};
        uint32_t ah[4], al[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float h = sm100::tf32_hi(a[i]);
            ah[i] = __float_as_uint(h);
            al[i] = __float_as_uint(a[i] - h);
        }
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
            const float b[2] = {Y[swz(ka, 8 * nt + g)], Y[swz(kb, 8 * nt + g)]};
            uint32_t bh[2], bl[2];
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const float h = sm100::tf32_hi(b[i]);
                bh[i] = __float_as_uint(h);
                bl[i] = __float_as_uint(b[i] - h);
            }
            sm100::mma_16x8x8_tf32(acc[nt], ah, bh);
            sm100::mma_16x8x8_tf32(acc[nt], ah, bl);
            sm100::mma_16x8x8_tf32(acc[nt], al, bh);
        }
    }
}

// The near-field sources of leaf (I, J) in super-block (A, C): the leaves above in this and the
// adjacent super-block (vertical, via E) and to the left (horizontal, via U); the older ones
// first, (I-1, J) and (I, J-1), which finish last, close the list.
struct NearField {
    int I, J, va, ha, nvs, nhs, nv, nh, nold, nsrc;
    __device__ NearField(int I_, int J_, int A, int C) : I(I_), J(J_) {
        va = max(0, (A - 1) * LPB);
        ha = max(0, (C - 1) * LPB);
        nvs = I - va;
        nhs = J - ha;
        nv = max(nvs - 1, 0);
        nh = max(nhs - 1, 0);
        nold = nv + nh;
        nsrc = nvs + nhs;
    }
    __device__ bool source(int idx, int& Is, int& Js) const {   // true: vertical
        if (idx < nv) { Is = va + idx; Js = J; return true; }
        if (idx < nold) { Is = I; Js = ha + (idx - nv); return false; }
        if (idx == nold && nvs > 0) { Is = I - 1; Js = J; return true; }
        Is = I; Js = J - 1;
        return false;
    }
};

// ------------------------------------------------------------------------------ leaf loaders
// The two loader warps of group g stage leaf k into buffer k & 1: W*, the diagonal blocks of
// L_O and L_I and the scales first, then (after the far-field counters) T_far / R_far plus the
// near-field contributions (one 32 x 32 x 32 product per source on CUDA cores). With box
// loads, one thread keeps NRING sources in flight through a ring of shared-memory stages.
__device__ void leaf_loaders(const FusedArgs& a, const LeafMaps* maps, LeafGroupSmem& sm, int g,
                             int lw, int lane, int slot, int nslots, const float* qcb) {
    const int lt = lw * 32 + lane;
    const bool lead = lt == 0;
    const int m = a.m, n = a.n;
    const long long total = (long long)a.Mt * a.Nt;
    const bool box = a.box_loads != 0;
    float* sA = &sm.ring[0][0][0];              // plain path staging (row stride LB)
    float* sB = sA + LB * LB;
    LeafWalker wk;
    wk.init();
    uint32_t rq = 0;                             // ring stages used so far (box path)
    int prevI = -1, prevJ = -1;                  // the group's previous leaf
    int k = 0;
    for (long long gi = slot; gi < total; gi += nslots, ++k) {
        const int b = k & 1;
        LeafBuf& B = sm.buf[b];
        if (k >= 2) {
            if (lead && !sm100::mbar_wait(&sm.empty[b], ((k >> 1) - 1) & 1, a.status, a.limit_ns)) {
                atomicExch(a.abort_word, 1);
                sm.stop = 1;
            }
            group_sync(g);
            if (*(volatile int*)&sm.stop) break;
            publish_rest(a, B, lt, qcb);   // leaf k - 2, solved from this buffer
            group_sync(g);            // its meta is read before it is overwritten
        }
        int I, J;
        wk.find(a.Mt, a.Nt, gi, I, J);
        const int A = I / LPB, C = J / LPB;
        const int i0 = I * LB, j0 = J * LB;
        const int rows = min(LB, m - i0), cols = min(LB, n - j0);
        // what does not depend on other leaves: W*, the diagonal blocks, the scales. With box
        // loads the diagonal blocks land in B.T / B.R (row-major), which the far-field sums
        // overwrite once the blocks are skewed into LOr / LIc, after the older near-field
        // products (so that those start right away).
        const float* dLO = sA;                   // plain path: diagonal blocks, swizzled tiles
        const float* dLI = sB;
        if (box) {
            if (lead) {
                sm100::mbar_arrive_expect_tx(&sm.sbar, 3 * kBox * 4);
                sm100::tma_load_2d(B.W, &maps->ws, j0, i0, &sm.sbar);
                sm100::tma_load_2d(B.T, &maps->lod, i0, i0, &sm.sbar);
                sm100::tma_load_2d(B.R, &maps->lid, j0, j0, &sm.sbar);
            }
        } else {
#pragma unroll 4
            for (int q = 0; q < (LB * LB) / NLOAD; ++q) {
                const int e = lt + q * NLOAD, r = e >> 5, c = e & 31;
                B.W[e] = (r < rows && c < cols) ? __ldg(&a.Ws[(size_t)(i0 + r) * n + j0 + c]) : 0.f;
                sA[swz(r, c)] = (r < rows && c < rows) ? __ldg(&a.LO[(size_t)(i0 + r) * m + i0 + c]) : 0.f;
                sB[swz(r, c)] = (r < cols && c < cols) ? __ldg(&a.LI[(size_t)(j0 + r) * n + j0 + c]) : 0.f;
            }
        }
        if (lt < LB) {
            // the leaf's grid step: per row, or per row and column group (one group per leaf)
            const float sv = (lt < rows)
                ? __ldg(&a.sc[(size_t)(i0 + lt) * a.n_groups + j0 / a.group_size]) : 0.f;
            B.S[lt] = sv;
            B.S[LB + lt] = sv > 0.f ? __frcp_rn(sv) : 0.f;
        }
        if (lead) { B.meta[0] = I; B.meta[1] = J; B.meta[2] = rows; B.meta[3] = cols; }
        if (a.stoch) {
            // the variates: thread lt takes row lt / 2 and the 16 columns from 16 (lt % 2), one
            // Philox block keyed (seed, 0) at counter (column / 16, row, 0, 0); the block's four
            // words, little-endian, are the 16 fields of those columns in order
            const int r = lt >> 1, cb = lt & 1;
            uint64_t w[4];
            philox4x64_10((uint64_t)((j0 >> 4) + cb), (uint64_t)(i0 + r), 0, 0, a.seed, 0, w);
            ulonglong2* dst = reinterpret_cast<ulonglong2*>(&B.oC[r * LB + 16 * cb]);
            dst[0] = make_ulonglong2(w[0], w[1]);
            dst[1] = make_ulonglong2(w[2], w[3]);
        }
        // far field: every super-block at least two steps above / to the left has been added
        // (the box path waits for it after its older near-field products, see below)
        const int ftile = (I * LB / TB) * a.TN + (J * LB / TB);
        auto far_ready = [&]() -> bool {
            bool ok = true;
            if (A >= 2)
                ok = wait_geq(&a.cntT[ftile], n_batches(A), a.abort_word, a.status, a.limit_ns);
            if (ok && C >= 2)
                ok = wait_geq(&a.cntR[ftile], n_batches(C), a.abort_word, a.status, a.limit_ns);
            return ok;
        };
        if (!box) {
            if (lead) sm.stop = far_ready() ? 0 : 1;
            group_sync(g);
            if (*(volatile int*)&sm.stop) break;
            for (int e = lt; e < LB * LS; e += NLOAD) {
                const int x = e / LS, dd = e % LS;
                B.LOr[e] = (dd >= 1 && dd < LB && x + dd < LB) ? dLO[swz(x, x + dd)] : 0.f;
                B.LIc[e] = (dd >= 1 && dd < LB && x - dd >= 0) ? dLI[swz(x - dd, x)] : 0.f;
            }
        }
        // this thread's accumulator elements (m16n8 layout, see product_mma)
        const int eg = lane >> 2, et = lane & 3;
        float accT[4][4], accR[4][4];
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int r = 16 * lw + eg + 8 * (q >> 1), c = 8 * nt + 2 * et + (q & 1);
                float tv = 0.f, rv = 0.f;
                if (!box) {
                    const bool ok = r < rows && c < cols;
                    const size_t o = (size_t)(i0 + r) * n + j0 + c;
                    tv = ok ? __ldcg(&a.Tf[o]) : 0.f;
                    rv = ok ? __ldcg(&a.Rf[o]) : 0.f;
                }
                accT[nt][q] = tv;
                accR[nt][q] = rv;
            }
        const NearField nf(I, J, A, C);
        // the recent horizontal source (I, J-1) is usually this group's previous leaf: its U is
        // still in the other buffer, so it needs no global round trip (box path only)
        const bool local_h = box && nf.nhs > 0 && prevI == I && prevJ == J - 1;
        const int hloc = nf.nsrc - 1;            // its index in the source list
        const LeafBuf& P = sm.buf[b ^ 1];        // the previous leaf's buffer
        // the older sources finished at least a diagonal ago: warp 0's lanes check their flags
        if (lw == 0) {
            bool ok = true;
            for (int idx = lane; idx < nf.nold && ok; idx += 32) {
                int Is, Js;
                nf.source(idx, Is, Js);
                ok = wait_flag(&a.flags[(size_t)Is * a.Nt + Js], a.abort_word, a.status, a.limit_ns);
            }
            ok = __all_sync(0xffffffffu, ok);
            if (lane == 0) sm.stop = ok ? 0 : 1;
        }
        group_sync(g);   // plain path: also, the skew is done with the diagonal blocks in sA / sB
        if (*(volatile int*)&sm.stop) break;
        bool stop = false;
        float acc[2][4][4];                      // box path: this warp's direction, all 32 rows
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int q = 0; q < 4; ++q) acc[mt][nt][q] = 0.f;
        if (box) {
            // loader warp lw takes one direction with its own two ring stages (2 lw, 2 lw + 1):
            // lw = 0 the vertical sources (E, into T), lw = 1 the horizontal ones (U, into R);
            // each source's product covers all 32 rows, so the warps never wait for each other
            const bool vdir = lw == 0;
            const int nold_d = vdir ? nf.nv : nf.nh;
            const int ns = nold_d + ((vdir ? nf.nvs : nf.nhs) > 0 ? 1 : 0);
            const bool loc = !vdir && local_h;   // the recent horizontal source is local
            auto srcd = [&](int i) -> int {      // the source's leaf index along the direction
                return i < nold_d ? (vdir ? nf.va : nf.ha) + i : (vdir ? I : J) - 1;
            };
            auto issue = [&](int i) {
                const uint32_t q = rq + i, st = 2 * lw + (q & 1);
                const int sl = srcd(i);
                if (loc && i == nold_d) {        // only L_I[sl cols][leaf cols]; U is in P
                    sm100::mbar_arrive_expect_tx(&sm.rfull[st], kBox * 4);
                    sm100::tma_load_2d(sm.ring[st][1], &maps->li, j0, sl * LB, &sm.rfull[st]);
                    return;
                }
                sm100::mbar_arrive_expect_tx(&sm.rfull[st], 2 * kBox * 4);
                if (vdir) {   // L_O[sl rows][leaf rows], E[sl rows][leaf cols]
                    sm100::tma_load_2d(sm.ring[st][0], &maps->lo, i0, sl * LB, &sm.rfull[st]);
                    sm100::tma_load_2d(sm.ring[st][1], &maps->e, j0, sl * LB, &sm.rfull[st]);
                } else {      // U^T[sl cols][leaf rows], L_I[sl cols][leaf cols]
                    sm100::tma_load_2d(sm.ring[st][0], &maps->ut, i0, sl * LB, &sm.rfull[st]);
                    sm100::tma_load_2d(sm.ring[st][1], &maps->li, j0, sl * LB, &sm.rfull[st]);
                }
            };
            // one source's product; false when a wait gave up
            auto product = [&](int i) -> bool {
                const bool recent = i == nold_d;
                if (recent) {   // its flag first (the local one needs none)
                    int okr = 1;
                    if (lane == 0) {
                        if (loc) {
                            issue(i);
                        } else {
                            const int sl = srcd(i);
                            const int* f = vdir ? &a.flags[(size_t)sl * a.Nt + J]
                                                : &a.flags[(size_t)I * a.Nt + sl];
                            okr = wait_flag(f, a.abort_word, a.status, a.limit_ns) ? 1 : 0;
                            if (okr) {
                                asm volatile("fence.proxy.async.global;" ::: "memory");
                                issue(i);
                            }
                        }
                    }
                    if (!__shfl_sync(0xffffffffu, okr, 0)) return false;
                }
                const uint32_t q = rq + i, st = 2 * lw + (q & 1);
                bool okw = sm100::mbar_wait(&sm.rfull[st], (q >> 1) & 1, a.status, a.limit_ns);
                if (okw && loc && recent)   // the previous leaf's wavefront is done
                    okw = sm100::mbar_wait(&sm.solved[b ^ 1], ((k - 1) >> 1) & 1, a.status,
                                           a.limit_ns);
                if (!__all_sync(0xffffffffu, okw)) return false;
                const float* X = (loc && recent) ? P.oUt : sm.ring[st][0];
                product_mma(X, sm.ring[st][1], 0, lane, acc[0]);
                product_mma(X, sm.ring[st][1], 1, lane, acc[1]);
                __syncwarp();   // the stage is free again
                if (lane == 0 && i + 2 < nold_d) issue(i + 2);
                return true;
            };
            if (lane == 0) {
                // the older sources' flags were acquired before the group barrier above
                asm volatile("fence.proxy.async.global;" ::: "memory");
                for (int i = 0; i < min(2, nold_d); ++i) issue(i);
            }
            for (int i = 0; i < nold_d && !stop; ++i) stop = !product(i);
            if (!vdir && !stop) {
                // the horizontal warp (whose older sources finish first), between its older and
                // its recent source: the diagonal blocks (in B.T / B.R) into LOr / LIc, then the
                // far field into B.T / B.R
                int ok = 1;
                if (lane == 0) ok = sm100::mbar_wait(&sm.sbar, k & 1, a.status, a.limit_ns);
                if (__shfl_sync(0xffffffffu, ok, 0)) {
                    for (int e = lane; e < LB * LS; e += 32) {
                        const int x = e / LS, dd = e % LS;
                        B.LOr[e] = (dd >= 1 && dd < LB && x + dd < LB) ? B.T[x * LB + x + dd] : 0.f;
                        B.LIc[e] = (dd >= 1 && dd < LB && x - dd >= 0) ? B.R[(x - dd) * LB + x] : 0.f;
                    }
                    __syncwarp();
                    if (lane == 0) {
                        ok = far_ready();
                        if (ok) {
                            // the skew's reads of B.T / B.R (generic proxy) come before the
                            // copies that overwrite them; T_far / R_far were written through
                            // the generic proxy on other SMs
                            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                            asm volatile("fence.proxy.async.global;" ::: "memory");
                            sm100::mbar_arrive_expect_tx(&sm.tbar, 2 * kBox * 4);
                            sm100::tma_load_2d(B.T, &maps->tf, j0, i0, &sm.tbar);
                            sm100::tma_load_2d(B.R, &maps->rf, j0, i0, &sm.tbar);
                        }
                    }
                }
                if (!__shfl_sync(0xffffffffu, ok, 0)) stop = true;
            }
            if (!stop && ns > nold_d) stop = !product(nold_d);
            if (!vdir && !stop && lane == 0 &&
                !sm100::mbar_wait(&sm.tbar, k & 1, a.status, a.limit_ns))
                stop = true;   // the far-field sums have landed in B.T / B.R
            stop = __shfl_sync(0xffffffffu, stop ? 1 : 0, 0) != 0;
            rq += ns;
            if (stop && lane == 0) {
                atomicExch(a.abort_word, 1);
                sm.stop = 1;
            }
        } else {
            // plain loads: the next source's blocks are fetched into registers while the
            // current one is multiplied; element e = lt + 64 q sits at (e >> 5, e & 31)
            float pf[32];
            auto fetch = [&](int idx) {
                int Is, Js;
                const bool vert = nf.source(idx, Is, Js);
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    const int e = lt + q * NLOAD, r = e >> 5, c = e & 31;
                    if (vert) {
                        const size_t kr = (size_t)Is * LB + r;
                        pf[q] = (c < rows) ? __ldg(&a.LO[kr * m + i0 + c]) : 0.f;
                        pf[16 + q] = (c < cols) ? __ldcg(&a.E[kr * n + j0 + c]) : 0.f;
                    } else {   // r = source column, c = leaf row (U^T) / leaf column (L_I)
                        const size_t l = (size_t)Js * LB;
                        pf[q] = (c < rows) ? __ldcg(&a.Ut[(l + r) * a.ldm + i0 + c]) : 0.f;
                        pf[16 + q] = (c < cols) ? __ldg(&a.LI[(l + r) * n + j0 + c]) : 0.f;
                    }
                }
            };
            auto wait_recent = [&](int idx) -> bool {
                if (idx < nf.nold) return true;
                if (lead) {
                    int Is, Js;
                    nf.source(idx, Is, Js);
                    sm.stop = wait_flag(&a.flags[(size_t)Is * a.Nt + Js], a.abort_word, a.status,
                                        a.limit_ns) ? 0 : 1;
                }
                group_sync(g);
                return !*(volatile int*)&sm.stop;
            };
            if (nf.nsrc > 0) {
                if (!wait_recent(0)) stop = true;
                else fetch(0);
            }
            for (int idx = 0; idx < nf.nsrc && !stop; ++idx) {
                int Is, Js;
                const bool vert = nf.source(idx, Is, Js);
                group_sync(g);   // the previous product is done with sA / sB
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    const int e = lt + q * NLOAD, r = e >> 5, c = e & 31;
                    sA[swz(r, c)] = pf[q];         // sA[k = source row / column][leaf row]
                    sB[swz(r, c)] = pf[16 + q];    // sB[k][leaf col]
                }
                if (idx + 1 < nf.nsrc) {
                    if (!wait_recent(idx + 1)) { stop = true; break; }
                    fetch(idx + 1);
                }
                group_sync(g);   // sA / sB complete
                if (vert) product_mma(sA, sB, lw, lane, accT);
                else product_mma(sA, sB, lw, lane, accR);
            }
        }
        // box path: the two warps may stop independently; they agree through sm.stop after the
        // barrier below (a warp leaving alone would strand the other at a named barrier)
        if (stop && !box) break;
        group_sync(g);
        if (*(volatile int*)&sm.stop) break;
        if (box) {
            // B.T / B.R hold the far sums; warp lw adds its direction's near field
            float* dst = lw == 0 ? B.T : B.R;
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int r = 16 * mt + eg + 8 * (q >> 1), c = 8 * nt + 2 * et + (q & 1);
                        const int o = r * LB + c;
                        dst[o] = (r < rows && c < cols) ? dst[o] + acc[mt][nt][q] : 0.f;
                    }
        } else {
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int r = 16 * lw + eg + 8 * (q >> 1), c = 8 * nt + 2 * et + (q & 1);
                    const int o = r * LB + c;
                    const bool ok = r < rows && c < cols;
                    B.T[o] = ok ? accT[nt][q] : 0.f;
                    B.R[o] = ok ? accR[nt][q] : 0.f;
                }
        }
        group_sync(g);
        if (lead) sm100::mbar_arrive(&sm.full[b]);
        prevI = I;
        prevJ = J;
    }
    if (lead && *(volatile int*)&sm.stop) atomicExch(a.abort_word, 1);
    // the last (up to) two leaves: wait until they are done with, then publish the rest
    if (!*(volatile int*)&sm.stop) {
        for (int kk = (k >= 2 ? k - 2 : 0); kk < k; ++kk) {
            const int b = kk & 1;
            if (lead && !sm100::mbar_wait(&sm.empty[b], (kk >> 1) & 1, a.status, a.limit_ns)) {
                atomicExch(a.abort_word, 1);
                sm.stop = 1;
            }
            group_sync(g);
            if (*(volatile int*)&sm.stop) break;
            publish_rest(a, sm.buf[b], lt, qcb);
        }
    }
}

// ------------------------------------------------------------------------------ leaf solver
__device__ void leaf_solver(const FusedArgs& a, LeafGroupSmem& sm, int lane, int slot,
                            int nslots, int bar, const float* qcb) {
    const int n = a.n;
    const long long total = (long long)a.Mt * a.Nt;
    int k = 0;
    for (long long gi = slot; gi < total; gi += nslots, ++k) {
        const int b = k & 1;
        LeafBuf& B = sm.buf[b];
        bool ok = true;
        if (lane == 0) ok = sm100::mbar_wait(&sm.full[b], (k >> 1) & 1, a.status, a.limit_ns);
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (ok && ld_acquire_gpu(a.abort_word) != 0) ok = false;
        // the helper follows this decision (it never waits on anything but the pair barrier)
        if (lane == 0) sm.go = ok ? 1 : 0;
        leaf::pair_sync(bar);
        if (!ok) {
            if (lane == 0) atomicExch(a.abort_word, 1);
            break;
        }
        const int I = B.meta[0], J = B.meta[1], rows = B.meta[2], cols = B.meta[3];
        const int i0 = I * LB, j0 = J * LB;
        if (a.ncb > 0)
            solve_leaf_chain<QKind::kCodebook>(lane, rows, cols, a.qlo, a.qhi, B, sm.xch, bar,
                                               a.status, qcb, a.cbmid);
        else if (a.stoch)
            solve_leaf_chain<QKind::kStochastic>(lane, rows, cols, a.qlo, a.qhi, B, sm.xch, bar,
                                                 a.status);
        else
            solve_leaf_chain<QKind::kNearest>(lane, rows, cols, a.qlo, a.qhi, B, sm.xch, bar,
                                              a.status);
        __syncwarp();
        if (lane == 0) sm100::mbar_arrive(&sm.solved[b]);
        // what the next leaves read: E (vertical pulls, lane = column) and U^T (horizontal pulls,
        // lane = row), then the flag; the loaders publish the rest
        if (lane < cols) {
            for (int r = 0; r < rows; ++r)
                __stcg(&a.E[(size_t)(i0 + r) * n + j0 + lane], B.oE[r * LB + lane]);
        }
        if (lane < rows) {
            for (int c = 0; c < cols; ++c)
                __stcg(&a.Ut[(size_t)(j0 + c) * a.ldm + i0 + lane], B.oUt[swz(c, lane)]);
        }
        __threadfence();
        __syncwarp();
        if (lane == 0) {
            st_release_gpu(&a.flags[(size_t)I * a.Nt + J], 1);
            sm100::mbar_arrive(&sm.empty[b]);
        }
    }
}

__device__ void leaf_helper(const FusedArgs& a, LeafGroupSmem& sm, int lane, int slot, int nslots,
                            int bar) {
    const long long total = (long long)a.Mt * a.Nt;
    int k = 0;
    for (long long gi = slot; gi < total; gi += nslots, ++k) {
        leaf::pair_sync(bar);             // the solver has decided (and seen the buffer full)
        if (!*(volatile int*)&sm.go) break;
        const int b = k & 1;
        LeafBuf& B = sm.buf[b];
        solve_leaf_pushes(lane, B, sm.xch, bar);
        // what the pushes read: the U planes (lane = column) and the E^T planes (lane = row),
        // then the leaf counts into its super-block; this depends on the leaf's own solve only
        const int I = B.meta[0], J = B.meta[1], rows = B.meta[2], cols = B.meta[3];
        const int i0 = I * LB, j0 = J * LB;
        if (lane < cols) {
            for (int r = 0; r < rows; ++r) {
                const float u = B.oU[r * LB + lane], uh = sm100::tf32_hi(u);
                const size_t ou = (size_t)(i0 + r) * a.ldn + j0 + lane;
                __stcg(&a.u_hi[ou], uh);
                __stcg(&a.u_lo[ou], u - uh);
            }
        }
        if (lane < rows) {
            for (int c = 0; c < cols; ++c) {
                const float x = B.oEt[c * LB + lane], xh = sm100::tf32_hi(x);
                const size_t ot = (size_t)(j0 + c) * a.ldm + i0 + lane;
                __stcg(&a.et_hi[ot], xh);
                __stcg(&a.et_lo[ot], x - xh);
            }
        }
        __threadfence();
        __syncwarp();
        if (lane == 0) {
            red_add_release_gpu(&a.sb_done[(I / LPB) * a.NS + (J / LPB)], 1);
            sm100::mbar_arrive(&sm.empty[b]);
        }
    }
}

__device__ void leaf_role(const FusedArgs& a, const LeafMaps* maps, uint8_t* smem) {
    LeafCtaSmem& cs = *reinterpret_cast<LeafCtaSmem*>(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int g = 0; g < 2; ++g) {
            for (int b = 0; b < 2; ++b) {
                sm100::mbar_init(&cs.g[g].full[b], 1);
                sm100::mbar_init(&cs.g[g].empty[b], 2);   // solver and helper
                sm100::mbar_init(&cs.g[g].solved[b], 1);
            }
            for (int r = 0; r < NRING; ++r) sm100::mbar_init(&cs.g[g].rfull[r], 1);
            sm100::mbar_init(&cs.g[g].sbar, 1);
            sm100::mbar_init(&cs.g[g].tbar, 1);
            cs.g[g].stop = 0;
        }
        sm100::fence_mbar_init();
    }
    if (threadIdx.x < kMaxCodebook) cs.qcb[threadIdx.x] = a.cb[threadIdx.x];
    __syncthreads();
    // warp w runs on SM sub-partition w % 4. Group g: helper warp g, solver warp 2 + g, loader
    // warps 4 + g and 6 + g, so the solver and its helper issue from different
    // sub-partitions and each sub-partition holds one of them plus one loader warp.
    // Named barriers: 1 + g for the loaders of group g, 3 + g for its solver and helper.
    const int g = warp & 1;
    const int slot = blockIdx.x * 2 + g, nslots = a.leaf_ctas * 2;
    if (warp < 2) leaf_helper(a, cs.g[g], lane, slot, nslots, 3 + g);
    else if (warp < 4) leaf_solver(a, cs.g[g], lane, slot, nslots, 3 + g, cs.qcb);
    else leaf_loaders(a, maps, cs.g[g], g, (warp - 4) >> 1, lane, slot, nslots, cs.qcb);
}

// ------------------------------------------------------------------------------ push tasks
struct PushTask {
    bool valid;
    bool vert;      // E into T_far (else U into R_far)
    int src_lo;     // the batch's source super-blocks along the column (vert) / row ...
    int src_hi;     // ... src_lo .. src_hi, src_hi the newest
    int pos;        // the batch's place in the tile's order of additions
    int A, C;       // target super-block
    int tr, tc;     // target 128 x 128 tile
    int k0;         // first K index (row / column of the sources)
    int nkb;        // k-blocks of 32
};

// Task t: its newest source super-block (A', C') by binary search over the prefix, then
// (target, tile) inside it: the targets (A' + bd_min(j), C') of the vertical push
// (j < n_ready(A', MS)) and (A', C' + bd_min(j)) of the horizontal one, nearest first
// (vertical, horizontal, then the next batch), 4 tiles each.
__device__ __forceinline__ PushTask decode_task(const FusedArgs& a, int t) {
    int lo = 0, hi = a.nsb - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (__ldg(&a.task_pre[mid]) <= t) lo = mid;
        else hi = mid - 1;
    }
    const int2 sc = __ldg(&a.task_sb[lo]);
    const int local = t - __ldg(&a.task_pre[lo]);
    const int nvj = n_ready(sc.x, a.MS), nhj = n_ready(sc.y, a.NS);
    const int mn = min(nvj, nhj);
    const int u = local >> 2, q = local & 3;
    int j;
    bool vert;
    if (u < 2 * mn) { j = u >> 1; vert = (u & 1) == 0; }
    else { j = mn + (u - 2 * mn); vert = nvj > nhj; }
    PushTask p;
    p.vert = vert;
    const int X = (vert ? sc.x : sc.y) + bd_min(j);       // the target along the direction
    p.A = vert ? X : sc.x;
    p.C = vert ? sc.y : X;
    p.src_hi = vert ? sc.x : sc.y;
    p.src_lo = max(0, X - bd_max(j));
    p.pos = n_batches(X) - 1 - j;                         // oldest batch first
    p.tr = 2 * p.A + (q >> 1);
    p.tc = 2 * p.C + (q & 1);
    p.valid = p.tr * TB < a.m && p.tc * TB < a.n;
    const int dim = vert ? a.m : a.n;
    p.k0 = p.src_lo * SB;
    p.nkb = (min((p.src_hi + 1) * SB, dim) - p.k0 + tc::BK - 1) / tc::BK;
    return p;
}

__device__ __forceinline__ void gemm_sync() {   // the six warps of the push pipeline
    asm volatile("bar.sync 2, 192;" ::: "memory");
}

__device__ __forceinline__ void epi_sync() {
    asm volatile("bar.sync 1, 128;" ::: "memory");
}

// Task ids travel from the producer (which takes them from the global counter) to the MMA
// issuer and the epilogue through a ring of kTaskFifo slots; -1 ends the stream.
constexpr int kTaskFifo = 8;
struct TaskFifo {
    int id[kTaskFifo];
    uint64_t full[kTaskFifo];    // the producer wrote the slot (1 arrival)
    uint64_t empty[kTaskFifo];   // the MMA issuer and the epilogue read it (2 arrivals)
};

// The consumer side: the n-th task id (or -1 at the end, -2 if a wait gave up).
__device__ __forceinline__ int fifo_pop(TaskFifo& q, int nth, int* status, uint64_t limit_ns,
                                        volatile int* s_abort) {
    const int f = nth % kTaskFifo;
    if (!tc::wait_or_abort(&q.full[f], (nth / kTaskFifo) & 1, status, limit_ns, s_abort))
        return -2;
    const int t = q.id[f];
    sm100::mbar_arrive(&q.empty[f]);
    return t;
}

// Tensor-core far-field pushes (same warp roles as the GEMM engine: warp 0 TMA, warp 1 MMA,
// warps 2-5 epilogue). The producer waits until the task's source super-block is complete; the
// epilogue waits until the output tile has taken every earlier source, adds the tile, and
// advances the tile's counter.
__device__ void gemm_role(const CUtensorMap* loth, const CUtensorMap* lotl, const CUtensorMap* eth,
                          const CUtensorMap* etl, const CUtensorMap* uh, const CUtensorMap* ul,
                          const CUtensorMap* lith, const CUtensorMap* litl, const FusedArgs& a,
                          uint8_t* smem_raw) {
    using Cf = tc::Cfg<BN>;
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float* epi_stage = reinterpret_cast<float*>(smem + STAGES * Cf::kStageBytes);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * Cf::kStageBytes + Cf::kEpiBytes);
    uint64_t* empty = full + STAGES;
    uint64_t* acc_full = empty + STAGES;
    uint64_t* acc_empty = acc_full + 2;
    uint64_t* drain = acc_empty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* s_abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
    volatile int* s_go = s_abort + 1;
    volatile int* s_task = s_go + 1;
    TaskFifo& fifo = *reinterpret_cast<TaskFifo*>(
        (reinterpret_cast<uintptr_t>(s_task + 1) + 7) & ~uintptr_t(7));

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp >= 6) return;   // the push pipeline uses warps 0 .. 5
    const int total = __ldg(&a.task_pre[a.nsb]);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            sm100::mbar_init(&full[s], 1);
            sm100::mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            sm100::mbar_init(&acc_full[b], 1);
            sm100::mbar_init(&acc_empty[b], 4);
        }
        sm100::mbar_init(drain, 1);
        for (int f = 0; f < kTaskFifo; ++f) {
            sm100::mbar_init(&fifo.full[f], 1);
            sm100::mbar_init(&fifo.empty[f], 2);
        }
        *s_abort = 0;
        *s_go = 0;
        sm100::fence_mbar_init();
    }
    if (warp == 1) {
        sm100::tmem_alloc(tmem_slot, Cf::kTmemCols);
        sm100::tmem_relinquish();
    }
    sm100::tc_fence_before();
    gemm_sync();
    sm100::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    auto stage_ptr = [&](int s, int which) -> uint8_t* {
        uint8_t* base = smem + (size_t)s * Cf::kStageBytes;
        return which < 2 ? base + which * Cf::kABytes : base + 2 * Cf::kABytes + (which - 2) * Cf::kBBytes;
    };

    if (warp == 0) {
        // ---------------- TMA producer
        if (lane == 0) {
            sm100::prefetch_tmap(loth); sm100::prefetch_tmap(lotl);
            sm100::prefetch_tmap(eth);  sm100::prefetch_tmap(etl);
            sm100::prefetch_tmap(uh);   sm100::prefetch_tmap(ul);
            sm100::prefetch_tmap(lith); sm100::prefetch_tmap(litl);
            uint32_t g = 0;
            for (int nt = 0; !*s_abort; ++nt) {
                // the next valid task from the global counter, or the end of the stream
                int t;
                PushTask p;
                do {
                    t = atomicAdd(a.task_next, 1);
                    if (t >= total) break;
                    p = decode_task(a, t);
                } while (!p.valid);
                const int f = nt % kTaskFifo;
                if (nt >= kTaskFifo &&
                    !tc::wait_or_abort(&fifo.empty[f], ((nt / kTaskFifo) & 1) ^ 1, a.status,
                                       a.limit_ns, s_abort))
                    break;
                fifo.id[f] = t < total ? t : -1;
                sm100::mbar_arrive(&fifo.full[f]);
                if (t >= total) break;
                bool ready = true;      // every source super-block of the batch is complete
                for (int sx = p.src_lo; sx <= p.src_hi && ready; ++sx) {
                    const int sA = p.vert ? sx : p.A, sC = p.vert ? p.C : sx;
                    const int need = leaves_in(a.Mt, sA) * leaves_in(a.Nt, sC);
                    ready = wait_geq(&a.sb_done[sA * a.NS + sC], need, a.abort_word, a.status,
                                     a.limit_ns);
                }
                if (!ready) {
                    *s_abort = 1;
                    break;
                }
                // the source planes were written through the generic proxy on other SMs
                asm volatile("fence.proxy.async.global;" ::: "memory");
                const CUtensorMap* ma_h = p.vert ? loth : uh;
                const CUtensorMap* ma_l = p.vert ? lotl : ul;
                const CUtensorMap* mb_h = p.vert ? eth : lith;
                const CUtensorMap* mb_l = p.vert ? etl : litl;
                bool ok = true;
                for (int kb = 0; kb < p.nkb; ++kb, ++g) {
                    const int s = g % STAGES;
                    if (g >= STAGES &&
                        !tc::wait_or_abort(&empty[s], ((g / STAGES) & 1) ^ 1, a.status, a.limit_ns, s_abort)) {
                        ok = false;
                        break;
                    }
                    sm100::mbar_arrive_expect_tx(&full[s], Cf::kStageBytes);
                    const int kx = p.k0 + kb * tc::BK;
                    sm100::tma_load_2d(stage_ptr(s, 0), ma_h, kx, p.tr * TB, &full[s]);
                    sm100::tma_load_2d(stage_ptr(s, 1), ma_l, kx, p.tr * TB, &full[s]);
                    sm100::tma_load_2d(stage_ptr(s, 2), mb_h, kx, p.tc * TB, &full[s]);
                    sm100::tma_load_2d(stage_ptr(s, 3), mb_l, kx, p.tc * TB, &full[s]);
                }
                if (!ok) break;
            }
            if (*s_abort) {
                atomicExch(a.abort_word, 1);
                for (uint32_t q = (g > (uint32_t)STAGES ? g - STAGES : 0); q < g; ++q)
                    sm100::mbar_wait(&full[q % STAGES], (q / STAGES) & 1, a.status, a.limit_ns);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = sm100::idesc_tf32(tc::BM, BN);
            uint32_t g = 0;
            int i = 0;
            for (int nt = 0; !*s_abort; ++nt) {
                const int t = fifo_pop(fifo, nt, a.status, a.limit_ns, s_abort);
                if (t < 0) break;
                const PushTask p = decode_task(a, t);
                const int b = i & 1;
                if (i >= 2 &&
                    !tc::wait_or_abort(&acc_empty[b], ((i >> 1) & 1) ^ 1, a.status, a.limit_ns, s_abort))
                    break;
                sm100::tc_fence_after();
                const uint32_t acc = tmem + (uint32_t)(b * BN);
                bool ok = true;
                for (int kb = 0; kb < p.nkb; ++kb, ++g) {
                    const int s = g % STAGES;
                    if (!tc::wait_or_abort(&full[s], (g / STAGES) & 1, a.status, a.limit_ns, s_abort)) {
                        ok = false;
                        break;
                    }
                    sm100::tc_fence_after();
                    const uint32_t ah = sm100::smem_u32(stage_ptr(s, 0));
                    const uint32_t al = sm100::smem_u32(stage_ptr(s, 1));
                    const uint32_t bh = sm100::smem_u32(stage_ptr(s, 2));
                    const uint32_t bl = sm100::smem_u32(stage_ptr(s, 3));
#pragma unroll
                    for (int kk = 0; kk < tc::BK / 8; ++kk) {
                        const uint32_t off = kk * 32;
                        const uint64_t dah = sm100::desc_kmajor_sw128(ah + off);
                        const uint64_t dal = sm100::desc_kmajor_sw128(al + off);
                        const uint64_t dbh = sm100::desc_kmajor_sw128(bh + off);
                        const uint64_t dbl = sm100::desc_kmajor_sw128(bl + off);
                        const uint32_t acc0 = (kb > 0 || kk > 0) ? 1u : 0u;
                        sm100::mma_tf32(acc, dah, dbh, idesc, acc0);
                        sm100::mma_tf32(acc, dah, dbl, idesc, 1u);
                        sm100::mma_tf32(acc, dal, dbh, idesc, 1u);
                    }
                    sm100::mma_commit(&empty[s]);
                }
                if (!ok) break;
                sm100::mma_commit(&acc_full[b]);
                ++i;
            }
            if (*s_abort) {
                sm100::mma_commit(drain);
                sm100::mbar_wait(drain, 0, a.status, a.limit_ns);
            }
        }
    } else {
        // ---------------- epilogue (warps 2 .. 5): T_far / R_far tile += accumulator
        const int quarter = warp & 3;
        float* stage = epi_stage + (warp - tc::kEpiWarp0) * (32 * 33);
        int i = 0;
        for (int nt = 0;; ++nt) {
            const int b = i & 1;
            if (threadIdx.x == tc::kEpiWarp0 * 32) {
                const int t = fifo_pop(fifo, nt, a.status, a.limit_ns, s_abort);
                bool ok = t >= 0;
                if (ok) {
                    const PushTask q = decode_task(a, t);
                    int* c = (q.vert ? a.cntT : a.cntR) + (size_t)q.tr * a.TN + q.tc;
                    ok = tc::wait_or_abort(&acc_full[b], (i >> 1) & 1, a.status, a.limit_ns,
                                           s_abort);
                    // the tile takes its batches in order
                    if (ok) ok = wait_geq(c, q.pos, a.abort_word, a.status, a.limit_ns);
                    if (!ok) { *s_abort = 1; atomicExch(a.abort_word, 1); }
                } else if (t == -2) {
                    atomicExch(a.abort_word, 1);
                }
                *s_task = t;
                *s_go = ok ? 1 : 0;
            }
            epi_sync();
            if (!*s_go) break;
            const PushTask p = decode_task(a, *s_task);
            int* cnt = (p.vert ? a.cntT : a.cntR) + (size_t)p.tr * a.TN + p.tc;
            sm100::tc_fence_after();
            float* Cm = p.vert ? a.Tf : a.Rf;
            const int row0 = p.tr * TB + quarter * 32;
#pragma unroll 1
            for (int c0 = 0; c0 < BN; c0 += 32) {
                float v[32];
                sm100::tmem_ld32(tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(b * BN + c0), v);
#pragma unroll
                for (int q = 0; q < 32; ++q) stage[lane * 33 + q] = v[q];
                __syncwarp();
                const int gc = p.tc * TB + c0 + lane;
                if (gc < a.n) {
                    // one fp32 add per element and source, in source order (the tile counter):
                    // the same sums as a load-add-store, without waiting for the loads
#pragma unroll
                    for (int rr = 0; rr < 32; ++rr)
                        if (row0 + rr < a.m)
                            red_add_f32(&Cm[(size_t)(row0 + rr) * a.n + gc], stage[rr * 33 + lane]);
                }
                __syncwarp();
            }
            __threadfence();
            sm100::tc_fence_before();
            epi_sync();
            if (threadIdx.x == tc::kEpiWarp0 * 32) st_release_gpu(cnt, p.pos + 1);
            if (lane == 0) sm100::mbar_arrive(&acc_empty[b]);
            ++i;
        }
    }
    __syncwarp();
    sm100::tc_fence_before();
    gemm_sync();
    if (warp == 1) sm100::tmem_dealloc(tmem, Cf::kTmemCols);
}

__global__ void __launch_bounds__(NTH, 1)
round_kernel(const __grid_constant__ CUtensorMap loth, const __grid_constant__ CUtensorMap lotl,
             const __grid_constant__ CUtensorMap eth, const __grid_constant__ CUtensorMap etl,
             const __grid_constant__ CUtensorMap uh, const __grid_constant__ CUtensorMap ul,
             const __grid_constant__ CUtensorMap lith, const __grid_constant__ CUtensorMap litl,
             const __grid_constant__ LeafMaps lmaps, const __grid_constant__ FusedArgs a) {
    extern __shared__ __align__(1024) uint8_t round_smem[];
    if ((int)blockIdx.x < a.leaf_ctas) {
        // swizzled box-copy destinations need 1024-byte alignment of the leaf layout's base
        uint8_t* base = reinterpret_cast<uint8_t*>(
            (reinterpret_cast<uintptr_t>(round_smem) + 1023) & ~uintptr_t(1023));
        leaf_role(a, &lmaps, base);
        return;
    }
    gemm_role(&loth, &lotl, &eth, &etl, &uh, &ul, &lith, &litl, a, round_smem);
}

// Push tasks per source super-block, in the order the sources finish (anti-diagonal, then row):
// pre[idx] = the first task of the idx-th source, sb[idx] its (A, C). One block: each thread
// takes a contiguous range of source indices, counts their tasks, and a block scan of the
// per-thread counts gives every range its first task.
constexpr int kPrefixThreads = 1024;
__global__ void __launch_bounds__(kPrefixThreads)
task_prefix_kernel(int MS, int NS, int* pre, int2* sb) {
    __shared__ int part[kPrefixThreads];
    const int nsb = MS * NS, tid = threadIdx.x;
    const int per = (nsb + kPrefixThreads - 1) / kPrefixThreads;
    const int i0 = min(nsb, tid * per), i1 = min(nsb, i0 + per);
    // the diagonal d of source index i0 and the index of that diagonal's first source
    int d = 0, base = 0;
    while (true) {
        const int cnt = min(d, MS - 1) - max(0, d - NS + 1) + 1;
        if (i0 < base + cnt || d >= MS + NS - 2) break;
        base += cnt;
        ++d;
    }
    auto walk = [&](auto&& f) {   // visits (idx, A, C) for idx in [i0, i1), in order
        int dd = d, bb = base;
        for (int i = i0; i < i1; ++i) {
            int lo = max(0, dd - NS + 1), hi = min(dd, MS - 1);
            while (i >= bb + hi - lo + 1) {
                bb += hi - lo + 1;
                ++dd;
                lo = max(0, dd - NS + 1);
                hi = min(dd, MS - 1);
            }
            const int A = lo + (i - bb);
            f(i, A, dd - A);
        }
    };
    int mine = 0;
    walk([&](int, int A, int C) { mine += 4 * (n_ready(A, MS) + n_ready(C, NS)); });
    part[tid] = mine;
    __syncthreads();
    for (int off = 1; off < kPrefixThreads; off <<= 1) {   // inclusive scan
        const int v = tid >= off ? part[tid - off] : 0;
        __syncthreads();
        part[tid] += v;
        __syncthreads();
    }
    int acc = part[tid] - mine;
    walk([&](int i, int A, int C) {
        pre[i] = acc;
        sb[i] = make_int2(A, C);
        acc += 4 * (n_ready(A, MS) + n_ready(C, NS));
    });
    if (tid == kPrefixThreads - 1) pre[nsb] = part[tid];
}

struct Layout {
    int Mt, Nt, MS, NS, TM, TN, ldm, ldn, nsb;
    size_t mn;
};

Layout layout(int m, int n) {
    Layout L;
    L.Mt = (m + LB - 1) / LB;
    L.Nt = (n + LB - 1) / LB;
    L.MS = (m + SB - 1) / SB;
    L.NS = (n + SB - 1) / SB;
    L.TM = (m + TB - 1) / TB;
    L.TN = (n + TB - 1) / TB;
    L.ldm = tc::plane_ld(m);
    L.ldn = tc::plane_ld(n);
    L.nsb = L.MS * L.NS;
    L.mn = (size_t)m * n;
    return L;
}

// the int region: leaf flags, super-block counts, tile counters, abort word (zeroed per call)
size_t sync_ints(const Layout& L) {
    return (size_t)L.Mt * L.Nt + (size_t)L.nsb + 2 * (size_t)L.TM * L.TN + 64;
}

template <class F>
void round_ws_layout(const Layout& L, int m, int n, F&& take) {
    take((size_t)L.mn * 4);                         // E (row-major, first: see bakron.h)
    take((size_t)m * L.ldm * 4); take((size_t)m * L.ldm * 4);   // L_O^T planes
    take((size_t)n * L.ldn * 4); take((size_t)n * L.ldn * 4);   // L_I^T planes
    take((size_t)n * L.ldm * 4); take((size_t)n * L.ldm * 4);   // E^T planes
    take((size_t)m * L.ldn * 4); take((size_t)m * L.ldn * 4);   // U planes
    take((size_t)n * L.ldm * 4);                    // U^T (full precision)
    take((size_t)L.mn * 4);                         // T_far
    take((size_t)L.mn * 4);                         // R_far
    take(sync_ints(L) * 4);                         // flags and counters
    take(((size_t)L.nsb + 1) * 4);                  // push-task prefix
    take((size_t)L.nsb * 8);                        // target super-blocks
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

namespace {

// The base quantizer of one call: the grid-step layout and the optional codebook.
struct QuantSpec {
    int group_size;              // columns per grid step (>= n: one per row)
    const float* codebook;       // host, 2^bits sorted entries, or nullptr (integer grid)
};

int round_impl(const float* Wstar, int m, int n, const float* L_O, const float* L_I,
               const float* scales, int bits, int stoch, unsigned long long seed,
               QuantSpec qs, int8_t* codes, float* W, void* ws, size_t ws_bytes,
               int* dev_status, void* stream) {
    if (m < 1 || n < 1 || (long long)m * n >= (1LL << 31) || !Wstar || !L_O || !L_I ||
        !scales || !codes || !W || !dev_status)
        return BAKRON_ERR_INVALID_ARG;
    if (qs.codebook ? (bits < 1 || bits > 4 || stoch) : (bits < 2 || bits > 8))
        return BAKRON_ERR_INVALID_ARG;
    if (qs.group_size < 1 || (qs.group_size < n && qs.group_size % LB != 0))
        return BAKRON_ERR_INVALID_ARG;
    const int group_size = std::min(qs.group_size, n);
    const int n_groups = (n + group_size - 1) / group_size;
    int ncb = 0;
    float cb[kMaxCodebook], cbmid[kMaxCodebook];
    if (qs.codebook) {
        ncb = 1 << bits;
        for (int k = 0; k < ncb; ++k) {
            const float c = qs.codebook[k];
            if (!(c > -3.0e38f && c < 3.0e38f) || (k > 0 && !(c > qs.codebook[k - 1])))
                return BAKRON_ERR_INVALID_ARG;   // non-finite or not strictly increasing
        }
    }
    for (int k = 0; k < kMaxCodebook; ++k) {
        cb[k] = ncb ? qs.codebook[std::min(k, ncb - 1)] : 0.f;
        const float sum = (k + 1 < ncb) ? qs.codebook[k] + qs.codebook[k + 1] : 0.f;
        cbmid[k] = (k + 1 < ncb) ? sum * 0.5f : std::numeric_limits<float>::infinity();
    }
    if (!ws_ok(ws, ws_bytes, bakron_round_workspace_bytes(m, n))) return BAKRON_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const Layout L = layout(m, n);
    WsCarver c(ws);
    char* p[15];
    int k = 0;
    round_ws_layout(L, m, n, [&](size_t bytes) { p[k++] = c.take<char>(bytes); });
    float* E = (float*)p[0];
    float *lot_hi = (float*)p[1], *lot_lo = (float*)p[2];
    float *lit_hi = (float*)p[3], *lit_lo = (float*)p[4];
    float *et_hi = (float*)p[5], *et_lo = (float*)p[6];
    float *u_hi = (float*)p[7], *u_lo = (float*)p[8];
    float* Ut = (float*)p[9];
    float *Tf = (float*)p[10], *Rf = (float*)p[11];
    int* ints = (int*)p[12];
    int* task_pre = (int*)p[13];
    int2* task_sb = (int2*)p[14];

    int e;
    if ((e = cuda_err(cudaMemsetAsync(ints, 0, sync_ints(L) * 4, st)))) return e;
    if ((e = cuda_err(cudaMemsetAsync(Tf, 0, L.mn * 4, st)))) return e;
    if ((e = cuda_err(cudaMemsetAsync(Rf, 0, L.mn * 4, st)))) return e;
    // static operands of the pushes: L_O^T and L_I^T as hi/lo planes
    tc::split_planes(L_O, m, m, m, lot_hi, lot_lo, L.ldm, 1, st);
    tc::split_planes(L_I, n, n, n, lit_hi, lit_lo, L.ldn, 1, st);
    task_prefix_kernel<<<1, kPrefixThreads, 0, st>>>(L.MS, L.NS, task_pre, task_sb);
    count_launches(1);

    CUtensorMap m_loth, m_lotl, m_eth, m_etl, m_uh, m_ul, m_lith, m_litl;
    if ((e = tc::make_kmajor_map(&m_loth, lot_hi, m, m, L.ldm, tc::BM))) return e;
    if ((e = tc::make_kmajor_map(&m_lotl, lot_lo, m, m, L.ldm, tc::BM))) return e;
    if ((e = tc::make_kmajor_map(&m_eth, et_hi, n, m, L.ldm, BN))) return e;
    if ((e = tc::make_kmajor_map(&m_etl, et_lo, n, m, L.ldm, BN))) return e;
    if ((e = tc::make_kmajor_map(&m_uh, u_hi, m, n, L.ldn, tc::BM))) return e;
    if ((e = tc::make_kmajor_map(&m_ul, u_lo, m, n, L.ldn, tc::BM))) return e;
    if ((e = tc::make_kmajor_map(&m_lith, lit_hi, n, n, L.ldn, BN))) return e;
    if ((e = tc::make_kmajor_map(&m_litl, lit_lo, n, n, L.ldn, BN))) return e;

    FusedArgs a;
    a.Ws = Wstar; a.LO = L_O; a.LI = L_I; a.sc = scales;
    a.m = m; a.n = n;
    a.qlo = (float)(-(1 << (bits - 1)));
    a.qhi = (float)((1 << (bits - 1)) - 1);
    a.codes = codes; a.Wq = W; a.E = E;
    a.et_hi = et_hi; a.et_lo = et_lo; a.ldm = L.ldm;
    a.u_hi = u_hi; a.u_lo = u_lo; a.ldn = L.ldn;
    a.Tf = Tf; a.Rf = Rf; a.Ut = Ut;
    a.flags = ints;
    a.sb_done = a.flags + (size_t)L.Mt * L.Nt;
    a.cntT = a.sb_done + L.nsb;
    a.cntR = a.cntT + (size_t)L.TM * L.TN;
    a.abort_word = a.cntR + (size_t)L.TM * L.TN;
    a.task_next = a.abort_word + 32;   // in the zeroed slack at the end of the int region
    a.status = dev_status;
    a.task_pre = task_pre;
    a.task_sb = task_sb;
    a.nsb = L.nsb;
    a.Mt = L.Mt; a.Nt = L.Nt; a.MS = L.MS; a.NS = L.NS; a.TN = L.TN;
    a.limit_ns = spin_limit_ns();
    a.stoch = stoch;
    a.seed = seed;
    a.n_groups = n_groups;
    a.group_size = group_size;
    a.ncb = ncb;
    for (int k = 0; k < kMaxCodebook; ++k) {
        a.cb[k] = cb[k];
        a.cbmid[k] = cbmid[k];
    }

    // box loads for the leaves when every row stride is a multiple of 16 bytes
    LeafMaps lm;
    memset(&lm, 0, sizeof(lm));
    auto al16 = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15) == 0; };
    a.box_loads = (m % 4 == 0 && n % 4 == 0 && al16(Wstar) && al16(L_O) && al16(L_I)) ? 1 : 0;
    if (a.box_loads) {
        if ((e = tc::make_box_map(&lm.lo, L_O, m, m, m, LB, true))) return e;
        if ((e = tc::make_box_map(&lm.li, L_I, n, n, n, LB, true))) return e;
        if ((e = tc::make_box_map(&lm.lod, L_O, m, m, m, LB))) return e;
        if ((e = tc::make_box_map(&lm.lid, L_I, n, n, n, LB))) return e;
        if ((e = tc::make_box_map(&lm.e, E, m, n, n, LB, true))) return e;
        if ((e = tc::make_box_map(&lm.ut, Ut, n, m, L.ldm, LB, true))) return e;
        if ((e = tc::make_box_map(&lm.ws, Wstar, m, n, n, LB))) return e;
        if ((e = tc::make_box_map(&lm.tf, Tf, m, n, n, LB))) return e;
        if ((e = tc::make_box_map(&lm.rf, Rf, m, n, n, LB))) return e;
    }

    if (cudaFuncSetAttribute(round_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kSmem) != cudaSuccess)
        return BAKRON_ERR_CUDA;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, round_kernel, NTH, kSmem) !=
            cudaSuccess || per_sm < 1)
        return BAKRON_ERR_CUDA;
    const int resident = per_sm * tc::sm_count();
    if (resident < 2) return BAKRON_ERR_CUDA;
    // two solver slots per leaf CTA, enough for one leaf anti-diagonal; the rest push
    const int diag = std::min(L.Mt, L.Nt);
    a.leaf_ctas = std::min({(diag + 1) / 2, kMaxLeafCtas, resident - 1});
    void* params[] = {&m_loth, &m_lotl, &m_eth, &m_etl, &m_uh, &m_ul, &m_lith, &m_litl, &lm, &a};
    count_launches(1);
    if ((e = cuda_err(cudaLaunchCooperativeKernel((const void*)round_kernel, dim3(resident),
                                                  dim3(NTH), params, kSmem, st))))
        return e;
    return cuda_err(cudaGetLastError());
}

}  // namespace

extern "C" int bakron_round(const float* Wstar, int m, int n, const float* L_O, const float* L_I,
                            const float* scales, int bits, int8_t* codes, float* W, void* ws,
                            size_t ws_bytes, int* dev_status, void* stream) {
    return round_impl(Wstar, m, n, L_O, L_I, scales, bits, 0, 0ull, QuantSpec{n, nullptr},
                      codes, W, ws, ws_bytes, dev_status, stream);
}

extern "C" int bakron_round_ex(const float* Wstar, int m, int n, const float* L_O,
                               const float* L_I, const float* scales, int group_size,
                               const float* codebook, int bits, int8_t* codes, float* W,
                               void* ws, size_t ws_bytes, int* dev_status, void* stream) {
    return round_impl(Wstar, m, n, L_O, L_I, scales, bits, 0, 0ull,
                      QuantSpec{group_size, codebook}, codes, W, ws, ws_bytes, dev_status,
                      stream);
}

extern "C" int bakron_round_stochastic(const float* Wstar, int m, int n, const float* L_O,
                                       const float* L_I, const float* scales, int bits,
                                       uint64_t seed, int8_t* codes, float* W, void* ws,
                                       size_t ws_bytes, int* dev_status, void* stream) {
    return round_impl(Wstar, m, n, L_O, L_I, scales, bits, 1, (unsigned long long)seed,
                      QuantSpec{n, nullptr}, codes, W, ws, ws_bytes, dev_status, stream);
}
