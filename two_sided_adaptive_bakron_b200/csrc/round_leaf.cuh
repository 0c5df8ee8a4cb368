// round_leaf.cuh -- the in-leaf wavefront of the BaKron solve (32 x 32 leaf, a warp pair).
//
// YAQA article, section 4, rounding rule, with U = (I + L_O)^T E:
//   pre_ij = W*_ij + T_ij + R_ij,  T_ij = sum_{k<i} L_O[k,i] E_kj,  R_ij = sum_{l<j} U_il L_I[l,j],
//   W_ij = s_i clamp(rint(pre_ij / s_i)),  E_ij = W*_ij - W_ij,  U_ij = T_ij + E_ij,
// or, with stochastic Q (the same section's alternative),
//   W_ij = s_i clamp(floor(pre_ij / s_i + u_ij)),  u_ij uniform on (0, 1),
// or, with a scalar codebook c_0 < ... < c_{K-1} (the BaKron page, summary: the solver is
// modular in the base quantizer), W_ij = s_ij c_k for the entry k nearest to pre_ij / s_ij.
// The grid step s may be per row or per row and column group (one group per leaf).
// T and R arrive holding everything from outside the leaf; the wavefront adds the in-leaf part.
#pragma once

#include <cstddef>

#include "sm100.cuh"

namespace bakron {
namespace leaf {

constexpr int LB = 32;          // leaf edge
constexpr int NSLOT = 2 * LB - 1;
constexpr int UW = 4;            // wavefront steps per unrolled group
constexpr int WIN = LB + UW;     // register window of slots
constexpr int LS = LB + 4;       // row stride of the skewed diagonal blocks (16-byte rows)

// Element (r, c) of a 32 x 32 fp32 tile in the layout a tensor copy with 128-byte swizzle
// gives (a 1024-byte aligned tile of 128-byte rows): the 16-byte chunk c / 4 of row r sits at
// chunk (c / 4) ^ (r % 8). The near-field fragment loads (a K index 2t or 2t + 1 against a row
// or column index g, see product_mma) then touch 32 distinct banks.
__device__ __forceinline__ int swz(int r, int c) {
    return r * LB + ((((c >> 2) ^ r) & 7) << 2) + (c & 3);
}

// One staging buffer: a leaf's inputs and outputs (shared memory, floats). LOr and LIc rows
// are read as float4 (16-byte rows); W, T and R may be filled by tensor (box) copies, whose
// shared-memory destination must sit on a 128-byte boundary.
struct alignas(128) LeafBuf {
    float W[LB * LB];            // W* of the leaf, row stride LB
    float T[LB * LB];            // vertical sums (everything above the leaf)
    float R[LB * LB];            // horizontal sums (everything left of the leaf)
    float LOr[LB * LS];          // LOr[r*LS + d] = L_O[i0+r][i0+r+d]
    float LIc[LB * LS];          // LIc[c*LS + d] = L_I[j0+c-d][j0+c]
    float S[2 * LB];             // s_r and its reciprocal
    float oE[LB * LB], oU[LB * LB];
    float oEt[LB * LB];          // E transposed (for the transposed planes)
    float oUt[LB * LB];          // U transposed, element (c, r) at swz(c, r)
    // the codes; before the wavefront, with stochastic Q, the 16-bit fields k of the leaf's
    // variates u = (k + 1/2) / 2^16 (each is read by the lane that then writes the code there)
    alignas(16) int16_t oC[LB * LB];
    int meta[4];                 // I, J, rows, cols
};
static_assert(offsetof(LeafBuf, LOr) % 16 == 0 && offsetof(LeafBuf, LIc) % 16 == 0 &&
                  (LS * 4) % 16 == 0 && offsetof(LeafBuf, W) % 128 == 0 &&
                  offsetof(LeafBuf, oC) % 16 == 0 &&
                  offsetof(LeafBuf, T) % 128 == 0 && offsetof(LeafBuf, R) % 128 == 0 &&
                  sizeof(LeafBuf) % 128 == 0,
              "staging buffer: 16-byte float4 rows, 128-byte box destinations");


// ------------------------------------------------------------------------------ the wavefront
// The in-leaf wavefront: lane j owns column j and the element of row r is handled at step
// s = r + j. Leaf arrays use row stride LB, element (r, c) at r*LB + c, so an anti-diagonal and a
// row both touch 32 distinct banks. Per lane, slot s of a window holds the vertical / horizontal
// sum of its element of step s; a step reads slot s, then pushes E down its column into slots
// s+1..s+31 (in-lane) and U along its row into slot s+d of lane j+d (warp shuffles). LIc is
// zero for d > j and LOr for r + d >= 32, so no push needs a guard (a lane j < d gets its own
// u back from the shuffle and multiplies it by zero). The step loop stays rolled (4 steps per
// iteration) over a sliding window of 36 slot registers, so every register index is static.
// Q decides on the real quotient pre / s_r of the fp32 pre. It is estimated as
// x = pre * (1/s_r), within 1.2e-7 |x| of the real quotient (two correctly rounded steps);
// where x lies more than 1e-6 max(1,|x|) from every rounding boundary b, the estimate decides.
// Inside that zone the side is taken from the sign of r = fmaf(-b, s_r, pre): b * s_r is exact
// inside the fma (b has at most 24 significant bits) and the single rounding of the fma keeps
// the sign of the exact residual pre - b s_r, so the decision is the real one (r == 0 is an
// exact tie). The boundaries: k + 1/2 for nearest rounding (a tie goes to the even code); for
// stochastic Q (kStochastic, floor(pre/s + u)) the points pre/s = k - u, k an integer, with
// k - u exact in fp32 for |k| <= 128 (u has 17 significant bits), which covers every k that the
// clamp does not absorb, and y = x + u estimated within 1.2e-7 |x| + 2^-24 |y| <= 5e-7 max(1,|y|);
// for a codebook its fp32 midpoints.
//
// The wavefront runs on two warps: the solver warp runs the element chain (the slot's sum, Q,
// e, u and the distance-1 terms), the helper warp the distance >= 2 pushes one step behind.
// Round rho: the solver computes step rho from the helper's partial sums of slot rho
// (everything from steps <= rho - 2 on top of T, R) plus its own distance-1 terms of step
// rho - 1; the helper pushes step rho - 1 and publishes slot rho + 1. One named barrier of the
// two warps closes each round.
// The base quantizer of the wavefront.
enum class QKind { kNearest, kStochastic, kCodebook };
constexpr int kMaxCodebook = 16;

struct LeafXchg {
    float part[2][2][LB];        // [slot & 1][T, R][lane]: the helper's partial sums
    float eu[2][2][LB];          // [step & 1][e, u][lane]: the solver's step results
};

__device__ __forceinline__ void pair_sync(int id) {
    asm volatile("bar.sync %0, 64;" ::"r"(id) : "memory");
}

// Codebook Q: cb (shared memory) holds the entries, mid (any memory, read once per leaf) the
// decision thresholds fl32((c_k + c_{k+1}) / 2), +inf past the last one; the code is the number
// of thresholds below x (a tie goes to the lower entry), found by independent compares that
// also give the distance to the nearest threshold for the exact decision near one.
template <QKind kQ>
__device__ __forceinline__ void solve_leaf_chain(int lane, int rows, int cols, float qlo,
                                                 float qhi, LeafBuf& B, LeafXchg& X, int bar,
                                                 int* status, const float* cb = nullptr,
                                                 const float* mid = nullptr) {
    const int j = lane;
    const bool colok = j < cols;
    const float li1 = B.LIc[j * LS + 1];
    float lo1p = 0.f, ep = 0.f, usp = 0.f;   // distance-1 terms of the previous step
    bool bad = false;
    float md[kMaxCodebook - 1];
    if constexpr (kQ == QKind::kCodebook) {
#pragma unroll
        for (int t = 0; t < kMaxCodebook - 1; ++t) md[t] = mid[t];
    }
    pair_sync(bar);                          // the helper's slots 0 and 1 are in place
#pragma unroll 1
    for (int s = 0; s < NSLOT; ++s) {
        const int r = s - j;
        const bool inleaf = (r >= 0) && (r < LB);
        const int rr = inleaf ? r : 0;
        const bool act = inleaf && (r < rows) && colok;
        const float tT = fmaf(lo1p, ep, X.part[s & 1][0][j]);
        const float tR = fmaf(usp, li1, X.part[s & 1][1][j]);
        const float lo1 = B.LOr[rr * LS + 1];
        const float w_star = B.W[rr * LB + j];
        const float sr = B.S[rr], inv = B.S[LB + rr];
        float e = 0.f, u = 0.f;
        if (act) {
            const float pre = w_star + tT + tR;
            float q = 0.f, qv = 0.f;         // the code and its grid value
            if (sr > 0.f) {
                if constexpr (kQ == QKind::kCodebook) {
                    const float x = pre * inv;
                    int k = 0;
                    float dmin = __int_as_float(0x7f800000);
#pragma unroll
                    for (int t = 0; t < kMaxCodebook - 1; ++t) {
                        k += (x > md[t]) ? 1 : 0;
                        dmin = fminf(dmin, fabsf(x - md[t]));
                    }
                    if (dmin < 1e-6f * fmaxf(1.f, fabsf(x))) {
                        // exact: pre/s > mu_t iff pre - mu_t s > 0 (+inf thresholds give -inf)
                        k = 0;
#pragma unroll
                        for (int t = 0; t < kMaxCodebook - 1; ++t)
                            k += (__fmaf_rn(-md[t], sr, pre) > 0.f) ? 1 : 0;
                    }
                    q = (float)k;
                    qv = cb[k];
                } else if constexpr (kQ == QKind::kStochastic) {
                    const float uv = ((float)(uint16_t)B.oC[rr * LB + j] + 0.5f) * (1.f / 65536.f);
                    const float y = __fadd_rn(__fmul_rn(pre, inv), uv);
                    const float k = rintf(y);
                    float f = floorf(y);
                    if (fabsf(y - k) < 1e-6f * fmaxf(1.f, fabsf(y)))
                        // exact: pre/s + u >= k iff pre - (k - u) s >= 0
                        f = (__fmaf_rn(-__fsub_rn(k, uv), sr, pre) >= 0.f) ? k : k - 1.f;
                    q = fminf(fmaxf(f, qlo), qhi);
                    qv = q;
                } else {
                    const float x = pre * inv;
                    float c = rintf(x);
                    const float t = fabsf(x - c);
                    if (0.5f - t < 1e-6f * fmaxf(1.f, fabsf(x))) {
                        // exact: the side of b = floor(x) + 1/2 from the sign of pre - b s; a
                        // zero residual is a tie, which goes to the even neighbour
                        const float lo = floorf(x), r = __fmaf_rn(-(lo + 0.5f), sr, pre);
                        c = r > 0.f ? lo + 1.f : (r < 0.f ? lo : rintf(lo + 0.5f));
                    }
                    q = fminf(fmaxf(c, qlo), qhi);
                    qv = q;
                }
            }
            bad |= !isfinite(pre);
            const float w = sr * qv;
            e = w_star - w;
            u = tT + e;
            B.oC[rr * LB + j] = (int16_t)q;
            B.oE[rr * LB + j] = e;
            B.oEt[j * LB + rr] = e;
            B.oU[rr * LB + j] = u;
            B.oUt[swz(j, rr)] = u;
        }
        X.eu[s & 1][0][j] = e;
        X.eu[s & 1][1][j] = u;
        lo1p = lo1;
        ep = e;
        usp = __shfl_up_sync(0xffffffffu, u, 1);
        pair_sync(bar);
    }
    pair_sync(bar);                          // the helper's last round
    if (bad) set_status(status, BAKRON_ERR_NONFINITE);
}

__device__ __forceinline__ void solve_leaf_pushes(int lane, LeafBuf& B, LeafXchg& X, int bar) {
    const int j = lane;
    float li[LB];
#pragma unroll
    for (int q = 0; q < LB / 4; ++q) {
        const float4 v = *reinterpret_cast<const float4*>(&B.LIc[j * LS + 4 * q]);
        li[4 * q] = v.x; li[4 * q + 1] = v.y; li[4 * q + 2] = v.z; li[4 * q + 3] = v.w;
    }
    float wT[WIN], wR[WIN];
#pragma unroll
    for (int t = 0; t < WIN; ++t) {
        const int r = t - j;
        const bool ok = (r >= 0) && (r < LB);
        const int rr = ok ? r : 0;
        wT[t] = ok ? B.T[rr * LB + j] : 0.f;
        wR[t] = ok ? B.R[rr * LB + j] : 0.f;
    }
    X.part[0][0][j] = wT[0];
    X.part[0][1][j] = wR[0];
    X.part[1][0][j] = wT[1];
    X.part[1][1][j] = wR[1];
    pair_sync(bar);                          // slots 0 and 1 are in place
    pair_sync(bar);                          // first exchange: step 0 is being computed
#pragma unroll 1
    for (int s0 = 0; s0 < NSLOT; s0 += UW) {
#pragma unroll
        for (int k = 0; k < UW; ++k) {
            const int s = s0 + k;            // step pushed in round s + 1
            if (s < NSLOT) {
                const int r = s - j;
                const bool inleaf = (r >= 0) && (r < LB);
                const int rr = inleaf ? r : 0;
                float lo[LB];
#pragma unroll
                for (int q = 0; q < LB / 4; ++q) {
                    const float4 v = *reinterpret_cast<const float4*>(&B.LOr[rr * LS + 4 * q]);
                    lo[4 * q] = v.x; lo[4 * q + 1] = v.y; lo[4 * q + 2] = v.z; lo[4 * q + 3] = v.w;
                }
                const float e = X.eu[s & 1][0][j], u = X.eu[s & 1][1][j];
#pragma unroll
                for (int d = 2; d < LB; ++d) wT[k + d] = fmaf(lo[d], e, wT[k + d]);
#pragma unroll
                for (int d = 2; d < LB; ++d)
                    wR[k + d] = fmaf(__shfl_up_sync(0xffffffffu, u, d), li[d], wR[k + d]);
                // slot s + 2 has all its distance >= 2 terms now
                X.part[(s + 2) & 1][0][j] = wT[k + 2];
                X.part[(s + 2) & 1][1][j] = wR[k + 2];
                pair_sync(bar);
            }
        }
#pragma unroll
        for (int t = 0; t < WIN - UW; ++t) {
            wT[t] = wT[t + UW];
            wR[t] = wR[t + UW];
        }
#pragma unroll
        for (int t = WIN - UW; t < WIN; ++t) {
            const int r = s0 + UW + t - j;
            const bool ok = (r >= 0) && (r < LB);
            const int rr = ok ? r : 0;
            wT[t] = ok ? B.T[rr * LB + j] : 0.f;
            wR[t] = ok ? B.R[rr * LB + j] : 0.f;
        }
    }
}

}  // namespace leaf
}  // namespace bakron
