// ldl_diag.cuh -- U D U^T of one diagonal block of the blocked LDL (fp64, register tiles),
// together with W = U^{-1}, which the panel step multiplies by.
//
// YAQA article, section 4: the factorisation H = (L + I) D (L + I)^T with L strictly upper.
// For one symmetric block A (upper triangle valid) the right-looking recurrence, last index
// first, is: d_k = A[k][k]; u_r = A[r][k] / d_k (r < k) is column k of U; the rows r <= c < k of
// the Schur complement lose u_r d_k u_c = u_r A[c][k].
//
// One matrix X holds both unknowns: at step k its columns < k are the Schur complement A (upper
// triangle) and its columns >= k are W's rows above the diagonal. W's row k is final at step k
// and W[r][c] -= U[r][k] W[k][c], so with v_c = A[c][k] (c < k), v_c = W[k][c] (c > k) a step
// is the single rank-1 update X[r][c] -= u_r v_c of the rows r < k (c != k), after which column k
// becomes W's column k: X[r][k] = -u_r. The lower triangle collects values that are never read.
//
// 512 threads; thread (warp w, lane 16 s + t) owns rows 8w + 4s + [0, 4) and columns 8t + [0, 8)
// of the 128 x 128 block. After step k + 1 the owners of column k, row k and pivot k write v, d_k
// and 1 / d_k into row k of a shared history, so a step costs one barrier; U and D are written
// out from that history at the end (u_r = v_r / d_k). Every thread forms the next pivot's
// candidate and its reciprocal right after its loads, so the reciprocal of the one thread whose
// candidate is the pivot is off the step's critical path. Rows that are done (>= k) drop out.
#pragma once

#include "sm100.cuh"

namespace bakron {
namespace ldl_diag {

constexpr int NB = 128;        // block width
constexpr int THREADS = 512;
constexpr int TR = 4, TC = 8;  // thread tile
constexpr int VS = NB + 2;     // history row stride (doubles): 16-byte rows, few bank conflicts
constexpr size_t kSmemBytes = ((size_t)NB * VS + 2 * NB) * sizeof(double);

// position of element c in a history row: pairs (8t + 2p, 8t + 2p + 1) at (16 p + t), so that a
// thread's 8 columns are 4 conflict-free double2 loads and its 4 rows are 2
__device__ __forceinline__ int vpos(int c) {
    return ((((c & 7) >> 1) << 4) + (c >> 3)) * 2 + (c & 1);
}

// 1 / d by two Newton-Raphson steps x <- x + x (1 - d x) from the correctly rounded
// single-precision reciprocal (relative error 2^-24 -> 2^-48 -> fp64 rounding); outside the
// single-precision normal range the division itself.
__device__ __forceinline__ double recip(double d) {
    const double a = fabs(d);
    if (!(a > 1e-36 && a < 1e36)) return 1.0 / d;
    double x = (double)__frcp_rn((float)d);
    double e = fma(-d, x, 1.0);
    x = fma(x, e, x);
    e = fma(-d, x, 1.0);
    return fma(x, e, x);
}

struct Ctx {
    int b;
    int* status;
    double (*vh)[VS];   // vh[k]: v of step k
    double* dh;         // pivots
    double* rdh;        // their reciprocals
    int warp, s, t, r0, c0;
    int orow;           // history offset of the thread's rows r0, r0 + 1 (r0 + 2, + 3 at +32)
    int ocol;           // history offset of its columns c0, c0 + 1 (pair p at +32 p)
};

__device__ __forceinline__ double checked_pivot(const Ctx& c, double d, int k) {
    const bool bad = !(d > 0.0) || !isfinite(d);
    if (bad && k < c.b) set_status(c.status, BAKRON_ERR_NOT_PD);
    return bad ? 1.0 : d;
}

// history offsets (see vpos) of tile row i and tile column q
__device__ __forceinline__ int rowpos(const Ctx& c, int i) { return c.orow + (i >> 1) * 32 + (i & 1); }
__device__ __forceinline__ int colpos(const Ctx& c, int q) { return c.ocol + (q >> 1) * 32 + (q & 1); }

// v of step kn (QN = kn & 7) from the owners' registers; the pivot's reciprocal comes in rd
template <int QN>
__device__ __forceinline__ void publish(const Ctx& c, const double (&X)[TR][TC], int kn, double d,
                                        double rd) {
    constexpr int IN = QN & 3;
    double* v = c.vh[kn];
    if (c.t == (kn >> 3)) {             // column kn, rows < kn
#pragma unroll
        for (int i = 0; i < TR; ++i)
            if (c.r0 + i < kn) v[rowpos(c, i)] = X[i][QN];
    }
    if (c.r0 == (kn & ~3)) {            // row kn, columns > kn; pivot kn
#pragma unroll
        for (int q = 0; q < TC; ++q)
            if (c.c0 + q > kn) v[colpos(c, q)] = X[IN][q];
        if (c.t == (kn >> 3)) {
            c.dh[kn] = d;
            c.rdh[kn] = rd;
        }
    }
}

// the update of step k for one warp. EDGE: the warp holding row k - 1, the only one whose rows
// straddle k; it also forms the next pivot (exactly as its update leaves it) and its reciprocal.
template <int Q, bool EDGE>
__device__ __forceinline__ void update(const Ctx& c, double (&X)[TR][TC], int k, double& dn,
                                       double& rn) {
    constexpr int QN = (Q + 7) & 7, IN = QN & 3;    // index k - 1 inside a tile
    const double* v = c.vh[k];
    const double rd = c.rdh[k];
    double u[TR], vc[TC];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const double2 a = *reinterpret_cast<const double2*>(&v[c.orow + 32 * h]);
        u[2 * h] = a.x;
        u[2 * h + 1] = a.y;
    }
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const double2 w = *reinterpret_cast<const double2*>(&v[c.ocol + 32 * p]);
        vc[2 * p] = w.x;
        vc[2 * p + 1] = w.y;
    }
#pragma unroll
    for (int i = 0; i < TR; ++i) u[i] = (!EDGE || c.r0 + i < k) ? u[i] * rd : 0.0;
    if (EDGE) {
        const bool piv = (c.r0 == ((k - 1) & ~3)) && (c.t == ((k - 1) >> 3));
        dn = checked_pivot(c, piv ? fma(-u[IN], vc[QN], X[IN][QN]) : 1.0, piv ? k - 1 : NB);
        rn = recip(dn);
    }
#pragma unroll
    for (int i = 0; i < TR; ++i)
#pragma unroll
        for (int q = 0; q < TC; ++q) X[i][q] = fma(-u[i], vc[q], X[i][q]);
    if (c.t == (k >> 3)) {              // column k becomes W's column k
#pragma unroll
        for (int i = 0; i < TR; ++i) X[i][Q] = -u[i];
    }
}

// step k (Q = k & 7, k >= 1), then the owners of index k - 1 publish
template <int Q>
__device__ __forceinline__ void step(const Ctx& c, double (&X)[TR][TC], int k) {
    __syncthreads();
    double dn = 1.0, rn = 1.0;
    const int edge = (k - 1) >> 3;      // warps below it have no rows < k left
    if (c.warp < edge) update<Q, false>(c, X, k, dn, rn);
    else if (c.warp == edge) update<Q, true>(c, X, k, dn, rn);
    publish<(Q + 7) & 7>(c, X, k - 1, dn, rn);
}

// L holds the block's upper triangle on entry (row stride n, block origin k0, size b <= 128,
// indices >= b padded with the identity); on exit its strict upper part holds U, D[k0 + .] the
// pivots and inv_hi / inv_lo (128 x 128, row stride 128) the tf32 hi/lo split of W = U^{-1}
// (zero outside the b x b block). A pivot that is not positive and finite sets
// BAKRON_ERR_NOT_PD and continues as 1. Dynamic shared memory: kSmemBytes.
__global__ void __launch_bounds__(THREADS) diag_block_kernel(float* __restrict__ L, int n, int k0,
                                                             int b, float* __restrict__ D,
                                                             float* __restrict__ inv_hi,
                                                             float* __restrict__ inv_lo,
                                                             int* status) {
    extern __shared__ __align__(16) double dsm[];
    double(*vh)[VS] = reinterpret_cast<double(*)[VS]>(dsm);
    double* dh = dsm + (size_t)NB * VS;
    double* rdh = dh + NB;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int s = lane >> 4, t = lane & 15;
    const int r0 = warp * 8 + s * 4, c0 = t * TC;
    const Ctx c{b, status, vh, dh, rdh, warp, s, t, r0, c0, ((2 * s) * 16 + warp) * 2, 2 * t};
    double X[TR][TC];
#pragma unroll
    for (int i = 0; i < TR; ++i)
#pragma unroll
        for (int q = 0; q < TC; ++q) {
            const int r = r0 + i, cc = c0 + q;
            double v = (r == cc) ? 1.0 : 0.0;
            if (r < b && cc < b) v = (cc >= r) ? (double)L[(size_t)(k0 + r) * n + k0 + cc] : 0.0;
            X[i][q] = v;
        }
    {
        const bool piv = (r0 == NB - 4) && (t == NB / TC - 1);
        const double d = checked_pivot(c, piv ? X[3][7] : 1.0, piv ? NB - 1 : NB);
        publish<7>(c, X, NB - 1, d, recip(d));
    }
#pragma unroll 1
    for (int kb = NB - 8; kb >= 8; kb -= 8) {
        step<7>(c, X, kb + 7);
        step<6>(c, X, kb + 6);
        step<5>(c, X, kb + 5);
        step<4>(c, X, kb + 4);
        step<3>(c, X, kb + 3);
        step<2>(c, X, kb + 2);
        step<1>(c, X, kb + 1);
        step<0>(c, X, kb);
    }
    step<7>(c, X, 7);
    step<6>(c, X, 6);
    step<5>(c, X, 5);
    step<4>(c, X, 4);
    step<3>(c, X, 3);
    step<2>(c, X, 2);
    step<1>(c, X, 1);
    // W = U^{-1}: strict upper part of X, unit diagonal, zero outside the b x b block
#pragma unroll
    for (int i = 0; i < TR; ++i) {
        const int r = r0 + i;
        float h[TC], l[TC];
#pragma unroll
        for (int q = 0; q < TC; ++q) {
            const int cc = c0 + q;
            const float x =
                (r < b && cc < b) ? (cc > r ? (float)X[i][q] : (cc == r ? 1.f : 0.f)) : 0.f;
            h[q] = sm100::tf32_hi(x);
            l[q] = x - h[q];
        }
        float4* ph = reinterpret_cast<float4*>(inv_hi + (size_t)r * NB + c0);
        float4* pl = reinterpret_cast<float4*>(inv_lo + (size_t)r * NB + c0);
        ph[0] = make_float4(h[0], h[1], h[2], h[3]);
        ph[1] = make_float4(h[4], h[5], h[6], h[7]);
        pl[0] = make_float4(l[0], l[1], l[2], l[3]);
        pl[1] = make_float4(l[4], l[5], l[6], l[7]);
    }
    __syncthreads();
    // U[r][k] = v_r / d_k (the u of step k) and the pivots, from the history
    for (int e = tid; e < b * b; e += THREADS) {
        const int r = e / b, k = e % b;
        if (k > r) L[(size_t)(k0 + r) * n + k0 + k] = (float)(vh[k][vpos(r)] * rdh[k]);
    }
    for (int k = tid; k < b; k += THREADS) D[k0 + k] = (float)dh[k];
}

}  // namespace ldl_diag
}  // namespace bakron
