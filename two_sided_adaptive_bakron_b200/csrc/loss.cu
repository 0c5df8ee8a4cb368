// loss.cu -- bakron_proxy_loss: tr(H_O dW H_I dW^T) = vec(dW)^T (H_O (x) H_I) vec(dW).
//
// YAQA article (news.43b.com.cn/a/479517.html), section 4: the layer proxy error
// dW (H_O (x) H_I) dW^T that the section bounds by tr(D_I) tr(D_O) sigma^2; section 2: the
// second-order objective (its factor 1/2 is not applied here).
//
// With X (p x q) oriented so that p <= q (X = dW, Ha = H_O, Hb = H_I when m <= n, otherwise
// X = dW^T, Ha = H_I, Hb = H_O; the trace is the same):
//   V = X^T Ha                       (q x p, K = p; 3xTF32 tensor-core GEMM, stored as planes)
//   Z = V' X = X^T Ha X              (q x q, K = p; only the upper block triangle is formed,
//                                     Z being symmetric)
//   loss = sum_{j,l} Hb[j][l] Z[j][l] (fused into the second GEMM's epilogue, fp64 per tile,
//                                     off-diagonal tiles counted twice, tiles summed in a
//                                     fixed order)
// Work 2 p^2 q + p q^2 flops (the minimum of the two orientations).
#include <algorithm>

#include "tcgemm_host.cuh"

namespace bakron {
namespace {

constexpr int BN = 128;       // square tiles (BM == BN) for the symmetric block triangle
constexpr int STAGES = 3;

// Sums the per-tile partials in a fixed order; a failed engine run yields NaN.
__global__ void final_sum_kernel(const double* __restrict__ partial, size_t count,
                                 const int* __restrict__ status, double* __restrict__ loss) {
    __shared__ double red[1024];
    double s = 0.0;
    for (size_t e = threadIdx.x; e < count; e += blockDim.x) s += partial[e];
    red[threadIdx.x] = s;
    __syncthreads();
    for (int w = blockDim.x / 2; w > 0; w >>= 1) {
        if ((int)threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x == 0) *loss = (*status == BAKRON_OK) ? red[0] : __longlong_as_double(-1LL);
}

struct LossLayout {
    int p, q, ldp;
    size_t xt, ha, v, tiles2;
};

LossLayout loss_layout(int m, int n) {
    LossLayout L;
    L.p = std::min(m, n);
    L.q = std::max(m, n);
    L.ldp = tc::plane_ld(L.p);
    L.xt = (size_t)L.q * L.ldp;
    L.ha = (size_t)L.p * L.ldp;
    L.v = (size_t)L.q * L.ldp;
    const size_t t = (L.q + BN - 1) / BN;
    L.tiles2 = t * (t + 1) / 2;   // upper block triangle of Z
    return L;
}

}  // namespace
}  // namespace bakron

using namespace bakron;

extern "C" size_t bakron_proxy_loss_workspace_bytes(int m, int n) {
    if (m < 1 || n < 1) return 0;
    const LossLayout L = loss_layout(m, n);
    WsSizer z;
    z.take<float>(L.xt); z.take<float>(L.xt);
    z.take<float>(L.ha); z.take<float>(L.ha);
    z.take<float>(L.v);  z.take<float>(L.v);
    z.take<double>(4 * L.tiles2);   // one partial per tile and epilogue warp
    z.take<int>(64);
    return z.bytes();
}

extern "C" int bakron_proxy_loss(const float* dW, int m, int n, const float* H_O,
                                 const float* H_I, double* loss, void* ws, size_t ws_bytes,
                                 void* stream) {
    if (m < 1 || n < 1 || !dW || !H_O || !H_I || !loss) return BAKRON_ERR_INVALID_ARG;
    if (!ws_ok(ws, ws_bytes, bakron_proxy_loss_workspace_bytes(m, n))) return BAKRON_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const LossLayout L = loss_layout(m, n);
    WsCarver c(ws);
    float* xt_hi = c.take<float>(L.xt);
    float* xt_lo = c.take<float>(L.xt);
    float* ha_hi = c.take<float>(L.ha);
    float* ha_lo = c.take<float>(L.ha);
    float* v_hi = c.take<float>(L.v);
    float* v_lo = c.take<float>(L.v);
    double* partial = c.take<double>(4 * L.tiles2);
    int* status = c.take<int>(64);   // engine timeouts (never expected) land here
    int e;
    if ((e = cuda_err(cudaMemsetAsync(status, 0, sizeof(int), st)))) return e;

    const bool dw_is_x = (m <= n);   // X = dW (p = m) or X = dW^T (p = n)
    const float* Ha = dw_is_x ? H_O : H_I;
    const float* Hb = dw_is_x ? H_I : H_O;
    const int p = L.p, q = L.q, ldp = L.ldp;
    // X^T (q x p): dW^T when X = dW, dW itself when X = dW^T
    tc::split_planes(dW, m, n, n, xt_hi, xt_lo, ldp, dw_is_x ? 1 : 0, st);
    tc::split_planes(Ha, p, p, p, ha_hi, ha_lo, ldp, 0, st);

    CUtensorMap m_xth, m_xtl, m_hah, m_hal, m_vh, m_vl;
    if ((e = tc::make_kmajor_map(&m_xth, xt_hi, q, p, ldp, tc::BM))) return e;
    if ((e = tc::make_kmajor_map(&m_xtl, xt_lo, q, p, ldp, tc::BM))) return e;
    if ((e = tc::make_kmajor_map(&m_hah, ha_hi, p, p, ldp, BN))) return e;
    if ((e = tc::make_kmajor_map(&m_hal, ha_lo, p, p, ldp, BN))) return e;
    if ((e = tc::make_kmajor_map(&m_vh, v_hi, q, p, ldp, BN))) return e;
    if ((e = tc::make_kmajor_map(&m_vl, v_lo, q, p, ldp, BN))) return e;

    // V[j][i] = sum_k X^T[j][k] Ha[i][k]
    tc::ProblemList g1(BN);
    g1.add(0, 0, 0, 0, q, p, p, 0, 0);
    tc::EpiStoreSplit epi1{v_hi, v_lo, ldp};
    if ((e = tc::launch_gemm3x<BN, STAGES>(m_xth, m_xtl, m_hah, m_hal, g1, epi1, status, st)))
        return e;
    // Z[j][l] = sum_i X^T[j][i] V[l][i], upper block triangle, dotted with Hb
    tc::ProblemList g2(BN);
    g2.add(0, 0, 0, 0, q, q, p, 0, 0, 1.f, /*upper_only=*/1);
    tc::EpiDot epi2{Hb, q, partial, 2.f, 0.0};
    if ((e = tc::launch_gemm3x<BN, STAGES>(m_xth, m_xtl, m_vh, m_vl, g2, epi2, status, st)))
        return e;
    final_sum_kernel<<<1, 1024, 0, st>>>(partial, 4 * L.tiles2, status, loss);
    count_launches(1);
    return cuda_err(cudaGetLastError());
}
