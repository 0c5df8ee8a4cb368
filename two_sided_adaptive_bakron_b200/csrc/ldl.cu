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
//   H'_BB = U_BB D_B U_BB^T                  one CTA per 128-index block (fp64 register
//                                             tiles, ldl_diag.cuh), which also forms U_BB^{-1};
//   X     = H'_AB U_BB^{-T},  U_AB = X D_B^{-1} 3xTF32 tensor-core GEMM (K = 128) whose
//                                             epilogue writes U_AB into L and the hi/lo planes
//                                             of X and U_AB;
//   H'_AA -= X U_AB^T                        split in two: columns inside the current 512-index
//                                             outer block right away (K = 128), the rest once
//                                             per outer block (K = 512, upper block triangle),
//                                             so the trailing matrix is streamed n/512 times.
// Look-ahead (n > kLookaheadMin): the diagonal blocks form a chain of single-CTA kernels that
// would leave the GPU mostly idle, so each outer block's trailing update is split and moved to
// a side stream. There, (a) the next outer block's 512 columns are updated first, on the whole
// GPU, and the caller's stream waits only for that before it goes on with the next block's
// diagonal chain; (b) the rest of the trailing matrix follows on all but kReserveSms SMs, which
// stay free for that chain. The side stream runs (a) of outer block o - 1 after (b) of o, the
// only other update of those columns. The panel planes alternate between two sets, so (b) can
// still read outer block o's planes while o - 1's panels are written.
// Inside an outer block, likewise, the caller's stream applies a panel only to the next
// diagonal block before factoring it; a second side stream applies the same panel to the next
// panel's input columns (which the caller's stream waits for before that panel; this update
// also writes that panel's hi/lo operand planes, so the panel needs no split pass) and then to
// the later columns of the outer block (waited for before the diagonal block after next).
#include <algorithm>
#include <atomic>
#include <mutex>

#include "ldl_diag.cuh"
#include "tcgemm_host.cuh"

namespace bakron {
namespace {

constexpr int NBI = 128;   // inner block: diagonal factorisation in one CTA
static_assert(NBI == ldl_diag::NB, "diagonal kernel block width");
constexpr int NBO = 512;   // outer block: K of the trailing update
constexpr int BN = 128;
constexpr int BNP = 64;    // panel tiles 128 x 64: twice the CTAs on the chain's critical path
constexpr int STAGES = 3;

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

// Panel epilogue: x = (H'_AB U_BB^{-T})[i][c]; U_AB = x (1 / D_c) goes to L; x and U_AB also go
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
        const float rdc = 1.0f / D[kb0 + c];
#pragma unroll 8
        for (int rr = 0; rr < 32; ++rr) {
            const int row = row0 + rr;
            if (row >= P.M) break;
            const float x = v[rr * 33];
            const float u = x * rdc;
            L[(size_t)row * n + kb0 + c] = u;
            const size_t o = (size_t)row * ldx + c_off + c;
            const float xh_ = sm100::tf32_hi(x), uh_ = sm100::tf32_hi(u);
            xh[o] = xh_;
            xl[o] = x - xh_;
            uh[o] = uh_;
            ul[o] = u - uh_;
        }
    }
    __device__ void tile_done(const tc::Problem&, int, int) {}
};

// C += weight * acc (as tc::EpiStore with accumulation; `upper`: only entries with global
// column >= global row), and every result at global (row, col) with row < pcol0 <= col also as
// hi/lo planes at (row, col - pcol0), row stride ldp: the update of the next panel's input
// columns leaves that panel's operand planes behind, so the panel needs no separate split pass
// on the chain.
struct EpiStorePlanes {
    float* C;
    int ldc;
    int upper;
    float* hi;
    float* lo;
    int ldp;
    int pcol0;
    __device__ void chunk(const tc::Problem& P, int row0, int col, int, int, const float* v) {
        if (col >= P.N) return;
        const int gc = P.c_col0 + col;
        float old[32];
#pragma unroll
        for (int rr = 0; rr < 32; ++rr) {
            const int gr = P.c_row0 + row0 + rr;
            const bool ok = (row0 + rr < P.M) && (!upper || gc >= gr);
            old[rr] = ok ? C[(size_t)gr * ldc + gc] : 0.f;
        }
#pragma unroll
        for (int rr = 0; rr < 32; ++rr) {
            const int gr = P.c_row0 + row0 + rr;
            if ((row0 + rr < P.M) && (!upper || gc >= gr)) {
                const float x = old[rr] + P.weight * v[rr * 33];
                C[(size_t)gr * ldc + gc] = x;
                if (gr < pcol0 && gc >= pcol0) {
                    const size_t o = (size_t)gr * ldp + (gc - pcol0);
                    const float h = sm100::tf32_hi(x);
                    hi[o] = h;
                    lo[o] = x - h;
                }
            }
        }
    }
    __device__ void tile_done(const tc::Problem&, int, int) {}
};

// Above this size the factorisation runs with look-ahead (two plane sets, a side stream);
// at or below it, sequentially on the caller's stream with one plane set.
constexpr int kLookaheadMin = 2048;
constexpr int kReserveSms = 24;   // SMs the bulk update leaves to the diagonal chain

inline int plane_sets(int n) { return n > kLookaheadMin ? 2 : 1; }

struct Planes {
    float *x_hi, *x_lo, *u_hi, *u_lo;   // X and U_AB of an outer block (n x NBO each)
};

struct LdlWs {
    float *inv_hi, *inv_lo, *p_hi, *p_lo;
    Planes set[2];
};

template <class F>
void ldl_ws_layout(int n, F&& take) {
    take((size_t)NBI * NBI);        // inv_hi
    take((size_t)NBI * NBI);        // inv_lo
    take((size_t)n * NBI);          // p_hi  (panel of H')
    take((size_t)n * NBI);          // p_lo
    for (int k = 0; k < plane_sets(n); ++k) {
        take((size_t)n * NBO);      // x_hi  (X of the outer block)
        take((size_t)n * NBO);      // x_lo
        take((size_t)n * NBO);      // u_hi  (U_AB of the outer block)
        take((size_t)n * NBO);      // u_lo
    }
}

// Side streams for the look-ahead, created once per device and never destroyed (a small pool,
// taken round robin, so that factorisations enqueued at the same time on different streams do
// not all share one side stream).
constexpr int kSidePool = 4;
constexpr int kMaxDevices = 64;
std::mutex g_side_mu;
cudaStream_t g_side[kMaxDevices][kSidePool] = {};
std::atomic<unsigned> g_side_next{0};

// Two distinct side streams of the current device's pool.
int side_streams(cudaStream_t* a, cudaStream_t* b) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return BAKRON_ERR_CUDA;
    const unsigned k = g_side_next.fetch_add(2, std::memory_order_relaxed) % kSidePool;
    std::lock_guard<std::mutex> lock(g_side_mu);
    cudaStream_t* out[2] = {a, b};
    for (unsigned i = 0; i < 2; ++i) {
        cudaStream_t& s = g_side[dev][(k + i) % kSidePool];
        if (!s && cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking) != cudaSuccess) {
            s = nullptr;
            return BAKRON_ERR_CUDA;
        }
        *out[i] = s;
    }
    return BAKRON_OK;
}

// Events of one call, released when the call has enqueued everything (their pending waits
// still complete).
struct CallEvents {
    static constexpr int kCount = 6;
    cudaEvent_t ev[kCount] = {};
    int n = 0;
    ~CallEvents() {
        for (int i = 0; i < n; ++i) cudaEventDestroy(ev[i]);
    }
    int make() {
        for (n = 0; n < kCount; ++n)
            if (cudaEventCreateWithFlags(&ev[n], cudaEventDisableTiming) != cudaSuccess)
                return BAKRON_ERR_CUDA;
        return BAKRON_OK;
    }
};

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
    float* bufs[12];
    int bi = 0;
    ldl_ws_layout(n, [&](size_t k) { bufs[bi++] = c.take<float>(k); });
    const int nsets = plane_sets(n);
    LdlWs w{bufs[0], bufs[1], bufs[2], bufs[3], {}};
    for (int k = 0; k < nsets; ++k)
        w.set[k] = Planes{bufs[4 + 4 * k], bufs[5 + 4 * k], bufs[6 + 4 * k], bufs[7 + 4 * k]};

    if (cudaFuncSetAttribute(ldl_diag::diag_block_kernel,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)ldl_diag::kSmemBytes) != cudaSuccess)
        return BAKRON_ERR_CUDA;
    int e;
    // Tensor maps over the outer-block planes (fixed for the whole call).
    CUtensorMap m_xh[2], m_xl[2], m_uh[2], m_ul[2];
    for (int k = 0; k < nsets; ++k) {
        if ((e = tc::make_kmajor_map(&m_xh[k], w.set[k].x_hi, n, NBO, NBO, tc::BM))) return e;
        if ((e = tc::make_kmajor_map(&m_xl[k], w.set[k].x_lo, n, NBO, NBO, tc::BM))) return e;
        if ((e = tc::make_kmajor_map(&m_uh[k], w.set[k].u_hi, n, NBO, NBO, BN))) return e;
        if ((e = tc::make_kmajor_map(&m_ul[k], w.set[k].u_lo, n, NBO, NBO, BN))) return e;
    }
    // look-ahead: two side streams and the call's events (ready: an outer block's panels are
    // written; next: the next outer block's columns are updated; join: the side stream's end;
    // panel: a panel is written; npanel: the next panel's input columns are updated; rest:
    // the later columns of the outer block are updated)
    const bool ahead = nsets == 2;
    cudaStream_t side = nullptr, s3 = nullptr;
    CallEvents evs;
    if (ahead) {
        if ((e = side_streams(&side, &s3))) return e;
        if ((e = evs.make())) return e;
    }
    cudaEvent_t ev_ready = evs.ev[0], ev_next = evs.ev[1], ev_join = evs.ev[2];
    cudaEvent_t ev_panel = evs.ev[3], ev_npanel = evs.ev[4], ev_rest = evs.ev[5];
    bool npanel_pending = false, rest_pending = false;
    bool first_planes = false;   // the look-ahead update left the next first panel's planes

    const int eb = 1184;
    copy_upper_kernel<<<eb, 256, 0, st>>>(H, L, n);
    count_launches(1);
    for (int ko1 = n, o = 0; ko1 > 0; ko1 -= NBO, ++o) {
        const int ko0 = std::max(0, ko1 - NBO);
        const int ps = ahead ? (o & 1) : 0;      // this outer block's plane set
        const Planes& pw = w.set[ps];
        for (int t = 0, kb1 = ko1; kb1 > ko0; ++t, kb1 -= NBI) {
            // plane columns of this inner block, counted from the end of the outer block so
            // that they stay 128-aligned even when the outer block is a partial one
            const int kb0 = std::max(ko0, kb1 - NBI), b = kb1 - kb0, c_off = NBO - NBI * (t + 1);
            ldl_diag::diag_block_kernel<<<1, ldl_diag::THREADS, ldl_diag::kSmemBytes, st>>>(L, n, kb0, b, D, w.inv_hi,
                                                                  w.inv_lo, dev_status);
            count_launches(1);
            if (kb0 == 0) continue;
            // panel: X = H'[0:kb0, B] U_BB^{-T}; with look-ahead its operand planes come from
            // the last update of these columns (the previous panel's, or for an outer block's
            // first panel the previous outer block's look-ahead update), else from a split here
            if (npanel_pending) {
                if ((e = cuda_err(cudaStreamWaitEvent(st, ev_npanel, 0)))) return e;
                npanel_pending = false;
            } else if (!(first_planes && t == 0)) {
                tc::split_planes(L + kb0, kb0, b, n, w.p_hi, w.p_lo, NBI, 0, st);
            }
            first_planes = false;
            CUtensorMap m_ph, m_pl, m_ih, m_il;
            if ((e = tc::make_kmajor_map(&m_ph, w.p_hi, kb0, b, NBI, tc::BM))) return e;
            if ((e = tc::make_kmajor_map(&m_pl, w.p_lo, kb0, b, NBI, tc::BM))) return e;
            if ((e = tc::make_kmajor_map(&m_ih, w.inv_hi, NBI, b, NBI, BNP))) return e;
            if ((e = tc::make_kmajor_map(&m_il, w.inv_lo, NBI, b, NBI, BNP))) return e;
            tc::ProblemList pl(BNP);
            pl.add(0, 0, 0, 0, kb0, b, b, 0, 0);
            EpiPanel ep{L, n, D, kb0, pw.x_hi, pw.x_lo, pw.u_hi, pw.u_lo, NBO, c_off};
            if ((e = tc::launch_gemm3x<BNP, STAGES>(m_ph, m_pl, m_ih, m_il, pl, ep, dev_status, st)))
                return e;
            // columns of the outer block still pending: H'[0:kb0, ko0:kb0] -= X U_AB^T
            if (kb0 > ko0) {
                tc::EpiStore es{L, n, 1, 1};
                if (!ahead) {
                    tc::ProblemList wl(BN);
                    wl.add(0, c_off, ko0, c_off, kb0, kb0 - ko0, b, 0, ko0, -1.f);
                    if ((e = tc::launch_gemm3x<BN, STAGES>(m_xh[ps], m_xl[ps], m_uh[ps],
                                                           m_ul[ps], wl, es, dev_status, st)))
                        return e;
                    continue;
                }
                // the next inner block [nb0, kb0): its input columns above it and the later
                // columns [ko0, nb0) on the second side stream, its diagonal block here
                const int nb0 = std::max(ko0, kb0 - NBI);
                if ((e = cuda_err(cudaEventRecord(ev_panel, st)))) return e;
                if ((e = cuda_err(cudaStreamWaitEvent(s3, ev_panel, 0)))) return e;
                tc::ProblemList nl(BN);
                nl.add(0, c_off, nb0, c_off, nb0, kb0 - nb0, b, 0, nb0, -1.f);
                EpiStorePlanes ep_next{L, n, 1, w.p_hi, w.p_lo, NBI, nb0};
                if ((e = tc::launch_gemm3x<BN, STAGES>(m_xh[ps], m_xl[ps], m_uh[ps], m_ul[ps], nl,
                                                       ep_next, dev_status, s3)))
                    return e;
                if ((e = cuda_err(cudaEventRecord(ev_npanel, s3)))) return e;
                npanel_pending = true;
                if (nb0 > ko0) {
                    tc::ProblemList rl(BN);
                    rl.add(0, c_off, ko0, c_off, nb0, nb0 - ko0, b, 0, ko0, -1.f);
                    if ((e = tc::launch_gemm3x<BN, STAGES>(m_xh[ps], m_xl[ps], m_uh[ps],
                                                           m_ul[ps], rl, es, dev_status, s3)))
                        return e;
                }
                // the previous panel's later columns hold the next diagonal block: they go first
                if (rest_pending && (e = cuda_err(cudaStreamWaitEvent(st, ev_rest, 0)))) return e;
                if ((e = cuda_err(cudaEventRecord(ev_rest, s3)))) return e;
                rest_pending = true;
                tc::ProblemList tl(BN);
                tl.add(nb0, c_off, nb0, c_off, kb0 - nb0, kb0 - nb0, b, nb0, nb0, -1.f,
                       /*upper_only=*/1);
                if ((e = tc::launch_gemm3x<BN, STAGES>(m_xh[ps], m_xl[ps], m_uh[ps], m_ul[ps], tl,
                                                       es, dev_status, st)))
                    return e;
            }
        }
        if (rest_pending) {   // everything the second side stream did for this outer block
            if ((e = cuda_err(cudaStreamWaitEvent(st, ev_rest, 0)))) return e;
            rest_pending = npanel_pending = false;
        }
        if (ko0 == 0) continue;
        // the rest of the trailing matrix, once per outer block: upper block triangle of
        // [0, ko0)^2, K = this outer block's columns
        const int K = ko1 - ko0;
        tc::EpiStore es{L, n, 1, 1};
        if (!ahead) {
            tc::ProblemList tl(BN);
            tl.add(0, 0, 0, 0, ko0, ko0, K, 0, 0, -1.f, /*upper_only=*/1);
            if ((e = tc::launch_gemm3x<BN, STAGES>(m_xh[0], m_xl[0], m_uh[0], m_ul[0], tl, es,
                                                   dev_status, st)))
                return e;
            continue;
        }
        // look-ahead, on the side stream once this outer block's panels are written: (a) the
        // columns [ca, ko0) of the next outer block (after (b) of the previous outer block,
        // which updated them too and read the plane set the next panels overwrite), then (b)
        // the bulk [0, ca)^2
        const int ca = std::max(0, ko0 - NBO);
        if ((e = cuda_err(cudaEventRecord(ev_ready, st)))) return e;
        if ((e = cuda_err(cudaStreamWaitEvent(side, ev_ready, 0)))) return e;
        tc::ProblemList al(BN);
        al.add(0, 0, ca, 0, ca, ko0 - ca, K, 0, ca, -1.f);                      // rows above
        al.add(ca, 0, ca, 0, ko0 - ca, ko0 - ca, K, ca, ca, -1.f, /*upper_only=*/1);
        // it also leaves the operand planes of the next outer block's first panel (columns
        // [fb0, ko0), rows above them)
        const int fb0 = std::max(ca, ko0 - NBI);
        EpiStorePlanes ep_first{L, n, 1, w.p_hi, w.p_lo, NBI, fb0};
        if ((e = tc::launch_gemm3x<BN, STAGES>(m_xh[ps], m_xl[ps], m_uh[ps], m_ul[ps], al,
                                               ep_first, dev_status, side)))
            return e;
        first_planes = true;
        if ((e = cuda_err(cudaEventRecord(ev_next, side)))) return e;
        if (ca > 0) {
            tc::ProblemList bl(BN);
            bl.add(0, 0, 0, 0, ca, ca, K, 0, 0, -1.f, /*upper_only=*/1);
            if ((e = tc::launch_gemm3x<BN, STAGES>(m_xh[ps], m_xl[ps], m_uh[ps], m_ul[ps], bl, es,
                                                   dev_status, side,
                                                   std::max(1, tc::sm_count() - kReserveSms))))
                return e;
        }
        if ((e = cuda_err(cudaStreamWaitEvent(st, ev_next, 0)))) return e;
    }
    if (ahead) {   // the side stream's last work joins the caller's stream
        if ((e = cuda_err(cudaEventRecord(ev_join, side)))) return e;
        if ((e = cuda_err(cudaStreamWaitEvent(st, ev_join, 0)))) return e;
    }
    clear_lower_kernel<<<eb, 256, 0, st>>>(L, n);
    count_launches(1);
    return cuda_err(cudaGetLastError());
}
