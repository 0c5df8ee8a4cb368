// internal.cu -- test hooks (see include/bakron_internal.h).
#include "bakron_internal.h"
#include "tcgemm_host.cuh"

using namespace bakron;

namespace {
constexpr int BN = 128;
constexpr int STAGES = 3;
}

extern "C" size_t bakron_internal_gemm3x_workspace_bytes(int M, int N, int K) {
    if (M < 1 || N < 1 || K < 0) return 0;
    const int ldk = tc::plane_ld(K > 0 ? K : 1);
    WsSizer z;
    z.take<float>((size_t)M * ldk); z.take<float>((size_t)M * ldk);
    z.take<float>((size_t)N * ldk); z.take<float>((size_t)N * ldk);
    return z.bytes();
}

extern "C" int bakron_internal_gemm3x(const float* A, int M, int K, int lda, const float* B,
                                      int N, int ldb, float* C, int ldc, void* ws,
                                      size_t ws_bytes, int* dev_status, void* stream) {
    if (M < 1 || N < 1 || K < 0 || !A || !B || !C || !dev_status) return BAKRON_ERR_INVALID_ARG;
    if (!ws_ok(ws, ws_bytes, bakron_internal_gemm3x_workspace_bytes(M, N, K)))
        return BAKRON_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int ldk = tc::plane_ld(K > 0 ? K : 1);
    WsCarver c(ws);
    float* ah = c.take<float>((size_t)M * ldk);
    float* al = c.take<float>((size_t)M * ldk);
    float* bh = c.take<float>((size_t)N * ldk);
    float* bl = c.take<float>((size_t)N * ldk);
    if (K > 0) {
        tc::split_planes(A, M, K, lda, ah, al, ldk, 0, st);
        tc::split_planes(B, N, K, ldb, bh, bl, ldk, 0, st);
    }
    const int kc = K > 0 ? K : 1;
    CUtensorMap mah, mal, mbh, mbl;
    int e;
    if ((e = tc::make_kmajor_map(&mah, ah, M, kc, ldk, tc::BM))) return e;
    if ((e = tc::make_kmajor_map(&mal, al, M, kc, ldk, tc::BM))) return e;
    if ((e = tc::make_kmajor_map(&mbh, bh, N, kc, ldk, BN))) return e;
    if ((e = tc::make_kmajor_map(&mbl, bl, N, kc, ldk, BN))) return e;
    tc::ProblemList L(BN);
    L.add(0, 0, 0, 0, M, N, K, 0, 0);
    tc::EpiStore epi{C, ldc, 0, 0};
    return tc::launch_gemm3x<BN, STAGES>(mah, mal, mbh, mbl, L, epi, dev_status, st);
}
