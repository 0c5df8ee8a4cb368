// tcgemm_host.cuh -- host-side helpers of the 3xTF32 GEMM engine: tensor maps, hi/lo plane
// splitting, epilogue functors and the launcher.
#pragma once

#include <cudaTypedefs.h>

#include "tcgemm.cuh"

namespace bakron {
namespace tc {

// Leading dimension of every hi/lo plane: a multiple of 32 fp32 (128 bytes), which satisfies
// the tensor-map stride rule (multiple of 16 bytes) and keeps rows on 128-byte boundaries.
inline int plane_ld(int cols) { return (cols + 31) / 32 * 32; }

// 2-D K-major fp32 tensor map: `rows` rows of `kcols` valid fp32 values, row stride `ld`
// elements (ld % 4 == 0, base 16-byte aligned), box of 32 x box_rows, 128-byte swizzle,
// out-of-range elements read as zero.
int make_kmajor_map(CUtensorMap* map, const float* base, int rows, int kcols, int ld,
                    int box_rows);

// 2-D fp32 tensor map of a row-major matrix (rows x cols, row stride ld elements, ld % 4 == 0,
// base 16-byte aligned) with a box x box box, out-of-range elements read as zero. Without
// swizzle the box lands as a dense row-major tile; with swizzle128 (box = 32: 128-byte rows)
// the 16-byte chunk c of row r lands at chunk c ^ (r % 8), and the destination must be
// 1024-byte aligned.
int make_box_map(CUtensorMap* map, const float* base, int rows, int cols, int ld, int box,
                 bool swizzle128 = false);

// Splits an fp32 matrix (rows x cols, row stride ld_src) into hi/lo planes (row stride
// ld_dst). transpose = 1 writes the planes of the transposed matrix (cols x rows).
void split_planes(const float* src, int rows, int cols, int ld_src, float* hi, float* lo,
                  int ld_dst, int transpose, cudaStream_t st);

// ---------------------------------------------------------------------------- epilogues
// An epilogue functor's chunk() is called once per 32 x 32 accumulator chunk of a warp:
// row0 is the chunk's first row, col = this lane's column (both relative to the problem
// origin), element rr of the lane's column is v[rr * 33]; m0, n0 give the tile origin.
// Global loads of a chunk are all issued before its stores (32 in flight per thread).
// tile_done(P, tile, quarter) runs after a tile's chunks, once per epilogue warp (all lanes);
// quarter (0..3) says which 32 rows of the tile the warp held.

// out = weight * acc, written as hi/lo planes at (c_row0 + r, c_col0 + c).
struct EpiStoreSplit {
    float* hi;
    float* lo;
    int ld;
    __device__ void chunk(const Problem& P, int row0, int col, int, int, const float* v) {
        if (col >= P.N) return;
#pragma unroll
        for (int rr = 0; rr < 32; ++rr) {
            if (row0 + rr < P.M) {
                const size_t o = (size_t)(P.c_row0 + row0 + rr) * ld + P.c_col0 + col;
                const float x = P.weight * v[rr * 33];
                const float h = sm100::tf32_hi(x);
                hi[o] = h;
                lo[o] = x - h;
            }
        }
    }
    __device__ void tile_done(const Problem&, int, int) {}
};

// C (+)= weight * acc at (c_row0 + r, c_col0 + c); `accumulate` selects += over =; with
// `upper` set only entries whose global column >= global row are touched.
struct EpiStore {
    float* C;
    int ldc;
    int accumulate;
    int upper;
    __device__ void chunk(const Problem& P, int row0, int col, int, int, const float* v) {
        if (col >= P.N) return;
        const int gc = P.c_col0 + col;
        float old[32];
#pragma unroll
        for (int rr = 0; rr < 32; ++rr) {
            const int gr = P.c_row0 + row0 + rr;
            const bool ok = (row0 + rr < P.M) && (!upper || gc >= gr);
            old[rr] = (ok && accumulate) ? C[(size_t)gr * ldc + gc] : 0.f;
        }
#pragma unroll
        for (int rr = 0; rr < 32; ++rr) {
            const int gr = P.c_row0 + row0 + rr;
            const bool ok = (row0 + rr < P.M) && (!upper || gc >= gr);
            if (ok) C[(size_t)gr * ldc + gc] = old[rr] + P.weight * v[rr * 33];
        }
    }
    __device__ void tile_done(const Problem&, int, int) {}
};

// partial[4 tile + quarter] = w * sum over the warp's 32 rows of the tile of acc[r][c] G[r][c]
// in fp64, w = 1 on diagonal tiles (m0 == n0) and `offdiag_weight` elsewhere (symmetric
// products computed on one triangle). The partials are summed in a fixed order afterwards.
struct EpiDot {
    const float* G;
    int ldg;
    double* partial;
    float offdiag_weight;
    double acc;
    __device__ void chunk(const Problem& P, int row0, int col, int m0, int n0, const float* v) {
        if (col >= P.N) return;
        float g[32];
#pragma unroll
        for (int rr = 0; rr < 32; ++rr)
            g[rr] = (row0 + rr < P.M) ? G[(size_t)(row0 + rr) * ldg + col] : 0.f;
        double s = 0.0;
#pragma unroll
        for (int rr = 0; rr < 32; ++rr) s += (double)v[rr * 33] * (double)g[rr];
        acc += (m0 == n0) ? s : (double)offdiag_weight * s;
    }
    __device__ void tile_done(const Problem&, int tile, int quarter) {
        double s = acc;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_down_sync(0xffffffffu, s, o);
        if ((threadIdx.x & 31) == 0) partial[(size_t)tile * 4 + quarter] = s;
        acc = 0.0;
    }
};

// ---------------------------------------------------------------------------- problems
struct ProblemList {
    Problems P{};
    int BN;
    explicit ProblemList(int bn) : BN(bn) { P.count = 0; P.total_tiles = 0; }
    // returns false when the list is full
    bool add(int a_row0, int a_k0, int b_row0, int b_k0, int M, int N, int K, int c_row0,
             int c_col0, float weight = 1.f, int upper_only = 0) {
        if (M <= 0 || N <= 0) return true;
        if (P.count == kMaxProblems) return false;
        Problem& p = P.p[P.count++];
        p.a_row0 = a_row0; p.a_k0 = a_k0; p.b_row0 = b_row0; p.b_k0 = b_k0;
        p.M = M; p.N = N; p.K = K; p.c_row0 = c_row0; p.c_col0 = c_col0;
        p.tiles_n = (N + BN - 1) / BN;
        const int tiles_m = (M + BM - 1) / BM;
        p.upper_only = upper_only;
        p.tiles = upper_only ? p.tiles_n * (p.tiles_n + 1) / 2 : tiles_m * p.tiles_n;
        p.tile_begin = P.total_tiles;
        p.weight = weight;
        P.total_tiles += p.tiles;
        return true;
    }
    bool empty() const { return P.total_tiles == 0; }
};

// Number of SMs of the current device (cached per device).
int sm_count();

// Launches the grouped GEMM with min(tiles, max_ctas) persistent CTAs (max_ctas <= 0: one per
// SM). A smaller max_ctas leaves SMs free for work on other streams. CHUNK > 0 restarts the
// accumulator every CHUNK k-blocks and sums the partials in round-to-nearest fp32.
template <int BN, int STAGES, int CHUNK = 0, class Epi>
int launch_gemm3x(const CUtensorMap& ah, const CUtensorMap& al, const CUtensorMap& bh,
                  const CUtensorMap& bl, const ProblemList& L, const Epi& epi, int* status,
                  cudaStream_t st, int max_ctas = 0) {
    if (L.empty()) return BAKRON_OK;
    // A TMA tile load must start on a 16-byte boundary: every K origin a multiple of 4 fp32.
    for (int i = 0; i < L.P.count; ++i)
        if ((L.P.p[i].a_k0 & 3) || (L.P.p[i].b_k0 & 3)) return BAKRON_ERR_INVALID_ARG;
    constexpr size_t smem = gemm_smem_bytes<BN, STAGES>();
    static_assert(smem <= 227 * 1024, "GEMM shared memory above the per-CTA limit");
    auto kern = gemm3x_kernel<BN, STAGES, Epi, CHUNK>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
        return BAKRON_ERR_CUDA;
    const int nsm = sm_count();
    if (nsm <= 0) return BAKRON_ERR_CUDA;
    int grid = (max_ctas > 0 && max_ctas < nsm) ? max_ctas : nsm;
    if (grid > L.P.total_tiles) grid = L.P.total_tiles;
    kern<<<grid, kThreads, smem, st>>>(ah, al, bh, bl, L.P, epi, status, spin_limit_ns());
    count_launches(1);
    return cuda_err(cudaGetLastError());
}

}  // namespace tc
}  // namespace bakron
