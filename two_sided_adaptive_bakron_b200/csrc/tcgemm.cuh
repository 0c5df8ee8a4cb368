// tcgemm.cuh -- 3xTF32 tensor-core GEMM engine for sm_100a (tcgen05 + TMA + TMEM).
//
//   C_tile (BM x BN) = sum_k A[m][k] * B[n][k]        (both operands K-major, fp32 values)
//
// Each fp32 operand is stored as two planes, hi = x with its 13 low mantissa bits cleared
// (exact in tf32) and lo = x - hi (exact in fp32). The product is accumulated as
//   A_hi B_hi + A_hi B_lo + A_lo B_hi
// in fp32 TMEM accumulators, which keeps about 22 significant bits per product (the dropped
// A_lo B_lo term and the tf32 truncation of lo are both below 2^-21 relative).
//
// Persistent pipeline (at most one 192-thread CTA per SM, tiles t = blockIdx.x + i * gridDim.x):
//   warp 0 / lane 0 : TMA producer, STAGES-deep ring of {A_hi, A_lo, B_hi, B_lo} k-blocks of
//                     32 fp32 (one 128-byte swizzle row) that runs on across tiles;
//   warp 1 / lane 0 : MMA issuer, 4 k-steps of 8 x 3 tcgen05.mma per k-block into one of the
//                     TMEM accumulators (two of BN columns); tcgen05.commit frees the stage and,
//                     after a tile's last k-block, hands the accumulator to the epilogue;
//   warps 2 .. 5    : epilogue, tcgen05.ld of the accumulator (warp w reads TMEM lanes
//                     32 (w % 4) .. + 31 = tile rows), then the Epi functor, then the
//                     accumulator goes back to the MMA issuer, so a tile's epilogue overlaps
//                     the next tile's MMAs.
// Chunked accumulation (CHUNK > 0): the tensor core's fp32 accumulator does not round to
// nearest, so its error grows with the number of MMAs summed into it. With CHUNK > 0 the issuer
// restarts the accumulator every CHUNK k-blocks and hands each partial sum over like a tile;
// the epilogue adds the partials in registers (fp32, round to nearest, in k order) and runs the
// Epi functor once per tile on their sum. The accumulator then never holds more than
// 3 CHUNK BK / 8 instructions' worth of products, whatever K is. This mode takes four TMEM
// accumulators (4 x BN columns), so the issuer can fill up to three chunks while the epilogue
// is still writing out the previous tile.
// A launch may hold several problems (a grouped GEMM): the operand tensor maps cover whole
// planes and every problem only moves the tile origins.
// Every mbarrier wait is bounded and also gives up when another role has raised the CTA's
// abort word; on expiry the status word gets BAKRON_ERR_TIMEOUT, in-flight copies and MMAs are
// drained (with a bound) and the TMEM is released before returning.
#pragma once

#include "sm100.cuh"

namespace bakron {
namespace tc {

constexpr int BM = 128;
constexpr int BK = 32;
constexpr int kMaxProblems = 48;
constexpr int kThreads = 192;
constexpr int kEpiWarp0 = 2;       // first of the 4 epilogue warps

struct Problem {
    int a_row0, a_k0;   // origin of the A tile rows (M) and of K in the A planes
    int b_row0, b_k0;   // origin of the B tile rows (N) and of K in the B planes
    int M, N, K;        // problem extents
    int c_row0, c_col0; // origin of the output (handed to the epilogue)
    int tiles_n;        // ceil(N / BN)
    int tile_begin;     // first linear tile index of this problem in the launch
    int tiles;          // number of tiles of this problem in the launch
    int upper_only;     // 1: only tiles with tile_m <= tile_n (square tiles, BM == BN)
    float weight;       // epilogue scalar
};

struct Problems {
    Problem p[kMaxProblems];
    int count;
    int total_tiles;
};

template <int BN>
struct Cfg {
    static constexpr uint32_t kABytes = BM * BK * 4;          // one A plane k-block
    static constexpr uint32_t kBBytes = BN * BK * 4;          // one B plane k-block
    static constexpr uint32_t kStageBytes = 2 * kABytes + 2 * kBBytes;
    static constexpr uint32_t kTmemCols = 2 * BN;             // two accumulators
    static constexpr uint32_t kEpiBytes = 4 * 32 * 33 * 4;    // per-warp 32 x 33 staging
    static_assert(kTmemCols >= 32 && kTmemCols <= 512 && (kTmemCols & (kTmemCols - 1)) == 0,
                  "TMEM allocation must be a power of two in [32, 512]");
};

template <int BN, int STAGES>
constexpr size_t gemm_smem_bytes() {
    return 1024 /*alignment slack*/ + (size_t)STAGES * Cfg<BN>::kStageBytes + Cfg<BN>::kEpiBytes +
           256;
}

// Bounded wait that also gives up once *abort is set (by any role of the CTA).
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, int* status,
                                              uint64_t limit_ns, volatile int* abort) {
    if (sm100::mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (!sm100::mbar_try_wait(bar, parity)) {
        if (*abort) return false;
        if (globaltimer_ns() - t0 > limit_ns) {
            set_status(status, BAKRON_ERR_TIMEOUT);
            *abort = 1;
            return false;
        }
    }
    return true;
}

// Maps a linear tile index of the launch to (problem, m0, n0). Returns false if out of range.
__device__ __forceinline__ bool decode_tile(const Problems& P, int BNv, int t, int& pi, int& m0,
                                            int& n0) {
    for (int i = 0; i < P.count; ++i) {
        const Problem& p = P.p[i];
        if (t >= p.tile_begin && t < p.tile_begin + p.tiles) {
            int local = t - p.tile_begin;
            int tm, tn;
            if (p.upper_only) {
                // enumerate (tm, tn) with tm <= tn < tiles_n row by row
                tm = 0;
                int rowlen = p.tiles_n;
                while (local >= rowlen) { local -= rowlen; ++tm; --rowlen; }
                tn = tm + local;
            } else {
                tm = local / p.tiles_n;
                tn = local % p.tiles_n;
            }
            pi = i;
            m0 = tm * BM;
            n0 = tn * BNv;
            return true;
        }
    }
    return false;
}

// k-blocks per accumulator hand-off and hand-offs per tile (K = 0: one, of zeros)
template <int CHUNK>
__device__ __forceinline__ int chunk_len(int nkb) { return CHUNK > 0 ? CHUNK : (nkb > 0 ? nkb : 1); }
template <int CHUNK>
__device__ __forceinline__ int chunk_count(int nkb) {
    return nkb > 0 ? (nkb + chunk_len<CHUNK>(nkb) - 1) / chunk_len<CHUNK>(nkb) : 1;
}

template <int BN, int STAGES, class Epi, int CHUNK = 0>
__global__ void __launch_bounds__(kThreads, 1)
gemm3x_kernel(const __grid_constant__ CUtensorMap a_hi, const __grid_constant__ CUtensorMap a_lo,
              const __grid_constant__ CUtensorMap b_hi, const __grid_constant__ CUtensorMap b_lo,
              const __grid_constant__ Problems probs, const Epi epi, int* status,
              uint64_t limit_ns) {
    using C = Cfg<BN>;
    // accumulators in TMEM: two, or four for chunked accumulation, so that the epilogue may
    // still be writing a finished tile while the issuer fills the next tile's first chunks
    constexpr int NACC = (CHUNK > 0 && 4 * BN <= 512) ? 4 : 2;
    constexpr uint32_t kTmemCols = NACC * BN;
    static_assert((2 * STAGES + 2 * NACC + 1) * 8 + 8 <= 256, "barrier area");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float* epi_stage = reinterpret_cast<float*>(smem + STAGES * C::kStageBytes);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * C::kStageBytes + C::kEpiBytes);
    uint64_t* empty = full + STAGES;
    uint64_t* acc_full = empty + STAGES;   // [NACC] accumulator ready for the epilogue
    uint64_t* acc_empty = acc_full + NACC; // [NACC] accumulator read out (4 epilogue warps)
    uint64_t* drain = acc_empty + NACC;    // error path: all MMAs retired
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* s_abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int total = probs.total_tiles;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            sm100::mbar_init(&full[s], 1);
            sm100::mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < NACC; ++b) {
            sm100::mbar_init(&acc_full[b], 1);
            sm100::mbar_init(&acc_empty[b], 4);
        }
        sm100::mbar_init(drain, 1);
        *s_abort = 0;
        sm100::fence_mbar_init();
    }
    if (warp == 1) {
        sm100::tmem_alloc(tmem_slot, kTmemCols);
        sm100::tmem_relinquish();
    }
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    auto stage_ptr = [&](int s, int which) -> uint8_t* {
        // which: 0 A_hi, 1 A_lo, 2 B_hi, 3 B_lo
        uint8_t* base = smem + (size_t)s * C::kStageBytes;
        return which < 2 ? base + which * C::kABytes : base + 2 * C::kABytes + (which - 2) * C::kBBytes;
    };

    if (warp == 0) {
        // ---------------- TMA producer
        if (lane == 0) {
            sm100::prefetch_tmap(&a_hi);
            sm100::prefetch_tmap(&a_lo);
            sm100::prefetch_tmap(&b_hi);
            sm100::prefetch_tmap(&b_lo);
            uint32_t g = 0;   // k-blocks issued by this CTA
            for (int t = blockIdx.x; t < total && !*s_abort; t += gridDim.x) {
                int pi, m0, n0;
                if (!decode_tile(probs, BN, t, pi, m0, n0)) break;
                const Problem& P = probs.p[pi];
                const int nkb = (P.K + BK - 1) / BK;
                for (int kb = 0; kb < nkb; ++kb, ++g) {
                    const int s = g % STAGES;
                    if (g >= STAGES &&
                        !wait_or_abort(&empty[s], ((g / STAGES) & 1) ^ 1, status, limit_ns, s_abort))
                        break;
                    sm100::mbar_arrive_expect_tx(&full[s], C::kStageBytes);
                    const int ka = P.a_k0 + kb * BK, kbb = P.b_k0 + kb * BK;
                    sm100::tma_load_2d(stage_ptr(s, 0), &a_hi, ka, P.a_row0 + m0, &full[s]);
                    sm100::tma_load_2d(stage_ptr(s, 1), &a_lo, ka, P.a_row0 + m0, &full[s]);
                    sm100::tma_load_2d(stage_ptr(s, 2), &b_hi, kbb, P.b_row0 + n0, &full[s]);
                    sm100::tma_load_2d(stage_ptr(s, 3), &b_lo, kbb, P.b_row0 + n0, &full[s]);
                }
            }
            // Error path: let every issued copy land before the CTA can exit.
            if (*s_abort) {
                for (uint32_t q = (g > (uint32_t)STAGES ? g - STAGES : 0); q < g; ++q)
                    sm100::mbar_wait(&full[q % STAGES], (q / STAGES) & 1, status, limit_ns);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = sm100::idesc_tf32(BM, BN);
            uint32_t g = 0;   // k-blocks consumed
            uint32_t u = 0;   // accumulator hand-offs (one per tile, or per chunk)
            bool ok = true;
            for (int t = blockIdx.x; t < total && ok && !*s_abort; t += gridDim.x) {
                int pi, m0, n0;
                if (!decode_tile(probs, BN, t, pi, m0, n0)) break;
                const int nkb = (probs.p[pi].K + BK - 1) / BK;
                const int per = chunk_len<CHUNK>(nkb), nch = chunk_count<CHUNK>(nkb);
                for (int j = 0; j < nch; ++j, ++u) {
                    const int b = u % NACC;
                    if (u >= NACC &&
                        !wait_or_abort(&acc_empty[b], ((u / NACC) & 1) ^ 1, status, limit_ns,
                                       s_abort)) {
                        ok = false;
                        break;
                    }
                    sm100::tc_fence_after();
                    const uint32_t acc = tmem + (uint32_t)(b * BN);
                    const int kb0 = j * per, kb1 = min(nkb, kb0 + per);
                    for (int kb = kb0; kb < kb1; ++kb, ++g) {
                        const int s = g % STAGES;
                        if (!wait_or_abort(&full[s], (g / STAGES) & 1, status, limit_ns, s_abort)) {
                            ok = false;
                            break;
                        }
                        sm100::tc_fence_after();
                        const uint32_t ah = sm100::smem_u32(stage_ptr(s, 0));
                        const uint32_t al = sm100::smem_u32(stage_ptr(s, 1));
                        const uint32_t bh = sm100::smem_u32(stage_ptr(s, 2));
                        const uint32_t bl = sm100::smem_u32(stage_ptr(s, 3));
#pragma unroll
                        for (int kk = 0; kk < BK / 8; ++kk) {
                            const uint32_t off = kk * 32;  // 8 tf32 = 32 bytes along the swizzled row
                            const uint64_t dah = sm100::desc_kmajor_sw128(ah + off);
                            const uint64_t dal = sm100::desc_kmajor_sw128(al + off);
                            const uint64_t dbh = sm100::desc_kmajor_sw128(bh + off);
                            const uint64_t dbl = sm100::desc_kmajor_sw128(bl + off);
                            const uint32_t acc0 = (kb > kb0 || kk > 0) ? 1u : 0u;
                            sm100::mma_tf32(acc, dah, dbh, idesc, acc0);
                            sm100::mma_tf32(acc, dah, dbl, idesc, 1u);
                            sm100::mma_tf32(acc, dal, dbh, idesc, 1u);
                        }
                        sm100::mma_commit(&empty[s]);
                    }
                    if (!ok) break;
                    if (nkb > 0) sm100::mma_commit(&acc_full[b]);
                    else sm100::mbar_arrive(&acc_full[b]);   // K = 0: the epilogue writes zeros
                }
            }
            if (*s_abort) {
                sm100::mma_commit(drain);
                sm100::mbar_wait(drain, 0, status, limit_ns);
            }
        }
    } else {
        // ---------------- epilogue (warps 2 .. 5)
        Epi e = epi;
        const int quarter = warp & 3;   // TMEM lanes this warp may read
        float* stage = epi_stage + (warp - kEpiWarp0) * (32 * 33);
        uint32_t u = 0;   // accumulator hand-offs, in the issuer's order
        bool ok = true;
        // lane 0 waits for hand-off u; the warp learns the outcome
        auto take = [&](uint32_t uu) {
            bool r = true;
            if (lane == 0)
                r = wait_or_abort(&acc_full[uu % NACC], (uu / NACC) & 1, status, limit_ns, s_abort);
            r = __shfl_sync(0xffffffffu, r ? 1 : 0, 0) != 0;
            if (r) sm100::tc_fence_after();
            return r;
        };
        auto give_back = [&](uint32_t uu) {
            sm100::tc_fence_before();
            __syncwarp();
            if (lane == 0) sm100::mbar_arrive(&acc_empty[uu % NACC]);
        };
        auto taddr = [&](uint32_t uu, int c0) {
            return tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)((uu % NACC) * BN + c0);
        };
        for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
            int pi, m0, n0;
            if (!decode_tile(probs, BN, t, pi, m0, n0)) break;
            const Problem& P = probs.p[pi];
            const bool have = P.K > 0;
            if constexpr (CHUNK == 0) {
                if (!(ok = take(u))) break;
#pragma unroll 1
                for (int c0 = 0; c0 < BN; c0 += 32) {
                    float v[32];
                    if (have) {
                        sm100::tmem_ld32(taddr(u, c0), v);
                    } else {
#pragma unroll
                        for (int q = 0; q < 32; ++q) v[q] = 0.f;
                    }
#pragma unroll
                    for (int q = 0; q < 32; ++q) stage[lane * 33 + q] = v[q];
                    __syncwarp();
                    // lane = column n0 + c0 + lane, element rr of the chunk at stage[rr * 33 + lane]
                    e.chunk(P, m0 + quarter * 32, n0 + c0 + lane, m0, n0, stage + lane);
                    __syncwarp();
                }
                give_back(u++);
            } else {
                const int nch = chunk_count<CHUNK>((P.K + BK - 1) / BK);
                float sum[BN / 32][32];
#pragma unroll
                for (int c = 0; c < BN / 32; ++c)
#pragma unroll
                    for (int q = 0; q < 32; ++q) sum[c][q] = 0.f;
                for (int j = 0; j < nch; ++j) {
                    if (!(ok = take(u))) break;
                    if (have) {
#pragma unroll
                        for (int c = 0; c < BN / 32; ++c) {
                            float v[32];
                            sm100::tmem_ld32(taddr(u, c * 32), v);
#pragma unroll
                            for (int q = 0; q < 32; ++q) sum[c][q] += v[q];
                        }
                    }
                    give_back(u++);
                }
                if (!ok) break;
#pragma unroll
                for (int c = 0; c < BN / 32; ++c) {
#pragma unroll
                    for (int q = 0; q < 32; ++q) stage[lane * 33 + q] = sum[c][q];
                    __syncwarp();
                    e.chunk(P, m0 + quarter * 32, n0 + c * 32 + lane, m0, n0, stage + lane);
                    __syncwarp();
                }
            }
            e.tile_done(P, t, quarter);
        }
    }
    __syncwarp();   // the producer and MMA warps reconverge with their idle lanes
    sm100::tc_fence_before();
    __syncthreads();
    if (warp == 1) sm100::tmem_dealloc(tmem, kTmemCols);
}

}  // namespace tc
}  // namespace bakron
