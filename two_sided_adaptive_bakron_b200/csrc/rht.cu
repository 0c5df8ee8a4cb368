// rht.cu -- incoherence processing: the randomised Hadamard transform on both sides of a
// matrix (bakron_rht) and the grid steps of a matrix (bakron_row_scales).
//
// YAQA article (news.43b.com.cn/a/479517.html), section 4: the error bound of the rounding
// rule grows with the incoherence of H_O and H_I, so, as with LDLQ, the factors' incoherence is
// lowered before quantising. The transform is T_d = H_d S_d / sqrt(d): S_d random signs, H_d
// Sylvester's Hadamard matrix for d = 2^k, or H_28 (x) H_{2^k} for d = 28 2^k with H_28
// Paley's skew Hadamard matrix of order 28 (from the quadratic character of GF(27)). Applied
// as W~ = T_m W T_n^T, H_O~ = T_m H_O T_m^T, H_I~ = T_n H_I T_n^T, and W = T_m^T W~_q T_n after
// rounding; the proxy loss is the same in both bases.
//
// One CTA transforms one row with the row in registers: the signs (one Philox4x64-10 block per
// 256 indices, keyed (seed, 0) at counter (i / 256, 0, 1, 0), bit i % 256, set = -1; drawn once
// per call by rht_signs_kernel, copied by every row's CTA), the
// Sylvester butterflies over each 2^k segment (the fast Walsh-Hadamard transform: a pair
// (i, i ^ h) with 2h <= 2^k never leaves its segment), by warp shuffles, shared memory or
// inside a thread depending on the stride, then the order-28 stage across segments, and the
// 1/sqrt(d) scale. Rows of 28 * 2^k >= 1792 take a variant that stages the row in shared
// memory and forms the order-28 stage on the tensor cores (rht_rows28_kernel). The column
// transform runs in place on the result in two more passes, on tiles of 32 columns (one
// 128-byte segment per row): the butterflies of strides below B = min(2^k, 512) inside 512-row
// tiles (registers, one shared-memory exchange), then, one thread per column and row residue
// mod B, the larger strides, the order-28 stage and the scale. Every pass reads and writes the
// matrix once: HBM-bound. The butterflies and the column passes' order-28 sums are formed in
// the textbook order (strides 1, 2, 4, ..., then the order-28 sums in index order).
#include <cmath>
#include <cstring>

#include "bakron_internal.h"
#include "common.cuh"
#include "philox.cuh"
#include "sm100.cuh"

namespace bakron {
namespace {

constexpr int kMaxLen = 32768;        // 2^15, or 28 * 2^10 = 28672

struct H28 {
    signed char h[28][28];
};

// Paley's construction over GF(27) = GF(3)[t] / (t^3 + 2t + 1): element e has coefficients
// (e mod 3, e / 3 mod 3, e / 9) of 1, t, t^2; H[0][*] = 1, H[1+x][0] = -1,
// H[1+x][1+y] = chi(x - y) + [x == y], chi the quadratic character (0, +1 square, -1 not).
H28 make_h28() {
    auto mul = [](const int* a, const int* b, int* out) {
        int c[5] = {0, 0, 0, 0, 0};
        for (int i = 0; i < 3; ++i)
            for (int j = 0; j < 3; ++j) c[i + j] += a[i] * b[j];
        for (int k = 4; k >= 3; --k) {   // t^3 = t + 2
            c[k - 2] += c[k];
            c[k - 3] += 2 * c[k];
            c[k] = 0;
        }
        for (int i = 0; i < 3; ++i) out[i] = c[i] % 3;
    };
    int el[27][3];
    for (int e = 0; e < 27; ++e) {
        el[e][0] = e % 3;
        el[e][1] = (e / 3) % 3;
        el[e][2] = e / 9;
    }
    bool square[27] = {};
    for (int e = 1; e < 27; ++e) {
        int sq[3];
        mul(el[e], el[e], sq);
        square[sq[0] + 3 * sq[1] + 9 * sq[2]] = true;
    }
    H28 H;
    for (int y = 0; y < 28; ++y) H.h[0][y] = 1;
    for (int x = 0; x < 27; ++x) {
        H.h[1 + x][0] = -1;
        for (int y = 0; y < 27; ++y) {
            int d = 0, p = 1;
            for (int k = 0; k < 3; ++k, p *= 3) d += ((el[x][k] - el[y][k] + 3) % 3) * p;
            const int chi = d == 0 ? 0 : (square[d] ? 1 : -1);
            H.h[1 + x][1 + y] = (signed char)(chi + (x == y ? 1 : 0));
        }
    }
    return H;
}

// d = 28 * 2^k (returns 28, sets seg = 2^k) or 2^k (returns 1, seg = d); 0 otherwise.
int factor(int d, int& seg) {
    const bool pow2 = d > 0 && (d & (d - 1)) == 0;
    if (pow2 && d <= kMaxLen) { seg = d; return 1; }
    if (d > 0 && d % 28 == 0) {
        const int k = d / 28;
        if ((k & (k - 1)) == 0 && d <= kMaxLen) { seg = k; return 28; }
    }
    return 0;
}

// H_28 as +-1.0f for the order-28 stage (fmaf(+-1, x, acc) rounds exactly like acc +- x).
struct H28f {
    float h[28][28];
};

// Row r of Y = T X_r (inverse: T^T X_r), rows of length d = OUTER * seg, in place allowed.
// Thread t of T threads holds the E = OUTER * U elements j = t + T e in registers, T = seg / U:
// e = a U + u is element t + T u of segment a. A butterfly of stride h pairs j with j ^ h: for
// h < T the partner is thread t ^ h with the same e (a warp shuffle for h < 32, shared memory
// above); for T <= h < seg it is element e ^ (h / T) of the same thread (same segment). The
// order-28 stage then mixes the 28 segments in registers. The additions are those of the
// textbook order (strides 1, 2, 4, ..., then the order-28 sums in index order).
constexpr int kRowThreads = 512;

// x * (bit ? -1 : +1), as a flip of the sign bit: the same bits as the multiplication
__device__ __forceinline__ float flip_if(float x, uint64_t bit) {
    return __uint_as_float(__float_as_uint(x) ^ ((uint32_t)bit << 31));
}

// The sign words of T_d: words[4 b + q] = word q of the Philox4x64-10 block keyed (seed, 0) at
// counter (b, 0, 1, 0), for the (d + 255) / 256 blocks b; bit i % 64 of word i / 64 is index i.
__global__ void rht_signs_kernel(int d, unsigned long long seed, uint64_t* __restrict__ words) {
    const int nblk = (d + 255) / 256;
    for (int b = blockIdx.x * blockDim.x + threadIdx.x; b < nblk; b += gridDim.x * blockDim.x) {
        uint64_t w[4];
        philox4x64_10((uint64_t)b, 0, 1, 0, seed, 0, w);
        for (int q = 0; q < 4; ++q) words[4 * b + q] = w[q];
    }
}

template <int U, int OUTER, bool kInverse>
__global__ void __launch_bounds__(kRowThreads)
rht_rows_kernel(const float* __restrict__ X, float* __restrict__ Y, int d, int T,
                const uint64_t* __restrict__ signs, float scale,
                const __grid_constant__ H28f H) {
    constexpr int E = OUTER * U;
    extern __shared__ __align__(16) uint8_t rht_smem[];
    float* buf = reinterpret_cast<float*>(rht_smem);                    // d floats (exchange)
    uint64_t* sw = reinterpret_cast<uint64_t*>(buf + ((d + 3) & ~3));   // sign words
    const size_t row = blockIdx.x;
    const int t = threadIdx.x;
    const bool own = t < T;                   // blockDim.x = max(T, 32)
    const int nwords = 4 * ((d + 255) / 256);
    for (int q = t; q < nwords; q += blockDim.x) sw[q] = __ldg(&signs[q]);
    const float* x = X + row * (size_t)d;
    float v[E];
#pragma unroll
    for (int e = 0; e < E; ++e) v[e] = own ? x[t + T * e] : 0.f;
    __syncthreads();                          // the sign words are in place
    auto sbit = [&](int j) { return (sw[j >> 6] >> (j & 63)) & 1ull; };
    if (!kInverse && own) {
#pragma unroll
        for (int e = 0; e < E; ++e) v[e] = flip_if(v[e], sbit(t + T * e));
    }
    for (int h = 1; h < T && h < 32; h <<= 1) {
        const bool hi = (t & h) != 0;
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const float p = __shfl_xor_sync(0xffffffffu, v[e], h);
            v[e] = hi ? p - v[e] : v[e] + p;
        }
    }
    for (int h = 32; h < T; h <<= 1) {        // T >= 64 here, every thread owns elements
        const bool hi = (t & h) != 0;
#pragma unroll
        for (int e = 0; e < E; ++e) buf[t + T * e] = v[e];
        __syncthreads();
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const float p = buf[(t ^ h) + T * e];
            v[e] = hi ? p - v[e] : v[e] + p;
        }
        __syncthreads();
    }
#pragma unroll
    for (int q = 1; q < U; q <<= 1) {         // strides T, 2T, ... < seg: inside the thread
#pragma unroll
        for (int e = 0; e < E; ++e) {
            if ((e & q) == 0) {
                const float a = v[e], b = v[e | q];
                v[e] = a + b;
                v[e | q] = a - b;
            }
        }
    }
    if (OUTER == 28) {                        // v[a U + u] <- sum_c H[a][c] v[c U + u] (or H^T)
#pragma unroll
        for (int u = 0; u < U; ++u) {
            float out[28];
#pragma unroll
            for (int a = 0; a < 28; ++a) {
                float acc = 0.f;
#pragma unroll
                for (int c = 0; c < 28; ++c)
                    acc = fmaf(kInverse ? H.h[c][a] : H.h[a][c], v[c * U + u], acc);
                out[a] = acc;
            }
#pragma unroll
            for (int a = 0; a < 28; ++a) v[a * U + u] = out[a];
        }
    }
    if (!own) return;
    float* y = Y + row * (size_t)d;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int j = t + T * e;
        y[j] = (kInverse ? flip_if(v[e], sbit(j)) : v[e]) * scale;
    }
}

// Row pass for d = 28 S, S = 32 NQ = 2^k between 64 and 1024 (the order-28 stage on the tensor
// cores). One CTA per row; the row is staged in shared memory as 28 segments of NQ chunks of
// 32 positions, a chunk padded to 33 floats and a segment to SP = 33 NQ + pad floats with
// SP = 8 (mod 32), so that the accesses of all three phases spread over the banks.
//   phase 0: the row into shared memory with coalesced float4 loads;
//   phase 1: one thread per chunk: the chunk's 32 positions in registers, the signs (forward),
//            the butterflies of strides 1 .. 16;
//   phase 2: one thread per segment and position residue mod 32: its NQ positions, strides
//            32 .. S / 2;
//   phase 3: out[a][p] = sum_c G[a][c] v[c][p] (G = gtab: H_28 forward, H_28^T inverse,
//            zero-padded to 32 x 32) as m16n8k8 tf32 MMAs, 8 positions per tile: G is exact in tf32 and
//            v = hi + lo (hi the tf32 truncation), two MMAs per tile, so a product is within
//            2^-21 of exact; then the scale, the inverse's signs and the store.
// The butterflies are those of the textbook order; the order-28 sums are accumulated by the
// tensor core (not the fmaf chain of rht_rows_kernel), which moves the last bits only.
constexpr int kRows28Threads = 256;

template <int NQ>
__host__ __device__ constexpr int rows28_sp() { return 33 * NQ + ((8 - NQ % 32) + 32) % 32; }
template <int NQ>
constexpr size_t rows28_smem() { return (size_t)28 * rows28_sp<NQ>() * sizeof(float); }

template <int NQ, bool kInverse>
__global__ void __launch_bounds__(kRows28Threads, 2)
rht_rows28_kernel(const float* __restrict__ X, float* __restrict__ Y,
                  const uint64_t* __restrict__ signs, float scale,
                  const float* __restrict__ gtab) {
    constexpr int S = 32 * NQ, D = 28 * S, NCH = 28 * NQ, SP = rows28_sp<NQ>();
    static_assert(SP % 32 == 8, "segment stride");
    extern __shared__ __align__(16) float seg[];   // [28][SP]
    const size_t row = blockIdx.x;
    const float* x = X + row * D;
    float* y = Y + row * D;
    const int t = threadIdx.x, lane = t & 31, w = t >> 5;
    // phase 0: the row into shared memory, coalesced (lane q takes positions 4 q .. 4 q + 3)
    const float4* src = reinterpret_cast<const float4*>(x);
#pragma unroll 4
    for (int q = t; q < D / 4; q += kRows28Threads) {
        const float4 f = src[q];
        const int j = 4 * q;
        float* d = seg + (j / S) * SP + 33 * ((j % S) >> 5) + (j & 31);
        d[0] = f.x;
        d[1] = f.y;
        d[2] = f.z;
        d[3] = f.w;
    }
    __syncthreads();
    // phase 1
    for (int ch = t; ch < NCH; ch += kRows28Threads) {
        float* cp = seg + (ch / NQ) * SP + 33 * (ch % NQ);
        float v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = cp[i];
        if (!kInverse) {
            const uint64_t sw = __ldg(&signs[(32 * ch) >> 6]);
            const int sb = (32 * ch) & 63;
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = flip_if(v[i], (sw >> (sb + i)) & 1ull);
        }
#pragma unroll
        for (int q = 1; q < 32; q <<= 1) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                if ((i & q) == 0) {
                    const float a = v[i], b = v[i | q];
                    v[i] = a + b;
                    v[i | q] = a - b;
                }
            }
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) cp[i] = v[i];
    }
    __syncthreads();
    // phase 2
    if (NQ > 1) {
        for (int gi = t; gi < 28 * 32; gi += kRows28Threads) {
            float* base = seg + (gi >> 5) * SP + (gi & 31);
            float v[NQ];
#pragma unroll
            for (int i = 0; i < NQ; ++i) v[i] = base[33 * i];
#pragma unroll
            for (int q = 1; q < NQ; q <<= 1) {
#pragma unroll
                for (int i = 0; i < NQ; ++i) {
                    if ((i & q) == 0) {
                        const float a = v[i], b = v[i | q];
                        v[i] = a + b;
                        v[i | q] = a - b;
                    }
                }
            }
#pragma unroll
            for (int i = 0; i < NQ; ++i) base[33 * i] = v[i];
        }
        __syncthreads();
    }
    // phase 3: fragments as laid out by mma.m16n8k8 (g = lane / 4, tq = lane % 4): A rows g,
    // g + 8 and columns tq, tq + 4 of a 16 x 8 tile; B rows (k) tq, tq + 4 of column (n) g;
    // C rows g, g + 8 and columns 2 tq, 2 tq + 1
    const int g = lane >> 2, tq = lane & 3;
    auto gval = [&](int m, int k) {
        return (m < 28 && k < 28) ? __ldg(&gtab[28 * m + k]) : 0.f;
    };
    uint32_t af[2][4][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int s4 = 0; s4 < 4; ++s4) {
            const int m0 = 16 * mt + g, k0 = 8 * s4 + tq;
            af[mt][s4][0] = __float_as_uint(gval(m0, k0));
            af[mt][s4][1] = __float_as_uint(gval(m0 + 8, k0));
            af[mt][s4][2] = __float_as_uint(gval(m0, k0 + 4));
            af[mt][s4][3] = __float_as_uint(gval(m0 + 8, k0 + 4));
        }
    for (int ng = w; ng < S / 8; ng += kRows28Threads / 32) {
        const int p = 8 * ng + g;                 // this lane's B column: position p
        const float* colp = seg + 33 * (p >> 5) + (p & 31);
        uint32_t bh[4][2], bl[4][2];
#pragma unroll
        for (int s4 = 0; s4 < 4; ++s4)
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                const int k = 8 * s4 + tq + 4 * hf;
                const float xv = k < 28 ? colp[k * SP] : 0.f;
                const float hv = sm100::tf32_hi(xv);
                bh[s4][hf] = __float_as_uint(hv);
                bl[s4][hf] = __float_as_uint(xv - hv);
            }
        float acc[2][4] = {};
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int s4 = 0; s4 < 4; ++s4) {
                sm100::mma_16x8x8_tf32(acc[mt], af[mt][s4], bh[s4]);
                sm100::mma_16x8x8_tf32(acc[mt], af[mt][s4], bl[s4]);
            }
        const int p0 = 8 * ng + 2 * tq;
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int a = 16 * mt + g + 8 * hh;
                if (a >= 28) continue;
                const int j = a * S + p0;         // even: j and j + 1 share a sign word
                float v0 = acc[mt][2 * hh], v1 = acc[mt][2 * hh + 1];
                if (kInverse) {
                    const uint64_t sw = __ldg(&signs[j >> 6]);
                    v0 = flip_if(v0, (sw >> (j & 63)) & 1ull);
                    v1 = flip_if(v1, (sw >> ((j & 63) + 1)) & 1ull);
                }
                *reinterpret_cast<float2*>(y + j) = make_float2(v0 * scale, v1 * scale);
            }
    }
}

// Column transform, first pass: Y (r x c, in place) along its rows i, the signs (forward)
// and the butterflies of strides 1 .. B / 2 of every B-row slab (B = min(2^k, 512), so a slab
// never leaves a 512-row tile). CTA = 512 consecutive rows x 32 columns, thread (w, lane) =
// column lane. Phase 1: rows 32 w + e (e < 32) in registers, strides 1 .. 16 inside the thread;
// phase 2 (B > 32), after one exchange through shared memory: rows w + 16 e, strides
// 32 .. 256 inside the thread. kFinal (d = 2^k <= 512, nothing left for the second pass): the
// scale and, inverse, the signs.
constexpr int kSlabRows = 512;
constexpr int kSlabThreads = 512;
constexpr size_t kSlabSmem = (size_t)kSlabRows * 32 * sizeof(float);

__device__ __forceinline__ uint64_t sign_bit(const uint64_t* __restrict__ words, int i) {
    return (__ldg(&words[i >> 6]) >> (i & 63)) & 1ull;
}

template <bool kInverse, bool kFinal>
__global__ void __launch_bounds__(kSlabThreads)
rht_cols_slab_kernel(float* __restrict__ Y, int r, int c, int B,
                     const uint64_t* __restrict__ signs, float scale) {
    extern __shared__ __align__(16) float slab[];   // [512][32]
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r0 = blockIdx.y * kSlabRows, col = blockIdx.x * 32 + lane;
    const bool cok = col < c;
    float v[32];
    // the thread's 32 rows share one sign word (rows 32 w .. 32 w + 31 of a 64-aligned tile)
    const uint64_t sw = (r0 + 32 * w < r) ? __ldg(&signs[(r0 + 32 * w) >> 6]) : 0ull;
    const int sb = (r0 + 32 * w) & 63;
#pragma unroll
    for (int e = 0; e < 32; ++e) {
        const int row = r0 + 32 * w + e;
        v[e] = (cok && row < r) ? Y[(size_t)row * c + col] : 0.f;
        if (!kInverse) v[e] = flip_if(v[e], (sw >> (sb + e)) & 1ull);
    }
#pragma unroll
    for (int q = 1; q < 32; q <<= 1) {        // strides 1 .. 16 (row bits 0 .. 4)
        if (q >= B) break;
#pragma unroll
        for (int e = 0; e < 32; ++e) {
            if ((e & q) == 0) {
                const float a = v[e], b = v[e | q];
                v[e] = a + b;
                v[e | q] = a - b;
            }
        }
    }
    const bool two = B > 32;
    if (two) {                                // rows w + 16 e: row bits 4 .. 8 in the thread
#pragma unroll
        for (int e = 0; e < 32; ++e) slab[(32 * w + e) * 32 + lane] = v[e];
        __syncthreads();
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = slab[(w + 16 * e) * 32 + lane];
#pragma unroll
        for (int q = 2; q < 32; q <<= 1) {    // strides 32 .. 256 (e bits 1 .. 4)
            if (16 * q >= B) break;
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                if ((e & q) == 0) {
                    const float a = v[e], b = v[e | q];
                    v[e] = a + b;
                    v[e | q] = a - b;
                }
            }
        }
    }
    if (!cok) return;
#pragma unroll
    for (int e = 0; e < 32; ++e) {
        const int row = r0 + (two ? w + 16 * e : 32 * w + e);
        if (row >= r) continue;
        float y = v[e];
        if (kFinal) y = (kInverse ? flip_if(y, sign_bit(signs, row)) : y) * scale;
        Y[(size_t)row * c + col] = y;
    }
}

// Column transform, second pass, for d = OUTER * 2^k rows with 2^k = HI * B: thread = one
// column and one row residue i0 < B, holding the A = OUTER * HI rows i0 + B (q HI + h) (q <
// OUTER: the order-28 index, h < HI). The butterflies of strides B .. 2^k / 2 (the h bits), the
// order-28 stage across q, then the scale and, inverse, the signs. No shared memory, no barrier.
// G is H_28^T forward and H_28 inverse, read as G[c][a] (a column of G per output: the same
// access pattern in both directions, which keeps the table in the constant bank).
constexpr int kStridedThreads = 64;   // small CTAs: several per SM, their phases interleave

template <int OUTER, int HI, bool kInverse>
__global__ void __launch_bounds__(kStridedThreads)
rht_cols_strided_kernel(float* __restrict__ Y, int c, int B, const uint64_t* __restrict__ signs,
                        float scale, const __grid_constant__ H28f G) {
    constexpr int A = OUTER * HI;
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int i0 = blockIdx.y * (kStridedThreads / 32) + w;
    const int col = blockIdx.x * 32 + lane;
    if (i0 >= B || col >= c) return;
    // 32-bit element offsets (r c < 2^31): one register per row instead of a 64-bit address
    const unsigned off0 = (unsigned)i0 * (unsigned)c + (unsigned)col;
    const unsigned step = (unsigned)B * (unsigned)c;
    float v[A];
#pragma unroll
    for (int a = 0; a < A; ++a) v[a] = Y[off0 + a * step];
#pragma unroll
    for (int q = 1; q < HI; q <<= 1) {
#pragma unroll
        for (int a = 0; a < A; ++a) {
            if ((a & q) == 0) {
                const float x = v[a], y = v[a | q];
                v[a] = x + y;
                v[a | q] = x - y;
            }
        }
    }
    // each output row is written as soon as it is formed: sum_c G[c][a] v[c HI + h] for the
    // order-28 stage, v itself otherwise
    auto put = [&](int a, float y) {
        const int row = i0 + B * a;
        Y[off0 + a * step] = (kInverse ? flip_if(y, sign_bit(signs, row)) : y) * scale;
    };
    if (OUTER == 28) {
#pragma unroll
        for (int h = 0; h < HI; ++h) {
#pragma unroll
            for (int a = 0; a < 28; ++a) {
                float acc = 0.f;
#pragma unroll
                for (int cc = 0; cc < 28; ++cc)
                    acc = fmaf(G.h[cc][a], v[cc * HI + h], acc);
                put(a * HI + h, acc);
            }
        }
    } else {
#pragma unroll
        for (int a = 0; a < A; ++a) put(a, v[a]);
    }
}

// The second column pass for d = 28 * 2^k rows with 2^k = 2 B (28672 rows): the same work as
// rht_cols_strided_kernel<28, 2> split over a lane pair, so that each thread carries one
// order-28 stage (half the unrolled code, which otherwise overflows the instruction cache).
// Lanes l and l + 16 share column 16 * blockIdx.x + (l & 15) and row residue i0; lane half h
// holds the 28 rows i0 + B (2 q + h). The stride-B butterfly takes the partner's value by a
// shuffle (lower half a + b, upper half a - b, as in the textbook order).
template <bool kInverse>
__global__ void __launch_bounds__(kStridedThreads)
rht_cols_strided28x2_kernel(float* __restrict__ Y, int c, int B,
                            const uint64_t* __restrict__ signs, float scale,
                            const __grid_constant__ H28f G) {
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31, h = lane >> 4;
    const int i0 = blockIdx.y * (kStridedThreads / 32) + w;
    const int col = blockIdx.x * 16 + (lane & 15);
    if (i0 >= B) return;                      // the whole warp
    const bool ok = col < c;                  // inactive lanes still take part in the shuffles
    const unsigned off0 = (unsigned)(i0 + B * h) * (unsigned)c + (unsigned)col;
    const unsigned step = 2u * (unsigned)B * (unsigned)c;
    float v[28];
#pragma unroll
    for (int q = 0; q < 28; ++q) v[q] = ok ? Y[off0 + q * step] : 0.f;
#pragma unroll
    for (int q = 0; q < 28; ++q) {
        const float p = __shfl_xor_sync(0xffffffffu, v[q], 16);
        v[q] = h ? p - v[q] : v[q] + p;
    }
    if (!ok) return;
#pragma unroll
    for (int a = 0; a < 28; ++a) {
        float acc = 0.f;
#pragma unroll
        for (int cc = 0; cc < 28; ++cc) acc = fmaf(G.h[cc][a], v[cc], acc);
        const int row = i0 + B * (2 * a + h);
        Y[off0 + a * step] = (kInverse ? flip_if(acc, sign_bit(signs, row)) : acc) * scale;
    }
}

// scales[i * G + g] = max_{j in group g} |W[i][j]| / divisor; one CTA per row, one warp per
// group at a time.
__global__ void row_scales_kernel(const float* __restrict__ W, int n, int group, int G,
                                  float divisor, float* __restrict__ scales) {
    const size_t i = blockIdx.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    for (int g = warp; g < G; g += nw) {
        const int j0 = g * group, j1 = min(n, j0 + group);
        float mx = 0.f;
        for (int j = j0 + lane; j < j1; j += 32) mx = fmaxf(mx, fabsf(W[i * n + j]));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        if (lane == 0) scales[i * G + g] = mx / divisor;
    }
}

template <int U, int OUTER, bool kInverse>
int launch_rows(const float* X, float* Y, int rows, int d, const uint64_t* signs,
                const H28f& H, cudaStream_t st) {
    const int T = d / (OUTER * U);
    const size_t smem = (size_t)((d + 3) & ~3) * sizeof(float) +
                        (size_t)4 * ((d + 255) / 256) * sizeof(uint64_t);
    auto kern = rht_rows_kernel<U, OUTER, kInverse>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
        return BAKRON_ERR_CUDA;
    const float scale = 1.0f / sqrtf((float)d);
    kern<<<rows, T < 32 ? 32 : T, smem, st>>>(X, Y, d, T, signs, scale, H);
    count_launches(1);
    return cuda_err(cudaGetLastError());
}

template <int NQ, bool kInverse>
int launch_rows28(const float* X, float* Y, int rows, const uint64_t* signs, const float* gtab,
                  cudaStream_t st) {
    constexpr size_t smem = rows28_smem<NQ>();
    auto kern = rht_rows28_kernel<NQ, kInverse>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
        return BAKRON_ERR_CUDA;
    const float scale = 1.0f / sqrtf((float)(28 * 32 * NQ));
    kern<<<rows, kRows28Threads, smem, st>>>(X, Y, signs, scale, gtab);
    count_launches(1);
    return cuda_err(cudaGetLastError());
}

// Rows of 28 S with S >= 64 (and 16-byte aligned matrices): the tensor-core row pass;
// otherwise T = min(seg, 512) threads, U = seg / T columns of each segment per thread.
template <bool kInverse>
int rows_pass_dir(const float* X, float* Y, int rows, int d, const uint64_t* signs,
                  const H28f& H, const float* gtab, cudaStream_t st) {
    int seg = 0;
    const int outer = factor(d, seg);
    const int U = seg <= kRowThreads ? 1 : seg / kRowThreads;
    const bool aligned = ((reinterpret_cast<uintptr_t>(X) | reinterpret_cast<uintptr_t>(Y)) & 15) == 0;
    if (outer == 28 && aligned) {
        switch (seg) {
            case 64: return launch_rows28<2, kInverse>(X, Y, rows, signs, gtab, st);
            case 128: return launch_rows28<4, kInverse>(X, Y, rows, signs, gtab, st);
            case 256: return launch_rows28<8, kInverse>(X, Y, rows, signs, gtab, st);
            case 512: return launch_rows28<16, kInverse>(X, Y, rows, signs, gtab, st);
            case 1024: return launch_rows28<32, kInverse>(X, Y, rows, signs, gtab, st);
            default: break;
        }
    }
    if (outer == 28) {
        switch (U) {
            case 1: return launch_rows<1, 28, kInverse>(X, Y, rows, d, signs, H, st);
            case 2: return launch_rows<2, 28, kInverse>(X, Y, rows, d, signs, H, st);
            default: return BAKRON_ERR_INVALID_ARG;
        }
    }
    switch (U) {
        case 1: return launch_rows<1, 1, kInverse>(X, Y, rows, d, signs, H, st);
        case 2: return launch_rows<2, 1, kInverse>(X, Y, rows, d, signs, H, st);
        case 4: return launch_rows<4, 1, kInverse>(X, Y, rows, d, signs, H, st);
        case 8: return launch_rows<8, 1, kInverse>(X, Y, rows, d, signs, H, st);
        case 16: return launch_rows<16, 1, kInverse>(X, Y, rows, d, signs, H, st);
        case 32: return launch_rows<32, 1, kInverse>(X, Y, rows, d, signs, H, st);
        case 64: return launch_rows<64, 1, kInverse>(X, Y, rows, d, signs, H, st);
        default: return BAKRON_ERR_INVALID_ARG;
    }
}

int rows_pass(const float* X, float* Y, int rows, int d, const uint64_t* signs, int inverse,
              const H28f& H, const float* gtab, cudaStream_t st) {
    return inverse ? rows_pass_dir<true>(X, Y, rows, d, signs, H, gtab, st)
                   : rows_pass_dir<false>(X, Y, rows, d, signs, H, gtab, st);
}

template <bool kInverse, bool kFinal>
int launch_slab(float* Y, int r, int c, int B, const uint64_t* signs, float scale,
                cudaStream_t st) {
    auto kern = rht_cols_slab_kernel<kInverse, kFinal>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kSlabSmem) != cudaSuccess)
        return BAKRON_ERR_CUDA;
    kern<<<dim3((c + 31) / 32, (r + kSlabRows - 1) / kSlabRows), kSlabThreads, kSlabSmem, st>>>(
        Y, r, c, B, signs, scale);
    count_launches(1);
    return cuda_err(cudaGetLastError());
}

template <int OUTER, int HI, bool kInverse>
int launch_strided(float* Y, int c, int B, const uint64_t* signs, float scale, const H28f& H,
                   cudaStream_t st) {
    H28f G;   // H^T forward, H inverse
    for (int a = 0; a < 28; ++a)
        for (int cc = 0; cc < 28; ++cc) G.h[cc][a] = kInverse ? H.h[cc][a] : H.h[a][cc];
    rht_cols_strided_kernel<OUTER, HI, kInverse>
        <<<dim3((c + 31) / 32, (B + kStridedThreads / 32 - 1) / (kStridedThreads / 32)),
           kStridedThreads, 0, st>>>(Y, c, B, signs, scale, G);
    count_launches(1);
    return cuda_err(cudaGetLastError());
}

template <bool kInverse>
int launch_strided28x2(float* Y, int c, int B, const uint64_t* signs, float scale,
                       const H28f& H, cudaStream_t st) {
    H28f G;   // H^T forward, H inverse
    for (int a = 0; a < 28; ++a)
        for (int cc = 0; cc < 28; ++cc) G.h[cc][a] = kInverse ? H.h[cc][a] : H.h[a][cc];
    rht_cols_strided28x2_kernel<kInverse>
        <<<dim3((c + 15) / 16, (B + kStridedThreads / 32 - 1) / (kStridedThreads / 32)),
           kStridedThreads, 0, st>>>(Y, c, B, signs, scale, G);
    count_launches(1);
    return cuda_err(cudaGetLastError());
}

// Y <- T_r Y (inverse: T_r^T Y) for Y (r x c), in place: the slab pass, then (unless d = 2^k
// <= 512) the strided pass.
template <bool kInverse>
int cols_pass_dir(float* Y, int r, int c, const uint64_t* signs, const H28f& H,
                  cudaStream_t st) {
    int seg = 0;
    const int outer = factor(r, seg);
    const int B = seg < kSlabRows ? seg : kSlabRows;
    const int hi = seg / B;
    const float scale = 1.0f / sqrtf((float)r);
    const bool final_slab = outer == 1 && hi == 1;
    int e = final_slab ? launch_slab<kInverse, true>(Y, r, c, B, signs, scale, st)
                       : launch_slab<kInverse, false>(Y, r, c, B, signs, scale, st);
    if (e || final_slab) return e;
    if (outer == 28) {
        switch (hi) {
            case 1: return launch_strided<28, 1, kInverse>(Y, c, B, signs, scale, H, st);
            case 2: return launch_strided28x2<kInverse>(Y, c, B, signs, scale, H, st);
            default: return BAKRON_ERR_INVALID_ARG;
        }
    }
    switch (hi) {
        case 2: return launch_strided<1, 2, kInverse>(Y, c, B, signs, scale, H, st);
        case 4: return launch_strided<1, 4, kInverse>(Y, c, B, signs, scale, H, st);
        case 8: return launch_strided<1, 8, kInverse>(Y, c, B, signs, scale, H, st);
        case 16: return launch_strided<1, 16, kInverse>(Y, c, B, signs, scale, H, st);
        case 32: return launch_strided<1, 32, kInverse>(Y, c, B, signs, scale, H, st);
        case 64: return launch_strided<1, 64, kInverse>(Y, c, B, signs, scale, H, st);
        default: return BAKRON_ERR_INVALID_ARG;
    }
}

int cols_pass(float* Y, int r, int c, const uint64_t* signs, int inverse, const H28f& H,
              cudaStream_t st) {
    return inverse ? cols_pass_dir<true>(Y, r, c, signs, H, st)
                   : cols_pass_dir<false>(Y, r, c, signs, H, st);
}

}  // namespace
}  // namespace bakron

using namespace bakron;

extern "C" void bakron_internal_hadamard28(signed char* out) {
    const H28 H = make_h28();
    memcpy(out, H.h, sizeof(H.h));
}

extern "C" int bakron_rht_supported(int d) {
    int seg = 0;
    return factor(d, seg) != 0 ? 1 : 0;
}

inline size_t sign_words(int d) { return 4 * (size_t)((d + 255) / 256); }

// gtab[28 m + k] = the order-28 matrix applied in this call: H_28 forward, H_28^T inverse. The
// tensor-core row pass builds its fragments from it with per-lane loads from global memory
// (per-lane reads of a kernel parameter would serialise on the constant cache).
__global__ void rht_h28_table_kernel(const __grid_constant__ H28f H, int inverse, float* gtab) {
    const int t = threadIdx.x;
    if (t < 28 * 28) gtab[t] = inverse ? H.h[t % 28][t / 28] : H.h[t / 28][t % 28];
}

extern "C" size_t bakron_rht_workspace_bytes(int rows, int cols) {
    if (rows < 1 || cols < 1) return 0;
    WsSizer z;
    z.take<uint64_t>(sign_words(cols));
    z.take<uint64_t>(sign_words(rows));
    z.take<float>(28 * 28);
    return z.bytes();
}

extern "C" int bakron_rht(const float* X, int rows, int cols, uint64_t seed_rows,
                          uint64_t seed_cols, int inverse, float* Y, void* ws, size_t ws_bytes,
                          void* stream) {
    int seg = 0;
    if (rows < 1 || cols < 1 || !factor(rows, seg) || !factor(cols, seg) || !X || !Y ||
        (inverse != 0 && inverse != 1) || (long long)rows * cols >= (1LL << 31))
        return BAKRON_ERR_INVALID_ARG;
    if (!ws_ok(ws, ws_bytes, bakron_rht_workspace_bytes(rows, cols))) return BAKRON_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    static const H28f H = [] {
        const H28 h = make_h28();
        H28f f;
        for (int a = 0; a < 28; ++a)
            for (int c = 0; c < 28; ++c) f.h[a][c] = (float)h.h[a][c];
        return f;
    }();
    WsCarver c(ws);
    uint64_t* sc_words = c.take<uint64_t>(sign_words(cols));
    uint64_t* sr_words = c.take<uint64_t>(sign_words(rows));
    float* gtab = c.take<float>(28 * 28);
    rht_h28_table_kernel<<<1, 28 * 28, 0, st>>>(H, inverse, gtab);
    count_launches(1);
    // the signs of T_c and T_r, drawn once for every row
    rht_signs_kernel<<<(cols / 256 + 64) / 64, 64, 0, st>>>(cols, seed_cols, sc_words);
    rht_signs_kernel<<<(rows / 256 + 64) / 64, 64, 0, st>>>(rows, seed_rows, sr_words);
    count_launches(2);
    int e;
    // Y = X T_c^T (inverse: X T_c): each row x -> T_c x (inverse: T_c^T x)
    if ((e = rows_pass(X, Y, rows, cols, sc_words, inverse, H, gtab, st))) return e;
    // then T_r Y (inverse: T_r^T Y) along the columns, in place
    if ((e = cols_pass(Y, rows, cols, sr_words, inverse, H, st))) return e;
    return cuda_err(cudaGetLastError());
}

extern "C" int bakron_row_scales(const float* W, int m, int n, int group_size, float divisor,
                                 float* scales, void* stream) {
    if (m < 1 || n < 1 || group_size < 1 || !(divisor > 0.f && divisor < 3.0e38f) || !W ||
        !scales)
        return BAKRON_ERR_INVALID_ARG;
    const int group = group_size < n ? group_size : n;
    const int G = (n + group - 1) / group;
    row_scales_kernel<<<m, 256, 0, static_cast<cudaStream_t>(stream)>>>(W, n, group, G, divisor,
                                                                       scales);
    count_launches(1);
    return cuda_err(cudaGetLastError());
}
