/*
 * bakron.h -- C ABI of the BaKron two-sided adaptive rounding library (CUDA, sm_100a).
 *
 * The library rounds an m x n weight matrix W* (rows = output features, columns = input
 * features) under a Kronecker-factored Hessian H ~ H_O (x) H_I, H_O m x m, H_I n x n
 * (YAQA article, news.43b.com.cn/a/479517.html, section 2: Kronecker approximation of the
 * Fisher; BaKron page "BaKron: Efficient Quantization with Kronecker-Factored Hessians",
 * abstract: the two-sided adaptive-rounding formulation of BoA/YAQA).
 *
 * Conventions for every entry point:
 *   - All array pointers are DEVICE pointers unless stated otherwise. Matrices are dense,
 *     row-major, leading dimension = number of columns. fp32 unless stated otherwise.
 *   - The caller owns every buffer, including the workspace; the library never allocates
 *     device memory. Outputs must not alias inputs or the workspace.
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t passed as void*; NULL is the
 *     legacy default stream). The return value reports host-side argument checks and launch
 *     errors only. Errors found on the device (non-positive pivot, non-finite input, a
 *     dependency wait that timed out) are written to `*dev_status`, a device int that the
 *     caller owns and initialises to 0 (BAKRON_OK). Calls never reset it: the first error of
 *     a chain of calls sticks, and bakron_read_status() reads it.
 *   - Nothing traps: device-side waits are bounded and give up with BAKRON_ERR_TIMEOUT.
 *   - Identical inputs give bitwise identical outputs.
 *   - Host threads: any entry point may be called from several host threads at once (the
 *     library's own host state, e.g. the SM count per device, is set up once under a lock);
 *     calls whose buffers, workspaces or status words overlap race on the device unless the
 *     caller orders their streams.
 */
#ifndef BAKRON_H_
#define BAKRON_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    BAKRON_OK = 0,
    BAKRON_ERR_INVALID_ARG = -1,  /* bad size, NULL pointer, unsupported bits          */
    BAKRON_ERR_NOT_PD = -2,       /* a pivot D_j <= 0 or non-finite in bakron_ldl        */
    BAKRON_ERR_CUDA = -3,         /* a CUDA launch or runtime call failed                */
    BAKRON_ERR_TIMEOUT = -4,      /* a device-side dependency wait gave up               */
    BAKRON_ERR_WORKSPACE = -5,    /* workspace NULL, too small or misaligned (256 B)     */
    BAKRON_ERR_NONFINITE = -6,    /* a non-finite value met on the device                */
    BAKRON_ERR_CAPTURE = -7       /* a set-up step that cannot run under stream capture  */
} bakron_status;

/* ------------------------------------------------------------------------------------------
 * bakron_ldl -- U D U^T factorisation of one damped Kronecker factor.
 *
 * Computes H = (I + L) D (I + L)^T with L strictly UPPER triangular and D diagonal > 0
 * (YAQA article, section 4: the factor L_O of the rounding rule is taken from the LDL
 * decomposition H_O = (L_O + I) D_O (L_O + I)^T; the rule of the same section makes L_O
 * strictly upper triangular, since a_i, the i-th column of L_O, only has entries above row i).
 * Equivalently it is the LDL^T factorisation of H with its index order reversed.
 *
 *   H        [in]  n x n, symmetric positive definite, already damped by the caller. Only the
 *                  upper triangle (j >= i) is read.
 *   n        [in]  1 <= n <= 65536.
 *   L        [out] n x n; written in full: the strictly upper part holds L, every entry on
 *                  and below the diagonal is 0.
 *   D        [out] n pivots.
 *   ws       [in]  workspace of at least bakron_ldl_workspace_bytes(n) bytes, 256-B aligned.
 *   dev_status [out] device int; BAKRON_ERR_NOT_PD if a pivot is <= 0 or non-finite (L and D
 *                  are then unspecified).
 * ---------------------------------------------------------------------------------------- */
size_t bakron_ldl_workspace_bytes(int n);
int bakron_ldl(const float* H, int n, float* L, float* D,
               void* ws, size_t ws_bytes, int* dev_status, void* stream);

/* ------------------------------------------------------------------------------------------
 * bakron_ldl_noalloc -- bakron_ldl without a caller workspace. (The pages have no counterpart:
 * this serves callers that cannot allocate device memory, e.g. a process whose framework
 * allocator already holds the device's memory, or a latency-critical loop that must not call
 * cudaMalloc / cudaFree, which can synchronise the device.)
 *
 * Same contract and results as bakron_ldl, with the scratch in a fixed array that is part of
 * the library (20 MiB, held on every GPU that loads the library until the process exits).
 *   n        [in]  1 <= n <= bakron_ldl_noalloc_max_n() (2048); larger n returns
 *                  BAKRON_ERR_INVALID_ARG without touching the device.
 * The first call on a device looks up the array's device address (cudaGetSymbolAddress) with
 * that device current, and caches it with the id of the device's current CUDA context; a call
 * that finds a different context current (the context was destroyed and created again, e.g.
 * by cudaDeviceReset) looks the address up again. Make the first call on a device, and the
 * first after such a reset, before any stream capture: a lookup while `stream` is capturing is
 * refused with BAKRON_ERR_CAPTURE, the capture untouched. Calls share the array: two calls that
 * overlap on the GPU (different streams or host threads) race. Nothing in the array needs to
 * start at zero. Allocates nothing.
 * ---------------------------------------------------------------------------------------- */
int bakron_ldl_noalloc(const float* H, int n, float* L, float* D, int* dev_status,
                       void* stream);
int bakron_ldl_noalloc_max_n(void);

/* ------------------------------------------------------------------------------------------
 * bakron_round -- the BaKron solve of the two-sided adaptive rounding rule.
 *
 * For every entry, in any order compatible with "(k,l) before (i,j) when k <= i and l <= j"
 * (the anti-diagonal order of the BaKron page, abstract: O(m+n) sequential steps):
 *
 *   pre_ij = W*_ij + a_i^T E[:i,:j] b_j + a_i^T E[:i,j] + E[i,:j] b_j      (YAQA, section 4)
 *   code_ij = clamp(round_half_even(pre_ij / s_i), -2^(bits-1), 2^(bits-1) - 1)
 *   W_ij    = s_i * code_ij,      E_ij = W*_ij - W_ij
 *
 * where a_i is column i of L_O (entries k < i), b_j is column j of L_I (entries l < j), and
 * ":i" means indices 0..i-1. Equivalently W = Q(W* + (I+L_O)^T E (I+L_I) - E) holds at every
 * entry (the closed form used to check results). pre_ij is accumulated in fp32 (products as
 * 3xTF32 on the tensor cores); the rounding decision is exact for that fp32 value, i.e. it
 * rounds the real quotient pre_ij / s_i, not an fp32 approximation of it.
 *
 *   Wstar    [in]  m x n.
 *   m, n     [in]  1 <= m, n; m*n < 2^31.
 *   L_O      [in]  m x m, strictly upper part used (the output format of bakron_ldl).
 *   L_I      [in]  n x n, strictly upper part used.
 *   scales   [in]  m per-row grid steps s_i >= 0 (s_i == 0: the row gets code 0, W 0).
 *   bits     [in]  2..8.
 *   codes    [out] m x n int8.
 *   W        [out] m x n dequantised weights s_i * code_ij.
 *   ws       [in/out] at least bakron_round_workspace_bytes(m, n) bytes, 256-B aligned. When
 *                  the call has run, its first m*n floats hold the residual E = W* - W
 *                  (row-major), ready to be passed to bakron_proxy_loss as dW.
 *   dev_status [out] BAKRON_ERR_TIMEOUT if a dependency wait gave up, BAKRON_ERR_NONFINITE if a
 *                  pre-rounding value was not finite.
 * ---------------------------------------------------------------------------------------- */
size_t bakron_round_workspace_bytes(int m, int n);
int bakron_round(const float* Wstar, int m, int n, const float* L_O, const float* L_I,
                 const float* scales, int bits, int8_t* codes, float* W,
                 void* ws, size_t ws_bytes, int* dev_status, void* stream);

/* ------------------------------------------------------------------------------------------
 * bakron_round_stochastic -- bakron_round with stochastic Q in place of nearest rounding (the
 * YAQA article's rounding rule, section 4, takes Q as nearest or stochastic rounding).
 *
 *   code_ij = clamp(floor(x_ij + u_ij), -2^(bits-1), 2^(bits-1) - 1),   x_ij = pre_ij / s_i,
 *
 * so that, away from the clamp, s_i code_ij is an unbiased rounding of pre_ij: it takes the
 * grid point above with probability frac(x_ij). The decision is exact for the kernel's fp32
 * pre_ij: floor of the real x_ij + u_ij. The variate u_ij = (k_ij + 1/2) / 2^16, where k_ij is the
 * 16-bit field (j mod 16) (least significant first: word (j mod 16) / 4, bits 16 (j mod 4)
 * and up) of the Philox4x64-10 block (Salmon, Moraes, Dror, Shaw, "Parallel random numbers:
 * as easy as 1, 2, 3", SC 2011) with key (seed, 0) and counter (j / 16, i, 0, 0).
 *
 *   seed     [in]  64-bit key of the variates; the same seed gives bitwise the same result.
 * Every other argument, the workspace (bakron_round_workspace_bytes) and the error behaviour
 * are those of bakron_round.
 * ---------------------------------------------------------------------------------------- */
int bakron_round_stochastic(const float* Wstar, int m, int n, const float* L_O,
                            const float* L_I, const float* scales, int bits, uint64_t seed,
                            int8_t* codes, float* W, void* ws, size_t ws_bytes, int* dev_status,
                            void* stream);

/* ------------------------------------------------------------------------------------------
 * bakron_round_ex -- bakron_round with the base quantizer chosen by the caller (the BaKron
 * page, summary: the solver is modular in the base quantizer): per-group grid steps and/or a
 * sorted scalar codebook. The rule and its order are those of bakron_round; only Q changes:
 *
 *   s_ij   = scales[i * G + j / group_size],   G = ceil(n / group_size)
 *   without a codebook: code_ij = clamp(round_half_even(pre_ij / s_ij)), W_ij = s_ij code_ij
 *   with a codebook c_0 < ... < c_{K-1}, K = 2^bits:
 *            code_ij = the index k of the entry nearest to x = pre_ij / s_ij, decided against
 *                      the fp32 midpoints fl32((c_k + c_{k+1}) / 2) (a tie goes to the lower
 *                      entry; x is the real quotient of the kernel's fp32 pre_ij),
 *            W_ij    = s_ij c_k.
 *
 *   scales   [in]  m x G grid steps (device), s_ij >= 0 (0: code 0 and W 0 on that row part;
 *                  with a codebook, code 0 is the index of c_0 and W is still 0).
 *   group_size [in] columns per grid step: a multiple of 32, or >= n (one step per row, the
 *                  layout of bakron_round).
 *   codebook [in]  HOST pointer to 2^bits finite, strictly increasing fp32 entries, copied
 *                  during the call; NULL selects the integer grid.
 *   bits     [in]  1..4 with a codebook (codes are entry indices 0 .. 2^bits - 1), else 2..8.
 * Every other argument, the workspace (bakron_round_workspace_bytes) and the error behaviour
 * are those of bakron_round; an invalid group_size or codebook returns BAKRON_ERR_INVALID_ARG.
 * ---------------------------------------------------------------------------------------- */
int bakron_round_ex(const float* Wstar, int m, int n, const float* L_O, const float* L_I,
                    const float* scales, int group_size, const float* codebook, int bits,
                    int8_t* codes, float* W, void* ws, size_t ws_bytes, int* dev_status,
                    void* stream);

/* ------------------------------------------------------------------------------------------
 * bakron_proxy_loss -- tr(H_O dW H_I dW^T) = vec(dW)^T (H_O (x) H_I) vec(dW).
 *
 * The layer proxy of the YAQA article (section 4 error bound, section 2 second-order
 * objective without its factor 1/2), row-major vec.
 *
 *   dW       [in]  m x n (e.g. W* - W).
 *   H_O, H_I [in]  m x m and n x n, symmetric (both triangles are read).
 *   loss     [out] one DEVICE double.
 *   ws       [in]  at least bakron_proxy_loss_workspace_bytes(m, n) bytes, 256-B aligned.
 * ---------------------------------------------------------------------------------------- */
size_t bakron_proxy_loss_workspace_bytes(int m, int n);
int bakron_proxy_loss(const float* dW, int m, int n, const float* H_O, const float* H_I,
                      double* loss, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------------------------
 * bakron_damped_gram -- one damped Kronecker factor from samples: the input second moment.
 *
 *   H = X^T X / N + damp * mean_i (X^T X / N)_ii * I
 *
 * (YAQA article, section 3: H_1 = E[x^T x] over the input rows x, the one-sided factor and
 * Sketch A's starting point; the same call gives E[g^T g] over output-gradient rows g. The
 * relative damping is that of the solver's inputs.) The product runs as 3xTF32 on the tensor
 * cores over the upper block triangle; H is then made exactly symmetric. Accuracy: each
 * product is within 3 * 2^-20 of exact, and the fp32 accumulation over the N samples loses
 * up to about 2^-24 N sqrt(H_aa H_bb) per entry (the tensor core rounds its accumulator
 * toward zero; 1.6e-4 sqrt(H_aa H_bb) at N = 8192).
 *
 *   X        [in]  N x d samples (rows), fp32.
 *   N, d     [in]  1 <= N <= 2097120, 1 <= d <= 65536.
 *   damp     [in]  relative damping >= 0 (0.01 for the solver's inputs).
 *   H        [out] d x d, symmetric, written in full; ready for bakron_ldl.
 *   ws       [in]  at least bakron_damped_gram_workspace_bytes(N, d) bytes, 256-B aligned.
 *   dev_status [out] BAKRON_ERR_TIMEOUT if a pipeline wait of the product gave up.
 * ---------------------------------------------------------------------------------------- */
size_t bakron_damped_gram_workspace_bytes(int N, int d);
int bakron_damped_gram(const float* X, int N, int d, float damp, float* H, void* ws,
                       size_t ws_bytes, int* dev_status, void* stream);

/* ------------------------------------------------------------------------------------------
 * bakron_sketch_b -- both Kronecker factors from per-sequence weight gradients (YAQA article,
 * section 3, Sketch B: one power-iteration round on the Fisher from H_O = H_I = I), damped:
 *
 *   H_O = (1/S) sum_s G_s G_s^T / n  + damp * mean(diag) * I      (m x m)
 *   H_I = (1/S) sum_s G_s^T G_s / m  + damp * mean(diag) * I      (n x n)
 *
 *   G        [in]  S x m x n: the gradient of the loss of sequence s w.r.t. the m x n weight
 *                  is G + s*m*n, row-major.
 *   S, m, n  [in]  1 <= m, n <= 65536, S*m <= 2097120, S*n <= 2^30.
 *   damp     [in]  relative damping >= 0.
 *   H_O, H_I [out] symmetric, written in full.
 *   ws       [in]  at least bakron_sketch_b_workspace_bytes(S, m, n) bytes, 256-B aligned.
 *   dev_status [out] as for bakron_damped_gram.
 * ---------------------------------------------------------------------------------------- */
size_t bakron_sketch_b_workspace_bytes(int S, int m, int n);
int bakron_sketch_b(const float* G, int S, int m, int n, float damp, float* H_O, float* H_I,
                    void* ws, size_t ws_bytes, int* dev_status, void* stream);

/* ------------------------------------------------------------------------------------------
 * bakron_rht -- the randomised Hadamard transform on both sides of a matrix (incoherence
 * processing; YAQA article, section 4: the bound on the rounding error grows with the
 * incoherence of H_O and H_I, which is lowered before quantising, as for LDLQ).
 *
 *   T_d = H_d S_d / sqrt(d),  S_d = diag(+-1),
 *   H_d = Sylvester's Hadamard matrix ((-1)^popcount(i & j)) for d = 2^k, and
 *         H_28 (x) H_{2^k} for d = 28 * 2^k, H_28 Paley's skew Hadamard matrix from the
 *         quadratic character chi of GF(27) = GF(3)[t] / (t^3 + 2t + 1) (element e <->
 *         (e mod 3) + (e/3 mod 3) t + (e/9) t^2; H_28[0][*] = 1, H_28[1+x][0] = -1,
 *         H_28[1+x][1+y] = chi(x - y) + [x = y]);
 *   S_d[i] = -1 when bit (i mod 256) of the Philox4x64-10 block keyed (seed, 0) at counter
 *         (i / 256, 0, 1, 0) is set (word (i mod 256) / 64, bit i mod 64), else +1;
 *   Y = T_rows X T_cols^T   (inverse = 0),    Y = T_rows^T X T_cols   (inverse = 1).
 *
 * The layer is processed as W~ = rht(W*, seed_o, seed_i), H_O~ = rht(H_O, seed_o, seed_o),
 * H_I~ = rht(H_I, seed_i, seed_i); after rounding W~, W = rht(W~_q, seed_o, seed_i, inverse).
 *
 *   X        [in]  rows x cols; may be the same buffer as Y.
 *   rows, cols [in] each 2^k or 28 * 2^k, at most 32768 (bakron_rht_supported tells).
 *   Y        [out] rows x cols.
 *   ws       [in]  at least bakron_rht_workspace_bytes(rows, cols) bytes, 256-B aligned.
 * Returns BAKRON_ERR_INVALID_ARG for an unsupported size. Three passes over the matrix: the
 * signs, butterflies and order-28 stage along each row (one CTA per row), then the same along
 * the columns in place on Y, on 32-column tiles: strides below 512 in one pass, the larger
 * strides and the order-28 stage in the next. The workspace holds the sign words and the
 * 28 x 28 matrix of the order-28 stage.
 * ---------------------------------------------------------------------------------------- */
int bakron_rht_supported(int d);
size_t bakron_rht_workspace_bytes(int rows, int cols);
int bakron_rht(const float* X, int rows, int cols, uint64_t seed_rows, uint64_t seed_cols,
               int inverse, float* Y, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------------------------
 * bakron_row_scales -- grid steps from a matrix: scales[i * G + g] = max over the columns j of
 * group g of |W[i][j]|, divided by `divisor` (one correctly rounded fp32 division);
 * G = ceil(n / group_size), group_size >= n gives one step per row. With divisor
 * 2^(bits-1) - 0.5 these are the per-row max-abs grid steps of the integer grid.
 *   W [in] m x n; scales [out] m x G (device); divisor > 0.
 * ---------------------------------------------------------------------------------------- */
int bakron_row_scales(const float* W, int m, int n, int group_size, float divisor,
                      float* scales, void* stream);

/* Synchronises `stream`, then returns the device status word (a bakron_status value), or
 * BAKRON_ERR_CUDA if the synchronisation itself failed. */
int bakron_read_status(const int* dev_status, void* stream);

/* Static, NUL-terminated description of a bakron_status value. */
const char* bakron_status_string(int code);

/* Number of CUDA kernels this library has launched in the calling process so far
 * (diagnostics: lets a benchmark count its launches). */
unsigned long long bakron_kernel_launches(void);

/* Library version as 10000*major + 100*minor + patch (0.2.0: stochastic Q, the pluggable
 * base quantizer, the Kronecker-factor and incoherence-processing entry points). */
int bakron_version(void);

#ifdef __cplusplus
}
#endif

#endif /* BAKRON_H_ */
