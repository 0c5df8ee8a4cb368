// tcgemm.cu -- tensor maps and hi/lo plane splitting for the 3xTF32 GEMM engine.
#include <mutex>

#include "tcgemm_host.cuh"

namespace bakron {
namespace tc {

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 32 x 32 tiles through shared memory; hi/lo computed on the way out.
__global__ void split_kernel(const float* __restrict__ src, int rows, int cols, int ld_src,
                             float* __restrict__ hi, float* __restrict__ lo, int ld_dst,
                             int transpose) {
    __shared__ float t[32][33];
    const int r0 = blockIdx.y * 32, c0 = blockIdx.x * 32;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8
    for (int k = ty; k < 32; k += 8) {
        const int r = r0 + k, c = c0 + tx;
        t[k][tx] = (r < rows && c < cols) ? src[(size_t)r * ld_src + c] : 0.f;
    }
    __syncthreads();
    for (int k = ty; k < 32; k += 8) {
        float x;
        size_t o;
        bool ok;
        if (transpose) {   // output row = source column c0 + k, output col = source row r0 + tx
            x = t[tx][k];
            ok = (c0 + k < cols) && (r0 + tx < rows);
            o = (size_t)(c0 + k) * ld_dst + r0 + tx;
        } else {
            x = t[k][tx];
            ok = (r0 + k < rows) && (c0 + tx < cols);
            o = (size_t)(r0 + k) * ld_dst + c0 + tx;
        }
        if (ok) {
            const float h = sm100::tf32_hi(x);
            hi[o] = h;
            lo[o] = x - h;
        }
    }
}

}  // namespace

int sm_count() {
    static std::mutex mu;
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 0;
    if (dev >= 64) {
        int v = 0;
        return cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess ? v : 0;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (cached[dev] == 0) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
        cached[dev] = v;
    }
    return cached[dev];
}

int make_box_map(CUtensorMap* map, const float* base, int rows, int cols, int ld, int box,
                 bool swizzle128) {
    auto fn = encode_fn();
    if (!fn) return BAKRON_ERR_CUDA;
    if (swizzle128 && box * sizeof(float) != 128) return BAKRON_ERR_INVALID_ARG;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)ld * sizeof(float)};
    cuuint32_t boxd[2] = {(cuuint32_t)box, (cuuint32_t)box};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims,
                    strides, boxd, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? BAKRON_OK : BAKRON_ERR_CUDA;
}

int make_kmajor_map(CUtensorMap* map, const float* base, int rows, int kcols, int ld,
                    int box_rows) {
    auto fn = encode_fn();
    if (!fn) return BAKRON_ERR_CUDA;
    cuuint64_t dims[2] = {(cuuint64_t)kcols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)ld * sizeof(float)};
    cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? BAKRON_OK : BAKRON_ERR_CUDA;
}

void split_planes(const float* src, int rows, int cols, int ld_src, float* hi, float* lo,
                  int ld_dst, int transpose, cudaStream_t st) {
    dim3 grid((cols + 31) / 32, (rows + 31) / 32);
    split_kernel<<<grid, 256, 0, st>>>(src, rows, cols, ld_src, hi, lo, ld_dst, transpose);
    count_launches(1);
}

}  // namespace tc
}  // namespace bakron
