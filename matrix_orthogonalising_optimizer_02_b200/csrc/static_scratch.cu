// Frobenius pre-scaling with library-owned scratch: X_out[i] = X0[i] / (||X0[i]||_F + eps),
// X0 = bf16(X_in) (or fp32 X_in in fp32 mode), for callers that cannot allocate device
// memory.  Same arithmetic, in the same order, as ns_orthogonalize with zero iterations:
// per 8192-element block a fp32 sum of squares per thread, reduced in fp64 (warp shuffle,
// then warps in order); per matrix the block sums strided over 32 lanes and shuffle-
// reduced; then the scaled cast with round-to-nearest-even.
//
// The scratch (block partial sums and per-matrix scales) is one file-scope __device__
// array, allocated when the library is loaded and held by every GPU that loads it until
// the process exits.  Host code cannot pass the array's name to a kernel (it names a host
// shadow, not device memory): the device address is fetched with cudaGetSymbolAddress on
// the first call made on each device, with that device current, and cached.
#include <cmath>
#include <mutex>

#include "../../include/muon_b200.h"
#include "kernels.cuh"
#include "ptx_sm100.cuh"

namespace muon {
namespace {

constexpr int kStaticBlockElems = 8192;
constexpr int kStaticThreads = 256;

struct StaticScratch {
    double partials[MUON_STATIC_MAX_BLOCKS];
    float scale[MUON_STATIC_MAX_BATCH];
};

static __device__ __align__(256) StaticScratch g_static_scratch;

std::mutex g_static_mu;
StaticScratch* g_static_ptr[256] = {};

muon_status static_scratch_address(StaticScratch** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 256) return MUON_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_static_mu);
    if (g_static_ptr[dev] == nullptr) {
        StaticScratch* p = nullptr;
        if (cudaGetSymbolAddress(reinterpret_cast<void**>(&p), g_static_scratch) != cudaSuccess || p == nullptr)
            return MUON_ERR_CUDA;
        g_static_ptr[dev] = p;
    }
    *out = g_static_ptr[dev];
    return MUON_OK;
}

__device__ __forceinline__ float load_in(const void* p, long long e, int f32) {
    return f32 ? static_cast<const float*>(p)[e] : __bfloat162float(static_cast<const __nv_bfloat16*>(p)[e]);
}
// The Newton-Schulz input: bf16-rounded (bf16 mode) or the fp32 value itself.
__device__ __forceinline__ float to_x0(float v, int fp32_mode) {
    return fp32_mode ? v : __bfloat162float(__float2bfloat16_rn(v));
}

// partials[b * blocks + lb] = sum of X0^2 over block lb of matrix b.
__global__ void __launch_bounds__(kStaticThreads)
static_sumsq_kernel(const void* X, int in_f32, int fp32_mode, long long n, int blocks, StaticScratch* sc) {
    const int lb = blockIdx.x, b = blockIdx.y;
    const size_t es = in_f32 ? 4 : 2;
    const void* x = static_cast<const uint8_t*>(X) + static_cast<size_t>(b) * n * es;
    const long long start = static_cast<long long>(lb) * kStaticBlockElems;
    float ss = 0.f;
    for (int i = 0; i < kStaticBlockElems / (kStaticThreads * 8); ++i) {
        const long long e = start + (static_cast<long long>(i) * kStaticThreads + threadIdx.x) * 8;
        const long long end = e + 8 < n ? e + 8 : n;
        for (long long k = e; k < end; ++k) {
            const float u = to_x0(load_in(x, k, in_f32), fp32_mode);
            ss = fmaf(u, u, ss);
        }
    }
    __shared__ double red[kStaticThreads / 32];
    double v = ss;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    if (threadIdx.x == 0) {
        double s = 0.0;
        for (int w = 0; w < kStaticThreads / 32; ++w) s += red[w];
        sc->partials[static_cast<long long>(b) * blocks + lb] = s;
    }
}

// scale[b] = 1 / (sqrt(sum of matrix b's partials) + eps); one warp per matrix.
__global__ void static_scale_kernel(int batch, int blocks, float eps, StaticScratch* sc, float* scale_out) {
    const int b = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (b >= batch) return;
    double s = 0.0;
    for (int i = lane; i < blocks; i += 32) s += sc->partials[static_cast<long long>(b) * blocks + i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) {
        const float f = static_cast<float>(1.0 / (sqrt(s) + static_cast<double>(eps)));
        sc->scale[b] = f;
        if (scale_out != nullptr) scale_out[b] = f;
    }
}

// X_out = scale[b] * X0, stored as out dtype (round to nearest even for bf16).
__global__ void __launch_bounds__(kStaticThreads)
static_apply_kernel(const void* X, int in_f32, int fp32_mode, void* Y, int out_f32, long long n,
                    const StaticScratch* sc) {
    const int lb = blockIdx.x, b = blockIdx.y;
    const void* x = static_cast<const uint8_t*>(X) + static_cast<size_t>(b) * n * (in_f32 ? 4 : 2);
    void* y = static_cast<uint8_t*>(Y) + static_cast<size_t>(b) * n * (out_f32 ? 4 : 2);
    const float f = sc->scale[b];
    const long long start = static_cast<long long>(lb) * kStaticBlockElems;
    for (int i = 0; i < kStaticBlockElems / (kStaticThreads * 8); ++i) {
        const long long e = start + (static_cast<long long>(i) * kStaticThreads + threadIdx.x) * 8;
        const long long end = e + 8 < n ? e + 8 : n;
        for (long long k = e; k < end; ++k) {
            const float v = f * to_x0(load_in(x, k, in_f32), fp32_mode);
            if (out_f32) static_cast<float*>(y)[k] = v;
            else static_cast<__nv_bfloat16*>(y)[k] = __float2bfloat16_rn(v);
        }
    }
}

}  // namespace
}  // namespace muon

using namespace muon;

extern "C" {

muon_status muon_frobenius_prescale_static(const void* X_in, int in_dtype, void* X_out, int out_dtype, int batch,
                                           int rows, int cols, int fp32_mode, float eps, float* scale_out,
                                           void* stream_) {
    if (X_in == nullptr || X_out == nullptr) return MUON_ERR_INVALID_ARG;
    if ((in_dtype != MUON_BF16 && in_dtype != MUON_F32) || (out_dtype != MUON_BF16 && out_dtype != MUON_F32))
        return MUON_ERR_INVALID_ARG;
    if (fp32_mode != 0 && fp32_mode != 1) return MUON_ERR_INVALID_ARG;
    if (!(eps > 0.f) || !std::isfinite(eps)) return MUON_ERR_INVALID_ARG;
    if (batch <= 0 || rows <= 0 || cols <= 0) return MUON_ERR_INVALID_ARG;
    const long long n = static_cast<long long>(rows) * cols;
    const long long blocks = (n + kStaticBlockElems - 1) / kStaticBlockElems;
    if (batch > MUON_STATIC_MAX_BATCH || blocks * batch > MUON_STATIC_MAX_BLOCKS) return MUON_ERR_UNSUPPORTED_SHAPE;
    StaticScratch* sc = nullptr;
    const muon_status st = static_scratch_address(&sc);
    if (st != MUON_OK) return st;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    const int in_f32 = in_dtype == MUON_F32, out_f32 = out_dtype == MUON_F32;
    const dim3 grid(static_cast<unsigned>(blocks), static_cast<unsigned>(batch));
    static_sumsq_kernel<<<grid, kStaticThreads, 0, stream>>>(X_in, in_f32, fp32_mode, n, static_cast<int>(blocks), sc);
    if (cudaGetLastError() != cudaSuccess) return MUON_ERR_CUDA;
    static_scale_kernel<<<(batch * 32 + 255) / 256, 256, 0, stream>>>(batch, static_cast<int>(blocks), eps, sc,
                                                                       scale_out);
    if (cudaGetLastError() != cudaSuccess) return MUON_ERR_CUDA;
    static_apply_kernel<<<grid, kStaticThreads, 0, stream>>>(X_in, in_f32, fp32_mode, X_out, out_f32, n, sc);
    if (cudaGetLastError() != cudaSuccess) return MUON_ERR_CUDA;
    return MUON_OK;
}

}  // extern "C"
