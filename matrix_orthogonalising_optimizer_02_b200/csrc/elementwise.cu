// HBM-bound elementwise kernels of the Muon step ("Muon优化器" page, "Muon 算法伪代码与
// PyTorch 实现"): momentum + bf16 cast + Frobenius partial sums in one pass, the per-matrix
// Frobenius scale, and scale + decoupled weight decay + update in one pass.
// 128-bit loads/stores, 8 elements per thread per step, one (matrix, 8192-element chunk)
// per block, deterministic per-block partial sums (no atomics), warp-shuffle reductions.
#include "kernels.cuh"
#include "ptx_sm100.cuh"

namespace muon {
namespace {

constexpr int VEC = 8;
constexpr int ITERS = kEwElemsPerBlock / (kEwThreads * VEC);

template <class Item>
__device__ __forceinline__ int find_item(const Item* __restrict__ items, int count, long long b) {
    int lo = 0, hi = count - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (items[mid].block0 <= b) lo = mid; else hi = mid - 1;
    }
    return lo;
}

__device__ __forceinline__ void load8(const void* p, long long e, int f32, float* v) {
    if (f32) {
        const float4* q = reinterpret_cast<const float4*>(static_cast<const float*>(p) + e);
        const float4 a = __ldg(q), b = __ldg(q + 1);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    } else {
        const uint4 w = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p) + e));
        v[0] = bf16_lo_to_f32(w.x); v[1] = bf16_hi_to_f32(w.x); v[2] = bf16_lo_to_f32(w.y); v[3] = bf16_hi_to_f32(w.y);
        v[4] = bf16_lo_to_f32(w.z); v[5] = bf16_hi_to_f32(w.z); v[6] = bf16_lo_to_f32(w.w); v[7] = bf16_hi_to_f32(w.w);
    }
}
// Stores v (rounded to bf16 RNE when !f32) and returns the stored values in v.
__device__ __forceinline__ void store8(void* p, long long e, int f32, float* v) {
    if (f32) {
        float4* q = reinterpret_cast<float4*>(static_cast<float*>(p) + e);
        q[0] = make_float4(v[0], v[1], v[2], v[3]);
        q[1] = make_float4(v[4], v[5], v[6], v[7]);
    } else {
        uint4 w;
        w.x = pack_bf16x2(v[0], v[1]); w.y = pack_bf16x2(v[2], v[3]);
        w.z = pack_bf16x2(v[4], v[5]); w.w = pack_bf16x2(v[6], v[7]);
        *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p) + e) = w;
        v[0] = bf16_lo_to_f32(w.x); v[1] = bf16_hi_to_f32(w.x); v[2] = bf16_lo_to_f32(w.y); v[3] = bf16_hi_to_f32(w.y);
        v[4] = bf16_lo_to_f32(w.z); v[5] = bf16_hi_to_f32(w.z); v[6] = bf16_lo_to_f32(w.w); v[7] = bf16_hi_to_f32(w.w);
    }
}
__device__ __forceinline__ float load1(const void* p, long long e, int f32) {
    return f32 ? static_cast<const float*>(p)[e] : __bfloat162float(static_cast<const __nv_bfloat16*>(p)[e]);
}
__device__ __forceinline__ float store1(void* p, long long e, int f32, float v) {
    if (f32) {
        static_cast<float*>(p)[e] = v;
        return v;
    }
    const __nv_bfloat16 h = __float2bfloat16_rn(v);
    static_cast<__nv_bfloat16*>(p)[e] = h;
    return __bfloat162float(h);
}

__device__ __forceinline__ double block_sum(double v) {
    __shared__ double red[kEwThreads / 32];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int w = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) red[w] = v;
    __syncthreads();
    double s = 0.0;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kEwThreads / 32; ++i) s += red[i];
    }
    return s;
}

// M <- beta*M + G; U = nesterov ? beta*M + G : M; X0 = cast(U); partial[b] = sum X0^2.
__global__ void __launch_bounds__(kEwThreads)
momentum_cast_kernel(const MomentumItem* __restrict__ items, int count, float beta, int nesterov,
                     double* __restrict__ partials) {
    const long long b = blockIdx.x;
    const MomentumItem& it = items[find_item(items, count, b)];
    const long long start = (b - it.block0) * kEwElemsPerBlock;
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < ITERS; ++i) {
        const long long e = start + (static_cast<long long>(i) * kEwThreads + threadIdx.x) * VEC;
        if (it.vec && e + VEC <= it.n) {
            float g[VEC], u[VEC];
            load8(it.G, e, it.g_f32, g);
            if (it.M != nullptr) {
                float m[VEC];
                load8(it.M, e, 1, m);
#pragma unroll
                for (int j = 0; j < VEC; ++j) {
                    m[j] = fmaf(beta, m[j], g[j]);
                    u[j] = nesterov ? fmaf(beta, m[j], g[j]) : m[j];
                }
                store8(it.M, e, 1, m);
            } else {
#pragma unroll
                for (int j = 0; j < VEC; ++j) u[j] = g[j];
            }
            store8(it.X0, e, it.x_f32, u);
#pragma unroll
            for (int j = 0; j < VEC; ++j) ss = fmaf(u[j], u[j], ss);
        } else if (e < it.n) {
            const long long end = e + VEC < it.n ? e + VEC : it.n;
            for (long long k = e; k < end; ++k) {
                const float g = load1(it.G, k, it.g_f32);
                float u = g;
                if (it.M != nullptr) {
                    const float m = fmaf(beta, it.M[k], g);
                    it.M[k] = m;
                    u = nesterov ? fmaf(beta, m, g) : m;
                }
                const float x = store1(it.X0, k, it.x_f32, u);
                ss = fmaf(x, x, ss);
            }
        }
    }
    const double tot = block_sum(static_cast<double>(ss));
    if (threadIdx.x == 0) partials[b] = tot;
}

__global__ void frob_scale_kernel(const long long* __restrict__ block0, const long long* __restrict__ nblocks,
                                  int count, const double* __restrict__ partials, float eps,
                                  float* __restrict__ scale, unsigned* status) {
    const int w = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (w >= count) return;
    double s = 0.0;
    for (long long i = lane; i < nblocks[w]; i += 32) s += partials[block0[w] + i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) {
        if (!isfinite(s)) atomicOr(status, kDevErrNonfinite);
        scale[w] = static_cast<float>(1.0 / (sqrt(s) + static_cast<double>(eps)));
    }
}

// W <- decay*W + step*(f*O); optional O_out = f*O.
__global__ void __launch_bounds__(kEwThreads)
update_kernel(const UpdateItem* __restrict__ items, int count) {
    const long long b = blockIdx.x;
    const UpdateItem& it = items[find_item(items, count, b)];
    const long long start = (b - it.block0) * kEwElemsPerBlock;
    const float f = it.dscale != nullptr ? __ldg(it.dscale) : 1.f;
#pragma unroll
    for (int i = 0; i < ITERS; ++i) {
        const long long e = start + (static_cast<long long>(i) * kEwThreads + threadIdx.x) * VEC;
        if (it.vec && e + VEC <= it.n) {
            float w[VEC], o[VEC];
            load8(it.W, e, it.w_f32, w);
            load8(it.O, e, it.o_f32, o);
#pragma unroll
            for (int j = 0; j < VEC; ++j) o[j] *= f;
            // A scaled O keeps its storage precision (the page's X /= norm leaves X in bf16).
            if (it.dscale != nullptr && !it.o_f32) {
#pragma unroll
                for (int j = 0; j < VEC; ++j) o[j] = __bfloat162float(__float2bfloat16_rn(o[j]));
            }
            if (it.O_out != nullptr) {
                float oc[VEC];
#pragma unroll
                for (int j = 0; j < VEC; ++j) oc[j] = o[j];
                store8(it.O_out, e, it.o_f32, oc);
            }
#pragma unroll
            for (int j = 0; j < VEC; ++j) w[j] = fmaf(it.step, o[j], it.decay * w[j]);
            store8(it.W, e, it.w_f32, w);
        } else if (e < it.n) {
            const long long end = e + VEC < it.n ? e + VEC : it.n;
            for (long long k = e; k < end; ++k) {
                float o = f * load1(it.O, k, it.o_f32);
                if (it.dscale != nullptr && !it.o_f32) o = __bfloat162float(__float2bfloat16_rn(o));
                if (it.O_out != nullptr) store1(it.O_out, k, it.o_f32, o);
                store1(it.W, k, it.w_f32, fmaf(it.step, o, it.decay * load1(it.W, k, it.w_f32)));
            }
        }
    }
}

__global__ void __launch_bounds__(kEwThreads)
cast_kernel(const CastItem* __restrict__ items, int count) {
    const long long b = blockIdx.x;
    const CastItem& it = items[find_item(items, count, b)];
    const long long start = (b - it.block0) * kEwElemsPerBlock;
    const float f = it.dscale != nullptr ? __ldg(it.dscale) : 1.f;
#pragma unroll
    for (int i = 0; i < ITERS; ++i) {
        const long long e = start + (static_cast<long long>(i) * kEwThreads + threadIdx.x) * VEC;
        if (it.vec && e + VEC <= it.n) {
            float v[VEC];
            load8(it.src, e, it.src_f32, v);
#pragma unroll
            for (int j = 0; j < VEC; ++j) v[j] *= f;
            store8(it.dst, e, it.dst_f32, v);
        } else if (e < it.n) {
            const long long end = e + VEC < it.n ? e + VEC : it.n;
            for (long long k = e; k < end; ++k) store1(it.dst, k, it.dst_f32, f * load1(it.src, k, it.src_f32));
        }
    }
}

}  // namespace

cudaError_t momentum_cast_launch(const MomentumItem* d_items, int count, long long total_blocks, float beta,
                                 int nesterov, double* d_partials, cudaStream_t stream) {
    if (total_blocks <= 0) return cudaSuccess;
    momentum_cast_kernel<<<static_cast<unsigned>(total_blocks), kEwThreads, 0, stream>>>(d_items, count, beta,
                                                                                          nesterov, d_partials);
    return cudaGetLastError();
}

cudaError_t frob_scale_launch(const long long* d_block0, const long long* d_nblocks, int count,
                              const double* d_partials, float eps, float* d_scale, unsigned* d_status,
                              cudaStream_t stream) {
    if (count <= 0) return cudaSuccess;
    const int threads = 256;
    const int blocks = (count * 32 + threads - 1) / threads;
    frob_scale_kernel<<<blocks, threads, 0, stream>>>(d_block0, d_nblocks, count, d_partials, eps, d_scale, d_status);
    return cudaGetLastError();
}

cudaError_t update_launch(const UpdateItem* d_items, int count, long long total_blocks, cudaStream_t stream) {
    if (total_blocks <= 0) return cudaSuccess;
    update_kernel<<<static_cast<unsigned>(total_blocks), kEwThreads, 0, stream>>>(d_items, count);
    return cudaGetLastError();
}

cudaError_t cast_launch(const CastItem* d_items, int count, long long total_blocks, cudaStream_t stream) {
    if (total_blocks <= 0) return cudaSuccess;
    cast_kernel<<<static_cast<unsigned>(total_blocks), kEwThreads, 0, stream>>>(d_items, count);
    return cudaGetLastError();
}

}  // namespace muon
