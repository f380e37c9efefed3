// The whole fp32 Muon step of a small matrix in one launch: momentum, Frobenius pre-scale,
// the Newton-Schulz iterations and the update ("Muon优化器" page, "Newton-Schulz 迭代" and
// "Muon 算法伪代码与 PyTorch 实现"), for fp32 mode and r = min(rows, cols) <= 128,
// s = max(rows, cols) <= 1024.  On such a matrix every product is far too small to fill the
// GPU, and the SIMT chain spends its time in 18 dependent launches; here one cluster of
// kSmallCluster CTAs (on as many SMs) runs the whole step.
//
// X (r x s, the page's orientation: X = U, or U^T when rows > cols) is cut along s into
// kSmallCluster column slabs, one per CTA, held transposed in shared memory (XT[c][i] =
// X[i][c0 + c]).  Per iteration:
//   1. every CTA forms the partial Gram P_j = X_j X_j^T of its slab;
//   2. CTA j sums rows R_j of all P_p (distributed shared memory, fixed order p = 0, 1, ...)
//      and writes them into the A of every CTA;
//   3. CTA j forms rows R_j of B = bA + c A A and writes them into the B of every CTA;
//   4. every CTA updates its slab, X_j <- a X_j + B X_j.
// Three cluster barriers per iteration separate the steps.  All arithmetic is fp32 FMA
// (no TF32); the Frobenius sum goes through fp64, like the other paths.  A and every
// partial are bitwise symmetric (commutative products, the same order of accumulation), so
// X B with B symmetric equals the page's B X of the transposed problem.
#include <cooperative_groups.h>

#include "kernels.cuh"

namespace cg = cooperative_groups;

namespace muon {
namespace {

constexpr int C = kSmallCluster;
constexpr int THREADS = kSmallThreads;
constexpr int PITCH = kSmallMaxR + 4;   // floats per row of A, B and XT (16-byte aligned rows)

__device__ __forceinline__ int ridx(int t, int q) { return q < 4 ? t * 4 + q : 64 + t * 4 + (q - 4); }

__device__ __forceinline__ float ld_in(const void* p, long long e, int f32) {
    return f32 ? static_cast<const float*>(p)[e] : __bfloat162float(static_cast<const __nv_bfloat16*>(p)[e]);
}
__device__ __forceinline__ void st_out(void* p, long long e, int f32, float v) {
    if (f32) static_cast<float*>(p)[e] = v;
    else static_cast<__nv_bfloat16*>(p)[e] = __float2bfloat16_rn(v);
}

__global__ void __cluster_dims__(kSmallCluster, 1, 1) __launch_bounds__(kSmallThreads, 1)
ns_small_kernel(const SmallItem* __restrict__ items, SmallParams prm, unsigned* dev_status) {
    extern __shared__ __align__(16) float smem[];
    float* A = smem;                          // r x r (pitch PITCH)
    float* B = A + kSmallMaxR * PITCH;        // r x r: the Gram partial, then B
    float* XT = B + kSmallMaxR * PITCH;       // w x r: this CTA's slab, transposed
    __shared__ double red[THREADS / 32];
    __shared__ double part;

    cg::cluster_group cluster = cg::this_cluster();
    const int j = static_cast<int>(cluster.block_rank());
    const SmallItem& it = items[blockIdx.x / C];
    const int rows = it.rows, cols = it.cols;
    const bool tall = rows > cols;
    const int r = tall ? cols : rows, s = tall ? rows : cols;
    const int wmax = (s + C - 1) / C;
    const int c0 = min(s, j * wmax), w = min(s, c0 + wmax) - c0;
    const int rb = (r + C - 1) / C;
    const int i0 = min(r, j * rb), i1 = min(r, i0 + rb);
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    // element (i, c) of the slab <-> flat index of the rows x cols matrix
    auto flat = [&](int i, int c) -> long long {
        return tall ? static_cast<long long>(c0 + c) * cols + i : static_cast<long long>(i) * cols + c0 + c;
    };

    // ---- momentum (elementwise on the slab's elements), NS input, Frobenius partial
    float ss = 0.f;
    for (int e = tid; e < r * w; e += THREADS) {
        // consecutive threads walk the contiguous direction of the matrix
        const int i = tall ? e % r : e / w;
        const int c = tall ? e / r : e % w;
        const long long f = flat(i, c);
        const float g = ld_in(it.G, f, it.g_f32);
        float u = g;
        if (it.M != nullptr) {
            const float m = fmaf(prm.beta, it.M[f], g);
            it.M[f] = m;
            u = prm.nesterov ? fmaf(prm.beta, m, g) : m;
        }
        XT[c * PITCH + i] = u;
        ss = fmaf(u, u, ss);
    }
    double v = ss;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if ((tid & 31) == 0) red[tid >> 5] = v;
    __syncthreads();
    if (tid == 0) {
        double t = 0.0;
        for (int q = 0; q < THREADS / 32; ++q) t += red[q];
        part = t;
    }
    cluster.sync();
    double tot = 0.0;
    for (int p = 0; p < C; ++p) tot += *cluster.map_shared_rank(&part, p);
    if (tid == 0 && j == 0 && !isfinite(tot)) atomicOr(dev_status, kDevErrNonfinite);
    const float scale = static_cast<float>(1.0 / (sqrt(tot) + static_cast<double>(prm.eps)));
    for (int e = tid; e < r * w; e += THREADS) {
        const int c = e / r, i = e % r;
        XT[c * PITCH + i] *= scale;
    }
    __syncthreads();

    for (int t = 0; t < prm.n_iters; ++t) {
        const float a = prm.coeffs[3 * t], b = prm.coeffs[3 * t + 1], cc = prm.coeffs[3 * t + 2];
        // 1. P_j = X_j X_j^T into B (8 x 8 per thread; rows/cols past r are never read)
        {
            float acc[8][8];
#pragma unroll
            for (int p = 0; p < 8; ++p)
#pragma unroll
                for (int q = 0; q < 8; ++q) acc[p][q] = 0.f;
            for (int c = 0; c < w; ++c) {
                const float* x = XT + c * PITCH;
                const float4 a0 = *reinterpret_cast<const float4*>(x + ty * 4);
                const float4 a1 = *reinterpret_cast<const float4*>(x + 64 + ty * 4);
                const float4 b0 = *reinterpret_cast<const float4*>(x + tx * 4);
                const float4 b1 = *reinterpret_cast<const float4*>(x + 64 + tx * 4);
                const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
                const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
                for (int p = 0; p < 8; ++p)
#pragma unroll
                    for (int q = 0; q < 8; ++q) acc[p][q] = fmaf(av[p], bv[q], acc[p][q]);
            }
#pragma unroll
            for (int p = 0; p < 8; ++p) {
                const int i = ridx(ty, p);
                if (i >= r) continue;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int k = h * 64 + tx * 4;
                    if (k < r)
                        *reinterpret_cast<float4*>(B + i * PITCH + k) =
                            make_float4(acc[p][4 * h], acc[p][4 * h + 1], acc[p][4 * h + 2], acc[p][4 * h + 3]);
                }
            }
        }
        cluster.sync();
        // 2. rows R_j of A = sum_p P_p, broadcast into every CTA's A
        for (int e = tid; e < (i1 - i0) * (r / 4); e += THREADS) {
            const int i = i0 + e / (r / 4), k = 4 * (e % (r / 4));
            float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int p = 0; p < C; ++p) {
                const float4 q = *reinterpret_cast<const float4*>(cluster.map_shared_rank(B + i * PITCH + k, p));
                sum.x += q.x; sum.y += q.y; sum.z += q.z; sum.w += q.w;
            }
            for (int p = 0; p < C; ++p) *reinterpret_cast<float4*>(cluster.map_shared_rank(A + i * PITCH + k, p)) = sum;
        }
        cluster.sync();
        // 3. rows R_j of B = b A + c A A (A symmetric), broadcast into every CTA's B
        for (int e = tid; e < (i1 - i0) * (r / 8); e += THREADS) {
            const int i = i0 + e / (r / 8), k = 8 * (e % (r / 8));
            float acc[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) acc[q] = 0.f;
            for (int m = 0; m < r; ++m) {
                const float aim = A[i * PITCH + m];
                const float4 b0 = *reinterpret_cast<const float4*>(A + m * PITCH + k);
                const float4 b1 = *reinterpret_cast<const float4*>(A + m * PITCH + k + 4);
                acc[0] = fmaf(aim, b0.x, acc[0]); acc[1] = fmaf(aim, b0.y, acc[1]);
                acc[2] = fmaf(aim, b0.z, acc[2]); acc[3] = fmaf(aim, b0.w, acc[3]);
                acc[4] = fmaf(aim, b1.x, acc[4]); acc[5] = fmaf(aim, b1.y, acc[5]);
                acc[6] = fmaf(aim, b1.z, acc[6]); acc[7] = fmaf(aim, b1.w, acc[7]);
            }
            float o[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) o[q] = fmaf(b, A[i * PITCH + k + q], cc * acc[q]);
            for (int p = 0; p < C; ++p) {
                float* dst = cluster.map_shared_rank(B + i * PITCH + k, p);
                *reinterpret_cast<float4*>(dst) = make_float4(o[0], o[1], o[2], o[3]);
                *reinterpret_cast<float4*>(dst + 4) = make_float4(o[4], o[5], o[6], o[7]);
            }
        }
        cluster.sync();
        // 4. X_j <- a X_j + B X_j, i.e. XT <- a XT + XT B (B symmetric): rows c = ty + 16 q of
        // XT, columns ridx(tx, .) ; computed in registers, written after a barrier
        {
            float acc[8][8];
#pragma unroll
            for (int p = 0; p < 8; ++p)
#pragma unroll
                for (int q = 0; q < 8; ++q) acc[p][q] = 0.f;
            const int nq = (w - ty + 15) / 16;   // rows of XT this thread owns
            for (int m = 0; m < r; ++m) {
                const float4 b0 = *reinterpret_cast<const float4*>(B + m * PITCH + tx * 4);
                const float4 b1 = *reinterpret_cast<const float4*>(B + m * PITCH + 64 + tx * 4);
                const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
                for (int p = 0; p < 8; ++p) {
                    if (p < nq) {
                        const float xm = XT[(ty + 16 * p) * PITCH + m];
#pragma unroll
                        for (int q = 0; q < 8; ++q) acc[p][q] = fmaf(xm, bv[q], acc[p][q]);
                    }
                }
            }
#pragma unroll
            for (int p = 0; p < 8; ++p) {
                if (p < nq) {
                    const float* x = XT + (ty + 16 * p) * PITCH;
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const int i = ridx(tx, q);
                        if (i < r) acc[p][q] = fmaf(a, x[i], acc[p][q]);
                    }
                }
            }
            __syncthreads();   // every thread has read the old slab
#pragma unroll
            for (int p = 0; p < 8; ++p) {
                if (p < nq) {
                    float* x = XT + (ty + 16 * p) * PITCH;
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const int i = ridx(tx, q);
                        if (i < r) x[i] = acc[p][q];
                    }
                }
            }
            __syncthreads();
        }
    }

    // ---- update (or output) of the slab's elements: O = X (U^T's orientation back for tall)
    for (int e = tid; e < r * w; e += THREADS) {
        const int i = tall ? e % r : e / w;
        const int c = tall ? e / r : e % w;
        const long long f = flat(i, c);
        const float o = XT[c * PITCH + i];
        if (it.O != nullptr) st_out(it.O, f, it.o_f32, o);
        if (it.W != nullptr) st_out(it.W, f, it.w_f32, fmaf(it.step, o, it.decay * ld_in(it.W, f, it.w_f32)));
    }
    // no CTA leaves while another may still read its shared memory (steps 2 and 3 are
    // followed by barriers, so this only matters for the last iteration's remote writes)
    cluster.sync();
}

}  // namespace

size_t ns_small_smem_bytes() { return static_cast<size_t>(3) * kSmallMaxR * PITCH * sizeof(float); }

bool ns_small_fits(int rows, int cols) {
    const int r = rows < cols ? rows : cols, s = rows < cols ? cols : rows;
    return r <= kSmallMaxR && r % 8 == 0 && (s + C - 1) / C <= kSmallMaxR;
}

cudaError_t ns_small_launch(const SmallItem* d_items, int count, const SmallParams& prm, unsigned* d_status,
                            cudaStream_t stream) {
    if (count <= 0) return cudaSuccess;
    static bool set_on[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!set_on[dev]) {   // per device, once (launches run under the plan cache's lock)
        e = cudaFuncSetAttribute(ns_small_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(ns_small_smem_bytes()));
        if (e != cudaSuccess) return e;
        set_on[dev] = true;
    }
    ns_small_kernel<<<C * count, THREADS, ns_small_smem_bytes(), stream>>>(d_items, prm, d_status);
    return cudaGetLastError();
}

}  // namespace muon
