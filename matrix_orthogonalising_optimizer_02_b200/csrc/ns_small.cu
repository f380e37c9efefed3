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

constexpr int THREADS = kSmallThreads;
constexpr int PITCH = kSmallMaxR + 4;   // floats per row of A, B and XT (16-byte aligned rows)
constexpr int kUnroll = 16;             // elements per thread per round of the element loops

__device__ __forceinline__ int ridx(int t, int q) { return q < 4 ? t * 4 + q : 64 + t * 4 + (q - 4); }

__device__ __forceinline__ float ld_in(const void* p, long long e, int f32) {
    return f32 ? static_cast<const float*>(p)[e] : __bfloat162float(static_cast<const __nv_bfloat16*>(p)[e]);
}
__device__ __forceinline__ void st_out(void* p, long long e, int f32, float v) {
    if (f32) static_cast<float*>(p)[e] = v;
    else static_cast<__nv_bfloat16*>(p)[e] = __float2bfloat16_rn(v);
}

// C: CTAs per cluster (per matrix), 8 or 16; the cluster shape is given at launch.
template <int C>
__global__ void __launch_bounds__(kSmallThreads, 1)
ns_small_kernel(const SmallItem* __restrict__ items, SmallParams prm, unsigned* dev_status) {
    extern __shared__ __align__(16) float smem[];
    float* A = smem;                          // r x r (pitch PITCH)
    float* B = A + kSmallMaxR * PITCH;        // r x r: the Gram partial, then B
    float* XT = B + kSmallMaxR * PITCH;       // w x r: this CTA's slab, transposed
    __shared__ double red[THREADS / 32];
    __shared__ double part;

    cg::cluster_group cluster = cg::this_cluster();
    const int j = static_cast<int>(cluster.block_rank());
    const SmallItem it = items[blockIdx.x / C];   // by value: stores through its pointers cannot alias it
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
    // consecutive threads walk the contiguous direction of the matrix; kUnroll elements per
    // thread per round, their loads issued before any is used
    for (int e0 = tid; e0 < r * w; e0 += kUnroll * THREADS) {
        long long f[kUnroll];
        float g[kUnroll], mo[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int e = min(e0 + u * THREADS, r * w - 1);
            const int i = tall ? e % r : e / w;
            const int c = tall ? e / r : e % w;
            f[u] = flat(i, c);
            g[u] = ld_in(it.G, f[u], it.g_f32);
            mo[u] = it.M != nullptr ? it.M[f[u]] : 0.f;
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int e = e0 + u * THREADS;
            if (e >= r * w) break;
            const int i = tall ? e % r : e / w;
            const int c = tall ? e / r : e % w;
            float x = g[u];
            if (it.M != nullptr) {
                const float m = fmaf(prm.beta, mo[u], g[u]);
                it.M[f[u]] = m;
                x = prm.nesterov ? fmaf(prm.beta, m, g[u]) : m;
            }
            XT[c * PITCH + i] = x;
            ss = fmaf(x, x, ss);
        }
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
        // 2. rows R_j of A = sum_p P_p, broadcast into every CTA's A.  Per round a thread's NU
        // 16-byte pieces: every remote load is issued before any sum or store.
        constexpr int NU = C >= 16 ? 1 : 2;   // pieces per round: NU x C remote loads in flight
        for (int e0 = tid; e0 < (i1 - i0) * (r / 4); e0 += NU * THREADS) {
            float4 q[NU][C];
#pragma unroll
            for (int u = 0; u < NU; ++u) {
                const int e = min(e0 + u * THREADS, (i1 - i0) * (r / 4) - 1);
                const int i = i0 + e / (r / 4), k = 4 * (e % (r / 4));
#pragma unroll
                for (int p = 0; p < C; ++p)
                    q[u][p] = *reinterpret_cast<const float4*>(cluster.map_shared_rank(B + i * PITCH + k, p));
            }
#pragma unroll
            for (int u = 0; u < NU; ++u) {
                const int e = e0 + u * THREADS;
                if (e >= (i1 - i0) * (r / 4)) break;
                const int i = i0 + e / (r / 4), k = 4 * (e % (r / 4));
                float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int p = 0; p < C; ++p) {   // fixed order: every element summed alike
                    sum.x += q[u][p].x; sum.y += q[u][p].y; sum.z += q[u][p].z; sum.w += q[u][p].w;
                }
#pragma unroll
                for (int p = 0; p < C; ++p)
                    *reinterpret_cast<float4*>(cluster.map_shared_rank(A + i * PITCH + k, (j + p) % C)) = sum;
            }
        }
        cluster.sync();
        // 3. rows R_j of B = b A + c A A.  A is symmetric, so (A A)[i][k] is the dot product
        // of rows i and k.  Work items are (row pair, half of the columns): a warp takes rows
        // ib, ib + 1 (warp-uniform, broadcast loads), lane L the columns k = L + 32 q, q in its
        // half (consecutive rows across lanes: the 528-byte pitch puts 8 lanes on 8 different
        // bank groups).  The rows go to the local B first (every CTA has read its partials:
        // barrier above), then to the other CTAs.
        {
            const int wid = tid >> 5, lane = tid & 31;
            const int nitem = 2 * ((i1 - i0 + 1) / 2);
            for (int item = wid; item < nitem; item += THREADS / 32) {
                const int ib = i0 + 2 * (item >> 1), qh = 2 * (item & 1);
                const int nrow = min(2, i1 - ib);
                float acc[2][2];
#pragma unroll
                for (int p = 0; p < 2; ++p)
#pragma unroll
                    for (int q = 0; q < 2; ++q) acc[p][q] = 0.f;
                for (int m = 0; m < r; m += 4) {
                    const float4 x0 = *reinterpret_cast<const float4*>(A + ib * PITCH + m);
                    const float4 x1 = *reinterpret_cast<const float4*>(A + min(ib + 1, r - 1) * PITCH + m);
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const int k = min(lane + 32 * (qh + q), r - 1);
                        const float4 y = *reinterpret_cast<const float4*>(A + k * PITCH + m);
                        acc[0][q] = fmaf(x0.x, y.x, acc[0][q]); acc[0][q] = fmaf(x0.y, y.y, acc[0][q]);
                        acc[0][q] = fmaf(x0.z, y.z, acc[0][q]); acc[0][q] = fmaf(x0.w, y.w, acc[0][q]);
                        acc[1][q] = fmaf(x1.x, y.x, acc[1][q]); acc[1][q] = fmaf(x1.y, y.y, acc[1][q]);
                        acc[1][q] = fmaf(x1.z, y.z, acc[1][q]); acc[1][q] = fmaf(x1.w, y.w, acc[1][q]);
                    }
                }
#pragma unroll
                for (int p = 0; p < 2; ++p) {
                    if (p >= nrow) break;
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const int k = lane + 32 * (qh + q);
                        if (k < r) B[(ib + p) * PITCH + k] = fmaf(b, A[(ib + p) * PITCH + k], cc * acc[p][q]);
                    }
                }
            }
            __syncthreads();
            for (int e = tid; e < (i1 - i0) * (r / 4); e += THREADS) {
                const int i = i0 + e / (r / 4), k = 4 * (e % (r / 4));
                const float4 val = *reinterpret_cast<const float4*>(B + i * PITCH + k);
                for (int p = 1; p < C; ++p)
                    *reinterpret_cast<float4*>(cluster.map_shared_rank(B + i * PITCH + k, (j + p) % C)) = val;
            }
        }
        cluster.sync();
        // 4. X_j <- a X_j + B X_j, i.e. XT[c][i] <- a XT[c][i] + sum_m XT[c][m] B[i][m] (B
        // symmetric): dot products of slab rows and B rows, both contiguous in m.  Work items
        // are (4 slab rows, half of the columns): a warp takes rows c = cb .. cb + 3 (broadcast
        // loads), lane L the columns i = L + 32 q, q in its half.  Two warps share slab rows, so
        // every product is formed before any is written (barrier).
        {
            constexpr int MAXI = 8;   // items per warp: ceil(w / 4) * 2 <= 64 = 8 warps x 8
            const int wid = tid >> 5, lane = tid & 31;
            const int nitem = 2 * ((w + 3) / 4);
            float acc[MAXI][4][2];
#pragma unroll
            for (int t = 0; t < MAXI; ++t) {
                const int item = wid + t * (THREADS / 32);
                if (item >= nitem) break;
                const int cb = 4 * (item >> 1), qh = 2 * (item & 1);
#pragma unroll
                for (int p = 0; p < 4; ++p)
#pragma unroll
                    for (int q = 0; q < 2; ++q) acc[t][p][q] = 0.f;
                for (int m = 0; m < r; m += 4) {
                    float4 x[4];
#pragma unroll
                    for (int p = 0; p < 4; ++p)
                        x[p] = *reinterpret_cast<const float4*>(XT + min(cb + p, w - 1) * PITCH + m);
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const int i = min(lane + 32 * (qh + q), r - 1);
                        const float4 y = *reinterpret_cast<const float4*>(B + i * PITCH + m);
#pragma unroll
                        for (int p = 0; p < 4; ++p) {
                            acc[t][p][q] = fmaf(x[p].x, y.x, acc[t][p][q]); acc[t][p][q] = fmaf(x[p].y, y.y, acc[t][p][q]);
                            acc[t][p][q] = fmaf(x[p].z, y.z, acc[t][p][q]); acc[t][p][q] = fmaf(x[p].w, y.w, acc[t][p][q]);
                        }
                    }
                }
            }
            __syncthreads();   // every product of the slab is formed
#pragma unroll
            for (int t = 0; t < MAXI; ++t) {
                const int item = wid + t * (THREADS / 32);
                if (item >= nitem) break;
                const int cb = 4 * (item >> 1), qh = 2 * (item & 1);
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    if (cb + p >= w) break;
                    float* xr = XT + (cb + p) * PITCH;
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const int i = lane + 32 * (qh + q);
                        if (i < r) xr[i] = fmaf(a, xr[i], acc[t][p][q]);
                    }
                }
            }
            __syncthreads();
        }
    }

    // ---- update (or output) of the slab's elements: O = X (U^T's orientation back for tall)
    for (int e0 = tid; e0 < r * w; e0 += kUnroll * THREADS) {
        long long f[kUnroll];
        float wv[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int e = min(e0 + u * THREADS, r * w - 1);
            const int i = tall ? e % r : e / w;
            const int c = tall ? e / r : e % w;
            f[u] = flat(i, c);
            wv[u] = it.W != nullptr ? ld_in(it.W, f[u], it.w_f32) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int e = e0 + u * THREADS;
            if (e >= r * w) break;
            const int i = tall ? e % r : e / w;
            const int c = tall ? e / r : e % w;
            const float o = XT[c * PITCH + i];
            if (it.O != nullptr) st_out(it.O, f[u], it.o_f32, o);
            if (it.W != nullptr) st_out(it.W, f[u], it.w_f32, fmaf(it.step, o, it.decay * wv[u]));
        }
    }
    // no CTA leaves while another may still read its shared memory (steps 2 and 3 are
    // followed by barriers, so this only matters for the last iteration's remote writes)
    cluster.sync();
}

}  // namespace

size_t ns_small_smem_bytes() { return static_cast<size_t>(3) * kSmallMaxR * PITCH * sizeof(float); }

bool ns_small_fits(int rows, int cols) {
    const int r = rows < cols ? rows : cols, s = rows < cols ? cols : rows;
    return r <= kSmallMaxR && r % 8 == 0 && (s + kSmallCluster - 1) / kSmallCluster <= kSmallMaxR;
}

// Cluster size per device: 16 CTAs when the device can schedule such a cluster with this
// kernel's shared memory (a non-portable size), else 8.
int small_cluster_size(int dev) {
    static int size_of[64] = {};
    if (dev < 0 || dev >= 64) return kSmallCluster;
    if (size_of[dev] != 0) return size_of[dev];
    int chosen = kSmallCluster;
    const size_t smem = ns_small_smem_bytes();
    if (cudaFuncSetAttribute(ns_small_kernel<16>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess &&
        cudaFuncSetAttribute(ns_small_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) ==
            cudaSuccess) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(16, 1, 1);
        cfg.blockDim = dim3(THREADS, 1, 1);
        cfg.dynamicSmemBytes = smem;
        cudaLaunchAttribute attr;
        attr.id = cudaLaunchAttributeClusterDimension;
        attr.val.clusterDim.x = 16;
        attr.val.clusterDim.y = 1;
        attr.val.clusterDim.z = 1;
        cfg.attrs = &attr;
        cfg.numAttrs = 1;
        int clusters = 0;
        if (cudaOccupancyMaxActiveClusters(&clusters, ns_small_kernel<16>, &cfg) == cudaSuccess && clusters > 0)
            chosen = 16;
    }
    cudaGetLastError();   // a refused attribute or query leaves no error pending
    size_of[dev] = chosen;
    return chosen;
}

template <int C>
cudaError_t launch_clusters(const SmallItem* d_items, int count, const SmallParams& prm, unsigned* d_status,
                            cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(C * count), 1, 1);
    cfg.blockDim = dim3(THREADS, 1, 1);
    cfg.dynamicSmemBytes = ns_small_smem_bytes();
    cfg.stream = stream;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = C;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, ns_small_kernel<C>, d_items, prm, d_status);
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
        e = cudaFuncSetAttribute(ns_small_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(ns_small_smem_bytes()));
        if (e != cudaSuccess) return e;
        set_on[dev] = true;
    }
    e = small_cluster_size(dev) == 16 ? launch_clusters<16>(d_items, count, prm, d_status, stream)
                                      : launch_clusters<8>(d_items, count, prm, d_status, stream);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace muon
