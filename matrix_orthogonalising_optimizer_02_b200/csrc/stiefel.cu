// Stiefel-manifold step ("Muon 在 Stiefel 流形上的精确闭式更新", mlqm.cn/news/1339166):
//   §1.3/§3.2  V = G - W sym(W^T G)
//   §6.2       Cayley retraction W <- (I + cA)^-1 (I - cA) W, A = V W^T - W V^T = U B with
//              U = [V, W], B = [W^T; -V^T], c = lr/2, through the 2k x 2k system
//              C = I + c B U = [[I + cP, cQ], [-cR, I - cP^T]]   (P = W^T V, Q = W^T W, R = V^T V)
//              The page's Woodbury steps (b = W - c U B W, y = B b, z = C^-1 y,
//              W_new = b - c U z) are taken through the identity
//              (I + cA)^-1 (I - cA) = 2 (I + cA)^-1 - I, which gives the same map with y
//              replaced by c B W = [cQ; -cP^T] (the right block column of C - I, no product):
//              z = C^-1 [cQ; -cP^T],  W_new = W - 2 (V z_top + W z_bot).
//              That drops the products for b and y, half the n x k fp32 work.
// No TF32 anywhere.  The n x k panel products run on the FMA pipes in fp32; the reductions
// over n (W^T G and the blocks P, Q, R) are split into 512-row chunks accumulated in fp32
// in parallel and summed in fp64.  The augmented 2k x (2k + k)
// matrix [C | c B W] is held and eliminated in fp64 (Gaussian elimination with partial
// pivoting, blocked: panel factorisation in shared memory, row swaps + unit-lower solve on
// the right-hand columns, rank-nb GEMM update), then blocked back substitution: C has
// condition numbers around 1e3 at n = 4096, k = 1024, and an fp32 solve alone lets the
// orthogonality defect ||W^T W - I|| grow by ~1e-7 per step.
#include <algorithm>
#include <cmath>

#include <cooperative_groups.h>

#include "runtime.cuh"
#include "simt_async.cuh"

namespace muon {
namespace {

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ---------------------------------------------------------------- small kernels
// S <- (S + S^T) / 2 in place (k x k per matrix), 32 x 32 tile pairs through shared memory so
// both the tile and its mirror are read and written along rows.  Block (bj, bi, matrix) with
// bi <= bj takes tiles (bi, bj) and (bj, bi); the diagonal is left as it is.
__global__ void __launch_bounds__(256) symmetrize_kernel(float* S, int k, long long stride) {
    const int bj = blockIdx.x, bi = blockIdx.y;
    if (bi > bj) return;
    __shared__ float up[32][33], lo[32][33];
    float* s = S + blockIdx.z * stride;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;   // 32 x 8
    for (int r = ty; r < 32; r += 8) {
        const int i = bi * 32 + r, j = bj * 32 + tx;   // upper tile, row-wise
        const int i2 = bj * 32 + r, j2 = bi * 32 + tx; // its mirror, row-wise
        up[r][tx] = (i < k && j < k) ? s[static_cast<long long>(i) * k + j] : 0.f;
        lo[r][tx] = (i2 < k && j2 < k) ? s[static_cast<long long>(i2) * k + j2] : 0.f;
    }
    __syncthreads();
    for (int r = ty; r < 32; r += 8) {
        // (i, j) in the upper tile with j > i: s[i][j] = s[j][i] = 0.5 (s[i][j] + s[j][i]),
        // s[j][i] being lo[tx][r]
        const int i = bi * 32 + r, j = bj * 32 + tx;
        if (i < k && j < k && j > i) s[static_cast<long long>(i) * k + j] = 0.5f * (up[r][tx] + lo[tx][r]);
        // mirror row i2 = bj*32 + r, column j2 = bi*32 + tx: the value of (j2, i2) upper pair
        const int i2 = bj * 32 + r, j2 = bi * 32 + tx;
        if (i2 < k && j2 < k && i2 > j2) s[static_cast<long long>(i2) * k + j2] = 0.5f * (up[tx][r] + lo[r][tx]);
    }
}

__global__ void aug_neg_transpose_kernel(double* Aug, int k, long long ld, long long stride) {
    double* a = Aug + blockIdx.y * stride;
    const long long total = static_cast<long long>(k) * k;
    for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < total;
         e += static_cast<long long>(gridDim.x) * blockDim.x) {
        const int i = static_cast<int>(e / k), j = static_cast<int>(e % k);
        a[(k + static_cast<long long>(i)) * ld + k + j] = -a[static_cast<long long>(j) * ld + i];
    }
}

// Right-hand side of the Woodbury solve: columns 2k..3k-1 <- columns k..2k-1, all 2k rows.
__global__ void aug_copy_rhs_kernel(double* Aug, int k, long long ld, long long stride) {
    double* a = Aug + blockIdx.y * stride;
    const long long total = 2LL * k * k;
    for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < total;
         e += static_cast<long long>(gridDim.x) * blockDim.x) {
        const long long i = e / k, j = e % k;
        a[i * ld + 2LL * k + j] = a[i * ld + k + j];
    }
}

// Adds the identity to the first 2k columns: Aug[i][i] += 1.
__global__ void aug_add_identity_kernel(double* Aug, int n2k, long long ld, long long stride) {
    double* a = Aug + blockIdx.y * stride;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n2k; i += gridDim.x * blockDim.x)
        a[static_cast<long long>(i) * ld + i] += 1.0;
}

// MuonCayley momentum (§4.3): M <- beta*M + (1 - beta)*G, elementwise over the batch.
__global__ void ema_kernel(float* __restrict__ M, const float* __restrict__ G, long long total, float beta) {
    const float omb = 1.0f - beta;
    for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < total;
         e += static_cast<long long>(gridDim.x) * blockDim.x)
        M[e] = fmaf(beta, M[e], omb * G[e]);
}

// cm[b][j] = mean over the n rows of column j of M[b] (fp64 sum), one thread per column.
__global__ void column_mean_kernel(const float* __restrict__ M, double* __restrict__ cm, int n, int k) {
    const int j = blockIdx.x * blockDim.x + threadIdx.x;
    const int b = blockIdx.y;
    if (j >= k) return;
    const float* m = M + static_cast<long long>(b) * n * k;
    double s = 0.0;
    for (int i = 0; i < n; ++i) s += m[static_cast<long long>(i) * k + j];
    cm[static_cast<long long>(b) * k + j] = s / n;
}

// D[b] = M[b] - cm[b] broadcast over rows (or a copy of M when cm is null).
__global__ void center_kernel(const float* __restrict__ M, const double* __restrict__ cm, float* __restrict__ D,
                              int n, int k, long long total) {
    for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < total;
         e += static_cast<long long>(gridDim.x) * blockDim.x) {
        if (cm == nullptr) {
            D[e] = M[e];
        } else {
            const long long b = e / (static_cast<long long>(n) * k);
            const int j = static_cast<int>(e % k);
            D[e] = static_cast<float>(static_cast<double>(M[e]) - cm[b * k + j]);
        }
    }
}

// Batched fp32 transpose, out[b] (cols x rows) = in[b]^T with in[b] rows x cols: 32 x 32
// tiles staged in shared memory (one padding column against bank conflicts) so that both
// the reads and the writes are row-contiguous.  Block 32 x 8, grid
// (ceil(cols/32), ceil(rows/32), batch).
__global__ void __launch_bounds__(256) transpose_kernel(const float* __restrict__ in, float* __restrict__ out,
                                                        int rows, int cols) {
    __shared__ float t[32][33];
    const long long off = static_cast<long long>(blockIdx.z) * rows * cols;
    const int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
    for (int i = threadIdx.y; i < 32; i += 8) {
        const int r = r0 + i, c = c0 + threadIdx.x;
        if (r < rows && c < cols) t[i][threadIdx.x] = in[off + static_cast<long long>(r) * cols + c];
    }
    __syncthreads();
    for (int i = threadIdx.y; i < 32; i += 8) {
        const int c = c0 + i, r = r0 + threadIdx.x;
        if (c < cols && r < rows) out[off + static_cast<long long>(c) * rows + r] = t[threadIdx.x][i];
    }
}

// out = alpha * sum_j part_j + beta * E, the chunk partials summed in fp64 in order j = 0..
struct SplitKItem {
    const float* part;   // nsplit consecutive M x N fp32 partials
    void* out;
    const void* E;
    long long ld_out, ld_e;
    long long block0;
    int M, N, nsplit;
    float alpha, beta;
    int out_f64, e_f64;
    int vec4;   // four consecutive elements per thread (N % 4 == 0, 16-byte aligned rows)
};
__global__ void splitk_reduce_kernel(const SplitKItem* __restrict__ items, int count) {
    const long long b = blockIdx.x;
    int lo = 0, hi = count - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (items[mid].block0 <= b) lo = mid; else hi = mid - 1;
    }
    const SplitKItem& it = items[lo];
    const long long mn = static_cast<long long>(it.M) * it.N;
    if (it.vec4) {   // the same sums, four columns of one row per thread
        const long long e = ((b - it.block0) * blockDim.x + threadIdx.x) * 4;
        if (e >= mn) return;
        double s4[4] = {0.0, 0.0, 0.0, 0.0};
        for (int j = 0; j < it.nsplit; ++j) {
            const float4 q = *reinterpret_cast<const float4*>(it.part + j * mn + e);
            s4[0] += static_cast<double>(q.x); s4[1] += static_cast<double>(q.y);
            s4[2] += static_cast<double>(q.z); s4[3] += static_cast<double>(q.w);
        }
        const long long m = e / it.N, nn = e % it.N;
        double v[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = static_cast<double>(it.alpha) * s4[i];
        if (it.beta != 0.f) {
            const long long eo = m * it.ld_e + nn;
#pragma unroll
            for (int i = 0; i < 4; ++i)
                v[i] += static_cast<double>(it.beta) * (it.e_f64 ? static_cast<const double*>(it.E)[eo + i]
                                                              : static_cast<double>(static_cast<const float*>(it.E)[eo + i]));
        }
        const long long oo = m * it.ld_out + nn;
        if (it.out_f64) {
            double2* o = reinterpret_cast<double2*>(static_cast<double*>(it.out) + oo);
            o[0] = make_double2(v[0], v[1]);
            o[1] = make_double2(v[2], v[3]);
        } else {
            *reinterpret_cast<float4*>(static_cast<float*>(it.out) + oo) =
                make_float4(static_cast<float>(v[0]), static_cast<float>(v[1]), static_cast<float>(v[2]), static_cast<float>(v[3]));
        }
        return;
    }
    const long long e = (b - it.block0) * blockDim.x + threadIdx.x;
    if (e >= mn) return;
    double sum = 0.0;
    for (int j = 0; j < it.nsplit; ++j) sum += static_cast<double>(it.part[j * mn + e]);
    const long long m = e / it.N, nn = e % it.N;
    double v = static_cast<double>(it.alpha) * sum;
    if (it.beta != 0.f) {
        const long long eo = m * it.ld_e + nn;
        v += static_cast<double>(it.beta) *
             (it.e_f64 ? static_cast<const double*>(it.E)[eo] : static_cast<double>(static_cast<const float*>(it.E)[eo]));
    }
    const long long oo = m * it.ld_out + nn;
    if (it.out_f64) static_cast<double*>(it.out)[oo] = v;
    else static_cast<float*>(it.out)[oo] = static_cast<float>(v);
}

// Exact three-way bf16 split of an fp32 value (fp64 sources are first rounded to fp32):
// x = hi + mid + lo with hi = bf16(x), mid = bf16(x - hi), lo = x - hi - mid (8 bits each).
struct Split3Item {
    const void* src;
    __nv_bfloat16* dst;   // 3 planes of rows x cols, contiguous
    long long ld;
    long long block0;
    int rows, cols;
    int src_f64;
    int vec4;   // four consecutive elements per thread (cols % 4 == 0, aligned rows)
};
__global__ void split3_kernel(const Split3Item* __restrict__ items, int count) {
    const long long b = blockIdx.x;
    int lo = 0, hi = count - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (items[mid].block0 <= b) lo = mid; else hi = mid - 1;
    }
    const Split3Item& it = items[lo];
    const long long n = static_cast<long long>(it.rows) * it.cols;
    auto split = [](float x, __nv_bfloat16& h, __nv_bfloat16& m, __nv_bfloat16& l) {
        h = __float2bfloat16_rn(x);
        const float r1 = x - __bfloat162float(h);
        m = __float2bfloat16_rn(r1);
        const float r2 = r1 - __bfloat162float(m);
        l = __float2bfloat16_rn(r2);
    };
    if (it.vec4) {   // four columns of one row per thread
        const long long e = ((b - it.block0) * blockDim.x + threadIdx.x) * 4;
        if (e >= n) return;
        const long long r = e / it.cols, c = e % it.cols;
        float x[4];
        if (it.src_f64) {
            const double2* p = reinterpret_cast<const double2*>(static_cast<const double*>(it.src) + r * it.ld + c);
            const double2 a = p[0], d = p[1];
            x[0] = static_cast<float>(a.x); x[1] = static_cast<float>(a.y);
            x[2] = static_cast<float>(d.x); x[3] = static_cast<float>(d.y);
        } else {
            const float4 q = *reinterpret_cast<const float4*>(static_cast<const float*>(it.src) + r * it.ld + c);
            x[0] = q.x; x[1] = q.y; x[2] = q.z; x[3] = q.w;
        }
        __nv_bfloat16 h[4], m[4], l[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) split(x[i], h[i], m[i], l[i]);
        auto put = [&](__nv_bfloat16* dst, const __nv_bfloat16 (&v)[4]) {
            __nv_bfloat162 p0, p1;
            p0.x = v[0]; p0.y = v[1]; p1.x = v[2]; p1.y = v[3];
            uint2 u;
            u.x = *reinterpret_cast<const uint32_t*>(&p0);
            u.y = *reinterpret_cast<const uint32_t*>(&p1);
            *reinterpret_cast<uint2*>(dst + e) = u;
        };
        put(it.dst, h);
        put(it.dst + n, m);
        put(it.dst + 2 * n, l);
        return;
    }
    const long long e = (b - it.block0) * blockDim.x + threadIdx.x;
    if (e >= n) return;
    const long long r = e / it.cols, c = e % it.cols;
    const float x = it.src_f64 ? static_cast<float>(static_cast<const double*>(it.src)[r * it.ld + c])
                               : static_cast<const float*>(it.src)[r * it.ld + c];
    __nv_bfloat16 h, m, l;
    split(x, h, m, l);
    it.dst[e] = h;
    it.dst[n + e] = m;
    it.dst[2 * n + e] = l;
}

// fp32 copy of a k x k block of an fp64 matrix (the same round-to-nearest the SIMT GEMM
// applies when it loads an fp64 operand), so the product that reads it can take the fp32
// multi-stage GEMM.
struct BlockCastItem {
    const double* src;
    float* dst;           // rows x cols, contiguous
    long long ld;         // source row pitch
    long long block0;
    int rows, cols;
    int vec4;             // four consecutive elements per thread (cols % 4 == 0, aligned rows)
};
__global__ void block_cast_kernel(const BlockCastItem* __restrict__ items, int count) {
    const long long b = blockIdx.x;
    int lo = 0, hi = count - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (items[mid].block0 <= b) lo = mid; else hi = mid - 1;
    }
    const BlockCastItem& it = items[lo];
    const long long n = static_cast<long long>(it.rows) * it.cols;
    if (it.vec4) {
        const long long e = ((b - it.block0) * blockDim.x + threadIdx.x) * 4;
        if (e >= n) return;
        const long long r = e / it.cols, c = e % it.cols;
        const double2* p = reinterpret_cast<const double2*>(it.src + r * it.ld + c);
        const double2 a = p[0], d = p[1];
        *reinterpret_cast<float4*>(it.dst + e) =
            make_float4(static_cast<float>(a.x), static_cast<float>(a.y), static_cast<float>(d.x), static_cast<float>(d.y));
        return;
    }
    const long long e = (b - it.block0) * blockDim.x + threadIdx.x;
    if (e >= n) return;
    const long long r = e / it.cols, c = e % it.cols;
    it.dst[e] = static_cast<float>(it.src[r * it.ld + c]);
}

// Panel factorisation (partial pivoting) of rows j0..N-1, columns j0..j0+nb-1, held in
// shared memory column by column with an odd pitch (consecutive rows in consecutive words,
// so the per-row sweeps are free of bank conflicts).  Records the pivot row of each column
// in piv (absolute row indices).
__host__ __device__ constexpr int panel_pitch(int rows) { return rows | 1; }
constexpr int kPanelMax = 32;   // widest panel (columns)
// 8-byte global -> shared copy, zero-filled beyond src_bytes (0 or 8).
__device__ __forceinline__ void cp_async8(double* smem_dst, const double* gmem_src, int src_bytes) {
    const unsigned d = static_cast<unsigned>(__cvta_generic_to_shared(smem_dst));
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(d), "l"(gmem_src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Warp-wide argmax: every lane ends with the largest v and, among lanes holding it, the
// smallest i (v >= -1, never NaN).
__device__ __forceinline__ void warp_argmax(double& v, int& i) {
    double m = v;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, o));
    i = static_cast<int>(__reduce_min_sync(0xffffffffu, v == m ? static_cast<unsigned>(i) : 0x7fffffffu));
    v = m;
}

// One CTA per system; with the cluster kernel taking the block columns over 1000 rows, 512
// threads (two rows each) measured faster than 1024 or 256.
constexpr int kPanelThreads = 512;
__global__ void __launch_bounds__(kPanelThreads)
lu_panel_kernel(double* Aug, long long ld, long long stride, int N, int j0, int nb, int* piv, long long piv_stride,
                unsigned* status) {
    extern __shared__ double pan[];  // nb columns of panel_pitch(N - j0)
    __shared__ double red_v[32];
    __shared__ int red_i[32];
    __shared__ int s_p;
    double* a = Aug + blockIdx.x * stride;
    int* pv = piv + blockIdx.x * piv_stride;
    const int rows = N - j0;
    const int pitch = panel_pitch(rows);
    const int tid = threadIdx.x, nt = blockDim.x;
    // cp.async: every copy in flight at once (a register round trip per element would order
    // each global load behind the previous shared store)
    for (int e = tid; e < rows * nb; e += nt) {
        const int r = e / nb, c = e % nb;
        cp_async8(pan + c * pitch + r, a + (j0 + static_cast<long long>(r)) * ld + j0 + c, 8);
    }
    cp_async_wait_all();
    __syncthreads();
    for (int jj = 0; jj < nb; ++jj) {
        const double* colj = pan + jj * pitch;
        // argmax |pan(r, jj)| over r >= jj (ties: smallest row)
        double best = -1.0;
        int bi = jj;
        for (int r = jj + tid; r < rows; r += nt) {
            const double v = fabs(colj[r]);
            if (v > best) { best = v; bi = r; }
        }
        warp_argmax(best, bi);   // (largest |a|, then smallest row) over the warp
        if ((tid & 31) == 0) { red_v[tid >> 5] = best; red_i[tid >> 5] = bi; }
        __syncthreads();
        if (tid < 32) {
            best = tid < (nt >> 5) ? red_v[tid] : -1.0;
            bi = tid < (nt >> 5) ? red_i[tid] : jj;
            warp_argmax(best, bi);
            if (tid == 0) {
                s_p = bi;
                pv[j0 + jj] = j0 + bi;
                if (!(best > 0.0) || !isfinite(best)) atomicOr(status, kDevErrNonfinite);
            }
        }
        __syncthreads();
        const int p = s_p;
        if (p != jj && tid < nb) {
            double* cc = pan + tid * pitch;
            const double t = cc[jj];
            cc[jj] = cc[p];
            cc[p] = t;
        }
        __syncthreads();
        // rows in pairs (r, r + nt): each pivot-row value is read once for both, and the column
        // loop runs four columns per trip (the kernel is issue-bound)
        const double piv_v = colj[jj];
        for (int r = jj + 1 + tid; r < rows; r += 2 * nt) {
            const int r1 = r + nt;
            const bool two = r1 < rows;
            const double l0 = colj[r] / piv_v;
            const double l1 = two ? colj[r1] / piv_v : 0.0;
            pan[jj * pitch + r] = l0;
            if (two) pan[jj * pitch + r1] = l1;
            double* p0 = pan + (jj + 1) * pitch + r;
            const double* u = pan + (jj + 1) * pitch + jj;
            int c = jj + 1;
            for (; c + 3 < nb; c += 4, p0 += 4 * pitch, u += 4 * pitch) {
                const double u0 = u[0], u1 = u[pitch], u2 = u[2 * pitch], u3 = u[3 * pitch];
                const double a0 = p0[0], a1 = p0[pitch], a2 = p0[2 * pitch], a3 = p0[3 * pitch];
                p0[0] = fma(-l0, u0, a0);
                p0[pitch] = fma(-l0, u1, a1);
                p0[2 * pitch] = fma(-l0, u2, a2);
                p0[3 * pitch] = fma(-l0, u3, a3);
                if (two) {
                    double* q = p0 + nt;
                    const double b0 = q[0], b1 = q[pitch], b2 = q[2 * pitch], b3 = q[3 * pitch];
                    q[0] = fma(-l1, u0, b0);
                    q[pitch] = fma(-l1, u1, b1);
                    q[2 * pitch] = fma(-l1, u2, b2);
                    q[3 * pitch] = fma(-l1, u3, b3);
                }
            }
            for (; c < nb; ++c, p0 += pitch, u += pitch) {
                const double uc = u[0];
                p0[0] = fma(-l0, uc, p0[0]);
                if (two) p0[nt] = fma(-l1, uc, p0[nt]);
            }
        }
        __syncthreads();
    }
    for (int e = tid; e < rows * nb; e += nt) {
        const int r = e / nb, c = e % nb;
        a[(j0 + static_cast<long long>(r)) * ld + j0 + c] = pan[c * pitch + r];
    }
}

// The same panel factorisation spread over a cluster of kPanelCluster CTAs per system: CTA c
// holds panel rows [c * rp, (c + 1) * rp) in shared memory (column by column, odd pitch),
// each with its logical row index (a pivot swaps two logical indices; the rows stay where
// they are, and the write-back puts every row at its logical place).  Per column, one cluster
// barrier: before it, each CTA writes its candidate (largest |a| over its live rows, smallest
// logical row on ties) together with that row's nb values into every CTA's shared memory
// (two buffers, alternating by column); after it, every CTA takes the same pivot, reads the
// pivot row from its own copy, and eliminates its own live rows.  The pivot choice and the
// arithmetic per element are those of lu_panel_kernel (l = a / pivot, then a - l u column by
// column), so results equal it for the same panel width.
constexpr int kPanelCluster = 8, kPanelClusterThreads = 256;
__host__ __device__ constexpr int panel_cluster_rows(int rows) { return (rows + kPanelCluster - 1) / kPanelCluster; }
// Shared memory of lu_panel_cluster_kernel beyond the nb panel columns: the candidate rows,
// then the rows' logical indices.
__host__ __device__ constexpr size_t panel_cluster_extra_bytes(int rp) {
    return static_cast<size_t>(2 * kPanelCluster * kPanelMax) * sizeof(double) + static_cast<size_t>(rp) * sizeof(int);
}
__global__ void __launch_bounds__(kPanelClusterThreads)
lu_panel_cluster_kernel(double* Aug, long long ld, long long stride, int N, int j0, int nb, int* piv,
                        long long piv_stride, unsigned* status) {
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    extern __shared__ double pan[];   // nb columns of panel_pitch(rp), candidate rows, logical rows
    constexpr int W = kPanelClusterThreads / 32;
    __shared__ double red_v[W];
    __shared__ int red_i[W], red_r[W];
    __shared__ double cand_v[2][kPanelCluster];
    __shared__ int cand_i[2][kPanelCluster];
    __shared__ int s_row;   // this CTA's candidate row (local index)
    const int me = static_cast<int>(cluster.block_rank());
    const int sys = static_cast<int>(blockIdx.x) / kPanelCluster;
    double* a = Aug + sys * stride;
    int* pv = piv + sys * piv_stride;
    const int rows = N - j0;
    const int rp = panel_cluster_rows(rows);
    const int pitch = panel_pitch(rp);
    const int r_lo = me * rp;
    const int nr = max(0, min(rows - r_lo, rp));   // this CTA's rows
    double* cand_row = pan + static_cast<size_t>(nb) * pitch;             // [2][kPanelCluster][kPanelMax]
    int* lidx = reinterpret_cast<int*>(cand_row + 2 * kPanelCluster * kPanelMax);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int e = tid; e < nr * nb; e += kPanelClusterThreads) {
        const int r = e / nb, c = e % nb;
        cp_async8(pan + c * pitch + r, a + (j0 + static_cast<long long>(r_lo + r)) * ld + j0 + c, 8);
    }
    for (int r = tid; r < nr; r += kPanelClusterThreads) lidx[r] = r_lo + r;
    cp_async_wait_all();
    __syncthreads();
    for (int jj = 0; jj < nb; ++jj) {
        const int buf = jj & 1;
        const double* colj = pan + jj * pitch;
        // this CTA's candidate; a NaN ranks as -1, so an all-NaN column pivots on logical row jj
        double best = -1.0;
        int bl = 0x7fffffff, br = 0;
        for (int r = tid; r < nr; r += kPanelClusterThreads) {
            const int li = lidx[r];
            if (li < jj) continue;
            double v = fabs(colj[r]);
            if (!(v >= 0.0)) v = -1.0;
            if (v > best || (v == best && li < bl)) { best = v; bl = li; br = r; }
        }
        double wv = best;
        int wl = bl;
        warp_argmax(wv, wl);
        const int wr = __shfl_sync(0xffffffffu, br, __ffs(__ballot_sync(0xffffffffu, best == wv && bl == wl)) - 1);
        if (lane == 0) { red_v[warp] = wv; red_i[warp] = wl; red_r[warp] = wr; }
        __syncthreads();
        if (warp == 0) {
            double v = lane < W ? red_v[lane] : -1.0;
            int l = lane < W ? red_i[lane] : 0x7fffffff;
            const double v0 = v;
            const int l0 = l;
            warp_argmax(v, l);
            const int src = __ffs(__ballot_sync(0xffffffffu, v0 == v && l0 == l)) - 1;
            const int r = __shfl_sync(0xffffffffu, lane < W ? red_r[lane] : 0, src);
            if (lane == 0) s_row = r;
            if (lane < kPanelCluster) {   // this CTA's candidate into every CTA's slot `me`
                *cluster.map_shared_rank(&cand_v[buf][me], lane) = v;
                *cluster.map_shared_rank(&cand_i[buf][me], lane) = l;
            }
        }
        __syncthreads();
        {   // the candidate row's values into every CTA's slot `me` (zeros when this CTA has no live row)
            const int r = s_row;
            const bool any = nr > 0;
            for (int e = tid; e < nb * kPanelCluster; e += kPanelClusterThreads) {
                const int c = e % nb, dst = e / nb;
                const double val = any ? pan[c * pitch + r] : 0.0;
                *cluster.map_shared_rank(cand_row + (buf * kPanelCluster + me) * kPanelMax + c, dst) = val;
            }
        }
        cluster.sync();
        double gv = lane < kPanelCluster ? cand_v[buf][lane] : -1.0;
        int lp = lane < kPanelCluster ? cand_i[buf][lane] : 0x7fffffff;
        const double gv0 = gv;
        const int lp0 = lp;
        warp_argmax(gv, lp);   // every warp of every CTA reaches the same pivot
        const int w = __ffs(__ballot_sync(0xffffffffu, gv0 == gv && lp0 == lp)) - 1;   // the CTA holding it
        const double* prow = cand_row + (buf * kPanelCluster + w) * kPanelMax;
        if (me == 0 && tid == 0) {
            pv[j0 + jj] = j0 + lp;
            if (!(gv > 0.0) || !isfinite(gv)) atomicOr(status, kDevErrNonfinite);
        }
        const int pr = (w == me) ? s_row : -1;   // the pivot row here (local index), if any
        const double piv_v = prow[jj];
        for (int r = tid; r < nr; r += kPanelClusterThreads) {
            const int li = lidx[r];
            if (r == pr) { lidx[r] = jj; continue; }
            if (li < jj) continue;
            if (li == jj) lidx[r] = lp;   // the row the pivot displaces takes its logical place
            const double l = colj[r] / piv_v;
            pan[jj * pitch + r] = l;
            for (int c = jj + 1; c < nb; ++c) pan[c * pitch + r] = fma(-l, prow[c], pan[c * pitch + r]);
        }
        __syncthreads();
    }
    for (int e = tid; e < nr * nb; e += kPanelClusterThreads) {
        const int r = e / nb, c = e % nb;
        a[(j0 + static_cast<long long>(lidx[r])) * ld + j0 + c] = pan[c * pitch + r];
    }
    cluster.sync();   // no CTA leaves while a peer may still write into its shared memory
}

// Triangular solves on right-hand columns held in registers.  Each column is shared by G
// consecutive lanes of a warp: lane h of the group holds rows G*m + h (m < R/G), so every
// lane keeps R/G values and all indices are compile-time.  The triangle sits in shared
// memory column by column (element (i, l) at T[l * P + i]), zero beyond its live size, so
// padded rows stay zero.  Both solves are right-looking: once x_l is final its owner lane
// hands it to the group (one shuffle) and all remaining rows take its term at once.
template <int R, int G, int P>
__device__ __forceinline__ void solve_unit_lower(double (&x)[R / G], const double* __restrict__ T, int h) {
    const int lane = threadIdx.x & 31;
    const double* Th = T + h;
#pragma unroll
    for (int l = 0; l < R - 1; ++l) {
        const double xl = __shfl_sync(0xffffffffu, x[l / G], (lane & ~(G - 1)) | (l % G));
#pragma unroll
        for (int m = 0; m < R / G; ++m) {
            if (G * m + G - 1 <= l) continue;               // all rows of slot m are at or above l
            if (G * m > l || h > l - G * m) x[m] = fma(-Th[l * P + G * m], xl, x[m]);
        }
    }
}
// Upper triangle; dinv holds the reciprocals of its diagonal (zero on padded rows).
template <int R, int G, int P>
__device__ __forceinline__ void solve_upper(double (&x)[R / G], const double* __restrict__ T,
                                            const double* __restrict__ dinv, int h) {
    const int lane = threadIdx.x & 31;
    const double* Th = T + h;
#pragma unroll
    for (int l = R - 1; l >= 0; --l) {
        if (h == l % G) x[l / G] *= dinv[l];
        const double xl = __shfl_sync(0xffffffffu, x[l / G], (lane & ~(G - 1)) | (l % G));
#pragma unroll
        for (int m = 0; m < R / G; ++m) {
            if (G * m >= l) continue;                       // all rows of slot m are at or below l
            if (G * m + G - 1 < l || h < l - G * m) x[m] = fma(-Th[l * P + G * m], xl, x[m]);
        }
    }
}

// Copies the w x w block at (r0, r0) of a into T column by column (pitch P, zero-padded to
// R x R); reads run along rows of a.
template <int R, int P>
__device__ __forceinline__ void load_block_cols(double* T, const double* a, long long ld, int r0, int w) {
    for (int e = threadIdx.x; e < R * R; e += blockDim.x) {
        const int i = e / R, l = e % R;
        const bool in = i < w && l < w;
        cp_async8(T + l * P + i, in ? a + (r0 + static_cast<long long>(i)) * ld + r0 + l : a, in ? 8 : 0);
    }
    cp_async_wait_all();
}

// Lane h's rows r0 + G*m + h (< r0 + w) of the column starting at p (pitch ld), zero beyond.
template <int R, int G>
__device__ __forceinline__ void load_column(double (&x)[R / G], const double* p, long long ld, int w, int h) {
    p += h * ld;
#pragma unroll
    for (int m = 0; m < R / G; ++m) {
        x[m] = G * m + h < w ? *p : 0.0;
        p += G * ld;
    }
}
template <int R, int G>
__device__ __forceinline__ void store_column(const double (&x)[R / G], double* p, long long ld, int w, int h) {
    p += h * ld;
#pragma unroll
    for (int m = 0; m < R / G; ++m) {
        if (G * m + h < w) *p = x[m];
        p += G * ld;
    }
}

// Row swaps then unit-lower solve U12 = L11^-1 A12 with the w x w triangle at (r0, r0), for
// the columns [c_lo, ncols) -- blockDim.x / G columns per block.  The interchanges of rows
// r0..r0+w-1 (in order) are applied as one permutation: thread 0 replays them on row indices
// in shared memory (cur[x - r0] = the original row that ends at row x), then every column
// gathers its w rows, and the rows below the block that receive one, with independent loads
// before it stores anything.  (Applied swap by swap, each column's 2w loads would wait on one
// another through the stores between them.)  iw holds nrows - r0 + 2R ints of shared memory;
// every lane of a warp reaches the shuffles.
template <int R, int G>
__device__ __forceinline__ void swap_trsm_block(double* a, long long ld, const int* pv, int r0, int w, int c_first,
                                                int c_end, bool solve, int nrows, double* T, int* iw) {
    constexpr int P = R + 2;
    __shared__ int s_nm;
    int* mv = iw;              // R destinations, then R sources, of rows below the block
    int* cur = iw + 2 * R;     // nrows - r0 entries
    for (int x = threadIdx.x; x < nrows - r0; x += blockDim.x) cur[x] = r0 + x;
    for (int i = threadIdx.x; i < w; i += blockDim.x) mv[i] = pv[r0 + i];   // the pivots, for thread 0
    if (solve) load_block_cols<R, P>(T, a, ld, r0, w);
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int i = 0; i < w; ++i) {
            const int p = mv[i];
            if (p != r0 + i && p > r0 + i && p < nrows) {
                const int t = cur[i];
                cur[i] = cur[p - r0];
                cur[p - r0] = t;
            }
        }
        int nm = 0;
        for (int i = 0; i < w; ++i) {
            const int p = mv[i];
            if (p >= r0 + w && p < nrows && cur[p - r0] != p) {
                mv[R + nm] = cur[p - r0];   // source (mv[nm] below is overwritten only after mv[i] is read)
                cur[p - r0] = p;            // recorded once
                mv[nm] = p;
                ++nm;
            }
        }
        s_nm = nm;
    }
    __syncthreads();
    const int nm = s_nm;
    const int c = c_first + static_cast<int>(threadIdx.x) / G;
    const int h = static_cast<int>(threadIdx.x) % G;
    const bool live = c < c_end;
    double* col = a + (live ? c : c_first);
    double x[R / G], y[R / G];
#pragma unroll
    for (int m = 0; m < R / G; ++m) {
        const int row = G * m + h;
        x[m] = (live && row < w) ? col[static_cast<long long>(cur[row]) * ld] : 0.0;
        y[m] = (live && row < nm) ? col[static_cast<long long>(mv[R + row]) * ld] : 0.0;
    }
#pragma unroll
    for (int m = 0; m < R / G; ++m) {
        const int j = G * m + h;
        if (live && j < nm) col[static_cast<long long>(mv[j]) * ld] = y[m];
    }
    if (solve) solve_unit_lower<R, G, P>(x, T, h);   // uniform across the block
#pragma unroll
    for (int m = 0; m < R / G; ++m) {
        const int row = G * m + h;
        if (live && row < w) col[(r0 + static_cast<long long>(row)) * ld] = x[m];
    }
}

// Shared memory of swap_trsm_block beyond the triangle: 2R ints plus one per row from r0 on.
__host__ __device__ constexpr size_t swap_ints_bytes(int R, int rows_from_r0) {
    return (2 * static_cast<size_t>(R) + static_cast<size_t>(rows_from_r0)) * sizeof(int);
}

// After a panel j0..j0+nb-1 of the block column starting at c_left: the panel's row swaps,
// applied to the block's earlier multiplier columns [c_left, j0) (blocks 0 .. left_blocks - 1)
// and, with the solve U12 = L11^-1 A12 by the unit-lower nb x nb triangle L11, to the block's
// columns [j0 + nb, ncols) (the remaining blocks).  nb <= kPanelMax.
constexpr int kPanelLanes = 2, kPanelSwapThreads = 128;
constexpr int kPanelSwapCols = kPanelSwapThreads / kPanelLanes;
constexpr size_t kPanelTriangleBytes = static_cast<size_t>(kPanelMax) * (kPanelMax + 2) * sizeof(double);
__global__ void __launch_bounds__(kPanelSwapThreads)
lu_swap_trsm_kernel(double* Aug, long long ld, long long stride, int c_left, int left_blocks, int j0, int nb,
                    int ncols, const int* piv, long long piv_stride) {
    extern __shared__ __align__(16) double T[];
    int* iw = reinterpret_cast<int*>(T + kPanelMax * (kPanelMax + 2));
    const bool left = static_cast<int>(blockIdx.x) < left_blocks;
    const int c_first = left ? c_left + static_cast<int>(blockIdx.x) * kPanelSwapCols
                             : j0 + nb + (static_cast<int>(blockIdx.x) - left_blocks) * kPanelSwapCols;
    swap_trsm_block<kPanelMax, kPanelLanes>(Aug + blockIdx.y * stride, ld, piv + blockIdx.y * piv_stride, j0, nb,
                                            c_first, left ? j0 : ncols, !left, static_cast<int>(piv_stride), T, iw);
}

// After a block column J0..J0+JB-1 is factorised: for every column c >= c_lo, apply the
// block's JB row swaps in order, then solve with the JB x JB unit-lower L11 (U12 = L11^-1 A12).
// The 128 x 128 triangle (133 KB) is in dynamic shared memory, shared by the block's 128
// columns (512 threads, 4 lanes per column, 32 rows per lane: measured faster than 8 or 16
// lanes, whose blocks reload the triangle and replay the swaps for fewer columns).
constexpr int kLuBlock = 128, kLuLanes = 4, kTrsmThreads = 512;
constexpr size_t kLuTriangleBytes = static_cast<size_t>(kLuBlock) * (kLuBlock + 2) * sizeof(double);
constexpr int kMaxAugRows = 2 * 4096;   // 2k for the largest k the entry points accept
__global__ void __launch_bounds__(kTrsmThreads)
lu_block_swap_trsm_kernel(double* Aug, long long ld, long long stride, int J0, int JB, int c_lo, int ncols,
                          const int* piv, long long piv_stride) {
    extern __shared__ __align__(16) double T[];
    int* iw = reinterpret_cast<int*>(T + kLuBlock * (kLuBlock + 2));
    swap_trsm_block<kLuBlock, kLuLanes>(Aug + blockIdx.y * stride, ld, piv + blockIdx.y * piv_stride, J0, JB,
                                        c_lo + static_cast<int>(blockIdx.x) * (kTrsmThreads / kLuLanes), ncols, true,
                                        static_cast<int>(piv_stride), T, iw);
}

// Back substitution on one diagonal block: rows i0..i0+bs-1 of the right-hand columns
// (starting at column rhs0, nrhs of them) <- U_ii^-1 (same rows); 128 columns per block of 512
// threads, the triangle and the reciprocals of its diagonal in dynamic shared memory.
constexpr int kBackBlock = 128, kBackLanes = 4, kBackPitch = kBackBlock + 2;
constexpr size_t kBackSmemBytes = (static_cast<size_t>(kBackBlock) * kBackPitch + kBackBlock) * sizeof(double);
__global__ void __launch_bounds__(kTrsmThreads)
back_diag_kernel(double* Aug, long long ld, long long stride, int i0, int bs, int rhs0, int nrhs) {
    extern __shared__ __align__(16) double T[];
    double* dinv = T + kBackBlock * kBackPitch;
    double* a = Aug + blockIdx.y * stride;
    load_block_cols<kBackBlock, kBackPitch>(T, a, ld, i0, bs);
    for (int l = threadIdx.x; l < kBackBlock; l += blockDim.x)
        dinv[l] = l < bs ? 1.0 / a[(i0 + static_cast<long long>(l)) * ld + i0 + l] : 0.0;
    __syncthreads();
    const int c = static_cast<int>(blockIdx.x * (blockDim.x / kBackLanes) + threadIdx.x / kBackLanes);
    const int h = static_cast<int>(threadIdx.x) % kBackLanes;
    const bool live = c < nrhs;
    double* col = a + rhs0 + (live ? c : 0) + i0 * ld;
    const int wl = live ? bs : 0;
    double x[kBackBlock / kBackLanes];
    load_column<kBackBlock, kBackLanes>(x, col, ld, wl, h);
    solve_upper<kBackBlock, kBackLanes, kBackPitch>(x, T, dinv, h);
    store_column<kBackBlock, kBackLanes>(x, col, ld, wl, h);
}

// Shared memory of a panel: nb fp64 columns of panel_pitch(rows).  The widest panel (<= 32
// columns) that fits in kPanelSmem is used.
constexpr size_t kPanelSmem = 200 * 1024;
size_t lu_panel_smem(int rows, int nb) { return static_cast<size_t>(panel_pitch(rows)) * nb * sizeof(double); }
// Shared memory of the cluster panel kernel: this CTA's nb columns of panel_pitch(rows / 8),
// then the candidate rows and the logical row indices.
size_t lu_panel_cluster_smem(int rows, int nb) {
    const int rp = panel_cluster_rows(rows);
    return static_cast<size_t>(panel_pitch(rp)) * nb * sizeof(double) + panel_cluster_extra_bytes(rp);
}
int lu_panel_cluster_width(int rows) {
    const size_t per_col = static_cast<size_t>(panel_pitch(panel_cluster_rows(rows))) * sizeof(double);
    const int nb = static_cast<int>((kPanelSmem - panel_cluster_extra_bytes(panel_cluster_rows(rows))) / per_col);
    return std::max(1, std::min(kPanelMax, nb));
}
// Block columns taller than this factorise their panels on a cluster of kPanelCluster CTAs per
// system (32 columns wide, about 2.8 us per column whatever the height); shorter ones on one
// CTA per system, whose time per column falls with the height (about 3.6 us at 2048 rows,
// 1.8 us at 384).  Measured on 16 x 4096 x 1024: 1000 rows 37.44-37.55 ms per step, 1400 37.70,
// 1800 38.22, 800 37.44, 600 37.51, all on clusters 38.08, none 38.58.
constexpr int kPanelClusterMinRows = 1000;
int lu_panel_width(int rows) {
    const int nb = static_cast<int>(kPanelSmem / (static_cast<size_t>(panel_pitch(rows)) * sizeof(double)));
    return std::max(1, std::min(kPanelMax, nb));
}

struct StiefelLayout {
    size_t V, b, S, Aug, piv, cm, part, planes, table_offset, data_bytes;
    bool tc;
};

// The tensor-core plan needs 16-byte bf16 row pitches for TMA.
bool stiefel_tc_ok(int n, int k) { return n % 8 == 0 && k % 8 == 0; }
// bf16 planes per matrix: W, G (n x k) and S (k x k), 3 planes each.
size_t stiefel_plane_elems(int n, int k) {
    return 3 * (2 * static_cast<size_t>(n) * k + static_cast<size_t>(k) * k);
}

// Split-K for the reductions over n: chunks of kSplitK rows summed in fp32, chunk partial
// sums added in fp64 in a fixed order.
constexpr int kSplitK = 512;
int splitk_parts(int n) { return (n + kSplitK - 1) / kSplitK; }
StiefelLayout stiefel_layout(int batch, int n, int k) {
    Arena ar;
    StiefelLayout L;
    const size_t nk = static_cast<size_t>(n) * k * 4, kk = static_cast<size_t>(k) * k * 4;
    L.V = ar.take(nk * batch);
    L.b = ar.take(nk * batch);
    L.S = ar.take(kk * batch);
    L.Aug = ar.take(static_cast<size_t>(2 * k) * (3 * k) * sizeof(double) * batch);
    L.piv = ar.take(static_cast<size_t>(2 * k) * 4 * batch);
    L.cm = ar.take(static_cast<size_t>(k) * sizeof(double) * batch);
    // largest split-K group: the three k x k blocks P, Q, R of every matrix
    L.part = ar.take(static_cast<size_t>(3) * batch * splitk_parts(n) * k * k * sizeof(float));
    L.tc = stiefel_tc_ok(n, k);
    L.planes = L.tc ? ar.take(stiefel_plane_elems(n, k) * sizeof(__nv_bfloat16) * batch) : 0;
    L.data_bytes = align_up(ar.used, kAlign);
    L.table_offset = kHeaderBytes + L.data_bytes;
    return L;
}

// MuonCayley on a wide parameter (rows < cols) runs on the transpose: the Stiefel layout of
// the transposed shape plus the transposed W and momentum, ahead of the plan tables.
struct CayleyLayout {
    StiefelLayout st;
    size_t Wt = 0, Mt = 0;
};
CayleyLayout cayley_layout(int batch, int rows, int cols) {
    const bool wide = rows < cols;
    CayleyLayout C;
    C.st = stiefel_layout(batch, wide ? cols : rows, wide ? rows : cols);
    if (wide) {
        const size_t nk = static_cast<size_t>(rows) * cols * sizeof(float) * batch;
        C.Wt = C.st.data_bytes;
        C.Mt = align_up(C.Wt + nk, kAlign);
        C.st.data_bytes = align_up(C.Mt + nk, kAlign);
        C.st.table_offset = kHeaderBytes + C.st.data_bytes;
    }
    return C;
}

size_t stiefel_tables_bound(int batch, int n, int k) {
    const int N = 2 * k, nb = lu_panel_width(N);
    const int outer = (N + kLuBlock - 1) / kLuBlock;
    const int panels = outer * ((kLuBlock + nb - 1) / nb);   // panels never straddle a block column
    const int back = (N + kBackBlock - 1) / kBackBlock;
    auto tiles = [](long long M, long long Nn) { return ((M + kSimtBM - 1) / kSimtBM) * ((Nn + kSimtBN - 1) / kSimtBN); };
    long long t = 0;
    t += tiles(k, k) * 1 + tiles(n, k) * 1 + tiles(k, k) * 3 + tiles(n, k) * 2 + tiles(k, k) * 2 + tiles(n, k) * 2;
    for (int p = 0; p < panels; ++p) t += tiles(N, kLuBlock);
    for (int q = 0; q < outer; ++q) t += tiles(N - q * kLuBlock, 3LL * k - q * kLuBlock);
    for (int q = 0; q < back; ++q) t += tiles(static_cast<long long>(q) * kBackBlock, k);
    const int ns = splitk_parts(n);
    t += tiles(k, k) * 6LL * ns;                     // split-K partial products (S, P, Q, R, y)
    const long long probs = 12 + panels + outer + back + 6LL * ns + 6;
    // tensor-core products (S split-K chunks, V): tiles, tensor maps of 3 plane sets x 3
    // planes x 2 box shapes, split items
    t += (tiles(k, k) * ns + tiles(n, k)) * 2LL;
    const size_t tmaps = static_cast<size_t>(batch) * 3 * 3 * 2 * (sizeof(CUtensorMap) + 128);
    const size_t prob_bytes = std::max(sizeof(SimtProblem), sizeof(TcProblem)) + 16;
    size_t b = static_cast<size_t>(t) * batch * sizeof(uint32_t) + static_cast<size_t>(probs) * batch * prob_bytes +
               static_cast<size_t>(probs) * 2 * kAlign + tmaps + static_cast<size_t>(batch) * 16 * 64 + 64 * kAlign +
               static_cast<size_t>(batch) * 4 * sizeof(BlockCastItem) + 2 * kAlign;   // fp32 block copies
    return align_up(b + 4096, kAlign);
}

// Appends grouped SIMT GEMM launches to the plan (f64_acc: fp64 accumulation), at most
// kMaxTileProblems problems per launch.
void add_gemm(Plan& plan, TableImage& img, const std::vector<SimtProblem>& all, bool f64_acc = false) {
    for (size_t first = 0; first < all.size(); first += kMaxTileProblems) {
        const size_t last = std::min(all.size(), first + static_cast<size_t>(kMaxTileProblems));
        const std::vector<SimtProblem> probs(all.begin() + first, all.begin() + last);
        std::vector<uint32_t> tiles;
        double flops = 0;
        for (size_t p = 0; p < probs.size(); ++p) {
            const SimtProblem& P = probs[p];
            if (P.M <= 0 || P.N <= 0) continue;
            const int mbs = (P.M + kSimtBM - 1) / kSimtBM, nbs = (P.N + kSimtBN - 1) / kSimtBN;
            for (int nb = 0; nb < nbs; ++nb)
                for (int mb = 0; mb < mbs; ++mb)
                    if (!P.sym || nb >= mb) tiles.push_back(tile_code(static_cast<int>(p), mb, nb));
            flops += (P.sym ? 1.0 : 2.0) * P.M * P.N * P.K;
        }
        if (tiles.empty()) continue;
        const SimtProblem* dp = img.dev<SimtProblem>(img.add(probs.data(), probs.size() * sizeof(SimtProblem), kAlign));
        const uint32_t* dt = img.dev<uint32_t>(img.add(tiles.data(), tiles.size() * sizeof(uint32_t), kAlign));
        const int nt = static_cast<int>(tiles.size());
        bool a_kc = false;
        const bool async = !f64_acc && simt_async_suits(probs, &a_kc);
        const bool dmma = f64_acc && dmma_gemm_suits(probs);
        plan.steps.push_back({f64_acc ? MUON_KERNEL_SIMT_GEMM_F64 : MUON_KERNEL_SIMT_GEMM, flops, [=](cudaStream_t s) {
                                  if (dmma) return dmma_gemm_launch(dp, dt, nt, s);
                                  return async ? simt_gemm_async_launch(dp, dt, nt, s, a_kc)
                                               : simt_gemm_launch(dp, dt, nt, s, f64_acc);
                              }});
    }
}

// The same products with the reduction dimension split into kSplitK chunks: every chunk's
// fp32 partial goes to `part`, then one launch sums the partials in fp64 and applies
// alpha, beta and the output type of each original problem.
// Whether a split-K reduce item / a plane split may take four elements per thread (whole
// 16-byte vectors on every row), and the blocks of 256 threads it then needs.
bool splitk_vec4(const SplitKItem& it) {
    auto a16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    if (it.N % 4 != 0 || !a16(it.part) || !a16(it.out)) return false;
    return it.out_f64 ? it.ld_out % 2 == 0 : it.ld_out % 4 == 0;
}
bool split3_vec4(const Split3Item& it) {
    auto a16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    if (it.cols % 4 != 0 || (reinterpret_cast<uintptr_t>(it.dst) & 7u) != 0 || !a16(it.src)) return false;
    return it.src_f64 ? it.ld % 2 == 0 : it.ld % 4 == 0;
}
long long elementwise_blocks(long long n, bool vec4) { return vec4 ? (n + 1023) / 1024 : (n + 255) / 256; }

void add_gemm_splitk(Plan& plan, TableImage& img, const std::vector<SimtProblem>& probs, float* part) {
    std::vector<SimtProblem> chunks;
    std::vector<SplitKItem> items;
    long long block0 = 0;
    float* cur = part;
    for (const SimtProblem& P : probs) {
        const int ns = (P.K + kSplitK - 1) / kSplitK;
        const long long mn = static_cast<long long>(P.M) * P.N;
        for (int j = 0; j < ns; ++j) {
            SimtProblem C = P;
            const long long k0 = static_cast<long long>(j) * kSplitK;
            C.A = static_cast<const uint8_t*>(P.A) + k0 * P.sak * (P.a_f64 ? 8 : 4);
            C.B = static_cast<const uint8_t*>(P.B) + k0 * P.sbk * (P.b_f64 ? 8 : 4);
            C.K = static_cast<int>(std::min<long long>(kSplitK, P.K - k0));
            C.out = cur + j * mn;
            C.out_f64 = 0;
            C.ld_out = P.N;
            C.E = nullptr;
            C.alpha = 1.f;
            C.beta = 0.f;
            C.dscale = nullptr;
            // vector loads stay legal: chunk offsets are multiples of 512 elements
            chunks.push_back(C);
        }
        SplitKItem it;
        std::memset(&it, 0, sizeof(it));
        it.part = cur; it.out = P.out; it.E = P.E; it.ld_out = P.ld_out; it.ld_e = P.ld_e;
        it.M = P.M; it.N = P.N; it.nsplit = ns; it.alpha = P.alpha; it.beta = P.beta;
        it.out_f64 = P.out_f64; it.e_f64 = P.e_f64;
        it.vec4 = splitk_vec4(it) ? 1 : 0;
        it.block0 = block0;
        block0 += elementwise_blocks(mn, it.vec4 != 0);
        items.push_back(it);
        cur += ns * mn;
    }
    add_gemm(plan, img, chunks, false);
    const SplitKItem* di = img.dev<SplitKItem>(img.add(items.data(), items.size() * sizeof(SplitKItem), kAlign));
    const int ni = static_cast<int>(items.size());
    const long long nb = block0;
    double bytes = 0;
    for (const auto& it : items) bytes += 4.0 * it.nsplit * it.M * it.N + (it.out_f64 ? 8.0 : 4.0) * it.M * it.N;
    plan.steps.push_back({MUON_KERNEL_MISC, bytes, [=](cudaStream_t s) {
                              splitk_reduce_kernel<<<static_cast<unsigned>(nb), 256, 0, s>>>(di, ni);
                              return cudaGetLastError();
                          }});
}

// out(M x N) = alpha * A(M x K) B(K x N) + beta * E, all row-major with the given pitches;
// ta / tb: operand stored transposed (A given as K x M, B as N x K); *64: fp64 storage.
struct Mat {
    const void* p;
    long long ld;
    bool t;
    bool f64;
};
SimtProblem gemm(Mat A, Mat B, void* out, long long ldo, bool o64, const void* E, long long lde, bool e64, int M,
                 int N, int K, float alpha, float beta) {
    SimtProblem P;
    std::memset(&P, 0, sizeof(P));
    P.A = A.p; P.B = B.p; P.E = E; P.out = out;
    if (!A.t) { P.sam = A.ld; P.sak = 1; } else { P.sam = 1; P.sak = A.ld; }
    if (!B.t) { P.sbk = B.ld; P.sbn = 1; } else { P.sbk = 1; P.sbn = B.ld; }
    P.ld_out = ldo; P.ld_e = lde;
    P.M = M; P.N = N; P.K = K;
    P.alpha = alpha; P.beta = beta;
    P.vec_a = al16(A.p) && A.ld % 4 == 0;
    P.vec_b = al16(B.p) && B.ld % 4 == 0;
    P.a_f64 = A.f64; P.b_f64 = B.f64; P.e_f64 = e64; P.out_f64 = o64;
    return P;
}

// Allows `kernel` `bytes` of dynamic shared memory on the current device (once per device;
// launches run under the plan cache's lock).
template <auto Kernel>
cudaError_t big_smem(size_t bytes) {
    static bool set_on[64] = {};   // one flag set per kernel (template argument)
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!set_on[dev]) {
        e = cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
        if (e != cudaSuccess) return e;
        set_on[dev] = true;
    }
    return cudaSuccess;
}

// True if lu_panel_cluster_kernel can run on this device with its largest shared memory (one
// cluster of kPanelCluster CTAs resident); else the plan keeps every panel on one CTA.
bool panel_clusters_available() {
    static int state[64] = {};   // 0 unknown, 1 yes, 2 no (plans are built under the cache's lock)
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
    if (state[dev] == 0) {
        bool ok = cudaFuncSetAttribute(lu_panel_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kPanelSmem)) == cudaSuccess;
        if (ok) {
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(kPanelCluster, 1, 1);
            cfg.blockDim = dim3(kPanelClusterThreads, 1, 1);
            cfg.dynamicSmemBytes = kPanelSmem;
            cudaLaunchAttribute attr;
            attr.id = cudaLaunchAttributeClusterDimension;
            attr.val.clusterDim.x = kPanelCluster;
            attr.val.clusterDim.y = 1;
            attr.val.clusterDim.z = 1;
            cfg.attrs = &attr;
            cfg.numAttrs = 1;
            int clusters = 0;
            ok = cudaOccupancyMaxActiveClusters(&clusters, lu_panel_cluster_kernel, &cfg) == cudaSuccess && clusters > 0;
        }
        cudaGetLastError();   // a refused query leaves no error pending
        state[dev] = ok ? 1 : 2;
    }
    return state[dev] == 1;
}

// Gaussian elimination with partial pivoting on the augmented fp64 systems [C | y]
// (N x ncols, row pitch ld, batch B), then back substitution: z overwrites y.
void add_lu_solve(Plan& plan, TableImage& img, double* Aug, int* piv, int N, int ncols, int k, int B, long long ld,
                  long long aug_stride, unsigned* d_status) {
    auto Ai = [&](int i) { return Aug + i * aug_stride; };
    std::vector<SimtProblem> pr;
    // Gaussian elimination with partial pivoting on [C | y], fp64, two levels: kLuBlock-wide
    // block columns factorised with panels (updates confined to the block column), then one
    // row-swap + unit-lower solve over the trailing columns and one K = kLuBlock trailing
    // update per block column.  A panel holds its rows from the block column's top down in
    // shared memory, so the lower block columns take wider panels (fewer, up to kPanelMax
    // columns), split evenly across the block column.  Widths are even, so the in-block updates
    // (K = the width, N = the block's remaining columns) suit the fp64 tensor-core kernel.
    const bool clusters = panel_clusters_available();
    for (int J0 = 0; J0 < N; J0 += kLuBlock) {
        const int JB = std::min(kLuBlock, N - J0);
        const bool on_cluster = clusters && N - J0 > kPanelClusterMinRows;
        const int widest = std::max(2, (on_cluster ? lu_panel_cluster_width(N - J0) : lu_panel_width(N - J0)) & ~1);
        const int npan = (JB + widest - 1) / widest;
        const int nb = std::min(widest, ((JB + npan - 1) / npan + 1) & ~1);
        for (int j0 = J0; j0 < J0 + JB; j0 += nb) {
            const int w = std::min(nb, J0 + JB - j0);
            const size_t smem = lu_panel_smem(N - j0, w);
            const double lu_flops = 2.0 * (N - j0) * w * w * B;
            if (on_cluster) {
                const size_t csmem = lu_panel_cluster_smem(N - j0, w);
                plan.steps.push_back({MUON_KERNEL_LU, lu_flops, [=](cudaStream_t s) {
                    static bool attr_set[64] = {};
                    int dev = 0;
                    cudaError_t e = cudaGetDevice(&dev);
                    if (e != cudaSuccess) return e;
                    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
                    if (!attr_set[dev]) {
                        e = cudaFuncSetAttribute(lu_panel_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 static_cast<int>(kPanelSmem));
                        if (e != cudaSuccess) return e;
                        attr_set[dev] = true;
                    }
                    cudaLaunchConfig_t cfg = {};
                    cfg.gridDim = dim3(B * kPanelCluster, 1, 1);
                    cfg.blockDim = dim3(kPanelClusterThreads, 1, 1);
                    cfg.dynamicSmemBytes = csmem;
                    cfg.stream = s;
                    cudaLaunchAttribute attr;
                    attr.id = cudaLaunchAttributeClusterDimension;
                    attr.val.clusterDim.x = kPanelCluster;
                    attr.val.clusterDim.y = 1;
                    attr.val.clusterDim.z = 1;
                    cfg.attrs = &attr;
                    cfg.numAttrs = 1;
                    return cudaLaunchKernelEx(&cfg, lu_panel_cluster_kernel, Aug, static_cast<long long>(ld), aug_stride,
                                              N, j0, w, piv, static_cast<long long>(N), d_status);
                }});
            } else
            plan.steps.push_back({MUON_KERNEL_LU, lu_flops, [=](cudaStream_t s) {
                // the function attribute is per device: set once on each (launches run under
                // the plan cache's lock)
                static bool attr_set[64] = {};
                int dev = 0;
                cudaError_t e = cudaGetDevice(&dev);
                if (e != cudaSuccess) return e;
                if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
                if (!attr_set[dev]) {
                    e = cudaFuncSetAttribute(lu_panel_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kPanelSmem));
                    if (e != cudaSuccess) return e;
                    attr_set[dev] = true;
                }
                lu_panel_kernel<<<B, kPanelThreads, smem, s>>>(Aug, ld, aug_stride, N, j0, w, piv, N, d_status);
                return cudaGetLastError();
            }});
            // the panel's swaps on the block's earlier columns, swaps + solve on its later ones
            const int right_in = J0 + JB - (j0 + w);
            const int left_blocks = (j0 - J0 + kPanelSwapCols - 1) / kPanelSwapCols;
            const int right_blocks = (right_in + kPanelSwapCols - 1) / kPanelSwapCols;
            if (left_blocks + right_blocks > 0) {
                const int block_end = J0 + JB;
                plan.steps.push_back({MUON_KERNEL_LU, 1.0 * w * w * std::max(right_in, 0) * B, [=](cudaStream_t s) {
                    const size_t smem = kPanelTriangleBytes + swap_ints_bytes(kPanelMax, N - j0);
                    lu_swap_trsm_kernel<<<dim3(left_blocks + right_blocks, B), kPanelSwapThreads, smem, s>>>(
                        Aug, ld, aug_stride, J0, left_blocks, j0, w, block_end, piv, N);
                    return cudaGetLastError();
                }});
            }
            if (right_in > 0) {
                for (int i = 0; i < B; ++i) {
                    double* base = Ai(i);
                    pr.push_back(gemm(Mat{base + (j0 + w) * ld + j0, ld, false, true}, Mat{base + j0 * ld + j0 + w, ld, false, true},
                                      base + (j0 + w) * ld + j0 + w, ld, true, base + (j0 + w) * ld + j0 + w, ld, true,
                                      N - j0 - w, right_in, w, -1.f, 1.f));
                }
                add_gemm(plan, img, pr, true); pr.clear();
            }
        }
        const int right = ncols - (J0 + JB);
        if (right > 0) {
            const int c_lo = J0 + JB;
            plan.steps.push_back({MUON_KERNEL_LU, 1.0 * JB * JB * right * B, [=](cudaStream_t s) {
                constexpr int cols_per_block = kTrsmThreads / kLuLanes;
                cudaError_t e = big_smem<lu_block_swap_trsm_kernel>(kLuTriangleBytes + swap_ints_bytes(kLuBlock, kMaxAugRows));
                if (e != cudaSuccess) return e;
                const size_t smem = kLuTriangleBytes + swap_ints_bytes(kLuBlock, N - J0);
                lu_block_swap_trsm_kernel<<<dim3((right + cols_per_block - 1) / cols_per_block, B), kTrsmThreads,
                                            smem, s>>>(Aug, ld, aug_stride, J0, JB, c_lo, ncols, piv, N);
                return cudaGetLastError();
            }});
            if (N - J0 - JB > 0) {
                for (int i = 0; i < B; ++i) {
                    double* base = Ai(i);
                    pr.push_back(gemm(Mat{base + (J0 + JB) * ld + J0, ld, false, true}, Mat{base + J0 * ld + J0 + JB, ld, false, true},
                                      base + (J0 + JB) * ld + J0 + JB, ld, true, base + (J0 + JB) * ld + J0 + JB, ld, true,
                                      N - J0 - JB, right, JB, -1.f, 1.f));
                }
                add_gemm(plan, img, pr, true); pr.clear();
            }
        }
    }
    // back substitution U z = y' (fp64)
    const int nblk = (N + kBackBlock - 1) / kBackBlock;
    for (int q = nblk - 1; q >= 0; --q) {
        const int i0 = q * kBackBlock, bs = std::min(kBackBlock, N - i0);
        plan.steps.push_back({MUON_KERNEL_LU, 1.0 * bs * bs * k * B, [=](cudaStream_t s) {
            constexpr int cols_per_block = kTrsmThreads / kBackLanes;
            cudaError_t e = big_smem<back_diag_kernel>(kBackSmemBytes);
            if (e != cudaSuccess) return e;
            back_diag_kernel<<<dim3((k + cols_per_block - 1) / cols_per_block, B), kTrsmThreads, kBackSmemBytes, s>>>(
                Aug, ld, aug_stride, i0, bs, N, k);
            return cudaGetLastError();
        }});
        if (i0 > 0) {
            for (int i = 0; i < B; ++i) {
                double* base = Ai(i);
                pr.push_back(gemm(Mat{base + i0, ld, false, true}, Mat{base + i0 * ld + N, ld, false, true}, base + N, ld, true,
                                  base + N, ld, true, i0, k, bs, -1.f, 1.f));
            }
            add_gemm(plan, img, pr, true); pr.clear();
        }
    }
}

// ---------------------------------------------------------------- tensor-core plan
// fp32 products on the tensor cores: each fp32 operand is held as three bf16 planes and a
// product is the sum of the six plane products with indices summing to <= 2 (the dropped
// ones are below 2^-24 of the result), accumulated in fp32 TMEM.
struct Planes {
    __nv_bfloat16* p;   // 3 contiguous planes of rows x cols
    int rows, cols;
};
struct TcOperand {
    const CUtensorMap* tm[kTcMaxPlanes];
    bool mn;
};

// K-major operand: rows are the M (or N) index, columns the K index; MN-major: rows are K.
TcOperand tc_operand(TmapPool& pool, const Planes& pl, bool mn) {
    TcOperand o;
    o.mn = mn;
    const size_t plane = static_cast<size_t>(pl.rows) * pl.cols;
    for (int i = 0; i < kTcMaxPlanes; ++i) o.tm[i] = pool.get(pl.p + i * plane, pl.rows, pl.cols, mn ? 64 : kTcBM / 2);
    return o;
}

TcProblem tc_problem(const TcOperand& a, const TcOperand& b, float* out, const float* E, int ld, int M, int N, int K,
                     float alpha, float beta, bool sym) {
    TcProblem P;
    std::memset(&P, 0, sizeof(P));
    for (int i = 0; i < kTcMaxPlanes; ++i) {
        P.tmA[i] = a.tm[i];
        P.tmB[i] = b.tm[i];
    }
    P.out[0] = out;
    P.E[0] = E;
    P.ld = ld;
    P.M = M; P.N = N; P.K = K;
    P.alpha = alpha; P.beta = beta;
    P.flags = (a.mn ? kProbAMn : 0u) | (b.mn ? kProbBMn : 0u) | (sym ? kProbSym : 0u) | kProbOutF32 |
              (E != nullptr ? kProbEF32 : 0u);
    tc_set_segments(P, kTcMaxPlanes, kTcMaxPlanes, 2);
    return P;
}

void add_tc(Plan& plan, TableImage& img, const std::vector<TcProblem>& all, unsigned* d_status) {
    const int sms = device_sm_count();
    for (size_t first = 0; first < all.size(); first += kMaxTileProblems) {
        const size_t last = std::min(all.size(), first + static_cast<size_t>(kMaxTileProblems));
        const std::vector<TcProblem> probs(all.begin() + first, all.begin() + last);
        std::vector<uint32_t> tiles;
        double flops = 0;
        for (size_t p = 0; p < probs.size(); ++p) {
            const TcProblem& P = probs[p];
            const int mbs = (P.M + kTcBM - 1) / kTcBM, nbs = (P.N + kTcBN - 1) / kTcBN;
            const bool sym = (P.flags & kProbSym) != 0;
            for (int nb = 0; nb < nbs; ++nb)
                for (int mb = 0; mb < mbs; ++mb)
                    if (!sym || nb >= mb) tiles.push_back(tile_code(static_cast<int>(p), mb, nb));
            flops += (sym ? 1.0 : 2.0) * P.M * P.N * P.K;
        }
        const TcProblem* dp = img.dev<TcProblem>(img.add(probs.data(), probs.size() * sizeof(TcProblem), kAlign));
        const uint32_t* dt = img.dev<uint32_t>(img.add(tiles.data(), tiles.size() * sizeof(uint32_t), kAlign));
        const int nt = static_cast<int>(tiles.size());
        plan.steps.push_back({MUON_KERNEL_TC_F32, flops, [=](cudaStream_t s) {
                                  return tc_gemm_launch(dp, dt, nt, d_status, sms, s);
                              }});
    }
}

// Destination of a split-K product: out = alpha * sum of the chunk partials.
struct SplitTarget {
    void* out;
    long long ld;
    int out_f64;
    float alpha;
};

void add_tc_splitk(Plan& plan, TableImage& img, const std::vector<TcProblem>& probs,
                   const std::vector<SplitTarget>& targets, float* part, unsigned* d_status) {
    std::vector<TcProblem> chunks;
    std::vector<SplitKItem> items;
    long long block0 = 0;
    float* cur = part;
    for (size_t p = 0; p < probs.size(); ++p) {
        const TcProblem& P = probs[p];
        const int ns = (P.K + kSplitK - 1) / kSplitK;
        const long long mn = static_cast<long long>(P.M) * P.N;
        for (int j = 0; j < ns; ++j) {
            TcProblem C = P;
            C.k_begin = j * kSplitK;
            C.K = std::min(kSplitK, P.K - j * kSplitK);
            C.out[0] = cur + j * mn;
            C.E[0] = nullptr;
            C.ld = P.N;
            C.alpha = 1.f;
            C.beta = 0.f;
            C.flags = (P.flags & ~kProbEF32) | kProbOutF32;
            chunks.push_back(C);
        }
        SplitKItem it;
        std::memset(&it, 0, sizeof(it));
        it.part = cur; it.out = targets[p].out; it.ld_out = targets[p].ld;
        it.M = P.M; it.N = P.N; it.nsplit = ns; it.alpha = targets[p].alpha;
        it.out_f64 = targets[p].out_f64;
        it.vec4 = splitk_vec4(it) ? 1 : 0;
        it.block0 = block0;
        block0 += elementwise_blocks(mn, it.vec4 != 0);
        items.push_back(it);
        cur += ns * mn;
    }
    add_tc(plan, img, chunks, d_status);
    const SplitKItem* di = img.dev<SplitKItem>(img.add(items.data(), items.size() * sizeof(SplitKItem), kAlign));
    const int ni = static_cast<int>(items.size());
    const long long nb = block0;
    double bytes = 0;
    for (const auto& it : items) bytes += 4.0 * it.nsplit * it.M * it.N + (it.out_f64 ? 8.0 : 4.0) * it.M * it.N;
    plan.steps.push_back({MUON_KERNEL_MISC, bytes, [=](cudaStream_t s) {
                              splitk_reduce_kernel<<<static_cast<unsigned>(nb), 256, 0, s>>>(di, ni);
                              return cudaGetLastError();
                          }});
}

void add_block_cast(Plan& plan, TableImage& img, const std::vector<BlockCastItem>& in) {
    std::vector<BlockCastItem> items(in);
    long long block0 = 0;
    double bytes = 0;
    for (auto& it : items) {
        it.vec4 = (it.cols % 4 == 0 && it.ld % 2 == 0 && (reinterpret_cast<uintptr_t>(it.src) & 15u) == 0 &&
                   (reinterpret_cast<uintptr_t>(it.dst) & 15u) == 0) ? 1 : 0;
        it.block0 = block0;
        const long long n = static_cast<long long>(it.rows) * it.cols;
        block0 += elementwise_blocks(n, it.vec4 != 0);
        bytes += 12.0 * n;
    }
    const BlockCastItem* di = img.dev<BlockCastItem>(img.add(items.data(), items.size() * sizeof(BlockCastItem), kAlign));
    const int ni = static_cast<int>(items.size());
    const long long nb = block0;
    plan.steps.push_back({MUON_KERNEL_MISC, bytes, [=](cudaStream_t s) {
                              block_cast_kernel<<<static_cast<unsigned>(nb), 256, 0, s>>>(di, ni);
                              return cudaGetLastError();
                          }});
}

void add_split3(Plan& plan, TableImage& img, const std::vector<Split3Item>& in) {
    std::vector<Split3Item> items(in);
    long long block0 = 0;
    double bytes = 0;
    for (auto& it : items) {
        it.vec4 = split3_vec4(it) ? 1 : 0;
        it.block0 = block0;
        const long long n = static_cast<long long>(it.rows) * it.cols;
        block0 += elementwise_blocks(n, it.vec4 != 0);
        bytes += n * ((it.src_f64 ? 8.0 : 4.0) + 6.0);
    }
    const Split3Item* di = img.dev<Split3Item>(img.add(items.data(), items.size() * sizeof(Split3Item), kAlign));
    const int ni = static_cast<int>(items.size());
    const long long nb = block0;
    plan.steps.push_back({MUON_KERNEL_MISC, bytes, [=](cudaStream_t s) {
                              split3_kernel<<<static_cast<unsigned>(nb), 256, 0, s>>>(di, ni);
                              return cudaGetLastError();
                          }});
}

// Appends the projection + Woodbury-Cayley launches for W (batch x n x k) with direction
// source G (may be the workspace V buffer itself: V = G - W sym(W^T G) is then formed in
// place, each element read and written by one thread).
muon_status build_stiefel(Plan& plan, TableImage& img, const StiefelLayout& L, uint8_t* ws, unsigned* d_status,
                          float* W, const float* G, int batch, int n, int k, float lr, size_t ws_bytes) {
    // With 16-byte bf16 row pitches, the two products that only shape the direction V (S = W^T G
    // and V = G - W sym(S)) run on the tensor cores from three bf16 planes.  Every product that
    // enters C, y, b or the final update stays on the FMA pipes in fp32 with round-to-nearest:
    // the retraction preserves W^T W = I only as well as those are computed, and the tensor
    // cores' fp32 accumulation over thousands of MMA steps drifted the 100-step orthogonality
    // defect to 7e-5 when they carried all products.  A = V W^T - W V^T stays skew for any V,
    // so the direction's own rounding does not leave the manifold.
    float* V = reinterpret_cast<float*>(ws + kHeaderBytes + L.V);
    float* bb = reinterpret_cast<float*>(ws + kHeaderBytes + L.b);
    float* S = reinterpret_cast<float*>(ws + kHeaderBytes + L.S);
    double* Aug = reinterpret_cast<double*>(ws + kHeaderBytes + L.Aug);
    int* piv = reinterpret_cast<int*>(ws + kHeaderBytes + L.piv);
    float* part = reinterpret_cast<float*>(ws + kHeaderBytes + L.part);
    const long long nk = static_cast<long long>(n) * k, kk = static_cast<long long>(k) * k;
    const int N = 2 * k, ncols = 3 * k;
    const long long ld = ncols, aug_stride = static_cast<long long>(N) * ncols;
    const float c = 0.5f * lr;
    const int B = batch;
    auto Wm = [&](int i, bool t = false) { return Mat{W + i * nk, k, t, false}; };
    auto Gm = [&](int i) { return Mat{G + i * nk, k, false, false}; };
    auto Vm = [&](int i, bool t = false) { return Mat{V + i * nk, k, t, false}; };
    auto Sm = [&](int i) { return Mat{S + i * kk, k, false, false}; };
    auto Ai = [&](int i) { return Aug + i * aug_stride; };

    std::vector<SimtProblem> pr;
    const bool tc = L.tc;
    __nv_bfloat16* planes = tc ? reinterpret_cast<__nv_bfloat16*>(ws + kHeaderBytes + L.planes) : nullptr;
    TmapPool pool(img);
    // planes per matrix: W, G (n x k) and S (k x k), three bf16 planes each
    const size_t per = stiefel_plane_elems(n, k);
    auto pl = [&](int i, int which) {
        __nv_bfloat16* base = planes + i * per;
        if (which < 2) return Planes{base + which * 3 * nk, n, k};
        return Planes{base + 2 * 3 * nk, k, k};
    };
    if (tc) {
        std::vector<Split3Item> sp;
        for (int i = 0; i < B; ++i) {
            for (int which = 0; which < 2; ++which) {
                Split3Item it;
                std::memset(&it, 0, sizeof(it));
                it.src = which == 0 ? static_cast<const void*>(W + i * nk) : static_cast<const void*>(G + i * nk);
                it.ld = k; it.rows = n; it.cols = k; it.dst = pl(i, which).p;
                sp.push_back(it);
            }
        }
        add_split3(plan, img, sp);
        // S = W^T G (split-K over n, fp64 sum of the chunk partials)
        std::vector<TcProblem> tp;
        std::vector<SplitTarget> tg;
        for (int i = 0; i < B; ++i) {
            tp.push_back(tc_problem(tc_operand(pool, pl(i, 0), true), tc_operand(pool, pl(i, 1), true), nullptr, nullptr,
                                    k, k, k, n, 1.f, 0.f, false));
            tg.push_back({S + i * kk, k, 0, 1.f});
        }
        add_tc_splitk(plan, img, tp, tg, part, d_status);
    } else {
        // S = W^T G (split-K), then sym(S)
        for (int i = 0; i < B; ++i) pr.push_back(gemm(Wm(i, true), Gm(i), S + i * kk, k, false, nullptr, 0, false, k, k, n, 1.f, 0.f));
        add_gemm_splitk(plan, img, pr, part); pr.clear();
    }
    plan.steps.push_back({MUON_KERNEL_MISC, 8.0 * kk * B, [=](cudaStream_t s) {
        const int tk = (k + 31) / 32;
        symmetrize_kernel<<<dim3(tk, tk, B), 256, 0, s>>>(S, k, kk);
        return cudaGetLastError();
    }});
    // V = G - W sym(S)
    if (tc) {
        std::vector<Split3Item> sp;
        for (int i = 0; i < B; ++i) {
            Split3Item it;
            std::memset(&it, 0, sizeof(it));
            it.src = S + i * kk; it.ld = k; it.rows = k; it.cols = k; it.dst = pl(i, 2).p;
            sp.push_back(it);
        }
        add_split3(plan, img, sp);
        std::vector<TcProblem> tp;
        for (int i = 0; i < B; ++i)
            tp.push_back(tc_problem(tc_operand(pool, pl(i, 0), false), tc_operand(pool, pl(i, 2), true), V + i * nk,
                                    G + i * nk, k, n, k, k, -1.f, 1.f, false));
        add_tc(plan, img, tp, d_status);
    } else {
        for (int i = 0; i < B; ++i) pr.push_back(gemm(Wm(i), Sm(i), V + i * nk, k, false, G + i * nk, k, false, n, k, k, -1.f, 1.f));
        add_gemm(plan, img, pr); pr.clear();
    }
    // fp64 blocks (split-K sums): [0,0] = c P = c W^T V, [0,k] = c Q = c W^T W, [k,0] = -c R = -c V^T V
    for (int i = 0; i < B; ++i) {
        pr.push_back(gemm(Wm(i, true), Vm(i), Ai(i), ld, true, nullptr, 0, false, k, k, n, c, 0.f));
        pr.push_back(gemm(Wm(i, true), Wm(i), Ai(i) + k, ld, true, nullptr, 0, false, k, k, n, c, 0.f));
        pr.back().sym = 1;                                   // Q = W^T W
        pr.push_back(gemm(Vm(i, true), Vm(i), Ai(i) + k * ld, ld, true, nullptr, 0, false, k, k, n, -c, 0.f));
        pr.back().sym = 1;                                   // R = V^T V
    }
    add_gemm_splitk(plan, img, pr, part); pr.clear();
    // [k,k] = -c P^T
    plan.steps.push_back({MUON_KERNEL_MISC, 16.0 * kk * B, [=](cudaStream_t s) {
        aug_neg_transpose_kernel<<<dim3(std::max(1, std::min<int>(1024, static_cast<int>((kk + 255) / 256))), B), 256, 0, s>>>(Aug, k, ld, aug_stride);
        return cudaGetLastError();
    }});
    // fp32 copies of two k x k blocks of each augmented matrix (into the split-K scratch, free
    // between the reductions), as the B operands of the n x k products that follow
    auto blocks32 = [&](int i, int which) { return part + (2LL * i + which) * kk; };
    auto cast_blocks = [&](long long off0, long long off1) {
        std::vector<BlockCastItem> items;
        for (int i = 0; i < B; ++i)
            for (int which = 0; which < 2; ++which)
                items.push_back({Ai(i) + (which == 0 ? off0 : off1), blocks32(i, which), ld, 0, k, k});
        add_block_cast(plan, img, items);
    };
    auto Bm32 = [&](int i, int which) { return Mat{blocks32(i, which), k, false, false}; };
    // right-hand side [cQ; -cP^T] = c B W: the right block column of cBU, copied before the
    // identity is added
    plan.steps.push_back({MUON_KERNEL_MISC, 32.0 * kk * B, [=](cudaStream_t s) {
        aug_copy_rhs_kernel<<<dim3(std::max(1, std::min<int>(1024, static_cast<int>((2 * kk + 255) / 256))), B), 256, 0, s>>>(Aug, k, ld, aug_stride);
        return cudaGetLastError();
    }});
    // C = I + c B U
    plan.steps.push_back({MUON_KERNEL_MISC, 16.0 * N * B, [=](cudaStream_t s) {
        aug_add_identity_kernel<<<dim3((N + 255) / 256, B), 256, 0, s>>>(Aug, N, ld, aug_stride);
        return cudaGetLastError();
    }});
    add_lu_solve(plan, img, Aug, piv, N, ncols, k, B, ld, aug_stride, d_status);
    // W_new = W - 2 (V z_top + W z_bot), z = C^-1 (c B W), through the workspace b, then into W
    cast_blocks(N, k * ld + N);
    for (int i = 0; i < B; ++i) pr.push_back(gemm(Vm(i), Bm32(i, 0), bb + i * nk, k, false, W + i * nk, k, false, n, k, k, -2.f, 1.f));
    add_gemm(plan, img, pr); pr.clear();
    for (int i = 0; i < B; ++i) pr.push_back(gemm(Wm(i), Bm32(i, 1), bb + i * nk, k, false, bb + i * nk, k, false, n, k, k, -2.f, 1.f));
    add_gemm(plan, img, pr); pr.clear();
    const size_t bytes = static_cast<size_t>(nk) * B * sizeof(float);
    plan.steps.push_back({MUON_KERNEL_MISC, 2.0 * bytes, [=](cudaStream_t s) {
        return cudaMemcpyAsync(W, bb, bytes, cudaMemcpyDeviceToDevice, s);
    }});
    if (L.table_offset + img.bytes.size() > ws_bytes) return MUON_ERR_WORKSPACE_TOO_SMALL;
    return MUON_OK;
}

}  // namespace
}  // namespace muon

using namespace muon;

extern "C" {

size_t stiefel_workspace_size(int batch, int n, int k) {
    if (batch <= 0 || n <= 0 || k <= 0 || n < k || k > 4096 || n > kMaxTileBlocks * kSimtBM) return 0;
    const StiefelLayout L = stiefel_layout(batch, n, k);
    return L.table_offset + stiefel_tables_bound(batch, n, k);
}

muon_status stiefel_cayley_step(float* W, const float* G, int batch, int n, int k, float lr, void* workspace,
                                size_t ws_bytes, void* stream_) {
    if (W == nullptr || G == nullptr || workspace == nullptr) return MUON_ERR_INVALID_ARG;
    if (batch <= 0 || batch > kMaxTileProblems / 4 || n <= 0 || k <= 0 || !std::isfinite(lr))
        return MUON_ERR_INVALID_ARG;
    if (n < k || k > 4096 || n > kMaxTileBlocks * kSimtBM) return MUON_ERR_UNSUPPORTED_SHAPE;
    if (!al16(W) || !al16(G) || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return MUON_ERR_ALIGNMENT;
    if (ws_bytes < stiefel_workspace_size(batch, n, k)) return MUON_ERR_WORKSPACE_TOO_SMALL;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    const StiefelLayout L = stiefel_layout(batch, n, k);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    unsigned* d_status = static_cast<unsigned*>(workspace);

    KeyWriter kw;
    kw.put(3);  // plan kind: stiefel
    kw.put(W); kw.put(G); kw.put(batch); kw.put(n); kw.put(k); kw.put(lr); kw.put(ws_bytes);

    auto build = [&](Plan& plan, TableImage& img) -> muon_status {
        return build_stiefel(plan, img, L, ws, d_status, W, G, batch, n, k, lr, ws_bytes);
    };
    return run_plan(kw.k, workspace, L.table_offset, build, stream);
}

size_t muon_cayley_workspace_size(int batch, int n, int k) {
    if (batch <= 0 || n <= 0 || k <= 0) return 0;
    const int nt = n < k ? k : n, kt = n < k ? n : k;
    if (kt > 4096 || nt > kMaxTileBlocks * kSimtBM) return 0;
    const CayleyLayout C = cayley_layout(batch, n, k);
    return C.st.table_offset + stiefel_tables_bound(batch, nt, kt);
}

muon_status muon_cayley_step(float* W, const float* G, float* M, int batch, int n, int k, float lr, float beta,
                             int center, void* workspace, size_t ws_bytes, void* stream_) {
    if (M == nullptr || !std::isfinite(beta) || (center != 0 && center != 1)) return MUON_ERR_INVALID_ARG;
    if (W == nullptr || G == nullptr || workspace == nullptr) return MUON_ERR_INVALID_ARG;
    if (batch <= 0 || batch > kMaxTileProblems / 4 || n <= 0 || k <= 0 || !std::isfinite(lr))
        return MUON_ERR_INVALID_ARG;
    // A wide parameter (n < k) is updated as its transpose (k x n, column-orthonormal).
    const bool wide = n < k;
    const int nt = wide ? k : n, kt = wide ? n : k;
    if (kt > 4096 || nt > kMaxTileBlocks * kSimtBM) return MUON_ERR_UNSUPPORTED_SHAPE;
    if (!al16(W) || !al16(G) || !al16(M) || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return MUON_ERR_ALIGNMENT;
    if (ws_bytes < muon_cayley_workspace_size(batch, n, k)) return MUON_ERR_WORKSPACE_TOO_SMALL;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    const CayleyLayout C = cayley_layout(batch, n, k);
    const StiefelLayout& L = C.st;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    unsigned* d_status = static_cast<unsigned*>(workspace);

    KeyWriter kw;
    kw.put(4);  // plan kind: MuonCayley
    kw.put(W); kw.put(G); kw.put(M); kw.put(batch); kw.put(n); kw.put(k); kw.put(lr); kw.put(beta); kw.put(center);
    kw.put(ws_bytes);

    auto build = [&](Plan& plan, TableImage& img) -> muon_status {
        float* V = reinterpret_cast<float*>(ws + kHeaderBytes + L.V);
        double* cm = center ? reinterpret_cast<double*>(ws + kHeaderBytes + L.cm) : nullptr;
        float* Wt = wide ? reinterpret_cast<float*>(ws + kHeaderBytes + C.Wt) : W;
        float* Mt = wide ? reinterpret_cast<float*>(ws + kHeaderBytes + C.Mt) : M;
        const long long total = static_cast<long long>(batch) * n * k;
        const int grid = static_cast<int>(std::min<long long>((total + 255) / 256, 148LL * 16));
        const float b = beta;
        // transposes of one batch: rows x cols -> cols x rows
        auto transpose = [&](const float* in, float* out, int rows, int cols) {
            const dim3 tg((cols + 31) / 32, (rows + 31) / 32, batch);
            plan.steps.push_back({MUON_KERNEL_MISC, 8.0 * total, [=](cudaStream_t s) {
                transpose_kernel<<<tg, dim3(32, 8), 0, s>>>(in, out, rows, cols);
                return cudaGetLastError();
            }});
        };
        plan.steps.push_back({MUON_KERNEL_MOMENTUM, 12.0 * total, [=](cudaStream_t s) {
            ema_kernel<<<grid, 256, 0, s>>>(M, G, total, b);
            return cudaGetLastError();
        }});
        if (wide) transpose(M, Mt, n, k);
        if (cm != nullptr) {
            plan.steps.push_back({MUON_KERNEL_MISC, 4.0 * total, [=](cudaStream_t s) {
                column_mean_kernel<<<dim3((kt + 127) / 128, batch), 128, 0, s>>>(Mt, cm, nt, kt);
                return cudaGetLastError();
            }});
        }
        plan.steps.push_back({MUON_KERNEL_MISC, 8.0 * total, [=](cudaStream_t s) {
            center_kernel<<<grid, 256, 0, s>>>(Mt, cm, V, nt, kt, total);
            return cudaGetLastError();
        }});
        if (wide) transpose(W, Wt, n, k);
        const muon_status st = build_stiefel(plan, img, L, ws, d_status, Wt, V, batch, nt, kt, lr, ws_bytes);
        if (st != MUON_OK) return st;
        if (wide) transpose(Wt, W, k, n);
        return MUON_OK;
    };
    return run_plan(kw.k, workspace, L.table_offset, build, stream);
}

}  // extern "C"
