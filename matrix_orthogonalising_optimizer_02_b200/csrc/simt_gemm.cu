// Grouped fp32 GEMM on the FMA pipes (no TF32): the fp32 Newton-Schulz mode and every
// product of the Stiefel/Woodbury path, where the result must carry fp32 accuracy.
// 128 x 128 tiles, K-step 8, 256 threads with an 8 x 8 register block each, double-
// buffered shared memory.  Operands are addressed by (row, column) strides, so transposed
// operands (W^T G, X^T X) need no copies.
#include "kernels.cuh"

namespace muon {
namespace {

constexpr int BM = kSimtBM, BN = kSimtBN, BK = kSimtBK;
constexpr int PAD = 4;

struct Frag {
    float a[4];
    float b[4];
};

// Thread -> element mapping of a tile load.  If the operand is contiguous along K the
// 256 threads cover 128 rows x 2 quads of K; otherwise 8 K-rows x 32 quads of M (or N).
__device__ __forceinline__ void load_tile(const float* __restrict__ base, long long s_mn, long long s_k, int mn0,
                                          int k0, int MN, int K, int vec, int tid, float (&r)[4]) {
    const bool k_contig = (s_k == 1);
    int mn, k;
    if (k_contig) {
        mn = tid >> 1;
        k = (tid & 1) * 4;
    } else {
        k = tid >> 5;
        mn = (tid & 31) * 4;
    }
    const int gm = mn0 + mn, gk = k0 + k;
    if (k_contig) {
        if (vec && gm < MN && gk + 3 < K) {
            const float4 v = __ldg(reinterpret_cast<const float4*>(base + gm * s_mn + gk));
            r[0] = v.x; r[1] = v.y; r[2] = v.z; r[3] = v.w;
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) r[i] = (gm < MN && gk + i < K) ? __ldg(base + gm * s_mn + (gk + i) * s_k) : 0.f;
        }
    } else {
        if (vec && gk < K && gm + 3 < MN) {
            const float4 v = __ldg(reinterpret_cast<const float4*>(base + gm * s_mn + gk * s_k));
            r[0] = v.x; r[1] = v.y; r[2] = v.z; r[3] = v.w;
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) r[i] = (gk < K && gm + i < MN) ? __ldg(base + (gm + i) * s_mn + gk * s_k) : 0.f;
        }
    }
}

__device__ __forceinline__ void store_tile(float (*s)[BM + PAD], bool k_contig, int tid, const float (&r)[4]) {
    if (k_contig) {
        const int mn = tid >> 1, k = (tid & 1) * 4;
#pragma unroll
        for (int i = 0; i < 4; ++i) s[k + i][mn] = r[i];
    } else {
        const int k = tid >> 5, mn = (tid & 31) * 4;
        *reinterpret_cast<float4*>(&s[k][mn]) = make_float4(r[0], r[1], r[2], r[3]);
    }
}

__global__ void __launch_bounds__(kSimtThreads)
simt_gemm_kernel(const SimtProblem* __restrict__ probs, const uint32_t* __restrict__ tiles, int num_tiles) {
    __shared__ __align__(16) float As[2][BK][BM + PAD];
    __shared__ __align__(16) float Bs[2][BK][BN + PAD];
    const int tid = threadIdx.x;
    const int tx = tid & 15, ty = tid >> 4;

    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x) {
        const uint32_t code = tiles[t];
        const SimtProblem& P = probs[code >> 20];
        const int m0 = static_cast<int>((code >> 10) & 1023u) * BM;
        const int n0 = static_cast<int>(code & 1023u) * BN;
        const bool a_kc = (P.sak == 1);
        const bool b_kc = (P.sbk == 1);

        float acc[8][8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

        float ra[4], rb[4];
        // A(m, k) = A[m*sam + k*sak]; B(k, n) = B[k*sbk + n*sbn] -> as an (n, k) operand.
        load_tile(P.A, P.sam, P.sak, m0, 0, P.M, P.K, P.vec_a, tid, ra);
        load_tile(P.B, P.sbn, P.sbk, n0, 0, P.N, P.K, P.vec_b, tid, rb);
        __syncthreads();  // previous tile's readers are done with buffer 0
        store_tile(As[0], a_kc, tid, ra);
        store_tile(Bs[0], b_kc, tid, rb);
        __syncthreads();

        const int ksteps = (P.K + BK - 1) / BK;
        for (int ks = 0; ks < ksteps; ++ks) {
            const int cur = ks & 1;
            const bool more = ks + 1 < ksteps;
            if (more) {
                load_tile(P.A, P.sam, P.sak, m0, (ks + 1) * BK, P.M, P.K, P.vec_a, tid, ra);
                load_tile(P.B, P.sbn, P.sbk, n0, (ks + 1) * BK, P.N, P.K, P.vec_b, tid, rb);
            }
#pragma unroll
            for (int k = 0; k < BK; ++k) {
                const float4 a0 = *reinterpret_cast<const float4*>(&As[cur][k][ty * 4]);
                const float4 a1 = *reinterpret_cast<const float4*>(&As[cur][k][64 + ty * 4]);
                const float4 b0 = *reinterpret_cast<const float4*>(&Bs[cur][k][tx * 4]);
                const float4 b1 = *reinterpret_cast<const float4*>(&Bs[cur][k][64 + tx * 4]);
                const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
                const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
                for (int i = 0; i < 8; ++i)
#pragma unroll
                    for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
            }
            if (more) {
                store_tile(As[cur ^ 1], a_kc, tid, ra);
                store_tile(Bs[cur ^ 1], b_kc, tid, rb);
            }
            __syncthreads();
        }

        float f = 1.f;
        if (P.dscale != nullptr && P.scale_pow > 0) {
            const float s = __ldg(P.dscale);
            f = (P.scale_pow == 1) ? s : s * s;
        }
        const float alpha = P.alpha * f, beta = P.beta * f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int m = m0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + (i - 4));
            if (m >= P.M) continue;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int n = n0 + (j < 4 ? tx * 4 + j : 64 + tx * 4 + (j - 4));
                if (n >= P.N) continue;
                float v = alpha * acc[i][j];
                if (beta != 0.f) v = fmaf(beta, P.E[m * P.ld_e + n], v);
                P.out[m * P.ld_out + n] = v;
            }
        }
    }
}

}  // namespace

cudaError_t simt_gemm_launch(const SimtProblem* d_probs, const uint32_t* d_tiles, int num_tiles, cudaStream_t stream) {
    if (num_tiles <= 0) return cudaSuccess;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int per_sm = 2;
    const int grid = num_tiles < sms * per_sm ? num_tiles : sms * per_sm;
    simt_gemm_kernel<<<grid, kSimtThreads, 0, stream>>>(d_probs, d_tiles, num_tiles);
    return cudaGetLastError();
}

}  // namespace muon
