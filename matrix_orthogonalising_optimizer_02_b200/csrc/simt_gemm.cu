// Grouped fp32 GEMM on the FMA pipes (no TF32): the fp32 Newton-Schulz mode and every
// product of the Stiefel/Woodbury path, where the result must carry fp32 accuracy.
// 128 x 128 tiles, K-step 8, 256 threads with an 8 x 8 register block each, double-
// buffered shared memory.  Operands are addressed by (row, column) strides, so transposed
// operands (W^T G, X^T X) need no copies.  The Acc = double instantiation stages the fp32
// operands as fp64 and accumulates with DFMA: used for long reductions (K = n) whose
// rounding would otherwise accumulate sequentially over thousands of terms.
#include "kernels.cuh"

namespace muon {
namespace {

constexpr int BM = kSimtBM, BN = kSimtBN, BK = kSimtBK;
constexpr int PAD = 4;

template <class T>
__device__ __forceinline__ T ld1(const void* base, long long off, int f64) {
    return f64 ? static_cast<T>(__ldg(static_cast<const double*>(base) + off))
               : static_cast<T>(__ldg(static_cast<const float*>(base) + off));
}
template <class T>
__device__ __forceinline__ void ld4(const void* base, long long off, int f64, T (&r)[4]) {
    if (f64) {
        const double2 a = __ldg(reinterpret_cast<const double2*>(static_cast<const double*>(base) + off));
        const double2 b = __ldg(reinterpret_cast<const double2*>(static_cast<const double*>(base) + off) + 1);
        r[0] = static_cast<T>(a.x); r[1] = static_cast<T>(a.y); r[2] = static_cast<T>(b.x); r[3] = static_cast<T>(b.y);
    } else {
        const float4 v = __ldg(reinterpret_cast<const float4*>(static_cast<const float*>(base) + off));
        r[0] = static_cast<T>(v.x); r[1] = static_cast<T>(v.y); r[2] = static_cast<T>(v.z); r[3] = static_cast<T>(v.w);
    }
}

// Thread -> element mapping of a tile load.  If the operand is contiguous along K the
// 256 threads cover 128 rows x 2 quads of K; otherwise 8 K-rows x 32 quads of M (or N).
// Values arrive in the accumulator type T (fp64 sources are rounded when T is float).
template <class T>
__device__ __forceinline__ void load_tile(const void* __restrict__ base, int f64, long long s_mn, long long s_k,
                                          int mn0, int k0, int MN, int K, int vec, int tid, T (&r)[4]) {
    const bool k_contig = (s_k == 1);
    int mn, k;
    if (k_contig) {
        mn = tid >> 1;
        k = (tid & 1) * 4;
    } else {
        k = tid >> 5;
        mn = (tid & 31) * 4;
    }
    const long long gm = mn0 + mn, gk = k0 + k;
    if (k_contig) {
        if (vec && gm < MN && gk + 3 < K) {
            ld4(base, gm * s_mn + gk, f64, r);
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) r[i] = (gm < MN && gk + i < K) ? ld1<T>(base, gm * s_mn + (gk + i) * s_k, f64) : T(0);
        }
    } else {
        if (vec && gk < K && gm + 3 < MN) {
            ld4(base, gm * s_mn + gk * s_k, f64, r);
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) r[i] = (gk < K && gm + i < MN) ? ld1<T>(base, (gm + i) * s_mn + gk * s_k, f64) : T(0);
        }
    }
}

template <class Acc>
__device__ __forceinline__ void store_tile(Acc (*s)[BM + PAD], bool k_contig, int tid, const Acc (&r)[4]) {
    if (k_contig) {
        const int mn = tid >> 1, k = (tid & 1) * 4;
#pragma unroll
        for (int i = 0; i < 4; ++i) s[k + i][mn] = static_cast<Acc>(r[i]);
    } else {
        const int k = tid >> 5, mn = (tid & 31) * 4;
        if constexpr (sizeof(Acc) == sizeof(float)) {
            *reinterpret_cast<float4*>(&s[k][mn]) = make_float4(r[0], r[1], r[2], r[3]);
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) s[k][mn + i] = static_cast<Acc>(r[i]);
        }
    }
}

__device__ __forceinline__ void load4(const double* p, double (&v)[8], int o) {
    const double2 a = *reinterpret_cast<const double2*>(p);
    const double2 b = *reinterpret_cast<const double2*>(p + 2);
    v[o] = a.x; v[o + 1] = a.y; v[o + 2] = b.x; v[o + 3] = b.y;
}
__device__ __forceinline__ void load4(const float* p, float (&v)[8], int o) {
    const float4 q = *reinterpret_cast<const float4*>(p);
    v[o] = q.x; v[o + 1] = q.y; v[o + 2] = q.z; v[o + 3] = q.w;
}

// fp32: two CTAs (16 warps) per SM; fp64: one (its 8 x 8 fp64 block needs the registers).
template <class Acc>
__global__ void __launch_bounds__(kSimtThreads, sizeof(Acc) == sizeof(float) ? 2 : 1)
simt_gemm_kernel(const SimtProblem* __restrict__ probs, const uint32_t* __restrict__ tiles, int num_tiles) {
    __shared__ __align__(16) Acc As[2][BK][BM + PAD];
    __shared__ __align__(16) Acc Bs[2][BK][BN + PAD];
    const int tid = threadIdx.x;
    const int tx = tid & 15, ty = tid >> 4;

    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x) {
        const uint32_t code = tiles[t];
        const SimtProblem& P = probs[code >> 20];
        const int m0 = static_cast<int>((code >> 10) & 1023u) * BM;
        const int n0 = static_cast<int>(code & 1023u) * BN;
        const bool a_kc = (P.sak == 1);
        const bool b_kc = (P.sbk == 1);

        Acc acc[8][8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[i][j] = Acc(0);

        Acc ra[4], rb[4];
        // A(m, k) = A[m*sam + k*sak]; B(k, n) = B[k*sbk + n*sbn] -> as an (n, k) operand.
        load_tile(P.A, P.a_f64, P.sam, P.sak, m0, 0, P.M, P.K, P.vec_a, tid, ra);
        load_tile(P.B, P.b_f64, P.sbn, P.sbk, n0, 0, P.N, P.K, P.vec_b, tid, rb);
        __syncthreads();  // previous tile's readers are done with buffer 0
        store_tile(As[0], a_kc, tid, ra);
        store_tile(Bs[0], b_kc, tid, rb);
        __syncthreads();

        const int ksteps = (P.K + BK - 1) / BK;
        for (int ks = 0; ks < ksteps; ++ks) {
            const int cur = ks & 1;
            const bool more = ks + 1 < ksteps;
            if (more) {
                load_tile(P.A, P.a_f64, P.sam, P.sak, m0, (ks + 1) * BK, P.M, P.K, P.vec_a, tid, ra);
                load_tile(P.B, P.b_f64, P.sbn, P.sbk, n0, (ks + 1) * BK, P.N, P.K, P.vec_b, tid, rb);
            }
#pragma unroll
            for (int k = 0; k < BK; ++k) {
                Acc av[8], bv[8];
                load4(&As[cur][k][ty * 4], av, 0);
                load4(&As[cur][k][64 + ty * 4], av, 4);
                load4(&Bs[cur][k][tx * 4], bv, 0);
                load4(&Bs[cur][k][64 + tx * 4], bv, 4);
#pragma unroll
                for (int i = 0; i < 8; ++i)
#pragma unroll
                    for (int j = 0; j < 8; ++j) acc[i][j] = fma(av[i], bv[j], acc[i][j]);
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
        if constexpr (sizeof(Acc) == sizeof(double)) {
            // The fp64 kernel's short-K launches (the LU updates) are dominated by this
            // epilogue.  With an fp64 output and addend on 16-byte aligned rows, each of the
            // thread's two groups of 4 consecutive columns per row goes as 32-byte accesses,
            // so a warp touches whole sectors.
            const bool has_e = beta != 0.f;
            const bool vec_ok = !P.sym && P.out_f64 && (reinterpret_cast<uintptr_t>(P.out) & 15u) == 0 &&
                                P.ld_out % 2 == 0 &&
                                (!has_e || (P.e_f64 && (reinterpret_cast<uintptr_t>(P.E) & 15u) == 0 && P.ld_e % 2 == 0));
            if (vec_ok) {
                const double* E = static_cast<const double*>(P.E);
                double* O = static_cast<double*>(P.out);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int m = m0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + (i - 4));
                    if (m >= P.M) continue;
#pragma unroll
                    for (int g = 0; g < 2; ++g) {
                        const int nq = n0 + g * 64 + tx * 4;
                        const long long eo = static_cast<long long>(m) * P.ld_e + nq;
                        const long long oo = static_cast<long long>(m) * P.ld_out + nq;
                        double v[4];
#pragma unroll
                        for (int j = 0; j < 4; ++j) v[j] = static_cast<double>(alpha) * acc[i][4 * g + j];
                        if (nq + 3 < P.N) {
                            if (has_e) {
                                const double2 e0 = *reinterpret_cast<const double2*>(E + eo);
                                const double2 e1 = *reinterpret_cast<const double2*>(E + eo + 2);
                                const double b = beta;
                                v[0] = fma(b, e0.x, v[0]); v[1] = fma(b, e0.y, v[1]);
                                v[2] = fma(b, e1.x, v[2]); v[3] = fma(b, e1.y, v[3]);
                            }
                            *reinterpret_cast<double2*>(O + oo) = make_double2(v[0], v[1]);
                            *reinterpret_cast<double2*>(O + oo + 2) = make_double2(v[2], v[3]);
                        } else {
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                if (nq + j >= P.N) continue;
                                O[oo + j] = has_e ? fma(static_cast<double>(beta), E[eo + j], v[j]) : v[j];
                            }
                        }
                    }
                }
                continue;
            }
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int m = m0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + (i - 4));
            if (m >= P.M) continue;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int n = n0 + (j < 4 ? tx * 4 + j : 64 + tx * 4 + (j - 4));
                if (n >= P.N) continue;
                if (P.sym && n < m) continue;   // written by the mirror of (n, m)
                Acc v = static_cast<Acc>(alpha) * acc[i][j];
                if (beta != 0.f) {
                    const long long eo = static_cast<long long>(m) * P.ld_e + n;
                    const Acc e = P.e_f64 ? static_cast<Acc>(static_cast<const double*>(P.E)[eo])
                                          : static_cast<Acc>(static_cast<const float*>(P.E)[eo]);
                    v = fma(static_cast<Acc>(beta), e, v);
                }
                const long long oo = static_cast<long long>(m) * P.ld_out + n;
                const long long om = static_cast<long long>(n) * P.ld_out + m;
                if (P.out_f64) {
                    static_cast<double*>(P.out)[oo] = static_cast<double>(v);
                    if (P.sym && n > m) static_cast<double*>(P.out)[om] = static_cast<double>(v);
                } else {
                    static_cast<float*>(P.out)[oo] = static_cast<float>(v);
                    if (P.sym && n > m) static_cast<float*>(P.out)[om] = static_cast<float>(v);
                }
            }
        }
    }
}

}  // namespace

cudaError_t simt_gemm_launch(const SimtProblem* d_probs, const uint32_t* d_tiles, int num_tiles, cudaStream_t stream,
                             bool f64_acc) {
    if (num_tiles <= 0) return cudaSuccess;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int per_sm = f64_acc ? 1 : 2;
    const int grid = num_tiles < sms * per_sm ? num_tiles : sms * per_sm;
    if (f64_acc)
        simt_gemm_kernel<double><<<grid, kSimtThreads, 0, stream>>>(d_probs, d_tiles, num_tiles);
    else
        simt_gemm_kernel<float><<<grid, kSimtThreads, 0, stream>>>(d_probs, d_tiles, num_tiles);
    return cudaGetLastError();
}

}  // namespace muon
