// Grouped SIMT GEMM with a multi-stage cp.async pipeline: the same products, tile codes and
// arithmetic as simt_gemm.cu (every thread accumulates its 8 x 8 block in K order, so results
// are bitwise those of that kernel), for fp32 operands with B row-major along N and A
// row-major along K or along M.  The templates also take Acc = double, but that
// instantiation measured 20% slower than the register-staged fp64 kernel on the LU updates
// (its 8 x 8 fp64 block leaves too few warps per SM), so only fp32 is launched.  Operand
// tiles go from global to shared memory by cp.async in 16-byte chunks, zero-filled past the
// matrix edges, through a 2-deep ring of K-steps of 32 (measured faster than 3 or 4 stages):
// the next K-step loads while the current one computes, with no staging registers.  (The
// register-staged kernel, profiled on these products, stalled mostly on global-load latency:
// its loads pass through registers.)
#include <cstdint>

#include "simt_async.cuh"

namespace muon {
namespace {

constexpr int BM = kSimtBM, BN = kSimtBN, THREADS = kSimtThreads, STAGES = 2;
static_assert(BM == BN, "square tiles: the A and B tiles share one layout");

template <class Acc>
struct Cfg {
    static constexpr int V = 16 / static_cast<int>(sizeof(Acc));      // elements per 16-byte chunk
    static constexpr int BK = sizeof(Acc) == sizeof(float) ? 32 : 8;  // K per stage
    static constexpr int PITCH_MN = BM + V;                           // row pitch of [k][mn] tiles
    static constexpr int PITCH_K = BK + V;                            // row pitch of [m][k] tiles
    static constexpr int A_ELEMS = BK * PITCH_MN > BM * PITCH_K ? BK * PITCH_MN : BM * PITCH_K;
    static constexpr int B_ELEMS = BK * PITCH_MN;
    static constexpr size_t SMEM = static_cast<size_t>(STAGES) * (A_ELEMS + B_ELEMS) * sizeof(Acc);
    static_assert((BK * BN / V) % THREADS == 0 && (BM * BK / V) % THREADS == 0, "whole chunks per thread");
};

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, int src_bytes) {
    const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// The fields of a problem the main loop reads, held in registers.
template <class Acc>
struct Ops {
    const Acc* A;
    const Acc* B;
    long long sa;   // A's row pitch: along M for an [m][k] A, along K for a [k][m] A
    long long sbk;
    int M, N, K;
};

// Row (within the tile) of the thread's register-block row i, and column of column j: fp32
// columns come in two groups of 4 (one 16-byte load each), fp64 columns in four groups of 2
// (one 16-byte load each, half a warp reading 256 contiguous bytes).
__device__ __forceinline__ int row_of(int ty, int i) { return i < 4 ? ty * 4 + i : 64 + ty * 4 + (i - 4); }
template <class Acc>
__device__ __forceinline__ int col_of(int tx, int j) {
    if constexpr (sizeof(Acc) == sizeof(double)) return 32 * (j >> 1) + 2 * tx + (j & 1);
    else return j < 4 ? tx * 4 + j : 64 + tx * 4 + (j - 4);
}

// Rows [r0, r0 + R) x contiguous columns [c0, c0 + C) of a row-major matrix (pitch ld, extent
// rows x cols) into a shared tile with row pitch `pitch`, as 16-byte chunks.
template <class Acc, int R, int C>
__device__ __forceinline__ void copy_block(Acc* dst, int pitch, const Acc* src, long long ld, int r0, int c0, int rows,
                                           int cols, int tid) {
    constexpr int V = Cfg<Acc>::V, CHUNKS_PER_ROW = C / V;
#pragma unroll
    for (int q = 0; q < (R * C / V) / THREADS; ++q) {
        const int c = tid + q * THREADS;
        const int r = c / CHUNKS_PER_ROW, col = (c % CHUNKS_PER_ROW) * V;
        const int gr = r0 + r, gc = c0 + col;
        int bytes = 0;
        const Acc* p = src;
        if (gr < rows && gc < cols) {
            bytes = (cols - gc < V ? cols - gc : V) * static_cast<int>(sizeof(Acc));
            p = src + static_cast<long long>(gr) * ld + gc;
        }
        cp_async16(dst + r * pitch + col, p, bytes);
    }
}

template <class Acc, bool A_KC>
__device__ __forceinline__ void load_stage(const Ops<Acc>& o, Acc* as, Acc* bs, int m0, int n0, int k0, int tid) {
    using C = Cfg<Acc>;
    copy_block<Acc, C::BK, BN>(bs, C::PITCH_MN, o.B, o.sbk, k0, n0, o.K, o.N, tid);
    if constexpr (A_KC) copy_block<Acc, BM, C::BK>(as, C::PITCH_K, o.A, o.sa, m0, k0, o.M, o.K, tid);
    else copy_block<Acc, C::BK, BM>(as, C::PITCH_MN, o.A, o.sa, k0, m0, o.K, o.M, tid);
}

template <class Acc>
__device__ __forceinline__ void load_b(const Acc* row, int tx, Acc (&bv)[8]) {
    if constexpr (sizeof(Acc) == sizeof(double)) {
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            const double2 q = *reinterpret_cast<const double2*>(row + 32 * g + 2 * tx);
            bv[2 * g] = q.x;
            bv[2 * g + 1] = q.y;
        }
    } else {
#pragma unroll
        for (int g = 0; g < 2; ++g) {
            const float4 q = *reinterpret_cast<const float4*>(row + 64 * g + 4 * tx);
            bv[4 * g] = q.x; bv[4 * g + 1] = q.y; bv[4 * g + 2] = q.z; bv[4 * g + 3] = q.w;
        }
    }
}

template <class Acc, bool A_KC>
__device__ __forceinline__ void compute_stage(const Acc* as, const Acc* bs, int tx, int ty, Acc (&acc)[8][8]) {
    using C = Cfg<Acc>;
    if constexpr (!A_KC) {
#pragma unroll
        for (int k = 0; k < C::BK; ++k) {
            Acc av[8], bv[8];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const Acc* p = as + k * C::PITCH_MN + 64 * h + ty * 4;
                if constexpr (sizeof(Acc) == sizeof(double)) {
                    const double2 q0 = *reinterpret_cast<const double2*>(p);
                    const double2 q1 = *reinterpret_cast<const double2*>(p + 2);
                    av[4 * h] = q0.x; av[4 * h + 1] = q0.y; av[4 * h + 2] = q1.x; av[4 * h + 3] = q1.y;
                } else {
                    const float4 q = *reinterpret_cast<const float4*>(p);
                    av[4 * h] = q.x; av[4 * h + 1] = q.y; av[4 * h + 2] = q.z; av[4 * h + 3] = q.w;
                }
            }
            load_b(bs + k * C::PITCH_MN, tx, bv);
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[i][j] = fma(av[i], bv[j], acc[i][j]);
        }
    } else {
        // [m][k] A: two consecutive K values of each of the thread's rows per load
#pragma unroll
        for (int k = 0; k < C::BK; k += 2) {
            Acc a2[8][2];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const Acc* p = as + row_of(ty, i) * C::PITCH_K + k;
                if constexpr (sizeof(Acc) == sizeof(double)) {
                    const double2 q = *reinterpret_cast<const double2*>(p);
                    a2[i][0] = q.x; a2[i][1] = q.y;
                } else {
                    const float2 q = *reinterpret_cast<const float2*>(p);
                    a2[i][0] = q.x; a2[i][1] = q.y;
                }
            }
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
                Acc bv[8];
                load_b(bs + (k + kk) * C::PITCH_MN, tx, bv);
#pragma unroll
                for (int i = 0; i < 8; ++i)
#pragma unroll
                    for (int j = 0; j < 8; ++j) acc[i][j] = fma(a2[i][kk], bv[j], acc[i][j]);
            }
        }
    }
}

// out = f * (alpha * acc + beta * E), out and E in the accumulator type; symmetric problems
// store the upper triangle and its mirror.
template <class Acc>
__device__ __forceinline__ void store_tile(const SimtProblem& P, const Acc (&acc)[8][8], int m0, int n0, int tx,
                                           int ty) {
    constexpr int V = Cfg<Acc>::V;
    constexpr int GW = sizeof(Acc) == sizeof(double) ? 2 : 4, NG = 8 / GW;   // columns per group, groups
    float f = 1.f;
    if (P.dscale != nullptr && P.scale_pow > 0) {
        const float s = __ldg(P.dscale);
        f = (P.scale_pow == 1) ? s : s * s;
    }
    const Acc alpha = static_cast<Acc>(P.alpha * f), beta = static_cast<Acc>(P.beta * f);
    const bool has_e = P.beta * f != 0.f;
    Acc* O = static_cast<Acc*>(P.out);
    const Acc* E = static_cast<const Acc*>(P.E);
    const bool vec = !P.sym && (reinterpret_cast<uintptr_t>(O) & 15u) == 0 && P.ld_out % V == 0 &&
                     (!has_e || ((reinterpret_cast<uintptr_t>(E) & 15u) == 0 && P.ld_e % V == 0));
    if constexpr (sizeof(Acc) == sizeof(float)) {
        if (vec) {
            // Four rows at a time, every E load issued before the first store: E is either the
            // output itself (each element read and written by this thread) or a disjoint array,
            // and loads placed after stores would each wait out a full memory latency.
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float4 e[4][NG];
#pragma unroll
                for (int ii = 0; ii < 4; ++ii) {
                    const int m = m0 + row_of(ty, 4 * half + ii);
#pragma unroll
                    for (int g = 0; g < NG; ++g) {
                        const int nq = n0 + col_of<Acc>(tx, GW * g);
                        e[ii][g] = (has_e && m < P.M && nq + GW - 1 < P.N)
                                       ? *reinterpret_cast<const float4*>(E + static_cast<long long>(m) * P.ld_e + nq)
                                       : make_float4(0.f, 0.f, 0.f, 0.f);
                    }
                }
#pragma unroll
                for (int ii = 0; ii < 4; ++ii) {
                    const int i = 4 * half + ii;
                    const int m = m0 + row_of(ty, i);
                    if (m >= P.M) continue;
#pragma unroll
                    for (int g = 0; g < NG; ++g) {
                        const int nq = n0 + col_of<Acc>(tx, GW * g);
                        if (nq >= P.N) continue;
                        const long long oo = static_cast<long long>(m) * P.ld_out + nq;
                        if (nq + GW - 1 < P.N) {
                            float4 v;
                            v.x = fmaf(beta, e[ii][g].x, alpha * acc[i][GW * g]);
                            v.y = fmaf(beta, e[ii][g].y, alpha * acc[i][GW * g + 1]);
                            v.z = fmaf(beta, e[ii][g].z, alpha * acc[i][GW * g + 2]);
                            v.w = fmaf(beta, e[ii][g].w, alpha * acc[i][GW * g + 3]);
                            *reinterpret_cast<float4*>(O + oo) = v;
                        } else {
                            const long long eo = static_cast<long long>(m) * P.ld_e + nq;
#pragma unroll
                            for (int j = 0; j < GW; ++j) {
                                if (nq + j >= P.N) continue;
                                Acc w = alpha * acc[i][GW * g + j];
                                if (has_e) w = fmaf(beta, E[eo + j], w);
                                O[oo + j] = w;
                            }
                        }
                    }
                }
            }
            return;
        }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int m = m0 + row_of(ty, i);
        if (m >= P.M) continue;
#pragma unroll
        for (int g = 0; g < NG; ++g) {
            const int nq = n0 + col_of<Acc>(tx, GW * g);
            if (nq >= P.N) continue;
            const long long eo = static_cast<long long>(m) * P.ld_e + nq;
            const long long oo = static_cast<long long>(m) * P.ld_out + nq;
            Acc v[GW];
#pragma unroll
            for (int j = 0; j < GW; ++j) v[j] = alpha * acc[i][GW * g + j];
            if (vec && nq + GW - 1 < P.N) {
                if constexpr (sizeof(Acc) == sizeof(double)) {
                    if (has_e) {
                        const double2 e = *reinterpret_cast<const double2*>(E + eo);
                        v[0] = fma(beta, e.x, v[0]);
                        v[1] = fma(beta, e.y, v[1]);
                    }
                    *reinterpret_cast<double2*>(O + oo) = make_double2(v[0], v[1]);
                } else {
                    if (has_e) {
                        const float4 e = *reinterpret_cast<const float4*>(E + eo);
                        v[0] = fmaf(beta, e.x, v[0]); v[1] = fmaf(beta, e.y, v[1]);
                        v[2] = fmaf(beta, e.z, v[2]); v[3] = fmaf(beta, e.w, v[3]);
                    }
                    *reinterpret_cast<float4*>(O + oo) = make_float4(v[0], v[1], v[2], v[3]);
                }
                continue;
            }
#pragma unroll
            for (int j = 0; j < GW; ++j) {
                const int n = nq + j;
                if (n >= P.N) continue;
                if (P.sym && n < m) continue;   // written by the mirror of (n, m)
                Acc w = v[j];
                if (has_e) w = fma(beta, E[eo + j], w);
                O[oo + j] = w;
                if (P.sym && n > m) O[static_cast<long long>(n) * P.ld_out + m] = w;
            }
        }
    }
}

// fp32: two CTAs (16 warps) per SM; fp64: one (its 8 x 8 fp64 block needs the registers).
template <class Acc, bool A_KC>
__global__ void __launch_bounds__(THREADS, sizeof(Acc) == sizeof(float) ? 2 : 1)
simt_gemm_async_kernel(const SimtProblem* __restrict__ probs, const uint32_t* __restrict__ tiles, int num_tiles) {
    using C = Cfg<Acc>;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    Acc* As = reinterpret_cast<Acc*>(smem_raw);
    Acc* Bs = As + STAGES * C::A_ELEMS;
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x) {
        const uint32_t code = tiles[t];
        const SimtProblem& P = probs[code >> 20];
        const int m0 = static_cast<int>((code >> 10) & 1023u) * BM;
        const int n0 = static_cast<int>(code & 1023u) * BN;
        Ops<Acc> o;
        o.A = static_cast<const Acc*>(P.A);
        o.B = static_cast<const Acc*>(P.B);
        o.sa = A_KC ? P.sam : P.sak;
        o.sbk = P.sbk;
        o.M = P.M; o.N = P.N; o.K = P.K;
        Acc acc[8][8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[i][j] = Acc(0);
        const int ksteps = (o.K + C::BK - 1) / C::BK;
        __syncthreads();   // every thread is done reading the ring for the previous tile
#pragma unroll
        for (int s = 0; s < STAGES - 1; ++s) {
            if (s < ksteps) load_stage<Acc, A_KC>(o, As + s * C::A_ELEMS, Bs + s * C::B_ELEMS, m0, n0, s * C::BK, tid);
            cp_async_commit();
        }
        for (int ks = 0; ks < ksteps; ++ks) {
            cp_async_wait<STAGES - 2>();   // stage ks has landed (for this thread's copies)
            __syncthreads();               // ... for every thread's; slot (ks - 1) % STAGES is free
            const int nx = ks + STAGES - 1;
            if (nx < ksteps) {
                const int slot = nx % STAGES;
                load_stage<Acc, A_KC>(o, As + slot * C::A_ELEMS, Bs + slot * C::B_ELEMS, m0, n0, nx * C::BK, tid);
            }
            cp_async_commit();
            const int cur = ks % STAGES;
            compute_stage<Acc, A_KC>(As + cur * C::A_ELEMS, Bs + cur * C::B_ELEMS, tx, ty, acc);
        }
        cp_async_wait<0>();
        store_tile<Acc>(P, acc, m0, n0, tx, ty);
    }
}

template <class Acc, bool A_KC>
cudaError_t launch_one(const SimtProblem* d_probs, const uint32_t* d_tiles, int num_tiles, cudaStream_t stream) {
    // The shared-memory attribute is per device: set once on each (launches run under the
    // plan cache's lock).
    static bool set_on[64] = {};
    int dev = 0, sms = 148;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!set_on[dev]) {
        e = cudaFuncSetAttribute(simt_gemm_async_kernel<Acc, A_KC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(Cfg<Acc>::SMEM));
        if (e != cudaSuccess) return e;
        set_on[dev] = true;
    }
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const int per_sm = sizeof(Acc) == sizeof(float) ? 2 : 1;
    const int grid = num_tiles < sms * per_sm ? num_tiles : sms * per_sm;
    simt_gemm_async_kernel<Acc, A_KC><<<grid, THREADS, Cfg<Acc>::SMEM, stream>>>(d_probs, d_tiles, num_tiles);
    return cudaGetLastError();
}

}  // namespace

bool simt_async_suits(const std::vector<SimtProblem>& probs, bool* a_kc) {
    if (probs.empty()) return false;
    const long long elt = 4;
    const int want = 0;
    auto al = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    int kc = -1;
    for (const SimtProblem& P : probs) {
        if (P.a_f64 != want || P.b_f64 != want || P.out_f64 != want) return false;
        if (P.beta != 0.f && P.E != nullptr && P.e_f64 != want) return false;
        if (P.sbn != 1 || !al(P.B) || (P.sbk * elt) % 16 != 0 || !al(P.A)) return false;
        int this_kc;
        if (P.sak == 1 && (P.sam * elt) % 16 == 0) this_kc = 1;
        else if (P.sam == 1 && (P.sak * elt) % 16 == 0) this_kc = 0;
        else return false;
        if (kc < 0) kc = this_kc;
        else if (kc != this_kc) return false;
    }
    *a_kc = kc == 1;
    return true;
}

cudaError_t simt_gemm_async_launch(const SimtProblem* d_probs, const uint32_t* d_tiles, int num_tiles,
                                   cudaStream_t stream, bool a_kc) {
    if (num_tiles <= 0) return cudaSuccess;
    return a_kc ? launch_one<float, true>(d_probs, d_tiles, num_tiles, stream)
                : launch_one<float, false>(d_probs, d_tiles, num_tiles, stream);
}

}  // namespace muon
