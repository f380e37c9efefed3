// Grouped fp64 GEMM on the double-precision tensor cores (mma.sync m16n8k4, fp64 operands,
// fp64 accumulation) for the fp64 products of the Stiefel step's 2k x 2k solve: the LU's
// trailing updates and the blocked back substitution, C <- alpha A B + beta E with A
// row-major along K and B row-major along N.  Same problems, tile codes (128 x 128) and
// results up to the order of the fp64 additions as the FMA-pipe kernel of simt_gemm.cu.
//
// 256 threads = 8 warps in a 2 (M) x 4 (N) grid, each warp 64 x 32 = 4 x 4 tiles of 16 x 8.
// Operand tiles go global -> shared by cp.async in 16-byte chunks (zero-filled outside the
// matrices) through a 2-stage ring of K-steps of 16 (measured faster than 3 or 4 stages,
// likely because the smaller shared-memory footprint leaves more L1 to the epilogue).  The
// first K-step of a CTA's next tile is issued before the epilogue of the current one, so its
// latency hides behind it, and
// the epilogue reads a half tile of E before it stores any result: E may be the output itself,
// so loads placed after stores would each wait out a full memory latency (the LU's K = 128
// updates spend about as long in the epilogue as in the MMAs).  Shared pitches are chosen so
// that every fragment load of a warp touches each bank group once per 16 lanes:
//   A as [m][k], 20 doubles per row (160 B: rows of a quarter-warp land 32 B apart mod 128),
//   B as [k][n], 132 doubles per row (1056 B = 32 B mod 128).
#include <cuda_runtime.h>

#include "simt_async.cuh"

namespace muon {
namespace {

constexpr int BM = 128, BN = 128, BKD = 16, STAGES = 2, THREADS = 256;
constexpr int PA = BKD + 4;     // doubles per A row ([m][k])
constexpr int PB = BN + 4;      // doubles per B row ([k][n])
constexpr int A_ELEMS = BM * PA, B_ELEMS = BKD * PB;
constexpr size_t SMEM = static_cast<size_t>(STAGES) * (A_ELEMS + B_ELEMS) * sizeof(double);
static_assert(BM == kSimtBM && BN == kSimtBN, "tile codes are shared with the FMA-pipe kernel");

__device__ __forceinline__ void cp16(double* smem_dst, const double* gmem_src, int src_bytes) {
    const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem_dst));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(s), "l"(gmem_src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void wait_group() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// D (16 x 8) += A (16 x 4, row) * B (4 x 8, col); lane = 4 g + t holds a0 = A[g][t],
// a1 = A[g + 8][t], b0 = B[t][g], d = D[g][2t], D[g][2t + 1], D[g + 8][2t], D[g + 8][2t + 1].
__device__ __forceinline__ void dmma(double (&d)[4], double a0, double a1, double b0) {
    asm volatile("mma.sync.aligned.m16n8k4.row.col.f64.f64.f64.f64 {%0,%1,%2,%3}, {%4,%5}, {%6}, {%0,%1,%2,%3};"
                 : "+d"(d[0]), "+d"(d[1]), "+d"(d[2]), "+d"(d[3])
                 : "d"(a0), "d"(a1), "d"(b0));
}

// One K-step of operand tiles: A rows m0 .. m0 + 127, columns k0 .. k0 + 15 (64 chunks of 16
// bytes per 8 rows); B rows k0 .. k0 + 15, columns n0 .. n0 + 127.  4 + 4 chunks per thread.
__device__ __forceinline__ void load_stage(const SimtProblem& P, double* As, double* Bs, int m0, int n0, int k0,
                                           int tid) {
    const double* A = static_cast<const double*>(P.A);
    const double* B = static_cast<const double*>(P.B);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int c = tid + q * THREADS;               // 1024 chunks: 128 rows x 8 chunks
        const int r = c >> 3, kc = (c & 7) * 2;
        const int gm = m0 + r, gk = k0 + kc;
        const bool in = gm < P.M && gk < P.K;           // K is even: a chunk is wholly in or out
        cp16(As + r * PA + kc, in ? A + static_cast<long long>(gm) * P.sam + gk : A, in ? 16 : 0);
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int c = tid + q * THREADS;               // 1024 chunks: 16 rows x 64 chunks
        const int r = c >> 6, nc = (c & 63) * 2;
        const int gk = k0 + r, gn = n0 + nc;
        const bool in = gk < P.K && gn < P.N;           // N is even
        cp16(Bs + r * PB + nc, in ? B + static_cast<long long>(gk) * P.sbk + gn : B, in ? 16 : 0);
    }
}

// out = f * (alpha * acc + beta * E) for the rows of register-block rows i0, i0 + 1 of this
// thread (two consecutive columns per access).  All E values are loaded before the first
// store: E is either the output itself (the same element read and written by this thread)
// or a disjoint array.
__device__ __forceinline__ void store_half(const SimtProblem& P, const double (&acc)[4][4][4], int i0, int m_base,
                                           int n_base, int g, int t, double alpha, double beta, bool has_e) {
    double* O = static_cast<double*>(P.out);
    const double* E = static_cast<const double*>(P.E);
    double2 e[2][2][4];
#pragma unroll
    for (int ii = 0; ii < 2; ++ii)
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int m = m_base + 16 * (i0 + ii) + g + 8 * h, n = n_base + 8 * j + 2 * t;
                e[ii][h][j] = (has_e && m < P.M && n < P.N)
                                  ? *reinterpret_cast<const double2*>(E + static_cast<long long>(m) * P.ld_e + n)
                                  : make_double2(0.0, 0.0);
            }
#pragma unroll
    for (int ii = 0; ii < 2; ++ii)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int m = m_base + 16 * (i0 + ii) + g + 8 * h;
            if (m >= P.M) continue;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int n = n_base + 8 * j + 2 * t;
                if (n >= P.N) continue;
                const double v0 = fma(beta, e[ii][h][j].x, alpha * acc[i0 + ii][j][2 * h]);
                const double v1 = fma(beta, e[ii][h][j].y, alpha * acc[i0 + ii][j][2 * h + 1]);
                *reinterpret_cast<double2*>(O + static_cast<long long>(m) * P.ld_out + n) = make_double2(v0, v1);
            }
        }
}

__device__ __forceinline__ void decode_tile(uint32_t code, int& p, int& m0, int& n0) {
    p = static_cast<int>(code >> 20);
    m0 = static_cast<int>((code >> 10) & 1023u) * BM;
    n0 = static_cast<int>(code & 1023u) * BN;
}

// The first STAGES - 1 K-steps of a tile, one commit group each (empty past the end).
__device__ __forceinline__ void prologue(const SimtProblem& P, double* As, double* Bs, int m0, int n0, int tid) {
    const int ksteps = (P.K + BKD - 1) / BKD;
#pragma unroll
    for (int s = 0; s < STAGES - 1; ++s) {
        if (s < ksteps) load_stage(P, As + s * A_ELEMS, Bs + s * B_ELEMS, m0, n0, s * BKD, tid);
        commit();
    }
}

__global__ void __launch_bounds__(THREADS, 1)
dmma_gemm_kernel(const SimtProblem* __restrict__ probs, const uint32_t* __restrict__ tiles, int num_tiles) {
    extern __shared__ __align__(16) double smem[];
    double* As = smem;
    double* Bs = smem + STAGES * A_ELEMS;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    const int wm = (warp >> 2) * 64, wn = (warp & 3) * 32;   // warp tile origin in the CTA tile
    int tt = blockIdx.x;
    if (tt >= num_tiles) return;
    int p, m0, n0;
    decode_tile(tiles[tt], p, m0, n0);
    prologue(probs[p], As, Bs, m0, n0, tid);
    while (true) {
        const SimtProblem& P = probs[p];
        double acc[4][4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[i][j][e] = 0.0;
        const int ksteps = (P.K + BKD - 1) / BKD;
        for (int ks = 0; ks < ksteps; ++ks) {
            wait_group<STAGES - 2>();   // stage ks has landed (this thread's copies)
            __syncthreads();            // ... every thread's; slot (ks - 1) % STAGES is free
            const int nx = ks + STAGES - 1;
            if (nx < ksteps) load_stage(P, As + (nx % STAGES) * A_ELEMS, Bs + (nx % STAGES) * B_ELEMS, m0, n0, nx * BKD, tid);
            commit();
            const double* a = As + (ks % STAGES) * A_ELEMS;
            const double* b = Bs + (ks % STAGES) * B_ELEMS;
#pragma unroll
            for (int kk = 0; kk < BKD; kk += 4) {
                double af[4][2], bf[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    af[i][0] = a[(wm + 16 * i + g) * PA + kk + t];
                    af[i][1] = a[(wm + 16 * i + g + 8) * PA + kk + t];
                }
#pragma unroll
                for (int j = 0; j < 4; ++j) bf[j] = b[(kk + t) * PB + wn + 8 * j + g];
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) dmma(acc[i][j], af[i][0], af[i][1], bf[j]);
            }
        }
        // every thread is done reading the ring: start the next tile's loads, then run this
        // tile's epilogue while they land
        __syncthreads();
        const int next = tt + static_cast<int>(gridDim.x);
        int np = 0, nm0 = 0, nn0 = 0;
        if (next < num_tiles) {
            decode_tile(tiles[next], np, nm0, nn0);
            prologue(probs[np], As, Bs, nm0, nn0, tid);
        }
        float f = 1.f;
        if (P.dscale != nullptr && P.scale_pow > 0) {
            const float sc = __ldg(P.dscale);
            f = (P.scale_pow == 1) ? sc : sc * sc;
        }
        const double alpha = static_cast<double>(P.alpha * f), beta = static_cast<double>(P.beta * f);
        const bool has_e = P.beta * f != 0.f && P.E != nullptr;
        store_half(P, acc, 0, m0 + wm, n0 + wn, g, t, alpha, beta, has_e);
        store_half(P, acc, 2, m0 + wm, n0 + wn, g, t, alpha, beta, has_e);
        if (next >= num_tiles) break;
        tt = next; p = np; m0 = nm0; n0 = nn0;
    }
    wait_group<0>();
}

}  // namespace

bool dmma_gemm_suits(const std::vector<SimtProblem>& probs) {
    if (probs.empty()) return false;
    auto al = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    for (const SimtProblem& P : probs) {
        if (!P.a_f64 || !P.b_f64 || !P.out_f64 || P.sym) return false;
        if (P.beta != 0.f && P.E != nullptr && !P.e_f64) return false;
        if (P.sak != 1 || P.sbn != 1) return false;                        // A along K, B along N
        if ((P.K & 1) || (P.N & 1)) return false;                          // whole 16-byte chunks
        if (!al(P.A) || !al(P.B) || !al(P.out) || (P.sam & 1) || (P.sbk & 1) || (P.ld_out & 1)) return false;
        if (P.E != nullptr && (!al(P.E) || (P.ld_e & 1))) return false;
    }
    return true;
}

cudaError_t dmma_gemm_launch(const SimtProblem* d_probs, const uint32_t* d_tiles, int num_tiles, cudaStream_t stream) {
    if (num_tiles <= 0) return cudaSuccess;
    static bool set_on[64] = {};
    int dev = 0, sms = 148;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!set_on[dev]) {   // per device, once (launches run under the plan cache's lock)
        e = cudaFuncSetAttribute(dmma_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(SMEM));
        if (e != cudaSuccess) return e;
        set_on[dev] = true;
    }
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const int grid = num_tiles < sms ? num_tiles : sms;
    dmma_gemm_kernel<<<grid, THREADS, SMEM, stream>>>(d_probs, d_tiles, num_tiles);
    return cudaGetLastError();
}

}  // namespace muon
