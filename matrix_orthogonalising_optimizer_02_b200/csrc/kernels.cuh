// Kernel-level interfaces shared by the kernel files and the host orchestration.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace muon {

// Device status bits (first word of every workspace).
constexpr unsigned kDevErrTimeout = 1u;
constexpr unsigned kDevErrNonfinite = 2u;
// After a timeout, copies or MMAs already issued did not finish within the drain limit
// before the kernel released its shared and tensor memory.
constexpr unsigned kDevErrUndrained = 4u;

// ------------------------------------------------------------------ tcgen05 grouped GEMM
// One problem of a grouped launch: out = f * (alpha * (A_op x B_op) + beta * E), f = 1 or
// (*dscale)^scale_pow, on bf16 operands with fp32 accumulation in TMEM.  A_op is M x K,
// B_op is K x N; each is read through TMA tensor maps, K-major (contiguous along K) or
// MN-major (contiguous along M resp. N).  An operand may come as up to three bf16 planes
// (value = plane0 + plane1 + plane2); the K loop runs over a list of plane pairs
// ("segments"), e.g. (0,0),(0,1),(1,0) for split-bf16, or the six pairs with indices
// summing to <= 2 for an fp32 operand split into three planes.  K starts at k_begin
// (split-K chunks).  The output is bf16 (plane 0 = value, optional plane 1 = remainder)
// or fp32; E is bf16 (one or two planes) or fp32.  With kProbSym the output is
// symmetric: only tiles that reach the upper triangle are computed, and their elements
// above the diagonal are also stored mirrored.
constexpr uint32_t kProbAMn = 1u;
constexpr uint32_t kProbBMn = 2u;
constexpr uint32_t kProbSym = 4u;
constexpr uint32_t kProbOutF32 = 8u;
constexpr uint32_t kProbEF32 = 16u;
constexpr int kTcMaxPlanes = 3, kTcMaxSegments = 8;

struct alignas(16) TcProblem {
    const CUtensorMap* tmA[kTcMaxPlanes];
    const CUtensorMap* tmB[kTcMaxPlanes];
    const void* E[2];
    void* out[2];
    const float* dscale;
    int M, N, K;
    int k_begin;
    int ld;            // row pitch (elements) of out and E
    float alpha, beta;
    int scale_pow;
    uint32_t flags;
    int nseg;
    uint32_t segs;     // segment s: A plane = (segs >> 4s) & 3, B plane = (segs >> (4s + 2)) & 3
};

// Segment list of plane pairs (pa, pb) with pa < na, pb < nb and pa + pb <= max_order,
// ordered by pa + pb (largest terms first).
inline void tc_set_segments(TcProblem& P, int na, int nb, int max_order) {
    P.nseg = 0;
    P.segs = 0;
    for (int o = 0; o <= max_order; ++o)
        for (int pa = 0; pa <= o; ++pa) {
            const int pb = o - pa;
            if (pa < na && pb < nb && P.nseg < kTcMaxSegments) {
                P.segs |= static_cast<uint32_t>(pa | (pb << 2)) << (4 * P.nseg);
                ++P.nseg;
            }
        }
}

constexpr int kTcBM = 256, kTcBN = 256, kTcBK = 64;   // pair (2-CTA) tile
// Depth of the TMA ring.  On the power-capped part 4 stages measured fastest: a deeper ring
// keeps the tensor pipe busier per cycle but lowers the sustained clock by more.
constexpr int kTcStages = 4;
constexpr int kTcThreads = 384;            // 4 role warps + 8 epilogue warps
constexpr int kTcEpilogueThreads = 256;
// Tile code: problem (12 bits) | m block (10 bits) | n block (10 bits).
__host__ __device__ inline uint32_t tile_code(int p, int mb, int nb) {
    return (static_cast<uint32_t>(p) << 20) | (static_cast<uint32_t>(mb) << 10) | static_cast<uint32_t>(nb);
}
constexpr int kMaxTileProblems = 4096, kMaxTileBlocks = 1024;

size_t tc_gemm_smem_bytes();
cudaError_t tc_gemm_launch(const TcProblem* d_probs, const uint32_t* d_tiles, int num_tiles, unsigned* d_status,
                           int num_sms, cudaStream_t stream);

// ------------------------------------------------------------------ SIMT grouped GEMM
// out[m*ld_out + n] = f * (alpha * sum_k A(m,k) B(k,n) + beta * E[m*ld_e + n]),
// A(m,k) = A[m*sam + k*sak], B(k,n) = B[k*sbk + n*sbn], on the FMA pipes (no TF32).  Each
// of A, B, E, out is fp32 or fp64 (flags); the accumulator type is chosen per launch.
struct alignas(16) SimtProblem {
    const void* A;
    const void* B;
    const void* E;
    void* out;
    const float* dscale;
    long long sam, sak, sbk, sbn;
    long long ld_out, ld_e;
    int M, N, K;
    float alpha, beta;
    int scale_pow;
    int vec_a, vec_b;  // 16-byte vector loads allowed along the contiguous dimension
    int a_f64, b_f64, e_f64, out_f64;
    int sym;           // symmetric output: only tiles with n-block >= m-block; mirrored stores
};
constexpr int kSimtBM = 128, kSimtBN = 128, kSimtBK = 8, kSimtThreads = 256;
cudaError_t simt_gemm_launch(const SimtProblem* d_probs, const uint32_t* d_tiles, int num_tiles, cudaStream_t stream,
                             bool f64_acc = false);

// ------------------------------------------------------------------ elementwise
// Per matrix of a momentum/cast launch.
struct alignas(16) MomentumItem {
    const void* G;       // bf16 or fp32
    float* M;            // fp32, updated in place (nullable: then X0 = cast(G))
    void* X0;            // bf16 (or fp32 in fp32 mode)
    long long n;         // elements
    long long block0;    // first block index of this matrix
    int g_f32;           // G dtype
    int x_f32;           // X0 dtype
    int vec;             // all pointers 16-byte aligned: 128-bit accesses allowed
};
cudaError_t momentum_cast_launch(const MomentumItem* d_items, int count, long long total_blocks, float beta,
                                 int nesterov, double* d_partials, cudaStream_t stream);
constexpr int kEwThreads = 256;
constexpr int kEwElemsPerBlock = 8192;   // 256 threads x 8 elements x 4

// scale[i] = 1 / (sqrt(sum of partials of matrix i) + eps); flags non-finite sums.
cudaError_t frob_scale_launch(const long long* d_block0, const long long* d_nblocks, int count,
                              const double* d_partials, float eps, float* d_scale, unsigned* d_status,
                              cudaStream_t stream);

struct alignas(16) UpdateItem {
    void* W;             // bf16 or fp32, in place
    const void* O;       // bf16 or fp32 NS output (natural layout)
    void* O_out;         // optional copy of f*O (same dtype as O)
    const float* dscale; // nullable: O is multiplied by *dscale (NS with zero iterations)
    long long n;
    long long block0;
    float decay;         // 1 - lr*wd
    float step;          // -lr*scale
    int w_f32;
    int o_f32;
    int vec;
};
cudaError_t update_launch(const UpdateItem* d_items, int count, long long total_blocks, cudaStream_t stream);

// ------------------------------------------------------------------ fused small fp32 step
// One cluster of kSmallCluster CTAs per matrix runs momentum, Frobenius pre-scale, every
// Newton-Schulz iteration and the update of an fp32-mode matrix with r = min(rows, cols) <=
// kSmallMaxR (r % 8 == 0) and ceil(max(rows, cols) / kSmallCluster) <= kSmallMaxR.
constexpr int kSmallCluster = 8, kSmallThreads = 256, kSmallMaxR = 128;
struct alignas(16) SmallItem {
    const void* G;   // gradient (step) or input X (orthogonalisation only); bf16 or fp32
    float* M;        // momentum, updated in place; nullptr: X0 = G
    void* W;         // weights, updated in place; nullptr: no update
    void* O;         // optional copy of the orthogonalised matrix
    int rows, cols;
    int g_f32, w_f32, o_f32;
    float decay;     // 1 - lr*wd
    float step;      // -lr*scale
};
struct SmallParams {
    float beta;
    int nesterov;
    float eps;
    int n_iters;
    float coeffs[3 * 32];
};
bool ns_small_fits(int rows, int cols);
size_t ns_small_smem_bytes();
cudaError_t ns_small_launch(const SmallItem* d_items, int count, const SmallParams& prm, unsigned* d_status,
                            cudaStream_t stream);

// dst (dtype dst_f32) = f * src (bf16 or fp32), f = *dscale or 1; batched items.
struct alignas(16) CastItem {
    const void* src;
    void* dst;
    const float* dscale;
    long long n;
    long long block0;
    int src_f32;
    int dst_f32;
    int vec;
};
cudaError_t cast_launch(const CastItem* d_items, int count, long long total_blocks, cudaStream_t stream);

}  // namespace muon
