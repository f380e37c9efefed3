// Multi-stage (cp.async) variant of the grouped SIMT GEMM for the common operand layouts.
#pragma once
#include <cuda_runtime.h>

#include <vector>

#include "kernels.cuh"

namespace muon {

// True if every problem suits simt_gemm_async_launch: B row-major along N (sbn == 1), A
// row-major along K (sak == 1) for all problems or along M (sam == 1) for all problems, A, B,
// out (and E if beta != 0) stored as fp32, 16-byte aligned bases and row pitches.  *a_kc
// receives A's layout.
bool simt_async_suits(const std::vector<SimtProblem>& probs, bool* a_kc);

// Same contract and tile codes as simt_gemm_launch with fp32 accumulation (128 x 128 tiles),
// operand tiles staged by cp.async through a 2-deep shared-memory ring of K-steps of 32.
cudaError_t simt_gemm_async_launch(const SimtProblem* d_probs, const uint32_t* d_tiles, int num_tiles,
                                   cudaStream_t stream, bool a_kc);

// True if every problem suits dmma_gemm_launch: A, B, out (and E if used) fp64, A row-major
// along K, B row-major along N, not symmetric, K and N even, 16-byte aligned bases and even
// row pitches.
bool dmma_gemm_suits(const std::vector<SimtProblem>& probs);

// The same problems and 128 x 128 tile codes as simt_gemm_launch with fp64 accumulation, on
// the double-precision tensor cores (mma.sync m16n8k4 f64).
cudaError_t dmma_gemm_launch(const SimtProblem* d_probs, const uint32_t* d_tiles, int num_tiles, cudaStream_t stream);

}  // namespace muon
