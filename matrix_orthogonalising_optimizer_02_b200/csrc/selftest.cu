// Self-test of the bounded device waits: one CTA waits, through the same mbar_wait the
// tensor-core kernel uses, on an mbarrier that nothing ever completes.  The wait gives up
// after its limit (kWaitLimitNs), records kDevErrTimeout in the workspace status word and
// returns, so the kernel ends and the context stays usable: the failure path of every
// pipeline wait is exercised without a fault, a trap or a hang.
#include "../../include/muon_b200.h"
#include "kernels.cuh"
#include "ptx_sm100.cuh"
#include "runtime.cuh"

namespace muon {
namespace {

__global__ void wait_timeout_kernel(unsigned* dev_status) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    // phase 0 of a fresh barrier with one expected arrival that never comes
    if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, dev_status);
}

}  // namespace
}  // namespace muon

extern "C" {

muon_status muon_selftest_wait_timeout(void* workspace, size_t ws_bytes, void* stream_) {
    using namespace muon;
    if (workspace == nullptr || ws_bytes < kHeaderBytes) return MUON_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MUON_ERR_ALIGNMENT;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    unsigned* status = static_cast<unsigned*>(workspace);
    cudaError_t e = cudaMemsetAsync(status, 0, sizeof(unsigned), stream);
    if (e != cudaSuccess) return cuda_error(e, "status clear");
    wait_timeout_kernel<<<1, 32, 0, stream>>>(status);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_error(e, "wait_timeout_kernel launch");
    return MUON_OK;
}

}  // extern "C"
