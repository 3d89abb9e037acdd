// probe.cu -- exercises the bounded-wait path of the tensor-core kernels
// without faulting anything: one thread waits on an mbarrier that no one
// completes, with the same wait routine the kernels use, until its limit
// runs out; it then records IDX_ERR_TIMEOUT in the workspace status word
// and the kernel returns normally, leaving the context usable.
#include "../../include/idx.h"
#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace {

__global__ void wait_probe_kernel(unsigned *status, unsigned long long limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        idx::tc::mbar_init(&bar, 1);  // expects one arrival that never comes
        abort_flag = 0;
        idx::tc::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) idx::tc::mbar_wait(&bar, 0, &abort_flag, status, limit_ns);
    __syncthreads();
}

}  // namespace

extern "C" idx_status idx_debug_wait_probe(void *ws, unsigned limit_ms, idx_stream_t stream) {
    if (!ws || limit_ms == 0 || limit_ms > 10000) return IDX_ERR_INVALID;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(ws, 0, 4, st) != cudaSuccess) return IDX_ERR_CUDA;
    idx::TraceScope ts("wait_probe", st);
    wait_probe_kernel<<<1, 32, 0, st>>>(static_cast<unsigned *>(ws), (unsigned long long)limit_ms * 1000000ull);
    return cudaGetLastError() == cudaSuccess ? IDX_OK : IDX_ERR_CUDA;
}
