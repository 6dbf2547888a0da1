// Self-test of the bounded waits that every pipelined kernel of this library
// uses (the page has no counterpart: it is part of the library's failure
// detection). One thread arms an mbarrier that nothing will complete and waits
// on it through the same bounded wait; after the wait limit (1 s) the wait gives
// up, records QLORA_ERR_TIMEOUT in the device status word, and the kernel
// returns normally: no trap, and the context stays usable.
#include "launch.h"
#include "tc.cuh"

namespace qnf4 {
using namespace tc;

__global__ void k_selftest_wait() {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int s_abort;
    if (threadIdx.x == 0) {
        mbar_init(smem_addr(&bar), 1);
        s_abort = 0;
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) (void)mbar_wait(smem_addr(&bar), 0, &s_abort);
}

}  // namespace qnf4

extern "C" qlora_status qlora_selftest_wait_timeout(qlora_stream_t stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    QNF4_LAUNCH("k_selftest_wait", st, qnf4::k_selftest_wait<<<1, 32, 0, st>>>());
    return cudaGetLastError() == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}
