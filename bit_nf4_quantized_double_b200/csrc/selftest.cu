// Self-tests (the page has no counterpart).
//
// k_selftest_wait: the bounded waits that every pipelined kernel of this library
// uses (part of the library's failure detection). One thread arms an mbarrier
// that nothing will complete and waits on it through the same bounded wait; after
// the wait limit (1 s) the wait gives up, records QLORA_ERR_TIMEOUT in the device
// status word, and the kernel returns normally: no trap, and the context stays
// usable.
//
// k_selftest_rcp: the error of the reciprocal approximation that the quantiser's
// fast path relies on, over all 2^23 mantissas m in [1, 2): |r - 1/m| in units of
// r's ulp, exact in double, as a fixed-point maximum (1024 = one ulp).
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

__global__ void k_selftest_rcp(unsigned int *max_err) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (1 << 23)) return;
    const float m = __uint_as_float(0x3f800000u | (unsigned)i);
    const float r = rcp_approx(m);
    int ex = 0;
    (void)frexp((double)r, &ex);                       // r = f 2^ex, f in [0.5, 1)
    const double ulp = ldexp(1.0, ex - 24);
    const double err = fabs((double)r - 1.0 / (double)m) / ulp;
    atomicMax(max_err, (unsigned int)(err * 1024.0));
}

}  // namespace qnf4

extern "C" qlora_status qlora_selftest_wait_timeout(qlora_stream_t stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    QNF4_LAUNCH("k_selftest_wait", st, qnf4::k_selftest_wait<<<1, 32, 0, st>>>());
    return cudaGetLastError() == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

extern "C" qlora_status qlora_selftest_rcp_error(unsigned int *max_err_1024, qlora_stream_t stream) {
    if (!max_err_1024) return QLORA_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(max_err_1024, 0, sizeof(unsigned int), st) != cudaSuccess) return QLORA_ERR_CUDA;
    QNF4_LAUNCH("k_selftest_rcp", st, qnf4::k_selftest_rcp<<<(1 << 23) / 256, 256, 0, st>>>(max_err_1024));
    return cudaGetLastError() == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}
