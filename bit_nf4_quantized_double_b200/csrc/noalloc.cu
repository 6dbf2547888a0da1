// A quantiser entry point that allocates nothing.
//
// qlora_nf4_quantize needs scratch memory (the exact fp32 absmax of every
// 64-weight block and the fp64 partial sums of the offset) and asks the caller
// for it as a workspace. Some callers cannot provide one: code that runs where
// no allocator is reachable (a plugin that is only handed input and output
// buffers, an allocator-free runtime, a host that forbids cudaMalloc after
// start-up). qlora_nf4_quantize_noalloc serves them: its scratch is a
// fixed-size array in this library's device memory, so the call itself never
// allocates or frees device memory.
//
// Cost of that choice: every GPU that loads the library holds kScratchBytes
// (about 4.2 MiB) until the process exits, whether or not the entry point is
// used; tensors above kNoAllocMaxWeights weights are rejected.
#include "launch.h"

namespace qnf4 {
namespace {

constexpr int64_t kNoAllocMaxWeights = int64_t(1) << 26;                     // 67,108,864 weights
constexpr int64_t kNoAllocMaxBlocks = kNoAllocMaxWeights / kBlock1;          // 1,048,576 absmax blocks
constexpr int64_t kNoAllocMaxGroups = kNoAllocMaxBlocks / kBlock2;           // 4,096 second-level groups
constexpr size_t kC1Bytes = (size_t)kNoAllocMaxBlocks * sizeof(float);       // 4 MiB, 256-byte multiple
constexpr size_t kScratchBytes = kC1Bytes + (size_t)kNoAllocMaxGroups * 8 * sizeof(double);

// The scratch array. In host code this name only stands for the symbol; its
// device address is looked up below and passed to the kernels.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

// Device address of the scratch array in the current device's context, looked
// up on every call rather than cached: a context that the caller destroys and
// re-creates (cudaDeviceReset, a primary-context reset) reloads this library's
// device code, and the array may then sit at another address. The lookup is a
// host-side table read once the code is loaded; the first lookup in a context
// loads it.
cudaError_t scratch_address(void **out) {
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    *out = p;
    return cudaSuccess;
}

}  // namespace
}  // namespace qnf4

using namespace qnf4;

extern "C" qlora_status qlora_nf4_quantize_noalloc(const void *W, qlora_dtype dt, const qlora_nf4_tensor *out,
                                                   qlora_stream_t stream) {
    if (!W || !aligned16(W) || !out || (dt != QLORA_F32 && dt != QLORA_BF16)) return QLORA_ERR_INVALID_ARG;
    if (out->rows < 1 || out->cols < 1 || !out->codes || !out->scale8 || !out->scale2 || !out->offset ||
        !aligned16(out->codes) || (reinterpret_cast<uintptr_t>(out->scale2) & 3u) ||
        (reinterpret_cast<uintptr_t>(out->offset) & 3u))
        return QLORA_ERR_INVALID_ARG;
    if (out->cols > kNoAllocMaxWeights || out->rows > kNoAllocMaxWeights / out->cols)
        return QLORA_ERR_UNSUPPORTED_SHAPE;              // more than kNoAllocMaxWeights weights
    const int64_t n = out->rows * out->cols;
    void *scratch = nullptr;
    if (scratch_address(&scratch) != cudaSuccess) return QLORA_ERR_CUDA;
    // The kernels write every scratch element they later read (c1 of every
    // block, one partial per 32 blocks) within this call, so the array needs no
    // clearing between calls.
    float *c1 = static_cast<float *>(scratch);
    double *part = reinterpret_cast<double *>(static_cast<char *>(scratch) + kC1Bytes);
    return launch_quantize(W, dt, n, *out, c1, part, static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? QLORA_OK
               : QLORA_ERR_CUDA;
}
