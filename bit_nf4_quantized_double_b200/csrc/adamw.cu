// Optimizer step of the adapter: AdamW on fp32 master parameters with fp32
// moments, whose state may live in unified (managed) memory.
//
// Method: "QLoRA: put the large model in memory, then change it with a small
// adapter" (wq-win.github.io/llm/074-qlora): section 3's procedure ends every
// batch with "update LoRA with a paged optimizer"; section 2 describes paged
// optimizers as keeping their state in unified memory that is moved between
// GPU and CPU memory when needed. The frozen NF4 weight gets no update.
//
// One element per lane, four per thread (16-byte loads and stores), in this
// order, every step one IEEE binary32 operation (no contraction):
//   m = fl(fl(b1 m) + fl(c1 g)),  v = fl(fl(b2 v) + fl(c2 fl(g g))),  c = 1 - b
//   upd = fl(fl(m ib1) / fl(fl(sqrt(fl(v ib2))) + eps))
//   theta = fl(theta - fl(lr fl(upd + fl(wd theta))))
// The inverse bias corrections ib1 = 1 / (1 - b1^t) and ib2 = 1 / (1 - b2^t) are
// computed once on the host in double and rounded to float, so each parameter
// costs one division and one square root. The kernel is HBM-bound: 30 bytes per
// parameter (theta, m, v read and written, g read, the bf16 copy written).
#include <cmath>

#include "launch.h"

namespace qnf4 {

struct AdamwConsts {
    float lr, b1, b2, c1, c2, eps, wd, ib1, ib2;
};

__device__ __forceinline__ float adamw_one(float &theta, float g, float &m, float &v, const AdamwConsts &k) {
    const float mi = __fadd_rn(__fmul_rn(k.b1, m), __fmul_rn(k.c1, g));
    const float vi = __fadd_rn(__fmul_rn(k.b2, v), __fmul_rn(k.c2, __fmul_rn(g, g)));
    const float den = __fadd_rn(__fsqrt_rn(__fmul_rn(vi, k.ib2)), k.eps);
    const float upd = __fdiv_rn(__fmul_rn(mi, k.ib1), den);
    const float t = __fsub_rn(theta, __fmul_rn(k.lr, __fadd_rn(upd, __fmul_rn(k.wd, theta))));
    m = mi;
    v = vi;
    theta = t;
    return t;
}

__global__ void __launch_bounds__(256)
k_adamw(float *__restrict__ theta, const float *__restrict__ g, float *__restrict__ m, float *__restrict__ v,
        int64_t n, AdamwConsts k, __nv_bfloat16 *__restrict__ out_bf16) {
    const int64_t n4 = n / 4;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride) {
        float4 th = reinterpret_cast<const float4 *>(theta)[i];
        const float4 gg = __ldg(reinterpret_cast<const float4 *>(g) + i);
        float4 mm = reinterpret_cast<const float4 *>(m)[i];
        float4 vv = reinterpret_cast<const float4 *>(v)[i];
        adamw_one(th.x, gg.x, mm.x, vv.x, k);
        adamw_one(th.y, gg.y, mm.y, vv.y, k);
        adamw_one(th.z, gg.z, mm.z, vv.z, k);
        adamw_one(th.w, gg.w, mm.w, vv.w, k);
        reinterpret_cast<float4 *>(theta)[i] = th;
        reinterpret_cast<float4 *>(m)[i] = mm;
        reinterpret_cast<float4 *>(v)[i] = vv;
        if (out_bf16)
            reinterpret_cast<uint2 *>(out_bf16)[i] = make_uint2(pack_bf16x2(th.x, th.y), pack_bf16x2(th.z, th.w));
    }
    // the last n % 4 parameters
    if (blockIdx.x == 0 && (int64_t)threadIdx.x < n - 4 * n4) {
        const int64_t e = 4 * n4 + threadIdx.x;
        float th = theta[e], mm = m[e], vv = v[e];
        adamw_one(th, g[e], mm, vv, k);
        theta[e] = th;
        m[e] = mm;
        v[e] = vv;
        if (out_bf16) out_bf16[e] = __float2bfloat16_rn(th);
    }
}

cudaError_t launch_adamw(float *theta, const float *g, float *m, float *v, int64_t n, float lr, float b1, float b2,
                         float eps, float wd, int64_t step, __nv_bfloat16 *out_bf16, cudaStream_t st) {
    AdamwConsts k;
    k.lr = lr;
    k.b1 = b1;
    k.b2 = b2;
    k.c1 = 1.0f - b1;
    k.c2 = 1.0f - b2;
    k.eps = eps;
    k.wd = wd;
    k.ib1 = (float)(1.0 / (1.0 - std::pow((double)b1, (double)step)));
    k.ib2 = (float)(1.0 / (1.0 - std::pow((double)b2, (double)step)));
    int64_t grid = ceil_div(ceil_div(n, 4), 256);
    const int64_t cap = (int64_t)num_sms() * 8;
    if (grid > cap) grid = cap;
    if (grid < 1) grid = 1;
    QNF4_LAUNCH("k_adamw", st, k_adamw<<<(unsigned)grid, 256, 0, st>>>(theta, g, m, v, n, k, out_bf16));
    return cudaGetLastError();
}

cudaError_t launch_prefetch(const void *ptr, size_t bytes, bool to_device, cudaStream_t st) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    return cudaMemPrefetchAsync(ptr, bytes, to_device ? dev : cudaCpuDeviceId, st);
}

}  // namespace qnf4
