// Shared device helpers of the QLoRA NF4 library (sm_100a).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "qlora_nf4.h"

namespace qnf4 {

constexpr int kBlock1 = 64;    // weights per first-level absmax block
constexpr int kBlock2 = 256;   // first-level constants per second-level block

// Per-device status word: bit (1 << status) is set by a kernel that detects a
// condition; the host reads and clears it in qlora_get_device_status().
extern __device__ unsigned int g_status_bits;

__device__ __forceinline__ void raise_status(qlora_status s) {
    atomicOr(&g_status_bits, 1u << (unsigned)s);
}

// The codebook and its decision thresholds, passed by value to the kernels
// that need them (kernel parameters live in the constant bank).
struct Codebook {
    float q[16];   // ascending, q[7] = +0
    float t[15];   // t[i] = fl(fl(q[i] + q[i+1]) * 0.5)
};

// Device view of a stored tensor.
struct NF4View {
    const uint8_t *codes;
    const int8_t *scale8;
    const float *scale2;
    const float *offset;
    int64_t rows, cols;
};

// c^_b = fl(fl(q8 * fl(s2 / 127)) + mu), every step a separately rounded
// IEEE operation (no contraction into a fused multiply-add).
__device__ __forceinline__ float dq_constant(int8_t q8, float s2, float mu) {
    const float step = __fdiv_rn(s2, 127.0f);
    return __fadd_rn(__fmul_rn((float)q8, step), mu);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);   // .x = lo (low half), .y = hi
    return *reinterpret_cast<uint32_t *>(&v);
}

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

// The hardware reciprocal approximation (PTX rcp.approx.ftz.f32, documented to
// within 1 ulp; qlora_selftest_rcp_error measures it over every mantissa).
__device__ __forceinline__ float rcp_approx(float x) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ uint4 ldg_nc_v4(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
    return r;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

}  // namespace qnf4

// Host-side helpers shared by the launch code.
namespace qnf4 {
inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
const Codebook &host_codebook();
int num_sms();
// Launch bookkeeping (profile.cu): counts every launch and, when profiling is
// enabled, brackets it with CUDA events on its stream.
void note_launch_begin(const char *name, cudaStream_t st, void **token);
void note_launch_end(void *token, cudaStream_t st);
// True while per-launch event timing is on: launches then drop programmatic dependent
// launch, so that each kernel's events bracket its own run and not its overlap with the
// kernel before it.
bool profiling_launches();
}  // namespace qnf4

#define QNF4_LAUNCH(name, st, ...)                         \
    do {                                                   \
        void *qnf4_tok_ = nullptr;                         \
        ::qnf4::note_launch_begin(name, st, &qnf4_tok_);   \
        __VA_ARGS__;                                       \
        ::qnf4::note_launch_end(qnf4_tok_, st);            \
    } while (0)
