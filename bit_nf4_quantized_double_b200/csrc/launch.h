// Internal launch interface between the C-ABI layer and the kernel files.
#pragma once

#include "common.cuh"

namespace qnf4 {

cudaError_t launch_quantize(const void *W, qlora_dtype dt, int64_t n, const qlora_nf4_tensor &out,
                            float *c1, double *part, cudaStream_t st);
// One tensor of a grouped quantisation: input, weights, output buffers and its workspace slices.
struct QuantArgs {
    const void *W;
    int64_t n;
    qlora_nf4_tensor out;
    float *c1;
    double *part;
};
cudaError_t launch_quantize_grouped(const QuantArgs *a, int count, qlora_dtype dt, cudaStream_t st);
// ctas_per_sm caps the persistent grid (8 fills the SMs; fewer leave room for a kernel
// running beside it on another stream).
cudaError_t launch_dequant(const NF4View &q, __nv_bfloat16 *out, cudaStream_t st, int ctas_per_sm = 8);
cudaError_t launch_dequant_grouped(const NF4View *q, __nv_bfloat16 *const *out, int count, cudaStream_t st);
cudaError_t launch_fmt4_quantize(const void *W, qlora_dtype dt, int64_t n, qlora_fmt4 f, uint8_t *codes,
                                 float *absmax, cudaStream_t st);
cudaError_t launch_fmt4_dequant(const uint8_t *codes, const float *absmax, int64_t n, qlora_fmt4 f,
                                __nv_bfloat16 *out, cudaStream_t st);
cudaError_t launch_adamw(float *theta, const float *g, float *m, float *v, int64_t n, float lr, float b1, float b2,
                         float eps, float wd, int64_t step, __nv_bfloat16 *out_bf16, cudaStream_t st);
cudaError_t launch_prefetch(const void *ptr, size_t bytes, bool to_device, cudaStream_t st);
// Adapter merge: k_merge_prep (A^T and B widened to fp32 into `prep`, merge_prep_bytes)
// then k_merge_bf16.
size_t merge_prep_bytes(int64_t rows, int64_t cols);
cudaError_t launch_merge_bf16(const NF4View &q, const __nv_bfloat16 *A, const __nv_bfloat16 *B, int r, float s,
                              __nv_bfloat16 *out, void *prep, cudaStream_t st);

// Plain bf16 GEMM on CTA pairs (tcgen05 cta_group::2), see gemm2sm.cu.
int gemm2sm_pairs(int max_pairs);
int gemm2sm_max_splits();
cudaError_t launch_gemm2sm(const __nv_bfloat16 *A, const __nv_bfloat16 *Ae, const __nv_bfloat16 *B, bool b_mn,
                           const __nv_bfloat16 *Be, bool be_mn, __nv_bfloat16 *C, int64_t M, int64_t N, int64_t K,
                           int ke, int pairs, int splits, float *partial, bool pdl, bool wait_first,
                           cudaStream_t st);

size_t fwd_workspace_bytes(int64_t M, int64_t rows, int64_t cols, int r);

// One projection of a grouped forward (device pointers; validated by the caller).
struct LinearDesc {
    const __nv_bfloat16 *X = nullptr;
    NF4View W{};
    const __nv_bfloat16 *A = nullptr, *B = nullptr;
    int r = 0;
    float s = 0.0f;
    __nv_bfloat16 *Y = nullptr, *XA_save = nullptr;
};
size_t fwd_grouped_workspace_bytes(int64_t M, int count, const LinearDesc *d);
cudaError_t launch_linear_fwd_grouped(int64_t M, int count, const LinearDesc *d, void *ws, cudaStream_t st);
size_t bwd_workspace_bytes(int64_t M, int64_t rows, int64_t cols, int r);

cudaError_t launch_linear_fwd(const __nv_bfloat16 *X, int64_t M, const NF4View &W,
                              const __nv_bfloat16 *A, const __nv_bfloat16 *B, int r, float s,
                              __nv_bfloat16 *Y, __nv_bfloat16 *XA_save, void *ws, cudaStream_t st);

cudaError_t launch_linear_bwd(const __nv_bfloat16 *X, const __nv_bfloat16 *dY, int64_t M, const NF4View &W,
                              const __nv_bfloat16 *A, const __nv_bfloat16 *B, int r, float s,
                              const __nv_bfloat16 *XA, __nv_bfloat16 *dX, float *dA, float *dB,
                              void *ws, cudaStream_t st);

}  // namespace qnf4
