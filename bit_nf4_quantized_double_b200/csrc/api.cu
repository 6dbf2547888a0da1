// C-ABI entry points of the QLoRA NF4 library: argument checks, workspace
// layout and launch sequencing. Every step of the computation runs in the
// kernels of quant.cu, gemm_tc.cu and gemv.cu.
#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "launch.h"

namespace qnf4 {

// ---------------------------------------------------------------- codebook
// Upper standard-normal quantile by Newton's method on Phi(x) - p with
// Phi(x) = 1 - erfc(x / sqrt 2) / 2, started at x = 0. Phi is concave on
// x >= 0, so the iterates rise monotonically to the root.
static double upper_normal_quantile(double p) {
    const double q = 1.0 - p;
    double x = 0.0;
    for (int it = 0; it < 200; ++it) {
        const double tail = 0.5 * std::erfc(x / std::sqrt(2.0));
        const double dens = std::exp(-0.5 * x * x) / std::sqrt(2.0 * M_PI);
        const double dx = (tail - q) / dens;
        x += dx;
        if (std::fabs(dx) <= 1e-16 * (x > 1.0 ? x : 1.0)) break;
    }
    return x;
}

static Codebook derive_codebook() {
    // 8 positive and 7 negative quantiles at equally spaced probabilities that
    // end at delta, plus an exact zero, divided by the quantile at delta.
    const double delta = 1.0 - 0.5 * (1.0 / 32.0 + 1.0 / 30.0);
    const double top = upper_normal_quantile(delta);
    double v[16];
    for (int j = 1; j <= 7; ++j) v[7 - j] = -upper_normal_quantile(0.5 + (delta - 0.5) * ((double)j / 7.0)) / top;
    v[7] = 0.0;
    for (int j = 1; j <= 8; ++j) v[7 + j] = upper_normal_quantile(0.5 + (delta - 0.5) * ((double)j / 8.0)) / top;
    Codebook cb;
    for (int i = 0; i < 16; ++i) cb.q[i] = (float)v[i];
    for (int i = 0; i < 15; ++i) {
        volatile float s = cb.q[i] + cb.q[i + 1];   // one rounding for the sum,
        cb.t[i] = s * 0.5f;                          // one (exact) for the halving
    }
    return cb;
}

const Codebook &host_codebook() {
    static const Codebook cb = derive_codebook();
    return cb;
}

int num_sms() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

static qlora_status from_cuda(cudaError_t e) { return e == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA; }

static bool tensor_ok(const qlora_nf4_tensor *t) {
    return t && t->rows >= 1 && t->cols >= 1 && t->codes && t->scale8 && t->scale2 && t->offset &&
           aligned16(t->codes) && (reinterpret_cast<uintptr_t>(t->scale2) & 3u) == 0 &&
           (reinterpret_cast<uintptr_t>(t->offset) & 3u) == 0;
}

static NF4View view_of(const qlora_nf4_tensor *t) {
    return NF4View{t->codes, t->scale8, t->scale2, t->offset, t->rows, t->cols};
}

}  // namespace qnf4

using namespace qnf4;

extern "C" {

size_t qlora_nf4_storage_bytes(int64_t rows, int64_t cols) {
    if (rows < 1 || cols < 1) return 0;
    const int64_t n = rows * cols, nb = ceil_div(n, kBlock1), nb2 = ceil_div(nb, kBlock2);
    return (size_t)(ceil_div(n, 2) + nb + 4 * nb2 + 4);
}

size_t qlora_nf4_quantize_workspace(int64_t rows, int64_t cols) {
    if (rows < 1 || cols < 1) return 0;
    const int64_t n = rows * cols, nb = ceil_div(n, kBlock1), nb2 = ceil_div(nb, kBlock2);
    return align256((size_t)nb * 4) + align256((size_t)nb2 * 64);
}

qlora_status qlora_nf4_quantize(const void *W, qlora_dtype dt, const qlora_nf4_tensor *out,
                                void *ws, size_t ws_bytes, qlora_stream_t stream) {
    if (!W || !aligned16(W) || !tensor_ok(out) || (dt != QLORA_F32 && dt != QLORA_BF16))
        return QLORA_ERR_INVALID_ARG;
    const size_t need = qlora_nf4_quantize_workspace(out->rows, out->cols);
    if (!ws || ws_bytes < need || !aligned16(ws)) return QLORA_ERR_WORKSPACE;
    const int64_t n = out->rows * out->cols, nb = ceil_div(n, kBlock1), nb2 = ceil_div(nb, kBlock2);
    if (nb2 > 0x7fffffffLL) return QLORA_ERR_UNSUPPORTED_SHAPE;
    float *c1 = static_cast<float *>(ws);
    double *part = reinterpret_cast<double *>(static_cast<char *>(ws) + align256((size_t)nb * 4));
    return from_cuda(launch_quantize(W, dt, n, *out, c1, part, static_cast<cudaStream_t>(stream)));
}

constexpr int kMaxGroupedTensors = 4096;

size_t qlora_nf4_quantize_grouped_workspace(int count, const qlora_nf4_tensor *out) {
    if (count < 1 || count > kMaxGroupedTensors || !out) return 0;
    size_t b = 0;
    for (int i = 0; i < count; ++i) {
        if (out[i].rows < 1 || out[i].cols < 1) return 0;
        b += qlora_nf4_quantize_workspace(out[i].rows, out[i].cols);
    }
    return b;
}

qlora_status qlora_nf4_quantize_grouped(int count, const void *const *W, qlora_dtype dt, const qlora_nf4_tensor *out,
                                        void *ws, size_t ws_bytes, qlora_stream_t stream) {
    if (count < 1 || count > kMaxGroupedTensors || !W || !out || (dt != QLORA_F32 && dt != QLORA_BF16))
        return QLORA_ERR_INVALID_ARG;
    for (int i = 0; i < count; ++i) {
        if (!W[i] || !aligned16(W[i]) || !tensor_ok(&out[i])) return QLORA_ERR_INVALID_ARG;
        const int64_t n = out[i].rows * out[i].cols, nb = ceil_div(n, kBlock1), nb2 = ceil_div(nb, kBlock2);
        if (nb2 > 0x7fffffffLL) return QLORA_ERR_UNSUPPORTED_SHAPE;
    }
    const size_t need = qlora_nf4_quantize_grouped_workspace(count, out);
    if (!ws || ws_bytes < need || !aligned16(ws)) return QLORA_ERR_WORKSPACE;
    std::vector<QuantArgs> args((size_t)count);
    char *w = static_cast<char *>(ws);
    for (int i = 0; i < count; ++i) {
        const int64_t n = out[i].rows * out[i].cols, nb = ceil_div(n, kBlock1);
        args[i].W = W[i];
        args[i].n = n;
        args[i].out = out[i];
        args[i].c1 = reinterpret_cast<float *>(w);
        args[i].part = reinterpret_cast<double *>(w + align256((size_t)nb * 4));
        w += qlora_nf4_quantize_workspace(out[i].rows, out[i].cols);
    }
    return from_cuda(launch_quantize_grouped(args.data(), count, dt, static_cast<cudaStream_t>(stream)));
}

qlora_status qlora_nf4_dequant_grouped(int count, const qlora_nf4_tensor *q, void *const *W_out,
                                       qlora_stream_t stream) {
    if (count < 1 || count > kMaxGroupedTensors || !q || !W_out) return QLORA_ERR_INVALID_ARG;
    std::vector<NF4View> views((size_t)count);
    std::vector<__nv_bfloat16 *> outs((size_t)count);
    for (int i = 0; i < count; ++i) {
        if (!tensor_ok(&q[i]) || !W_out[i] || !aligned16(W_out[i])) return QLORA_ERR_INVALID_ARG;
        views[i] = view_of(&q[i]);
        outs[i] = static_cast<__nv_bfloat16 *>(W_out[i]);
    }
    return from_cuda(launch_dequant_grouped(views.data(), outs.data(), count, static_cast<cudaStream_t>(stream)));
}

qlora_status qlora_nf4_dequant(const qlora_nf4_tensor *q, void *W_out, qlora_stream_t stream) {
    if (!tensor_ok(q) || !W_out || !aligned16(W_out)) return QLORA_ERR_INVALID_ARG;
    return from_cuda(launch_dequant(view_of(q), static_cast<__nv_bfloat16 *>(W_out),
                                    static_cast<cudaStream_t>(stream)));
}

static qlora_status check_linear(int64_t M, const qlora_nf4_tensor *W, int r, float s) {
    if (!tensor_ok(W) || !std::isfinite(s)) return QLORA_ERR_INVALID_ARG;
    if (M < 1 || W->cols % 64 != 0 || W->rows % 16 != 0 || r < 0 || r > 256 || r % 8 != 0)
        return QLORA_ERR_UNSUPPORTED_SHAPE;
    if (M > (1LL << 31) || W->rows > (1LL << 31) || W->cols > (1LL << 31)) return QLORA_ERR_UNSUPPORTED_SHAPE;
    return QLORA_OK;
}

size_t qlora_linear_fwd_workspace(int64_t M, int64_t rows, int64_t cols, int r) {
    if (M < 1 || rows < 1 || cols < 1 || r < 0) return 0;
    return fwd_workspace_bytes(M, rows, cols, r);
}

qlora_status qlora_linear_fwd(const void *X, int64_t M, const qlora_nf4_tensor *W,
                              const void *A, const void *B, int r, float s,
                              void *Y, void *XA_save, void *ws, size_t ws_bytes,
                              qlora_stream_t stream) {
    qlora_status st = check_linear(M, W, r, s);
    if (st != QLORA_OK) return st;
    if (!X || !Y || !aligned16(X) || !aligned16(Y)) return QLORA_ERR_INVALID_ARG;
    if (r > 0 && (!A || !B || !aligned16(A) || !aligned16(B) || (XA_save && !aligned16(XA_save))))
        return QLORA_ERR_INVALID_ARG;
    const size_t need = fwd_workspace_bytes(M, W->rows, W->cols, r);
    if (need > 0 && (!ws || ws_bytes < need || !aligned16(ws))) return QLORA_ERR_WORKSPACE;
    return from_cuda(launch_linear_fwd(static_cast<const __nv_bfloat16 *>(X), M, view_of(W),
                                       static_cast<const __nv_bfloat16 *>(A), static_cast<const __nv_bfloat16 *>(B),
                                       r, s, static_cast<__nv_bfloat16 *>(Y), static_cast<__nv_bfloat16 *>(XA_save),
                                       ws, static_cast<cudaStream_t>(stream)));
}

// Validates one grouped item as qlora_linear_fwd validates its arguments and fills
// the internal descriptor.
static qlora_status grouped_item(int64_t M, const qlora_linear_desc &in, LinearDesc &out) {
    if (!in.W) return QLORA_ERR_INVALID_ARG;
    qlora_status st = check_linear(M, in.W, in.r, in.s);
    if (st != QLORA_OK) return st;
    if (!in.X || !in.Y || !aligned16(in.X) || !aligned16(in.Y)) return QLORA_ERR_INVALID_ARG;
    if (in.r > 0 && (!in.A || !in.B || !aligned16(in.A) || !aligned16(in.B) || (in.XA_save && !aligned16(in.XA_save))))
        return QLORA_ERR_INVALID_ARG;
    out.X = static_cast<const __nv_bfloat16 *>(in.X);
    out.W = view_of(in.W);
    out.A = static_cast<const __nv_bfloat16 *>(in.A);
    out.B = static_cast<const __nv_bfloat16 *>(in.B);
    out.r = in.r;
    out.s = in.s;
    out.Y = static_cast<__nv_bfloat16 *>(in.Y);
    out.XA_save = static_cast<__nv_bfloat16 *>(in.XA_save);
    return QLORA_OK;
}
constexpr int kMaxGrouped = 64;

size_t qlora_linear_fwd_grouped_workspace(int64_t M, int count, const qlora_linear_desc *d) {
    if (M < 1 || count < 1 || count > kMaxGrouped || !d) return 0;
    LinearDesc items[kMaxGrouped];
    for (int i = 0; i < count; ++i) {
        if (!d[i].W || d[i].W->rows < 1 || d[i].W->cols < 1 || d[i].r < 0) return 0;
        items[i].W.rows = d[i].W->rows;
        items[i].W.cols = d[i].W->cols;
        items[i].r = d[i].r;
    }
    return fwd_grouped_workspace_bytes(M, count, items);
}

qlora_status qlora_linear_fwd_grouped(int64_t M, int count, const qlora_linear_desc *d, void *ws,
                                      size_t ws_bytes, qlora_stream_t stream) {
    if (count < 1 || count > kMaxGrouped || !d) return QLORA_ERR_INVALID_ARG;
    LinearDesc items[kMaxGrouped];
    for (int i = 0; i < count; ++i) {
        qlora_status st = grouped_item(M, d[i], items[i]);
        if (st != QLORA_OK) return st;
    }
    const size_t need = fwd_grouped_workspace_bytes(M, count, items);
    if (need > 0 && (!ws || ws_bytes < need || !aligned16(ws))) return QLORA_ERR_WORKSPACE;
    return from_cuda(launch_linear_fwd_grouped(M, count, items, ws, static_cast<cudaStream_t>(stream)));
}

size_t qlora_nf4_merge_workspace(int64_t rows, int64_t cols) {
    if (rows < 1 || cols < 1) return 0;
    return align256((size_t)rows * (size_t)cols * 2) + merge_prep_bytes(rows, cols) +
           qlora_nf4_quantize_workspace(rows, cols);
}

qlora_status qlora_nf4_merge_adapter(const qlora_nf4_tensor *W, const void *A, const void *B, int r, float s,
                                     void *W_bf16, const qlora_nf4_tensor *W_out, void *ws, size_t ws_bytes,
                                     qlora_stream_t stream) {
    if (!tensor_ok(W) || !tensor_ok(W_out) || W_out->rows != W->rows || W_out->cols != W->cols)
        return QLORA_ERR_INVALID_ARG;
    if (W->cols % 64 != 0 || r < 1 || r > 256) return QLORA_ERR_UNSUPPORTED_SHAPE;
    if (!A || !B || !aligned16(A) || !aligned16(B) || (W_bf16 && !aligned16(W_bf16)) || !std::isfinite(s))
        return QLORA_ERR_INVALID_ARG;
    const size_t need = qlora_nf4_merge_workspace(W->rows, W->cols);
    if (!ws || ws_bytes < need || !aligned16(ws)) return QLORA_ERR_WORKSPACE;
    const int64_t n = W->rows * W->cols, nb = ceil_div(n, kBlock1), nb2 = ceil_div(nb, kBlock2);
    if (nb2 > 0x7fffffffLL) return QLORA_ERR_UNSUPPORTED_SHAPE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    char *w = static_cast<char *>(ws);
    __nv_bfloat16 *merged = W_bf16 ? static_cast<__nv_bfloat16 *>(W_bf16) : reinterpret_cast<__nv_bfloat16 *>(w);
    w += align256((size_t)n * 2);
    void *prep = w;
    w += merge_prep_bytes(W->rows, W->cols);
    float *c1 = reinterpret_cast<float *>(w);
    double *part = reinterpret_cast<double *>(w + align256((size_t)nb * 4));
    cudaError_t e = launch_merge_bf16(view_of(W), static_cast<const __nv_bfloat16 *>(A),
                                      static_cast<const __nv_bfloat16 *>(B), r, s, merged, prep, st);
    if (e != cudaSuccess) return from_cuda(e);
    return from_cuda(launch_quantize(merged, QLORA_BF16, n, *W_out, c1, part, st));
}

size_t qlora_linear_bwd_workspace(int64_t M, int64_t rows, int64_t cols, int r) {
    if (M < 1 || rows < 1 || cols < 1 || r < 0) return 0;
    return bwd_workspace_bytes(M, rows, cols, r);
}

qlora_status qlora_linear_bwd(const void *X, const void *dY, int64_t M, const qlora_nf4_tensor *W,
                              const void *A, const void *B, int r, float s, const void *XA,
                              void *dX, float *dA, float *dB, void *ws, size_t ws_bytes,
                              qlora_stream_t stream) {
    qlora_status st = check_linear(M, W, r, s);
    if (st != QLORA_OK) return st;
    if (!dY || !dX || !aligned16(dY) || !aligned16(dX)) return QLORA_ERR_INVALID_ARG;
    if (r > 0 && (!X || !A || !B || !dA || !dB || !aligned16(X) || !aligned16(A) || !aligned16(B) ||
                  !aligned16(dA) || !aligned16(dB) || (XA && !aligned16(XA))))
        return QLORA_ERR_INVALID_ARG;
    const size_t need = bwd_workspace_bytes(M, W->rows, W->cols, r);
    if (need > 0 && (!ws || ws_bytes < need || !aligned16(ws))) return QLORA_ERR_WORKSPACE;
    return from_cuda(launch_linear_bwd(static_cast<const __nv_bfloat16 *>(X), static_cast<const __nv_bfloat16 *>(dY), M,
                                       view_of(W), static_cast<const __nv_bfloat16 *>(A),
                                       static_cast<const __nv_bfloat16 *>(B), r, s,
                                       static_cast<const __nv_bfloat16 *>(XA), static_cast<__nv_bfloat16 *>(dX), dA, dB,
                                       ws, static_cast<cudaStream_t>(stream)));
}

qlora_status qlora_adamw_step(float *theta, const float *grad, float *m, float *v, int64_t n,
                              const qlora_adamw_hparams *h, void *theta_bf16, qlora_stream_t stream) {
    if (!theta || !grad || !m || !v || !h || !aligned16(theta) || !aligned16(grad) || !aligned16(m) || !aligned16(v) ||
        (theta_bf16 && !aligned16(theta_bf16)) || n < 1)
        return QLORA_ERR_INVALID_ARG;
    if (h->step < 1 || !std::isfinite(h->lr) || !std::isfinite(h->eps) || !std::isfinite(h->weight_decay) ||
        !(h->beta1 >= 0.0f && h->beta1 < 1.0f) || !(h->beta2 >= 0.0f && h->beta2 < 1.0f) || h->eps < 0.0f)
        return QLORA_ERR_INVALID_ARG;
    return from_cuda(launch_adamw(theta, grad, m, v, n, h->lr, h->beta1, h->beta2, h->eps, h->weight_decay, h->step,
                                  static_cast<__nv_bfloat16 *>(theta_bf16), static_cast<cudaStream_t>(stream)));
}

qlora_status qlora_adamw_prefetch(const void *ptr, size_t bytes, int to_device, qlora_stream_t stream) {
    if (!ptr || bytes == 0) return QLORA_ERR_INVALID_ARG;
    return from_cuda(launch_prefetch(ptr, bytes, to_device != 0, static_cast<cudaStream_t>(stream)));
}

static bool fmt4_ok(qlora_fmt4 f) {
    return f == QLORA_FMT4_INT4 || f == QLORA_FMT4_FP4_E2M1 || f == QLORA_FMT4_FP4_E3M0;
}

qlora_status qlora_fmt4_quantize(const void *W, qlora_dtype dt, int64_t n, qlora_fmt4 fmt, uint8_t *codes,
                                 float *absmax, qlora_stream_t stream) {
    const uintptr_t wa = reinterpret_cast<uintptr_t>(W);
    if (!W || !codes || !absmax || n < 1 || !fmt4_ok(fmt) || (dt != QLORA_F32 && dt != QLORA_BF16) ||
        (wa & (dt == QLORA_F32 ? 3u : 1u)) || (reinterpret_cast<uintptr_t>(absmax) & 3u))
        return QLORA_ERR_INVALID_ARG;
    return from_cuda(launch_fmt4_quantize(W, dt, n, fmt, codes, absmax, static_cast<cudaStream_t>(stream)));
}

qlora_status qlora_fmt4_dequant(const uint8_t *codes, const float *absmax, int64_t n, qlora_fmt4 fmt,
                                void *W_out, qlora_stream_t stream) {
    if (!codes || !absmax || !W_out || n < 1 || !fmt4_ok(fmt) || (reinterpret_cast<uintptr_t>(absmax) & 3u) ||
        !aligned16(codes) || !aligned16(W_out))
        return QLORA_ERR_INVALID_ARG;
    return from_cuda(launch_fmt4_dequant(codes, absmax, n, fmt, static_cast<__nv_bfloat16 *>(W_out),
                                         static_cast<cudaStream_t>(stream)));
}

qlora_status qlora_get_device_status(qlora_stream_t stream) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return QLORA_ERR_CUDA;
    unsigned int bits = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&bits, g_status_bits, sizeof(bits)) != cudaSuccess) return QLORA_ERR_CUDA;
    if (bits && cudaMemcpyToSymbol(g_status_bits, &zero, sizeof(zero)) != cudaSuccess) return QLORA_ERR_CUDA;
    for (int s = 1; s < 32; ++s)
        if (bits & (1u << s)) return (qlora_status)s;
    return QLORA_OK;
}

const char *qlora_status_string(qlora_status s) {
    switch (s) {
        case QLORA_OK: return "ok";
        case QLORA_ERR_INVALID_ARG: return "invalid argument (null or misaligned pointer, bad dtype or scale)";
        case QLORA_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
        case QLORA_ERR_WORKSPACE: return "workspace missing or too small";
        case QLORA_ERR_NONFINITE: return "non-finite weight in quantiser input";
        case QLORA_ERR_TIMEOUT: return "a bounded device wait ran out";
        case QLORA_ERR_CUDA: return "CUDA error";
    }
    return "unknown status";
}

void qlora_nf4_codebook(float out[16]) {
    if (!out) return;
    std::memcpy(out, host_codebook().q, sizeof(float) * 16);
}

}  // extern "C"
