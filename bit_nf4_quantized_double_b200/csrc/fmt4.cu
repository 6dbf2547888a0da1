// Blockwise 4-bit reference formats that the NF4 + double-quantisation format is compared
// with: Int4, FP4 E2M1 and FP4 E3M0 (page "QLoRA: put the large model in memory, then change
// it with a small adapter", wq-win.github.io/llm/074-qlora, section 4, evidence 1, the
// paper's Table 2). The pages name the formats without defining them. This file follows these
// readings:
//   64-weight blocks, each scaled by its absmax c (fp32, not double-quantised), with |w| = c
//     mapped to the format's largest magnitude S;
//   Int4: magnitudes 0..7 (S = 7);
//   E2M1: sign, 2 exponent bits (bias 1), 1 mantissa bit, with subnormals: magnitudes
//     0, 0.5, 1, 1.5, 2, 3, 4, 6 (S = 6);
//   E3M0: sign, 3 exponent bits, exponent field 0 = zero: magnitudes 0 and 2^(e-7) for
//     e = 1..7 (S = 1);
//   x' = fl(fl(w / c) * S); the magnitude index is the count of midpoints below |x'|, with a
//     tie exactly on a midpoint going to the even index; bit 3 holds the sign (none for zero);
//   w^ = bf16(fl(v * fl(c / S))).
// Codes are packed two per byte as in the NF4 format: byte k = code[2k] << 4 | code[2k + 1].
//
// k_fmt4_quantize: one warp per 64-block, each lane two consecutive weights (one output byte),
// absmax by a butterfly of shuffles. k_fmt4_dequant: one thread per 16 weights. Both stream
// HBM.
#include "launch.h"

namespace qnf4 {

struct Fmt4Table {
    float mag[8];   // magnitudes, ascending
    float mid[7];   // midpoints of consecutive magnitudes (exact in fp32)
    float S;        // largest magnitude
};

static Fmt4Table fmt4_table(qlora_fmt4 f) {
    Fmt4Table t;
    switch (f) {
        case QLORA_FMT4_INT4:
            for (int i = 0; i < 8; ++i) t.mag[i] = (float)i;
            break;
        case QLORA_FMT4_FP4_E2M1: {
            const float m[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};
            for (int i = 0; i < 8; ++i) t.mag[i] = m[i];
            break;
        }
        default:   // QLORA_FMT4_FP4_E3M0
            t.mag[0] = 0.0f;
            for (int e = 1; e <= 7; ++e) t.mag[e] = std::ldexp(1.0f, e - 7);
            break;
    }
    for (int i = 0; i < 7; ++i) t.mid[i] = (t.mag[i] + t.mag[i + 1]) * 0.5f;   // exact for all three
    t.S = t.mag[7];
    return t;
}

__device__ __forceinline__ float load_f32(const float *p) { return __ldg(p); }
__device__ __forceinline__ float load_f32(const __nv_bfloat16 *p) { return __bfloat162float(p[0]); }

__device__ __forceinline__ uint32_t fmt4_code(float w, float c, const Fmt4Table &t) {
    const float x = c > 0.0f ? __fmul_rn(__fdiv_rn(w, c), t.S) : 0.0f;
    const float m = fabsf(x);
    uint32_t idx = 0;
#pragma unroll
    for (int i = 0; i < 7; ++i) idx += (t.mid[i] < m) ? 1u : 0u;
    if (idx < 7 && (idx & 1u) && m == t.mid[idx]) ++idx;       // a tie goes to the even index
    return idx | ((x < 0.0f && idx > 0) ? 8u : 0u);
}

template <typename T>
__global__ void __launch_bounds__(256) k_fmt4_quantize(const T *__restrict__ w, int64_t n, const __grid_constant__ Fmt4Table t,
                                                      uint8_t *__restrict__ codes, float *__restrict__ absmax) {
    const int64_t blk = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t nb = (n + 63) / 64;
    if (blk >= nb) return;                                       // whole warps leave together
    const int64_t i0 = blk * 64 + 2 * lane;
    const float a = i0 < n ? load_f32(w + i0) : 0.0f;
    const float b = i0 + 1 < n ? load_f32(w + i0 + 1) : 0.0f;
    float c = fmaxf(fabsf(a), fabsf(b));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) c = fmaxf(c, __shfl_xor_sync(0xffffffffu, c, o));
    if (i0 < n) codes[i0 >> 1] = (uint8_t)((fmt4_code(a, c, t) << 4) | fmt4_code(b, c, t));
    if (lane == 0) absmax[blk] = c;
}

// Dequantisation: one thread per 16 weights (an 8-byte code word, all of it in one
// 64-block: one division for the step), signed values from a 16-entry table in shared
// memory (16 words in 16 banks: lookups never conflict), two 16-byte bf16 stores. The
// last n % 16 weights are written element by element by thread 0 of CTA 0.
__global__ void __launch_bounds__(256) k_fmt4_dequant(const uint8_t *__restrict__ codes,
                                                     const float *__restrict__ absmax, int64_t n,
                                                     const __grid_constant__ Fmt4Table t,
                                                     __nv_bfloat16 *__restrict__ out) {
    __shared__ float s_v[16];   // code c -> sign (bit 3) times magnitude mag[c & 7]
    if (threadIdx.x < 16) s_v[threadIdx.x] = (threadIdx.x & 8u) ? -t.mag[threadIdx.x & 7u] : t.mag[threadIdx.x & 7u];
    __syncthreads();
    const int64_t words = n / 16;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t w = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; w < words; w += stride) {
        const uint2 cw = __ldg(reinterpret_cast<const uint2 *>(codes) + w);
        const float step = __fdiv_rn(__ldg(absmax + w / 4), t.S);
        uint32_t o[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const uint32_t byte = ((k < 4 ? cw.x : cw.y) >> (8 * (k & 3))) & 0xffu;
            o[k] = pack_bf16x2(__fmul_rn(s_v[byte >> 4], step), __fmul_rn(s_v[byte & 15u], step));
        }
        uint4 *dst = reinterpret_cast<uint4 *>(out + 16 * w);
        dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
        dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        for (int64_t e = words * 16; e < n; ++e) {
            const uint32_t byte = codes[e / 2];
            const uint32_t c = (e % 2 == 0) ? (byte >> 4) : (byte & 15u);
            out[e] = __float2bfloat16_rn(__fmul_rn(s_v[c], __fdiv_rn(absmax[e / 64], t.S)));
        }
    }
}

cudaError_t launch_fmt4_quantize(const void *W, qlora_dtype dt, int64_t n, qlora_fmt4 f, uint8_t *codes,
                                 float *absmax, cudaStream_t st) {
    const int64_t nb = (n + 63) / 64;
    const unsigned grid = (unsigned)ceil_div(nb * 32, 256);
    const Fmt4Table t = fmt4_table(f);
    if (dt == QLORA_F32)
        QNF4_LAUNCH("k_fmt4_quantize", st,
                    k_fmt4_quantize<float><<<grid, 256, 0, st>>>(static_cast<const float *>(W), n, t, codes, absmax));
    else
        QNF4_LAUNCH("k_fmt4_quantize", st,
                    k_fmt4_quantize<__nv_bfloat16><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16 *>(W), n, t,
                                                                        codes, absmax));
    return cudaGetLastError();
}

cudaError_t launch_fmt4_dequant(const uint8_t *codes, const float *absmax, int64_t n, qlora_fmt4 f,
                                __nv_bfloat16 *out, cudaStream_t st) {
    int64_t grid = ceil_div(n / 16, (int64_t)256);
    const int64_t cap = (int64_t)num_sms() * 8;
    if (grid > cap) grid = cap;
    if (grid < 1) grid = 1;
    QNF4_LAUNCH("k_fmt4_dequant", st,
                k_fmt4_dequant<<<(unsigned)grid, 256, 0, st>>>(codes, absmax, n, fmt4_table(f), out));
    return cudaGetLastError();
}

}  // namespace qnf4
