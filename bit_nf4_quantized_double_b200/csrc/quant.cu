// NF4 quantisation, double quantisation and dequantisation kernels (sm_100a).
//
// Method: "QLoRA: put the large model in memory, then change it with a small
// adapter" (wq-win.github.io/llm/074-qlora), section 2 (64-weight absmax
// blocks, 16-value normal-quantile codebook, 8-bit constants with an offset and
// one fp32 constant per 256 constants) and section 3 (quantise W, then the
// constants; dequantise to BF16 on demand).
//
// Launch sequence of a quantisation (all HBM-bound):
//   k_quantize_codes  one CTA per second-level group (256 blocks = 16384 weights):
//                     absmax per 64-block by warp shuffles, IEEE division, 4-step
//                     threshold search, nibble packing; writes the exact fp32
//                     absmax and the group's fp64 pairwise partial sum;
//   k_offset          one CTA: the upper levels of the fp64 pairwise tree -> mean;
//   k_double_quant    one warp per group: s2 = max |c1 - mu|, int8 constants.

#include <cmath>

#include "common.cuh"

namespace qnf4 {

__device__ unsigned int g_status_bits = 0;

// Number of thresholds strictly below x (t ascending, 15 entries in shared
// memory): a 4-step binary search that returns the same count as comparing
// against all 15. A value equal to a threshold stays on the lower code.
__device__ __forceinline__ int nf4_code(float x, const float *t) {
    int c = (x > t[7]) ? 8 : 0;
    c += (x > t[c + 3]) ? 4 : 0;
    c += (x > t[c + 1]) ? 2 : 0;
    c += (x > t[c]) ? 1 : 0;
    return c;
}

// Code table over 256 equal bins of [-1, 1): bin k = [-1 + k/128, -1 + (k+1)/128)
// holds base[k] = number of thresholds below the bin and thr[k] = the one
// threshold inside the bin (4.0 if none). Valid when no threshold lies within
// kBinMargin of a bin edge (checked on the host).
struct CodeBins {
    int base[256];
    float thr[256];
};
constexpr double kBinMargin = 1e-5;

static bool build_code_bins(const Codebook &cb, CodeBins &b) {
    for (int k = 0; k < 256; ++k) {
        const double lo = -1.0 + k / 128.0, hi = lo + 1.0 / 128.0;
        int base = 0;
        float thr = 4.0f;
        int inside = 0;
        for (int t = 0; t < 15; ++t) {
            const double T = cb.t[t];
            if (std::fabs(T - lo) < kBinMargin || std::fabs(T - hi) < kBinMargin) return false;
            if (T < lo) ++base;
            else if (T < hi) { thr = cb.t[t]; ++inside; }
        }
        if (inside > 1) return false;
        b.base[k] = base;
        b.thr[k] = thr;
    }
    return true;
}

template <typename T> __device__ __forceinline__ float to_f32(T v);
template <> __device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T, int VEC>
__device__ __forceinline__ void load_vec(const T *p, float (&v)[VEC]) {
    const uint4 raw = *reinterpret_cast<const uint4 *>(p);
    if constexpr (sizeof(T) == 4) {
        v[0] = __uint_as_float(raw.x); v[1] = __uint_as_float(raw.y);
        v[2] = __uint_as_float(raw.z); v[3] = __uint_as_float(raw.w);
    } else {
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) { v[2 * k] = bf16_lo(w[k]); v[2 * k + 1] = bf16_hi(w[k]); }
    }
}

// One CTA of 256 threads per second-level group j (blocks 256j .. 256j+255).
// Warp w handles blocks 256j + 32w .. +31; a 64-block is spread over
// LPB = 64 / VEC lanes that each load 16 bytes.
//
// With BINS, a lane divides by one correctly rounded reciprocal of its block's
// absmax (x' = fl(w * fl(1/c1)), within 1.5 ulp of the exact quotient x =
// fl(w / c1)) and reads the code from the bin table through the float bits of
// x' + 3 (in [2, 4): the top 8 mantissa bits are the bin). Where x' lies within
// 4 ulp of the bin's threshold the exact quotient and the full search decide, so
// the codes are those of x bit for bit. Without BINS every weight is divided.
template <typename T, bool BINS>
__global__ void __launch_bounds__(256, 4)
k_quantize_codes(const T *__restrict__ W, int64_t n, int64_t nb, Codebook cb,
                 const __grid_constant__ CodeBins bins,
                 float *__restrict__ c1_out, double *__restrict__ part_out,
                 uint8_t *__restrict__ codes) {
    constexpr int VEC = 16 / sizeof(T);   // elements per 16-byte lane load
    constexpr int LPB = kBlock1 / VEC;    // lanes per block
    constexpr int BPI = 32 / LPB;         // blocks per warp iteration
    constexpr int ITERS = 32 / BPI;       // iterations per warp (32 blocks)
    constexpr int NBYTES = VEC / 2;       // code bytes per lane per iteration

    __shared__ float s_t[16];
    __shared__ float s_c1[kBlock2];
    __shared__ double s_part[8];
    __shared__ int2 s_bin[256];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x < 15) s_t[threadIdx.x] = cb.t[threadIdx.x];
    if (BINS) s_bin[threadIdx.x] = make_int2(bins.base[threadIdx.x], __float_as_int(bins.thr[threadIdx.x]));
    __syncthreads();

    const int64_t group = blockIdx.x;
    const int sub = lane / LPB, li = lane % LPB;
    const int64_t ncode = (n + 1) / 2;
    bool nonfinite = false;

    // the lane's 16-byte loads are issued in batches of 8 before any arithmetic
    // (one memory round trip per batch instead of one per iteration)
    constexpr int BATCH = ITERS < 8 ? ITERS : 8;
#pragma unroll 1
    for (int it0 = 0; it0 < ITERS; it0 += BATCH) {
    uint4 raw[BATCH];
#pragma unroll
    for (int j = 0; j < BATCH; ++j) {
        const int it = it0 + j;
        const int64_t e0 = ((group * kBlock2 + warp * 32 + it * BPI + sub) * kBlock1) + (int64_t)li * VEC;
        raw[j] = (e0 + VEC <= n) ? __ldg(reinterpret_cast<const uint4 *>(W + e0)) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int j = 0; j < BATCH; ++j) {
        const int it = it0 + j;
        const int local = warp * 32 + it * BPI + sub;          // block index within the group
        const int64_t b = group * kBlock2 + local;
        const int64_t e0 = b * kBlock1 + (int64_t)li * VEC;     // first element of this lane
        float v[VEC];
        if (e0 + VEC <= n) {
            if constexpr (sizeof(T) == 4) {
                v[0] = __uint_as_float(raw[j].x); v[1] = __uint_as_float(raw[j].y);
                v[2] = __uint_as_float(raw[j].z); v[3] = __uint_as_float(raw[j].w);
            } else {
                const uint32_t w4[4] = {raw[j].x, raw[j].y, raw[j].z, raw[j].w};
#pragma unroll
                for (int k = 0; k < 4; ++k) { v[2 * k] = bf16_lo(w4[k]); v[2 * k + 1] = bf16_hi(w4[k]); }
            }
        } else {
#pragma unroll
            for (int k = 0; k < VEC; ++k) v[k] = (e0 + k < n) ? to_f32<T>(W[e0 + k]) : 0.0f;
        }
        float m = 0.0f;
#pragma unroll
        for (int k = 0; k < VEC; ++k) {
            nonfinite |= !isfinite(v[k]);
            m = fmaxf(m, fabsf(v[k]));
        }
#pragma unroll
        for (int o = LPB / 2; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (li == 0) {
            s_c1[local] = m;
            if (b < nb) c1_out[b] = m;
        }
        // codes of the lane's VEC elements: NBYTES bytes, byte k = hi << 4 | lo
        uint32_t packed = 0;
        if (BINS) {
            const float rcp = __frcp_rn(m);
#pragma unroll
            for (int k = 0; k < VEC; ++k) {
                const float xa = __fmul_rn(v[k], rcp);
                const float y = fminf(fmaxf(__fadd_rn(xa, 3.0f), 2.0f), 3.99999976f);
                const int2 e = s_bin[(__float_as_uint(y) >> 15) & 0xffu];
                const float thr = __int_as_float(e.y);
                int c = e.x + (xa > thr ? 1 : 0);
                if (fabsf(__fsub_rn(xa, thr)) <= __fmul_rn(fabsf(thr), 0x1p-21f)) c = nf4_code(__fdiv_rn(v[k], m), s_t);
                if (m == 0.0f) c = 7;
                packed |= (uint32_t)c << (8 * (k / 2) + ((k & 1) ? 0 : 4));
            }
        } else {
#pragma unroll
            for (int k = 0; k < VEC; k += 2) {
                const float x0 = (m == 0.0f) ? 0.0f : __fdiv_rn(v[k], m);
                const float x1 = (m == 0.0f) ? 0.0f : __fdiv_rn(v[k + 1], m);
                const uint32_t byte = ((uint32_t)nf4_code(x0, s_t) << 4) | (uint32_t)nf4_code(x1, s_t);
                packed |= byte << (8 * (k / 2));
            }
        }
        const int64_t c0 = e0 / 2;
        if (c0 + NBYTES <= ncode) {
            if constexpr (NBYTES == 4) *reinterpret_cast<uint32_t *>(codes + c0) = packed;
            else *reinterpret_cast<uint16_t *>(codes + c0) = (uint16_t)packed;
        } else {
#pragma unroll
            for (int k = 0; k < NBYTES; ++k)
                if (c0 + k < ncode) codes[c0 + k] = (uint8_t)(packed >> (8 * k));
        }
    }
    }
    if (__any_sync(0xffffffffu, nonfinite) && lane == 0) raise_status(QLORA_ERR_NONFINITE);
    __syncthreads();

    // fp64 pairwise tree over the group's 256 leaves (blocks past nb are 0):
    // node i of level l+1 = node 2i + node 2i+1 of level l.
    double v = (double)s_c1[threadIdx.x];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const double u = __shfl_down_sync(0xffffffffu, v, o);
        if ((lane & (2 * o - 1)) == 0) v = v + u;
    }
    if (lane == 0) s_part[warp] = v;
    __syncthreads();
    if (warp == 0) {
        v = (lane < 8) ? s_part[lane] : 0.0;
#pragma unroll
        for (int o = 1; o < 8; o <<= 1) {
            const double u = __shfl_down_sync(0xffffffffu, v, o);
            if ((lane & (2 * o - 1)) == 0) v = v + u;
        }
        if (lane == 0) part_out[group] = v;
    }
}

// Upper levels of the pairwise tree over the nb2 group partials, zero-padded
// to a power of two (>= 1024): thread t first reduces leaves [tC, tC+C) with
// a binary-counter stack (which forms exactly the subtree of those leaves),
// then the 1024 subtree sums are combined level by level. mu = fl(S / nb).
__global__ void __launch_bounds__(1024)
k_offset(const double *__restrict__ part, int64_t nb2, int64_t nb, float *__restrict__ offset_out) {
    __shared__ double s_w[32];
    int64_t L = 1024;
    while (L < nb2) L <<= 1;
    const int64_t C = L / 1024;
    const int64_t i0 = (int64_t)threadIdx.x * C;
    double v = 0.0;
    if (i0 < nb2) {
        double stack[48];
        int level[48];
        int sp = 0;
        for (int64_t i = 0; i < C; ++i) {
            double x = (i0 + i < nb2) ? part[i0 + i] : 0.0;
            int l = 0;
            while (sp > 0 && level[sp - 1] == l) { x = stack[--sp] + x; ++l; }
            stack[sp] = x;
            level[sp] = l;
            ++sp;
        }
        v = stack[0];
    }
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const double u = __shfl_down_sync(0xffffffffu, v, o);
        if ((lane & (2 * o - 1)) == 0) v = v + u;
    }
    if (lane == 0) s_w[warp] = v;
    __syncthreads();
    if (warp == 0) {
        v = s_w[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const double u = __shfl_down_sync(0xffffffffu, v, o);
            if ((lane & (2 * o - 1)) == 0) v = v + u;
        }
        if (lane == 0) *offset_out = __double2float_rn(__ddiv_rn(v, (double)nb));
    }
}

// One warp per second-level group: d_b = fl(c1_b - mu), s2 = max |d_b|,
// q8_b = rint(fl(fl(d_b / s2) * 127)) (0 when s2 == 0).
__global__ void __launch_bounds__(256)
k_double_quant(const float *__restrict__ c1, int64_t nb, int64_t nb2, const float *__restrict__ offset,
               int8_t *__restrict__ q8, float *__restrict__ s2) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t j = (int64_t)blockIdx.x * 8 + warp;
    if (j >= nb2) return;
    const float mu = *offset;
    float d[8];
    float m = 0.0f;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const int64_t b = j * kBlock2 + k * 32 + lane;
        d[k] = (b < nb) ? __fsub_rn(c1[b], mu) : 0.0f;
        m = fmaxf(m, fabsf(d[k]));
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) s2[j] = m;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const int64_t b = j * kBlock2 + k * 32 + lane;
        if (b < nb) {
            int q = 0;
            if (m != 0.0f) q = __float2int_rn(__fmul_rn(__fdiv_rn(d[k], m), 127.0f));
            q8[b] = (int8_t)q;
        }
    }
}

// Dequantisation: each thread expands two 32-bit words of codes (16 weights, a
// quarter block) into two 16-byte bf16 stores; a warp reads 256 contiguous code
// bytes and writes 1 KB, and four such pairs per thread are in flight at once.
// Codebook in shared memory (16 distinct words: lookups never conflict). A
// ragged tail (n % 16 != 0) is written element by element.
constexpr int kDequantUnroll = 4;
__global__ void __launch_bounds__(256, 4)
k_dequant(NF4View q, int64_t n, Codebook cb, __nv_bfloat16 *__restrict__ out) {
    __shared__ float s_q[16];
    if (threadIdx.x < 16) s_q[threadIdx.x] = cb.q[threadIdx.x];
    __syncthreads();
    const float mu = *q.offset;
    const int64_t n16 = n / 16;
    const int64_t nthr = (int64_t)gridDim.x * blockDim.x;
    const uint2 *codes = reinterpret_cast<const uint2 *>(q.codes);
    for (int64_t g0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g0 < n16; g0 += kDequantUnroll * nthr) {
        uint2 w[kDequantUnroll];
        int8_t q8[kDequantUnroll];
        float s2[kDequantUnroll];
#pragma unroll
        for (int u = 0; u < kDequantUnroll; ++u) {
            const int64_t g = g0 + u * nthr;
            if (g < n16) {
                const int64_t b = g / (kBlock1 / 16);
                w[u] = __ldg(codes + g);
                q8[u] = __ldg(q.scale8 + b);
                s2[u] = __ldg(q.scale2 + b / kBlock2);
            }
        }
#pragma unroll
        for (int u = 0; u < kDequantUnroll; ++u) {
            const int64_t g = g0 + u * nthr;
            if (g < n16) {
                const float ch = dq_constant(q8[u], s2[u], mu);
                uint32_t o[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t byte = ((k < 4 ? w[u].x : w[u].y) >> (8 * (k & 3))) & 0xffu;
                    o[k] = pack_bf16x2(__fmul_rn(s_q[byte >> 4], ch), __fmul_rn(s_q[byte & 15u], ch));
                }
                uint4 *dst = reinterpret_cast<uint4 *>(out + 16 * g);
                dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
                dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
            }
        }
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        for (int64_t e = 16 * n16; e < n; ++e) {
            const int64_t b = e / kBlock1;
            const float ch = dq_constant(q.scale8[b], q.scale2[b / kBlock2], mu);
            const uint8_t byte = q.codes[e / 2];
            const uint32_t code = (e % 2 == 0) ? (byte >> 4) : (byte & 15u);
            out[e] = __float2bfloat16_rn(__fmul_rn(s_q[code], ch));
        }
    }
}

// ---------------------------------------------------------------- adapter merge
// Merged BF16 weight (the page's sections 5 and 6: merging the adapter into the
// weight and re-quantising can change outputs; the merge is done in BF16):
//   w'[n,k] = bf16( fl( w^[n,k] + fl(s * d[n,k]) ) ),
//   d[n,k]  = fused multiply-adds of A[k,j] * B[j,n] over j = 0 .. r-1 in order, from 0,
// with w^ the dequantised weight computed in place (step 7 of the format). A CTA
// takes 64 x 64 tiles (rows x inputs: one 64-block per row); the tile's A rows and
// B columns are staged in shared memory as fp32, transposed so that a thread reads
// its 16 consecutive inputs of one j with four 16-byte loads.
__global__ void __launch_bounds__(256)
k_merge_bf16(NF4View q, const __nv_bfloat16 *__restrict__ A, const __nv_bfloat16 *__restrict__ B, int r, float s,
             Codebook cb, __nv_bfloat16 *__restrict__ out) {
    extern __shared__ __align__(16) float msm[];
    float *As = msm;                 // [r][64]: As[j][kk] = A[k0 + kk][j]
    float *Bs = msm + r * 64;        // [r][64]: Bs[j][nn] = B[j][n0 + nn]
    __shared__ float s_q[16];
    if (threadIdx.x < 16) s_q[threadIdx.x] = cb.q[threadIdx.x];
    const int64_t rows = q.rows, cols = q.cols, kbs = cols / 64;
    const float mu = *q.offset;
    const int nn = threadIdx.x >> 2, kk0 = (threadIdx.x & 3) * 16;
    const int64_t tiles_n = (rows + 63) / 64, tiles = tiles_n * kbs;
    for (int64_t tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
        const int64_t n0 = (tile % tiles_n) * 64, k0 = (tile / tiles_n) * 64;
        __syncthreads();   // previous tile's readers are done
        for (int i = threadIdx.x; i < r * 64; i += blockDim.x) {
            const int j = i / 64, c = i % 64;
            As[j * 64 + c] = __bfloat162float(A[(k0 + c) * r + j]);
            Bs[j * 64 + c] = (n0 + c < rows) ? __bfloat162float(B[(int64_t)j * rows + n0 + c]) : 0.0f;
        }
        __syncthreads();
        const int64_t n = n0 + nn;
        if (n >= rows) continue;
        float d[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) d[e] = 0.0f;
        for (int j = 0; j < r; ++j) {
            const float b = Bs[j * 64 + nn];
            const float4 *a4 = reinterpret_cast<const float4 *>(As + j * 64 + kk0);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                const float4 a = a4[v];
                d[4 * v + 0] = fmaf(a.x, b, d[4 * v + 0]);
                d[4 * v + 1] = fmaf(a.y, b, d[4 * v + 1]);
                d[4 * v + 2] = fmaf(a.z, b, d[4 * v + 2]);
                d[4 * v + 3] = fmaf(a.w, b, d[4 * v + 3]);
            }
        }
        // dequantise the 16 weights (one 64-block: block n * kbs + k0 / 64) and add
        const int64_t e0 = n * cols + k0 + kk0;
        const int64_t blk = n * kbs + k0 / 64;
        const float ch = dq_constant(q.scale8[blk], q.scale2[blk / kBlock2], mu);
        const uint2 cw = *reinterpret_cast<const uint2 *>(q.codes + e0 / 2);
        uint32_t o[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const uint32_t byte = ((k < 4 ? cw.x : cw.y) >> (8 * (k & 3))) & 0xffu;
            const float w_hi = __bfloat162float(__float2bfloat16_rn(__fmul_rn(s_q[byte >> 4], ch)));
            const float w_lo = __bfloat162float(__float2bfloat16_rn(__fmul_rn(s_q[byte & 15u], ch)));
            o[k] = pack_bf16x2(__fadd_rn(w_hi, __fmul_rn(s, d[2 * k])), __fadd_rn(w_lo, __fmul_rn(s, d[2 * k + 1])));
        }
        uint4 *dst = reinterpret_cast<uint4 *>(out + e0);
        dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
        dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
    }
}

cudaError_t launch_merge_bf16(const NF4View &q, const __nv_bfloat16 *A, const __nv_bfloat16 *B, int r, float s,
                              __nv_bfloat16 *out, cudaStream_t st) {
    const int64_t tiles = ceil_div(q.rows, (int64_t)64) * (q.cols / 64);
    int64_t grid = tiles;
    const int64_t cap = (int64_t)num_sms() * 4;
    if (grid > cap) grid = cap;
    const size_t sm = (size_t)r * 64 * 4 * 2;
    cudaError_t e = cudaFuncSetAttribute(k_merge_bf16, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    QNF4_LAUNCH("k_merge_bf16", st, k_merge_bf16<<<(unsigned)grid, 256, sm, st>>>(q, A, B, r, s, host_codebook(), out));
    return cudaGetLastError();
}

// ---------------------------------------------------------------- launchers
cudaError_t launch_quantize(const void *W, qlora_dtype dt, int64_t n, const qlora_nf4_tensor &out,
                            float *c1, double *part, cudaStream_t st) {
    const int64_t nb = ceil_div(n, kBlock1), nb2 = ceil_div(nb, kBlock2);
    const Codebook &cb = host_codebook();
    static CodeBins bins;
    static const bool use_bins = build_code_bins(cb, bins);
    if (dt == QLORA_F32) {
        if (use_bins)
            QNF4_LAUNCH("k_quantize_codes", st, k_quantize_codes<float, true><<<(unsigned)nb2, 256, 0, st>>>(static_cast<const float *>(W), n, nb, cb, bins, c1, part, out.codes));
        else
            QNF4_LAUNCH("k_quantize_codes", st, k_quantize_codes<float, false><<<(unsigned)nb2, 256, 0, st>>>(static_cast<const float *>(W), n, nb, cb, bins, c1, part, out.codes));
    } else {
        if (use_bins)
            QNF4_LAUNCH("k_quantize_codes", st, k_quantize_codes<__nv_bfloat16, true><<<(unsigned)nb2, 256, 0, st>>>(static_cast<const __nv_bfloat16 *>(W), n, nb, cb, bins, c1, part, out.codes));
        else
            QNF4_LAUNCH("k_quantize_codes", st, k_quantize_codes<__nv_bfloat16, false><<<(unsigned)nb2, 256, 0, st>>>(static_cast<const __nv_bfloat16 *>(W), n, nb, cb, bins, c1, part, out.codes));
    }
    QNF4_LAUNCH("k_offset", st, k_offset<<<1, 1024, 0, st>>>(part, nb2, nb, out.offset));
    QNF4_LAUNCH("k_double_quant", st, k_double_quant<<<(unsigned)ceil_div(nb2, 8), 256, 0, st>>>(c1, nb, nb2, out.offset, out.scale8, out.scale2));
    return cudaGetLastError();
}

cudaError_t launch_dequant(const NF4View &q, __nv_bfloat16 *out, cudaStream_t st) {
    const int64_t n = q.rows * q.cols;
    int64_t grid = ceil_div(ceil_div(n, 16 * kDequantUnroll), 256);
    const int64_t cap = (int64_t)num_sms() * 8;
    if (grid < 1) grid = 1;
    if (grid > cap) grid = cap;
    QNF4_LAUNCH("k_dequant", st, k_dequant<<<(unsigned)grid, 256, 0, st>>>(q, n, host_codebook(), out));
    return cudaGetLastError();
}

}  // namespace qnf4
