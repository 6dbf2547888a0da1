// NF4 quantisation, double quantisation and dequantisation kernels (sm_100a).
//
// Method: "QLoRA: put the large model in memory, then change it with a small
// adapter" (wq-win.github.io/llm/074-qlora), section 2 (64-weight absmax
// blocks, 16-value normal-quantile codebook, 8-bit constants with an offset and
// one fp32 constant per 256 constants) and section 3 (quantise W, then the
// constants; dequantise to BF16 on demand).
//
// Launch sequence of a quantisation (all HBM-bound):
//   k_quantize_codes  persistent CTAs over the second-level groups (256 blocks =
//                     16384 weights): absmax per 64-block by warp shuffles, codes
//                     from a bin table with an exact-quotient fallback, nibble
//                     packing; writes the exact fp32 absmax and the group's fp64
//                     pairwise partial sum;
//   k_offset          one CTA per tensor: the upper levels of the fp64 pairwise
//                     tree -> mean;
//   k_double_quant    one warp per group: s2 = max |c1 - mu|, int8 constants.

#include <atomic>
#include <cmath>
#include <cstring>
#include <type_traits>

#include "launch.h"

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

// Code table of the quantiser's fast path. A weight is mapped to u in [0, 1], an
// approximation of x / 2 + 1/2 with x its exact normalised value (see k_quantize_codes;
// NaN to 0), and to its bin k = z - 2^23 with z = fl(u 255 + 2^23), an integer in
// [0, 255]. The rounding is monotone, so each bin holds an interval of u. Entry k holds
// the one threshold inside bin k in the same domain, U = fl(T / 2 + 1/2) (4.0 if none),
// and base = the number of thresholds below bin k, both as floats; the code is
// base + (u > U). Valid when no bin holds two thresholds and every threshold's
// neighbourhood T +- 2^-16 lies inside its own bin (checked on the host), so that a
// threshold can sit between u and the exact value only if it is the threshold of u's bin.
struct CodeTable {
    float thr[256];
    float base[256];
};

static int host_bin(float x) {
    float u = std::fmaf(x, 0.5f, 0.5f);
    u = u < 0.0f ? 0.0f : (u > 1.0f ? 1.0f : u);
    return (int)(std::fmaf(u, 255.0f, 8388608.0f) - 8388608.0f);
}

static bool build_code_table(const Codebook &cb, CodeTable &tb) {
    int owner[256];
    for (int k = 0; k < 256; ++k) owner[k] = -1;
    for (int t = 0; t < 15; ++t) {
        const float T = cb.t[t];
        const int k = host_bin(T);
        if (host_bin(T - 0x1p-16f) != k || host_bin(T + 0x1p-16f) != k) return false;
        if (owner[k] != -1) return false;
        if (!(std::fabs(T) >= 0x1p-5f && std::fabs(T) < 1.0f)) return false;   // the band below assumes it
        owner[k] = t;
    }
    for (int k = 0; k < 256; ++k) {
        int base = 0;
        for (int t = 0; t < 15; ++t) base += host_bin(cb.t[t]) < k ? 1 : 0;
        if (owner[k] >= 0 && owner[k] != base) return false;
        tb.thr[k] = owner[k] >= 0 ? std::fmaf(cb.t[owner[k]], 0.5f, 0.5f) : 4.0f;
        tb.base[k] = (float)base;
    }
    return true;
}

__device__ __forceinline__ float fma_sat(float a, float b, float c) {
    float d;
    asm("fma.rn.sat.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

__device__ __forceinline__ float mul_sat(float a, float b) {
    float d;
    asm("mul.rn.sat.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
    return d;
}

__device__ __forceinline__ void lds_f2(uint32_t addr, float &x, float &y) {
    asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(x), "=f"(y) : "r"(addr));
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

template <typename T> __device__ __forceinline__ float to_f32(T v);
template <> __device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

__device__ __forceinline__ uint32_t vmax_u16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// 16 input bytes of a lane from element e0 on, zero past n (the partial lane of a
// tensor's tail).
template <typename T>
__device__ __forceinline__ uint4 load_partial(const T *W, int64_t e0, int64_t n) {
    uint32_t w[4] = {0u, 0u, 0u, 0u};
    constexpr int VEC = 16 / sizeof(T);
#pragma unroll
    for (int k = 0; k < VEC; ++k) {
        if (e0 + k < n) {
            if constexpr (sizeof(T) == 4) w[k] = __float_as_uint(reinterpret_cast<const float *>(W)[e0 + k]);
            else w[k / 2] |= (uint32_t)__bfloat16_as_ushort(W[e0 + k]) << (16 * (k & 1));
        }
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// Store a lane's NBYTES code bytes at code byte c0 (bytes past ncode are dropped).
template <int NBYTES>
__device__ __forceinline__ void store_codes(uint8_t *codes, int64_t c0, int64_t ncode, uint32_t packed) {
    if (c0 + NBYTES <= ncode) {
        if constexpr (NBYTES == 4) *reinterpret_cast<uint32_t *>(codes + c0) = packed;
        else *reinterpret_cast<uint16_t *>(codes + c0) = (uint16_t)packed;
    } else {
#pragma unroll
        for (int k = 0; k < NBYTES; ++k)
            if (c0 + k < ncode) codes[c0 + k] = (uint8_t)(packed >> (8 * k));
    }
}

// A list of tensors quantised by one sequence of launches: group ranges per tensor
// (second-level groups in k_quantize_codes, blocks of eight groups in
// k_double_quant), one CTA per tensor in k_offset.
constexpr int kQuantMaxItems = 64;
struct QuantItem {
    const void *W;
    int64_t n, nb, nb2;
    float *c1;                   // [nb] exact absmax (workspace)
    double *part;                // [8 nb2] partial sums of the groups' 32-block eighths (workspace)
    uint8_t *codes;
    int8_t *scale8;
    float *scale2;
    float *offset;
    int64_t cta0;                // first group of this tensor in k_quantize_codes' numbering
    int64_t dq0;                 // first CTA of this tensor in k_double_quant
};
struct QuantGroup {
    QuantItem it[kQuantMaxItems];
    int count;
    int64_t groups;              // total second-level groups of the list
};
// The tensor whose range holds unit b (ranges ascending from 0).
__device__ __forceinline__ int quant_item(const QuantGroup &g, int64_t b, bool dq) {
    int lo = 0, hi = g.count - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if ((dq ? g.it[mid].dq0 : g.it[mid].cta0) <= b) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// Codes, exact absmax and group partial sums. A persistent grid of 256-thread CTAs
// walks the second-level groups (256 blocks = 16384 weights); warp w handles blocks
// 32w .. 32w+31 of a group, a 64-block spread over LPB = 64 / VEC lanes that each
// load 16 bytes, eight loads in flight per lane before any arithmetic.
//
// Absmax c1 = max |w| is taken on the weights' bit patterns with the sign cleared
// (integer order equals float order there; inf and NaN compare above every finite
// value, which also flags a non-finite block).
//
// With BINS (default), a lane takes an approximate reciprocal r of c1 (within 1 ulp)
// and forms u = sat(fl(w (r/2) + 1/2)) with one fused multiply-add (r/2 is exact). Then
// |u - (w/c1)/2 - 1/2| <= 2^-25 + 2^-24, and the table's U = fl(T/2 + 1/2) is within
// 2^-25 of T/2 + 1/2, so wherever |u - U| > 2^-22 the exact value w/c1 lies on the
// same side of T as u does of U, more than 2^-25 (half an ulp of T) away from it, and
// so does its rounded quotient x = fl(w / c1): the code is that of x bit for bit. The
// code is base + (u > U) from the lane's own copy of the code table (entry k of lane l
// at byte 256 k + 8 l: the 32 lanes never meet in one bank; the address is one integer
// multiply-add of z's bit pattern). The per-weight work stays on the FMA pipe: the
// compare is sat(fl(u - U) 2^100), the codes are summed into the mantissa of 2^23
// (16 bits per float, joined by one byte permutation), and the lane keeps the smallest
// |u - U| of its weights. Where that is <= 2^-22, or where c1 is outside [2^-126, 2^125)
// (a reciprocal that is not a normal number), the lane's 8 or 4 codes are recomputed
// after the batch from the exact quotient and the threshold search, out of the
// unrolled path. Without BINS every weight is divided.
template <typename T, bool BINS>
__global__ void __launch_bounds__(256, 3)
k_quantize_codes(const __grid_constant__ QuantGroup grp, const __grid_constant__ Codebook cb, const __grid_constant__ CodeTable tab) {
    constexpr int VEC = 16 / sizeof(T);   // elements per 16-byte lane load
    constexpr int LPB = kBlock1 / VEC;    // lanes per block
    constexpr int BPI = 32 / LPB;         // blocks per warp iteration
    constexpr int ITERS = 32 / BPI;       // iterations per warp (32 blocks)
    constexpr int NBYTES = VEC / 2;       // code bytes per lane per iteration
    constexpr int BATCH = ITERS < 8 ? ITERS : 8;

    __shared__ float s_t[16];
    __shared__ float s_c1[kBlock2];
    extern __shared__ __align__(16) float2 s_tab[];   // BINS: [256][32] (64 KB)

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x < 15) s_t[threadIdx.x] = cb.t[threadIdx.x];
    if constexpr (BINS) {
        for (int i = threadIdx.x; i < 256 * 32; i += blockDim.x) s_tab[i] = make_float2(tab.thr[i >> 5], tab.base[i >> 5]);
    }
    __syncthreads();
    // z's bit pattern is 0x4B000000 + k and 0x4B000000 * 256 = 0 mod 2^32, so
    // bits(z) * 256 + tab_lane is the byte address of entry k of this lane
    const uint32_t tab_lane = static_cast<uint32_t>(__cvta_generic_to_shared(s_tab)) + (uint32_t)lane * 8u;
    const int sub = lane / LPB, li = lane % LPB;
    bool nonfinite = false;

    for (int64_t unit = blockIdx.x; unit < grp.groups; unit += gridDim.x) {
    const QuantItem &item = grp.it[quant_item(grp, unit, false)];
    const T *__restrict__ W = static_cast<const T *>(item.W);
    const int64_t n = item.n, nb = item.nb;
    const int64_t group = unit - item.cta0;
    const int64_t ncode = (n + 1) / 2;

    // FULL: the whole group lies inside the tensor (every group but a tensor's last):
    // no bounds checks, fixed offsets from per-lane base pointers
    auto run_group = [&](auto full_tag) {
    constexpr bool FULL = decltype(full_tag)::value;
    const int64_t lane_e = (group * kBlock2 + warp * 32 + sub) * kBlock1 + (int64_t)li * VEC;
    const T *__restrict__ Wl = W + lane_e;
    uint8_t *__restrict__ cl = item.codes + lane_e / 2;
#pragma unroll 1
    for (int it0 = 0; it0 < ITERS; it0 += BATCH) {
        uint4 raw[BATCH];
#pragma unroll
        for (int j = 0; j < BATCH; ++j) {
            const int off = (it0 + j) * BPI * kBlock1;
            if constexpr (FULL) {
                raw[j] = __ldg(reinterpret_cast<const uint4 *>(Wl + off));
            } else {
                const int64_t e0 = lane_e + off;
                raw[j] = (e0 + VEC <= n) ? __ldg(reinterpret_cast<const uint4 *>(W + e0))
                                         : (e0 < n ? load_partial<T>(W, e0, n) : make_uint4(0u, 0u, 0u, 0u));
            }
        }
        [[maybe_unused]] uint32_t redo = 0;
#pragma unroll
        for (int j = 0; j < BATCH; ++j) {
            const int local = warp * 32 + (it0 + j) * BPI + sub;   // block index within the group
            const int off = (it0 + j) * BPI * kBlock1;             // elements from the lane's first
            const uint32_t r4[4] = {raw[j].x, raw[j].y, raw[j].z, raw[j].w};
            float v[VEC];
            uint32_t mbits;
            if constexpr (sizeof(T) == 4) {
#pragma unroll
                for (int k = 0; k < 4; ++k) v[k] = __uint_as_float(r4[k]);
                mbits = max(max(r4[0] & 0x7fffffffu, r4[1] & 0x7fffffffu), max(r4[2] & 0x7fffffffu, r4[3] & 0x7fffffffu));
#pragma unroll
                for (int o = LPB / 2; o >= 1; o >>= 1) mbits = max(mbits, __shfl_xor_sync(0xffffffffu, mbits, o));
            } else {
#pragma unroll
                for (int k = 0; k < 4; ++k) { v[2 * k] = bf16_lo(r4[k]); v[2 * k + 1] = bf16_hi(r4[k]); }
                uint32_t h = vmax_u16x2(vmax_u16x2(r4[0] & 0x7fff7fffu, r4[1] & 0x7fff7fffu),
                                        vmax_u16x2(r4[2] & 0x7fff7fffu, r4[3] & 0x7fff7fffu));
#pragma unroll
                for (int o = LPB / 2; o >= 1; o >>= 1) h = vmax_u16x2(h, __shfl_xor_sync(0xffffffffu, h, o));
                mbits = max(h & 0xffffu, h >> 16) << 16;
            }
            const float m = __uint_as_float(mbits);
            nonfinite |= mbits >= 0x7f800000u;
            if (li == 0) {
                s_c1[local] = m;
                const int64_t b = group * kBlock2 + local;
                if (FULL || b < nb) item.c1[b] = m;
            }
            // codes of the lane's VEC elements: NBYTES bytes, byte k = hi << 4 | lo
            uint32_t packed = 0;
            if constexpr (BINS) {
                const float rh = mbits == 0u ? 0.0f : __fmul_rn(rcp_approx(m), 0.5f);
                const bool odd = mbits != 0u && (mbits - 0x00800000u) >= (0x7e000000u - 0x00800000u);
                constexpr float kNibble[4] = {16.0f, 1.0f, 4096.0f, 256.0f};   // byte = code(2i) << 4 | code(2i+1)
                float pf[(VEC + 3) / 4];
#pragma unroll
                for (int h = 0; h < (VEC + 3) / 4; ++h) pf[h] = 8388608.0f;
                float near = 1.0f;
#pragma unroll
                for (int k = 0; k < VEC; ++k) {
                    const float u = fma_sat(v[k], rh, 0.5f);
                    const float z = __fmaf_rn(u, 255.0f, 8388608.0f);
                    float thr, base;
                    lds_f2(__float_as_uint(z) * 256u + tab_lane, thr, base);
                    const float d = __fsub_rn(u, thr);
                    const float c = __fadd_rn(base, mul_sat(d, 0x1p100f));
                    pf[k / 4] = __fmaf_rn(c, kNibble[k % 4], pf[k / 4]);
                    near = fminf(near, fabsf(d));
                }
                if constexpr (VEC == 8) packed = prmt(__float_as_uint(pf[0]), __float_as_uint(pf[1]), 0x5410u);
                else packed = __float_as_uint(pf[0]) & 0xffffu;
                redo |= (odd || near <= 0x1p-22f) ? (1u << j) : 0u;
            } else {
#pragma unroll
                for (int k = 0; k < VEC; k += 2) {
                    const float x0 = (m == 0.0f) ? 0.0f : __fdiv_rn(v[k], m);
                    const float x1 = (m == 0.0f) ? 0.0f : __fdiv_rn(v[k + 1], m);
                    const uint32_t byte = ((uint32_t)nf4_code(x0, s_t) << 4) | (uint32_t)nf4_code(x1, s_t);
                    packed |= byte << (8 * (k / 2));
                }
            }
            if constexpr (FULL) {
                if constexpr (NBYTES == 4) *reinterpret_cast<uint32_t *>(cl + off / 2) = packed;
                else *reinterpret_cast<uint16_t *>(cl + off / 2) = (uint16_t)packed;
            } else {
                store_codes<NBYTES>(item.codes, (lane_e + off) / 2, ncode, packed);
            }
        }
        if constexpr (BINS) {
            __syncwarp();
            // exact codes of the lanes whose normalised weights came near a threshold
#pragma unroll 1
            for (; redo != 0u; redo &= redo - 1u) {
                const int j = __ffs(redo) - 1;
                const int local = warp * 32 + (it0 + j) * BPI + sub;
                const int64_t e0 = lane_e + (it0 + j) * BPI * kBlock1;
                const float m = s_c1[local];
                uint32_t packed = 0;
#pragma unroll 1
                for (int k = 0; k < VEC; ++k) {
                    const float w = (e0 + k < n) ? to_f32<T>(W[e0 + k]) : 0.0f;
                    const float x = (m == 0.0f) ? 0.0f : __fdiv_rn(w, m);
                    packed |= (uint32_t)nf4_code(x, s_t) << (8 * (k / 2) + ((k & 1) ? 0 : 4));
                }
                store_codes<NBYTES>(item.codes, e0 / 2, ncode, packed);
            }
        }
    }
    };
    if ((group + 1) * (int64_t)(kBlock1 * kBlock2) <= n) run_group(std::true_type{});
    else run_group(std::false_type{});
    __syncwarp();

    // fp64 pairwise tree over the warp's 32 leaves, the group's blocks 32 w .. 32 w + 31
    // (blocks past nb are 0): node i of level l+1 = node 2i + node 2i+1 of level l. The
    // group's eight warp sums are leaves 8 group .. 8 group + 7 of the tree that k_offset
    // completes, so no warp waits for another.
    double v = (double)s_c1[threadIdx.x];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const double u = __shfl_down_sync(0xffffffffu, v, o);
        if ((lane & (2 * o - 1)) == 0) v = v + u;
    }
    if (lane == 0) item.part[group * 8 + warp] = v;
    }
    if (__any_sync(0xffffffffu, nonfinite) && lane == 0) raise_status(QLORA_ERR_NONFINITE);
}

// Upper levels of the pairwise tree over the 8 nb2 partials (32 blocks each), zero-padded
// to a power of two (>= 1024): thread t first reduces leaves [tC, tC+C) with
// a binary-counter stack (which forms exactly the subtree of those leaves),
// then the 1024 subtree sums are combined level by level. mu = fl(S / nb).
__global__ void __launch_bounds__(1024)
k_offset(const __grid_constant__ QuantGroup grp) {
    __shared__ double s_w[32];
    const QuantItem &item = grp.it[blockIdx.x];
    const double *__restrict__ part = item.part;
    const int64_t nl = 8 * item.nb2, nb = item.nb;
    float *__restrict__ offset_out = item.offset;
    int64_t L = 1024;
    while (L < nl) L <<= 1;
    const int64_t C = L / 1024;
    const int64_t i0 = (int64_t)threadIdx.x * C;
    double v = 0.0;
    if (i0 < nl) {
        double stack[48];
        int level[48];
        int sp = 0;
        for (int64_t i = 0; i < C; ++i) {
            double x = (i0 + i < nl) ? part[i0 + i] : 0.0;
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
k_double_quant(const __grid_constant__ QuantGroup grp) {
    const QuantItem &item = grp.it[quant_item(grp, blockIdx.x, true)];
    const float *__restrict__ c1 = item.c1;
    const int64_t nb = item.nb, nb2 = item.nb2;
    const float *__restrict__ offset = item.offset;
    int8_t *__restrict__ q8 = item.scale8;
    float *__restrict__ s2 = item.scale2;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t j = (int64_t)(blockIdx.x - item.dq0) * 8 + warp;
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

// Dequantisation, over one tensor or a list of them in one launch. The codes of
// every tensor are cut into chunks of 256 32-bit words (2048 weights, 32 blocks;
// chunks never straddle a second-level group of 2048 words), numbered across the
// list; warps walk the chunks grid-stride. Lane l of a warp expands words
// 32 u + l (u = 0..7) of its chunk: eight coalesced 4-byte code loads and eight
// coalesced 16-byte bf16 stores, all loads issued before any arithmetic. Each word
// is one eighth of a 64-block: c^ = fl(fl(q8 * fl(s2 / 127)) + mu) with the step
// divided once per chunk, then w^ = bf16(fl(Q[code] * c^)) from the codebook in
// shared memory (16 distinct words: the lookups never conflict). The last n % 8
// weights of a tensor, if any, are written element by element.
constexpr int kDeqChunkWords = 256;
constexpr int kDeqMaxItems = 64;
struct DeqItem {
    const uint32_t *codes;
    const int8_t *scale8;
    const float *scale2;
    const float *offset;
    __nv_bfloat16 *out;
    int64_t n;              // weights
    int64_t chunk0;         // first chunk of this tensor in the list's numbering
};
struct DeqGroup {
    DeqItem it[kDeqMaxItems];
    int count;
    int64_t chunks;         // total
};

__device__ __forceinline__ uint32_t dequant_pair(const float *s_q, uint32_t byte, float ch) {
    return pack_bf16x2(__fmul_rn(s_q[byte >> 4], ch), __fmul_rn(s_q[byte & 15u], ch));
}

__global__ void __launch_bounds__(256)
k_dequant(const __grid_constant__ DeqGroup grp, const __grid_constant__ Codebook cb) {
    __shared__ float s_q[16];
    if (threadIdx.x < 16) s_q[threadIdx.x] = cb.q[threadIdx.x];
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
    int ii = 0;
    float mu = __ldg(grp.it[0].offset);
    for (int64_t c = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; c < grp.chunks; c += nwarps) {
        if (c >= grp.it[ii].chunk0 + ((grp.it[ii].n / 8 + kDeqChunkWords - 1) / kDeqChunkWords)) {
            do { ++ii; } while (ii + 1 < grp.count && c >= grp.it[ii + 1].chunk0);
            mu = __ldg(grp.it[ii].offset);
        }
        const DeqItem &it = grp.it[ii];
        const int64_t nw = it.n / 8;                       // whole code words
        const int64_t w0 = (c - it.chunk0) * kDeqChunkWords;
        uint32_t w[8];
        int8_t q8[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int64_t wi = w0 + 32 * u + lane;
            w[u] = wi < nw ? __ldg(it.codes + wi) : 0u;
            q8[u] = wi < nw ? __ldg(it.scale8 + (wi >> 3)) : (int8_t)0;
        }
        const float step = __fdiv_rn(__ldg(it.scale2 + (w0 >> 11)), 127.0f);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int64_t wi = w0 + 32 * u + lane;
            if (wi < nw) {
                const float ch = __fadd_rn(__fmul_rn((float)q8[u], step), mu);
                uint4 o;
                o.x = dequant_pair(s_q, w[u] & 0xffu, ch);
                o.y = dequant_pair(s_q, (w[u] >> 8) & 0xffu, ch);
                o.z = dequant_pair(s_q, (w[u] >> 16) & 0xffu, ch);
                o.w = dequant_pair(s_q, w[u] >> 24, ch);
                reinterpret_cast<uint4 *>(it.out)[wi] = o;
            }
        }
    }
    // the last n % 8 weights of tensor blockIdx.x (the code word is read byte by byte)
    if ((int)blockIdx.x < grp.count && threadIdx.x == 0) {
        const DeqItem &it = grp.it[blockIdx.x];
        const uint8_t *cbytes = reinterpret_cast<const uint8_t *>(it.codes);
        const float m = __ldg(it.offset);
        for (int64_t e = (it.n / 8) * 8; e < it.n; ++e) {
            const int64_t b = e / kBlock1;
            const float ch = dq_constant(it.scale8[b], it.scale2[b / kBlock2], m);
            const uint8_t byte = cbytes[e / 2];
            const uint32_t code = (e % 2 == 0) ? (byte >> 4) : (byte & 15u);
            it.out[e] = __float2bfloat16_rn(__fmul_rn(s_q[code], ch));
        }
    }
}

// ---------------------------------------------------------------- adapter merge
// Merged BF16 weight (the page's sections 5 and 6: merging the adapter into the
// weight and re-quantising can change outputs; the merge is done in BF16):
//   w'[n,k] = bf16( fl( w^[n,k] + fl(s * d[n,k]) ) ),
//   d[n,k]  = fused multiply-adds of A[k,j] * B[j,n] over j = 0 .. r-1 in order, from 0,
// with w^ the dequantised weight computed in place (step 7 of the format). The fixed
// order of the r multiply-adds keeps this on the fp32 FMA pipes (r FMAs per weight;
// the bound is the FMA rate, not HBM).
//
// k_merge_prep widens A and B to fp32 once, A transposed (At[j][k]) and B with rows
// padded to a multiple of four (Bf[j][n]), so that k_merge_bf16 stages both with
// 16-byte asynchronous copies. k_merge_bf16: persistent, two 256-thread CTAs per SM
// over 128 x 128 tiles of W; each thread keeps an 8 x 8 block of d in registers (rows
// 8t..8t+7, inputs 4t..4t+3 and 64+4t..+3 of the tile, so that a warp's 16-byte
// shared loads of At are contiguous). At and Bf come in chunks of 32 j through two
// shared-memory buffers: the copies of the next (tile, chunk) step are in flight
// while the current one is multiplied (four 16-byte shared loads per 64 FMAs).
constexpr int kMergeTile = 128;
constexpr int kMergeJ = 32;
constexpr int kMergeBuf = kMergeJ * kMergeTile;                       // floats per operand per buffer
constexpr size_t kMergeSmem = (size_t)2 * 2 * kMergeBuf * sizeof(float);   // 64 KB

__global__ void k_merge_prep(const __nv_bfloat16 *__restrict__ A, const __nv_bfloat16 *__restrict__ B, int r,
                             int64_t K, int64_t N, int64_t ldb, float *__restrict__ At, float *__restrict__ Bf) {
    const int64_t j = blockIdx.y;                   // one adapter rank per grid row
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; k < K; k += stride)
        At[j * K + k] = __bfloat162float(A[k * r + j]);
    for (int64_t n = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; n < ldb; n += stride)
        Bf[j * ldb + n] = n < N ? __bfloat162float(B[j * N + n]) : 0.0f;
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__global__ void __launch_bounds__(256, 2)
k_merge_bf16(NF4View q, const float *__restrict__ At, const float *__restrict__ Bf, int64_t ldb, int r, float s,
             const __grid_constant__ Codebook cb, __nv_bfloat16 *__restrict__ out) {
    extern __shared__ __align__(16) float msm[];   // [buf][At chunk | Bf chunk], each [kMergeJ][kMergeTile]
    __shared__ float s_q[16];
    __shared__ float s_ch[2 * kMergeTile];         // c^ of (row n0 + i, 64-block g of the tile) at 2 i + g
    if (threadIdx.x < 16) s_q[threadIdx.x] = cb.q[threadIdx.x];
    const int64_t rows = q.rows, cols = q.cols, kbs = cols / 64;
    const float mu = __ldg(q.offset);
    const int tn = threadIdx.x >> 4, tk = threadIdx.x & 15;
    const int64_t tiles_n = (rows + kMergeTile - 1) / kMergeTile;
    const int64_t tiles_k = (cols + kMergeTile - 1) / kMergeTile;
    const int64_t tiles = tiles_n * tiles_k;
    const int nj = (r + kMergeJ - 1) / kMergeJ;
    const uint32_t sm0 = static_cast<uint32_t>(__cvta_generic_to_shared(msm));

    // copies of step (tile, chunk) into buffer buf: 2048 16-byte pieces, 8 per thread
    auto issue = [&](int64_t tile, int c, int buf) {
        const int64_t n0 = (tile % tiles_n) * kMergeTile, k0 = (tile / tiles_n) * kMergeTile;
        const int j0 = c * kMergeJ;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int piece = threadIdx.x + 256 * (u & 3);          // [jj][c4] of one operand
            const int jj = piece >> 5, c4 = piece & 31;
            const int j = j0 + jj;
            const uint32_t dst = sm0 + (uint32_t)(((buf * 2 + (u >> 2)) * kMergeBuf + jj * kMergeTile + 4 * c4) * 4);
            if (u < 4) {
                const int64_t k = k0 + 4 * c4;
                const bool ok = j < r && k < cols;
                cp_async16(dst, ok ? At + (int64_t)j * cols + k : At, ok ? 16u : 0u);
            } else {
                const int64_t n = n0 + 4 * c4;
                const bool ok = j < r && n < ldb;
                cp_async16(dst, ok ? Bf + (int64_t)j * ldb + n : Bf, ok ? 16u : 0u);
            }
        }
        cp_async_commit();
    };

    int64_t tile = blockIdx.x;
    if (tile < tiles) issue(tile, 0, 0);
    int step = 0;
    for (; tile < tiles; tile += gridDim.x) {
        const int64_t n0 = (tile % tiles_n) * kMergeTile, k0 = (tile / tiles_n) * kMergeTile;
        // d[i][2p], d[i][2p + 1] as one 64-bit pair dd[i][p] (low half first): two fused
        // multiply-adds per instruction (fma.rn.f32x2, each half one IEEE fma)
        uint64_t dd[8][4];
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int c = 0; c < 4; ++c) dd[i][c] = 0ull;
        for (int c = 0; c < nj; ++c, ++step) {
            // the next step's copies go out before this step's wait
            const bool more = c + 1 < nj || tile + gridDim.x < tiles;
            if (more) {
                if (c + 1 < nj) issue(tile, c + 1, (step + 1) & 1);
                else issue(tile + gridDim.x, 0, (step + 1) & 1);
                cp_async_wait<1>();
            } else {
                cp_async_wait<0>();
            }
            __syncthreads();   // this step's buffer is complete for every thread
            if (c == 0) {
                const int64_t n = n0 + (threadIdx.x >> 1), blkk = k0 / 64 + (threadIdx.x & 1);
                s_ch[threadIdx.x] = (n < rows && blkk < kbs)
                                        ? dq_constant(q.scale8[n * kbs + blkk], q.scale2[(n * kbs + blkk) / kBlock2], mu)
                                        : 0.0f;
            }
            // this thread's columns of the chunk: fixed offsets from two base pointers
            const float *Ap = msm + (size_t)((step & 1) * 2) * kMergeBuf + 4 * tk;
            const float *Bp = msm + (size_t)((step & 1) * 2 + 1) * kMergeBuf + 8 * tn;
            const int jn = r - c * kMergeJ < kMergeJ ? r - c * kMergeJ : kMergeJ;
            auto fma_step = [&](int jj) {
                const ulonglong2 a0 = *reinterpret_cast<const ulonglong2 *>(Ap + jj * kMergeTile);
                const ulonglong2 a1 = *reinterpret_cast<const ulonglong2 *>(Ap + jj * kMergeTile + 64);
                const float4 b0 = *reinterpret_cast<const float4 *>(Bp + jj * kMergeTile);
                const float4 b1 = *reinterpret_cast<const float4 *>(Bp + jj * kMergeTile + 4);
                const uint64_t ap[4] = {a0.x, a0.y, a1.x, a1.y};      // inputs (2p, 2p + 1)
                const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    uint64_t bb;
                    asm("mov.b64 %0, {%1, %1};" : "=l"(bb) : "f"(b[i]));
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(dd[i][c]) : "l"(ap[c]), "l"(bb));
                }
            };
            if (jn == kMergeJ) {
#pragma unroll
                for (int jj = 0; jj < kMergeJ; ++jj) fma_step(jj);
            } else {
#pragma unroll 1
                for (int jj = 0; jj < jn; ++jj) fma_step(jj);
            }
            __syncthreads();   // every thread is done with this buffer before it is refilled
        }
        // dequantise the thread's weights and add: rows n0 + 8 tn + i, inputs
        // k0 + 64 g + 4 tk .. + 3 (g = 0, 1; each group inside one 64-block)
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int64_t n = n0 + 8 * tn + i;
            if (n >= rows) break;
#pragma unroll
            for (int g = 0; g < 2; ++g) {
                const int64_t k = k0 + 64 * g + 4 * tk;
                if (k >= cols) continue;
                const int64_t e0 = n * cols + k;
                const float ch = s_ch[2 * (8 * tn + i) + g];
                const uint32_t cw = *reinterpret_cast<const uint16_t *>(q.codes + e0 / 2);
                uint32_t o[2];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint32_t byte = (cw >> (8 * h)) & 0xffu;
                    const float w_hi = __bfloat162float(__float2bfloat16_rn(__fmul_rn(s_q[byte >> 4], ch)));
                    const float w_lo = __bfloat162float(__float2bfloat16_rn(__fmul_rn(s_q[byte & 15u], ch)));
                    float d0, d1;                                   // inputs 4g + 2h and 4g + 2h + 1
                    asm("mov.b64 {%0, %1}, %2;" : "=f"(d0), "=f"(d1) : "l"(dd[i][2 * g + h]));
                    o[h] = pack_bf16x2(__fadd_rn(w_hi, __fmul_rn(s, d0)), __fadd_rn(w_lo, __fmul_rn(s, d1)));
                }
                *reinterpret_cast<uint2 *>(out + e0) = make_uint2(o[0], o[1]);
            }
        }
    }
}

size_t merge_prep_bytes(int64_t rows, int64_t cols) {
    return align256((size_t)256 * (size_t)cols * 4) + align256((size_t)256 * (size_t)((rows + 3) / 4 * 4) * 4);
}

cudaError_t launch_merge_bf16(const NF4View &q, const __nv_bfloat16 *A, const __nv_bfloat16 *B, int r, float s,
                              __nv_bfloat16 *out, void *prep, cudaStream_t st) {
    const int64_t ldb = (q.rows + 3) / 4 * 4;
    float *At = static_cast<float *>(prep);
    float *Bf = reinterpret_cast<float *>(static_cast<char *>(prep) + align256((size_t)256 * (size_t)q.cols * 4));
    int64_t px = ceil_div(q.cols > ldb ? q.cols : ldb, (int64_t)256);
    if (px > 64) px = 64;
    QNF4_LAUNCH("k_merge_prep", st,
                k_merge_prep<<<dim3((unsigned)px, (unsigned)r), 256, 0, st>>>(A, B, r, q.cols, q.rows, ldb, At, Bf));
    const int64_t tiles = ceil_div(q.rows, (int64_t)kMergeTile) * ceil_div(q.cols, (int64_t)kMergeTile);
    int64_t grid = tiles;
    const int64_t cap = (int64_t)num_sms() * 2;
    if (grid > cap) grid = cap;
    static const cudaError_t attr =
        cudaFuncSetAttribute(k_merge_bf16, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kMergeSmem);
    if (attr != cudaSuccess) return attr;
    QNF4_LAUNCH("k_merge_bf16", st,
                k_merge_bf16<<<(unsigned)grid, 256, kMergeSmem, st>>>(q, At, Bf, ldb, r, s, host_codebook(), out));
    return cudaGetLastError();
}

// ---------------------------------------------------------------- launchers
// Code search of the quantiser: the bin table with its exact fallback (default) or a
// division for every weight; both give the same codes (the second exists so that the
// tests can compare the two).
static std::atomic<int> g_divide_every_weight{0};

// Three launches over up to kQuantMaxItems tensors of one input dtype.
static cudaError_t quantize_launch(const QuantArgs *a, int count, qlora_dtype dt, cudaStream_t st) {
    const Codebook &cb = host_codebook();
    static CodeTable table;
    static const bool table_ok = build_code_table(cb, table);
    const bool use_bins = table_ok && g_divide_every_weight.load() == 0;
    QuantGroup g;
    g.count = count;
    int64_t groups = 0, dq = 0;
    for (int i = 0; i < count; ++i) {
        QuantItem &it = g.it[i];
        it.W = a[i].W;
        it.n = a[i].n;
        it.nb = ceil_div(it.n, kBlock1);
        it.nb2 = ceil_div(it.nb, kBlock2);
        it.c1 = a[i].c1;
        it.part = a[i].part;
        it.codes = a[i].out.codes;
        it.scale8 = a[i].out.scale8;
        it.scale2 = a[i].out.scale2;
        it.offset = a[i].out.offset;
        it.cta0 = groups;
        it.dq0 = dq;
        groups += it.nb2;
        dq += ceil_div(it.nb2, 8);
    }
    g.groups = groups;
    if (dq > 0x7fffffffLL) return cudaErrorInvalidValue;
    // persistent: three 256-thread CTAs per SM (65 KB of shared memory each)
    int64_t grid = groups;
    const int64_t cap = (int64_t)num_sms() * 3;
    if (grid > cap) grid = cap;
    if (grid < 1) grid = 1;
    const unsigned gx = (unsigned)grid;
    const size_t tab_bytes = (size_t)256 * 32 * sizeof(float2);
    static const bool attr_ok =
        cudaFuncSetAttribute(k_quantize_codes<float, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)tab_bytes) == cudaSuccess &&
        cudaFuncSetAttribute(k_quantize_codes<__nv_bfloat16, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)tab_bytes) == cudaSuccess;
    if (!attr_ok) return cudaErrorInvalidValue;
    if (dt == QLORA_F32) {
        if (use_bins)
            QNF4_LAUNCH("k_quantize_codes", st, k_quantize_codes<float, true><<<gx, 256, tab_bytes, st>>>(g, cb, table));
        else
            QNF4_LAUNCH("k_quantize_codes", st, k_quantize_codes<float, false><<<gx, 256, 0, st>>>(g, cb, table));
    } else {
        if (use_bins)
            QNF4_LAUNCH("k_quantize_codes", st, k_quantize_codes<__nv_bfloat16, true><<<gx, 256, tab_bytes, st>>>(g, cb, table));
        else
            QNF4_LAUNCH("k_quantize_codes", st, k_quantize_codes<__nv_bfloat16, false><<<gx, 256, 0, st>>>(g, cb, table));
    }
    QNF4_LAUNCH("k_offset", st, k_offset<<<(unsigned)count, 1024, 0, st>>>(g));
    QNF4_LAUNCH("k_double_quant", st, k_double_quant<<<(unsigned)dq, 256, 0, st>>>(g));
    return cudaGetLastError();
}

cudaError_t launch_quantize(const void *W, qlora_dtype dt, int64_t n, const qlora_nf4_tensor &out,
                            float *c1, double *part, cudaStream_t st) {
    const QuantArgs a{W, n, out, c1, part};
    return quantize_launch(&a, 1, dt, st);
}

cudaError_t launch_quantize_grouped(const QuantArgs *a, int count, qlora_dtype dt, cudaStream_t st) {
    for (int i = 0; i < count; i += kQuantMaxItems) {
        const int n = count - i < kQuantMaxItems ? count - i : kQuantMaxItems;
        cudaError_t e = quantize_launch(a + i, n, dt, st);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

// One launch over up to kDeqMaxItems tensors; a persistent grid of up to eight
// 256-thread CTAs per SM.
static cudaError_t dequant_launch(const NF4View *q, __nv_bfloat16 *const *out, int count, int ctas_per_sm,
                                  cudaStream_t st) {
    DeqGroup g;
    g.count = count;
    int64_t chunks = 0;
    for (int i = 0; i < count; ++i) {
        DeqItem &it = g.it[i];
        it.codes = reinterpret_cast<const uint32_t *>(q[i].codes);
        it.scale8 = q[i].scale8;
        it.scale2 = q[i].scale2;
        it.offset = q[i].offset;
        it.out = out[i];
        it.n = q[i].rows * q[i].cols;
        it.chunk0 = chunks;
        chunks += ceil_div(it.n / 8, kDeqChunkWords);
    }
    g.chunks = chunks;
    int64_t grid = ceil_div(chunks, 8);                   // eight warps per CTA
    const int64_t cap = (int64_t)num_sms() * ctas_per_sm;
    if (grid > cap) grid = cap;
    if (grid < count) grid = count;                       // one CTA per tensor writes its tail
    QNF4_LAUNCH("k_dequant", st, k_dequant<<<(unsigned)grid, 256, 0, st>>>(g, host_codebook()));
    return cudaGetLastError();
}

cudaError_t launch_dequant(const NF4View &q, __nv_bfloat16 *out, cudaStream_t st, int ctas_per_sm) {
    return dequant_launch(&q, &out, 1, ctas_per_sm, st);
}

cudaError_t launch_dequant_grouped(const NF4View *q, __nv_bfloat16 *const *out, int count, cudaStream_t st) {
    for (int i = 0; i < count; i += kDeqMaxItems) {
        const int n = count - i < kDeqMaxItems ? count - i : kDeqMaxItems;
        cudaError_t e = dequant_launch(q + i, out + i, n, 8, st);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace qnf4

extern "C" void qlora_nf4_set_code_search(int divide_every_weight) {
    qnf4::g_divide_every_weight.store(divide_every_weight ? 1 : 0);
}
