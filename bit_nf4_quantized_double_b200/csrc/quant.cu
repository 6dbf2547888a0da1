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

#include <atomic>
#include <cmath>

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
// A list of tensors quantised by one sequence of launches: CTA ranges per tensor
// (groups in k_quantize_codes, blocks of eight groups in k_double_quant), one CTA
// per tensor in k_offset.
constexpr int kQuantMaxItems = 64;
struct QuantItem {
    const void *W;
    int64_t n, nb, nb2;
    float *c1;                   // [nb] exact absmax (workspace)
    double *part;                // [nb2] group partial sums (workspace)
    uint8_t *codes;
    int8_t *scale8;
    float *scale2;
    float *offset;
    int64_t cta0;                // first CTA of this tensor in k_quantize_codes
    int64_t dq0;                 // first CTA of this tensor in k_double_quant
};
struct QuantGroup {
    QuantItem it[kQuantMaxItems];
    int count;
};
// The tensor whose CTA range holds block b (ranges ascending from 0).
__device__ __forceinline__ int quant_item(const QuantGroup &g, int64_t b, bool dq) {
    int lo = 0, hi = g.count - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if ((dq ? g.it[mid].dq0 : g.it[mid].cta0) <= b) lo = mid; else hi = mid - 1;
    }
    return lo;
}

template <typename T, bool BINS>
__global__ void __launch_bounds__(256, 4)
k_quantize_codes(const __grid_constant__ QuantGroup grp, Codebook cb, const __grid_constant__ CodeBins bins) {
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

    const QuantItem &item = grp.it[quant_item(grp, blockIdx.x, false)];
    const T *__restrict__ W = static_cast<const T *>(item.W);
    const int64_t n = item.n, nb = item.nb;
    float *__restrict__ c1_out = item.c1;
    double *__restrict__ part_out = item.part;
    uint8_t *__restrict__ codes = item.codes;
    const int64_t group = blockIdx.x - item.cta0;
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
k_offset(const __grid_constant__ QuantGroup grp) {
    __shared__ double s_w[32];
    const QuantItem &item = grp.it[blockIdx.x];
    const double *__restrict__ part = item.part;
    const int64_t nb2 = item.nb2, nb = item.nb;
    float *__restrict__ offset_out = item.offset;
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
k_dequant(const __grid_constant__ DeqGroup grp, Codebook cb) {
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
// Code search of the quantiser: the bin table with its exact fallback (default) or a
// division for every weight; both give the same codes (the second exists so that the
// tests can compare the two).
static std::atomic<int> g_divide_every_weight{0};

// Three launches over up to kQuantMaxItems tensors of one input dtype.
static cudaError_t quantize_launch(const QuantArgs *a, int count, qlora_dtype dt, cudaStream_t st) {
    const Codebook &cb = host_codebook();
    static CodeBins bins;
    static const bool bins_ok = build_code_bins(cb, bins);
    const bool use_bins = bins_ok && g_divide_every_weight.load() == 0;
    QuantGroup g;
    g.count = count;
    int64_t ctas = 0, dq = 0;
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
        it.cta0 = ctas;
        it.dq0 = dq;
        ctas += it.nb2;
        dq += ceil_div(it.nb2, 8);
    }
    if (ctas > 0x7fffffffLL || dq > 0x7fffffffLL) return cudaErrorInvalidValue;
    if (dt == QLORA_F32) {
        if (use_bins)
            QNF4_LAUNCH("k_quantize_codes", st, k_quantize_codes<float, true><<<(unsigned)ctas, 256, 0, st>>>(g, cb, bins));
        else
            QNF4_LAUNCH("k_quantize_codes", st, k_quantize_codes<float, false><<<(unsigned)ctas, 256, 0, st>>>(g, cb, bins));
    } else {
        if (use_bins)
            QNF4_LAUNCH("k_quantize_codes", st, k_quantize_codes<__nv_bfloat16, true><<<(unsigned)ctas, 256, 0, st>>>(g, cb, bins));
        else
            QNF4_LAUNCH("k_quantize_codes", st, k_quantize_codes<__nv_bfloat16, false><<<(unsigned)ctas, 256, 0, st>>>(g, cb, bins));
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
static cudaError_t dequant_launch(const NF4View *q, __nv_bfloat16 *const *out, int count, cudaStream_t st) {
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
    const int64_t cap = (int64_t)num_sms() * 8;
    if (grid > cap) grid = cap;
    if (grid < count) grid = count;                       // one CTA per tensor writes its tail
    QNF4_LAUNCH("k_dequant", st, k_dequant<<<(unsigned)grid, 256, 0, st>>>(g, host_codebook()));
    return cudaGetLastError();
}

cudaError_t launch_dequant(const NF4View &q, __nv_bfloat16 *out, cudaStream_t st) {
    return dequant_launch(&q, &out, 1, st);
}

cudaError_t launch_dequant_grouped(const NF4View *q, __nv_bfloat16 *const *out, int count, cudaStream_t st) {
    for (int i = 0; i < count; i += kDeqMaxItems) {
        const int n = count - i < kDeqMaxItems ? count - i : kDeqMaxItems;
        cudaError_t e = dequant_launch(q + i, out + i, n, st);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace qnf4

extern "C" void qlora_nf4_set_code_search(int divide_every_weight) {
    qnf4::g_divide_every_weight.store(divide_every_weight ? 1 : 0);
}
