// Small-M (M <= 16 tokens) forward: a streaming NF4 GEMV on the warp-level
// tensor-core path, and the dispatch between it and the tcgen05 GEMMs.
//
// Layer: Y = X W^ + s (X A) B (page "QLoRA: put the large model in memory,
// then change it with a small adapter", wq-win.github.io/llm/074-qlora,
// section 1), at decode-sized M where the packed 4-bit codes dominate HBM
// traffic (section 2: about 4.127 bits per weight).
//
// Three launches, each chained to the previous one by programmatic dependent
// launch so that it starts while its predecessor still runs:
//   k_gemv         persistent, one CTA per SM, over work units of 16 RG weight rows
//                  x 2048 inputs (1 KB of codes per row), ordered (projection, K
//                  chunk, row block) and cut into contiguous ranges of equal weight
//                  count, one per CTA; writes each unit's fp32 sums to the workspace.
//                  RG = 2 row groups for M <= 8, 1 for larger M (whose X fragments
//                  need twice the registers);
//   k_gemv_xa      one warp per (adapter, 128 inputs): the X A partial sums, run
//                  beside the GEMV (no shared memory, so its warps fit next to a
//                  GEMV CTA);
//   k_gemv_finish  one thread per output element: Y = the K chunks' sums in chunk order
//                  + (s XA) B with XA = its chunk partials in chunk order, rounded to
//                  bf16; the first CTA of a projection also saves XA as bf16.
// In k_gemv a producer warp loads each unit's codes with TMA (one 3D box of
// 8 K slices x 16 RG rows x 128 bytes, 128-byte swizzle, or eight 2D boxes when a
// row is not a whole number of 128-byte slices) and computes the unit's
// dequantised block constants c^ (double quantisation, section 3) into the stage
// from int8 constants it fetched three units earlier.
// 8 RG compute warps, RG row groups of 16 x 8 K slices of 256 inputs, keep
// their slice of X in registers as mma B fragments for as long as the units
// stay in one (projection, K chunk), turn each code byte into a bf16 pair
// (Q[hi], Q[lo]) with one byte permute (address = byte * 256 + lane * 4) and one
// load from a per-lane replicated table, accumulate sum_k Q[code] x_k per
// 64-block with mma.sync m16n8k16 (16 weight rows x 8 tokens) and scale each
// block's partial dot product by its c^. The eight K slices of a row group are
// added in slice order through shared memory by one of them (the role rotates
// from unit to unit). Every output is thus a fixed-order sum, whichever CTA
// computes it.
#include "launch.h"
#include "tc.cuh"
#include "tmap.h"

namespace qnf4 {

using namespace tc;

cudaError_t launch_linear_fwd_large(const __nv_bfloat16 *X, int64_t M, const NF4View &W, const __nv_bfloat16 *A,
                                    const __nv_bfloat16 *B, int r, float s, __nv_bfloat16 *Y,
                                    __nv_bfloat16 *XA_save, void *ws, cudaStream_t st);

constexpr int kGemvMaxM = 16;
constexpr int kGemvSlice = 256;                 // inputs per compute warp (4 blocks of 64)
constexpr int kGemvMaxSlices = 8;               // slices per K chunk (one per compute warp)
constexpr int kGemvMaxItems = 8;
constexpr int kGemvMaxGrid = 160;
// Shared memory: a 64 KB region whose 256 rows of 256 bytes hold the lookup table in
// their first 128 bytes (one word per lane) and, in the second 128 bytes ("holes"),
// the c^ of the stages (one hole per stage row) and then the K-slice reduction
// buffer (32 RG NT holes); then the stages; then barriers.
constexpr int kLutRegion = 65536;

// Row groups of 16 per unit, by token tiles of 8: the M <= 8 variant has 16 compute
// warps (17 with the producer: at most 96 registers a thread), the 9..16 variant 8
// (9 warps: room for its 64 registers of X fragments).
__host__ __device__ constexpr int gemv_rg(int nt) { return nt == 1 ? 2 : 1; }
__host__ __device__ constexpr int gemv_rows(int nt) { return 16 * gemv_rg(nt); }
constexpr int kGemvProducers = 2;              // producer warps, taking alternate units
__host__ __device__ constexpr int gemv_threads(int nt) { return 256 * gemv_rg(nt) + 32 * kGemvProducers; }
__host__ __device__ constexpr int gemv_box_bytes(int nt) { return gemv_rows(nt) * 128; }
__host__ __device__ constexpr int gemv_stage_bytes(int nt) { return 8 * gemv_box_bytes(nt); }
__host__ __device__ constexpr int gemv_stages(int nt) { return nt == 1 ? 4 : 8; }
__host__ __device__ constexpr int gemv_red_hole0(int nt) { return gemv_rows(nt) * gemv_stages(nt); }
// holes of one of the two reduction buffers (a warp's slice sums: 32 lanes x NT float4)
__host__ __device__ constexpr int gemv_red_holes(int nt) { return 32 * gemv_rg(nt) * nt; }
__host__ __device__ constexpr int gemv_smem(int nt) {
    return 1024 + kLutRegion + gemv_stages(nt) * gemv_stage_bytes(nt) + 512;
}
static_assert(gemv_smem(1) <= 232448 && gemv_smem(2) <= 232448, "shared memory");
static_assert(gemv_red_hole0(1) + 2 * gemv_red_holes(1) <= 256 && gemv_red_hole0(2) + 2 * gemv_red_holes(2) <= 256,
              "holes");

__device__ __forceinline__ uint32_t hole(int h) { return (uint32_t)h * 256u + 128u; }

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack2_bf16(const __nv_bfloat16 *p0, const __nv_bfloat16 *p1) {
    const uint32_t lo = *reinterpret_cast<const uint16_t *>(p0), hi = *reinterpret_cast<const uint16_t *>(p1);
    return lo | (hi << 16);
}


__device__ __forceinline__ void sts128f(uint32_t a, float4 v) {
    asm volatile("st.shared.v4.f32 [%0], {%1,%2,%3,%4};" ::"r"(a), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w) : "memory");
}
__device__ __forceinline__ void sts128u(uint32_t a, uint4 v) {
    asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}

// ---------------------------------------------------------------- adapter product
constexpr int kXaChunk = 128;                   // inputs per k_gemv_xa warp
struct XaItem {
    const __nv_bfloat16 *X;      // [M, K]
    const __nv_bfloat16 *A;      // [K, r]
    float *xpart;                // [nchunks][M][r] partial sums of X A
    int K, r, cta0;
};
struct XaGroup {
    XaItem it[kGemvMaxItems];
    int n, M;
};

// X A over one 128-input chunk: mma m16n8k16 with X rows (tokens, zero past M) as A
// and the adapter's columns as B, the chunk's 32 16-input steps in order.
__global__ void __launch_bounds__(32) k_gemv_xa(const __grid_constant__ XaGroup grp) {
    griddep_launch_dependents();
    int ii = 0;
    while (ii + 1 < grp.n && (int)blockIdx.x >= grp.it[ii + 1].cta0) ++ii;
    const XaItem &it = grp.it[ii];
    const int M = grp.M, K = it.K, r = it.r;
    const int c = blockIdx.x - it.cta0;
    const int k_begin = c * kXaChunk, k_end = min(K, k_begin + kXaChunk);
    const int lane = threadIdx.x, g = lane >> 2, t = lane & 3;
    float *dst = it.xpart + (int64_t)c * M * r;
    for (int nt0 = 0; nt0 < r / 8; nt0 += 4) {
        const int nts = min(4, r / 8 - nt0);
        float acc[4][4];
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[q][0] = acc[q][1] = acc[q][2] = acc[q][3] = 0.0f;
#pragma unroll 8
        for (int k0 = k_begin; k0 < k_end; k0 += 16) {
            uint32_t a[4] = {0u, 0u, 0u, 0u};
            if (g < M) {
                a[0] = __ldg(reinterpret_cast<const unsigned int *>(it.X + (int64_t)g * K + k0 + 2 * t));
                a[2] = __ldg(reinterpret_cast<const unsigned int *>(it.X + (int64_t)g * K + k0 + 8 + 2 * t));
            }
            if (g + 8 < M) {
                a[1] = __ldg(reinterpret_cast<const unsigned int *>(it.X + (int64_t)(g + 8) * K + k0 + 2 * t));
                a[3] = __ldg(reinterpret_cast<const unsigned int *>(it.X + (int64_t)(g + 8) * K + k0 + 8 + 2 * t));
            }
            uint32_t bb[4][2];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                bb[q][0] = bb[q][1] = 0u;
                if (q < nts) {
                    const __nv_bfloat16 *ak = it.A + (int64_t)(k0 + 2 * t) * r + (nt0 + q) * 8 + g;
                    bb[q][0] = pack2_bf16(ak, ak + r);
                    bb[q][1] = pack2_bf16(ak + 8 * r, ak + 9 * r);
                }
            }
#pragma unroll
            for (int q = 0; q < 4; ++q)
                if (q < nts) mma_bf16_16816(acc[q], a, bb[q][0], bb[q][1]);
        }
        // c[0], c[1]: token g, tile columns 2t, 2t+1; c[2], c[3]: token g + 8
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            if (q >= nts) continue;
            const int j0 = (nt0 + q) * 8 + 2 * t;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int tok = g + (e >= 2 ? 8 : 0);
                if (tok < M) dst[tok * r + j0 + (e & 1)] = acc[q][e];
            }
        }
    }
    griddep_wait();                                  // this grid ends after the GEMV
}

// ---------------------------------------------------------------- main kernel
// The K range of a projection is cut into nch chunks of (nearly) equal numbers of
// 256-input slices, at most 8: with nsl = q nch + rem, chunk c starts at slice
// c q + min(c, rem) (the first rem chunks have q + 1 slices).
__host__ __device__ __forceinline__ int chunk_slice0(int ch, int q, int rem) { return ch * q + min(ch, rem); }

struct GemvItem {
    CUtensorMap codes;           // 3D: box of zbig slices; 2D: box 128 B x 16 RG rows; 128-byte swizzle
    CUtensorMap codes_small;     // 3D only: box of zbig - 1 slices (chunks one slice shorter)
    const int8_t *scale8;
    const float *scale2;
    const float *offset;
    const __nv_bfloat16 *X;      // [M, K]
    float *partial;              // [nch][N][M] K-chunk sums
    int N, K, kbs, nch, nrb;     // rows, inputs, 64-blocks per row, K chunks, row blocks
    int nsl, zbig;               // 256-input slices; slices of the longest chunk
    int sq, srem;                // nsl = sq nch + srem
    int unit0;                   // first unit of this item
    int map3d;                   // codes maps are 3D (K % 256 == 0): one box per unit
};
struct GemvGroup {
    GemvItem it[kGemvMaxItems];
    int n, M;
    int ustart[kGemvMaxGrid + 1];  // CTA c takes units ustart[c] .. ustart[c+1] - 1
};
struct FinishItem {
    const float *partial;        // [nch][N][M]
    const float *xpart;          // [nxa][M][r] X A chunk partials, or null
    const __nv_bfloat16 *B;      // [r, N], or null
    __nv_bfloat16 *Y;            // [M, N]
    __nv_bfloat16 *XA_save;      // [M, r], or null
    float s;
    int N, nch, r, nxa, cta0;
};
struct FinishGroup {
    FinishItem it[kGemvMaxItems];
    int n, M;
};

struct UnitPos {
    int item, ch, rb;
};
__device__ __forceinline__ UnitPos unit_pos(const GemvGroup &g, int u) {
    int i = 0;
    while (i + 1 < g.n && u >= g.it[i + 1].unit0) ++i;
    const int lu = u - g.it[i].unit0, nrb = g.it[i].nrb;
    const int ch = lu / nrb;
    return {i, ch, lu - ch * nrb};
}
__device__ __forceinline__ UnitPos unit_next(const GemvGroup &g, UnitPos p) {
    if (++p.rb == g.it[p.item].nrb) {
        p.rb = 0;
        if (++p.ch == g.it[p.item].nch) {
            p.ch = 0;
            ++p.item;
        }
    }
    return p;
}

// The int8 constants of one row of a unit (32 blocks), prefetched a unit ahead.
struct Q8Row {
    uint32_t w[8];               // blocks 4k .. 4k+3, little-endian
    float s2a, s2b, mu;
    int split, nblk;             // blocks < split in the first second-level group; valid blocks
};
template <int ROWS>
__device__ __forceinline__ void q8_fetch(const GemvGroup &grp, UnitPos p, int lane, Q8Row &q) {
    const GemvItem &it = grp.it[p.item];
    const int row = p.rb * ROWS + lane;
    const int sl0 = chunk_slice0(p.ch, it.sq, it.srem), sl1 = chunk_slice0(p.ch + 1, it.sq, it.srem);
    const int nblk = min(4 * (sl1 - sl0), it.kbs - 4 * sl0);
    const bool valid = lane < ROWS && row < it.N;
    const int64_t b0 = (int64_t)row * it.kbs + 4 * sl0;
    const int8_t *src = it.scale8 + b0;
#pragma unroll
    for (int k = 0; k < 8; ++k) q.w[k] = 0u;
    if (valid) {
        const uintptr_t a = reinterpret_cast<uintptr_t>(src);
        if (nblk == 32 && (a & 15u) == 0) {
            const uint4 v0 = __ldg(reinterpret_cast<const uint4 *>(src));
            const uint4 v1 = __ldg(reinterpret_cast<const uint4 *>(src) + 1);
            q.w[0] = v0.x; q.w[1] = v0.y; q.w[2] = v0.z; q.w[3] = v0.w;
            q.w[4] = v1.x; q.w[5] = v1.y; q.w[6] = v1.z; q.w[7] = v1.w;
        } else {
            const bool w4 = (a & 3u) == 0;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                if (w4 && 4 * k + 4 <= nblk) {
                    q.w[k] = __ldg(reinterpret_cast<const unsigned int *>(src) + k);
                } else {
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        if (4 * k + e < nblk) q.w[k] |= (uint32_t)(uint8_t)__ldg(src + 4 * k + e) << (8 * e);
                }
            }
        }
    }
    const int64_t g0 = b0 >> 8;
    q.split = 256 - (int)(b0 & 255);
    q.nblk = valid ? nblk : 0;
    q.s2a = valid ? __ldg(it.scale2 + g0) : 0.0f;
    q.s2b = (valid && q.split < nblk) ? __ldg(it.scale2 + g0 + 1) : q.s2a;
    q.mu = __ldg(it.offset);
}
// c^ = fl(fl(q8 * fl(s2 / 127)) + mu) of the row's 32 blocks (zero past K or N), stored
// in the row's hole with the 16-byte chunks XOR-swizzled by the row (conflict-free reads).
template <int ROWS>
__device__ __forceinline__ void chat_store(uint32_t lut_base, int stage, int lane, const Q8Row &q) {
    if (lane >= ROWS) return;
    const float st0 = __fdiv_rn(q.s2a, 127.0f);
    const float st1 = q.split < q.nblk ? __fdiv_rn(q.s2b, 127.0f) : st0;
    const uint32_t base = lut_base + hole(stage * ROWS + lane);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        float c[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int b = 4 * k + e;
            const float qv = (float)(int8_t)(q.w[k] >> (8 * e));
            c[e] = b < q.nblk ? __fadd_rn(__fmul_rn(qv, b < q.split ? st0 : st1), q.mu) : 0.0f;
        }
        sts128f(base + (uint32_t)((k ^ (lane & 7)) << 4), make_float4(c[0], c[1], c[2], c[3]));
    }
}

// X fragments of a warp's K slice for the mma B operand: xf[nt][b][2j], xf[nt][b][2j+1] hold
// X[nt * 8 + lane / 4][k0 + 64 b + 16 (lane % 4) + 4 j + 0..3], the four inputs whose codes
// are bytes 2j and 2j + 1 of the lane's 8-byte code word of block b (zero past M or K).
template <int NT>
__device__ __forceinline__ void x_load(const GemvGroup &grp, UnitPos p, int ks, int lane, uint32_t (&xf)[NT][4][8]) {
    const GemvItem &it = grp.it[p.item];
    const int g = lane >> 2, t = lane & 3;
    const int sl0 = chunk_slice0(p.ch, it.sq, it.srem), sl1 = chunk_slice0(p.ch + 1, it.sq, it.srem);
    const int k0 = (sl0 + ks) * kGemvSlice;
    const bool in_chunk = sl0 + ks < sl1;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const int tok = nt * 8 + g, kb = k0 + 64 * b;
            uint4 v0 = make_uint4(0u, 0u, 0u, 0u), v1 = v0;
            if (in_chunk && tok < grp.M && kb < it.K) {
                const uint4 *src = reinterpret_cast<const uint4 *>(it.X + (int64_t)tok * it.K + kb + 16 * t);
                v0 = __ldg(src);
                v1 = __ldg(src + 1);
            }
            xf[nt][b][0] = v0.x; xf[nt][b][1] = v0.y; xf[nt][b][2] = v0.z; xf[nt][b][3] = v0.w;
            xf[nt][b][4] = v1.x; xf[nt][b][5] = v1.y; xf[nt][b][6] = v1.z; xf[nt][b][7] = v1.w;
        }
}

// Y[tok][R] = sum over K chunks c in order of partial[c][R][tok] + sum_j (s XA)[tok][j] B[j][R]
// (fused multiply-adds in increasing j), one thread per row R and group of up to four
// tokens (tokens fastest), so that a B value serves up to four tokens. XA = its X A chunk
// partials added in chunk order, staged in shared memory (times s); the first CTA of a
// projection also saves XA as bf16. Every sum issues its loads (up to eight) before the
// adds, so a thread waits for memory about three times.
constexpr int kFinishThreads = 256;
__global__ void __launch_bounds__(kFinishThreads) k_gemv_finish(const __grid_constant__ FinishGroup grp) {
    __shared__ float sx[kGemvMaxM * 256];
    griddep_wait();                                  // the chunk sums and X A partials are complete
    int ii = 0;
    while (ii + 1 < grp.n && (int)blockIdx.x >= grp.it[ii + 1].cta0) ++ii;
    const FinishItem &it = grp.it[ii];
    const int M = grp.M, N = it.N, r = it.r;
    for (int i = threadIdx.x; i < M * r; i += blockDim.x) {
        float v = 0.0f;
        for (int c0 = 0; c0 < it.nxa; c0 += 8) {
            float pv[8];
#pragma unroll
            for (int c = 0; c < 8; ++c)
                pv[c] = c0 + c < it.nxa ? __ldcg(it.xpart + (int64_t)(c0 + c) * M * r + i) : 0.0f;
#pragma unroll
            for (int c = 0; c < 8; ++c)
                if (c0 + c < it.nxa) v += pv[c];
        }
        sx[i] = it.s * v;
        if (blockIdx.x == it.cta0 && it.XA_save) it.XA_save[i] = __float2bfloat16_rn(v);
    }
    __syncthreads();
    const int MQ = (M + 3) / 4;                      // token groups of four
    const int64_t e = (int64_t)(blockIdx.x - it.cta0) * kFinishThreads + threadIdx.x;
    if (e >= (int64_t)N * MQ) return;
    const int R = (int)(e / MQ), m0 = 4 * (int)(e - (int64_t)R * MQ);
    const int mn = M - m0 < 4 ? M - m0 : 4;
    float y[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    for (int c0 = 0; c0 < it.nch; c0 += 4) {
        float pv[4][4];
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int q = 0; q < 4; ++q)
                pv[c][q] = (c0 + c < it.nch && q < mn) ? __ldcg(it.partial + ((int64_t)(c0 + c) * N + R) * M + m0 + q)
                                                       : 0.0f;
#pragma unroll
        for (int c = 0; c < 4; ++c)
            if (c0 + c < it.nch)
#pragma unroll
                for (int q = 0; q < 4; ++q) y[q] += pv[c][q];
    }
    if (r > 0) {
        float a[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        for (int j0 = 0; j0 < r; j0 += 8) {          // r % 8 == 0: eight B loads in flight
            float bv[8];
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) bv[jj] = __bfloat162float(it.B[(int64_t)(j0 + jj) * N + R]);
#pragma unroll
            for (int jj = 0; jj < 8; ++jj)
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    if (q < mn) a[q] = fmaf(sx[(m0 + q) * r + j0 + jj], bv[jj], a[q]);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) y[q] += a[q];
    }
#pragma unroll
    for (int q = 0; q < 4; ++q)
        if (q < mn) it.Y[(int64_t)(m0 + q) * N + R] = __float2bfloat16_rn(y[q]);
}

// Compute warps of k_gemv (warp w < 8 RG): row group w / 8, K slice w % 8.
template <int NT>
__device__ __forceinline__ void gemv_compute(const GemvGroup &grp, const uint8_t *base, uint32_t full0,
                                             uint32_t empty0, uint32_t redf0, uint32_t rede0, volatile int *abort,
                                             int u_begin, int count, int warp, int lane) {
    constexpr int S = gemv_stages(NT), ROWS = gemv_rows(NT);
    constexpr int BOX = gemv_box_bytes(NT), STAGE = gemv_stage_bytes(NT);
    // shared memory is read through ordinary loads, which the compiler may interleave
    // (they are ordered after the barrier waits, whose asm clobbers memory)
    const uint8_t *lut = base;
    const uint8_t *stages = base + kLutRegion;
    auto ld32 = [&](uint32_t off) { return *reinterpret_cast<const uint32_t *>(lut + off); };
    auto ld128 = [&](uint32_t off) { return *reinterpret_cast<const float4 *>(lut + off); };
    const int rg = warp >> 3, ks = warp & 7, g = lane >> 2, t = lane & 3;
    const uint32_t lane4 = lane * 4;
    // this lane's 8-byte code words of rows rg*16 + g and + 8 in box ks: chunk (2b + t/2) ^ g
    const uint32_t box_row0 = ks * BOX + (rg * 16 + g) * 128 + (t & 1) * 8;
    const uint32_t box_row1 = box_row0 + 8 * 128;
    // two reduction buffers, used by alternate units: a warp that is ahead waits for the
    // reducer of the unit before last only
    const uint32_t red_mine = hole(gemv_red_hole0(NT) + (rg * 8 + ks) * NT * 4 + (lane >> 3)) + (lane & 7) * 16;
    constexpr uint32_t kRedBuf = gemv_red_holes(NT) * 256u;
    bool ok = true;

    uint32_t xf[NT][4][8];
    UnitPos pos = unit_pos(grp, u_begin);
    int xkey = -1, nblk = 0;
    float acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.0f;

    for (int i = 0; i < count && ok; ++i) {
        const int s = i % S, n = i / S;
        const GemvItem &it = grp.it[pos.item];
        const int key = pos.item * 4096 + pos.ch;
        if (key != xkey) {
            x_load<NT>(grp, pos, ks, lane, xf);
            xkey = key;
            const int sl0 = chunk_slice0(pos.ch, it.sq, it.srem);
            const int kslice = (sl0 + ks) * kGemvSlice;
            nblk = ks < it.sq + (pos.ch < it.srem ? 1 : 0) ? min(4, (it.K - kslice) / 64) : 0;
        }
        if (!mbar_wait(full0 + 8 * s, n & 1, abort)) { ok = false; break; }
        if (nblk > 0) {
            const float4 c0 = ld128(hole(s * ROWS + rg * 16 + g) + ((ks ^ g) << 4));
            const float4 c1 = ld128(hole(s * ROWS + rg * 16 + g + 8) + ((ks ^ g) << 4));
            const float ch0[4] = {c0.x, c0.y, c0.z, c0.w}, ch1[4] = {c1.x, c1.y, c1.z, c1.w};
            const uint8_t *sb = stages + s * STAGE;
            // one 64-block: 16 table lookups, 4 NT MMAs, the block's c^ on the partial sums
            auto block = [&](int b) {
                const uint32_t off = (uint32_t)(((2 * b + (t >> 1)) ^ g) << 4);
                const uint2 w0 = *reinterpret_cast<const uint2 *>(sb + box_row0 + off);
                const uint2 w1 = *reinterpret_cast<const uint2 *>(sb + box_row1 + off);
                float cbk[NT][4];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) cbk[nt][0] = cbk[nt][1] = cbk[nt][2] = cbk[nt][3] = 0.0f;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint32_t r0 = (j < 2) ? w0.x : w0.y;
                    const uint32_t r1 = (j < 2) ? w1.x : w1.y;
                    // byte k of the word, times 256, plus lane * 4: one permute
                    const uint32_t slo = 0x5504u | ((uint32_t)(2 * (j & 1)) << 4), shi = slo + 0x10u;
                    uint32_t a[4];
                    a[0] = ld32(prmt(r0, lane4, slo));
                    a[2] = ld32(prmt(r0, lane4, shi));
                    a[1] = ld32(prmt(r1, lane4, slo));
                    a[3] = ld32(prmt(r1, lane4, shi));
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(cbk[nt], a, xf[nt][b][2 * j], xf[nt][b][2 * j + 1]);
                }
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    acc[nt][0] = fmaf(ch0[b], cbk[nt][0], acc[nt][0]);
                    acc[nt][1] = fmaf(ch0[b], cbk[nt][1], acc[nt][1]);
                    acc[nt][2] = fmaf(ch1[b], cbk[nt][2], acc[nt][2]);
                    acc[nt][3] = fmaf(ch1[b], cbk[nt][3], acc[nt][3]);
                }
            };
            if (nblk == 4) {
#pragma unroll
                for (int b = 0; b < 4; ++b) block(b);
            } else {
#pragma unroll
                for (int b = 0; b < 4; ++b)
                    if (b < nblk) block(b);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty0 + 8 * s);

        // ---------------- the row group's eight slices: written, then summed by warp ks == i % 8
        const int rb_ = i & 1, use = i >> 1;             // reduction buffer and its use count
        if (use > 0 && !mbar_wait(rede0 + 16 * rg + 8 * rb_, (use - 1) & 1, abort)) { ok = false; break; }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            *reinterpret_cast<float4 *>(const_cast<uint8_t *>(lut) + red_mine + rb_ * kRedBuf + nt * 4 * 256) =
                make_float4(acc[nt][0], acc[nt][1], acc[nt][2], acc[nt][3]);
            acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.0f;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(redf0 + 16 * rg + 8 * rb_);
        if (ks == (i & 7)) {
            if (!mbar_wait(redf0 + 16 * rg + 8 * rb_, use & 1, abort)) { ok = false; break; }
            float sum[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                sum[nt][0] = sum[nt][1] = sum[nt][2] = sum[nt][3] = 0.0f;
#pragma unroll
                for (int k2 = 0; k2 < 8; ++k2) {
                    const float4 v =
                        ld128(hole(gemv_red_hole0(NT) + ((rg * 8 + k2) * NT + nt) * 4 + (lane >> 3)) + (lane & 7) * 16 +
                              rb_ * kRedBuf);
                    sum[nt][0] += v.x; sum[nt][1] += v.y; sum[nt][2] += v.z; sum[nt][3] += v.w;
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(rede0 + 16 * rg + 8 * rb_);
            const int M = grp.M, N = it.N;
            const int R0 = pos.rb * ROWS + rg * 16 + g;
            float *pp = it.partial + (int64_t)pos.ch * N * M;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int tok = nt * 8 + 2 * t + (q & 1), R = R0 + (q >= 2 ? 8 : 0);
                    if (tok < M && R < N) pp[(int64_t)R * M + tok] = sum[nt][q];
                }
        }
        pos = unit_next(grp, pos);
    }
}

template <int NT>
__global__ void __launch_bounds__(gemv_threads(NT), 1)
k_gemv(const __grid_constant__ GemvGroup grp, const __grid_constant__ Codebook cb) {
    constexpr int S = gemv_stages(NT), RG = gemv_rg(NT), ROWS = gemv_rows(NT);
    constexpr int BOX = gemv_box_bytes(NT), STAGE = gemv_stage_bytes(NT);
    extern __shared__ __align__(16) uint8_t smem_raw[];
    uint8_t *base = align1024(smem_raw);
    const uint32_t lut = smem_addr(base);
    const uint32_t stages = lut + kLutRegion;
    uint64_t *bars = reinterpret_cast<uint64_t *>(base + kLutRegion + S * STAGE);
    int *flags = reinterpret_cast<int *>(bars + 2 * S + 4 * RG);
    const uint32_t full0 = smem_addr(bars), empty0 = full0 + 8 * S;
    const uint32_t redf0 = full0 + 16 * S, rede0 = redf0 + 16 * RG;   // per row group and buffer
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    // lookup table: word (e * 64 + lane) = bf16 pair (Q[e >> 4] low half, Q[e & 15] high half)
    for (int i = tid; i < 256 * 8; i += blockDim.x) {
        const int e = i >> 3, q = i & 7;
        const uint32_t v = pack_bf16x2(cb.q[e >> 4], cb.q[e & 15]);
        sts128u(lut + e * 256 + q * 16, make_uint4(v, v, v, v));
    }
    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full0 + 8 * s, 33);           // producer's expect-tx arrival + 32 lanes after c^
            mbar_init(empty0 + 8 * s, 8 * RG);      // one arrival per compute warp
        }
        for (int b = 0; b < 2 * RG; ++b) {
            mbar_init(redf0 + 8 * b, 8);            // the row group's eight slices written
            mbar_init(rede0 + 8 * b, 1);            // the reducer has read them
        }
        flags[0] = 0;
        fence_barrier_init();
    }
    __syncthreads();
    volatile int *abort = flags;

    griddep_launch_dependents();
    const int u_begin = grp.ustart[blockIdx.x];
    const int count = grp.ustart[blockIdx.x + 1] - u_begin;
    if (count <= 0) return;

    if (warp >= 8 * RG) {
        // ---------------- producers: TMA of the codes, c^ of every row into the stage's holes.
        // Producer w takes units w, w + 2, ... of the CTA's range. The int8 constants of a unit
        // are fetched while its three predecessors of the same producer are produced, into a
        // ring of four register sets that the unrolled loop names statically (copying a set
        // whose loads are in flight would wait for them).
        const int pw = warp - 8 * RG;
        int last = -1;
        UnitPos p = unit_pos(grp, u_begin);
        if (pw < count) {
            for (int j = 0; j < pw; ++j) p = unit_next(grp, p);
        }
        UnitPos pf = p;
        auto advance = [&](UnitPos x) {
#pragma unroll
            for (int j = 0; j < kGemvProducers; ++j) x = unit_next(grp, x);
            return x;
        };
        Q8Row qa, qb, qc, qd;
        if (pw < count) q8_fetch<ROWS>(grp, pf, lane, qa);
        pf = advance(pf);
        if (pw + kGemvProducers < count) q8_fetch<ROWS>(grp, pf, lane, qb);
        pf = advance(pf);
        if (pw + 2 * kGemvProducers < count) q8_fetch<ROWS>(grp, pf, lane, qc);
        pf = advance(pf);
        // produce unit i from `cur`; fetch unit i + 3 producer strides on into `nxt`
        auto step = [&](int i, const Q8Row &cur, Q8Row &nxt) -> bool {
            if (i >= count) return false;
            if (i + 3 * kGemvProducers < count) q8_fetch<ROWS>(grp, pf, lane, nxt);
            pf = advance(pf);
            const int s = i % S, n = i / S;
            if (!mbar_wait(empty0 + 8 * s, (n & 1) ^ 1, abort)) return false;
            const GemvItem &it = grp.it[p.item];
            if (lane == 0) {
                const int sl0 = chunk_slice0(p.ch, it.sq, it.srem);
                const int nsl = it.sq + (p.ch < it.srem ? 1 : 0);
                if (it.map3d) {
                    mbar_arrive_expect_tx(full0 + 8 * s, nsl * BOX);
                    tma_load_3d(stages + s * STAGE, nsl == it.zbig ? &it.codes : &it.codes_small, full0 + 8 * s, 0,
                                p.rb * ROWS, sl0);
                } else {
                    mbar_arrive_expect_tx(full0 + 8 * s, nsl * BOX);
                    for (int b = 0; b < nsl; ++b)
                        tma_load_2d(stages + s * STAGE + b * BOX, &it.codes, full0 + 8 * s, (sl0 + b) * 128,
                                    p.rb * ROWS);
                }
            }
            chat_store<ROWS>(lut, s, lane, cur);
            mbar_arrive(full0 + 8 * s);
            last = i;
            p = advance(p);
            return true;
        };
        constexpr int P = kGemvProducers;
        for (int i = pw; i < count; i += 4 * P) {
            if (!step(i, qa, qd)) break;
            if (!step(i + P, qb, qa)) break;
            if (!step(i + 2 * P, qc, qb)) break;
            if (!step(i + 3 * P, qd, qc)) break;
        }
        if (lane == 0) flags[1 + pw] = last;           // the last unit this producer issued
    } else {
        gemv_compute<NT>(grp, base, full0, empty0, redf0, rede0, abort, u_begin, count, warp, lane);
    }
    // The CTA does not exit with a copy in flight: once every role is done, wait for the last
    // unit issued on each stage (no later unit reuses a stage, so its phase is the stage's last).
    __syncthreads();
    if (tid == 0) {
        const uint64_t t0 = global_timer_ns();
        for (int s = 0; s < S; ++s) {
            int u = -1;
            for (int pw = 0; pw < kGemvProducers; ++pw) {
                const int lastp = flags[1 + pw];
                for (int i = lastp; i >= 0 && i > lastp - S * kGemvProducers; i -= kGemvProducers)
                    if (i % S == s) { u = max(u, i); break; }
            }
            if (u < 0) continue;
            while (!mbar_try_wait(full0 + 8 * s, (u / S) & 1))
                if (global_timer_ns() - t0 > kWaitLimitNs) {
                    raise_status(QLORA_ERR_TIMEOUT);
                    return;
                }
        }
    }
}

// ---------------------------------------------------------------- host side
static int rows_for(int64_t M) { return M <= 8 ? gemv_rows(1) : gemv_rows(2); }

// Workspace of one launch group: fp32 K-chunk sums [nch][N][M] per projection and
// X A chunk partials [K/128][M][r] per adapter, each region 256-byte aligned.
static size_t group_workspace(int64_t M, int count, const LinearDesc *d) {
    size_t b = 0;
    for (int i = 0; i < count; ++i) {
        b += align256((size_t)ceil_div(ceil_div(d[i].W.cols, kGemvSlice), kGemvMaxSlices) * d[i].W.rows * M * 4);
        if (d[i].r > 0) b += align256((size_t)ceil_div(d[i].W.cols, kXaChunk) * M * d[i].r * 4);
    }
    return b;
}

size_t fwd_workspace_bytes_large(int64_t M, int64_t rows, int64_t cols, int r);

size_t fwd_workspace_bytes(int64_t M, int64_t rows, int64_t cols, int r) {
    if (M <= kGemvMaxM) {
        LinearDesc d{};
        d.W.rows = rows;
        d.W.cols = cols;
        d.r = r;
        return group_workspace(M, 1, &d);
    }
    return fwd_workspace_bytes_large(M, rows, cols, r);
}

size_t fwd_grouped_workspace_bytes(int64_t M, int count, const LinearDesc *d) {
    size_t b = 0;
    for (int i = 0; i < count; i += (M <= kGemvMaxM ? kGemvMaxItems : 1)) {
        const int n = M <= kGemvMaxM ? (count - i < kGemvMaxItems ? count - i : kGemvMaxItems) : 1;
        const size_t x = M <= kGemvMaxM ? group_workspace(M, n, d + i)
                                        : fwd_workspace_bytes_large(M, d[i].W.rows, d[i].W.cols, d[i].r);
        if (x > b) b = x;
    }
    return b;
}

// Small-M forward of count <= kGemvMaxItems projections: the X A pre-pass, the GEMV, the finish.
static cudaError_t gemv_group(int64_t M, int count, const LinearDesc *d, void *ws, cudaStream_t st) {
    GemvGroup grp;
    XaGroup xg;
    FinishGroup fg;
    const int rows = rows_for(M);
    grp.n = fg.n = count;
    grp.M = xg.M = fg.M = (int)M;
    xg.n = 0;
    char *wsp = static_cast<char *>(ws);
    int u0 = 0, fc = 0;
    int64_t total = 0;
    for (int i = 0; i < count; ++i) {
        GemvItem &it = grp.it[i];
        FinishItem &fi = fg.it[i];
        const NF4View &w = d[i].W;
        it.nsl = (int)ceil_div(w.cols, kGemvSlice);
        it.nch = (int)ceil_div(it.nsl, kGemvMaxSlices);
        it.zbig = (int)ceil_div(it.nsl, it.nch);
        it.sq = it.nsl / it.nch;
        it.srem = it.nsl % it.nch;
        // rows of whole 128-byte slices: one 3D box (slice x row x byte) per unit, of the
        // chunk's slice count (two maps: chunks differ by at most one slice); else 2D boxes
        it.map3d = (w.cols % 256 == 0) ? 1 : 0;
        if (it.map3d) {
            const uint64_t dims[3] = {128, (uint64_t)w.rows, (uint64_t)w.cols / 256};
            const uint64_t strides[2] = {(uint64_t)w.cols / 2, 128};
            const uint32_t box[3] = {128, (uint32_t)rows, (uint32_t)it.zbig};
            const uint32_t box_small[3] = {128, (uint32_t)rows, (uint32_t)(it.zbig > 1 ? it.zbig - 1 : 1)};
            if (!make_map_3d(&it.codes, w.codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, dims, strides, box,
                             CU_TENSOR_MAP_SWIZZLE_128B) ||
                !make_map_3d(&it.codes_small, w.codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, dims, strides, box_small,
                             CU_TENSOR_MAP_SWIZZLE_128B))
                return cudaErrorInvalidValue;
        } else if (!make_map(&it.codes, w.codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, (uint64_t)w.cols / 2,
                             (uint64_t)w.rows, (uint64_t)w.cols / 2, 128, (uint32_t)rows, CU_TENSOR_MAP_SWIZZLE_128B)) {
            return cudaErrorInvalidValue;
        }
        it.scale8 = w.scale8;
        it.scale2 = w.scale2;
        it.offset = w.offset;
        it.X = d[i].X;
        it.N = (int)w.rows;
        it.K = (int)w.cols;
        it.kbs = (int)(w.cols / 64);
        it.nrb = (int)ceil_div(w.rows, rows);
        it.unit0 = u0;
        it.partial = reinterpret_cast<float *>(wsp);
        wsp += align256((size_t)it.nch * w.rows * M * 4);
        u0 += it.nch * it.nrb;
        total += (int64_t)w.rows * w.cols;
        fi.partial = it.partial;
        fi.B = d[i].B;
        fi.Y = d[i].Y;
        fi.N = it.N;
        fi.nch = it.nch;
        fi.r = d[i].r > 0 ? d[i].r : 0;
        fi.s = d[i].s;
        fi.xpart = nullptr;
        fi.XA_save = d[i].r > 0 ? d[i].XA_save : nullptr;
        fi.nxa = 0;
        fi.cta0 = fc;
        fc += (int)ceil_div(w.rows * ceil_div(M, (int64_t)4), (int64_t)kFinishThreads);
    }
    int xc = 0;
    for (int i = 0; i < count; ++i) {
        if (d[i].r <= 0) continue;
        XaItem &xi = xg.it[xg.n++];
        const int nxa = (int)ceil_div(d[i].W.cols, kXaChunk);
        xi.X = d[i].X;
        xi.A = d[i].A;
        xi.K = (int)d[i].W.cols;
        xi.r = d[i].r;
        xi.cta0 = xc;
        xi.xpart = reinterpret_cast<float *>(wsp);
        wsp += align256((size_t)nxa * M * d[i].r * 4);
        xc += nxa;
        fg.it[i].xpart = xi.xpart;
        fg.it[i].nxa = nxa;
    }
    // contiguous unit ranges of (nearly) equal weight count, one per CTA
    const int units = u0;
    int grid = num_sms();
    if (grid > kGemvMaxGrid) grid = kGemvMaxGrid;
    if (grid > units) grid = units;
    {
        int c = 0;
        int64_t acc = 0;
        grp.ustart[0] = 0;
        for (int i = 0; i < count; ++i) {
            const GemvItem &it = grp.it[i];
            for (int ch = 0; ch < it.nch; ++ch) {
                const int64_t sl0 = chunk_slice0(ch, it.sq, it.srem), sl1 = chunk_slice0(ch + 1, it.sq, it.srem);
                const int64_t kin = std::min<int64_t>(sl1 * kGemvSlice, it.K) - sl0 * kGemvSlice;
                for (int rb = 0; rb < it.nrb; ++rb) {
                    const int64_t nr = std::min<int64_t>(rows, it.N - (int64_t)rb * rows);
                    acc += nr * kin;
                    const int u = it.unit0 + ch * it.nrb + rb;
                    // CTA c ends after the unit that brings the running sum to c+1 shares
                    while (c < grid - 1 && acc * grid >= (int64_t)(c + 1) * total) grp.ustart[++c] = u + 1;
                }
            }
        }
        while (c < grid) grp.ustart[++c] = units;
    }
    cudaError_t e;
    if (M <= 8) {
        if ((e = set_smem(k_gemv<1>, gemv_smem(1))) != cudaSuccess) return e;
        QNF4_LAUNCH("k_gemv", st,
                    e = launch_pdl(k_gemv<1>, grid, gemv_threads(1), gemv_smem(1), st, false, grp, host_codebook()));
    } else {
        if ((e = set_smem(k_gemv<2>, gemv_smem(2))) != cudaSuccess) return e;
        QNF4_LAUNCH("k_gemv", st,
                    e = launch_pdl(k_gemv<2>, grid, gemv_threads(2), gemv_smem(2), st, false, grp, host_codebook()));
    }
    if (e != cudaSuccess) return e;
    if (xc > 0) {
        QNF4_LAUNCH("k_gemv_xa", st, e = launch_pdl(k_gemv_xa, xc, 32, 0, st, true, xg));
        if (e != cudaSuccess) return e;
    }
    QNF4_LAUNCH("k_gemv_finish", st, e = launch_pdl(k_gemv_finish, fc, kFinishThreads, 0, st, true, fg));
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t launch_linear_fwd_grouped(int64_t M, int count, const LinearDesc *d, void *ws, cudaStream_t st) {
    if (M > kGemvMaxM) {
        for (int i = 0; i < count; ++i) {
            cudaError_t e = launch_linear_fwd_large(d[i].X, M, d[i].W, d[i].A, d[i].B, d[i].r, d[i].s, d[i].Y,
                                                    d[i].XA_save, ws, st);
            if (e != cudaSuccess) return e;
        }
        return cudaSuccess;
    }
    // groups of at most kGemvMaxItems projections, one after the other in the same workspace
    for (int i = 0; i < count; i += kGemvMaxItems) {
        const int n = count - i < kGemvMaxItems ? count - i : kGemvMaxItems;
        cudaError_t e = gemv_group(M, n, d + i, ws, st);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

cudaError_t launch_linear_fwd(const __nv_bfloat16 *X, int64_t M, const NF4View &W, const __nv_bfloat16 *A,
                              const __nv_bfloat16 *B, int r, float s, __nv_bfloat16 *Y, __nv_bfloat16 *XA_save,
                              void *ws, cudaStream_t st) {
    if (M > kGemvMaxM) return launch_linear_fwd_large(X, M, W, A, B, r, s, Y, XA_save, ws, st);
    LinearDesc d;
    d.X = X;
    d.W = W;
    d.A = A;
    d.B = B;
    d.r = r;
    d.s = s;
    d.Y = Y;
    d.XA_save = XA_save;
    return launch_linear_fwd_grouped(M, 1, &d, ws, st);
}

}  // namespace qnf4
