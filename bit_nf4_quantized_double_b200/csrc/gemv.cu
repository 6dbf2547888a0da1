// Small-M (M <= 16 tokens) forward: a streaming NF4 GEMV on the warp-level
// tensor-core path, and the dispatch between it and the tcgen05 GEMMs.
//
// Layer: Y = X W^ + s (X A) B (page "QLoRA: put the large model in memory,
// then change it with a small adapter", wq-win.github.io/llm/074-qlora,
// section 1), at decode-sized M where the packed 4-bit codes dominate HBM
// traffic (section 2: about 4.127 bits per weight).
//
// Three launches, the last two chained by programmatic dependent launch so that
// they start while their predecessor still runs:
//   k_gemv_xa    per (projection, 512-input chunk): XA partial sums [M, r];
//   k_gemv_lora  per (projection, 256 outputs): XA = sum of the partials in chunk
//                order, L = (s XA) B in fp32; also clears the main kernel's
//                row-block counters;
//   k_gemv       persistent, one CTA per SM over work units of 128 weight rows x
//                512 inputs, ordered (projection, row block, K chunk) and cut into
//                equal contiguous ranges, one per CTA.
// In k_gemv, one producer warp per pipeline stage loads the unit's packed codes
// with TMA (two 128-byte-swizzled boxes of 128 rows x 128 bytes) and computes the
// unit's dequantised block constants c^ (double quantisation, section 3) into the
// stage. Sixteen compute warps (8 row groups of 16 x 2 halves of the K chunk)
// turn each code byte into a bf16 pair (Q[hi], Q[lo]) with one byte permute
// (address = byte * 256 + lane * 4) and one load from a per-lane replicated table,
// accumulate sum_k Q[code] x_k per 64-block with mma.sync m16n8k16 (16 weight rows
// x 8 tokens) and scale each block's partial dot product by its c^. A row block
// ends in the CTA that holds its last K chunk: (half 0 + half 1) + L rounded to
// bf16; a row block cut between two or more CTAs is combined by whichever CTA
// finishes last, adding the parts in CTA order (reproducible).
#include "launch.h"
#include "tc.cuh"
#include "tmap.h"

namespace qnf4 {

using namespace tc;

cudaError_t launch_linear_fwd_large(const __nv_bfloat16 *X, int64_t M, const NF4View &W, const __nv_bfloat16 *A,
                                    const __nv_bfloat16 *B, int r, float s, __nv_bfloat16 *Y,
                                    __nv_bfloat16 *XA_save, void *ws, cudaStream_t st);

constexpr int kGemvMaxM = 16;
constexpr int kGemvRows = 128;                  // weight rows per unit (8 row groups of 16)
constexpr int kGemvKChunk = 512;                // inputs per unit (8 blocks of 64)
constexpr int kGemvCompute = 512;               // compute threads (16 warps)
constexpr int kGemvMaxItems = 8;
constexpr int kLutBytes = 256 * 256;            // 256 code bytes x 64 words (32 used: one per lane)
constexpr int kBoxBytes = kGemvRows * 128;      // one TMA box: 128 rows x 128 code bytes
constexpr int kChatBytes = kGemvRows * 8 * 4;   // c^ of 128 rows x 8 blocks
constexpr int kStageBytes = 2 * kBoxBytes + kChatBytes;
constexpr int kXaChunk = 512;                   // inputs per k_gemv_xa CTA
constexpr int kLoraCols = 256;                  // outputs per k_gemv_lora CTA

__host__ __device__ constexpr int gemv_stages(int nt) { return nt == 1 ? 4 : 3; }
__host__ __device__ constexpr int gemv_threads(int nt) { return kGemvCompute + 32 * gemv_stages(nt); }
__host__ __device__ constexpr int gemv_xs_bytes(int nt) { return nt * 8 * 4 * 32 * 8; }   // one X buffer
__host__ __device__ constexpr int gemv_smem(int nt) {
    return kLutBytes + 1024 + gemv_stages(nt) * kStageBytes + 2 * gemv_xs_bytes(nt) + 128;
}

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint2 ldg_nc_v2(const void *p) {
    uint2 r;
    asm volatile("ld.global.nc.v2.u32 {%0,%1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(p));
    return r;
}

__device__ __forceinline__ uint32_t pack2_bf16(const __nv_bfloat16 *p0, const __nv_bfloat16 *p1) {
    const uint32_t lo = *reinterpret_cast<const uint16_t *>(p0), hi = *reinterpret_cast<const uint16_t *>(p1);
    return lo | (hi << 16);
}

__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;"); }

// ---------------------------------------------------------------- adapter kernels
struct LoraItem {
    const __nv_bfloat16 *X;      // [M, K]
    const __nv_bfloat16 *A;      // [K, r]
    const __nv_bfloat16 *B;      // [r, N]
    __nv_bfloat16 *XA_save;      // [M, r] or null
    float *part;                 // [nchunks][M][r]
    float *L;                    // [M][N]
    float s;
    int K, N, r, nchunks;
    int cta_xa, cta_lora;        // first CTA of this item in either kernel
};
struct LoraGroup {
    LoraItem it[kGemvMaxItems];
    int n, M;
    int *counters;
    int ncounters;
};

// XA partial of one 512-input chunk: part[c][m][j] = sum over the chunk of X[m][k] A[k][j].
// mma m16n8k16 with X rows (tokens, zero past M) as A and A_lora columns as B; warp w
// takes the chunk's 16-wide k steps w, w + 8, ...; the eight warps' sums are added in
// warp order through shared memory.
__global__ void __launch_bounds__(256) k_gemv_xa(const __grid_constant__ LoraGroup grp) {
    __shared__ float4 red[8 * 4 * 32];
    griddep_launch_dependents();
    int ii = 0;
    while (ii + 1 < grp.n && (int)blockIdx.x >= grp.it[ii + 1].cta_xa) ++ii;
    const LoraItem &it = grp.it[ii];
    const int M = grp.M, K = it.K, r = it.r;
    const int c = blockIdx.x - it.cta_xa;
    const int kbase = c * kXaChunk;
    const int ksteps = (min(K, kbase + kXaChunk) - kbase) / 16;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const int ntiles = r / 8;
    float *dst = it.part + (int64_t)c * M * r;
    for (int nt0 = 0; nt0 < ntiles; nt0 += 4) {
        const int nts = min(4, ntiles - nt0);
        float acc[4][4];
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[q][0] = acc[q][1] = acc[q][2] = acc[q][3] = 0.0f;
#pragma unroll
        for (int st = 0; st < kXaChunk / 16 / 8; ++st) {
            const int kstep = warp + 8 * st;
            if (kstep >= ksteps) break;
            const int k0 = kbase + 16 * kstep;
            uint32_t a[4] = {0u, 0u, 0u, 0u};
            if (g < M) {
                a[0] = *reinterpret_cast<const uint32_t *>(it.X + (int64_t)g * K + k0 + 2 * t);
                a[2] = *reinterpret_cast<const uint32_t *>(it.X + (int64_t)g * K + k0 + 8 + 2 * t);
            }
            if (g + 8 < M) {
                a[1] = *reinterpret_cast<const uint32_t *>(it.X + (int64_t)(g + 8) * K + k0 + 2 * t);
                a[3] = *reinterpret_cast<const uint32_t *>(it.X + (int64_t)(g + 8) * K + k0 + 8 + 2 * t);
            }
            uint32_t bb[4][2];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
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
#pragma unroll
        for (int q = 0; q < 4; ++q)
            if (q < nts) red[(warp * 4 + q) * 32 + lane] = make_float4(acc[q][0], acc[q][1], acc[q][2], acc[q][3]);
        __syncthreads();
        // c[0], c[1]: token g, tile columns 2t, 2t+1; c[2], c[3]: token g + 8
        for (int i = threadIdx.x; i < nts * 32; i += blockDim.x) {
            const int q = i >> 5, ln = i & 31;
            float4 v = red[q * 32 + ln];
            for (int ww = 1; ww < 8; ++ww) {
                const float4 x = red[(ww * 4 + q) * 32 + ln];
                v.x += x.x; v.y += x.y; v.z += x.z; v.w += x.w;
            }
            const int gg = ln >> 2, tt = ln & 3, j0 = (nt0 + q) * 8 + 2 * tt;
            if (gg < M) { dst[gg * r + j0] = v.x; dst[gg * r + j0 + 1] = v.y; }
            if (gg + 8 < M) { dst[(gg + 8) * r + j0] = v.z; dst[(gg + 8) * r + j0 + 1] = v.w; }
        }
        __syncthreads();
    }
}

// XA = sum of the chunk partials (chunk order), saved as bf16; L[m][n] = sum_j (s XA[m][j]) B[j][n]
// (fused multiply-adds in increasing j). CTA 0 also clears the main kernel's counters.
__global__ void __launch_bounds__(256) k_gemv_lora(const __grid_constant__ LoraGroup grp) {
    __shared__ float sx[kGemvMaxM * 256];          // s XA, r <= 256
    griddep_launch_dependents();
    if (blockIdx.x == 0)
        for (int i = threadIdx.x; i < grp.ncounters; i += blockDim.x) grp.counters[i] = 0;
    if (grp.n == 0) return;
    griddep_wait();                                  // the XA partials are complete
    int ii = 0;
    while (ii + 1 < grp.n && (int)blockIdx.x >= grp.it[ii + 1].cta_lora) ++ii;
    const LoraItem &it = grp.it[ii];
    const int M = grp.M, r = it.r, N = it.N;
    const int slice = blockIdx.x - it.cta_lora;
    for (int i = threadIdx.x; i < M * r; i += blockDim.x) {
        float v = 0.0f;
        for (int c0 = 0; c0 < it.nchunks; c0 += 8) {         // eight partial loads in flight
            float pv[8];
#pragma unroll
            for (int c = 0; c < 8; ++c)
                pv[c] = c0 + c < it.nchunks ? __ldcg(it.part + (int64_t)(c0 + c) * M * r + i) : 0.0f;
#pragma unroll
            for (int c = 0; c < 8; ++c)
                if (c0 + c < it.nchunks) v += pv[c];
        }
        sx[i] = it.s * v;
        if (slice == 0 && it.XA_save) it.XA_save[i] = __float2bfloat16_rn(v);
    }
    __syncthreads();
    const int n = slice * kLoraCols + threadIdx.x;
    if (n >= N) return;
    float acc[kGemvMaxM];
#pragma unroll
    for (int m = 0; m < kGemvMaxM; ++m) acc[m] = 0.0f;
    for (int j0 = 0; j0 < r; j0 += 8) {             // r % 8 == 0: eight B loads in flight
        float b[8];
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) b[jj] = __bfloat162float(it.B[(int64_t)(j0 + jj) * N + n]);
#pragma unroll
        for (int jj = 0; jj < 8; ++jj)
#pragma unroll
            for (int m = 0; m < kGemvMaxM; ++m)
                if (m < M) acc[m] = fmaf(sx[m * r + j0 + jj], b[jj], acc[m]);
    }
#pragma unroll
    for (int m = 0; m < kGemvMaxM; ++m)
        if (m < M) it.L[(int64_t)m * N + n] = acc[m];
}

// ---------------------------------------------------------------- main kernel
struct GemvItem {
    CUtensorMap codes;           // codes as bytes [N][K/2], box 128 B x 128 rows, 128-byte swizzle
    const int8_t *scale8;
    const float *scale2;
    const float *offset;
    const __nv_bfloat16 *X;      // [M, K]
    __nv_bfloat16 *Y;            // [M, N]
    const float *L;              // [M, N] adapter term, or null
    int N, K, kbs, nks, nrb;     // rows, inputs, 64-blocks per row, K chunks, row blocks
    int unit0;                   // first unit of this item
    int rb0;                     // first counter of this item
};
struct GemvGroup {
    GemvItem it[kGemvMaxItems];
    int n, M;
    int units, per_cta;          // total units; contiguous units per CTA
    int *counters;               // one per row block, zero on entry (k_gemv_lora)
    float *partial;              // [grid][2 slots][128 rows][M]
};

struct UnitPos {
    int item, rb, ks;
};
__device__ __forceinline__ UnitPos unit_pos(const GemvGroup &g, int u) {
    int i = 0;
    while (i + 1 < g.n && u >= g.it[i + 1].unit0) ++i;
    const int lu = u - g.it[i].unit0, nks = g.it[i].nks;
    const int rb = lu / nks;
    return {i, rb, lu - rb * nks};
}
__device__ __forceinline__ UnitPos unit_next(const GemvGroup &g, UnitPos p) {
    if (++p.ks == g.it[p.item].nks) {
        p.ks = 0;
        if (++p.rb == g.it[p.item].nrb) {
            p.rb = 0;
            ++p.item;
        }
    }
    return p;
}

// Stage producer: TMA of the unit's codes and the unit's c^ (128 rows x 8 blocks;
// lane l takes rows l, l + 32, l + 64, l + 96). Every load is issued before any
// arithmetic. c^ = fl(fl(q8 * fl(s2 / 127)) + mu), zero for rows past N and blocks past K.
__device__ __forceinline__ void gemv_produce(const GemvGroup &grp, const UnitPos p, uint32_t stage, float *chat,
                                             uint32_t full_bar, int lane) {
    const GemvItem &it = grp.it[p.item];
    if (lane == 0) {
        mbar_arrive_expect_tx(full_bar, 2 * kBoxBytes);
        tma_load_2d(stage, &it.codes, full_bar, p.ks * 256, p.rb * kGemvRows);
        tma_load_2d(stage + kBoxBytes, &it.codes, full_bar, p.ks * 256 + 128, p.rb * kGemvRows);
    }
    const int nblk = min(8, it.K / 64 - p.ks * 8);
    const float mu = __ldg(it.offset);
    uint32_t qw[4][2];           // the row's eight int8 constants, little-endian
    float s2a[4], s2b[4];
    int split[4];                // blocks b < split[i] are in the first second-level group
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int row = p.rb * kGemvRows + lane + 32 * i;
        const bool valid = row < it.N;
        const int64_t b0 = (int64_t)row * it.kbs + p.ks * 8;
        const int8_t *q8 = it.scale8 + b0;
        qw[i][0] = qw[i][1] = 0u;
        if (valid) {
            if (nblk == 8 && (reinterpret_cast<uintptr_t>(q8) & 3u) == 0) {
                qw[i][0] = __ldg(reinterpret_cast<const unsigned int *>(q8));
                qw[i][1] = __ldg(reinterpret_cast<const unsigned int *>(q8) + 1);
            } else {
#pragma unroll
                for (int b = 0; b < 8; ++b)
                    if (b < nblk) qw[i][b >> 2] |= (uint32_t)(uint8_t)__ldg(q8 + b) << (8 * (b & 3));
            }
        }
        const int64_t g0 = b0 >> 8;
        split[i] = 256 - (int)(b0 & 255);
        s2a[i] = valid ? __ldg(it.scale2 + g0) : 0.0f;
        s2b[i] = (valid && split[i] < nblk) ? __ldg(it.scale2 + g0 + 1) : s2a[i];
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float st0 = __fdiv_rn(s2a[i], 127.0f);
        const float st1 = split[i] < nblk ? __fdiv_rn(s2b[i], 127.0f) : st0;
        float c[8];
#pragma unroll
        for (int b = 0; b < 8; ++b) {
            const float q = (float)(int8_t)(qw[i][b >> 2] >> (8 * (b & 3)));
            c[b] = (b < nblk) ? __fadd_rn(__fmul_rn(q, b < split[i] ? st0 : st1), mu) : 0.0f;
        }
        if (p.rb * kGemvRows + lane + 32 * i >= it.N)
#pragma unroll
            for (int b = 0; b < 8; ++b) c[b] = 0.0f;
        float4 *dst = reinterpret_cast<float4 *>(chat + (lane + 32 * i) * 8);
        dst[0] = make_float4(c[0], c[1], c[2], c[3]);
        dst[1] = make_float4(c[4], c[5], c[6], c[7]);
    }
}

// X fragments of one unit for the mma B operand: entry ((nt * 8 + b) * 4 + j) * 32 + lane
// holds X[nt * 8 + lane / 4][kbase + 64 b + 16 (lane % 4) + 4 j + 0..3], the four inputs whose
// codes are bytes 2j and 2j + 1 of that lane's 8-byte code word of block b (zero past M or K).
template <int NT>
__device__ __forceinline__ void x_fetch(const GemvGroup &grp, UnitPos p, int ctid, uint2 (&v)[2 * NT]) {
    const GemvItem &it = grp.it[p.item];
    const int kbase = p.ks * kGemvKChunk;
#pragma unroll
    for (int q = 0; q < 2 * NT; ++q) {
        const int e = ctid + kGemvCompute * q;
        const int nt = e >> 10, b = (e >> 7) & 7, j = (e >> 5) & 3, ln = e & 31;
        const int tok = nt * 8 + (ln >> 2);
        const int k = kbase + b * 64 + 16 * (ln & 3) + 4 * j;
        v[q] = (tok < grp.M && k < it.K) ? ldg_nc_v2(it.X + (int64_t)tok * it.K + k) : make_uint2(0u, 0u);
    }
}
template <int NT>
__device__ __forceinline__ void x_store(uint2 *xs, int ctid, const uint2 (&v)[2 * NT]) {
#pragma unroll
    for (int q = 0; q < 2 * NT; ++q) xs[ctid + kGemvCompute * q] = v[q];
}

template <int NT>
__global__ void __launch_bounds__(gemv_threads(NT), 1)
k_gemv(const __grid_constant__ GemvGroup grp, const __grid_constant__ Codebook cb) {
    constexpr int S = gemv_stages(NT);
    extern __shared__ __align__(16) uint8_t smem_raw[];
    uint32_t *lut = reinterpret_cast<uint32_t *>(smem_raw);
    uint8_t *stages = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + kLutBytes + 1023) & ~uintptr_t(1023));
    uint2 *xs = reinterpret_cast<uint2 *>(stages + S * kStageBytes);          // [2][NT][8][4][32]
    uint64_t *bars = reinterpret_cast<uint64_t *>(stages + S * kStageBytes + 2 * gemv_xs_bytes(NT));
    int *flags = reinterpret_cast<int *>(bars + 2 * S);                       // abort, last
    const uint32_t full0 = smem_addr(bars), empty0 = smem_addr(bars + S);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    // lookup table: word (e * 64 + lane) = bf16 pair (Q[e >> 4] low half, Q[e & 15] high half)
    for (int i = tid; i < 256 * 32; i += blockDim.x) {
        const int e = i >> 5;
        lut[e * 64 + (i & 31)] = pack_bf16x2(cb.q[e >> 4], cb.q[e & 15]);
    }
    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full0 + 8 * s, 33);           // producer's expect-tx arrival + 32 lanes after c^
            mbar_init(empty0 + 8 * s, 16);          // one arrival per compute warp
        }
        flags[0] = 0;
        fence_barrier_init();
    }
    __syncthreads();
    volatile int *abort = flags;

    const int u_begin = blockIdx.x * grp.per_cta;
    const int count = min(grp.units, u_begin + grp.per_cta) - u_begin;
    if (count <= 0) return;

    if (warp >= 16) {
        // ---------------- producer of stage s: units s, s + S, ... of this CTA's range
        const int s = warp - 16;
        const uint32_t st_addr = smem_addr(stages + s * kStageBytes);
        float *chat = reinterpret_cast<float *>(stages + s * kStageBytes + 2 * kBoxBytes);
        int last = -1;
        for (int i = s, n = 0; i < count; i += S, ++n) {
            if (!mbar_wait(empty0 + 8 * s, (n & 1) ^ 1, abort)) break;
            gemv_produce(grp, unit_pos(grp, u_begin + i), st_addr, chat, full0 + 8 * s, lane);
            mbar_arrive(full0 + 8 * s);
            last = n;
        }
        // the CTA does not exit with this stage's copy in flight
        if (last >= 0 && lane == 0) {
            const uint64_t t0 = global_timer_ns();
            while (!mbar_try_wait(full0 + 8 * s, last & 1))
                if (global_timer_ns() - t0 > kWaitLimitNs) {
                    raise_status(QLORA_ERR_TIMEOUT);
                    break;
                }
        }
        return;
    }

    // ---------------- compute warps
    const int h = warp >> 3, wr = warp & 7, g = lane >> 2, t = lane & 3;
    const int Rl0 = wr * 16 + g;                                    // rows Rl0 and Rl0 + 8 of the unit
    const uint32_t lane4 = lane * 4;
    const uint32_t xg = (uint32_t)((t >> 1) ^ g) << 4, tb = (t & 1) * 8;
    const char *lut_b = reinterpret_cast<const char *>(lut);
    bool ok = true, dep_done = false;

    UnitPos pos = unit_pos(grp, u_begin);
    {
        uint2 v[2 * NT];
        x_fetch<NT>(grp, pos, tid, v);
        x_store<NT>(xs, tid, v);
    }
    named_bar_sync(1, kGemvCompute);

    float acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.0f;

    for (int i = 0; i < count; ++i) {
        const int s = i % S, n = i / S, cur = i & 1;
        const bool has_next = i + 1 < count;
        const UnitPos nxt = unit_next(grp, pos);
        uint2 xv[2 * NT];
        if (has_next) x_fetch<NT>(grp, nxt, tid, xv);

        const GemvItem &it = grp.it[pos.item];
        const int nblk = min(8, it.K / 64 - pos.ks * 8);
        uint2 cw[4][2];
        float4 c0 = make_float4(0.f, 0.f, 0.f, 0.f), c1 = c0;
        ok = ok && mbar_wait(full0 + 8 * s, n & 1, abort);
        if (ok) {
            const uint8_t *box = stages + s * kStageBytes + h * kBoxBytes;
#pragma unroll
            for (int bb = 0; bb < 4; ++bb) {
                const uint32_t off = (((uint32_t)bb << 5) ^ xg) + tb;
                cw[bb][0] = *reinterpret_cast<const uint2 *>(box + Rl0 * 128 + off);
                cw[bb][1] = *reinterpret_cast<const uint2 *>(box + (Rl0 + 8) * 128 + off);
            }
            const float *chat = reinterpret_cast<const float *>(stages + s * kStageBytes + 2 * kBoxBytes);
            c0 = *reinterpret_cast<const float4 *>(chat + Rl0 * 8 + 4 * h);
            c1 = *reinterpret_cast<const float4 *>(chat + (Rl0 + 8) * 8 + 4 * h);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty0 + 8 * s);

        if (ok) {
            const uint2 *xc = xs + cur * (NT * 1024);
            const float ch0[4] = {c0.x, c0.y, c0.z, c0.w}, ch1[4] = {c1.x, c1.y, c1.z, c1.w};
#pragma unroll
            for (int bb = 0; bb < 4; ++bb) {
                const int b = 4 * h + bb;
                if (b >= nblk) break;
                float cb[NT][4];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) cb[nt][0] = cb[nt][1] = cb[nt][2] = cb[nt][3] = 0.0f;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint32_t w0 = (j < 2) ? cw[bb][0].x : cw[bb][0].y;
                    const uint32_t w1 = (j < 2) ? cw[bb][1].x : cw[bb][1].y;
                    // byte k of w, times 256, plus lane * 4: one permute
                    const uint32_t slo = 0x5504u | ((uint32_t)(2 * (j & 1)) << 4), shi = slo + 0x10u;
                    uint32_t a[4];
                    a[0] = *reinterpret_cast<const uint32_t *>(lut_b + __byte_perm(w0, lane4, slo));
                    a[2] = *reinterpret_cast<const uint32_t *>(lut_b + __byte_perm(w0, lane4, shi));
                    a[1] = *reinterpret_cast<const uint32_t *>(lut_b + __byte_perm(w1, lane4, slo));
                    a[3] = *reinterpret_cast<const uint32_t *>(lut_b + __byte_perm(w1, lane4, shi));
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        const uint2 bx = xc[((nt * 8 + b) * 4 + j) * 32 + lane];
                        mma_bf16_16816(cb[nt], a, bx.x, bx.y);
                    }
                }
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    acc[nt][0] = fmaf(ch0[bb], cb[nt][0], acc[nt][0]);
                    acc[nt][1] = fmaf(ch0[bb], cb[nt][1], acc[nt][1]);
                    acc[nt][2] = fmaf(ch1[bb], cb[nt][2], acc[nt][2]);
                    acc[nt][3] = fmaf(ch1[bb], cb[nt][3], acc[nt][3]);
                }
            }
        }
        if (has_next) x_store<NT>(xs + (cur ^ 1) * (NT * 1024), tid, xv);
        named_bar_sync(1, kGemvCompute);

        if (!has_next || nxt.ks == 0) {
            // ---------------- row block done in this CTA: combine halves, parts, adapter term
            if (!dep_done) {
                griddep_wait();                        // L and the cleared counters are visible
                dep_done = true;
            }
            const int M = grp.M, N = it.N;
            float *ex = reinterpret_cast<float *>(xs + cur * (NT * 1024));   // free until the next unit ends
            if (h == 1)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
                    reinterpret_cast<float4 *>(ex)[(nt * 8 + wr) * 32 + lane] =
                        make_float4(acc[nt][0], acc[nt][1], acc[nt][2], acc[nt][3]);
            named_bar_sync(1, kGemvCompute);
            const int ru0 = it.unit0 + pos.rb * it.nks;                      // first unit of the row block
            const int c_first = ru0 / grp.per_cta, c_last = (ru0 + it.nks - 1) / grp.per_cta;
            const int nparts = c_last - c_first + 1;
            const int row0 = pos.rb * kGemvRows + Rl0, row1 = row0 + 8;
            float tot[NT][4];
            if (h == 0) {
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const float4 o = reinterpret_cast<const float4 *>(ex)[(nt * 8 + wr) * 32 + lane];
                    tot[nt][0] = acc[nt][0] + o.x;
                    tot[nt][1] = acc[nt][1] + o.y;
                    tot[nt][2] = acc[nt][2] + o.z;
                    tot[nt][3] = acc[nt][3] + o.w;
                }
            }
            bool write_y = nparts == 1;
            if (nparts > 1) {
                if (h == 0) {
                    const int slot = ru0 < u_begin ? 0 : 1;
                    float *pp = grp.partial + ((int64_t)(blockIdx.x * 2 + slot) * kGemvRows) * M;
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        const int t0 = nt * 8 + 2 * t;
                        if (t0 < M) { pp[Rl0 * M + t0] = tot[nt][0]; pp[(Rl0 + 8) * M + t0] = tot[nt][2]; }
                        if (t0 + 1 < M) { pp[Rl0 * M + t0 + 1] = tot[nt][1]; pp[(Rl0 + 8) * M + t0 + 1] = tot[nt][3]; }
                    }
                    __threadfence();
                }
                named_bar_sync(1, kGemvCompute);
                if (tid == 0) {
                    const int old = atomicAdd(grp.counters + it.rb0 + pos.rb, 1);
                    flags[1] = (old == nparts - 1) ? 1 : 0;
                }
                named_bar_sync(1, kGemvCompute);
                write_y = flags[1] != 0;
                if (write_y && h == 0) {
                    __threadfence();
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) tot[nt][0] = tot[nt][1] = tot[nt][2] = tot[nt][3] = 0.0f;
                    for (int pi = 0; pi < nparts; ++pi) {
                        const int c = c_first + pi;
                        const int slot = ru0 < c * grp.per_cta ? 0 : 1;
                        const float *pp = grp.partial + ((int64_t)(c * 2 + slot) * kGemvRows) * M;
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            const int t0 = min(nt * 8 + 2 * t, M - 1), t1 = min(nt * 8 + 2 * t + 1, M - 1);
                            tot[nt][0] += __ldcg(pp + Rl0 * M + t0);
                            tot[nt][1] += __ldcg(pp + Rl0 * M + t1);
                            tot[nt][2] += __ldcg(pp + (Rl0 + 8) * M + t0);
                            tot[nt][3] += __ldcg(pp + (Rl0 + 8) * M + t1);
                        }
                    }
                    if (tid == 0) grp.counters[it.rb0 + pos.rb] = 0;   // ready for the next launch
                }
            }
            if (write_y && h == 0 && ok) {
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int tok = nt * 8 + 2 * t + (q & 1), row = (q < 2) ? row0 : row1;
                        if (tok < M && row < N) {
                            float y = tot[nt][q];
                            if (it.L) y += __ldcg(it.L + (int64_t)tok * N + row);
                            it.Y[(int64_t)tok * N + row] = __float2bfloat16_rn(y);
                        }
                    }
                }
            }
            named_bar_sync(1, kGemvCompute);              // ex is reused by the next unit
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.0f;
        }
        pos = nxt;
    }
}

// ---------------------------------------------------------------- host side
static int gemv_grid(int units) {
    int ctas = num_sms();
    if (ctas > units) ctas = units;
    const int per = (int)ceil_div(units, ctas);
    return (int)ceil_div(units, per);
}
static int item_units(const LinearDesc &d) {
    return (int)(ceil_div(d.W.rows, kGemvRows) * ceil_div(d.W.cols, kGemvKChunk));
}

// Workspace of one launch group: counters, partial slots, XA partials, L.
static size_t group_workspace(int64_t M, int count, const LinearDesc *d) {
    int units = 0, nrb = 0;
    size_t lora = 0;
    for (int i = 0; i < count; ++i) {
        units += item_units(d[i]);
        nrb += (int)ceil_div(d[i].W.rows, kGemvRows);
        if (d[i].r > 0) {
            lora += align256((size_t)ceil_div(d[i].W.cols, kXaChunk) * M * d[i].r * 4);
            lora += align256((size_t)M * d[i].W.rows * 4);
        }
    }
    const int grid = units > 0 ? gemv_grid(units) : 0;
    return align256((size_t)nrb * 4) + align256((size_t)grid * 2 * kGemvRows * M * 4) + lora;
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

template <typename... KArgs, typename... Args>
static cudaError_t launch_pdl(void (*kernel)(KArgs...), int grid, int block, size_t smem, cudaStream_t st, bool pdl,
                              Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3((unsigned)block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Small-M forward of count <= kGemvMaxItems projections: adapter kernels and one GEMV launch.
static cudaError_t gemv_group(int64_t M, int count, const LinearDesc *d, void *ws, cudaStream_t st) {
    GemvGroup grp;
    LoraGroup lg;
    grp.n = count;
    grp.M = (int)M;
    lg.n = 0;
    lg.M = (int)M;
    char *wsp = static_cast<char *>(ws);
    int units = 0, nrb = 0;
    for (int i = 0; i < count; ++i) {
        units += item_units(d[i]);
        nrb += (int)ceil_div(d[i].W.rows, kGemvRows);
    }
    const int grid = gemv_grid(units);
    grp.units = units;
    grp.per_cta = (int)ceil_div(units, grid);
    grp.counters = reinterpret_cast<int *>(wsp);
    wsp += align256((size_t)nrb * 4);
    grp.partial = reinterpret_cast<float *>(wsp);
    wsp += align256((size_t)grid * 2 * kGemvRows * M * 4);
    lg.counters = grp.counters;
    lg.ncounters = nrb;
    int u0 = 0, rb0 = 0, cta_xa = 0, cta_lora = 0;
    for (int i = 0; i < count; ++i) {
        GemvItem &it = grp.it[i];
        const NF4View &w = d[i].W;
        if (!make_map(&it.codes, w.codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, (uint64_t)w.cols / 2, (uint64_t)w.rows,
                      (uint64_t)w.cols / 2, 128, kGemvRows, CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
        it.scale8 = w.scale8;
        it.scale2 = w.scale2;
        it.offset = w.offset;
        it.X = d[i].X;
        it.Y = d[i].Y;
        it.L = nullptr;
        it.N = (int)w.rows;
        it.K = (int)w.cols;
        it.kbs = (int)(w.cols / 64);
        it.nks = (int)ceil_div(w.cols, kGemvKChunk);
        it.nrb = (int)ceil_div(w.rows, kGemvRows);
        it.unit0 = u0;
        it.rb0 = rb0;
        u0 += it.nks * it.nrb;
        rb0 += it.nrb;
        if (d[i].r > 0) {
            LoraItem &li = lg.it[lg.n++];
            li.X = d[i].X;
            li.A = d[i].A;
            li.B = d[i].B;
            li.XA_save = d[i].XA_save;
            li.s = d[i].s;
            li.K = it.K;
            li.N = it.N;
            li.r = d[i].r;
            li.nchunks = (int)ceil_div(w.cols, kXaChunk);
            li.part = reinterpret_cast<float *>(wsp);
            wsp += align256((size_t)li.nchunks * M * li.r * 4);
            li.L = reinterpret_cast<float *>(wsp);
            wsp += align256((size_t)M * w.rows * 4);
            li.cta_xa = cta_xa;
            li.cta_lora = cta_lora;
            cta_xa += li.nchunks;
            cta_lora += (int)ceil_div(w.rows, kLoraCols);
            it.L = li.L;
        }
    }
    cudaError_t e;
    const bool xa = lg.n > 0;
    if (xa) QNF4_LAUNCH("k_gemv_xa", st, k_gemv_xa<<<cta_xa, 256, 0, st>>>(lg));
    QNF4_LAUNCH("k_gemv_lora", st, e = launch_pdl(k_gemv_lora, xa ? cta_lora : 1, 256, 0, st, xa, lg));
    if (e != cudaSuccess) return e;
    if (M <= 8) {
        if ((e = set_smem(k_gemv<1>, gemv_smem(1))) != cudaSuccess) return e;
        QNF4_LAUNCH("k_gemv", st,
                    e = launch_pdl(k_gemv<1>, grid, gemv_threads(1), gemv_smem(1), st, true, grp, host_codebook()));
    } else {
        if ((e = set_smem(k_gemv<2>, gemv_smem(2))) != cudaSuccess) return e;
        QNF4_LAUNCH("k_gemv", st,
                    e = launch_pdl(k_gemv<2>, grid, gemv_threads(2), gemv_smem(2), st, true, grp, host_codebook()));
    }
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
