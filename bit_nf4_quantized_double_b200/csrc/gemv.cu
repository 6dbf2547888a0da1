// Small-M (M <= 16 tokens) forward: a streaming NF4 GEMV on the warp-level
// tensor-core path, and the dispatch between it and the fused tcgen05 GEMM.
//
// Layer: Y = X W^ + s (X A) B (page "QLoRA: put the large model in memory,
// then change it with a small adapter", wq-win.github.io/llm/074-qlora,
// section 1), at decode-sized M where the packed 4-bit codes dominate HBM
// traffic (section 2: about 4.127 bits per weight).
//
// k_gemv is persistent: each CTA builds, once, a 256-entry table byte ->
// bf16 pair (Q[hi], Q[lo]) replicated per lane (a warp's lookups never
// conflict), then takes work units of 128 weight rows x 512 inputs. For a unit
// it stages the X chunk as mma.sync B fragments, issues every code load (8 bytes
// per thread per 64-block: the four threads of a row cover one 32-byte sector)
// and every block-constant load of the unit before any arithmetic, and
// accumulates sum_k Q[code] x_k per 64-block with mma.sync m16n8k16 (16 weight
// rows x 8 tokens); the block's dequantised constant c^ then multiplies that
// block's partial dot product, so the per-weight work is one table lookup.
// Extra units compute the split-K partials of X*A for the adapter in the same
// launch. k_gemv_finish sums both kinds of partials in split order (fixed
// order: reproducible), adds s*(XA)*B and rounds to bf16.
#include "launch.h"

namespace qnf4 {

cudaError_t launch_linear_fwd_large(const __nv_bfloat16 *X, int64_t M, const NF4View &W, const __nv_bfloat16 *A,
                                    const __nv_bfloat16 *B, int r, float s, __nv_bfloat16 *Y,
                                    __nv_bfloat16 *XA_save, void *ws, cudaStream_t st);

constexpr int kGemvMaxM = 16;
constexpr int kGemvRows = 128;      // weight rows per unit (8 warps x 16)
constexpr int kGemvKChunk = 512;    // inputs per unit (8 blocks of 64)
constexpr int kGemvBlk = kGemvKChunk / 64;

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint2 ldg_nc_v2(const void *p) {
    uint2 r;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(p));
    return r;
}

__device__ __forceinline__ uint32_t pack2_bf16(const __nv_bfloat16 *p0, const __nv_bfloat16 *p1) {
    const uint32_t lo = *reinterpret_cast<const uint16_t *>(p0), hi = *reinterpret_cast<const uint16_t *>(p1);
    return lo | (hi << 16);
}

// One projection of a grouped small-M forward.
struct GemvItem {
    NF4View w;
    const __nv_bfloat16 *X;      // [M, K]
    const __nv_bfloat16 *A;      // [K, r] or null
    const __nv_bfloat16 *B;      // [r, N] or null
    __nv_bfloat16 *Y;            // [M, N]
    __nv_bfloat16 *XA_save;      // [M, r] or null
    float s;
    int r, splits, nrb;
    int unit0;                   // first unit of this item; main units then adapter units
    int out0;                    // first output element (M * N per item)
    int xa0;                     // first s*XA value in the finish kernel's table (M * r per item)
    float *partial;              // [splits][M][N]
    float *partial_xa;           // [splits][M][r]
};
constexpr int kGemvMaxItems = 8;
struct GemvGroup {
    GemvItem it[kGemvMaxItems];
    int n, M;
    int units, per_cta;          // total units; contiguous units per CTA
    int outs, xas;               // total outputs; total s*XA values
};

__device__ __forceinline__ int find_item(const GemvGroup &g, int u) {
    int i = 0;
#pragma unroll 1
    while (i + 1 < g.n && u >= g.it[i + 1].unit0) ++i;
    return i;
}

// Token tiles of 8 (NT = 1: M <= 8, NT = 2: M <= 16). Each CTA takes a contiguous
// range of units ordered (item, K split, row block), so it stages an X chunk once
// for all the row blocks of that split it handles.
template <int NT>
__global__ void __launch_bounds__(256, 2)
k_gemv(const __grid_constant__ GemvGroup grp, Codebook cb) {
    extern __shared__ __align__(16) uint8_t smem[];
    uint32_t *lut = reinterpret_cast<uint32_t *>(smem);                  // [256 entries][32 lanes]
    uint2 *xs = reinterpret_cast<uint2 *>(smem + 256 * 32 * 4);           // [NT][kGemvBlk][4][32]
    __shared__ float s_q[16];
    const int M = grp.M;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;

    if (threadIdx.x < 16) s_q[threadIdx.x] = cb.q[threadIdx.x];
    __syncthreads();
    for (int i = threadIdx.x; i < 256 * 32; i += blockDim.x) {
        const int e = i >> 5;
        const __nv_bfloat162 pr = __floats2bfloat162_rn(s_q[e >> 4], s_q[e & 15]);
        lut[i] = *reinterpret_cast<const uint32_t *>(&pr);
    }
    // lookup of code byte c: lut word (c * 32 + lane); byte address c * 128 + lane * 4
    const char *lut_b = reinterpret_cast<const char *>(lut) + lane * 4;
    int staged = -1;                 // (item, split) whose X chunk is in xs

    const int u_begin = blockIdx.x * grp.per_cta;
    const int u_end = min(grp.units, u_begin + grp.per_cta);
    for (int u = u_begin; u < u_end; ++u) {
        const int ii = find_item(grp, u);
        const GemvItem &it = grp.it[ii];
        const NF4View &w = it.w;
        const int K = (int)w.cols, N = (int)w.rows;
        const int lu = u - it.unit0;
        const int main_units = it.nrb * it.splits;
        const int ks = lu < main_units ? lu / it.nrb : lu - main_units;
        const int kbase = ks * kGemvKChunk;
        const int nblk = (min(K, kbase + kGemvKChunk) - kbase) / 64;
        if (lu >= main_units) {
            // ---------------- adapter partial: XA_ks[m][j] = sum over this K chunk of X[m][k] A[k][j]
            // mma m16n8k16 with X rows (tokens, zero past M) as A and A_lora columns as B.
            // Warp w takes 16-wide k steps w, w + 8, ...; all loads are issued before the
            // MMAs, and the eight warps' sums are added in warp order through shared memory.
            float *red = reinterpret_cast<float *>(xs);           // [8 warps][4 tiles][32 lanes][4]
            const int ntiles = it.r / 8;
            const int ksteps = nblk * 4;
            __syncthreads();                                      // xs is free
            staged = -1;
            for (int nt0 = 0; nt0 < ntiles; nt0 += 4) {           // at most 4 tiles per pass (smem)
                const int nts = min(4, ntiles - nt0);
                float c[4][4];
#pragma unroll
                for (int q = 0; q < 4; ++q) c[q][0] = c[q][1] = c[q][2] = c[q][3] = 0.0f;
                for (int kstep = warp; kstep < ksteps; kstep += 8) {
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
                            const __nv_bfloat16 *ak = it.A + (int64_t)(k0 + 2 * t) * it.r + (nt0 + q) * 8 + g;
                            bb[q][0] = pack2_bf16(ak, ak + it.r);
                            bb[q][1] = pack2_bf16(ak + 8 * it.r, ak + 9 * it.r);
                        }
                    }
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        if (q < nts) mma_bf16_16816(c[q], a, bb[q][0], bb[q][1]);
                }
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    if (q < nts)
                        *reinterpret_cast<float4 *>(red + ((warp * 4 + q) * 32 + lane) * 4) =
                            make_float4(c[q][0], c[q][1], c[q][2], c[q][3]);
                __syncthreads();
                // c[0], c[1]: token g, tile columns 2t, 2t+1; c[2], c[3]: token g + 8
                for (int i = threadIdx.x; i < nts * 32; i += blockDim.x) {
                    const int q = i >> 5, ln = i & 31;
                    float4 v = *reinterpret_cast<const float4 *>(red + (q * 32 + ln) * 4);
                    for (int ww = 1; ww < 8; ++ww) {
                        const float4 x = *reinterpret_cast<const float4 *>(red + ((ww * 4 + q) * 32 + ln) * 4);
                        v.x += x.x; v.y += x.y; v.z += x.z; v.w += x.w;
                    }
                    const int gg = ln >> 2, tt = ln & 3, j0 = (nt0 + q) * 8 + 2 * tt;
                    float *dst = it.partial_xa + (int64_t)ks * M * it.r;
                    if (gg < M) { dst[gg * it.r + j0] = v.x; dst[gg * it.r + j0 + 1] = v.y; }
                    if (gg + 8 < M) { dst[(gg + 8) * it.r + j0] = v.z; dst[(gg + 8) * it.r + j0 + 1] = v.w; }
                }
                __syncthreads();
            }
            continue;
        }
        const int rb = lu % it.nrb;
        const int key = ii * 4096 + ks;
        if (key != staged) {
            // ---------------- stage the X chunk as B fragments (k order matches the code bytes below)
            __syncthreads();   // every warp is done with the previous chunk
            for (int i = threadIdx.x; i < NT * nblk * 128; i += blockDim.x) {
                const int nt = i / (nblk * 128), rem = i % (nblk * 128);
                const int b = rem >> 7, j = (rem >> 5) & 3, ln = rem & 31;
                const int tok = nt * 8 + (ln >> 2), tt = ln & 3;
                const int k = kbase + b * 64 + 16 * tt + 4 * j;
                uint2 v = make_uint2(0u, 0u);
                if (tok < M) v = *reinterpret_cast<const uint2 *>(it.X + (int64_t)tok * K + k);
                xs[((nt * kGemvBlk + b) * 4 + j) * 32 + ln] = v;
            }
            __syncthreads();
            staged = key;
        }

        const int64_t kbs = K / 64;
        const float mu = *w.offset;
        const int r0 = rb * kGemvRows + warp * 16 + g, r1 = r0 + 8;
        const bool v0 = r0 < N, v1 = r1 < N;
        const uint8_t *c0p = w.codes + ((int64_t)r0 * K + kbase) / 2 + 8 * t;
        const uint8_t *c1p = w.codes + ((int64_t)r1 * K + kbase) / 2 + 8 * t;
        // every load of the unit in flight before any arithmetic
        uint2 u0[kGemvBlk], u1[kGemvBlk];
        int8_t q0[kGemvBlk], q1[kGemvBlk];
        const int64_t b0g = (int64_t)r0 * kbs + kbase / 64, b1g = (int64_t)r1 * kbs + kbase / 64;
#pragma unroll
        for (int b = 0; b < kGemvBlk; ++b) {
            const bool in = b < nblk;
            u0[b] = (in && v0) ? ldg_nc_v2(c0p + 32 * b) : make_uint2(0x77777777u, 0x77777777u);
            u1[b] = (in && v1) ? ldg_nc_v2(c1p + 32 * b) : make_uint2(0x77777777u, 0x77777777u);
            q0[b] = (in && v0) ? __ldg(w.scale8 + b0g + b) : (int8_t)0;
            q1[b] = (in && v1) ? __ldg(w.scale8 + b1g + b) : (int8_t)0;
        }
        // second-level steps: a unit's 8 blocks of one row touch at most two 256-block groups
        const int64_t g0a = b0g >> 8, g1a = b1g >> 8;
        const bool split0 = ((b0g + nblk - 1) >> 8) != g0a, split1 = ((b1g + nblk - 1) >> 8) != g1a;
        const float s0a = v0 ? __fdiv_rn(__ldg(w.scale2 + g0a), 127.0f) : 0.0f;
        const float s1a = v1 ? __fdiv_rn(__ldg(w.scale2 + g1a), 127.0f) : 0.0f;
        float s0b = s0a, s1b = s1a;
        if (split0) s0b = __fdiv_rn(__ldg(w.scale2 + g0a + 1), 127.0f);
        if (split1) s1b = __fdiv_rn(__ldg(w.scale2 + g1a + 1), 127.0f);

        float acc[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[nt][i] = 0.0f;
#pragma unroll
        for (int b = 0; b < kGemvBlk; ++b) {
            if (b >= nblk) break;
            const float st0 = ((b0g + b) >> 8) == g0a ? s0a : s0b;
            const float st1 = ((b1g + b) >> 8) == g1a ? s1a : s1b;
            const float ch0 = __fadd_rn(__fmul_rn((float)q0[b], st0), mu);
            const float ch1 = __fadd_rn(__fmul_rn((float)q1[b], st1), mu);
            float cblk[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i) cblk[nt][i] = 0.0f;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t w0 = (j < 2) ? u0[b].x : u0[b].y;
                const uint32_t w1 = (j < 2) ? u1[b].x : u1[b].y;
                // byte k of a word, times 128: ((w >> 8k) & 0xff) << 7 in two operations
                uint32_t a[4];
                if ((j & 1) == 0) {
                    a[0] = *reinterpret_cast<const uint32_t *>(lut_b + ((w0 << 7) & 0x7f80u));
                    a[2] = *reinterpret_cast<const uint32_t *>(lut_b + ((w0 >> 1) & 0x7f80u));
                    a[1] = *reinterpret_cast<const uint32_t *>(lut_b + ((w1 << 7) & 0x7f80u));
                    a[3] = *reinterpret_cast<const uint32_t *>(lut_b + ((w1 >> 1) & 0x7f80u));
                } else {
                    a[0] = *reinterpret_cast<const uint32_t *>(lut_b + ((w0 >> 9) & 0x7f80u));
                    a[2] = *reinterpret_cast<const uint32_t *>(lut_b + ((w0 >> 17) & 0x7f80u));
                    a[1] = *reinterpret_cast<const uint32_t *>(lut_b + ((w1 >> 9) & 0x7f80u));
                    a[3] = *reinterpret_cast<const uint32_t *>(lut_b + ((w1 >> 17) & 0x7f80u));
                }
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const uint2 bx = xs[((nt * kGemvBlk + b) * 4 + j) * 32 + lane];
                    mma_bf16_16816(cblk[nt], a, bx.x, bx.y);
                }
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                acc[nt][0] = fmaf(ch0, cblk[nt][0], acc[nt][0]);
                acc[nt][1] = fmaf(ch0, cblk[nt][1], acc[nt][1]);
                acc[nt][2] = fmaf(ch1, cblk[nt][2], acc[nt][2]);
                acc[nt][3] = fmaf(ch1, cblk[nt][3], acc[nt][3]);
            }
        }
        float *dst = it.partial + (int64_t)ks * M * N;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int t0 = nt * 8 + 2 * t, t1 = t0 + 1;
            if (v0 && t0 < M) dst[(int64_t)t0 * N + r0] = acc[nt][0];
            if (v0 && t1 < M) dst[(int64_t)t1 * N + r0] = acc[nt][1];
            if (v1 && t0 < M) dst[(int64_t)t0 * N + r1] = acc[nt][2];
            if (v1 && t1 < M) dst[(int64_t)t1 * N + r1] = acc[nt][3];
        }
    }
}

// For every item: Y[m, n] = bf16( sum_split partial[split][m][n] + sum_j (s XA[m, j]) B[j, n] ),
// XA[m, j] = sum_split partial_xa[split][m][j] (also written as bf16 to XA_save).
constexpr int kFinishMaxSplits = 32;
__global__ void __launch_bounds__(256)
k_gemv_finish(const __grid_constant__ GemvGroup grp) {
    extern __shared__ float sxa[];                // s * XA of every item, [xa0 + m * r + j]
    const int M = grp.M;
    for (int i = threadIdx.x; i < grp.xas; i += blockDim.x) {
        int ii = 0;
        while (ii + 1 < grp.n && i >= grp.it[ii + 1].xa0) ++ii;
        const GemvItem &it = grp.it[ii];
        const int li = i - it.xa0;
        float pv[kFinishMaxSplits];
#pragma unroll
        for (int sp = 0; sp < kFinishMaxSplits; ++sp)
            if (sp < it.splits) pv[sp] = __ldg(it.partial_xa + sp * M * it.r + li);
        float v = 0.0f;
#pragma unroll
        for (int sp = 0; sp < kFinishMaxSplits; ++sp)
            if (sp < it.splits) v += pv[sp];
        sxa[i] = it.s * v;
        if (it.XA_save && blockIdx.x == 0) it.XA_save[li] = __float2bfloat16_rn(v);
    }
    __syncthreads();
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < grp.outs; i += gridDim.x * blockDim.x) {
        int ii = 0;
        while (ii + 1 < grp.n && i >= grp.it[ii + 1].out0) ++ii;
        const GemvItem &it = grp.it[ii];
        const int N = (int)it.w.rows;
        const int64_t li = i - it.out0, count = (int64_t)M * N;
        const int m = (int)(li / N), n = (int)(li % N);
        float pv[kFinishMaxSplits];
#pragma unroll
        for (int sp = 0; sp < kFinishMaxSplits; ++sp)
            if (sp < it.splits) pv[sp] = __ldg(it.partial + sp * count + li);
        float v = 0.0f;
#pragma unroll
        for (int sp = 0; sp < kFinishMaxSplits; ++sp)
            if (sp < it.splits) v += pv[sp];
        const float *sx = sxa + it.xa0 + m * it.r;
        for (int j = 0; j < it.r; ++j) v = fmaf(sx[j], __bfloat162float(it.B[(int64_t)j * N + n]), v);
        it.Y[li] = __float2bfloat16_rn(v);
    }
}

static int gemv_splits(int64_t cols) { return (int)ceil_div(cols, kGemvKChunk); }
// lookup table + the larger of the X fragments and the adapter unit's reduction buffer
static size_t gemv_smem(int nt) {
    const size_t xs = (size_t)nt * kGemvBlk * 128 * 8, red = 8 * 4 * 32 * 4 * 4;
    return 256 * 32 * 4 + (xs > red ? xs : red);
}
constexpr size_t kFinishSmemMax = 48 * 1024;

static size_t item_workspace(int64_t M, int64_t rows, int64_t cols, int r) {
    const size_t sp = (size_t)gemv_splits(cols);
    size_t b = (sp * M * rows * 4 + 255) & ~size_t(255);
    if (r > 0) b += (sp * M * r * 4 + 255) & ~size_t(255);
    return b;
}

size_t fwd_workspace_bytes_large(int64_t M, int64_t rows, int64_t cols, int r);

size_t fwd_workspace_bytes(int64_t M, int64_t rows, int64_t cols, int r) {
    if (M <= kGemvMaxM) return item_workspace(M, rows, cols, r);
    return fwd_workspace_bytes_large(M, rows, cols, r);
}

size_t fwd_grouped_workspace_bytes(int64_t M, int count, const LinearDesc *d) {
    size_t b = 0;
    if (M <= kGemvMaxM) {
        for (int i = 0; i < count; ++i) b += item_workspace(M, d[i].W.rows, d[i].W.cols, d[i].r);
    } else {
        for (int i = 0; i < count; ++i) {
            const size_t x = fwd_workspace_bytes_large(M, d[i].W.rows, d[i].W.cols, d[i].r);
            if (x > b) b = x;
        }
    }
    return b;
}

// Small-M forward of count projections in one GEMV launch and one finish launch
// (count <= kGemvMaxItems and the s*XA table fits the finish kernel's shared memory;
// larger groups go in chunks).
static cudaError_t gemv_group(int64_t M, int count, const LinearDesc *d, void *ws, cudaStream_t st) {
    GemvGroup grp;
    grp.n = count;
    grp.M = (int)M;
    char *wsp = static_cast<char *>(ws);
    int units = 0, outs = 0, xas = 0;
    for (int i = 0; i < count; ++i) {
        GemvItem &it = grp.it[i];
        it.w = d[i].W;
        it.X = d[i].X;
        it.A = d[i].A;
        it.B = d[i].B;
        it.Y = d[i].Y;
        it.XA_save = d[i].r > 0 ? d[i].XA_save : nullptr;
        it.s = d[i].s;
        it.r = d[i].r;
        it.splits = gemv_splits(it.w.cols);
        if (it.splits > kFinishMaxSplits) return cudaErrorInvalidValue;
        it.nrb = (int)ceil_div(it.w.rows, kGemvRows);
        it.unit0 = units;
        it.out0 = outs;
        it.xa0 = xas;
        it.partial = reinterpret_cast<float *>(wsp);
        wsp += ((size_t)it.splits * M * it.w.rows * 4 + 255) & ~size_t(255);
        it.partial_xa = reinterpret_cast<float *>(wsp);
        if (it.r > 0) wsp += ((size_t)it.splits * M * it.r * 4 + 255) & ~size_t(255);
        units += it.nrb * it.splits + (it.r > 0 ? it.splits : 0);
        outs += (int)(M * it.w.rows);
        xas += (int)(M * it.r);
    }
    grp.units = units;
    grp.outs = outs;
    grp.xas = xas;
    int ctas = 2 * num_sms();
    if (ctas > units) ctas = units;
    grp.per_cta = (int)ceil_div(units, ctas);
    ctas = (int)ceil_div(units, grp.per_cta);
    cudaError_t e;
    if (M <= 8) {
        const size_t sm = gemv_smem(1);
        e = cudaFuncSetAttribute(k_gemv<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        if (e != cudaSuccess) return e;
        QNF4_LAUNCH("k_gemv", st, k_gemv<1><<<ctas, 256, sm, st>>>(grp, host_codebook()));
    } else {
        const size_t sm = gemv_smem(2);
        e = cudaFuncSetAttribute(k_gemv<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        if (e != cudaSuccess) return e;
        QNF4_LAUNCH("k_gemv", st, k_gemv<2><<<ctas, 256, sm, st>>>(grp, host_codebook()));
    }
    // at least one CTA per SM (32 outputs each at the smallest): the finish is latency bound
    int64_t g = ceil_div(outs, 32);
    if (g > (int64_t)num_sms()) g = ceil_div(outs, 256) > num_sms() ? ceil_div(outs, 256) : num_sms();
    if (g > (int64_t)num_sms() * 4) g = (int64_t)num_sms() * 4;
    const size_t fsm = (size_t)(xas > 0 ? xas : 1) * 4;
    QNF4_LAUNCH("k_gemv_finish", st, k_gemv_finish<<<(unsigned)g, 256, fsm, st>>>(grp));
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
    // chunks that fit one launch: at most kGemvMaxItems items and an s*XA table within the
    // finish kernel's shared memory
    char *wsp = static_cast<char *>(ws);
    int i = 0;
    while (i < count) {
        int n = 0;
        size_t xas = 0;
        while (i + n < count && n < kGemvMaxItems && (xas + (size_t)M * d[i + n].r) * 4 <= kFinishSmemMax) {
            xas += (size_t)M * d[i + n].r;
            ++n;
        }
        if (n == 0) return cudaErrorInvalidValue;
        cudaError_t e = gemv_group(M, n, d + i, wsp, st);
        if (e != cudaSuccess) return e;
        for (int k = 0; k < n; ++k) wsp += item_workspace(M, d[i + k].W.rows, d[i + k].W.cols, d[i + k].r);
        i += n;
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
