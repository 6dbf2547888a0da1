// Small-M (M <= 16 tokens) forward: a streaming NF4 GEMV on the warp-level
// tensor-core path, and the dispatch between it and the fused tcgen05 GEMM.
//
// Layer: Y = X W^ + s (X A) B (page "QLoRA: put the large model in memory,
// then change it with a small adapter", wq-win.github.io/llm/074-qlora,
// section 1), at decode-sized M where the packed 4-bit codes dominate HBM
// traffic (section 2: about 4.127 bits per weight).
//
// k_gemv streams each weight row's codes once with 8-byte loads (the four
// threads of a row cover one 32-byte sector per 64-block), turns code bytes
// into bf16 pairs (Q[hi], Q[lo]) through a 256-entry table replicated once
// per lane (so a warp's lookups never conflict), and accumulates
// sum_k Q[code]*x_k per 64-block with mma.sync m16n8k16 (16 weight rows x 8
// tokens). The block's dequantised constant c^ multiplies each block's partial
// dot product (sum Q*x) * c^, so the per-weight work is one table lookup.
// The K dimension is split across CTAs; k_gemv_finish sums the partials in
// split order, adds the adapter term s*XA*B and rounds to bf16.
#include "launch.h"

namespace qnf4 {

cudaError_t launch_linear_fwd_large(const __nv_bfloat16 *X, int64_t M, const NF4View &W, const __nv_bfloat16 *A,
                                    const __nv_bfloat16 *B, int r, float s, __nv_bfloat16 *Y,
                                    __nv_bfloat16 *XA_save, void *ws, cudaStream_t st);
cudaError_t launch_xa_small(const __nv_bfloat16 *X, int64_t M, int64_t cols, const __nv_bfloat16 *A, int r, float s,
                            __nv_bfloat16 *XA_save, __nv_bfloat16 *XAs, void *part_ws, cudaStream_t st);
size_t xa_small_workspace(int64_t M, int64_t cols, int r);

constexpr int kGemvMaxM = 16;
constexpr int kGemvRows = 128;      // weight rows per CTA (8 warps x 16)
constexpr int kGemvKChunk = 512;    // K per CTA
constexpr int kGemvUnroll = 4;      // 64-blocks in flight per thread

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

// Dequantised block constant of block b, with the second-level step cached
// while consecutive blocks stay in the same 256-block group.
struct StepCache {
    int64_t grp = -1;
    float step = 0.0f;
    __device__ __forceinline__ float chat(const NF4View &w, int64_t b, float mu) {
        const int64_t g = b >> 8;
        if (g != grp) {
            grp = g;
            step = __fdiv_rn(w.scale2[g], 127.0f);
        }
        return __fadd_rn(__fmul_rn((float)w.scale8[b], step), mu);
    }
};

// Token tiles of 8 (NT = 1: M <= 8, NT = 2: M <= 16). Grid: (row blocks, K splits).
template <int NT>
__global__ void __launch_bounds__(256)
k_gemv(NF4View w, const __nv_bfloat16 *__restrict__ X, int M, Codebook cb, float *__restrict__ partial) {
    extern __shared__ __align__(16) uint8_t smem[];
    uint32_t *lut = reinterpret_cast<uint32_t *>(smem);                  // [256 entries][32 lanes]
    uint2 *xs = reinterpret_cast<uint2 *>(smem + 256 * 32 * 4);           // [NT][nblk][4][32]
    const int K = (int)w.cols, N = (int)w.rows;
    const int kbase = blockIdx.y * kGemvKChunk;
    const int kend = min(K, kbase + kGemvKChunk);
    const int nblk = (kend - kbase) / 64;

    for (int i = threadIdx.x; i < 256 * 32; i += blockDim.x) {
        const int e = i >> 5;
        const __nv_bfloat162 pr = __floats2bfloat162_rn(cb.q[e >> 4], cb.q[e & 15]);
        lut[i] = *reinterpret_cast<const uint32_t *>(&pr);
    }
    const int units = NT * nblk * 128;
    for (int u = threadIdx.x; u < units; u += blockDim.x) {
        const int nt = u / (nblk * 128), rem = u % (nblk * 128);
        const int b = rem >> 7, j = (rem >> 5) & 3, ln = rem & 31;
        const int tok = nt * 8 + (ln >> 2), t = ln & 3;
        const int k = kbase + b * 64 + 16 * t + 4 * j;
        uint2 v = make_uint2(0u, 0u);
        if (tok < M) v = *reinterpret_cast<const uint2 *>(X + (int64_t)tok * K + k);
        xs[u] = v;
    }
    __syncthreads();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int r0 = blockIdx.x * kGemvRows + warp * 16 + g, r1 = r0 + 8;
    const bool v0 = r0 < N, v1 = r1 < N;
    const int64_t kbs = K / 64;
    const float mu = *w.offset;
    const uint8_t *c0p = w.codes + ((int64_t)r0 * K + kbase) / 2 + 8 * t;
    const uint8_t *c1p = w.codes + ((int64_t)r1 * K + kbase) / 2 + 8 * t;
    const uint32_t *lut_l = lut + lane;
    StepCache sc0, sc1;
    float acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[nt][i] = 0.0f;

    for (int b0 = 0; b0 < nblk; b0 += kGemvUnroll) {
        uint2 u0[kGemvUnroll], u1[kGemvUnroll];
#pragma unroll
        for (int u = 0; u < kGemvUnroll; ++u) {
            const bool in = b0 + u < nblk;
            u0[u] = (in && v0) ? ldg_nc_v2(c0p + 32 * (b0 + u)) : make_uint2(0x77777777u, 0x77777777u);
            u1[u] = (in && v1) ? ldg_nc_v2(c1p + 32 * (b0 + u)) : make_uint2(0x77777777u, 0x77777777u);
        }
#pragma unroll
        for (int u = 0; u < kGemvUnroll; ++u) {
            const int b = b0 + u;
            if (b >= nblk) break;
            const int64_t kb = kbase / 64 + b;
            const float ch0 = v0 ? sc0.chat(w, (int64_t)r0 * kbs + kb, mu) : 0.0f;
            const float ch1 = v1 ? sc1.chat(w, (int64_t)r1 * kbs + kb, mu) : 0.0f;
            float cblk[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i) cblk[nt][i] = 0.0f;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t w0 = (j < 2) ? u0[u].x : u0[u].y;
                const uint32_t w1 = (j < 2) ? u1[u].x : u1[u].y;
                const int sh = (j & 1) * 16;
                uint32_t a[4];
                a[0] = lut_l[((w0 >> sh) & 0xffu) << 5];
                a[2] = lut_l[((w0 >> (sh + 8)) & 0xffu) << 5];
                a[1] = lut_l[((w1 >> sh) & 0xffu) << 5];
                a[3] = lut_l[((w1 >> (sh + 8)) & 0xffu) << 5];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const uint2 bx = xs[((nt * nblk + b) * 4 + j) * 32 + lane];
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
    }
    float *dst = partial + (int64_t)blockIdx.y * M * N;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int t0 = nt * 8 + 2 * t, t1 = t0 + 1;
        if (v0 && t0 < M) dst[(int64_t)t0 * N + r0] = acc[nt][0];
        if (v0 && t1 < M) dst[(int64_t)t1 * N + r0] = acc[nt][1];
        if (v1 && t0 < M) dst[(int64_t)t0 * N + r1] = acc[nt][2];
        if (v1 && t1 < M) dst[(int64_t)t1 * N + r1] = acc[nt][3];
    }
}

// Y[m, n] = bf16( sum_split partial[split][m][n] + sum_j XAs[m, j] * B[j, n] ).
__global__ void k_gemv_finish(const float *__restrict__ partial, int splits, int M, int N,
                              const __nv_bfloat16 *__restrict__ XAs, const __nv_bfloat16 *__restrict__ B, int r,
                              __nv_bfloat16 *__restrict__ Y) {
    const int64_t count = (int64_t)M * N;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count; i += (int64_t)gridDim.x * blockDim.x) {
        const int m = (int)(i / N), n = (int)(i % N);
        float v = 0.0f;
        for (int sp = 0; sp < splits; ++sp) v += partial[sp * count + i];
        for (int j = 0; j < r; ++j)
            v = fmaf(__bfloat162float(XAs[(int64_t)m * r + j]), __bfloat162float(B[(int64_t)j * N + n]), v);
        Y[i] = __float2bfloat16_rn(v);
    }
}

static int gemv_splits(int64_t cols) { return (int)ceil_div(cols, kGemvKChunk); }
static size_t gemv_smem(int nt) { return 256 * 32 * 4 + (size_t)nt * (kGemvKChunk / 64) * 128 * 8; }

static size_t small_workspace(int64_t M, int64_t rows, int64_t cols, int r) {
    size_t b = ((size_t)gemv_splits(cols) * M * rows * 4 + 255) & ~size_t(255);
    if (r > 0) b += xa_small_workspace(M, cols, r);
    return b;
}

size_t fwd_workspace_bytes_large(int64_t M, int64_t rows, int64_t cols, int r);

size_t fwd_workspace_bytes(int64_t M, int64_t rows, int64_t cols, int r) {
    if (M <= kGemvMaxM) return small_workspace(M, rows, cols, r);
    return fwd_workspace_bytes_large(M, rows, cols, r);
}

cudaError_t launch_linear_fwd(const __nv_bfloat16 *X, int64_t M, const NF4View &W, const __nv_bfloat16 *A,
                              const __nv_bfloat16 *B, int r, float s, __nv_bfloat16 *Y, __nv_bfloat16 *XA_save,
                              void *ws, cudaStream_t st) {
    if (M > kGemvMaxM) return launch_linear_fwd_large(X, M, W, A, B, r, s, Y, XA_save, ws, st);
    const int splits = gemv_splits(W.cols);
    float *partial = static_cast<float *>(ws);
    char *rest = static_cast<char *>(ws) + (((size_t)splits * M * W.rows * 4 + 255) & ~size_t(255));
    __nv_bfloat16 *XAs = nullptr;
    cudaError_t e;
    if (r > 0) {
        XAs = reinterpret_cast<__nv_bfloat16 *>(rest);
        e = launch_xa_small(X, M, W.cols, A, r, s, XA_save, XAs, rest + (((size_t)M * r * 2 + 255) & ~size_t(255)), st);
        if (e != cudaSuccess) return e;
    }
    const dim3 grid((unsigned)ceil_div(W.rows, kGemvRows), (unsigned)splits);
    if (M <= 8) {
        const size_t sm = gemv_smem(1);
        e = cudaFuncSetAttribute(k_gemv<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        if (e != cudaSuccess) return e;
        QNF4_LAUNCH("k_gemv", st, k_gemv<1><<<grid, 256, sm, st>>>(W, X, (int)M, host_codebook(), partial));
    } else {
        const size_t sm = gemv_smem(2);
        e = cudaFuncSetAttribute(k_gemv<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        if (e != cudaSuccess) return e;
        QNF4_LAUNCH("k_gemv", st, k_gemv<2><<<grid, 256, sm, st>>>(W, X, (int)M, host_codebook(), partial));
    }
    const int64_t count = M * W.rows;
    int64_t g = ceil_div(count, 256);
    if (g > (int64_t)num_sms() * 8) g = (int64_t)num_sms() * 8;
    QNF4_LAUNCH("k_gemv_finish", st, k_gemv_finish<<<(unsigned)g, 256, 0, st>>>(partial, splits, (int)M, (int)W.rows, XAs, B, r, Y));
    return cudaGetLastError();
}

}  // namespace qnf4
