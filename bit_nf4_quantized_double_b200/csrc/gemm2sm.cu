// Two-SM tcgen05 GEMM for the large-batch path of the QLoRA linear layer
// (page "QLoRA: put the large model in memory, then change it with a small
// adapter", wq-win.github.io/llm/074-qlora, section 1 equation and section 3
// "dequantise to BF16 on demand").
//
// When many token tiles share one weight, dequantising inside the GEMM repeats
// the per-weight table lookups once per token tile, and those integer
// instructions, not the tensor core, set the pace. For such batches the layer
// dequantises W once into a bf16 scratch matrix (qnf4 dequant kernel) and runs
// this plain GEMM:
//   C[M, N] = A[M, K] * B[N, K]^T + Ae[M, Ke] * Be[N, Ke]^T        (fp32 accumulate)
// The extension operands carry the adapter term as extra K blocks of the same
// accumulator: forward  A = X,  B = W^ (d_out x d_in),  Ae = s*XA, Be = B_lora^T;
//                 dgrad A = dY, B = W^ read transposed,   Ae = s*G,  Be = A_lora.
//
// Tiling: a cluster of two CTAs computes a 256 x 256 tile with
// tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 16 per instruction). CTA r
// stages rows [128r, 128r + 128) of A and rows [128r, 128r + 128) of B; the MMA
// issued by rank 0 reads both CTAs' halves, and each CTA's TMEM receives its
// 128 accumulator rows. Per SM that is 8 KB of operand reads per K16 step, half
// of what a one-SM 128 x 256 tile with both operands in shared memory needs.
// Persistent: pair p takes work items p, p + pairs, p + 2 pairs, ..., so that at any
// moment the pairs work on neighbouring tiles, which share the operand panels in L2.
// An item is a whole tile, or, when the tiles are too few to occupy the SMs, one of
// `splits` equal ranges of a tile's K blocks: those write fp32 partial tiles that
// k_gemm2sm_reduce adds in split order. Two accumulators in TMEM let the epilogue of one
// item overlap the main loop of the next.
#include "launch.h"
#include "tc.cuh"
#include "tmap.h"

namespace qnf4 {
using namespace tc;

namespace g2 {
constexpr int kStages = 6;
constexpr int kTileM = 256, kTileN = 256, kHalf = 128;
constexpr int kStageA = kHalf * 128;          // 16 KB: 128 rows x 64 K, 128-byte swizzle
constexpr int kStageB = kHalf * 128;          // 16 KB: K-major, or MN-major as two 64-wide chunks
constexpr int kStage = kStageA + kStageB;
constexpr int kPart = kHalf * 128;            // epilogue staging: 128 rows x 64 columns bf16 (16 KB)
constexpr int kSmem = 1024 + kStages * kStage + 2 * kPart;
constexpr int kThreads = 192;                 // warp 0 TMA, warp 1 MMA + TMEM, warps 2..5 epilogue
constexpr uint32_t kTmemCols = 512;           // two 256-column accumulators
}  // namespace g2

struct G2Params {
    int M, N;          // output rows and columns
    int KB, KBE;       // main and extension K blocks of 64
    int ke;            // extension K extent (the extension blocks' MMAs stop at it)
    int tiles_m, tiles_n;
    int splits;        // K ranges per tile (1: the epilogue writes C directly)
    float *partial;    // [splits][M][N] fp32 when splits > 1
    int wait_first;    // B (not only the extension) comes from the kernel launched before
};

template <bool B_MN, bool BE_MN>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(g2::kThreads, 1)
k_gemm2sm(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_ae,
          const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_be,
          const __grid_constant__ CUtensorMap tm_c, G2Params p) {
    using namespace g2;
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t bars[2 * kStages + 5];
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;

    uint8_t *smem = align1024(smem_raw);
    uint8_t *staging = smem + kStages * kStage;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const uint32_t bar0 = smem_addr(bars);
    // full: only rank 0's is used (both CTAs' copies count on it); empty, tfull: both
    // CTAs' copies receive the multicast commits; tempty: rank 0's, 4 epilogue warps x 2 CTAs
    auto full = [&](uint32_t s) { return bar0 + 8u * s; };
    auto empty = [&](uint32_t s) { return bar0 + 8u * (kStages + s); };
    auto tfull = [&](uint32_t b) { return bar0 + 8u * (2 * kStages + b); };
    auto tempty = [&](uint32_t b) { return bar0 + 8u * (2 * kStages + 2 + b); };
    const uint32_t fin = bar0 + 8u * (2 * kStages + 4);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) { mbar_init(full(s), 1); mbar_init(empty(s), 1); }
        for (int b = 0; b < 2; ++b) { mbar_init(tfull(b), 1); mbar_init(tempty(b), 8); }
        mbar_init(fin, 1);
        s_abort = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tm_a);
        tma_prefetch_desc(&tm_ae);
        tma_prefetch_desc(&tm_b);
        tma_prefetch_desc(&tm_be);
        tma_prefetch_desc(&tm_c);
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_addr(&s_tmem), kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();   // both CTAs' barriers initialised and TMEM allocated before any cross-CTA use
    tc_fence_after();
    const uint32_t tmem = s_tmem;
    volatile int *abort = &s_abort;

    const int KBT = p.KB + p.KBE;
    const int ntiles = p.tiles_m * p.tiles_n;
    const int nitems = ntiles * p.splits;           // item i: tile i % ntiles, K range i / ntiles
    const int pair = (int)(blockIdx.x >> 1), npairs = (int)(gridDim.x >> 1);

    if (warp == 0) {
        // ------------------------------------------------ TMA producer (both CTAs)
        if (lane == 0) {
            uint32_t st = 0, ph = 0;
            bool ok = true, ext_ready = false;
            if (p.wait_first) {
                // B is written by the kernel before this one (programmatic dependent launch):
                // only this prologue overlapped it
                griddep_wait();
                fence_proxy_async_global();
                ext_ready = true;
            }
            for (int item = pair; item < nitems && ok; item += npairs) {
                const int tile = item % ntiles, sp = item / ntiles;
                const int kb_lo = sp * KBT / p.splits, kb_hi = (sp + 1) * KBT / p.splits;
                const int m0 = (tile % p.tiles_m) * kTileM + (int)rank * kHalf;
                const int n0 = (tile / p.tiles_m) * kTileN + (int)rank * kHalf;
                for (int kb = kb_lo; kb < kb_hi; ++kb) {
                    if (kb >= p.KB && !ext_ready) {
                        // the extension operand (s XA or s G) comes from the kernel launched just
                        // before this one, which may still run (programmatic dependent launch):
                        // the main K blocks above needed only inputs that were complete
                        griddep_wait();
                        fence_proxy_async_global();
                        ext_ready = true;
                    }
                    if (!mbar_wait(empty(st), ph ^ 1u, abort)) { ok = false; break; }
                    const uint32_t fb = map_to_rank(full(st), 0);
                    if (rank == 0) mbar_arrive_expect_tx(full(st), 2 * kStage);
                    const uint32_t da = smem_addr(smem + st * kStage), db = da + kStageA;
                    if (kb < p.KB) {
                        const int k0 = kb * 64;
                        tma_load_2d_pair(da, &tm_a, fb, k0, m0);
                        if (B_MN) {
                            tma_load_2d_pair(db, &tm_b, fb, n0, k0);
                            tma_load_2d_pair(db + 8192, &tm_b, fb, n0 + 64, k0);
                        } else {
                            tma_load_2d_pair(db, &tm_b, fb, k0, n0);
                        }
                    } else {
                        const int k0 = (kb - p.KB) * 64;
                        tma_load_2d_pair(da, &tm_ae, fb, k0, m0);
                        if (BE_MN) {
                            tma_load_2d_pair(db, &tm_be, fb, n0, k0);
                            tma_load_2d_pair(db + 8192, &tm_be, fb, n0 + 64, k0);
                        } else {
                            tma_load_2d_pair(db, &tm_be, fb, k0, n0);
                        }
                    }
                    if (++st == (uint32_t)kStages) { st = 0; ph ^= 1u; }
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (rank 0)
        if (rank == 0 && lane == 0) {
            const uint32_t idesc_main = idesc_bf16(kTileM, kTileN, false, B_MN);
            const uint32_t idesc_ext = idesc_bf16(kTileM, kTileN, false, BE_MN);
            const uint64_t adesc0 = sw128_desc(smem_addr(smem), 16, 1024);           // +2 per K16
            const uint64_t bk0 = sw128_desc(smem_addr(smem) + kStageA, 16, 1024);    // K-major B: +2 per K16
            const uint64_t bm0 = sw128_desc(smem_addr(smem) + kStageA, 8192, 1024);  // MN-major B: +128 per K16
            constexpr uint32_t kStageDesc = kStage >> 4;
            uint32_t st = 0, ph = 0, lt = 0;
            bool ok = true;
            for (int item = pair; item < nitems && ok; item += npairs, ++lt) {
                const int sp = item / ntiles;
                const int kb_lo = sp * KBT / p.splits, kb_hi = (sp + 1) * KBT / p.splits;
                const uint32_t acc = lt & 1u, use = lt >> 1;
                if (!mbar_wait_cluster(tempty(acc), (use & 1u) ^ 1u, abort)) break;
                tc_fence_after();
                const uint32_t d = tmem + acc * 256u;
                for (int kb = kb_lo; kb < kb_hi; ++kb) {
                    if (!mbar_wait(full(st), ph, abort)) { ok = false; break; }
                    tc_fence_after();
                    const uint64_t ad = adesc0 + st * kStageDesc;
                    if (kb < p.KB) {
                        const uint64_t bd = (B_MN ? bm0 : bk0) + st * kStageDesc;
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            mma_pair_ss(d, ad + 2u * k, bd + (B_MN ? 128u : 2u) * k, idesc_main,
                                        (kb != kb_lo || k != 0) ? 1u : 0u);
                    } else {
                        const uint64_t bd = (BE_MN ? bm0 : bk0) + st * kStageDesc;
                        const int nk = min(4, (p.ke - (kb - p.KB) * 64 + 15) / 16);
                        for (int k = 0; k < nk; ++k)
                            mma_pair_ss(d, ad + 2u * k, bd + (BE_MN ? 128u : 2u) * k, idesc_ext,
                                        (kb != kb_lo || k != 0) ? 1u : 0u);
                    }
                    mma_pair_commit(empty(st), 0x3);
                    if (++st == (uint32_t)kStages) { st = 0; ph ^= 1u; }
                }
                if (!ok) break;
                mma_pair_commit(tfull(acc), 0x3);
            }
            mma_pair_commit(fin, 0x1);   // every MMA has completed before TMEM is released
            const uint64_t t0 = global_timer_ns();
            while (!mbar_try_wait(fin, 0)) {
                if (global_timer_ns() - t0 > kWaitLimitNs) { raise_status(QLORA_ERR_TIMEOUT); break; }
            }
        }
    } else {
        // ------------------------------------------------ epilogue (warps 2..5, both CTAs)
        const int q = warp & 3, et = threadIdx.x - 64;
        const int row = q * 32 + lane;                 // TMEM lane = tile row within this CTA
        const uint32_t tempty0 = map_to_rank(tempty(0), 0), tempty1 = map_to_rank(tempty(1), 0);
        uint32_t lt = 0;
        for (int item = pair; item < nitems; item += npairs, ++lt) {
            const int tile = item % ntiles, sp = item / ntiles;
            const uint32_t acc = lt & 1u, use = lt >> 1;
            if (!mbar_wait(tfull(acc), use & 1u, abort)) break;
            tc_fence_after();
            const int m0 = (tile % p.tiles_m) * kTileM + (int)rank * kHalf;
            const int n0 = (tile / p.tiles_m) * kTileN;
            const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + acc * 256u;
#pragma unroll 1
            for (int part = 0; part < 4; ++part) {     // 64 output columns each
                uint32_t v[32], w[32];
                tmem_ld32(taddr + part * 64, v);
                tmem_ld32(taddr + part * 64 + 32, w);
                tmem_wait_ld();
                if (part == 3) {
                    // the accumulator is in registers: hand it back to the MMA issuer
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(acc ? tempty1 : tempty0);
                }
                if (p.splits > 1) {
                    // fp32 partial of this K range: row m0 + row, columns n0 + 64 part .. + 63
                    const int mg = m0 + row;
                    if (mg < p.M) {
                        float *dst = p.partial + ((int64_t)sp * p.M + mg) * p.N + n0 + part * 64;
#pragma unroll
                        for (int i = 0; i < 64; i += 4) {
                            if (n0 + part * 64 + i >= p.N) break;
                            const uint32_t *src = i < 32 ? v + i : w + (i - 32);
                            *reinterpret_cast<float4 *>(dst + i) =
                                make_float4(__uint_as_float(src[0]), __uint_as_float(src[1]), __uint_as_float(src[2]),
                                            __uint_as_float(src[3]));
                        }
                    }
                    continue;
                }
                uint8_t *stg = staging + (part & 1) * kPart;
                if (et == 0) bulk_wait_read1();        // the store that last read this buffer is done
                named_bar_sync(1, 128);
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint32_t *src = c < 4 ? v + 8 * c : w + 8 * (c - 4);
                    const uint4 o = make_uint4(pack_bf16x2(__uint_as_float(src[0]), __uint_as_float(src[1])),
                                               pack_bf16x2(__uint_as_float(src[2]), __uint_as_float(src[3])),
                                               pack_bf16x2(__uint_as_float(src[4]), __uint_as_float(src[5])),
                                               pack_bf16x2(__uint_as_float(src[6]), __uint_as_float(src[7])));
                    *reinterpret_cast<uint4 *>(stg + sw128_offset((uint32_t)row, (uint32_t)c)) = o;
                }
                fence_proxy_async_smem();
                named_bar_sync(1, 128);
                if (et == 0) {
                    tma_store_2d(&tm_c, smem_addr(stg), n0 + part * 64, m0);
                    bulk_commit();
                }
            }
        }
        if (et == 0) bulk_wait0();
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();   // neither CTA leaves while the pair's MMAs or arrivals may still touch it
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, kTmemCols);
    }
}

// C = bf16 of the sum of the splits' fp32 partials, added in split order; four consecutive
// elements per thread, every split's load issued before the adds.
constexpr int kMaxGemmSplits = 16;
__global__ void __launch_bounds__(256) k_gemm2sm_reduce(const float *__restrict__ part, int splits, int64_t count,
                                                        __nv_bfloat16 *__restrict__ C) {
    const int64_t stride = 4 * (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = 4 * ((int64_t)blockIdx.x * blockDim.x + threadIdx.x); i < count; i += stride) {
        float4 v[kMaxGemmSplits];
#pragma unroll
        for (int sp = 0; sp < kMaxGemmSplits; ++sp)
            if (sp < splits) v[sp] = __ldcg(reinterpret_cast<const float4 *>(part + sp * count + i));
        float4 a = v[0];
#pragma unroll
        for (int sp = 1; sp < kMaxGemmSplits; ++sp)
            if (sp < splits) {
                a.x += v[sp].x;
                a.y += v[sp].y;
                a.z += v[sp].z;
                a.w += v[sp].w;
            }
        *reinterpret_cast<uint2 *>(C + i) = make_uint2(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w));
    }
}

int gemm2sm_max_splits() { return kMaxGemmSplits; }

int gemm2sm_pairs(int max_pairs) {
    const int all = num_sms() / 2;
    return (max_pairs > 0 && max_pairs < all) ? max_pairs : all;
}

// C[M, N] (bf16, row-major, ldc = N) = A[M, K] B[N, K]^T + Ae[M, ke] Be[N, ke]^T.
// A, Ae: K-major bf16 (row strides K and ke). B: K-major [N][K] or, with
// b_mn, stored [K][N]. Be likewise with be_mn. ke == 0: no extension.
// K, N, ke multiples of 8 (16-byte row strides); all pointers 16-byte aligned.
// `pairs` CTA pairs (at most gemm2sm_pairs(0)) share the work items. With splits > 1, each
// tile's K blocks are cut into `splits` ranges whose fp32 partials go to `partial`
// ([splits][M][N]), and k_gemm2sm_reduce writes C. With pdl, the launch may begin while the
// previous kernel on the stream still runs, and only the extension operands Ae, Be are read
// after that kernel completes (it must produce nothing else this GEMM reads), unless
// wait_first, when that kernel also writes B and every load waits for it.
cudaError_t launch_gemm2sm(const __nv_bfloat16 *A, const __nv_bfloat16 *Ae, const __nv_bfloat16 *B, bool b_mn,
                           const __nv_bfloat16 *Be, bool be_mn, __nv_bfloat16 *C, int64_t M, int64_t N, int64_t K,
                           int ke, int pairs, int splits, float *partial, bool pdl, bool wait_first,
                           cudaStream_t st) {
    using namespace g2;
    if (M < 1 || N < 1 || K < 1 || K % 8 != 0 || N % 8 != 0 || ke < 0 || ke % 8 != 0 || pairs < 1 || splits < 1 ||
        splits > kMaxGemmSplits || (splits > 1 && !partial))
        return cudaErrorInvalidValue;
    CUtensorMap ta, tae, tb, tbe, tcm;
    bool ok = map_bf16(&ta, A, (uint64_t)K, (uint64_t)M, 64, kHalf);
    if (b_mn) ok = ok && map_bf16(&tb, B, (uint64_t)N, (uint64_t)K, 64, 64);
    else ok = ok && map_bf16(&tb, B, (uint64_t)K, (uint64_t)N, 64, kHalf);
    if (ke > 0) {
        ok = ok && map_bf16(&tae, Ae, (uint64_t)ke, (uint64_t)M, 64, kHalf);
        if (be_mn) ok = ok && map_bf16(&tbe, Be, (uint64_t)N, (uint64_t)ke, 64, 64);
        else ok = ok && map_bf16(&tbe, Be, (uint64_t)ke, (uint64_t)N, 64, kHalf);
    } else {
        tae = ta;
        tbe = tb;
    }
    ok = ok && map_bf16(&tcm, C, (uint64_t)N, (uint64_t)M, 64, kHalf);
    if (!ok) return cudaErrorInvalidValue;
    G2Params p;
    p.M = (int)M;
    p.N = (int)N;
    p.KB = (int)ceil_div(K, 64);   // a ragged last block reads zeros past K
    p.KBE = (int)ceil_div(ke, 64);
    p.ke = ke;
    p.tiles_m = (int)ceil_div(M, kTileM);
    p.tiles_n = (int)ceil_div(N, kTileN);
    p.splits = splits;
    p.partial = partial;
    p.wait_first = wait_first ? 1 : 0;
    const int nitems = p.tiles_m * p.tiles_n * splits;
    if (pairs > nitems) pairs = nitems;            // at least one item per pair
    cudaError_t e;
#define QNF4_G2(BM, BEM)                                                                                  \
    e = set_smem(k_gemm2sm<BM, BEM>, kSmem);                                                            \
    if (e != cudaSuccess) return e;                                                                      \
    QNF4_LAUNCH("k_gemm2sm", st,                                                                         \
                e = launch_pdl(k_gemm2sm<BM, BEM>, 2 * pairs, kThreads, kSmem, st, pdl, ta, tae, tb, tbe, tcm, p)); \
    if (e != cudaSuccess) return e;
    if (b_mn && be_mn) { QNF4_G2(true, true) }
    else if (b_mn) { QNF4_G2(true, false) }
    else if (be_mn) { QNF4_G2(false, true) }
    else { QNF4_G2(false, false) }
#undef QNF4_G2
    if (splits > 1) {
        const int64_t count = M * N;                   // N % 8 == 0: whole float4 groups
        int64_t grid = ceil_div(count, (int64_t)4 * 256);
        const int64_t cap = (int64_t)num_sms() * 8;
        if (grid > cap) grid = cap;
        QNF4_LAUNCH("k_gemm2sm_reduce", st,
                    k_gemm2sm_reduce<<<(unsigned)grid, 256, 0, st>>>(partial, splits, count, C));
    }
    return cudaGetLastError();
}

}  // namespace qnf4
