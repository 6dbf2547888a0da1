// tcgen05 / TMEM kernels of the QLoRA linear layer (sm_100a).
//
// Layer (page "QLoRA: put the large model in memory, then change it with a
// small adapter", wq-win.github.io/llm/074-qlora, section 1 equation):
//   Y  = X W^ + s X A B                 (forward)
//   dX = dY W^T + s (dY B^T) A^T        (backward; W^ gets no gradient)
//   dA = s X^T (dY B^T),  dB = s (X A)^T dY
// with W^ = Dequant(W4, scales) = (stored [d_out, d_in] matrix)^T, dequantised
// to bf16 on the fly (section 3).
//
// Kernels
//   k_fused_fwd   persistent; tile = 128 weight rows x 256 tokens. Dequant warps
//                 turn each 64-weight block of a weight row into bf16 through a
//                 16-entry per-block table (prmt lookups) and store it straight
//                 into TMEM with tcgen05.st; tcgen05.mma takes that as its A
//                 operand and the TMA-staged X tile (128-byte swizzle) as B, so
//                 the dequantised weight never touches shared memory. One extra
//                 K block multiplies B_lora^T (TMEM) by s*XA (TMA), which adds
//                 the adapter term inside the same accumulator.
//   k_fused_dgrad the transposed twin: the dequant warps write W^ tiles into
//                 shared memory in the MN-major 128-byte-swizzled layout
//                 tcgen05.mma reads directly, dY streams through TMA; the extra
//                 K block multiplies A_lora (TMA) by s*G (TMA).
//   k_skinny      TMA-fed tcgen05 GEMM for the rank-r products X*A, dY*B^T,
//                 X^T*(sG), dY^T*XA, split over K across the CTAs of a thread-block
//                 cluster that add their accumulators in a fixed order through
//                 distributed shared memory and apply scale/layout. Before a pair
//                 GEMM its CTAs may also carry extra warps that dequantise the
//                 weight into the GEMM's bf16 operand (skinny_dequant).
// Both fused kernels keep the accumulator tile D[row, token] in TMEM and store
// it transposed (out[token, row]) through a shared-memory staging tile and a
// TMA store.
#include <atomic>
#include <mutex>

#include "launch.h"
#include "tc.cuh"
#include "tmap.h"

namespace qnf4 {
using namespace tc;

// ------------------------------------------------------------------ dequant
// Per-block bf16 table T[c] = bf16(fl(Q[c] * c^)) split into byte planes:
// L[i] holds the low bytes of T[4i..4i+3], H[i] the high bytes.
__device__ __forceinline__ void make_table(const Codebook &cb, float chat, uint32_t (&L)[4], uint32_t (&H)[4]) {
    uint32_t tw[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) tw[j] = pack_bf16x2(__fmul_rn(cb.q[2 * j], chat), __fmul_rn(cb.q[2 * j + 1], chat));
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        L[i] = prmt(tw[2 * i], tw[2 * i + 1], 0x6420u);
        H[i] = prmt(tw[2 * i], tw[2 * i + 1], 0x7531u);
    }
}

// One 32-bit word of packed codes (8 elements e0..e7 in memory order, byte k =
// e[2k] << 4 | e[2k+1]) -> four bf16x2 words (e0|e1<<16, e2|e3<<16, ...).
// prmt selects bytes by 3-bit index; bit 3 of each code picks the table half.
__device__ __forceinline__ void lookup8(uint32_t w, const uint32_t (&L)[4], const uint32_t (&H)[4], uint32_t *out) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const uint32_t v = h ? (w >> 16) : w;
        const uint32_t sel = v & 0x7777u;
        const uint32_t sel2 = ((v >> 1) & 0x4444u) | 0x3210u;
        const uint32_t lo = prmt(prmt(L[0], L[1], sel), prmt(L[2], L[3], sel), sel2);
        const uint32_t hi = prmt(prmt(H[0], H[1], sel), prmt(H[2], H[3], sel), sel2);
        // nibble order inside the half-word is e1, e0, e3, e2
        out[2 * h] = prmt(lo, hi, 0x4051u);
        out[2 * h + 1] = prmt(lo, hi, 0x6273u);
    }
}

// 64 codes (32 bytes) of one block -> 32 bf16x2 words in element order.
__device__ __forceinline__ void dequant_block(const uint4 &c0, const uint4 &c1, const Codebook &cb, float chat,
                                              uint32_t (&o)[32]) {
    uint32_t L[4], H[4];
    make_table(cb, chat, L, H);
    lookup8(c0.x, L, H, o + 0);
    lookup8(c0.y, L, H, o + 4);
    lookup8(c0.z, L, H, o + 8);
    lookup8(c0.w, L, H, o + 12);
    lookup8(c1.x, L, H, o + 16);
    lookup8(c1.y, L, H, o + 20);
    lookup8(c1.z, L, H, o + 24);
    lookup8(c1.w, L, H, o + 28);
}

// Bounded wait without the abort short-cut, for draining in-flight copies.
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity) {
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - t0 > kWaitLimitNs) {
            raise_status(QLORA_ERR_TIMEOUT);
            return;
        }
    }
}

// Prefetched per-block constants (scale8, scale2) of the next kRing blocks a
// dequant thread will handle, so their global-memory latency overlaps the
// work on earlier blocks. Indexed with compile-time slots only.
constexpr int kRing = 4;
struct ScaleRing {
    int8_t q8[kRing];
    float s2[kRing];
    __device__ __forceinline__ void load(int slot, const NF4View &w, bool valid, int64_t row, int64_t kbs, int kb,
                                         int KB) {
        int8_t a = 0;
        float b = 0.0f;
        if (valid && kb < KB) {
            const int64_t blk = row * kbs + kb;
            a = __ldg(w.scale8 + blk);
            b = __ldg(w.scale2 + (blk >> 8));
        }
        q8[slot] = a;
        s2[slot] = b;
    }
    __device__ __forceinline__ void load_blk(int slot, const NF4View &w, bool valid, int64_t blk) {
        q8[slot] = valid ? __ldg(w.scale8 + blk) : (int8_t)0;
        s2[slot] = valid ? __ldg(w.scale2 + (blk >> 8)) : 0.0f;
    }
};

struct FusedParams {
    NF4View w;        // stored weight [rows, cols]
    int M;            // tokens
    int rows, cols;   // d_out, d_in
    int r;            // adapter rank (0: none)
    int tiles_tok;    // token tiles (256 each)
    int tiles_row;    // output-row tiles (128 each): weight rows (fwd) or d_in columns (dgrad)
    const __nv_bfloat16 *lora_t;  // fwd: B_lora [r, rows] (read transposed by the dequant warps)
};

constexpr int kTileRows = 128;   // TMEM lanes / MMA M
constexpr int kTileTok = 256;    // MMA N
constexpr int kTokStage = kTileTok * 128;          // 32 KB: 256 tokens x 64 bf16
// Epilogue shared by both fused kernels: TMEM D[row, token] -> bf16 staging
// [token][row] -> TMA store at (x = row0, y = tok0), in PARTS slices of
// 256 / PARTS tokens through one staging tile. The accumulator is released
// (tempty) as soon as its last columns are in registers.
template <int PARTS>
__device__ __forceinline__ void fused_epilogue(uint32_t tmem_d, int q, int lane, int et, uint8_t *staging,
                                               const CUtensorMap *tm_out, int row0, int tok0, uint32_t tempty) {
    constexpr int kPartTok = kTileTok / PARTS;
    uint16_t *st16 = reinterpret_cast<uint16_t *>(staging);
    const int row_local = q * 32 + lane;
#pragma unroll 1
    for (int h = 0; h < PARTS; ++h) {
        if (et == 0) bulk_wait_read0();      // the previous store has finished reading the staging tile
        named_bar_sync(1, 128);
#pragma unroll 1
        for (int c = 0; c < kPartTok / 32; ++c) {
            uint32_t v[32];
            tmem_ld32(tmem_d + ((uint32_t)(q * 32) << 16) + (uint32_t)(h * kPartTok + 32 * c), v);
            tmem_wait_ld();
            if (h == PARTS - 1 && c == kPartTok / 32 - 1) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(tempty);
            }
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const __nv_bfloat16 b = __float2bfloat16_rn(__uint_as_float(v[i]));
                st16[(32 * c + i) * kTileRows + row_local] = *reinterpret_cast<const uint16_t *>(&b);
            }
        }
        fence_proxy_async_smem();
        named_bar_sync(1, 128);
        if (et == 0) {
            tma_store_2d(tm_out, smem_addr(staging), row0, tok0 + h * kPartTok);
            bulk_commit();
        }
    }
}

// ================================================================ forward
// Warp roles (15 warps): 0 X producer (TMA), 1 MMA issuer + TMEM owner,
// 2..5 epilogue, 6..13 dequant (two groups of four; group g takes the K blocks
// of iteration parity g), 14 code-tile producer (TMA). Three decoupled rings:
// X tiles (SX), code tiles (SC, small, fetched far ahead) and dequantised
// weight tiles in TMEM (SA), so dequantisation runs up to SA K blocks ahead of
// the tensor core. The X and weight rings share one pair of barriers per K
// block (stage ring of SA entries): `full` completes when the X tile has landed
// and all four dequant warps have stored the weight tile, `empty` when the MMAs
// of that block have completed. The MMA thread therefore tests one barrier and
// commits once per block.
namespace fwd {
constexpr int SX = 5;
constexpr int SCG = 4;                       // code-tile slots per dequant group (two rings)
constexpr int SA = 8;                        // even: each TMEM slot always serves the same group
constexpr int SC = 2 * SCG;
constexpr int kCodeStage = kTileRows * 32;   // 4 KB: 128 rows x 32 code bytes (32-byte swizzle)
constexpr int kParts = 2;                    // output staging: 128 tokens x 128 rows (32 KB)
constexpr int kStaging = kTileTok / kParts * kTileRows * 2;
constexpr int kSmem = 1024 + SX * kTokStage + SC * kCodeStage + kStaging;
constexpr int kThreads = 480;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemD = 0, kTmemA = 256;  // A stage s at columns 256 + 32 s
}  // namespace fwd

__global__ void __launch_bounds__(fwd::kThreads, 1)
k_fused_fwd(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_codes,
            const __grid_constant__ CUtensorMap tm_xa, const __grid_constant__ CUtensorMap tm_y,
            FusedParams p, const __grid_constant__ Codebook cb) {
    using namespace fwd;
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t bars[2 * (SA + SC) + 3];
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;

    uint8_t *smem = align1024(smem_raw);
    uint8_t *xs = smem;
    uint8_t *cs = xs + SX * kTokStage;
    uint8_t *staging = cs + SC * kCodeStage;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t bar0 = smem_addr(bars);
    // stage barriers: block `it` uses full/empty(it % SA)
    auto full = [&](uint32_t s) { return bar0 + 8u * s; };
    auto empty = [&](uint32_t s) { return bar0 + 8u * (SA + s); };
    auto c_full = [&](int s) { return bar0 + 8u * (2 * SA + s); };
    auto c_empty = [&](int s) { return bar0 + 8u * (2 * SA + SC + s); };
    const uint32_t tfull = bar0 + 8u * (2 * (SA + SC)), tempty = tfull + 8u, fin = tfull + 16u;

    if (threadIdx.x == 0) {
        // full: the X producer's expect_tx arrival plus one arrival per dequant warp
        for (int s = 0; s < SA; ++s) { mbar_init(full(s), 5); mbar_init(empty(s), 1); }
        for (int s = 0; s < SC; ++s) { mbar_init(c_full(s), 1); mbar_init(c_empty(s), 4); }
        mbar_init(tfull, 1);
        mbar_init(tempty, 4);
        mbar_init(fin, 1);
        s_abort = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tm_x);
        tma_prefetch_desc(&tm_codes);
        tma_prefetch_desc(&tm_xa);
        tma_prefetch_desc(&tm_y);
    }
    if (warp == 1) {
        tmem_alloc(smem_addr(&s_tmem), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;
    volatile int *abort = &s_abort;

    const int KB = p.cols / 64;
    const int LKB = (p.r + 63) / 64;
    const int KBT = KB + LKB;
    const int ntiles = p.tiles_tok * p.tiles_row;

    if (warp == 0) {
        // ------------------------------------------------ X / s*XA producer
        if (lane == 0) {
            // X slot it % SX is free once block it - SX has been consumed
            uint32_t it = 0, sx = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
                const int tok0 = (tile % p.tiles_tok) * kTileTok;
                for (int kb = 0; kb < KBT; ++kb, ++it) {
                    if (it >= (uint32_t)SX) {
                        const uint32_t b = it - SX;
                        if (!mbar_wait(empty(b % SA), (b / SA) & 1u, abort)) { ok = false; break; }
                    }
                    const uint32_t bar = full(it % SA), dst = smem_addr(xs + sx * kTokStage);
                    mbar_arrive_expect_tx(bar, kTokStage);
                    if (kb < KB) tma_load_2d(dst, &tm_x, bar, kb * 64, tok0);
                    else tma_load_2d(dst, &tm_xa, bar, (kb - KB) * 64, tok0);
                    sx = sx + 1 == (uint32_t)SX ? 0u : sx + 1;
                }
            }
            // the last SX copies may still be in flight: wait for their stages
            const uint32_t first = it > (uint32_t)SX ? it - SX : 0;
            for (uint32_t i = first; i < it; ++i) drain_wait(full(i % SA), (i / SA) & 1u);
        }
    } else if (warp == 14) {
        // ------------------------------------------------ code-tile producer
        if (lane == 0) {
            // one ring per dequant group: the block of iteration it goes to ring it % 2
            uint32_t it = 0, ig[2] = {0u, 0u};
            bool ok = true;
            for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
                const int row0 = (tile / p.tiles_tok) * kTileRows;
                for (int kb = 0; kb < KB; ++kb) {
                    const int gg = (int)((it + (uint32_t)kb) & 1u);
                    const uint32_t i = ig[gg]++;
                    const int s = gg * SCG + (int)(i % SCG);
                    if (!mbar_wait(c_empty(s), ((i / SCG) & 1u) ^ 1u, abort)) { ok = false; break; }
                    mbar_arrive_expect_tx(c_full(s), kCodeStage);
                    tma_load_2d(smem_addr(cs + s * kCodeStage), &tm_codes, c_full(s), kb * 32, row0);
                }
                it += (uint32_t)KBT;
            }
            for (int gg = 0; gg < 2; ++gg) {
                const uint32_t first = ig[gg] > (uint32_t)SCG ? ig[gg] - SCG : 0;
                for (uint32_t i = first; i < ig[gg]; ++i) drain_wait(c_full(gg * SCG + (int)(i % SCG)), (i / SCG) & 1u);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            // The tensor core queues only about two MMAs, and each instruction of this
            // thread costs tens of cycles, so its own work per K block (4 MMAs, ~512 cycles
            // of tensor work) has to stay small: ring positions are counters, descriptors
            // advance by constants, one barrier is tested (without blocking, between
            // MMAs) and one commit releases the previous block's stage.
            static_assert((SA & (SA - 1)) == 0 && SX <= SA, "stage ring: power of two, at least the X ring");
            const uint32_t idesc = idesc_bf16(kTileRows, kTileTok, false, false);
            const uint64_t xdesc0 = sw128_desc(smem_addr(xs), 16, 1024);   // +2048 per 32 KB stage, +2 per K16
            const uint32_t dD = tmem + kTmemD, dA0 = tmem + kTmemA;
            uint32_t st = 0, ph = 0, sx = 0;   // stage slot (= TMEM slot) and parity, X slot
            uint32_t pst = 0;                  // stage slot of the previous block
            uint32_t lt = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++lt) {
                if (!mbar_wait(tempty, (lt & 1u) ^ 1u, abort) || !mbar_wait(full(st), ph, abort)) { ok = false; break; }
                tc_fence_after();
                for (int kb = 0; kb < KBT; ++kb) {
                    const uint64_t xd = xdesc0 + ((uint64_t)sx << 11);
                    const uint32_t ad = dA0 + (st << 5);
                    const uint32_t nst = (st + 1) & (SA - 1), nph = ph ^ (nst == 0 ? 1u : 0u);
                    const uint32_t nsx = sx + 1 == (uint32_t)SX ? 0u : sx + 1;
                    const bool first = kb == 0, has_next = kb + 1 < KBT;
                    bool next_ready = !has_next;
                    if (kb < KB) {
                        mma_ts(dD, ad, xd, idesc, first ? 0u : 1u);
                        if (!first) mma_commit(empty(pst));
                        mma_ts(dD, ad + 8u, xd + 2u, idesc, 1u);
                        if (has_next) next_ready = mbar_test(full(nst), nph);
                        mma_ts(dD, ad + 16u, xd + 4u, idesc, 1u);
                        mma_ts(dD, ad + 24u, xd + 6u, idesc, 1u);
                    } else {
                        // adapter block (kb >= KB >= 1): up to four K16 steps of the rank
                        const int nk = min(4, (p.r - (kb - KB) * 64 + 15) / 16);
                        for (int k = 0; k < nk; ++k) mma_ts(dD, ad + 8u * k, xd + 2u * k, idesc, 1u);
                        mma_commit(empty(pst));
                    }
                    if (has_next) {
                        if (!next_ready && !mbar_wait(full(nst), nph, abort)) { ok = false; break; }
                        tc_fence_after();
                    }
                    pst = st; st = nst; ph = nph; sx = nsx;
                }
                if (!ok) break;
                mma_commit(empty(pst));
                mma_commit(tfull);
            }
            mma_commit(fin);          // every MMA of this CTA has completed before TMEM is released
            drain_wait(fin, 0);
        }
    } else if (warp < 6) {
        // ------------------------------------------------ epilogue (warps 2..5)
        const int q = warp & 3, et = threadIdx.x - 64;
        uint32_t lt = 0;
        for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++lt) {
            const int tok0 = (tile % p.tiles_tok) * kTileTok, row0 = (tile / p.tiles_tok) * kTileRows;
            if (!mbar_wait(tfull, lt & 1u, abort)) break;
            tc_fence_after();
            fused_epilogue<kParts>(tmem + kTmemD, q, lane, et, staging, &tm_y, row0, tok0, tempty);
        }
        if (et == 0) bulk_wait0();
    } else {
        // ------------------------------------------------ dequant (warps 6..13)
        const int g = (warp - 6) >> 2;          // takes the iterations with it % 2 == g
        const int q = warp & 3;                 // TMEM lane quarter
        const int row_local = q * 32 + lane;
        const float mu = *p.w.offset;
        const int64_t kbs = p.cols / 64;        // 64-blocks per weight row
        // code tile rows are 32 bytes, stored with the 32-byte TMA swizzle
        const uint32_t src_off0 = row_local * 32 + ((0u ^ ((row_local >> 2) & 1u)) << 4);
        const uint32_t src_off1 = row_local * 32 + ((1u ^ ((row_local >> 2) & 1u)) << 4);
        uint32_t it = 0, ic = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
            const int row0 = (tile / p.tiles_tok) * kTileRows;
            const int n = row0 + row_local;
            const bool valid = n < p.rows;
            const uint32_t it0 = it, ic0 = ic;
            const int kb_first = (int)((uint32_t)g - it0) & 1;
            const int J = (KBT - kb_first + 1) / 2;
            ScaleRing ring;
#pragma unroll
            for (int d = 0; d < kRing; ++d) ring.load(d, p.w, valid, n, kbs, kb_first + 2 * d, KB);
            for (int j0 = 0; j0 < J && ok; j0 += kRing) {
#pragma unroll
                for (int u = 0; u < kRing; ++u) {
                    const int j = j0 + u;
                    if (j >= J) break;
                    const int kb = kb_first + 2 * j;
                    const uint32_t itj = it0 + (uint32_t)kb;
                    const uint32_t sa = itj % SA;
                    const int8_t q8 = ring.q8[u];
                    const float s2 = ring.s2[u];
                    ring.load(u, p.w, valid, n, kbs, kb + 2 * kRing, KB);
                    uint32_t v[32];
                    int code_slot = -1;
                    if (kb < KB) {
                        const uint32_t icj = ic0 + (uint32_t)j;          // this group's main blocks so far
                        const int sc = g * SCG + (int)(icj % SCG);
                        if (!mbar_wait(c_full(sc), (icj / SCG) & 1u, abort)) { ok = false; break; }
                        const uint8_t *src = cs + sc * kCodeStage;
                        const uint4 c0 = *reinterpret_cast<const uint4 *>(src + src_off0);
                        const uint4 c1 = *reinterpret_cast<const uint4 *>(src + src_off1);
                        code_slot = sc;
                        if (valid) {
                            dequant_block(c0, c1, cb, dq_constant(q8, s2, mu), v);
                        } else {
#pragma unroll
                            for (int i = 0; i < 32; ++i) v[i] = 0u;
                        }
                    } else {
                        // adapter block: A operand row n = B_lora[:, n] (rank index along K)
                        const int jr = (kb - KB) * 64;
                        const uint16_t *bl = reinterpret_cast<const uint16_t *>(p.lora_t);
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            const int k = jr + 2 * i;
                            const uint32_t lo = (valid && k < p.r) ? bl[(int64_t)k * p.rows + n] : 0u;
                            const uint32_t hi = (valid && k + 1 < p.r) ? bl[(int64_t)(k + 1) * p.rows + n] : 0u;
                            v[i] = lo | (hi << 16);
                        }
                    }
                    if (!mbar_wait(empty(sa), ((itj / SA) & 1u) ^ 1u, abort)) { ok = false; break; }
                    tc_fence_after();
                    tmem_st32(tmem + ((uint32_t)(q * 32) << 16) + kTmemA + 32u * sa, v);
                    tmem_wait_st();
                    tc_fence_before();
                    __syncwarp();
                    // the code slot is released only now: the values stored above depend on
                    // the codes read from it, so those reads have certainly completed
                    if (lane == 0) {
                        if (code_slot >= 0) mbar_arrive(c_empty(code_slot));
                        mbar_arrive(full(sa));
                    }
                }
            }
            it = it0 + (uint32_t)KBT;
            ic = ic0 + (uint32_t)((KB - kb_first + 1) / 2);  // main blocks this group handled
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ================================================================ dgrad
// Same warp roles; the dequant warps write W^ tiles (64 weight rows x 128
// d_in) into shared memory in the MN-major 128-byte-swizzled layout and the
// MMA reads them as its A operand; dY tiles come by TMA as B. The dY and W^
// rings have the same size and share one full/empty barrier pair per K block.
namespace dg {
constexpr int SX = 4;                        // dY / s*G tiles (32 KB); SX == SA
constexpr int SCG = 2;                       // code tiles per dequant group (4 KB: 64 rows x 64 bytes, 64-byte swizzle)
constexpr int SA = 4;                        // dequantised A tiles (16 KB: 2 MN chunks of 64 d_in x 64 K rows); even
constexpr int SC = 2 * SCG;
constexpr int kAStage = kTileRows * 128;
constexpr int kCodeStage = 64 * 64;
constexpr int kParts = 4;                    // output staging: 64 tokens x 128 rows (16 KB)
constexpr int kStaging = kTileTok / kParts * kTileRows * 2;
constexpr int kSmem = 1024 + SA * kAStage + SX * kTokStage + SC * kCodeStage + kStaging;
constexpr int kThreads = 480;
constexpr uint32_t kTmemCols = 256;
}  // namespace dg

__global__ void __launch_bounds__(dg::kThreads, 1)
k_fused_dgrad(const __grid_constant__ CUtensorMap tm_dy, const __grid_constant__ CUtensorMap tm_codes,
              const __grid_constant__ CUtensorMap tm_alora, const __grid_constant__ CUtensorMap tm_gs,
              const __grid_constant__ CUtensorMap tm_dx, FusedParams p, const __grid_constant__ Codebook cb) {
    using namespace dg;
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t bars[2 * (SA + SC) + 3];
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;

    uint8_t *smem = align1024(smem_raw);
    uint8_t *as = smem;
    uint8_t *bs = as + SA * kAStage;
    uint8_t *cs = bs + SX * kTokStage;
    uint8_t *staging = cs + SC * kCodeStage;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t bar0 = smem_addr(bars);
    static_assert(SX == SA && (SA & (SA - 1)) == 0, "one stage ring for dY and W^ tiles");
    auto full = [&](uint32_t s) { return bar0 + 8u * s; };
    auto empty = [&](uint32_t s) { return bar0 + 8u * (SA + s); };
    auto c_full = [&](int s) { return bar0 + 8u * (2 * SA + s); };
    auto c_empty = [&](int s) { return bar0 + 8u * (2 * SA + SC + s); };
    const uint32_t tfull = bar0 + 8u * (2 * (SA + SC)), tempty = tfull + 8u, fin = tfull + 16u;

    if (threadIdx.x == 0) {
        // full: the producer's expect_tx arrival plus one arrival per dequant warp. The
        // A tile of an adapter block comes by TMA; its dequant group still arrives.
        for (int s = 0; s < SA; ++s) { mbar_init(full(s), 5); mbar_init(empty(s), 1); }
        for (int s = 0; s < SC; ++s) { mbar_init(c_full(s), 1); mbar_init(c_empty(s), 4); }
        mbar_init(tfull, 1);
        mbar_init(tempty, 4);
        mbar_init(fin, 1);
        s_abort = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tm_dy);
        tma_prefetch_desc(&tm_codes);
        tma_prefetch_desc(&tm_alora);
        tma_prefetch_desc(&tm_gs);
        tma_prefetch_desc(&tm_dx);
    }
    if (warp == 1) {
        tmem_alloc(smem_addr(&s_tmem), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;
    volatile int *abort = &s_abort;

    const int KB = (p.rows + 63) / 64;           // contraction over d_out in blocks of 64 rows
    const int LKB = (p.r + 63) / 64;
    const int KBT = KB + LKB;
    const int ntiles = p.tiles_tok * p.tiles_row;

    if (warp == 0) {
        // ------------------------------------------------ dY / s*G producer (+ A_lora for adapter blocks)
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
                const int tok0 = (tile % p.tiles_tok) * kTileTok, col0 = (tile / p.tiles_tok) * kTileRows;
                for (int kb = 0; kb < KBT; ++kb, ++it) {
                    const uint32_t s = it % SA;
                    if (!mbar_wait(empty(s), ((it / SA) & 1u) ^ 1u, abort)) { ok = false; break; }
                    if (kb < KB) {
                        mbar_arrive_expect_tx(full(s), kTokStage);
                        tma_load_2d(smem_addr(bs + s * kTokStage), &tm_dy, full(s), kb * 64, tok0);
                    } else {
                        // the adapter A tile goes into the A slot of this stage
                        mbar_arrive_expect_tx(full(s), kTokStage + kAStage);
                        tma_load_2d(smem_addr(as + s * kAStage), &tm_alora, full(s), (kb - KB) * 64, col0);
                        tma_load_2d(smem_addr(bs + s * kTokStage), &tm_gs, full(s), (kb - KB) * 64, tok0);
                    }
                }
            }
            const uint32_t first = it > (uint32_t)SA ? it - SA : 0;
            for (uint32_t i = first; i < it; ++i) drain_wait(full(i % SA), (i / SA) & 1u);
        }
    } else if (warp == 14) {
        // ------------------------------------------------ code-tile producer
        if (lane == 0) {
            uint32_t it = 0, ig[2] = {0u, 0u};
            bool ok = true;
            for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
                const int col0 = (tile / p.tiles_tok) * kTileRows;
                for (int kb = 0; kb < KB; ++kb) {
                    const int gg = (int)((it + (uint32_t)kb) & 1u);
                    const uint32_t i = ig[gg]++;
                    const int s = gg * SCG + (int)(i % SCG);
                    if (!mbar_wait(c_empty(s), ((i / SCG) & 1u) ^ 1u, abort)) { ok = false; break; }
                    mbar_arrive_expect_tx(c_full(s), kCodeStage);
                    tma_load_2d(smem_addr(cs + s * kCodeStage), &tm_codes, c_full(s), col0 / 2, kb * 64);
                }
                it += (uint32_t)KBT;
            }
            for (int gg = 0; gg < 2; ++gg) {
                const uint32_t first = ig[gg] > (uint32_t)SCG ? ig[gg] - SCG : 0;
                for (uint32_t i = first; i < ig[gg]; ++i) drain_wait(c_full(gg * SCG + (int)(i % SCG)), (i / SCG) & 1u);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // the same lean issue loop as the forward kernel
            const uint32_t idesc_main = idesc_bf16(kTileRows, kTileTok, true, false);
            const uint32_t idesc_lora = idesc_bf16(kTileRows, kTileTok, false, false);
            const uint64_t adesc0 = sw128_desc(smem_addr(as), 8192, 1024);   // MN-major W^: +1024 per 16 KB stage, +128 per K16
            const uint64_t ldesc0 = sw128_desc(smem_addr(as), 16, 1024);     // K-major adapter tile: +2 per K16
            const uint64_t bdesc0 = sw128_desc(smem_addr(bs), 16, 1024);     // +2048 per 32 KB stage, +2 per K16
            uint32_t st = 0, ph = 0, pst = 0;
            uint32_t lt = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++lt) {
                if (!mbar_wait(tempty, (lt & 1u) ^ 1u, abort) || !mbar_wait(full(st), ph, abort)) { ok = false; break; }
                tc_fence_after();
                for (int kb = 0; kb < KBT; ++kb) {
                    const uint64_t bd = bdesc0 + ((uint64_t)st << 11);
                    const uint32_t nst = (st + 1) & (SA - 1), nph = ph ^ (nst == 0 ? 1u : 0u);
                    const bool first = kb == 0, has_next = kb + 1 < KBT;
                    bool next_ready = !has_next;
                    if (kb < KB) {
                        const uint64_t ad = adesc0 + ((uint64_t)st << 10);
                        mma_ss(tmem, ad, bd, idesc_main, first ? 0u : 1u);
                        if (!first) mma_commit(empty(pst));
                        mma_ss(tmem, ad + 128u, bd + 2u, idesc_main, 1u);
                        if (has_next) next_ready = mbar_test(full(nst), nph);
                        mma_ss(tmem, ad + 256u, bd + 4u, idesc_main, 1u);
                        mma_ss(tmem, ad + 384u, bd + 6u, idesc_main, 1u);
                    } else {
                        const uint64_t ad = ldesc0 + ((uint64_t)st << 10);
                        const int nk = min(4, (p.r - (kb - KB) * 64 + 15) / 16);
                        for (int k = 0; k < nk; ++k) mma_ss(tmem, ad + 2u * k, bd + 2u * k, idesc_lora, 1u);
                        mma_commit(empty(pst));
                    }
                    if (has_next) {
                        if (!next_ready && !mbar_wait(full(nst), nph, abort)) { ok = false; break; }
                        tc_fence_after();
                    }
                    pst = st; st = nst; ph = nph;
                }
                if (!ok) break;
                mma_commit(empty(pst));
                mma_commit(tfull);
            }
            mma_commit(fin);
            drain_wait(fin, 0);
        }
    } else if (warp < 6) {
        const int q = warp & 3, et = threadIdx.x - 64;
        uint32_t lt = 0;
        for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++lt) {
            const int tok0 = (tile % p.tiles_tok) * kTileTok, col0 = (tile / p.tiles_tok) * kTileRows;
            if (!mbar_wait(tfull, lt & 1u, abort)) break;
            tc_fence_after();
            fused_epilogue<kParts>(tmem, q, lane, et, staging, &tm_dx, col0, tok0, tempty);
        }
        if (et == 0) bulk_wait0();
    } else {
        // dequant: thread tg = (warp % 4) * 32 + lane -> weight row kb*64 + (tg % 64), d_in chunk tg / 64
        const int g = (warp - 6) >> 2;
        const int tg = (warp & 3) * 32 + lane;
        const int n_local = tg & 63, chunk = tg >> 6;
        const float mu = *p.w.offset;
        const int64_t kbs = p.cols / 64;
        // code tile rows are 64 bytes, stored with the 64-byte TMA swizzle
        const uint32_t sw = ((uint32_t)n_local >> 1) & 3u;
        const uint32_t src_off0 = n_local * 64 + (((2u * chunk) ^ sw) << 4);
        const uint32_t src_off1 = n_local * 64 + (((2u * chunk + 1u) ^ sw) << 4);
        uint32_t it = 0, ic = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
            const int col0 = (tile / p.tiles_tok) * kTileRows;
            const int kcol = col0 + 64 * chunk;
            const bool col_ok = kcol < p.cols;
            const uint32_t it0 = it, ic0 = ic;
            const int kb_first = (int)((uint32_t)g - it0) & 1;
            const int J = (KBT - kb_first + 1) / 2;
            // the block of (row kb*64 + n_local, column chunk kcol/64)
            auto blk_of = [&](int kb, bool &v) {
                const int n = kb * 64 + n_local;
                v = kb < KB && n < p.rows && col_ok;
                return (int64_t)n * kbs + kcol / 64;
            };
            ScaleRing ring;
#pragma unroll
            for (int d = 0; d < kRing; ++d) {
                bool v;
                const int64_t b = blk_of(kb_first + 2 * d, v);
                ring.load_blk(d, p.w, v, b);
            }
            for (int j0 = 0; j0 < J && ok; j0 += kRing) {
#pragma unroll
                for (int u = 0; u < kRing; ++u) {
                    const int j = j0 + u;
                    if (j >= J) break;
                    const int kb = kb_first + 2 * j;
                    const uint32_t itj = it0 + (uint32_t)kb;
                    const uint32_t sa = itj % SA;
                    bool valid;
                    blk_of(kb, valid);
                    const int8_t q8 = ring.q8[u];
                    const float s2 = ring.s2[u];
                    {
                        bool v;
                        const int64_t b = blk_of(kb + 2 * kRing, v);
                        ring.load_blk(u, p.w, v, b);
                    }
                    int code_slot = -1;
                    if (kb < KB) {
                        const uint32_t icj = ic0 + (uint32_t)j;          // this group's main blocks so far
                        const int sc = g * SCG + (int)(icj % SCG);
                        if (!mbar_wait(c_full(sc), (icj / SCG) & 1u, abort)) { ok = false; break; }
                        const uint8_t *src = cs + sc * kCodeStage;
                        const uint4 c0 = *reinterpret_cast<const uint4 *>(src + src_off0);
                        const uint4 c1 = *reinterpret_cast<const uint4 *>(src + src_off1);
                        code_slot = sc;
                        uint32_t v[32];
                        if (valid) {
                            dequant_block(c0, c1, cb, dq_constant(q8, s2, mu), v);
                        } else {
#pragma unroll
                            for (int i = 0; i < 32; ++i) v[i] = 0u;
                        }
                        if (!mbar_wait(empty(sa), ((itj / SA) & 1u) ^ 1u, abort)) { ok = false; break; }
                        uint8_t *dst = as + sa * kAStage + chunk * 8192;
#pragma unroll
                        for (int c = 0; c < 8; ++c)
                            *reinterpret_cast<uint4 *>(dst + sw128_offset(n_local, c)) =
                                make_uint4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
                        fence_proxy_async_smem();
                    } else {
                        // adapter block: the producer's TMA fills the A slot; the group only
                        // keeps the stage's arrival count
                        if (!mbar_wait(empty(sa), ((itj / SA) & 1u) ^ 1u, abort)) { ok = false; break; }
                    }
                    __syncwarp();
                    // the code slot is released only after the A-tile stores that depend on the
                    // codes read from it, so those reads have certainly completed
                    if (lane == 0) {
                        if (code_slot >= 0) mbar_arrive(c_empty(code_slot));
                        mbar_arrive(full(sa));
                    }
                }
            }
            it = it0 + (uint32_t)KBT;
            ic = ic0 + (uint32_t)((KB - kb_first + 1) / 2);  // main blocks this group handled
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ================================================================ skinny
// D[128 x BN] = sum over K of A[128 x K] * B[BN x K]^T, operands by TMA in
// 128-byte-swizzled tiles of 64 K; A and B each K-major or MN-major. The K blocks of an
// M tile are split over the S CTAs of one thread-block cluster (1 x S, S <= 8). Each
// CTA stages its fp32 accumulator in its own shared memory; CTA q of the cluster then
// adds rows q/S .. (q+1)/S of the tile over the S accumulators in split order (reading
// the peers' shared memory), scales, converts and writes the outputs. No partial sums
// go through HBM and no second kernel runs.
struct SkinnyParams {
    int Mp, Np, BN;        // output rows, columns (r), MMA N (Np rounded up to 16)
    int kb_total, kb_per_split;
    int stages;
    int nb;                // K blocks per stage: 2 with a K-major A read by one 3D box, else 1
    int transpose;         // the fp32 output as [Np][Mp] instead of [Mp][Np]
    float s;               // scale of out_s and out_f32
    __nv_bfloat16 *out;    // bf16 [Mp][Np] of the sum, or null
    __nv_bfloat16 *out_s;  // bf16 [Mp][Np] of s times the sum, or null
    float *out_f32;        // fp32 s times the sum, or null
    // dequantisation carried by the same CTAs (only with extra warps, see k_skinny)
    const uint32_t *dq_codes;    // packed codes, 8 weights per word
    const int8_t *dq_scale8;
    const float *dq_scale2, *dq_offset;
    uint4 *dq_out;               // bf16 weights, 8 per uint4
    int64_t dq_words;            // whole code words (n / 8)
    float dq_q[16];              // codebook
};
constexpr int kSkinnyMaxSplits = 8;    // a portable cluster
// dequantisation warps beside a product (one CTA per SM; 20 warps x 82 registers fill the
// register file; measured at 4096^2 fwd + bwd: 8 warps 247.6, 12 warps 242.2, 16 warps 239.3 us)
constexpr int kPrepDeqWarps = 16;

__device__ __forceinline__ float4 ld_cluster_f4(uint32_t caddr) {
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(caddr) : "memory");
    return v;
}

// With DW > 0 the CTA has DW more warps, which dequantise one share of a weight into bf16
// (the page's section 3: c^ = fl(fl(q8 fl(s2/127)) + mu), w^ = bf16(fl(Q[code] c^)), the
// same roundings as the dequantisation kernel) while warps 0..3 run the product: the two
// memory-bound passes in the same CTAs, so that their streams overlap. Used when the
// product has at most one CTA per SM. Warp-chunks of 256 code words (2048 weights) are
// taken grid-stride over all CTAs' extra warps; each lane expands words 32 u + lane,
// u = 0..7, of a chunk: eight coalesced 4-byte code loads issued before any arithmetic,
// eight coalesced 16-byte stores.
template <int DW>
__device__ __forceinline__ void skinny_dequant(const SkinnyParams &p, float *s_q) {
    const int lane = threadIdx.x & 31, dw = (threadIdx.x >> 5) - 4;
    // this warp's own copy of the codebook: the warp starts without waiting for the CTA
    if (lane < 16) s_q[lane] = p.dq_q[lane];
    __syncwarp();
    const int64_t cta = (int64_t)blockIdx.y * gridDim.x + blockIdx.x;
    const int64_t nw = p.dq_words;
    const int64_t chunks = (nw + 255) / 256;
    const int64_t stride = (int64_t)gridDim.x * gridDim.y * DW;
    const float mu = __ldg(p.dq_offset);
    for (int64_t c = cta * DW + dw; c < chunks; c += stride) {
        const int64_t w0 = c * 256;
        uint32_t w[8];
        int8_t q8[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int64_t wi = w0 + 32 * u + lane;
            w[u] = wi < nw ? __ldg(p.dq_codes + wi) : 0u;
            q8[u] = wi < nw ? __ldg(p.dq_scale8 + (wi >> 3)) : (int8_t)0;
        }
        const float step = __fdiv_rn(__ldg(p.dq_scale2 + (w0 >> 11)), 127.0f);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int64_t wi = w0 + 32 * u + lane;
            if (wi < nw) {
                const float ch = __fadd_rn(__fmul_rn((float)q8[u], step), mu);
                const uint32_t b = w[u];
                uint4 o;
                o.x = pack_bf16x2(__fmul_rn(s_q[(b >> 4) & 15u], ch), __fmul_rn(s_q[b & 15u], ch));
                o.y = pack_bf16x2(__fmul_rn(s_q[(b >> 12) & 15u], ch), __fmul_rn(s_q[(b >> 8) & 15u], ch));
                o.z = pack_bf16x2(__fmul_rn(s_q[(b >> 20) & 15u], ch), __fmul_rn(s_q[(b >> 16) & 15u], ch));
                o.w = pack_bf16x2(__fmul_rn(s_q[(b >> 28) & 15u], ch), __fmul_rn(s_q[(b >> 24) & 15u], ch));
                p.dq_out[wi] = o;
            }
        }
    }
}

template <bool A_MN, bool B_MN, int DW>
__global__ void __launch_bounds__(128 + 32 * DW, DW > 0 ? 1 : 2)
k_skinny(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
         const __grid_constant__ SkinnyParams p) {
    griddep_launch_dependents();                     // a following GEMM may start its main K blocks
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t bars[2 * 8 + 2];
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;
    __shared__ float s_q[DW > 0 ? DW * 16 : 1];
    uint8_t *smem = align1024(smem_raw);
    const int S = p.stages, NB = p.nb;
    const int a_bytes = 128 * 128;
    const int b_chunks = B_MN ? (p.BN + 63) / 64 : 1;
    const int b_bytes = B_MN ? b_chunks * 8192 : p.BN * 128;
    const int b_alloc = (b_bytes + 1023) & ~1023;
    // stage s: NB A tiles (16 KB each, consecutive K blocks) at as + s NB a_bytes, then the
    // NB B tiles at bs + s NB b_alloc
    uint8_t *as = smem;
    uint8_t *bs = smem + S * NB * a_bytes;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t bar0 = smem_addr(bars);
    auto full = [&](int s) { return bar0 + 8u * s; };
    auto empty = [&](int s) { return bar0 + 8u * (8 + s); };
    const uint32_t done = bar0 + 8u * 16, fin = done + 8u;
    uint32_t ncols = 32;
    while ((int)ncols < p.BN) ncols <<= 1;

    const int m0 = blockIdx.x * 128;
    const int split = blockIdx.y;                    // also the CTA's rank in its cluster
    const int nsplit = gridDim.y;
    const int kb0 = split * p.kb_per_split;
    const int kb1 = min(p.kb_total, kb0 + p.kb_per_split);
    volatile int *abort = &s_abort;

    // One stage's loads (the stage is free): NB K blocks of A and B from K block kb on. A box
    // past the split's last block (or past K, zero-filled) is loaded whole and left unused
    // by the MMAs.
    auto issue = [&](int kb, int s) {
        mbar_arrive_expect_tx(full(s), NB * (a_bytes + b_bytes));
        const uint32_t a = smem_addr(as + s * NB * a_bytes), b = smem_addr(bs + s * NB * b_alloc);
        if (A_MN) {
            tma_load_2d(a, &tm_a, full(s), m0, kb * 64);
            tma_load_2d(a + 8192, &tm_a, full(s), m0 + 64, kb * 64);
        } else if (NB > 1) {
            tma_load_3d(a, &tm_a, full(s), 0, m0, kb);     // NB K blocks of 128 rows: 128 NB-byte row runs
        } else {
            tma_load_2d(a, &tm_a, full(s), kb * 64, m0);
        }
        for (int bi = 0; bi < NB; ++bi) {
            const uint32_t bb = b + (uint32_t)(bi * b_alloc);
            if (B_MN) {
                for (int c = 0; c < b_chunks; ++c) tma_load_2d(bb + 8192u * c, &tm_b, full(s), 64 * c, (kb + bi) * 64);
            } else {
                tma_load_2d(bb, &tm_b, full(s), (kb + bi) * 64, 0);
            }
        }
    };

    // Thread 0 initialises the barriers and at once fills the S free stages (their loads need
    // nothing else), while warp 1 allocates TMEM; the product's warps then meet at a named
    // barrier of their own. The dequantisation warps never wait for it.
    uint32_t issued = 0;
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), 1);
        }
        mbar_init(done, 1);
        mbar_init(fin, 1);
        s_abort = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tm_a);
        tma_prefetch_desc(&tm_b);
        for (int kb = kb0; kb < kb1 && (int)issued < S; kb += NB, ++issued) issue(kb, (int)issued);
    }
    if (DW > 0 && warp >= 4) {
        skinny_dequant<DW>(p, s_q + (warp - 4) * 16);
    } else {
        if (warp == 1) {
            tmem_alloc(smem_addr(&s_tmem), ncols);
            tmem_relinquish();
        }
        tc_fence_before();
        named_bar_sync(1, 128);
        tc_fence_after();
    }
    const uint32_t tmem = s_tmem;

    if (warp == 0 && lane == 0) {
        uint32_t it = issued;
        for (int kb = kb0 + (int)issued * NB; kb < kb1; kb += NB, ++it) {
            const int s = it % S;
            const uint32_t ph = (it / S) & 1u;
            if (!mbar_wait(empty(s), ph ^ 1u, abort)) break;
            issue(kb, s);
        }
        const uint32_t first = it > (uint32_t)S ? it - S : 0;
        for (uint32_t i = first; i < it; ++i) drain_wait(full(i % S), (i / S) & 1u);
    } else if (warp == 1 && lane == 0) {
        const uint32_t idesc = idesc_bf16(128, p.BN, A_MN, B_MN);
        uint32_t it = 0;
        bool ok = true;
        for (int kb = kb0; kb < kb1; kb += NB, ++it) {
            const int s = it % S;
            const uint32_t ph = (it / S) & 1u;
            if (!mbar_wait(full(s), ph, abort)) { ok = false; break; }
            tc_fence_after();
            for (int bi = 0; bi < NB && kb + bi < kb1; ++bi) {
                const uint32_t a = smem_addr(as + (s * NB + bi) * a_bytes), b = smem_addr(bs + (s * NB + bi) * b_alloc);
                for (int k = 0; k < 4; ++k) {
                    const uint64_t ad =
                        A_MN ? sw128_desc(a + 2048u * k, 8192, 1024) : sw128_desc(a + 32u * k, 16, 1024);
                    const uint64_t bd =
                        B_MN ? sw128_desc(b + 2048u * k, 8192, 1024) : sw128_desc(b + 32u * k, 16, 1024);
                    mma_ss(tmem, ad, bd, idesc, (kb + bi != kb0 || k != 0) ? 1u : 0u);
                }
            }
            mma_commit(empty(s));
        }
        if (ok) mma_commit(done);
        mma_commit(fin);
        drain_wait(fin, 0);
    }
    __syncwarp();
    // the accumulator into this CTA's shared memory (the stages are free now): fp32
    // [128 rows][BN + 4], warp w holding TMEM lanes (rows) 32w .. 32w + 31
    const int ld = p.BN + 4;
    float *acc_s = reinterpret_cast<float *>(smem);
    if (warp < 4) {
        // TMEM lanes 0..127 belong to warps 0..3
        if (kb1 > kb0 && mbar_wait(done, 0, abort)) {
            tc_fence_after();
            const int rl = warp * 32 + lane;
            for (int c = 0; c < p.BN; c += 16) {
                uint32_t v[16];
                tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)c, v);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; i += 4)
                    *reinterpret_cast<float4 *>(acc_s + rl * ld + c + i) =
                        make_float4(__uint_as_float(v[i]), __uint_as_float(v[i + 1]), __uint_as_float(v[i + 2]),
                                    __uint_as_float(v[i + 3]));
            }
        } else {
            // no K blocks for this split (or an expired wait): it adds zero
            for (int i = threadIdx.x; i < 128 * ld; i += 128) acc_s[i] = 0.0f;
        }
    }
    cluster_sync();   // every CTA's accumulator is in its shared memory
    {
        const int rpc = (128 + nsplit - 1) / nsplit;
        const int r0 = split * rpc, r1 = min(128, r0 + rpc);
        const int nvec = p.Np / 4;
        const uint32_t base = smem_addr(acc_s);
        for (int e = threadIdx.x; e < (r1 - r0) * nvec; e += blockDim.x) {
            const int rl = r0 + e / nvec, c = (e % nvec) * 4;
            const int row = m0 + rl;
            if (row >= p.Mp) continue;
            const uint32_t off = base + (uint32_t)((rl * ld + c) * 4);
            // every peer's value is requested before the first add (the adds stay in rank order)
            float4 w[kSkinnyMaxSplits];
#pragma unroll
            for (int k = 0; k < kSkinnyMaxSplits; ++k)
                if (k < nsplit) w[k] = ld_cluster_f4(map_to_rank(off, (uint32_t)k));
            float4 v = w[0];
#pragma unroll
            for (int k = 1; k < kSkinnyMaxSplits; ++k)
                if (k < nsplit) {
                    v.x += w[k].x;
                    v.y += w[k].y;
                    v.z += w[k].z;
                    v.w += w[k].w;
                }
            const int64_t o = (int64_t)row * p.Np + c;
            if (p.out) *reinterpret_cast<uint2 *>(p.out + o) = make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
            if (p.out_s)
                *reinterpret_cast<uint2 *>(p.out_s + o) =
                    make_uint2(pack_bf16x2(p.s * v.x, p.s * v.y), pack_bf16x2(p.s * v.z, p.s * v.w));
            if (p.out_f32) {
                const float4 w = make_float4(p.s * v.x, p.s * v.y, p.s * v.z, p.s * v.w);
                if (p.transpose) {
                    p.out_f32[(int64_t)(c + 0) * p.Mp + row] = w.x;
                    p.out_f32[(int64_t)(c + 1) * p.Mp + row] = w.y;
                    p.out_f32[(int64_t)(c + 2) * p.Mp + row] = w.z;
                    p.out_f32[(int64_t)(c + 3) * p.Mp + row] = w.w;
                } else {
                    *reinterpret_cast<float4 *>(p.out_f32 + o) = w;
                }
            }
        }
    }
    tc_fence_before();
    cluster_sync();   // the peers have read this CTA's shared memory
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, ncols);
    }
}

// ================================================================ host side
// Split-K sizing: at most two CTAs per SM, all resident at once, at most
// kSkinnyMaxSplits CTAs (one cluster) per M tile, and at most four when four CTAs per
// M tile already reach three quarters of the SMs and K is at most 64 blocks.
constexpr int kSkinnyStages = 4;

struct SplitPlan { int kb_total, kb_per_split, splits; };
static SplitPlan plan_splits(int64_t Mp, int64_t Kp, int sms) {
    SplitPlan sp;
    sp.kb_total = (int)ceil_div(Kp, 64);
    const int mt = (int)ceil_div(Mp, 128);
    int want = (2 * sms) / mt;
    if (want > kSkinnyMaxSplits) want = kSkinnyMaxSplits;
    // four-CTA clusters once the tiles alone give most SMs a CTA and K is short: each tile's
    // reduction and cluster barrier then span half as many CTAs (measured at M = 4096: 248
    // against 253 us for the 4096^2 layer's fwd + bwd step; with K = 8192 and more, the
    // streaming outweighs those fixed costs and two CTAs per SM stream faster)
    if (want > 4 && 4 * mt >= (3 * sms) / 4 && sp.kb_total <= 64) want = 4;
    if (want < 1) want = 1;
    if (want > sp.kb_total) want = sp.kb_total;
    sp.kb_per_split = (int)ceil_div(sp.kb_total, want);
    sp.splits = (int)ceil_div(sp.kb_total, sp.kb_per_split);
    return sp;
}

// Outputs of one skinny product (any of them may be null): bf16 sum, bf16 s * sum,
// fp32 s * sum (transposed when f32_transposed).
struct SkinnyOut {
    __nv_bfloat16 *bf16 = nullptr, *bf16_s = nullptr;
    float *f32 = nullptr;
    bool f32_transposed = false;
    float s = 1.0f;
    // optional: a weight the same launch dequantises into deq_out (see skinny_takes_dequant)
    const NF4View *deq = nullptr;
    __nv_bfloat16 *deq_out = nullptr;
};

// Whether a product of Mp rows over Kp inputs runs one CTA on most SMs and never two, and
// streams at least 32 K blocks, so that its CTAs can carry the dequantisation warps
// (kPrepDeqWarps) of a weight as well with the whole GPU's memory parallelism (measured
// at 4096^2, M = 4096: fwd + bwd 240.9 against 247.1 us with twelve such warps; the
// 70B-like layer, whose only such product has K = 1024, measured 12.6 against 12.3 ms
// with it, so shorter products keep the two streams).
static bool skinny_takes_dequant(int64_t Mp, int64_t Kp) {
    const SplitPlan sp = plan_splits(Mp, Kp, num_sms());
    const int64_t ctas = ceil_div(Mp, (int64_t)128) * sp.splits;
    return ctas <= num_sms() && 4 * ctas >= 3 * (int64_t)num_sms() && sp.kb_total >= 32;
}

// Launch one skinny product on `sms` SMs' worth of CTAs (all of them, or those a
// concurrent GEMM leaves free). A operand: K-major [Mp rows, Kp] or MN-major [Kp rows, Mp];
// B operand: K-major [r rows, Kp] or MN-major [Kp rows, r].
static cudaError_t run_skinny(bool a_mn, const void *a, bool b_mn, const void *b, int64_t Mp, int64_t Kp, int r,
                              const SkinnyOut &out, cudaStream_t st, int sms = 0) {
    CUtensorMap ta, tb;
    const int BN = (int)ceil_div(r, 16) * 16;
    // a K-major A whose rows are whole 64-element blocks is read two blocks per 3D box
    // ([64 elements][Mp rows][Kp/64 blocks], block stride 128 bytes): 256-byte row runs
    const int nb = (!a_mn && Kp % 64 == 0) ? 2 : 1;
    bool ok;
    if (a_mn) {
        ok = map_bf16(&ta, a, (uint64_t)Mp, (uint64_t)Kp, 64, 64);
    } else if (nb > 1) {
        const uint64_t dims[3] = {64, (uint64_t)Mp, (uint64_t)(Kp / 64)};
        const uint64_t strides[2] = {(uint64_t)Kp * 2, 128};
        const uint32_t box[3] = {64, 128, (uint32_t)nb};
        ok = make_map_3d(&ta, a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
    } else {
        ok = map_bf16(&ta, a, (uint64_t)Kp, (uint64_t)Mp, 64, 128);
    }
    if (b_mn) ok = ok && map_bf16(&tb, b, (uint64_t)r, (uint64_t)Kp, 64, 64);
    else ok = ok && map_bf16(&tb, b, (uint64_t)Kp, (uint64_t)r, 64, (uint32_t)BN);
    if (!ok) return cudaErrorInvalidValue;
    const SplitPlan sp = plan_splits(Mp, Kp, sms > 0 ? sms : num_sms());
    SkinnyParams p;
    p.Mp = (int)Mp;
    p.Np = r;
    p.BN = BN;
    p.kb_total = sp.kb_total;
    p.kb_per_split = sp.kb_per_split;
    p.transpose = out.f32_transposed ? 1 : 0;
    p.s = out.s;
    p.out = out.bf16;
    p.out_s = out.bf16_s;
    p.out_f32 = out.f32;
    const bool with_deq = out.deq != nullptr;
    if (with_deq) {
        if (sms > 0 || !skinny_takes_dequant(Mp, Kp)) return cudaErrorInvalidValue;
        p.dq_codes = reinterpret_cast<const uint32_t *>(out.deq->codes);
        p.dq_scale8 = out.deq->scale8;
        p.dq_scale2 = out.deq->scale2;
        p.dq_offset = out.deq->offset;
        p.dq_out = reinterpret_cast<uint4 *>(out.deq_out);
        p.dq_words = out.deq->rows * out.deq->cols / 8;
        for (int i = 0; i < 16; ++i) p.dq_q[i] = host_codebook().q[i];
    } else {
        p.dq_codes = nullptr;
        p.dq_scale8 = nullptr;
        p.dq_scale2 = p.dq_offset = nullptr;
        p.dq_out = nullptr;
        p.dq_words = 0;
        for (int i = 0; i < 16; ++i) p.dq_q[i] = 0.0f;
    }
    const int b_bytes = b_mn ? (int)ceil_div(BN, 64) * 8192 : BN * 128;
    const int stage = nb * (128 * 128 + ((b_bytes + 1023) & ~1023));
    const int groups = (int)ceil_div(sp.kb_per_split, nb);      // stage loads per split
    int stages = (100 * 1024) / stage;
    if (stages > kSkinnyStages) stages = kSkinnyStages;
    if (stages > groups) stages = groups < 2 ? 2 : groups;
    if (stages < 1) stages = 1;
    p.stages = stages;
    p.nb = nb;
    const int acc_bytes = 128 * (BN + 4) * 4;       // the staged accumulator reuses the stages
    const int smem = 1024 + (stages * stage > acc_bytes ? stages * stage : acc_bytes);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)ceil_div(Mp, 128), (unsigned)sp.splits);
    cfg.blockDim = dim3(with_deq ? 128 + 32 * kPrepDeqWarps : 128);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 1;
    at[0].val.clusterDim.y = (unsigned)sp.splits;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    cudaError_t e;
#define QNF4_SK(AM, BM, DW)                                                  \
    e = set_smem(k_skinny<AM, BM, DW>, smem);                                \
    if (e != cudaSuccess) return e;                                          \
    QNF4_LAUNCH("k_skinny", st, e = cudaLaunchKernelEx(&cfg, k_skinny<AM, BM, DW>, ta, tb, p)); \
    if (e != cudaSuccess) return e;
    if (with_deq) {
        // the products that precede a pair GEMM: X A and dY B^T (K-major A)
        if (a_mn) return cudaErrorInvalidValue;
        if (b_mn) { QNF4_SK(false, true, kPrepDeqWarps) }
        else { QNF4_SK(false, false, kPrepDeqWarps) }
    } else if (a_mn && b_mn) { QNF4_SK(true, true, 0) }
    else if (a_mn) { QNF4_SK(true, false, 0) }
    else if (b_mn) { QNF4_SK(false, true, 0) }
    else { QNF4_SK(false, false, 0) }
#undef QNF4_SK
    return cudaGetLastError();
}

static size_t mr_bytes(int64_t M, int r) { return align256((size_t)M * (size_t)r * 2); }

// From this many tokens on (default 128), the layer dequantises W once into bf16
// scratch and runs the CTA-pair GEMM: the fused kernel repeats the dequantisation for
// every 256-token tile and runs at the rate of its integer work. Timed per direction at
// M = 128 .. 480 on 4096^2, 16384 x 1024, 1024 x 16384, 11008 x 4096 and 4096 x 11008
// weights (r = 64), the pair route was up to 30 % faster (the 16384 x 1024 forward at
// M = 480: 40.9 against 57.5 us) and at most 1.4 us slower (the 4096^2 forward at M = 384:
// 51.3 against 49.9 us); below 128 tokens the bf16 copy costs more than the fused kernel.
// With a larger P, from 128 tokens on a direction whose fused kernel would have fewer
// 128 x 256 output tiles than half the SMs still takes the pair GEMM, whose K blocks then
// split over the idle SMs. Settable so that both routes can be compared at any M
// (qlora_linear_set_pair_min_m; INT64_MAX keeps every M > 16 on the fused kernels).
constexpr int64_t kFewTilesMinM = 128;
static std::atomic<int64_t> g_pair_min_m{128};
// CTAs per SM of the dequantisation beside an adapter product of Mp rows over Kp inputs:
// three 256-thread CTAs when the product has at most one CTA per SM (they leave it the
// registers for one), else two, so that the product's CTAs are scheduled next to the
// dequantisation instead of after it (measured at 4096^2: 247.8 against 249.1 us per
// fwd + bwd step for three against two).
static int side_dequant_ctas(int64_t Mp, int64_t Kp) {
    const SplitPlan sp = plan_splits(Mp, Kp, num_sms());
    return ceil_div(Mp, (int64_t)128) * sp.splits <= num_sms() ? 3 : 2;
}
// out_rows: the output dimension the fused kernel tiles by 128 (the weight rows for the
// forward, its columns for the dgrad).
static bool pair_route(int64_t M, int64_t out_rows) {
    const int64_t P = g_pair_min_m.load(std::memory_order_relaxed);
    if (M >= P) return true;
    if (P == INT64_MAX || M < kFewTilesMinM) return false;
    const int64_t fused_tiles = ceil_div(M, (int64_t)kTileTok) * ceil_div(out_rows, (int64_t)kTileRows);
    return 2 * fused_tiles < num_sms();
}
static size_t wd_bytes(int64_t rows, int64_t cols) { return align256((size_t)rows * (size_t)cols * 2); }

static size_t fwd_adapter_bytes(int64_t M, int64_t cols, int r) {
    (void)cols;
    return r == 0 ? 0 : mr_bytes(M, r);                      // s XA
}

// Work plan of the pair GEMM for an [M, N] output over K inputs plus the r adapter ones.
// With at least half as many 256 x 256 tiles as CTA pairs, whole tiles and as few pairs as
// give the same number of tile rounds: the GEMM is bound by the power cap more than by the
// SM count (measured: a stream-K split of the K blocks over every SM was 0.6 % slower at
// 4096^2 than 64 pairs of four whole tiles, and its contiguous per-pair runs lost the L2
// reuse of the strided tile order on the 70B-like projections), and the SMs left over run
// the side stream's adapter gradients beside the dgrad GEMM. With fewer tiles, each tile's
// K blocks are split (at least eight per range, at most gemm2sm_max_splits ranges) so that
// the items fill the pairs, and a reduction adds the fp32 partials.
struct PairPlan {
    int pairs, splits;
};
static PairPlan pair_plan(int64_t M, int64_t N, int64_t K, int r) {
    const int64_t ntiles = ceil_div(M, 256) * ceil_div(N, 256);
    const int max_pairs = gemm2sm_pairs(0);
    const int kbt = (int)(ceil_div(K, 64) + ceil_div((int64_t)r, 64));
    int splits = 1;
    if (2 * ntiles <= max_pairs) {
        splits = (int)(max_pairs / ntiles);
        if (splits > kbt / 8) splits = kbt / 8;
        if (splits > gemm2sm_max_splits()) splits = gemm2sm_max_splits();
        if (splits < 1) splits = 1;
    }
    const int64_t items = ntiles * splits;
    const int64_t rounds = ceil_div(items, (int64_t)max_pairs);
    return {(int)ceil_div(items, rounds), splits};
}
static size_t split_bytes(const PairPlan &pp, int64_t M, int64_t N) {
    return pp.splits > 1 ? align256((size_t)pp.splits * (size_t)M * (size_t)N * 4) : 0;
}

size_t fwd_workspace_bytes_large(int64_t M, int64_t rows, int64_t cols, int r) {
    if (!pair_route(M, rows)) return fwd_adapter_bytes(M, cols, r);
    return fwd_adapter_bytes(M, cols, r) + wd_bytes(rows, cols) + split_bytes(pair_plan(M, rows, cols, r), M, rows);
}

static size_t bwd_adapter_bytes(int64_t M, int64_t rows, int64_t cols, int r) {
    (void)rows;
    (void)cols;
    return r == 0 ? 0 : 2 * mr_bytes(M, r);                  // s G, and X A when it is recomputed
}

size_t bwd_workspace_bytes(int64_t M, int64_t rows, int64_t cols, int r) {
    if (!pair_route(M, cols)) return bwd_adapter_bytes(M, rows, cols, r);
    return bwd_adapter_bytes(M, rows, cols, r) + wd_bytes(rows, cols) + split_bytes(pair_plan(M, cols, rows, r), M, cols);
}

static cudaError_t run_fused_fwd(const __nv_bfloat16 *X, int64_t M, const NF4View &W, const __nv_bfloat16 *XAs,
                                 const __nv_bfloat16 *Blora, int r, __nv_bfloat16 *Y, cudaStream_t st) {
    CUtensorMap tx, tc_, txa, ty;
    bool ok = map_bf16(&tx, X, (uint64_t)W.cols, (uint64_t)M, 64, kTileTok);
    ok = ok && make_map(&tc_, W.codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, (uint64_t)(W.cols / 2), (uint64_t)W.rows,
                        (uint64_t)(W.cols / 2), 32, kTileRows, CU_TENSOR_MAP_SWIZZLE_32B);
    if (r > 0) ok = ok && map_bf16(&txa, XAs, (uint64_t)r, (uint64_t)M, 64, kTileTok);
    else txa = tx;
    ok = ok && map_bf16(&ty, Y, (uint64_t)W.rows, (uint64_t)M, kTileRows, kTileTok / fwd::kParts,
                        CU_TENSOR_MAP_SWIZZLE_NONE);
    if (!ok) return cudaErrorInvalidValue;
    FusedParams p;
    p.w = W;
    p.M = (int)M;
    p.rows = (int)W.rows;
    p.cols = (int)W.cols;
    p.r = r;
    p.tiles_tok = (int)ceil_div(M, kTileTok);
    p.tiles_row = (int)ceil_div(W.rows, kTileRows);
    p.lora_t = Blora;
    const int ntiles = p.tiles_tok * p.tiles_row;
    const int grid = ntiles < num_sms() ? ntiles : num_sms();
    cudaError_t e = set_smem(k_fused_fwd, fwd::kSmem);
    if (e != cudaSuccess) return e;
    QNF4_LAUNCH("k_fused_fwd", st, k_fused_fwd<<<grid, fwd::kThreads, fwd::kSmem, st>>>(tx, tc_, txa, ty, p, host_codebook()));
    return cudaGetLastError();
}

static cudaError_t run_fused_dgrad(const __nv_bfloat16 *dY, int64_t M, const NF4View &W, const __nv_bfloat16 *Alora,
                                   const __nv_bfloat16 *Gs, int r, __nv_bfloat16 *dX, cudaStream_t st) {
    CUtensorMap tdy, tc_, ta, tg, tdx;
    bool ok = map_bf16(&tdy, dY, (uint64_t)W.rows, (uint64_t)M, 64, kTileTok);
    ok = ok && make_map(&tc_, W.codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, (uint64_t)(W.cols / 2), (uint64_t)W.rows,
                        (uint64_t)(W.cols / 2), 64, 64, CU_TENSOR_MAP_SWIZZLE_64B);
    if (r > 0) {
        ok = ok && map_bf16(&ta, Alora, (uint64_t)r, (uint64_t)W.cols, 64, kTileRows);
        ok = ok && map_bf16(&tg, Gs, (uint64_t)r, (uint64_t)M, 64, kTileTok);
    } else {
        ta = tdy;
        tg = tdy;
    }
    ok = ok && map_bf16(&tdx, dX, (uint64_t)W.cols, (uint64_t)M, kTileRows, kTileTok / dg::kParts,
                        CU_TENSOR_MAP_SWIZZLE_NONE);
    if (!ok) return cudaErrorInvalidValue;
    FusedParams p;
    p.w = W;
    p.M = (int)M;
    p.rows = (int)W.rows;
    p.cols = (int)W.cols;
    p.r = r;
    p.tiles_tok = (int)ceil_div(M, kTileTok);
    p.tiles_row = (int)ceil_div(W.cols, kTileRows);
    p.lora_t = nullptr;
    const int ntiles = p.tiles_tok * p.tiles_row;
    const int grid = ntiles < num_sms() ? ntiles : num_sms();
    cudaError_t e = set_smem(k_fused_dgrad, dg::kSmem);
    if (e != cudaSuccess) return e;
    QNF4_LAUNCH("k_fused_dgrad", st, k_fused_dgrad<<<grid, dg::kThreads, dg::kSmem, st>>>(tdy, tc_, ta, tg, tdx, p, host_codebook()));
    return cudaGetLastError();
}

// A second stream per device for work that can run beside other kernels: the
// pair GEMM leaves SMs free (it uses as few CTA pairs as give the same number of
// tile rounds) and is bound by the tensor pipe, while the adapter products and
// the dequantisation are bound by memory. The mutex keeps each fork/join
// sequence of events whole when several host threads call the library.
struct SideStream {
    cudaStream_t s = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
};
static std::mutex g_side_mu;
static SideStream *side_stream_locked() {
    static SideStream tab[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    SideStream &x = tab[dev];
    if (!x.s) {
        if (cudaStreamCreateWithFlags(&x.s, cudaStreamNonBlocking) != cudaSuccess ||
            cudaEventCreateWithFlags(&x.fork, cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&x.join, cudaEventDisableTiming) != cudaSuccess) {
            x = SideStream();
            return nullptr;
        }
    }
    return &x;
}

cudaError_t launch_linear_fwd_large(const __nv_bfloat16 *X, int64_t M, const NF4View &W, const __nv_bfloat16 *A,
                                    const __nv_bfloat16 *B, int r, float s, __nv_bfloat16 *Y,
                                    __nv_bfloat16 *XA_save, void *ws, cudaStream_t st) {
    __nv_bfloat16 *XAs = nullptr;
    const bool pair = pair_route(M, W.rows);
    __nv_bfloat16 *Wd = pair ? reinterpret_cast<__nv_bfloat16 *>(static_cast<char *>(ws) + fwd_adapter_bytes(M, W.cols, r))
                             : nullptr;
    cudaError_t e;
    std::unique_lock<std::mutex> lock(g_side_mu, std::defer_lock);
    SideStream *side = nullptr;
    // the dequantisation and X*A are independent memory-bound passes: run them in the same
    // CTAs when the product has at most one CTA per SM, else on two streams
    const bool prep = pair && r > 0 && skinny_takes_dequant(M, W.cols);
    if (pair && r > 0 && !prep) {
        lock.lock();
        side = side_stream_locked();
        if (side) {
            if ((e = cudaEventRecord(side->fork, st)) != cudaSuccess) return e;
            if ((e = cudaStreamWaitEvent(side->s, side->fork, 0)) != cudaSuccess) return e;
            if ((e = launch_dequant(W, Wd, side->s, side_dequant_ctas(M, W.cols))) != cudaSuccess) return e;
            if ((e = cudaEventRecord(side->join, side->s)) != cudaSuccess) return e;
        }
    }
    // the pair GEMM follows the X*A product directly (programmatic dependent launch: its
    // main K blocks may start while the product finishes), so the dequantised weight is
    // produced before the product or joined after it
    if (pair && !side && !prep && (e = launch_dequant(W, Wd, st)) != cudaSuccess) return e;
    if (r > 0) {
        XAs = static_cast<__nv_bfloat16 *>(ws);
        SkinnyOut o;
        o.bf16 = XA_save;
        o.bf16_s = XAs;
        o.s = s;
        if (prep) {
            o.deq = &W;
            o.deq_out = Wd;
        }
        e = run_skinny(false, X, true, A, M, W.cols, r, o, st);
        if (e != cudaSuccess) return e;
        if (side && (e = cudaStreamWaitEvent(st, side->join, 0)) != cudaSuccess) return e;
    }
    if (pair) {
        // Y = X W^T + (s XA) B: W^ [d_out, d_in] is the K-major B operand, B_lora [r, d_out]
        // the MN-major extension
        const PairPlan pp = pair_plan(M, W.rows, W.cols, r);
        float *part = reinterpret_cast<float *>(reinterpret_cast<char *>(Wd) + wd_bytes(W.rows, W.cols));
        return launch_gemm2sm(X, XAs, Wd, false, B, true, Y, M, W.rows, W.cols, r, pp.pairs, pp.splits, part, r > 0,
                              prep, st);
    }
    return run_fused_fwd(X, M, W, XAs, B, r, Y, st);
}

// dA = X^T (sG) and dB = s (XA)^T dY on stream `st`, sized for `sms` SMs.
static cudaError_t adapter_grads(const __nv_bfloat16 *X, const __nv_bfloat16 *dY, int64_t M, const NF4View &W,
                                 const __nv_bfloat16 *Gs, const __nv_bfloat16 *XA, int r, float s, float *dA,
                                 float *dB, cudaStream_t st, int sms = 0) {
    SkinnyOut oa;
    oa.f32 = dA;
    oa.s = 1.0f;
    cudaError_t e = run_skinny(true, X, true, Gs, W.cols, M, r, oa, st, sms);
    if (e != cudaSuccess) return e;
    // computed as (dY^T XA)^T, the fp32 output written transposed
    SkinnyOut ob;
    ob.f32 = dB;
    ob.f32_transposed = true;
    ob.s = s;
    e = run_skinny(true, dY, true, XA, W.rows, M, r, ob, st, sms);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t launch_linear_bwd(const __nv_bfloat16 *X, const __nv_bfloat16 *dY, int64_t M, const NF4View &W,
                              const __nv_bfloat16 *A, const __nv_bfloat16 *B, int r, float s,
                              const __nv_bfloat16 *XA, __nv_bfloat16 *dX, float *dA, float *dB, void *ws,
                              cudaStream_t st) {
    __nv_bfloat16 *Gs = nullptr;
    cudaError_t e;
    const bool pair = pair_route(M, W.cols);
    __nv_bfloat16 *Wd = pair ? reinterpret_cast<__nv_bfloat16 *>(static_cast<char *>(ws) +
                                                                bwd_adapter_bytes(M, W.rows, W.cols, r))
                             : nullptr;
    std::unique_lock<std::mutex> lock(g_side_mu, std::defer_lock);
    SideStream *side = nullptr;
    // the dequantisation overlaps the dY*B^T pass (in the same CTAs, or on a second
    // stream); after the dgrad GEMM is launched, the adapter gradients run beside it
    const bool prep = pair && r > 0 && skinny_takes_dequant(M, W.rows);
    if (pair && r > 0) {
        lock.lock();
        side = side_stream_locked();
        if (side && !prep) {
            if ((e = cudaEventRecord(side->fork, st)) != cudaSuccess) return e;
            if ((e = cudaStreamWaitEvent(side->s, side->fork, 0)) != cudaSuccess) return e;
            if ((e = launch_dequant(W, Wd, side->s, side_dequant_ctas(M, W.rows))) != cudaSuccess) return e;
            if ((e = cudaEventRecord(side->join, side->s)) != cudaSuccess) return e;
        }
    }
    // as in the forward, the pair GEMM follows the dY*B^T reduction directly
    if (pair && !side && !prep && (e = launch_dequant(W, Wd, st)) != cudaSuccess) return e;
    if (r > 0) {
        Gs = static_cast<__nv_bfloat16 *>(ws);
        __nv_bfloat16 *XAbuf = reinterpret_cast<__nv_bfloat16 *>(static_cast<char *>(ws) + mr_bytes(M, r));
        if (!XA) {
            SkinnyOut ox;
            ox.bf16 = XAbuf;
            e = run_skinny(false, X, true, A, M, W.cols, r, ox, st);
            if (e != cudaSuccess) return e;
            XA = XAbuf;
        }
        // G = dY B^T -> sG (bf16)
        SkinnyOut og;
        og.bf16_s = Gs;
        og.s = s;
        if (prep) {
            og.deq = &W;
            og.deq_out = Wd;
        }
        e = run_skinny(false, dY, false, B, M, W.rows, r, og, st);
        if (e != cudaSuccess) return e;
        if (side && !prep && (e = cudaStreamWaitEvent(st, side->join, 0)) != cudaSuccess) return e;
    }
    if (pair) {
        // dX = dY W^ + (s G) A^T: W^ [d_out, d_in] read as the MN-major B operand
        // ([K = d_out][N = d_in]), A_lora [d_in, r] the K-major extension
        const PairPlan pp = pair_plan(M, W.cols, W.rows, r);
        float *part = reinterpret_cast<float *>(reinterpret_cast<char *>(Wd) + wd_bytes(W.rows, W.cols));
        if (r > 0) {
            // the adapter gradients need only Gs and XA: they run on the side stream
            // while the dgrad GEMM occupies the tensor cores
            if (side) {
                if ((e = cudaEventRecord(side->fork, st)) != cudaSuccess) return e;
                e = launch_gemm2sm(dY, Gs, Wd, true, A, false, dX, M, W.cols, W.rows, r, pp.pairs, pp.splits, part,
                                   true, prep, st);
                if (e != cudaSuccess) return e;
                if ((e = cudaStreamWaitEvent(side->s, side->fork, 0)) != cudaSuccess) return e;
                // sized for the SMs the dgrad GEMM leaves free
                int free_sms = num_sms() - 2 * pp.pairs;
                if (free_sms < 2) free_sms = 2;
                e = adapter_grads(X, dY, M, W, Gs, XA, r, s, dA, dB, side->s, free_sms);
                if (e != cudaSuccess) return e;
                if ((e = cudaEventRecord(side->join, side->s)) != cudaSuccess) return e;
                return cudaStreamWaitEvent(st, side->join, 0);
            }
        }
        e = launch_gemm2sm(dY, Gs, Wd, true, A, false, dX, M, W.cols, W.rows, r, pp.pairs, pp.splits, part, r > 0,
                           prep, st);
    } else {
        e = run_fused_dgrad(dY, M, W, A, Gs, r, dX, st);
    }
    if (e != cudaSuccess) return e;
    if (r > 0) return adapter_grads(X, dY, M, W, Gs, XA, r, s, dA, dB, st);
    return cudaGetLastError();
}

}  // namespace qnf4

extern "C" void qlora_linear_set_pair_min_m(int64_t m) {
    qnf4::g_pair_min_m.store(m < 17 ? 17 : m, std::memory_order_relaxed);
}
