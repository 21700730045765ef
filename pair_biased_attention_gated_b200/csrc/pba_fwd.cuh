// Forward kernel: out = sigmoid(G) * softmax(scale * Q K^T + bias + mask) V, and the
// logsumexp of every query row.
//
// Pair-biased attention as described on the "AlphaFold3 open-source implementation" page,
// Model Efficiency section: the pair bias is added after the key-query dot product and
// is shared by every broadcast row b (triangle rows, MSA sequences, diffusion copies).
//
// Work item = (head h, 128-query tile, chunk of BC broadcast rows).  The kernel is
// persistent: two CTAs per SM, each walking the items blockIdx.x, blockIdx.x + gridDim.x,
// ... with one pipeline that runs across item boundaries (every ring and barrier counts
// steps and tiles of the CTA, not of the item), so the next item's loads and Q K^T
// overlap the current item's last steps and epilogue.  Within an item the loop runs over
// key tiles j (outer) and the chunk's rows b (inner): each 128x128 bias tile is moved into
// shared memory once and reused by all rows of the chunk.  The chunk's Q tiles are
// reloaded per item once the previous item's last Q K^T is done; K and V tiles stream
// through two rings: a K stage is refilled as soon as its Q K^T is done, a V stage only
// after its P V.
//
// Warp roles (256 threads, two warpgroups):
//   warps 0-3  softmax and epilogue: thread = query row = TMEM lane
//   warp 4     TMA producer (Q, K, V, bias tiles) and per-row key-mask words
//   warp 5     TMEM allocator and, on lane 0, the issuer of the Q K^T MMAs
//   warp 6     lane 0 issues the P V MMAs
//   warp 7     folds the key mask into each bias tile (masked keys -> -inf), or builds the
//              tile when there is no bias, so the softmax never tests mask bits
// A tcgen05.mma issue occupies the issuing thread about as long as the MMA runs, so the
// two products have separate issuers: Q K^T of the next step never queues behind P V.
// The second warpgroup hands registers to the first through setmaxnreg.
//
// Tensor memory (256 columns): S [0,128), P as packed bf16 [128,192), then one
// CP-column fp32 O accumulator per row of the chunk [192,256).  S and P are separate, so
// the next Q K^T runs while the softmax turns the current S into P: step k's softmax
// frees S right after reading it, and P only has to wait for the previous P V.  The O
// slots start over with the first P V of the next item, which waits for the P of that
// step, written only after the softmax warps have read this item's O out.
#pragma once

#include "pba_device.cuh"

namespace pba {

struct FwdArgs {
    int B, H, Nq, Nk, C;
    int nI, nJ, nChunks;
    int items;       // H * nI * nChunks work items, walked by a grid of at most 2 CTAs per SM
    int win;         // local attention: query tile t visits key tiles [t - win, t + win] (clamped);
                     // < 0: every key tile
    float scale;
    int has_bias;
    int mask_shared;  // the key mask (if any) is one row shared by every b
    const uint8_t *mask;
    long long smask_b;
    const __nv_bfloat16 *gate;
    long long sg0, sg1, sg2;
    __nv_bfloat16 *out;
    long long so0, so1, so2;
    float *lse;
    int skip_step;   // test hook: the producer skips this step's K load (-1: never)
};

template <int CP>
struct FwdTraits {
    static constexpr int BC = 64 / CP;                         // rows b per CTA (O slots)
    static constexpr int KVS = (CP == 16) ? 3 : 2;             // stages of each of the K and V rings
    static constexpr int BS = (CP == 64) ? 1 : 2;              // bias tile buffers
    static constexpr int TILE_BYTES = 128 * CP * 2;            // Q, K or V tile
    static constexpr int BIAS_BYTES = 128 * 128 * 2;           // two 64-key halves
    static constexpr int OFF_BIAS = 0;                         // 1024-byte aligned (SW128)
    static constexpr int OFF_Q = OFF_BIAS + BS * BIAS_BYTES;
    static constexpr int OFF_K = OFF_Q + BC * TILE_BYTES;
    static constexpr int OFF_V = OFF_K + KVS * TILE_BYTES;
    static constexpr int OFF_MASK = OFF_V + KVS * TILE_BYTES;  // u32 [KVS][8] per-row words (V ring)
    static constexpr int NBAR = 2 + 4 * KVS + 3 * BS + 6;
    static constexpr int OFF_BAR = OFF_MASK + KVS * 32;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;        // TMEM base, abort flag
    static constexpr int SMEM_BYTES = OFF_MISC + 16;
    static constexpr uint32_t SWZ = CP == 64 ? kSw128 : (CP == 32 ? kSw64 : kSw32);
    static constexpr uint32_t ROWB = CP * 2;                   // bytes per tile row
    static constexpr int THREADS = 256;
    // register split through setmaxnreg: 128 x 200 + 128 x 56 = 256 x 128, the registers
    // the CTA is launched with at two CTAs per SM (the build checks that ptxas reports 128)
    static constexpr int REGS_SOFTMAX = 200;
    static constexpr int REGS_OTHER = 56;
    static constexpr int TMEM_COLS = 256;
    static constexpr uint32_t T_S = 0, T_P = 128, T_O = 192;
};
// two CTAs per SM: 2 x (shared memory + the 1 KB the system reserves per CTA) <= 228 KB
static_assert(2 * (FwdTraits<16>::SMEM_BYTES + 1024) <= 233472, "smem");
static_assert(2 * (FwdTraits<32>::SMEM_BYTES + 1024) <= 233472, "smem");
static_assert(2 * (FwdTraits<64>::SMEM_BYTES + 1024) <= 233472, "smem");

// Online-softmax rescale threshold (natural-log units, = 8 in log2 units): the running
// maximum is only moved, and O and l rescaled, when a row's maximum grows by more than
// this.  Exponentials are then bounded by 2^8, harmless in fp32 and bf16; the final
// O / l is exact regardless of the reference point.
constexpr float kRescaleThresh = 5.545177444479562f;
constexpr float kLog2e = 1.4426950408889634f;

enum : unsigned {
    SITE_FWD_PROD = 0x101, SITE_FWD_MMA = 0x102, SITE_FWD_SOFTMAX = 0x103,
    SITE_FWD_EPI = 0x104, SITE_FWD_FOLD = 0x105,
    SITE_FWD_ALIGN = 0x1FF   // refused: dynamic shared memory not 1024-byte aligned
};

// byte offset of bias element (row r, key c) in a tile: two 64-key halves of 128 rows x
// 128 bytes, 16-byte chunks swizzled by the row (the TMA 128-byte swizzle)
__device__ __forceinline__ uint32_t bias_off(int r, int c) {
    return (uint32_t)((c >> 6) * 16384 + r * 128 + ((((c & 63) >> 3) ^ (r & 7)) << 4) + (c & 7) * 2);
}

template <int CP>
__global__ void __launch_bounds__(256, 2)
pba_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV,
               const __grid_constant__ CUtensorMap tmBias, const FwdArgs a) {
    using T = FwdTraits<CP>;
    constexpr int KVS = T::KVS, BS = T::BS, BC = T::BC;
    extern __shared__ __align__(1024) uint8_t dsmem[];
    const uint32_t sbase = smem_u32(dsmem);
    if (sbase & 1023u) {
        // the swizzled tiles need a 1024-byte aligned base and there is no room to
        // realign at two CTAs per SM: refuse before touching anything
        if (threadIdx.x == 0) watchdog_fire(SITE_FWD_ALIGN);
        return;
    }

    uint64_t *bars = reinterpret_cast<uint64_t *>(dsmem + T::OFF_BAR);
    const uint32_t b_q_full = smem_u32(&bars[0]);    // the item's Q tiles landed
    const uint32_t b_q_empty = smem_u32(&bars[1]);   // the item's last Q K^T done
    auto b_k_full = [&](int st) { return smem_u32(&bars[2 + st]); };
    auto b_k_empty = [&](int st) { return smem_u32(&bars[2 + KVS + st]); };
    auto b_v_full = [&](int st) { return smem_u32(&bars[2 + 2 * KVS + st]); };
    auto b_v_empty = [&](int st) { return smem_u32(&bars[2 + 3 * KVS + st]); };
    constexpr int OBB = 2 + 4 * KVS;
    auto b_bias_full = [&](int x) { return smem_u32(&bars[OBB + x]); };            // landed
    auto b_bias_ready = [&](int x) { return smem_u32(&bars[OBB + BS + x]); };      // folded
    auto b_bias_empty = [&](int x) { return smem_u32(&bars[OBB + 2 * BS + x]); };
    constexpr int OB = OBB + 3 * BS;
    const uint32_t b_s_full = smem_u32(&bars[OB + 0]);   // Q K^T in S
    const uint32_t b_s_free = smem_u32(&bars[OB + 1]);   // S read out
    const uint32_t b_p_full = smem_u32(&bars[OB + 2]);   // P in TMEM, O rescaled
    const uint32_t b_p_free = smem_u32(&bars[OB + 3]);   // P V done
    const uint32_t b_ofinal = smem_u32(&bars[OB + 4]);   // every P V of the item done
    const uint32_t b_drain = smem_u32(&bars[OB + 5]);    // abort path
    uint32_t *s_tmem_base = reinterpret_cast<uint32_t *>(dsmem + T::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(dsmem + T::OFF_MISC + 4);

    const int warp = warp_id(), lane = lane_id();
    const bool row_mask = a.mask != nullptr && !a.mask_shared;
    // item n of this CTA is blockIdx.x + n gridDim.x: query tile fastest, then the head, then
    // the chunk of rows.  CTAs running at the same time share K/V tiles in L2, and they cover
    // every head of the rows they read: one 128-byte line of Q, K, V or the gate holds the
    // channels of several heads (c = 32: 64 bytes per head), so with the heads apart in time
    // each line would be fetched from DRAM once per head that reads it.
    struct FItem {
        int h, i0, b0, nb;
        int jlo, nj;   // the item's key tiles [jlo, jlo + nj)
    };
    auto item = [&](int n) {
        int idx = blockIdx.x + n * gridDim.x;
        const int itile = idx % a.nI;
        idx /= a.nI;
        FItem it;
        it.h = idx % a.H;
        const int chunk = idx / a.H;
        it.i0 = itile * 128;
        it.b0 = chunk * BC;
        it.nb = min(BC, a.B - it.b0);
        it.jlo = a.win < 0 ? 0 : max(0, itile - a.win);
        it.nj = (a.win < 0 ? a.nJ : min(a.nJ, itile + a.win + 1)) - it.jlo;   // >= 1 (host check)
        return it;
    };
    const int n_items = (int)blockIdx.x < a.items ? (a.items - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    // steps of an item: (key tile jlo + j, row s), local index j * nb + s; k below is the
    // CTA's step count

    if (threadIdx.x == 0) {
        mbar_init(b_q_full, 1);
        mbar_init(b_q_empty, 1);
        for (int st = 0; st < KVS; ++st) {
            mbar_init(b_k_full(st), 1);
            mbar_init(b_k_empty(st), 1);
            mbar_init(b_v_full(st), 1);
            mbar_init(b_v_empty(st), 1);
        }
        for (int x = 0; x < BS; ++x) {
            mbar_init(b_bias_full(x), 1);
            mbar_init(b_bias_ready(x), 32);
            mbar_init(b_bias_empty(x), 128);
        }
        mbar_init(b_s_full, 1);
        mbar_init(b_s_free, 128);
        mbar_init(b_p_full, 128);
        mbar_init(b_p_free, 1);
        mbar_init(b_ofinal, 1);
        mbar_init(b_drain, 2);   // one commit from each issuer
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 5) {
        tmem_alloc(smem_u32(s_tmem_base), T::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *s_tmem_base;

    // K loads issued for steps [0, k_done), V loads for [0, v_done), bias tiles
    // [0, n_bias), Q for items [0, q_done): what has to land before the CTA may exit after
    // an abort
    int k_done = 0, v_done = 0, n_bias = 0, q_done = 0;

    if (warp >= 4) reg_dealloc<T::REGS_OTHER>();   // the whole second warpgroup, same point
    if (warp == 4) {
        // ------------------------------------------------------------------ producer
        if (lane == 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            if (a.has_bias) tma_prefetch_desc(&tmBias);
        }
        // Load order of an item: B(0), K(0), the item's Q tiles (once the previous item's
        // last Q K^T is done), then for every step k: K(k + 1), V(k), and the bias tile of
        // the next key tile once step k + 1 starts one.  K runs a step ahead of V; a bias
        // tile (which waits for the softmax to leave the buffer's previous tile) comes
        // after the V loads whose mask words that softmax may be waiting for.
        auto load_bias = [&](int jg, int j, const FItem &it) -> bool {
            const int bs = jg % BS;
            bool ok = true;
            if (jg >= BS)
                ok = mbar_wait(b_bias_empty(bs), ((jg / BS) - 1) & 1, abort_flag,
                               SITE_FWD_PROD | 0x20 | (jg << 12));
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) return false;
            if (lane == 0) {
                if (a.has_bias) {
                    const uint32_t dst = sbase + T::OFF_BIAS + bs * T::BIAS_BYTES;
                    mbar_arrive_tx(b_bias_full(bs), T::BIAS_BYTES);
                    tma_load_3d(dst, &tmBias, b_bias_full(bs), j * 128, it.i0, it.h);
                    tma_load_3d(dst + 16384, &tmBias, b_bias_full(bs), j * 128 + 64, it.i0, it.h);
                } else {
                    mbar_arrive(b_bias_full(bs));   // buffer free: the fold warps build it
                }
            }
            n_bias = jg + 1;
            return true;
        };
        auto load_q = [&](int n, const FItem &it) -> bool {
            bool ok = true;
            if (n >= 1) ok = mbar_wait(b_q_empty, (n - 1) & 1, abort_flag, SITE_FWD_PROD | 0x30 | (n << 12));
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) return false;
            if (lane == 0) {
                mbar_arrive_tx(b_q_full, it.nb * T::TILE_BYTES);
                for (int s = 0; s < it.nb; ++s)
                    tma_load_4d(sbase + T::OFF_Q + s * T::TILE_BYTES, &tmQ, b_q_full, 0, it.h, it.i0, it.b0 + s);
            }
            q_done = n + 1;
            return true;
        };
        auto load_k = [&](int k, int kl, const FItem &it) -> bool {
            const int st = k % KVS, use = k / KVS;
            bool ok = true;
            if (use >= 1)
                ok = mbar_wait(b_k_empty(st), (use - 1) & 1, abort_flag, SITE_FWD_PROD | (k << 12));
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) return false;
            if (lane == 0 && k != a.skip_step) {
                mbar_arrive_tx(b_k_full(st), T::TILE_BYTES);
                tma_load_4d(sbase + T::OFF_K + st * T::TILE_BYTES, &tmK, b_k_full(st), 0, it.h,
                            (it.jlo + kl / it.nb) * 128, it.b0 + kl % it.nb);
            }
            k_done = k + 1;
            return true;
        };
        auto load_v = [&](int k, int kl, const FItem &it) -> bool {
            const int st = k % KVS, use = k / KVS;
            bool ok = true;
            if (use >= 1)
                ok = mbar_wait(b_v_empty(st), (use - 1) & 1, abort_flag, SITE_FWD_PROD | 0x10 | (k << 12));
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) return false;
            const int j = it.jlo + kl / it.nb, b = it.b0 + kl % it.nb;
            if (row_mask) {
                // words of row b: word q bit t <-> key 128 j + 32 q + t attended
                uint32_t w[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int key = j * 128 + q * 32 + lane;
                    const bool valid = key < a.Nk && a.mask[(long long)b * a.smask_b + key] != 0;
                    w[q] = __ballot_sync(0xffffffffu, valid);
                }
                if (lane == 0) {
                    uint32_t *mw = reinterpret_cast<uint32_t *>(dsmem + T::OFF_MASK) + st * 8;
                    mw[0] = w[0];
                    mw[1] = w[1];
                    mw[2] = w[2];
                    mw[3] = w[3];
                    mw[4] = (w[0] & w[1] & w[2] & w[3]) == 0xffffffffu;
                }
            }
            if (lane == 0) {
                mbar_arrive_tx(b_v_full(st), T::TILE_BYTES);
                tma_load_4d(sbase + T::OFF_V + st * T::TILE_BYTES, &tmV, b_v_full(st), 0, it.h, j * 128, b);
            }
            v_done = k + 1;
            return true;
        };
        bool ok = true;
        int kg = 0, jg = 0;   // the CTA's steps and bias tiles before this item
        for (int n = 0; n < n_items && ok; ++n) {
            const FItem it = item(n);
            const int Kn = it.nj * it.nb;
            ok = load_bias(jg, it.jlo, it) && load_k(kg, 0, it) && load_q(n, it);
            for (int kl = 0; kl < Kn && ok; ++kl) {
                if (kl + 1 < Kn) ok = load_k(kg + kl + 1, kl + 1, it);
                if (ok) ok = load_v(kg + kl, kl, it);
                if (ok && kl + 1 < Kn && (kl + 1) % it.nb == 0)
                    ok = load_bias(jg + (kl + 1) / it.nb, it.jlo + (kl + 1) / it.nb, it);
            }
            kg += Kn;
            jg += it.nj;
        }
    } else if (warp == 5) {
        // ------------------------------------------------------------------ Q K^T issuer
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16(128, 128, false, false);
            constexpr uint32_t SBO = 8 * T::ROWB;
            bool ok = true;
            int kg = 0;
            for (int n = 0; n < n_items && ok; ++n) {
                const FItem it = item(n);
                const int nb = it.nb, Kn = it.nj * nb;
                ok = mbar_wait(b_q_full, n & 1, abort_flag, SITE_FWD_MMA | 0x50 | (n << 12));
                // step k: S must have been read out by the softmax of step k - 1
                for (int kl = 0; kl < Kn && ok; ++kl) {
                    const int k = kg + kl, s = kl % nb, st = k % KVS;
                    ok = mbar_wait_all(abort_flag, b_s_free, (k - 1) & 1, k > 0, SITE_FWD_MMA | 0x20 | (k << 12),
                                       b_k_full(st), (k / KVS) & 1, true, SITE_FWD_MMA | 0x10 | (k << 12));
                    if (!ok) break;
                    tc_fence_after();
                    const uint64_t dq = sdesc(sbase + T::OFF_Q + s * T::TILE_BYTES, 16, SBO, T::SWZ);
                    const uint64_t dk = sdesc(sbase + T::OFF_K + st * T::TILE_BYTES, 16, SBO, T::SWZ);
#pragma unroll
                    for (int kk = 0; kk < CP / 16; ++kk)   // K steps of 16 channels: 32 bytes on
                        umma_ss(tbase + T::T_S, sdesc_add(dq, kk * 32), sdesc_add(dk, kk * 32), idesc_qk,
                                kk > 0 ? 1u : 0u);
                    umma_commit(b_s_full);
                    umma_commit(b_k_empty(st));
                    if (kl == Kn - 1) umma_commit(b_q_empty);   // the next item's Q may load
                }
                kg += Kn;
            }
        }
    } else if (warp == 6) {
        // ------------------------------------------------------------------ P V issuer
        if (lane == 0) {
            constexpr uint32_t idesc_pv = idesc_bf16(128, CP, false, true);
            constexpr uint32_t SBO = 8 * T::ROWB;
            bool ok = true;
            int kg = 0;
            for (int n = 0; n < n_items && ok; ++n) {
                const FItem it = item(n);
                const int nb = it.nb, Kn = it.nj * nb;
                // step k: P of step k written (and O[s] rescaled) by the softmax, V landed
                for (int kl = 0; kl < Kn && ok; ++kl) {
                    const int k = kg + kl, j = kl / nb, s = kl % nb, st = k % KVS;
                    ok = mbar_wait_all(abort_flag, b_p_full, k & 1, true, SITE_FWD_MMA | 0x30 | (k << 12),
                                       b_v_full(st), (k / KVS) & 1, true, SITE_FWD_MMA | 0x40 | (k << 12));
                    if (!ok) break;
                    tc_fence_after();
                    const uint64_t dv = sdesc(sbase + T::OFF_V + st * T::TILE_BYTES, T::TILE_BYTES, SBO, T::SWZ);
                    const uint32_t d = tbase + T::T_O + s * CP;
                    // K steps of 16 keys: P advances 8 TMEM columns, V 16 rows
                    umma_ts(d, tbase + T::T_P, dv, idesc_pv, j > 0 ? 1u : 0u);
#pragma unroll
                    for (int kk = 1; kk < 8; ++kk)
                        umma_ts(d, tbase + T::T_P + kk * 8, sdesc_add(dv, kk * 16 * T::ROWB), idesc_pv, 1u);
                    umma_commit(b_p_free);
                    umma_commit(b_v_empty(st));
                }
                if (ok) umma_commit(b_ofinal);
                kg += Kn;
            }
        }
    } else if (warp == 7) {
        // ------------------------------------------------------------------ mask fold
        const int t = lane;   // rows t, t + 32, t + 64, t + 96 of every bias tile
        bool ok = true;
        int jg = 0;   // the CTA's bias tiles
        for (int n = 0; n < n_items && ok; ++n) {
            const FItem it = item(n);
            for (int jl = 0; jl < it.nj && ok; ++jl, ++jg) {
                const int bs = jg % BS, j = it.jlo + jl;
                // word q bit l <-> key 128 j + 32 q + l attended by every row of the chunk
                uint32_t w[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int key = j * 128 + q * 32 + lane;
                    bool valid = key < a.Nk;
                    if (valid && a.mask && !row_mask) valid = a.mask[key] != 0;
                    w[q] = __ballot_sync(0xffffffffu, valid);
                }
                ok = mbar_wait(b_bias_full(bs), (jg / BS) & 1, abort_flag, SITE_FWD_FOLD | (jg << 12));
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                uint8_t *tile = dsmem + T::OFF_BIAS + bs * T::BIAS_BYTES;
                if (a.has_bias) {
                    if ((w[0] & w[1] & w[2] & w[3]) != 0xffffffffu) {
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            uint32_t m = ~w[q];
                            while (m) {
                                const int c = q * 32 + __ffs(m) - 1;
                                m &= m - 1;
#pragma unroll
                                for (int r = t; r < 128; r += 32)
                                    *reinterpret_cast<uint16_t *>(tile + bias_off(r, c)) = 0xFF80u;
                            }
                        }
                    }
                } else {
                    // no bias: 0 for attended keys, -inf for the rest
#pragma unroll 1
                    for (int ch = 0; ch < 16; ++ch) {   // 16-byte chunk ch: keys 8 ch .. 8 ch + 7
                        const int qw = ch >> 2;
                        const uint32_t wq = qw == 0 ? w[0] : qw == 1 ? w[1] : qw == 2 ? w[2] : w[3];
                        const uint32_t bits = wq >> ((ch & 3) * 8);
                        uint32_t v4[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const uint32_t lo = ((bits >> (2 * e)) & 1u) ? 0u : 0xFF80u;
                            const uint32_t hi = ((bits >> (2 * e + 1)) & 1u) ? 0u : 0xFF80u;
                            v4[e] = lo | (hi << 16);
                        }
                        const uint4 val = make_uint4(v4[0], v4[1], v4[2], v4[3]);
                        const uint32_t tb = sbase + T::OFF_BIAS + bs * T::BIAS_BYTES;
#pragma unroll
                        for (int r = t; r < 128; r += 32) sts128(tb + bias_off(r, ch * 8), val);
                    }
                }
                // these generic writes precede a later TMA refill of the same buffer
                fence_proxy_async();
                mbar_arrive(b_bias_ready(bs));
            }
        }
    } else {
        // ------------------------------------------------------------------ softmax
        reg_alloc<T::REGS_SOFTMAX>();
        const int row = warp * 32 + lane;
        const uint32_t lane_off = ((uint32_t)(warp * 32)) << 16;
        const uint32_t tS = tbase + T::T_S + lane_off;
        const uint32_t tP = tbase + T::T_P + lane_off;
        const float2 sc2 = make_float2(a.scale, a.scale);
        const float2 l2e2 = make_float2(kLog2e, kLog2e);
        bool ok = true;
        int k = 0, jg = 0;   // the CTA's steps and bias tiles before this one
        for (int n = 0; n < n_items && ok; ++n) {
            const FItem it = item(n);
            const int nb = it.nb;
            float m_run[BC], l_run[BC];   // running (max, sum) of this row in every slot
#pragma unroll
            for (int t = 0; t < BC; ++t) {
                m_run[t] = -INFINITY;
                l_run[t] = 0.f;
            }
            // the epilogue's gate rows: into L2 now, so that their loads after the item's
            // last step do not wait for DRAM
            if (a.gate && it.i0 + row < a.Nq) {
#pragma unroll
                for (int t = 0; t < BC; ++t)
                    if (t < nb)
                        prefetch_l2(a.gate + (it.b0 + t) * a.sg0 + (long long)(it.i0 + row) * a.sg1 +
                                    it.h * a.sg2);
            }
            for (int j = 0; j < it.nj && ok; ++j, ++jg) {   // j: the item's key tile jlo + j
                const int bs = jg % BS;
                for (int s = 0; s < nb; ++s, ++k) {
                    const int st = k % KVS;
                    // S of the step, the folded bias tile at a tile's first row, and with
                    // per-row masks the step's V stage (its mask words come with it): probed
                    // together
                    ok = mbar_wait_all(abort_flag, b_s_full, k & 1, true, SITE_FWD_SOFTMAX | (k << 12),
                                       b_bias_ready(bs), (jg / BS) & 1, s == 0, SITE_FWD_SOFTMAX | 0x10 | (k << 12),
                                       b_v_full(st), (k / KVS) & 1, row_mask, SITE_FWD_SOFTMAX | 0x20 | (k << 12));
                    ok = __all_sync(0xffffffffu, ok);
                    if (!ok) break;
                    tc_fence_after();

                    // the first half of this row's bias words: their shared-memory loads are in
                    // flight while the TMEM load of S below waits
                    const uint32_t bias_row = sbase + T::OFF_BIAS + bs * T::BIAS_BYTES + row * 128;
                    uint4 bw0[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q) bw0[q] = lds128(bias_row + (((q & 7) ^ (row & 7)) << 4));

                    // S of this row, then hand the S columns back for the next Q K^T
                    uint32_t xr[128];
                    tmem_ld128(tS, xr);
                    tc_fence_before();
                    mbar_arrive(b_s_free);
                    // the second half's bias words, all issued before any of them is used
                    uint4 bw1[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q) bw1[q] = lds128(bias_row + 16384 + ((q ^ (row & 7)) << 4));

                    // logits in place: x = scale * S + bias (natural-log units; -inf if masked)
                    {
#pragma unroll
                        for (int q = 0; q < 16; ++q) {  // 16-byte chunk q holds keys 8q .. 8q+7
                            const uint4 bw = q < 8 ? bw0[q & 7] : bw1[q & 7];
                            const uint32_t bb[4] = {bw.x, bw.y, bw.z, bw.w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int c = q * 8 + 2 * e;
                                const float2 v = ffma2(make_float2(__uint_as_float(xr[c]), __uint_as_float(xr[c + 1])),
                                                       sc2, make_float2(bf16lo(bb[e]), bf16hi(bb[e])));
                                xr[c] = __float_as_uint(v.x);
                                xr[c + 1] = __float_as_uint(v.y);
                            }
                        }
                    }
                    if (s == nb - 1) mbar_arrive(b_bias_empty(bs));   // last reader of the tile
                    float *x = reinterpret_cast<float *>(xr);
                    if (row_mask) {
                        const uint32_t *mw = reinterpret_cast<const uint32_t *>(dsmem + T::OFF_MASK) + st * 8;
                        if (mw[4] == 0u) {
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                const uint32_t wd = mw[q];
#pragma unroll
                                for (int t = 0; t < 32; ++t)
                                    if (!((wd >> t) & 1u)) x[q * 32 + t] = -INFINITY;
                            }
                        }
                    }
                    // row maximum: four independent chains of three-input max
                    float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                    for (int c = 0; c < 128; c += 8) {
                        m4[0] = max3(m4[0], x[c], x[c + 1]);
                        m4[1] = max3(m4[1], x[c + 2], x[c + 3]);
                        m4[2] = max3(m4[2], x[c + 4], x[c + 5]);
                        m4[3] = max3(m4[3], x[c + 6], x[c + 7]);
                    }
                    const float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));

                    float m_use = m_run[0], l_prev = l_run[0];
#pragma unroll
                    for (int t = 1; t < BC; ++t)
                        if (s == t) {
                            m_use = m_run[t];
                            l_prev = l_run[t];
                        }
                    float alpha = 1.f;
                    bool resc = false;
                    if (j == 0) {
                        m_use = mx;
                        l_prev = 0.f;
                    } else if (mx > m_use + kRescaleThresh) {
                        alpha = (m_use == -INFINITY) ? 0.f : ex2((m_use - mx) * kLog2e);
                        m_use = mx;
                        resc = true;
                    }
                    const float nm = (m_use == -INFINITY) ? 0.f : -m_use * kLog2e;
                    const float2 nm2 = make_float2(nm, nm);

                    // The exponentials go into registers first: only the store of P (and a
                    // rescale of O[s]) has to wait for the previous P V, so the exponential
                    // unit's share of the step overlaps that product instead of following it.
                    // P and O[s] may only be written once the previous P V is done: probe that
                    // now, so the probe's latency overlaps the exponentials (a phase found
                    // complete stays complete: the next one needs this step's P)
                    const bool pv_done = k == 0 || mbar_test(b_p_free, (k - 1) & 1);
                    float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
                    uint32_t p0[32], p1[32];   // P of keys 0..63 and 64..127 as bf16 pairs
#pragma unroll
                    for (int c = 0; c < 64; ++c) {
                        const float2 tt = ffma2(make_float2(x[2 * c], x[2 * c + 1]), l2e2, nm2);
                        const float2 pv = make_float2(ex2(tt.x), ex2(tt.y));
                        if (c & 1) acc1 = fadd2(acc1, pv);
                        else acc0 = fadd2(acc0, pv);
                        if (c < 32) p0[c] = pack_bf16x2(pv.x, pv.y);
                        else p1[c - 32] = pack_bf16x2(pv.x, pv.y);
                    }
                    const float sum = (acc0.x + acc0.y) + (acc1.x + acc1.y);
                    if (!__all_sync(0xffffffffu, pv_done)) {
                        ok = mbar_wait(b_p_free, (k - 1) & 1, abort_flag, SITE_FWD_SOFTMAX | 0x30 | (k << 12));
                        ok = __all_sync(0xffffffffu, ok);
                        if (!ok) break;
                    }
                    tc_fence_after();
                    tmem_st32(tP, p0);
                    tmem_st32(tP + 32, p1);
                    if (__any_sync(0xffffffffu, resc)) {
                        const uint32_t tO = tbase + T::T_O + s * CP + lane_off;
                        uint32_t o[CP];
                        tmem_ld_cols<CP>(tO, o);
#pragma unroll
                        for (int c = 0; c < CP; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
                        tmem_st_cols<CP>(tO, o);
                    }
                    tmem_wait_st();
                    const float l_new = l_prev * alpha + sum;
#pragma unroll
                    for (int t = 0; t < BC; ++t)
                        if (s == t) {
                            m_run[t] = m_use;
                            l_run[t] = l_new;
                        }
                    tc_fence_before();
                    mbar_arrive(b_p_full);
                }
            }
            // ------------------------------------------------------------------ epilogue
            // The gate does not depend on O: fetch it for all slots before waiting for the
            // last P V products, so its latency overlaps theirs.
            uint4 gw[BC][CP / 8];
            const int i = it.i0 + row;
            const bool row_ok = i < a.Nq;
#pragma unroll
            for (int t = 0; t < BC; ++t) {
#pragma unroll
                for (int c8 = 0; c8 < CP / 8; ++c8) {
                    gw[t][c8] = make_uint4(0, 0, 0, 0);
                    if (ok && a.gate && row_ok && t < nb && c8 * 8 < a.C)
                        gw[t][c8] = *reinterpret_cast<const uint4 *>(
                            a.gate + (it.b0 + t) * a.sg0 + (long long)i * a.sg1 + it.h * a.sg2 + c8 * 8);
                }
            }
            if (ok) {
                ok = mbar_wait(b_ofinal, n & 1, abort_flag, SITE_FWD_EPI | (n << 12));
                ok = __all_sync(0xffffffffu, ok);
            }
            if (ok) {
                tc_fence_after();
#pragma unroll
                for (int t = 0; t < BC; ++t) {
                    if (t >= nb) break;
                    uint32_t o[CP];
                    tmem_ld_cols<CP>(tbase + T::T_O + t * CP + lane_off, o);
                    if (!row_ok) continue;
                    const int b = it.b0 + t;
                    const bool live = l_run[t] > 0.f;
                    const float inv = live ? rcp_approx(l_run[t]) : 0.f;
                    __nv_bfloat16 *op = a.out + b * a.so0 + (long long)i * a.so1 + it.h * a.so2;
#pragma unroll
                    for (int c8 = 0; c8 < CP / 8; ++c8) {
                        if (c8 * 8 < a.C) {
                            const uint32_t g4[4] = {gw[t][c8].x, gw[t][c8].y, gw[t][c8].z, gw[t][c8].w};
                            uint32_t ow[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                float lo = __uint_as_float(o[c8 * 8 + 2 * e]) * inv;
                                float hi = __uint_as_float(o[c8 * 8 + 2 * e + 1]) * inv;
                                if (a.gate) {
                                    lo *= sigmoid_fast(bf16lo(g4[e]));
                                    hi *= sigmoid_fast(bf16hi(g4[e]));
                                }
                                ow[e] = pack_bf16x2(lo, hi);
                            }
                            *reinterpret_cast<uint4 *>(op + c8 * 8) = make_uint4(ow[0], ow[1], ow[2], ow[3]);
                        }
                    }
                    a.lse[((long long)b * a.H + it.h) * a.Nq + i] =
                        live ? m_run[t] + lg2_approx(l_run[t]) * 0.6931471805599453f : -INFINITY;
                }
            }
        }
    }

    // ---------------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (*abort_flag) {
        // Some wait ran out.  Every role has stopped; before shared memory and TMEM are
        // released, let the copies and MMAs already issued finish (bounded waits).
        if (warp == 4 && lane == 0) {
            if (q_done > 0) mbar_wait_drain(b_q_full, (q_done - 1) & 1);
            for (int kk = max(0, k_done - KVS); kk < k_done; ++kk)
                if (kk != a.skip_step) mbar_wait_drain(b_k_full(kk % KVS), (kk / KVS) & 1);
            for (int kk = max(0, v_done - KVS); kk < v_done; ++kk)
                mbar_wait_drain(b_v_full(kk % KVS), (kk / KVS) & 1);
            for (int jj = max(0, n_bias - BS); jj < n_bias; ++jj)
                mbar_wait_drain(b_bias_full(jj % BS), (jj / BS) & 1);
        }
        if ((warp == 5 || warp == 6) && lane == 0) {
            umma_commit(b_drain);   // each issuer's own MMAs
            mbar_wait_drain(b_drain, 0);
        }
        tc_fence_before();
        __syncthreads();
    }
    if (warp == 5) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tbase, T::TMEM_COLS);
    }
}

}  // namespace pba
