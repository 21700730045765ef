// Forward kernel: out = sigmoid(G) * softmax(scale * Q K^T + bias + mask) V, and the
// logsumexp of every query row.
//
// Pair-biased attention as described on the "AlphaFold3 open-source implementation" page,
// Model Efficiency section: the pair bias is added after the key-query dot product and
// is shared by every broadcast row b (triangle rows, MSA sequences, diffusion copies).
//
// Work item = (head h, 128-query tile, chunk of BC = 128 / CP broadcast rows: 8, 4 or 2).
// The kernel is persistent, one CTA per SM walking the items blockIdx.x, blockIdx.x +
// gridDim.x, ... with one pipeline that runs across item boundaries (every ring and barrier
// counts steps and tiles of the CTA, not of the item).  Within an item the loop runs over
// key tiles j (outer) and the chunk's rows b (inner, "slots" s = 0 .. BC - 1): each
// 128 x 128 bias tile is moved into shared memory once and reused by all BC rows.
//
// The softmax is done by two row groups: group g takes the slots s with s & 1 == g, so
// the two groups alternate on the tensor core (one group's exponentials run while the
// other group's P V and next Q K^T do).  Each group is two warpgroups, one per 64-key half
// of the score tile (thread = query row = TMEM lane, 64 scores each): sixteen softmax warps,
// four per SM sub-partition, keep the exponential unit fed.  The two halves of a row agree
// on the running maximum through shared memory at every step and add their partial row
// sums at the end of the item.
//
// Warp roles (640 threads):
//   warps 0-15  softmax and epilogue: group g = warp / 8, key half e = (warp / 4) % 2
//   warp 16     TMA producer (Q, K, V, bias tiles) and per-row key-mask words
//   warp 17     TMEM allocator and, on lane 0, the MMA issuer of row group 0
//   warp 18     lane 0: the MMA issuer of row group 1
//   warp 19     folds the key mask into each bias tile (masked keys -> -inf), or builds the
//               tile when there is no bias, so the softmax never tests mask bits
// One thread issues a tcgen05.mma only every ~200 cycles whatever its shape (measured: M =
// 128, K = 16, N = 32 to 256), while separate issuing threads proceed at that rate each, so
// each row group has its own issuer: Q K^T of the group's step, then P V of its previous
// step.  Each group also has its own K and V rings, consumed in order by its issuer only
// (a ring shared by two independent issuers could see one of them run a full ring ahead of
// the other, where a parity wait passes on the wrong phase).  The last warpgroup hands
// registers to the softmax warpgroups through setmaxnreg.
//
// Tensor memory (512 columns): S of group g at [128 g, 128 g + 128), P of group g (packed
// bf16) at [256 + 64 g, 320 + 64 g), then one CP-column fp32 O accumulator per slot at
// [384 + CP s, ...).  S and P are separate, so a group's next Q K^T runs while its softmax
// turns the current S into P.
#pragma once

#include "pba_device.cuh"

namespace pba {

struct FwdArgs {
    int B, H, Nq, Nk, C;
    int nI, nJ, nChunks;
    int items;       // H * nI * nChunks work items, walked by a grid of at most one CTA per SM
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
    static constexpr int BC = 128 / CP;                        // rows b per item (O slots)
    static constexpr int SPG = BC / 2;                         // slots per row group
    static constexpr int KVG = (CP == 64) ? 1 : 2;             // K and V stages of each row group's rings
    static constexpr int BS = 2;                               // bias tile buffers
    static constexpr int TILE_BYTES = 128 * CP * 2;            // Q, K or V tile
    static constexpr int BIAS_BYTES = 128 * 128 * 2;           // two 64-key halves
    static constexpr int OFF_BIAS = 0;                         // 1024-byte aligned (SW128)
    static constexpr int OFF_Q = OFF_BIAS + BS * BIAS_BYTES;   // + s * TILE_BYTES
    static constexpr int OFF_K = OFF_Q + BC * TILE_BYTES;      // + (g KVG + st) * TILE_BYTES
    static constexpr int OFF_V = OFF_K + 2 * KVG * TILE_BYTES; // + (g KVG + st) * TILE_BYTES
    static constexpr int OFF_MASK = OFF_V + 2 * KVG * TILE_BYTES;  // u32 [2][KVG][8] per-row words (V rings)
    // row-statistics exchange between the two key halves: float [group][parity][half][SPG][128]
    static constexpr int OFF_X = OFF_MASK + 2 * KVG * 32;
    static constexpr int X_GROUP = 2 * 2 * SPG * 128;          // floats per group
    // barriers
    static constexpr int B_QF = 0, B_QE = BC, B_KF = 2 * BC, B_KE = B_KF + 2 * KVG, B_VF = B_KE + 2 * KVG,
                         B_VE = B_VF + 2 * KVG, B_BF = B_VE + 2 * KVG, B_BR = B_BF + BS, B_BE = B_BR + BS,
                         B_SF = B_BE + BS, B_SE = B_SF + 2, B_PF = B_SE + 2, B_PE = B_PF + 2,
                         B_OF = B_PE + 2, B_X = B_OF + 2, B_DRAIN = B_X + 16, NBAR = B_DRAIN + 1;
    static constexpr int OFF_BAR = OFF_X + 2 * X_GROUP * 4;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;        // TMEM base, abort flag
    static constexpr int SMEM_BYTES = OFF_MISC + 16;
    static constexpr int SMEM_LAUNCH = SMEM_BYTES + 1024;      // room to align the base to 1 KB
    static constexpr uint32_t SWZ = CP == 64 ? kSw128 : (CP == 32 ? kSw64 : kSw32);
    static constexpr uint32_t ROWB = CP * 2;                   // bytes per tile row
    static constexpr int THREADS = 640;
    static constexpr int W_PROD = 16, W_ISS0 = 17, W_ISS1 = 18, W_FOLD = 19;
    // register split through setmaxnreg: 512 x 104 + 128 x 64 = 640 x 96, the registers the
    // CTA is launched with (the build checks that ptxas reports 96)
    static constexpr int REGS_SOFTMAX = 104;
    static constexpr int REGS_OTHER = 64;
    static constexpr int TMEM_COLS = 512;
    static constexpr uint32_t T_S = 0, T_P = 256, T_O = 384;
    static_assert(T_O + BC * CP <= 512, "TMEM");
};
static_assert(FwdTraits<16>::SMEM_LAUNCH <= 232448, "smem");
static_assert(FwdTraits<32>::SMEM_LAUNCH <= 232448, "smem");
static_assert(FwdTraits<64>::SMEM_LAUNCH <= 232448, "smem");
static_assert(512 * FwdTraits<32>::REGS_SOFTMAX + 128 * FwdTraits<32>::REGS_OTHER == 640 * 96, "regs");

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
__global__ void __launch_bounds__(640, 1)
pba_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV,
               const __grid_constant__ CUtensorMap tmBias, const FwdArgs a) {
    using T = FwdTraits<CP>;
    constexpr int KVG = T::KVG, BS = T::BS, BC = T::BC, SPG = T::SPG;
    extern __shared__ uint8_t dsmem[];
    const uint32_t raw = smem_u32(dsmem);
    const uint32_t sbase = (raw + 1023u) & ~1023u;   // the swizzled tiles need 1 KB alignment
    uint8_t *gbase = dsmem + (sbase - raw);

    uint64_t *bars = reinterpret_cast<uint64_t *>(gbase + T::OFF_BAR);
    auto bar = [&](int i) { return smem_u32(&bars[i]); };
    auto b_q_full = [&](int s) { return bar(T::B_QF + s); };    // slot s's Q tile landed
    auto b_q_empty = [&](int s) { return bar(T::B_QE + s); };   // slot s's last Q K^T done
    // K and V rings of row group g, stage st
    auto b_k_full = [&](int g, int st) { return bar(T::B_KF + g * KVG + st); };
    auto b_k_empty = [&](int g, int st) { return bar(T::B_KE + g * KVG + st); };
    auto b_v_full = [&](int g, int st) { return bar(T::B_VF + g * KVG + st); };
    auto b_v_empty = [&](int g, int st) { return bar(T::B_VE + g * KVG + st); };
    auto b_bias_full = [&](int x) { return bar(T::B_BF + x); };    // landed
    auto b_bias_ready = [&](int x) { return bar(T::B_BR + x); };   // folded
    auto b_bias_empty = [&](int x) { return bar(T::B_BE + x); };
    auto b_s_full = [&](int g) { return bar(T::B_SF + g); };      // Q K^T in S of group g
    auto b_s_free = [&](int g) { return bar(T::B_SE + g); };      // S of group g read out
    auto b_p_full = [&](int g) { return bar(T::B_PF + g); };      // P of group g in TMEM, O rescaled
    auto b_p_free = [&](int g) { return bar(T::B_PE + g); };      // P V of group g done
    auto b_ofinal = [&](int g) { return bar(T::B_OF + g); };      // group g's P V of the item done
    const uint32_t b_drain = bar(T::B_DRAIN);                      // abort path
    uint32_t *s_tmem_base = reinterpret_cast<uint32_t *>(gbase + T::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(gbase + T::OFF_MISC + 4);

    const int warp = warp_id(), lane = lane_id();
    const bool row_mask = a.mask != nullptr && !a.mask_shared;
    // item n of this CTA is blockIdx.x + n gridDim.x: query tile fastest, then the chunk of
    // rows, then the head (CTAs running at the same time share K/V tiles in L2)
    struct FItem {
        int h, i0, b0, nb;
        int jlo, nj;   // the item's key tiles [jlo, jlo + nj)
    };
    auto item = [&](int n) {
        int idx = blockIdx.x + n * gridDim.x;
        const int itile = idx % a.nI;
        idx /= a.nI;
        const int chunk = idx % a.nChunks;
        FItem it;
        it.h = idx / a.nChunks;
        it.i0 = itile * 128;
        it.b0 = chunk * BC;
        it.nb = min(BC, a.B - it.b0);
        it.jlo = a.win < 0 ? 0 : max(0, itile - a.win);
        it.nj = (a.win < 0 ? a.nJ : min(a.nJ, itile + a.win + 1)) - it.jlo;   // >= 1 (host check)
        return it;
    };
    const int n_items = (int)blockIdx.x < a.items ? (a.items - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    // Steps of an item: (key tile jlo + j, slot s), local index j * nb + s, in this order in
    // every role; k below is the CTA's step count.  Step (j, s) belongs to row group s & 1.

    if (threadIdx.x == 0) {
        for (int s = 0; s < BC; ++s) {
            mbar_init(b_q_full(s), 1);
            mbar_init(b_q_empty(s), 1);
        }
        for (int g = 0; g < 2; ++g)
            for (int st = 0; st < KVG; ++st) {
                mbar_init(b_k_full(g, st), 1);
                mbar_init(b_k_empty(g, st), 1);
                mbar_init(b_v_full(g, st), 1);
                mbar_init(b_v_empty(g, st), 1);
            }
        for (int x = 0; x < BS; ++x) {
            mbar_init(b_bias_full(x), 1);
            mbar_init(b_bias_ready(x), 32);
            mbar_init(b_bias_empty(x), 512);   // every softmax thread, once per tile
        }
        for (int g = 0; g < 2; ++g) {
            mbar_init(b_s_full(g), 1);
            mbar_init(b_s_free(g), 256);
            mbar_init(b_p_full(g), 256);
            mbar_init(b_p_free(g), 1);
            mbar_init(b_ofinal(g), 1);
        }
        for (int x = 0; x < 16; ++x) mbar_init(bar(T::B_X + x), 64);   // the two warps of a row quad
        mbar_init(b_drain, 2);   // one commit from each group's issuer
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == T::W_ISS0) {
        tmem_alloc(smem_u32(s_tmem_base), T::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *s_tmem_base;

    // K loads issued for group g's steps [0, k_done[g]), V loads for [0, v_done[g]), bias
    // tiles [0, n_bias), q_loads[s] Q loads of slot s: what has to land before the CTA may
    // exit after an abort
    int k_done[2] = {0, 0}, v_done[2] = {0, 0}, n_bias = 0;
    int skipped_g = -1, skipped_gs = -1;   // the K load the test hook skipped (never lands)
    int q_loads[BC];
#pragma unroll
    for (int s = 0; s < BC; ++s) q_loads[s] = 0;

    if (warp >= 16) reg_dealloc<T::REGS_OTHER>();   // the whole last warpgroup, same point
    if (warp == T::W_PROD) {
        // ------------------------------------------------------------------ producer
        if (lane == 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            if (a.has_bias) tma_prefetch_desc(&tmBias);
        }
        // Load order of an item: B(0), K(0), the Q tile of every slot (each once the
        // previous item's last Q K^T on that slot is done), then for every step k:
        // K(k + 1), V(k), and the bias tile of the next key tile once step k + 1 starts
        // one.  K runs a step ahead of V; a bias tile (which waits for the softmax to leave
        // the buffer's previous tile) comes after the V loads whose mask words that softmax
        // may be waiting for.
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
                    mbar_arrive(b_bias_full(bs));   // buffer free: the fold warp builds it
                }
            }
            n_bias = jg + 1;
            return true;
        };
        auto load_q = [&](const FItem &it) -> bool {
            for (int s = 0; s < it.nb; ++s) {
                bool ok = true;
                if (q_loads[s] >= 1)
                    ok = mbar_wait(b_q_empty(s), (q_loads[s] - 1) & 1, abort_flag, SITE_FWD_PROD | 0x30 | (s << 12));
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) return false;
                if (lane == 0) {
                    mbar_arrive_tx(b_q_full(s), T::TILE_BYTES);
                    tma_load_4d(sbase + T::OFF_Q + s * T::TILE_BYTES, &tmQ, b_q_full(s), 0, it.h, it.i0, it.b0 + s);
                }
                ++q_loads[s];
            }
            return true;
        };
        // K and V of the CTA's step k (item step kl): into the ring of the step's row group g,
        // whose gs-th step it is
        auto load_k = [&](int k, int kl, const FItem &it, int g, int gs) -> bool {
            const int st = gs % KVG, use = gs / KVG;
            bool ok = true;
            if (use >= 1)
                ok = mbar_wait(b_k_empty(g, st), (use - 1) & 1, abort_flag, SITE_FWD_PROD | (k << 12));
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) return false;
            if (k == a.skip_step) {
                skipped_g = g;
                skipped_gs = gs;
            }
            if (lane == 0 && k != a.skip_step) {
                mbar_arrive_tx(b_k_full(g, st), T::TILE_BYTES);
                tma_load_4d(sbase + T::OFF_K + (g * KVG + st) * T::TILE_BYTES, &tmK, b_k_full(g, st), 0, it.h,
                            (it.jlo + kl / it.nb) * 128, it.b0 + kl % it.nb);
            }
            k_done[g] = gs + 1;
            return true;
        };
        auto load_v = [&](int k, int kl, const FItem &it, int g, int gs) -> bool {
            const int st = gs % KVG, use = gs / KVG;
            bool ok = true;
            if (use >= 1)
                ok = mbar_wait(b_v_empty(g, st), (use - 1) & 1, abort_flag, SITE_FWD_PROD | 0x10 | (k << 12));
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
                    uint32_t *mw = reinterpret_cast<uint32_t *>(gbase + T::OFF_MASK) + (g * KVG + st) * 8;
                    mw[0] = w[0];
                    mw[1] = w[1];
                    mw[2] = w[2];
                    mw[3] = w[3];
                }
            }
            if (lane == 0) {
                mbar_arrive_tx(b_v_full(g, st), T::TILE_BYTES);
                tma_load_4d(sbase + T::OFF_V + (g * KVG + st) * T::TILE_BYTES, &tmV, b_v_full(g, st), 0, it.h,
                            j * 128, b);
            }
            v_done[g] = gs + 1;
            return true;
        };
        bool ok = true;
        int kg = 0, jg = 0;    // the CTA's steps and bias tiles before this item
        int gs[2] = {0, 0};    // each row group's steps before this item
        for (int n = 0; n < n_items && ok; ++n) {
            const FItem it = item(n);
            const int nb = it.nb, Kn = it.nj * nb;
            // step kl of the item is row group (kl % nb) & 1's step number gs0[g] + (its
            // steps before kl): per key tile the group has (nb - g + 1) / 2 of them
            const int per_tile[2] = {(nb + 1) / 2, nb / 2};
            auto gstep = [&](int kl, int &g) {
                const int j = kl / nb, s = kl % nb;
                g = s & 1;
                return gs[g] + j * per_tile[g] + (s >> 1);
            };
            int g0;
            const int s0 = gstep(0, g0);
            ok = load_bias(jg, it.jlo, it) && load_k(kg, 0, it, g0, s0) && load_q(it);
            for (int kl = 0; kl < Kn && ok; ++kl) {
                int gn, gc;
                if (kl + 1 < Kn) {
                    const int sn = gstep(kl + 1, gn);
                    ok = load_k(kg + kl + 1, kl + 1, it, gn, sn);
                }
                const int sc = gstep(kl, gc);
                if (ok) ok = load_v(kg + kl, kl, it, gc, sc);
                if (ok && kl + 1 < Kn && (kl + 1) % nb == 0)
                    ok = load_bias(jg + (kl + 1) / nb, it.jlo + (kl + 1) / nb, it);
            }
            kg += Kn;
            jg += it.nj;
            gs[0] += it.nj * per_tile[0];
            gs[1] += it.nj * per_tile[1];
        }
    } else if (warp == T::W_ISS0 || warp == T::W_ISS1) {
        // ------------------------------------------------------------------ row group issuers
        // Row group g's issuer: Q K^T of each of the group's steps, then P V of the group's
        // previous step, so that a step's scores never wait behind the previous P V.
        if (lane == 0) {
            const int g = warp - T::W_ISS0;
            constexpr uint32_t idesc_qk = idesc_bf16(128, 128, false, false);
            constexpr uint32_t idesc_pv = idesc_bf16(128, CP, false, true);
            constexpr uint32_t SBO = 8 * T::ROWB;
            bool ok = true;
            int kg = 0;
            int gk = 0;   // the group's steps so far
            int quse[BC];
#pragma unroll
            for (int s = 0; s < BC; ++s) quse[s] = 0;
            struct Pend { int k, j, s, gk, nj, nb; };
            Pend pend;
            bool has_pend = false;
            // P V of the group's step pd: its P written (and O[s] rescaled) by the softmax,
            // its V landed; the group's last step of its item releases the epilogue
            auto issue_pv = [&](const Pend &pd) -> bool {
                const int st = pd.gk % KVG;
                bool okp = mbar_wait(b_p_full(g), pd.gk & 1, abort_flag, SITE_FWD_MMA | 0x30 | (pd.k << 12));
                if (okp) okp = mbar_wait(b_v_full(g, st), (pd.gk / KVG) & 1, abort_flag, SITE_FWD_MMA | 0x40 | (pd.k << 12));
                if (!okp) return false;
                tc_fence_after();
                const uint32_t va = sbase + T::OFF_V + (g * KVG + st) * T::TILE_BYTES;
                const uint32_t d = tbase + T::T_O + pd.s * CP;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    umma_ts(d, tbase + T::T_P + g * 64 + kk * 8,
                            sdesc(va + kk * 16 * T::ROWB, T::TILE_BYTES, SBO, T::SWZ), idesc_pv,
                            (pd.j > 0 || kk > 0) ? 1u : 0u);
                umma_commit(b_p_free(g));
                umma_commit(b_v_empty(g, st));
                if (pd.j == pd.nj - 1 && pd.s + 2 >= pd.nb) umma_commit(b_ofinal(g));
                return true;
            };
            for (int n = 0; n < n_items && ok; ++n) {
                const FItem it = item(n);
                const int nb = it.nb, Kn = it.nj * nb;
                if (nb <= g) {
                    // no row of this group in the item: its last P V goes out now (the
                    // group's epilogue waits for it, and this item's loads wait for that
                    // group to hand back the previous tiles)
                    if (has_pend) ok = issue_pv(pend);
                    has_pend = false;
                    kg += Kn;
                    continue;
                }
                for (int kl = 0; kl < Kn && ok; ++kl) {
                    const int k = kg + kl, j = kl / nb, s = kl % nb;
                    if ((s & 1) != g) continue;
                    const int st = gk % KVG;
                    // the group's S must have been read out by its previous step's softmax
                    if (gk > 0)
                        ok = mbar_wait(b_s_free(g), (gk - 1) & 1, abort_flag, SITE_FWD_MMA | 0x20 | (k << 12));
                    if (ok) ok = mbar_wait(b_k_full(g, st), (gk / KVG) & 1, abort_flag, SITE_FWD_MMA | 0x10 | (k << 12));
                    if (ok && j == 0)
                        ok = mbar_wait(b_q_full(s), quse[s] & 1, abort_flag, SITE_FWD_MMA | 0x50 | (k << 12));
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t qa = sbase + T::OFF_Q + s * T::TILE_BYTES;
                    const uint32_t ka = sbase + T::OFF_K + (g * KVG + st) * T::TILE_BYTES;
#pragma unroll
                    for (int kk = 0; kk < CP / 16; ++kk)
                        umma_ss(tbase + T::T_S + g * 128, sdesc(qa + kk * 32, 16, SBO, T::SWZ),
                                sdesc(ka + kk * 32, 16, SBO, T::SWZ), idesc_qk, kk > 0 ? 1u : 0u);
                    umma_commit(b_s_full(g));
                    umma_commit(b_k_empty(g, st));
                    if (j == it.nj - 1) umma_commit(b_q_empty(s));   // the next item's Q of slot s may load
                    if (has_pend) ok = issue_pv(pend);
                    pend = {k, j, s, gk, it.nj, nb};
                    has_pend = true;
                    ++gk;
                }
                for (int s = 0; s < nb; ++s) ++quse[s];
                kg += Kn;
            }
            if (ok && has_pend) issue_pv(pend);
        }
    } else if (warp == T::W_FOLD) {
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
                uint8_t *tile = gbase + T::OFF_BIAS + bs * T::BIAS_BYTES;
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
        const int g = warp >> 3, e = (warp >> 2) & 1, q4 = warp & 3;
        const int row = q4 * 32 + lane;
        const uint32_t lane_off = ((uint32_t)(q4 * 32)) << 16;
        const uint32_t tS = tbase + T::T_S + g * 128 + e * 64 + lane_off;
        const uint32_t tP = tbase + T::T_P + g * 64 + e * 32 + lane_off;
        constexpr int HC = CP / 2;   // this half's output channels [e HC, e HC + HC)
        const float2 sc2 = make_float2(a.scale, a.scale);
        const float2 l2e2 = make_float2(kLog2e, kLog2e);
        // Exchange with the other key half of the same rows: both publish N values into a
        // slot of the group's buffer (alternating between two slots, so a slot is rewritten
        // only after the partner has read it), arrive on the row quad's barrier of that slot
        // and read the partner's values once all 64 threads have arrived.  Bounded waits.
        float *xbuf = reinterpret_cast<float *>(gbase + T::OFF_X) + g * T::X_GROUP;
        int xc = 0;   // exchanges so far (the same sequence in both halves)
        auto exchange = [&](const auto &mine, auto &theirs) -> bool {
            constexpr int NV = sizeof(mine) / sizeof(float);
            const int par = xc & 1;
            float *slot = xbuf + par * (2 * SPG * 128);
#pragma unroll
            for (int i = 0; i < NV; ++i) slot[(e * SPG + i) * 128 + row] = mine[i];
            const uint32_t xb = bar(T::B_X + (g * 4 + q4) * 2 + par);
            mbar_arrive(xb);
            bool okx = mbar_wait(xb, (xc >> 1) & 1, abort_flag, SITE_FWD_SOFTMAX | 0x50 | (xc << 12));
            okx = __all_sync(0xffffffffu, okx);
            if (okx) {
#pragma unroll
                for (int i = 0; i < NV; ++i) theirs[i] = slot[((1 - e) * SPG + i) * 128 + row];
            }
            ++xc;
            return okx;
        };
        bool ok = true;
        int k = 0, jg = 0;   // the CTA's steps and bias tiles before this item
        int gk = 0;          // this group's steps so far
        int gitems = 0;      // items with a row of this group so far (its ofinal phases)
        for (int n = 0; n < n_items && ok; ++n) {
            const FItem it = item(n);
            const int nb = it.nb;
            const int nmine = nb > g ? (nb - g + 1) / 2 : 0;   // slots g, g + 2, ... below nb
            float m_run[SPG], l_run[SPG];   // running (max, partial sum over my keys) per slot
#pragma unroll
            for (int t = 0; t < SPG; ++t) {
                m_run[t] = -INFINITY;
                l_run[t] = 0.f;
            }
            // the epilogue's gate rows: into L2 now, so that their loads after the item's
            // last step do not wait for DRAM
            if (a.gate && e == 0 && it.i0 + row < a.Nq) {
#pragma unroll
                for (int t = 0; t < SPG; ++t)
                    if (t < nmine)
                        prefetch_l2(a.gate + (it.b0 + g + 2 * t) * a.sg0 + (long long)(it.i0 + row) * a.sg1 +
                                    it.h * a.sg2);
            }
            for (int j = 0; j < it.nj && ok; ++j, ++jg) {   // j: the item's key tile jlo + j
                const int bs = jg % BS;
                if (nmine == 0) {
                    // this group has no row in the item: it only hands each bias tile back
                    ok = mbar_wait(b_bias_ready(bs), (jg / BS) & 1, abort_flag, SITE_FWD_SOFTMAX | 0x60 | (jg << 12));
                    ok = __all_sync(0xffffffffu, ok);
                    if (ok) mbar_arrive(b_bias_empty(bs));
                    continue;
                }
                for (int t = 0; t < nmine; ++t, ++gk) {
                    const int s = g + 2 * t;
                    const int ks = k + j * nb + s;   // the CTA's step of (j, s)
                    const int st = gk % KVG;         // its stage in the group's rings
                    ok = mbar_wait(b_s_full(g), gk & 1, abort_flag, SITE_FWD_SOFTMAX | (ks << 12));
                    if (ok && t == 0)
                        ok = mbar_wait(b_bias_ready(bs), (jg / BS) & 1, abort_flag,
                                       SITE_FWD_SOFTMAX | 0x10 | (ks << 12));
                    if (ok && row_mask)   // this step's mask words come with its V tile
                        ok = mbar_wait(b_v_full(g, st), (gk / KVG) & 1, abort_flag,
                                       SITE_FWD_SOFTMAX | 0x20 | (ks << 12));
                    ok = __all_sync(0xffffffffu, ok);
                    if (!ok) break;
                    tc_fence_after();

                    // S of this row's 64 keys, then hand the S columns back for the next Q K^T
                    uint32_t xr[64];
                    tmem_ld64(tS, xr);
                    tc_fence_before();
                    mbar_arrive(b_s_free(g));

                    // logits in place: x = scale * S + bias (natural-log units; -inf if masked)
                    {
                        const uint32_t bias_row = sbase + T::OFF_BIAS + bs * T::BIAS_BYTES + e * 16384 + row * 128;
#pragma unroll
                        for (int q = 0; q < 8; ++q) {  // 16-byte chunk q holds keys 8q .. 8q+7 of the half
                            const uint4 bw = lds128(bias_row + ((q ^ (row & 7)) << 4));
                            const uint32_t bb[4] = {bw.x, bw.y, bw.z, bw.w};
#pragma unroll
                            for (int u = 0; u < 4; ++u) {
                                const int c = q * 8 + 2 * u;
                                const float2 v = ffma2(make_float2(__uint_as_float(xr[c]), __uint_as_float(xr[c + 1])),
                                                       sc2, make_float2(bf16lo(bb[u]), bf16hi(bb[u])));
                                xr[c] = __float_as_uint(v.x);
                                xr[c + 1] = __float_as_uint(v.y);
                            }
                        }
                    }
                    if (t == nmine - 1) mbar_arrive(b_bias_empty(bs));   // the group's last reader of the tile
                    float *x = reinterpret_cast<float *>(xr);
                    if (row_mask) {
                        const uint32_t *mw = reinterpret_cast<const uint32_t *>(gbase + T::OFF_MASK) +
                                             (g * KVG + st) * 8 + 2 * e;
                        const uint32_t w0 = mw[0], w1 = mw[1];
                        if ((w0 & w1) != 0xffffffffu) {
#pragma unroll
                            for (int c = 0; c < 32; ++c) {
                                if (!((w0 >> c) & 1u)) x[c] = -INFINITY;
                                if (!((w1 >> c) & 1u)) x[32 + c] = -INFINITY;
                            }
                        }
                    }
                    // maximum over this half's keys: four independent chains of three-input max
                    float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                    for (int c = 0; c < 64; c += 8) {
                        m4[0] = max3(m4[0], x[c], x[c + 1]);
                        m4[1] = max3(m4[1], x[c + 2], x[c + 3]);
                        m4[2] = max3(m4[2], x[c + 4], x[c + 5]);
                        m4[3] = max3(m4[3], x[c + 6], x[c + 7]);
                    }
                    float mxh[1] = {fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]))}, mxo[1] = {-INFINITY};
                    // the row's maximum over both halves (the same value in both)
                    ok = exchange(mxh, mxo);
                    if (!ok) break;
                    const float mx = fmaxf(mxh[0], mxo[0]);

                    float m_use = m_run[0], l_prev = l_run[0];
#pragma unroll
                    for (int u = 1; u < SPG; ++u)
                        if (t == u) {
                            m_use = m_run[u];
                            l_prev = l_run[u];
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
                    // rescale of O[s]) has to wait for the group's previous P V.
                    float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
                    uint32_t p[32];   // P of this half's 64 keys as bf16 pairs
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        const float2 tt = ffma2(make_float2(x[2 * c], x[2 * c + 1]), l2e2, nm2);
                        const float2 pv = make_float2(ex2(tt.x), ex2(tt.y));
                        if (c & 1) acc1 = fadd2(acc1, pv);
                        else acc0 = fadd2(acc0, pv);
                        p[c] = pack_bf16x2(pv.x, pv.y);
                    }
                    const float sum = (acc0.x + acc0.y) + (acc1.x + acc1.y);
                    // P and O[s] may only be written once the group's previous P V is done
                    if (gk > 0) {
                        ok = mbar_wait(b_p_free(g), (gk - 1) & 1, abort_flag, SITE_FWD_SOFTMAX | 0x30 | (ks << 12));
                        ok = __all_sync(0xffffffffu, ok);
                        if (!ok) break;
                        tc_fence_after();
                    }
                    tmem_st32(tP, p);
                    if (__any_sync(0xffffffffu, resc)) {
                        const uint32_t tO = tbase + T::T_O + s * CP + e * HC + lane_off;
                        uint32_t o[HC];
                        tmem_ld_cols<HC>(tO, o);
#pragma unroll
                        for (int c = 0; c < HC; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
                        tmem_st_cols<HC>(tO, o);
                    }
                    tmem_wait_st();
                    const float l_new = l_prev * alpha + sum;
#pragma unroll
                    for (int u = 0; u < SPG; ++u)
                        if (t == u) {
                            m_run[u] = m_use;
                            l_run[u] = l_new;
                        }
                    tc_fence_before();
                    mbar_arrive(b_p_full(g));
                }
            }
            k += it.nj * nb;
            if (!ok) break;
            if (nmine == 0) continue;   // no row of this group in the item: nothing to write
            // ------------------------------------------------------------------ epilogue
            ok = mbar_wait(b_ofinal(g), gitems & 1, abort_flag, SITE_FWD_EPI | (n << 12));
            ++gitems;
            ok = __all_sync(0xffffffffu, ok);
            // the row sum over both halves, added in the same order in both
            float lo_[SPG];
#pragma unroll
            for (int t = 0; t < SPG; ++t) lo_[t] = 0.f;
            if (ok) ok = exchange(l_run, lo_);
            if (!ok) break;
            // the gate rows were brought into L2 at the item's start
            const int i = it.i0 + row;
            const bool row_ok = i < a.Nq;
            uint4 gw[SPG][HC / 8];
#pragma unroll
            for (int t = 0; t < SPG; ++t) {
#pragma unroll
                for (int c8 = 0; c8 < HC / 8; ++c8) {
                    const int ch = e * HC + c8 * 8;
                    gw[t][c8] = make_uint4(0, 0, 0, 0);
                    if (a.gate && row_ok && t < nmine && ch < a.C)
                        gw[t][c8] = *reinterpret_cast<const uint4 *>(
                            a.gate + (it.b0 + g + 2 * t) * a.sg0 + (long long)i * a.sg1 + it.h * a.sg2 + ch);
                }
            }
            tc_fence_after();
#pragma unroll
            for (int t = 0; t < SPG; ++t) {
                if (t >= nmine) break;
                const int s = g + 2 * t;
                const float l_tot = e == 0 ? l_run[t] + lo_[t] : lo_[t] + l_run[t];
                uint32_t o[HC];
                tmem_ld_cols<HC>(tbase + T::T_O + s * CP + e * HC + lane_off, o);
                if (!row_ok) continue;
                const int b = it.b0 + s;
                const bool live = l_tot > 0.f;
                const float inv = live ? rcp_approx(l_tot) : 0.f;
                __nv_bfloat16 *op = a.out + b * a.so0 + (long long)i * a.so1 + it.h * a.so2;
#pragma unroll
                for (int c8 = 0; c8 < HC / 8; ++c8) {
                    const int ch = e * HC + c8 * 8;
                    if (ch < a.C) {
                        const uint32_t g4[4] = {gw[t][c8].x, gw[t][c8].y, gw[t][c8].z, gw[t][c8].w};
                        uint32_t ow[4];
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            float lo = __uint_as_float(o[c8 * 8 + 2 * u]) * inv;
                            float hi = __uint_as_float(o[c8 * 8 + 2 * u + 1]) * inv;
                            if (a.gate) {
                                lo *= sigmoid_fast(bf16lo(g4[u]));
                                hi *= sigmoid_fast(bf16hi(g4[u]));
                            }
                            ow[u] = pack_bf16x2(lo, hi);
                        }
                        *reinterpret_cast<uint4 *>(op + ch) = make_uint4(ow[0], ow[1], ow[2], ow[3]);
                    }
                }
                if (e == 0)
                    a.lse[((long long)b * a.H + it.h) * a.Nq + i] =
                        live ? m_run[t] + lg2_approx(l_tot) * 0.6931471805599453f : -INFINITY;
            }
        }
    }

    // ---------------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (*abort_flag) {
        // Some wait ran out.  Every role has stopped; before shared memory and TMEM are
        // released, let the copies and MMAs already issued finish (bounded waits).
        if (warp == T::W_PROD && lane == 0) {
            for (int s = 0; s < BC; ++s)
                if (q_loads[s] > 0) mbar_wait_drain(b_q_full(s), (q_loads[s] - 1) & 1);
            for (int g = 0; g < 2; ++g) {
                for (int kk = max(0, k_done[g] - KVG); kk < k_done[g]; ++kk)
                    if (g != skipped_g || kk != skipped_gs) mbar_wait_drain(b_k_full(g, kk % KVG), (kk / KVG) & 1);
                for (int kk = max(0, v_done[g] - KVG); kk < v_done[g]; ++kk)
                    mbar_wait_drain(b_v_full(g, kk % KVG), (kk / KVG) & 1);
            }
            for (int jj = max(0, n_bias - BS); jj < n_bias; ++jj)
                mbar_wait_drain(b_bias_full(jj % BS), (jj / BS) & 1);
        }
        if ((warp == T::W_ISS0 || warp == T::W_ISS1) && lane == 0) {
            umma_commit(b_drain);   // each issuer's own MMAs
            mbar_wait_drain(b_drain, 0);
        }
        tc_fence_before();
        __syncthreads();
    }
    if (warp == T::W_ISS0) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tbase, T::TMEM_COLS);
    }
}

}  // namespace pba
