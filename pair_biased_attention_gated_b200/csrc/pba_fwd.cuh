// Forward kernel: out = sigmoid(G) * softmax(scale * Q K^T + bias + mask) V, and the
// logsumexp of every query row.
//
// Pair-biased attention as described on the "AlphaFold3 open-source implementation" page,
// Model Efficiency section: the pair bias is added after the key-query dot product and
// is shared by every broadcast row b (triangle rows, MSA sequences, diffusion copies).
//
// One CTA owns one (head h, 128-query tile, chunk of `bc` broadcast rows).  Its loop runs
// over key tiles j (outer) and the chunk's rows b (inner), so each 128x128 bias tile is
// moved into shared memory once and reused by all rows of the chunk.  The Q tiles of the
// chunk stay resident; K/V tiles stream through a ring.
//
// Warp roles (384 threads, three warpgroups):
//   warps 0-3  softmax warpgroup 0: the chunk's even rows (slot s = 0, 2, ...)
//   warps 4-7  softmax warpgroup 1: the odd rows
//   warp 8     TMA producer (Q, K, V, bias tiles) and key-mask bits
//   warp 9     TMEM allocator and, on lane 0, the tcgen05 MMA issuer
//   warps 10-11 idle: they complete the third warpgroup, whose registers the softmax
//              warpgroups take over (setmaxnreg)
// Tensor memory (512 columns): S/P buffer of warpgroup 0 [0,128), of warpgroup 1
// [128,256), then one CP-column fp32 O accumulator per slot of the chunk.
// The two warpgroups alternate: while one computes exp() of its S tile the MMA issuer
// runs the other's Q K^T and P V products.
#pragma once

#include "pba_device.cuh"

namespace pba {

struct FwdArgs {
    int B, H, Nq, Nk, C;
    int nI, nJ, nChunks, bc;
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
    int skip_step;   // test hook: the producer skips this step's K/V load (-1: never)
};

template <int CP>
struct FwdTraits {
    static constexpr int BCMAX = (CP == 64) ? 4 : 8;           // O slots in TMEM
    static constexpr int KV_STAGES = (CP == 64) ? 2 : 3;
    static constexpr int TILE_BYTES = 128 * CP * 2;            // Q, K or V tile
    static constexpr int BIAS_BYTES = 128 * 128 * 2;           // two 64-key halves
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_KV = OFF_Q + BCMAX * TILE_BYTES;
    static constexpr int OFF_BIAS = OFF_KV + KV_STAGES * 2 * TILE_BYTES;
    static constexpr int OFF_STATS = OFF_BIAS + 2 * BIAS_BYTES;  // float2 [BCMAX][128]
    static constexpr int OFF_MASK = OFF_STATS + BCMAX * 128 * 8; // u32 [KV_STAGES][8] (per row b)
    static constexpr int OFF_BMASK = OFF_MASK + KV_STAGES * 32;  // u32 [2][8] (shared by all b)
    static constexpr int SMEM_BYTES = OFF_BMASK + 2 * 32 + 1024;
    static constexpr uint32_t SWZ = CP == 64 ? kSw128 : (CP == 32 ? kSw64 : kSw32);
    static constexpr uint32_t ROWB = CP * 2;                   // bytes per tile row
    static constexpr int THREADS = 384;
    // register split through setmaxnreg: 2 x 128 x 216 + 128 x 72 = 384 x 168, the
    // registers the CTA is launched with (the build checks that ptxas reports 168)
    static constexpr int REGS_SOFTMAX = 216;
    static constexpr int REGS_OTHER = 72;
};

// Online-softmax rescale threshold (natural-log units, = 8 in log2 units): the running
// maximum is only moved, and O and l rescaled, when a row's maximum grows by more than
// this.  Exponentials are then bounded by 2^8, harmless in fp32 and bf16; the final
// O / l is exact regardless of the reference point.
constexpr float kRescaleThresh = 5.545177444479562f;
constexpr float kLog2e = 1.4426950408889634f;

enum : unsigned {
    SITE_FWD_PROD = 0x101, SITE_FWD_MMA = 0x102, SITE_FWD_SOFTMAX = 0x103,
    SITE_FWD_EPI = 0x104
};

template <int CP>
__global__ void __launch_bounds__(384, 1)
pba_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV,
               const __grid_constant__ CUtensorMap tmBias, const FwdArgs a) {
    using T = FwdTraits<CP>;
    constexpr int KVS = T::KV_STAGES;
    extern __shared__ uint8_t dsmem[];
    __shared__ __align__(8) uint64_t bars[6 + 2 * KVS + 2 + 2 + 2 + 2];
    __shared__ uint32_t s_tmem_base;
    __shared__ int s_abort;

    // barrier slots
    const uint32_t b_q = smem_u32(&bars[0]);
    const uint32_t b_ofinal = smem_u32(&bars[1]);
    const uint32_t b_drain = smem_u32(&bars[2]);
    auto b_kv_full = [&](int st) { return smem_u32(&bars[6 + st]); };
    auto b_kv_empty = [&](int st) { return smem_u32(&bars[6 + KVS + st]); };
    auto b_bias_full = [&](int x) { return smem_u32(&bars[6 + 2 * KVS + x]); };
    auto b_bias_empty = [&](int x) { return smem_u32(&bars[6 + 2 * KVS + 2 + x]); };
    auto b_s_full = [&](int x) { return smem_u32(&bars[6 + 2 * KVS + 4 + x]); };
    auto b_p_full = [&](int x) { return smem_u32(&bars[6 + 2 * KVS + 6 + x]); };

    const uint32_t raw = smem_u32(dsmem);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    uint8_t *gbase = dsmem + (sbase - raw);

    const int warp = warp_id(), lane = lane_id();
    int idx = blockIdx.x;
    const int itile = idx % a.nI;
    idx /= a.nI;
    const int chunk = idx % a.nChunks;
    const int h = idx / a.nChunks;
    const int i0 = itile * 128, b0 = chunk * a.bc;
    const int nb = min(a.bc, a.B - b0);
    const int nJ = a.nJ;
    const int nW = nb >= 2 ? 2 : 1;

    if (threadIdx.x == 0) {
        mbar_init(b_q, 1);
        mbar_init(b_ofinal, 1);
        mbar_init(b_drain, 1);
        for (int st = 0; st < KVS; ++st) {
            mbar_init(b_kv_full(st), 1);
            mbar_init(b_kv_empty(st), 1);
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(b_bias_full(x), 1);
            mbar_init(b_bias_empty(x), 128 * nW);
            mbar_init(b_s_full(x), 1);
            mbar_init(b_p_full(x), 128);
        }
        s_abort = 0;
        fence_mbar_init();
    }
    if (warp < 8) {
        // per-slot running (max, sum) of this thread's row
        float2 *stats = reinterpret_cast<float2 *>(gbase + T::OFF_STATS);
        const int row = (warp & 3) * 32 + lane;
        for (int s = warp >> 2; s < T::BCMAX; s += 2) stats[s * 128 + row] = make_float2(-INFINITY, 0.f);
    }
    if (warp == 9) {
        tmem_alloc(smem_u32(&s_tmem_base), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = s_tmem_base;
    volatile int *abort_flag = &s_abort;

    // K/V loads issued for steps [0, kv_done), bias tiles [0, n_bias): what has to land
    // before the CTA may exit after an abort
    int kv_done = 0, n_bias = 0;

    if (warp >= 8) reg_dealloc<T::REGS_OTHER>();   // the whole third warpgroup, same point
    if (warp == 8) {
        // ------------------------------------------------------------------ producer
        if (lane == 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            if (a.has_bias) tma_prefetch_desc(&tmBias);
            mbar_arrive_tx(b_q, nb * T::TILE_BYTES);
            for (int s = 0; s < nb; ++s)
                tma_load_4d(sbase + T::OFF_Q + s * T::TILE_BYTES, &tmQ, b_q, 0, h, i0, b0 + s);
        }
        // mask bits of key tile j for row b: word q bit t <-> key 128 j + 32 q + t attended
        auto mask_words = [&](int b, int j, uint32_t (&w)[4]) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int key = j * 128 + q * 32 + lane;
                bool valid = key < a.Nk;
                if (valid && a.mask) valid = a.mask[(long long)b * a.smask_b + key] != 0;
                w[q] = __ballot_sync(0xffffffffu, valid);
            }
        };
        auto put_words = [&](uint32_t *mw, const uint32_t (&w)[4]) {
            mw[0] = w[0];
            mw[1] = w[1];
            mw[2] = w[2];
            mw[3] = w[3];
            mw[4] = (w[0] & w[1] & w[2] & w[3]) == 0xffffffffu;
        };
        bool ok = true;
        int k = 0;
        for (int j = 0; j < nJ && ok; ++j) {
            const int bs = j & 1;
            if (j >= 2) ok = mbar_wait(b_bias_empty(bs), ((j >> 1) - 1) & 1, abort_flag, SITE_FWD_PROD | 0x20 | (j << 12));
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            uint32_t wj[4] = {0, 0, 0, 0};
            if (a.mask_shared) mask_words(0, j, wj);
            if (lane == 0) {
                if (a.mask_shared)
                    put_words(reinterpret_cast<uint32_t *>(gbase + T::OFF_BMASK) + bs * 8, wj);
                if (a.has_bias) {
                    const uint32_t dst = sbase + T::OFF_BIAS + bs * T::BIAS_BYTES;
                    mbar_arrive_tx(b_bias_full(bs), T::BIAS_BYTES);
                    tma_load_3d(dst, &tmBias, b_bias_full(bs), j * 128, i0, h);
                    tma_load_3d(dst + 16384, &tmBias, b_bias_full(bs), j * 128 + 64, i0, h);
                } else {
                    mbar_arrive(b_bias_full(bs));
                }
            }
            n_bias = j + 1;
            for (int s = 0; s < nb; ++s, ++k) {
                const int st = k % KVS, use = k / KVS;
                if (use >= 1) ok = mbar_wait(b_kv_empty(st), (use - 1) & 1, abort_flag, SITE_FWD_PROD | (k << 12));
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                const int b = b0 + s;
                uint32_t w[4] = {0, 0, 0, 0};
                if (!a.mask_shared) mask_words(b, j, w);
                if (lane == 0 && k != a.skip_step) {
                    if (!a.mask_shared)
                        put_words(reinterpret_cast<uint32_t *>(gbase + T::OFF_MASK) + st * 8, w);
                    const uint32_t dst = sbase + T::OFF_KV + st * 2 * T::TILE_BYTES;
                    mbar_arrive_tx(b_kv_full(st), 2 * T::TILE_BYTES);
                    tma_load_4d(dst, &tmK, b_kv_full(st), 0, h, j * 128, b);
                    tma_load_4d(dst + T::TILE_BYTES, &tmV, b_kv_full(st), 0, h, j * 128, b);
                }
                kv_done = k + 1;
            }
        }
    } else if (warp == 9) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16(128, 128, false, false);
            constexpr uint32_t idesc_pv = idesc_bf16(128, CP, false, true);
            constexpr uint32_t SBO = 8 * T::ROWB;
            bool ok = mbar_wait(b_q, 0, abort_flag, SITE_FWD_MMA);
            int pending[2] = {-1, -1};
            int pcount[2] = {0, 0};
            const int K = nJ * nb;
            auto issue_pv = [&](int kp) {
                const int jp = kp / nb, sp = kp % nb, wp = sp & 1, stp = kp % KVS;
                const uint32_t va = sbase + T::OFF_KV + stp * 2 * T::TILE_BYTES + T::TILE_BYTES;
                const uint32_t d = tbase + 256 + sp * CP;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    umma_ts(d, tbase + wp * 128 + kk * 8,
                            sdesc(va + kk * 16 * T::ROWB, T::TILE_BYTES, SBO, T::SWZ), idesc_pv,
                            (jp > 0 || kk > 0) ? 1u : 0u);
                umma_commit(b_kv_empty(stp));
            };
            // Serve whichever softmax warpgroup is ready: issue its pending P V as soon as
            // its P is in TMEM, then its next Q K^T as soon as that step's K/V tile landed.
            // Steps of warpgroup w: slots s = w, w + 2, ... of key tile j, j = 0, 1, ...
            int next[2] = {0, 1 < nb ? 1 : K};
            if (next[1] >= K) next[1] = K;
            auto step_after = [&](int k) {
                const int s = k % nb, j = k / nb;
                return (s + 2 < nb) ? k + 2 : (j + 1) * nb + (s & 1);
            };
            long long t_idle = 0;
            while (ok && (next[0] < K || next[1] < K || pending[0] >= 0 || pending[1] >= 0)) {
                bool progress = false;
#pragma unroll
                for (int w = 0; w < 2; ++w) {
                    if (pending[w] >= 0 && mbar_test(b_p_full(w), pcount[w] & 1)) {
                        ++pcount[w];
                        tc_fence_after();
                        issue_pv(pending[w]);
                        pending[w] = -1;
                        progress = true;
                    }
                    const int k = next[w];
                    if (pending[w] < 0 && k < K && mbar_test(b_kv_full(k % KVS), (k / KVS) & 1)) {
                        tc_fence_after();
                        const int s = k % nb, st = k % KVS;
                        const uint32_t qa = sbase + T::OFF_Q + s * T::TILE_BYTES;
                        const uint32_t ka = sbase + T::OFF_KV + st * 2 * T::TILE_BYTES;
#pragma unroll
                        for (int kk = 0; kk < CP / 16; ++kk)
                            umma_ss(tbase + w * 128, sdesc(qa + kk * 32, 16, SBO, T::SWZ),
                                    sdesc(ka + kk * 32, 16, SBO, T::SWZ), idesc_qk, kk > 0 ? 1u : 0u);
                        umma_commit(b_s_full(w));
                        pending[w] = k;
                        int n2 = step_after(k);
                        next[w] = n2 < K ? n2 : K;
                        progress = true;
                    }
                }
                if (progress) {
                    t_idle = 0;
                } else if (t_idle == 0) {
                    t_idle = sm_cycles();
                } else if (*abort_flag) {
                    ok = false;
                } else if (sm_cycles() - t_idle > kWaitLimitCycles) {
                    *abort_flag = 1;
                    watchdog_fire(SITE_FWD_MMA | ((next[0] < next[1] ? next[0] : next[1]) << 12));
                    ok = false;
                }
            }
            if (ok) umma_commit(b_ofinal);
        }
    } else if (warp < 8) {
        // ------------------------------------------------------------------ softmax
        reg_alloc<T::REGS_SOFTMAX>();
        const int w = warp >> 2;
        const int row = (warp & 3) * 32 + lane;
        const uint32_t lane_off = ((uint32_t)((warp & 3) * 32)) << 16;
        const uint32_t tS = tbase + w * 128 + lane_off;
        float2 *stats = reinterpret_cast<float2 *>(gbase + T::OFF_STATS);
        const float2 sc2 = make_float2(a.scale, a.scale);
        const float2 l2e2 = make_float2(kLog2e, kLog2e);
        int ns = 0;
        bool ok = true;
        for (int j = 0; j < nJ && ok; ++j) {
            bool bias_ready = false;
            for (int s = w; s < nb; s += 2) {
                const int k = j * nb + s, st = k % KVS;
                ok = mbar_wait(b_s_full(w), ns & 1, abort_flag, SITE_FWD_SOFTMAX | (k << 12));
                ++ns;
                if (ok && !a.mask_shared)
                    ok = mbar_wait(b_kv_full(st), (k / KVS) & 1, abort_flag, SITE_FWD_SOFTMAX);
                if (ok && !bias_ready) {
                    ok = mbar_wait(b_bias_full(j & 1), (j >> 1) & 1, abort_flag, SITE_FWD_SOFTMAX);
                    bias_ready = true;
                }
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                tc_fence_after();

                // logits of this row, in place: x = scale * S + bias (natural-log units)
                uint32_t xr[128];
                tmem_ld128(tS, xr);
                {
                    const uint32_t bias_row = sbase + T::OFF_BIAS + (j & 1) * T::BIAS_BYTES + row * 128;
#pragma unroll
                    for (int q = 0; q < 16; ++q) {  // 16-byte chunk q holds keys 8q .. 8q+7
                        uint4 bw = make_uint4(0, 0, 0, 0);
                        if (a.has_bias)
                            bw = lds128(bias_row + (q >> 3) * 16384 + (((q & 7) ^ (row & 7)) << 4));
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
                float *x = reinterpret_cast<float *>(xr);
                const uint32_t *mw = a.mask_shared
                                         ? reinterpret_cast<const uint32_t *>(gbase + T::OFF_BMASK) + (j & 1) * 8
                                         : reinterpret_cast<const uint32_t *>(gbase + T::OFF_MASK) + st * 8;
                if (mw[4] == 0u) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint32_t wd = mw[q];
#pragma unroll
                        for (int t = 0; t < 32; ++t)
                            if (!((wd >> t) & 1u)) x[q * 32 + t] = -INFINITY;
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

                const float2 stv = stats[s * 128 + row];
                float m_use = stv.x, l_prev = stv.y, alpha = 1.f;
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
                float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    uint32_t p[32];
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        const int i2 = hf * 64 + 2 * c;
                        const float2 t = ffma2(make_float2(x[i2], x[i2 + 1]), l2e2, nm2);
                        const float2 pv = make_float2(ex2(t.x), ex2(t.y));
                        if (c & 1) acc1 = fadd2(acc1, pv);
                        else acc0 = fadd2(acc0, pv);
                        p[c] = pack_bf16x2(pv.x, pv.y);
                    }
                    tmem_st32(tS + hf * 32, p);
                }
                const float sum = (acc0.x + acc0.y) + (acc1.x + acc1.y);
                // O must be rescaled before P V of this step is issued, i.e. before p_full
                if (__any_sync(0xffffffffu, resc)) {
                    const uint32_t tO = tbase + 256 + s * CP + lane_off;
                    uint32_t o[CP];
                    tmem_ld_cols<CP>(tO, o);
#pragma unroll
                    for (int c = 0; c < CP; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
                    tmem_st_cols<CP>(tO, o);
                }
                tmem_wait_st();
                stats[s * 128 + row] = make_float2(m_use, l_prev * alpha + sum);
                tc_fence_before();
                mbar_arrive(b_p_full(w));
                if (s + 2 >= nb) mbar_arrive(b_bias_empty(j & 1));
            }
        }
        // ------------------------------------------------------------------ epilogue
        // The gate does not depend on O: fetch it for all of this warpgroup's slots before
        // waiting for the last P V products, so its latency overlaps theirs.
        constexpr int NSL = T::BCMAX / 2;                  // slots per warpgroup
        uint4 gw[NSL][CP / 8];
        const int i = i0 + row;
        const bool row_ok = i < a.Nq;
#pragma unroll
        for (int t = 0; t < NSL; ++t) {
            const int s = w + 2 * t;
#pragma unroll
            for (int c8 = 0; c8 < CP / 8; ++c8) {
                gw[t][c8] = make_uint4(0, 0, 0, 0);
                if (ok && a.gate && row_ok && s < nb && c8 * 8 < a.C)
                    gw[t][c8] = *reinterpret_cast<const uint4 *>(
                        a.gate + (b0 + s) * a.sg0 + (long long)i * a.sg1 + h * a.sg2 + c8 * 8);
            }
        }
        if (ok && w < nb) {
            ok = mbar_wait(b_ofinal, 0, abort_flag, SITE_FWD_EPI);
            ok = __all_sync(0xffffffffu, ok);
        }
        if (ok) {
            tc_fence_after();
#pragma unroll
            for (int t = 0; t < NSL; ++t) {
                const int s = w + 2 * t;
                if (s >= nb) break;
                uint32_t o[CP];
                tmem_ld_cols<CP>(tbase + 256 + s * CP + lane_off, o);
                const float2 stv = stats[s * 128 + row];
                if (!row_ok) continue;
                const int b = b0 + s;
                const bool live = stv.y > 0.f;
                const float inv = live ? rcp_approx(stv.y) : 0.f;
                __nv_bfloat16 *op = a.out + b * a.so0 + (long long)i * a.so1 + h * a.so2;
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
                a.lse[((long long)b * a.H + h) * a.Nq + i] =
                    live ? stv.x + lg2_approx(stv.y) * 0.6931471805599453f : -INFINITY;
            }
        }
    }

    // ---------------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (*abort_flag) {
        // Some wait ran out.  Every role has stopped; before shared memory and TMEM are
        // released, let the copies and MMAs already issued finish (bounded waits).
        if (warp == 8 && lane == 0) {
            mbar_wait_drain(b_q, 0);
            for (int kk = max(0, kv_done - KVS); kk < kv_done; ++kk)
                if (kk != a.skip_step) mbar_wait_drain(b_kv_full(kk % KVS), (kk / KVS) & 1);
            for (int jj = max(0, n_bias - 2); jj < n_bias; ++jj) mbar_wait_drain(b_bias_full(jj & 1), (jj >> 1) & 1);
        }
        if (warp == 9 && lane == 0) {
            umma_commit(b_drain);
            mbar_wait_drain(b_drain, 0);
        }
        tc_fence_before();
        __syncthreads();
    }
    if (warp == 9) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tbase, 512);
    }
}

}  // namespace pba
