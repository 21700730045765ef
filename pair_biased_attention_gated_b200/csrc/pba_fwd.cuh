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
// Warp roles (320 threads):
//   warps 0-3  softmax warpgroup 0: the chunk's even rows (slot s = 0, 2, ...)
//   warps 4-7  softmax warpgroup 1: the odd rows
//   warp 8     TMA producer (Q, K, V, bias tiles) and key-mask bits
//   warp 9     TMEM allocator and, on lane 0, the tcgen05 MMA issuer
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
    const uint8_t *mask;
    long long smask_b;
    const __nv_bfloat16 *gate;
    long long sg0, sg1, sg2;
    __nv_bfloat16 *out;
    long long so0, so1, so2;
    float *lse;
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
    static constexpr int OFF_MASK = OFF_STATS + BCMAX * 128 * 8; // u32 [KV_STAGES][8]
    static constexpr int SMEM_BYTES = OFF_MASK + KV_STAGES * 32 + 1024;
    static constexpr uint32_t SWZ = CP == 64 ? kSw128 : (CP == 32 ? kSw64 : kSw32);
    static constexpr uint32_t ROWB = CP * 2;                   // bytes per tile row
    static constexpr int THREADS = 320;
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
__global__ void __launch_bounds__(320, 1)
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
        bool ok = true;
        int k = 0;
        for (int j = 0; j < nJ && ok; ++j) {
            const int bs = j & 1;
            if (j >= 2) ok = mbar_wait(b_bias_empty(bs), ((j >> 1) - 1) & 1, abort_flag, SITE_FWD_PROD);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            if (lane == 0) {
                if (a.has_bias) {
                    const uint32_t dst = sbase + T::OFF_BIAS + bs * T::BIAS_BYTES;
                    mbar_arrive_tx(b_bias_full(bs), T::BIAS_BYTES);
                    tma_load_3d(dst, &tmBias, b_bias_full(bs), j * 128, i0, h);
                    tma_load_3d(dst + 16384, &tmBias, b_bias_full(bs), j * 128 + 64, i0, h);
                } else {
                    mbar_arrive(b_bias_full(bs));
                }
            }
            for (int s = 0; s < nb; ++s, ++k) {
                const int st = k % KVS, use = k / KVS;
                if (use >= 1) ok = mbar_wait(b_kv_empty(st), (use - 1) & 1, abort_flag, SITE_FWD_PROD);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                const int b = b0 + s;
                uint32_t words[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int key = j * 128 + q * 32 + lane;
                    bool valid = key < a.Nk;
                    if (valid && a.mask) valid = a.mask[(long long)b * a.smask_b + key] != 0;
                    words[q] = __ballot_sync(0xffffffffu, valid);
                }
                if (lane == 0) {
                    uint32_t *mw = reinterpret_cast<uint32_t *>(gbase + T::OFF_MASK) + st * 8;
                    mw[0] = words[0];
                    mw[1] = words[1];
                    mw[2] = words[2];
                    mw[3] = words[3];
                    mw[4] = (words[0] & words[1] & words[2] & words[3]) == 0xffffffffu;
                    const uint32_t dst = sbase + T::OFF_KV + st * 2 * T::TILE_BYTES;
                    mbar_arrive_tx(b_kv_full(st), 2 * T::TILE_BYTES);
                    tma_load_4d(dst, &tmK, b_kv_full(st), 0, h, j * 128, b);
                    tma_load_4d(dst + T::TILE_BYTES, &tmV, b_kv_full(st), 0, h, j * 128, b);
                }
            }
        }
        if (!ok && lane == 0) {
            // let every copy already issued land before the CTA's shared memory goes away
            mbar_wait_drain(b_q, 0);
            for (int kk = max(0, k - KVS); kk < k; ++kk) mbar_wait_drain(b_kv_full(kk % KVS), (kk / KVS) & 1);
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
            for (int k = 0; k < K && ok; ++k) {
                const int s = k % nb, w = s & 1, st = k % KVS;
                if (pending[w] >= 0) {
                    ok = mbar_wait(b_p_full(w), pcount[w] & 1, abort_flag, SITE_FWD_MMA);
                    ++pcount[w];
                    if (!ok) break;
                    tc_fence_after();
                    issue_pv(pending[w]);
                    pending[w] = -1;
                }
                ok = mbar_wait(b_kv_full(st), (k / KVS) & 1, abort_flag, SITE_FWD_MMA);
                if (!ok) break;
                tc_fence_after();
                const uint32_t qa = sbase + T::OFF_Q + s * T::TILE_BYTES;
                const uint32_t ka = sbase + T::OFF_KV + st * 2 * T::TILE_BYTES;
#pragma unroll
                for (int kk = 0; kk < CP / 16; ++kk)
                    umma_ss(tbase + w * 128, sdesc(qa + kk * 32, 16, SBO, T::SWZ),
                            sdesc(ka + kk * 32, 16, SBO, T::SWZ), idesc_qk, kk > 0 ? 1u : 0u);
                umma_commit(b_s_full(w));
                pending[w] = k;
            }
            for (int w = 0; w < 2 && ok; ++w) {
                if (pending[w] < 0) continue;
                ok = mbar_wait(b_p_full(w), pcount[w] & 1, abort_flag, SITE_FWD_MMA);
                ++pcount[w];
                if (!ok) break;
                tc_fence_after();
                issue_pv(pending[w]);
            }
            if (ok) {
                umma_commit(b_ofinal);
            } else {
                umma_commit(b_drain);
                mbar_wait_drain(b_drain, 0);
            }
        }
    } else {
        // ------------------------------------------------------------------ softmax
        const int w = warp >> 2;
        const int row = (warp & 3) * 32 + lane;
        const uint32_t lane_off = ((uint32_t)((warp & 3) * 32)) << 16;
        const uint32_t tS = tbase + w * 128 + lane_off;
        float2 *stats = reinterpret_cast<float2 *>(gbase + T::OFF_STATS);
        const float scale = a.scale;
        int ns = 0;
        bool ok = true;
        for (int j = 0; j < nJ && ok; ++j) {
            bool bias_ready = false;
            for (int s = w; s < nb; s += 2) {
                const int k = j * nb + s, st = k % KVS;
                ok = mbar_wait(b_s_full(w), ns & 1, abort_flag, SITE_FWD_SOFTMAX);
                ++ns;
                if (ok) ok = mbar_wait(b_kv_full(st), (k / KVS) & 1, abort_flag, SITE_FWD_SOFTMAX);
                if (ok && !bias_ready) {
                    ok = mbar_wait(b_bias_full(j & 1), (j >> 1) & 1, abort_flag, SITE_FWD_SOFTMAX);
                    bias_ready = true;
                }
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                tc_fence_after();

                // logits of this row: x = scale * S + bias (natural-log units)
                float x[128];
                const uint32_t bias_row = sbase + T::OFF_BIAS + (j & 1) * T::BIAS_BYTES + row * 128;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint32_t r[32];
                    tmem_ld32(tS + q * 32, r);
#pragma unroll
                    for (int c4 = 0; c4 < 4; ++c4) {
                        const int c8 = (q & 1) * 4 + c4;  // 16-byte chunk within a 64-key half
                        uint4 bw = make_uint4(0, 0, 0, 0);
                        if (a.has_bias)
                            bw = lds128(bias_row + (q >> 1) * 16384 + ((c8 ^ (row & 7)) << 4));
                        const uint32_t bb[4] = {bw.x, bw.y, bw.z, bw.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int c = q * 32 + c4 * 8 + 2 * e;
                            x[c] = fmaf(__uint_as_float(r[c4 * 8 + 2 * e]), scale, bf16lo(bb[e]));
                            x[c + 1] = fmaf(__uint_as_float(r[c4 * 8 + 2 * e + 1]), scale, bf16hi(bb[e]));
                        }
                    }
                }
                const uint32_t *mw = reinterpret_cast<const uint32_t *>(gbase + T::OFF_MASK) + st * 8;
                if (mw[4] == 0u) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint32_t wd = mw[q];
#pragma unroll
                        for (int t = 0; t < 32; ++t)
                            if (!((wd >> t) & 1u)) x[q * 32 + t] = -INFINITY;
                    }
                }
                float mx = x[0];
#pragma unroll
                for (int c = 1; c < 128; ++c) mx = fmaxf(mx, x[c]);

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
                float sum = 0.f;
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    uint32_t p[32];
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        const float p0 = ex2(fmaf(x[hf * 64 + 2 * c], kLog2e, nm));
                        const float p1 = ex2(fmaf(x[hf * 64 + 2 * c + 1], kLog2e, nm));
                        sum += p0 + p1;
                        p[c] = pack_bf16x2(p0, p1);
                    }
                    tmem_st32(tS + hf * 32, p);
                }
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
        if (ok && w < nb) {
            ok = mbar_wait(b_ofinal, 0, abort_flag, SITE_FWD_EPI);
            ok = __all_sync(0xffffffffu, ok);
        }
        if (ok) {
            tc_fence_after();
            for (int s = w; s < nb; s += 2) {
                uint32_t o[CP];
                tmem_ld_cols<CP>(tbase + 256 + s * CP + lane_off, o);
                const float2 stv = stats[s * 128 + row];
                const int i = i0 + row, b = b0 + s;
                if (i < a.Nq) {
                    const bool live = stv.y > 0.f;
                    const float inv = live ? 1.f / stv.y : 0.f;
                    const __nv_bfloat16 *gp =
                        a.gate ? a.gate + b * a.sg0 + (long long)i * a.sg1 + h * a.sg2 : nullptr;
                    __nv_bfloat16 *op = a.out + b * a.so0 + (long long)i * a.so1 + h * a.so2;
#pragma unroll
                    for (int c8 = 0; c8 < CP / 8; ++c8) {
                        if (c8 * 8 < a.C) {
                            uint32_t gw[4] = {0, 0, 0, 0};
                            if (gp) {
                                const uint4 g4 = *reinterpret_cast<const uint4 *>(gp + c8 * 8);
                                gw[0] = g4.x; gw[1] = g4.y; gw[2] = g4.z; gw[3] = g4.w;
                            }
                            uint32_t ow[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                float lo = __uint_as_float(o[c8 * 8 + 2 * e]) * inv;
                                float hi = __uint_as_float(o[c8 * 8 + 2 * e + 1]) * inv;
                                if (gp) {
                                    lo *= 1.f / (1.f + __expf(-bf16lo(gw[e])));
                                    hi *= 1.f / (1.f + __expf(-bf16hi(gw[e])));
                                }
                                if (!live) lo = hi = 0.f;
                                ow[e] = pack_bf16x2(lo, hi);
                            }
                            *reinterpret_cast<uint4 *>(op + c8 * 8) = make_uint4(ow[0], ow[1], ow[2], ow[3]);
                        }
                    }
                    a.lse[((long long)b * a.H + h) * a.Nq + i] = live ? stv.x + logf(stv.y) : -INFINITY;
                }
            }
        }
    }

    // ---------------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tbase, 512);
    }
}

}  // namespace pba
