// Forward kernel: out = sigmoid(G) * softmax(scale * Q K^T + bias + mask) V, and the
// logsumexp of every query row.
//
// Pair-biased attention as described on the "AlphaFold3 open-source implementation" page,
// Model Efficiency section: the pair bias is added after the key-query dot product and
// is shared by every broadcast row b (triangle rows, MSA sequences, diffusion copies).
//
// One CTA owns one (head h, 128-query tile, chunk of `bc` broadcast rows).  Its loop runs
// over key tiles j (outer) and the chunk's rows b (inner), so each 128x128 bias tile is
// moved into shared memory once and reused by all rows of the chunk.  Each step (j, b)
// streams the Q and K tiles of row b through one ring of stages, released as soon as
// Q K^T is done, and the V tile through a deeper ring, released after P V.
//
// Warp roles (384 threads, three warpgroups):
//   warps 0-3  softmax warpgroup 0: the chunk's even rows (slot s = 0, 2, ...)
//   warps 4-7  softmax warpgroup 1: the odd rows
//   warp 8     TMA producer (Q, K, V, bias tiles) and key-mask bits
//   warp 9     TMEM allocator; lane 0 issues the tcgen05 MMAs of softmax warpgroup 0
//   warp 10    lane 0 issues the tcgen05 MMAs of softmax warpgroup 1
//   warp 11    idle: it completes the third warpgroup, whose registers the softmax
//              warpgroups take over (setmaxnreg)
// Tensor memory (512 columns): S buffer of warpgroup 0 [0,128), of warpgroup 1 [128,256),
// then one CP-column fp32 O accumulator per slot of the chunk.
//
// Per step a softmax warpgroup loads its S tile from TMEM and at once hands the buffer
// back, so the next Q K^T of that warpgroup runs while it computes exp(); it then writes
// P (bf16) to a shared-memory tile, from which the P V product reads.  Neither MMA is on
// the warpgroup's critical path.
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
    int skip_step;   // test hook: the producer skips this step's Q/K load (-1: never)
};

template <int CP>
struct FwdTraits {
    static constexpr int BCMAX = (CP == 64) ? 4 : 8;           // O slots in TMEM
    static constexpr int QKS = (CP == 64) ? 2 : (CP == 32 ? 3 : 4);  // Q+K stages
    static constexpr int VS = (CP == 64) ? 3 : (CP == 32 ? 5 : 6);   // V stages
    static constexpr int BS = (CP == 64) ? 1 : 2;              // bias stages
    static constexpr int TILE_BYTES = 128 * CP * 2;            // Q, K or V tile
    static constexpr int BIAS_BYTES = 128 * 128 * 2;           // two 64-key halves
    static constexpr int P_BYTES = 128 * 128 * 2;              // P tile, two 64-key halves
    static constexpr int OFF_QK = 0;                           // [QKS] x (Q, K)
    static constexpr int OFF_V = OFF_QK + QKS * 2 * TILE_BYTES; // [VS] x V
    static constexpr int OFF_BIAS = OFF_V + VS * TILE_BYTES;
    static constexpr int OFF_P = OFF_BIAS + BS * BIAS_BYTES;   // [2 warpgroups]
    static constexpr int OFF_STATS = OFF_P + 2 * P_BYTES;      // float2 [BCMAX][128]
    static constexpr int OFF_MASK = OFF_STATS + BCMAX * 128 * 8; // u32 [VS][8] (per row b)
    static constexpr int OFF_BMASK = OFF_MASK + VS * 32;         // u32 [BS][8] (shared by all b)
    static constexpr int SMEM_BYTES = OFF_BMASK + BS * 32 + 1024;
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
    constexpr int QKS = T::QKS, VS = T::VS, BS = T::BS;
    extern __shared__ uint8_t dsmem[];
    __shared__ __align__(8) uint64_t bars[4 + 2 * QKS + 2 * VS + 2 * BS + 8 + T::BCMAX];
    __shared__ uint32_t s_tmem_base;
    __shared__ int s_abort;

    // barrier slots
    const uint32_t b_ofinal = smem_u32(&bars[0]);
    auto b_drain = [&](int w) { return smem_u32(&bars[1 + w]); };             // abort path
    auto b_qk_full = [&](int st) { return smem_u32(&bars[4 + st]); };          // Q, K landed
    auto b_qk_empty = [&](int st) { return smem_u32(&bars[4 + QKS + st]); };   // Q K^T done
    auto b_v_full = [&](int st) { return smem_u32(&bars[4 + 2 * QKS + st]); }; // V landed
    auto b_v_empty = [&](int st) { return smem_u32(&bars[4 + 2 * QKS + VS + st]); };  // P V done
    constexpr int OBB = 4 + 2 * QKS + 2 * VS;
    auto b_bias_full = [&](int x) { return smem_u32(&bars[OBB + x]); };
    auto b_bias_empty = [&](int x) { return smem_u32(&bars[OBB + BS + x]); };
    constexpr int OB = OBB + 2 * BS;
    auto b_s_full = [&](int w) { return smem_u32(&bars[OB + w]); };        // S in TMEM
    auto b_s_free = [&](int w) { return smem_u32(&bars[OB + 2 + w]); };    // S read out
    auto b_p_full = [&](int w) { return smem_u32(&bars[OB + 4 + w]); };    // P in smem
    auto b_p_free = [&](int w) { return smem_u32(&bars[OB + 6 + w]); };    // P V done reading P
    auto b_o_ready = [&](int s) { return smem_u32(&bars[OB + 8 + s]); };   // P V into O[s] done

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
        mbar_init(b_ofinal, nW);  // one commit from each MMA issuer
        mbar_init(b_drain(0), 1);
        mbar_init(b_drain(1), 1);
        for (int st = 0; st < QKS; ++st) {
            mbar_init(b_qk_full(st), 1);
            mbar_init(b_qk_empty(st), 1);
        }
        for (int st = 0; st < VS; ++st) {
            mbar_init(b_v_full(st), 1);
            mbar_init(b_v_empty(st), 1);
        }
        for (int x = 0; x < BS; ++x) {
            mbar_init(b_bias_full(x), 1);
            mbar_init(b_bias_empty(x), 128 * nW);
        }
        for (int w = 0; w < 2; ++w) {
            mbar_init(b_s_full(w), 1);
            mbar_init(b_s_free(w), 128);
            mbar_init(b_p_full(w), 128);
            mbar_init(b_p_free(w), 1);
        }
        for (int s = 0; s < T::BCMAX; ++s) mbar_init(b_o_ready(s), 1);
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

    // steps whose Q/K (V) loads the producer issued are [0, qk_done) ([0, v_done)); bias
    // tiles [0, n_bias): what has to land before the CTA may exit after an abort
    int qk_done = 0, v_done = 0, n_bias = 0;

    if (warp >= 8) reg_dealloc<T::REGS_OTHER>();   // the whole third warpgroup, same point
    if (warp == 8) {
        // ------------------------------------------------------------------ producer
        if (lane == 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            if (a.has_bias) tma_prefetch_desc(&tmBias);
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
            const int bs = j % BS;
            if (j >= BS) ok = mbar_wait(b_bias_empty(bs), ((j / BS) - 1) & 1, abort_flag, SITE_FWD_PROD | 0x20 | (j << 12));
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
            ++n_bias;
            for (int s = 0; s < nb; ++s, ++k) {
                const int sq = k % QKS, uq = k / QKS, sv = k % VS, uv = k / VS;
                if (uq >= 1) ok = mbar_wait(b_qk_empty(sq), (uq - 1) & 1, abort_flag, SITE_FWD_PROD | (k << 12));
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                const int b = b0 + s;
                if (lane == 0 && k != a.skip_step) {
                    const uint32_t dst = sbase + T::OFF_QK + sq * 2 * T::TILE_BYTES;
                    mbar_arrive_tx(b_qk_full(sq), 2 * T::TILE_BYTES);
                    tma_load_4d(dst, &tmQ, b_qk_full(sq), 0, h, i0, b);
                    tma_load_4d(dst + T::TILE_BYTES, &tmK, b_qk_full(sq), 0, h, j * 128, b);
                }
                qk_done = k + 1;
                if (uv >= 1) ok = mbar_wait(b_v_empty(sv), (uv - 1) & 1, abort_flag, SITE_FWD_PROD | 0x10 | (k << 12));
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                // a per-row mask travels with the V stage: it is released only after P V,
                // i.e. after the softmax of this step has read the mask
                uint32_t w[4] = {0, 0, 0, 0};
                if (!a.mask_shared) mask_words(b, j, w);
                if (lane == 0) {
                    if (!a.mask_shared)
                        put_words(reinterpret_cast<uint32_t *>(gbase + T::OFF_MASK) + sv * 8, w);
                    mbar_arrive_tx(b_v_full(sv), T::TILE_BYTES);
                    tma_load_4d(sbase + T::OFF_V + sv * T::TILE_BYTES, &tmV, b_v_full(sv), 0, h, j * 128, b);
                }
                v_done = k + 1;
            }
        }
    } else if (warp == 9 || warp == 10) {
        // ------------------------------------------------------------------ MMA issuers
        // Lane 0 of warp 9 issues every MMA of softmax warpgroup 0, lane 0 of warp 10 those
        // of warpgroup 1.  Each keeps the Q K^T of the warpgroup's next step one step ahead
        // of its P V: S(k+1) as soon as S(k) was read out of TMEM, P V(k) once P(k) is in
        // shared memory.  All waits suspend the thread.
        const int w = warp - 9;
        if (lane == 0 && w < nW) {
            constexpr uint32_t idesc_qk = idesc_bf16(128, 128, false, false);
            constexpr uint32_t idesc_pv = idesc_bf16(128, CP, false, true);
            constexpr uint32_t SBO = 8 * T::ROWB;
            const int K = nJ * nb;
            // steps of warpgroup w: slots s = w, w + 2, ... of key tile j, j = 0, 1, ...
            auto step_after = [&](int k) {
                const int s = k % nb, j = k / nb;
                const int n = (s + 2 < nb) ? k + 2 : (j + 1) * nb + (s & 1);
                return n < K ? n : K;
            };
            auto issue_s = [&](int k, int n) -> bool {   // n = how many S this warpgroup issued
                if (n > 0 && !mbar_wait(b_s_free(w), (n - 1) & 1, abort_flag, SITE_FWD_MMA | (k << 12))) return false;
                if (!mbar_wait(b_qk_full(k % QKS), (k / QKS) & 1, abort_flag, SITE_FWD_MMA | 0x10 | (k << 12))) return false;
                tc_fence_after();
                const uint32_t qa = sbase + T::OFF_QK + (k % QKS) * 2 * T::TILE_BYTES;
                const uint32_t ka = qa + T::TILE_BYTES;
#pragma unroll
                for (int kk = 0; kk < CP / 16; ++kk)
                    umma_ss(tbase + w * 128, sdesc(qa + kk * 32, 16, SBO, T::SWZ),
                            sdesc(ka + kk * 32, 16, SBO, T::SWZ), idesc_qk, kk > 0 ? 1u : 0u);
                umma_commit(b_s_full(w));
                umma_commit(b_qk_empty(k % QKS));
                return true;
            };
            auto issue_pv = [&](int k, int n) -> bool {  // n = how many P V this warpgroup issued
                if (!mbar_wait(b_p_full(w), n & 1, abort_flag, SITE_FWD_MMA | 0x20 | (k << 12))) return false;
                if (!mbar_wait(b_v_full(k % VS), (k / VS) & 1, abort_flag, SITE_FWD_MMA | 0x30 | (k << 12))) return false;
                tc_fence_after();
                const int jp = k / nb, sp = k % nb;
                const uint32_t pa = sbase + T::OFF_P + w * T::P_BYTES;
                const uint32_t va = sbase + T::OFF_V + (k % VS) * T::TILE_BYTES;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    umma_ss(tbase + 256 + sp * CP,
                            sdesc(pa + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024, kSw128),
                            sdesc(va + kk * 16 * T::ROWB, T::TILE_BYTES, SBO, T::SWZ), idesc_pv,
                            (jp > 0 || kk > 0) ? 1u : 0u);
                umma_commit(b_v_empty(k % VS));
                umma_commit(b_p_free(w));
                umma_commit(b_o_ready(sp));
                return true;
            };
            bool ok = true;
            int k = w;                 // this warpgroup's first step
            int n = 0;
            if (k < K) ok = issue_s(k, n);
            while (ok && k < K) {
                const int kn = step_after(k);
                // The producer reaches step kn only after the P V of step kn - 1 - VS (the
                // V ring).  When that is this warpgroup's step k, its P V has to go first.
                if (kn < K && kn - 1 - VS >= k) {
                    ok = issue_pv(k, n);
                    if (ok) ok = issue_s(kn, n + 1);
                } else {
                    if (kn < K) ok = issue_s(kn, n + 1);
                    if (ok) ok = issue_pv(k, n);
                }
                k = kn;
                ++n;
            }
            if (ok) umma_commit(b_ofinal);   // each issuer arrives once (count = nW)
        }
    } else if (warp < 8) {
        // ------------------------------------------------------------------ softmax
        reg_alloc<T::REGS_SOFTMAX>();
        const int w = warp >> 2;
        const int row = (warp & 3) * 32 + lane;
        const uint32_t lane_off = ((uint32_t)((warp & 3) * 32)) << 16;
        const uint32_t tS = tbase + w * 128 + lane_off;
        const uint32_t prow = sbase + T::OFF_P + w * T::P_BYTES + row * 128;
        float2 *stats = reinterpret_cast<float2 *>(gbase + T::OFF_STATS);
        const float2 sc2 = make_float2(a.scale, a.scale);
        const float2 l2e2 = make_float2(kLog2e, kLog2e);
        int ns = 0;
        bool ok = true;
        for (int j = 0; j < nJ && ok; ++j) {
            bool bias_ready = false;
            for (int s = w; s < nb; s += 2) {
                const int k = j * nb + s, st = k % VS;
                ok = mbar_wait(b_s_full(w), ns & 1, abort_flag, SITE_FWD_SOFTMAX | (k << 12));
                if (ok && !a.mask_shared)
                    ok = mbar_wait(b_v_full(st), (k / VS) & 1, abort_flag, SITE_FWD_SOFTMAX);
                if (ok && !bias_ready) {
                    ok = mbar_wait(b_bias_full(j % BS), (j / BS) & 1, abort_flag, SITE_FWD_SOFTMAX | 0x10 | (k << 12));
                    bias_ready = true;
                }
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                tc_fence_after();

                // S of this row, then the buffer goes back to the MMA issuer
                uint32_t xr[128];
                tmem_ld128(tS, xr);
                tc_fence_before();
                mbar_arrive(b_s_free(w));

                // logits in place: x = scale * S + bias (natural-log units)
                {
                    const uint32_t bias_row = sbase + T::OFF_BIAS + (j % BS) * T::BIAS_BYTES + row * 128;
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
                                         ? reinterpret_cast<const uint32_t *>(gbase + T::OFF_BMASK) + (j % BS) * 8
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
                // P = exp(x - m) in bf16, written over x as packed pairs
#pragma unroll
                for (int c = 0; c < 64; ++c) {
                    const float2 t = ffma2(make_float2(x[2 * c], x[2 * c + 1]), l2e2, nm2);
                    const float2 pv = make_float2(ex2(t.x), ex2(t.y));
                    if (c & 1) acc1 = fadd2(acc1, pv);
                    else acc0 = fadd2(acc0, pv);
                    xr[c] = pack_bf16x2(pv.x, pv.y);
                }
                const float sum = (acc0.x + acc0.y) + (acc1.x + acc1.y);
                // the previous P of this warpgroup must have been consumed by its P V
                if (ns > 0) {
                    ok = mbar_wait(b_p_free(w), (ns - 1) & 1, abort_flag, SITE_FWD_SOFTMAX | 0x20 | (k << 12));
                    ok = __all_sync(0xffffffffu, ok);
                    if (!ok) break;
                }
#pragma unroll
                for (int q = 0; q < 16; ++q)
                    sts128(prow + (q >> 3) * 16384 + (((q & 7) ^ (row & 7)) << 4),
                           make_uint4(xr[4 * q], xr[4 * q + 1], xr[4 * q + 2], xr[4 * q + 3]));
                // generic-proxy writes -> visible to the tensor core's async proxy
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                // O[s] must be rescaled before this step's P V, after the previous one
                if (__any_sync(0xffffffffu, resc)) {
                    ok = mbar_wait(b_o_ready(s), (j - 1) & 1, abort_flag, SITE_FWD_SOFTMAX | 0x30 | (k << 12));
                    ok = __all_sync(0xffffffffu, ok);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t tO = tbase + 256 + s * CP + lane_off;
                    uint32_t o[CP];
                    tmem_ld_cols<CP>(tO, o);
#pragma unroll
                    for (int c = 0; c < CP; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
                    tmem_st_cols<CP>(tO, o);
                    tmem_wait_st();
                    tc_fence_before();
                }
                stats[s * 128 + row] = make_float2(m_use, l_prev * alpha + sum);
                mbar_arrive(b_p_full(w));
                ++ns;
                if (s + 2 >= nb) mbar_arrive(b_bias_empty(j % BS));
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
            for (int kk = max(0, qk_done - QKS); kk < qk_done; ++kk)
                if (kk != a.skip_step) mbar_wait_drain(b_qk_full(kk % QKS), (kk / QKS) & 1);
            for (int kk = max(0, v_done - VS); kk < v_done; ++kk) mbar_wait_drain(b_v_full(kk % VS), (kk / VS) & 1);
            for (int jj = max(0, n_bias - BS); jj < n_bias; ++jj) mbar_wait_drain(b_bias_full(jj % BS), (jj / BS) & 1);
        }
        if ((warp == 9 || warp == 10) && lane == 0 && warp - 9 < nW) {
            umma_commit(b_drain(warp - 9));
            mbar_wait_drain(b_drain(warp - 9), 0);
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
