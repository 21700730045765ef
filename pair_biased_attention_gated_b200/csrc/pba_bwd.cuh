// Backward kernels of pair-biased gated attention.
//
// The bias gradient is the gradient of the scaled logits, and because the bias is
// broadcast over the rows b in the forward pass it is summed over b in the backward pass
// ("AlphaFold3 open-source implementation" page, Model Efficiency section).
//
// With o = softmax(s) v, out = sigmoid(g) o, P recomputed from the saved logsumexp:
//   dOa = dout * sigmoid(g)           dg = dout * out * (1 - sigmoid(g))
//   D_i = sum_c dout * out            (= sum_j P_ij dP_ij)
//   dP  = dOa V^T      dS = P (dP - D)
//   dV  = P^T dOa      dK = scale dS^T Q      dQ = scale dS K      dbias = sum_b dS
//
// Kernels, in launch order on one stream:
//   pba_bwd_pre_kernel      per query row: dOa (bf16), dg, and (lse * log2 e, D) row stats
//   pba_bwd_main_kernel     CTA = (b, h, 128-key tile): loops over query tiles; dK, dV
//                           accumulate in TMEM; each step's dQ partial is added to an fp32
//                           accumulator in global memory
//   pba_dbias_kernel        CTA = (h, query tile, key tile, split of b): loops over its rows
//                           b with the bias tile resident; dS summed in registers; one fp32
//                           partial tile per split
//   pba_dbias_reduce_kernel sums the split partials in split order (bit-stable dbias)
//   pba_dq_convert_kernel   fp32 dQ accumulator -> bf16 dq (times scale)
#pragma once

#include "pba_device.cuh"

namespace pba {

struct BwdArgs {
    int B, H, Nq, Nk, C;
    int nI, nJ, NqPad, NkPad;
    int splits, rows_per_split;
    float scale;
    int has_bias, has_gate;
    const uint8_t *mask;
    long long smask_b;
    // forward tensors (user layouts)
    const __nv_bfloat16 *gate, *out, *dout;
    long long sg0, sg1, sg2, so0, so1, so2;
    const float *lse;
    // outputs
    __nv_bfloat16 *dq, *dk, *dv, *dgate;
    long long sq0, sq1, sq2, sk0, sk1, sk2, sv0, sv1, sv2;
    float *dbias;
    // workspace
    float2 *rowstats;          // [B][H][NqPad]: (lse * log2 e, or +inf for a dead row; D)
    __nv_bfloat16 *doa;        // [B][Nq][H][C] (only with a gate)
    float *dqacc;              // [B][Nq][H][C]
    float *dbias_part;         // [splits][H][NqPad][NkPad]
};

enum : unsigned {
    SITE_BWD_PROD = 0x201, SITE_BWD_MMA = 0x202, SITE_BWD_EW = 0x203,
    SITE_DB_PROD = 0x301, SITE_DB_MMA = 0x302, SITE_DB_EW = 0x303
};

constexpr float kLog2eB = 1.4426950408889634f;

// ---------------------------------------------------------------------------------------
// pre: one thread per (b, i, h) query row, i < NqPad (padded rows only get row stats)
// ---------------------------------------------------------------------------------------
template <int CP>
__global__ void __launch_bounds__(256) pba_bwd_pre_kernel(const BwdArgs a) {
    const long long n = (long long)a.B * a.NqPad * a.H;
    for (long long r = blockIdx.x * (long long)blockDim.x + threadIdx.x; r < n;
         r += (long long)gridDim.x * blockDim.x) {
        const int h = (int)(r % a.H);
        const long long bi = r / a.H;
        const int i = (int)(bi % a.NqPad);
        const int b = (int)(bi / a.NqPad);
        float2 rs = make_float2(INFINITY, 0.f);
        if (i < a.Nq) {
            const __nv_bfloat16 *op = a.out + b * a.so0 + (long long)i * a.so1 + h * a.so2;
            const __nv_bfloat16 *dp = a.dout + b * a.so0 + (long long)i * a.so1 + h * a.so2;
            const __nv_bfloat16 *gp = a.has_gate ? a.gate + b * a.sg0 + (long long)i * a.sg1 + h * a.sg2 : nullptr;
            __nv_bfloat16 *dgp = a.has_gate ? a.dgate + b * a.sg0 + (long long)i * a.sg1 + h * a.sg2 : nullptr;
            __nv_bfloat16 *dap = a.has_gate ? a.doa + (((long long)b * a.Nq + i) * a.H + h) * a.C : nullptr;
            float D = 0.f;
#pragma unroll
            for (int c8 = 0; c8 < CP / 8; ++c8) {
                if (c8 * 8 >= a.C) break;
                const uint4 o4 = *reinterpret_cast<const uint4 *>(op + c8 * 8);
                const uint4 d4 = *reinterpret_cast<const uint4 *>(dp + c8 * 8);
                const uint32_t ow[4] = {o4.x, o4.y, o4.z, o4.w};
                const uint32_t dw[4] = {d4.x, d4.y, d4.z, d4.w};
                uint32_t gw[4] = {0, 0, 0, 0};
                if (gp) {
                    const uint4 g4 = *reinterpret_cast<const uint4 *>(gp + c8 * 8);
                    gw[0] = g4.x; gw[1] = g4.y; gw[2] = g4.z; gw[3] = g4.w;
                }
                uint32_t dgw[4], daw[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float o0 = bf16lo(ow[e]), o1 = bf16hi(ow[e]);
                    const float d0 = bf16lo(dw[e]), d1 = bf16hi(dw[e]);
                    D = fmaf(d0, o0, D);
                    D = fmaf(d1, o1, D);
                    if (gp) {
                        const float s0 = 1.f / (1.f + __expf(-bf16lo(gw[e])));
                        const float s1 = 1.f / (1.f + __expf(-bf16hi(gw[e])));
                        daw[e] = pack_bf16x2(d0 * s0, d1 * s1);
                        dgw[e] = pack_bf16x2(d0 * o0 * (1.f - s0), d1 * o1 * (1.f - s1));
                    }
                }
                if (gp) {
                    *reinterpret_cast<uint4 *>(dap + c8 * 8) = make_uint4(daw[0], daw[1], daw[2], daw[3]);
                    *reinterpret_cast<uint4 *>(dgp + c8 * 8) = make_uint4(dgw[0], dgw[1], dgw[2], dgw[3]);
                }
            }
            const float l = a.lse[((long long)b * a.H + h) * a.Nq + i];
            rs.x = (l == -INFINITY) ? INFINITY : l * kLog2eB;
            rs.y = D;
        }
        a.rowstats[((long long)b * a.H + h) * a.NqPad + i] = rs;
    }
}

// ---------------------------------------------------------------------------------------
// shared helpers for the two tcgen05 backward kernels
// ---------------------------------------------------------------------------------------

// Mask bits of one 128-key tile for row b, computed by a whole warp:
// word q bit t <-> key j0 + 32 q + t attended (keys >= Nk are never attended).
__device__ __forceinline__ void mask_words(const BwdArgs &a, int b, int j0, uint32_t (&w)[4]) {
    const int lane = lane_id();
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int key = j0 + q * 32 + lane;
        bool valid = key < a.Nk;
        if (valid && a.mask) valid = a.mask[(long long)b * a.smask_b + key] != 0;
        w[q] = __ballot_sync(0xffffffffu, valid);
    }
}

// P and dS of 64 keys (one half of a 128-key tile) for one query row.
//   S, dP: this lane's 64 fp32 values from TMEM; bias: the row's 64 bf16 in a 128-byte
//   swizzled shared-memory row; mask: two 32-bit words for those 64 keys.
// Returns P (fp32) in p[], dS (fp32) in ds[].
__device__ __forceinline__ void p_ds_half(uint32_t tS, uint32_t tdP, uint32_t bias_row, int row,
                                          bool has_bias, uint32_t mw0, uint32_t mw1, bool full,
                                          float scale, float lse2, float D, float (&p)[64],
                                          float (&ds)[64]) {
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        uint32_t r[32];
        tmem_ld32(tS + q * 32, r);
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
            const int c8 = q * 4 + c4;
            uint4 bw = make_uint4(0, 0, 0, 0);
            if (has_bias) bw = lds128(bias_row + ((c8 ^ (row & 7)) << 4));
            const uint32_t bb[4] = {bw.x, bw.y, bw.z, bw.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int c = q * 32 + c4 * 8 + 2 * e;
                const float t0 = fmaf(__uint_as_float(r[c4 * 8 + 2 * e]), scale, bf16lo(bb[e]));
                const float t1 = fmaf(__uint_as_float(r[c4 * 8 + 2 * e + 1]), scale, bf16hi(bb[e]));
                p[c] = ex2(fmaf(t0, kLog2eB, -lse2));
                p[c + 1] = ex2(fmaf(t1, kLog2eB, -lse2));
            }
        }
    }
    if (!full) {
#pragma unroll
        for (int c = 0; c < 64; ++c) {
            const uint32_t wd = c < 32 ? mw0 : mw1;
            if (!((wd >> (c & 31)) & 1u)) p[c] = 0.f;
        }
    }
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        uint32_t r[32];
        tmem_ld32(tdP + q * 32, r);
#pragma unroll
        for (int c = 0; c < 32; ++c) ds[q * 32 + c] = p[q * 32 + c] * (__uint_as_float(r[c]) - D);
    }
}

// ---------------------------------------------------------------------------------------
// main backward kernel: dQ, dK, dV
//
// Persistent: one CTA per SM walks the items (b, h, 128-key tile) n = blockIdx.x,
// blockIdx.x + gridDim.x, ...; an item's steps are its query tiles.  The step pipeline
// (S/dP -> P/dS -> dV, dK, dQ) runs on across item boundaries: the next item's K/V tiles
// load into the other stage while the current item finishes, and dK/dV accumulate in one
// of two TMEM buffers, so an item's dK/dV epilogue (written by the element-wise warps right
// after the next item's first step) overlaps the next item's MMAs.
// ---------------------------------------------------------------------------------------
template <int CP>
struct BwdTraits {
    static constexpr int QS = 2;                                // Q/dOa/row-stat stages
    static constexpr int BS = (CP == 64) ? 1 : 2;               // bias stages
    static constexpr int KVB = (CP == 64) ? 1 : 2;              // K/V stages (items)
    static constexpr int DKB = (CP == 64) ? 1 : 2;              // dK/dV TMEM buffers (items)
    static constexpr int TILE_BYTES = 128 * CP * 2;
    static constexpr int BIAS_BYTES = 128 * 128 * 2;
    static constexpr int PS_BYTES = 128 * 128 * 2;              // P or dS tile (bf16)
    static constexpr int OFF_K = 0;                             // + x * TILE_BYTES
    static constexpr int OFF_V = OFF_K + KVB * TILE_BYTES;      // + x * TILE_BYTES
    static constexpr int OFF_Q = OFF_V + KVB * TILE_BYTES;      // + st * 2 * TILE_BYTES
    static constexpr int OFF_P = OFF_Q + QS * 2 * TILE_BYTES;
    static constexpr int OFF_DS = OFF_P + PS_BYTES;
    static constexpr int OFF_BIAS = OFF_DS + PS_BYTES;          // + bs * BIAS_BYTES
    static constexpr int OFF_RS = OFF_BIAS + BS * BIAS_BYTES;   // float2 [QS][128]
    static constexpr int OFF_MASK = OFF_RS + QS * 1024;         // u32 [KVB][8]
    static constexpr int SMEM_BYTES = OFF_MASK + KVB * 32 + 1024;
    static constexpr uint32_t SWZ = CP == 64 ? kSw128 : (CP == 32 ? kSw64 : kSw32);
    static constexpr uint32_t ROWB = CP * 2;
    // TMEM columns: S, dP, then per dK/dV buffer x: dK at T_DK + 2 CP x, dV after it, then
    // the two dQ buffers
    static constexpr int T_S = 0, T_DP = 128, T_DK = 256, T_DQ = 256 + DKB * 2 * CP;
    static_assert(T_DQ + 2 * CP <= 512, "TMEM");
};
static_assert(BwdTraits<64>::SMEM_BYTES <= 232448 && BwdTraits<32>::SMEM_BYTES <= 232448, "smem");

template <int CP>
__global__ void __launch_bounds__(320, 1)
pba_bwd_main_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                    const __grid_constant__ CUtensorMap tmBias, const BwdArgs a) {
    using T = BwdTraits<CP>;
    constexpr int QS = T::QS, BS = T::BS, KVB = T::KVB, DKB = T::DKB;
    extern __shared__ uint8_t dsmem[];
    __shared__ __align__(8) uint64_t bars[16 + 2 * QS + 2 * BS + 2 * KVB + 2 * DKB];
    __shared__ uint32_t s_tmem_base;
    __shared__ int s_abort;

    const uint32_t b_sd_full = smem_u32(&bars[1]);
    const uint32_t b_sd_free = smem_u32(&bars[2]);
    const uint32_t b_ps_full = smem_u32(&bars[3]);
    const uint32_t b_ps_free = smem_u32(&bars[4]);
    const uint32_t b_drain = smem_u32(&bars[6]);
    auto b_dq_full = [&](int x) { return smem_u32(&bars[8 + x]); };
    auto b_dq_free = [&](int x) { return smem_u32(&bars[10 + x]); };
    auto b_q_full = [&](int x) { return smem_u32(&bars[16 + x]); };
    auto b_q_empty = [&](int x) { return smem_u32(&bars[16 + QS + x]); };
    auto b_bias_full = [&](int x) { return smem_u32(&bars[16 + 2 * QS + x]); };
    auto b_bias_empty = [&](int x) { return smem_u32(&bars[16 + 2 * QS + BS + x]); };
    constexpr int OK_ = 16 + 2 * QS + 2 * BS;
    auto b_kv_full = [&](int x) { return smem_u32(&bars[OK_ + x]); };          // K, V, mask words
    auto b_kv_empty = [&](int x) { return smem_u32(&bars[OK_ + KVB + x]); };   // item's MMAs done
    auto b_dkv_full = [&](int x) { return smem_u32(&bars[OK_ + 2 * KVB + x]); };        // dK/dV final
    auto b_dkv_free = [&](int x) { return smem_u32(&bars[OK_ + 2 * KVB + DKB + x]); };  // read out

    const uint32_t raw = smem_u32(dsmem);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    uint8_t *gbase = dsmem + (sbase - raw);

    const int warp = warp_id(), lane = lane_id();
    const int nI = a.nI;
    const long long n_items = (long long)a.B * a.H * a.nJ;
    // items of this CTA: blockIdx.x + m * gridDim.x, m < M; steps t = m * nI + i
    const int M = blockIdx.x < n_items ? (int)((n_items - 1 - blockIdx.x) / gridDim.x) + 1 : 0;
    const int Tn = M * nI;
    struct Item { int b, h, jt; };
    auto item = [&](int m) {
        long long n = blockIdx.x + (long long)m * gridDim.x;
        Item it;
        it.jt = (int)(n % a.nJ);
        n /= a.nJ;
        it.h = (int)(n % a.H);
        it.b = (int)(n / a.H);
        return it;
    };

    if (threadIdx.x == 0) {
        mbar_init(b_sd_full, 1);
        mbar_init(b_sd_free, 256);
        mbar_init(b_ps_full, 256);
        mbar_init(b_ps_free, 1);
        mbar_init(b_drain, 1);
        for (int x = 0; x < 2; ++x) {
            mbar_init(b_dq_full(x), 1);
            mbar_init(b_dq_free(x), 256);
        }
        for (int x = 0; x < QS; ++x) {
            mbar_init(b_q_full(x), 1);
            mbar_init(b_q_empty(x), 1 + 256);
        }
        for (int x = 0; x < BS; ++x) {
            mbar_init(b_bias_full(x), 1);
            mbar_init(b_bias_empty(x), 256);
        }
        for (int x = 0; x < KVB; ++x) {
            mbar_init(b_kv_full(x), 1);
            mbar_init(b_kv_empty(x), 1);
        }
        for (int x = 0; x < DKB; ++x) {
            mbar_init(b_dkv_full(x), 1);
            mbar_init(b_dkv_free(x), 256);
        }
        s_abort = 0;
        fence_mbar_init();
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
    // loads issued: items [0, kv_done), steps [0, q_done) (Q/dOa/row stats), [0, bias_done)
    int kv_done = 0, q_done = 0, bias_done = 0;

    if (warp == 8) {
        // ------------------------------------------------------------------ producer
        if (lane == 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            tma_prefetch_desc(&tmDO);
            if (a.has_bias) tma_prefetch_desc(&tmBias);
        }
        bool ok = true;
        for (int m = 0; m < M && ok; ++m) {
            const Item it = item(m);
            const int x = m % KVB, j0 = it.jt * 128;
            if (m >= KVB)
                ok = mbar_wait(b_kv_empty(x), ((m / KVB) - 1) & 1, abort_flag, SITE_BWD_PROD | 0x10 | (m << 12));
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            uint32_t w[4];
            mask_words(a, it.b, j0, w);
            if (lane == 0) {
                uint32_t *mw = reinterpret_cast<uint32_t *>(gbase + T::OFF_MASK) + x * 8;
                mw[0] = w[0]; mw[1] = w[1]; mw[2] = w[2]; mw[3] = w[3];
                mw[4] = (w[0] & w[1]) == 0xffffffffu;
                mw[5] = (w[2] & w[3]) == 0xffffffffu;
                mbar_arrive_tx(b_kv_full(x), 2 * T::TILE_BYTES);
                tma_load_4d(sbase + T::OFF_K + x * T::TILE_BYTES, &tmK, b_kv_full(x), 0, it.h, j0, it.b);
                tma_load_4d(sbase + T::OFF_V + x * T::TILE_BYTES, &tmV, b_kv_full(x), 0, it.h, j0, it.b);
            }
            kv_done = m + 1;
            for (int i = 0; i < nI && ok; ++i) {
                const int t = m * nI + i, st = t % QS, bs = t % BS, i0 = i * 128;
                if (t >= QS) ok = mbar_wait(b_q_empty(st), ((t / QS) - 1) & 1, abort_flag, SITE_BWD_PROD | (t << 12));
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                if (lane == 0) {
                    const uint32_t qdst = sbase + T::OFF_Q + st * 2 * T::TILE_BYTES;
                    mbar_arrive_tx(b_q_full(st), 2 * T::TILE_BYTES + 1024);
                    tma_load_4d(qdst, &tmQ, b_q_full(st), 0, it.h, i0, it.b);
                    tma_load_4d(qdst + T::TILE_BYTES, &tmDO, b_q_full(st), 0, it.h, i0, it.b);
                    bulk_load(sbase + T::OFF_RS + st * 1024,
                              a.rowstats + ((long long)it.b * a.H + it.h) * a.NqPad + i0, 1024, b_q_full(st));
                }
                q_done = t + 1;
                if (t >= BS) ok = mbar_wait(b_bias_empty(bs), ((t / BS) - 1) & 1, abort_flag, SITE_BWD_PROD | 0x20 | (t << 12));
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                if (lane == 0) {
                    if (a.has_bias) {
                        const uint32_t dst = sbase + T::OFF_BIAS + bs * T::BIAS_BYTES;
                        mbar_arrive_tx(b_bias_full(bs), T::BIAS_BYTES);
                        tma_load_3d(dst, &tmBias, b_bias_full(bs), j0, i0, it.h);
                        tma_load_3d(dst + 16384, &tmBias, b_bias_full(bs), j0 + 64, i0, it.h);
                    } else {
                        mbar_arrive(b_bias_full(bs));
                    }
                }
                bias_done = t + 1;
            }
        }
    } else if (warp == 9) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t SBO = 8 * T::ROWB;
            constexpr uint32_t id_s = idesc_bf16(128, 128, false, false);   // S = Q K^T, dP = dOa V^T
            constexpr uint32_t id_kv = idesc_bf16(128, CP, true, true);     // dV = P^T dOa, dK = dS^T Q
            constexpr uint32_t id_q = idesc_bf16(128, CP, false, true);     // dQ = dS K
            const uint32_t sP = sbase + T::OFF_P, sDS = sbase + T::OFF_DS;
            auto issue_sdp = [&](int t) {
                const int st = t % QS, x = (t / nI) % KVB;
                const uint32_t sQ = sbase + T::OFF_Q + st * 2 * T::TILE_BYTES;
                const uint32_t sDO = sQ + T::TILE_BYTES;
                const uint32_t sK = sbase + T::OFF_K + x * T::TILE_BYTES;
                const uint32_t sV = sbase + T::OFF_V + x * T::TILE_BYTES;
#pragma unroll
                for (int kk = 0; kk < CP / 16; ++kk) {
                    umma_ss(tbase + T::T_S, sdesc(sQ + kk * 32, 16, SBO, T::SWZ),
                            sdesc(sK + kk * 32, 16, SBO, T::SWZ), id_s, kk > 0);
                    umma_ss(tbase + T::T_DP, sdesc(sDO + kk * 32, 16, SBO, T::SWZ),
                            sdesc(sV + kk * 32, 16, SBO, T::SWZ), id_s, kk > 0);
                }
                umma_commit(b_sd_full);
            };
            bool ok = true;
            if (Tn > 0) {
                ok = mbar_wait(b_kv_full(0), 0, abort_flag, SITE_BWD_MMA | 0x10);
                if (ok) ok = mbar_wait(b_q_full(0), 0, abort_flag, SITE_BWD_MMA);
                if (ok) {
                    tc_fence_after();
                    issue_sdp(0);
                }
            }
            for (int t = 0; t < Tn && ok; ++t) {
                const int m = t / nI, i = t % nI, st = t % QS;
                const int x = m % KVB, d = m % DKB;
                ok = mbar_wait(b_ps_full, t & 1, abort_flag, SITE_BWD_MMA | 0x20 | (t << 12));
                if (!ok) break;
                // S/dP of the next step go ahead of this step's products, except when the
                // next step starts an item whose K/V reuse this item's stage: those tiles
                // only load once this item's MMAs are done, so they follow them.
                const int m1 = (t + 1) / nI;
                const bool late = t + 1 < Tn && m1 != m && m1 % KVB == x;
                auto next_sdp = [&]() -> bool {
                    bool okn = true;
                    if (m1 != m)
                        okn = mbar_wait(b_kv_full(m1 % KVB), (m1 / KVB) & 1, abort_flag, SITE_BWD_MMA | 0x30 | (t << 12));
                    if (okn) okn = mbar_wait(b_q_full((t + 1) % QS), ((t + 1) / QS) & 1, abort_flag, SITE_BWD_MMA | 0x40 | (t << 12));
                    if (okn) okn = mbar_wait(b_sd_free, t & 1, abort_flag, SITE_BWD_MMA | 0x50 | (t << 12));
                    if (!okn) return false;
                    tc_fence_after();
                    issue_sdp(t + 1);
                    return true;
                };
                if (t + 1 < Tn && !late) {
                    ok = next_sdp();
                    if (!ok) break;
                }
                if (i == 0 && m >= DKB) {
                    // this item's dK/dV buffer: the epilogue of item m - DKB has read it
                    ok = mbar_wait(b_dkv_free(d), ((m / DKB) - 1) & 1, abort_flag, SITE_BWD_MMA | 0x60 | (t << 12));
                    if (!ok) break;
                }
                if (t >= 2) {
                    ok = mbar_wait(b_dq_free(t & 1), ((t >> 1) - 1) & 1, abort_flag, SITE_BWD_MMA | 0x70 | (t << 12));
                    if (!ok) break;
                }
                tc_fence_after();
                const uint32_t sQ = sbase + T::OFF_Q + st * 2 * T::TILE_BYTES;
                const uint32_t sDO = sQ + T::TILE_BYTES;
                const uint32_t sK = sbase + T::OFF_K + x * T::TILE_BYTES;
                const uint32_t tDK = tbase + T::T_DK + d * 2 * CP, tDV = tDK + CP;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    // K steps over 16 queries: A (P^T / dS^T, MN-major) rows advance 2 KB,
                    // B (dOa / Q, MN-major) rows advance 16 rows
                    const uint32_t acc = (i > 0 || kk > 0) ? 1u : 0u;
                    umma_ss(tDV, sdesc(sP + kk * 2048, 16384, 1024, kSw128),
                            sdesc(sDO + kk * 16 * T::ROWB, T::TILE_BYTES, SBO, T::SWZ), id_kv, acc);
                    umma_ss(tDK, sdesc(sDS + kk * 2048, 16384, 1024, kSw128),
                            sdesc(sQ + kk * 16 * T::ROWB, T::TILE_BYTES, SBO, T::SWZ), id_kv, acc);
                }
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    // K steps over 16 keys: A (dS, K-major) advances 32 B within a 64-key half
                    const uint32_t a_addr = sDS + (kk >> 2) * 16384 + (kk & 3) * 32;
                    umma_ss(tbase + T::T_DQ + (t & 1) * CP, sdesc(a_addr, 16, 1024, kSw128),
                            sdesc(sK + kk * 16 * T::ROWB, T::TILE_BYTES, SBO, T::SWZ), id_q, kk > 0);
                }
                umma_commit(b_ps_free);
                umma_commit(b_q_empty(st));
                umma_commit(b_dq_full(t & 1));
                if (i == nI - 1) {
                    umma_commit(b_dkv_full(d));
                    umma_commit(b_kv_empty(x));
                }
                if (late) ok = next_sdp();
            }
        }
    } else {
        // ------------------------------------------------------------------ elementwise
        // warpgroup e owns keys [64 e, 64 e + 64) of the tile for all 128 query rows
        const int e = warp >> 2;
        const int row = (warp & 3) * 32 + lane;
        const uint32_t lane_off = ((uint32_t)((warp & 3) * 32)) << 16;
        const float scale = a.scale;
        bool ok = true;
        auto flush_dq = [&](int t) -> bool {
            // dQ(t): this thread's query row, channels [e CP/2, (e+1) CP/2), added to dqacc
            bool okf = mbar_wait(b_dq_full(t & 1), (t >> 1) & 1, abort_flag, SITE_BWD_EW | 0x10 | (t << 12));
            okf = __all_sync(0xffffffffu, okf);
            if (!okf) return false;
            tc_fence_after();
            uint32_t r[CP / 2];
            const uint32_t taddr = tbase + T::T_DQ + (t & 1) * CP + e * (CP / 2) + lane_off;
            if constexpr (CP / 2 == 8) {
                uint32_t r16[16];
                tmem_ld16(taddr, r16);  // reads 16 columns; only the first 8 are this half's
#pragma unroll
                for (int c = 0; c < 8; ++c) r[c] = r16[c];
            } else if constexpr (CP / 2 == 16) {
                tmem_ld16(taddr, r);
            } else {
                tmem_ld32(taddr, r);
            }
            tc_fence_before();
            mbar_arrive(b_dq_free(t & 1));
            const Item it = item(t / nI);
            const int i = (t % nI) * 128 + row;
            if (i < a.Nq) {
                float *dst = a.dqacc + (((long long)it.b * a.Nq + i) * a.H + it.h) * a.C;
#pragma unroll
                for (int c4 = 0; c4 < CP / 8; ++c4) {
                    const int c = e * (CP / 2) + c4 * 4;
                    if (c < a.C)
                        atomicAdd(reinterpret_cast<float4 *>(dst + c),
                                  make_float4(__uint_as_float(r[c4 * 4]), __uint_as_float(r[c4 * 4 + 1]),
                                              __uint_as_float(r[c4 * 4 + 2]), __uint_as_float(r[c4 * 4 + 3])));
                }
            }
            return true;
        };
        auto epilogue = [&](int m) -> bool {
            // dK/dV of item m: warpgroup 0 writes dK (times scale), warpgroup 1 dV; lane = key
            bool oke = mbar_wait(b_dkv_full(m % DKB), (m / DKB) & 1, abort_flag, SITE_BWD_EW | 0x20 | (m << 12));
            oke = __all_sync(0xffffffffu, oke);
            if (!oke) return false;
            tc_fence_after();
            uint32_t r[CP];
            tmem_ld_cols<CP>(tbase + T::T_DK + (m % DKB) * 2 * CP + e * CP + lane_off, r);
            tc_fence_before();
            mbar_arrive(b_dkv_free(m % DKB));
            const Item it = item(m);
            const int j = it.jt * 128 + row;
            if (j < a.Nk) {
                __nv_bfloat16 *dst = e == 0 ? a.dk + it.b * a.sk0 + (long long)j * a.sk1 + it.h * a.sk2
                                            : a.dv + it.b * a.sv0 + (long long)j * a.sv1 + it.h * a.sv2;
                const float mul = e == 0 ? a.scale : 1.f;
#pragma unroll
                for (int c8 = 0; c8 < CP / 8; ++c8) {
                    if (c8 * 8 < a.C) {
                        uint32_t ow[4];
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            ow[q] = pack_bf16x2(__uint_as_float(r[c8 * 8 + 2 * q]) * mul,
                                                __uint_as_float(r[c8 * 8 + 2 * q + 1]) * mul);
                        *reinterpret_cast<uint4 *>(dst + c8 * 8) = make_uint4(ow[0], ow[1], ow[2], ow[3]);
                    }
                }
            }
            return true;
        };
        uint32_t mw0 = 0, mw1 = 0;
        bool full = true;
        for (int t = 0; t < Tn && ok; ++t) {
            const int m = t / nI, i = t % nI, st = t % QS, bs = t % BS;
            if (i == 0) {
                // this item's mask words come with its K/V tiles
                ok = mbar_wait(b_kv_full(m % KVB), (m / KVB) & 1, abort_flag, SITE_BWD_EW | 0x30 | (t << 12));
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                const uint32_t *mw = reinterpret_cast<const uint32_t *>(gbase + T::OFF_MASK) + (m % KVB) * 8;
                mw0 = mw[2 * e];
                mw1 = mw[2 * e + 1];
                full = mw[4 + e] != 0;
            }
            ok = mbar_wait(b_sd_full, t & 1, abort_flag, SITE_BWD_EW | (t << 12));
            if (ok) ok = mbar_wait(b_q_full(st), (t / QS) & 1, abort_flag, SITE_BWD_EW | 0x40 | (t << 12));
            if (ok) ok = mbar_wait(b_bias_full(bs), (t / BS) & 1, abort_flag, SITE_BWD_EW | 0x50 | (t << 12));
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            const float2 rs = reinterpret_cast<const float2 *>(gbase + T::OFF_RS + st * 1024)[row];
            float p[64], ds[64];
            const uint32_t bias_row = sbase + T::OFF_BIAS + bs * T::BIAS_BYTES + e * 16384 + row * 128;
            p_ds_half(tbase + T::T_S + e * 64 + lane_off, tbase + T::T_DP + e * 64 + lane_off, bias_row,
                      row, a.has_bias != 0, mw0, mw1, full, scale, rs.x, rs.y, p, ds);
            tc_fence_before();
            mbar_arrive(b_sd_free);
            mbar_arrive(b_bias_empty(bs));
            mbar_arrive(b_q_empty(st));
            if (t > 0) {
                ok = mbar_wait(b_ps_free, (t - 1) & 1, abort_flag, SITE_BWD_EW | 0x60 | (t << 12));
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
            }
            // P and dS (bf16) into their 128-byte swizzled tiles: half e, row `row`
            const uint32_t prow = sbase + T::OFF_P + e * 16384 + row * 128;
            const uint32_t drow = sbase + T::OFF_DS + e * 16384 + row * 128;
#pragma unroll
            for (int c8 = 0; c8 < 8; ++c8) {
                const uint32_t sw = (uint32_t)((c8 ^ (row & 7)) << 4);
                sts128(prow + sw, make_uint4(pack_bf16x2(p[c8 * 8 + 0], p[c8 * 8 + 1]),
                                             pack_bf16x2(p[c8 * 8 + 2], p[c8 * 8 + 3]),
                                             pack_bf16x2(p[c8 * 8 + 4], p[c8 * 8 + 5]),
                                             pack_bf16x2(p[c8 * 8 + 6], p[c8 * 8 + 7])));
                sts128(drow + sw, make_uint4(pack_bf16x2(ds[c8 * 8 + 0], ds[c8 * 8 + 1]),
                                             pack_bf16x2(ds[c8 * 8 + 2], ds[c8 * 8 + 3]),
                                             pack_bf16x2(ds[c8 * 8 + 4], ds[c8 * 8 + 5]),
                                             pack_bf16x2(ds[c8 * 8 + 6], ds[c8 * 8 + 7])));
            }
            // generic-proxy writes -> visible to the tensor core's async proxy
            fence_proxy_async();
            mbar_arrive(b_ps_full);
            if (t > 0) ok = flush_dq(t - 1);
            if (ok && i == 0 && m > 0) ok = epilogue(m - 1);
        }
        if (ok && Tn > 0) ok = flush_dq(Tn - 1);
        if (ok && M > 0) ok = epilogue(M - 1);
    }

    tc_fence_before();
    __syncthreads();
    if (*abort_flag) {
        // a wait ran out: let the copies and MMAs already issued finish before shared memory
        // and TMEM are released (bounded waits)
        if (warp == 8 && lane == 0) {
            for (int mm = max(0, kv_done - KVB); mm < kv_done; ++mm)
                mbar_wait_drain(b_kv_full(mm % KVB), (mm / KVB) & 1);
            for (int tt = max(0, q_done - QS); tt < q_done; ++tt) mbar_wait_drain(b_q_full(tt % QS), (tt / QS) & 1);
            for (int tt = max(0, bias_done - BS); tt < bias_done; ++tt)
                mbar_wait_drain(b_bias_full(tt % BS), (tt / BS) & 1);
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

// ---------------------------------------------------------------------------------------
// dbias kernel: CTA = (h, query tile, key tile, split s); loops over its rows b
// ---------------------------------------------------------------------------------------
template <int CP>
struct DbTraits {
    static constexpr int NS = (CP == 64) ? 2 : 3;                 // stages (one row b each)
    static constexpr int TILE_BYTES = 128 * CP * 2;
    static constexpr int STAGE_BYTES = 4 * TILE_BYTES + 1024;     // Q, dOa, K, V, row stats
    static constexpr int OFF_BIAS = 0;
    static constexpr int OFF_STAGE = 128 * 128 * 2;               // + st * STAGE_BYTES
    static constexpr int OFF_MASK = OFF_STAGE + NS * STAGE_BYTES; // u32 [NS][8]
    static constexpr int SMEM_BYTES = OFF_MASK + NS * 32 + 1024;
    static constexpr uint32_t SWZ = CP == 64 ? kSw128 : (CP == 32 ? kSw64 : kSw32);
    static constexpr uint32_t ROWB = CP * 2;
};

template <int CP>
__global__ void __launch_bounds__(320, 1)
pba_dbias_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                 const __grid_constant__ CUtensorMap tmBias, const BwdArgs a) {
    using T = DbTraits<CP>;
    constexpr int NS = T::NS;
    extern __shared__ uint8_t dsmem[];
    __shared__ __align__(8) uint64_t bars[8 + 2 * NS];
    __shared__ uint32_t s_tmem_base;
    __shared__ int s_abort;

    const uint32_t b_bias = smem_u32(&bars[0]);
    const uint32_t b_drain = smem_u32(&bars[1]);
    auto b_sd_full = [&](int x) { return smem_u32(&bars[2 + x]); };
    auto b_sd_free = [&](int x) { return smem_u32(&bars[4 + x]); };
    auto b_full = [&](int x) { return smem_u32(&bars[8 + x]); };
    auto b_empty = [&](int x) { return smem_u32(&bars[8 + NS + x]); };

    const uint32_t raw = smem_u32(dsmem);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    uint8_t *gbase = dsmem + (sbase - raw);

    const int warp = warp_id(), lane = lane_id();
    int idx = blockIdx.x;
    const int jt = idx % a.nJ;
    idx /= a.nJ;
    const int it = idx % a.nI;
    idx /= a.nI;
    const int h = idx % a.H;
    const int sp = idx / a.H;
    const int i0 = it * 128, j0 = jt * 128;
    const int bstart = sp * a.rows_per_split;
    const int nb = max(0, min(a.rows_per_split, a.B - bstart));

    if (threadIdx.x == 0) {
        mbar_init(b_bias, 1);
        mbar_init(b_drain, 1);
        for (int x = 0; x < 2; ++x) {
            mbar_init(b_sd_full(x), 1);
            mbar_init(b_sd_free(x), 256);
        }
        for (int x = 0; x < NS; ++x) {
            mbar_init(b_full(x), 1);
            mbar_init(b_empty(x), 1 + 256);
        }
        s_abort = 0;
        fence_mbar_init();
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
    int n_done = 0;   // rows b whose stage loads were issued: [0, n_done)

    if (warp == 8) {
        // ------------------------------------------------------------------ producer
        if (lane == 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            tma_prefetch_desc(&tmDO);
            if (a.has_bias) {
                tma_prefetch_desc(&tmBias);
                mbar_arrive_tx(b_bias, 128 * 128 * 2);
                tma_load_3d(sbase + T::OFF_BIAS, &tmBias, b_bias, j0, i0, h);
                tma_load_3d(sbase + T::OFF_BIAS + 16384, &tmBias, b_bias, j0 + 64, i0, h);
            } else {
                mbar_arrive(b_bias);
            }
        }
        bool ok = true;
        int n = 0;
        for (; n < nb; ++n) {
            const int st = n % NS, b = bstart + n;
            if (n >= NS) ok = mbar_wait(b_empty(st), ((n / NS) - 1) & 1, abort_flag, SITE_DB_PROD);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            uint32_t w[4];
            mask_words(a, b, j0, w);
            if (lane == 0) {
                uint32_t *mw = reinterpret_cast<uint32_t *>(gbase + T::OFF_MASK) + st * 8;
                mw[0] = w[0]; mw[1] = w[1]; mw[2] = w[2]; mw[3] = w[3];
                mw[4] = (w[0] & w[1]) == 0xffffffffu;
                mw[5] = (w[2] & w[3]) == 0xffffffffu;
                const uint32_t s0 = sbase + T::OFF_STAGE + st * T::STAGE_BYTES;
                mbar_arrive_tx(b_full(st), 4 * T::TILE_BYTES + 1024);
                tma_load_4d(s0, &tmQ, b_full(st), 0, h, i0, b);
                tma_load_4d(s0 + T::TILE_BYTES, &tmDO, b_full(st), 0, h, i0, b);
                tma_load_4d(s0 + 2 * T::TILE_BYTES, &tmK, b_full(st), 0, h, j0, b);
                tma_load_4d(s0 + 3 * T::TILE_BYTES, &tmV, b_full(st), 0, h, j0, b);
                bulk_load(s0 + 4 * T::TILE_BYTES, a.rowstats + ((long long)b * a.H + h) * a.NqPad + i0,
                          1024, b_full(st));
            }
            n_done = n + 1;
        }
    } else if (warp == 9) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t SBO = 8 * T::ROWB;
            constexpr uint32_t id_s = idesc_bf16(128, 128, false, false);
            bool ok = true;
            for (int n = 0; n < nb && ok; ++n) {
                const int st = n % NS, x = n & 1;
                ok = mbar_wait(b_full(st), (n / NS) & 1, abort_flag, SITE_DB_MMA);
                if (ok && n >= 2) ok = mbar_wait(b_sd_free(x), ((n >> 1) - 1) & 1, abort_flag, SITE_DB_MMA);
                if (!ok) break;
                tc_fence_after();
                const uint32_t s0 = sbase + T::OFF_STAGE + st * T::STAGE_BYTES;
                const uint32_t sQ = s0, sDO = s0 + T::TILE_BYTES, sK = s0 + 2 * T::TILE_BYTES,
                               sV = s0 + 3 * T::TILE_BYTES;
#pragma unroll
                for (int kk = 0; kk < CP / 16; ++kk) {
                    umma_ss(tbase + x * 256, sdesc(sQ + kk * 32, 16, SBO, T::SWZ),
                            sdesc(sK + kk * 32, 16, SBO, T::SWZ), id_s, kk > 0);
                    umma_ss(tbase + x * 256 + 128, sdesc(sDO + kk * 32, 16, SBO, T::SWZ),
                            sdesc(sV + kk * 32, 16, SBO, T::SWZ), id_s, kk > 0);
                }
                umma_commit(b_sd_full(x));
                umma_commit(b_empty(st));
            }
        }
    } else {
        // ------------------------------------------------------------------ elementwise
        const int e = warp >> 2;
        const int row = (warp & 3) * 32 + lane;
        const uint32_t lane_off = ((uint32_t)((warp & 3) * 32)) << 16;
        const float scale = a.scale;
        float acc[64];
#pragma unroll
        for (int c = 0; c < 64; ++c) acc[c] = 0.f;
        bool ok = mbar_wait(b_bias, 0, abort_flag, SITE_DB_EW);
        ok = __all_sync(0xffffffffu, ok);
        const uint32_t bias_row = sbase + T::OFF_BIAS + e * 16384 + row * 128;
        for (int n = 0; n < nb && ok; ++n) {
            const int st = n % NS, x = n & 1;
            ok = mbar_wait(b_sd_full(x), (n >> 1) & 1, abort_flag, SITE_DB_EW);
            if (ok) ok = mbar_wait(b_full(st), (n / NS) & 1, abort_flag, SITE_DB_EW);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            const uint8_t *s0 = gbase + T::OFF_STAGE + st * T::STAGE_BYTES;
            const float2 rs = reinterpret_cast<const float2 *>(s0 + 4 * T::TILE_BYTES)[row];
            const uint32_t *mw = reinterpret_cast<const uint32_t *>(gbase + T::OFF_MASK) + st * 8;
            float p[64], ds[64];
            p_ds_half(tbase + x * 256 + e * 64 + lane_off, tbase + x * 256 + 128 + e * 64 + lane_off,
                      bias_row, row, a.has_bias != 0, mw[2 * e], mw[2 * e + 1], mw[4 + e] != 0, scale,
                      rs.x, rs.y, p, ds);
            tc_fence_before();
            mbar_arrive(b_sd_free(x));
            mbar_arrive(b_empty(st));
#pragma unroll
            for (int c = 0; c < 64; ++c) acc[c] += ds[c];
        }
        if (ok) {
            // this split's partial tile, padded layout: [split][h][NqPad][NkPad]
            float *dst = a.dbias_part +
                         ((((long long)sp * a.H + h) * a.NqPad + i0 + row) * a.NkPad + j0 + e * 64);
#pragma unroll
            for (int c = 0; c < 64; c += 4)
                *reinterpret_cast<float4 *>(dst + c) = make_float4(acc[c], acc[c + 1], acc[c + 2], acc[c + 3]);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (*abort_flag) {
        if (warp == 8 && lane == 0) {
            mbar_wait_drain(b_bias, 0);
            for (int nn = max(0, n_done - NS); nn < n_done; ++nn) mbar_wait_drain(b_full(nn % NS), (nn / NS) & 1);
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

// dbias[h][i][j] = sum over splits s = 0, 1, ... of the partial tiles, in that order.
__global__ void __launch_bounds__(256) pba_dbias_reduce_kernel(const BwdArgs a) {
    const long long n = (long long)a.H * a.Nq * a.Nk;
    const long long plane = (long long)a.H * a.NqPad * a.NkPad;
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n;
         e += (long long)gridDim.x * blockDim.x) {
        const int j = (int)(e % a.Nk);
        const long long hi = e / a.Nk;
        const int i = (int)(hi % a.Nq);
        const int h = (int)(hi / a.Nq);
        const float *src = a.dbias_part + ((long long)h * a.NqPad + i) * a.NkPad + j;
        float s = 0.f;
        for (int sp = 0; sp < a.splits; ++sp) s += src[sp * plane];
        a.dbias[e] = s;
    }
}

// dq = bf16(scale * dqacc), eight channels per thread.
__global__ void __launch_bounds__(256) pba_dq_convert_kernel(const BwdArgs a) {
    const int c8n = a.C / 8;
    const long long n = (long long)a.B * a.Nq * a.H * c8n;
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n;
         e += (long long)gridDim.x * blockDim.x) {
        const int c8 = (int)(e % c8n);
        const long long r = e / c8n;
        const int h = (int)(r % a.H);
        const long long bi = r / a.H;
        const int i = (int)(bi % a.Nq);
        const int b = (int)(bi / a.Nq);
        const float4 *src = reinterpret_cast<const float4 *>(a.dqacc + r * a.C + c8 * 8);
        const float4 x0 = src[0], x1 = src[1];
        const float s = a.scale;
        __nv_bfloat16 *dst = a.dq + b * a.sq0 + (long long)i * a.sq1 + h * a.sq2 + c8 * 8;
        *reinterpret_cast<uint4 *>(dst) =
            make_uint4(pack_bf16x2(x0.x * s, x0.y * s), pack_bf16x2(x0.z * s, x0.w * s),
                       pack_bf16x2(x1.x * s, x1.y * s), pack_bf16x2(x1.z * s, x1.w * s));
    }
}

}  // namespace pba
