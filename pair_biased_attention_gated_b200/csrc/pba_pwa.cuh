// MSA pair-weighted averaging ("AlphaFold3 open-source implementation" page, sections "MSA
// Pair Averaging" and "Model Efficiency"): the value rows of every MSA sequence b are averaged
// with weights from the pair representation alone, shared by all sequences:
//
//   w[h,i,j] = softmax_j(bias[h,i,j] + mask_j)     (once per (h, i), not per b)
//   out[b,i,h,:] = sigmoid(g) * sum_j w[h,i,j] v[b,j,h,:]
//   backward: dOa = dout sigmoid(g); dg = dout out (1 - sigmoid(g));
//             dv[b,j,h,:] = sum_i w[h,i,j] dOa[b,i,h,:];
//             dW[h,i,j] = sum_b sum_c dOa[b,i,h,c] v[b,j,h,c];
//             dbias = w (dW - sum_j w dW)
//
// Kernels:
//   pba_pwa_weights_kernel  one warp per (h, i): w as bf16 (the MMA operand) and lse_w
//   pba_pwa_gemm_kernel<CP, DV>
//                           the two contractions with w on the tensor cores, as one
//                           template: out[b] = sigmoid(g) (W V[b])  (DV = false, rows i) and
//                           dv[b] = W^T dOa[b]  (DV = true, rows j).  CTA = (h, 128 output
//                           rows, chunk of BC rows b); the W tile of each reduction tile is
//                           loaded once and reused by the chunk's rows.
//   pba_pwa_pre_kernel      dOa and dg
//   pba_pwa_dw_kernel<CP>   dW partials: CTA = (h, query tile, key tile, split of b), dW
//                           accumulates over the split's rows in TMEM
//   pba_pwa_dbias_kernel    one warp per (h, i): dW = sum of the split partials in split
//                           order, w recomputed in fp32 from bias and lse_w, dbias = w (dW - r)
//                           with r reduced in a fixed order (bit-stable)
#pragma once

#include "pba_device.cuh"

namespace pba {

struct PwaArgs {
    int B, H, N, C;
    int nT, nChunks, NPad, Wld;   // tiles of 128 rows, chunks of rows b, N rounded up to 128,
                                  // row length of the w buffer (N rounded up to 8)
    int splits, rows_per_split;
    int has_bias, has_gate;
    const __nv_bfloat16 *bias;
    long long sb0, sb1;           // bias strides (head, row); key stride 1
    const uint8_t *mask;          // [N] shared by every b, or null
    const __nv_bfloat16 *gate;
    long long sg0, sg1, sg2;
    __nv_bfloat16 *out;           // out (forward) or dv (dv pass)
    long long so0, so1, so2;
    const __nv_bfloat16 *oin, *dout;   // pre: gated output and its gradient
    long long si0, si1, si2;
    __nv_bfloat16 *w;             // [H][N][Wld] bf16
    float *lse;                   // [H][N]
    __nv_bfloat16 *doa;           // [B][N][H][C] bf16 (with a gate)
    __nv_bfloat16 *dgate;
    float *dw_part;               // [splits][H][NPad][NPad]
    float *dbias;                 // [H][N][N]
};

enum : unsigned { SITE_PWA_PROD = 0x401, SITE_PWA_MMA = 0x402, SITE_PWA_EPI = 0x403, SITE_PWA_ALIGN = 0x4FF };

// ---------------------------------------------------------------------------------------
// weights: one warp per (h, i) row
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) pba_pwa_weights_kernel(const PwaArgs a) {
    const int lane = threadIdx.x & 31;
    const long long nrows = (long long)a.H * a.N;
    const long long wstride = (long long)gridDim.x * (blockDim.x >> 5);
    for (long long r = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < nrows; r += wstride) {
        const int h = (int)(r / a.N), i = (int)(r % a.N);
        const __nv_bfloat16 *brow = a.has_bias ? a.bias + h * a.sb0 + (long long)i * a.sb1 : nullptr;
        auto logit = [&](int j) -> float {
            if (a.mask && !a.mask[j]) return -INFINITY;
            return brow ? __bfloat162float(brow[j]) : 0.f;
        };
        float m = -INFINITY;
        for (int j = lane; j < a.N; j += 32) m = fmaxf(m, logit(j));
#pragma unroll
        for (int x = 16; x > 0; x >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, x));
        float l = 0.f;
        if (m != -INFINITY)
            for (int j = lane; j < a.N; j += 32) l += __expf(logit(j) - m);
#pragma unroll
        for (int x = 16; x > 0; x >>= 1) l += __shfl_xor_sync(0xffffffffu, l, x);
        const float inv = l > 0.f ? 1.f / l : 0.f;
        __nv_bfloat16 *wrow = a.w + r * a.Wld;
        for (int j = lane; j < a.Wld; j += 32)
            wrow[j] = __float2bfloat16_rn(j < a.N && l > 0.f ? __expf(logit(j) - m) * inv : 0.f);
        if (lane == 0) a.lse[r] = l > 0.f ? m + logf(l) : -INFINITY;
    }
}

// ---------------------------------------------------------------------------------------
// the two contractions with w
// ---------------------------------------------------------------------------------------
template <int CP>
struct PwaTraits {
    static constexpr int BC = 256 / CP;                        // rows b per CTA (TMEM slots)
    static constexpr int KH = 64;                              // reduction rows per stage
    static constexpr int XT_BYTES = KH * CP * 2;               // one row b's V / dOa tile
    static constexpr int W_BYTES = 128 * 64 * 2;               // the stage's 128 x 64 block of w
    static constexpr int STAGE_BYTES = W_BYTES + BC * XT_BYTES;   // 48 KB at every CP
    static constexpr int NS = 2;                               // stages
    static constexpr int OFF_ST = 0;                           // 1024-byte aligned (SW128)
    static constexpr int NBAR = 2 * NS + 2;
    static constexpr int OFF_BAR = OFF_ST + NS * STAGE_BYTES;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int SMEM_BYTES = OFF_MISC + 16;
    static constexpr uint32_t SWZ = CP == 64 ? kSw128 : (CP == 32 ? kSw64 : kSw32);
    static constexpr uint32_t ROWB = CP * 2;
};
static_assert(2 * (PwaTraits<16>::SMEM_BYTES + 1024) <= 233472, "smem");
static_assert(2 * (PwaTraits<32>::SMEM_BYTES + 1024) <= 233472, "smem");
static_assert(2 * (PwaTraits<64>::SMEM_BYTES + 1024) <= 233472, "smem");

// Warp roles (192 threads): warps 0-3 epilogue (thread = output row = TMEM lane), warp 4
// TMA producer, warp 5 TMEM allocator and (lane 0) MMA issuer.
//
// One MMA covers every row b of the chunk: the chunk's BC tiles of V (or dOa) sit side by
// side in a stage and form one B operand of N = BC * CP = 256 columns (MN-major, one
// swizzle atom per row b, LBO = one tile), so each 64-row reduction stage takes four
// M = 128, N = 256, K = 16 instructions instead of four per row b; the accumulator of row
// b is TMEM columns [b CP, (b + 1) CP).
template <int CP, bool DV>
__global__ void __launch_bounds__(192, 2)
pba_pwa_gemm_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                    const PwaArgs a) {
    using T = PwaTraits<CP>;
    constexpr int NS = T::NS, BC = T::BC;
    extern __shared__ __align__(1024) uint8_t dsmem[];
    const uint32_t sbase = smem_u32(dsmem);
    if (sbase & 1023u) {
        if (threadIdx.x == 0) watchdog_fire(SITE_PWA_ALIGN);
        return;
    }
    uint64_t *bars = reinterpret_cast<uint64_t *>(dsmem + T::OFF_BAR);
    auto b_full = [&](int st) { return smem_u32(&bars[st]); };
    auto b_empty = [&](int st) { return smem_u32(&bars[NS + st]); };
    const uint32_t b_done = smem_u32(&bars[2 * NS]);
    const uint32_t b_drain = smem_u32(&bars[2 * NS + 1]);
    uint32_t *s_tmem_base = reinterpret_cast<uint32_t *>(dsmem + T::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(dsmem + T::OFF_MISC + 4);

    const int warp = warp_id(), lane = lane_id();
    int idx = blockIdx.x;
    const int tile = idx % a.nT;
    idx /= a.nT;
    const int chunk = idx % a.nChunks;
    const int h = idx / a.nChunks;
    const int t0 = tile * 128, b0 = chunk * BC;
    const int nb = min(BC, a.B - b0);
    const int nK = (a.N + T::KH - 1) / T::KH;   // reduction stages (the problem is square)

    if (threadIdx.x == 0) {
        for (int st = 0; st < NS; ++st) {
            mbar_init(b_full(st), 1);
            mbar_init(b_empty(st), 1);
        }
        mbar_init(b_done, 1);
        mbar_init(b_drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 5) {
        tmem_alloc(smem_u32(s_tmem_base), 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *s_tmem_base;
    int k_done = 0;   // stages loaded: [0, k_done)

    if (warp == 4) {
        // ------------------------------------------------------------------ producer
        if (lane == 0) {
            tma_prefetch_desc(&tmW);
            tma_prefetch_desc(&tmX);
            bool ok = true;
            for (int r = 0; r < nK && ok; ++r) {
                const int st = r % NS;
                if (r >= NS) ok = mbar_wait(b_empty(st), ((r / NS) - 1) & 1, abort_flag, SITE_PWA_PROD | (r << 12));
                if (!ok) break;
                const uint32_t sw = sbase + T::OFF_ST + st * T::STAGE_BYTES;
                mbar_arrive_tx(b_full(st), T::W_BYTES + nb * T::XT_BYTES);
                if (DV) {
                    // w rows i = reduction rows [64 r, 64 r + 64), columns j = output rows
                    tma_load_3d(sw, &tmW, b_full(st), t0, r * 64, h);
                    tma_load_3d(sw + 8192, &tmW, b_full(st), t0 + 64, r * 64, h);
                } else {
                    // w rows i = output rows, columns j = reduction rows [64 r, 64 r + 64)
                    tma_load_3d(sw, &tmW, b_full(st), r * 64, t0, h);
                }
                for (int s = 0; s < nb; ++s)
                    tma_load_4d(sw + T::W_BYTES + s * T::XT_BYTES, &tmX, b_full(st), 0, h, r * 64, b0 + s);
                k_done = r + 1;
            }
        }
    } else if (warp == 5) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            // forward: A = w (rows i, K = j) K-major; dv: A = w^T (rows j, K = i) MN-major;
            // B = the chunk's V / dOa tiles (K = reduction rows, N = rows b x channels)
            constexpr uint32_t idesc = idesc_bf16(128, 256, DV, true);
            constexpr uint32_t SBO = 8 * T::ROWB;
            bool ok = true;
            for (int r = 0; r < nK && ok; ++r) {
                const int st = r % NS;
                ok = mbar_wait(b_full(st), (r / NS) & 1, abort_flag, SITE_PWA_MMA | (r << 12));
                if (!ok) break;
                tc_fence_after();
                const uint32_t sw = sbase + T::OFF_ST + st * T::STAGE_BYTES;
                const uint32_t sx = sw + T::W_BYTES;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t adesc = DV ? sdesc(sw + kk * 2048, 8192, 1024, kSw128)
                                              : sdesc(sw + kk * 32, 16, 1024, kSw128);
                    umma_ss(tbase, adesc, sdesc(sx + kk * 16 * T::ROWB, T::XT_BYTES, SBO, T::SWZ), idesc,
                            (r > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(b_empty(st));
            }
            if (ok) umma_commit(b_done);
        }
    } else {
        // ------------------------------------------------------------------ epilogue
        const int row = warp * 32 + lane;
        const uint32_t lane_off = ((uint32_t)(warp * 32)) << 16;
        const int n = t0 + row;   // output row: i (forward) or j (dv)
        const bool row_ok = n < a.N;
        // The forward's gate rows do not depend on the products: the first GA slots are
        // fetched before the MMAs are waited for, and every later one GA slots ahead of
        // its use, so the loads' latency overlaps the MMAs and the stores.
        constexpr int GA = CP == 64 ? 1 : BC / 2;
        uint4 gq[GA][CP / 8];
        auto fetch_gate = [&](int s, uint4 (&g)[CP / 8]) {
#pragma unroll
            for (int c8 = 0; c8 < CP / 8; ++c8) {
                g[c8] = make_uint4(0, 0, 0, 0);
                if (!DV && a.has_gate && row_ok && s < nb && c8 * 8 < a.C)
                    g[c8] = *reinterpret_cast<const uint4 *>(a.gate + (b0 + s) * a.sg0 + (long long)n * a.sg1 +
                                                             h * a.sg2 + c8 * 8);
            }
        };
#pragma unroll
        for (int s = 0; s < GA; ++s) fetch_gate(s, gq[s]);
        bool ok = mbar_wait(b_done, 0, abort_flag, SITE_PWA_EPI);
        ok = __all_sync(0xffffffffu, ok);
        if (ok) {
            tc_fence_after();
#pragma unroll
            for (int s = 0; s < BC; ++s) {
                if (s >= nb) break;   // uniform: the TMEM loads below are warp-collective
                uint32_t o[CP];
                tmem_ld_cols<CP>(tbase + s * CP + lane_off, o);
                uint4 g[CP / 8];
#pragma unroll
                for (int c8 = 0; c8 < CP / 8; ++c8) g[c8] = gq[s % GA][c8];
                if (s + GA < BC) fetch_gate(s + GA, gq[s % GA]);
                if (!row_ok) continue;
                const int b = b0 + s;
                __nv_bfloat16 *op = a.out + b * a.so0 + (long long)n * a.so1 + h * a.so2;
                const bool gated = !DV && a.has_gate;
#pragma unroll
                for (int c8 = 0; c8 < CP / 8; ++c8) {
                    if (c8 * 8 < a.C) {
                        const uint32_t gw[4] = {g[c8].x, g[c8].y, g[c8].z, g[c8].w};
                        uint32_t ow[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            float lo = __uint_as_float(o[c8 * 8 + 2 * e]);
                            float hi = __uint_as_float(o[c8 * 8 + 2 * e + 1]);
                            if (gated) {
                                lo *= sigmoid_fast(bf16lo(gw[e]));
                                hi *= sigmoid_fast(bf16hi(gw[e]));
                            }
                            ow[e] = pack_bf16x2(lo, hi);
                        }
                        *reinterpret_cast<uint4 *>(op + c8 * 8) = make_uint4(ow[0], ow[1], ow[2], ow[3]);
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (*abort_flag) {
        if (warp == 4 && lane == 0) {
            for (int rr = max(0, k_done - NS); rr < k_done; ++rr) mbar_wait_drain(b_full(rr % NS), (rr / NS) & 1);
        }
        if (warp == 5 && lane == 0) {
            umma_commit(b_drain);
            mbar_wait_drain(b_drain, 0);
        }
        tc_fence_before();
        __syncthreads();
    }
    if (warp == 5) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tbase, 256);
    }
}

// ---------------------------------------------------------------------------------------
// pre: dOa = dout sigmoid(g), dg = dout out (1 - sigmoid(g)); eight channels per thread
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) pba_pwa_pre_kernel(const PwaArgs a) {
    const int c8n = a.C / 8;
    const long long n = (long long)a.B * a.N * a.H * c8n;
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n;
         e += (long long)gridDim.x * blockDim.x) {
        const int r = (int)(e / c8n), c0 = (int)(e - (long long)r * c8n) * 8;   // r = (b, i, h)
        const int h = r % a.H, bi = r / a.H, i = bi % a.N, b = bi / a.N;
        const uint4 d4 = *reinterpret_cast<const uint4 *>(a.dout + b * a.si0 + (long long)i * a.si1 + h * a.si2 + c0);
        const uint4 o4 = *reinterpret_cast<const uint4 *>(a.oin + b * a.si0 + (long long)i * a.si1 + h * a.si2 + c0);
        const uint4 g4 = *reinterpret_cast<const uint4 *>(a.gate + b * a.sg0 + (long long)i * a.sg1 + h * a.sg2 + c0);
        const uint32_t dw[4] = {d4.x, d4.y, d4.z, d4.w}, ow[4] = {o4.x, o4.y, o4.z, o4.w};
        const uint32_t gw[4] = {g4.x, g4.y, g4.z, g4.w};
        uint32_t da[4], dg[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float s0 = 1.f / (1.f + __expf(-bf16lo(gw[q]))), s1 = 1.f / (1.f + __expf(-bf16hi(gw[q])));
            da[q] = pack_bf16x2(bf16lo(dw[q]) * s0, bf16hi(dw[q]) * s1);
            dg[q] = pack_bf16x2(bf16lo(dw[q]) * bf16lo(ow[q]) * (1.f - s0), bf16hi(dw[q]) * bf16hi(ow[q]) * (1.f - s1));
        }
        *reinterpret_cast<uint4 *>(a.doa + (long long)r * a.C + c0) = make_uint4(da[0], da[1], da[2], da[3]);
        *reinterpret_cast<uint4 *>(a.dgate + b * a.sg0 + (long long)i * a.sg1 + h * a.sg2 + c0) =
            make_uint4(dg[0], dg[1], dg[2], dg[3]);
    }
}

// ---------------------------------------------------------------------------------------
// dW partials: CTA = (h, query tile, key tile, split of b)
// ---------------------------------------------------------------------------------------
template <int CP>
struct PwaDwTraits {
    static constexpr int S = 4;                                // (dOa, V) stages
    static constexpr int TILE_BYTES = 128 * CP * 2;
    static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
    static constexpr int OFF_ST = 0;
    static constexpr int NBAR = 2 * S + 2;
    static constexpr int OFF_BAR = OFF_ST + S * STAGE_BYTES;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int SMEM_BYTES = OFF_MISC + 16;
    static constexpr uint32_t SWZ = CP == 64 ? kSw128 : (CP == 32 ? kSw64 : kSw32);
    static constexpr uint32_t ROWB = CP * 2;
};

template <int CP>
__global__ void __launch_bounds__(192, 2)
pba_pwa_dw_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmV,
                  const PwaArgs a) {
    using T = PwaDwTraits<CP>;
    constexpr int S = T::S;
    extern __shared__ __align__(1024) uint8_t dsmem[];
    const uint32_t sbase = smem_u32(dsmem);
    if (sbase & 1023u) {
        if (threadIdx.x == 0) watchdog_fire(SITE_PWA_ALIGN);
        return;
    }
    uint64_t *bars = reinterpret_cast<uint64_t *>(dsmem + T::OFF_BAR);
    auto b_full = [&](int st) { return smem_u32(&bars[st]); };
    auto b_empty = [&](int st) { return smem_u32(&bars[S + st]); };
    const uint32_t b_done = smem_u32(&bars[2 * S]);
    const uint32_t b_drain = smem_u32(&bars[2 * S + 1]);
    uint32_t *s_tmem_base = reinterpret_cast<uint32_t *>(dsmem + T::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(dsmem + T::OFF_MISC + 4);

    const int warp = warp_id(), lane = lane_id();
    int idx = blockIdx.x;
    const int jt = idx % a.nT;
    idx /= a.nT;
    const int it = idx % a.nT;
    idx /= a.nT;
    const int h = idx % a.H;
    const int sp = idx / a.H;
    const int i0 = it * 128, j0 = jt * 128;
    const int bstart = sp * a.rows_per_split;
    const int nb = max(0, min(a.rows_per_split, a.B - bstart));

    if (threadIdx.x == 0) {
        for (int st = 0; st < S; ++st) {
            mbar_init(b_full(st), 1);
            mbar_init(b_empty(st), 1);
        }
        mbar_init(b_done, 1);
        mbar_init(b_drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 5) {
        tmem_alloc(smem_u32(s_tmem_base), 128);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *s_tmem_base;
    int n_done = 0;

    if (warp == 4) {
        if (lane == 0) {
            tma_prefetch_desc(&tmA);
            tma_prefetch_desc(&tmV);
            bool ok = true;
            for (int n = 0; n < nb && ok; ++n) {
                const int st = n % S, b = bstart + n;
                if (n >= S) ok = mbar_wait(b_empty(st), ((n / S) - 1) & 1, abort_flag, SITE_PWA_PROD | (n << 12));
                if (!ok) break;
                const uint32_t s0 = sbase + T::OFF_ST + st * T::STAGE_BYTES;
                mbar_arrive_tx(b_full(st), 2 * T::TILE_BYTES);
                tma_load_4d(s0, &tmA, b_full(st), 0, h, i0, b);
                tma_load_4d(s0 + T::TILE_BYTES, &tmV, b_full(st), 0, h, j0, b);
                n_done = n + 1;
            }
        }
    } else if (warp == 5) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16(128, 128, false, false);   // dW += dOa V^T
            constexpr uint32_t SBO = 8 * T::ROWB;
            bool ok = true;
            for (int n = 0; n < nb && ok; ++n) {
                const int st = n % S;
                ok = mbar_wait(b_full(st), (n / S) & 1, abort_flag, SITE_PWA_MMA | (n << 12));
                if (!ok) break;
                tc_fence_after();
                const uint32_t s0 = sbase + T::OFF_ST + st * T::STAGE_BYTES;
#pragma unroll
                for (int kk = 0; kk < CP / 16; ++kk)
                    umma_ss(tbase, sdesc(s0 + kk * 32, 16, SBO, T::SWZ),
                            sdesc(s0 + T::TILE_BYTES + kk * 32, 16, SBO, T::SWZ), idesc,
                            (n > 0 || kk > 0) ? 1u : 0u);
                umma_commit(b_empty(st));
            }
            if (ok) umma_commit(b_done);
        }
    } else {
        // this split's partial tile, padded layout [split][h][NPad][NPad]; a split without
        // rows (nb = 0) writes zeros
        const int row = warp * 32 + lane;
        const uint32_t lane_off = ((uint32_t)(warp * 32)) << 16;
        float *dst = a.dw_part + ((((long long)sp * a.H + h) * a.NPad + i0 + row) * a.NPad + j0);
        bool ok = true;
        if (nb > 0) {
            ok = mbar_wait(b_done, 0, abort_flag, SITE_PWA_EPI);
            ok = __all_sync(0xffffffffu, ok);
            if (ok) tc_fence_after();
        }
        if (ok) {
#pragma unroll 1
            for (int q = 0; q < 4; ++q) {
                uint32_t r[32];
                if (nb > 0) {
                    tmem_ld32(tbase + q * 32 + lane_off, r);
                } else {
#pragma unroll
                    for (int c = 0; c < 32; ++c) r[c] = 0u;
                }
#pragma unroll
                for (int c = 0; c < 32; c += 4)
                    *reinterpret_cast<float4 *>(dst + q * 32 + c) =
                        make_float4(__uint_as_float(r[c]), __uint_as_float(r[c + 1]), __uint_as_float(r[c + 2]),
                                    __uint_as_float(r[c + 3]));
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (*abort_flag) {
        if (warp == 4 && lane == 0)
            for (int nn = max(0, n_done - S); nn < n_done; ++nn) mbar_wait_drain(b_full(nn % S), (nn / S) & 1);
        if (warp == 5 && lane == 0) {
            umma_commit(b_drain);
            mbar_wait_drain(b_drain, 0);
        }
        tc_fence_before();
        __syncthreads();
    }
    if (warp == 5) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tbase, 128);
    }
}

// ---------------------------------------------------------------------------------------
// dbias = w (dW - sum_j w dW): one warp per (h, i); fixed summation orders (bit-stable)
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) pba_pwa_dbias_kernel(const PwaArgs a) {
    const int lane = threadIdx.x & 31;
    const long long nrows = (long long)a.H * a.N;
    const long long plane = (long long)a.H * a.NPad * a.NPad;
    const long long wstride = (long long)gridDim.x * (blockDim.x >> 5);
    constexpr int U = 8;   // keys per lane per round: their loads are all issued before any is used
    for (long long r = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < nrows; r += wstride) {
        const int h = (int)(r / a.N), i = (int)(r % a.N);
        const float lse = a.lse[r];
        const __nv_bfloat16 *brow = a.has_bias ? a.bias + h * a.sb0 + (long long)i * a.sb1 : nullptr;
        const float *prow = a.dw_part + ((long long)h * a.NPad + i) * a.NPad;
        // keys j0 + 32 u + lane, u < U: w in fp32 (recomputed from bias and lse_w) and dW (the
        // split partials summed in split order)
        auto round = [&](int j0, float (&wv)[U], float (&dv)[U]) {
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int j = j0 + 32 * u + lane;
                const bool in = j < a.N;
                const float b = (in && brow) ? __bfloat162float(brow[j]) : 0.f;
                const bool keep = in && lse != -INFINITY && !(a.mask && !a.mask[j]);
                wv[u] = keep ? __expf(b - lse) : 0.f;
                dv[u] = 0.f;
            }
            for (int q = 0; q < a.splits; ++q) {
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int j = j0 + 32 * u + lane;
                    if (j < a.N) dv[u] += prow[q * plane + j];
                }
            }
        };
        // r = sum_j w dW: each lane over its keys in increasing order, then a fixed butterfly
        float rs = 0.f;
        for (int j0 = 0; j0 < a.N; j0 += 32 * U) {
            float wv[U], dv[U];
            round(j0, wv, dv);
#pragma unroll
            for (int u = 0; u < U; ++u)
                if (j0 + 32 * u + lane < a.N) rs += wv[u] * dv[u];
        }
#pragma unroll
        for (int x = 16; x > 0; x >>= 1) rs += __shfl_xor_sync(0xffffffffu, rs, x);
        float *drow = a.dbias + r * a.N;
        for (int j0 = 0; j0 < a.N; j0 += 32 * U) {
            float wv[U], dv[U];
            round(j0, wv, dv);
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int j = j0 + 32 * u + lane;
                if (j < a.N) drow[j] = wv[u] * (dv[u] - rs);
            }
        }
    }
}

}  // namespace pba
