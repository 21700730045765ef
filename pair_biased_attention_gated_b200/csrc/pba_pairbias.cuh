// Pair-bias projection: the prologue that makes every pair-biased attention's bias from the
// pair representation z ("AlphaFold3 open-source implementation" page, Model Efficiency
// section: each attention projects its pair bias from the pair representation; the
// Protenix page, scalability section: LayerNorm over the pair representation is the op
// worth a custom kernel).  Read as a LayerNorm over the channels of z[i,j,:] followed by a
// linear map without bias:
//
//   xh = (z - mean) / sqrt(var + eps),  y = gamma xh + beta,  bias[h,i,j] = sum_c y_c w[c,h]
//
// and its backward for a given dbias:
//   dz_c = rstd (dxh_c - mean_c dxh - xh_c mean_c(dxh xh)),  dxh_c = gamma_c sum_h w[c,h] g_h
//   dw[c,h] = sum_pos y_c g_h,  dgamma_c = sum_pos dy_c xh_c,  dbeta_c = sum_pos dy_c
//
// The kernels rewrite the sums so that one pass over a row suffices.  With w' = gamma w
// (columns padded with zeros to HP), S_h = sum_c w'[c,h] and acc_h = sum_c w'[c,h](z_c - mean):
//   bias_h = rstd acc_h + sum_c beta_c w[c,h]
//   mean_c dxh = sum_h g_h S_h / Cz,  mean_c(dxh xh) = rstd sum_h g_h acc_h / Cz
// and the parameter gradients need only A[c,h] = sum_pos xh_c g_h and G_h = sum_pos g_h:
//   dw[c,h] = gamma_c A[c,h] + beta_c G_h,  dgamma_c = sum_h w[c,h] A[c,h],
//   dbeta_c = sum_h w[c,h] G_h.
//
// Work unit: a tile of 128 consecutive positions j of one row i.  Every block (thread =
// position where a thread owns a row) is persistent over tiles blockIdx.x, blockIdx.x +
// gridDim.x, ...; tiles arrive by TMA (the Cz channels as 64-channel boxes with the 128-byte
// swizzle, so that each thread reads its own row without bank conflicts, and the layout the
// tensor core reads) into two buffers, the next but one tile loading while the current one is
// processed.  HBM-bound: z is read once and the bias (or dz) written once.  The forward, and
// the backward at Cz = 128, run their contractions on the tensor core (tcgen05, TMEM
// accumulators); the backward at the other widths on the CUDA cores.  The backward's
// parameter sums are added per block in tile order, then over the blocks in block order by
// two small kernels (bit-stable).
#pragma once

#include "pba_device.cuh"

namespace pba {

struct PbArgs {
    int Ni, Nj, Cz, H;
    int nJt, tiles;                 // tiles of 128 positions along j per row, all tiles
    float eps;
    const float *gamma, *beta, *w;  // [Cz], [Cz], [Cz][H]
    __nv_bfloat16 *bias;            // forward output [H][Ni][Nj], strides (sb0, sb1), j stride 1
    long long sb0, sb1;
    const float *dbias;             // backward input, strides (sd0, sd1), j stride 1
    long long sd0, sd1;
    __nv_bfloat16 *dz;              // backward output, the layout of z: strides (sz0, sz1)
    long long sz0, sz1;
    float *part;                    // [gridDim.x][Cz * HP + HP] per-block sums A, G
    float *sums;                    // [Cz * HP + HP] their sums over the blocks
    float *dw, *dgamma, *dbeta;
    int nparts, hp;
};

enum : unsigned { SITE_PB_FWD = 0x501, SITE_PB_BWD = 0x502, SITE_PB_ALIGN = 0x5FF };

template <int CZ, int HP>
struct PbTraits {
    static constexpr int TILE_BYTES = 128 * CZ * 2;            // CZ / 64 boxes of 16 KB
    static constexpr int OFF_Z = 0;                            // 1024-byte aligned (SW128)
    static constexpr int OFF_W = OFF_Z + 2 * TILE_BYTES;       // w' fp32, channel pairs interleaved
    static constexpr int OFF_S = OFF_W + CZ * HP * 4;          // S [HP]
    static constexpr int OFF_BB = OFF_S + HP * 4;              // sum_c beta_c w[c,h] [HP]
    static constexpr int OFF_MU = OFF_BB + HP * 4;             // bwd: mean per position [128]
    static constexpr int OFF_G1 = OFF_MU + 128 * 4;            // bwd: rstd g [128][HP]
    static constexpr int OFF_G0 = OFF_G1 + 128 * HP * 4;       // bwd: g [128][HP]
    static constexpr int OFF_BAR = OFF_G0 + 128 * HP * 4;      // full[2]
    static constexpr int OFF_MISC = OFF_BAR + 16;              // abort flag
    static constexpr int SMEM_BYTES = OFF_MISC + 16;
};

// 16-byte chunk q (channels 8q .. 8q+7) of row r in a swizzled tile buffer
__device__ __forceinline__ uint32_t pb_chunk(uint32_t buf, int r, int q) {
    return buf + (uint32_t)((q >> 3) * 16384 + r * 128 + (((q & 7) ^ (r & 7)) << 4));
}

// w'[c,h] sits at ((c / 2) HP + h) 2 + c % 2: one 16-byte load gives columns h, h + 1 of
// the channel pair (c, c + 1) as two float2, the operands of the packed fp32 FMA.
__device__ __forceinline__ int pb_widx(int c, int h, int HP) { return ((c >> 1) * HP + h) * 2 + (c & 1); }

// Block setup: w' = gamma w (zero-padded to HP columns), its column sums S and the beta
// projection; initialises the two tile barriers.
template <int CZ, int HP, typename T = PbTraits<CZ, HP>>
__device__ __forceinline__ void pb_setup(const PbArgs &a, uint8_t *dsmem, bool with_bb) {
    float *sW = reinterpret_cast<float *>(dsmem + T::OFF_W);
    float *sS = reinterpret_cast<float *>(dsmem + T::OFF_S);
    float *sB = reinterpret_cast<float *>(dsmem + T::OFF_BB);
    const int tid = threadIdx.x;
    if (tid == 0) {
        uint64_t *bars = reinterpret_cast<uint64_t *>(dsmem + T::OFF_BAR);
        mbar_init(smem_u32(&bars[0]), 1);
        mbar_init(smem_u32(&bars[1]), 1);
        *reinterpret_cast<volatile int *>(dsmem + T::OFF_MISC) = 0;
        fence_mbar_init();
    }
    for (int e = tid; e < CZ * HP; e += blockDim.x) {
        const int c = e / HP, h = e % HP;
        sW[pb_widx(c, h, HP)] = h < a.H ? a.gamma[c] * a.w[c * a.H + h] : 0.f;
    }
    __syncthreads();
    // column sums: warp w takes columns h = w, w + 4, ...; lanes stride over the channels,
    // then a fixed butterfly
    const int warp = tid >> 5, lane = tid & 31;
    for (int h = warp; h < HP; h += 4) {
        float s = 0.f, bb = 0.f;
        for (int c = lane; c < CZ; c += 32) {
            s += sW[pb_widx(c, h, HP)];
            if (with_bb && h < a.H) bb = fmaf(a.beta[c], a.w[c * a.H + h], bb);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            s += __shfl_xor_sync(0xffffffffu, s, o);
            bb += __shfl_xor_sync(0xffffffffu, bb, o);
        }
        if (lane == 0) {
            sS[h] = s;
            sB[h] = bb;
        }
    }
    __syncthreads();
}

template <int CZ>
__device__ __forceinline__ void pb_issue(const CUtensorMap *tm, uint32_t dst, uint32_t bar, int tile,
                                         int nJt) {
    const int i = tile / nJt, j0 = (tile % nJt) * 128;
    mbar_arrive_tx(bar, CZ * 128 * 2);
#pragma unroll
    for (int hf = 0; hf < CZ / 64; ++hf) tma_load_3d(dst + hf * 16384, tm, bar, hf * 64, j0, i);
}

// Row r of a tile buffer: its mean (first pass), then in one second pass over the row
// 1 / sqrt(var + eps) and acc_h = sum_c w'[c,h] (x_c - mean).  The row is read from shared
// memory, not held in registers, which keeps Cz = 256 spill-free.
template <int CZ, int HP>
__device__ __forceinline__ void pb_row_stats(const float *sW, uint32_t buf, int r, float eps, float &mu,
                                             float &rstd, float (&acc)[HP]) {
    float s0 = 0.f, s1 = 0.f;
#pragma unroll 4
    for (int q = 0; q < CZ / 8; ++q) {
        const uint4 v = lds128(pb_chunk(buf, r, q));
        const uint32_t x[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            s0 += bf16lo(x[e]);
            s1 += bf16hi(x[e]);
        }
    }
    mu = (s0 + s1) * (1.f / CZ);
    float2 acc2[HP];   // (even channel, odd channel) partial sums of acc_h
#pragma unroll
    for (int h = 0; h < HP; ++h) acc2[h] = make_float2(0.f, 0.f);
    float2 var2 = make_float2(0.f, 0.f);
    const float2 nmu = make_float2(-mu, -mu);
#pragma unroll 1
    for (int q = 0; q < CZ / 8; ++q) {
        const uint4 v = lds128(pb_chunk(buf, r, q));
        const uint32_t x[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float4 *wp = reinterpret_cast<const float4 *>(sW + pb_widx(q * 8 + 2 * e, 0, HP));
            const float2 d = fadd2(make_float2(bf16lo(x[e]), bf16hi(x[e])), nmu);
            var2 = ffma2(d, d, var2);
#pragma unroll
            for (int h2 = 0; h2 < HP / 2; ++h2) {
                const float4 w4 = wp[h2];   // columns 2 h2, 2 h2 + 1 of channels (c, c + 1)
                acc2[2 * h2] = ffma2(make_float2(w4.x, w4.y), d, acc2[2 * h2]);
                acc2[2 * h2 + 1] = ffma2(make_float2(w4.z, w4.w), d, acc2[2 * h2 + 1]);
            }
        }
    }
#pragma unroll
    for (int h = 0; h < HP; ++h) acc[h] = acc2[h].x + acc2[h].y;
    rstd = rsqrtf((var2.x + var2.y) * (1.f / CZ) + eps);
}

// Forward on the tensor core: per tile, acc[p,h] = sum_c z[p,c] w'[c,h] is one M = 128, N = 32
// product per 16 channels, accumulated in TMEM: w' = gamma w as two bf16 terms for fp32
// accuracy, hi in columns 0-15 and lo in columns 16-31 (heads padded with zeros to 16), added
// in the epilogue, so the two terms cost no extra MMA instructions; the threads only make each row's
// mean and 1 / sqrt(var + eps) and the epilogue bias_h = rstd (acc_h - mean S_h) + sum_c beta_c w[c,h].
// Warp roles (160 threads): warps 0-3 thread = position (TMEM lane); warp 4 allocates TMEM and,
// on lane 0, loads the tiles and issues the products.
template <int CZ>
struct PbFwdTraits {
    static constexpr int TILE_BYTES = 128 * CZ * 2;            // CZ / 64 boxes of 16 KB
    // tile buffers (a ring): more than two measured no faster, the kernel being issue-bound
    static constexpr int NBUF = 2;
    static constexpr int WT_BYTES = 32 * CZ * 2;               // w'^T: rows 0-15 hi, 16-31 lo, x CZ
    static constexpr int OFF_Z = 0;                            // 1024-byte aligned (SW128)
    static constexpr int OFF_WT = OFF_Z + NBUF * TILE_BYTES;   // 1024-byte aligned (SW128)
    static constexpr int OFF_S = OFF_WT + WT_BYTES;            // S_h [16]
    static constexpr int OFF_BB = OFF_S + 64;                  // sum_c beta_c w[c,h] [16]
    static constexpr int OFF_BAR = OFF_BB + 64;   // full[NBUF] z_free[NBUF] mma_done[2] acc_free[2] drain
    static constexpr int OFF_MISC = OFF_BAR + 8 * (2 * NBUF + 5);   // abort flag, TMEM base
    static constexpr int SMEM_BYTES = OFF_MISC + 16;
    static constexpr int THREADS = 160;
    static_assert(WT_BYTES % 1024 == 0, "w' terms stay 1024-byte aligned");
    static_assert(SMEM_BYTES + 1024 <= 233472, "one CTA per SM at least");
};

// byte offset of w'^T element (row n, channel c) in a 32 x CZ K-major tile: 64-channel blocks
// of 32 rows x 128 bytes, 16-byte chunks swizzled by the row (the 128-byte swizzle)
__device__ __forceinline__ uint32_t pb_wt_off(int n, int c) {
    return (uint32_t)((c >> 6) * 4096 + n * 128 + ((((c & 63) >> 3) ^ (n & 7)) << 4) + (c & 7) * 2);
}

template <int CZ, int HP>
__global__ void __launch_bounds__(160) pba_pair_bias_fwd_kernel(const __grid_constant__ CUtensorMap tmZ,
                                                                 const PbArgs a) {
    using T = PbFwdTraits<CZ>;
    static_assert(HP <= 16, "heads");
    extern __shared__ __align__(1024) uint8_t dsmem[];
    const uint32_t sbase = smem_u32(dsmem);
    if (sbase & 1023u) {
        if (threadIdx.x == 0) watchdog_fire(SITE_PB_ALIGN);
        return;
    }
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    float *sS = reinterpret_cast<float *>(dsmem + T::OFF_S);
    float *sB = reinterpret_cast<float *>(dsmem + T::OFF_BB);
    uint64_t *bars = reinterpret_cast<uint64_t *>(dsmem + T::OFF_BAR);
    constexpr int NB = T::NBUF;
    auto b_full = [&](int y) { return smem_u32(&bars[y]); };             // tile buffer y landed
    auto b_zfree = [&](int y) { return smem_u32(&bars[NB + y]); };       // its rows read by the threads
    auto b_mma = [&](int x) { return smem_u32(&bars[2 * NB + x]); };     // products into accumulator x done
    auto b_afree = [&](int x) { return smem_u32(&bars[2 * NB + 2 + x]); };   // accumulator x read out
    const uint32_t b_drain = smem_u32(&bars[2 * NB + 4]);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(dsmem + T::OFF_MISC);
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(dsmem + T::OFF_MISC + 4);
    const int n_items = (int)blockIdx.x < a.tiles ? (a.tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    auto tile_of = [&](int n) { return (int)blockIdx.x + n * (int)gridDim.x; };

    if (tid == 0) {
        for (int y = 0; y < NB; ++y) {
            mbar_init(b_full(y), 1);
            mbar_init(b_zfree(y), 128);
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(b_mma(x), 1);
            mbar_init(b_afree(x), 128);
        }
        mbar_init(b_drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    // w'^T as hi + lo bf16 terms (zero rows for padded heads), and the per-head constants
    for (int e = tid; e < 16 * CZ; e += blockDim.x) {
        const int n = e / CZ, c = e % CZ;
        const float wv = n < a.H ? a.gamma[c] * a.w[c * a.H + n] : 0.f;
        const __nv_bfloat16 hi = __float2bfloat16_rn(wv);
        const __nv_bfloat16 lo = __float2bfloat16_rn(wv - __bfloat162float(hi));
        *reinterpret_cast<__nv_bfloat16 *>(dsmem + T::OFF_WT + pb_wt_off(n, c)) = hi;
        *reinterpret_cast<__nv_bfloat16 *>(dsmem + T::OFF_WT + pb_wt_off(16 + n, c)) = lo;
    }
    if (warp < 4) {
        // S_h = sum_c gamma_c w[c,h] and sum_c beta_c w[c,h]: warp w takes heads w, w + 4, ...
        for (int h = warp; h < 16; h += 4) {
            float sv = 0.f, bb = 0.f;
            if (h < a.H)
                for (int c = lane; c < CZ; c += 32) {
                    sv = fmaf(a.gamma[c], a.w[c * a.H + h], sv);
                    bb = fmaf(a.beta[c], a.w[c * a.H + h], bb);
                }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                sv += __shfl_xor_sync(0xffffffffu, sv, o);
                bb += __shfl_xor_sync(0xffffffffu, bb, o);
            }
            if (lane == 0) {
                sS[h] = sv;
                sB[h] = bb;
            }
        }
    } else {
        tmem_alloc(smem_u32(s_tmem), 64);
        tmem_relinquish();
    }
    fence_proxy_async();   // the w' terms are read by the tensor core
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *s_tmem;
    int issued = 0;        // warp 4, lane 0: tiles whose loads were issued

    if (warp == 4) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16(128, 32, false, false);
            tma_prefetch_desc(&tmZ);
            for (; issued < NB && issued < n_items; ++issued)
                pb_issue<CZ>(&tmZ, sbase + T::OFF_Z + issued * T::TILE_BYTES, b_full(issued), tile_of(issued), a.nJt);
            bool ok = true;
            for (int n = 0; n < n_items && ok; ++n) {
                const int x = n & 1, y = n % NB;   // accumulator, tile buffer
                ok = mbar_wait_all(abort_flag, b_full(y), (n / NB) & 1, true, SITE_PB_FWD | (n << 12),
                                   b_afree(x), ((n >> 1) - 1) & 1, n >= 2, SITE_PB_FWD | 0x10 | (n << 12));
                if (!ok) break;
                tc_fence_after();
                const uint32_t zb = sbase + T::OFF_Z + y * T::TILE_BYTES;
                const uint64_t dz = sdesc(zb, 16, 1024, kSw128);
                const uint64_t dw = sdesc(sbase + T::OFF_WT, 16, 1024, kSw128);
#pragma unroll
                for (int kk = 0; kk < CZ / 16; ++kk) {
                    const uint32_t za = (kk >> 2) * 16384 + (kk & 3) * 32, wa = (kk >> 2) * 4096 + (kk & 3) * 32;
                    umma_ss(tbase + x * 32, sdesc_add(dz, za), sdesc_add(dw, wa), idesc, kk > 0);
                }
                umma_commit(b_mma(x));
                // the previous tile's buffer, once its rows are read and its products done,
                // takes tile n - 1 + NB
                if (n >= 1 && issued < n_items) {
                    const int m = n - 1, ym = m % NB;
                    ok = mbar_wait_all(abort_flag, b_zfree(ym), (m / NB) & 1, true, SITE_PB_FWD | 0x20 | (n << 12),
                                       b_mma(m & 1), (m >> 1) & 1, true, SITE_PB_FWD | 0x30 | (n << 12));
                    if (!ok) break;
                    pb_issue<CZ>(&tmZ, sbase + T::OFF_Z + ym * T::TILE_BYTES, b_full(ym), tile_of(issued), a.nJt);
                    ++issued;
                }
            }
        }
    } else {
        // thread = position p of the tile = TMEM lane
        const uint32_t lane_off = ((uint32_t)(warp * 32)) << 16;
        bool ok = true;
        for (int n = 0; n < n_items && ok; ++n) {
            const int x = n & 1, y = n % NB;
            const uint32_t zb = sbase + T::OFF_Z + y * T::TILE_BYTES;
            ok = mbar_wait(b_full(y), (n / NB) & 1, abort_flag, SITE_PB_FWD | 0x40 | (n << 12));
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            // the row's mean, then 1 / sqrt(var + eps) in a second pass
            float s0 = 0.f, s1 = 0.f;
#pragma unroll 4
            for (int q = 0; q < CZ / 8; ++q) {
                const uint4 v = lds128(pb_chunk(zb, tid, q));
                const uint32_t xw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    s0 += bf16lo(xw[e]);
                    s1 += bf16hi(xw[e]);
                }
            }
            const float mu = (s0 + s1) * (1.f / CZ);
            float2 var2 = make_float2(0.f, 0.f);
            const float2 nmu = make_float2(-mu, -mu);
#pragma unroll 4
            for (int q = 0; q < CZ / 8; ++q) {
                const uint4 v = lds128(pb_chunk(zb, tid, q));
                const uint32_t xw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 d = fadd2(make_float2(bf16lo(xw[e]), bf16hi(xw[e])), nmu);
                    var2 = ffma2(d, d, var2);
                }
            }
            const float rstd = rsqrtf((var2.x + var2.y) * (1.f / CZ) + a.eps);
            mbar_arrive(b_zfree(y));
            ok = mbar_wait(b_mma(x), (n >> 1) & 1, abort_flag, SITE_PB_FWD | 0x50 | (n << 12));
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            uint32_t acc[32];   // sum_c z w'_hi in columns 0-15, sum_c z w'_lo in 16-31
            tmem_ld32(tbase + x * 32 + lane_off, acc);
            tc_fence_before();
            mbar_arrive(b_afree(x));
            const int t = tile_of(n), i = t / a.nJt, j = (t % a.nJt) * 128 + tid;
            if (j < a.Nj) {
                __nv_bfloat16 *dst = a.bias + (long long)i * a.sb1 + j;
#pragma unroll
                for (int h = 0; h < HP; ++h)
                    if (h < a.H)
                        dst[h * a.sb0] = __float2bfloat16_rn(
                            fmaf(rstd, fmaf(-mu, sS[h], __uint_as_float(acc[h]) + __uint_as_float(acc[16 + h])), sB[h]));
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (*abort_flag && warp == 4 && lane == 0) {
        // loads issued for tiles not yet consumed may still land, products may still run
        for (int m = max(0, issued - NB); m < issued; ++m) mbar_wait_drain(b_full(m % NB), (m / NB) & 1);
        umma_commit(b_drain);
        mbar_wait_drain(b_drain, 0);
    }
    __syncthreads();
    if (warp == 4) {
        tc_fence_after();
        tmem_dealloc(tbase, 64);
    }
}

template <int CZ, int HP>
__global__ void __launch_bounds__(128) pba_pair_bias_bwd_kernel(const __grid_constant__ CUtensorMap tmZ,
                                                                 const PbArgs a) {
    using T = PbTraits<CZ, HP>;
    extern __shared__ __align__(1024) uint8_t dsmem[];
    const uint32_t sbase = smem_u32(dsmem);
    if (sbase & 1023u) {
        if (threadIdx.x == 0) watchdog_fire(SITE_PB_ALIGN);
        return;
    }
    const int tid = threadIdx.x;
    const float *sW = reinterpret_cast<const float *>(dsmem + T::OFF_W);
    const float *sS = reinterpret_cast<const float *>(dsmem + T::OFF_S);
    float *sMu = reinterpret_cast<float *>(dsmem + T::OFF_MU);
    float *sG1 = reinterpret_cast<float *>(dsmem + T::OFF_G1);
    float *sG0 = reinterpret_cast<float *>(dsmem + T::OFF_G0);
    uint64_t *bars = reinterpret_cast<uint64_t *>(dsmem + T::OFF_BAR);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(dsmem + T::OFF_MISC);
    const int n_items = (int)blockIdx.x < a.tiles ? (a.tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    auto tile_of = [&](int n) { return (int)blockIdx.x + n * (int)gridDim.x; };
    constexpr int CPT = (CZ + 127) / 128;   // channels per thread in phase 2

    pb_setup<CZ, HP>(a, dsmem, false);
    float A[CPT][HP];   // this block's sum over positions of xh_c g_h, channels c = tid + 128 k
    float G = 0.f;      // threads h < HP: sum over positions of g_h
#pragma unroll
    for (int k = 0; k < CPT; ++k)
#pragma unroll
        for (int h = 0; h < HP; ++h) A[k][h] = 0.f;
    int issued = 0;
    if (tid == 0) {
        tma_prefetch_desc(&tmZ);
        for (; issued < 2 && issued < n_items; ++issued)
            pb_issue<CZ>(&tmZ, sbase + T::OFF_Z + issued * T::TILE_BYTES, smem_u32(&bars[issued]),
                         tile_of(issued), a.nJt);
    }
    int n = 0;
    for (; n < n_items; ++n) {
        const int buf = n & 1;
        const uint32_t zb = sbase + T::OFF_Z + buf * T::TILE_BYTES;
        bool ok = mbar_wait(smem_u32(&bars[buf]), (n >> 1) & 1, abort_flag, SITE_PB_BWD | (n << 12));
        if (!__syncthreads_and(ok)) break;
        const int t = tile_of(n), i = t / a.nJt, j = (t % a.nJt) * 128 + tid;
        const bool valid = j < a.Nj;
        // ---- phase 1: thread = position j; dz of its row
        {
            float mu, rstd, acc[HP];
            pb_row_stats<CZ, HP>(sW, zb, tid, a.eps, mu, rstd, acc);
            float g[HP];
#pragma unroll
            for (int h = 0; h < HP; ++h)
                g[h] = (valid && h < a.H) ? a.dbias[h * a.sd0 + (long long)i * a.sd1 + j] : 0.f;
            float s1 = 0.f, s2 = 0.f;
#pragma unroll
            for (int h = 0; h < HP; ++h) {
                s1 = fmaf(g[h], sS[h], s1);
                s2 = fmaf(g[h], acc[h], s2);
            }
            const float m1 = s1 * (1.f / CZ);             // mean_c dxh
            const float m2r = s2 * rstd * rstd * (1.f / CZ);   // mean_c(dxh xh) * rstd
            if (valid) {
                __nv_bfloat16 *dst = a.dz + (long long)i * a.sz0 + (long long)j * a.sz1;
#pragma unroll 1
                for (int q = 0; q < CZ / 8; ++q) {
                    const uint4 v = lds128(pb_chunk(zb, tid, q));
                    const uint32_t x[4] = {v.x, v.y, v.z, v.w};
                    uint32_t ow[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float4 *wp = reinterpret_cast<const float4 *>(sW + pb_widx(q * 8 + 2 * e, 0, HP));
                        float2 dx = make_float2(0.f, 0.f);   // dxh of the channel pair
#pragma unroll
                        for (int h2 = 0; h2 < HP / 2; ++h2) {
                            const float4 w4 = wp[h2];
                            dx = ffma2(make_float2(w4.x, w4.y), make_float2(g[2 * h2], g[2 * h2]), dx);
                            dx = ffma2(make_float2(w4.z, w4.w), make_float2(g[2 * h2 + 1], g[2 * h2 + 1]), dx);
                        }
                        const float d0 = bf16lo(x[e]) - mu, d1 = bf16hi(x[e]) - mu;
                        ow[e] = pack_bf16x2(rstd * (dx.x - m1 - d0 * m2r), rstd * (dx.y - m1 - d1 * m2r));
                    }
                    *reinterpret_cast<uint4 *>(dst + q * 8) = make_uint4(ow[0], ow[1], ow[2], ow[3]);
                }
            }
            sMu[tid] = mu;
#pragma unroll
            for (int h = 0; h < HP; ++h) {
                sG1[tid * HP + h] = valid ? rstd * g[h] : 0.f;
                sG0[tid * HP + h] = g[h];
            }
        }
        __syncthreads();
        // ---- phase 2: thread = channel; A[c,h] += (z - mean) rstd g over the tile's positions
#pragma unroll 2
        for (int p = 0; p < 128; ++p) {
            const float mu = sMu[p];
            const float4 *g1 = reinterpret_cast<const float4 *>(sG1 + p * HP);
#pragma unroll
            for (int k = 0; k < CPT; ++k) {
                const int c = tid + 128 * k;
                if (c < CZ) {
                    const uint32_t addr = pb_chunk(zb, p, c >> 3) + (c & 7) * 2;
                    uint16_t raw;
                    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(raw) : "r"(addr));
                    const float d = __uint_as_float((uint32_t)raw << 16) - mu;
#pragma unroll
                    for (int h4 = 0; h4 < HP / 4; ++h4) {
                        const float4 gg = g1[h4];
                        A[k][4 * h4] = fmaf(d, gg.x, A[k][4 * h4]);
                        A[k][4 * h4 + 1] = fmaf(d, gg.y, A[k][4 * h4 + 1]);
                        A[k][4 * h4 + 2] = fmaf(d, gg.z, A[k][4 * h4 + 2]);
                        A[k][4 * h4 + 3] = fmaf(d, gg.w, A[k][4 * h4 + 3]);
                    }
                }
            }
            if (tid < HP) G += sG0[p * HP + tid];
        }
        __syncthreads();   // the tile buffer and the per-position arrays are free again
        if (tid == 0 && issued < n_items) {
            pb_issue<CZ>(&tmZ, zb, smem_u32(&bars[buf]), tile_of(issued), a.nJt);
            ++issued;
        }
    }
    const bool aborted = *abort_flag != 0;
    if (aborted && tid == 0) {
        for (int m = n; m < issued; ++m) mbar_wait_drain(smem_u32(&bars[m & 1]), (m >> 1) & 1);
    }
    if (!aborted) {
        float *dst = a.part + (long long)blockIdx.x * (CZ * HP + HP);
#pragma unroll
        for (int k = 0; k < CPT; ++k) {
            const int c = tid + 128 * k;
            if (c < CZ) {
#pragma unroll
                for (int h = 0; h < HP; ++h) dst[c * HP + h] = A[k][h];
            }
        }
        if (tid < HP) dst[CZ * HP + tid] = G;
    }
    __syncthreads();
}

// Backward for Cz = 128 with its three contractions on the tensor core; the threads keep the
// LayerNorm statistics and the elementwise part of dz.  Per tile of 128 positions:
//   acc[p,h]  = sum_c z[p,c] w'[c,h]         M = 128 positions, N = 32, K = 128 channels (the
//               z tile as the K-major A operand; w' as hi and lo bf16 rows, as in the forward)
//   dxh[p,c]  = sum_h g[p,h] w'[c,h]         M = 128 positions, N = 128 channels, K = 3 x 16:
//               g_hi w_hi + g_hi w_lo + g_lo w_hi (fp32 accuracy), one 64-wide K block
//   A[c,h]   += sum_p z[p,c] G1[p,h]          M = 128 channels, N = 32, K = 16 positions per
//               product: the z tile as the MN-major A operand (rows = positions of 128 bytes of
//               channels, the 128-byte swizzle, 64-channel blocks 16 KB apart), G1 = rstd g as
//               hi and lo rows, accumulated in TMEM over all of the block's tiles
// and A = sum_p (z - mean) G1 = that sum - sum_p mean_p G1[p,:].  The per-block partials have the
// layout of the kernel above, so their reduction stays bit-stable.
template <int HP>
struct PbBwdTcTraits {
    static constexpr int CZ = 128;
    static constexpr int TILE_BYTES = 128 * CZ * 2;
    static constexpr int OFF_Z = 0;                            // 2 tiles, 1024-byte aligned (SW128)
    static constexpr int OFF_GT = OFF_Z + 2 * TILE_BYTES;      // G1^T: 32 rows x 128 positions bf16
    static constexpr int OFF_WF = OFF_GT + 32 * 128 * 2;       // w'^T: 32 rows (hi, lo) x 128 channels
    static constexpr int OFF_G = OFF_WF + 32 * 128 * 2;        // g: 128 positions x 64 (g_hi, g_hi, g_lo, 0)
    static constexpr int OFF_WB = OFF_G + 128 * 128;           // w': 128 channels x 64 (w_hi, w_lo, w_hi, 0)
    static constexpr int OFF_S = OFF_WB + 128 * 128;           // S_h = sum_c w'[c,h] [16]
    static constexpr int OFF_RED = OFF_S + 64;                 // setup: per-warp head sums [4][16]
    static constexpr int OFF_BAR = OFF_RED + 256;              // full[2], acc, dx, all, drain
    static constexpr int OFF_MISC = OFF_BAR + 48;              // abort flag, TMEM base
    static constexpr int SMEM_BYTES = OFF_MISC + 16;
    static constexpr uint32_t T_ACC = 0, T_A = 32, T_DX = 128;   // TMEM columns (256 allocated)
    static_assert(OFF_GT % 1024 == 0 && OFF_WF % 1024 == 0 && OFF_G % 1024 == 0 && OFF_WB % 1024 == 0,
                  "operands 1024-byte aligned");
    static_assert(2 * TILE_BYTES >= 128 * 2 * HP * 4 + 2 * HP * 4, "the tile buffers hold the final sums");
    static_assert(2 * (SMEM_BYTES + 1024) <= 233472, "two blocks per SM");
};

// byte offset of element (row r, k) of a 128-row x 64 K-major tile with the 128-byte swizzle
__device__ __forceinline__ uint32_t pb_k64_off(int r, int k) {
    return (uint32_t)(r * 128 + (((k >> 3) ^ (r & 7)) << 4) + (k & 7) * 2);
}

template <int HP>
__global__ void __launch_bounds__(128) pba_pair_bias_bwd_tc_kernel(const __grid_constant__ CUtensorMap tmZ,
                                                                    const PbArgs a) {
    constexpr int CZ = 128;
    using T = PbBwdTcTraits<HP>;
    extern __shared__ __align__(1024) uint8_t dsmem[];
    const uint32_t sbase = smem_u32(dsmem);
    if (sbase & 1023u) {
        if (threadIdx.x == 0) watchdog_fire(SITE_PB_ALIGN);
        return;
    }
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    float *sS = reinterpret_cast<float *>(dsmem + T::OFF_S);
    uint64_t *bars = reinterpret_cast<uint64_t *>(dsmem + T::OFF_BAR);
    auto b_full = [&](int x) { return smem_u32(&bars[x]); };
    const uint32_t b_acc = smem_u32(&bars[2]), b_dx = smem_u32(&bars[3]), b_all = smem_u32(&bars[4]),
                   b_drain = smem_u32(&bars[5]);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(dsmem + T::OFF_MISC);
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(dsmem + T::OFF_MISC + 4);
    const int n_items = (int)blockIdx.x < a.tiles ? (a.tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    auto tile_of = [&](int n) { return (int)blockIdx.x + n * (int)gridDim.x; };

    int issued = 0;   // thread 0: tiles whose loads were issued
    if (tid == 0) {
        mbar_init(b_full(0), 1);
        mbar_init(b_full(1), 1);
        mbar_init(b_acc, 1);
        mbar_init(b_dx, 1);
        mbar_init(b_all, 1);
        mbar_init(b_drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmZ);
        for (; issued < 2 && issued < n_items; ++issued)
            pb_issue<CZ>(&tmZ, sbase + T::OFF_Z + issued * T::TILE_BYTES, b_full(issued), tile_of(issued), a.nJt);
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(s_tmem), 256);
        tmem_relinquish();
    }
    // operand tiles: w' = gamma w as hi and lo bf16 terms, zeros elsewhere (padded heads, the
    // unused K slice); thread = channel c; all its loads issued before any is used
    {
        const int c = tid;
        const float gc = __ldg(a.gamma + c);
        float wv[16];
#pragma unroll
        for (int h = 0; h < 16; ++h) wv[h] = h < a.H ? __ldg(a.w + c * a.H + h) : 0.f;
        float *red = reinterpret_cast<float *>(dsmem + T::OFF_RED);
#pragma unroll
        for (int h = 0; h < 16; ++h) {
            const float v = gc * wv[h];
            const __nv_bfloat16 hi = __float2bfloat16_rn(v);
            const __nv_bfloat16 lo = __float2bfloat16_rn(v - __bfloat162float(hi));
            *reinterpret_cast<__nv_bfloat16 *>(dsmem + T::OFF_WF + pb_wt_off(h, c)) = hi;
            *reinterpret_cast<__nv_bfloat16 *>(dsmem + T::OFF_WF + pb_wt_off(16 + h, c)) = lo;
            *reinterpret_cast<__nv_bfloat16 *>(dsmem + T::OFF_WB + pb_k64_off(c, h)) = hi;
            *reinterpret_cast<__nv_bfloat16 *>(dsmem + T::OFF_WB + pb_k64_off(c, 16 + h)) = lo;
            *reinterpret_cast<__nv_bfloat16 *>(dsmem + T::OFF_WB + pb_k64_off(c, 32 + h)) = hi;
            *reinterpret_cast<__nv_bfloat16 *>(dsmem + T::OFF_WB + pb_k64_off(c, 48 + h)) = __float2bfloat16_rn(0.f);
            // S_h = sum_c w'[c,h]: each warp's butterfly, then the warps in order
            float sv = v;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) sv += __shfl_xor_sync(0xffffffffu, sv, o);
            if (lane == 0) red[warp * 16 + h] = sv;
        }
        // G1^T and g start zero (padded heads, the unused K slice)
        for (int e = tid; e < 32 * 128 * 2 / 16; e += 128) sts128(sbase + T::OFF_GT + e * 16, make_uint4(0, 0, 0, 0));
        for (int e = tid; e < 128 * 128 / 16; e += 128) sts128(sbase + T::OFF_G + e * 16, make_uint4(0, 0, 0, 0));
        __syncthreads();
        if (tid < 16) sS[tid] = ((red[tid] + red[16 + tid]) + red[32 + tid]) + red[48 + tid];
    }
    fence_proxy_async();   // the operand tiles are read by the tensor core
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *s_tmem;
    const uint32_t lane_off = ((uint32_t)(warp * 32)) << 16;
    float Gs[HP], Ms[HP];   // this thread's positions: sum of g_h, sum of mean G1_h
#pragma unroll
    for (int h = 0; h < HP; ++h) Gs[h] = Ms[h] = 0.f;
    constexpr uint32_t id_acc = idesc_bf16(128, 32, false, false);
    constexpr uint32_t id_dx = idesc_bf16(128, 128, false, false);
    constexpr uint32_t id_a = idesc_bf16(128, 32, true, false);
    int n = 0;
    for (; n < n_items; ++n) {
        const int buf = n & 1;
        const uint32_t zb = sbase + T::OFF_Z + buf * T::TILE_BYTES;
        bool ok = mbar_wait(b_full(buf), (n >> 1) & 1, abort_flag, SITE_PB_BWD | (n << 12));
        if (!__syncthreads_and(ok)) break;
        if (tid == 0) {   // acc = z w' for the tile
            tc_fence_after();
            const uint64_t dz = sdesc(zb, 16, 1024, kSw128), dw = sdesc(sbase + T::OFF_WF, 16, 1024, kSw128);
#pragma unroll
            for (int kk = 0; kk < CZ / 16; ++kk)
                umma_ss(tbase + T::T_ACC, sdesc_add(dz, (kk >> 2) * 16384 + (kk & 3) * 32),
                        sdesc_add(dw, (kk >> 2) * 4096 + (kk & 3) * 32), id_acc, kk > 0);
            umma_commit(b_acc);
        }
        const int t = tile_of(n), i = t / a.nJt, j = (t % a.nJt) * 128 + tid;
        const bool valid = j < a.Nj;
        float g[HP];
#pragma unroll
        for (int h = 0; h < HP; ++h)
            g[h] = (valid && h < a.H) ? a.dbias[h * a.sd0 + (long long)i * a.sd1 + j] : 0.f;
        // the row's mean, then 1 / sqrt(var + eps) in a second pass (thread = position)
        float s0 = 0.f, s1p = 0.f;
#pragma unroll 4
        for (int q = 0; q < CZ / 8; ++q) {
            const uint4 v = lds128(pb_chunk(zb, tid, q));
            const uint32_t xw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                s0 += bf16lo(xw[e]);
                s1p += bf16hi(xw[e]);
            }
        }
        const float mu = (s0 + s1p) * (1.f / CZ);
        float2 var2 = make_float2(0.f, 0.f);
        const float2 nmu = make_float2(-mu, -mu);
#pragma unroll 4
        for (int q = 0; q < CZ / 8; ++q) {
            const uint4 v = lds128(pb_chunk(zb, tid, q));
            const uint32_t xw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 d = fadd2(make_float2(bf16lo(xw[e]), bf16hi(xw[e])), nmu);
                var2 = ffma2(d, d, var2);
            }
        }
        const float rstd = rsqrtf((var2.x + var2.y) * (1.f / CZ) + a.eps);
        ok = mbar_wait(b_acc, n & 1, abort_flag, SITE_PB_BWD | 0x10 | (n << 12));
        ok = __all_sync(0xffffffffu, ok);
        float s1 = 0.f, s2 = 0.f;
        if (ok) {
            tc_fence_after();
            uint32_t d[32];
            tmem_ld32(tbase + T::T_ACC + lane_off, d);
#pragma unroll
            for (int h = 0; h < HP; ++h) {
                const float acc = fmaf(-mu, sS[h], __uint_as_float(d[h]) + __uint_as_float(d[16 + h]));
                s1 = fmaf(g[h], sS[h], s1);
                s2 = fmaf(g[h], acc, s2);
            }
        }
        const float m1 = s1 * (1.f / CZ);                  // mean_c dxh
        const float m2r = s2 * rstd * rstd * (1.f / CZ);   // mean_c(dxh xh) * rstd
        // this position's g (for dxh) and G1 = rstd g (for A), as hi and lo bf16 terms
#pragma unroll
        for (int h = 0; h < HP; ++h) {
            const float g1 = valid ? rstd * g[h] : 0.f;
            Gs[h] += g[h];
            Ms[h] = fmaf(mu, g1, Ms[h]);
            const __nv_bfloat16 ghi = __float2bfloat16_rn(g[h]);
            const __nv_bfloat16 glo = __float2bfloat16_rn(g[h] - __bfloat162float(ghi));
            *reinterpret_cast<__nv_bfloat16 *>(dsmem + T::OFF_G + pb_k64_off(tid, h)) = ghi;
            *reinterpret_cast<__nv_bfloat16 *>(dsmem + T::OFF_G + pb_k64_off(tid, 16 + h)) = ghi;
            *reinterpret_cast<__nv_bfloat16 *>(dsmem + T::OFF_G + pb_k64_off(tid, 32 + h)) = glo;
            const __nv_bfloat16 hi = __float2bfloat16_rn(g1);
            const __nv_bfloat16 lo = __float2bfloat16_rn(g1 - __bfloat162float(hi));
            *reinterpret_cast<__nv_bfloat16 *>(dsmem + T::OFF_GT + pb_wt_off(h, tid)) = hi;
            *reinterpret_cast<__nv_bfloat16 *>(dsmem + T::OFF_GT + pb_wt_off(16 + h, tid)) = lo;
        }
        fence_proxy_async();   // read by the tensor core
        tc_fence_before();
        if (!__syncthreads_and(ok)) break;
        if (tid == 0) {   // dxh = g w'^T, then A += z^T G1
            tc_fence_after();
            const uint64_t dg = sdesc(sbase + T::OFF_G, 16, 1024, kSw128), dwb = sdesc(sbase + T::OFF_WB, 16, 1024, kSw128);
#pragma unroll
            for (int kk = 0; kk < 3; ++kk)
                umma_ss(tbase + T::T_DX, sdesc_add(dg, kk * 32), sdesc_add(dwb, kk * 32), id_dx, kk > 0);
            umma_commit(b_dx);
            const uint64_t da = sdesc(zb, 16384, 1024, kSw128), dt = sdesc(sbase + T::OFF_GT, 16, 1024, kSw128);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                umma_ss(tbase + T::T_A, sdesc_add(da, kk * 2048), sdesc_add(dt, (kk >> 2) * 4096 + (kk & 3) * 32), id_a,
                        (n > 0 || kk > 0) ? 1u : 0u);
            umma_commit(b_all);
        }
        // dz = rstd (dxh - mean dxh - xh mean(dxh xh)), 32 channels at a time
        ok = mbar_wait(b_dx, n & 1, abort_flag, SITE_PB_BWD | 0x20 | (n << 12));
        ok = __all_sync(0xffffffffu, ok);
        if (ok) {
            tc_fence_after();
            __nv_bfloat16 *dst = a.dz + (long long)i * a.sz0 + (long long)j * a.sz1;
#pragma unroll 1
            for (int cb = 0; cb < CZ / 32; ++cb) {
                uint32_t dxr[32];
                tmem_ld32(tbase + T::T_DX + cb * 32 + lane_off, dxr);
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const int q = cb * 4 + q4;   // 16-byte chunk: channels 8 q .. 8 q + 7
                    const uint4 v = lds128(pb_chunk(zb, tid, q));
                    const uint32_t xw[4] = {v.x, v.y, v.z, v.w};
                    uint32_t ow[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float dx0 = __uint_as_float(dxr[q4 * 8 + 2 * e]), dx1 = __uint_as_float(dxr[q4 * 8 + 2 * e + 1]);
                        const float d0 = bf16lo(xw[e]) - mu, d1 = bf16hi(xw[e]) - mu;
                        ow[e] = pack_bf16x2(rstd * (dx0 - m1 - d0 * m2r), rstd * (dx1 - m1 - d1 * m2r));
                    }
                    if (valid) *reinterpret_cast<uint4 *>(dst + q * 8) = make_uint4(ow[0], ow[1], ow[2], ow[3]);
                }
            }
        }
        tc_fence_before();
        if (!__syncthreads_and(ok)) break;   // the tile's rows are read: its buffer may be refilled
        if (tid == 0) {
            ok = mbar_wait(b_all, n & 1, abort_flag, SITE_PB_BWD | 0x30 | (n << 12));
            if (ok && issued < n_items) {
                pb_issue<CZ>(&tmZ, zb, b_full(buf), tile_of(issued), a.nJt);
                ++issued;
            }
        }
    }
    __syncthreads();
    const bool aborted = *abort_flag != 0;
    if (aborted && tid == 0) {
        for (int m = max(0, issued - 2); m < issued; ++m) mbar_wait_drain(b_full(m & 1), (m >> 1) & 1);
        umma_commit(b_drain);
        mbar_wait_drain(b_drain, 0);
    }
    if (!aborted) {
        // the block's sums of g and of mean G1 over its positions: per thread, then over the
        // threads in order (through the idle tile buffers)
        float *red = reinterpret_cast<float *>(dsmem + T::OFF_Z);
#pragma unroll
        for (int h = 0; h < HP; ++h) {
            red[tid * 2 * HP + h] = Gs[h];
            red[tid * 2 * HP + HP + h] = Ms[h];
        }
        __syncthreads();
        float *tot = red + 128 * 2 * HP;   // [2 HP]
        if (tid < 2 * HP) {
            float v = 0.f;
            for (int r = 0; r < 128; ++r) v += red[r * 2 * HP + tid];
            tot[tid] = v;
        }
        __syncthreads();
        // thread = channel = TMEM lane: A[c,h] = (Z^T G1_hi)[c,h] + (Z^T G1_lo)[c,h] - sum mean G1_h
        float *dst = a.part + (long long)blockIdx.x * (CZ * HP + HP);
        uint32_t d[32];
        if (n_items > 0) {
            tc_fence_after();
            tmem_ld32(tbase + T::T_A + lane_off, d);
        }
#pragma unroll
        for (int h = 0; h < HP; ++h)
            dst[tid * HP + h] = n_items > 0 ? (__uint_as_float(d[h]) + __uint_as_float(d[16 + h])) - tot[HP + h] : 0.f;
        if (tid < HP) dst[CZ * HP + tid] = tot[tid];
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tbase, 256);
    }
}

// Sums of the per-block partials, column by column: block = 32 columns x 16 warps; warp w
// adds the partials of blocks [w R, (w + 1) R) in order, then warp 0 adds the 16 warp sums
// in order (bit-stable).  sums[e] for e < Cz * HP + HP: A[c,h] at c * HP + h, then G_h.
__global__ void __launch_bounds__(512) pba_pair_bias_reduce_kernel(const PbArgs a) {
    __shared__ float red[16][33];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int cols = a.Cz * a.hp + a.hp;
    const int e = blockIdx.x * 32 + lane;
    const int R = (a.nparts + 15) / 16;
    const int b_lo = warp * R, b_hi = min(a.nparts, b_lo + R);
    float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
    if (e < cols) {
        const float *src = a.part + e;
        int b = b_lo;
        for (; b + 4 <= b_hi; b += 4) {
            s0 += src[(long long)b * cols];
            s1 += src[(long long)(b + 1) * cols];
            s2 += src[(long long)(b + 2) * cols];
            s3 += src[(long long)(b + 3) * cols];
        }
        for (; b < b_hi; ++b) s0 += src[(long long)b * cols];
    }
    red[warp][lane] = (s0 + s1) + (s2 + s3);
    __syncthreads();
    if (warp == 0 && e < cols) {
        float t = 0.f;
#pragma unroll
        for (int w = 0; w < 16; ++w) t += red[w][lane];
        a.sums[e] = t;
    }
}

// dw[c,h] = gamma_c A[c,h] + beta_c G_h, dgamma_c = sum_h w[c,h] A[c,h], dbeta_c = sum_h w[c,h] G_h
__global__ void __launch_bounds__(128) pba_pair_bias_param_kernel(const PbArgs a) {
    const int c = blockIdx.x * blockDim.x + threadIdx.x;
    if (c >= a.Cz) return;
    const int HP = a.hp;
    float dg = 0.f, db = 0.f;
    for (int h = 0; h < a.H; ++h) {
        const float A = a.sums[c * HP + h], G = a.sums[a.Cz * HP + h];
        const float wch = a.w[c * a.H + h];
        a.dw[c * a.H + h] = a.gamma[c] * A + a.beta[c] * G;
        dg = fmaf(wch, A, dg);
        db = fmaf(wch, G, db);
    }
    a.dgamma[c] = dg;
    a.dbeta[c] = db;
}

}  // namespace pba
