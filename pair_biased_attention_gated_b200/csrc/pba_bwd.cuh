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
// Kernels, in launch order (the dbias kernel runs on a second stream, beside the dq
// conversion, once the main kernel is done):
//   pba_bwd_pre_kernel      per query row: dOa (bf16), dg, and (lse * log2 e, D) row stats
//   pba_bwd_main_kernel     persistent, items (b, h, 128-key tile): steps over query tiles;
//                           dK, dV accumulate in TMEM; each step's dQ partial is added to an
//                           fp32 accumulator in global memory
//   pba_dbias_zero_kernel   local attention only: zeros of dbias outside the window
//   pba_dbias_kernel        CTA = (h, dbias tile, split of b): loops over its rows b with the
//                           bias tile resident; dS summed in registers by three element-wise
//                           warpgroups (48, 48 and 32 keys); one fp32 partial tile
//                           per split; the tile's last CTA to finish sums the partials in
//                           split order (bit-stable dbias)
//   pba_dq_convert_kernel   fp32 dQ accumulator -> bf16 dq (times scale)
// Local attention (win >= 0): key tile j is seen only by query tiles [j - win, j + win]; the
// main kernel's items step over those, the dbias kernel covers only those tile pairs.
#pragma once

#include <type_traits>

#include "pba_device.cuh"

namespace pba {

struct BwdArgs {
    int B, H, Nq, Nk, C;
    int nI, nJ, NqPad, NkPad;
    int splits, rows_per_split;
    int win;                   // local attention: key tile j is seen by query tiles [j - win,
                               // j + win] (clamped); < 0: every query tile
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
    float *dbias_part;         // [splits][H][ntiles][128][128]
    int ntiles;                // dbias tiles computed: nI nJ, or those within the window
    int *tile_count;           // [H][nI][nJ]: splits done (zeroed before the launch)
};

enum : unsigned {
    SITE_BWD_PROD = 0x201, SITE_BWD_MMA = 0x202, SITE_BWD_EW = 0x203, SITE_BWD_EPI = 0x204,
    SITE_DB_PROD = 0x301, SITE_DB_MMA = 0x302, SITE_DB_EW = 0x303
};

constexpr float kLog2eB = 1.4426950408889634f;

// ---------------------------------------------------------------------------------------
// pre: CP/8 lanes per query row (16 bytes of each tensor per lane), rows r = (b, i, h) with
// h fastest, so a warp's rows are contiguous in the [B][N][H][C] tensors; padded rows
// (i >= Nq) only get row stats
// ---------------------------------------------------------------------------------------
// It also clears the dQ accumulator and the dbias tile counters for the kernels after it.
template <int CP>
__global__ void __launch_bounds__(256) pba_bwd_pre_kernel(const BwdArgs a) {
    {
        const int ntiles = a.H * a.nI * a.nJ;
        for (int x = blockIdx.x * blockDim.x + threadIdx.x; x < ntiles; x += gridDim.x * blockDim.x)
            a.tile_count[x] = 0;
    }
    constexpr int LPR = CP / 8;        // lanes per row
    constexpr int RPW = 32 / LPR;      // rows per warp
    const int lane = threadIdx.x & 31, sub = lane % LPR, rw = lane / LPR;
    const long long nrows = (long long)a.B * a.H * a.NqPad;
    const long long wstride = (long long)gridDim.x * (blockDim.x >> 5) * RPW;
    for (long long r0 = ((long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * RPW; r0 < nrows;
         r0 += wstride) {
        const long long r = r0 + rw;
        const bool in = r < nrows;
        int i = 0, h = 0, b = 0;
        if (in) {   // nrows < 2^31 (checked on the host): 32-bit index arithmetic
            const int r32 = (int)r;
            h = r32 % a.H;
            const int bi = r32 / a.H;
            i = bi % a.NqPad;
            b = bi / a.NqPad;
        }
        float D = 0.f;
        const int c0 = sub * 8;
        if (in && i < a.Nq && c0 < a.C) {
            float4 *acc = reinterpret_cast<float4 *>(a.dqacc + (((long long)b * a.Nq + i) * a.H + h) * a.C + c0);
            acc[0] = make_float4(0.f, 0.f, 0.f, 0.f);
            acc[1] = make_float4(0.f, 0.f, 0.f, 0.f);
            const long long orow = b * a.so0 + (long long)i * a.so1 + h * a.so2 + c0;
            const uint4 o4 = *reinterpret_cast<const uint4 *>(a.out + orow);
            const uint4 d4 = *reinterpret_cast<const uint4 *>(a.dout + orow);
            const uint32_t ow[4] = {o4.x, o4.y, o4.z, o4.w};
            const uint32_t dw[4] = {d4.x, d4.y, d4.z, d4.w};
            if (a.has_gate) {
                const long long grow = b * a.sg0 + (long long)i * a.sg1 + h * a.sg2 + c0;
                const uint4 g4 = *reinterpret_cast<const uint4 *>(a.gate + grow);
                const uint32_t gw[4] = {g4.x, g4.y, g4.z, g4.w};
                uint32_t dgw[4], daw[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float o0 = bf16lo(ow[e]), o1 = bf16hi(ow[e]);
                    const float d0 = bf16lo(dw[e]), d1 = bf16hi(dw[e]);
                    D = fmaf(d0, o0, D);
                    D = fmaf(d1, o1, D);
                    // the forward epilogue's sigmoid, so both passes use the same gate values
                    const float s0 = sigmoid_fast(bf16lo(gw[e]));
                    const float s1 = sigmoid_fast(bf16hi(gw[e]));
                    daw[e] = pack_bf16x2(d0 * s0, d1 * s1);
                    dgw[e] = pack_bf16x2(d0 * o0 * (1.f - s0), d1 * o1 * (1.f - s1));
                }
                *reinterpret_cast<uint4 *>(a.doa + (((long long)b * a.Nq + i) * a.H + h) * a.C + c0) =
                    make_uint4(daw[0], daw[1], daw[2], daw[3]);
                *reinterpret_cast<uint4 *>(a.dgate + grow) = make_uint4(dgw[0], dgw[1], dgw[2], dgw[3]);
            } else {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    D = fmaf(bf16lo(dw[e]), bf16lo(ow[e]), D);
                    D = fmaf(bf16hi(dw[e]), bf16hi(ow[e]), D);
                }
            }
        }
#pragma unroll
        for (int x = 1; x < LPR; x <<= 1) D += __shfl_xor_sync(0xffffffffu, D, x);
        if (in && sub == 0) {
            float2 rs = make_float2(INFINITY, 0.f);
            if (i < a.Nq) {
                const float l = a.lse[((long long)b * a.H + h) * a.Nq + i];
                rs.x = (l == -INFINITY) ? INFINITY : l * kLog2eB;
                rs.y = D;
            }
            a.rowstats[((long long)b * a.H + h) * a.NqPad + i] = rs;   // [B][H][NqPad]
        }
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

// P and dS of 64 keys (one half of a 128-key tile) for one query row, in KC-key chunks.
//   tS, tdP: this lane's S and dP columns in TMEM; bias_row: the row's 64 bf16 bias values
//   in a 128-byte swizzled shared-memory row; mw0, mw1: mask words of those 64 keys (all
//   ones when `full`); sl2e = scale log2 e; lse2 = lse log2 e; D = sum_c dout out.
//   P = exp2(S sl2e + bias log2 e - lse2) (0 for masked keys), dS = P (dP - D).
// For each pair of keys (c, c + 1), c even, `use(c, p, dpd)` receives the two P and dP - D
// (dS = P (dP - D) is formed by the caller: a product, or a fused multiply-add into a sum);
// `loaded()` is called once the last chunk's S and dP are in registers (the TMEM columns
// may then be handed back before the chunk is computed).
template <int KC, typename Use, typename Loaded>
__device__ __forceinline__ void p_ds_half(uint32_t tS, uint32_t tdP, uint32_t bias_row, int row,
                                          bool has_bias, uint32_t mw0, uint32_t mw1, bool full,
                                          float sl2e, float lse2, float D, Use &&use, Loaded &&loaded) {
    // KC-key chunks (32 or 16): S and dP of one chunk take 2 KC registers; the main kernel
    // uses 16 to stay within the 128 registers a thread has at 512 threads per CTA
    static_assert(KC == 16 || KC == 32, "chunk");
    const float2 sl2 = make_float2(sl2e, sl2e), l2e2 = make_float2(kLog2eB, kLog2eB);
    const float2 nl2 = make_float2(-lse2, -lse2), nD2 = make_float2(-D, -D);
#pragma unroll
    for (int q = 0; q < 64 / KC; ++q) {
        // the chunk's bias words first: their shared-memory loads are then in flight while
        // the TMEM load below waits
        uint4 bws[KC / 8];
#pragma unroll
        for (int c2 = 0; c2 < KC / 8; ++c2) {
            bws[c2] = make_uint4(0, 0, 0, 0);
            if (has_bias) bws[c2] = lds128(bias_row + (((q * (KC / 8) + c2) ^ (row & 7)) << 4));
        }
        uint32_t r[2 * KC];   // S of keys KC q .. KC q + KC - 1 in r[0, KC), dP in r[KC, 2 KC)
        if constexpr (KC == 32) tmem_ld32x2(tS + q * KC, tdP + q * KC, r);
        else tmem_ld16x2(tS + q * KC, tdP + q * KC, r);
        if (q == 64 / KC - 1) loaded();
        const uint32_t mw = ((q * KC) < 32 ? mw0 : mw1) >> ((q * KC) & 31);
#pragma unroll
        for (int c2 = 0; c2 < KC / 8; ++c2) {
            const uint4 bw = bws[c2];
            const uint32_t bb[4] = {bw.x, bw.y, bw.z, bw.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int k = c2 * 8 + 2 * e;   // key within the chunk
                float2 u = ffma2(make_float2(bf16lo(bb[e]), bf16hi(bb[e])), l2e2, nl2);
                u = ffma2(make_float2(__uint_as_float(r[k]), __uint_as_float(r[k + 1])), sl2, u);
                float2 p = make_float2(ex2(u.x), ex2(u.y));
                if (!full) {
                    p.x = ((mw >> k) & 1u) ? p.x : 0.f;
                    p.y = ((mw >> (k + 1)) & 1u) ? p.y : 0.f;
                }
                const float2 dpd = fadd2(make_float2(__uint_as_float(r[KC + k]), __uint_as_float(r[KC + 1 + k])), nD2);
                use(q * KC + k, p, dpd);
            }
        }
    }
}

// The bits of mask word w (keys 32 w .. 32 w + 31) that fall in the keys k0 .. k0 + nk - 1.
__host__ __device__ constexpr uint32_t key_bits(int k0, int nk, int w) {
    const int lo = (k0 > 32 * w ? k0 : 32 * w) - 32 * w;
    const int hi = (k0 + nk < 32 * w + 32 ? k0 + nk : 32 * w + 32) - 32 * w;
    return hi <= lo ? 0u : (hi - lo == 32 ? 0xffffffffu : ((1u << (hi - lo)) - 1u) << lo);
}
static_assert(key_bits(48, 48, 1) == 0xffff0000u && key_bits(48, 48, 2) == 0xffffffffu &&
              key_bits(0, 48, 1) == 0x0000ffffu && key_bits(96, 32, 3) == 0xffffffffu &&
              key_bits(96, 32, 2) == 0u, "key_bits");

// P and dS of the NK keys K0 .. K0 + NK - 1 of a 128-key tile for one query row, in 16-key
// chunks (as p_ds_half, for a key range that need not be a half):
//   tS, tdP: this lane's S and dP column 0 in TMEM; bias_row: the row in the first 64-key
//   half of the bias tile (128-byte swizzled rows, the second half 16 KB further); mw: the
//   four mask words of the tile's keys (all ones when `full`).
// `use(c, p, dpd)` receives keys K0 + c and K0 + c + 1 (c even); `loaded()` is called once the
// last chunk's S and dP are in registers.
template <int K0, int NK, typename Use, typename Loaded>
__device__ __forceinline__ void p_ds_keys(uint32_t tS, uint32_t tdP, uint32_t bias_row, int row,
                                          bool has_bias, const uint32_t *mw, bool full, float sl2e,
                                          float lse2, float D, Use &&use, Loaded &&loaded) {
    static_assert(K0 % 16 == 0 && NK % 16 == 0 && K0 + NK <= 128, "key range");
    const float2 sl2 = make_float2(sl2e, sl2e), l2e2 = make_float2(kLog2eB, kLog2eB);
    const float2 nl2 = make_float2(-lse2, -lse2), nD2 = make_float2(-D, -D);
#pragma unroll
    for (int q = 0; q < NK / 16; ++q) {
        const int kc = K0 + 16 * q;   // first key of the chunk
        uint4 bws[2];
#pragma unroll
        for (int c2 = 0; c2 < 2; ++c2) {
            const int k8 = kc + 8 * c2;
            bws[c2] = make_uint4(0, 0, 0, 0);
            if (has_bias)
                bws[c2] = lds128(bias_row + (k8 >> 6) * 16384 + ((((k8 & 63) >> 3) ^ (row & 7)) << 4));
        }
        uint32_t r[32];   // S of the chunk's keys in r[0, 16), dP in r[16, 32)
        tmem_ld16x2(tS + kc, tdP + kc, r);
        if (q == NK / 16 - 1) loaded();
        const uint32_t m = full ? 0xffffffffu : (mw[kc >> 5] >> (kc & 31));
#pragma unroll
        for (int c2 = 0; c2 < 2; ++c2) {
            const uint4 bw = bws[c2];
            const uint32_t bb[4] = {bw.x, bw.y, bw.z, bw.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int k = c2 * 8 + 2 * e;   // key within the chunk
                float2 u = ffma2(make_float2(bf16lo(bb[e]), bf16hi(bb[e])), l2e2, nl2);
                u = ffma2(make_float2(__uint_as_float(r[k]), __uint_as_float(r[k + 1])), sl2, u);
                float2 p = make_float2(ex2(u.x), ex2(u.y));
                if (!full) {
                    p.x = ((m >> k) & 1u) ? p.x : 0.f;
                    p.y = ((m >> (k + 1)) & 1u) ? p.y : 0.f;
                }
                const float2 dpd = fadd2(make_float2(__uint_as_float(r[16 + k]), __uint_as_float(r[17 + k])), nD2);
                use(kc - K0 + k, p, dpd);
            }
        }
    }
}

// ---------------------------------------------------------------------------------------
// main backward kernel: dQ, dK, dV
//
// Persistent: one CTA per SM walks the items (b, h, 128-key tile) n = blockIdx.x,
// blockIdx.x + gridDim.x, ...; an item's steps are its query tiles.  The step pipeline
// (S/dP -> P/dS -> dV, dK, dQ) runs on across item boundaries: the next item's K/V tiles
// load into the other stage while the current item finishes, and dK/dV accumulate in one
// of two TMEM buffers, so an item's dK/dV epilogue overlaps the next item's MMAs.  The dQ
// flushes and the dK/dV epilogues belong to a warpgroup of their own, so the element-wise
// warps only turn S/dP into P/dS.
// ---------------------------------------------------------------------------------------
template <int CP>
struct BwdTraits {
    // dQ partials (CP = 32): written into a 128-byte-swizzled fp32 staging tile and added to
    // the accumulator by one TMA tensor reduction per step; otherwise vector reductions
    static constexpr bool DQ_TMA = CP == 32;
    static constexpr int QS = (CP == 16) ? 3 : 2;               // Q/dOa/row-stat stages
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
    static constexpr int OFF_DQS = OFF_MASK + 1024;             // fp32 [128][CP] staging (DQ_TMA)
    static constexpr int SMEM_BYTES = OFF_DQS + (DQ_TMA ? 128 * CP * 4 : 0) + 1024;
    static constexpr uint32_t SWZ = CP == 64 ? kSw128 : (CP == 32 ? kSw64 : kSw32);
    static constexpr uint32_t ROWB = CP * 2;
    // TMEM columns: S, dP, then per dK/dV buffer x: dK at T_DK + 2 CP x, dV after it, then
    // the two dQ buffers
    static constexpr int T_S = 0, T_DP = 128, T_DK = 256, T_DQ = 256 + DKB * 2 * CP;
    static_assert(T_DQ + 2 * CP <= 512, "TMEM");
};
static_assert(BwdTraits<64>::SMEM_BYTES <= 232448 && BwdTraits<32>::SMEM_BYTES <= 232448, "smem");

// Warp roles (512 threads, four warpgroups): warps 0-7 element-wise (two warpgroups, one
// 64-key half each), warp 8 TMA producer, warp 9 TMEM allocator and (lane 0) issuer of the
// dV products, warp 10 (lane 0) issuer of S = Q K^T and dP = dOa V^T of each step and then
// of the previous step's dQ products, warp 11 (lane 0) issuer of the dK products, warps
// 12-15 the dQ flushes and dK/dV epilogues (thread = TMEM lane).  One thread issues a
// tcgen05.mma only every ~200 cycles whatever the shape (measured: M = 128, K = 16, N = 32
// to 256), while several issuing threads proceed at that rate each; the 28 MMAs of a step
// are therefore spread over three threads (12, 8 and 8).  Every thread has 128 registers
// (512 threads on one SM).
template <int CP>
__global__ void __launch_bounds__(512, 1)
pba_bwd_main_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                    const __grid_constant__ CUtensorMap tmBias, const __grid_constant__ CUtensorMap tmDQ,
                    const BwdArgs a) {
    using T = BwdTraits<CP>;
    constexpr int QS = T::QS, BS = T::BS, KVB = T::KVB, DKB = T::DKB;
    extern __shared__ uint8_t dsmem[];
    __shared__ __align__(8) uint64_t bars[16 + 2 * QS + 2 * BS + 2 * KVB + 2 * DKB + 2];
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
    const uint32_t b_stg_full = smem_u32(&bars[OK_ + 2 * KVB + 2 * DKB]);       // dQ staging written
    const uint32_t b_stg_free = smem_u32(&bars[OK_ + 2 * KVB + 2 * DKB + 1]);   // staging read by TMA

    const uint32_t raw = smem_u32(dsmem);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    uint8_t *gbase = dsmem + (sbase - raw);

    const int warp = warp_id(), lane = lane_id();
    const long long n_items = (long long)a.B * a.H * a.nJ;
    // items of this CTA: blockIdx.x + m * gridDim.x, m < M; an item's steps are its query
    // tiles ilo .. ilo + ni - 1, and t counts the CTA's steps
    const int M = blockIdx.x < n_items ? (int)((n_items - 1 - blockIdx.x) / gridDim.x) + 1 : 0;
    struct Item { int b, h, jt, ilo, ni; };
    auto item = [&](int m) {   // n_items < 2^31 (checked on the host)
        int n = (int)blockIdx.x + m * (int)gridDim.x;
        Item it;
        it.jt = n % a.nJ;
        n /= a.nJ;
        it.h = n % a.H;
        it.b = n / a.H;
        it.ilo = a.win < 0 ? 0 : max(0, it.jt - a.win);
        it.ni = (a.win < 0 ? a.nI : min(a.nI, it.jt + a.win + 1)) - it.ilo;   // >= 1 (host check)
        return it;
    };

    if (threadIdx.x == 0) {
        mbar_init(b_sd_full, 1);
        mbar_init(b_sd_free, 256);
        mbar_init(b_ps_full, 256);
        mbar_init(b_ps_free, 3);   // the dV, dK and dQ issuers' commits
        mbar_init(b_drain, 3);     // one commit from each issuer
        for (int x = 0; x < 2; ++x) {
            mbar_init(b_dq_full(x), 1);
            mbar_init(b_dq_free(x), 128);
        }
        for (int x = 0; x < QS; ++x) {
            mbar_init(b_q_full(x), 1);
            mbar_init(b_q_empty(x), 2 + 256);   // the dV and dK commits, the element-wise warps
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
            mbar_init(b_dkv_full(x), 2);   // the dV and dK commits
            mbar_init(b_dkv_free(x), 128);
        }
        mbar_init(b_stg_full, 128);
        mbar_init(b_stg_free, 1);
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
        int t = 0;
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
            for (int ii = 0; ii < it.ni && ok; ++ii, ++t) {
                const int st = t % QS, bs = t % BS, i0 = (it.ilo + ii) * 128;
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
    } else if (warp == 10) {
        // ------------------------------------------------------------------ S/dP and dQ issuer
        // S/dP of step t, then the dQ products of step t - 1, so that the next step's scores
        // are never queued behind this step's products.  With one K/V stage the previous
        // item's last dQ (which frees the stage) goes first at an item's first step.
        if (lane == 0) {
            constexpr uint32_t SBO = 8 * T::ROWB;
            constexpr uint32_t id_s = idesc_bf16(128, 128, false, false);   // S = Q K^T, dP = dOa V^T
            constexpr uint32_t id_q = idesc_bf16(128, CP, false, true);     // dQ = dS K
            const uint32_t sDS = sbase + T::OFF_DS;
            bool ok = true;
            // S/dP of step t: its item's K/V, its Q/dOa, and S/dP of step t - 1 read out
            auto issue_sdp = [&](int t, int m, int ii) -> bool {
                const int st = t % QS, x = m % KVB;
                const bool okk = mbar_wait_all(abort_flag,
                                               b_kv_full(x), (m / KVB) & 1, ii == 0, SITE_BWD_MMA | 0x80 | (t << 12),
                                               b_q_full(st), (t / QS) & 1, true, SITE_BWD_MMA | 0x90 | (t << 12),
                                               b_sd_free, (t - 1) & 1, t > 0, SITE_BWD_MMA | 0xA0 | (t << 12));
                if (!okk) return false;
                tc_fence_after();
                const uint32_t sQ = sbase + T::OFF_Q + st * 2 * T::TILE_BYTES;
                const uint64_t dQd = sdesc(sQ, 16, SBO, T::SWZ), dDO = sdesc(sQ + T::TILE_BYTES, 16, SBO, T::SWZ);
                const uint64_t dK = sdesc(sbase + T::OFF_K + x * T::TILE_BYTES, 16, SBO, T::SWZ);
                const uint64_t dV = sdesc(sbase + T::OFF_V + x * T::TILE_BYTES, 16, SBO, T::SWZ);
#pragma unroll
                for (int kk = 0; kk < CP / 16; ++kk) {   // K steps of 16 channels: 32 bytes on
                    umma_ss(tbase + T::T_S, sdesc_add(dQd, kk * 32), sdesc_add(dK, kk * 32), id_s, kk > 0);
                    umma_ss(tbase + T::T_DP, sdesc_add(dDO, kk * 32), sdesc_add(dV, kk * 32), id_s, kk > 0);
                }
                umma_commit(b_sd_full);
                return true;
            };
            // dQ of step t (item m, its step i of ni): P/dS written, the dQ buffer free
            auto issue_dq = [&](int t, int m, int i, int ni) -> bool {
                const int x = m % KVB;
                const bool okk = mbar_wait_all(abort_flag,
                                               b_ps_full, t & 1, true, SITE_BWD_MMA | 0x20 | (t << 12),
                                               b_dq_free(t & 1), ((t >> 1) - 1) & 1, t >= 2, SITE_BWD_MMA | 0x70 | (t << 12));
                if (!okk) return false;
                tc_fence_after();
                const uint64_t dA = sdesc(sDS, 16, 1024, kSw128);
                const uint64_t dB = sdesc(sbase + T::OFF_K + x * T::TILE_BYTES, T::TILE_BYTES, SBO, T::SWZ);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    // K steps over 16 keys: A (dS, K-major) advances 32 B within a 64-key half,
                    // B (K, MN-major) 16 rows
                    umma_ss(tbase + T::T_DQ + (t & 1) * CP, sdesc_add(dA, (kk >> 2) * 16384 + (kk & 3) * 32),
                            sdesc_add(dB, kk * 16 * T::ROWB), id_q, kk > 0);
                }
                umma_commit(b_ps_free);
                umma_commit(b_dq_full(t & 1));
                if (i == ni - 1) umma_commit(b_kv_empty(x));   // the item's last reader of K/V
                return true;
            };
            int t = 0;
            int pm = -1, pi = 0, pni = 0;   // the previous step: item, step within it, its steps
            for (int m = 0; m < M && ok; ++m) {
                const int ni = item(m).ni;
                for (int ii = 0; ii < ni && ok; ++ii, ++t) {
                    const bool dq_first = KVB == 1 && ii == 0;
                    if (dq_first && t > 0) ok = issue_dq(t - 1, pm, pi, pni);
                    if (ok) ok = issue_sdp(t, m, ii);
                    if (ok && !dq_first && t > 0) ok = issue_dq(t - 1, pm, pi, pni);
                    pm = m; pi = ii; pni = ni;
                }
            }
            if (ok && t > 0) issue_dq(t - 1, pm, pi, pni);
        }
    } else if (warp == 9 || warp == 11) {
        // ------------------------------------------------------------------ dV / dK issuers
        // warp 9 issues dV += P^T dOa, warp 11 dK += dS^T Q: one issuing thread per product,
        // so that each MMA stream goes at its own thread's issue rate
        if (lane == 0) {
            constexpr uint32_t SBO = 8 * T::ROWB;
            constexpr uint32_t id_kv = idesc_bf16(128, CP, true, true);
            const bool is_dv = warp == 9;
            const uint32_t sA = sbase + (is_dv ? T::OFF_P : T::OFF_DS);
            bool ok = true;
            // step t: P/dS written (S/dP of the step were read out before that, so its S/dP
            // MMAs are complete); this item's dK/dV buffer free
            int t = 0;
            for (int m = 0; m < M && ok; ++m) {
                const int ni = item(m).ni;
                for (int i = 0; i < ni && ok; ++i, ++t) {   // i: the item's step (query tile ilo + i)
                    const int st = t % QS, d = m % DKB;
                    // P/dS of the step, and at an item's first step its dK/dV buffer (read out by
                    // the epilogue of item m - DKB)
                    ok = mbar_wait_all(abort_flag,
                                       b_ps_full, t & 1, true, SITE_BWD_MMA | 0x20 | (t << 12),
                                       b_dkv_free(d), ((m / DKB) - 1) & 1, i == 0 && m >= DKB, SITE_BWD_MMA | 0x60 | (t << 12));
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t sQ = sbase + T::OFF_Q + st * 2 * T::TILE_BYTES;
                    const uint64_t dA = sdesc(sA, 16384, 1024, kSw128);
                    const uint64_t dB = sdesc(is_dv ? sQ + T::TILE_BYTES : sQ, T::TILE_BYTES, SBO, T::SWZ);   // dOa or Q
                    const uint32_t tD = tbase + T::T_DK + d * 2 * CP + (is_dv ? CP : 0);
                    // K steps over 16 queries: A (P^T / dS^T, MN-major) rows advance 2 KB,
                    // B (dOa / Q, MN-major) rows advance 16 rows
                    umma_ss(tD, dA, dB, id_kv, i > 0 ? 1u : 0u);
#pragma unroll
                    for (int kk = 1; kk < 8; ++kk)
                        umma_ss(tD, sdesc_add(dA, kk * 2048), sdesc_add(dB, kk * 16 * T::ROWB), id_kv, 1u);
                    umma_commit(b_ps_free);
                    umma_commit(b_q_empty(st));
                    if (i == ni - 1) umma_commit(b_dkv_full(d));
                }
            }
        }
    } else if (warp < 8) {
        // ------------------------------------------------------------------ elementwise
        // warpgroup e owns keys [64 e, 64 e + 64) of the tile for all 128 query rows
        const int e = warp >> 2;
        const int row = (warp & 3) * 32 + lane;
        const uint32_t lane_off = ((uint32_t)((warp & 3) * 32)) << 16;
        const float sl2e = a.scale * kLog2eB;
        bool ok = true;
        uint32_t mw0 = 0, mw1 = 0;
        bool full = true;
        int t = 0;
        for (int m = 0; m < M && ok; ++m) {
            const int ni = item(m).ni;
            for (int i = 0; i < ni && ok; ++i, ++t) {
                const int st = t % QS, bs = t % BS;
                // the item's K/V tiles (with its mask words) at its first step, the step's S/dP,
                // Q stage (row statistics) and bias tile: probed together
                ok = mbar_wait_all(abort_flag,
                                   b_kv_full(m % KVB), (m / KVB) & 1, i == 0, SITE_BWD_EW | 0x30 | (t << 12),
                                   b_sd_full, t & 1, true, SITE_BWD_EW | (t << 12),
                                   b_q_full(st), (t / QS) & 1, true, SITE_BWD_EW | 0x40 | (t << 12),
                                   b_bias_full(bs), (t / BS) & 1, true, SITE_BWD_EW | 0x50 | (t << 12));
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                if (i == 0) {
                    const uint32_t *mw = reinterpret_cast<const uint32_t *>(gbase + T::OFF_MASK) + (m % KVB) * 8;
                    mw0 = mw[2 * e];
                    mw1 = mw[2 * e + 1];
                    full = mw[4 + e] != 0;
                }
                tc_fence_after();
                const float2 rs = reinterpret_cast<const float2 *>(gbase + T::OFF_RS + st * 1024)[row];
                uint32_t pp[32], dsp[32];   // P and dS as bf16 pairs, keys 2 c and 2 c + 1
                bool prod_done = t == 0;    // the previous step's products, probed below
                const uint32_t bias_row = sbase + T::OFF_BIAS + bs * T::BIAS_BYTES + e * 16384 + row * 128;
                p_ds_half<16>(tbase + T::T_S + e * 64 + lane_off, tbase + T::T_DP + e * 64 + lane_off, bias_row,
                          row, a.has_bias != 0, mw0, mw1, full, sl2e, rs.x, rs.y,
                          [&](int c, float2 p, float2 dpd) {
                              const float2 ds = fmul2(p, dpd);
                              pp[c >> 1] = pack_bf16x2(p.x, p.y);
                              dsp[c >> 1] = pack_bf16x2(ds.x, ds.y);
                          },
                          [&]() {   // S/dP read out: the next step's S/dP MMAs may start
                              tc_fence_before();
                              mbar_arrive(b_sd_free);
                              // probe the previous step's products now, so that the probe's
                              // latency overlaps the last chunk (a complete phase stays
                              // complete: the next one needs this step's P/dS)
                              if (t > 0) prod_done = mbar_test(b_ps_free, (t - 1) & 1);
                          });
                mbar_arrive(b_bias_empty(bs));
                mbar_arrive(b_q_empty(st));
                if (!__all_sync(0xffffffffu, prod_done)) {
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
                    sts128(prow + sw, make_uint4(pp[c8 * 4], pp[c8 * 4 + 1], pp[c8 * 4 + 2], pp[c8 * 4 + 3]));
                    sts128(drow + sw, make_uint4(dsp[c8 * 4], dsp[c8 * 4 + 1], dsp[c8 * 4 + 2], dsp[c8 * 4 + 3]));
                }
                // generic-proxy writes -> visible to the tensor core's async proxy
                fence_proxy_async();
                mbar_arrive(b_ps_full);
            }
        }
    } else if (warp >= 12) {
        // ------------------------------------------------------------------ dQ and dK/dV
        // thread = TMEM lane = query row (dQ) or key row (dK/dV); the warpgroup's first
        // thread issues the dQ tile's TMA reductions
        const int row = (warp & 3) * 32 + lane;
        const uint32_t lane_off = ((uint32_t)((warp & 3) * 32)) << 16;
        const bool issuer = threadIdx.x == 384;
        bool ok = true;
        auto flush_dq = [&](int t, int i0, const Item &it) -> bool {
            // dQ(t): this thread's query row, all CP channels, added to dqacc
            bool okf = mbar_wait(b_dq_full(t & 1), (t >> 1) & 1, abort_flag, SITE_BWD_EPI | 0x10 | (t << 12));
            okf = __all_sync(0xffffffffu, okf);
            if (!okf) return false;
            tc_fence_after();
            const uint32_t tq = tbase + T::T_DQ + (t & 1) * CP + lane_off;
            const int i = i0 + row;
            if constexpr (T::DQ_TMA) {
                uint32_t r[32];
                tmem_ld32(tq, r);
                tc_fence_before();
                mbar_arrive(b_dq_free(t & 1));
                // the staging tile of the previous flush has been read by its TMA reduction:
                // the thread that issued it checks that here (a step later, so it no longer
                // waits) and releases the tile
                if (t > 0) {
                    if (issuer) {
                        bulk_wait_read_all();
                        mbar_arrive(b_stg_free);
                    }
                    okf = mbar_wait(b_stg_free, (t - 1) & 1, abort_flag, SITE_BWD_EPI | 0x70 | (t << 12));
                    okf = __all_sync(0xffffffffu, okf);
                    if (!okf) return false;
                }
                // row `row` of the 128 x 32 fp32 staging tile: eight 16-byte chunks, swizzled
                const uint32_t srow = sbase + T::OFF_DQS + row * 128;
#pragma unroll
                for (int q4 = 0; q4 < 8; ++q4)
                    sts128(srow + ((q4 ^ (row & 7)) << 4),
                           make_uint4(r[q4 * 4], r[q4 * 4 + 1], r[q4 * 4 + 2], r[q4 * 4 + 3]));
                fence_proxy_async();
                mbar_arrive(b_stg_full);
                bool oki = true;
                if (issuer) {
                    // rows >= Nq and channels >= C fall outside the map and are skipped
                    oki = mbar_wait(b_stg_full, t & 1, abort_flag, SITE_BWD_EPI | 0x80 | (t << 12));
                    if (oki) {
                        tma_reduce_add_4d(&tmDQ, sbase + T::OFF_DQS, 0, it.h, i0, it.b);
                        bulk_commit();
                    }
                }
                if (!__all_sync(0xffffffffu, oki)) return false;   // the issuer's warp leaves together
            } else {
                float *dst = a.dqacc + (((long long)it.b * a.Nq + i) * a.H + it.h) * a.C;
#pragma unroll
                for (int h32 = 0; h32 < (CP + 31) / 32; ++h32) {
                    constexpr int W = CP < 32 ? CP : 32;   // columns per TMEM load
                    uint32_t r[W];
                    if constexpr (W == 16) tmem_ld16(tq, r);
                    else tmem_ld32(tq + h32 * 32, r);
                    if (h32 == (CP + 31) / 32 - 1) {
                        tc_fence_before();
                        mbar_arrive(b_dq_free(t & 1));
                    }
                    if (i < a.Nq) {
#pragma unroll
                        for (int c4 = 0; c4 < W / 4; ++c4) {
                            const int c = h32 * 32 + c4 * 4;
                            if (c < a.C)
                                red_add_v4(dst + c, __uint_as_float(r[c4 * 4]), __uint_as_float(r[c4 * 4 + 1]),
                                           __uint_as_float(r[c4 * 4 + 2]), __uint_as_float(r[c4 * 4 + 3]));
                        }
                    }
                }
            }
            return true;
        };
        auto epilogue = [&](int m, const Item &it) -> bool {
            // dK (times scale) and dV of item m; lane = key row
            bool oke = mbar_wait(b_dkv_full(m % DKB), (m / DKB) & 1, abort_flag, SITE_BWD_EPI | 0x20 | (m << 12));
            oke = __all_sync(0xffffffffu, oke);
            if (!oke) return false;
            tc_fence_after();
            const int j = it.jt * 128 + row;
            const uint32_t tdk = tbase + T::T_DK + (m % DKB) * 2 * CP + lane_off;
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                __nv_bfloat16 *dst = e == 0 ? a.dk + it.b * a.sk0 + (long long)j * a.sk1 + it.h * a.sk2
                                            : a.dv + it.b * a.sv0 + (long long)j * a.sv1 + it.h * a.sv2;
                const float mul = e == 0 ? a.scale : 1.f;
#pragma unroll
                for (int h32 = 0; h32 < (CP + 31) / 32; ++h32) {
                    constexpr int W = CP < 32 ? CP : 32;
                    uint32_t r[W];
                    if constexpr (W == 16) tmem_ld16(tdk + e * CP, r);
                    else tmem_ld32(tdk + e * CP + h32 * 32, r);
                    if (e == 1 && h32 == (CP + 31) / 32 - 1) {
                        tc_fence_before();
                        mbar_arrive(b_dkv_free(m % DKB));
                    }
                    if (j < a.Nk) {
#pragma unroll
                        for (int c8 = 0; c8 < W / 8; ++c8) {
                            const int c = h32 * 32 + c8 * 8;
                            if (c < a.C) {
                                uint32_t ow[4];
#pragma unroll
                                for (int q = 0; q < 4; ++q)
                                    ow[q] = pack_bf16x2(__uint_as_float(r[c8 * 8 + 2 * q]) * mul,
                                                        __uint_as_float(r[c8 * 8 + 2 * q + 1]) * mul);
                                *reinterpret_cast<uint4 *>(dst + c) = make_uint4(ow[0], ow[1], ow[2], ow[3]);
                            }
                        }
                    }
                }
            }
            return true;
        };
        int t = 0;
        for (int m = 0; m < M && ok; ++m) {
            const Item cur = item(m);
            for (int i = 0; i < cur.ni && ok; ++i, ++t) {
                ok = flush_dq(t, (cur.ilo + i) * 128, cur);
                if (ok && i == cur.ni - 1) ok = epilogue(m, cur);
            }
        }
        if (T::DQ_TMA && issuer) bulk_wait_all();   // its TMA reductions are done
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
        if ((warp == 9 || warp == 10 || warp == 11) && lane == 0) {
            umma_commit(b_drain);   // each issuer's own MMAs
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

// dbias tile number bt -> (query tile, key tile): row-major over the tile pairs the kernels
// visit (every pair, or under a window the pairs with |query tile - key tile| <= win)
__device__ __forceinline__ void dbias_tile(const BwdArgs &a, int bt, int &it, int &jt) {
    if (a.win < 0) {
        it = bt / a.nJ;
        jt = bt % a.nJ;
        return;
    }
    it = a.nI - 1;
    jt = a.nJ - 1;
    for (int i = 0; i < a.nI; ++i) {
        const int lo = max(0, i - a.win), hi = min(a.nJ, i + a.win + 1);
        if (bt < hi - lo) {
            it = i;
            jt = lo + bt;
            return;
        }
        bt -= hi - lo;
    }
}

// local attention: dbias is 0 at every pair outside the window (no query of such a pair's
// tile sees its key); the dbias kernel writes the tiles inside it
__global__ void __launch_bounds__(256) pba_dbias_zero_kernel(const BwdArgs a) {
    // one dbias row (h, i) per block: the keys before and after the row's window
    for (long long r = blockIdx.x; r < (long long)a.H * a.Nq; r += gridDim.x) {
        const int t = (int)(r % a.Nq) >> 7;
        const int lo = max(0, t - a.win) * 128, hi = min(a.Nk, (t + a.win + 1) * 128);
        float *row = a.dbias + r * a.Nk;
        for (int j = threadIdx.x; j < lo; j += blockDim.x) row[j] = 0.f;
        for (int j = hi + threadIdx.x; j < a.Nk; j += blockDim.x) row[j] = 0.f;
    }
}

// ---------------------------------------------------------------------------------------
// dbias kernel: CTA = (h, dbias tile, split s); loops over its rows b
// ---------------------------------------------------------------------------------------
template <int CP>
struct DbTraits {
    // element-wise warpgroups: keys 0-47, 48-95 and 96-127 (three warps per SM
    // sub-partition, for latency hiding), then the producer and the MMA issuer warps
    static constexpr int NWG = 3;
    static constexpr int THREADS = 32 * (4 * NWG + 2);
    static constexpr int W_PROD = 4 * NWG, W_MMA = 4 * NWG + 1;
    // stages (one row b each): as many as fit beside the bias tile, so that the TMA loads of
    // several rows are in flight
    static constexpr int NS = (CP == 64) ? 2 : (CP == 32 ? 5 : 8);
    static constexpr int TILE_BYTES = 128 * CP * 2;
    static constexpr int STAGE_BYTES = 4 * TILE_BYTES + 1024;     // Q, dOa, K, V, row stats
    static constexpr int OFF_BIAS = 0;
    static constexpr int OFF_STAGE = 128 * 128 * 2;               // + st * STAGE_BYTES
    static constexpr int OFF_MASK = OFF_STAGE + NS * STAGE_BYTES; // u32 [NS][8]
    static constexpr int SMEM_BYTES = OFF_MASK + NS * 32 + 1024;
    static constexpr uint32_t SWZ = CP == 64 ? kSw128 : (CP == 32 ? kSw64 : kSw32);
    static constexpr uint32_t ROWB = CP * 2;
};

// one CTA per SM: the dynamic shared memory (with its alignment slack) within the 227 KB a
// CTA may have
static_assert(DbTraits<16>::SMEM_BYTES <= 232448 && DbTraits<32>::SMEM_BYTES <= 232448 &&
              DbTraits<64>::SMEM_BYTES <= 232448, "dbias shared memory");

template <int CP>
__global__ void __launch_bounds__(DbTraits<CP>::THREADS, 1)
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
    const int bt = idx % a.ntiles;   // the tile, in dbias_tile order
    idx /= a.ntiles;
    const int h = idx % a.H;
    const int sp = idx / a.H;
    int it, jt;
    dbias_tile(a, bt, it, jt);
    const int i0 = it * 128, j0 = jt * 128;
    const int bstart = sp * a.rows_per_split;
    const int nb = max(0, min(a.rows_per_split, a.B - bstart));

    if (threadIdx.x == 0) {
        mbar_init(b_bias, 1);
        mbar_init(b_drain, 1);
        for (int x = 0; x < 2; ++x) {
            mbar_init(b_sd_full(x), 1);
            mbar_init(b_sd_free(x), 128 * T::NWG);
        }
        for (int x = 0; x < NS; ++x) {
            mbar_init(b_full(x), 1);
            mbar_init(b_empty(x), 1 + 128 * T::NWG);
        }
        s_abort = 0;
        fence_mbar_init();
    }
    if (warp == T::W_MMA) {
        tmem_alloc(smem_u32(&s_tmem_base), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = s_tmem_base;
    volatile int *abort_flag = &s_abort;
    int n_done = 0;   // rows b whose stage loads were issued: [0, n_done)

    if (warp == T::W_PROD) {
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
        // a row's mask words are read before its stage is free, so that their global loads
        // overlap the wait
        uint32_t w[4];
        if (nb > 0) mask_words(a, bstart, j0, w);
        for (; n < nb; ++n) {
            const int st = n % NS, b = bstart + n;
            if (n >= NS) ok = mbar_wait(b_empty(st), ((n / NS) - 1) & 1, abort_flag, SITE_DB_PROD);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
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
            if (n + 1 < nb) mask_words(a, b + 1, j0, w);
        }
    } else if (warp == T::W_MMA) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t SBO = 8 * T::ROWB;
            constexpr uint32_t id_s = idesc_bf16(128, 128, false, false);
            bool ok = true;
            for (int n = 0; n < nb && ok; ++n) {
                const int st = n % NS, x = n & 1;
                ok = mbar_wait_all(abort_flag, b_full(st), (n / NS) & 1, true, SITE_DB_MMA,
                                   b_sd_free(x), ((n >> 1) - 1) & 1, n >= 2, SITE_DB_MMA);
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
        // warpgroup g: keys 48 g .. 48 g + 47 (g < 2) or 96 .. 127 (g = 2) of its 32 rows
        const int g = warp >> 2;
        const int row = (warp & 3) * 32 + lane;
        const uint32_t lane_off = ((uint32_t)((warp & 3) * 32)) << 16;
        const float sl2e = a.scale * kLog2eB;
        const uint32_t bias_row = sbase + T::OFF_BIAS + row * 128;
        bool ok = mbar_wait(b_bias, 0, abort_flag, SITE_DB_EW);
        ok = __all_sync(0xffffffffu, ok);
        auto run = [&](auto k0c, auto nkc) {
            constexpr int K0 = decltype(k0c)::value, NK = decltype(nkc)::value;
            float2 acc[NK / 2];   // sum over this split's rows b of dS, keys K0 + 2 c and K0 + 2 c + 1
#pragma unroll
            for (int c = 0; c < NK / 2; ++c) acc[c] = make_float2(0.f, 0.f);
            for (int n = 0; n < nb && ok; ++n) {
                const int st = n % NS, x = n & 1;
                ok = mbar_wait_all(abort_flag, b_sd_full(x), (n >> 1) & 1, true, SITE_DB_EW,
                                   b_full(st), (n / NS) & 1, true, SITE_DB_EW);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                tc_fence_after();
                const uint8_t *s0 = gbase + T::OFF_STAGE + st * T::STAGE_BYTES;
                const float2 rs = reinterpret_cast<const float2 *>(s0 + 4 * T::TILE_BYTES)[row];
                const uint32_t *mw = reinterpret_cast<const uint32_t *>(gbase + T::OFF_MASK) + st * 8;
                // every key of the range attended
                bool full = true;
#pragma unroll
                for (int w = K0 >> 5; w <= (K0 + NK - 1) >> 5; ++w) {
                    const uint32_t bits = key_bits(K0, NK, w);
                    full = full && (mw[w] & bits) == bits;
                }
                p_ds_keys<K0, NK>(tbase + x * 256 + lane_off, tbase + x * 256 + 128 + lane_off, bias_row, row,
                                  a.has_bias != 0, mw, full, sl2e, rs.x, rs.y,
                                  [&](int c, float2 p, float2 dpd) { acc[c >> 1] = ffma2(p, dpd, acc[c >> 1]); },
                                  []() {});
                tc_fence_before();
                mbar_arrive(b_sd_free(x));
                mbar_arrive(b_empty(st));
            }
            if (ok) {
                // this split's partial tile: [split][h][tile][128][128]
                float *dst = a.dbias_part +
                             ((((long long)sp * a.H + h) * a.ntiles + bt) * 128 + row) * 128 + K0;
#pragma unroll
                for (int c = 0; c < NK / 2; c += 2)
                    *reinterpret_cast<float4 *>(dst + 2 * c) = make_float4(acc[c].x, acc[c].y, acc[c + 1].x, acc[c + 1].y);
                __threadfence();   // this thread's partial row, before the tile counter moves
            }
        };
        if (g == 0) run(std::integral_constant<int, 0>(), std::integral_constant<int, 48>());
        else if (g == 1) run(std::integral_constant<int, 48>(), std::integral_constant<int, 48>());
        else run(std::integral_constant<int, 96>(), std::integral_constant<int, 32>());
    }

    tc_fence_before();
    __syncthreads();
    if (*abort_flag) {
        if (warp == T::W_PROD && lane == 0) {
            mbar_wait_drain(b_bias, 0);
            for (int nn = max(0, n_done - NS); nn < n_done; ++nn) mbar_wait_drain(b_full(nn % NS), (nn / NS) & 1);
        }
        if (warp == T::W_MMA && lane == 0) {
            umma_commit(b_drain);
            mbar_wait_drain(b_drain, 0);
        }
        tc_fence_before();
        __syncthreads();
    }
    if (warp == T::W_MMA) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tbase, 512);
    }
    if (*abort_flag) return;
    // Every partial of this CTA is written and fenced.  The tile's last CTA to get here sums
    // the partials of all splits, in split order, into dbias.
    __shared__ int s_last;
    if (threadIdx.x == 0) {
        __threadfence();
        const int tile = (h * a.nI + it) * a.nJ + jt;
        s_last = atomicAdd(a.tile_count + tile, 1) == a.splits - 1;
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    // Only the tile's valid part (rows i < Nq, four-key groups starting below Nk) is summed,
    // four positions per thread at a time.  Every position adds its partials in split order,
    // starting from zero; the loads of four splits of the four positions are all issued
    // before their additions, so their latencies overlap.
    const long long plane = (long long)a.H * a.ntiles * 128 * 128;
    const float *part = a.dbias_part + ((long long)h * a.ntiles + bt) * 128 * 128;
    const int groups = (min(128, a.Nk - j0) + 3) >> 2;
    const int nv = min(128, a.Nq - i0) * groups;
    for (int v0 = threadIdx.x; v0 < nv; v0 += 4 * blockDim.x) {
        int off[4];   // row * 128 + column within the tile, or -1
        float4 sum[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int v = v0 + u * blockDim.x;
            off[u] = v < nv ? (v / groups) * 128 + (v % groups) * 4 : -1;
            sum[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        int q = 0;
        for (; q + 4 <= a.splits; q += 4) {
            float4 x[4][4];
#pragma unroll
            for (int s = 0; s < 4; ++s)
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    x[s][u] = off[u] >= 0 ? __ldcg(reinterpret_cast<const float4 *>(part + (q + s) * plane + off[u]))
                                          : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int s = 0; s < 4; ++s)
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    sum[u].x += x[s][u].x;
                    sum[u].y += x[s][u].y;
                    sum[u].z += x[s][u].z;
                    sum[u].w += x[s][u].w;
                }
        }
        for (; q < a.splits; ++q) {
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                if (off[u] < 0) continue;
                const float4 x = __ldcg(reinterpret_cast<const float4 *>(part + q * plane + off[u]));
                sum[u].x += x.x;
                sum[u].y += x.y;
                sum[u].z += x.z;
                sum[u].w += x.w;
            }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            if (off[u] < 0) continue;
            const int i = i0 + (off[u] >> 7), j = j0 + (off[u] & 127);
            float *dst = a.dbias + ((long long)h * a.Nq + i) * a.Nk + j;
            dst[0] = sum[u].x;
            if (j + 1 < a.Nk) dst[1] = sum[u].y;
            if (j + 2 < a.Nk) dst[2] = sum[u].z;
            if (j + 3 < a.Nk) dst[3] = sum[u].w;
        }
    }
}

// out[i] = ordered sum over the parts of parts[p][i] (part 0 first).  With `vec` (n a
// multiple of 4, so that every part starts 16-byte aligned) four elements per thread and
// load, otherwise one.
__global__ void __launch_bounds__(256) pba_dbias_sum_kernel(const float *parts, int n_parts, long long n,
                                                            float *out, int vec) {
    const long long stride = (long long)gridDim.x * blockDim.x;
    if (vec) {
        const long long n4 = n >> 2;
        for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n4; e += stride) {
            float4 acc = __ldcs(reinterpret_cast<const float4 *>(parts) + e);
            for (int p = 1; p < n_parts; ++p) {
                const float4 x = __ldcs(reinterpret_cast<const float4 *>(parts + p * n) + e);
                acc.x += x.x;
                acc.y += x.y;
                acc.z += x.z;
                acc.w += x.w;
            }
            reinterpret_cast<float4 *>(out)[e] = acc;
        }
        return;
    }
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += stride) {
        float acc = parts[i];
        for (int p = 1; p < n_parts; ++p) acc += parts[p * n + i];
        out[i] = acc;
    }
}

// dq = bf16(scale * dqacc), eight channels per thread.
__global__ void __launch_bounds__(256) pba_dq_convert_kernel(const BwdArgs a) {
    // element groups e = (row r, c8) with r = (b, i, h) < 2^31 rows (checked on the host):
    // 32-bit index arithmetic
    const int c8n = a.C / 8;
    const int nrows = a.B * a.Nq * a.H;
    const long long n = (long long)nrows * c8n;
    const float s = a.scale;
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n;
         e += (long long)gridDim.x * blockDim.x) {
        const int r = (int)(e / c8n);
        const int c8 = (int)(e - (long long)r * c8n);
        const int h = r % a.H;
        const int bi = r / a.H;
        const int i = bi % a.Nq;
        const int b = bi / a.Nq;
        const float4 *src = reinterpret_cast<const float4 *>(a.dqacc + (long long)r * a.C + c8 * 8);
        const float4 x0 = __ldcs(src), x1 = __ldcs(src + 1);
        __nv_bfloat16 *dst = a.dq + b * a.sq0 + (long long)i * a.sq1 + h * a.sq2 + c8 * 8;
        *reinterpret_cast<uint4 *>(dst) =
            make_uint4(pack_bf16x2(x0.x * s, x0.y * s), pack_bf16x2(x0.z * s, x0.w * s),
                       pack_bf16x2(x1.x * s, x1.y * s), pack_bf16x2(x1.z * s, x1.w * s));
    }
}

}  // namespace pba
