// libpba host side: argument validation, TMA tensor maps, launches, the C ABI of pba.h.
//
// The library allocates nothing per call.  The CUDA driver's tensor-map encoder is
// fetched through the runtime's entry-point query on first use, so the shared library
// itself loads (and its symbols can be inspected) on a machine without a GPU.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <climits>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/pba.h"
#include "pba_bwd.cuh"
#include "pba_fwd.cuh"
#include "pba_pairbias.cuh"
#include "pba_pwa.cuh"

namespace {

thread_local std::string g_last_error;
int g_debug_skip_step = -1;   // test hook, see pba_debug_skip_load

pba_status fail(pba_status s, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return s;
}

pba_status cuda_fail(cudaError_t e, const char *what) {
    return fail(PBA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// ---------------------------------------------------------------------------- profiling
enum KernelId { K_FWD = 0, K_BWD_PRE, K_BWD_MAIN, K_DBIAS, K_DQ_CONVERT, K_ZERO_ROWS,
                K_PWA_WEIGHTS, K_PWA_FWD, K_PWA_PRE, K_PWA_DV, K_PWA_DW, K_PWA_DBIAS,
                K_PB_FWD, K_PB_BWD, K_PB_REDUCE, K_PB_PARAM, K_DBIAS_ZERO, K_DBIAS_SUM, K_PB_BWD_TC,
                K_COUNT };
const char *const kKernelNames[K_COUNT] = {"pba_fwd_kernel", "pba_bwd_pre_kernel", "pba_bwd_main_kernel",
                                           "pba_dbias_kernel",
                                           "pba_dq_convert_kernel", "zero_rows_kernel",
                                           "pba_pwa_weights_kernel", "pba_pwa_gemm_kernel (out)",
                                           "pba_pwa_pre_kernel", "pba_pwa_gemm_kernel (dv)",
                                           "pba_pwa_dw_kernel", "pba_pwa_dbias_kernel",
                                           "pba_pair_bias_fwd_kernel", "pba_pair_bias_bwd_kernel",
                                           "pba_pair_bias_reduce_kernel", "pba_pair_bias_param_kernel",
                                           "pba_dbias_zero_kernel", "pba_dbias_sum_kernel",
                                           "pba_pair_bias_bwd_tc_kernel"};
struct ProfRec {
    int kid;
    cudaEvent_t a, b;
};
std::mutex g_prof_mu;
bool g_prof_on = false;
std::vector<ProfRec> g_prof_recs;
std::vector<cudaEvent_t> g_prof_pool;

cudaEvent_t prof_event() {
    if (!g_prof_pool.empty()) {
        cudaEvent_t e = g_prof_pool.back();
        g_prof_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
}

// Brackets one kernel launch with events when profiling is on.
struct ProfScope {
    int kid;
    cudaStream_t s;
    cudaEvent_t a = nullptr;
    ProfScope(int k, cudaStream_t st) : kid(k), s(st) {
        std::lock_guard<std::mutex> g(g_prof_mu);
        if (!g_prof_on) return;
        a = prof_event();
        if (a) cudaEventRecord(a, s);
    }
    ~ProfScope() {
        if (!a) return;
        std::lock_guard<std::mutex> g(g_prof_mu);
        cudaEvent_t b = prof_event();
        if (!b) return;
        cudaEventRecord(b, s);
        g_prof_recs.push_back({kid, a, b});
    }
};

// ---------------------------------------------------------------------------- tensor maps
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;
cudaError_t g_encode_err = cudaSuccess;

pba_status get_encoder() {
    std::call_once(g_encode_once, [] {
        cudaDriverEntryPointQueryResult q;
        void *fn = nullptr;
        g_encode_err = cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000,
                                                        cudaEnableDefault, &q);
        if (g_encode_err == cudaSuccess && q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    if (!g_encode) return fail(PBA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable (%s)",
                               cudaGetErrorString(g_encode_err));
    return PBA_OK;
}

CUtensorMapSwizzle swizzle_for_row_bytes(int rowb) {
    return rowb == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                       : (rowb == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
}

// A [B, N, H, C] bf16 tensor (C stride 1) as a 4-D map (C, H, N, B), box (CP, 1, 128, 1).
pba_status map_bnhc(CUtensorMap *m, const void *base, int B, int N, int H, int C,
                    const int64_t s[3], int CP, const char *name, int rows = 128) {
    cuuint64_t dims[4] = {(cuuint64_t)C, (cuuint64_t)H, (cuuint64_t)(N > 0 ? N : 1),
                          (cuuint64_t)(B > 0 ? B : 1)};
    // a dimension of extent 1 is never stepped along: give it a harmless legal stride
    cuuint64_t strides[3] = {(cuuint64_t)(H > 1 ? s[2] * 2 : 16),
                             (cuuint64_t)(N > 1 ? s[1] * 2 : 16),
                             (cuuint64_t)(B > 1 ? s[0] * 2 : 16)};
    cuuint32_t box[4] = {(cuuint32_t)CP, 1, (cuuint32_t)rows, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          swizzle_for_row_bytes(CP * 2), CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(PBA_ERR_CUDA, "tensor map for %s failed (CUresult %d)", name, (int)r);
    return PBA_OK;
}

// The dense fp32 [B, Nq, H, C] dQ accumulator as a 4-D map (C, H, Nq, B), box (32, 1, 128, 1),
// 128-byte swizzle (rows of 32 fp32), for the backward's TMA reductions.
pba_status map_dqacc(CUtensorMap *m, void *base, int B, int Nq, int H, int C) {
    cuuint64_t dims[4] = {(cuuint64_t)C, (cuuint64_t)H, (cuuint64_t)(Nq > 0 ? Nq : 1), (cuuint64_t)(B > 0 ? B : 1)};
    cuuint64_t strides[3] = {(cuuint64_t)C * 4, (cuuint64_t)H * C * 4, (cuuint64_t)Nq * H * C * 4};
    cuuint32_t box[4] = {32, 1, 128, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, base, dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(PBA_ERR_CUDA, "tensor map for the dQ accumulator failed (CUresult %d)", (int)r);
    return PBA_OK;
}

// The [H, Nq, Nk] bias as a 3-D map (Nk, Nq, H), box (64, 128, 1), 128-byte swizzle.
pba_status map_bias(CUtensorMap *m, const void *base, int H, int Nq, int Nk, const int64_t s[2]) {
    cuuint64_t dims[3] = {(cuuint64_t)(Nk > 0 ? Nk : 1), (cuuint64_t)(Nq > 0 ? Nq : 1), (cuuint64_t)H};
    cuuint64_t strides[2] = {(cuuint64_t)(Nq > 1 ? s[1] * 2 : 16), (cuuint64_t)(H > 1 ? s[0] * 2 : 16)};
    cuuint32_t box[3] = {64, 128, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(PBA_ERR_CUDA, "tensor map for bias failed (CUresult %d)", (int)r);
    return PBA_OK;
}

// ---------------------------------------------------------------------------- validation
bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

pba_status check_strides(const int64_t s[3], int B, int N, int H, const char *name) {
    const int ext[3] = {B, N, H};
    for (int d = 0; d < 3; ++d) {
        if (ext[d] <= 1) continue;
        if (s[d] <= 0 || (s[d] % 8) != 0)
            return fail(PBA_ERR_INVALID_ARG,
                        "%s: stride of dim %d is %lld elements; must be a positive multiple of 8",
                        name, d, (long long)s[d]);
        if (s[d] * 2 >= (int64_t(1) << 40))
            return fail(PBA_ERR_UNSUPPORTED, "%s: stride of dim %d too large", name, d);
    }
    return PBA_OK;
}

pba_status check_dims(const pba_dims *d) {
    if (!d) return fail(PBA_ERR_INVALID_ARG, "dims is NULL");
    if (d->B < 0 || d->H < 0 || d->Nq < 0 || d->Nk < 0 || d->C < 0)
        return fail(PBA_ERR_INVALID_ARG, "negative size");
    if (d->C < 8 || d->C > 64 || (d->C % 8) != 0)
        return fail(PBA_ERR_UNSUPPORTED, "C=%d: head dim must be a multiple of 8 in [8, 64]", d->C);
    if (d->H < 1) return fail(PBA_ERR_INVALID_ARG, "H must be >= 1");
    if (d->Nq > (1 << 24) || d->Nk > (1 << 24) || d->B > (1 << 24) || d->H > 4096)
        return fail(PBA_ERR_UNSUPPORTED, "sizes too large");
    if (!(d->scale >= 0.f) || !std::isfinite(d->scale))
        return fail(PBA_ERR_INVALID_ARG, "scale must be finite and >= 0 (0 = 1/sqrt(C))");
    return PBA_OK;
}

pba_status check_layouts(const pba_dims *d) {
    pba_status st;
    if ((st = check_strides(d->sq, d->B, d->Nq, d->H, "q")) != PBA_OK) return st;
    if ((st = check_strides(d->sk, d->B, d->Nk, d->H, "k")) != PBA_OK) return st;
    if ((st = check_strides(d->sv, d->B, d->Nk, d->H, "v")) != PBA_OK) return st;
    if ((st = check_strides(d->so, d->B, d->Nq, d->H, "out")) != PBA_OK) return st;
    return PBA_OK;
}

pba_status check_bias(const pba_dims *d) {
    if (d->H > 1 && (d->sbias[0] <= 0 || d->sbias[0] % 8))
        return fail(PBA_ERR_INVALID_ARG, "bias: H stride must be a positive multiple of 8");
    if (d->Nq > 1 && (d->sbias[1] <= 0 || d->sbias[1] % 8))
        return fail(PBA_ERR_INVALID_ARG, "bias: Nq stride must be a positive multiple of 8");
    return PBA_OK;
}

int padded_c(int C) { return C <= 16 ? 16 : (C <= 32 ? 32 : 64); }

float eff_scale(const pba_dims *d) {
    return d->scale > 0.f ? d->scale : 1.0f / std::sqrt((float)d->C);
}

// Local attention: query tile t visits key tiles [t - window, t + window]; every query tile
// must keep at least one key tile and every key tile at least one query tile (window < 0:
// dense, always fine).
pba_status check_window(const pba_dims *d, int window) {
    if (window < 0) return PBA_OK;
    const long long nI = (d->Nq + 127) / 128, nJ = (d->Nk + 127) / 128;
    if (d->Nq > 0 && d->Nk > 0 && (nI > nJ + window || nJ > nI + window))
        return fail(PBA_ERR_UNSUPPORTED, "window %d leaves a query or key tile with no partner "
                                         "(%lld query tiles, %lld key tiles)", window, nI, nJ);
    return PBA_OK;
}

template <typename K>
pba_status set_smem(K kernel, int bytes) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
    return PBA_OK;
}

long long num_sms();

template <int CP>
pba_status launch_fwd(const pba_bf16 *q, const pba_bf16 *k, const pba_bf16 *v,
                      const pba_bf16 *bias, const uint8_t *mask, const pba_bf16 *gate,
                      pba_bf16 *out, float *lse, const pba_dims *d, int win, cudaStream_t stream) {
    using T = pba::FwdTraits<CP>;
    CUtensorMap tq, tk, tv, tb;
    pba_status st;
    if ((st = map_bnhc(&tq, q, d->B, d->Nq, d->H, d->C, d->sq, CP, "q")) != PBA_OK) return st;
    if ((st = map_bnhc(&tk, k, d->B, d->Nk, d->H, d->C, d->sk, CP, "k")) != PBA_OK) return st;
    if ((st = map_bnhc(&tv, v, d->B, d->Nk, d->H, d->C, d->sv, CP, "v")) != PBA_OK) return st;
    if (bias) {
        if ((st = map_bias(&tb, bias, d->H, d->Nq, d->Nk, d->sbias)) != PBA_OK) return st;
    } else {
        std::memset(&tb, 0, sizeof(tb));
    }
    pba::FwdArgs a;
    a.B = d->B; a.H = d->H; a.Nq = d->Nq; a.Nk = d->Nk; a.C = d->C;
    a.nI = (d->Nq + 127) / 128;
    a.nJ = (d->Nk + 127) / 128;
    a.nChunks = (d->B + T::BC - 1) / T::BC;
    const long long tiles = (long long)a.nI * d->H;
    a.scale = eff_scale(d);
    a.has_bias = bias != nullptr;
    a.mask = mask;
    a.smask_b = d->smask_b;
    a.mask_shared = (mask == nullptr || d->smask_b == 0 || d->B == 1) ? 1 : 0;
    a.gate = reinterpret_cast<const __nv_bfloat16 *>(gate);
    a.sg0 = d->sg[0]; a.sg1 = d->sg[1]; a.sg2 = d->sg[2];
    a.out = reinterpret_cast<__nv_bfloat16 *>(out);
    a.so0 = d->so[0]; a.so1 = d->so[1]; a.so2 = d->so[2];
    a.lse = lse;
    a.skip_step = g_debug_skip_step;
    a.win = win;
    if ((st = set_smem(pba::pba_fwd_kernel<CP>, T::SMEM_BYTES)) != PBA_OK) return st;
    // two CTAs per SM need (almost) all of the unified L1 / shared memory as shared memory
    cudaError_t ce = cudaFuncSetAttribute(pba::pba_fwd_kernel<CP>,
                                          cudaFuncAttributePreferredSharedMemoryCarveout,
                                          cudaSharedmemCarveoutMaxShared);
    if (ce != cudaSuccess) return cuda_fail(ce, "cudaFuncSetAttribute (carveout)");
    const long long items = tiles * a.nChunks;
    if (items > INT_MAX) return fail(PBA_ERR_UNSUPPORTED, "too many forward work items");
    a.items = (int)items;
    // persistent: at most two CTAs per SM (their shared memory allows no more)
    const long long grid = std::min<long long>(items, 2LL * num_sms());
    {
        ProfScope ps(K_FWD, stream);
        pba::pba_fwd_kernel<CP><<<(unsigned)grid, T::THREADS, T::SMEM_BYTES, stream>>>(tq, tk, tv, tb, a);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "pba_fwd_kernel launch");
    return PBA_OK;
}

// ---------------------------------------------------------------------------- backward
constexpr long long kSmCount = 148;   // SMs of a B200

struct BwdPlan {
    int nI, nJ, NqPad, NkPad, splits, rows_per_split, ntiles;
    size_t off_rs, off_doa, off_dq, off_cnt, off_part, total;
};

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// the split count that minimises waves x (rows + 3) for `tiles` dbias tiles, at most
// `max_part` split partial tiles (splits x tiles)
void choose_splits(const pba_dims *d, long long tiles, long long max_part, int *splits, int *rows_per_split);

BwdPlan plan_bwd(const pba_dims *d, int win = -1) {
    BwdPlan p;
    p.nI = (d->Nq + 127) / 128;
    p.nJ = (d->Nk + 127) / 128;
    p.NqPad = p.nI * 128;
    p.NkPad = p.nJ * 128;
    p.ntiles = p.nI * p.nJ;
    if (win >= 0) {   // local attention: the (query tile, key tile) pairs within the window
        long long n = 0;
        for (int i = 0; i < p.nI; ++i) n += std::min(p.nJ, i + win + 1) - std::max(0, i - win);
        p.ntiles = (int)n;
    }
    // splits of the broadcast rows for the dbias kernel: a fixed function of the sizes,
    // so the reduction order (and every bit of dbias) depends on nothing else.  A CTA
    // handles one (head, query tile, key tile, split); its time grows with the rows of its
    // split plus a fixed cost (bias tile, pipeline fill, the partial tile's store) of about
    // three rows, so pick the split count that minimises waves x (rows + 3) on 148 SMs.
    // The workspace is sized for the dense problem, so a window's plan holds at most as many
    // partial tiles as the dense plan.
    int dense_splits, dense_rows;
    choose_splits(d, (long long)d->H * p.nI * p.nJ, -1, &dense_splits, &dense_rows);
    if (win < 0) {
        p.splits = dense_splits;
        p.rows_per_split = dense_rows;
    } else {
        choose_splits(d, (long long)d->H * p.ntiles, (long long)dense_splits * p.nI * p.nJ * d->H,
                      &p.splits, &p.rows_per_split);
    }
    const size_t rows = (size_t)d->B * d->H * p.NqPad;
    const size_t elems = (size_t)d->B * d->Nq * d->H * d->C;
    p.off_rs = 0;
    p.off_doa = align256(p.off_rs + rows * sizeof(float2));
    p.off_dq = align256(p.off_doa + elems * 2);
    // per-tile counters of the dbias kernel (cleared by the pre kernel)
    p.off_cnt = align256(p.off_dq + elems * 4);
    p.off_part = align256(p.off_cnt + (size_t)d->H * p.nI * p.nJ * sizeof(int));
    p.total = align256(p.off_part + (size_t)p.splits * d->H * p.ntiles * 128 * 128 * 4);
    return p;
}

void choose_splits(const pba_dims *d, long long tiles, long long max_part, int *splits, int *rows_per_split) {
    const long long maxs = d->B < 64 ? (d->B > 0 ? d->B : 1) : 64;
    long long best_cost = -1;
    *splits = 1;
    *rows_per_split = d->B > 0 ? d->B : 1;
    for (long long sp = 1; sp <= maxs; ++sp) {
        const long long rows = d->B > 0 ? (d->B + sp - 1) / sp : 1;
        const long long actual = d->B > 0 ? (d->B + rows - 1) / rows : 1;
        if (max_part >= 0 && actual * tiles > max_part) break;
        const long long waves = (tiles * actual + kSmCount - 1) / kSmCount;
        const long long cost = waves * (rows + 3);
        if (best_cost < 0 || cost < best_cost) {
            best_cost = cost;
            *splits = (int)actual;
            *rows_per_split = (int)rows;
        }
    }
}

__global__ void zero_rows_kernel(__nv_bfloat16 *dk, __nv_bfloat16 *dv, pba::BwdArgs a) {
    const int c8n = a.C / 8;
    const long long n = (long long)a.B * a.Nk * a.H * c8n;
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n;
         e += (long long)gridDim.x * blockDim.x) {
        const int c8 = (int)(e % c8n);
        const long long r = e / c8n;
        const int h = (int)(r % a.H);
        const long long bj = r / a.H;
        const int j = (int)(bj % a.Nk);
        const int b = (int)(bj / a.Nk);
        *reinterpret_cast<uint4 *>(dk + b * a.sk0 + (long long)j * a.sk1 + h * a.sk2 + c8 * 8) = make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4 *>(dv + b * a.sv0 + (long long)j * a.sv1 + h * a.sv2 + c8 * 8) = make_uint4(0, 0, 0, 0);
    }
}

// SMs of the current device (one CTA each for the persistent kernels)
long long num_sms() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        return kSmCount;
    return n;
}

unsigned grid_for(long long n, int threads) {
    long long g = (n + threads - 1) / threads;
    if (g > 148LL * 32) g = 148LL * 32;
    return (unsigned)(g > 0 ? g : 1);
}

pba_status launch_zero_rows(pba_bf16 *dk, pba_bf16 *dv, const pba_dims *d, cudaStream_t s) {
    if (!aligned16(dk) || !aligned16(dv)) return fail(PBA_ERR_INVALID_ARG, "dk, dv must be 16-byte aligned");
    pba::BwdArgs a;
    std::memset(&a, 0, sizeof(a));
    a.B = d->B; a.H = d->H; a.Nk = d->Nk; a.C = d->C;
    a.sk0 = d->sk[0]; a.sk1 = d->sk[1]; a.sk2 = d->sk[2];
    a.sv0 = d->sv[0]; a.sv1 = d->sv[1]; a.sv2 = d->sv[2];
    const long long n = (long long)d->B * d->Nk * d->H * (d->C / 8);
    {
        ProfScope ps(K_ZERO_ROWS, s);
        zero_rows_kernel<<<grid_for(n, 256), 256, 0, s>>>(reinterpret_cast<__nv_bfloat16 *>(dk),
                                                           reinterpret_cast<__nv_bfloat16 *>(dv), a);
    }
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? PBA_OK : cuda_fail(e, "zero_rows_kernel launch");
}

// ---------------------------------------------------------------------------- side stream
// The dbias kernel needs only the pre kernel's row statistics and the dq conversion only the
// dq/dk/dv kernel, and the two share an SM well (the dbias kernel is bound by the exponential
// unit and instruction issue, the conversion by DRAM).  So once the dq/dk/dv kernel is done the
// dbias kernel runs on a second stream of higher priority (its CTAs are placed first) while
// the conversion runs on the caller's stream, which then waits for the second stream.  The
// stream and its two events are created once per CUDA context (keyed by the context's unique
// id, outside any stream capture) and shared by every call in that context under g_side_mu,
// which also keeps each call's event record and the wait on it together.  Inside a capture the
// fork and the join become graph dependencies.
struct SideStream {
    unsigned long long ctx;
    cudaStream_t s;
    cudaEvent_t fork, join;
};
std::mutex g_side_mu;
std::vector<SideStream> g_side;
// The side stream of the current context (created on first use; never while `s` is being
// captured); false if it does not exist and cannot be made, and the caller then stays on `s`.
// The caller holds g_side_mu.
bool side_stream(cudaStream_t s, SideStream *out);

template <int CP>
pba_status launch_bwd(const pba_bf16 *q, const pba_bf16 *k, const pba_bf16 *v,
                      const pba_bf16 *bias, const uint8_t *mask, const pba_bf16 *gate,
                      const pba_bf16 *out, const float *lse, const pba_bf16 *dout,
                      pba_bf16 *dq, pba_bf16 *dk, pba_bf16 *dv, float *dbias, pba_bf16 *dgate,
                      void *ws, const BwdPlan &pl, const pba_dims *d, int win, cudaStream_t s) {
    using MT = pba::BwdTraits<CP>;
    using DT = pba::DbTraits<CP>;
    uint8_t *w = static_cast<uint8_t *>(ws);
    pba::BwdArgs a;
    std::memset(&a, 0, sizeof(a));
    a.B = d->B; a.H = d->H; a.Nq = d->Nq; a.Nk = d->Nk; a.C = d->C;
    a.nI = pl.nI; a.nJ = pl.nJ; a.NqPad = pl.NqPad; a.NkPad = pl.NkPad;
    a.splits = pl.splits; a.rows_per_split = pl.rows_per_split;
    a.win = win;
    a.ntiles = pl.ntiles;
    a.scale = eff_scale(d);
    a.has_bias = bias != nullptr;
    a.has_gate = gate != nullptr;
    a.mask = mask;
    a.smask_b = d->smask_b;
    a.gate = reinterpret_cast<const __nv_bfloat16 *>(gate);
    a.out = reinterpret_cast<const __nv_bfloat16 *>(out);
    a.dout = reinterpret_cast<const __nv_bfloat16 *>(dout);
    a.sg0 = d->sg[0]; a.sg1 = d->sg[1]; a.sg2 = d->sg[2];
    a.so0 = d->so[0]; a.so1 = d->so[1]; a.so2 = d->so[2];
    a.lse = lse;
    a.dq = reinterpret_cast<__nv_bfloat16 *>(dq);
    a.dk = reinterpret_cast<__nv_bfloat16 *>(dk);
    a.dv = reinterpret_cast<__nv_bfloat16 *>(dv);
    a.dgate = reinterpret_cast<__nv_bfloat16 *>(dgate);
    a.sq0 = d->sq[0]; a.sq1 = d->sq[1]; a.sq2 = d->sq[2];
    a.sk0 = d->sk[0]; a.sk1 = d->sk[1]; a.sk2 = d->sk[2];
    a.sv0 = d->sv[0]; a.sv1 = d->sv[1]; a.sv2 = d->sv[2];
    a.dbias = dbias;
    a.rowstats = reinterpret_cast<float2 *>(w + pl.off_rs);
    a.doa = reinterpret_cast<__nv_bfloat16 *>(w + pl.off_doa);
    a.dqacc = reinterpret_cast<float *>(w + pl.off_dq);
    a.dbias_part = reinterpret_cast<float *>(w + pl.off_part);
    a.tile_count = reinterpret_cast<int *>(w + pl.off_cnt);

    pba_status st;
    CUtensorMap tq, tk, tv, tdo, tb, tdq;
    if ((st = map_bnhc(&tq, q, d->B, d->Nq, d->H, d->C, d->sq, CP, "q")) != PBA_OK) return st;
    if ((st = map_bnhc(&tk, k, d->B, d->Nk, d->H, d->C, d->sk, CP, "k")) != PBA_OK) return st;
    if ((st = map_bnhc(&tv, v, d->B, d->Nk, d->H, d->C, d->sv, CP, "v")) != PBA_OK) return st;
    if (gate) {
        const int64_t sd[3] = {(int64_t)d->Nq * d->H * d->C, (int64_t)d->H * d->C, d->C};
        if ((st = map_bnhc(&tdo, a.doa, d->B, d->Nq, d->H, d->C, sd, CP, "dOa")) != PBA_OK) return st;
    } else {
        if ((st = map_bnhc(&tdo, dout, d->B, d->Nq, d->H, d->C, d->so, CP, "dout")) != PBA_OK) return st;
    }
    if (bias) {
        if ((st = map_bias(&tb, bias, d->H, d->Nq, d->Nk, d->sbias)) != PBA_OK) return st;
    } else {
        std::memset(&tb, 0, sizeof(tb));
    }
    if (MT::DQ_TMA) {
        if ((st = map_dqacc(&tdq, a.dqacc, d->B, d->Nq, d->H, d->C)) != PBA_OK) return st;
    } else {
        std::memset(&tdq, 0, sizeof(tdq));
    }
    cudaError_t e;
    const size_t elems = (size_t)d->B * d->Nq * d->H * d->C;
    // (the pre kernel clears the dQ accumulator and the dbias tile counters)
    const long long pre_rows = (long long)d->B * pl.NqPad * d->H;
    if (pre_rows >= (1LL << 31)) return fail(PBA_ERR_UNSUPPORTED, "B * Nq * H must be below 2^31");
    {
        ProfScope ps(K_BWD_PRE, s);
        pba::pba_bwd_pre_kernel<CP><<<grid_for(pre_rows * (CP / 8), 256), 256, 0, s>>>(a);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "pba_bwd_pre_kernel launch");
    if (pl.nJ > 0) {
        if ((st = set_smem(pba::pba_bwd_main_kernel<CP>, MT::SMEM_BYTES)) != PBA_OK) return st;
        // persistent: one CTA per SM (at most one per item)
        const long long items = (long long)d->B * d->H * pl.nJ;
        if (items >= (1LL << 31)) return fail(PBA_ERR_UNSUPPORTED, "B * H * key tiles must be below 2^31");
        const long long grid = items < num_sms() ? items : num_sms();
        {
            ProfScope ps(K_BWD_MAIN, s);
            pba::pba_bwd_main_kernel<CP><<<(unsigned)grid, 512, MT::SMEM_BYTES, s>>>(tq, tk, tv, tdo, tb, tdq, a);
        }
        if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "pba_bwd_main_kernel launch");
        if (dbias) {
            if ((st = set_smem(pba::pba_dbias_kernel<CP>, DT::SMEM_BYTES)) != PBA_OK) return st;
            std::lock_guard<std::mutex> g(g_side_mu);
            SideStream side;
            const bool fork = side_stream(s, &side);
            cudaStream_t ds = s;   // the dbias kernels' stream
            if (fork) {
                if ((e = cudaEventRecord(side.fork, s)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
                if ((e = cudaStreamWaitEvent(side.s, side.fork, 0)) != cudaSuccess) return cuda_fail(e, "cudaStreamWaitEvent");
                ds = side.s;
            }
            const long long g2 = (long long)pl.splits * d->H * pl.ntiles;
            if (win >= 0) {
                ProfScope ps(K_DBIAS_ZERO, ds);
                const long long rows = (long long)d->H * d->Nq;
                pba::pba_dbias_zero_kernel<<<(unsigned)std::min<long long>(rows, 8 * kSmCount), 256, 0, ds>>>(a);
            }
            if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "pba_dbias_zero_kernel launch");
            {
                ProfScope ps(K_DBIAS, ds);
                pba::pba_dbias_kernel<CP><<<(unsigned)g2, DT::THREADS, DT::SMEM_BYTES, ds>>>(tq, tk, tv, tdo, tb, a);
            }
            if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "pba_dbias_kernel launch");
            // (the last CTA of every tile sums the split partials in split order)
            {
                ProfScope ps(K_DQ_CONVERT, s);
                pba::pba_dq_convert_kernel<<<grid_for((long long)elems / 8, 256), 256, 0, s>>>(a);
            }
            if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "pba_dq_convert_kernel launch");
            if (fork) {
                if ((e = cudaEventRecord(side.join, side.s)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
                if ((e = cudaStreamWaitEvent(s, side.join, 0)) != cudaSuccess) return cuda_fail(e, "cudaStreamWaitEvent");
            }
            return PBA_OK;
        }
    }
    {
        ProfScope ps(K_DQ_CONVERT, s);
        pba::pba_dq_convert_kernel<<<grid_for((long long)elems / 8, 256), 256, 0, s>>>(a);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "pba_dq_convert_kernel launch");
    return PBA_OK;
}

// ---------------------------------------------------------------------------- no-alloc
// Scratch of pba_bwd_noalloc: a file-scope device array, so callers that cannot allocate
// can still run the backward pass.  In host code its name is only a stand-in; the
// device address comes from cudaGetSymbolAddress.  A __device__ symbol's address belongs
// to the CUDA context that loaded the module, so it is looked up once per context (the
// first call in a context, with that context's device current) and cached under the
// context's unique id, which a re-created context (after cudaDeviceReset, or another
// context on the same device) does not share.
constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;
__device__ __align__(256) unsigned char g_pba_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
std::vector<std::pair<unsigned long long, void *>> g_noalloc_addr;   // (context id, address)

typedef CUresult (*PFN_ctxGetCurrent)(CUcontext *);
typedef CUresult (*PFN_ctxGetId)(CUcontext, unsigned long long *);

pba_status current_context_id(unsigned long long *id) {
    static PFN_ctxGetCurrent get_cur = nullptr;
    static PFN_ctxGetId get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        cudaDriverEntryPointQueryResult q;
        void *fn = nullptr;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &fn, 12000, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            get_cur = reinterpret_cast<PFN_ctxGetCurrent>(fn);
        fn = nullptr;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &fn, 12000, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<PFN_ctxGetId>(fn);
    });
    if (!get_cur || !get_id) return fail(PBA_ERR_CUDA, "cuCtxGetCurrent / cuCtxGetId unavailable");
    CUcontext ctx = nullptr;
    if (get_cur(&ctx) != CUDA_SUCCESS || !ctx) return fail(PBA_ERR_CUDA, "no current CUDA context");
    if (get_id(ctx, id) != CUDA_SUCCESS) return fail(PBA_ERR_CUDA, "cuCtxGetId failed");
    return PBA_OK;
}

pba_status noalloc_scratch(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    // makes the device's primary context current if the caller has none yet
    if ((e = cudaSetDevice(dev)) != cudaSuccess) return cuda_fail(e, "cudaSetDevice");
    unsigned long long ctx_id = 0;
    pba_status st = current_context_id(&ctx_id);
    if (st != PBA_OK) return st;
    std::lock_guard<std::mutex> g(g_noalloc_mu);
    for (const auto &ent : g_noalloc_addr)
        if (ent.first == ctx_id) {
            *out = ent.second;
            return PBA_OK;
        }
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_pba_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress of the built-in scratch");
    g_noalloc_addr.emplace_back(ctx_id, p);
    *out = p;
    return PBA_OK;
}


bool side_stream(cudaStream_t s, SideStream *out) {
    unsigned long long id = 0;
    {
        // a failure here only means no side stream: keep the caller's last error untouched
        const std::string keep = g_last_error;
        const pba_status st = current_context_id(&id);
        g_last_error = keep;
        if (st != PBA_OK) return false;
    }
    for (const auto &ent : g_side)
        if (ent.ctx == id) {
            *out = ent;
            return true;
        }
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone) return false;
    int lo = 0, hi = 0;
    if (cudaDeviceGetStreamPriorityRange(&lo, &hi) != cudaSuccess) return false;
    SideStream ent{id, nullptr, nullptr, nullptr};
    if (cudaStreamCreateWithPriority(&ent.s, cudaStreamNonBlocking, hi) != cudaSuccess) return false;
    if (cudaEventCreateWithFlags(&ent.fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&ent.join, cudaEventDisableTiming) != cudaSuccess) {
        if (ent.fork) cudaEventDestroy(ent.fork);
        cudaStreamDestroy(ent.s);
        cudaGetLastError();
        return false;
    }
    g_side.push_back(ent);
    *out = ent;
    return true;
}

// ---------------------------------------------------------------------------- pair-weighted
// The [H, N, Wld] bf16 weights as a 3-D map (N, N, H), box (64, 128, 1), 128-byte swizzle:
// the same tiles as the bias.
pba_status map_w(CUtensorMap *m, void *base, int H, int N, int Wld, int rows = 128) {
    cuuint64_t dims[3] = {(cuuint64_t)N, (cuuint64_t)N, (cuuint64_t)H};
    cuuint64_t strides[2] = {(cuuint64_t)Wld * 2, (cuuint64_t)N * Wld * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(PBA_ERR_CUDA, "tensor map for the weights failed (CUresult %d)", (int)r);
    return PBA_OK;
}

struct PwaPlan {
    int N, Wld, NPad, nT, splits, rows_per_split;
    size_t off_w, off_lse, off_doa, off_part, fwd_total, bwd_total;
};

PwaPlan plan_pwa(const pba_dims *d) {
    PwaPlan p;
    p.N = d->Nq;
    p.Wld = (p.N + 7) / 8 * 8;
    p.nT = (p.N + 127) / 128;
    p.NPad = p.nT * 128;
    // splits of the rows b for the dW partials: a function of the sizes only (bit-stable
    // dbias), chosen like the attention's dbias splits
    const long long tiles = (long long)d->H * p.nT * p.nT;
    const long long maxs = d->B < 64 ? (d->B > 0 ? d->B : 1) : 64;
    long long best = -1;
    p.splits = 1;
    p.rows_per_split = d->B > 0 ? d->B : 1;
    for (long long sp = 1; sp <= maxs; ++sp) {
        const long long rows = d->B > 0 ? (d->B + sp - 1) / sp : 1;
        const long long actual = d->B > 0 ? (d->B + rows - 1) / rows : 1;
        const long long waves = (tiles * actual + 2 * kSmCount - 1) / (2 * kSmCount);   // 2 CTAs per SM
        const long long cost = waves * (rows + 3);
        if (best < 0 || cost < best) {
            best = cost;
            p.splits = (int)actual;
            p.rows_per_split = (int)rows;
        }
    }
    p.off_w = 0;
    p.fwd_total = align256((size_t)d->H * p.N * p.Wld * 2);
    p.off_lse = p.fwd_total;
    p.off_doa = align256(p.off_lse + (size_t)d->H * p.N * 4);
    p.off_part = align256(p.off_doa + (size_t)d->B * p.N * d->H * d->C * 2);
    p.bwd_total = align256(p.off_part + (size_t)p.splits * d->H * p.NPad * p.NPad * 4);
    return p;
}

pba_status check_pwa_dims(const pba_dims *d) {
    pba_status st = check_dims(d);
    if (st != PBA_OK) return st;
    if (d->Nq != d->Nk) return fail(PBA_ERR_UNSUPPORTED, "pair-weighted averaging needs Nq == Nk");
    if (d->smask_b != 0 && d->B > 1)
        return fail(PBA_ERR_UNSUPPORTED, "pair-weighted averaging needs a key mask shared by every row (smask_b = 0)");
    return PBA_OK;
}

void fill_pwa_args(pba::PwaArgs &a, const PwaPlan &pl, const pba_dims *d, const pba_bf16 *bias,
                   const uint8_t *mask, const pba_bf16 *gate, uint8_t *ws) {
    std::memset(&a, 0, sizeof(a));
    a.B = d->B; a.H = d->H; a.N = pl.N; a.C = d->C;
    a.nT = pl.nT; a.NPad = pl.NPad; a.Wld = pl.Wld;
    a.splits = pl.splits; a.rows_per_split = pl.rows_per_split;
    a.has_bias = bias != nullptr;
    a.has_gate = gate != nullptr;
    a.bias = reinterpret_cast<const __nv_bfloat16 *>(bias);
    a.sb0 = d->sbias[0]; a.sb1 = d->sbias[1];
    a.mask = mask;
    a.gate = reinterpret_cast<const __nv_bfloat16 *>(gate);
    a.sg0 = d->sg[0]; a.sg1 = d->sg[1]; a.sg2 = d->sg[2];
    a.w = reinterpret_cast<__nv_bfloat16 *>(ws + pl.off_w);
}

template <int CP>
pba_status launch_pwa_gemm(const CUtensorMap &tw, const CUtensorMap &tx, const pba::PwaArgs &a0, bool dv,
                           cudaStream_t s) {
    using T = pba::PwaTraits<CP>;
    pba::PwaArgs a = a0;
    a.nChunks = (a.B + T::BC - 1) / T::BC;
    const long long grid = (long long)a.H * a.nT * a.nChunks;
    if (dv) {
        pba_status st = set_smem(pba::pba_pwa_gemm_kernel<CP, true>, T::SMEM_BYTES);
        if (st != PBA_OK) return st;
        cudaFuncSetAttribute(pba::pba_pwa_gemm_kernel<CP, true>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
        ProfScope ps(K_PWA_DV, s);
        pba::pba_pwa_gemm_kernel<CP, true><<<(unsigned)grid, 192, T::SMEM_BYTES, s>>>(tw, tx, a);
    } else {
        pba_status st = set_smem(pba::pba_pwa_gemm_kernel<CP, false>, T::SMEM_BYTES);
        if (st != PBA_OK) return st;
        cudaFuncSetAttribute(pba::pba_pwa_gemm_kernel<CP, false>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
        ProfScope ps(K_PWA_FWD, s);
        pba::pba_pwa_gemm_kernel<CP, false><<<(unsigned)grid, 192, T::SMEM_BYTES, s>>>(tw, tx, a);
    }
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? PBA_OK : cuda_fail(e, "pba_pwa_gemm_kernel launch");
}

pba_status launch_pwa_weights(const pba::PwaArgs &a, cudaStream_t s) {
    {
        ProfScope ps(K_PWA_WEIGHTS, s);
        pba::pba_pwa_weights_kernel<<<grid_for((long long)a.H * a.N * 32, 256), 256, 0, s>>>(a);
    }
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? PBA_OK : cuda_fail(e, "pba_pwa_weights_kernel launch");
}

template <int CP>
pba_status launch_pwa_fwd(const pba_bf16 *v, const pba_bf16 *bias, const uint8_t *mask, const pba_bf16 *gate,
                          pba_bf16 *out, float *lse, uint8_t *ws, const PwaPlan &pl, const pba_dims *d,
                          cudaStream_t s) {
    pba::PwaArgs a;
    fill_pwa_args(a, pl, d, bias, mask, gate, ws);
    a.lse = lse;
    a.out = reinterpret_cast<__nv_bfloat16 *>(out);
    a.so0 = d->so[0]; a.so1 = d->so[1]; a.so2 = d->so[2];
    pba_status st;
    CUtensorMap tw, tv;
    // the GEMM's stages: 128 output rows x 64 reduction columns of w, 64 rows of each V tile
    if ((st = map_w(&tw, a.w, d->H, pl.N, pl.Wld, 128)) != PBA_OK) return st;
    if ((st = map_bnhc(&tv, v, d->B, pl.N, d->H, d->C, d->sv, CP, "v", 64)) != PBA_OK) return st;
    if ((st = launch_pwa_weights(a, s)) != PBA_OK) return st;
    return launch_pwa_gemm<CP>(tw, tv, a, false, s);
}

template <int CP>
pba_status launch_pwa_bwd(const pba_bf16 *v, const pba_bf16 *bias, const uint8_t *mask, const pba_bf16 *gate,
                          const pba_bf16 *out, const pba_bf16 *dout, pba_bf16 *dv, float *dbias, pba_bf16 *dgate,
                          uint8_t *ws, const PwaPlan &pl, const pba_dims *d, cudaStream_t s) {
    using DT = pba::PwaDwTraits<CP>;
    pba::PwaArgs a;
    fill_pwa_args(a, pl, d, bias, mask, gate, ws);
    a.lse = reinterpret_cast<float *>(ws + pl.off_lse);
    a.doa = reinterpret_cast<__nv_bfloat16 *>(ws + pl.off_doa);
    a.dw_part = reinterpret_cast<float *>(ws + pl.off_part);
    a.dbias = dbias;
    a.dgate = reinterpret_cast<__nv_bfloat16 *>(dgate);
    a.oin = reinterpret_cast<const __nv_bfloat16 *>(out);
    a.dout = reinterpret_cast<const __nv_bfloat16 *>(dout);
    a.si0 = d->so[0]; a.si1 = d->so[1]; a.si2 = d->so[2];
    pba_status st;
    // dW partials: 128-row tiles of dOa and V; dv GEMM: 64 x 128 blocks of w (rows i =
    // reduction, columns j = output) and 64-row tiles of dOa
    CUtensorMap tw, tv, tdo, tdo64;
    if ((st = map_w(&tw, a.w, d->H, pl.N, pl.Wld, 64)) != PBA_OK) return st;
    if ((st = map_bnhc(&tv, v, d->B, pl.N, d->H, d->C, d->sv, CP, "v")) != PBA_OK) return st;
    if (gate) {
        const int64_t sd[3] = {(int64_t)pl.N * d->H * d->C, (int64_t)d->H * d->C, d->C};
        if ((st = map_bnhc(&tdo, a.doa, d->B, pl.N, d->H, d->C, sd, CP, "dOa")) != PBA_OK) return st;
        if ((st = map_bnhc(&tdo64, a.doa, d->B, pl.N, d->H, d->C, sd, CP, "dOa", 64)) != PBA_OK) return st;
    } else {
        if ((st = map_bnhc(&tdo, dout, d->B, pl.N, d->H, d->C, d->so, CP, "dout")) != PBA_OK) return st;
        if ((st = map_bnhc(&tdo64, dout, d->B, pl.N, d->H, d->C, d->so, CP, "dout", 64)) != PBA_OK) return st;
    }
    if ((st = launch_pwa_weights(a, s)) != PBA_OK) return st;
    cudaError_t e;
    if (gate) {
        {
            ProfScope ps(K_PWA_PRE, s);
            pba::pba_pwa_pre_kernel<<<grid_for((long long)d->B * pl.N * d->H * (d->C / 8), 256), 256, 0, s>>>(a);
        }
        if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "pba_pwa_pre_kernel launch");
    }
    // dv = W^T dOa (rows j)
    pba::PwaArgs av = a;
    av.out = reinterpret_cast<__nv_bfloat16 *>(dv);
    av.so0 = d->sv[0]; av.so1 = d->sv[1]; av.so2 = d->sv[2];
    if ((st = launch_pwa_gemm<CP>(tw, tdo64, av, true, s)) != PBA_OK) return st;
    if (dbias) {
        if ((st = set_smem(pba::pba_pwa_dw_kernel<CP>, DT::SMEM_BYTES)) != PBA_OK) return st;
        cudaFuncSetAttribute(pba::pba_pwa_dw_kernel<CP>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
        const long long g2 = (long long)pl.splits * d->H * pl.nT * pl.nT;
        {
            ProfScope ps(K_PWA_DW, s);
            pba::pba_pwa_dw_kernel<CP><<<(unsigned)g2, 192, DT::SMEM_BYTES, s>>>(tdo, tv, a);
        }
        if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "pba_pwa_dw_kernel launch");
        {
            ProfScope ps(K_PWA_DBIAS, s);
            pba::pba_pwa_dbias_kernel<<<grid_for((long long)d->H * pl.N * 32, 256), 256, 0, s>>>(a);
        }
        if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "pba_pwa_dbias_kernel launch");
    }
    return PBA_OK;
}

pba_status check_pwa_common(const pba_bf16 *v, const pba_bf16 *bias, const uint8_t *mask, const pba_bf16 *gate,
                            const pba_dims *d) {
    pba_status st;
    if ((st = check_strides(d->sv, d->B, d->Nk, d->H, "v")) != PBA_OK) return st;
    if ((st = check_strides(d->so, d->B, d->Nq, d->H, "out")) != PBA_OK) return st;
    if (!v) return fail(PBA_ERR_INVALID_ARG, "v is required");
    if (!aligned16(v)) return fail(PBA_ERR_INVALID_ARG, "v must be 16-byte aligned");
    if (gate) {
        if (!aligned16(gate)) return fail(PBA_ERR_INVALID_ARG, "gate must be 16-byte aligned");
        if ((st = check_strides(d->sg, d->B, d->Nq, d->H, "gate")) != PBA_OK) return st;
    }
    if (bias && d->H > 1 && d->sbias[0] <= 0) return fail(PBA_ERR_INVALID_ARG, "bias: H stride must be positive");
    if (bias && d->Nq > 1 && d->sbias[1] <= 0) return fail(PBA_ERR_INVALID_ARG, "bias: row stride must be positive");
    (void)mask;
    return get_encoder();
}

// ------------------------------------------------------------------ pair-bias projection
int pb_hp(int H) { return H <= 4 ? 4 : (H <= 8 ? 8 : 16); }

pba_status check_pb_dims(const pba_pair_bias_dims *d) {
    if (!d) return fail(PBA_ERR_INVALID_ARG, "dims is NULL");
    if (d->Ni < 0 || d->Nj < 0 || d->Cz < 0 || d->H < 0) return fail(PBA_ERR_INVALID_ARG, "negative size");
    if (d->Cz != 64 && d->Cz != 128 && d->Cz != 192 && d->Cz != 256)
        return fail(PBA_ERR_UNSUPPORTED, "Cz=%d: must be 64, 128, 192 or 256", d->Cz);
    if (d->H < 1 || d->H > 16) return fail(PBA_ERR_UNSUPPORTED, "H=%d: must be in [1, 16]", d->H);
    if (!(d->eps > 0.f) || !std::isfinite(d->eps)) return fail(PBA_ERR_INVALID_ARG, "eps must be finite and > 0");
    if (d->Ni > (1 << 24) || d->Nj > (1 << 24)) return fail(PBA_ERR_UNSUPPORTED, "sizes too large");
    if ((long long)d->Ni * ((d->Nj + 127) / 128) > INT_MAX) return fail(PBA_ERR_UNSUPPORTED, "too many tiles");
    const int ext[2] = {d->Ni, d->Nj};
    for (int k = 0; k < 2; ++k) {
        if (ext[k] > 1 && (d->sz[k] <= 0 || d->sz[k] % 8 != 0))
            return fail(PBA_ERR_INVALID_ARG, "z: stride %d must be a positive multiple of 8 elements", k);
        if (d->sz[k] * 2 >= (int64_t(1) << 40)) return fail(PBA_ERR_UNSUPPORTED, "z: stride too large");
    }
    return PBA_OK;
}

long long pb_grid(const pba_pair_bias_dims *d, int smem_bytes) {
    const long long tiles = (long long)d->Ni * ((d->Nj + 127) / 128);
    long long per_sm = 233472 / (smem_bytes + 1024);
    per_sm = per_sm < 1 ? 1 : (per_sm > 4 ? 4 : per_sm);
    // a fixed function of the sizes (not of the device): the order of the backward's sums
    // depends on it
    const long long g = per_sm * kSmCount;
    return tiles < g ? tiles : g;
}

template <int CZ, int HP>
int pb_smem() {
    // the backward's layout (its grid fixes the partials): Cz = 128 has its own kernel
    if constexpr (CZ == 128) return pba::PbBwdTcTraits<HP>::SMEM_BYTES;
    else return pba::PbTraits<CZ, HP>::SMEM_BYTES;
}

int pb_smem_for(int Cz, int HP) {
#define PB_CASE(cz, hp) if (Cz == cz && HP == hp) return pb_smem<cz, hp>();
    PB_CASE(64, 4) PB_CASE(64, 8) PB_CASE(64, 16) PB_CASE(128, 4) PB_CASE(128, 8) PB_CASE(128, 16)
    PB_CASE(192, 4) PB_CASE(192, 8) PB_CASE(192, 16) PB_CASE(256, 4) PB_CASE(256, 8) PB_CASE(256, 16)
#undef PB_CASE
    return 0;
}

// workspace: the per-block partials [grid][Cz * HP + HP], then their sums [Cz * HP + HP]
size_t pb_ws_bytes(const pba_pair_bias_dims *d) {
    const int HP = pb_hp(d->H);
    const long long g = pb_grid(d, pb_smem_for(d->Cz, HP));
    return (size_t)((g > 0 ? g : 1) + 1) * ((size_t)d->Cz * HP + HP) * 4;
}

// z as a 3-D map (Cz, Nj, Ni), box (64, 128, 1), 128-byte swizzle
pba_status map_z(CUtensorMap *m, const void *z, const pba_pair_bias_dims *d) {
    cuuint64_t dims[3] = {(cuuint64_t)d->Cz, (cuuint64_t)(d->Nj > 0 ? d->Nj : 1), (cuuint64_t)(d->Ni > 0 ? d->Ni : 1)};
    cuuint64_t strides[2] = {(cuuint64_t)(d->Nj > 1 ? d->sz[1] * 2 : 16), (cuuint64_t)(d->Ni > 1 ? d->sz[0] * 2 : 16)};
    cuuint32_t box[3] = {64, 128, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(z), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(PBA_ERR_CUDA, "tensor map for z failed (CUresult %d)", (int)r);
    return PBA_OK;
}

pba::PbArgs pb_args(const pba_pair_bias_dims *d, const float *gamma, const float *beta, const float *w) {
    pba::PbArgs a;
    std::memset(&a, 0, sizeof(a));
    a.Ni = d->Ni; a.Nj = d->Nj; a.Cz = d->Cz; a.H = d->H;
    a.nJt = (d->Nj + 127) / 128;
    a.tiles = (int)((long long)d->Ni * a.nJt);
    a.eps = d->eps;
    a.gamma = gamma; a.beta = beta; a.w = w;
    a.sz0 = d->sz[0]; a.sz1 = d->sz[1];
    a.sb0 = d->sbias[0]; a.sb1 = d->sbias[1];
    a.sd0 = d->sdbias[0]; a.sd1 = d->sdbias[1];
    a.hp = pb_hp(d->H);
    return a;
}

template <int CZ, int HP>
pba_status launch_pb(bool bwd, const CUtensorMap &tm, pba::PbArgs a, const pba_pair_bias_dims *d, cudaStream_t s) {
    using T = pba::PbTraits<CZ, HP>;
    const int bwd_smem = pb_smem<CZ, HP>();
    const long long grid = pb_grid(d, bwd_smem);
    a.nparts = (int)grid;
    pba_status st;
    cudaError_t e;
    if (!bwd) {
        // the forward has its own shared-memory layout (and so its own grid); nothing of the
        // backward's reduction order depends on it
        using F = pba::PbFwdTraits<CZ>;
        const long long fgrid = pb_grid(d, F::SMEM_BYTES);
        if ((st = set_smem(pba::pba_pair_bias_fwd_kernel<CZ, HP>, F::SMEM_BYTES)) != PBA_OK) return st;
        ProfScope ps(K_PB_FWD, s);
        pba::pba_pair_bias_fwd_kernel<CZ, HP><<<(unsigned)fgrid, F::THREADS, F::SMEM_BYTES, s>>>(tm, a);
        if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "pba_pair_bias_fwd_kernel launch");
        return PBA_OK;
    }
    if constexpr (CZ == 128) {
        // parameter sums on the tensor core
        if ((st = set_smem(pba::pba_pair_bias_bwd_tc_kernel<HP>, bwd_smem)) != PBA_OK) return st;
        ProfScope ps(K_PB_BWD_TC, s);
        pba::pba_pair_bias_bwd_tc_kernel<HP><<<(unsigned)grid, 128, bwd_smem, s>>>(tm, a);
    } else {
        if ((st = set_smem(pba::pba_pair_bias_bwd_kernel<CZ, HP>, T::SMEM_BYTES)) != PBA_OK) return st;
        ProfScope ps(K_PB_BWD, s);
        pba::pba_pair_bias_bwd_kernel<CZ, HP><<<(unsigned)grid, 128, T::SMEM_BYTES, s>>>(tm, a);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "pba_pair_bias_bwd_kernel launch");
    a.sums = a.part + grid * ((long long)CZ * HP + HP);
    {
        ProfScope ps(K_PB_REDUCE, s);
        pba::pba_pair_bias_reduce_kernel<<<(unsigned)((CZ * HP + HP + 31) / 32), 512, 0, s>>>(a);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "pba_pair_bias_reduce_kernel launch");
    {
        ProfScope ps(K_PB_PARAM, s);
        pba::pba_pair_bias_param_kernel<<<(unsigned)((CZ + 127) / 128), 128, 0, s>>>(a);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "pba_pair_bias_param_kernel launch");
    return PBA_OK;
}

pba_status dispatch_pb(bool bwd, const CUtensorMap &tm, const pba::PbArgs &a, const pba_pair_bias_dims *d,
                       cudaStream_t s) {
    const int HP = pb_hp(d->H);
#define PB_CASE(cz, hp) if (d->Cz == cz && HP == hp) return launch_pb<cz, hp>(bwd, tm, a, d, s);
    PB_CASE(64, 4) PB_CASE(64, 8) PB_CASE(64, 16) PB_CASE(128, 4) PB_CASE(128, 8) PB_CASE(128, 16)
    PB_CASE(192, 4) PB_CASE(192, 8) PB_CASE(192, 16) PB_CASE(256, 4) PB_CASE(256, 8) PB_CASE(256, 16)
#undef PB_CASE
    return fail(PBA_ERR_UNSUPPORTED, "unsupported Cz / H");
}

}  // namespace

extern "C" {

void pba_dims_dense(pba_dims *d, int32_t B, int32_t H, int32_t Nq, int32_t Nk, int32_t C,
                    float scale) {
    std::memset(d, 0, sizeof(*d));
    d->B = B; d->H = H; d->Nq = Nq; d->Nk = Nk; d->C = C;
    d->scale = scale;
    const int64_t q3[3] = {(int64_t)Nq * H * C, (int64_t)H * C, C};
    const int64_t k3[3] = {(int64_t)Nk * H * C, (int64_t)H * C, C};
    for (int i = 0; i < 3; ++i) {
        d->sq[i] = q3[i]; d->sg[i] = q3[i]; d->so[i] = q3[i];
        d->sk[i] = k3[i]; d->sv[i] = k3[i];
    }
    d->sbias[0] = (int64_t)Nq * Nk;
    d->sbias[1] = Nk;
    d->smask_b = 0;
}

pba_status pba_fwd(const pba_bf16 *q, const pba_bf16 *k, const pba_bf16 *v,
                   const pba_bf16 *bias, const uint8_t *key_mask, const pba_bf16 *gate,
                   pba_bf16 *out, float *lse, const pba_dims *d, void *stream) {
    return pba_fwd_local(q, k, v, bias, key_mask, gate, out, lse, d, -1, stream);
}

pba_status pba_fwd_local(const pba_bf16 *q, const pba_bf16 *k, const pba_bf16 *v,
                         const pba_bf16 *bias, const uint8_t *key_mask, const pba_bf16 *gate,
                         pba_bf16 *out, float *lse, const pba_dims *d, int window, void *stream) {
    g_last_error.clear();
    pba_status st = check_dims(d);
    if (st != PBA_OK) return st;
    if ((st = check_window(d, window)) != PBA_OK) return st;
    if (d->B == 0 || d->Nq == 0) return PBA_OK;  // nothing to compute
    if ((st = check_layouts(d)) != PBA_OK) return st;
    if (!q || !k || !v || !out || !lse) return fail(PBA_ERR_INVALID_ARG, "q, k, v, out and lse are required");
    if (d->Nk > 0 && (!aligned16(q) || !aligned16(k) || !aligned16(v)))
        return fail(PBA_ERR_INVALID_ARG, "q, k, v must be 16-byte aligned");
    if (!aligned16(out)) return fail(PBA_ERR_INVALID_ARG, "out must be 16-byte aligned");
    if (gate) {
        if (!aligned16(gate)) return fail(PBA_ERR_INVALID_ARG, "gate must be 16-byte aligned");
        if ((st = check_strides(d->sg, d->B, d->Nq, d->H, "gate")) != PBA_OK) return st;
    }
    if (bias) {
        if (!aligned16(bias)) return fail(PBA_ERR_INVALID_ARG, "bias must be 16-byte aligned");
        if ((st = check_bias(d)) != PBA_OK) return st;
    }
    if (key_mask && d->smask_b < 0) return fail(PBA_ERR_INVALID_ARG, "smask_b must be >= 0");
    if ((st = get_encoder()) != PBA_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    switch (padded_c(d->C)) {
        case 16: return launch_fwd<16>(q, k, v, bias, key_mask, gate, out, lse, d, window, s);
        case 32: return launch_fwd<32>(q, k, v, bias, key_mask, gate, out, lse, d, window, s);
        default: return launch_fwd<64>(q, k, v, bias, key_mask, gate, out, lse, d, window, s);
    }
}

size_t pba_bwd_workspace_size(const pba_dims *d) {
    if (!d || check_dims(d) != PBA_OK) return 0;
    return plan_bwd(d).total;
}

pba_status pba_bwd(const pba_bf16 *q, const pba_bf16 *k, const pba_bf16 *v,
                   const pba_bf16 *bias, const uint8_t *key_mask, const pba_bf16 *gate,
                   const pba_bf16 *out, const float *lse, const pba_bf16 *dout,
                   pba_bf16 *dq, pba_bf16 *dk, pba_bf16 *dv, float *dbias, pba_bf16 *dgate,
                   void *workspace, size_t workspace_bytes, const pba_dims *d, void *stream) {
    return pba_bwd_local(q, k, v, bias, key_mask, gate, out, lse, dout, dq, dk, dv, dbias, dgate,
                         workspace, workspace_bytes, d, -1, stream);
}

// Every check of the backward's arguments except the workspace: shared by pba_bwd_local and
// pba_bwd_noalloc, so both report an argument error before any question of scratch size.
pba_status check_bwd_args(const pba_bf16 *q, const pba_bf16 *k, const pba_bf16 *v,
                          const pba_bf16 *bias, const uint8_t *key_mask, const pba_bf16 *gate,
                          const pba_bf16 *out, const float *lse, const pba_bf16 *dout,
                          pba_bf16 *dq, pba_bf16 *dk, pba_bf16 *dv, pba_bf16 *dgate,
                          const pba_dims *d, int window) {
    pba_status st = check_dims(d);
    if (st != PBA_OK) return st;
    if ((st = check_window(d, window)) != PBA_OK) return st;
    if (d->B == 0) return PBA_OK;
    if (d->Nq == 0) {
        if (d->Nk == 0) return PBA_OK;
        if (!dk || !dv) return fail(PBA_ERR_INVALID_ARG, "dk and dv are required");
        if ((st = check_strides(d->sk, d->B, d->Nk, d->H, "k")) != PBA_OK) return st;
        return check_strides(d->sv, d->B, d->Nk, d->H, "v");
    }
    if ((st = check_layouts(d)) != PBA_OK) return st;
    if (!q || !k || !v || !out || !lse || !dout || !dq || !dk || !dv)
        return fail(PBA_ERR_INVALID_ARG, "q, k, v, out, lse, dout, dq, dk and dv are required");
    if (gate && !dgate) return fail(PBA_ERR_INVALID_ARG, "dgate is required when gate is given");
    const void *aligned_ptrs[] = {q, k, v, out, dout, dq, dk, dv};
    for (const void *p : aligned_ptrs)
        if (!aligned16(p)) return fail(PBA_ERR_INVALID_ARG, "bf16 tensors must be 16-byte aligned");
    if (gate) {
        if (!aligned16(gate) || !aligned16(dgate))
            return fail(PBA_ERR_INVALID_ARG, "gate and dgate must be 16-byte aligned");
        if ((st = check_strides(d->sg, d->B, d->Nq, d->H, "gate")) != PBA_OK) return st;
    }
    if (bias) {
        if (!aligned16(bias)) return fail(PBA_ERR_INVALID_ARG, "bias must be 16-byte aligned");
        if ((st = check_bias(d)) != PBA_OK) return st;
    }
    if (key_mask && d->smask_b < 0) return fail(PBA_ERR_INVALID_ARG, "smask_b must be >= 0");
    return PBA_OK;
}

pba_status pba_bwd_local(const pba_bf16 *q, const pba_bf16 *k, const pba_bf16 *v,
                         const pba_bf16 *bias, const uint8_t *key_mask, const pba_bf16 *gate,
                         const pba_bf16 *out, const float *lse, const pba_bf16 *dout,
                         pba_bf16 *dq, pba_bf16 *dk, pba_bf16 *dv, float *dbias, pba_bf16 *dgate,
                         void *workspace, size_t workspace_bytes, const pba_dims *d, int window,
                         void *stream) {
    g_last_error.clear();
    pba_status st = check_bwd_args(q, k, v, bias, key_mask, gate, out, lse, dout, dq, dk, dv, dgate, d, window);
    if (st != PBA_OK) return st;
    if (d->B == 0) return PBA_OK;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (d->Nq == 0) {
        // no query: every key gradient is zero, there is no dq, dgate or dbias element
        if (d->Nk == 0) return PBA_OK;
        if ((st = get_encoder()) != PBA_OK) return st;  // (keeps error handling uniform)
        return launch_zero_rows(dk, dv, d, s);
    }
    const BwdPlan pl = plan_bwd(d, window);
    if (!workspace || workspace_bytes < pl.total)
        return fail(PBA_ERR_WORKSPACE, "workspace of %zu bytes given, %zu needed", workspace_bytes,
                    pl.total);
    if (reinterpret_cast<uintptr_t>(workspace) & 255u)
        return fail(PBA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    if ((st = get_encoder()) != PBA_OK) return st;
    switch (padded_c(d->C)) {
        case 16: return launch_bwd<16>(q, k, v, bias, key_mask, gate, out, lse, dout, dq, dk, dv, dbias, dgate, workspace, pl, d,
                                  window, s);
        case 32: return launch_bwd<32>(q, k, v, bias, key_mask, gate, out, lse, dout, dq, dk, dv, dbias, dgate, workspace, pl, d,
                                  window, s);
        default: return launch_bwd<64>(q, k, v, bias, key_mask, gate, out, lse, dout, dq, dk, dv, dbias, dgate, workspace, pl, d,
                                  window, s);
    }
}

pba_status pba_bwd_noalloc(const pba_bf16 *q, const pba_bf16 *k, const pba_bf16 *v,
                           const pba_bf16 *bias, const uint8_t *key_mask, const pba_bf16 *gate,
                           const pba_bf16 *out, const float *lse, const pba_bf16 *dout,
                           pba_bf16 *dq, pba_bf16 *dk, pba_bf16 *dv, float *dbias,
                           pba_bf16 *dgate, const pba_dims *d, void *stream) {
    g_last_error.clear();
    // the same argument checks as pba_bwd first, then the scratch size
    pba_status st = check_bwd_args(q, k, v, bias, key_mask, gate, out, lse, dout, dq, dk, dv, dgate, d, -1);
    if (st != PBA_OK) return st;
    if (d->B > 0 && d->Nq > 0) {
        const size_t need = plan_bwd(d).total;
        if (need > kNoAllocScratchBytes)
            return fail(PBA_ERR_UNSUPPORTED,
                        "pba_bwd_noalloc: these sizes need %zu bytes of scratch, more than the %zu "
                        "built into the library; call pba_bwd with a workspace instead",
                        need, kNoAllocScratchBytes);
    }
    void *scratch = nullptr;
    if ((st = noalloc_scratch(&scratch)) != PBA_OK) return st;
    return pba_bwd(q, k, v, bias, key_mask, gate, out, lse, dout, dq, dk, dv, dbias, dgate,
                   scratch, kNoAllocScratchBytes, d, stream);
}

pba_status pba_dbias_sum(const float *parts, int n_parts, int64_t n, float *out, void *stream) {
    g_last_error.clear();
    if (n_parts < 1 || n < 0) return fail(PBA_ERR_INVALID_ARG, "n_parts must be >= 1 and n >= 0");
    if (n == 0) return PBA_OK;
    if (!parts || !out) return fail(PBA_ERR_INVALID_ARG, "parts and out are required");
    if (!aligned16(parts) || !aligned16(out)) return fail(PBA_ERR_INVALID_ARG, "parts and out must be 16-byte aligned");
    const uintptr_t lo = reinterpret_cast<uintptr_t>(parts), hi = lo + (uintptr_t)n_parts * (uintptr_t)n * 4;
    const uintptr_t o0 = reinterpret_cast<uintptr_t>(out), o1 = o0 + (uintptr_t)n * 4;
    if (o0 < hi && lo < o1) return fail(PBA_ERR_INVALID_ARG, "out overlaps parts");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int vec = (n & 3) == 0;
    {
        ProfScope ps(K_DBIAS_SUM, s);
        pba::pba_dbias_sum_kernel<<<grid_for(vec ? n / 4 : n, 256), 256, 0, s>>>(parts, n_parts, n, out, vec);
    }
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? PBA_OK : cuda_fail(e, "pba_dbias_sum_kernel launch");
}

pba_status pba_device_status(void *stream) {
    cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    unsigned int w = 0, site = 0, zero = 0;
    e = cudaMemcpyFromSymbol(&w, pba::g_pba_watchdog, sizeof(w));
    if (e != cudaSuccess) return cuda_fail(e, "reading the watchdog word");
    if (w) {
        cudaMemcpyFromSymbol(&site, pba::g_pba_watchdog_site, sizeof(site));
        cudaMemcpyToSymbol(pba::g_pba_watchdog, &zero, sizeof(zero));
        cudaMemcpyToSymbol(pba::g_pba_watchdog_site, &zero, sizeof(zero));
        if ((site & 0xFFFu) == pba::SITE_FWD_ALIGN || (site & 0xFFFu) == pba::SITE_PWA_ALIGN ||
            (site & 0xFFFu) == pba::SITE_PB_ALIGN)
            return fail(PBA_ERR_UNSUPPORTED, "forward kernel refused: dynamic shared memory "
                                             "is not 1024-byte aligned");
        return fail(PBA_ERR_TIMEOUT, "a bounded in-kernel wait ran out (site 0x%x)", site);
    }
    return PBA_OK;
}

pba_status pba_profile_enable(int on) {
    std::lock_guard<std::mutex> g(g_prof_mu);
    g_prof_on = on != 0;
    return PBA_OK;
}

int pba_profile_read(pba_kernel_stat *out, int max) {
    std::vector<ProfRec> recs;
    {
        std::lock_guard<std::mutex> g(g_prof_mu);
        recs.swap(g_prof_recs);
    }
    int64_t launches[K_COUNT] = {0};
    double ms[K_COUNT] = {0};
    bool err = false;
    for (const ProfRec &r : recs) {
        float t = 0.f;
        if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess)
            err = true;
        launches[r.kid] += 1;
        ms[r.kid] += t;
    }
    {
        std::lock_guard<std::mutex> g(g_prof_mu);
        for (const ProfRec &r : recs) {
            g_prof_pool.push_back(r.a);
            g_prof_pool.push_back(r.b);
        }
    }
    if (err) return -1;
    int n = 0;
    for (int k = 0; k < K_COUNT; ++k) {
        if (!launches[k]) continue;
        if (out && n < max) {
            std::memset(&out[n], 0, sizeof(out[n]));
            std::snprintf(out[n].name, sizeof(out[n].name), "%s", kKernelNames[k]);
            out[n].launches = launches[k];
            out[n].total_ms = ms[k];
        }
        ++n;
    }
    return n < max ? n : max;
}

size_t pba_pwa_fwd_workspace_size(const pba_dims *d) {
    if (!d || check_pwa_dims(d) != PBA_OK) return 0;
    return plan_pwa(d).fwd_total;
}

size_t pba_pwa_bwd_workspace_size(const pba_dims *d) {
    if (!d || check_pwa_dims(d) != PBA_OK) return 0;
    return plan_pwa(d).bwd_total;
}

pba_status pba_pwa_fwd(const pba_bf16 *v, const pba_bf16 *bias, const uint8_t *key_mask, const pba_bf16 *gate,
                       pba_bf16 *out, float *lse_w, void *workspace, size_t workspace_bytes,
                       const pba_dims *d, void *stream) {
    g_last_error.clear();
    pba_status st = check_pwa_dims(d);
    if (st != PBA_OK) return st;
    if (d->B == 0 || d->Nq == 0 || d->H == 0) return PBA_OK;
    if (!out || !lse_w) return fail(PBA_ERR_INVALID_ARG, "out and lse_w are required");
    if (!aligned16(out)) return fail(PBA_ERR_INVALID_ARG, "out must be 16-byte aligned");
    if ((st = check_pwa_common(v, bias, key_mask, gate, d)) != PBA_OK) return st;
    const PwaPlan pl = plan_pwa(d);
    if (!workspace || workspace_bytes < pl.fwd_total)
        return fail(PBA_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", pl.fwd_total, workspace_bytes);
    if (reinterpret_cast<uintptr_t>(workspace) & 255u)
        return fail(PBA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    switch (padded_c(d->C)) {
        case 16: return launch_pwa_fwd<16>(v, bias, key_mask, gate, out, lse_w, ws, pl, d, s);
        case 32: return launch_pwa_fwd<32>(v, bias, key_mask, gate, out, lse_w, ws, pl, d, s);
        default: return launch_pwa_fwd<64>(v, bias, key_mask, gate, out, lse_w, ws, pl, d, s);
    }
}

pba_status pba_pwa_bwd(const pba_bf16 *v, const pba_bf16 *bias, const uint8_t *key_mask, const pba_bf16 *gate,
                       const pba_bf16 *out, const pba_bf16 *dout, pba_bf16 *dv, float *dbias, pba_bf16 *dgate,
                       void *workspace, size_t workspace_bytes, const pba_dims *d, void *stream) {
    g_last_error.clear();
    pba_status st = check_pwa_dims(d);
    if (st != PBA_OK) return st;
    if (d->B == 0 || d->Nq == 0 || d->H == 0) return PBA_OK;
    if (!dout || !dv) return fail(PBA_ERR_INVALID_ARG, "dout and dv are required");
    if (gate && (!out || !dgate)) return fail(PBA_ERR_INVALID_ARG, "out and dgate are required with a gate");
    const void *al[] = {dout, dv, out, dgate};
    for (const void *p : al)
        if (p && !aligned16(p)) return fail(PBA_ERR_INVALID_ARG, "bf16 tensors must be 16-byte aligned");
    if ((st = check_pwa_common(v, bias, key_mask, gate, d)) != PBA_OK) return st;
    const PwaPlan pl = plan_pwa(d);
    if (!workspace || workspace_bytes < pl.bwd_total)
        return fail(PBA_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", pl.bwd_total, workspace_bytes);
    if (reinterpret_cast<uintptr_t>(workspace) & 255u)
        return fail(PBA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    switch (padded_c(d->C)) {
        case 16: return launch_pwa_bwd<16>(v, bias, key_mask, gate, out, dout, dv, dbias, dgate, ws, pl, d, s);
        case 32: return launch_pwa_bwd<32>(v, bias, key_mask, gate, out, dout, dv, dbias, dgate, ws, pl, d, s);
        default: return launch_pwa_bwd<64>(v, bias, key_mask, gate, out, dout, dv, dbias, dgate, ws, pl, d, s);
    }
}

pba_status pba_pair_bias_fwd(const pba_bf16 *z, const float *gamma, const float *beta, const float *w,
                             pba_bf16 *bias, const pba_pair_bias_dims *d, void *stream) {
    g_last_error.clear();
    pba_status st = check_pb_dims(d);
    if (st != PBA_OK) return st;
    if (d->Ni == 0 || d->Nj == 0) return PBA_OK;
    if (!z || !gamma || !beta || !w || !bias) return fail(PBA_ERR_INVALID_ARG, "z, gamma, beta, w and bias are required");
    if (!aligned16(z)) return fail(PBA_ERR_INVALID_ARG, "z must be 16-byte aligned");
    if ((d->H > 1 && d->sbias[0] <= 0) || (d->Ni > 1 && d->sbias[1] <= 0))
        return fail(PBA_ERR_INVALID_ARG, "bias strides must be positive");
    if ((st = get_encoder()) != PBA_OK) return st;
    CUtensorMap tm;
    if ((st = map_z(&tm, z, d)) != PBA_OK) return st;
    pba::PbArgs a = pb_args(d, gamma, beta, w);
    a.bias = reinterpret_cast<__nv_bfloat16 *>(bias);
    return dispatch_pb(false, tm, a, d, reinterpret_cast<cudaStream_t>(stream));
}

size_t pba_pair_bias_bwd_workspace_size(const pba_pair_bias_dims *d) {
    if (check_pb_dims(d) != PBA_OK) return 0;
    return pb_ws_bytes(d);
}

pba_status pba_pair_bias_bwd(const pba_bf16 *z, const float *gamma, const float *beta, const float *w,
                             const float *dbias, pba_bf16 *dz, float *dw, float *dgamma, float *dbeta,
                             void *workspace, size_t workspace_bytes, const pba_pair_bias_dims *d, void *stream) {
    g_last_error.clear();
    pba_status st = check_pb_dims(d);
    if (st != PBA_OK) return st;
    if (!gamma || !beta || !w || !dw || !dgamma || !dbeta)
        return fail(PBA_ERR_INVALID_ARG, "gamma, beta, w, dw, dgamma and dbeta are required");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (d->Ni == 0 || d->Nj == 0) {
        // no position: every parameter gradient is an empty sum
        cudaError_t e;
        if ((e = cudaMemsetAsync(dw, 0, sizeof(float) * (size_t)d->Cz * d->H, s)) != cudaSuccess ||
            (e = cudaMemsetAsync(dgamma, 0, sizeof(float) * (size_t)d->Cz, s)) != cudaSuccess ||
            (e = cudaMemsetAsync(dbeta, 0, sizeof(float) * (size_t)d->Cz, s)) != cudaSuccess)
            return cuda_fail(e, "cudaMemsetAsync");
        return PBA_OK;
    }
    if (!z || !dbias || !dz) return fail(PBA_ERR_INVALID_ARG, "z, dbias and dz are required");
    if (!aligned16(z) || !aligned16(dz)) return fail(PBA_ERR_INVALID_ARG, "z and dz must be 16-byte aligned");
    if ((d->H > 1 && d->sdbias[0] <= 0) || (d->Ni > 1 && d->sdbias[1] <= 0))
        return fail(PBA_ERR_INVALID_ARG, "dbias strides must be positive");
    const size_t need = pb_ws_bytes(d);
    if (!workspace || workspace_bytes < need)
        return fail(PBA_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, workspace_bytes);
    if (reinterpret_cast<uintptr_t>(workspace) & 255u)
        return fail(PBA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    if ((st = get_encoder()) != PBA_OK) return st;
    CUtensorMap tm;
    if ((st = map_z(&tm, z, d)) != PBA_OK) return st;
    pba::PbArgs a = pb_args(d, gamma, beta, w);
    a.dbias = dbias;
    a.dz = reinterpret_cast<__nv_bfloat16 *>(dz);
    a.part = static_cast<float *>(workspace);
    a.dw = dw; a.dgamma = dgamma; a.dbeta = dbeta;
    return dispatch_pb(true, tm, a, d, s);
}

const char *pba_status_string(pba_status s) {
    switch (s) {
        case PBA_OK: return "PBA_OK";
        case PBA_ERR_INVALID_ARG: return "PBA_ERR_INVALID_ARG";
        case PBA_ERR_UNSUPPORTED: return "PBA_ERR_UNSUPPORTED";
        case PBA_ERR_CUDA: return "PBA_ERR_CUDA";
        case PBA_ERR_TIMEOUT: return "PBA_ERR_TIMEOUT";
        case PBA_ERR_WORKSPACE: return "PBA_ERR_WORKSPACE";
    }
    return "PBA_ERR_UNKNOWN";
}

const char *pba_last_error(void) { return g_last_error.c_str(); }

int pba_version(void) { return PBA_VERSION; }

void pba_debug_skip_load(int step) { g_debug_skip_step = step < 0 ? -1 : step; }

}  // extern "C"
