/*
 * libpba: pair-biased gated attention for NVIDIA B200 (sm_100a).
 *
 * The operation is the attention of AlphaFold3-style models as described on the
 * "AlphaFold3 open-source implementation" page (Ligo Biosciences README), section
 * "Model Efficiency": a pair bias, projected from the pair representation, is added
 * after the key-query dot product; the bias is broadcast over a batch-like axis (the
 * rows of a triangle attention, the sequences of an MSA, or the 48 noise-level copies
 * of the diffusion module, which that section folds into the batch dimension), so its
 * gradient is the gradient of the scaled logits summed over that axis.  With the
 * sigmoid gate, for every broadcast row b, head h and query i:
 *
 *   s[b,h,i,j] = scale * <q[b,i,h,:], k[b,j,h,:]> + bias[h,i,j]   (masked keys: -inf)
 *   out[b,i,h,:] = sigmoid(gate[b,i,h,:]) * sum_j softmax_j(s[b,h,i,:]) v[b,j,h,:]
 *   lse[b,h,i]   = ln sum_j exp(s[b,h,i,j])
 *
 * and the backward pass returns dq, dk, dv, dgate and dbias[h,i,j] = sum_b dS[b,h,i,j].
 * A query row whose keys are all masked gets out = 0, lse = -inf and no gradient.
 *
 * Conventions for every entry point:
 *  - Element types: q, k, v, gate, out, dout, dq, dk, dv, dgate and bias are bf16 (passed
 *    as uint16_t bit patterns); lse and dbias are fp32; key_mask is uint8 (nonzero = the
 *    key is attended, 0 = masked).  Arithmetic is bf16 x bf16 -> fp32 on the tensor
 *    cores, fp32 elsewhere.
 *  - All pointers are DEVICE pointers, owned by the caller; the library keeps none of
 *    them after a call returns and allocates nothing per call.  Outputs are written in
 *    full (never accumulated into).
 *  - Calls are asynchronous and ordered on `stream` (a cudaStream_t; NULL = the legacy
 *    default stream).  Argument errors are detected on the host and returned before
 *    anything is launched.
 *  - Every wait inside the kernels is bounded (about two seconds of SM cycles).  A wait that runs out
 *    makes the kernel stop early and record a device error word; pba_device_status()
 *    reports it as PBA_ERR_TIMEOUT.
 */
#ifndef PBA_H
#define PBA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define PBA_VERSION 1

typedef uint16_t pba_bf16; /* bf16 bit pattern */

typedef enum {
    PBA_OK = 0,
    PBA_ERR_INVALID_ARG = 1,  /* null required pointer, negative size, bad stride/alignment */
    PBA_ERR_UNSUPPORTED = 2,  /* valid request outside what the kernels implement (e.g. C>64) */
    PBA_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed (see pba_last_error) */
    PBA_ERR_TIMEOUT = 4,      /* a bounded in-kernel wait ran out (device watchdog) */
    PBA_ERR_WORKSPACE = 5     /* workspace too small */
} pba_status;

/*
 * Problem sizes and layouts.
 *  q, gate, out, dout, dq, dgate : [B, Nq, H, C]      k, v, dk, dv : [B, Nk, H, C]
 *  The channel (C) stride is 1; s?[0], s?[1], s?[2] are the element strides of the
 *  B, N and H dimensions (so = out and dout, sq = q and dq, sk = k and dk, sv = v and
 *  dv, sg = gate and dgate).  Every such stride must be a multiple of 8 elements and
 *  every base pointer 16-byte aligned (the tiles are moved by the Tensor Memory
 *  Accelerator), C a multiple of 8 in [8, 64].
 *  bias : [H, Nq, Nk], key stride 1; sbias[0], sbias[1] = element strides of H and Nq
 *         (multiples of 8).
 *  key_mask : [B, Nk] uint8, key stride 1, row stride smask_b (0 = one row for all b).
 *  lse : [B, H, Nq] fp32, contiguous.      dbias : [H, Nq, Nk] fp32, contiguous.
 *  scale : multiplier of <q,k>; 0 selects 1/sqrt(C) (the true C, not a padded one).
 */
typedef struct {
    int32_t B, H, Nq, Nk, C;
    float scale;
    int64_t sq[3], sk[3], sv[3], sg[3], so[3];
    int64_t sbias[2];
    int64_t smask_b;
} pba_dims;

/* Fill `d` with dense strides for the layouts above (mask shared by all b). */
void pba_dims_dense(pba_dims *d, int32_t B, int32_t H, int32_t Nq, int32_t Nk, int32_t C,
                    float scale);

/*
 * Forward pass (the operator stated in the header comment).
 *  bias may be NULL (no pair bias), key_mask may be NULL (every key attended), gate
 *  may be NULL (no gate: out = softmax(s) v).  out and lse are required.
 * Returns PBA_OK once the kernel is queued on `stream`.
 */
pba_status pba_fwd(const pba_bf16 *q, const pba_bf16 *k, const pba_bf16 *v,
                   const pba_bf16 *bias, const uint8_t *key_mask, const pba_bf16 *gate,
                   pba_bf16 *out, float *lse, const pba_dims *dims, void *stream);

/* Bytes of device workspace pba_bwd needs for these dims (0 for an empty problem). */
size_t pba_bwd_workspace_size(const pba_dims *dims);

/*
 * Backward pass: given the forward inputs, the forward outputs (out, lse) and dout,
 * writes dq, dk, dv (required), dgate (required iff gate is not NULL, else ignored)
 * and dbias (may be NULL to skip it; computed even when bias is NULL, as the gradient
 * with respect to a zero bias).  dbias is the sum over the B broadcast rows of the
 * logits' gradient, reduced in a fixed order, so it is bit-identical from run to run.
 * workspace: caller-owned device memory of at least pba_bwd_workspace_size(dims) bytes,
 * 256-byte aligned; its contents on entry do not matter and on return are undefined.
 * With dbias, the dbias kernel runs on a second stream of the library's beside the dq
 * conversion; `stream` waits for it before the call's work ends, so everything stays
 * ordered on `stream` (in a stream capture both become part of the graph).  That stream and
 * its two events are created by the first such call in a CUDA context and kept for the
 * context's lifetime; if that first call is made while `stream` is being captured, the call
 * runs on `stream` alone (same results), so make one call before capturing to get the overlap.
 */
pba_status pba_bwd(const pba_bf16 *q, const pba_bf16 *k, const pba_bf16 *v,
                   const pba_bf16 *bias, const uint8_t *key_mask, const pba_bf16 *gate,
                   const pba_bf16 *out, const float *lse, const pba_bf16 *dout,
                   pba_bf16 *dq, pba_bf16 *dk, pba_bf16 *dv, float *dbias, pba_bf16 *dgate,
                   void *workspace, size_t workspace_bytes, const pba_dims *dims,
                   void *stream);

/*
 * Block-sparse local attention (the sequence-local atom attention of the AlphaFold3 family,
 * "AlphaFold3 open-source implementation" page, Model Efficiency section, which names the
 * atom attention encoder and decoder among the attention-with-pair-bias modules): query
 * tile t (rows 128 t .. 128 t + 127) attends only the key tiles [t - window, t + window]
 * (clamped to the problem); every other key is masked for its rows and never read.  A
 * finer local pattern inside the visited tiles is expressed through the bias (-inf) or the
 * key mask.  The results equal pba_fwd / pba_bwd with those keys masked; dbias is 0 for the
 * pairs outside the band.  window < 0 is pba_fwd / pba_bwd.  Every query tile must keep a
 * key tile and every key tile a query tile (ceil(Nq/128) <= ceil(Nk/128) + window and the
 * reverse), else PBA_ERR_UNSUPPORTED.  Other arguments, layouts and errors as pba_fwd /
 * pba_bwd; the workspace is pba_bwd_workspace_size(dims).
 */
pba_status pba_fwd_local(const pba_bf16 *q, const pba_bf16 *k, const pba_bf16 *v,
                         const pba_bf16 *bias, const uint8_t *key_mask, const pba_bf16 *gate,
                         pba_bf16 *out, float *lse, const pba_dims *dims, int window,
                         void *stream);
pba_status pba_bwd_local(const pba_bf16 *q, const pba_bf16 *k, const pba_bf16 *v,
                         const pba_bf16 *bias, const uint8_t *key_mask, const pba_bf16 *gate,
                         const pba_bf16 *out, const float *lse, const pba_bf16 *dout,
                         pba_bf16 *dq, pba_bf16 *dk, pba_bf16 *dv, float *dbias, pba_bf16 *dgate,
                         void *workspace, size_t workspace_bytes, const pba_dims *dims,
                         int window, void *stream);

/*
 * Backward pass for callers that cannot allocate device memory.  The method's sources have
 * no counterpart: this entry point exists for users of the library, not for the method.
 * Some callers have no way to obtain scratch memory: a plugin running inside another
 * framework's executor that owns all device memory and forbids cudaMalloc while it
 * runs, or a binding from a language with no device allocator.  This variant takes the
 * same arguments as pba_bwd except the workspace, and uses instead a scratch array built
 * into the library (64 MiB in device global memory, held by every GPU that loads the
 * library until the process exits).  It allocates nothing: no cudaMalloc, no cudaFree.
 *  - Arguments are checked exactly as pba_bwd checks them (PBA_ERR_INVALID_ARG and the
 *    like come first); then sizes whose workspace (pba_bwd_workspace_size) exceeds 64 MiB
 *    are rejected with PBA_ERR_UNSUPPORTED before anything is launched; use pba_bwd for
 *    those.
 *  - The first call in a CUDA context looks up the scratch array's device address in that
 *    context (one cudaGetSymbolAddress, with the calling thread's current device and
 *    context) and keeps it under the context's unique id, so a context created later (a
 *    second context on the device, or the one after cudaDeviceReset) gets its own lookup.
 *    Make the first call in each context before any stream capture.
 *  - Every call on a device shares the one array and leaves the last call's contents in
 *    it (the parts that must start at zero are cleared by each call).  Calls whose
 *    execution overlaps on the GPU (different streams, no ordering between them) race on
 *    the array and give wrong results: order them.
 */
pba_status pba_bwd_noalloc(const pba_bf16 *q, const pba_bf16 *k, const pba_bf16 *v,
                           const pba_bf16 *bias, const uint8_t *key_mask, const pba_bf16 *gate,
                           const pba_bf16 *out, const float *lse, const pba_bf16 *dout,
                           pba_bf16 *dq, pba_bf16 *dk, pba_bf16 *dv, float *dbias,
                           pba_bf16 *dgate, const pba_dims *dims, void *stream);

/*
 * MSA pair-weighted averaging ("AlphaFold3 open-source implementation" page, sections "MSA
 * Pair Averaging" and "Model Efficiency"): the value rows of every broadcast row b (MSA
 * sequence) are averaged with weights taken from the pair representation alone, shared by
 * all rows -- the operator above without its key-query term:
 *   w[h,i,j] = softmax_j(bias[h,i,j] + mask_j),  lse_w[h,i] = ln sum_j exp(bias + mask)
 *   out[b,i,h,:] = sigmoid(gate[b,i,h,:]) * sum_j w[h,i,j] v[b,j,h,:]      (no gate: no factor)
 * The weights are computed once per (h, i), not per b.  Arguments follow pba_fwd with
 * Nq = Nk = N (else PBA_ERR_UNSUPPORTED): v, gate, out use dims->sv, sg, so; bias (nullable,
 * = 0) dims->sbias; key_mask (nullable) is one [N] row shared by every b (dims->smask_b must
 * be 0 when B > 1, else PBA_ERR_UNSUPPORTED).  dims->scale and q/k strides are ignored.
 * lse_w: fp32 [H, N], written; -inf for a row whose keys are all masked (its out is 0).
 * workspace: caller-owned device memory of pba_pwa_fwd_workspace_size(dims) bytes,
 * 256-byte aligned (PBA_ERR_WORKSPACE if smaller); it holds the bf16 weights.
 */
size_t pba_pwa_fwd_workspace_size(const pba_dims *dims);
pba_status pba_pwa_fwd(const pba_bf16 *v, const pba_bf16 *bias, const uint8_t *key_mask,
                       const pba_bf16 *gate, pba_bf16 *out, float *lse_w, void *workspace,
                       size_t workspace_bytes, const pba_dims *dims, void *stream);

/*
 * Backward of pba_pwa_fwd, given v, bias, key_mask, gate, the forward output `out` (only
 * needed with a gate) and dout:
 *   dOa = dout * sigmoid(gate);  dgate = dout * out * (1 - sigmoid(gate))
 *   dv[b,j,h,:] = sum_i w[h,i,j] dOa[b,i,h,:]
 *   dW[h,i,j] = sum_b sum_c dOa[b,i,h,c] v[b,j,h,c];  dbias = w * (dW - sum_j w dW)
 * dv (required, strides of v), dgate (required iff gate), dbias (fp32 [H,N,N], may be NULL
 * to skip it; bit-identical from run to run: fixed reduction orders).  The weights are
 * recomputed from bias and key_mask.  workspace: pba_pwa_bwd_workspace_size(dims) bytes,
 * 256-byte aligned.
 */
size_t pba_pwa_bwd_workspace_size(const pba_dims *dims);
pba_status pba_pwa_bwd(const pba_bf16 *v, const pba_bf16 *bias, const uint8_t *key_mask,
                       const pba_bf16 *gate, const pba_bf16 *out, const pba_bf16 *dout,
                       pba_bf16 *dv, float *dbias, pba_bf16 *dgate, void *workspace,
                       size_t workspace_bytes, const pba_dims *dims, void *stream);

/*
 * Pair-bias projection, the prologue that makes an attention's bias from the pair
 * representation ("AlphaFold3 open-source implementation" page, Model Efficiency section:
 * every attention projects its pair bias from the pair representation; the Protenix page,
 * scalability section: the LayerNorm of the pair representation is worth a custom
 * kernel).  A LayerNorm over the Cz channels of z[i,j,:], then a linear map without bias:
 *   bias[h,i,j] = sum_c (gamma_c (z[i,j,c] - mean) / sqrt(var + eps) + beta_c) w[c,h]
 * (mean and biased variance over the channels of one position).  The output feeds
 * pba_fwd / pba_bwd as their bias (Ni = Nq, Nj = Nk); a transposed bias (the ending-node
 * triangle attention) is the same call with the two z strides exchanged.
 *
 * Sizes: Cz in {64, 128, 192, 256}; 1 <= H <= 16; eps finite and > 0; Ni, Nj >= 0.
 * z: bf16, element (i, j, c) at z[i * sz[0] + j * sz[1] + c]; base 16-byte aligned,
 * sz[0] and sz[1] positive multiples of 8 (the Tensor Memory Accelerator's rule).
 * gamma, beta: fp32 [Cz]; w: fp32 [Cz][H] (row c, column h), all device pointers.
 * bias: bf16, element (h, i, j) at bias[h * sbias[0] + i * sbias[1] + j].
 */
typedef struct {
    int Ni, Nj, Cz, H;
    float eps;
    int64_t sz[2];      /* z (and dz) strides of i and j, in elements; channel stride 1 */
    int64_t sbias[2];   /* bias strides of h and i, in elements; j stride 1 */
    int64_t sdbias[2];  /* dbias strides of h and i, in elements; j stride 1 */
} pba_pair_bias_dims;

pba_status pba_pair_bias_fwd(const pba_bf16 *z, const float *gamma, const float *beta,
                             const float *w, pba_bf16 *bias, const pba_pair_bias_dims *dims,
                             void *stream);

/*
 * Backward of pba_pair_bias_fwd for a given dbias (fp32, e.g. the dbias of pba_bwd):
 *   dz (bf16, the layout of z), dw (fp32 [Cz][H]), dgamma, dbeta (fp32 [Cz]), all written
 *   in full.  dw, dgamma and dbeta are sums over all Ni * Nj positions, added in an order
 *   that depends only on the sizes: bit-identical from run to run.
 * workspace: caller-owned device memory of pba_pair_bias_bwd_workspace_size(dims) bytes,
 * 256-byte aligned (PBA_ERR_WORKSPACE if smaller).
 */
size_t pba_pair_bias_bwd_workspace_size(const pba_pair_bias_dims *dims);
pba_status pba_pair_bias_bwd(const pba_bf16 *z, const float *gamma, const float *beta,
                             const float *w, const float *dbias, pba_bf16 *dz, float *dw,
                             float *dgamma, float *dbeta, void *workspace,
                             size_t workspace_bytes, const pba_pair_bias_dims *dims,
                             void *stream);

/*
 * Ordered sum of bias-gradient partials, for the row-sharded backward pass across GPUs.
 * The Design-CP page ("Context Parallelism for Design of Protein Nanoparticles", Method)
 * shards each attention block's rows over GPUs and exchanges activations between blocks;
 * for pair-biased attention the bias gradient is a sum over the broadcast rows
 * ("AlphaFold3 open-source implementation" page, Model Efficiency), so row shards each
 * hold a partial of it.  Given n_parts partials of n fp32 elements each, stored one after
 * the other in `parts` (device memory, part p at parts + p * n), writes
 *   out[i] = (...((parts[0][i] + parts[1][i]) + parts[2][i]) ... + parts[n_parts-1][i])
 * in exactly that order, so the result depends only on the partials and their order, not
 * on which GPU computed which.  `out` may not overlap `parts`.  n_parts >= 1, n >= 0;
 * pointers 16-byte aligned.  Asynchronous on `stream`; allocates nothing.
 */
pba_status pba_dbias_sum(const float *parts, int n_parts, int64_t n, float *out, void *stream);

/*
 * Synchronizes `stream`, then reports and clears the device watchdog word of the
 * current device: PBA_ERR_TIMEOUT if any kernel of this library gave up a bounded wait
 * since the last call, PBA_ERR_CUDA if the synchronization itself failed, else PBA_OK.
 */
pba_status pba_device_status(void *stream);

/*
 * Kernel timing for benchmarks.  While enabled, every kernel this library launches is
 * bracketed by two CUDA events recorded on the kernel's own stream, and counted.
 * pba_profile_read() waits for the recorded events, writes one entry per kernel name
 * (launch count and summed device time) into `out` (at most `max` entries), clears the
 * records and returns the number of entries (or -1 on a CUDA error).  The events are
 * CUDA event objects owned by the library and reused; no device memory is allocated.
 */
typedef struct {
    char name[48];
    int64_t launches;
    double total_ms;
} pba_kernel_stat;

pba_status pba_profile_enable(int on);
int pba_profile_read(pba_kernel_stat *out, int max);

/*
 * Test hook for the device watchdog (no production use).  With step >= 0, the next
 * pba_fwd calls make their TMA producer skip the K load of that step of every CTA, so
 * the barrier it would have completed never does: the MMA issuer's bounded wait runs
 * out (about one second), every role of the CTA drains what it issued and returns, and
 * pba_device_status() then reports PBA_ERR_TIMEOUT.  No GPU fault is raised and the
 * context stays usable.  step < 0 switches the hook off (the default).
 */
void pba_debug_skip_load(int step);

/* Static description of a status code. */
const char *pba_status_string(pba_status s);

/* Detail of the last error returned on the calling host thread ("" if none). */
const char *pba_last_error(void);

int pba_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PBA_H */
