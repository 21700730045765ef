/*
 * Oracle for pair-biased gated attention: plain, slow, fp64 CPU loops.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call this code: only the
 * tests, the package's smoke check and the benchmark's CPU-baseline leg use it.  It
 * shares no code, header, table or helper with the CUDA library.
 *
 * What it computes (the plain definition, fully materialised, no tiling):
 *
 *   The operator is the one described on the "AlphaFold3 open-source implementation"
 *   page (Ligo Biosciences README), section "Model Efficiency": every attention
 *   projects a pair bias from the pair representation and adds it after the key-query
 *   dot product; the bias needs a gradient, which equals the gradient of the scaled
 *   QK^T logits; and because the bias is broadcast over a batch-like axis in the
 *   forward pass, its gradient is a reduction over that axis in the backward pass.
 *   The same page's Model Efficiency section folds the 48 diffusion noise-level copies
 *   into that batch axis.  The pages do not print the formula; the readings used are:
 *
 *     s[b,h,i,j]   = scale * sum_c q[b,i,h,c] k[b,j,h,c] + bias[h,i,j]     (unmasked j)
 *     P[b,h,i,j]   = exp(s - m_i) / sum_j' exp(s_ij' - m_i),  m_i = max_j s_ij  (masked j: P = 0)
 *     o[b,i,h,c]   = sum_j P v[b,j,h,c]
 *     out          = sigmoid(g) * o                     (elementwise over c)
 *     lse[b,h,i]   = m_i + ln sum_j exp(s_ij - m_i)     (natural log, includes scale/bias/mask)
 *
 *   Backward, for a given dout:
 *     dOa  = dout * sigmoid(g)
 *     dg   = dout * o * sigmoid(g) * (1 - sigmoid(g))
 *     dP   = dOa_i . v_j
 *     D_i  = sum_j P_ij dP_ij
 *     dS   = P * (dP - D_i)
 *     dq_i = scale * sum_j dS_ij k_j ;  dk_j = scale * sum_i dS_ij q_i ;  dv_j = sum_i P_ij dOa_i
 *     dbias[h,i,j] = sum_b dS[b,h,i,j]          (the broadcast over b becomes a sum over b)
 *
 *   A row whose keys are all masked has no softmax: out = 0, lse = -inf, and it sends
 *   no gradient anywhere (reading of a case the pages do not cover).
 *
 * Layouts: q, k, v, g, out, dout, dq, dk, dv, dg are [B, N, H, C] (C innermost);
 * bias and dbias are [H, Nq, Nk]; keep is [B, Nk] with a row stride keep_sb (0 = one
 * row shared by all b), 1 = attended, 0 = masked; lse is [B, H, Nq].  Slice entry points
 * take one (b, h) problem as dense [N][C] / [Nq][Nk] arrays.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Number of OpenMP threads the parallel loops below may use. */
int pba_oracle_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

/* ---------------------------------------------------------------------------------- */
/* one (b, h) problem                                                                  */
/* ---------------------------------------------------------------------------------- */

/* Logits and softmax of one query row i: fills s[Nk] and p[Nk]; returns the logsumexp
   (-inf when every key is masked, in which case p is all zero). */
static double row_softmax(int i, int Nk, int C, double scale, const double *q,
                          const double *k, const double *bias, const uint8_t *keep,
                          double *s, double *p)
{
    double m = -INFINITY;
    for (int j = 0; j < Nk; ++j) {
        double dot = 0.0;
        for (int c = 0; c < C; ++c) dot += q[(size_t)i * C + c] * k[(size_t)j * C + c];
        s[j] = scale * dot + (bias ? bias[(size_t)i * Nk + j] : 0.0);
        if ((!keep || keep[j]) && s[j] > m) m = s[j];
    }
    if (m == -INFINITY) {
        for (int j = 0; j < Nk; ++j) p[j] = 0.0;
        return -INFINITY;
    }
    double z = 0.0;
    for (int j = 0; j < Nk; ++j)
        if (!keep || keep[j]) z += exp(s[j] - m);
    for (int j = 0; j < Nk; ++j) p[j] = (!keep || keep[j]) ? exp(s[j] - m) / z : 0.0;
    return m + log(z);
}

void pba_oracle_fwd_slice(int Nq, int Nk, int C, double scale, const double *q,
                          const double *k, const double *v, const double *bias,
                          const uint8_t *keep, const double *g, double *out, double *lse,
                          double *P /* optional [Nq][Nk] */)
{
    double *s = (double *)malloc(sizeof(double) * (size_t)(Nk > 0 ? Nk : 1));
    double *p = (double *)malloc(sizeof(double) * (size_t)(Nk > 0 ? Nk : 1));
    for (int i = 0; i < Nq; ++i) {
        lse[i] = row_softmax(i, Nk, C, scale, q, k, bias, keep, s, p);
        for (int c = 0; c < C; ++c) {
            double o = 0.0;
            for (int j = 0; j < Nk; ++j) o += p[j] * v[(size_t)j * C + c];
            double gate = g ? sigmoid(g[(size_t)i * C + c]) : 1.0;
            out[(size_t)i * C + c] = gate * o;
        }
        if (P) memcpy(P + (size_t)i * Nk, p, sizeof(double) * (size_t)Nk);
    }
    free(s);
    free(p);
}

/* Backward of one (b, h) problem.  Writes dq, dk, dv, dg (dg may be NULL when g is NULL)
   and, when ds is not NULL, this slice's dS[Nq][Nk]. */
void pba_oracle_bwd_slice(int Nq, int Nk, int C, double scale, const double *q,
                          const double *k, const double *v, const double *bias,
                          const uint8_t *keep, const double *g, const double *dout,
                          double *dq, double *dk, double *dv, double *dg, double *ds)
{
    size_t nP = (size_t)(Nq > 0 ? Nq : 1) * (size_t)(Nk > 0 ? Nk : 1);
    double *P = (double *)malloc(sizeof(double) * nP);
    double *dP = (double *)malloc(sizeof(double) * nP);
    double *dS = (double *)malloc(sizeof(double) * nP);
    double *o = (double *)malloc(sizeof(double) * (size_t)(Nq > 0 ? Nq : 1) * (C > 0 ? C : 1));
    double *dOa = (double *)malloc(sizeof(double) * (size_t)(Nq > 0 ? Nq : 1) * (C > 0 ? C : 1));
    double *s = (double *)malloc(sizeof(double) * (size_t)(Nk > 0 ? Nk : 1));

    /* forward quantities: P and the ungated o */
    for (int i = 0; i < Nq; ++i) {
        row_softmax(i, Nk, C, scale, q, k, bias, keep, s, P + (size_t)i * Nk);
        for (int c = 0; c < C; ++c) {
            double acc = 0.0;
            for (int j = 0; j < Nk; ++j) acc += P[(size_t)i * Nk + j] * v[(size_t)j * C + c];
            o[(size_t)i * C + c] = acc;
        }
    }
    /* gate */
    for (int i = 0; i < Nq; ++i)
        for (int c = 0; c < C; ++c) {
            size_t e = (size_t)i * C + c;
            double sg = g ? sigmoid(g[e]) : 1.0;
            dOa[e] = dout[e] * sg;
            if (dg) dg[e] = g ? dout[e] * o[e] * sg * (1.0 - sg) : 0.0;
        }
    /* dP, D, dS */
    for (int i = 0; i < Nq; ++i) {
        double D = 0.0;
        for (int j = 0; j < Nk; ++j) {
            double acc = 0.0;
            for (int c = 0; c < C; ++c) acc += dOa[(size_t)i * C + c] * v[(size_t)j * C + c];
            dP[(size_t)i * Nk + j] = acc;
            D += P[(size_t)i * Nk + j] * acc;
        }
        for (int j = 0; j < Nk; ++j)
            dS[(size_t)i * Nk + j] = P[(size_t)i * Nk + j] * (dP[(size_t)i * Nk + j] - D);
    }
    /* dq, dk, dv */
    for (int i = 0; i < Nq; ++i)
        for (int c = 0; c < C; ++c) {
            double acc = 0.0;
            for (int j = 0; j < Nk; ++j) acc += dS[(size_t)i * Nk + j] * k[(size_t)j * C + c];
            dq[(size_t)i * C + c] = scale * acc;
        }
    for (int j = 0; j < Nk; ++j)
        for (int c = 0; c < C; ++c) {
            double acck = 0.0, accv = 0.0;
            for (int i = 0; i < Nq; ++i) {
                acck += dS[(size_t)i * Nk + j] * q[(size_t)i * C + c];
                accv += P[(size_t)i * Nk + j] * dOa[(size_t)i * C + c];
            }
            dk[(size_t)j * C + c] = scale * acck;
            dv[(size_t)j * C + c] = accv;
        }
    if (ds) memcpy(ds, dS, sizeof(double) * (size_t)Nq * (size_t)Nk);
    free(P); free(dP); free(dS); free(o); free(dOa); free(s);
}

/* ---------------------------------------------------------------------------------- */
/* full tensors in the library layout                                                  */
/* ---------------------------------------------------------------------------------- */

static void gather(const double *src, int b, int h, int N, int H, int C, double *dst)
{
    for (int n = 0; n < N; ++n)
        memcpy(dst + (size_t)n * C, src + (((size_t)b * N + n) * H + h) * C, sizeof(double) * C);
}

static void scatter(double *dst, int b, int h, int N, int H, int C, const double *src)
{
    for (int n = 0; n < N; ++n)
        memcpy(dst + (((size_t)b * N + n) * H + h) * C, src + (size_t)n * C, sizeof(double) * C);
}

void pba_oracle_fwd(int B, int H, int Nq, int Nk, int C, double scale, const double *q,
                    const double *k, const double *v, const double *bias,
                    const uint8_t *keep, long long keep_sb, const double *g, double *out,
                    double *lse)
{
    #pragma omp parallel for schedule(dynamic)
    for (long long bh = 0; bh < (long long)B * H; ++bh) {
        int b = (int)(bh / H), h = (int)(bh % H);
        double *qs = malloc(sizeof(double) * (size_t)Nq * C + 8);
        double *ks = malloc(sizeof(double) * (size_t)Nk * C + 8);
        double *vs = malloc(sizeof(double) * (size_t)Nk * C + 8);
        double *gs = g ? malloc(sizeof(double) * (size_t)Nq * C + 8) : NULL;
        double *os = malloc(sizeof(double) * (size_t)Nq * C + 8);
        gather(q, b, h, Nq, H, C, qs);
        gather(k, b, h, Nk, H, C, ks);
        gather(v, b, h, Nk, H, C, vs);
        if (g) gather(g, b, h, Nq, H, C, gs);
        pba_oracle_fwd_slice(Nq, Nk, C, scale, qs, ks, vs,
                             bias ? bias + (size_t)h * Nq * Nk : NULL,
                             keep ? keep + (size_t)b * keep_sb : NULL, gs, os,
                             lse + ((size_t)b * H + h) * Nq, NULL);
        scatter(out, b, h, Nq, H, C, os);
        free(qs); free(ks); free(vs); free(gs); free(os);
    }
}

void pba_oracle_bwd(int B, int H, int Nq, int Nk, int C, double scale, const double *q,
                    const double *k, const double *v, const double *bias,
                    const uint8_t *keep, long long keep_sb, const double *g,
                    const double *dout, double *dq, double *dk, double *dv, double *dg,
                    double *dbias)
{
    /* one thread per head: the dbias sum over b runs in order b = 0, 1, ... */
    #pragma omp parallel for schedule(dynamic)
    for (int h = 0; h < H; ++h) {
        double *qs = malloc(sizeof(double) * (size_t)Nq * C + 8);
        double *ks = malloc(sizeof(double) * (size_t)Nk * C + 8);
        double *vs = malloc(sizeof(double) * (size_t)Nk * C + 8);
        double *gs = g ? malloc(sizeof(double) * (size_t)Nq * C + 8) : NULL;
        double *dos = malloc(sizeof(double) * (size_t)Nq * C + 8);
        double *dqs = malloc(sizeof(double) * (size_t)Nq * C + 8);
        double *dks = malloc(sizeof(double) * (size_t)Nk * C + 8);
        double *dvs = malloc(sizeof(double) * (size_t)Nk * C + 8);
        double *dgs = g ? malloc(sizeof(double) * (size_t)Nq * C + 8) : NULL;
        double *dss = malloc(sizeof(double) * (size_t)Nq * Nk + 8);
        double *dbh = dbias ? dbias + (size_t)h * Nq * Nk : NULL;
        if (dbh) for (size_t e = 0; e < (size_t)Nq * Nk; ++e) dbh[e] = 0.0;
        for (int b = 0; b < B; ++b) {
            gather(q, b, h, Nq, H, C, qs);
            gather(k, b, h, Nk, H, C, ks);
            gather(v, b, h, Nk, H, C, vs);
            if (g) gather(g, b, h, Nq, H, C, gs);
            gather(dout, b, h, Nq, H, C, dos);
            pba_oracle_bwd_slice(Nq, Nk, C, scale, qs, ks, vs,
                                 bias ? bias + (size_t)h * Nq * Nk : NULL,
                                 keep ? keep + (size_t)b * keep_sb : NULL, gs, dos, dqs, dks,
                                 dvs, dgs, dss);
            scatter(dq, b, h, Nq, H, C, dqs);
            scatter(dk, b, h, Nk, H, C, dks);
            scatter(dv, b, h, Nk, H, C, dvs);
            if (g && dg) scatter(dg, b, h, Nq, H, C, dgs);
            if (dbh) for (size_t e = 0; e < (size_t)Nq * Nk; ++e) dbh[e] += dss[e];
        }
        free(qs); free(ks); free(vs); free(gs); free(dos); free(dqs); free(dks); free(dvs);
        free(dgs); free(dss);
    }
}

/* dbias[h, i, :] = sum_b dS[b, h, i, :] for one query row: the softmax, dP and D of row
   i depend on row i only, so one row of dbias is computable without the full problem.
   Used to sample dbias at sizes where the full oracle would take too long. */
void pba_oracle_dbias_row(int B, int H, int Nq, int Nk, int C, double scale, int h, int i,
                          const double *q, const double *k, const double *v,
                          const double *bias, const uint8_t *keep, long long keep_sb,
                          const double *g, const double *dout, double *dbias_row)
{
    double *qi = malloc(sizeof(double) * (size_t)C + 8);
    double *dOa = malloc(sizeof(double) * (size_t)C + 8);
    double *ks = malloc(sizeof(double) * (size_t)Nk * C + 8);
    double *vs = malloc(sizeof(double) * (size_t)Nk * C + 8);
    double *s = malloc(sizeof(double) * (size_t)Nk + 8);
    double *p = malloc(sizeof(double) * (size_t)Nk + 8);
    double *dP = malloc(sizeof(double) * (size_t)Nk + 8);
    for (int j = 0; j < Nk; ++j) dbias_row[j] = 0.0;
    for (int b = 0; b < B; ++b) {
        size_t row = (((size_t)b * Nq + i) * H + h) * C;
        for (int c = 0; c < C; ++c) qi[c] = q[row + c];
        gather(k, b, h, Nk, H, C, ks);
        gather(v, b, h, Nk, H, C, vs);
        row_softmax(0, Nk, C, scale, qi, ks, bias ? bias + ((size_t)h * Nq + i) * Nk : NULL,
                    keep ? keep + (size_t)b * keep_sb : NULL, s, p);
        for (int c = 0; c < C; ++c) dOa[c] = dout[row + c] * (g ? sigmoid(g[row + c]) : 1.0);
        double D = 0.0;
        for (int j = 0; j < Nk; ++j) {
            double acc = 0.0;
            for (int c = 0; c < C; ++c) acc += dOa[c] * vs[(size_t)j * C + c];
            dP[j] = acc;
            D += p[j] * acc;
        }
        for (int j = 0; j < Nk; ++j) dbias_row[j] += p[j] * (dP[j] - D);
    }
    free(qi); free(dOa); free(ks); free(vs); free(s); free(p); free(dP);
}

/*
 * MSA pair-weighted averaging ("AlphaFold3 open-source implementation" page, sections
 * "MSA Pair Averaging" and "Model Efficiency"): the MSA module averages the value rows of
 * every MSA sequence with weights taken from the pair representation alone.  The pages
 * print no formula; the plainest reading, the gated operator above without its key-query
 * term, shared by all B rows (Nq = Nk = N, key mask one row shared by all b):
 *
 *   w[h,i,j]    = exp(bias[h,i,j] - m_i) / sum_j' exp(bias[h,i,j'] - m_i)  (masked j: w = 0)
 *   lse_w[h,i]  = m_i + ln sum_j exp(bias[h,i,j] - m_i)                    (-inf: all masked)
 *   o[b,i,h,c]  = sum_j w[h,i,j] v[b,j,h,c] ;   out = sigmoid(g) * o
 *
 *   Backward:  dOa = dout * sigmoid(g) ;  dg = dout * o * sigmoid(g) (1 - sigmoid(g))
 *              dv[b,j,h,c] = sum_i w[h,i,j] dOa[b,i,h,c]
 *              dW[h,i,j]   = sum_b sum_c dOa[b,i,h,c] v[b,j,h,c]
 *              dbias[h,i,j] = w[h,i,j] (dW[h,i,j] - sum_j' w[h,i,j'] dW[h,i,j'])
 *
 * Layouts: v, g, out, dout, dv, dg are [B, N, H, C]; bias, dbias are [H, N, N]; keep is
 * [N] (1 = attended) or NULL; lse_w is [H, N].
 */
static void pwa_weights(int N, const double *brow, const uint8_t *keep, double *w, double *lse)
{
    double m = -INFINITY;
    for (int j = 0; j < N; ++j)
        if (!keep || keep[j]) m = fmax(m, brow ? brow[j] : 0.0);
    if (m == -INFINITY) {   /* every key masked */
        for (int j = 0; j < N; ++j) w[j] = 0.0;
        *lse = -INFINITY;
        return;
    }
    double l = 0.0;
    for (int j = 0; j < N; ++j) {
        w[j] = (!keep || keep[j]) ? exp((brow ? brow[j] : 0.0) - m) : 0.0;
        l += w[j];
    }
    for (int j = 0; j < N; ++j) w[j] /= l;
    *lse = m + log(l);
}

void pba_oracle_pwa_fwd(int B, int H, int N, int C, const double *v, const double *bias,
                        const uint8_t *keep, const double *g, double *out, double *lse)
{
    #pragma omp parallel for schedule(dynamic)
    for (int h = 0; h < H; ++h) {
        double *w = malloc(sizeof(double) * (size_t)N + 8);
        for (int i = 0; i < N; ++i) {
            pwa_weights(N, bias ? bias + ((size_t)h * N + i) * N : NULL, keep, w,
                        lse + (size_t)h * N + i);
            for (int b = 0; b < B; ++b)
                for (int c = 0; c < C; ++c) {
                    double o = 0.0;
                    for (int j = 0; j < N; ++j) o += w[j] * v[(((size_t)b * N + j) * H + h) * C + c];
                    const size_t e = (((size_t)b * N + i) * H + h) * C + c;
                    out[e] = g ? sigmoid(g[e]) * o : o;
                }
        }
        free(w);
    }
}

void pba_oracle_pwa_bwd(int B, int H, int N, int C, const double *v, const double *bias,
                        const uint8_t *keep, const double *g, const double *dout, double *dv,
                        double *dg, double *dbias)
{
    #pragma omp parallel for schedule(dynamic)
    for (int h = 0; h < H; ++h) {
        double *w = malloc(sizeof(double) * (size_t)N * N + 8);
        double *lse = malloc(sizeof(double) * (size_t)N + 8);
        double *doa = malloc(sizeof(double) * (size_t)B * N * C + 8);   /* [b][i][c] */
        for (int i = 0; i < N; ++i)
            pwa_weights(N, bias ? bias + ((size_t)h * N + i) * N : NULL, keep, w + (size_t)i * N, lse + i);
        /* dOa and dg need the ungated o */
        for (int b = 0; b < B; ++b)
            for (int i = 0; i < N; ++i)
                for (int c = 0; c < C; ++c) {
                    const size_t e = (((size_t)b * N + i) * H + h) * C + c;
                    double o = 0.0;
                    for (int j = 0; j < N; ++j) o += w[(size_t)i * N + j] * v[(((size_t)b * N + j) * H + h) * C + c];
                    const double s = g ? sigmoid(g[e]) : 1.0;
                    doa[((size_t)b * N + i) * C + c] = dout[e] * s;
                    if (g && dg) dg[e] = dout[e] * o * s * (1.0 - s);
                }
        /* dv[b,j] = sum_i w[i,j] dOa[b,i] */
        for (int b = 0; b < B; ++b)
            for (int j = 0; j < N; ++j)
                for (int c = 0; c < C; ++c) {
                    double a = 0.0;
                    for (int i = 0; i < N; ++i) a += w[(size_t)i * N + j] * doa[((size_t)b * N + i) * C + c];
                    dv[(((size_t)b * N + j) * H + h) * C + c] = a;
                }
        /* dW[i,j] = sum_b sum_c dOa[b,i,c] v[b,j,c]; dbias = w (dW - sum_j w dW), row by row */
        if (dbias) {
            double *dw = malloc(sizeof(double) * (size_t)N + 8);
            for (int i = 0; i < N; ++i) {
                for (int j = 0; j < N; ++j) {
                    double a = 0.0;
                    for (int b = 0; b < B; ++b)
                        for (int c = 0; c < C; ++c)
                            a += doa[((size_t)b * N + i) * C + c] * v[(((size_t)b * N + j) * H + h) * C + c];
                    dw[j] = a;
                }
                double r = 0.0;
                for (int j = 0; j < N; ++j) r += w[(size_t)i * N + j] * dw[j];
                for (int j = 0; j < N; ++j)
                    dbias[((size_t)h * N + i) * N + j] = w[(size_t)i * N + j] * (dw[j] - r);
            }
            free(dw);
        }
        free(w); free(lse); free(doa);
    }
}

/*
 * Pair-bias projection, the prologue of every pair-biased attention: the bias is
 * projected from the pair representation ("AlphaFold3 open-source implementation" page,
 * section "Model Efficiency"), after a LayerNorm of that representation (the Protenix
 * page "Protenix: AlphaFold3的再现", section on scalability, which names LayerNorm as the
 * op its custom CUDA kernel speeds up).  The pages print no formula; the plainest reading
 * is a LayerNorm over the channels of z[i,j,:] followed by a linear map without bias:
 *
 *   mu = mean_c z[i,j,c],  var = mean_c (z - mu)^2,  xh_c = (z_c - mu) / sqrt(var + eps)
 *   y_c = gamma_c xh_c + beta_c
 *   bias[h,i,j] = sum_c y_c w[c,h]
 *
 * Backward for a given dbias[h,i,j] = g_h (the chain rule through the three steps):
 *   dw[c,h]   = sum_{i,j} y_c g_h
 *   dy_c      = sum_h w[c,h] g_h
 *   dgamma_c  = sum_{i,j} dy_c xh_c ;  dbeta_c = sum_{i,j} dy_c
 *   dxh_c     = gamma_c dy_c
 *   dz_c      = (dxh_c - mean_c dxh - xh_c mean_c(dxh xh)) / sqrt(var + eps)
 *
 * Layouts: z, dz [Ni][Nj][Cz]; w [Cz][H]; gamma, beta [Cz]; bias, dbias [H][Ni][Nj].
 */
static void pb_normalize(int Cz, double eps, const double *zr, double *xh, double *sigma)
{
    double mu = 0.0;
    for (int c = 0; c < Cz; ++c) mu += zr[c];
    mu /= Cz;
    double var = 0.0;
    for (int c = 0; c < Cz; ++c) var += (zr[c] - mu) * (zr[c] - mu);
    var /= Cz;
    *sigma = sqrt(var + eps);
    for (int c = 0; c < Cz; ++c) xh[c] = (zr[c] - mu) / *sigma;
}

void pba_oracle_pair_bias_fwd(int Ni, int Nj, int Cz, int H, double eps, const double *z,
                              const double *gamma, const double *beta, const double *w,
                              double *bias)
{
    #pragma omp parallel for schedule(dynamic)
    for (int i = 0; i < Ni; ++i) {
        double *xh = malloc(sizeof(double) * (size_t)Cz + 8);
        for (int j = 0; j < Nj; ++j) {
            double sigma;
            pb_normalize(Cz, eps, z + ((size_t)i * Nj + j) * Cz, xh, &sigma);
            for (int h = 0; h < H; ++h) {
                double s = 0.0;
                for (int c = 0; c < Cz; ++c) s += (gamma[c] * xh[c] + beta[c]) * w[(size_t)c * H + h];
                bias[((size_t)h * Ni + i) * Nj + j] = s;
            }
        }
        free(xh);
    }
}

void pba_oracle_pair_bias_bwd(int Ni, int Nj, int Cz, int H, double eps, const double *z,
                              const double *gamma, const double *beta, const double *w,
                              const double *dbias, double *dz, double *dw, double *dgamma,
                              double *dbeta)
{
    memset(dw, 0, sizeof(double) * (size_t)Cz * H);
    memset(dgamma, 0, sizeof(double) * (size_t)Cz);
    memset(dbeta, 0, sizeof(double) * (size_t)Cz);
    double *xh = malloc(sizeof(double) * (size_t)Cz + 8);
    double *dy = malloc(sizeof(double) * (size_t)Cz + 8);
    double *g = malloc(sizeof(double) * (size_t)H + 8);
    /* sums over (i, j) in the order i = 0, 1, ...; j = 0, 1, ... */
    for (int i = 0; i < Ni; ++i)
        for (int j = 0; j < Nj; ++j) {
            double sigma;
            pb_normalize(Cz, eps, z + ((size_t)i * Nj + j) * Cz, xh, &sigma);
            for (int h = 0; h < H; ++h) g[h] = dbias[((size_t)h * Ni + i) * Nj + j];
            for (int c = 0; c < Cz; ++c) {
                const double y = gamma[c] * xh[c] + beta[c];
                double s = 0.0;
                for (int h = 0; h < H; ++h) {
                    dw[(size_t)c * H + h] += y * g[h];
                    s += w[(size_t)c * H + h] * g[h];
                }
                dy[c] = s;
                dgamma[c] += s * xh[c];
                dbeta[c] += s;
            }
            double m1 = 0.0, m2 = 0.0;
            for (int c = 0; c < Cz; ++c) {
                m1 += gamma[c] * dy[c];
                m2 += gamma[c] * dy[c] * xh[c];
            }
            m1 /= Cz;
            m2 /= Cz;
            double *dzr = dz + ((size_t)i * Nj + j) * Cz;
            for (int c = 0; c < Cz; ++c) dzr[c] = (gamma[c] * dy[c] - m1 - xh[c] * m2) / sigma;
        }
    free(xh);
    free(dy);
    free(g);
}
