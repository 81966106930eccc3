/*
 * linattn_oracle.c — plain fp64 CPU oracle for kernelized linear attention
 * with the elu(x)+1 feature map.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file: only the tests, the package's smoke check and the bench's
 * CPU-baseline leg do.  It shares no code, header, table or helper with the
 * CUDA library; the two meet only through the seeded input arrays.
 *
 * Every function walks the tokens one at a time, in the order and notation
 * of the pages it follows, with no blocking, chunking or reordering:
 *
 *   phi(x)  = elu(x) + 1                       (Transformers-are-RNNs map;
 *             "Linear Attention" knowledge-base page, section 2, "Choice of
 *             phi"; linear-attention lesson, "What the pieces are for")
 *   S_t     = a_t * S_{t-1} + phi(k_t) v_t^T    (running state, section 2
 *   z_t     = a_t * z_{t-1} + phi(k_t)           "Causal recurrence"; decay
 *                                                 a_t from the concept card's
 *                                                 "Implementation sketch" and
 *                                                 its SSD variant, a_t = 1 is
 *                                                 the plain form)
 *   o_t     = phi(q_t)^T S_t / (phi(q_t)^T z_t + eps)
 *                                               (normalised read-out with the
 *                                                 1e-6 of the section 3 sketch)
 *
 * Gated form: an optional per-token gain b_t scales the new term,
 *   S_t = a_t S_{t-1} + b_t phi(k_t) v_t^T,  z_t = a_t z_{t-1} + b_t phi(k_t).
 * Random Feature Attention's sigmoid gate g_t is a_t = g_t, b_t = 1 - g_t
 * (concept card "Linear attention": RFA variant and the closing paragraph of
 * its "Implementation sketch", RFA eq. 7); b_t = 1 is the plain form.
 *
 * mLSTM read-out (concept card, "Matrix memory with exponential gates
 * (mLSTM)"; its implementation sketch: the identity as the feature map,
 * input-dependent gates and a normaliser read-out): C_t = f_t C_{t-1} +
 * i_t v_t k_t^T, n_t = f_t n_{t-1} + i_t k_t, h_t = C_t q_t / max(|n_t^T q_t|, 1).
 * With S = C^T this is the gated recurrence above with phi = identity,
 * a = f, b = i, and the denominator max(|q^T z|, 1) in place of q^T z + eps.
 *
 * Layouts (all row-major, C order, fp64):
 *   q, k     [B, H, T, d_k]      v [B, H, T, d_v]      out [B, H, T, d_v]
 *   decay    [B, H, T] (causal) or [B, H] (decode); NULL = no decay
 *   gain     same layout as decay; NULL = 1
 *   S        [B, H, d_k, d_v]    z [B, H, d_k]
 *
 * Parallelism: independent (b, h) heads are spread over OpenMP threads; the
 * arithmetic of one head is sequential and identical for any thread count.
 */
#include <math.h>
#include <stddef.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* elu(x) + 1 with alpha = 1.  For x <= 0, elu(x) + 1 = (e^x - 1) + 1, which
 * is e^x exactly in real arithmetic; writing e^x avoids the cancellation of
 * the -1/+1 pair.  At x = 0 both branches give 1. */
static double phi(double x) { return x > 0.0 ? x + 1.0 : exp(x); }

/* Feature map and read-out of one call: elu(x)+1 with (den + eps), or the
 * mLSTM form: the identity with max(|den|, 1). */
typedef struct { int mlstm; } form_t;
static double fmap(form_t f, double x) { return f.mlstm ? x : phi(x); }
static double denom(form_t f, double den, double eps) { return f.mlstm ? fmax(fabs(den), 1.0) : den + eps; }

void orc_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int orc_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* One head of the causal recurrence.  fk/fq are scratch of length dk.  The
 * gain multiplies the new key's features once (b * phi(k_t)), so it reaches
 * both the state and the normaliser; b = 1 leaves every value unchanged. */
static void causal_head(form_t form, const double *q, const double *k, const double *v,
                        const double *decay, const double *gain, long T, int dk, int dv,
                        double eps, double *S, double *z, double *out, double *fk, double *fq)
{
    for (long t = 0; t < T; ++t) {
        const double *qt = q + t * dk, *kt = k + t * dk, *vt = v + t * dv;
        const double b = gain ? gain[t] : 1.0;
        for (int i = 0; i < dk; ++i) { fk[i] = b * fmap(form, kt[i]); fq[i] = fmap(form, qt[i]); }
        if (decay) {
            /* decayed form: the old state is scaled first, the new token
             * enters undecayed */
            const double a = decay[t];
            for (int i = 0; i < dk; ++i) {
                for (int j = 0; j < dv; ++j) S[i * dv + j] = a * S[i * dv + j] + fk[i] * vt[j];
                z[i] = a * z[i] + fk[i];
            }
        } else {
            /* plain form: rank-one update and vector update */
            for (int i = 0; i < dk; ++i) {
                for (int j = 0; j < dv; ++j) S[i * dv + j] = S[i * dv + j] + fk[i] * vt[j];
                z[i] = z[i] + fk[i];
            }
        }
        double den = 0.0;
        for (int i = 0; i < dk; ++i) den += fq[i] * z[i];
        den = denom(form, den, eps);
        double *ot = out + t * dv;
        for (int j = 0; j < dv; ++j) {
            double num = 0.0;
            for (int i = 0; i < dk; ++i) num += fq[i] * S[i * dv + j];
            ot[j] = num / den;
        }
    }
}

/*
 * Causal linear attention over all heads.
 *   S_in/z_in  : initial state, or NULL for zeros.
 *   S_out/z_out: final state, or NULL to discard.
 * Returns 0, or -1 on a bad argument / allocation failure.
 */
int orc_causal_form(int mlstm, const double *q, const double *k, const double *v, const double *decay,
                    const double *gain, int B, int H, long T, int dk, int dv, double eps,
                    const double *S_in, const double *z_in,
                    double *out, double *S_out, double *z_out)
{
    const form_t form = {mlstm};
    if (B < 0 || H < 0 || T < 0 || dk <= 0 || dv <= 0) return -1;
    const long BH = (long)B * H;
    int err = 0;
#pragma omp parallel
    {
        double *S = (double *)malloc(sizeof(double) * (size_t)dk * dv);
        double *z = (double *)malloc(sizeof(double) * (size_t)dk);
        double *fk = (double *)malloc(sizeof(double) * (size_t)dk);
        double *fq = (double *)malloc(sizeof(double) * (size_t)dk);
        if (!S || !z || !fk || !fq) {
#pragma omp atomic write
            err = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (long bh = 0; bh < BH; ++bh) {
                if (S_in) memcpy(S, S_in + bh * dk * dv, sizeof(double) * (size_t)dk * dv);
                else memset(S, 0, sizeof(double) * (size_t)dk * dv);
                if (z_in) memcpy(z, z_in + bh * dk, sizeof(double) * (size_t)dk);
                else memset(z, 0, sizeof(double) * (size_t)dk);
                causal_head(form, q + bh * T * dk, k + bh * T * dk, v + bh * T * dv,
                            decay ? decay + bh * T : NULL, gain ? gain + bh * T : NULL, T, dk, dv,
                            eps, S, z, out + bh * T * dv, fk, fq);
                if (S_out) memcpy(S_out + bh * dk * dv, S, sizeof(double) * (size_t)dk * dv);
                if (z_out) memcpy(z_out + bh * dk, z, sizeof(double) * (size_t)dk);
            }
        }
        free(S); free(z); free(fk); free(fq);
    }
    return err ? -1 : 0;
}

int orc_causal_gated(const double *q, const double *k, const double *v, const double *decay,
                     const double *gain, int B, int H, long T, int dk, int dv, double eps,
                     const double *S_in, const double *z_in,
                     double *out, double *S_out, double *z_out)
{
    return orc_causal_form(0, q, k, v, decay, gain, B, H, T, dk, dv, eps, S_in, z_in, out, S_out, z_out);
}

int orc_causal(const double *q, const double *k, const double *v, const double *decay,
               int B, int H, long T, int dk, int dv, double eps,
               const double *S_in, const double *z_in,
               double *out, double *S_out, double *z_out)
{
    return orc_causal_form(0, q, k, v, decay, NULL, B, H, T, dk, dv, eps, S_in, z_in, out, S_out, z_out);
}

/*
 * Non-causal linear attention: the prefix sums collapse to global sums over
 * all Lk keys (knowledge-base page, section 3, first sketch):
 *   S = S_in + sum_j phi(k_j) v_j^T,  z = z_in + sum_j phi(k_j),
 *   o_i = phi(q_i)^T S / (phi(q_i)^T z + eps)  for each of the Lq queries.
 * S_out/z_out receive the totals (including the state in), or NULL.
 */
int orc_noncausal(const double *q, const double *k, const double *v,
                  int B, int H, long Lq, long Lk, int dk, int dv, double eps,
                  const double *S_in, const double *z_in,
                  double *out, double *S_out, double *z_out)
{
    if (B < 0 || H < 0 || Lq < 0 || Lk < 0 || dk <= 0 || dv <= 0) return -1;
    const long BH = (long)B * H;
    int err = 0;
#pragma omp parallel
    {
        double *S = (double *)malloc(sizeof(double) * (size_t)dk * dv);
        double *z = (double *)malloc(sizeof(double) * (size_t)dk);
        double *f = (double *)malloc(sizeof(double) * (size_t)dk);
        if (!S || !z || !f) {
#pragma omp atomic write
            err = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (long bh = 0; bh < BH; ++bh) {
                if (S_in) memcpy(S, S_in + bh * dk * dv, sizeof(double) * (size_t)dk * dv);
                else memset(S, 0, sizeof(double) * (size_t)dk * dv);
                if (z_in) memcpy(z, z_in + bh * dk, sizeof(double) * (size_t)dk);
                else memset(z, 0, sizeof(double) * (size_t)dk);
                const double *kh = k + bh * Lk * dk, *vh = v + bh * Lk * dv;
                for (long j = 0; j < Lk; ++j) {
                    for (int i = 0; i < dk; ++i) f[i] = phi(kh[j * dk + i]);
                    for (int i = 0; i < dk; ++i) {
                        for (int c = 0; c < dv; ++c) S[i * dv + c] += f[i] * vh[j * dv + c];
                        z[i] += f[i];
                    }
                }
                const double *qh = q + bh * Lq * dk;
                double *oh = out + bh * Lq * dv;
                for (long t = 0; t < Lq; ++t) {
                    for (int i = 0; i < dk; ++i) f[i] = phi(qh[t * dk + i]);
                    double den = 0.0;
                    for (int i = 0; i < dk; ++i) den += f[i] * z[i];
                    for (int c = 0; c < dv; ++c) {
                        double num = 0.0;
                        for (int i = 0; i < dk; ++i) num += f[i] * S[i * dv + c];
                        oh[t * dv + c] = num / (den + eps);
                    }
                }
                if (S_out) memcpy(S_out + bh * dk * dv, S, sizeof(double) * (size_t)dk * dv);
                if (z_out) memcpy(z_out + bh * dk, z, sizeof(double) * (size_t)dk);
            }
        }
        free(S); free(z); free(f);
    }
    return err ? -1 : 0;
}

/*
 * One constant-state decode step per head: the causal loop body applied once
 * to a carried (S, z), which are updated in place.
 *   q, k [B, H, dk], v [B, H, dv], decay and gain [B, H] or NULL, out [B, H, dv].
 */
int orc_decode_step_form(int mlstm, const double *q, const double *k, const double *v,
                         const double *decay, const double *gain, int B, int H, int dk, int dv,
                         double eps, double *S, double *z, double *out)
{
    const form_t form = {mlstm};
    if (B < 0 || H < 0 || dk <= 0 || dv <= 0 || !S || !z) return -1;
    const long BH = (long)B * H;
    int err = 0;
#pragma omp parallel
    {
        double *fk = (double *)malloc(sizeof(double) * (size_t)dk);
        double *fq = (double *)malloc(sizeof(double) * (size_t)dk);
        if (!fk || !fq) {
#pragma omp atomic write
            err = 1;
        } else {
#pragma omp for schedule(static)
            for (long bh = 0; bh < BH; ++bh) {
                causal_head(form, q + bh * dk, k + bh * dk, v + bh * dv,
                            decay ? decay + bh : NULL, gain ? gain + bh : NULL, 1, dk, dv, eps,
                            S + bh * dk * dv, z + bh * dk, out + bh * dv, fk, fq);
            }
        }
        free(fk); free(fq);
    }
    return err ? -1 : 0;
}

int orc_decode_step_gated(const double *q, const double *k, const double *v, const double *decay,
                          const double *gain, int B, int H, int dk, int dv, double eps,
                          double *S, double *z, double *out)
{
    return orc_decode_step_form(0, q, k, v, decay, gain, B, H, dk, dv, eps, S, z, out);
}

int orc_decode_step(const double *q, const double *k, const double *v, const double *decay,
                    int B, int H, int dk, int dv, double eps,
                    double *S, double *z, double *out)
{
    return orc_decode_step_form(0, q, k, v, decay, NULL, B, H, dk, dv, eps, S, z, out);
}

/*
 * FLASH chunk form, causal (concept card "Linear attention", "Chunked
 * attention: exact inside blocks, linear across them (FLASH)", and the
 * closing paragraph of its implementation sketch): the sequence is cut into
 * non-overlapping chunks of `chunk` tokens; inside a chunk, exact
 * squared-ReLU attention over the chunk's earlier tokens (j <= t); across
 * chunks, a linear term read from the summaries of the earlier chunks only,
 * the summary of chunk g being sum_{j in g} k_j v_j^T, added to the running
 * sum once the chunk is done.  Softmax-free: no feature map, no normaliser.
 *   scaled = 0: the equations' form, weight relu(q.k)^2, summaries unscaled;
 *   scaled = 1: the listings' form, scores divided by the chunk length before
 *               the squared ReLU and each summary divided by the chunk length
 *               (the nominal chunk, also for a shorter last chunk).
 * S_out (or NULL) receives the sum of every chunk's summary.
 */
int orc_flash(const double *q, const double *k, const double *v, int B, int H, long T, int dk, int dv,
              int chunk, int scaled, double *out, double *S_out)
{
    if (B < 0 || H < 0 || T < 0 || dk <= 0 || dv <= 0 || chunk <= 0) return -1;
    const long BH = (long)B * H;
    const double sc = scaled ? (double)chunk : 1.0;
    int err = 0;
#pragma omp parallel
    {
        double *M = (double *)malloc(sizeof(double) * (size_t)dk * dv);   /* earlier chunks' summaries */
        double *dM = (double *)malloc(sizeof(double) * (size_t)dk * dv);  /* this chunk's summary */
        if (!M || !dM) {
#pragma omp atomic write
            err = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (long bh = 0; bh < BH; ++bh) {
                const double *qh = q + bh * T * dk, *kh = k + bh * T * dk, *vh = v + bh * T * dv;
                double *oh = out + bh * T * dv;
                memset(M, 0, sizeof(double) * (size_t)dk * dv);
                for (long g0 = 0; g0 < T; g0 += chunk) {
                    const long g1 = g0 + chunk < T ? g0 + chunk : T;
                    for (long t = g0; t < g1; ++t) {
                        const double *qt = qh + t * dk;
                        double *ot = oh + t * dv;
                        /* linear term: the summaries of the earlier chunks */
                        for (int c = 0; c < dv; ++c) {
                            double acc = 0.0;
                            for (int i = 0; i < dk; ++i) acc += qt[i] * M[i * dv + c];
                            ot[c] = acc;
                        }
                        /* exact squared-ReLU attention inside the chunk */
                        for (long j = g0; j <= t; ++j) {
                            double s = 0.0;
                            for (int i = 0; i < dk; ++i) s += qt[i] * kh[j * dk + i];
                            s /= sc;
                            const double r = s > 0.0 ? s : 0.0;
                            const double w = r * r;
                            for (int c = 0; c < dv; ++c) ot[c] += w * vh[j * dv + c];
                        }
                    }
                    /* the chunk's summary joins the running sum */
                    memset(dM, 0, sizeof(double) * (size_t)dk * dv);
                    for (long j = g0; j < g1; ++j)
                        for (int i = 0; i < dk; ++i)
                            for (int c = 0; c < dv; ++c) dM[i * dv + c] += kh[j * dk + i] * vh[j * dv + c];
                    for (long e = 0; e < (long)dk * dv; ++e) M[e] += dM[e] / sc;
                }
                if (S_out) memcpy(S_out + bh * dk * dv, M, sizeof(double) * (size_t)dk * dv);
            }
        }
        free(M); free(dM);
    }
    return err ? -1 : 0;
}

