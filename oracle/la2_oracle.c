/*
 * la2_oracle.c -- fp64 CPU oracle for decayed causal linear attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file: only the tests, the package's smoke check and the CPU
 * baseline leg of the benchmark use it.  It shares no code, header, table or
 * helper with the CUDA library.
 *
 * What it computes (per batch b and head h, rows t = 0..L-1):
 *
 *   o_t = sum_{j <= t} lambda^(t-j) (q_t . k_j) v_j  (+ lambda^(t+1) q_t kv0)
 *
 * i.e. O = (Q K^T (.) M) V with M_tj = lambda^(t-j) for j <= t, 0 above the
 * diagonal.  lambda = 1 is plain causal linear attention.
 *
 * It is written as the token-by-token recurrence over a fixed-size d x e state
 * -- the "recurrent form" that the Lightning Attention glossary page
 * (jisaku.com, section "主な特徴・仕組み": recurrent and parallel forms, a
 * constant-size state for inference) names, and the running "cumulative
 * summation" of k^T v that the Lightning Attention-2 notes page
 * (phantomic12.github.io, opening paragraph) says the causal case needs:
 *
 *   kv_t = lambda * kv_{t-1} + k_t^T v_t      (kv_{-1} = kv0, or 0)
 *   o_t  = q_t kv_t                            (the state already holds token t)
 *
 * No blocking, no reordering: one token at a time, fp64 accumulation.
 * The pages give no decay, feature map, normalisation or scaling; the
 * attention takes its inputs as already mapped (the optional feature map is
 * its own pair of functions at the end of this file), and no denominator is
 * applied.
 *
 * Layout: q,k [B,H,L,d], v [B,H,L,e] contiguous row-major (float, which holds
 * bf16 and fp32 inputs exactly); lambda [H] double; states [B,H,d,e] double;
 * outputs double.  Every (b,h) problem is independent; OpenMP only spreads
 * those independent problems over host cores.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Forward: o (and optionally the final state kv_out) from the recurrence. */
void oracle_forward(int B, int H, long L, int d, int e,
                    const float *q, const float *k, const float *v,
                    const double *lambda, const double *kv0,
                    double *o, double *kv_out)
{
    long BH = (long)B * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (long bh = 0; bh < BH; bh++) {
        int h = (int)(bh % H);
        double lam = lambda[h];
        double *kv = (double *)malloc(sizeof(double) * d * e);
        if (kv0) memcpy(kv, kv0 + bh * d * e, sizeof(double) * d * e);
        else memset(kv, 0, sizeof(double) * d * e);
        const float *qb = q + bh * L * d, *kb = k + bh * L * d, *vb = v + bh * L * e;
        double *ob = o + bh * L * e;
        for (long t = 0; t < L; t++) {
            const float *qt = qb + t * d, *kt = kb + t * d, *vt = vb + t * e;
            /* state update: decay the old state, add the outer product k_t^T v_t */
            for (int i = 0; i < d; i++)
                for (int j = 0; j < e; j++)
                    kv[i * e + j] = lam * kv[i * e + j] + (double)kt[i] * (double)vt[j];
            /* read-out: o_t = q_t kv_t */
            for (int j = 0; j < e; j++) {
                double acc = 0.0;
                for (int i = 0; i < d; i++) acc += (double)qt[i] * kv[i * e + j];
                ob[t * e + j] = acc;
            }
        }
        if (kv_out) memcpy(kv_out + bh * d * e, kv, sizeof(double) * d * e);
        free(kv);
    }
}

/*
 * Backward of the same recurrence for an upstream gradient dO (the gradient
 * of a scalar loss with respect to o).  Applying the chain rule to the two
 * lines of the recurrence:
 *
 *   dq_t = dO_t kv_t^T                               (forward state kv_t)
 *   G_t  = q_t^T dO_t + lambda * G_{t+1},  G_L = 0    (adjoint of kv_t)
 *   dk_t = v_t G_t^T,   dv_t = k_t G_t
 *   dkv0 = lambda * G_0                               (gradient w.r.t. kv0)
 *
 * The "tiling in both forward and backward" of the Lightning Attention-2 notes
 * page ("Tiling." paragraph) is a faster schedule of exactly these sums.
 *
 * oracle_backward_end takes a terminal adjoint G_L = gend [B,H,d,e] (NULL:
 * zero): the part of the loss that depends on the state after the last
 * token through tokens that come later (the rows after a shard of a longer
 * sequence: G_L = sum_{s >= L} lambda^(s-L) q_s^T dO_s).  Same chain rule.
 */
void oracle_backward_end(int B, int H, long L, int d, int e,
                         const float *q, const float *k, const float *v,
                         const double *lambda, const double *kv0, const float *dO,
                         const double *gend,
                         double *dq, double *dk, double *dv, double *dkv0)
{
    long BH = (long)B * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (long bh = 0; bh < BH; bh++) {
        int h = (int)(bh % H);
        double lam = lambda[h];
        double *st = (double *)malloc(sizeof(double) * d * e);
        const float *qb = q + bh * L * d, *kb = k + bh * L * d, *vb = v + bh * L * e;
        const float *gb = dO + bh * L * e;

        /* forward sweep: rebuild kv_t, dq_t = dO_t kv_t^T */
        if (kv0) memcpy(st, kv0 + bh * d * e, sizeof(double) * d * e);
        else memset(st, 0, sizeof(double) * d * e);
        for (long t = 0; t < L; t++) {
            const float *kt = kb + t * d, *vt = vb + t * e, *gt = gb + t * e;
            for (int i = 0; i < d; i++)
                for (int j = 0; j < e; j++)
                    st[i * e + j] = lam * st[i * e + j] + (double)kt[i] * (double)vt[j];
            for (int i = 0; i < d; i++) {
                double acc = 0.0;
                for (int j = 0; j < e; j++) acc += (double)gt[j] * st[i * e + j];
                dq[(bh * L + t) * d + i] = acc;
            }
        }

        /* reverse sweep: G_t = q_t^T dO_t + lambda G_{t+1}, from G_L */
        if (gend) memcpy(st, gend + bh * d * e, sizeof(double) * d * e);
        else memset(st, 0, sizeof(double) * d * e);
        for (long t = L - 1; t >= 0; t--) {
            const float *qt = qb + t * d, *kt = kb + t * d, *vt = vb + t * e, *gt = gb + t * e;
            for (int i = 0; i < d; i++)
                for (int j = 0; j < e; j++)
                    st[i * e + j] = lam * st[i * e + j] + (double)qt[i] * (double)gt[j];
            for (int i = 0; i < d; i++) {          /* dk_t = v_t G_t^T */
                double acc = 0.0;
                for (int j = 0; j < e; j++) acc += (double)vt[j] * st[i * e + j];
                dk[(bh * L + t) * d + i] = acc;
            }
            for (int j = 0; j < e; j++) {          /* dv_t = k_t G_t */
                double acc = 0.0;
                for (int i = 0; i < d; i++) acc += (double)kt[i] * st[i * e + j];
                dv[(bh * L + t) * e + j] = acc;
            }
        }
        if (dkv0)
            for (int i = 0; i < d * e; i++) dkv0[bh * d * e + i] = lam * st[i];
        free(st);
    }
}

void oracle_backward(int B, int H, long L, int d, int e,
                     const float *q, const float *k, const float *v,
                     const double *lambda, const double *kv0, const float *dO,
                     double *dq, double *dk, double *dv, double *dkv0)
{
    oracle_backward_end(B, H, L, d, e, q, k, v, lambda, kv0, dO, NULL, dq, dk, dv, dkv0);
}

/*
 * One decode step: the recurrence above applied to a single new token per
 * (b,h), with the fixed-size state kept by the caller between calls (the
 * constant-size inference state of the glossary page, "主な特徴・仕組み").
 *   kv <- lambda kv + k^T v;  o = q kv.
 * q,k [B,H,d], v [B,H,e] float; kv [B,H,d,e] double, updated in place;
 * o [B,H,e] double.
 */
void oracle_decode_step(int B, int H, int d, int e,
                        const float *q, const float *k, const float *v,
                        const double *lambda, double *kv, double *o)
{
    long BH = (long)B * H;
#pragma omp parallel for schedule(static)
    for (long bh = 0; bh < BH; bh++) {
        int h = (int)(bh % H);
        double lam = lambda[h];
        double *s = kv + bh * d * e;
        const float *qt = q + bh * d, *kt = k + bh * d, *vt = v + bh * e;
        for (int i = 0; i < d; i++)
            for (int j = 0; j < e; j++)
                s[i * e + j] = lam * s[i * e + j] + (double)kt[i] * (double)vt[j];
        for (int j = 0; j < e; j++) {
            double acc = 0.0;
            for (int i = 0; i < d; i++) acc += (double)qt[i] * s[i * e + j];
            o[bh * e + j] = acc;
        }
    }
}

/*
 * Gradient of the loss sum(o * dO) with respect to each head's decay
 * lambda_h, summed over the batch: the chain rule through the recurrence
 * (the running state of the Lightning Attention-2 notes page, opening
 * paragraph, with the decay factor).  With kv_t = lambda kv_{t-1} + k_t^T
 * v_t (kv_{-1} = kv0, a constant) its derivative R_t = d kv_t / d lambda
 * obeys
 *   R_t = kv_{t-1} + lambda R_{t-1},   R_{-1} = 0,
 * and o_t = q_t kv_t gives d o_t / d lambda = q_t R_t, so
 *   dlambda_h = sum_b sum_t dO_t . (q_t R_t).
 * dlam [H] double (written, not accumulated).
 */
void oracle_dlambda(int B, int H, long L, int d, int e,
                    const float *q, const float *k, const float *v,
                    const double *lambda, const double *kv0, const float *dO,
                    double *dlam)
{
    long BH = (long)B * H;
    double *part = (double *)calloc((size_t)BH, sizeof(double));
#pragma omp parallel for schedule(dynamic, 1)
    for (long bh = 0; bh < BH; bh++) {
        int h = (int)(bh % H);
        double lam = lambda[h];
        double *st = (double *)malloc(sizeof(double) * d * e);
        double *rt = (double *)calloc((size_t)d * e, sizeof(double));
        const float *qb = q + bh * L * d, *kb = k + bh * L * d, *vb = v + bh * L * e;
        const float *gb = dO + bh * L * e;
        if (kv0) memcpy(st, kv0 + bh * d * e, sizeof(double) * d * e);
        else memset(st, 0, sizeof(double) * d * e);
        double acc = 0.0;
        for (long t = 0; t < L; t++) {
            const float *qt = qb + t * d, *kt = kb + t * d, *vt = vb + t * e, *gt = gb + t * e;
            for (int i = 0; i < d; i++)
                for (int j = 0; j < e; j++) {
                    rt[i * e + j] = st[i * e + j] + lam * rt[i * e + j];   /* uses kv_{t-1} */
                    st[i * e + j] = lam * st[i * e + j] + (double)kt[i] * (double)vt[j];
                }
            for (int j = 0; j < e; j++) {
                double s = 0.0;
                for (int i = 0; i < d; i++) s += (double)qt[i] * rt[i * e + j];
                acc += (double)gt[j] * s;
            }
        }
        part[bh] = acc;
        free(st);
        free(rt);
    }
    for (int h = 0; h < H; h++) dlam[h] = 0.0;
    for (long bh = 0; bh < BH; bh++) dlam[bh % H] += part[bh];
    free(part);
}

/*
 * Feature map, the optional prologue applied to q and k before the attention.
 *
 * The Lightning Attention glossary page (section "主な特徴・仕組み") has
 * linear attention replace softmax by a kernel feature map so that K^T V
 * can be aggregated first, but it names no map.  Reading taken here: the
 * exponential linear unit plus one, phi(x) = elu(x) + 1, the positive map
 * of "Transformers are RNNs", one of the works the Luna page lists as its
 * basis next to the ELU paper.  With elu's own definition (alpha = 1):
 *
 *   elu(x) = x              for x > 0,   exp(x) - 1   for x <= 0
 *   phi(x) = elu(x) + 1
 *
 * and, for the chain rule of the backward pass, elu's derivative
 *
 *   elu'(x) = 1             for x > 0,   exp(x)       for x <= 0
 *
 * so dL/dx = dL/dphi(x) * elu'(x).  Elementwise over n values; x float
 * (exact bf16 or fp32 inputs), results double.
 */
void oracle_feature_map(long n, const float *x, double *y)
{
#pragma omp parallel for schedule(static)
    for (long i = 0; i < n; i++) {
        double xi = (double)x[i];
        double elu = xi > 0.0 ? xi : expm1(xi);
        y[i] = elu + 1.0;
    }
}

void oracle_feature_map_grad(long n, const float *x, const double *dy, double *dx)
{
#pragma omp parallel for schedule(static)
    for (long i = 0; i < n; i++) {
        double xi = (double)x[i];
        double delu = xi > 0.0 ? 1.0 : exp(xi);
        dx[i] = dy[i] * delu;
    }
}
