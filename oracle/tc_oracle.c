/*
 * Tensor Cache layer -- CPU oracle (test infrastructure only).
 *
 * This file is the plain, slow, obviously-correct definition of what the layer
 * computes, written in float64 and looping token by token over a ring buffer
 * and the memory matrix A.  Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg load it.  It shares no code, header or table with the CUDA
 * library, and the library never calls it.
 *
 * Source: "Tensor Cache: Eviction-conditioned Associative Memory for
 * Transformers" (arXiv 2605.22884).
 *   - §3.1, eq. (1): the local window K_win, V_win holds the most recent W
 *     key/value pairs; y_local_t = Attn(q_t, K_win, V_win) is exact causal
 *     softmax attention over it (scaled by 1/sqrt(d_k)).
 *   - §3.2: A in R^{d_k x d_v} starts at zero; the KV cache is a FIFO ring
 *     buffer and the pair displaced when slot pos is overwritten is the write
 *     source ("write on evict").
 *   - §3.2, Fig. 2, one streaming step: (1) window full, (2) evict the oldest
 *     pair, (3) A <- lambda*A + eta*(k_old (x) v_old), (4) insert (k_t, v_t)
 *     into the freed slot, (5) read both paths and fuse:
 *     y_t = y_local_t + sigma(g) * m_t with m_t = q_t A.
 *   - abstract / §1: the read identity q (k (x) v) = <q,k> v, which fixes the
 *     orientation k (x) v = k v^T (d_k x d_v) and m = q A as a row vector.
 *   - abstract / §2 "training considerations": the chunk-mean shortcut
 *     A <- lambda*A + eta*(kbar (x) vbar) and the parallel weighted-sum chunk
 *     scan that equals per-token writes.
 *
 * Readings where the pages leave a step open:
 *   - the write (step 3) precedes the read (step 5) inside a step, so the query
 *     at step t sees token t-W through A and tokens t-W+1..t through the window;
 *   - the window includes the current token (inserted at step 4 before the
 *     read at step 5);
 *   - slots that were never filled (t < W) are excluded from the softmax;
 *   - the decay multiplies A once per eviction (it is part of the write rule);
 *   - sigma is the logistic function and g, lambda, eta are per head.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* One streaming step for one (batch, head): Fig. 2 steps (2)-(5) in order.
 * ring_k [W, dk], ring_v [W, dv], A [dk, dv] are updated in place.
 * s is scratch of length W.  y_local and m may be NULL. */
/* Write rules of step (3), A <- lam A + eta update(k_old, v_old) (Fig. 2):
 *   RULE_OUTER: update = k_old (x) v_old, the outer product;
 *   RULE_DELTA: update = k_old (x) (v_old - k_old^T A), the optional delta
 *     (Widrow-Hoff error-correcting) rule the figure mentions; the pages give
 *     no formula, and k_old^T A is read from A before this write (the memory's
 *     current prediction of v_old from k_old). */
enum { RULE_OUTER = 0, RULE_DELTA = 1 };

static void tc_step(int64_t t, int64_t dk, int64_t dv, int64_t W,
                    double *ring_k, double *ring_v, double *A,
                    const double *q, const double *k, const double *v,
                    double lam, double eta, double g,
                    double *y, double *y_local, double *m, double *s,
                    int rule, double *u)
{
    const int64_t pos = t % W;

    /* (2) + (3): once the window is full the slot about to be overwritten
     * holds the oldest pair; it is written into A before anything is read. */
    if (t >= W) {
        const double *k_old = ring_k + pos * dk;
        const double *v_old = ring_v + pos * dv;
        if (rule == RULE_DELTA) {
            for (int64_t c = 0; c < dv; ++c) {
                double pred = 0.0;
                for (int64_t r = 0; r < dk; ++r) pred += k_old[r] * A[r * dv + c];
                u[c] = v_old[c] - pred;
            }
        } else {
            for (int64_t c = 0; c < dv; ++c) u[c] = v_old[c];
        }
        for (int64_t r = 0; r < dk; ++r)
            for (int64_t c = 0; c < dv; ++c)
                A[r * dv + c] = lam * A[r * dv + c] + eta * (k_old[r] * u[c]);
    }

    /* (4): the new pair takes the freed slot. */
    memcpy(ring_k + pos * dk, k, (size_t)dk * sizeof(double));
    memcpy(ring_v + pos * dv, v, (size_t)dv * sizeof(double));

    /* (5a) L1: exact softmax over the filled slots (eq. (1)).  Before the
     * ring is full, slots 0..t hold tokens 0..t; afterwards all W do. */
    const int64_t n = (t + 1 < W) ? t + 1 : W;
    const double scale = 1.0 / sqrt((double)dk);
    double smax = -INFINITY;
    for (int64_t j = 0; j < n; ++j) {
        double dot = 0.0;
        for (int64_t r = 0; r < dk; ++r) dot += q[r] * ring_k[j * dk + r];
        s[j] = dot * scale;
        if (s[j] > smax) smax = s[j];
    }
    double denom = 0.0;
    for (int64_t j = 0; j < n; ++j) {
        s[j] = exp(s[j] - smax);
        denom += s[j];
    }

    /* (5b) L2: m = q A, m[c] = sum_r q[r] A[r][c]. */
    const double gate = 1.0 / (1.0 + exp(-g));
    for (int64_t c = 0; c < dv; ++c) {
        double acc = 0.0;
        for (int64_t j = 0; j < n; ++j) acc += s[j] * ring_v[j * dv + c];
        const double yl = acc / denom;
        double mc = 0.0;
        for (int64_t r = 0; r < dk; ++r) mc += q[r] * A[r * dv + c];
        /* (5c) fusion */
        y[c] = yl + gate * mc;
        if (y_local) y_local[c] = yl;
        if (m) m[c] = mc;
    }
}

static void set_threads(int nthreads)
{
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
}

/* Threads the oracle would use (for reporting). */
int oracle_max_threads(int nthreads)
{
#ifdef _OPENMP
    set_threads(nthreads);
    return omp_get_max_threads();
#else
    (void)nthreads;
    return 1;
#endif
}

/* Prefill: the streaming step applied to tokens 0..T-1 from an empty ring and
 * A = 0 (§3.2: A_0 = 0).  q,k: [B,H,T,dk]; v: [B,H,T,dv]; lam, eta, g: [H].
 * Outputs y: [B,H,T,dv], A_final: [B,H,dk,dv]; y_local and m (same shape as
 * y) may be NULL.  Returns 0, or -1 on bad sizes / allocation failure. */
int oracle_prefill_rule(int64_t B, int64_t H, int64_t T, int64_t dk, int64_t dv, int64_t W,
                        const double *q, const double *k, const double *v,
                        const double *lam, const double *eta, const double *g,
                        double *y, double *A_final, double *y_local, double *m,
                        int rule, int nthreads)
{
    if (B < 0 || H < 0 || T < 0 || dk < 1 || dv < 1 || W < 1) return -1;
    if (rule != RULE_OUTER && rule != RULE_DELTA) return -1;
    set_threads(nthreads);
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : err)
    for (int64_t bh = 0; bh < B * H; ++bh) {
        const int64_t h = bh % H;
        double *ring_k = (double *)calloc((size_t)(W * dk), sizeof(double));
        double *ring_v = (double *)calloc((size_t)(W * dv), sizeof(double));
        double *s = (double *)malloc((size_t)W * sizeof(double));
        double *u = (double *)malloc((size_t)dv * sizeof(double));
        double *A = A_final + bh * dk * dv;
        if (!ring_k || !ring_v || !s || !u) {
            err |= 1;
        } else {
            memset(A, 0, (size_t)(dk * dv) * sizeof(double));
            for (int64_t t = 0; t < T; ++t) {
                const int64_t rq = (bh * T + t) * dk, rv = (bh * T + t) * dv;
                tc_step(t, dk, dv, W, ring_k, ring_v, A, q + rq, k + rq, v + rv,
                        lam[h], eta[h], g[h], y + rv,
                        y_local ? y_local + rv : NULL, m ? m + rv : NULL, s, rule, u);
            }
        }
        free(ring_k);
        free(ring_v);
        free(s);
        free(u);
    }
    return err ? -1 : 0;
}

int oracle_prefill(int64_t B, int64_t H, int64_t T, int64_t dk, int64_t dv, int64_t W,
                   const double *q, const double *k, const double *v,
                   const double *lam, const double *eta, const double *g,
                   double *y, double *A_final, double *y_local, double *m,
                   int nthreads)
{
    return oracle_prefill_rule(B, H, T, dk, dv, W, q, k, v, lam, eta, g, y, A_final, y_local, m,
                               RULE_OUTER, nthreads);
}

/* Decode: nsteps streaming steps starting at clock t0 from a given state.
 * ring_k: [B,H,W,dk], ring_v: [B,H,W,dv], A: [B,H,dk,dv] (updated in place);
 * q,k: [nsteps,B,H,dk]; v: [nsteps,B,H,dv]; y: [nsteps,B,H,dv].
 * Slot j of the ring holds token j when t0 < W and token t with t mod W = j
 * otherwise (the layout a streaming run leaves behind). */
int oracle_decode_rule(int64_t B, int64_t H, int64_t dk, int64_t dv, int64_t W,
                       int64_t t0, int64_t nsteps,
                       double *ring_k, double *ring_v, double *A,
                       const double *q, const double *k, const double *v,
                       const double *lam, const double *eta, const double *g,
                       double *y, int rule, int nthreads)
{
    if (B < 0 || H < 0 || dk < 1 || dv < 1 || W < 1 || t0 < 0 || nsteps < 0) return -1;
    if (rule != RULE_OUTER && rule != RULE_DELTA) return -1;
    set_threads(nthreads);
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : err)
    for (int64_t bh = 0; bh < B * H; ++bh) {
        const int64_t h = bh % H;
        double *s = (double *)malloc((size_t)W * sizeof(double));
        double *u = (double *)malloc((size_t)dv * sizeof(double));
        if (!s || !u) {
            err |= 1;
        } else {
            for (int64_t i = 0; i < nsteps; ++i) {
                const int64_t rq = (i * B * H + bh) * dk, rv = (i * B * H + bh) * dv;
                tc_step(t0 + i, dk, dv, W, ring_k + bh * W * dk, ring_v + bh * W * dv,
                        A + bh * dk * dv, q + rq, k + rq, v + rv, lam[h], eta[h], g[h],
                        y + rv, NULL, NULL, s, rule, u);
            }
        }
        free(s);
        free(u);
    }
    return err ? -1 : 0;
}

int oracle_decode(int64_t B, int64_t H, int64_t dk, int64_t dv, int64_t W,
                  int64_t t0, int64_t nsteps,
                  double *ring_k, double *ring_v, double *A,
                  const double *q, const double *k, const double *v,
                  const double *lam, const double *eta, const double *g,
                  double *y, int nthreads)
{
    return oracle_decode_rule(B, H, dk, dv, W, t0, nsteps, ring_k, ring_v, A, q, k, v, lam, eta,
                              g, y, RULE_OUTER, nthreads);
}

/* ------------------------------------------------------------------------
 * State-only scans over a sequence of E evicted pairs (one head), used by the
 * property tests of the training form.  k: [E,dk], v: [E,dv], A out [dk,dv].
 * With fp32 != 0 every operation is rounded to float32 (the decay powers are
 * computed in float64 and rounded once); otherwise float64 throughout.
 * ------------------------------------------------------------------------ */

/* Per-token writes (§3.2, Fig. 2 step (3)) applied E times from A = 0. */
void oracle_scan_tokens(int64_t E, int64_t dk, int64_t dv,
                        const double *k, const double *v,
                        double lam, double eta, int fp32, double *A)
{
    if (fp32) {
        float *Af = (float *)calloc((size_t)(dk * dv), sizeof(float));
        const float l = (float)lam, e = (float)eta;
        for (int64_t i = 0; i < E; ++i)
            for (int64_t r = 0; r < dk; ++r) {
                const float kr = (float)k[i * dk + r];
                for (int64_t c = 0; c < dv; ++c) {
                    const float kv = kr * (float)v[i * dv + c];
                    const float a = l * Af[r * dv + c];
                    const float w = e * kv;
                    Af[r * dv + c] = a + w;
                }
            }
        for (int64_t x = 0; x < dk * dv; ++x) A[x] = (double)Af[x];
        free(Af);
        return;
    }
    memset(A, 0, (size_t)(dk * dv) * sizeof(double));
    for (int64_t i = 0; i < E; ++i)
        for (int64_t r = 0; r < dk; ++r)
            for (int64_t c = 0; c < dv; ++c)
                A[r * dv + c] = lam * A[r * dv + c] + eta * (k[i * dk + r] * v[i * dv + c]);
}

/* Parallel weighted-sum chunk scan (abstract; §1 contributions; §2): the
 * evictions are cut into chunks of C from the first one (the last chunk may
 * be shorter, length Cc) and each chunk applies
 *   A <- lambda^Cc * A + eta * sum_{i<Cc} lambda^(Cc-1-i) k_i (x) v_i,
 * which is the per-token recurrence unrolled over the chunk. */
void oracle_scan_chunks(int64_t E, int64_t C, int64_t dk, int64_t dv,
                        const double *k, const double *v,
                        double lam, double eta, int fp32, double *A)
{
    const int64_t n = dk * dv;
    double *Ad = (double *)calloc((size_t)n, sizeof(double));
    float *Af = (float *)calloc((size_t)n, sizeof(float));
    double *Sd = (double *)malloc((size_t)n * sizeof(double));
    float *Sf = (float *)malloc((size_t)n * sizeof(float));
    for (int64_t c0 = 0; c0 < E; c0 += C) {
        const int64_t Cc = (E - c0 < C) ? E - c0 : C;
        /* weighted sum of the chunk's outer products */
        memset(Sd, 0, (size_t)n * sizeof(double));
        memset(Sf, 0, (size_t)n * sizeof(float));
        for (int64_t i = 0; i < Cc; ++i) {
            const double wd = eta * pow(lam, (double)(Cc - 1 - i));
            const float wf = (float)wd;
            for (int64_t r = 0; r < dk; ++r)
                for (int64_t c = 0; c < dv; ++c) {
                    const double kk = k[(c0 + i) * dk + r], vv = v[(c0 + i) * dv + c];
                    if (fp32) {
                        const float kv = (float)kk * (float)vv;
                        const float t = wf * kv;
                        Sf[r * dv + c] = Sf[r * dv + c] + t;
                    } else {
                        Sd[r * dv + c] += wd * (kk * vv);
                    }
                }
        }
        const double dd = pow(lam, (double)Cc);
        const float df = (float)dd;
        for (int64_t x = 0; x < n; ++x) {
            if (fp32) {
                const float a = df * Af[x];
                Af[x] = a + Sf[x];
            } else {
                Ad[x] = dd * Ad[x] + Sd[x];
            }
        }
    }
    for (int64_t x = 0; x < n; ++x) A[x] = fp32 ? (double)Af[x] : Ad[x];
    free(Ad);
    free(Af);
    free(Sd);
    free(Sf);
}

/* The chunk-mean shortcut the pages identify as lossy (abstract; §1; §2):
 *   A <- lambda * A + eta * (kbar (x) vbar),  kbar, vbar = chunk means.
 * float64 throughout. */
void oracle_scan_chunk_mean(int64_t E, int64_t C, int64_t dk, int64_t dv,
                            const double *k, const double *v,
                            double lam, double eta, double *A)
{
    double *kb = (double *)malloc((size_t)dk * sizeof(double));
    double *vb = (double *)malloc((size_t)dv * sizeof(double));
    memset(A, 0, (size_t)(dk * dv) * sizeof(double));
    for (int64_t c0 = 0; c0 < E; c0 += C) {
        const int64_t Cc = (E - c0 < C) ? E - c0 : C;
        for (int64_t r = 0; r < dk; ++r) {
            double acc = 0.0;
            for (int64_t i = 0; i < Cc; ++i) acc += k[(c0 + i) * dk + r];
            kb[r] = acc / (double)Cc;
        }
        for (int64_t c = 0; c < dv; ++c) {
            double acc = 0.0;
            for (int64_t i = 0; i < Cc; ++i) acc += v[(c0 + i) * dv + c];
            vb[c] = acc / (double)Cc;
        }
        for (int64_t r = 0; r < dk; ++r)
            for (int64_t c = 0; c < dv; ++c)
                A[r * dv + c] = lam * A[r * dv + c] + eta * (kb[r] * vb[c]);
    }
    free(kb);
    free(vb);
}

/* ------------------------------------------------------------------------
 * Backward of the layer (outer-product write), by reverse-mode through the
 * token loop of Fig. 2.  For the scalar L = sum_t <dy_t, y_t> it returns
 * dq, dk, dv ([B,H,T,d], same layout as the inputs) and the per-head
 * dlam, deta, dg ([H], summed over the batch).  The forward is replayed with
 * every state A_t kept (T*dk*dv doubles per head: small inputs only).
 *   y_t = y_local_t + s m_t,  s = sigmoid(g),  m_t = q_t A_t,
 *   A_t = lam A_{t-1} + eta k_{t-W} v_{t-W}^T  (t >= W),  A_t = A_{t-1} else.
 * Reverse pass: G_t = dL/dA_t = q_t^T (s dy_t) + [t+1 >= W] lam G_{t+1}
 * (G_{t+1} unscaled when step t+1 has no write); each write at step t gives
 * dk_e += eta G_t v_e, dv_e += eta G_t^T k_e, deta += <G_t, k_e v_e^T>,
 * dlam += <G_t, A_{t-1}>.  The window softmax backward is the usual one:
 * dp_j = <dy_t, v_j>, ds_j = p_j (dp_j - sum_i p_i dp_i),
 * dq_t += sum_j ds_j k_j / sqrt(dk), dk_j += ds_j q_t / sqrt(dk), dv_j += p_j dy_t.
 * ------------------------------------------------------------------------ */
int oracle_backward(int64_t B, int64_t H, int64_t T, int64_t dk, int64_t dv, int64_t W,
                    const double *q, const double *k, const double *v,
                    const double *lam, const double *eta, const double *g,
                    const double *dy, double *dq, double *dkk, double *dvv,
                    double *dlam, double *deta, double *dg, int nthreads)
{
    if (B < 0 || H < 0 || T < 0 || dk < 1 || dv < 1 || W < 1) return -1;
    set_threads(nthreads);
    const int64_t nel = dk * dv;
    memset(dq, 0, (size_t)(B * H * T * dk) * sizeof(double));
    memset(dkk, 0, (size_t)(B * H * T * dk) * sizeof(double));
    memset(dvv, 0, (size_t)(B * H * T * dv) * sizeof(double));
    double *pdl = (double *)calloc((size_t)(B * H), sizeof(double));
    double *pde = (double *)calloc((size_t)(B * H), sizeof(double));
    double *pdg = (double *)calloc((size_t)(B * H), sizeof(double));
    if (!pdl || !pde || !pdg) {
        free(pdl); free(pde); free(pdg);
        return -1;
    }
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : err)
    for (int64_t bh = 0; bh < B * H; ++bh) {
        const int64_t h = bh % H;
        const double *qh = q + bh * T * dk, *kh = k + bh * T * dk, *vh = v + bh * T * dv;
        const double *dyh = dy + bh * T * dv;
        double *dqh = dq + bh * T * dk, *dkh = dkk + bh * T * dk, *dvh = dvv + bh * T * dv;
        double *As = (double *)calloc((size_t)((T + 1) * nel), sizeof(double)); /* As[t+1] = A_t */
        double *G = (double *)calloc((size_t)nel, sizeof(double));
        double *p = (double *)malloc((size_t)W * sizeof(double));
        if (!As || !G || !p) {
            err |= 1;
        } else {
            const double s = 1.0 / (1.0 + exp(-g[h]));
            const double scale = 1.0 / sqrt((double)dk);
            /* forward states */
            for (int64_t t = 0; t < T; ++t) {
                const double *Ap = As + t * nel;
                double *An = As + (t + 1) * nel;
                if (t >= W) {
                    const double *ke = kh + (t - W) * dk, *ve = vh + (t - W) * dv;
                    for (int64_t r = 0; r < dk; ++r)
                        for (int64_t c = 0; c < dv; ++c)
                            An[r * dv + c] = lam[h] * Ap[r * dv + c] + eta[h] * ke[r] * ve[c];
                } else {
                    memcpy(An, Ap, (size_t)nel * sizeof(double));
                }
            }
            /* L2: gate, dq, and the reverse state gradient */
            for (int64_t t = T - 1; t >= 0; --t) {
                const double *At = As + (t + 1) * nel;
                const double *qt = qh + t * dk, *dyt = dyh + t * dv;
                double mdy = 0.0;
                for (int64_t c = 0; c < dv; ++c) {
                    double mc = 0.0;
                    for (int64_t r = 0; r < dk; ++r) mc += qt[r] * At[r * dv + c];
                    mdy += mc * dyt[c];
                }
                pdg[bh] += s * (1.0 - s) * mdy;
                for (int64_t r = 0; r < dk; ++r) {
                    double acc = 0.0;
                    for (int64_t c = 0; c < dv; ++c) acc += At[r * dv + c] * s * dyt[c];
                    dqh[t * dk + r] += acc;
                }
                for (int64_t r = 0; r < dk; ++r)
                    for (int64_t c = 0; c < dv; ++c) G[r * dv + c] += qt[r] * s * dyt[c];
                if (t >= W) {
                    const int64_t e = t - W;
                    const double *ke = kh + e * dk, *ve = vh + e * dv;
                    const double *Ap = As + t * nel; /* A_{t-1} */
                    for (int64_t r = 0; r < dk; ++r) {
                        double acc = 0.0;
                        for (int64_t c = 0; c < dv; ++c) acc += G[r * dv + c] * ve[c];
                        dkh[e * dk + r] += eta[h] * acc;
                    }
                    for (int64_t c = 0; c < dv; ++c) {
                        double acc = 0.0;
                        for (int64_t r = 0; r < dk; ++r) acc += G[r * dv + c] * ke[r];
                        dvh[e * dv + c] += eta[h] * acc;
                    }
                    double gkv = 0.0, ga = 0.0;
                    for (int64_t r = 0; r < dk; ++r)
                        for (int64_t c = 0; c < dv; ++c) {
                            gkv += G[r * dv + c] * ke[r] * ve[c];
                            ga += G[r * dv + c] * Ap[r * dv + c];
                        }
                    pde[bh] += gkv;
                    pdl[bh] += ga;
                    for (int64_t x = 0; x < nel; ++x) G[x] *= lam[h];
                }
            }
            /* L1: window softmax backward */
            for (int64_t t = 0; t < T; ++t) {
                const double *qt = qh + t * dk, *dyt = dyh + t * dv;
                const int64_t j0 = t - W + 1 > 0 ? t - W + 1 : 0, n = t - j0 + 1;
                double smax = -INFINITY, den = 0.0;
                for (int64_t i = 0; i < n; ++i) {
                    double dot = 0.0;
                    for (int64_t r = 0; r < dk; ++r) dot += qt[r] * kh[(j0 + i) * dk + r];
                    p[i] = dot * scale;
                    if (p[i] > smax) smax = p[i];
                }
                for (int64_t i = 0; i < n; ++i) {
                    p[i] = exp(p[i] - smax);
                    den += p[i];
                }
                double Dt = 0.0;
                for (int64_t i = 0; i < n; ++i) {
                    p[i] /= den;
                    double dp = 0.0;
                    for (int64_t c = 0; c < dv; ++c) dp += dyt[c] * vh[(j0 + i) * dv + c];
                    Dt += p[i] * dp;
                }
                for (int64_t i = 0; i < n; ++i) {
                    const int64_t j = j0 + i;
                    double dp = 0.0;
                    for (int64_t c = 0; c < dv; ++c) dp += dyt[c] * vh[j * dv + c];
                    const double ds = p[i] * (dp - Dt);
                    for (int64_t r = 0; r < dk; ++r) {
                        dqh[t * dk + r] += ds * kh[j * dk + r] * scale;
                        dkh[j * dk + r] += ds * qt[r] * scale;
                    }
                    for (int64_t c = 0; c < dv; ++c) dvh[j * dv + c] += p[i] * dyt[c];
                }
            }
        }
        free(As);
        free(G);
        free(p);
    }
    for (int64_t h = 0; h < H; ++h) {
        dlam[h] = deta[h] = dg[h] = 0.0;
        for (int64_t b = 0; b < B; ++b) {
            dlam[h] += pdl[b * H + h];
            deta[h] += pde[b * H + h];
            dg[h] += pdg[b * H + h];
        }
    }
    free(pdl);
    free(pde);
    free(pdg);
    return err ? -1 : 0;
}
