/*
 * gdn_oracle.c -- fp64 CPU oracle for the gated delta rule.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or
 * calls this file; only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark do.  It shares no code, header or constant with the CUDA
 * library.
 *
 * What it computes (token by token, per (sequence b, head h), in double):
 *
 *   "Gated Delta Networks: Improving Mamba2 with Delta Rule" (paper review),
 *   section "Method":  S_t = S_{t-1} a_t (I - b_t k_t k_t^T) + b_t v_t k_t^T,
 *   with a data-dependent decay a_t in (0,1) and writing strength b_t.
 *
 * Expanded into the order used here (same value, no reassociation beyond
 * distributing S_{t-1} a_t over the bracket):
 *
 *   Sh  = S_{t-1} D_t          D_t = a_t (scalar gate) or Diag(a_t) (channel gate)
 *   p   = Sh k_t
 *   u   = b_t (v_t - p)
 *   S_t = Sh + u k_t^T
 *   o_t = S_t (scale q_t)      (read-out of the post-update state)
 *
 * a_t = exp(g_t) where g_t is the log-gate input.  The channel-gate
 * (Kimi-Delta-Attention) form replaces the scalar a_t by Diag(a_t) acting on
 * the key index, at the same position in the recurrence; the review pages
 * name that variant but do not print its equation, so this is the plain
 * reading.  With scale = 1 the read-out is o_t = S_t q_t.
 *
 * Backward: exact reverse-mode differentiation of the loop above (BPTT) for
 * the loss  L = sum_t <dO_t, o_t> + <dhT, S_T>.  States inside a chunk of
 * `ckpt` tokens are recomputed from a stored chunk-start state, so memory
 * stays at (ckpt+1) states per (b,h).
 *
 * Layouts (row-major, contiguous):
 *   q, k        [B,T,H,dk]        v, o      [B,T,H,dv]
 *   g           [B,T,H] (scalar)  or [B,T,H,dk] (channel gate)
 *   beta        [B,T,H]
 *   h0, hT, dh0 [B,H,dv,dk]       state row a = value index, column c = key index
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

int gdn_oracle_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Pointers to the token-t slices of one (b,h) stream. */
typedef struct {
    const double *q, *k, *v, *g;
    double beta;
} tok_t;

static inline tok_t token(int b, int t, int h, int T, int H, int dk, int dv,
                          int channel_gate, const double *q, const double *k,
                          const double *v, const double *g, const double *beta)
{
    tok_t r;
    size_t th = ((size_t)b * T + t) * H + h;
    r.q = q + th * dk;
    r.k = k + th * dk;
    r.v = v + th * dv;
    r.g = channel_gate ? g + th * dk : g + th;
    r.beta = beta[th];
    return r;
}

/* One token of the recurrence.  S (dv x dk) is overwritten with S_t.
 * If Sh_out is not NULL it receives the decayed state Sh; p_out receives p;
 * o (length dv) receives S_t (scale q) when not NULL. */
static void step(int dk, int dv, int channel_gate, double scale, tok_t x,
                 double *S, double *Sh_out, double *p_out, double *u_out,
                 double *o, double *work)
{
    double *p = p_out ? p_out : work;
    double *u = u_out ? u_out : work + dv;
    for (int a = 0; a < dv; ++a) {
        double *row = S + (size_t)a * dk;
        /* Sh = S D */
        if (channel_gate) {
            for (int c = 0; c < dk; ++c) row[c] *= exp(x.g[c]);
        } else {
            double al = exp(x.g[0]);
            for (int c = 0; c < dk; ++c) row[c] *= al;
        }
        if (Sh_out) memcpy(Sh_out + (size_t)a * dk, row, sizeof(double) * dk);
        double acc = 0.0;
        for (int c = 0; c < dk; ++c) acc += row[c] * x.k[c];
        p[a] = acc;
        u[a] = x.beta * (x.v[a] - acc);
        for (int c = 0; c < dk; ++c) row[c] += u[a] * x.k[c];
        if (o) {
            double oa = 0.0;
            for (int c = 0; c < dk; ++c) oa += row[c] * (scale * x.q[c]);
            o[a] = oa;
        }
    }
}

void gdn_oracle_fwd(int B, int T, int H, int dk, int dv, int channel_gate,
                    double scale, const double *q, const double *k,
                    const double *v, const double *g, const double *beta,
                    const double *h0, double *o, double *hT)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < B * H; ++bh) {
        int b = bh / H, h = bh % H;
        size_t ss = (size_t)dv * dk;
        double *S = (double *)malloc(sizeof(double) * ss);
        double *work = (double *)malloc(sizeof(double) * 2 * dv);
        if (h0) memcpy(S, h0 + (size_t)bh * ss, sizeof(double) * ss);
        else memset(S, 0, sizeof(double) * ss);
        for (int t = 0; t < T; ++t) {
            tok_t x = token(b, t, h, T, H, dk, dv, channel_gate, q, k, v, g, beta);
            size_t th = ((size_t)b * T + t) * H + h;
            step(dk, dv, channel_gate, scale, x, S, NULL, NULL, NULL,
                 o + th * dv, work);
        }
        if (hT) memcpy(hT + (size_t)bh * ss, S, sizeof(double) * ss);
        free(S);
        free(work);
    }
}

/* Single-token decode: the same step applied to N*H independent states held
 * by the caller.  q,k [N,H,dk], v,o [N,H,dv], g [N,H] or [N,H,dk],
 * beta [N,H], state [N,H,dv,dk] updated in place. */
void gdn_oracle_step(int N, int H, int dk, int dv, int channel_gate,
                     double scale, const double *q, const double *k,
                     const double *v, const double *g, const double *beta,
                     double *state, double *o)
{
#pragma omp parallel for schedule(static)
    for (int nh = 0; nh < N * H; ++nh) {
        double work[2 * 512];
        double *wk = dv <= 512 ? work : (double *)malloc(sizeof(double) * 2 * dv);
        int n = nh / H, h = nh % H;
        tok_t x = token(n, 0, h, 1, H, dk, dv, channel_gate, q, k, v, g, beta);
        step(dk, dv, channel_gate, scale, x, state + (size_t)nh * dv * dk,
             NULL, NULL, NULL, o + (size_t)nh * dv, wk);
        if (wk != work) free(wk);
    }
}

/*
 * Backward by reverse-mode differentiation of `step`, token by token, for
 * L = sum_t <dO_t, o_t> + <dhT, S_T>.  With dS the gradient w.r.t. S_t:
 *
 *   dS   += dO_t (scale q_t)^T          dq_t  = scale S_t^T dO_t
 *   du    = dS k_t                      dk_t  = dS^T u
 *   dbeta = <du, v_t - p>               dv_t  = beta du
 *   dp    = -beta du
 *   dSh   = dS + dp k_t^T               dk_t += Sh^T dp
 *   da    = sum(dSh .* S_{t-1})  (scalar) | column sums of dSh .* S_{t-1} (channel)
 *   dg_t  = da .* a_t                   dS_{t-1} = dSh D_t
 *
 * dh0 is the final dS.  `ckpt` tokens per recomputation chunk.
 */
void gdn_oracle_bwd(int B, int T, int H, int dk, int dv, int channel_gate,
                    double scale, const double *q, const double *k,
                    const double *v, const double *g, const double *beta,
                    const double *h0, const double *dO, const double *dhT,
                    double *dq, double *dkk, double *dvv, double *dg,
                    double *dbeta, double *dh0, int ckpt)
{
    if (ckpt < 1) ckpt = 64;
    int nck = (T + ckpt - 1) / ckpt;
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < B * H; ++bh) {
        int b = bh / H, h = bh % H;
        size_t ss = (size_t)dv * dk;
        double *starts = (double *)malloc(sizeof(double) * ss * (nck + 1));
        double *Sts = (double *)malloc(sizeof(double) * ss * (ckpt + 1)); /* S_{t0-1} .. S_{t1-1} */
        double *Shs = (double *)malloc(sizeof(double) * ss * ckpt);
        double *ps = (double *)malloc(sizeof(double) * dv * ckpt);
        double *us = (double *)malloc(sizeof(double) * dv * ckpt);
        double *dS = (double *)malloc(sizeof(double) * ss);
        double *work = (double *)malloc(sizeof(double) * 2 * dv);
        double *du = (double *)malloc(sizeof(double) * dv);
        double *dp = (double *)malloc(sizeof(double) * dv);
        double *da = (double *)malloc(sizeof(double) * dk);

        /* forward pass: store the state entering each checkpoint chunk */
        double *S = starts;
        if (h0) memcpy(S, h0 + (size_t)bh * ss, sizeof(double) * ss);
        else memset(S, 0, sizeof(double) * ss);
        for (int n = 0; n < nck; ++n) {
            memcpy(starts + (size_t)(n + 1) * ss, starts + (size_t)n * ss, sizeof(double) * ss);
            double *Sn = starts + (size_t)(n + 1) * ss;
            int t1 = (n + 1) * ckpt < T ? (n + 1) * ckpt : T;
            for (int t = n * ckpt; t < t1; ++t) {
                tok_t x = token(b, t, h, T, H, dk, dv, channel_gate, q, k, v, g, beta);
                step(dk, dv, channel_gate, scale, x, Sn, NULL, NULL, NULL, NULL, work);
            }
        }
        /* dS = dL/dS_T */
        if (dhT) memcpy(dS, dhT + (size_t)bh * ss, sizeof(double) * ss);
        else memset(dS, 0, sizeof(double) * ss);

        for (int n = nck - 1; n >= 0; --n) {
            int t0 = n * ckpt;
            int t1 = (n + 1) * ckpt < T ? (n + 1) * ckpt : T;
            int len = t1 - t0;
            /* recompute S_{t-1}, Sh_t, p_t, u_t inside the chunk */
            memcpy(Sts, starts + (size_t)n * ss, sizeof(double) * ss);
            for (int j = 0; j < len; ++j) {
                tok_t x = token(b, t0 + j, h, T, H, dk, dv, channel_gate, q, k, v, g, beta);
                memcpy(Sts + (size_t)(j + 1) * ss, Sts + (size_t)j * ss, sizeof(double) * ss);
                step(dk, dv, channel_gate, scale, x, Sts + (size_t)(j + 1) * ss,
                     Shs + (size_t)j * ss, ps + (size_t)j * dv, us + (size_t)j * dv,
                     NULL, work);
            }
            for (int j = len - 1; j >= 0; --j) {
                int t = t0 + j;
                tok_t x = token(b, t, h, T, H, dk, dv, channel_gate, q, k, v, g, beta);
                size_t th = ((size_t)b * T + t) * H + h;
                const double *St = Sts + (size_t)(j + 1) * ss;   /* S_t     */
                const double *Sp = Sts + (size_t)j * ss;         /* S_{t-1} */
                const double *Sh = Shs + (size_t)j * ss;
                const double *p = ps + (size_t)j * dv;
                const double *u = us + (size_t)j * dv;
                const double *dot = dO + th * dv;
                double *dqt = dq + th * dk, *dkt = dkk + th * dk, *dvt = dvv + th * dv;
                /* o_t = S_t (scale q_t) */
                for (int c = 0; c < dk; ++c) {
                    double acc = 0.0;
                    for (int a = 0; a < dv; ++a) acc += St[(size_t)a * dk + c] * dot[a];
                    dqt[c] = scale * acc;
                }
                for (int a = 0; a < dv; ++a)
                    for (int c = 0; c < dk; ++c)
                        dS[(size_t)a * dk + c] += dot[a] * scale * x.q[c];
                /* S_t = Sh + u k^T */
                for (int a = 0; a < dv; ++a) {
                    double acc = 0.0;
                    for (int c = 0; c < dk; ++c) acc += dS[(size_t)a * dk + c] * x.k[c];
                    du[a] = acc;
                }
                for (int c = 0; c < dk; ++c) {
                    double acc = 0.0;
                    for (int a = 0; a < dv; ++a) acc += dS[(size_t)a * dk + c] * u[a];
                    dkt[c] = acc;
                }
                /* u = beta (v - p) */
                double db = 0.0;
                for (int a = 0; a < dv; ++a) {
                    db += du[a] * (x.v[a] - p[a]);
                    dvt[a] = x.beta * du[a];
                    dp[a] = -x.beta * du[a];
                }
                dbeta[th] = db;
                /* p = Sh k:  dSh = dS + dp k^T ;  dk += Sh^T dp */
                for (int c = 0; c < dk; ++c) {
                    double acc = 0.0;
                    for (int a = 0; a < dv; ++a) acc += Sh[(size_t)a * dk + c] * dp[a];
                    dkt[c] += acc;
                }
                for (int a = 0; a < dv; ++a)
                    for (int c = 0; c < dk; ++c)
                        dS[(size_t)a * dk + c] += dp[a] * x.k[c];
                /* Sh = S_{t-1} D_t */
                for (int c = 0; c < dk; ++c) da[c] = 0.0;
                for (int a = 0; a < dv; ++a)
                    for (int c = 0; c < dk; ++c)
                        da[c] += dS[(size_t)a * dk + c] * Sp[(size_t)a * dk + c];
                if (channel_gate) {
                    for (int c = 0; c < dk; ++c) {
                        double al = exp(x.g[c]);
                        dg[th * dk + c] = da[c] * al;
                        for (int a = 0; a < dv; ++a) dS[(size_t)a * dk + c] *= al;
                    }
                } else {
                    double al = exp(x.g[0]), s = 0.0;
                    for (int c = 0; c < dk; ++c) s += da[c];
                    dg[th] = s * al;
                    for (size_t e = 0; e < ss; ++e) dS[e] *= al;
                }
            }
        }
        if (dh0) memcpy(dh0 + (size_t)bh * ss, dS, sizeof(double) * ss);
        free(starts); free(Sts); free(Shs); free(ps); free(us); free(dS);
        free(work); free(du); free(dp); free(da);
    }
}
