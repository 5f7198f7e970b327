/*
 * gdr2_oracle.c -- plain fp64 CPU oracle for the Gated Delta Rule-2 (GDR-2)
 * token mixer of "Gated DeltaNet-2: Decoupling Erase and Write in Linear
 * Attention" (Hatamizadeh, Choi, Kautz).
 *
 * TEST INFRASTRUCTURE. This file is the checker, not the product: only the
 * tests, the smoke check and the CPU-baseline leg of the benchmark load it.
 * It shares no code, header, table or constant with the CUDA library.
 *
 * What it computes (one independent recurrence per (batch, head)), written
 * token by token with no blocking, fusion or reordering:
 *
 *   a_t  = exp(log_alpha_t)          channel decay, in (0,1]^dk (0 allowed)
 *   e_t  = b_t (.) k_t               erase-gated key  (key side, dk)
 *   z_t  = w_t (.) v_t               write-gated value (value side, dv)
 *   Sb   = Diag(a_t) S_{t-1}         decayed state, S is dk x dv
 *   r_t  = Sb^T e_t                  read along the gated key
 *   S_t  = Sb + k_t (z_t - r_t)^T    = (I - k_t e_t^T) Sb + k_t z_t^T
 *   o_t  = S_t^T q_t                 output read by the query (post-update)
 *
 * Source passages (Gated DeltaNet-2 note, graygoo.forestry.md):
 *   - sec. 3 "Technical Architecture", forward-pass paragraph: the gated key
 *     e = b(.)k, the gated value z = w(.)v, the decay Sb = Diag(alpha) S and
 *     the read r = Sb^T e, in that order;
 *   - sec. 2 "Theoretical Framework", fast-weight objective: S_t minimises
 *     ||S - Sb||_F^2 - 2 <S^T k, z - Sb^T e>, whose stationary point is the
 *     update above with the erase outer product taken along k;
 *   - sec. 3, gate-aware backward paragraph: the asymmetric factor
 *     (I - k_t e_t^T).
 * The forward-pass paragraph writes the erase term as e_t r_t^T; read
 * literally, b would enter the erase squared and the KDA reduction stated in
 * sec. 2 (b = w = beta*1) would fail. The objective and the asymmetric
 * factor both place k_t on the left, and that is the reading taken here.
 *
 * Layouts (row-major, contiguous):
 *   q, k, log_alpha, b : [B, T, H, dk]     v, w, o : [B, T, H, dv]
 *   S0, S_T, dS0, dS_T : [B, H, dk, dv]   (row = key channel, col = value)
 * Decode-step layouts drop T: q,k,... [N, H, d], S [N, H, dk, dv].
 *
 * Every entry point returns 0 on success, 1 for invalid arguments and 2 when
 * scratch memory cannot be allocated. Nothing is clamped: log_alpha = -inf
 * (alpha = 0) is a full reset.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_BAD_ARG 1
#define ORACLE_NO_MEM 2

/* Token-major element offset of [b, t, h, :] in a [B, T, H, D] tensor. */
static size_t tok_off(int b, int t, int h, int T, int H, int D)
{
    return (((size_t)b * T + t) * H + h) * (size_t)D;
}

/* One token of the recurrence, in place on S (dk x dv, row-major).
 * Gated DeltaNet-2 note, sec. 3 forward-pass paragraph (gates, decay, read)
 * with the erase outer product along k (sec. 2 objective, sec. 3 backward
 * paragraph). Writes o_t = S_t^T q_t when o is not NULL.
 * scratch: 2*dk + 2*dv doubles. */
static void gdr2_token(int dk, int dv, double *S,
                       const double *q, const double *k, const double *v,
                       const double *la, const double *b, const double *w,
                       double *o, double *scratch)
{
    double *a = scratch;            /* dk */
    double *e = a + dk;             /* dk */
    double *z = e + dk;             /* dv */
    double *r = z + dv;             /* dv */
    for (int c = 0; c < dk; ++c) {
        a[c] = exp(la[c]);
        e[c] = b[c] * k[c];
    }
    for (int j = 0; j < dv; ++j) z[j] = w[j] * v[j];
    /* Sb = Diag(a) S */
    for (int c = 0; c < dk; ++c)
        for (int j = 0; j < dv; ++j) S[(size_t)c * dv + j] *= a[c];
    /* r = Sb^T e */
    for (int j = 0; j < dv; ++j) {
        double acc = 0.0;
        for (int c = 0; c < dk; ++c) acc += S[(size_t)c * dv + j] * e[c];
        r[j] = acc;
    }
    /* S = Sb + k (z - r)^T */
    for (int c = 0; c < dk; ++c)
        for (int j = 0; j < dv; ++j) S[(size_t)c * dv + j] += k[c] * (z[j] - r[j]);
    /* o = S^T q */
    if (o) {
        for (int j = 0; j < dv; ++j) {
            double acc = 0.0;
            for (int c = 0; c < dk; ++c) acc += S[(size_t)c * dv + j] * q[c];
            o[j] = acc;
        }
    }
}

static int resolve_threads(int nthreads)
{
#ifdef _OPENMP
    return nthreads > 0 ? nthreads : omp_get_max_threads();
#else
    (void)nthreads;
    return 1;
#endif
}

/* Full-sequence forward: for every (b, h), S starts at S0 (zeros when S0 is
 * NULL) and the token recurrence runs t = 0..T-1. o may be NULL (states only),
 * S_T may be NULL. Gated DeltaNet-2 note, sec. 2-3 (see file header). */
int gdr2_oracle_forward(int B, int T, int H, int dk, int dv,
                        const double *q, const double *k, const double *v,
                        const double *log_alpha, const double *b, const double *w,
                        const double *S0, double *o, double *S_T, int nthreads)
{
    if (B < 0 || T < 0 || H < 0 || dk <= 0 || dv <= 0) return ORACLE_BAD_ARG;
    if (T > 0 && (!q || !k || !v || !log_alpha || !b || !w)) return ORACLE_BAD_ARG;
    const int BH = B * H;
    const size_t SS = (size_t)dk * dv;
    int err = ORACLE_OK;
    int nt = resolve_threads(nthreads);
#pragma omp parallel for num_threads(nt) schedule(dynamic, 1)
    for (int bh = 0; bh < BH; ++bh) {
        const int bb = bh / H, h = bh % H;
        double *S = (double *)malloc(sizeof(double) * (SS + 2 * (size_t)dk + 2 * (size_t)dv));
        if (!S) {
#pragma omp atomic write
            err = ORACLE_NO_MEM;
            continue;
        }
        double *scratch = S + SS;
        if (S0) memcpy(S, S0 + (size_t)bh * SS, sizeof(double) * SS);
        else memset(S, 0, sizeof(double) * SS);
        for (int t = 0; t < T; ++t) {
            const size_t ok = tok_off(bb, t, h, T, H, dk), ov = tok_off(bb, t, h, T, H, dv);
            gdr2_token(dk, dv, S, q + ok, k + ok, v + ov, log_alpha + ok, b + ok, w + ov,
                       o ? o + ov : NULL, scratch);
        }
        if (S_T) memcpy(S_T + (size_t)bh * SS, S, sizeof(double) * SS);
        free(S);
    }
    return err;
}

/* One recurrent decode step (constant-memory inference, Gated DeltaNet-2 note
 * sec. 1): the same token update applied once to each of N*H resident states,
 * S updated in place, o = S_t^T q_t. */
int gdr2_oracle_decode_step(int N, int H, int dk, int dv,
                            const double *q, const double *k, const double *v,
                            const double *log_alpha, const double *b, const double *w,
                            double *S, double *o, int nthreads)
{
    if (N < 0 || H < 0 || dk <= 0 || dv <= 0) return ORACLE_BAD_ARG;
    if (N * H > 0 && (!q || !k || !v || !log_alpha || !b || !w || !S)) return ORACLE_BAD_ARG;
    const int NH = N * H;
    const size_t SS = (size_t)dk * dv;
    int err = ORACLE_OK;
    int nt = resolve_threads(nthreads);
#pragma omp parallel for num_threads(nt) schedule(static)
    for (int nh = 0; nh < NH; ++nh) {
        double *scratch = (double *)malloc(sizeof(double) * (2 * (size_t)dk + 2 * (size_t)dv));
        if (!scratch) {
#pragma omp atomic write
            err = ORACLE_NO_MEM;
            continue;
        }
        gdr2_token(dk, dv, S + (size_t)nh * SS, q + (size_t)nh * dk, k + (size_t)nh * dk,
                   v + (size_t)nh * dv, log_alpha + (size_t)nh * dk, b + (size_t)nh * dk,
                   w + (size_t)nh * dv, o ? o + (size_t)nh * dv : NULL, scratch);
        free(scratch);
    }
    return err;
}

/* Reverse-mode gradient of the token recurrence (the gate-aware backward of
 * Gated DeltaNet-2 note sec. 3, taken here token by token rather than per
 * chunk). With Sb = Diag(a) S_{t-1}, delta = z - Sb^T e, S_t = Sb + k delta^T,
 * o_t = S_t^T q and dS the gradient reaching S_t from later tokens:
 *   dS  += q dO_t^T            dq = S_t dO_t
 *   dk   = dS delta            ddelta = dS^T k
 *   dw   = ddelta (.) v        dv = ddelta (.) w
 *   de   = -Sb ddelta          db = de (.) k,   dk += de (.) b
 *   dSb  = dS - e ddelta^T     dlog_alpha_c = sum_j dSb[c,j] Sb[c,j]
 *   dS   = Diag(a) dSb          (gradient reaching S_{t-1})
 * dS starts at dS_T (zeros when NULL); dS0 receives the final dS.
 * States are checkpointed every CKPT tokens and recomputed forward inside
 * each segment, so memory is O((T/CKPT + CKPT) dk dv) per (b, h). */
#define CKPT 64
int gdr2_oracle_backward(int B, int T, int H, int dk, int dv,
                         const double *q, const double *k, const double *v,
                         const double *log_alpha, const double *b, const double *w,
                         const double *S0, const double *dO, const double *dS_T,
                         double *dq, double *dk_out, double *dv_out, double *dlog_alpha,
                         double *db, double *dw, double *dS0, int nthreads)
{
    if (B < 0 || T < 0 || H < 0 || dk <= 0 || dv <= 0) return ORACLE_BAD_ARG;
    if (T > 0 && (!q || !k || !v || !log_alpha || !b || !w || !dO || !dq || !dk_out ||
                  !dv_out || !dlog_alpha || !db || !dw))
        return ORACLE_BAD_ARG;
    const int BH = B * H;
    const size_t SS = (size_t)dk * dv;
    const int nseg = (T + CKPT - 1) / CKPT;
    int err = ORACLE_OK;
    int nt = resolve_threads(nthreads);
#pragma omp parallel for num_threads(nt) schedule(dynamic, 1)
    for (int bh = 0; bh < BH; ++bh) {
        const int bb = bh / H, h = bh % H;
        /* ckpt: nseg+1 states; seg: CKPT+1 states; dS, Sb, dSb; then the
         * per-token vectors a, e, de (dk each), delta, ddelta, z (dv each)
         * and the token-step scratch (2dk + 2dv). */
        size_t need = SS * ((size_t)nseg + 1 + CKPT + 1 + 3) + 5 * (size_t)dk + 5 * (size_t)dv;
        double *mem = (double *)malloc(sizeof(double) * need);
        if (!mem) {
#pragma omp atomic write
            err = ORACLE_NO_MEM;
            continue;
        }
        double *ckpt = mem;
        double *seg = ckpt + SS * ((size_t)nseg + 1);
        double *dS = seg + SS * (CKPT + 1);
        double *Sb = dS + SS;
        double *dSb = Sb + SS;
        double *a = dSb + SS, *e = a + dk, *de = e + dk;
        double *delta = de + dk, *ddelta = delta + dv, *zz = ddelta + dv;
        double *scratch = zz + dv;

        /* forward pass storing the state at every segment start */
        if (S0) memcpy(ckpt, S0 + (size_t)bh * SS, sizeof(double) * SS);
        else memset(ckpt, 0, sizeof(double) * SS);
        for (int s = 0; s < nseg; ++s) {
            double *S = ckpt + SS * ((size_t)s + 1);
            memcpy(S, ckpt + SS * (size_t)s, sizeof(double) * SS);
            const int t1 = (s + 1) * CKPT < T ? (s + 1) * CKPT : T;
            for (int t = s * CKPT; t < t1; ++t) {
                const size_t ok = tok_off(bb, t, h, T, H, dk), ov = tok_off(bb, t, h, T, H, dv);
                gdr2_token(dk, dv, S, q + ok, k + ok, v + ov, log_alpha + ok, b + ok, w + ov,
                           NULL, scratch);
            }
        }

        if (dS_T) memcpy(dS, dS_T + (size_t)bh * SS, sizeof(double) * SS);
        else memset(dS, 0, sizeof(double) * SS);

        for (int s = nseg - 1; s >= 0; --s) {
            const int t0 = s * CKPT;
            const int t1 = (s + 1) * CKPT < T ? (s + 1) * CKPT : T;
            /* seg[i] = state after tokens < t0 + i, i = 0..t1-t0 */
            memcpy(seg, ckpt + SS * (size_t)s, sizeof(double) * SS);
            for (int t = t0; t < t1; ++t) {
                double *Sn = seg + SS * ((size_t)(t - t0) + 1);
                memcpy(Sn, seg + SS * (size_t)(t - t0), sizeof(double) * SS);
                const size_t ok = tok_off(bb, t, h, T, H, dk), ov = tok_off(bb, t, h, T, H, dv);
                gdr2_token(dk, dv, Sn, q + ok, k + ok, v + ov, log_alpha + ok, b + ok, w + ov,
                           NULL, scratch);
            }
            for (int t = t1 - 1; t >= t0; --t) {
                const size_t ok = tok_off(bb, t, h, T, H, dk), ov = tok_off(bb, t, h, T, H, dv);
                const double *qt = q + ok, *kt = k + ok, *lat = log_alpha + ok, *bt = b + ok;
                const double *vt = v + ov, *wt = w + ov, *dOt = dO + ov;
                const double *Sprev = seg + SS * (size_t)(t - t0);
                const double *Scur = seg + SS * ((size_t)(t - t0) + 1);
                for (int c = 0; c < dk; ++c) {
                    a[c] = exp(lat[c]);
                    e[c] = bt[c] * kt[c];
                }
                for (int j = 0; j < dv; ++j) zz[j] = wt[j] * vt[j];
                for (int c = 0; c < dk; ++c)
                    for (int j = 0; j < dv; ++j) Sb[(size_t)c * dv + j] = a[c] * Sprev[(size_t)c * dv + j];
                for (int j = 0; j < dv; ++j) {
                    double acc = 0.0;
                    for (int c = 0; c < dk; ++c) acc += Sb[(size_t)c * dv + j] * e[c];
                    delta[j] = zz[j] - acc;
                }
                /* o_t = S_t^T q_t */
                for (int c = 0; c < dk; ++c)
                    for (int j = 0; j < dv; ++j) dS[(size_t)c * dv + j] += qt[c] * dOt[j];
                double *dqt = dq + ok, *dkt = dk_out + ok, *dbt = db + ok, *dlat = dlog_alpha + ok;
                double *dvt = dv_out + ov, *dwt = dw + ov;
                for (int c = 0; c < dk; ++c) {
                    double acc = 0.0;
                    for (int j = 0; j < dv; ++j) acc += Scur[(size_t)c * dv + j] * dOt[j];
                    dqt[c] = acc;
                }
                /* S_t = Sb + k delta^T */
                for (int c = 0; c < dk; ++c) {
                    double acc = 0.0;
                    for (int j = 0; j < dv; ++j) acc += dS[(size_t)c * dv + j] * delta[j];
                    dkt[c] = acc;
                }
                for (int j = 0; j < dv; ++j) {
                    double acc = 0.0;
                    for (int c = 0; c < dk; ++c) acc += dS[(size_t)c * dv + j] * kt[c];
                    ddelta[j] = acc;
                }
                /* delta = z - Sb^T e,  z = w (.) v */
                for (int j = 0; j < dv; ++j) {
                    dwt[j] = ddelta[j] * vt[j];
                    dvt[j] = ddelta[j] * wt[j];
                }
                for (int c = 0; c < dk; ++c) {
                    double acc = 0.0;
                    for (int j = 0; j < dv; ++j) acc += Sb[(size_t)c * dv + j] * ddelta[j];
                    de[c] = -acc;
                }
                /* e = b (.) k */
                for (int c = 0; c < dk; ++c) {
                    dbt[c] = de[c] * kt[c];
                    dkt[c] += de[c] * bt[c];
                }
                /* dSb = dS - e ddelta^T; Sb = Diag(a) S_{t-1} */
                for (int c = 0; c < dk; ++c) {
                    double acc = 0.0;
                    for (int j = 0; j < dv; ++j) {
                        const double g = dS[(size_t)c * dv + j] - e[c] * ddelta[j];
                        dSb[(size_t)c * dv + j] = g;
                        acc += g * Sb[(size_t)c * dv + j];
                    }
                    dlat[c] = acc;
                }
                for (int c = 0; c < dk; ++c)
                    for (int j = 0; j < dv; ++j) dS[(size_t)c * dv + j] = a[c] * dSb[(size_t)c * dv + j];
            }
        }
        if (dS0) memcpy(dS0 + (size_t)bh * SS, dS, sizeof(double) * SS);
        free(mem);
    }
    return err;
}
