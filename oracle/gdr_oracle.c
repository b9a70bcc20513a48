/*
 * CPU oracle for the gated delta-rule recurrence -- TEST INFRASTRUCTURE ONLY.
 *
 * Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may load
 * this library. It shares no code with the CUDA path.
 *
 * What it computes (plain definition, fp64, one token at a time):
 *
 *   S_t = (I - k_t^T (b_t . k_t)) Diag(alpha_t) S_{t-1} + (w_t . k_t)^T v_t
 *   o_t = q_t S_t
 *
 * with row vectors k, q, b, w, alpha (length d_k) and v, o (length d_v), and
 * the state S of size d_k x d_v ("." is the elementwise product).
 *
 * Sources:
 *   - write S <- S + k^T v and read o = q S, row-vector convention:
 *     "Recurrent Memory: Write, Erase, Decay, Read", section 01 (equations).
 *   - erase before write (delta rule, S <- (I - beta k^T k) S + beta k^T v):
 *     same page, section 03; "The Eraser Trilogy", "Eraser two".
 *   - decay Diag(alpha) with channel-wise alpha (KDA) and the unified
 *     equation: same page, sections 04-05; "The Eraser Trilogy", "Eraser three".
 *   - separate channel-wise erase gate b and write gate w, decay absorbed into
 *     the erase factor (decay applied before the erase): "Erase-then-Delta
 *     Attention" (Gated DeltaNet-2), abstract.
 *   - state S in R^{d_k x d_v}, read o_t from S_t: "How Linear Attention
 *     Remembers", Analytical Framework (state update and read equations).
 *
 * Gate conventions: a NULL alpha means alpha = 1; a NULL b means b = 0; a NULL
 * w means w = 1. A gate with per_channel = 0 holds one value per token-head
 * ([B,T,H]) used for every channel; per_channel = 1 holds [B,T,H,d_k].
 *
 * Layouts (contiguous, row-major): q,k [B,T,H,dk]; v,o [B,T,H,dv];
 * S0,S_T [B,H,dk,dv].
 */
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

static double gate_at(const double* g, int per_channel, long tok, int dk, int i, double dflt) {
    if (!g) return dflt;
    return per_channel ? g[tok * dk + i] : g[tok];
}

/* Runs the recurrence for one head (bi, hi) over all T tokens. */
static void run_head(int bi, int hi, int T, int H, int dk, int dv,
                     const double* q, const double* k, const double* v,
                     const double* alpha, int alpha_pc,
                     const double* b, int b_pc,
                     const double* w, int w_pc,
                     const double* S0, double* o, double* S_T,
                     double* S, double* r) {
    long head = (long)bi * H + hi;
    if (S0) memcpy(S, S0 + head * dk * dv, sizeof(double) * dk * dv);
    else memset(S, 0, sizeof(double) * dk * dv);
    for (int t = 0; t < T; ++t) {
        long tok = ((long)bi * T + t) * H + hi; /* index into [B,T,H] */
        const double* kt = k + tok * dk;
        const double* qt = q + tok * dk;
        const double* vt = v + tok * dv;
        /* decay: S <- Diag(alpha_t) S */
        for (int i = 0; i < dk; ++i) {
            double a = gate_at(alpha, alpha_pc, tok, dk, i, 1.0);
            for (int j = 0; j < dv; ++j) S[i * dv + j] *= a;
        }
        /* erase read: r = (b_t . k_t) S  (1 x dv) */
        for (int j = 0; j < dv; ++j) r[j] = 0.0;
        for (int i = 0; i < dk; ++i) {
            double bk = gate_at(b, b_pc, tok, dk, i, 0.0) * kt[i];
            for (int j = 0; j < dv; ++j) r[j] += bk * S[i * dv + j];
        }
        /* erase along k_t, write (w_t . k_t)^T v_t */
        for (int i = 0; i < dk; ++i) {
            double wk = gate_at(w, w_pc, tok, dk, i, 1.0) * kt[i];
            for (int j = 0; j < dv; ++j) S[i * dv + j] += -kt[i] * r[j] + wk * vt[j];
        }
        /* read: o_t = q_t S_t */
        double* ot = o + tok * dv;
        for (int j = 0; j < dv; ++j) ot[j] = 0.0;
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) ot[j] += qt[i] * S[i * dv + j];
    }
    if (S_T) memcpy(S_T + head * dk * dv, S, sizeof(double) * dk * dv);
}

/* Returns 0 on success, -1 on bad arguments, -2 on allocation failure. */
int gdr_oracle_forward(int B, int T, int H, int dk, int dv,
                       const double* q, const double* k, const double* v,
                       const double* alpha, int alpha_per_channel,
                       const double* b, int b_per_channel,
                       const double* w, int w_per_channel,
                       const double* S0, double* o, double* S_T, int nthreads) {
    if (B < 0 || T < 0 || H < 0 || dk <= 0 || dv <= 0) return -1;
    if ((T > 0 && (!q || !k || !v || !o))) return -1;
    int nheads = B * H;
    int err = 0;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel
#endif
    {
        double* S = (double*)malloc(sizeof(double) * (size_t)dk * dv);
        double* r = (double*)malloc(sizeof(double) * (size_t)dv);
        if (!S || !r) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
            err = -2;
        } else {
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
            for (int hd = 0; hd < nheads; ++hd)
                run_head(hd / H, hd % H, T, H, dk, dv, q, k, v, alpha, alpha_per_channel,
                         b, b_per_channel, w, w_per_channel, S0, o, S_T, S, r);
        }
        free(S);
        free(r);
    }
    (void)nthreads;
    return err;
}

/*
 * Backward pass: the gradient of a scalar loss L with respect to every input,
 * given dL/do_t (dO) and dL/dS_T (dS_T, NULL = 0).
 *
 * The pages ask for a gate-aware backward pass ("Erase-then-Delta Attention"
 * (Gated DeltaNet-2), abstract) but print no formula for it, so this is the
 * plain definition: reverse-mode differentiation of the token loop above,
 * one step at a time, with every state S_0 .. S_T of the forward kept. With
 * e = b . k (erase key), u = w . k (write key), S' = Diag(alpha) S_{t-1},
 * r = e S' and S_t = S' - k^T r + u^T v, o_t = q_t S_t, and G = dL/dS_t:
 *
 *   dq_t = dO_t S_t^T                 G += q_t^T dO_t
 *   dv_t = u G                        du = G v^T       dk <- -G r^T
 *   dr   = -k G                       de = S' dr^T     dS' = G + e^T dr
 *   dalpha_i = sum_j dS'_ij S_{t-1,ij}                 G <- Diag(alpha) dS'
 *   dk += b . de + w . du,  db = k . de,  dw = k . du
 *
 * ending with dS0 = G. A scalar gate's gradient is the sum over channels of
 * the per-channel one. Outputs dalpha / db / dw may be NULL (gate absent); the
 * caller handles tied gates (w := b) by passing b as w and adding dw to db.
 * Layouts: dq, dk [B,T,H,dk]; dv [B,T,H,dv]; gate gradients the gate's own
 * layout; dS0 [B,H,dk,dv] (may be NULL).
 */
static void bwd_head(int bi, int hi, int T, int H, int dk, int dv,
                     const double* q, const double* k, const double* v,
                     const double* alpha, int alpha_pc, const double* b, int b_pc,
                     const double* w, int w_pc, const double* S0, const double* dO,
                     const double* dS_T, double* dq, double* dk_out, double* dv_out,
                     double* dalpha, double* db, double* dw, double* dS0,
                     double* Sall, double* G, double* Sd, double* r, double* dr,
                     double* de, double* du) {
    const long head = (long)bi * H + hi;
    const long SZ = (long)dk * dv;
    /* forward, keeping S_0 .. S_T */
    if (S0) memcpy(Sall, S0 + head * SZ, sizeof(double) * SZ);
    else memset(Sall, 0, sizeof(double) * SZ);
    for (int t = 0; t < T; ++t) {
        long tok = ((long)bi * T + t) * H + hi;
        const double* kt = k + tok * dk;
        const double* vt = v + tok * dv;
        const double* Sp = Sall + (long)t * SZ;
        double* Sn = Sall + (long)(t + 1) * SZ;
        for (int i = 0; i < dk; ++i) {
            double a = gate_at(alpha, alpha_pc, tok, dk, i, 1.0);
            for (int j = 0; j < dv; ++j) Sd[i * dv + j] = a * Sp[i * dv + j];
        }
        for (int j = 0; j < dv; ++j) r[j] = 0.0;
        for (int i = 0; i < dk; ++i) {
            double e = gate_at(b, b_pc, tok, dk, i, 0.0) * kt[i];
            for (int j = 0; j < dv; ++j) r[j] += e * Sd[i * dv + j];
        }
        for (int i = 0; i < dk; ++i) {
            double u = gate_at(w, w_pc, tok, dk, i, 1.0) * kt[i];
            for (int j = 0; j < dv; ++j) Sn[i * dv + j] = Sd[i * dv + j] - kt[i] * r[j] + u * vt[j];
        }
    }
    /* reverse */
    if (dS_T) memcpy(G, dS_T + head * SZ, sizeof(double) * SZ);
    else memset(G, 0, sizeof(double) * SZ);
    for (int t = T - 1; t >= 0; --t) {
        long tok = ((long)bi * T + t) * H + hi;
        const double* qt = q + tok * dk;
        const double* kt = k + tok * dk;
        const double* vt = v + tok * dv;
        const double* dot = dO + tok * dv;
        const double* Sp = Sall + (long)t * SZ;       /* S_{t-1} */
        const double* St = Sall + (long)(t + 1) * SZ; /* S_t */
        /* o_t = q_t S_t */
        for (int i = 0; i < dk; ++i) {
            double acc = 0.0;
            for (int j = 0; j < dv; ++j) acc += St[i * dv + j] * dot[j];
            dq[tok * dk + i] = acc;
            for (int j = 0; j < dv; ++j) G[i * dv + j] += qt[i] * dot[j];
        }
        /* recompute S' and r of this step */
        for (int i = 0; i < dk; ++i) {
            double a = gate_at(alpha, alpha_pc, tok, dk, i, 1.0);
            for (int j = 0; j < dv; ++j) Sd[i * dv + j] = a * Sp[i * dv + j];
        }
        for (int j = 0; j < dv; ++j) r[j] = 0.0;
        for (int i = 0; i < dk; ++i) {
            double e = gate_at(b, b_pc, tok, dk, i, 0.0) * kt[i];
            for (int j = 0; j < dv; ++j) r[j] += e * Sd[i * dv + j];
        }
        /* S_t = S' - k^T r + u^T v */
        for (int j = 0; j < dv; ++j) {
            double accv = 0.0, accr = 0.0;
            for (int i = 0; i < dk; ++i) {
                double u = gate_at(w, w_pc, tok, dk, i, 1.0) * kt[i];
                accv += u * G[i * dv + j];
                accr += kt[i] * G[i * dv + j];
            }
            dv_out[tok * dv + j] = accv;
            dr[j] = -accr;
        }
        for (int i = 0; i < dk; ++i) {
            double accu = 0.0, acck = 0.0, acce = 0.0;
            for (int j = 0; j < dv; ++j) {
                accu += G[i * dv + j] * vt[j];
                acck += G[i * dv + j] * r[j];
                acce += Sd[i * dv + j] * dr[j]; /* r = e S' */
            }
            du[i] = accu;
            de[i] = acce;
            dk_out[tok * dk + i] = -acck;
        }
        /* dS' = G + e^T dr; S' = Diag(alpha) S_{t-1} */
        double dal_sum = 0.0, db_sum = 0.0, dw_sum = 0.0;
        for (int i = 0; i < dk; ++i) {
            double a = gate_at(alpha, alpha_pc, tok, dk, i, 1.0);
            double bi_ = gate_at(b, b_pc, tok, dk, i, 0.0);
            double wi = gate_at(w, w_pc, tok, dk, i, 1.0);
            double e = bi_ * kt[i];
            double dal = 0.0;
            for (int j = 0; j < dv; ++j) {
                double dsd = G[i * dv + j] + e * dr[j];
                dal += dsd * Sp[i * dv + j];
                G[i * dv + j] = a * dsd;
            }
            dk_out[tok * dk + i] += bi_ * de[i] + wi * du[i];
            if (dalpha && alpha_pc) dalpha[tok * dk + i] = dal;
            if (db && b_pc) db[tok * dk + i] = kt[i] * de[i];
            if (dw && w_pc) dw[tok * dk + i] = kt[i] * du[i];
            dal_sum += dal;
            db_sum += kt[i] * de[i];
            dw_sum += kt[i] * du[i];
        }
        if (dalpha && !alpha_pc) dalpha[tok] = dal_sum;
        if (db && !b_pc) db[tok] = db_sum;
        if (dw && !w_pc) dw[tok] = dw_sum;
    }
    if (dS0) memcpy(dS0 + head * SZ, G, sizeof(double) * SZ);
}

/* Returns 0 on success, -1 on bad arguments, -2 on allocation failure. */
int gdr_oracle_backward(int B, int T, int H, int dk, int dv,
                        const double* q, const double* k, const double* v,
                        const double* alpha, int alpha_per_channel,
                        const double* b, int b_per_channel,
                        const double* w, int w_per_channel,
                        const double* S0, const double* dO, const double* dS_T,
                        double* dq, double* dk_out, double* dv_out,
                        double* dalpha, double* db, double* dw, double* dS0, int nthreads) {
    if (B < 0 || T < 0 || H < 0 || dk <= 0 || dv <= 0) return -1;
    if (T > 0 && (!q || !k || !v || !dO || !dq || !dk_out || !dv_out)) return -1;
    int nheads = B * H;
    int err = 0;
    const size_t SZ = (size_t)dk * dv;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel
#endif
    {
        double* Sall = (double*)malloc(sizeof(double) * SZ * ((size_t)T + 1));
        double* G = (double*)malloc(sizeof(double) * SZ);
        double* Sd = (double*)malloc(sizeof(double) * SZ);
        double* vec = (double*)malloc(sizeof(double) * (size_t)(2 * dv + 3 * dk));
        if (!Sall || !G || !Sd || !vec) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
            err = -2;
        } else {
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
            for (int hd = 0; hd < nheads; ++hd)
                bwd_head(hd / H, hd % H, T, H, dk, dv, q, k, v, alpha, alpha_per_channel, b,
                         b_per_channel, w, w_per_channel, S0, dO, dS_T, dq, dk_out, dv_out,
                         dalpha, db, dw, dS0, Sall, G, Sd, vec, vec + dv, vec + 2 * dv,
                         vec + 2 * dv + dk);
        }
        free(Sall);
        free(G);
        free(Sd);
        free(vec);
    }
    (void)nthreads;
    return err;
}

/* Number of threads the oracle will use (1 without OpenMP). */
int gdr_oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
