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

/* Number of threads the oracle will use (1 without OpenMP). */
int gdr_oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
