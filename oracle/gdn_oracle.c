/*
 * Oracle for the causal gated delta-rule recurrence.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may call this code; the product path never
 * does.  It shares no code, header or constant with the CUDA library.
 *
 * What it computes (float64, token by token, one (b,h) head at a time), in the
 * column convention S in R^{dv x dk} (state stored [B,H,dv,dk]):
 *
 *   S_t = S_{t-1} Diag(alpha_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
 *   o_t = S_t q_t,
 *
 * written out as the three steps that this product expands to:
 *   1. decay:   S' = S_{t-1} Diag(alpha_t)        (column j scaled by alpha_t[j];
 *               alpha_t = exp(g_t), a scalar or a dk-vector; 1 without a gate)
 *   2. write:   additive / decay modes:  S_t = S' + v_t k_t^T
 *               delta mode:  u_t = beta_t (v_t - S' k_t),  S_t = S' + u_t k_t^T
 *   3. read:    o_t = S_t q_t
 *
 * Sources ("Linear Attention, Visualized"): section "Naive linear attention"
 * (additive state S_t = S_{t-1} + outer product, read o_t from S_t);
 * "RetNet: scalar decay" and "Mamba-2: input-dependent scalar decay" (the state
 * is shrunk by the gate before the write); "DeltaNet", subsection "Recurrent
 * form" (predict with the current state, write beta times the residual);
 * "Gated DeltaNet (GDN)" (scalar decay then delta write); "Gated Linear
 * Attention (GLA)" and "Kimi Delta Attention (KDA)" (per-channel decay along
 * the key dimension, applied before the delta correction).  "Beyond attention"
 * (learning.iampt.xyz), list "Three ways to update the state", names the same
 * three write rules.
 *
 * Mode numbering: update 0 = additive, 1 = decay, 2 = delta;
 *                 gate   0 = none,     1 = scalar, 2 = channel.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

#define ORC_ADDITIVE 0
#define ORC_DECAY 1
#define ORC_DELTA 2
#define ORC_GATE_NONE 0
#define ORC_GATE_SCALAR 1
#define ORC_GATE_CHANNEL 2

/* One head.  q,k: [T,dk]; v: [T,dv]; g: [T] or [T,dk] or NULL; beta: [T] or
 * NULL; S: [dv,dk] in/out; o: [T,dv]. */
static void run_head(int update, int gate, long T, long dk, long dv,
                     const double *q, const double *k, const double *v,
                     const double *g, const double *beta, double *S, double *o,
                     double *alpha, double *u)
{
    for (long t = 0; t < T; ++t) {
        const double *qt = q + t * dk;
        const double *kt = k + t * dk;
        const double *vt = v + t * dv;

        /* 1. decay: alpha_t = exp(g_t) */
        if (gate != ORC_GATE_NONE) {
            for (long j = 0; j < dk; ++j)
                alpha[j] = (gate == ORC_GATE_SCALAR) ? exp(g[t]) : exp(g[t * dk + j]);
            for (long i = 0; i < dv; ++i)
                for (long j = 0; j < dk; ++j)
                    S[i * dk + j] *= alpha[j];
        }

        /* 2. write */
        if (update == ORC_DELTA) {
            const double bt = beta[t];
            for (long i = 0; i < dv; ++i) {
                double pred = 0.0; /* (S' k_t)_i */
                for (long j = 0; j < dk; ++j)
                    pred += S[i * dk + j] * kt[j];
                u[i] = bt * (vt[i] - pred);
            }
        } else {
            for (long i = 0; i < dv; ++i)
                u[i] = vt[i];
        }
        for (long i = 0; i < dv; ++i)
            for (long j = 0; j < dk; ++j)
                S[i * dk + j] += u[i] * kt[j];

        /* 3. read */
        for (long i = 0; i < dv; ++i) {
            double acc = 0.0;
            for (long j = 0; j < dk; ++j)
                acc += S[i * dk + j] * qt[j];
            o[t * dv + i] = acc;
        }
    }
}

/*
 * Full forward over B*H heads.  Layouts (contiguous, float64):
 *   q,k [BH,T,dk]; v,o [BH,T,dv]; beta [BH,T] (delta only, else may be NULL);
 *   g [BH,T] (scalar) or [BH,T,dk] (channel) or NULL (none);
 *   S0 [BH,dv,dk] or NULL (zeros); ST [BH,dv,dk] or NULL (not written).
 * Returns 0, or -1 on an invalid mode.
 */
int oracle_gdn_forward(int update, int gate, long BH, long T, long dk, long dv,
                       const double *q, const double *k, const double *v,
                       const double *g, const double *beta, const double *S0,
                       double *o, double *ST)
{
    if (update < 0 || update > 2 || gate < 0 || gate > 2)
        return -1;
    if (update == ORC_DELTA && beta == NULL)
        return -1;
    if ((gate != ORC_GATE_NONE) != (g != NULL))
        return -1;
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (long bh = 0; bh < BH; ++bh) {
        double *S = (double *)malloc(sizeof(double) * (size_t)(dv * dk));
        double *alpha = (double *)malloc(sizeof(double) * (size_t)dk);
        double *u = (double *)malloc(sizeof(double) * (size_t)dv);
        if (!S || !alpha || !u) {
#pragma omp atomic write
            err = -2;
        } else {
            if (S0)
                memcpy(S, S0 + bh * dv * dk, sizeof(double) * (size_t)(dv * dk));
            else
                memset(S, 0, sizeof(double) * (size_t)(dv * dk));
            const double *gh = NULL;
            if (gate == ORC_GATE_SCALAR)
                gh = g + bh * T;
            else if (gate == ORC_GATE_CHANNEL)
                gh = g + bh * T * dk;
            run_head(update, gate, T, dk, dv, q + bh * T * dk, k + bh * T * dk,
                     v + bh * T * dv, gh, beta ? beta + bh * T : NULL, S,
                     o + bh * T * dv, alpha, u);
            if (ST)
                memcpy(ST + bh * dv * dk, S, sizeof(double) * (size_t)(dv * dk));
        }
        free(S);
        free(alpha);
        free(u);
    }
    return err;
}

int oracle_num_threads(void)
{
    int n = 1;
#pragma omp parallel
    {
#pragma omp single
        {
#ifdef _OPENMP
            extern int omp_get_num_threads(void);
            n = omp_get_num_threads();
#endif
        }
    }
    return n;
}
