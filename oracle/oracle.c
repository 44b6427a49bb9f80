/*
 * Float64 CPU oracle for the delta-rule sequence mixer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may load this
 * library: only tests/, the smoke check of the package entry file and the
 * CPU-baseline / reference arm of bench.py use it.  It shares no code, header,
 * table or helper with the CUDA library.
 *
 * Sources (web pages on the subject):
 *   [P1] "How a Baseten Engineer Traced 7 Years of Attention Mechanism
 *        Evolution -- From GPT-2 to Kimi K3, in Runable PyTorch" (wpnews.pro),
 *        paragraphs on the delta rule ("before writing, read what this key
 *        position currently stores"), on Gated DeltaNet ("decay first, then
 *        precise write") and on linear attention (Q' = ELU(Q)+1).
 *   [P3] "GPT-2 から Kimi K3 まで、AI モデルの進化を解説" (news.ainew.jp),
 *        sections "Linear attention" (the cached S, z forward),
 *        "DeltaNet (Fast weight programmers)" (the beta-weighted delta write)
 *        and "DeltaNet (Parallelizing linear transformers with delta rule)"
 *        (the direct per-token prefill loop).
 *
 * What is computed is the plain per-token recurrence, in float64, in the
 * order the pages give it.  Inputs are read in their stored precision
 * (float32, or bfloat16 bit patterns) and widened exactly to double.
 *
 * Parity: pinned.  tests/test_oracle_pins.py checks every function here
 * against properties the pages state (zero write strength, zero delta,
 * overwrite with unit keys, additive special case, decay 1 and 0), closed
 * forms (orthonormal keys, matmul form of causal linear attention) and
 * hand-derived golden fixtures under tests/golden/.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

/* Input element types understood by the oracle. */
enum { ORC_F32 = 0, ORC_BF16 = 1, ORC_F64 = 2 };

/* Options of the delta rule.
 *   ORC_PRESTEP: q and k are the raw projections and beta holds logits; each
 *     token first takes the DeltaNet layer's feature maps of [P3] "DeltaNet
 *     (Fast weight programmers)": q <- normalize(silu(q)), k <- normalize(silu(k))
 *     (L2 over the head dimension, divisor max(norm, 1e-12) as F.normalize),
 *     beta <- sigmoid(beta).
 *   ORC_ALPHA_PER_DIM: alpha is (B,H,T,Dk), one decay per key dimension: row i
 *     of the state decays by alpha_t[i] ([P1], the KDA paragraph: scalar gating
 *     replaced by per-dimension gating). */
enum { ORC_PRESTEP = 1, ORC_ALPHA_PER_DIM = 2 };

/* Widen one stored element to double.  A bfloat16 value is the upper 16 bits
 * of the float32 with the same value, so the widening is exact. */
static double widen(const void *p, int dtype, size_t i)
{
    if (dtype == ORC_F64)
        return ((const double *)p)[i];
    if (dtype == ORC_F32)
        return (double)((const float *)p)[i];
    uint32_t bits = (uint32_t)((const uint16_t *)p)[i] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* silu(x) = x * sigmoid(x) = x / (1 + e^-x) */
static double silu(double x)
{
    return x / (1.0 + exp(-x));
}

/* Read one token's Dk-vector (q or k) into out[], applying the pre-step map
 * normalize(silu(.)) when asked. */
static void load_key(const void *p, int dtype, size_t at, long Dk, int prestep, double *out)
{
    for (long i = 0; i < Dk; ++i)
        out[i] = prestep ? silu(widen(p, dtype, at + i)) : widen(p, dtype, at + i);
    if (prestep) {
        double ss = 0.0;
        for (long i = 0; i < Dk; ++i)
            ss += out[i] * out[i];
        double nrm = sqrt(ss);
        if (nrm < 1e-12)
            nrm = 1e-12;
        for (long i = 0; i < Dk; ++i)
            out[i] /= nrm;
    }
}

/* Problem description shared by the worker threads. */
typedef struct {
    const void *q, *k, *v;
    int dtype;
    const float *beta, *alpha;
    const double *S0, *z0;
    double *o, *S_out, *z_out;
    long B, H, T, Dk, Dv;
    int linear; /* 0: delta rule (optionally gated); 1: ELU+1 linear attention */
    int flags;  /* delta rule only: ORC_PRESTEP, ORC_ALPHA_PER_DIM */
    long next;  /* next (b,h) pair to process */
    pthread_mutex_t lock;
} job_t;

/*
 * One (b,h) sequence of the delta rule.
 *
 * [P3] "DeltaNet (Parallelizing linear transformers with delta rule)", the
 * direct loop over tokens: read v_old = k_t S, form u_t = beta_t (v_t - v_old),
 * write S += k_t^T u_t, then emit o_t = q_t S with the state after the write.
 * [P1] Gated DeltaNet: S_new = alpha * S_old + k^T delta, "decay first, then
 * precise write", so the read is taken from the decayed state alpha_t S.
 * alpha == NULL means alpha_t = 1 (plain DeltaNet); with ORC_ALPHA_PER_DIM the
 * decay of row i of S is alpha_t[i].  `kv` holds 2 Dk doubles (q_t, k_t).
 */
static void delta_sequence(const job_t *J, long bh, double *S, double *r, double *kv)
{
    const long T = J->T, Dk = J->Dk, Dv = J->Dv;
    const size_t qk0 = (size_t)bh * T * Dk, v0 = (size_t)bh * T * Dv, s0 = (size_t)bh * Dk * Dv;
    const int prestep = (J->flags & ORC_PRESTEP) != 0, per_dim = (J->flags & ORC_ALPHA_PER_DIM) != 0;
    double *qv = kv, *kk = kv + Dk;

    for (long i = 0; i < Dk * Dv; ++i)
        S[i] = J->S0 ? J->S0[s0 + i] : 0.0;

    for (long t = 0; t < T; ++t) {
        double beta = (double)J->beta[(size_t)bh * T + t];
        if (prestep)
            beta = 1.0 / (1.0 + exp(-beta));
        const size_t kt = qk0 + (size_t)t * Dk, vt = v0 + (size_t)t * Dv;
        load_key(J->q, J->dtype, kt, Dk, prestep, qv);
        load_key(J->k, J->dtype, kt, Dk, prestep, kk);

        /* decay first */
        if (J->alpha && per_dim) {
            for (long i = 0; i < Dk; ++i) {
                const double a = (double)J->alpha[kt + i];
                for (long j = 0; j < Dv; ++j)
                    S[i * Dv + j] *= a;
            }
        } else if (J->alpha) {
            const double alpha = (double)J->alpha[(size_t)bh * T + t];
            for (long i = 0; i < Dk * Dv; ++i)
                S[i] *= alpha;
        }
        /* read the value currently stored under k_t: v_old = k_t S */
        for (long j = 0; j < Dv; ++j)
            r[j] = 0.0;
        for (long i = 0; i < Dk; ++i)
            for (long j = 0; j < Dv; ++j)
                r[j] += kk[i] * S[i * Dv + j];
        /* the delta u_t = beta_t (v_t - v_old), written as an outer product */
        for (long j = 0; j < Dv; ++j)
            r[j] = beta * (widen(J->v, J->dtype, vt + j) - r[j]);
        for (long i = 0; i < Dk; ++i)
            for (long j = 0; j < Dv; ++j)
                S[i * Dv + j] += kk[i] * r[j];
        /* output with the updated state: o_t = q_t S */
        double *o = J->o + v0 + (size_t)t * Dv;
        for (long j = 0; j < Dv; ++j)
            o[j] = 0.0;
        for (long i = 0; i < Dk; ++i)
            for (long j = 0; j < Dv; ++j)
                o[j] += qv[i] * S[i * Dv + j];
    }
    if (J->S_out)
        memcpy(J->S_out + s0, S, sizeof(double) * (size_t)(Dk * Dv));
}

/* ELU(x) + 1, the positive feature map of [P1] and [P3] "Linear attention". */
static double elu_plus_one(double x)
{
    return (x > 0.0 ? x : expm1(x)) + 1.0;
}

/*
 * One (b,h) sequence of causal linear attention with the ELU+1 feature map.
 *
 * [P3] "Linear attention", the cached forward: q' = ELU(q)+1, k' = ELU(k)+1,
 * S += k'^T v, z += k', o = (q' S) / (q' . z).  Applied one token at a time,
 * so every query sees exactly the keys up to and including its own position.
 * v is not mapped.
 */
static void linear_sequence(const job_t *J, long bh, double *S, double *z, double *kp)
{
    const long T = J->T, Dk = J->Dk, Dv = J->Dv;
    const size_t qk0 = (size_t)bh * T * Dk, v0 = (size_t)bh * T * Dv, s0 = (size_t)bh * Dk * Dv;

    for (long i = 0; i < Dk * Dv; ++i)
        S[i] = J->S0 ? J->S0[s0 + i] : 0.0;
    for (long i = 0; i < Dk; ++i)
        z[i] = J->z0 ? J->z0[(size_t)bh * Dk + i] : 0.0;

    for (long t = 0; t < T; ++t) {
        const size_t kt = qk0 + (size_t)t * Dk, vt = v0 + (size_t)t * Dv;
        for (long i = 0; i < Dk; ++i)
            kp[i] = elu_plus_one(widen(J->k, J->dtype, kt + i));
        for (long i = 0; i < Dk; ++i) {
            for (long j = 0; j < Dv; ++j)
                S[i * Dv + j] += kp[i] * widen(J->v, J->dtype, vt + j);
            z[i] += kp[i];
        }
        double *o = J->o + v0 + (size_t)t * Dv;
        double den = 0.0;
        for (long j = 0; j < Dv; ++j)
            o[j] = 0.0;
        for (long i = 0; i < Dk; ++i) {
            const double qi = elu_plus_one(widen(J->q, J->dtype, kt + i));
            for (long j = 0; j < Dv; ++j)
                o[j] += qi * S[i * Dv + j];
            den += qi * z[i];
        }
        for (long j = 0; j < Dv; ++j)
            o[j] /= den;
    }
    if (J->S_out)
        memcpy(J->S_out + s0, S, sizeof(double) * (size_t)(Dk * Dv));
    if (J->z_out)
        memcpy(J->z_out + (size_t)bh * Dk, z, sizeof(double) * (size_t)Dk);
}

static void *worker(void *arg)
{
    job_t *J = (job_t *)arg;
    double *S = (double *)malloc(sizeof(double) * (size_t)(J->Dk * J->Dv));
    double *r = (double *)malloc(sizeof(double) * (size_t)(4 * J->Dk + J->Dv));
    if (!S || !r) {
        free(S);
        free(r);
        return (void *)1;
    }
    for (;;) {
        pthread_mutex_lock(&J->lock);
        const long bh = J->next++;
        pthread_mutex_unlock(&J->lock);
        if (bh >= J->B * J->H)
            break;
        if (J->linear)
            linear_sequence(J, bh, S, r, r + J->Dk);
        else
            delta_sequence(J, bh, S, r, r + J->Dv);
    }
    free(S);
    free(r);
    return NULL;
}

static int run(job_t *J, int nthreads)
{
    if (J->B < 0 || J->H < 0 || J->T < 0 || J->Dk <= 0 || J->Dv <= 0)
        return -1;
    if (nthreads <= 0)
        nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (nthreads < 1)
        nthreads = 1;
    if (nthreads > J->B * J->H)
        nthreads = (int)(J->B * J->H > 0 ? J->B * J->H : 1);
    pthread_mutex_init(&J->lock, NULL);
    J->next = 0;
    pthread_t *th = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
    if (!th)
        return -2;
    int rc = 0;
    for (int i = 0; i < nthreads; ++i)
        pthread_create(&th[i], NULL, worker, J);
    for (int i = 0; i < nthreads; ++i) {
        void *ret = NULL;
        pthread_join(th[i], &ret);
        if (ret)
            rc = -2;
    }
    free(th);
    pthread_mutex_destroy(&J->lock);
    return rc;
}

/*
 * Delta rule over whole sequences (a decode step is the case T = 1 with the
 * caller's state as S0).  q, k: (B,H,T,Dk); v, o: (B,H,T,Dv); beta, alpha:
 * (B,H,T) float32 (alpha may be NULL); S0, S_out: (B,H,Dk,Dv) float64 (S0 may
 * be NULL for a zero state; S_out may be NULL).  All row-major, contiguous.
 * Returns 0, or a negative value on bad sizes / allocation failure.
 */
int oracle_deltanet(const void *q, const void *k, const void *v, int dtype,
                    const float *beta, const float *alpha, const double *S0,
                    double *o, double *S_out,
                    long B, long H, long T, long Dk, long Dv, int nthreads)
{
    job_t J;
    memset(&J, 0, sizeof J);
    J.q = q; J.k = k; J.v = v; J.dtype = dtype;
    J.beta = beta; J.alpha = alpha; J.S0 = S0;
    J.o = o; J.S_out = S_out;
    J.B = B; J.H = H; J.T = T; J.Dk = Dk; J.Dv = Dv;
    J.linear = 0;
    return run(&J, nthreads);
}

/*
 * The delta rule with options (ORC_PRESTEP, ORC_ALPHA_PER_DIM; see above).
 * Shapes as oracle_deltanet, except alpha: (B,H,T,Dk) with ORC_ALPHA_PER_DIM;
 * with ORC_PRESTEP, q and k are the raw projections and beta the logits.
 */
int oracle_deltanet_ex(const void *q, const void *k, const void *v, int dtype,
                       const float *beta, const float *alpha, const double *S0,
                       double *o, double *S_out,
                       long B, long H, long T, long Dk, long Dv, int flags, int nthreads)
{
    job_t J;
    memset(&J, 0, sizeof J);
    J.q = q; J.k = k; J.v = v; J.dtype = dtype;
    J.beta = beta; J.alpha = alpha; J.S0 = S0;
    J.o = o; J.S_out = S_out;
    J.B = B; J.H = H; J.T = T; J.Dk = Dk; J.Dv = Dv;
    J.linear = 0;
    J.flags = flags;
    return run(&J, nthreads);
}

/*
 * ELU+1 causal linear attention.  Shapes as oracle_deltanet; z0, z_out:
 * (B,H,Dk) float64, nullable.
 */
int oracle_linear_attn(const void *q, const void *k, const void *v, int dtype,
                       const double *S0, const double *z0,
                       double *o, double *S_out, double *z_out,
                       long B, long H, long T, long Dk, long Dv, int nthreads)
{
    job_t J;
    memset(&J, 0, sizeof J);
    J.q = q; J.k = k; J.v = v; J.dtype = dtype;
    J.S0 = S0; J.z0 = z0;
    J.o = o; J.S_out = S_out; J.z_out = z_out;
    J.B = B; J.H = H; J.T = T; J.Dk = Dk; J.Dv = Dv;
    J.linear = 1;
    return run(&J, nthreads);
}


/* ------------------------------------------------------------------------ */
/* Gradient of the delta rule (reverse mode of the per-token loop).
 *
 * [P3] "DeltaNet (Parallelizing linear transformers with delta rule)" presents
 * the chunked form as what makes linear-time training hardware-efficient; the
 * training step needs the gradient of the same recurrence.  This is the plain
 * reverse sweep of the per-token loop above (gated as [P1]'s Gated DeltaNet),
 * written from the chain rule, one token at a time from the last:
 *
 *   forward   S'_t = a_t S_{t-1};  r_t = k_t S'_t;  u_t = b_t (v_t - r_t);
 *             S_t = S'_t + k_t^T u_t;  o_t = q_t S_t
 *   backward  G  <- G + q_t^T dO_t                  (G = dL/dS_t)
 *             dq_t = dO_t S_t^T
 *             du   = k_t G;     dk_t  = G u_t^T
 *             db_t = du . (v_t - r_t);   dv_t = b_t du;   dr = -b_t du
 *             dk_t += dr S'_t^T;  G' = G + k_t^T dr  (= dL/dS'_t)
 *             da_t = <G', S_{t-1}>;   G <- a_t G'     (= dL/dS_{t-1})
 *   dS0 = G after token 0.  The loss is sum(dO * o) + sum(dS_T * S_T).
 *
 * The forward states are kept for the sweep ((T+1) Dk Dv doubles per
 * sequence).  Inputs as oracle_deltanet (q, k, v may also be float64, dtype
 * 2); alpha is per token (or NULL); dO (B,H,T,Dv) and dS_T (B,H,Dk,Dv, nullable)
 * are float64; outputs dq, dk (B,H,T,Dk), dv (B,H,T,Dv), dbeta (B,H,T), dalpha
 * (B,H,T, nullable) and dS0 (B,H,Dk,Dv) are float64.
 */
typedef struct {
    const void *q, *k, *v;
    int dtype;
    const float *beta, *alpha;
    const double *S0, *dO, *dST;
    double *dq, *dk, *dv, *dbeta, *dalpha, *dS0;
    long B, H, T, Dk, Dv;
    long next;
    pthread_mutex_t lock;
} bjob_t;

static void delta_sequence_bwd(const bjob_t *J, long bh, double *Ss, double *G, double *w)
{
    const long T = J->T, Dk = J->Dk, Dv = J->Dv, DD = Dk * Dv;
    const size_t qk0 = (size_t)bh * T * Dk, v0 = (size_t)bh * T * Dv, s0 = (size_t)bh * DD;
    double *kk = w, *qq = w + Dk, *r = w + 2 * Dk, *u = r + Dv, *du = u + Dv, *dr = du + Dv;

    /* forward sweep: Ss holds S_{-1} = S0, S_0, ..., S_{T-1} */
    for (long i = 0; i < DD; ++i)
        Ss[i] = J->S0 ? J->S0[s0 + i] : 0.0;
    for (long t = 0; t < T; ++t) {
        const double *Sp = Ss + (size_t)t * DD;
        double *Sn = Ss + (size_t)(t + 1) * DD;
        const double beta = (double)J->beta[(size_t)bh * T + t];
        const double alpha = J->alpha ? (double)J->alpha[(size_t)bh * T + t] : 1.0;
        for (long i = 0; i < Dk; ++i)
            kk[i] = widen(J->k, J->dtype, qk0 + (size_t)t * Dk + i);
        for (long i = 0; i < DD; ++i)
            Sn[i] = alpha * Sp[i];
        for (long j = 0; j < Dv; ++j) {
            r[j] = 0.0;
            for (long i = 0; i < Dk; ++i)
                r[j] += kk[i] * Sn[i * Dv + j];
            u[j] = beta * (widen(J->v, J->dtype, v0 + (size_t)t * Dv + j) - r[j]);
        }
        for (long i = 0; i < Dk; ++i)
            for (long j = 0; j < Dv; ++j)
                Sn[i * Dv + j] += kk[i] * u[j];
    }
    /* reverse sweep */
    for (long i = 0; i < DD; ++i)
        G[i] = J->dST ? J->dST[s0 + i] : 0.0;
    for (long t = T - 1; t >= 0; --t) {
        const double *Sprev = Ss + (size_t)t * DD, *St = Ss + (size_t)(t + 1) * DD;
        const double beta = (double)J->beta[(size_t)bh * T + t];
        const double alpha = J->alpha ? (double)J->alpha[(size_t)bh * T + t] : 1.0;
        const double *dO = J->dO + v0 + (size_t)t * Dv;
        for (long i = 0; i < Dk; ++i) {
            kk[i] = widen(J->k, J->dtype, qk0 + (size_t)t * Dk + i);
            qq[i] = widen(J->q, J->dtype, qk0 + (size_t)t * Dk + i);
        }
        /* o_t = q_t S_t */
        for (long i = 0; i < Dk; ++i)
            for (long j = 0; j < Dv; ++j)
                G[i * Dv + j] += qq[i] * dO[j];
        double *dq = J->dq + qk0 + (size_t)t * Dk, *dk = J->dk + qk0 + (size_t)t * Dk;
        for (long i = 0; i < Dk; ++i) {
            double acc = 0.0;
            for (long j = 0; j < Dv; ++j)
                acc += dO[j] * St[i * Dv + j];
            dq[i] = acc;
        }
        /* recompute r_t, u_t from S'_t = alpha S_{t-1} */
        for (long j = 0; j < Dv; ++j) {
            r[j] = 0.0;
            for (long i = 0; i < Dk; ++i)
                r[j] += kk[i] * alpha * Sprev[i * Dv + j];
            u[j] = beta * (widen(J->v, J->dtype, v0 + (size_t)t * Dv + j) - r[j]);
        }
        /* S_t = S'_t + k_t^T u_t */
        for (long j = 0; j < Dv; ++j) {
            du[j] = 0.0;
            for (long i = 0; i < Dk; ++i)
                du[j] += kk[i] * G[i * Dv + j];
        }
        for (long i = 0; i < Dk; ++i) {
            double acc = 0.0;
            for (long j = 0; j < Dv; ++j)
                acc += G[i * Dv + j] * u[j];
            dk[i] = acc;
        }
        /* u_t = beta_t (v_t - r_t) */
        double db = 0.0;
        double *dv = J->dv + v0 + (size_t)t * Dv;
        for (long j = 0; j < Dv; ++j) {
            db += du[j] * (widen(J->v, J->dtype, v0 + (size_t)t * Dv + j) - r[j]);
            dv[j] = beta * du[j];
            dr[j] = -beta * du[j];
        }
        J->dbeta[(size_t)bh * T + t] = db;
        /* r_t = k_t S'_t */
        for (long i = 0; i < Dk; ++i) {
            double acc = 0.0;
            for (long j = 0; j < Dv; ++j)
                acc += dr[j] * alpha * Sprev[i * Dv + j];
            dk[i] += acc;
        }
        for (long i = 0; i < Dk; ++i)
            for (long j = 0; j < Dv; ++j)
                G[i * Dv + j] += kk[i] * dr[j];
        /* S'_t = alpha_t S_{t-1} */
        if (J->dalpha) {
            double da = 0.0;
            for (long i = 0; i < DD; ++i)
                da += G[i] * Sprev[i];
            J->dalpha[(size_t)bh * T + t] = da;
        }
        for (long i = 0; i < DD; ++i)
            G[i] *= alpha;
    }
    memcpy(J->dS0 + s0, G, sizeof(double) * (size_t)DD);
}

static void *bwd_worker(void *arg)
{
    bjob_t *J = (bjob_t *)arg;
    const size_t DD = (size_t)(J->Dk * J->Dv);
    double *Ss = (double *)malloc(sizeof(double) * DD * (size_t)(J->T + 1));
    double *G = (double *)malloc(sizeof(double) * DD);
    double *w = (double *)malloc(sizeof(double) * (size_t)(2 * J->Dk + 4 * J->Dv));
    void *rc = NULL;
    if (!Ss || !G || !w) {
        rc = (void *)1;
    } else {
        for (;;) {
            pthread_mutex_lock(&J->lock);
            const long bh = J->next++;
            pthread_mutex_unlock(&J->lock);
            if (bh >= J->B * J->H)
                break;
            delta_sequence_bwd(J, bh, Ss, G, w);
        }
    }
    free(Ss);
    free(G);
    free(w);
    return rc;
}

int oracle_deltanet_bwd(const void *q, const void *k, const void *v, int dtype,
                        const float *beta, const float *alpha, const double *S0,
                        const double *dO, const double *dST,
                        double *dq, double *dk, double *dv, double *dbeta, double *dalpha,
                        double *dS0, long B, long H, long T, long Dk, long Dv, int nthreads)
{
    if (B < 0 || H < 0 || T < 0 || Dk <= 0 || Dv <= 0)
        return -1;
    bjob_t J;
    memset(&J, 0, sizeof J);
    J.q = q; J.k = k; J.v = v; J.dtype = dtype;
    J.beta = beta; J.alpha = alpha; J.S0 = S0; J.dO = dO; J.dST = dST;
    J.dq = dq; J.dk = dk; J.dv = dv; J.dbeta = dbeta; J.dalpha = dalpha; J.dS0 = dS0;
    J.B = B; J.H = H; J.T = T; J.Dk = Dk; J.Dv = Dv;
    if (nthreads <= 0)
        nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (nthreads < 1)
        nthreads = 1;
    if (nthreads > B * H)
        nthreads = (int)(B * H > 0 ? B * H : 1);
    pthread_mutex_init(&J.lock, NULL);
    pthread_t *th = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
    if (!th)
        return -2;
    int rc = 0;
    for (int i = 0; i < nthreads; ++i)
        pthread_create(&th[i], NULL, bwd_worker, &J);
    for (int i = 0; i < nthreads; ++i) {
        void *ret = NULL;
        pthread_join(th[i], &ret);
        if (ret)
            rc = -2;
    }
    free(th);
    pthread_mutex_destroy(&J.lock);
    return rc;
}
