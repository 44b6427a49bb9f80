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
enum { ORC_F32 = 0, ORC_BF16 = 1 };

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
