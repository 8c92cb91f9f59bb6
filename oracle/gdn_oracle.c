/*
 * gdn_oracle.c -- plain, slow, sequential fp64 CPU oracle for the Gated DeltaNet layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and bench.py's
 * cpu_baseline / reference leg may load this library.  The CUDA product path shares no
 * code with it and never calls it.
 *
 * What it computes (sources):
 *   - Layer constants: "Qwen3-Coder-Next" model card (llm-atlas), raw config.json fields:
 *     linear_conv_kernel_dim 4, linear_key_head_dim 128, linear_num_key_heads 16,
 *     linear_num_value_heads 32, linear_value_head_dim 128, rms_norm_eps 1e-6, hidden_act silu.
 *   - Structure of the token mixer: hyper.ai story on Qwen3-Next in Transformers (the
 *     Gated DeltaNet paragraph): Q/K/V plus a separate Z projection, a causal convolution for
 *     local context, beta gating the strength of each update, kv_mem as the stored prior
 *     knowledge read out of the recurrent state, linear cost through a recurrent state update,
 *     and a zero-centred RMSNorm.
 *   - State independent of sequence length: Qwen3.5 teardown (rkmt.cn), section 3.2
 *     "Linear Attention layer".
 *   - fp32 recurrent state by default: "Qwen3-Next" SGLang cookbook, section 3.2
 *     Configuration Tips (--mamba-ssm-dtype).
 *   - The recurrence itself, as this library reads it:
 *        S_t = alpha_t * S_{t-1} * (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,   o_t = S_t q_t
 *     written out per token as: S <- alpha S; kv_mem = S k; u = beta (v - kv_mem);
 *     S <- S + u k^T; o = S q.  (Expanding the product shows the two forms are equal.)
 *
 * Readings where the pages are silent (each is a plain reading, stated once here):
 *   - conv: depthwise, no bias, weight w[c][i], tap K-1 multiplies the current token, history
 *     before the first token comes from the caller's conv state (zeros if none); SiLU after.
 *     With the conv switched off the input passes through unchanged (no SiLU).
 *   - channel order of the conv input: q (Hk*d) | k (Hk*d) | v (Hv*d).
 *   - q = q~ / sqrt(|q~|^2 + l2_eps) * q_scale, k = k~ / sqrt(|k~|^2 + l2_eps); v unchanged.
 *   - value head h reads key/query head h / (Hv/Hk).
 *   - alpha_t = exp(g_t) with g = log alpha supplied per (token, value head).
 *   - state layout S[v][k] (row = value index), fp64 here.
 *   - gated norm: y = o / sqrt(mean(o^2) + norm_eps) * w * silu(z), per (token, value head),
 *     w is the effective weight (a zero-centred caller passes 1 + w).
 *
 * Error scales (optional outputs, used by the tests to set element-wise tolerances).  Every
 * quantity gets a magnitude: the same computation with every term replaced by its absolute
 * value, so that nothing cancels.  The conv output y = silu(sum_i w_i x_i) gets
 * ym = 1.1 sum_i |w_i| |x_i| (1.1 bounds the slope of SiLU; ym >= |y|), or |x| with the conv
 * off; q and k get ym / |y~| after the L2 norm, v keeps ym.  Writing km, qm, vm for those, the
 * state runs
 *        M_t = alpha_t M_{t-1} + beta_t (vm_t + alpha_t |S_{t-1}| km_t) km_t^T,   M_0 = |S_0|
 * (|.| element-wise; the kv_mem term uses the actual state, so M stays finite like S).  By the
 * triangle inequality M_t >= |S_t| element-wise.  The scale of output element o_t[v] is
 * c_t[v] = sum_k M_t[v][k] qm_t[k] (>= |o_t[v]|): the size of the terms the dot product adds
 * up.  For the gated RMSNorm y = o r w silu(z), r = 1 / sqrt(m + eps), m = mean(o^2), a change
 * of each o[u] by c[u] moves y[v] by at most (to first order)
 *        s[v] = |w[v] silu(z[v])| r (c[v] + |o[v]| sum_u |o[u]| c[u] / (d (m + eps))),
 * which is the scale reported for normalised outputs.  Rounding an input or an intermediate of
 * the recurrence by a relative epsilon changes an element by a multiple of epsilon times its
 * scale, not of epsilon times its value: elements that are small sums of large terms (a query
 * nearly orthogonal to the state, a row whose RMSNorm divides by a small norm) carry large
 * scales.  The scales are outputs only; they change nothing in out, SN or convN.
 *
 * All inputs are converted exactly to fp64 (bf16 and fp32 values are exactly representable).
 * Independent (sequence, value head) units run on host threads; within a unit the arithmetic
 * is the sequential per-token recurrence above, in the order written.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* dtype codes of activation-like inputs */
enum { ORC_F32 = 0, ORC_BF16 = 1, ORC_F64 = 2 };

typedef struct {
    int32_t num_k_heads, num_v_heads, head_dim, conv_kernel;
    double q_scale, l2_eps, norm_eps;
} orc_dims;

static double ld_any(const void *p, int dtype, size_t i) {
    if (dtype == ORC_F64) return ((const double *)p)[i];
    if (dtype == ORC_F32) return (double)((const float *)p)[i];
    /* bf16: the upper 16 bits of an IEEE single */
    uint32_t u = ((uint32_t)((const uint16_t *)p)[i]) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }
static double silu(double x) { return x * sigmoid(x); }

/* ------------------------------------------------------------------------------------------ */
/* Causal depthwise conv + SiLU over packed variable-length sequences.                          */
/*   x        [T][C]     (dtype)                                                               */
/*   w        [C][K]     (dtype)                                                               */
/*   conv_in  [N][K-1][C] (dtype) or NULL (zeros): row j holds x_{j-(K-1)} of the sequence       */
/*   y        [T][C]     fp64 out: silu(sum_i w[c][i] * x_{t-(K-1)+i}[c])                         */
/*   conv_out [N][K-1][C] fp64 out or NULL: the last K-1 rows of the extended history          */
/* ------------------------------------------------------------------------------------------ */
int orc_conv1d_silu(int dtype, const void *x, const void *w, const int32_t *cu_seqlens, int N,
                    int T, int C, int K, const void *conv_in, double *y, double *conv_out) {
    if (K < 1 || C < 1 || N < 0 || T < 0) return -1;
    if (N > 0 && cu_seqlens[N] != T) return -1;
    double *hist = (double *)malloc(sizeof(double) * (size_t)(K - 1 + 1) * (size_t)C);
    if (!hist) return -2;
    for (int n = 0; n < N; ++n) {
        int t0 = cu_seqlens[n], t1 = cu_seqlens[n + 1];
        /* hist rows 0..K-2: the K-1 previous inputs, oldest first */
        for (int j = 0; j < K - 1; ++j)
            for (int c = 0; c < C; ++c)
                hist[(size_t)j * C + c] =
                    conv_in ? ld_any(conv_in, dtype, ((size_t)n * (K - 1) + j) * C + c) : 0.0;
        for (int t = t0; t < t1; ++t) {
            for (int c = 0; c < C; ++c) {
                double acc = 0.0;
                for (int i = 0; i < K - 1; ++i)
                    acc += ld_any(w, dtype, (size_t)c * K + i) * hist[(size_t)i * C + c];
                double xc = ld_any(x, dtype, (size_t)t * C + c);
                acc += ld_any(w, dtype, (size_t)c * K + (K - 1)) * xc;
                y[(size_t)t * C + c] = silu(acc);
            }
            /* shift the history by one token */
            for (int j = 0; j + 1 < K - 1; ++j)
                for (int c = 0; c < C; ++c) hist[(size_t)j * C + c] = hist[(size_t)(j + 1) * C + c];
            if (K - 1 > 0)
                for (int c = 0; c < C; ++c)
                    hist[(size_t)(K - 2) * C + c] = ld_any(x, dtype, (size_t)t * C + c);
        }
        if (conv_out)
            for (int j = 0; j < K - 1; ++j)
                for (int c = 0; c < C; ++c)
                    conv_out[((size_t)n * (K - 1) + j) * C + c] = hist[(size_t)j * C + c];
    }
    free(hist);
    return 0;
}

/* ------------------------------------------------------------------------------------------ */
/* Gated RMSNorm: y[r][:] = o[r][:] / sqrt(mean(o[r]^2) + eps) * w * silu(z[r][:])               */
/* w may be NULL (ones).  All of o, z, w in `dtype`; y fp64.                                    */
/* ------------------------------------------------------------------------------------------ */
int orc_gated_rmsnorm(int dtype, const void *o, const void *z, const void *w, double eps, int rows,
                      int dim, double *y) {
    if (rows < 0 || dim < 1) return -1;
    for (int r = 0; r < rows; ++r) {
        double ss = 0.0;
        for (int c = 0; c < dim; ++c) {
            double v = ld_any(o, dtype, (size_t)r * dim + c);
            ss += v * v;
        }
        double inv = 1.0 / sqrt(ss / dim + eps);
        for (int c = 0; c < dim; ++c) {
            double v = ld_any(o, dtype, (size_t)r * dim + c);
            double wc = w ? ld_any(w, dtype, (size_t)c) : 1.0;
            double zc = ld_any(z, dtype, (size_t)r * dim + c);
            y[(size_t)r * dim + c] = v * inv * wc * silu(zc);
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------------------------ */
/* One (sequence, value head) unit of the full layer, token by token.                          */
/* ------------------------------------------------------------------------------------------ */
typedef struct {
    const orc_dims *dm;
    int dtype;
    const void *x, *conv_w, *z, *norm_w;
    const float *beta, *g;
    const int32_t *cu_seqlens;
    int N, T;
    const float *S0;       /* [N][Hv][d][d] fp32 or NULL */
    const double *S0d;     /* same, fp64 (used by the decode entry point) */
    const void *conv0;     /* [N][K-1][Cc] dtype or NULL */
    const double *conv0d;  /* same, fp64 */
    long long out_t0;
    double *out;           /* [T - out_t0][Hv][d] */
    double *SN;            /* [N][Hv][d][d] or NULL */
    double *out_scale;     /* [T - out_t0][Hv][d] or NULL: element scales of out */
    double *SN_scale;      /* [N][Hv][d][d] or NULL: the magnitude M at the end */
    double *Md;            /* decode: [slots][Hv][d][d] magnitude, in/out, or NULL */
    const int32_t *slot;   /* decode: state slot of each sequence, or NULL */
    int next;              /* shared work counter */
    pthread_mutex_t mu;
} unit_job;

static int take_unit(unit_job *jb) {
    pthread_mutex_lock(&jb->mu);
    int u = jb->next++;
    pthread_mutex_unlock(&jb->mu);
    return u;
}

static void run_unit(unit_job *jb, int unit) {
    const orc_dims *dm = jb->dm;
    const int Hk = dm->num_k_heads, Hv = dm->num_v_heads, d = dm->head_dim, K = dm->conv_kernel;
    const int Cc = 2 * Hk * d + Hv * d;
    const int n = unit / Hv, h = unit % Hv;
    const int hk = h / (Hv / Hk);
    const int slot = jb->slot ? jb->slot[n] : n;
    /* channel offsets of the three groups this unit reads */
    const int cq = hk * d, ck = Hk * d + hk * d, cv = 2 * Hk * d + h * d;
    const int chans[3] = {cq, ck, cv};

    double *S = (double *)calloc((size_t)d * d, sizeof(double));
    double *hist = (double *)calloc((size_t)(K > 1 ? K - 1 : 1) * 3 * d, sizeof(double));
    double *q = (double *)malloc(sizeof(double) * d), *k = (double *)malloc(sizeof(double) * d);
    double *v = (double *)malloc(sizeof(double) * d), *o = (double *)malloc(sizeof(double) * d);
    double *u = (double *)malloc(sizeof(double) * d), *kv = (double *)malloc(sizeof(double) * d);
    double *yq = (double *)malloc(sizeof(double) * 3 * d);
    /* error scales: magnitudes of the conv outputs and of q, k, v, magnitude M of the state,
       |S| km and the output scales c */
    const int scales = jb->out_scale || jb->SN_scale || jb->Md;
    double *ym = scales ? (double *)malloc(sizeof(double) * 3 * d) : NULL;
    double *M = scales ? (double *)calloc((size_t)d * d, sizeof(double)) : NULL;
    double *ak = scales ? (double *)malloc(sizeof(double) * d) : NULL;
    double *cs = scales ? (double *)malloc(sizeof(double) * d) : NULL;

    const size_t sbase = ((size_t)slot * Hv + h) * (size_t)d * d;
    if (jb->S0)
        for (size_t i = 0; i < (size_t)d * d; ++i) S[i] = (double)jb->S0[sbase + i];
    if (jb->S0d)
        for (size_t i = 0; i < (size_t)d * d; ++i) S[i] = jb->S0d[sbase + i];
    if (scales) {
        for (size_t i = 0; i < (size_t)d * d; ++i) M[i] = fabs(S[i]);
        if (jb->Md)
            for (size_t i = 0; i < (size_t)d * d; ++i) M[i] = jb->Md[sbase + i];
    }
    /* conv history for the three channel groups, oldest row first */
    for (int j = 0; j < K - 1; ++j)
        for (int gi = 0; gi < 3; ++gi)
            for (int c = 0; c < d; ++c) {
                size_t src = ((size_t)slot * (K - 1) + j) * Cc + chans[gi] + c;
                double hv = 0.0;
                if (jb->conv0) hv = ld_any(jb->conv0, jb->dtype, src);
                if (jb->conv0d) hv = jb->conv0d[src];
                hist[((size_t)j * 3 + gi) * d + c] = hv;
            }

    const int t0 = jb->cu_seqlens[n], t1 = jb->cu_seqlens[n + 1];
    for (int t = t0; t < t1; ++t) {
        /* 1. causal conv + SiLU (or pass-through) for q | k | v of this unit */
        for (int gi = 0; gi < 3; ++gi)
            for (int c = 0; c < d; ++c) {
                double xc = ld_any(jb->x, jb->dtype, (size_t)t * Cc + chans[gi] + c);
                double yv;
                double mag = fabs(xc);
                if (jb->conv_w) {
                    const size_t wrow = (size_t)(chans[gi] + c) * K;
                    double acc = 0.0, am = 0.0;
                    for (int i = 0; i < K - 1; ++i) {
                        const double wi = ld_any(jb->conv_w, jb->dtype, wrow + i);
                        const double hi = hist[((size_t)i * 3 + gi) * d + c];
                        acc += wi * hi;
                        am += fabs(wi) * fabs(hi);
                    }
                    const double wl = ld_any(jb->conv_w, jb->dtype, wrow + K - 1);
                    acc += wl * xc;
                    am += fabs(wl) * fabs(xc);
                    yv = silu(acc);
                    mag = 1.1 * am;
                } else {
                    yv = xc;
                }
                yq[gi * d + c] = yv;
                if (scales) ym[gi * d + c] = mag;
            }
        for (int j = 0; j + 1 < K - 1; ++j)
            for (int i = 0; i < 3 * d; ++i) hist[(size_t)j * 3 * d + i] = hist[(size_t)(j + 1) * 3 * d + i];
        if (K - 1 > 0)
            for (int gi = 0; gi < 3; ++gi)
                for (int c = 0; c < d; ++c)
                    hist[((size_t)(K - 2) * 3 + gi) * d + c] =
                        ld_any(jb->x, jb->dtype, (size_t)t * Cc + chans[gi] + c);

        /* 2. L2 normalisation of q and k; v passes through */
        double sq = 0.0, sk = 0.0;
        for (int c = 0; c < d; ++c) {
            sq += yq[c] * yq[c];
            sk += yq[d + c] * yq[d + c];
        }
        double rq = dm->q_scale / sqrt(sq + dm->l2_eps), rk = 1.0 / sqrt(sk + dm->l2_eps);
        for (int c = 0; c < d; ++c) {
            q[c] = yq[c] * rq;
            k[c] = yq[d + c] * rk;
            v[c] = yq[2 * d + c];
        }
        if (scales)  /* magnitudes of q, k, v in place of the conv magnitudes */
            for (int c = 0; c < d; ++c) {
                ym[c] *= rq;
                ym[d + c] *= rk;
            }

        /* 3. gated delta rule, one token */
        const double alpha = exp((double)jb->g[(size_t)t * Hv + h]);
        const double beta = (double)jb->beta[(size_t)t * Hv + h];
        for (size_t i = 0; i < (size_t)d * d; ++i) S[i] *= alpha;       /* S <- alpha S      */
        if (scales) {                                   /* |alpha S_{t-1}| km, before the write */
            for (int r = 0; r < d; ++r) {
                double acc = 0.0;
                for (int c = 0; c < d; ++c) acc += fabs(S[(size_t)r * d + c]) * ym[d + c];
                ak[r] = acc;
            }
        }
        for (int r = 0; r < d; ++r) {                                      /* kv_mem = S k      */
            double acc = 0.0;
            for (int c = 0; c < d; ++c) acc += S[(size_t)r * d + c] * k[c];
            kv[r] = acc;
        }
        for (int r = 0; r < d; ++r) u[r] = beta * (v[r] - kv[r]);          /* u = beta(v - kv)  */
        for (int r = 0; r < d; ++r)                                        /* S <- S + u k^T    */
            for (int c = 0; c < d; ++c) S[(size_t)r * d + c] += u[r] * k[c];
        for (int r = 0; r < d; ++r) {                                      /* o = S q           */
            double acc = 0.0;
            for (int c = 0; c < d; ++c) acc += S[(size_t)r * d + c] * q[c];
            o[r] = acc;
        }
        if (scales) {                         /* M <- alpha M + beta (vm + |alpha S| km) km^T */
            for (int r = 0; r < d; ++r) {
                const double a = beta * (ym[2 * d + r] + ak[r]);
                for (int c = 0; c < d; ++c)
                    M[(size_t)r * d + c] = alpha * M[(size_t)r * d + c] + a * ym[d + c];
            }
            for (int r = 0; r < d; ++r) {                              /* c = M qm           */
                double acc = 0.0;
                for (int c = 0; c < d; ++c) acc += M[(size_t)r * d + c] * ym[c];
                cs[r] = acc;
            }
        }

        /* 4. z-gated RMSNorm */
        if (jb->z) {
            double ss = 0.0, oc = 0.0;
            for (int r = 0; r < d; ++r) {
                ss += o[r] * o[r];
                if (scales) oc += fabs(o[r]) * cs[r];
            }
            const double m_eps = ss / d + dm->norm_eps;
            double inv = 1.0 / sqrt(m_eps);
            for (int r = 0; r < d; ++r) {
                double wr = jb->norm_w ? ld_any(jb->norm_w, jb->dtype, (size_t)r) : 1.0;
                double zr = ld_any(jb->z, jb->dtype, ((size_t)t * Hv + h) * d + r);
                if (scales)   /* first-order change of the normalised element (header) */
                    cs[r] = fabs(wr * silu(zr)) * inv * (cs[r] + fabs(o[r]) * oc / (d * m_eps));
                o[r] = o[r] * inv * wr * silu(zr);
            }
        }
        if ((long long)t >= jb->out_t0) {
            double *dst = jb->out + (((size_t)(t - jb->out_t0)) * Hv + h) * d;
            memcpy(dst, o, sizeof(double) * d);
            if (jb->out_scale)
                memcpy(jb->out_scale + (((size_t)(t - jb->out_t0)) * Hv + h) * d, cs,
                       sizeof(double) * d);
        }
    }
    if (jb->SN) memcpy(jb->SN + sbase, S, sizeof(double) * (size_t)d * d);
    if (jb->SN_scale) memcpy(jb->SN_scale + sbase, M, sizeof(double) * (size_t)d * d);
    if (jb->Md) memcpy(jb->Md + sbase, M, sizeof(double) * (size_t)d * d);
    free(S); free(hist); free(q); free(k); free(v); free(o); free(u); free(kv); free(yq);
    free(M); free(ak); free(cs); free(ym);
}

static void *worker(void *arg) {
    unit_job *jb = (unit_job *)arg;
    const int total = jb->N * jb->dm->num_v_heads;
    for (int u = take_unit(jb); u < total; u = take_unit(jb)) run_unit(jb, u);
    return NULL;
}

static int run_units(unit_job *jb, int nthreads) {
    pthread_mutex_init(&jb->mu, NULL);
    jb->next = 0;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    pthread_t th[256];
    int started = 0;
    for (int i = 1; i < nthreads; ++i)
        if (pthread_create(&th[started], NULL, worker, jb) == 0) ++started;
    worker(jb);
    for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
    pthread_mutex_destroy(&jb->mu);
    return 0;
}

static int dims_ok(const orc_dims *dm) {
    return dm && dm->num_k_heads > 0 && dm->num_v_heads > 0 && dm->head_dim > 0 &&
           dm->conv_kernel >= 1 && dm->num_v_heads % dm->num_k_heads == 0;
}

/* Final conv history of each sequence: the last K-1 rows of [conv0 ; x_seq]. */
static void conv_final(const orc_dims *dm, int dtype, const void *x, const int32_t *cu, int N,
                       const void *conv0, const double *conv0d, const int32_t *slot,
                       double *convN) {
    const int K = dm->conv_kernel, Cc = 2 * dm->num_k_heads * dm->head_dim + dm->num_v_heads * dm->head_dim;
    for (int n = 0; n < N; ++n) {
        const int L = cu[n + 1] - cu[n], s = slot ? slot[n] : n;
        for (int j = 0; j < K - 1; ++j) {
            /* position of output row j in the extended history of length (K-1) + L */
            const int e = L + j; /* index into [conv0 rows 0..K-2, x rows 0..L-1] */
            for (int c = 0; c < Cc; ++c) {
                double val;
                if (e < K - 1) {
                    size_t src = ((size_t)s * (K - 1) + e) * Cc + c;
                    val = conv0 ? ld_any(conv0, dtype, src) : (conv0d ? conv0d[src] : 0.0);
                } else {
                    val = ld_any(x, dtype, (size_t)(cu[n] + e - (K - 1)) * Cc + c);
                }
                convN[((size_t)s * (K - 1) + j) * Cc + c] = val;
            }
        }
    }
}

/* ------------------------------------------------------------------------------------------ */
/* Full layer over packed variable-length sequences.                                          */
/*   x [T][Cc] dtype (pre-conv q|k|v), conv_w [Cc][K] dtype or NULL (conv and SiLU off),       */
/*   beta, g [T][Hv] fp32, z [T][Hv][d] dtype or NULL (norm off), norm_w [d] dtype or NULL,    */
/*   cu_seqlens [N+1], S0 [N][Hv][d][d] fp32 or NULL, conv0 [N][K-1][Cc] dtype or NULL.          */
/*   out [T-out_t0][Hv][d] fp64: outputs of tokens t >= out_t0 only.                            */
/*   SN [N][Hv][d][d] fp64 or NULL; convN [N][K-1][Cc] fp64 or NULL.                            */
/*   out_scale [T-out_t0][Hv][d], SN_scale [N][Hv][d][d] fp64 or NULL: the error scales of the   */
/*   header (element scales of out, magnitude M of the final states).                          */
/* ------------------------------------------------------------------------------------------ */
int orc_prefill(const orc_dims *dm, int dtype, const void *x, const void *conv_w, const float *beta,
                const float *g, const void *z, const void *norm_w, const int32_t *cu_seqlens, int N,
                int T, const float *S0, const void *conv0, long long out_t0, double *out, double *SN,
                double *convN, double *out_scale, double *SN_scale, int nthreads) {
    if (!dims_ok(dm) || N < 0 || T < 0 || out_t0 < 0 || out_t0 > T) return -1;
    if (N > 0 && (cu_seqlens[0] != 0 || cu_seqlens[N] != T)) return -1;
    for (int n = 0; n < N; ++n)
        if (cu_seqlens[n + 1] < cu_seqlens[n]) return -1;
    unit_job jb;
    memset(&jb, 0, sizeof jb);
    jb.dm = dm; jb.dtype = dtype; jb.x = x; jb.conv_w = conv_w; jb.z = z; jb.norm_w = norm_w;
    jb.beta = beta; jb.g = g; jb.cu_seqlens = cu_seqlens; jb.N = N; jb.T = T; jb.S0 = S0;
    jb.conv0 = conv0; jb.out_t0 = out_t0; jb.out = out; jb.SN = SN;
    jb.out_scale = out_scale; jb.SN_scale = SN_scale;
    run_units(&jb, nthreads);
    if (convN) conv_final(dm, dtype, x, cu_seqlens, N, conv0, NULL, NULL, convN);
    return 0;
}

/* ------------------------------------------------------------------------------------------ */
/* One decode step for B sequences (one token each), states updated in place (fp64).           */
/*   x [B][Cc] dtype, beta/g [B][Hv] fp32, z [B][Hv][d] dtype or NULL.                           */
/*   conv_state [slots][K-1][Cc] fp64 in/out, S [slots][Hv][d][d] fp64 in/out,                   */
/*   slot_idx [B] or NULL (sequence b uses slot b).  out [B][Hv][d] fp64.                         */
/*   M [slots][Hv][d][d] fp64 in/out or NULL: the state magnitude of the header, carried across  */
/*   steps like S (start from |S|); out_scale [B][Hv][d] fp64 (used only with M).                */
/* ------------------------------------------------------------------------------------------ */
int orc_decode_step(const orc_dims *dm, int dtype, const void *x, const void *conv_w,
                    const float *beta, const float *g, const void *z, const void *norm_w,
                    double *conv_state, double *S, const int32_t *slot_idx, int B, double *out,
                    double *M, double *out_scale, int nthreads) {
    if (!dims_ok(dm) || B < 0) return -1;
    const int K = dm->conv_kernel, Cc = 2 * dm->num_k_heads * dm->head_dim + dm->num_v_heads * dm->head_dim;
    int32_t *cu = (int32_t *)malloc(sizeof(int32_t) * (size_t)(B + 1));
    if (!cu) return -2;
    for (int b = 0; b <= B; ++b) cu[b] = b;
    unit_job jb;
    memset(&jb, 0, sizeof jb);
    jb.dm = dm; jb.dtype = dtype; jb.x = x; jb.conv_w = conv_w; jb.z = z; jb.norm_w = norm_w;
    jb.beta = beta; jb.g = g; jb.cu_seqlens = cu; jb.N = B; jb.T = B; jb.S0d = S;
    jb.conv0d = conv_state; jb.out_t0 = 0; jb.out = out; jb.SN = S; jb.slot = slot_idx;
    jb.Md = M; jb.out_scale = M ? out_scale : NULL;
    run_units(&jb, nthreads);
    /* new conv history of each slot: drop the oldest row, append this token's input
       (all units have finished reading the old history at this point) */
    for (int b = 0; b < B && K > 1; ++b) {
        const int s = slot_idx ? slot_idx[b] : b;
        double *hs = conv_state + (size_t)s * (K - 1) * Cc;
        for (int j = 0; j + 1 < K - 1; ++j)
            for (int c = 0; c < Cc; ++c) hs[(size_t)j * Cc + c] = hs[(size_t)(j + 1) * Cc + c];
        for (int c = 0; c < Cc; ++c) hs[(size_t)(K - 2) * Cc + c] = ld_any(x, dtype, (size_t)b * Cc + c);
    }
    free(cu);
    return 0;
}
