/*
 * ckda_oracle.c -- float64 sequential CPU oracle for the Complex KDA (CKDA) recurrence.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or call this file:
 * it exists so that tests/, the smoke check and bench.py's cpu_baseline leg have a plain,
 * slow, obviously correct definition to compare the CUDA library against.  It shares no
 * code, header, table or constant with gated_delta_rule_82_b200/csrc.
 *
 * What it computes (per batch b and head h, independently; sequentially over t):
 *
 *   S := h0[b,h] or 0                                  S in R^{dk x dv}
 *   for t = 0 .. T-1:
 *     q, k := q[b,t,h,:], k[b,t,h,:]
 *     if rope_theta > 0:  rotate (q, k) by angles p * rope_theta^(-2i/dk), p = pos_offset + t
 *     if l2norm:          x <- x / sqrt(sum x^2 + 1e-6)       (per head, for q and k)
 *     S <- Diag(alpha_t) S                              (row c of S scaled by alpha_t[c])
 *     w <- S^T k
 *     S <- S + beta_t k (v_t - w)^T                     i.e. S_t = (I - b k k^T) Diag(a) S_{t-1} + b k v^T
 *     out[b,t,h,:] <- scale * S^T q                     (S after the update)
 *   hT[b,h] := S
 *
 * Sources (page title, section / equation):
 *  - "Complex KDA" paper summary (picx.dev), Background: the gated delta-rule transition
 *    A_t = (I - beta_t k_t k_t^T) Diag(alpha_t); "CKDA Definition": alpha in [-1,1]^n, beta in [0,2].
 *  - the recurrence's write term beta k v^T and read-out scale dk^-1/2 * S_t^T q_t complete the
 *    transition into a layer (the FLA KDA operator the "RoPE into the KDA q/k path" review studies).
 *  - "RoPE into the KDA q/k path" review, sections 2-3: the q/k L2 norm is a kernel-side step and
 *    the rotation is applied before it; section 5: inverse frequencies 1/base^(2i/dim).
 *  - the same review, section 3 (rotate_half, optional interleaved pairing) and the ferrox "mla"
 *    module doc (interleaved convention): pair layout of the rotation.
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *  - L2 norm epsilon: x / sqrt(sum x^2 + 1e-6); the zero vector stays zero.
 *  - alpha gates the dk (key) rows of S; Diag(alpha) is applied before the rank-one correction.
 *  - the output reads S_t, after the update.
 *  - RoPE position p = pos_offset + t, 0-based.
 *
 * Gate activation (optional input form): the "Complex KDA" paper summary, Methodology, "CKDA
 * Definition", parameterises the gates from unconstrained logits as beta_t = 2 sigma(b_t) and the
 * signed gates alpha_{t,i} = 2 sigma(a_{t,i}) - 1, sigma the logistic function.
 *
 * Backward (ckda_oracle_bwd, at the end of this file): reverse-mode gradients of the same forward,
 * pinned to central finite differences of it.
 *
 * Planted mistakes (CKDA_ORACLE_MUTANT=n at compile time) exist only so that the test suite can
 * prove its pins catch each class of error; the default build (0) is the oracle.
 */
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

#ifndef CKDA_ORACLE_MUTANT
#define CKDA_ORACLE_MUTANT 0
#endif

/* mutant ids (see tests/test_oracle_mutants.py) */
#define MUT_DH_ORDER 1      /* apply Diag(alpha) after the Householder-like factor */
#define MUT_ABS_ALPHA 2     /* drop the sign of alpha */
#define MUT_BETA_CLAMP 3    /* clamp beta to [0,1] */
#define MUT_OUT_PREV 4      /* read the output from S_{t-1} */
#define MUT_NO_SCALE 5      /* forget the dk^-1/2 read-out scale */
#define MUT_FREQ_NO2 6      /* rope frequency exponent without its factor 2 */
#define MUT_ROPE_Q_ONLY 7   /* rotate q but not k */
#define MUT_THETA_1000 8    /* rope base 1000 instead of the given one */
#define MUT_NO_L2 9         /* skip the L2 norm */
#define MUT_NORM_AFTER 10   /* L2 norm over q and k jointly instead of per vector */
#define MUT_GATE_NO_AFFINE 11 /* alpha = sigma(a), the sigmoid without its 2x - 1 map */
#define MUT_BETA_NO2 12     /* beta = sigma(b), without the factor 2 */

#define L2_EPS 1e-6

static const int g_mutant = CKDA_ORACLE_MUTANT;

int ckda_oracle_mutant(void) { return g_mutant; }

/* logistic function, evaluated on the side where exp() cannot overflow */
static double logistic(double x) {
    if (x >= 0.0) return 1.0 / (1.0 + exp(-x));
    double e = exp(x);
    return e / (1.0 + e);
}

/*
 * Gates from logits: alpha[i] = 2 sigma(a[i]) - 1 for i < na, beta[j] = 2 sigma(b[j]) for j < nb
 * ("Complex KDA" paper summary, Methodology, CKDA Definition).  Either pair may be null.
 */
int ckda_oracle_gates(const double* a, double* alpha, long long na, const double* b, double* beta,
                      long long nb) {
    if (a && alpha)
        for (long long i = 0; i < na; ++i)
            alpha[i] = g_mutant == MUT_GATE_NO_AFFINE ? logistic(a[i]) : 2.0 * logistic(a[i]) - 1.0;
    if (b && beta)
        for (long long j = 0; j < nb; ++j)
            beta[j] = g_mutant == MUT_BETA_NO2 ? logistic(b[j]) : 2.0 * logistic(b[j]);
    return 0;
}

/* Rotate one head vector x[0..d) in place by position p (see header comment for the pairing). */
static void rope_rotate(double* x, int d, long long p, double theta, int convention) {
    if (g_mutant == MUT_THETA_1000) theta = 1000.0;
    int half = d / 2;
    for (int i = 0; i < half; ++i) {
        double expo = (g_mutant == MUT_FREQ_NO2) ? (double)i / (double)d : 2.0 * (double)i / (double)d;
        double omega = pow(theta, -expo);
        double phi = (double)p * omega;
        double c = cos(phi), s = sin(phi);
        int a, b;
        if (convention == 0) { a = i; b = i + half; }       /* half-split: (x_i, x_{i+d/2}) */
        else                 { a = 2 * i; b = 2 * i + 1; }  /* interleaved: (x_{2i}, x_{2i+1}) */
        double xa = x[a], xb = x[b];
        x[a] = xa * c - xb * s;
        x[b] = xb * c + xa * s;
    }
}

static void l2_normalise(double* x, int d) {
    double ss = 0.0;
    for (int i = 0; i < d; ++i) ss += x[i] * x[i];
    double r = 1.0 / sqrt(ss + L2_EPS);
    for (int i = 0; i < d; ++i) x[i] *= r;
}

/* The q/k prologue for one token of one head: optional rotation of the first `rot` channels
 * (a rotation of that sub-vector as a head of its own, the remaining channels carried through:
 * the partial rotation of the "RoPE review", section 3), then optional L2 norm over all dk. */
static void prologue_pair(double* q, double* k, int dk, int rot, long long p, int l2norm,
                          double theta, int convention) {
    if (theta > 0.0) {
        rope_rotate(q, rot, p, theta, convention);
        if (g_mutant != MUT_ROPE_Q_ONLY) rope_rotate(k, rot, p, theta, convention);
    }
    if (l2norm && g_mutant != MUT_NO_L2) {
        if (g_mutant == MUT_NORM_AFTER) {
            double ss = 0.0;
            for (int i = 0; i < dk; ++i) ss += q[i] * q[i] + k[i] * k[i];
            double r = 1.0 / sqrt(ss + L2_EPS);
            for (int i = 0; i < dk; ++i) { q[i] *= r; k[i] *= r; }
        } else {
            l2_normalise(q, dk);
            l2_normalise(k, dk);
        }
    }
}

/* One token of the recurrence on state S (dk x dv, row-major), given prepared q, k. */
static void recurrence_token(double* S, const double* q, const double* k, const double* v,
                             const double* alpha, double beta, double scale, int dk, int dv,
                             double* w, double* o) {
    if (g_mutant == MUT_BETA_CLAMP && beta > 1.0) beta = 1.0;
    if (g_mutant == MUT_OUT_PREV) {
        for (int j = 0; j < dv; ++j) {
            double acc = 0.0;
            for (int c = 0; c < dk; ++c) acc += S[(size_t)c * dv + j] * q[c];
            o[j] = scale * acc;
        }
    }
    if (g_mutant == MUT_DH_ORDER) {
        /* S <- Diag(a) (I - b k k^T) S + b k v^T  (factors in the wrong order) */
        for (int j = 0; j < dv; ++j) {
            double acc = 0.0;
            for (int c = 0; c < dk; ++c) acc += S[(size_t)c * dv + j] * k[c];
            w[j] = acc;
        }
        for (int c = 0; c < dk; ++c) {
            double a = alpha[c];
            for (int j = 0; j < dv; ++j) {
                double s = S[(size_t)c * dv + j] - beta * k[c] * w[j];
                S[(size_t)c * dv + j] = a * s + beta * k[c] * v[j];
            }
        }
    } else {
        /* Diag(alpha_t) S_{t-1} */
        for (int c = 0; c < dk; ++c) {
            double a = (g_mutant == MUT_ABS_ALPHA) ? fabs(alpha[c]) : alpha[c];
            for (int j = 0; j < dv; ++j) S[(size_t)c * dv + j] *= a;
        }
        /* w = S^T k */
        for (int j = 0; j < dv; ++j) {
            double acc = 0.0;
            for (int c = 0; c < dk; ++c) acc += S[(size_t)c * dv + j] * k[c];
            w[j] = acc;
        }
        /* S += beta k (v - w)^T */
        for (int c = 0; c < dk; ++c) {
            double bk = beta * k[c];
            for (int j = 0; j < dv; ++j) S[(size_t)c * dv + j] += bk * (v[j] - w[j]);
        }
    }
    if (g_mutant != MUT_OUT_PREV) {
        for (int j = 0; j < dv; ++j) {
            double acc = 0.0;
            for (int c = 0; c < dk; ++c) acc += S[(size_t)c * dv + j] * q[c];
            o[j] = scale * acc;
        }
    }
    if (g_mutant == MUT_NO_SCALE && scale != 0.0) {
        for (int j = 0; j < dv; ++j) o[j] /= scale;
    }
}

typedef struct {
    const double *q, *k, *v, *alpha, *beta, *h0;
    double *out, *hT;
    int B, T, H, dk, dv, l2norm, convention, rot;
    double theta, scale;
    long long pos_offset;
    const long long* cu;      /* packed sequences: token offsets [B + 1], or NULL (batched) */
    int next;                 /* next (b,h) pair to process */
    pthread_mutex_t lock;
    int status;
} fwd_job;

static int take_pair(fwd_job* J) {
    pthread_mutex_lock(&J->lock);
    int p = J->next++;
    pthread_mutex_unlock(&J->lock);
    return p;
}

static void* fwd_worker(void* arg) {
    fwd_job* J = (fwd_job*)arg;
    int dk = J->dk, dv = J->dv, H = J->H, T = J->T;
    double* S = (double*)malloc(sizeof(double) * (size_t)dk * dv);
    double* qb = (double*)malloc(sizeof(double) * dk);
    double* kb = (double*)malloc(sizeof(double) * dk);
    double* w = (double*)malloc(sizeof(double) * dv);
    double* o = (double*)malloc(sizeof(double) * dv);
    if (!S || !qb || !kb || !w || !o) {
        J->status = -2;
        free(S); free(qb); free(kb); free(w); free(o);
        return NULL;
    }
    for (;;) {
        int pair = take_pair(J);
        if (pair >= J->B * H) break;
        int b = pair / H, h = pair % H;
        /* sequence b: tokens first .. first + len - 1 of the token axis (a packed sequence, or
           row b of the batch); its positions start again at pos_offset */
        long long first = J->cu ? J->cu[b] : (long long)b * T;
        long long len = J->cu ? J->cu[b + 1] - J->cu[b] : T;
        size_t sofs = ((size_t)b * H + h) * (size_t)dk * dv;
        if (J->h0) memcpy(S, J->h0 + sofs, sizeof(double) * (size_t)dk * dv);
        else memset(S, 0, sizeof(double) * (size_t)dk * dv);
        for (long long t = 0; t < len; ++t) {
            size_t row = ((size_t)(first + t)) * H + h;
            memcpy(qb, J->q + row * dk, sizeof(double) * dk);
            memcpy(kb, J->k + row * dk, sizeof(double) * dk);
            prologue_pair(qb, kb, dk, J->rot, J->pos_offset + t, J->l2norm, J->theta, J->convention);
            recurrence_token(S, qb, kb, J->v + row * dv, J->alpha + row * dk, J->beta[row], J->scale,
                             dk, dv, w, o);
            memcpy(J->out + row * dv, o, sizeof(double) * dv);
        }
        if (J->hT) memcpy(J->hT + sofs, S, sizeof(double) * (size_t)dk * dv);
    }
    free(S); free(qb); free(kb); free(w); free(o);
    return NULL;
}

/* Runs the (sequence, head) pairs of J on nthreads threads (the caller's included). */
static int run_fwd_job(fwd_job* J, int nthreads) {
    J->next = 0;
    J->status = 0;
    pthread_mutex_init(&J->lock, NULL);
    int pairs = J->B * J->H;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > pairs) nthreads = pairs > 0 ? pairs : 1;
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
    if (!th) { pthread_mutex_destroy(&J->lock); return -2; }
    int started = 0;
    for (int i = 1; i < nthreads; ++i) {
        if (pthread_create(&th[i], NULL, fwd_worker, J) == 0) ++started; else break;
    }
    fwd_worker(J);
    for (int i = 1; i <= started; ++i) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&J->lock);
    return J->status;
}

static int check_rope(int dk, double rope_theta, int* rope_dims) {
    if (*rope_dims == 0) *rope_dims = dk;
    if (rope_theta > 0.0 && ((*rope_dims % 2) != 0 || *rope_dims < 0 || *rope_dims > dk)) return -1;
    return 0;
}

/*
 * Chunk-free forward over a whole sequence batch.
 *   q, k, alpha: [B, T, H, dk];  v, out: [B, T, H, dv];  beta: [B, T, H];
 *   h0, hT: [B, H, dk, dv] (h0 may be NULL for a zero state, hT may be NULL);
 *   rope_dims: channels rotated (0 = all dk; otherwise an even number up to dk).
 * Returns 0 on success, -1 on bad arguments, -2 on allocation failure.
 */
int ckda_oracle_fwd(const double* q, const double* k, const double* v, const double* alpha,
                    const double* beta, const double* h0, double* out, double* hT, int B, int T,
                    int H, int dk, int dv, int l2norm, double rope_theta, int rope_convention,
                    int rope_dims, double scale, long long pos_offset, int nthreads) {
    if (!q || !k || !v || !alpha || !beta || !out) return -1;
    if (B < 0 || T < 0 || H < 0 || dk <= 0 || dv <= 0) return -1;
    if (check_rope(dk, rope_theta, &rope_dims) != 0) return -1;
    fwd_job J;
    J.q = q; J.k = k; J.v = v; J.alpha = alpha; J.beta = beta; J.h0 = h0; J.out = out; J.hT = hT;
    J.B = B; J.T = T; J.H = H; J.dk = dk; J.dv = dv; J.l2norm = l2norm;
    J.convention = rope_convention; J.theta = rope_theta; J.scale = scale; J.rot = rope_dims;
    J.pos_offset = pos_offset; J.cu = NULL;
    return run_fwd_job(&J, nthreads);
}

/*
 * Forward over packed sequences of different lengths (the cu_seqlens layout of the rotary that
 * FLA's attention layer applies: "RoPE review", section 4).  Sequence s owns tokens
 * cu[s] .. cu[s+1] - 1 of the token axis; it starts from h0[s] (or zero), ends in hT[s], and its
 * rotary positions start again at pos_offset.  No state crosses from one sequence to the next.
 *   q, k, alpha: [T_total, H, dk];  v, out: [T_total, H, dv];  beta: [T_total, H];
 *   h0, hT: [n_seqs, H, dk, dv];  cu: [n_seqs + 1], cu[0] = 0, non-decreasing, cu[n_seqs] = T_total.
 * Returns 0 on success, -1 on bad arguments, -2 on allocation failure.
 */
int ckda_oracle_fwd_varlen(const double* q, const double* k, const double* v,
                           const double* alpha, const double* beta, const double* h0,
                           double* out, double* hT, const long long* cu, int n_seqs, int H,
                           int dk, int dv, int l2norm, double rope_theta, int rope_convention,
                           int rope_dims, double scale, long long pos_offset, int nthreads) {
    if (!cu || n_seqs < 0 || H < 0 || dk <= 0 || dv <= 0) return -1;
    if (cu[0] != 0) return -1;
    for (int s = 0; s < n_seqs; ++s)
        if (cu[s + 1] < cu[s]) return -1;
    if (cu[n_seqs] > 0 && (!q || !k || !v || !alpha || !beta || !out)) return -1;
    if (check_rope(dk, rope_theta, &rope_dims) != 0) return -1;
    fwd_job J;
    J.q = q; J.k = k; J.v = v; J.alpha = alpha; J.beta = beta; J.h0 = h0; J.out = out; J.hT = hT;
    J.B = n_seqs; J.T = 0; J.H = H; J.dk = dk; J.dv = dv; J.l2norm = l2norm;
    J.convention = rope_convention; J.theta = rope_theta; J.scale = scale; J.rot = rope_dims;
    J.pos_offset = pos_offset; J.cu = cu;
    return run_fwd_job(&J, nthreads);
}

/*
 * One decode step for N independent sequences: the same token body as the forward, applied
 * in place to state [N, H, dk, dv] with the rotation at position pos[n] (pos may be NULL when
 * rope_theta <= 0).  q, k, alpha: [N, H, dk]; v, out: [N, H, dv]; beta: [N, H].
 */
int ckda_oracle_decode(const double* q, const double* k, const double* v, const double* alpha,
                       const double* beta, double* state, double* out, const long long* pos,
                       int N, int H, int dk, int dv, int l2norm, double rope_theta,
                       int rope_convention, int rope_dims, double scale) {
    if (!q || !k || !v || !alpha || !beta || !state || !out) return -1;
    if (check_rope(dk, rope_theta, &rope_dims) != 0 || (rope_theta > 0.0 && !pos)) return -1;
    double* qb = (double*)malloc(sizeof(double) * dk);
    double* kb = (double*)malloc(sizeof(double) * dk);
    double* w = (double*)malloc(sizeof(double) * dv);
    if (!qb || !kb || !w) { free(qb); free(kb); free(w); return -2; }
    for (int n = 0; n < N; ++n) {
        for (int h = 0; h < H; ++h) {
            size_t row = (size_t)n * H + h;
            memcpy(qb, q + row * dk, sizeof(double) * dk);
            memcpy(kb, k + row * dk, sizeof(double) * dk);
            prologue_pair(qb, kb, dk, rope_dims, rope_theta > 0.0 ? pos[n] : 0, l2norm, rope_theta,
                          rope_convention);
            recurrence_token(state + row * (size_t)dk * dv, qb, kb, v + row * dv, alpha + row * dk,
                             beta[row], scale, dk, dv, w, out + row * dv);
        }
    }
    free(qb); free(kb); free(w);
    return 0;
}

/*
 * The q/k prologue alone on one tensor x [B, T, H, d] -> y: rotation at p = pos_offset + t
 * (if rope_theta > 0), then the per-head L2 norm (if l2norm).
 */
int ckda_oracle_prologue(const double* x, double* y, int B, int T, int H, int d, int l2norm,
                         double rope_theta, int rope_convention, int rope_dims,
                         long long pos_offset) {
    if (!x || !y || d <= 0) return -1;
    if (rope_dims == 0) rope_dims = d;
    if (rope_theta > 0.0 && ((rope_dims % 2) != 0 || rope_dims < 0 || rope_dims > d)) return -1;
    double* buf = (double*)malloc(sizeof(double) * d);
    if (!buf) return -2;
    for (int b = 0; b < B; ++b)
        for (int t = 0; t < T; ++t)
            for (int h = 0; h < H; ++h) {
                size_t row = ((size_t)b * T + t) * H + h;
                memcpy(buf, x + row * d, sizeof(double) * d);
                if (rope_theta > 0.0)
                    rope_rotate(buf, rope_dims, pos_offset + t, rope_theta, rope_convention);
                if (l2norm && g_mutant != MUT_NO_L2) l2_normalise(buf, d);
                memcpy(y + row * d, buf, sizeof(double) * d);
            }
    free(buf);
    return 0;
}

/*
 * Reverse-mode gradients of the forward above, by backpropagation through the token loop, for a
 * loss L with dL/dout = dout and dL/dhT = dhT (either may be NULL for zero).  Per (b, h) the
 * forward is replayed with every state S_0 .. S_T kept, then the tokens are walked backwards.
 * One token (q^, k^ the prepared vectors, S' = Diag(alpha) S_{t-1}, w = S'^T k^, u = v - w,
 * S_t = S' + beta k^ u^T, o = scale S_t^T q^) gives, with G the gradient of S_t (future tokens
 * plus this token's read-out, G += scale q^ do^T):
 *   dq^ = scale S_t do,  dbeta = k^T G u,  dv = du = beta G^T k^,  dk^ = beta G u + S' dw,
 *   dw = -du,  G' = G + k^ dw^T (gradient of S'),  dalpha_i = sum_j G'_ij S_{t-1,ij},
 *   gradient of S_{t-1} = Diag(alpha) G'.
 * The prologue is differentiated through: for the norm n(y) = y s, s = (|y|^2 + eps)^(-1/2),
 * dy = s dn - s^3 (y . dn) y; the rotation is orthogonal, so dx = R^T dy, the rotation by -p.
 * Outputs dq, dk, dalpha: [B, T, H, dk]; dv: [B, T, H, dv]; dbeta: [B, T, H]; dh0: [B, H, dk, dv]
 * (may be NULL).  Gates are taken as values (the logit form composes with dalpha / da =
 * (1 - alpha^2) / 2 and dbeta / db = beta (1 - beta / 2)).
 * Returns 0 on success, -1 on bad arguments, -2 on allocation failure.
 */
typedef struct {
    const double *q, *k, *v, *alpha, *beta, *h0, *dout, *dhT;
    double *dq, *dk, *dv, *dalpha, *dbeta, *dh0;
    int B, T, H, dk_, dv_, l2norm, convention, rot;
    double theta, scale;
    long long pos_offset;
    int next;
    pthread_mutex_t lock;
    int status;
} bwd_job;

/* Gradient through x^ = n(R x) for one head vector: y is R x (before the norm), g the gradient of
 * x^ on entry and of x on return. */
static void prologue_backward(double* g, const double* y, int d, int rot, long long p, int l2norm,
                              double theta, int convention) {
    if (l2norm) {
        double ss = 0.0, yg = 0.0;
        for (int i = 0; i < d; ++i) { ss += y[i] * y[i]; yg += y[i] * g[i]; }
        double s = 1.0 / sqrt(ss + L2_EPS);
        for (int i = 0; i < d; ++i) g[i] = s * g[i] - s * s * s * yg * y[i];
    }
    if (theta > 0.0) rope_rotate(g, rot, -p, theta, convention);
}

static void* bwd_worker(void* arg) {
    bwd_job* J = (bwd_job*)arg;
    const int dk = J->dk_, dv = J->dv_, H = J->H, T = J->T;
    const size_t SS = (size_t)dk * dv;
    double* St = (double*)malloc(sizeof(double) * SS * (size_t)(T + 1));   /* S_0 .. S_T */
    double* Y = (double*)malloc(sizeof(double) * (size_t)T * 2 * dk);      /* R q, R k per token */
    double* QK = (double*)malloc(sizeof(double) * (size_t)T * 2 * dk);     /* q^, k^ per token */
    double* G = (double*)malloc(sizeof(double) * SS);
    double* Sp = (double*)malloc(sizeof(double) * SS);
    double* w = (double*)malloc(sizeof(double) * dv);
    double* u = (double*)malloc(sizeof(double) * dv);
    double* du = (double*)malloc(sizeof(double) * dv);
    double* o = (double*)malloc(sizeof(double) * dv);
    double* gq = (double*)malloc(sizeof(double) * dk);
    double* gk = (double*)malloc(sizeof(double) * dk);
    if (!St || !Y || !QK || !G || !Sp || !w || !u || !du || !o || !gq || !gk) {
        J->status = -2;
        free(St); free(Y); free(QK); free(G); free(Sp); free(w); free(u); free(du); free(o);
        free(gq); free(gk);
        return NULL;
    }
    for (;;) {
        pthread_mutex_lock(&J->lock);
        int pair = J->next++;
        pthread_mutex_unlock(&J->lock);
        if (pair >= J->B * H) break;
        int b = pair / H, h = pair % H;
        size_t sofs = ((size_t)b * H + h) * SS;
        /* forward replay, keeping every state and the prepared vectors */
        if (J->h0) memcpy(St, J->h0 + sofs, sizeof(double) * SS);
        else memset(St, 0, sizeof(double) * SS);
        for (int t = 0; t < T; ++t) {
            size_t row = ((size_t)b * T + t) * H + h;
            double* yq = Y + (size_t)t * 2 * dk;
            double* yk = yq + dk;
            double* qh = QK + (size_t)t * 2 * dk;
            double* kh = qh + dk;
            memcpy(yq, J->q + row * dk, sizeof(double) * dk);
            memcpy(yk, J->k + row * dk, sizeof(double) * dk);
            if (J->theta > 0.0) {
                rope_rotate(yq, J->rot, J->pos_offset + t, J->theta, J->convention);
                rope_rotate(yk, J->rot, J->pos_offset + t, J->theta, J->convention);
            }
            memcpy(qh, yq, sizeof(double) * dk);
            memcpy(kh, yk, sizeof(double) * dk);
            if (J->l2norm) {
                l2_normalise(qh, dk);
                l2_normalise(kh, dk);
            }
            double* S = St + (size_t)(t + 1) * SS;
            memcpy(S, St + (size_t)t * SS, sizeof(double) * SS);
            recurrence_token(S, qh, kh, J->v + row * dv, J->alpha + row * dk, J->beta[row],
                             J->scale, dk, dv, w, o);
        }
        /* backward over the tokens */
        if (J->dhT) memcpy(G, J->dhT + sofs, sizeof(double) * SS);
        else memset(G, 0, sizeof(double) * SS);
        for (int t = T - 1; t >= 0; --t) {
            size_t row = ((size_t)b * T + t) * H + h;
            const double* S = St + (size_t)(t + 1) * SS;
            const double* S0 = St + (size_t)t * SS;
            const double* qh = QK + (size_t)t * 2 * dk;
            const double* kh = qh + dk;
            const double* a = J->alpha + row * dk;
            const double* vt = J->v + row * dv;
            const double bt = J->beta[row];
            const double* dot = J->dout ? J->dout + row * dv : NULL;
            /* read-out: dq^ = scale S_t do, G += scale q^ do^T */
            for (int i = 0; i < dk; ++i) {
                double acc = 0.0;
                if (dot)
                    for (int j = 0; j < dv; ++j) acc += S[(size_t)i * dv + j] * dot[j];
                gq[i] = J->scale * acc;
            }
            if (dot)
                for (int i = 0; i < dk; ++i)
                    for (int j = 0; j < dv; ++j) G[(size_t)i * dv + j] += J->scale * qh[i] * dot[j];
            /* S' = Diag(alpha) S_{t-1}, w = S'^T k^, u = v - w */
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j) Sp[(size_t)i * dv + j] = a[i] * S0[(size_t)i * dv + j];
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int i = 0; i < dk; ++i) acc += Sp[(size_t)i * dv + j] * kh[i];
                w[j] = acc;
                u[j] = vt[j] - acc;
            }
            /* rank-one write */
            double db = 0.0;
            for (int i = 0; i < dk; ++i) {
                double gu = 0.0;
                for (int j = 0; j < dv; ++j) gu += G[(size_t)i * dv + j] * u[j];
                db += kh[i] * gu;
                gk[i] = bt * gu;
            }
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int i = 0; i < dk; ++i) acc += G[(size_t)i * dv + j] * kh[i];
                du[j] = bt * acc;
            }
            J->dbeta[row] = db;
            for (int j = 0; j < dv; ++j) J->dv[row * dv + j] = du[j];
            /* w = S'^T k^ with dw = -du: G' = G + k^ dw^T, dk^ += S' dw */
            for (int i = 0; i < dk; ++i) {
                double acc = 0.0;
                for (int j = 0; j < dv; ++j) {
                    G[(size_t)i * dv + j] -= kh[i] * du[j];
                    acc -= Sp[(size_t)i * dv + j] * du[j];
                }
                gk[i] += acc;
            }
            /* S' = Diag(alpha) S_{t-1} */
            for (int i = 0; i < dk; ++i) {
                double acc = 0.0;
                for (int j = 0; j < dv; ++j) {
                    acc += G[(size_t)i * dv + j] * S0[(size_t)i * dv + j];
                    G[(size_t)i * dv + j] *= a[i];
                }
                J->dalpha[row * dk + i] = acc;
            }
            /* prologue */
            const double* yq = Y + (size_t)t * 2 * dk;
            const double* yk = yq + dk;
            prologue_backward(gq, yq, dk, J->rot, J->pos_offset + t, J->l2norm, J->theta, J->convention);
            prologue_backward(gk, yk, dk, J->rot, J->pos_offset + t, J->l2norm, J->theta, J->convention);
            memcpy(J->dq + row * dk, gq, sizeof(double) * dk);
            memcpy(J->dk + row * dk, gk, sizeof(double) * dk);
        }
        if (J->dh0) memcpy(J->dh0 + sofs, G, sizeof(double) * SS);
    }
    free(St); free(Y); free(QK); free(G); free(Sp); free(w); free(u); free(du); free(o);
    free(gq); free(gk);
    return NULL;
}

int ckda_oracle_bwd(const double* q, const double* k, const double* v, const double* alpha,
                    const double* beta, const double* h0, const double* dout, const double* dhT,
                    double* dq, double* dk_out, double* dv_out, double* dalpha, double* dbeta,
                    double* dh0, int B, int T, int H, int dk, int dv, int l2norm, double rope_theta,
                    int rope_convention, int rope_dims, double scale, long long pos_offset,
                    int nthreads) {
    if (!q || !k || !v || !alpha || !beta || !dq || !dk_out || !dv_out || !dalpha || !dbeta)
        return -1;
    if (B < 0 || T < 0 || H < 0 || dk <= 0 || dv <= 0) return -1;
    if (check_rope(dk, rope_theta, &rope_dims) != 0) return -1;
    bwd_job J;
    J.q = q; J.k = k; J.v = v; J.alpha = alpha; J.beta = beta; J.h0 = h0; J.dout = dout;
    J.dhT = dhT; J.dq = dq; J.dk = dk_out; J.dv = dv_out; J.dalpha = dalpha; J.dbeta = dbeta;
    J.dh0 = dh0; J.B = B; J.T = T; J.H = H; J.dk_ = dk; J.dv_ = dv; J.l2norm = l2norm;
    J.convention = rope_convention; J.rot = rope_dims; J.theta = rope_theta; J.scale = scale;
    J.pos_offset = pos_offset; J.next = 0; J.status = 0;
    pthread_mutex_init(&J.lock, NULL);
    int pairs = B * H;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > pairs) nthreads = pairs > 0 ? pairs : 1;
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
    if (!th) { pthread_mutex_destroy(&J.lock); return -2; }
    int started = 0;
    for (int i = 1; i < nthreads; ++i) {
        if (pthread_create(&th[i], NULL, bwd_worker, &J) == 0) ++started; else break;
    }
    bwd_worker(&J);
    for (int i = 1; i <= started; ++i) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&J.lock);
    return J.status;
}
