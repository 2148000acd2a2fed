/*
 * retention_oracle.c -- fp64 host reference for the retention contraction.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the checker the CUDA path is
 * compared against.  Only tests/, the smoke check and the CPU-baseline leg of
 * the benchmark load it.  It shares no code, header, table or constant with the
 * CUDA library (retnet_retention_chunkwise_b200/csrc), and it never includes
 * anything from there.
 *
 * What it computes (source: "Retentive Networks -- Microsoft Propone
 * l'Alternativa Architetturale ai Transformer", aimpact.prandi.net, section
 * "Il meccanismo: Multi-Scale Retention"):
 *
 *   retention sum       y_n = sum_{m<=n} gamma^(n-m) (q_n . k_m) v_m
 *   recurrent form      S_n = gamma S_{n-1} + k_n^T v_n ,   y_n = q_n S_n
 *   chunkwise form      blocks of length C: the parallel rule inside a block,
 *                       the recurrence between blocks (stated in words only)
 *
 * Row vectors: q_n, k_n in R^{1 x dk}, v_n, y_n in R^{1 x dv}, S in R^{dk x dv}
 * (the state shape "h x d" given in the author responses on paperhub.cn,
 * "Retentive Network: A Successor to Transformer ...", reply on inference cost).
 * One gamma per head (same page 1 section: each head has its own gamma).
 *
 * Readings where the pages are silent (all stated again in the design notes):
 *   - gamma^0 = 1 also for gamma = 0 (the diagonal term is kept);
 *   - the state before the first token is state_in, or zero when none is given;
 *   - state_out is S after the last token of the call;
 *   - no normalisation and no denominator (author responses on paperhub.cn,
 *     reply comparing Eq. (1) with RFA-Gate);
 *   - a chunk length that does not divide L leaves a shorter last chunk.
 *
 * Layout: q, k [B][H][L][dk], v, y [B][H][L][dv], state [B][H][dk][dv], all
 * row-major doubles.  gamma [H].  Heads are independent; threads take whole
 * (b, h) pairs.  Every function returns 0 on success, -1 on bad arguments.
 */
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

/* gamma^n for integer n >= 0, with gamma^0 = 1 for every gamma (0^0 = 1). */
static double gpow(double g, long n) {
    if (n == 0) return 1.0;
    return pow(g, (double)n);
}

typedef struct {
    int form;            /* 0 recurrent, 1 parallel (double sum), 2 chunkwise */
    int B, H, L, dk, dv, C;
    const double *q, *k, *v, *gamma, *state_in;
    double *y, *state_out;
    int next;            /* next (b,h) pair to take */
    pthread_mutex_t lock;
} job_t;

/* Recurrent form: S <- gamma S + k_n^T v_n, then y_n = q_n S (page 1, the
 * "forma ricorrente" sentence).  This is the definition itself: unrolling the
 * recurrence gives S_n = sum_{m<=n} gamma^(n-m) k_m^T v_m, so q_n S_n is the
 * retention sum plus gamma^(n+1) q_n S_in. */
static void head_recurrent(const job_t* J, const double* q, const double* k,
                           const double* v, double g, const double* s_in,
                           double* y, double* s_out) {
    const int L = J->L, dk = J->dk, dv = J->dv;
    double* S = (double*)calloc((size_t)dk * dv, sizeof(double));
    if (s_in) memcpy(S, s_in, sizeof(double) * (size_t)dk * dv);
    for (int n = 0; n < L; ++n) {
        const double* qn = q + (size_t)n * dk;
        const double* kn = k + (size_t)n * dk;
        const double* vn = v + (size_t)n * dv;
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j)
                S[(size_t)i * dv + j] = g * S[(size_t)i * dv + j] + kn[i] * vn[j];
        double* yn = y + (size_t)n * dv;
        for (int j = 0; j < dv; ++j) {
            double acc = 0.0;
            for (int i = 0; i < dk; ++i) acc += qn[i] * S[(size_t)i * dv + j];
            yn[j] = acc;
        }
    }
    if (s_out) memcpy(s_out, S, sizeof(double) * (size_t)dk * dv);
    free(S);
}

/* Parallel form as the plain double sum of the definition (page 1, the
 * "Y_n = sum_(m<=n) gamma^(n-m) Q_n K_m^T V_m" sentence), plus the carried-in
 * state term gamma^(n+1) q_n S_in. */
static void head_parallel(const job_t* J, const double* q, const double* k,
                          const double* v, double g, const double* s_in,
                          double* y, double* s_out) {
    const int L = J->L, dk = J->dk, dv = J->dv;
    for (int n = 0; n < L; ++n) {
        const double* qn = q + (size_t)n * dk;
        double* yn = y + (size_t)n * dv;
        for (int j = 0; j < dv; ++j) yn[j] = 0.0;
        for (int m = 0; m <= n; ++m) {
            const double* km = k + (size_t)m * dk;
            const double* vm = v + (size_t)m * dv;
            double s = 0.0;
            for (int i = 0; i < dk; ++i) s += qn[i] * km[i];
            s *= gpow(g, n - m);
            for (int j = 0; j < dv; ++j) yn[j] += s * vm[j];
        }
        if (s_in) {
            const double w = gpow(g, (long)n + 1);
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int i = 0; i < dk; ++i) acc += qn[i] * s_in[(size_t)i * dv + j];
                yn[j] += w * acc;
            }
        }
    }
    if (s_out) {
        /* S_{L-1} = gamma^L S_in + sum_m gamma^(L-1-m) k_m^T v_m */
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) {
                double acc = s_in ? gpow(g, L) * s_in[(size_t)i * dv + j] : 0.0;
                for (int m = 0; m < L; ++m)
                    acc += gpow(g, (long)L - 1 - m) * k[(size_t)m * dk + i] * v[(size_t)m * dv + j];
                s_out[(size_t)i * dv + j] = acc;
            }
    }
}

/* Chunkwise form (page 1, the "forma chunkwise" sentence: blocks of length C,
 * parallel inside the block, recurrence between blocks).  Splitting the
 * definition's sum at the block start t0 gives, for local index i < l:
 *   y_{t0+i} = sum_{j<=i} gamma^(i-j) (q_i . k_j) v_j  +  gamma^(i+1) q_i S_prev
 *   S_new    = gamma^l S_prev + sum_{j<l} gamma^(l-1-j) k_j^T v_j
 * with l = C, or the remainder for the last block. */
static void head_chunkwise(const job_t* J, const double* q, const double* k,
                           const double* v, double g, const double* s_in,
                           double* y, double* s_out) {
    const int L = J->L, dk = J->dk, dv = J->dv, C = J->C;
    double* S = (double*)calloc((size_t)dk * dv, sizeof(double));
    double* Sn = (double*)malloc(sizeof(double) * (size_t)dk * dv);
    if (s_in) memcpy(S, s_in, sizeof(double) * (size_t)dk * dv);
    for (int t0 = 0; t0 < L; t0 += C) {
        const int l = (L - t0 < C) ? (L - t0) : C;
        for (int i = 0; i < l; ++i) {
            const double* qi = q + (size_t)(t0 + i) * dk;
            double* yi = y + (size_t)(t0 + i) * dv;
            for (int c = 0; c < dv; ++c) yi[c] = 0.0;
            for (int j = 0; j <= i; ++j) {
                const double* kj = k + (size_t)(t0 + j) * dk;
                const double* vj = v + (size_t)(t0 + j) * dv;
                double s = 0.0;
                for (int d = 0; d < dk; ++d) s += qi[d] * kj[d];
                s *= gpow(g, i - j);
                for (int c = 0; c < dv; ++c) yi[c] += s * vj[c];
            }
            const double xi = gpow(g, (long)i + 1);
            for (int c = 0; c < dv; ++c) {
                double acc = 0.0;
                for (int d = 0; d < dk; ++d) acc += qi[d] * S[(size_t)d * dv + c];
                yi[c] += xi * acc;
            }
        }
        const double gl = gpow(g, l);
        for (int d = 0; d < dk; ++d)
            for (int c = 0; c < dv; ++c) {
                double acc = gl * S[(size_t)d * dv + c];
                for (int j = 0; j < l; ++j)
                    acc += gpow(g, (long)l - 1 - j) * k[(size_t)(t0 + j) * dk + d] *
                           v[(size_t)(t0 + j) * dv + c];
                Sn[(size_t)d * dv + c] = acc;
            }
        memcpy(S, Sn, sizeof(double) * (size_t)dk * dv);
    }
    if (s_out) memcpy(s_out, S, sizeof(double) * (size_t)dk * dv);
    free(Sn);
    free(S);
}

static void* worker(void* arg) {
    job_t* J = (job_t*)arg;
    const size_t qs = (size_t)J->L * J->dk, vs = (size_t)J->L * J->dv;
    const size_t ss = (size_t)J->dk * J->dv;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        const int p = J->next++;
        pthread_mutex_unlock(&J->lock);
        if (p >= J->B * J->H) break;
        const int h = p % J->H;
        const double* si = J->state_in ? J->state_in + (size_t)p * ss : NULL;
        double* so = J->state_out ? J->state_out + (size_t)p * ss : NULL;
        const double* q = J->q + (size_t)p * qs;
        const double* k = J->k + (size_t)p * qs;
        const double* v = J->v + (size_t)p * vs;
        double* y = J->y + (size_t)p * vs;
        if (J->form == 0) head_recurrent(J, q, k, v, J->gamma[h], si, y, so);
        else if (J->form == 1) head_parallel(J, q, k, v, J->gamma[h], si, y, so);
        else head_chunkwise(J, q, k, v, J->gamma[h], si, y, so);
    }
    return NULL;
}

static int run(int form, int B, int H, int L, int dk, int dv, int C,
               const double* q, const double* k, const double* v,
               const double* gamma, const double* state_in, double* y,
               double* state_out, int nthreads) {
    if (B < 0 || H < 1 || L < 0 || dk < 1 || dv < 1 || !gamma) return -1;
    if (form == 2 && C < 1) return -1;
    if (L > 0 && (!q || !k || !v || !y)) return -1;
    for (int h = 0; h < H; ++h)
        if (!(gamma[h] >= 0.0 && gamma[h] <= 1.0)) return -1;
    job_t J = {form, B, H, L, dk, dv, C, q, k, v, gamma, state_in, y, state_out, 0};
    pthread_mutex_init(&J.lock, NULL);
    if (nthreads <= 0) nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (nthreads > B * H) nthreads = B * H;
    if (nthreads < 1) nthreads = 1;
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
    for (int t = 1; t < nthreads; ++t) pthread_create(&th[t], NULL, worker, &J);
    worker(&J);
    for (int t = 1; t < nthreads; ++t) pthread_join(th[t], NULL);
    free(th);
    pthread_mutex_destroy(&J.lock);
    return 0;
}

int oracle_recurrent(int B, int H, int L, int dk, int dv, const double* q,
                     const double* k, const double* v, const double* gamma,
                     const double* state_in, double* y, double* state_out,
                     int nthreads) {
    return run(0, B, H, L, dk, dv, 1, q, k, v, gamma, state_in, y, state_out, nthreads);
}

int oracle_parallel(int B, int H, int L, int dk, int dv, const double* q,
                    const double* k, const double* v, const double* gamma,
                    const double* state_in, double* y, double* state_out,
                    int nthreads) {
    return run(1, B, H, L, dk, dv, 1, q, k, v, gamma, state_in, y, state_out, nthreads);
}

int oracle_chunkwise(int B, int H, int L, int dk, int dv, int C, const double* q,
                     const double* k, const double* v, const double* gamma,
                     const double* state_in, double* y, double* state_out,
                     int nthreads) {
    return run(2, B, H, L, dk, dv, C, q, k, v, gamma, state_in, y, state_out, nthreads);
}

/*
 * Group normalisation of the retention output, one group per head.  Source:
 * the author responses on paperhub.cn ("Retentive Network: A Successor to
 * Transformer for Large Language Models", reply comparing GroupNorm with
 * LayerNorm): heads carry different statistics, so each head is normalised on
 * its own.  Readings (the page gives no formula, eps or affine): for every
 * (b, h, n) the dv values of y_n of head h are taken as one group,
 *     mean = (1/dv) sum_c y_c ,   var = (1/dv) sum_c (y_c - mean)^2
 *     out_c = (y_c - mean) / sqrt(var + eps) * w[h*dv + c] + bias[h*dv + c]
 * with w and bias optional (NULL: 1 and 0).  Two passes in fp64.
 * Layout: y, out [B][H][L][dv]; w, bias [H*dv].  out may alias y.
 */
int oracle_groupnorm(int B, int H, int L, int dv, const double* y, double eps,
                     const double* w, const double* bias, double* out) {
    if (B < 0 || H < 1 || L < 0 || dv < 1 || !y || !out || !(eps >= 0.0)) return -1;
    for (long r = 0; r < (long)B * H * L; ++r) {
        const int h = (int)((r / L) % H);
        const double* yr = y + r * dv;
        double* o = out + r * dv;
        double mean = 0.0;
        for (int c = 0; c < dv; ++c) mean += yr[c];
        mean /= dv;
        double var = 0.0;
        for (int c = 0; c < dv; ++c) var += (yr[c] - mean) * (yr[c] - mean);
        var /= dv;
        const double inv = 1.0 / sqrt(var + eps);
        for (int c = 0; c < dv; ++c) {
            const double z = (yr[c] - mean) * inv;
            o[c] = z * (w ? w[(size_t)h * dv + c] : 1.0) + (bias ? bias[(size_t)h * dv + c] : 0.0);
        }
    }
    return 0;
}

/*
 * Gradients of the parallel form (no carried state) for an upstream gradient
 * dy [B][H][L][dv]: with y_n = sum_{m<=n} gamma^(n-m) (q_n . k_m) v_m (page
 * "Retentive Networks -- Microsoft Propone l'Alternativa Architetturale ai
 * Transformer", section "Il meccanismo: Multi-Scale Retention"), the chain
 * rule on each term of the double sum gives, for m <= n and w = gamma^(n-m),
 *     dq_n += w (dy_n . v_m) k_m
 *     dk_m += w (dy_n . v_m) q_n
 *     dv_m += w (q_n . k_m) dy_n
 * The pages give no backward pass; this is the derivative of their definition.
 * Outputs dq, dk [B][H][L][dk], dv [B][H][L][dv] are overwritten.
 */
int oracle_parallel_backward(int B, int H, int L, int dk, int dv, const double* q, const double* k,
                             const double* v, const double* gamma, const double* dy, double* dq,
                             double* dkk, double* dvv) {
    if (B < 0 || H < 1 || L < 0 || dk < 1 || dv < 1 || !q || !k || !v || !gamma || !dy || !dq || !dkk || !dvv)
        return -1;
    memset(dq, 0, sizeof(double) * (size_t)B * H * L * dk);
    memset(dkk, 0, sizeof(double) * (size_t)B * H * L * dk);
    memset(dvv, 0, sizeof(double) * (size_t)B * H * L * dv);
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            const size_t ok = ((size_t)b * H + h) * L * dk, ov = ((size_t)b * H + h) * L * dv;
            const double g = gamma[h];
            for (int n = 0; n < L; ++n)
                for (int m = 0; m <= n; ++m) {
                    const double w = gpow(g, n - m);
                    double qk = 0.0, dyv = 0.0;
                    for (int i = 0; i < dk; ++i) qk += q[ok + (size_t)n * dk + i] * k[ok + (size_t)m * dk + i];
                    for (int j = 0; j < dv; ++j) dyv += dy[ov + (size_t)n * dv + j] * v[ov + (size_t)m * dv + j];
                    for (int i = 0; i < dk; ++i) {
                        dq[ok + (size_t)n * dk + i] += w * dyv * k[ok + (size_t)m * dk + i];
                        dkk[ok + (size_t)m * dk + i] += w * dyv * q[ok + (size_t)n * dk + i];
                    }
                    for (int j = 0; j < dv; ++j) dvv[ov + (size_t)m * dv + j] += w * qk * dy[ov + (size_t)n * dv + j];
                }
        }
    return 0;
}

/*
 * The terms a carried state adds to the gradients.  With state_in S0 and
 * state_out S_out (same page and section: the recurrence S_n = gamma S_{n-1} +
 * k_n^T v_n started from S0), unrolling gives
 *     y_n   gains  gamma^(n+1) q_n S0
 *     S_out =      gamma^L S0 + sum_m gamma^(L-1-m) k_m^T v_m
 * and for upstream gradients dy [B][H][L][dv] and dS_out [B][H][dk][dv]:
 *     dq_n  += gamma^(n+1) dy_n S0^T
 *     dk_m  += gamma^(L-1-m) v_m dS_out^T
 *     dv_m  += gamma^(L-1-m) k_m dS_out
 *     dS0    = gamma^L dS_out + sum_n gamma^(n+1) q_n^T dy_n
 * s0 or dsout may be null (zero).  dq, dk, dv are ADDED to (call
 * oracle_parallel_backward first for the terms without state); ds0 may be
 * null, else it is overwritten.
 */
int oracle_state_backward(int B, int H, int L, int dk, int dv, const double* q, const double* k,
                          const double* v, const double* gamma, const double* dy, const double* s0,
                          const double* dsout, double* dq, double* dkk, double* dvv, double* ds0) {
    if (B < 0 || H < 1 || L < 0 || dk < 1 || dv < 1 || !q || !k || !v || !gamma || !dy || !dq || !dkk || !dvv)
        return -1;
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            const size_t ok = ((size_t)b * H + h) * L * dk, ov = ((size_t)b * H + h) * L * dv;
            const size_t os = ((size_t)b * H + h) * dk * dv;
            const double g = gamma[h];
            for (int n = 0; n < L; ++n) {
                const double wq = gpow(g, (long)n + 1), ws = gpow(g, (long)L - 1 - n);
                for (int i = 0; i < dk; ++i)
                    for (int j = 0; j < dv; ++j) {
                        if (s0) dq[ok + (size_t)n * dk + i] += wq * dy[ov + (size_t)n * dv + j] * s0[os + (size_t)i * dv + j];
                        if (dsout) {
                            const double d = dsout[os + (size_t)i * dv + j];
                            dkk[ok + (size_t)n * dk + i] += ws * v[ov + (size_t)n * dv + j] * d;
                            dvv[ov + (size_t)n * dv + j] += ws * k[ok + (size_t)n * dk + i] * d;
                        }
                    }
            }
            if (!ds0) continue;
            const double gL = gpow(g, (long)L);
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j) {
                    double acc = dsout ? gL * dsout[os + (size_t)i * dv + j] : 0.0;
                    for (int n = 0; n < L; ++n)
                        acc += gpow(g, (long)n + 1) * q[ok + (size_t)n * dk + i] * dy[ov + (size_t)n * dv + j];
                    ds0[os + (size_t)i * dv + j] = acc;
                }
        }
    return 0;
}

/*
 * Output gate of the retention layer.  The author responses on paperhub.cn
 * ("Retentive Network: A Successor to Transformer ...", reply on the
 * "transformer without softmax" remark) name gated multi-scale retention next
 * to group normalisation but give no formula.  Reading: the gate multiplies
 * the normalised output elementwise by an activation of a gate input g of the
 * same shape,
 *     out = act(g) * z,   act(x) = x (act 0), x sigmoid(x) (act 1, swish),
 *                         sigmoid(x) (act 2),  sigmoid(x) = 1 / (1 + exp(-x)).
 * n values; out may alias z.
 */
int oracle_gate(long n, const double* z, const double* g, int act, double* out) {
    if (n < 0 || !z || !g || !out || act < 0 || act > 2) return -1;
    for (long i = 0; i < n; ++i) {
        const double x = g[i];
        const double s = 1.0 / (1.0 + exp(-x));
        const double a = act == 0 ? x : (act == 1 ? x * s : s);
        out[i] = a * z[i];
    }
    return 0;
}
