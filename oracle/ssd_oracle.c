/*
 * ssd_oracle.c -- plain, slow, float64 CPU oracle of the Mamba-2 SSD layer core.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls
 * this file: only the test-suite, the smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no code, header, table or helper with the
 * CUDA library; it is written from the method's definition, not from kernels.
 *
 * What it computes (per batch b and head h, state of size N x P):
 *
 *   dt_t = softplus(dt_raw[t,h] + dt_bias[h])
 *   h_t  = exp(dt_t * A[h]) * h_{t-1} + dt_t * B_t x_t^T          (N x P)
 *   y_t  = C_t^T h_t + D[h] * x_t                                  (P)
 *
 * Sources (titles of the pages the method is described on):
 *  - "Mamba3" (Telegram post, ai_machinelearning_big_data), paragraph on
 *    Mamba-2: the state transition matrix is a scalar times the identity; and
 *    section "New discretisation scheme": Mamba-1/2 discretise with a mix of
 *    ZOH (here exp(dt*A) on the state) and Euler (here dt*B on the input).
 *  - "Mamba-3 : SSM optimise inference" (call-informatique.fr), section
 *    "Du training-first a l'inference-first": transition reduced to a scalar
 *    times identity.
 *  - "Mamba-2 vs Transformers / SSD" (axiomlogica.com), section "Mamba-2 and
 *    the SSD paper: what changed in practice": the layer is a semiseparable
 *    matrix; SSM recurrence and masked attention are two contraction orders of
 *    it; the blocked algorithm splits the sequence into chunks processed in
 *    parallel and recombines the per-chunk states.
 *
 * Readings where the pages are silent:
 *  - y_t uses the state AFTER the token-t update (so the diagonal of the
 *    semiseparable mask is exp(0) = 1).
 *  - softplus(z) = log(1 + e^z), evaluated exactly (no threshold).
 *  - head h reads group g = h / (H / G) of B and C (contiguous head blocks).
 *  - D and dt_bias are one scalar per head; NULL means zero.
 *  - init_state NULL means a zero initial state.
 *
 * Layouts (row-major, last index fastest):
 *   x, y [b][L][H][P]; dt_raw [b][L][H]; B, C [b][L][G][N];
 *   dt_bias, A, D [H]; init_state, final_state [b][H][N][P].
 *   Decode step: x, y [b][H][P]; dt_raw [b][H]; B, C [b][G][N]; state [b][H][N][P].
 *   MIMO decode step (rank R): x, y [b][H][R][P]; B, C [b][G][R][N].
 *
 * All functions return 0 on success, -1 on invalid arguments.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* softplus(z) = log(1 + exp(z)), written so that it neither overflows for
 * large z nor loses digits for very negative z. */
static double sp(double z) { return fmax(z, 0.0) + log1p(exp(-fabs(z))); }

double oracle_softplus(double z) { return sp(z); }

/* Round a double to the nearest bfloat16 value (8 significant bits, 8-bit
 * exponent like IEEE binary32), ties to even.  Used only where the API stores
 * a state in bf16 (the reading of "the oracle runs on the bf16-rounded
 * values" for a bf16 decode state). */
double oracle_round_bf16(double v) {
    if (v == 0.0 || !isfinite(v)) return v;
    int e2;
    (void)frexp(v, &e2);           /* |v| in [2^(e2-1), 2^e2) */
    int e = e2 - 1;
    if (e < -126) e = -126;        /* subnormal range: fixed spacing 2^-133 */
    double spacing = ldexp(1.0, e - 7);
    double q = nearbyint(v / spacing);   /* default mode: ties to even */
    double r = q * spacing;
    const double bf16_max = ldexp(255.0 / 128.0, 127);  /* (2 - 2^-7) * 2^127 */
    if (fabs(r) > bf16_max) return v > 0 ? INFINITY : -INFINITY;
    return r;
}

/* Element-wise oracle_round_bf16 over an array (out may equal in). */
void oracle_round_bf16_array(const double* in, double* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_round_bf16(in[i]);
}

static int set_threads(int nthreads) {
#ifdef _OPENMP
    if (nthreads > 0) return nthreads;
    return omp_get_max_threads();
#else
    (void)nthreads;
    return 1;
#endif
}

int oracle_num_threads(void) { return set_threads(0); }

static int check_dims(int64_t b, int64_t L, int64_t H, int64_t P, int64_t N, int64_t G) {
    if (b <= 0 || L < 0 || H <= 0 || P <= 0 || N <= 0 || G <= 0) return -1;
    if (H % G != 0) return -1;
    return 0;
}

/* ------------------------------------------------------------------------ */
/* 1. Sequential recurrence: the definition itself.                          */
/* ------------------------------------------------------------------------ */
int oracle_ssd_recurrent(int64_t batch, int64_t seqlen, int64_t nheads, int64_t headdim,
                         int64_t dstate, int64_t ngroups,
                         const double* x, const double* dt_raw, const double* dt_bias,
                         const double* A, const double* B, const double* C, const double* D,
                         const double* init_state, double* y, double* final_state,
                         int nthreads) {
    if (check_dims(batch, seqlen, nheads, headdim, dstate, ngroups)) return -1;
    if (!x || !dt_raw || !A || !B || !C) return -1;
    const int64_t H = nheads, P = headdim, N = dstate, G = ngroups, L = seqlen;
    const int64_t heads_per_group = H / G;
    const int nt = set_threads(nthreads);
    int64_t pair;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nt)
    for (pair = 0; pair < batch * H; ++pair) {
        const int64_t b = pair / H, h = pair % H, g = h / heads_per_group;
        double* st = (double*)malloc(sizeof(double) * N * P);
        if (init_state) memcpy(st, init_state + (b * H + h) * N * P, sizeof(double) * N * P);
        else memset(st, 0, sizeof(double) * N * P);
        const double bias = dt_bias ? dt_bias[h] : 0.0;
        const double d_skip = D ? D[h] : 0.0;
        for (int64_t t = 0; t < L; ++t) {
            const double dt = sp(dt_raw[(b * L + t) * H + h] + bias);
            const double decay = exp(dt * A[h]);
            const double* xt = x + ((b * L + t) * H + h) * P;
            const double* Bt = B + ((b * L + t) * G + g) * N;
            const double* Ct = C + ((b * L + t) * G + g) * N;
            /* h_t = decay * h_{t-1} + dt * B_t x_t^T */
            for (int64_t n = 0; n < N; ++n) {
                const double coef = dt * Bt[n];
                double* row = st + n * P;
                for (int64_t p = 0; p < P; ++p) row[p] = decay * row[p] + coef * xt[p];
            }
            /* y_t = C_t^T h_t + D x_t */
            if (y) {
                double* yt = y + ((b * L + t) * H + h) * P;
                for (int64_t p = 0; p < P; ++p) {
                    double acc = 0.0;
                    for (int64_t n = 0; n < N; ++n) acc += Ct[n] * st[n * P + p];
                    yt[p] = acc + d_skip * xt[p];
                }
            }
        }
        if (final_state) memcpy(final_state + (b * H + h) * N * P, st, sizeof(double) * N * P);
        free(st);
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* 2. Quadratic ("masked attention") form of the same semiseparable matrix:  */
/*    y = (Lmask o C B^T)(dt x) + D x + exp(cs_i) C_i^T h0,                  */
/*    Lmask[i][j] = exp(cs_i - cs_j) for j <= i, else 0,                     */
/*    cs_i = sum_{k<=i} dt_k A  (inclusive).                                 */
/*    final_state = exp(cs_{L-1}) h0 + sum_j exp(cs_{L-1}-cs_j) dt_j B_j x_j^T */
/* ------------------------------------------------------------------------ */
int oracle_ssd_quadratic(int64_t batch, int64_t seqlen, int64_t nheads, int64_t headdim,
                         int64_t dstate, int64_t ngroups,
                         const double* x, const double* dt_raw, const double* dt_bias,
                         const double* A, const double* B, const double* C, const double* D,
                         const double* init_state, double* y, double* final_state,
                         int nthreads) {
    if (check_dims(batch, seqlen, nheads, headdim, dstate, ngroups)) return -1;
    if (!x || !dt_raw || !A || !B || !C) return -1;
    const int64_t H = nheads, P = headdim, N = dstate, G = ngroups, L = seqlen;
    const int64_t heads_per_group = H / G;
    const int nt = set_threads(nthreads);
    int64_t pair;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nt)
    for (pair = 0; pair < batch * H; ++pair) {
        const int64_t b = pair / H, h = pair % H, g = h / heads_per_group;
        const double bias = dt_bias ? dt_bias[h] : 0.0;
        const double d_skip = D ? D[h] : 0.0;
        double* dt = (double*)malloc(sizeof(double) * (L + 1));
        double* cs = (double*)malloc(sizeof(double) * (L + 1));
        double run = 0.0;
        for (int64_t t = 0; t < L; ++t) {
            dt[t] = sp(dt_raw[(b * L + t) * H + h] + bias);
            run += dt[t] * A[h];
            cs[t] = run;
        }
        const double* h0 = init_state ? init_state + (b * H + h) * N * P : NULL;
        for (int64_t i = 0; y && i < L; ++i) {
            const double* Ci = C + ((b * L + i) * G + g) * N;
            double* yi = y + ((b * L + i) * H + h) * P;
            for (int64_t p = 0; p < P; ++p) yi[p] = 0.0;
            for (int64_t j = 0; j <= i; ++j) {
                const double* Bj = B + ((b * L + j) * G + g) * N;
                const double* xj = x + ((b * L + j) * H + h) * P;
                double cb = 0.0;
                for (int64_t n = 0; n < N; ++n) cb += Ci[n] * Bj[n];
                const double m = exp(cs[i] - cs[j]) * cb * dt[j];
                for (int64_t p = 0; p < P; ++p) yi[p] += m * xj[p];
            }
            if (h0) {
                const double e = exp(cs[i]);
                for (int64_t p = 0; p < P; ++p) {
                    double acc = 0.0;
                    for (int64_t n = 0; n < N; ++n) acc += Ci[n] * h0[n * P + p];
                    yi[p] += e * acc;
                }
            }
            const double* xi = x + ((b * L + i) * H + h) * P;
            for (int64_t p = 0; p < P; ++p) yi[p] += d_skip * xi[p];
        }
        if (final_state) {
            double* hf = final_state + (b * H + h) * N * P;
            const double last = L > 0 ? cs[L - 1] : 0.0;
            for (int64_t k = 0; k < N * P; ++k) hf[k] = h0 ? exp(last) * h0[k] : 0.0;
            for (int64_t j = 0; j < L; ++j) {
                const double w = exp(last - cs[j]) * dt[j];
                const double* Bj = B + ((b * L + j) * G + g) * N;
                const double* xj = x + ((b * L + j) * H + h) * P;
                for (int64_t n = 0; n < N; ++n)
                    for (int64_t p = 0; p < P; ++p) hf[n * P + p] += w * Bj[n] * xj[p];
            }
        }
        free(dt);
        free(cs);
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* 3. Chunked (blocked two-pass) restatement: the sequence is cut into       */
/*    chunks of `chunk` tokens (the last one may be shorter).  Per chunk:    */
/*    acs_l = chunk-local inclusive cumsum of dt*A;                          */
/*    intra-chunk quadratic block; chunk state                               */
/*    S_c = sum_s exp(acs_last - acs_s) dt_s B_s x_s^T;                      */
/*    state passing h_in[c+1] = exp(acs_last) h_in[c] + S_c (h_in[0] = h0);  */
/*    off-diagonal output exp(acs_l) C_l^T h_in[c].                          */
/* ------------------------------------------------------------------------ */
int oracle_ssd_chunked(int64_t batch, int64_t seqlen, int64_t nheads, int64_t headdim,
                       int64_t dstate, int64_t ngroups, int64_t chunk,
                       const double* x, const double* dt_raw, const double* dt_bias,
                       const double* A, const double* B, const double* C, const double* D,
                       const double* init_state, double* y, double* final_state,
                       int nthreads) {
    if (check_dims(batch, seqlen, nheads, headdim, dstate, ngroups)) return -1;
    if (chunk <= 0 || !x || !dt_raw || !A || !B || !C) return -1;
    const int64_t H = nheads, P = headdim, N = dstate, G = ngroups, L = seqlen, Q = chunk;
    const int64_t heads_per_group = H / G;
    const int64_t nchunks = (L + Q - 1) / Q;
    const int nt = set_threads(nthreads);
    int64_t pair;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nt)
    for (pair = 0; pair < batch * H; ++pair) {
        const int64_t b = pair / H, h = pair % H, g = h / heads_per_group;
        const double bias = dt_bias ? dt_bias[h] : 0.0;
        const double d_skip = D ? D[h] : 0.0;
        double* dt = (double*)malloc(sizeof(double) * (Q + 1));
        double* acs = (double*)malloc(sizeof(double) * (Q + 1));
        double* hin = (double*)malloc(sizeof(double) * N * P);   /* state entering the chunk */
        double* sc = (double*)malloc(sizeof(double) * N * P);    /* chunk's own state S_c */
        if (init_state) memcpy(hin, init_state + (b * H + h) * N * P, sizeof(double) * N * P);
        else memset(hin, 0, sizeof(double) * N * P);
        for (int64_t c = 0; c < nchunks; ++c) {
            const int64_t t0 = c * Q;
            const int64_t len = (t0 + Q <= L) ? Q : L - t0;
            double run = 0.0;
            for (int64_t l = 0; l < len; ++l) {
                dt[l] = sp(dt_raw[(b * L + t0 + l) * H + h] + bias);
                run += dt[l] * A[h];
                acs[l] = run;
            }
            /* outputs of the chunk: intra-chunk block + off-diagonal term + skip */
            for (int64_t l = 0; y && l < len; ++l) {
                const double* Cl = C + ((b * L + t0 + l) * G + g) * N;
                const double* xl = x + ((b * L + t0 + l) * H + h) * P;
                double* yl = y + ((b * L + t0 + l) * H + h) * P;
                for (int64_t p = 0; p < P; ++p) yl[p] = d_skip * xl[p];
                for (int64_t s = 0; s <= l; ++s) {
                    const double* Bs = B + ((b * L + t0 + s) * G + g) * N;
                    const double* xs = x + ((b * L + t0 + s) * H + h) * P;
                    double cb = 0.0;
                    for (int64_t n = 0; n < N; ++n) cb += Cl[n] * Bs[n];
                    const double m = cb * exp(acs[l] - acs[s]) * dt[s];
                    for (int64_t p = 0; p < P; ++p) yl[p] += m * xs[p];
                }
                const double e = exp(acs[l]);
                for (int64_t p = 0; p < P; ++p) {
                    double acc = 0.0;
                    for (int64_t n = 0; n < N; ++n) acc += Cl[n] * hin[n * P + p];
                    yl[p] += e * acc;
                }
            }
            /* chunk state S_c */
            memset(sc, 0, sizeof(double) * N * P);
            for (int64_t s = 0; s < len; ++s) {
                const double w = exp(acs[len - 1] - acs[s]) * dt[s];
                const double* Bs = B + ((b * L + t0 + s) * G + g) * N;
                const double* xs = x + ((b * L + t0 + s) * H + h) * P;
                for (int64_t n = 0; n < N; ++n)
                    for (int64_t p = 0; p < P; ++p) sc[n * P + p] += w * Bs[n] * xs[p];
            }
            /* state passing to the next chunk */
            const double chunk_decay = exp(acs[len - 1]);
            for (int64_t k = 0; k < N * P; ++k) hin[k] = chunk_decay * hin[k] + sc[k];
        }
        if (final_state) memcpy(final_state + (b * H + h) * N * P, hin, sizeof(double) * N * P);
        free(dt);
        free(acs);
        free(hin);
        free(sc);
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* 4. One decode step (recurrent mode, one token per sequence), in place on  */
/*    the state.  If round_state_bf16 != 0 the stored state is rounded to    */
/*    bf16 after the update (the API's bf16 state storage); y is taken from  */
/*    the unrounded float64 update.                                          */
/* ------------------------------------------------------------------------ */
int oracle_ssd_decode_step(int64_t batch, int64_t nheads, int64_t headdim, int64_t dstate,
                           int64_t ngroups, double* state, const double* x,
                           const double* dt_raw, const double* dt_bias, const double* A,
                           const double* B, const double* C, const double* D, double* y,
                           int round_state_bf16, int nthreads) {
    if (check_dims(batch, 1, nheads, headdim, dstate, ngroups)) return -1;
    if (!state || !x || !dt_raw || !A || !B || !C) return -1;
    const int64_t H = nheads, P = headdim, N = dstate, G = ngroups;
    const int64_t heads_per_group = H / G;
    const int nt = set_threads(nthreads);
    int64_t pair;
#pragma omp parallel for schedule(static) num_threads(nt)
    for (pair = 0; pair < batch * H; ++pair) {
        const int64_t b = pair / H, h = pair % H, g = h / heads_per_group;
        const double dt = sp(dt_raw[b * H + h] + (dt_bias ? dt_bias[h] : 0.0));
        const double decay = exp(dt * A[h]);
        const double* xt = x + (b * H + h) * P;
        const double* Bt = B + (b * G + g) * N;
        const double* Ct = C + (b * G + g) * N;
        double* st = state + (b * H + h) * N * P;
        double* yt = y ? y + (b * H + h) * P : NULL;
        if (yt) for (int64_t p = 0; p < P; ++p) yt[p] = (D ? D[h] : 0.0) * xt[p];
        for (int64_t n = 0; n < N; ++n) {
            for (int64_t p = 0; p < P; ++p) {
                const double v = decay * st[n * P + p] + dt * Bt[n] * xt[p];
                if (yt) yt[p] += Ct[n] * v;
                st[n * P + p] = round_state_bf16 ? oracle_round_bf16(v) : v;
            }
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* 5. One MIMO decode step: B, C widened to rank R ("Mamba3" (Telegram post), */
/*    section on the switch from SISO to MIMO: outer products become matrix  */
/*    products, the state size stays the same; "Mamba-3 : SSM optimise       */
/*    inference", section "Mode MIMO": several SSMs in parallel with extended */
/*    B and C matrices).  Reading, per (b, h), with X_t = [x_0 .. x_{R-1}]:   */
/*      h_t = exp(dt A) h_{t-1} + dt * sum_r B_r x_r^T                        */
/*      y_r = C_r^T h_t + D x_r          (r = 0 .. R-1)                       */
/*    Layouts: x, y [b][H][R][P]; dt_raw [b][H]; B, C [b][G][R][N].  R = 1 is */
/*    the decode step above.  round_state_bf16 as there.                      */
/* ------------------------------------------------------------------------ */
int oracle_ssd_decode_step_mimo(int64_t batch, int64_t nheads, int64_t headdim, int64_t dstate,
                                int64_t ngroups, int64_t rank, double* state, const double* x,
                                const double* dt_raw, const double* dt_bias, const double* A,
                                const double* B, const double* C, const double* D, double* y,
                                int round_state_bf16, int nthreads) {
    if (check_dims(batch, 1, nheads, headdim, dstate, ngroups) || rank < 1) return -1;
    if (!state || !x || !dt_raw || !A || !B || !C) return -1;
    const int64_t H = nheads, P = headdim, N = dstate, G = ngroups, R = rank;
    const int64_t heads_per_group = H / G;
    const int nt = set_threads(nthreads);
    int64_t pair;
#pragma omp parallel for schedule(static) num_threads(nt)
    for (pair = 0; pair < batch * H; ++pair) {
        const int64_t b = pair / H, h = pair % H, g = h / heads_per_group;
        const double dt = sp(dt_raw[b * H + h] + (dt_bias ? dt_bias[h] : 0.0));
        const double decay = exp(dt * A[h]);
        const double* Xt = x + (b * H + h) * R * P;          /* [R][P] */
        const double* Bt = B + (b * G + g) * R * N;          /* [R][N] */
        const double* Ct = C + (b * G + g) * R * N;
        double* st = state + (b * H + h) * N * P;
        double* yt = y ? y + (b * H + h) * R * P : NULL;
        if (yt)
            for (int64_t r = 0; r < R; ++r)
                for (int64_t p = 0; p < P; ++p) yt[r * P + p] = (D ? D[h] : 0.0) * Xt[r * P + p];
        for (int64_t n = 0; n < N; ++n) {
            for (int64_t p = 0; p < P; ++p) {
                double in = 0.0;                              /* sum_r B_r[n] x_r[p] */
                for (int64_t r = 0; r < R; ++r) in += Bt[r * N + n] * Xt[r * P + p];
                const double v = decay * st[n * P + p] + dt * in;
                if (yt)
                    for (int64_t r = 0; r < R; ++r) yt[r * P + p] += Ct[r * N + n] * v;
                st[n * P + p] = round_state_bf16 ? oracle_round_bf16(v) : v;
            }
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* 6. Backward pass: reverse-mode gradients of the sequential recurrence.    */
/* ------------------------------------------------------------------------ */
/* The pages only say that end-to-end training also needs the backward pass
 * ("Mamba-3 : SSM optimise inference", opening paragraph); what it computes is
 * fixed by the forward definition above.  For the scalar loss
 *     loss = sum_t <dy_t, y_t> + <dfinal, h_{L-1}>
 * the adjoint of the state, G_t = d loss / d h_t (N x P), obeys
 *     G_{L-1} = dfinal + C_{L-1} dy_{L-1}^T,
 *     G_t     = C_t dy_t^T + exp(dt_{t+1} A) G_{t+1},
 * and every gradient is a local product at token t (with hp = h_{t-1}):
 *     dx_t   = dt_t B_t^T G_t + D dy_t
 *     dB_t  += dt_t G_t x_t                 (summed over the heads of a group)
 *     dC_t  += h_t dy_t                     (same)
 *     d(dt A)_t = exp(dt_t A) <G_t, hp>
 *     d dt_t = <G_t, B_t x_t^T> + A d(dt A)_t
 *     d dt_raw_t = d dt_t * sigmoid(dt_raw_t + dt_bias)   (softplus' = sigmoid)
 *     dA += dt_t d(dt A)_t;  d dt_bias += d dt_raw_t;  dD += <dy_t, x_t>
 *     d init_state = exp(dt_0 A) G_0.
 * The states h_t are not all kept: one every SEG tokens is, and each segment
 * is recomputed from its checkpoint during the reverse sweep.
 * dinit, ddt_bias and dD may be NULL (not computed); dfinal, init_state, D and
 * dt_bias may be NULL (zero). */
#define ORACLE_BWD_SEG 64

static void step_state(double* dst, const double* src, double decay, double dt, const double* Bt,
                       const double* xt, int64_t N, int64_t P) {
    for (int64_t n = 0; n < N; ++n)
        for (int64_t p = 0; p < P; ++p) dst[n * P + p] = decay * src[n * P + p] + dt * Bt[n] * xt[p];
}

int oracle_ssd_backward(int64_t batch, int64_t seqlen, int64_t nheads, int64_t headdim, int64_t dstate,
                        int64_t ngroups, const double* x, const double* dt_raw, const double* dt_bias,
                        const double* A, const double* B, const double* C, const double* D,
                        const double* init_state, const double* dy, const double* dfinal, double* dx,
                        double* ddt_raw, double* ddt_bias, double* dA, double* dB, double* dC, double* dD,
                        double* dinit, int nthreads) {
    if (check_dims(batch, seqlen, nheads, headdim, dstate, ngroups)) return -1;
    if (!x || !dt_raw || !A || !B || !C || !dy || !dx || !ddt_raw || !dA || !dB || !dC) return -1;
    const int64_t H = nheads, P = headdim, N = dstate, G = ngroups, L = seqlen, NP = N * P;
    const int64_t heads_per_group = H / G, S = ORACLE_BWD_SEG, nseg = (L + S - 1) / S;
    /* per-head dB, dC and per-(b, h) partial sums, reduced in a fixed order below */
    double* dBh = (double*)calloc((size_t)(batch * L * H * N) + 1, sizeof(double));
    double* dCh = (double*)calloc((size_t)(batch * L * H * N) + 1, sizeof(double));
    double* part = (double*)calloc((size_t)(3 * batch * H), sizeof(double));
    if (!dBh || !dCh || !part) { free(dBh); free(dCh); free(part); return -1; }
    const int nt = set_threads(nthreads);
    int64_t pair;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nt)
    for (pair = 0; pair < batch * H; ++pair) {
        const int64_t b = pair / H, h = pair % H, g = h / heads_per_group;
        const double bias = dt_bias ? dt_bias[h] : 0.0, d_skip = D ? D[h] : 0.0, Ah = A[h];
        double* ck = (double*)malloc(sizeof(double) * (size_t)((nseg + 1) * NP));   /* h before each segment */
        double* seg = (double*)malloc(sizeof(double) * (size_t)((S + 1) * NP));     /* h_{t0-1} .. h_{t1-1} */
        double* Gs = (double*)malloc(sizeof(double) * (size_t)NP);
        /* forward sweep: keep the state entering every segment */
        double* cur = seg;
        if (init_state) memcpy(cur, init_state + (b * H + h) * NP, sizeof(double) * NP);
        else memset(cur, 0, sizeof(double) * NP);
        for (int64_t t = 0; t < L; ++t) {
            if (t % S == 0) memcpy(ck + (t / S) * NP, cur, sizeof(double) * NP);
            const double dt = sp(dt_raw[(b * L + t) * H + h] + bias);
            step_state(seg + NP, cur, exp(dt * Ah), dt, B + ((b * L + t) * G + g) * N,
                       x + ((b * L + t) * H + h) * P, N, P);
            memcpy(cur, seg + NP, sizeof(double) * NP);
        }
        /* reverse sweep */
        if (dfinal) memcpy(Gs, dfinal + (b * H + h) * NP, sizeof(double) * NP);
        else memset(Gs, 0, sizeof(double) * NP);
        double sum_dA = 0.0, sum_dbias = 0.0, sum_dD = 0.0;
        for (int64_t k = nseg - 1; k >= 0; --k) {
            const int64_t t0 = k * S, t1 = (t0 + S < L) ? t0 + S : L;
            memcpy(seg, ck + k * NP, sizeof(double) * NP);
            for (int64_t t = t0; t < t1; ++t) {
                const double dt = sp(dt_raw[(b * L + t) * H + h] + bias);
                step_state(seg + (t - t0 + 1) * NP, seg + (t - t0) * NP, exp(dt * Ah), dt,
                           B + ((b * L + t) * G + g) * N, x + ((b * L + t) * H + h) * P, N, P);
            }
            for (int64_t t = t1 - 1; t >= t0; --t) {
                const double* hp = seg + (t - t0) * NP;       /* h_{t-1} */
                const double* hc = seg + (t - t0 + 1) * NP;   /* h_t */
                const double z = dt_raw[(b * L + t) * H + h] + bias;
                const double dt = sp(z), decay = exp(dt * Ah);
                const double* xt = x + ((b * L + t) * H + h) * P;
                const double* dyt = dy + ((b * L + t) * H + h) * P;
                const double* Bt = B + ((b * L + t) * G + g) * N;
                const double* Ct = C + ((b * L + t) * G + g) * N;
                /* y_t reads h_t: G_t gains C_t dy_t^T */
                for (int64_t n = 0; n < N; ++n)
                    for (int64_t p = 0; p < P; ++p) Gs[n * P + p] += Ct[n] * dyt[p];
                double* dxt = dx + ((b * L + t) * H + h) * P;
                for (int64_t p = 0; p < P; ++p) {
                    double acc = 0.0;
                    for (int64_t n = 0; n < N; ++n) acc += Bt[n] * Gs[n * P + p];
                    dxt[p] = dt * acc + d_skip * dyt[p];
                }
                double* dBt = dBh + ((b * L + t) * H + h) * N;
                double* dCt = dCh + ((b * L + t) * H + h) * N;
                double gbx = 0.0, gh = 0.0;
                for (int64_t n = 0; n < N; ++n) {
                    double gx = 0.0, hy = 0.0;
                    for (int64_t p = 0; p < P; ++p) {
                        gx += Gs[n * P + p] * xt[p];
                        hy += hc[n * P + p] * dyt[p];
                        gh += Gs[n * P + p] * hp[n * P + p];
                    }
                    dBt[n] = dt * gx;
                    dCt[n] = hy;
                    gbx += Bt[n] * gx;
                }
                const double dlogdecay = decay * gh;            /* d loss / d (dt_t A) */
                const double ddt = gbx + Ah * dlogdecay;
                const double dz = ddt / (1.0 + exp(-z));
                ddt_raw[(b * L + t) * H + h] = dz;
                sum_dA += dt * dlogdecay;
                sum_dbias += dz;
                for (int64_t p = 0; p < P; ++p) sum_dD += dyt[p] * xt[p];
                /* G_{t-1} part that flows through the transition */
                for (int64_t i = 0; i < NP; ++i) Gs[i] *= decay;
            }
        }
        if (dinit) memcpy(dinit + (b * H + h) * NP, Gs, sizeof(double) * NP);
        part[3 * pair + 0] = sum_dA;
        part[3 * pair + 1] = sum_dbias;
        part[3 * pair + 2] = sum_dD;
        free(ck);
        free(seg);
        free(Gs);
    }
    for (int64_t bt = 0; bt < batch * L; ++bt)
        for (int64_t g = 0; g < G; ++g)
            for (int64_t n = 0; n < N; ++n) {
                double sb = 0.0, sc = 0.0;
                for (int64_t j = 0; j < heads_per_group; ++j) {
                    const int64_t h = g * heads_per_group + j;
                    sb += dBh[(bt * H + h) * N + n];
                    sc += dCh[(bt * H + h) * N + n];
                }
                dB[(bt * G + g) * N + n] = sb;
                dC[(bt * G + g) * N + n] = sc;
            }
    for (int64_t h = 0; h < H; ++h) {
        double sa = 0.0, sbias = 0.0, sd = 0.0;
        for (int64_t b = 0; b < batch; ++b) {
            sa += part[3 * (b * H + h) + 0];
            sbias += part[3 * (b * H + h) + 1];
            sd += part[3 * (b * H + h) + 2];
        }
        dA[h] = sa;
        if (ddt_bias) ddt_bias[h] = sbias;
        if (dD) dD[h] = sd;
    }
    free(dBh);
    free(dCh);
    free(part);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* 7. Mamba-3 recurrence: exponential-trapezoidal input, rotational state.   */
/* ------------------------------------------------------------------------ */
/* "Mamba3" (Telegram post), section "New discretisation scheme": the integral
 * over a step is approximated from both ends of the interval with a learned
 * mixing coefficient, which makes the recurrence an implicit convolution on
 * the input.  Reading: over the step t-1 -> t of length dt_t the input term is
 *     dt_t [ (1 - lam_t) exp(dt_t A) B_{t-1} x_{t-1}^T + lam_t B_t x_t^T ],
 * the left end transported over the interval like the state (lam = 1 is
 * Mamba-2's Euler input; there is no input before the first token).
 * Same post, section on complex-valued SSMs, and "Mamba-3 : SSM optimise
 * inference", section "Etats complexes via RoPE": the complex transition is a
 * scaling and a rotation.  Reading: state rows (2k, 2k+1) form the pair k of
 * a complex state component and the transition of step t rotates every pair
 * by theta[t][g][k] (the same angle for every head of group g) and scales by
 * exp(dt_t A):
 *     h_t = exp(dt_t A) R(theta_t) (h_{t-1} + (1 - lam_t) dt_t B_{t-1} x_{t-1}^T)
 *           + lam_t dt_t B_t x_t^T,
 *     y_t = C_t^T h_t + D x_t,
 * R rotating (h[2k], h[2k+1]) by the angle counter-clockwise.  lam [b][L][H]
 * and theta [b][L][G][N/2] may each be NULL (lam = 1, theta = 0). */
int oracle_ssd_mamba3_recurrent(int64_t batch, int64_t seqlen, int64_t nheads, int64_t headdim,
                                int64_t dstate, int64_t ngroups, const double* x, const double* dt_raw,
                                const double* dt_bias, const double* A, const double* B, const double* C,
                                const double* D, const double* lam, const double* theta,
                                const double* init_state, double* y, double* final_state, int nthreads) {
    if (check_dims(batch, seqlen, nheads, headdim, dstate, ngroups)) return -1;
    if (!x || !dt_raw || !A || !B || !C) return -1;
    if (theta && dstate % 2 != 0) return -1;
    const int64_t H = nheads, P = headdim, N = dstate, G = ngroups, L = seqlen;
    const int64_t heads_per_group = H / G;
    const int nt = set_threads(nthreads);
    int64_t pair;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nt)
    for (pair = 0; pair < batch * H; ++pair) {
        const int64_t b = pair / H, h = pair % H, g = h / heads_per_group;
        double* st = (double*)malloc(sizeof(double) * N * P);
        if (init_state) memcpy(st, init_state + (b * H + h) * N * P, sizeof(double) * N * P);
        else memset(st, 0, sizeof(double) * N * P);
        const double bias = dt_bias ? dt_bias[h] : 0.0;
        const double d_skip = D ? D[h] : 0.0;
        for (int64_t t = 0; t < L; ++t) {
            const double dt = sp(dt_raw[(b * L + t) * H + h] + bias);
            const double decay = exp(dt * A[h]);
            const double mix = lam ? lam[(b * L + t) * H + h] : 1.0;
            const double* xt = x + ((b * L + t) * H + h) * P;
            const double* Bt = B + ((b * L + t) * G + g) * N;
            const double* Ct = C + ((b * L + t) * G + g) * N;
            /* left end of the interval: the previous token's input, weighted 1 - lam_t */
            if (t > 0) {
                const double* xp = x + ((b * L + t - 1) * H + h) * P;
                const double* Bp = B + ((b * L + t - 1) * G + g) * N;
                for (int64_t n = 0; n < N; ++n)
                    for (int64_t p = 0; p < P; ++p) st[n * P + p] += (1.0 - mix) * dt * Bp[n] * xp[p];
            }
            /* transition: rotate each pair of rows, then scale */
            if (theta) {
                for (int64_t k = 0; k < N / 2; ++k) {
                    const double ang = theta[((b * L + t) * G + g) * (N / 2) + k];
                    const double c = cos(ang), s = sin(ang);
                    double* r0 = st + (2 * k) * P;
                    double* r1 = st + (2 * k + 1) * P;
                    for (int64_t p = 0; p < P; ++p) {
                        const double u = r0[p], v = r1[p];
                        r0[p] = c * u - s * v;
                        r1[p] = s * u + c * v;
                    }
                }
            }
            for (int64_t i = 0; i < N * P; ++i) st[i] *= decay;
            /* right end: the current token's input, weighted lam_t */
            for (int64_t n = 0; n < N; ++n)
                for (int64_t p = 0; p < P; ++p) st[n * P + p] += mix * dt * Bt[n] * xt[p];
            if (y) {
                double* yt = y + ((b * L + t) * H + h) * P;
                for (int64_t p = 0; p < P; ++p) {
                    double acc = 0.0;
                    for (int64_t n = 0; n < N; ++n) acc += Ct[n] * st[n * P + p];
                    yt[p] = acc + d_skip * xt[p];
                }
            }
        }
        if (final_state) memcpy(final_state + (b * H + h) * N * P, st, sizeof(double) * N * P);
        free(st);
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* 8. Mamba-3 decode step and MIMO sequence (references for later kernels). */
/* ------------------------------------------------------------------------ */
/* One token of the Mamba-3 recurrence of section 7, in place.  The trapezoid's
 * left end needs the previous token's input, so the decode state is the SSM
 * state plus that token's B [b][G][N] and x [b][H][P] (zero before the first
 * token); both are replaced by this token's.  lam [b][H], theta [b][G][N/2]
 * nullable as in section 7. */
int oracle_ssd_mamba3_decode_step(int64_t batch, int64_t nheads, int64_t headdim, int64_t dstate,
                                  int64_t ngroups, double* state, double* B_prev, double* x_prev,
                                  const double* x, const double* dt_raw, const double* dt_bias, const double* A,
                                  const double* B, const double* C, const double* D, const double* lam,
                                  const double* theta, double* y, int nthreads) {
    if (check_dims(batch, 1, nheads, headdim, dstate, ngroups)) return -1;
    if (!state || !B_prev || !x_prev || !x || !dt_raw || !A || !B || !C || !y) return -1;
    if (theta && dstate % 2 != 0) return -1;
    const int64_t H = nheads, P = headdim, N = dstate, G = ngroups;
    const int64_t heads_per_group = H / G;
    const int nt = set_threads(nthreads);
    int64_t pair;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nt)
    for (pair = 0; pair < batch * H; ++pair) {
        const int64_t b = pair / H, h = pair % H, g = h / heads_per_group;
        double* st = state + (b * H + h) * N * P;
        const double dt = sp(dt_raw[b * H + h] + (dt_bias ? dt_bias[h] : 0.0));
        const double decay = exp(dt * A[h]);
        const double mix = lam ? lam[b * H + h] : 1.0;
        const double* xp = x_prev + (b * H + h) * P;
        const double* Bp = B_prev + (b * G + g) * N;
        const double* xt = x + (b * H + h) * P;
        const double* Bt = B + (b * G + g) * N;
        const double* Ct = C + (b * G + g) * N;
        for (int64_t n = 0; n < N; ++n)
            for (int64_t p = 0; p < P; ++p) st[n * P + p] += (1.0 - mix) * dt * Bp[n] * xp[p];
        if (theta) {
            for (int64_t k = 0; k < N / 2; ++k) {
                const double ang = theta[(b * G + g) * (N / 2) + k];
                const double c = cos(ang), s = sin(ang);
                for (int64_t p = 0; p < P; ++p) {
                    const double u = st[(2 * k) * P + p], v = st[(2 * k + 1) * P + p];
                    st[(2 * k) * P + p] = c * u - s * v;
                    st[(2 * k + 1) * P + p] = s * u + c * v;
                }
            }
        }
        for (int64_t i = 0; i < N * P; ++i) st[i] *= decay;
        for (int64_t n = 0; n < N; ++n)
            for (int64_t p = 0; p < P; ++p) st[n * P + p] += mix * dt * Bt[n] * xt[p];
        double* yt = y + (b * H + h) * P;
        for (int64_t p = 0; p < P; ++p) {
            double acc = 0.0;
            for (int64_t n = 0; n < N; ++n) acc += Ct[n] * st[n * P + p];
            yt[p] = acc + (D ? D[h] : 0.0) * xt[p];
        }
    }
    /* the previous-token buffers take this token's inputs (after every head has read them) */
    memcpy(x_prev, x, sizeof(double) * (size_t)(batch * H * P));
    memcpy(B_prev, B, sizeof(double) * (size_t)(batch * G * N));
    return 0;
}

/* A sequence of MIMO (rank-R) tokens: per token the step of
 * oracle_ssd_decode_step_mimo, h_t = exp(dt_t A) h_{t-1} + dt_t sum_r B_{t,r} x_{t,r}^T,
 * y_{t,r} = C_{t,r}^T h_t + D x_{t,r}.  x, y [b][L][H][R][P]; B, C [b][L][G][R][N]. */
int oracle_ssd_mimo_recurrent(int64_t batch, int64_t seqlen, int64_t nheads, int64_t headdim, int64_t dstate,
                              int64_t ngroups, int64_t rank, const double* x, const double* dt_raw,
                              const double* dt_bias, const double* A, const double* B, const double* C,
                              const double* D, const double* init_state, double* y, double* final_state,
                              int nthreads) {
    if (check_dims(batch, seqlen, nheads, headdim, dstate, ngroups) || rank < 1) return -1;
    if (!x || !dt_raw || !A || !B || !C || !y) return -1;
    const int64_t H = nheads, P = headdim, N = dstate, G = ngroups, L = seqlen, R = rank;
    const int64_t heads_per_group = H / G;
    const int nt = set_threads(nthreads);
    int64_t pair;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nt)
    for (pair = 0; pair < batch * H; ++pair) {
        const int64_t b = pair / H, h = pair % H, g = h / heads_per_group;
        double* st = (double*)malloc(sizeof(double) * N * P);
        if (init_state) memcpy(st, init_state + (b * H + h) * N * P, sizeof(double) * N * P);
        else memset(st, 0, sizeof(double) * N * P);
        for (int64_t t = 0; t < L; ++t) {
            const double dt = sp(dt_raw[(b * L + t) * H + h] + (dt_bias ? dt_bias[h] : 0.0));
            const double decay = exp(dt * A[h]);
            const double* Xt = x + ((b * L + t) * H + h) * R * P;
            const double* Bt = B + ((b * L + t) * G + g) * R * N;
            const double* Ct = C + ((b * L + t) * G + g) * R * N;
            for (int64_t n = 0; n < N; ++n)
                for (int64_t p = 0; p < P; ++p) {
                    double in = 0.0;
                    for (int64_t r = 0; r < R; ++r) in += Bt[r * N + n] * Xt[r * P + p];
                    st[n * P + p] = decay * st[n * P + p] + dt * in;
                }
            double* Yt = y + ((b * L + t) * H + h) * R * P;
            for (int64_t r = 0; r < R; ++r)
                for (int64_t p = 0; p < P; ++p) {
                    double acc = 0.0;
                    for (int64_t n = 0; n < N; ++n) acc += Ct[r * N + n] * st[n * P + p];
                    Yt[r * P + p] = acc + (D ? D[h] : 0.0) * Xt[r * P + p];
                }
        }
        if (final_state) memcpy(final_state + (b * H + h) * N * P, st, sizeof(double) * N * P);
        free(st);
    }
    return 0;
}
