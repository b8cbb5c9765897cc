/*
 * gdn_oracle.c -- plain, slow, fp64 CPU oracle for the gated delta rule.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call
 * this file; only the tests, the package's smoke check and the bench's CPU
 * baseline do.  It shares no code, header, table or helper with the CUDA
 * library.
 *
 * What it computes, and where the pages fix it:
 *
 *  - Gates.  NVIDIA Megatron-Core API docs, "core.ssm.ops.gdp.decode_prepare",
 *    module description and the `softplus` entry: beta = sigmoid(b),
 *    g = -exp(A_log) * softplus(a + dt_bias), softplus(x) = log1p(exp(x)),
 *    the identity when x > 20 (strict, as torch's F.softplus at beta = 1).
 *    Reading: a + dt_bias is one IEEE fp32 add; every transcendental is taken
 *    in fp64 and the result is rounded to fp32 once.
 *
 *  - Recurrence.  The gated delta rule
 *        S_t = exp(g_t) S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
 *        o_t = S_t q_t,
 *    carried here as h = S^T (K x V, key-major, the layout of h0 / h_T).
 *    Expanding the product gives, token by token:
 *        h <- exp(g_t) h;  u = v_t - h^T k_t;  h <- h + beta_t k_t u^T;
 *        o_t = scale * h^T q_t.
 *    ZzCompute (Helion hackathon gallery entry 11), items 2-4, describe the
 *    chunked form of this same map (64-token chunks); the oracle does not
 *    chunk at all, it walks every token in order.
 *
 *  - Short convolution.  ZzCompute item 1 ("Causal Conv1d -- Depthwise
 *    Causal Convolution"): every channel is convolved on its own with its
 *    past context, filter width W = 4, boundaries by masked loads rather
 *    than padding.  Written out per sequence and channel:
 *        y[t,c] = bias[c] + sum_{i<W} w[c,i] x[t-(W-1)+i, c],
 *    so w[c,W-1] weighs the current input; taps before the sequence start
 *    read the sequence's initial conv state (its W-1 previous inputs, oldest
 *    first) or zero.  SiLU (y * sigmoid(y)) is an option.  The one-token
 *    decode update shifts the same W-1 input window; a request whose state
 *    slot is -1 is padding: its output is zero and no state is touched
 *    (Megatron-Core "gdp_decode_prepare": "a -1 slot zeroes its conv output").
 *
 *  - GDP decode.  Megatron-Core "gdp_decode_prepare" (function entry and
 *    parameter list): the post-conv row x = [value | key | query] with sizes
 *    M*H*P, M*G*N, G*N; ba = [b (M*H) | a (H)]; key/query GQA-expanded from
 *    G groups to H heads; query only on the last Householder copy, decay only
 *    on the first; outputs [n, M, H, *].  The step then runs the recurrence
 *    above over the M copies of each request, starting from its state.
 *
 * Parity status per function (see the pins in tests/test_oracle_pins.py):
 *    oracle_softplus / oracle_gate_prep : pinned (torch's softplus/sigmoid,
 *                                         saturation, denormal tail)
 *    oracle_gdn_fwd                     : pinned (brute-force transition
 *                                         products, closed forms, invariants)
 *    oracle_gdp_decode_prepare          : part boundaries, copy placement and
 *                                         GQA sharing pinned by properties;
 *                                         the order inside each part is a
 *                                         reading -- parity unpinned there.
 *    oracle_gdp_decode_step             : recurrence pinned through
 *                                         oracle_gdn_fwd (same token step);
 *                                         layout as decode_prepare.
 *    oracle_conv1d_fwd / _update        : pinned (impulse response, numpy's
 *                                         convolve, constant input, token-
 *                                         by-token update = whole sequence);
 *                                         the tap order w[c,W-1] = current
 *                                         input is a reading.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

/* ------------------------------------------------------------------ gates */

/* softplus at beta = 1, threshold 20, in fp64 on an fp32 argument. */
static double sp_f64(float x) {
    double xd = (double)x;
    return (xd > 20.0) ? xd : log1p(exp(xd));
}

void oracle_softplus(const float* x, int64_t n, double* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = sp_f64(x[i]);
}

static float gate_g(float a, float dt_bias, float A_log) {
    volatile float x = a + dt_bias; /* one IEEE fp32 add, no contraction */
    return (float)(-exp((double)A_log) * sp_f64(x));
}

static float gate_beta(float b) { return (float)(1.0 / (1.0 + exp(-(double)b))); }

/* a, b: [n_tok, H] (token stride a_stride / b_stride elements);
 * beta, g: [n_tok, H] contiguous. */
void oracle_gate_prep(const float* a, const float* b, int64_t n_tok, int H, int64_t a_stride,
                      int64_t b_stride, const float* A_log, const float* dt_bias, float* beta,
                      float* g) {
    for (int64_t t = 0; t < n_tok; ++t)
        for (int h = 0; h < H; ++h) {
            g[t * H + h] = gate_g(a[t * a_stride + h], dt_bias[h], A_log[h]);
            beta[t * H + h] = gate_beta(b[t * b_stride + h]);
        }
}

/* ------------------------------------------------------------- recurrence */

/* One token of the rule on the K x V state h (fp64, row-major [K][V]).
 * u is V doubles of scratch.  Returns nothing; o (V doubles) receives
 * scale * h^T q when q != NULL. */
static void token_step(double* h, int K, int V, const double* k, const double* v, double gt,
                       double bt, const double* q, double scale, double* u, double* o) {
    double e = exp(gt);
    for (int i = 0; i < K * V; ++i) h[i] *= e;
    for (int j = 0; j < V; ++j) u[j] = v[j];
    for (int i = 0; i < K; ++i) {
        double ki = k[i];
        const double* hr = h + (int64_t)i * V;
        for (int j = 0; j < V; ++j) u[j] -= hr[j] * ki;
    }
    for (int i = 0; i < K; ++i) {
        double c = bt * k[i];
        double* hr = h + (int64_t)i * V;
        for (int j = 0; j < V; ++j) hr[j] += c * u[j];
    }
    if (o) {
        for (int j = 0; j < V; ++j) o[j] = 0.0;
        for (int i = 0; i < K; ++i) {
            double qi = q[i];
            const double* hr = h + (int64_t)i * V;
            for (int j = 0; j < V; ++j) o[j] += hr[j] * qi;
        }
        for (int j = 0; j < V; ++j) o[j] *= scale;
    }
}

typedef struct {
    const float *q, *k, *v, *g, *beta, *h0;
    const int64_t* cu;
    int n_seq, H, K, V;
    double scale;
    double *o, *hT;
    int tid, nth;
} fwd_job;

static void* fwd_worker(void* arg) {
    fwd_job* J = (fwd_job*)arg;
    const int H = J->H, K = J->K, V = J->V;
    double* h = (double*)malloc(sizeof(double) * (size_t)K * V);
    double* u = (double*)malloc(sizeof(double) * V);
    double* kd = (double*)malloc(sizeof(double) * K);
    double* qd = (double*)malloc(sizeof(double) * K);
    double* vd = (double*)malloc(sizeof(double) * V);
    for (int64_t c = J->tid; c < (int64_t)J->n_seq * H; c += J->nth) {
        int s = (int)(c / H), hh = (int)(c % H);
        const size_t st = (size_t)K * V * ((size_t)s * H + hh);
        for (int i = 0; i < K * V; ++i) h[i] = J->h0 ? (double)J->h0[st + i] : 0.0;
        for (int64_t t = J->cu[s]; t < J->cu[s + 1]; ++t) {
            const int64_t row = t * H + hh;
            for (int i = 0; i < K; ++i) kd[i] = J->k[row * K + i];
            for (int i = 0; i < K; ++i) qd[i] = J->q[row * K + i];
            for (int j = 0; j < V; ++j) vd[j] = J->v[row * V + j];
            token_step(h, K, V, kd, vd, J->g[row], J->beta[row], qd, J->scale, u,
                       J->o + row * V);
        }
        if (J->hT)
            for (int i = 0; i < K * V; ++i) J->hT[st + i] = h[i];
    }
    free(h); free(u); free(kd); free(qd); free(vd);
    return NULL;
}

static int pick_threads(int want, int64_t work) {
    int n = want > 0 ? want : (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (n < 1) n = 1;
    if (n > work) n = (int)(work > 0 ? work : 1);
    return n;
}

/* Token-by-token fp64 recurrence over packed sequences.
 *   q, k  : [T_total, H, K]      v : [T_total, H, V]     (widened exactly to fp32)
 *   g, beta: [T_total, H]        h0: [n_seq, H, K, V] or NULL (zero state)
 *   cu    : [n_seq + 1] token offsets (dense B x T is cu = {0, T, 2T, ...})
 *   o     : [T_total, H, V] fp64 out;  hT : [n_seq, H, K, V] fp64 out or NULL.
 * Returns the number of threads used. */
int oracle_gdn_fwd(const float* q, const float* k, const float* v, const float* g,
                   const float* beta, const float* h0, const int64_t* cu, int n_seq, int H, int K,
                   int V, double scale, double* o, double* hT, int n_threads) {
    int nth = pick_threads(n_threads, (int64_t)n_seq * H);
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * nth);
    fwd_job* jobs = (fwd_job*)malloc(sizeof(fwd_job) * nth);
    for (int i = 0; i < nth; ++i) {
        fwd_job J = {q, k, v, g, beta, h0, cu, n_seq, H, K, V, scale, o, hT, i, nth};
        jobs[i] = J;
        pthread_create(&th[i], NULL, fwd_worker, &jobs[i]);
    }
    for (int i = 0; i < nth; ++i) pthread_join(th[i], NULL);
    free(th); free(jobs);
    return nth;
}

/* ------------------------------------------------------------- GDP decode */

static float bf16_to_f32(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* Split / GQA-expand / interleave / gate one decode step.
 *   x  : [n, x_n_stride] bf16 bits, each row [v: M*H*P | k: M*G*N | q: G*N]
 *   ba : [n, ba_n_stride] bf16 bits, each row [b: M*H | a: H]
 *   q, k: [n, M, H, N] bf16 bits;  v: [n, M, H, P] bf16 bits
 *   beta, g: [n, M, H] fp32.
 * Readings: inside each part the Householder copy is the outer index
 * ([M, H, P] for value, [M, G, N] for key, [M, H] for b); head h reads group
 * h / (H / G); query is placed on copy M-1 and is zero on the others; the
 * decay g is on copy 0 and zero on the others; beta is per copy. */
void oracle_gdp_decode_prepare(const uint16_t* x, int64_t x_n_stride, const uint16_t* ba,
                               int64_t ba_n_stride, const float* A_log, const float* dt_bias,
                               int n, int M, int H, int G, int P, int N, uint16_t* q, uint16_t* k,
                               uint16_t* v, float* beta, float* g) {
    const int hpg = H / G;
    const int64_t kbase = (int64_t)M * H * P, qbase = kbase + (int64_t)M * G * N;
    for (int r = 0; r < n; ++r) {
        const uint16_t* xr = x + (int64_t)r * x_n_stride;
        const uint16_t* br = ba + (int64_t)r * ba_n_stride;
        for (int m = 0; m < M; ++m)
            for (int h = 0; h < H; ++h) {
                const int grp = h / hpg;
                const int64_t o = ((int64_t)r * M + m) * H + h;
                for (int p = 0; p < P; ++p) v[o * P + p] = xr[((int64_t)m * H + h) * P + p];
                for (int i = 0; i < N; ++i) k[o * N + i] = xr[kbase + ((int64_t)m * G + grp) * N + i];
                for (int i = 0; i < N; ++i)
                    q[o * N + i] = (m == M - 1) ? xr[qbase + (int64_t)grp * N + i] : (uint16_t)0;
                beta[o] = gate_beta(bf16_to_f32(br[m * H + h]));
                g[o] = (m == 0) ? gate_g(bf16_to_f32(br[M * H + h]), dt_bias[h], A_log[h]) : 0.0f;
            }
    }
}

typedef struct {
    const uint16_t *q, *k, *v;
    const float *beta, *g, *state;
    int n, M, H, P, N, l2;
    double scale;
    double *state_out, *o;
    int tid, nth;
} dec_job;

static void l2n(double* x, int n) {
    double s = 0.0;
    for (int i = 0; i < n; ++i) s += x[i] * x[i];
    double r = 1.0 / sqrt(s + 1e-6);
    for (int i = 0; i < n; ++i) x[i] *= r;
}

static void* dec_worker(void* arg) {
    dec_job* J = (dec_job*)arg;
    const int N = J->N, P = J->P, H = J->H, M = J->M;
    double* h = (double*)malloc(sizeof(double) * (size_t)N * P);
    double* u = (double*)malloc(sizeof(double) * P);
    double* kd = (double*)malloc(sizeof(double) * N);
    double* qd = (double*)malloc(sizeof(double) * N);
    double* vd = (double*)malloc(sizeof(double) * P);
    for (int64_t c = J->tid; c < (int64_t)J->n * H; c += J->nth) {
        const int r = (int)(c / H), hh = (int)(c % H);
        const size_t st = (size_t)N * P * c;
        for (int i = 0; i < N * P; ++i) h[i] = J->state[st + i];
        for (int m = 0; m < M; ++m) {
            const int64_t o = ((int64_t)r * M + m) * H + hh;
            for (int i = 0; i < N; ++i) kd[i] = bf16_to_f32(J->k[o * N + i]);
            for (int i = 0; i < N; ++i) qd[i] = bf16_to_f32(J->q[o * N + i]);
            for (int p = 0; p < P; ++p) vd[p] = bf16_to_f32(J->v[o * P + p]);
            if (J->l2) { l2n(kd, N); l2n(qd, N); }
            token_step(h, N, P, kd, vd, J->g[o], J->beta[o], qd, J->scale, u,
                       (m == M - 1) ? J->o + c * P : NULL);
        }
        for (int i = 0; i < N * P; ++i) J->state_out[st + i] = h[i];
    }
    free(h); free(u); free(kd); free(qd); free(vd);
    return NULL;
}

/* Prepare, then run the rule over the M copies of each request from
 * state [n, H, N, P] (fp32 in).  state_out [n, H, N, P] and o [n, H, P] are
 * fp64 out; o is the output at the last copy.  With qk_l2norm, q and k of
 * every copy are divided by sqrt(sum x^2 + 1e-6) first (a reading: the pages
 * name no normalisation; the epsilon keeps the zero query rows at zero).
 * Returns the number of threads used. */
int oracle_gdp_decode_step(const uint16_t* x, int64_t x_n_stride, const uint16_t* ba,
                           int64_t ba_n_stride, const float* A_log, const float* dt_bias, int n,
                           int M, int H, int G, int P, int N, const float* state, double scale,
                           int qk_l2norm, double* state_out, double* o, int n_threads) {
    const size_t nq = (size_t)n * M * H;
    uint16_t* q = (uint16_t*)malloc(nq * N * 2);
    uint16_t* k = (uint16_t*)malloc(nq * N * 2);
    uint16_t* v = (uint16_t*)malloc(nq * P * 2);
    float* beta = (float*)malloc(nq * 4);
    float* g = (float*)malloc(nq * 4);
    oracle_gdp_decode_prepare(x, x_n_stride, ba, ba_n_stride, A_log, dt_bias, n, M, H, G, P, N, q,
                              k, v, beta, g);
    int nth = pick_threads(n_threads, (int64_t)n * H);
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * nth);
    dec_job* jobs = (dec_job*)malloc(sizeof(dec_job) * nth);
    for (int i = 0; i < nth; ++i) {
        dec_job J = {q, k, v, beta, g, state, n, M, H, P, N, qk_l2norm, scale, state_out, o, i, nth};
        jobs[i] = J;
        pthread_create(&th[i], NULL, dec_worker, &jobs[i]);
    }
    for (int i = 0; i < nth; ++i) pthread_join(th[i], NULL);
    free(th); free(jobs); free(q); free(k); free(v); free(beta); free(g);
    return nth;
}

/* ------------------------------------------------------------- short conv */

static double silu_f64(double y) { return y / (1.0 + exp(-y)); }

/* Causal depthwise conv1d over packed sequences (ZzCompute item 1).
 * x [rows, C] (fp32 values; bf16 inputs widened exactly), rows = cu[n_seq];
 * w [C, W]; bias [C] or NULL; init [n_seq, C, W-1] or NULL (zeros);
 * y [rows, C] fp64; final [n_seq, C, W-1] or NULL: the last W-1 inputs of each
 * sequence, oldest first (initial-state values where the sequence is shorter). */
void oracle_conv1d_fwd(const float* x, const float* w, const float* bias, int W,
                       const int64_t* cu, int n_seq, int C, const float* init, int act,
                       double* y, float* final_state) {
    const int H = W - 1;
    for (int s = 0; s < n_seq; ++s) {
        const int64_t t0 = cu[s], len = cu[s + 1] - cu[s];
        for (int c = 0; c < C; ++c) {
            /* input at sequence position tau (may be negative) */
#define XIN(tau) ((tau) >= 0 ? (double)x[(t0 + (tau)) * C + c] \
                             : (init ? (double)init[((int64_t)s * C + c) * H + (H + (tau))] : 0.0))
            for (int64_t t = 0; t < len; ++t) {
                double acc = bias ? (double)bias[c] : 0.0;
                for (int i = 0; i < W; ++i) acc += (double)w[(int64_t)c * W + i] * XIN(t - H + i);
                y[(t0 + t) * C + c] = act ? silu_f64(acc) : acc;
            }
            if (final_state)
                for (int j = 0; j < H; ++j)
                    final_state[((int64_t)s * C + c) * H + j] = (float)XIN(len - H + j);
#undef XIN
        }
    }
}

/* One-token update for n requests: x [n, C]; state [n_slots, C, W-1] in/out
 * (the W-1 previous inputs, oldest first); idx [n] slot per request, or NULL
 * for slot = request; a negative slot is padding (y = 0, no state change). */
void oracle_conv1d_update(const float* x, const float* w, const float* bias, int W,
                          float* state, const int32_t* idx, int n, int C, int act, double* y) {
    const int H = W - 1;
    for (int r = 0; r < n; ++r) {
        const int slot = idx ? idx[r] : r;
        for (int c = 0; c < C; ++c) {
            if (slot < 0) {
                y[(int64_t)r * C + c] = 0.0;
                continue;
            }
            float* st = state + ((int64_t)slot * C + c) * H;
            const double xin = (double)x[(int64_t)r * C + c];
            double acc = bias ? (double)bias[c] : 0.0;
            for (int i = 0; i < H; ++i) acc += (double)w[(int64_t)c * W + i] * (double)st[i];
            acc += (double)w[(int64_t)c * W + H] * xin;
            y[(int64_t)r * C + c] = act ? silu_f64(acc) : acc;
            for (int i = 0; i + 1 < H; ++i) st[i] = st[i + 1];
            if (H > 0) st[H - 1] = x[(int64_t)r * C + c];
        }
    }
}
