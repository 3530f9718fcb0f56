/*
 * ORACLE — test infrastructure only.  A plain, slow, obviously correct CPU
 * implementation of the ExpertsInt8 mixture-of-experts layer, in IEEE fp64
 * (fp32 where the method fixes fp32).  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load this library; the CUDA path shares no
 * code, header, table or helper with it.
 *
 * What it computes, and where that is defined:
 *   - oracle_quantize_rows: ExpertsInt8 weight quantization (Jamba-1.5 paper,
 *     §3.1 "ExpertsInt8": MoE/MLP weights are quantized to INT8 and stored in
 *     INT8, without calibration).  Readings of what the page leaves open:
 *     one fp32 scale per output channel (row of the [out][in] matrix),
 *     symmetric range [-127, 127], scale = amax / 127 in fp32 round-to-nearest,
 *     q = round-half-to-even of the exact quotient w / scale (taken in fp64,
 *     which decides every tie exactly for a bf16 w and an fp32 scale), and an
 *     all-zero row gets scale 1 and q = 0.
 *   - oracle_route: the MoE router (Jamba-1.5 paper, "Model Architecture":
 *     n = 16 experts, two of them serving every token).  Readings: logits
 *     z_e = sum_i x_i * Wr[e][i] (+ bias_e), softmax over all E experts,
 *     the K largest logits in descending order (equal logits: lower expert
 *     index first), weights = the softmax probabilities of the chosen experts,
 *     not renormalised.
 *   - oracle_moe_forward_bf16w: the same layer with unquantized bf16 weights (the comparator the
 *     Jamba-1.5 paper measures ExpertsInt8 against in §3.1), weights taken as their exact values.
 *   - oracle_moe_forward: y_t = sum_k w_tk * E_{e_tk}(x_t) with SwiGLU experts
 *     E_e(x) = W2_e (SiLU(W1_e x) * (W3_e x)) (GLU variants, Shazeer 2020,
 *     cited by the Jamba paper), where each weight is the dequantized value
 *     q * scale formed exactly in fp64 (Jamba-1.5 paper, §3.1: the int8 weights
 *     become BF16 values again for the arithmetic).  No intermediate rounding:
 *     the result is fp64.
 *   - oracle_quantize_rows_fp8, oracle_moe_forward_fp8: the FP8 (E4M3) layer the
 *     Jamba-1.5 paper compares ExpertsInt8 with (§3.1), per-channel weight scales and
 *     per-row dynamic activation scales (reading stated beside the functions).
 *   - oracle_mlp_forward: the dense MLP of the layers without MoE, whose weights
 *     ExpertsInt8 quantizes too (Jamba-1.5 paper, §3.1): the same SwiGLU block
 *     as one expert, every token with weight 1.
 *
 * Parity pins: every function here is checked by the `-m "not gpu"` tests
 * against exact rational arithmetic, closed forms, invariants and brute-force
 * special cases that do not reuse this code.
 *
 * Build: gcc -O2 -shared -fPIC -pthread oracle.c -lm   (no -ffast-math: the
 * rounding of every operation must be IEEE round-to-nearest-even).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

/* ---------------------------------------------------------------- helpers */

/* bf16 bit pattern -> the fp32 (hence fp64) value it denotes; exact. */
static float bf16_value(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

static int pick_threads(int threads, int64_t work_items) {
    if (threads <= 0) {
        long n = sysconf(_SC_NPROCESSORS_ONLN);
        threads = n > 0 ? (int)n : 1;
    }
    if (threads > 256) threads = 256;
    if (work_items < threads) threads = work_items > 0 ? (int)work_items : 1;
    return threads;
}

typedef void (*range_fn)(void* ctx, int64_t begin, int64_t end);

typedef struct {
    range_fn fn;
    void* ctx;
    int64_t begin, end;
} range_job;

static void* range_entry(void* p) {
    range_job* j = (range_job*)p;
    j->fn(j->ctx, j->begin, j->end);
    return NULL;
}

/* Run fn over [0, n) split into contiguous pieces on `threads` threads. */
static void parallel_for(int64_t n, int threads, range_fn fn, void* ctx) {
    threads = pick_threads(threads, n);
    range_job jobs[256];
    pthread_t tids[256];
    int64_t per = (n + threads - 1) / threads;
    for (int t = 0; t < threads; ++t) {
        int64_t b = per * t, e = b + per;
        if (b > n) b = n;
        if (e > n) e = n;
        jobs[t] = (range_job){fn, ctx, b, e};
    }
    for (int t = 1; t < threads; ++t) pthread_create(&tids[t], NULL, range_entry, &jobs[t]);
    range_entry(&jobs[0]);
    for (int t = 1; t < threads; ++t) pthread_join(tids[t], NULL);
}

/* ------------------------------------------------------------ quantization */

typedef struct {
    const uint16_t* w;
    int64_t cols;
    int8_t* q;
    float* s;
} quant_ctx;

/* One output channel: amax, scale = amax/127 (fp32), q = rne(w/scale) in fp64. */
static void quantize_row(const uint16_t* w, int64_t cols, int8_t* q, float* s) {
    float amax = 0.0f;
    for (int64_t i = 0; i < cols; ++i) {
        float a = fabsf(bf16_value(w[i]));
        if (a > amax) amax = a;
    }
    if (amax == 0.0f) {
        *s = 1.0f;
        memset(q, 0, (size_t)cols);
        return;
    }
    const float scale = amax / 127.0f; /* IEEE fp32 division, round to nearest even */
    *s = scale;
    for (int64_t i = 0; i < cols; ++i) {
        double r = nearbyint((double)bf16_value(w[i]) / (double)scale); /* default mode: ties to even */
        if (r > 127.0) r = 127.0;
        if (r < -127.0) r = -127.0;
        q[i] = (int8_t)r;
    }
}

static void quantize_range(void* p, int64_t b, int64_t e) {
    quant_ctx* c = (quant_ctx*)p;
    for (int64_t r = b; r < e; ++r) quantize_row(c->w + r * c->cols, c->cols, c->q + r * c->cols, c->s + r);
}

/* w: bf16 bits [rows][cols]; q: int8 [rows][cols]; s: fp32 [rows]. Returns 0, or -1 on bad args. */
int oracle_quantize_rows(const uint16_t* w, int64_t rows, int64_t cols, int8_t* q, float* s, int threads) {
    if (!w || !q || !s || rows < 0 || cols <= 0) return -1;
    quant_ctx c = {w, cols, q, s};
    parallel_for(rows, threads, quantize_range, &c);
    return 0;
}

/* ----------------------------------------------------------------- routing */

/* Logits in fp64, softmax over all E, top-K by logit (ties: lower index first),
 * weights = chosen probabilities (not renormalised). */
static void route_token(const uint16_t* x, int64_t d, const float* wr, const float* bias, int E, int K,
                        int32_t* ids, double* wts, double* logits) {
    double z[64];
    for (int e = 0; e < E; ++e) {
        double acc = 0.0;
        const float* row = wr + (int64_t)e * d;
        for (int64_t i = 0; i < d; ++i) acc += (double)bf16_value(x[i]) * (double)row[i];
        if (bias) acc += (double)bias[e];
        z[e] = acc;
        if (logits) logits[e] = acc;
    }
    double zmax = z[0];
    for (int e = 1; e < E; ++e)
        if (z[e] > zmax) zmax = z[e];
    double p[64], denom = 0.0;
    for (int e = 0; e < E; ++e) {
        p[e] = exp(z[e] - zmax);
        denom += p[e];
    }
    for (int e = 0; e < E; ++e) p[e] /= denom;
    int taken[64] = {0};
    for (int k = 0; k < K; ++k) {
        int best = -1;
        for (int e = 0; e < E; ++e) {
            if (taken[e]) continue;
            if (best < 0 || z[e] > z[best]) best = e; /* strict: equal logits keep the lower index */
        }
        taken[best] = 1;
        ids[k] = best;
        wts[k] = p[best];
    }
}

typedef struct {
    const uint16_t* x;
    int64_t d;
    const float* wr;
    const float* bias;
    int E, K;
    int32_t* ids;
    double* wts;
    double* logits;
} route_ctx;

static void route_range(void* p, int64_t b, int64_t e) {
    route_ctx* c = (route_ctx*)p;
    for (int64_t t = b; t < e; ++t)
        route_token(c->x + t * c->d, c->d, c->wr, c->bias, c->E, c->K, c->ids + t * c->K, c->wts + t * c->K,
                    c->logits ? c->logits + t * c->E : NULL);
}

/* x: bf16 bits [T][d]; wr: fp32 [E][d]; bias: fp32 [E] or NULL.
 * ids: int32 [T][K]; wts: fp64 [T][K]; logits: fp64 [T][E] or NULL.  Returns 0, or -1 on bad args. */
int oracle_route(const uint16_t* x, int64_t T, int64_t d, const float* wr, const float* bias, int E, int K,
                 int32_t* ids, double* wts, double* logits, int threads) {
    if (!x || !wr || !ids || !wts || T < 0 || d <= 0 || E < 1 || E > 64 || K < 1 || K > E) return -1;
    route_ctx c = {x, d, wr, bias, E, K, ids, wts, logits};
    parallel_for(T, threads, route_range, &c);
    return 0;
}

/* ----------------------------------------------------------------- experts */

typedef struct {
    const uint16_t* x;
    int64_t d, F;
    int E, K;
    const float* wr;
    const float* bias;
    const int8_t *q1, *q3, *q2;
    const float *s1, *s3, *s2;
    const int64_t* tokens;
    double* y;
    int32_t* ids;
    double* wts;
    double* h_out;
} fwd_ctx;

/* One SwiGLU expert on one token with dequantized weights w = q * s (exact in fp64):
 *   a1_j = sum_i w1[j][i] x_i,  a3_j = sum_i w3[j][i] x_i,
 *   h_j = SiLU(a1_j) * a3_j = a1_j / (1 + exp(-a1_j)) * a3_j,
 *   o_i = sum_j w2[i][j] h_j. */
static void expert_ffn(const fwd_ctx* c, int e, const double* xd, double* h, double* o) {
    const int64_t d = c->d, F = c->F;
    const int8_t* q1 = c->q1 + (int64_t)e * F * d;
    const int8_t* q3 = c->q3 + (int64_t)e * F * d;
    const int8_t* q2 = c->q2 + (int64_t)e * d * F;
    const float* s1 = c->s1 + (int64_t)e * F;
    const float* s3 = c->s3 + (int64_t)e * F;
    const float* s2 = c->s2 + (int64_t)e * d;
    for (int64_t j = 0; j < F; ++j) {
        double a1 = 0.0, a3 = 0.0;
        const double sc1 = (double)s1[j], sc3 = (double)s3[j];
        const int8_t* r1 = q1 + j * d;
        const int8_t* r3 = q3 + j * d;
        for (int64_t i = 0; i < d; ++i) {
            a1 += ((double)r1[i] * sc1) * xd[i];
            a3 += ((double)r3[i] * sc3) * xd[i];
        }
        h[j] = a1 / (1.0 + exp(-a1)) * a3;
    }
    for (int64_t i = 0; i < d; ++i) {
        double acc = 0.0;
        const double sc2 = (double)s2[i];
        const int8_t* r2 = q2 + i * F;
        for (int64_t j = 0; j < F; ++j) acc += ((double)r2[j] * sc2) * h[j];
        o[i] = acc;
    }
}

static void forward_range(void* p, int64_t b, int64_t e) {
    fwd_ctx* c = (fwd_ctx*)p;
    const int64_t d = c->d, F = c->F;
    double* xd = (double*)malloc(sizeof(double) * (size_t)d);
    double* h = (double*)malloc(sizeof(double) * (size_t)F);
    double* o = (double*)malloc(sizeof(double) * (size_t)d);
    int32_t ids[64];
    double wts[64];
    for (int64_t n = b; n < e; ++n) {
        const int64_t t = c->tokens ? c->tokens[n] : n;
        const uint16_t* xt = c->x + t * d;
        for (int64_t i = 0; i < d; ++i) xd[i] = (double)bf16_value(xt[i]);
        route_token(xt, d, c->wr, c->bias, c->E, c->K, ids, wts, NULL);
        double* yt = c->y + n * d;
        for (int64_t i = 0; i < d; ++i) yt[i] = 0.0;
        for (int k = 0; k < c->K; ++k) {
            expert_ffn(c, ids[k], xd, h, o);
            for (int64_t i = 0; i < d; ++i) yt[i] += wts[k] * o[i];
            if (c->h_out) memcpy(c->h_out + (n * c->K + k) * F, h, sizeof(double) * (size_t)F);
            if (c->ids) c->ids[n * c->K + k] = ids[k];
            if (c->wts) c->wts[n * c->K + k] = wts[k];
        }
    }
    free(xd);
    free(h);
    free(o);
}

/* The layer on a subset of tokens.
 *   x: bf16 bits [T][d]; wr fp32 [E][d]; bias fp32 [E] or NULL;
 *   q1, q3: int8 [E][F][d] with s1, s3 fp32 [E][F]; q2: int8 [E][d][F] with s2 fp32 [E][d];
 *   tokens: int64 [n_tokens] indices into x, or NULL for tokens 0..n_tokens-1;
 *   y: fp64 [n_tokens][d] (output);
 *   ids int32 [n_tokens][K], wts fp64 [n_tokens][K], h_out fp64 [n_tokens][K][F]: optional outputs.
 * Returns 0, or -1 on bad arguments. */
int oracle_moe_forward(const uint16_t* x, int64_t T, int64_t d, int64_t F, int E, int K, const float* wr,
                       const float* bias, const int8_t* q1, const float* s1, const int8_t* q3, const float* s3,
                       const int8_t* q2, const float* s2, const int64_t* tokens, int64_t n_tokens, double* y,
                       int32_t* ids, double* wts, double* h_out, int threads) {
    if (!x || !wr || !q1 || !s1 || !q3 || !s3 || !q2 || !s2 || !y) return -1;
    if (T < 0 || d <= 0 || F <= 0 || E < 1 || E > 64 || K < 1 || K > E || n_tokens < 0) return -1;
    if (tokens) {
        for (int64_t n = 0; n < n_tokens; ++n)
            if (tokens[n] < 0 || tokens[n] >= T) return -1;
    } else if (n_tokens > T) {
        return -1;
    }
    fwd_ctx c = {x, d, F, E, K, wr, bias, q1, q3, q2, s1, s3, s2, tokens, y, ids, wts, h_out};
    parallel_for(n_tokens, threads, forward_range, &c);
    return 0;
}

/* ------------------------------------------------------- bf16-weight layer */

typedef struct {
    const uint16_t* x;
    int64_t d, F;
    int E, K;
    const float* wr;
    const float* bias;
    const uint16_t *w1, *w3, *w2;
    const int64_t* tokens;
    double* y;
    int32_t* ids;
    double* wts;
    double* h_out;
} fwdb_ctx;

/* One SwiGLU expert on one token with bf16 weights (exact as doubles). */
static void expert_ffn_bf16w(const fwdb_ctx* c, int e, const double* xd, double* h, double* o) {
    const int64_t d = c->d, F = c->F;
    const uint16_t* w1 = c->w1 + (int64_t)e * F * d;
    const uint16_t* w3 = c->w3 + (int64_t)e * F * d;
    const uint16_t* w2 = c->w2 + (int64_t)e * d * F;
    for (int64_t j = 0; j < F; ++j) {
        double a1 = 0.0, a3 = 0.0;
        const uint16_t* r1 = w1 + j * d;
        const uint16_t* r3 = w3 + j * d;
        for (int64_t i = 0; i < d; ++i) {
            a1 += (double)bf16_value(r1[i]) * xd[i];
            a3 += (double)bf16_value(r3[i]) * xd[i];
        }
        h[j] = a1 / (1.0 + exp(-a1)) * a3;
    }
    for (int64_t i = 0; i < d; ++i) {
        double acc = 0.0;
        const uint16_t* r2 = w2 + i * F;
        for (int64_t j = 0; j < F; ++j) acc += (double)bf16_value(r2[j]) * h[j];
        o[i] = acc;
    }
}

static void forward_bf16w_range(void* p, int64_t b, int64_t e) {
    fwdb_ctx* c = (fwdb_ctx*)p;
    const int64_t d = c->d, F = c->F;
    double* xd = (double*)malloc(sizeof(double) * (size_t)d);
    double* h = (double*)malloc(sizeof(double) * (size_t)F);
    double* o = (double*)malloc(sizeof(double) * (size_t)d);
    int32_t ids[64];
    double wts[64];
    for (int64_t n = b; n < e; ++n) {
        const int64_t t = c->tokens ? c->tokens[n] : n;
        const uint16_t* xt = c->x + t * d;
        for (int64_t i = 0; i < d; ++i) xd[i] = (double)bf16_value(xt[i]);
        route_token(xt, d, c->wr, c->bias, c->E, c->K, ids, wts, NULL);
        double* yt = c->y + n * d;
        for (int64_t i = 0; i < d; ++i) yt[i] = 0.0;
        for (int k = 0; k < c->K; ++k) {
            expert_ffn_bf16w(c, ids[k], xd, h, o);
            for (int64_t i = 0; i < d; ++i) yt[i] += wts[k] * o[i];
            if (c->h_out) memcpy(c->h_out + (n * c->K + k) * F, h, sizeof(double) * (size_t)F);
            if (c->ids) c->ids[n * c->K + k] = ids[k];
            if (c->wts) c->wts[n * c->K + k] = wts[k];
        }
    }
    free(xd);
    free(h);
    free(o);
}

/* The layer with bf16 weights w1, w3 [E][F][d] and w2 [E][d][F] (bit patterns); other arguments as in
 * oracle_moe_forward.  Returns 0, or -1 on bad arguments. */
int oracle_moe_forward_bf16w(const uint16_t* x, int64_t T, int64_t d, int64_t F, int E, int K, const float* wr,
                             const float* bias, const uint16_t* w1, const uint16_t* w3, const uint16_t* w2,
                             const int64_t* tokens, int64_t n_tokens, double* y, int32_t* ids, double* wts,
                             double* h_out, int threads) {
    if (!x || !wr || !w1 || !w3 || !w2 || !y) return -1;
    if (T < 0 || d <= 0 || F <= 0 || E < 1 || E > 64 || K < 1 || K > E || n_tokens < 0) return -1;
    if (tokens) {
        for (int64_t n = 0; n < n_tokens; ++n)
            if (tokens[n] < 0 || tokens[n] >= T) return -1;
    } else if (n_tokens > T) {
        return -1;
    }
    fwdb_ctx c = {x, d, F, E, K, wr, bias, w1, w3, w2, tokens, y, ids, wts, h_out};
    parallel_for(n_tokens, threads, forward_bf16w_range, &c);
    return 0;
}

/* ------------------------------------------------------------- dense MLP */

/* The MLP of a layer without MoE, with ExpertsInt8 weights (Jamba-1.5 paper, §3.1 "ExpertsInt8":
 * the MLP weights are quantized like the experts'; "Model Architecture": one layer in e = 2 has
 * an MoE block, the other an MLP).  The MLP is the same SwiGLU block as one expert,
 *   y_t = W2 (SiLU(W1 x_t) * (W3 x_t)),  w = q * scale formed exactly in fp64,
 * taken by every token with weight 1: no router, no softmax, no sum over experts. */
static void mlp_range(void* p, int64_t b, int64_t e) {
    fwd_ctx* c = (fwd_ctx*)p;
    const int64_t d = c->d, F = c->F;
    double* xd = (double*)malloc(sizeof(double) * (size_t)d);
    double* h = (double*)malloc(sizeof(double) * (size_t)F);
    for (int64_t n = b; n < e; ++n) {
        const int64_t t = c->tokens ? c->tokens[n] : n;
        const uint16_t* xt = c->x + t * d;
        for (int64_t i = 0; i < d; ++i) xd[i] = (double)bf16_value(xt[i]);
        expert_ffn(c, 0, xd, h, c->y + n * d);
        if (c->h_out) memcpy(c->h_out + n * F, h, sizeof(double) * (size_t)F);
    }
    free(xd);
    free(h);
}

/* The dense MLP on a subset of tokens.
 *   x: bf16 bits [T][d]; q1, q3: int8 [F][d] with s1, s3 fp32 [F]; q2: int8 [d][F] with s2 fp32 [d];
 *   tokens: int64 [n_tokens] indices into x, or NULL for tokens 0..n_tokens-1;
 *   y: fp64 [n_tokens][d] (output); h_out: fp64 [n_tokens][F] (optional, the SwiGLU hidden).
 * Returns 0, or -1 on bad arguments. */
int oracle_mlp_forward(const uint16_t* x, int64_t T, int64_t d, int64_t F, const int8_t* q1, const float* s1,
                       const int8_t* q3, const float* s3, const int8_t* q2, const float* s2, const int64_t* tokens,
                       int64_t n_tokens, double* y, double* h_out, int threads) {
    if (!x || !q1 || !s1 || !q3 || !s3 || !q2 || !s2 || !y) return -1;
    if (T < 0 || d <= 0 || F <= 0 || n_tokens < 0) return -1;
    if (tokens) {
        for (int64_t n = 0; n < n_tokens; ++n)
            if (tokens[n] < 0 || tokens[n] >= T) return -1;
    } else if (n_tokens > T) {
        return -1;
    }
    fwd_ctx c = {x, d, F, 1, 1, NULL, NULL, q1, q3, q2, s1, s3, s2, tokens, y, NULL, NULL, h_out};
    parallel_for(n_tokens, threads, mlp_range, &c);
    return 0;
}

/* ------------------------------------------------ FP8 (E4M3) comparator layer */

/* The FP8 layer the Jamba-1.5 paper compares ExpertsInt8 with (§3.1: on H100 ExpertsInt8 "matches
 * FP8 in latency"; FP8 needs hardware FP8 and, unlike ExpertsInt8, does not keep BF16 activations).
 * The page defines no FP8 scheme; the reading taken: both GEMM operands in OCP FP8 E4M3 (1 sign,
 * 4 exponent bits with bias 7, 3 mantissa bits, no infinities, largest finite 448, subnormals
 * m * 2^-9), weights with one fp32 scale per output channel (amax / 448), activations (x, and the
 * SwiGLU intermediate h) with one dynamic fp32 scale per row (per token, per expert slot for h);
 * rounding to the nearest E4M3 value, ties to the even code, saturating at +-448. */

/* The value of an E4M3 code (never called with the NaN codes 0x7F, 0xFF). */
static double e4m3_value(uint8_t code) {
    const int e = (code >> 3) & 15, m = code & 7;
    const double v = (e == 0) ? ldexp((double)m, -9) : ldexp(8.0 + m, e - 10); /* (1 + m/8) 2^(e-7) */
    return (code & 0x80) ? -v : v;
}

/* The E4M3 code nearest to a finite v (ties: even code), saturating at +-448; -0 keeps its sign. */
static uint8_t e4m3_round(double v) {
    const uint8_t sign = signbit(v) ? 0x80 : 0;
    const double a = fabs(v);
    if (a >= 448.0) return sign | 0x7E;
    if (a == 0.0) return sign;
    int e2;
    frexp(a, &e2); /* a = f * 2^e2, f in [0.5, 1) */
    int eb = e2 - 1;   /* floor(log2 a) */
    if (eb < -6) eb = -6; /* below the smallest normal: the subnormal spacing 2^-9 */
    double n = nearbyint(ldexp(a, 3 - eb)); /* a / spacing, spacing = 2^(eb-3): exact scaling, ties to even */
    if (n >= 16.0) { /* rounded up into the next binade */
        eb += 1;
        n = 8.0;
    }
    if (eb == -6 && n < 8.0) return sign | (uint8_t)n; /* subnormal */
    return sign | (uint8_t)(((eb + 7) << 3) | ((int)n - 8));
}

/* Per-row FP8 quantization of bf16 values: scale = amax / 448 (fp32 division), code = the E4M3
 * rounding of the exact quotient (taken in fp64, which decides every tie exactly for a bf16 value
 * and an fp32 scale); a row of zeros gets scale 1 and code 0. */
static void quantize_row_fp8(const uint16_t* w, int64_t cols, uint8_t* q, float* s) {
    float amax = 0.0f;
    for (int64_t i = 0; i < cols; ++i) {
        float a = fabsf(bf16_value(w[i]));
        if (a > amax) amax = a;
    }
    if (amax == 0.0f) {
        *s = 1.0f;
        memset(q, 0, (size_t)cols);
        return;
    }
    const float scale = amax / 448.0f;
    *s = scale;
    for (int64_t i = 0; i < cols; ++i) q[i] = e4m3_round((double)bf16_value(w[i]) / (double)scale);
}

typedef struct {
    const uint16_t* w;
    int64_t cols;
    uint8_t* q;
    float* s;
} quant8_ctx;

static void quantize_fp8_range(void* p, int64_t b, int64_t e) {
    quant8_ctx* c = (quant8_ctx*)p;
    for (int64_t r = b; r < e; ++r) quantize_row_fp8(c->w + r * c->cols, c->cols, c->q + r * c->cols, c->s + r);
}

/* w: bf16 bits [rows][cols]; q: E4M3 codes [rows][cols]; s: fp32 [rows]. Returns 0, or -1. */
int oracle_quantize_rows_fp8(const uint16_t* w, int64_t rows, int64_t cols, uint8_t* q, float* s, int threads) {
    if (!w || !q || !s || rows < 0 || cols <= 0) return -1;
    quant8_ctx c = {w, cols, q, s};
    parallel_for(rows, threads, quantize_fp8_range, &c);
    return 0;
}

/* codes[i] = e4m3_round(v[i]) and values[i] = e4m3_value(codes[i]), for tests. */
int oracle_e4m3_round(const double* v, int64_t n, uint8_t* codes, double* values) {
    if (!v || !codes || n < 0) return -1;
    for (int64_t i = 0; i < n; ++i) {
        codes[i] = e4m3_round(v[i]);
        if (values) values[i] = e4m3_value(codes[i]);
    }
    return 0;
}

typedef struct {
    const uint16_t* x;
    int64_t d, F;
    int E, K;
    const float* wr;
    const float* bias;
    const uint8_t *q1, *q3, *q2;
    const float *s1, *s3, *s2;
    const int64_t* tokens;
    double* y;
    int32_t* ids;
    double* wts;
    double* h_out;
} fwd8_ctx;

/* fp32 -> bf16, round to nearest even (finite values). */
static double bf16_round(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    u = (u + 0x7FFFu + ((u >> 16) & 1u)) & 0xFFFF0000u;
    float r;
    memcpy(&r, &u, 4);
    return (double)r;
}

/* One FP8 expert on one token whose activations xd are already the dequantized E4M3 values:
 *   a1_j = sum_i (v(q1[j][i]) s1_j) xd_i, a3_j likewise, h_j = SiLU(a1_j) a3_j,
 *   h held in bf16 between the two GEMMs, as in the ExpertsInt8 layer (fp64 -> fp32 -> bf16, each
 *   to nearest even), then quantized per row (scale = amax_j |h_j| / 448 in fp32, codes of
 *   h_j / scale), o_i = sum_j (v(q2[i][j]) s2_i) hd_j with hd the dequantized h. */
static void expert_ffn_fp8(const fwd8_ctx* c, int e, const double* xd, double* h, uint8_t* h8, double* o) {
    const int64_t d = c->d, F = c->F;
    const uint8_t* q1 = c->q1 + (int64_t)e * F * d;
    const uint8_t* q3 = c->q3 + (int64_t)e * F * d;
    const uint8_t* q2 = c->q2 + (int64_t)e * d * F;
    const float* s1 = c->s1 + (int64_t)e * F;
    const float* s3 = c->s3 + (int64_t)e * F;
    const float* s2 = c->s2 + (int64_t)e * d;
    double amax = 0.0;
    for (int64_t j = 0; j < F; ++j) {
        double a1 = 0.0, a3 = 0.0;
        const double sc1 = (double)s1[j], sc3 = (double)s3[j];
        for (int64_t i = 0; i < d; ++i) {
            a1 += (e4m3_value(q1[j * d + i]) * sc1) * xd[i];
            a3 += (e4m3_value(q3[j * d + i]) * sc3) * xd[i];
        }
        h[j] = a1 / (1.0 + exp(-a1)) * a3;
        const double hb = bf16_round((float)h[j]);
        if (fabs(hb) > amax) amax = fabs(hb);
    }
    const float hs = (amax == 0.0) ? 1.0f : (float)amax / 448.0f;
    for (int64_t j = 0; j < F; ++j) h8[j] = (amax == 0.0) ? 0 : e4m3_round(bf16_round((float)h[j]) / (double)hs);
    for (int64_t i = 0; i < d; ++i) {
        double acc = 0.0;
        const double sc2 = (double)s2[i];
        for (int64_t j = 0; j < F; ++j) acc += (e4m3_value(q2[i * F + j]) * sc2) * (e4m3_value(h8[j]) * (double)hs);
        o[i] = acc;
    }
}

static void forward_fp8_range(void* p, int64_t b, int64_t e) {
    fwd8_ctx* c = (fwd8_ctx*)p;
    const int64_t d = c->d, F = c->F;
    double* xd = (double*)malloc(sizeof(double) * (size_t)d);
    uint8_t* xq = (uint8_t*)malloc((size_t)d);
    double* h = (double*)malloc(sizeof(double) * (size_t)F);
    uint8_t* h8 = (uint8_t*)malloc((size_t)F);
    double* o = (double*)malloc(sizeof(double) * (size_t)d);
    int32_t ids[64];
    double wts[64];
    for (int64_t n = b; n < e; ++n) {
        const int64_t t = c->tokens ? c->tokens[n] : n;
        const uint16_t* xt = c->x + t * d;
        float xs;
        quantize_row_fp8(xt, d, xq, &xs); /* per-token activation scale */
        for (int64_t i = 0; i < d; ++i) xd[i] = e4m3_value(xq[i]) * (double)xs;
        route_token(xt, d, c->wr, c->bias, c->E, c->K, ids, wts, NULL); /* the router sees the bf16 x */
        double* yt = c->y + n * d;
        for (int64_t i = 0; i < d; ++i) yt[i] = 0.0;
        for (int k = 0; k < c->K; ++k) {
            expert_ffn_fp8(c, ids[k], xd, h, h8, o);
            for (int64_t i = 0; i < d; ++i) yt[i] += wts[k] * o[i];
            if (c->h_out) memcpy(c->h_out + (n * c->K + k) * F, h, sizeof(double) * (size_t)F);
            if (c->ids) c->ids[n * c->K + k] = ids[k];
            if (c->wts) c->wts[n * c->K + k] = wts[k];
        }
    }
    free(xd);
    free(xq);
    free(h);
    free(h8);
    free(o);
}

/* The FP8 layer on a subset of tokens; arguments as oracle_moe_forward with E4M3 codes for q1, q3, q2
 * (scales from oracle_quantize_rows_fp8); h_out gets the SwiGLU intermediate before its quantization. */
int oracle_moe_forward_fp8(const uint16_t* x, int64_t T, int64_t d, int64_t F, int E, int K, const float* wr,
                           const float* bias, const uint8_t* q1, const float* s1, const uint8_t* q3, const float* s3,
                           const uint8_t* q2, const float* s2, const int64_t* tokens, int64_t n_tokens, double* y,
                           int32_t* ids, double* wts, double* h_out, int threads) {
    if (!x || !wr || !q1 || !s1 || !q3 || !s3 || !q2 || !s2 || !y) return -1;
    if (T < 0 || d <= 0 || F <= 0 || E < 1 || E > 64 || K < 1 || K > E || n_tokens < 0) return -1;
    if (tokens) {
        for (int64_t n = 0; n < n_tokens; ++n)
            if (tokens[n] < 0 || tokens[n] >= T) return -1;
    } else if (n_tokens > T) {
        return -1;
    }
    fwd8_ctx c = {x, d, F, E, K, wr, bias, q1, q3, q2, s1, s3, s2, tokens, y, ids, wts, h_out};
    parallel_for(n_tokens, threads, forward_fp8_range, &c);
    return 0;
}

/* Number of host threads the oracle uses when asked for "all" (threads <= 0). */
int oracle_default_threads(void) { return pick_threads(0, 1 << 30); }
