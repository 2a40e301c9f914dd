/*
 * moe_oracle.c -- plain, slow CPU oracle for the fused MXFP4 routed-MoE layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls
 * this file: only the test suite, the smoke check and the bench's CPU-baseline
 * leg do.  It shares no code, table or constant generator with the CUDA
 * library; it holds its own MX tables and its own quantiser.
 *
 * What it computes, step by step, for one token t (per-token evaluation; the
 * GPU reaches the same result by grouping tokens per expert):
 *   routing   : softmax over the E router logits, the k largest kept (lowest
 *               expert index wins ties), their probabilities renormalised to
 *               sum to 1.  [TokenSpeed-kernel README, "Public API" (moe_route);
 *               fusedtok package description, "Operators" (softmax, top-k) and
 *               "API stability" (lowest-index tie determinism)]
 *   FC1       : [g;u] = W1_e . a, W1_e dequantised from MXFP4 (E2M1 codes, one
 *               E8M0 scale per 32 elements along the reduction dim).
 *               [tokenspeed-situ package description, intro and "Supported
 *               contract" (MxE2m1 weights)]
 *   activation: h = silu(g) * u (SwiGLU).  [b12x package description, "What's
 *               in here"; mxfp6-sm120 package description, path table
 *               ("SiLU-and-mul")]
 *   FC2       : y = W2_e . h.
 *   combine   : out[t] = sum_j w_j * y_j, j ascending.  [TokenSpeed-kernel
 *               README, "Public API" (moe_combine)]
 *   w4a8      : the activation x[t] is quantised to MXFP8 E4M3 (E8M0 scale per
 *               32 along H) before FC1, and h is quantised to MXFP8 then
 *               dequantised to bf16 before FC2.  [tokenspeed-situ, "Activation
 *               precision (w4a16 vs w4a8)"; mxfp6-sm120, "Execution model"]
 * All arithmetic is IEEE double; bf16 roundings are explicit.
 *
 * MX element/scale encodings follow the OCP Microscaling Formats (MX) v1.0
 * specification (E2M1, E4M3, E8M0 definitions and the shared-scale rule
 * floor(log2(amax)) - emax_elem).
 *
 * Parity pins for every function live in tests/test_oracle_*.py (MX codecs, routing and
 * grouping, the layer, the routed form, the shared expert), with hand-derived fixtures in
 * tests/golden/.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/*
 * Mutation hook for the pin tests: building with -DORACLE_PLANT_MISTAKE=n plants
 * one deliberate mistake (listed at each use) so that the tests can show their
 * pins catch it.  The default build (0) plants nothing.
 */
#ifndef ORACLE_PLANT_MISTAKE
#define ORACLE_PLANT_MISTAKE 0
#endif

/* ------------------------------------------------------------------------ */
/* MX element decode                                                         */
/* ------------------------------------------------------------------------ */

/* E2M1 magnitudes in code order (codes 0..7); codes 8..15 are the negatives. */
static const double kE2M1Mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double oracle_e2m1_decode(uint8_t code)
{
    double m = kE2M1Mag[code & 7];
    return (code & 8) ? -m : m;
}

/* E4M3 ("fn" flavour): bias 7, no infinities, S.1111.111 is NaN. */
double oracle_e4m3_decode(uint8_t code)
{
    int sign = (code >> 7) & 1;
    int exp = (code >> 3) & 15;
    int man = code & 7;
    double v;
    if (exp == 15 && man == 7)
        return NAN;
    if (exp == 0)
        v = ldexp((double)man, -9);            /* subnormal: man/8 * 2^-6 */
    else
        v = ldexp(8.0 + (double)man, exp - 10); /* (1 + man/8) * 2^(exp-7) */
    return sign ? -v : v;
}

/* E8M0 scale: 2^(e-127); 0xFF is NaN. */
double oracle_e8m0_decode(uint8_t e)
{
    if (e == 0xFF)
        return NAN;
    return ldexp(1.0, (int)e - 127);
}

/* ------------------------------------------------------------------------ */
/* MX quantisation                                                           */
/* ------------------------------------------------------------------------ */

enum { ORACLE_FMT_E2M1 = 0, ORACLE_FMT_E4M3 = 1 };

static double g_e4m3_grid[127]; /* non-negative finite E4M3 magnitudes, codes 0..126 */
static pthread_once_t g_grid_once = PTHREAD_ONCE_INIT;

static void build_e4m3_grid(void)
{
    for (int c = 0; c < 127; ++c)
        g_e4m3_grid[c] = oracle_e4m3_decode((uint8_t)c);
}

/*
 * Round the non-negative magnitude t onto a monotone grid of n values
 * (grid[i] is the value of code i): nearest value, ties to the code whose
 * least significant bit is 0 (round-half-to-even on the element's mantissa),
 * and anything at or above the largest value saturates to it.
 */
static int round_to_grid(double t, const double *grid, int n)
{
    if (!(t < grid[n - 1]))
        return n - 1;
    int i = 0;
    while (i + 1 < n && grid[i + 1] <= t)
        ++i;
    double lo = t - grid[i];
    double hi = grid[i + 1] - t;
    if (lo < hi)
        return i;
    if (hi < lo)
        return i + 1;
    if (ORACLE_PLANT_MISTAKE == 1) /* plant: ties go to the odd code */
        return (i & 1) ? i : i + 1;
    return (i & 1) ? i + 1 : i;
}

/*
 * Quantise one block of n (<= 32) values to MX.  The shared scale exponent is
 * s = floor(log2(amax)) - emax (emax = 2 for E2M1, 8 for E4M3), clamped to
 * [-127, 127]; the scale byte is s + 127.  floor(log2) is read from frexp, not
 * from a libm log.  Each element is v * 2^-s rounded onto the element grid
 * (RNE, saturating); the sign is kept even when the magnitude rounds to 0.
 * All-zero block: s = -127 (byte 0x00), all codes +0.  NaN/Inf in the block:
 * scale byte 0xFF and all codes 0 (such inputs are never generated).
 * codes_out receives one code per element (unpacked).
 */
static void quantize_block(const double *v, int n, int fmt, uint8_t *codes_out, uint8_t *scale_out)
{
    pthread_once(&g_grid_once, build_e4m3_grid);
    const double *grid = (fmt == ORACLE_FMT_E2M1) ? kE2M1Mag : g_e4m3_grid;
    const int ngrid = (fmt == ORACLE_FMT_E2M1) ? 8 : 127;
    const int emax = ((fmt == ORACLE_FMT_E2M1) ? 2 : 8) + (ORACLE_PLANT_MISTAKE == 2); /* plant: emax + 1 */
    const uint8_t sign_bit = (fmt == ORACLE_FMT_E2M1) ? 0x8 : 0x80;

    double amax = 0.0;
    int finite = 1;
    for (int i = 0; i < n; ++i) {
        if (!isfinite(v[i]))
            finite = 0;
        else if (fabs(v[i]) > amax)
            amax = fabs(v[i]);
    }
    if (!finite) {
        *scale_out = 0xFF;
        memset(codes_out, 0, (size_t)n);
        return;
    }
    int s;
    if (amax == 0.0) {
        s = -127;
    } else {
        int ex;
        frexp(amax, &ex); /* amax = m * 2^ex, m in [0.5, 1) => floor(log2 amax) = ex - 1 */
        s = ex - 1 - emax;
        if (s < -127)
            s = -127;
        if (s > 127)
            s = 127;
    }
    *scale_out = (uint8_t)(s + 127);
    for (int i = 0; i < n; ++i) {
        double t = ldexp(fabs(v[i]), -s); /* exact power-of-two scaling */
        int c = round_to_grid(t, grid, ngrid);
        codes_out[i] = (uint8_t)c | (signbit(v[i]) ? sign_bit : 0);
    }
}

/* Quantise one row of K values (K % 32 == 0) given in double. */
static void quantize_row_d(const double *v, int64_t K, int fmt, uint8_t *codes, uint8_t *scales)
{
    uint8_t blk[32];
    for (int64_t b = 0; b < K / 32; ++b) {
        quantize_block(v + b * 32, 32, fmt, blk, &scales[b]);
        if (fmt == ORACLE_FMT_E2M1) {
            for (int i = 0; i < 16; ++i)
                codes[b * 16 + i] = (uint8_t)(blk[2 * i] | (blk[2 * i + 1] << 4));
        } else {
            memcpy(codes + b * 32, blk, 32);
        }
    }
}

typedef struct {
    const float *v;
    int64_t rows, K;
    int fmt;
    uint8_t *codes, *scales;
    int64_t r0, r1;
} quant_job;

static void *quant_worker(void *arg)
{
    quant_job *j = (quant_job *)arg;
    const int64_t code_stride = (j->fmt == ORACLE_FMT_E2M1) ? j->K / 2 : j->K;
    double *row = (double *)malloc(sizeof(double) * (size_t)j->K);
    for (int64_t r = j->r0; r < j->r1; ++r) {
        for (int64_t i = 0; i < j->K; ++i)
            row[i] = (double)j->v[r * j->K + i];
        quantize_row_d(row, j->K, j->fmt, j->codes + r * code_stride, j->scales + r * (j->K / 32));
    }
    free(row);
    return NULL;
}

/*
 * Quantise a row-major float32 matrix [rows, K] along K.
 * fmt 0 = MXFP4 (E2M1 codes packed two per byte, element 2i in the low nibble
 * of byte i; codes [rows, K/2]); fmt 1 = MXFP8 E4M3 (codes [rows, K]).
 * scales: [rows, K/32] E8M0 bytes.  Returns 0, or -1 on bad arguments.
 */
int oracle_mx_quantize(const float *v, int64_t rows, int64_t K, int fmt, uint8_t *codes,
                       uint8_t *scales, int nthreads)
{
    if (!v || !codes || !scales || rows < 0 || K <= 0 || K % 32 != 0 || (fmt != 0 && fmt != 1))
        return -1;
    if (nthreads < 1)
        nthreads = 1;
    if (nthreads > rows)
        nthreads = rows > 0 ? (int)rows : 1;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    quant_job *jobs = (quant_job *)malloc(sizeof(quant_job) * (size_t)nthreads);
    for (int i = 0; i < nthreads; ++i) {
        jobs[i] = (quant_job){v, rows, K, fmt, codes, scales, rows * i / nthreads, rows * (i + 1) / nthreads};
        pthread_create(&th[i], NULL, quant_worker, &jobs[i]);
    }
    for (int i = 0; i < nthreads; ++i)
        pthread_join(th[i], NULL);
    free(th);
    free(jobs);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* bf16 rounding                                                             */
/* ------------------------------------------------------------------------ */

/* Round a double directly to the nearest bf16 value (ties to even), returned
 * as a double.  bf16: 8 significant bits, exponent range of float32. */
double oracle_round_bf16(double v)
{
    if (!isfinite(v) || v == 0.0)
        return v;
    int ex;
    frexp(v, &ex); /* |v| = m * 2^ex, m in [0.5, 1) */
    int q = ex - 8; /* quantum of an 8-significant-bit number in this binade */
    if (q < -133)
        q = -133; /* bf16 subnormal quantum is 2^-133 */
    double r = nearbyint(ldexp(v, -q)); /* default rounding mode: nearest-even */
    double out = ldexp(r, q);
    if (fabs(out) >= ldexp(1.0, 128))
        return v > 0 ? INFINITY : -INFINITY;
    return out;
}

static inline double bf16_bits_to_double(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

static inline uint16_t double_to_bf16_bits(double v)
{
    /* v is already a bf16 value: the float conversion is exact. */
    float f = (float)oracle_round_bf16(v);
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(u >> 16);
}

uint16_t oracle_bf16_bits(double v) { return double_to_bf16_bits(v); }

/* ------------------------------------------------------------------------ */
/* Routing                                                                   */
/* ------------------------------------------------------------------------ */

/*
 * Top-k softmax routing for one token.  The k experts are the k largest
 * logits, ordered by descending logit, equal logits ordered by ascending expert
 * index (the selection is taken on the float32 logits: softmax is monotone, so
 * this is the same set as on the probabilities, without exp-rounding ties).
 * Weights: full softmax in double, the k selected probabilities renormalised
 * to sum to 1, rounded to float.
 */
void oracle_route(const float *logits, int E, int k, int32_t *ids, float *w)
{
    /* A NaN logit ranks below every number and gets probability 0: it is read as -inf (the
     * pages do not say; this keeps the selection a total order).  A row with no finite logit
     * has no defined softmax; its weights come out NaN. */
    double *l = (double *)malloc(sizeof(double) * (size_t)E);
    for (int e = 0; e < E; ++e)
        l[e] = isnan(logits[e]) ? -INFINITY : (double)logits[e];
    unsigned char *taken = (unsigned char *)calloc((size_t)E, 1);
    for (int j = 0; j < k; ++j) {
        int best = -1;
        for (int e = 0; e < E; ++e) {
            if (taken[e])
                continue;
            if (best < 0 || l[e] > l[best] ||
                (ORACLE_PLANT_MISTAKE == 3 && l[e] == l[best])) /* plant: highest index wins */
                best = e;
        }
        taken[best] = 1;
        ids[j] = best;
    }
    free(taken);
    double mx = -INFINITY;
    for (int e = 0; e < E; ++e)
        if (l[e] > mx)
            mx = l[e];
    double z = 0.0;
    for (int e = 0; e < E; ++e)
        z += exp(l[e] - mx);
    double p[1024];
    double psum = 0.0;
    for (int j = 0; j < k; ++j) {
        p[j] = exp(l[ids[j]] - mx) / z;
        psum += p[j];
    }
    free(l);
    for (int j = 0; j < k; ++j)
        w[j] = (float)(ORACLE_PLANT_MISTAKE == 8 ? p[j] : p[j] / psum); /* plant: no renormalisation */
}

/* ------------------------------------------------------------------------ */
/* Grouping                                                                  */
/* ------------------------------------------------------------------------ */

/*
 * Group the T*k (token, slot) pairs by expert.  Pair id p = t*k + j.
 * counts[e] = number of pairs routed to e; offsets = exclusive prefix sum
 * (E+1 entries); sorted_pair = stable counting sort of p by expert, i.e. within
 * one expert the pairs appear in ascending p (ascending token).
 */
void oracle_group(int T, int k, int E, const int32_t *ids, int32_t *counts, int32_t *offsets,
                  int32_t *sorted_pair)
{
    const int64_t P = (int64_t)T * k;
    memset(counts, 0, sizeof(int32_t) * (size_t)E);
    for (int64_t p = 0; p < P; ++p)
        counts[ids[p]]++;
    offsets[0] = 0;
    for (int e = 0; e < E; ++e)
        offsets[e + 1] = offsets[e] + counts[e];
    int32_t *fill = (int32_t *)malloc(sizeof(int32_t) * (size_t)E);
    memcpy(fill, offsets, sizeof(int32_t) * (size_t)E);
    if (ORACLE_PLANT_MISTAKE == 9) { /* plant: pairs placed in descending order within an expert */
        for (int e = 0; e < E; ++e)
            fill[e] = offsets[e + 1];
        for (int64_t p = 0; p < P; ++p)
            sorted_pair[--fill[ids[p]]] = (int32_t)p;
    } else {
        for (int64_t p = 0; p < P; ++p)
            sorted_pair[fill[ids[p]]++] = (int32_t)p;
    }
    free(fill);
}

/* ------------------------------------------------------------------------ */
/* Per-token layer evaluation                                                */
/* ------------------------------------------------------------------------ */

typedef struct {
    int T, H, I, E, k, act_mode;
    int n_shared;               /* shared-expert slots E..E+n_shared-1, weight 1 for every token */
    const uint16_t *x;
    const float *logits;        /* router logits [T,E], or NULL when the routing is given: */
    const int32_t *given_ids;   /* [T,k] global expert ids (routed form), */
    const float *given_w;       /* [T,k] their weights, */
    int local_offset;           /* and the first global id of the local experts [0,E) */
    const uint8_t *w1, *w1s, *w2, *w2s;
    const int32_t *tokens;
    uint16_t *out;
    double *out_exact;
    int32_t *ids_out;
    float *w_out;
    int64_t i0, i1;
} fwd_job;

/* Dequantised weight element (e, row, col) of an MXFP4 matrix with K columns. */
static inline double mx4_weight(const uint8_t *codes, const uint8_t *scales, int64_t row, int64_t K,
                                int64_t col)
{
    uint8_t byte = codes[row * (K / 2) + col / 2];
    int odd = (int)(col & 1) ^ (ORACLE_PLANT_MISTAKE == 4); /* plant: nibbles swapped */
    uint8_t code = odd ? (byte >> 4) : (byte & 0xF);
    return oracle_e2m1_decode(code) * oracle_e8m0_decode(scales[row * (K / 32) + col / 32]);
}

/* MXFP8-quantise a row of doubles and return the dequantised values in place. */
static void mxfp8_roundtrip(double *v, int64_t K)
{
    uint8_t blk[32], sc;
    for (int64_t b = 0; b < K / 32; ++b) {
        quantize_block(v + b * 32, 32, ORACLE_FMT_E4M3, blk, &sc);
        double s = oracle_e8m0_decode(sc);
        for (int i = 0; i < 32; ++i)
            v[b * 32 + i] = oracle_e4m3_decode(blk[i]) * s;
    }
}

static void forward_token(const fwd_job *jb, int64_t slot)
{
    const int H = jb->H, I = jb->I, E = jb->E, k = jb->k;
    const int t = jb->tokens ? jb->tokens[slot] : (int)slot;
    int32_t ids[1024];
    float w[1024];
    if (jb->logits) {
        oracle_route(jb->logits + (int64_t)t * E, E, k, ids, w);
    } else {
        /* routed form: global ids; only the experts of the local shard [offset, offset + E)
         * contribute, so the result is this shard's partial output */
        for (int j = 0; j < k; ++j) {
            const int64_t g = jb->given_ids[(int64_t)t * k + j];
            const int64_t off = ORACLE_PLANT_MISTAKE == 10 ? 0 : jb->local_offset; /* plant: offset ignored */
            ids[j] = (g >= off && g < off + E) ? (int32_t)(g - off) : -1;
            w[j] = jb->given_w[(int64_t)t * k + j];
        }
    }

    double *a = (double *)malloc(sizeof(double) * (size_t)H);
    double *h = (double *)malloc(sizeof(double) * (size_t)I);
    double *acc = (double *)calloc((size_t)H, sizeof(double));
    for (int c = 0; c < H; ++c)
        a[c] = bf16_bits_to_double(jb->x[(int64_t)t * H + c]);
    if (jb->act_mode == 1)
        mxfp8_roundtrip(a, H);

    /* the shared expert: slots k..k+n_shared-1 hold its n_shared chunks (experts E..), weight 1
     * [mxfp6-sm120 package description, path table: "shared-expert combine and routed/shared
     * reduction"] */
    const int S = jb->n_shared;
    for (int c = 0; c < S; ++c) {
        ids[k + c] = E + c;
        w[k + c] = ORACLE_PLANT_MISTAKE == 11 ? 0.5f : 1.0f; /* plant: shared expert half-weighted */
    }
    if (jb->ids_out)
        memcpy(jb->ids_out + slot * (k + S), ids, sizeof(int32_t) * (size_t)(k + S));
    if (jb->w_out)
        memcpy(jb->w_out + slot * (k + S), w, sizeof(float) * (size_t)(k + S));
    for (int j = 0; j < k + S - (ORACLE_PLANT_MISTAKE == 7); ++j) { /* plant: last slot dropped */
        const int64_t e = ids[j];
        if (e < 0)
            continue; /* routed form: an expert outside the local shard */
        const int64_t r1 = e * 2 * I; /* first W1 row of expert e */
        for (int i = 0; i < I; ++i) {
            double g = 0.0, u = 0.0;
            for (int c = 0; c < H; ++c) {
                g += mx4_weight(jb->w1, jb->w1s, r1 + i, H, c) * a[c];
                u += mx4_weight(jb->w1, jb->w1s, r1 + I + i, H, c) * a[c];
            }
            if (ORACLE_PLANT_MISTAKE == 5) { /* plant: gate and up halves swapped */
                double tmp = g;
                g = u;
                u = tmp;
            }
            if (ORACLE_PLANT_MISTAKE == 6) /* plant: sign error inside silu */
                h[i] = g / (1.0 + exp(g)) * u;
            else
                h[i] = g / (1.0 + exp(-g)) * u;
        }
        if (jb->act_mode == 1)
            mxfp8_roundtrip(h, I); /* dequantised MXFP8 values are exact bf16 values */
        else
            for (int i = 0; i < I; ++i)
                h[i] = oracle_round_bf16(h[i]);
        const int64_t r2 = e * H; /* first W2 row of expert e */
        for (int n = 0; n < H; ++n) {
            double y = 0.0;
            for (int i = 0; i < I; ++i)
                y += mx4_weight(jb->w2, jb->w2s, r2 + n, I, i) * h[i];
            acc[n] += (double)w[j] * y;
        }
    }
    for (int n = 0; n < H; ++n) {
        jb->out[slot * H + n] = double_to_bf16_bits(acc[n]);
        if (jb->out_exact)
            jb->out_exact[slot * H + n] = acc[n];
    }
    free(a);
    free(h);
    free(acc);
}

static void *forward_worker(void *arg)
{
    fwd_job *jb = (fwd_job *)arg;
    for (int64_t s = jb->i0; s < jb->i1; ++s)
        forward_token(jb, s);
    return NULL;
}

/*
 * Evaluate the layer for n_eval tokens.  tokens == NULL evaluates tokens
 * 0..n_eval-1; otherwise tokens[i] names the token whose output goes to row i
 * of out (bf16 bits, [n_eval, H]) and of ids_out/w_out ([n_eval, k], optional).
 * out_exact (optional, [n_eval, H]) receives the combined output before its
 * final rounding to bf16 (the exact value a rounded result is measured against).
 * act_mode 0 = bf16 activations (w4a16), 1 = MXFP8 activations (w4a8).
 * Layouts: x bf16 [T,H]; logits f32 [T,E]; w1 codes [E,2I,H/2] (gate rows
 * [0,I), up rows [I,2I)), w1s [E,2I,H/32]; w2 codes [E,H,I/2], w2s [E,H,I/32].
 * Returns 0, or -1 on bad arguments.
 */
static int run_forward(int T, int H, int I, int E, int S, int k, int act_mode, const uint16_t *x, const float *logits,
                       const int32_t *given_ids, const float *given_w, int local_offset, const uint8_t *w1,
                       const uint8_t *w1s, const uint8_t *w2, const uint8_t *w2s, const int32_t *tokens, int n_eval,
                       uint16_t *out, int32_t *ids_out, float *w_out, double *out_exact, int nthreads)
{
    if (T < 0 || H <= 0 || I <= 0 || H % 32 || I % 32 || E < 1 || S < 0 || E + S > 1024 || k < 1 ||
        k + S > 1024 || (logits && k > E) || (act_mode != 0 && act_mode != 1) || n_eval < 0 || !out)
        return -1;
    if (n_eval == 0)
        return 0;
    for (int i = 0; tokens && i < n_eval; ++i)
        if (tokens[i] < 0 || tokens[i] >= T)
            return -1;
    if (!tokens && n_eval > T)
        return -1;
    if (nthreads < 1)
        nthreads = 1;
    if (nthreads > n_eval)
        nthreads = n_eval;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    fwd_job *jobs = (fwd_job *)malloc(sizeof(fwd_job) * (size_t)nthreads);
    for (int i = 0; i < nthreads; ++i) {
        jobs[i] = (fwd_job){T, H, I, E, k, act_mode, S, x, logits, given_ids, given_w, local_offset, w1, w1s, w2, w2s,
                            tokens, out, out_exact, ids_out, w_out, (int64_t)n_eval * i / nthreads,
                            (int64_t)n_eval * (i + 1) / nthreads};
        pthread_create(&th[i], NULL, forward_worker, &jobs[i]);
    }
    for (int i = 0; i < nthreads; ++i)
        pthread_join(th[i], NULL);
    free(th);
    free(jobs);
    return 0;
}

int oracle_moe_forward(int T, int H, int I, int E, int k, int act_mode, const uint16_t *x,
                       const float *logits, const uint8_t *w1, const uint8_t *w1s, const uint8_t *w2,
                       const uint8_t *w2s, const int32_t *tokens, int n_eval, uint16_t *out,
                       int32_t *ids_out, float *w_out, double *out_exact, int nthreads)
{
    if (!logits)
        return -1;
    return run_forward(T, H, I, E, 0, k, act_mode, x, logits, NULL, NULL, 0, w1, w1s, w2, w2s, tokens, n_eval, out,
                       ids_out, w_out, out_exact, nthreads);
}

/*
 * The layer with a shared expert: every token also passes through the shared
 * expert, a SwiGLU MLP of intermediate size n_shared * I, and its output is added
 * to the routed sum with weight 1 (the routed/shared reduction of the mxfp6-sm120
 * package description's routed-MoE path).  The shared expert is held as n_shared
 * chunks of I in expert slots E..E+n_shared-1 of w1..w2s ([E + n_shared, ...]):
 * chunk c holds gate rows c*I..(c+1)*I-1 of the shared W1 followed by the matching
 * up rows, and columns c*I..(c+1)*I-1 of the shared W2.  (SwiGLU is elementwise
 * over the intermediate index, so the chunks' outputs add up to the shared MLP.)
 * The router sees the E routed experts only (logits [T, E]).  ids_out / w_out
 * ([n, k + n_shared]) list the routed slots, then the shared slots (ids E..,
 * weight 1).  Returns 0, or -1 on bad arguments.
 */
int oracle_moe_forward_shared(int T, int H, int I, int E, int n_shared, int k, int act_mode, const uint16_t *x,
                              const float *logits, const uint8_t *w1, const uint8_t *w1s, const uint8_t *w2,
                              const uint8_t *w2s, const int32_t *tokens, int n_eval, uint16_t *out, int32_t *ids_out,
                              float *w_out, double *out_exact, int nthreads)
{
    if (!logits)
        return -1;
    return run_forward(T, H, I, E, n_shared, k, act_mode, x, logits, NULL, NULL, 0, w1, w1s, w2, w2s, tokens, n_eval,
                       out, ids_out, w_out, out_exact, nthreads);
}

/*
 * The layer with the routing given instead of the router logits (precomputed,
 * unpacked top-k: global expert ids and their weights), for the local expert
 * shard [local_offset, local_offset + E) whose weights w1..w2s hold [E, ...].
 * Pairs routed to experts outside the shard contribute nothing, so the output
 * is the shard's partial sum; the partial outputs of all shards add up to the
 * whole layer.  [tokenspeed-situ package description, "Supported contract":
 * precomputed top-k routing, global expert ids, contiguous local expert shards
 * with a local expert offset, partial outputs that the caller all-reduces]
 * ids_out receives the local ids (-1: not in the shard), w_out the weights.
 * Returns 0, or -1 on bad arguments.
 */
int oracle_moe_forward_routed(int T, int H, int I, int E, int k, int act_mode, const uint16_t *x,
                              const int32_t *topk_ids, const float *topk_w, int local_offset, const uint8_t *w1,
                              const uint8_t *w1s, const uint8_t *w2, const uint8_t *w2s, const int32_t *tokens,
                              int n_eval, uint16_t *out, int32_t *ids_out, float *w_out, double *out_exact,
                              int nthreads)
{
    if (!topk_ids || !topk_w || k > 1024)
        return -1;
    return run_forward(T, H, I, E, 0, k, act_mode, x, NULL, topk_ids, topk_w, local_offset, w1, w1s, w2, w2s, tokens,
                       n_eval, out, ids_out, w_out, out_exact, nthreads);
}
