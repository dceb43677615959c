/*
 * Float64 CPU oracle of the Qwen3-0.6B decode-attention step.
 *
 * TEST INFRASTRUCTURE ONLY. This file is built into oracle/liboracle.so and is
 * loaded by the test suite, by the smoke check and by the benchmark's CPU
 * baseline leg. The CUDA library never links, loads or calls it, and it shares
 * no source, header, table or helper with the CUDA library.
 *
 * What it computes is the plain definition of the step, written out in double
 * precision in the order the specification states it, with no blocking, no
 * online softmax and no fusion:
 *
 *   qkv row -> split into 16 q heads | 8 k heads | 8 v heads of 128
 *        (Qwen3-0.6B Model Spec, "Compute-graph nodes", attn.qkv_proj N=4096;
 *         nnterp qwen3 page, "Queries and keys are normed per head, before the
 *         rotary": q_proj(x).view(..., num_heads, 128))
 *   q, k -> per-head RMSNorm over 128 dims with one shared gain vector
 *        (Model Spec, "Compute-graph nodes", attn.qk_norm, eps=1e-06)
 *   q, k -> RoPE: pairs (i, i+64), i < 64, rotated by pos * theta^(-2i/128)
 *        (Model Spec, "Compute-graph nodes", attn.rope, theta=1000000)
 *   k, v -> appended to the paged cache at slot seq_len-1
 *        (Model Spec, "At a glance", shape domain: page size 16;
 *         Supported models page, "What every spec covers": one new query per
 *         sequence over seq_lens[b] cached positions)
 *   o[b,h] = sum_{s < seq_lens[b]} softmax_s(<q[b,h], k[b,s,h/2]> / sqrt(128)) v[b,s,h/2]
 *        (Model Spec, "Compute-graph nodes", attn.core decodeGQA)
 *
 * Readings taken where the pages leave a step open (each one is listed with
 * its reason in the design notes of the repository):
 *   - the rotation is the counter-clockwise one: (a, b) -> (a cos - b sin,
 *     b cos + a sin) for the pair (x_i, x_{i+64});
 *   - seq_lens[b] counts the new token; the new token sits in cache slot
 *     seq_lens[b]-1 and, unless positions are given, has that position too;
 *   - the paged cache is [num_pages][16 slots][8 kv heads][128] bf16 and
 *     logical slot t of sequence b lives in page block_table[b][t/16], row t%16;
 *   - nothing is rounded until an output: k is rounded once, from double, to
 *     bf16 with round-to-nearest-even when it is written to the cache; the
 *     attention then reads the cache as stored (the rounded k); o stays double.
 *
 * It also holds the two nodes that produce the step's input, input_norm and
 * attn.qkv_proj (oracle_input_norm_qkv_proj), with nothing rounded before the
 * bf16 qkv row, and the node that consumes its output, attn.o_proj
 * (oracle_o_proj).
 *
 * Every function names the passage it follows. The pins that tie this file to
 * the pages and to mathematics (closed forms, invariants, library routines,
 * brute force) live in tests/test_oracle_pins.py.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Constants of the Qwen3-0.6B Model Spec ("Published configuration" and the
 * attn.* rows of "Compute-graph nodes"). */
enum {
    ORC_NUM_Q_HEADS = 16,
    ORC_NUM_KV_HEADS = 8,
    ORC_HEAD_DIM = 128,
    ORC_ROPE_PAIRS = 64,          /* attn.rope: active = 64, rot = 128 */
    ORC_PAGE = 16,                /* "At a glance": page size 16 */
    ORC_Q_WIDTH = ORC_NUM_Q_HEADS * ORC_HEAD_DIM,   /* 2048 */
    ORC_KV_WIDTH = ORC_NUM_KV_HEADS * ORC_HEAD_DIM, /* 1024 */
    ORC_PAGE_ELEMS = ORC_PAGE * ORC_KV_WIDTH,       /* elements in one page */
    ORC_MAX_BATCH = 256,          /* "At a glance": B in [1, 256] */
    ORC_MAX_SEQ = 40960           /* "At a glance": S in [1, 40960] */
};

enum {
    ORC_OK = 0,
    ORC_ERR_ARG = -1,      /* a null pointer or a size outside the domain */
    ORC_ERR_BOUNDS = -4    /* a seq_len or a block-table entry out of range */
};

/* ---- bf16 <-> double --------------------------------------------------- */

/* bf16 is the upper half of an IEEE binary32 word, so widening is exact. */
double oracle_bf16_to_f64(uint16_t bits)
{
    uint32_t w = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &w, sizeof f);
    return (double)f;
}

/* Round a double to the nearest bf16 value, ties to even, straight from the
 * double (no intermediate float rounding). bf16 keeps 8 significant bits and
 * the binary32 exponent range: normal numbers are spaced 2^(E-7) within the
 * binade [2^E, 2^(E+1)), subnormals are spaced 2^-133, and the largest finite
 * value is (2 - 2^-7) * 2^127. Scaling by the spacing is exact, nearbyint()
 * rounds half to even under the default rounding mode, and scaling back is
 * exact; what is left is an exact bf16 value that is re-encoded. */
uint16_t oracle_f64_to_bf16_rne(double x)
{
    uint16_t sign = signbit(x) ? 0x8000u : 0u;
    if (isnan(x)) return (uint16_t)(sign | 0x7FC0u);
    double a = fabs(x);
    if (a == 0.0) return sign;
    if (isinf(a)) return (uint16_t)(sign | 0x7F80u);

    int e2;
    (void)frexp(a, &e2);               /* a = f * 2^e2, f in [0.5, 1) */
    int E = e2 - 1;                    /* a in [2^E, 2^(E+1)) */
    int spacing_exp = (E < -126) ? -133 : E - 7;
    double q = ldexp(a, -spacing_exp); /* exact */
    double r = nearbyint(q);           /* round half to even */
    double v = ldexp(r, spacing_exp);  /* exact */

    const double bf16_max = ldexp(255.0, 120); /* (2 - 2^-7) * 2^127 */
    if (v > bf16_max) return (uint16_t)(sign | 0x7F80u);

    float f = (float)v; /* exact: v has at most 8 significant bits */
    uint32_t w;
    memcpy(&w, &f, sizeof w);
    return (uint16_t)(sign | (uint16_t)(w >> 16));
}

/* ---- attn.qk_norm ------------------------------------------------------- */

/* Model Spec, "Compute-graph nodes", rmsnorm row:
 *   y[i] = x[i] / sqrt(sum_j x[j]^2 / H + eps) * w[i]
 * with the sum running j = 0 .. n-1 in index order. */
void oracle_rmsnorm(const double *x, const double *w, int n, double eps, double *y)
{
    double ss = 0.0;
    for (int j = 0; j < n; ++j) ss += x[j] * x[j];
    double r = sqrt(ss / (double)n + eps);
    for (int i = 0; i < n; ++i) y[i] = x[i] / r * w[i];
}

/* ---- attn.rope ---------------------------------------------------------- */

/* Model Spec, "Compute-graph nodes", attn.rope row: rotate the pair
 * (x[i], x[i + d/2]) for i < d/2 by the angle pos * theta^(-2i/d); with
 * d = rot = 128 every coordinate is in a pair, so none is left unchanged.
 * The rotation is the counter-clockwise one (the reading named above). */
void oracle_rope(double *x, int d, double pos, double theta)
{
    int half = d / 2;
    for (int i = 0; i < half; ++i) {
        double angle = pos * pow(theta, -2.0 * (double)i / (double)d);
        double c = cos(angle), s = sin(angle);
        double a = x[i], b = x[i + half];
        x[i] = a * c - b * s;
        x[i + half] = b * c + a * s;
    }
}

/* ---- attn.core (decodeGQA) for one query head --------------------------- */

/* Model Spec, "Compute-graph nodes", attn.core row:
 *   o = sum_{s < L} softmax_s(<q, k_s> / sqrt(128)) v_s
 * k_s and v_s are kv head `kvh` of logical slot s, read through the block
 * table from the paged cache. The softmax is evaluated as exp(z - max z) / sum,
 * which equals the definition by the softmax_shift theorem (Supported models
 * page, "Facts proved about the specs"). `scores` must hold L doubles. */
void oracle_decode_head(const double *q, int L, const int32_t *bt_row,
                        const uint16_t *k_cache, const uint16_t *v_cache,
                        int kvh, double *scores, double *o)
{
    const double scale = 1.0 / sqrt((double)ORC_HEAD_DIM);
    double m = -INFINITY;
    for (int s = 0; s < L; ++s) {
        size_t base = (size_t)bt_row[s / ORC_PAGE] * ORC_PAGE_ELEMS
                    + (size_t)(s % ORC_PAGE) * ORC_KV_WIDTH + (size_t)kvh * ORC_HEAD_DIM;
        double dot = 0.0;
        for (int d = 0; d < ORC_HEAD_DIM; ++d)
            dot += q[d] * oracle_bf16_to_f64(k_cache[base + d]);
        scores[s] = dot * scale;
        if (scores[s] > m) m = scores[s];
    }
    double z = 0.0;
    for (int s = 0; s < L; ++s) {
        scores[s] = exp(scores[s] - m);
        z += scores[s];
    }
    for (int d = 0; d < ORC_HEAD_DIM; ++d) o[d] = 0.0;
    for (int s = 0; s < L; ++s) {
        size_t base = (size_t)bt_row[s / ORC_PAGE] * ORC_PAGE_ELEMS
                    + (size_t)(s % ORC_PAGE) * ORC_KV_WIDTH + (size_t)kvh * ORC_HEAD_DIM;
        double p = scores[s] / z;
        for (int d = 0; d < ORC_HEAD_DIM; ++d)
            o[d] += p * oracle_bf16_to_f64(v_cache[base + d]);
    }
}

/* ---- threads -------------------------------------------------------------- */

/* Threads the attention loop of the step may use (default 1). Test and
 * baseline infrastructure only: the timed CPU baseline reports both one
 * thread and every host core. */
static int g_threads = 1;

void oracle_set_threads(int n) { g_threads = n < 1 ? 1 : (n > 256 ? 256 : n); }

int oracle_get_threads(void) { return g_threads; }

/* ---- the whole step ------------------------------------------------------ */

/* The attention step for a batch with T new tokens per sequence, in the
 * order the specification gives it: for every sequence and new token, norm
 * and rotate q and k, append the new k and v to the cache; then, over the
 * cache as it stands after the appends, attend causally: new token t of
 * sequence b sits in cache slot L - T + t (L = seq_lens[b] counts the new
 * tokens) and its query reads slots 0 .. L - T + t (Model Spec, "What to
 * watch for": every layer is full causal attention; "At a glance": T tokens;
 * Supported models, forward_causal). T = 1 is decodeGQA (attn.core).
 * num_q_heads query heads share the 8 kv heads: 16 for Qwen3-0.6B and 1.7B,
 * 32 for 4B/8B, 40 for 14B, 64 for 32B (nnterp qwen3, "Grouped-query
 * attention, with 128-wide heads on every size"); query head h reads kv head
 * h / (num_q_heads / 8), which is h / 2 for 0.6B (Model Spec attn.core).
 *
 *   qkv          bf16 [B][T][(num_q_heads + 16) * 128], q | k | v, head-major
 *   q_norm_w     bf16 [128], k_norm_w bf16 [128] (one gain for every head)
 *   seq_lens     [B], counts the new tokens, T <= L <= 40960 and <= 16*bt_stride
 *   positions    [B] RoPE position of each sequence's first new token (token
 *                t has positions[b] + t), or NULL for L - T
 *   block_table  [B][bt_stride] page ids; entries past ceil(L/16) are not read
 *   k_cache, v_cache  bf16 [num_pages][16][8][128], updated in place
 *   o            double [B][T][num_q_heads][128] (output)
 *   q_out        double [B][T][num_q_heads][128] or NULL: q after norm and RoPE
 *   k_out        double [B][T][8][128] or NULL: new k after norm and RoPE,
 *                before its rounding to bf16
 *
 * Returns 0, ORC_ERR_ARG, or ORC_ERR_BOUNDS (nothing is written then). */
int oracle_append_and_attend_tokens(const uint16_t *qkv, const uint16_t *q_norm_w,
                                    const uint16_t *k_norm_w, const int32_t *seq_lens,
                                    const int32_t *positions, const int32_t *block_table,
                                    int bt_stride, uint16_t *k_cache, uint16_t *v_cache,
                                    int num_pages, double *o, int B, int T, int num_q_heads,
                                    double rope_theta, double rms_eps, double *q_out,
                                    double *k_out)
{
    if (!qkv || !q_norm_w || !k_norm_w || !seq_lens || !block_table || !k_cache ||
        !v_cache || !o || B < 1 || B > ORC_MAX_BATCH || bt_stride < 1 || num_pages < 1 ||
        T < 1 || T > ORC_MAX_SEQ ||
        num_q_heads < ORC_NUM_KV_HEADS || num_q_heads % ORC_NUM_KV_HEADS != 0 || num_q_heads > 64)
        return ORC_ERR_ARG;
    const int group = num_q_heads / ORC_NUM_KV_HEADS;
    const int q_width = num_q_heads * ORC_HEAD_DIM;
    const size_t row_width = (size_t)q_width + 2 * ORC_KV_WIDTH;

    /* Validate every index the step will use before touching anything. */
    for (int b = 0; b < B; ++b) {
        int L = seq_lens[b];
        if (L < T || L > ORC_MAX_SEQ || L > ORC_PAGE * bt_stride) return ORC_ERR_BOUNDS;
        for (int p = 0; p < (L + ORC_PAGE - 1) / ORC_PAGE; ++p) {
            int32_t id = block_table[(size_t)b * bt_stride + p];
            if (id < 0 || id >= num_pages) return ORC_ERR_BOUNDS;
        }
    }

    double wq[ORC_HEAD_DIM], wk[ORC_HEAD_DIM];
    for (int i = 0; i < ORC_HEAD_DIM; ++i) {
        wq[i] = oracle_bf16_to_f64(q_norm_w[i]);
        wk[i] = oracle_bf16_to_f64(k_norm_w[i]);
    }

    double *q_all = (double *)malloc(sizeof(double) * (size_t)B * T * q_width);
    if (!q_all) return ORC_ERR_ARG;

    /* Norm, rotation and append, sequence by sequence, token by token. */
    for (int b = 0; b < B; ++b) {
        int L = seq_lens[b];
        for (int t = 0; t < T; ++t) {
            const uint16_t *row = qkv + ((size_t)b * T + t) * row_width;
            int slot = L - T + t;
            double pos = positions ? (double)positions[b] + t : (double)slot;
            double x[ORC_HEAD_DIM], y[ORC_HEAD_DIM];

            for (int h = 0; h < num_q_heads; ++h) {
                for (int i = 0; i < ORC_HEAD_DIM; ++i)
                    x[i] = oracle_bf16_to_f64(row[h * ORC_HEAD_DIM + i]);
                oracle_rmsnorm(x, wq, ORC_HEAD_DIM, rms_eps, y);
                oracle_rope(y, ORC_HEAD_DIM, pos, rope_theta);
                memcpy(q_all + (((size_t)b * T + t) * num_q_heads + h) * ORC_HEAD_DIM, y, sizeof y);
            }

            int32_t page = block_table[(size_t)b * bt_stride + slot / ORC_PAGE];
            size_t slot_base = (size_t)page * ORC_PAGE_ELEMS + (size_t)(slot % ORC_PAGE) * ORC_KV_WIDTH;
            for (int j = 0; j < ORC_NUM_KV_HEADS; ++j) {
                for (int i = 0; i < ORC_HEAD_DIM; ++i)
                    x[i] = oracle_bf16_to_f64(row[q_width + j * ORC_HEAD_DIM + i]);
                oracle_rmsnorm(x, wk, ORC_HEAD_DIM, rms_eps, y);
                oracle_rope(y, ORC_HEAD_DIM, pos, rope_theta);
                if (k_out)
                    memcpy(k_out + (((size_t)b * T + t) * ORC_NUM_KV_HEADS + j) * ORC_HEAD_DIM, y, sizeof y);
                for (int i = 0; i < ORC_HEAD_DIM; ++i) {
                    k_cache[slot_base + (size_t)j * ORC_HEAD_DIM + i] = oracle_f64_to_bf16_rne(y[i]);
                    /* v has no norm and no rotation: its bits are copied. */
                    v_cache[slot_base + (size_t)j * ORC_HEAD_DIM + i] =
                        row[q_width + ORC_KV_WIDTH + j * ORC_HEAD_DIM + i];
                }
            }
        }
    }

    /* Causal attention over the cache as it stands after every append: new
     * token t reads the L - T + t + 1 slots up to and including its own.
     * Every (sequence, token, head) row is computed on its own, by the same
     * sequential code whatever the thread count (oracle_set_threads), so the
     * result does not depend on it. */
    int max_L = 0;
    for (int b = 0; b < B; ++b) if (seq_lens[b] > max_L) max_L = seq_lens[b];
    const int nthreads = g_threads;
    double *scores = (double *)malloc(sizeof(double) * (size_t)max_L * (size_t)nthreads);
    if (!scores) { free(q_all); return ORC_ERR_ARG; }
    const long rows = (long)B * T * num_q_heads;
#ifdef _OPENMP
#pragma omp parallel for num_threads(nthreads) schedule(dynamic, 1) if (nthreads > 1)
#endif
    for (long r = 0; r < rows; ++r) {
        const int h = (int)(r % num_q_heads);
        const int t = (int)((r / num_q_heads) % T);
        const int b = (int)(r / ((long)num_q_heads * T));
        const int visible = seq_lens[b] - T + t + 1;
#ifdef _OPENMP
        double *sc = scores + (size_t)omp_get_thread_num() * (size_t)max_L;
#else
        double *sc = scores;
#endif
        oracle_decode_head(q_all + (size_t)r * ORC_HEAD_DIM, visible, block_table + (size_t)b * bt_stride,
                           k_cache, v_cache, h / group, sc, o + (size_t)r * ORC_HEAD_DIM);
    }
    if (q_out) memcpy(q_out, q_all, sizeof(double) * (size_t)B * T * q_width);
    free(scores);
    free(q_all);
    return ORC_OK;
}

/* One new token per sequence (decodeGQA, Model Spec attn.core). */
int oracle_append_and_attend_gqa(const uint16_t *qkv, const uint16_t *q_norm_w,
                                 const uint16_t *k_norm_w, const int32_t *seq_lens,
                                 const int32_t *positions, const int32_t *block_table,
                                 int bt_stride, uint16_t *k_cache, uint16_t *v_cache,
                                 int num_pages, double *o, int B, int num_q_heads,
                                 double rope_theta, double rms_eps, double *q_out,
                                 double *k_out)
{
    return oracle_append_and_attend_tokens(qkv, q_norm_w, k_norm_w, seq_lens, positions, block_table,
                                           bt_stride, k_cache, v_cache, num_pages, o, B, 1, num_q_heads,
                                           rope_theta, rms_eps, q_out, k_out);
}

/* The Qwen3-0.6B step: 16 query heads over 8 kv heads (Model Spec attn.core). */
int oracle_append_and_attend(const uint16_t *qkv, const uint16_t *q_norm_w,
                             const uint16_t *k_norm_w, const int32_t *seq_lens,
                             const int32_t *positions, const int32_t *block_table,
                             int bt_stride, uint16_t *k_cache, uint16_t *v_cache,
                             int num_pages, double *o, int B, double rope_theta,
                             double rms_eps, double *q_out, double *k_out)
{
    return oracle_append_and_attend_gqa(qkv, q_norm_w, k_norm_w, seq_lens, positions, block_table,
                                        bt_stride, k_cache, v_cache, num_pages, o, B,
                                        ORC_NUM_Q_HEADS, rope_theta, rms_eps, q_out, k_out);
}

/* ---- input_norm + attn.qkv_proj (the step's input) ------------------------ */

/* The two nodes before the attention step, in the order of the Model Spec's
 * "Compute-graph nodes" table: input_norm (rmsnorm over H = hidden, eps) and
 * attn.qkv_proj (linear, y[t,n] = sum_k x[t,k] * w[n,k], K = hidden,
 * N = (num_q_heads + 16) * 128, no bias: the parameter count leaves none).
 * Rows t are the B sequences' new tokens.
 *
 *   x        bf16 [B][K]   the hidden state entering the layer
 *   norm_w   bf16 [K]      input_norm gain
 *   w        bf16 [N][K]   qkv_proj weight, row n = output feature n
 *   y_out    double [B][N] the exact (double) projection, or NULL
 *   y_bits   bf16 [B][N]   y rounded once to bf16 (nearest-even), or NULL
 *
 * Nothing is rounded before y (the normalised x stays double). The sum over
 * k runs in index order. Returns 0 or ORC_ERR_ARG. */
int oracle_input_norm_qkv_proj(const uint16_t *x, const uint16_t *norm_w, const uint16_t *w,
                               int B, int K, int N, double eps, double *y_out, uint16_t *y_bits)
{
    if (!x || !norm_w || !w || B < 1 || K < 1 || N < 1 || !(eps >= 0.0) || (!y_out && !y_bits))
        return ORC_ERR_ARG;
    double *g = (double *)malloc(sizeof(double) * (size_t)K);
    double *row = (double *)malloc(sizeof(double) * (size_t)K);
    double *xn = (double *)malloc(sizeof(double) * (size_t)K);
    if (!g || !row || !xn) { free(g); free(row); free(xn); return ORC_ERR_ARG; }
    for (int k = 0; k < K; ++k) g[k] = oracle_bf16_to_f64(norm_w[k]);
    for (int b = 0; b < B; ++b) {
        for (int k = 0; k < K; ++k) row[k] = oracle_bf16_to_f64(x[(size_t)b * K + k]);
        oracle_rmsnorm(row, g, K, eps, xn);                        /* input_norm */
        for (int n = 0; n < N; ++n) {                              /* attn.qkv_proj */
            const uint16_t *wn = w + (size_t)n * K;
            double acc = 0.0;
            for (int k = 0; k < K; ++k) acc += xn[k] * oracle_bf16_to_f64(wn[k]);
            if (y_out) y_out[(size_t)b * N + n] = acc;
            if (y_bits) y_bits[(size_t)b * N + n] = oracle_f64_to_bf16_rne(acc);
        }
    }
    free(g);
    free(row);
    free(xn);
    return 0;
}

/* ---- attn.o_proj (the step's consumer) ----------------------------------- */

/* The node after the attention core in the Model Spec's "Compute-graph
 * nodes" table: attn.o_proj, a linear map y[t,n] = sum_k x[t,k] * w[n,k] with
 * K = 2048, N = 1024 for Qwen3-0.6B and no bias. Its input x[t] is the core's
 * output o[b] of [16][128] read as one row of 16 * 128 (the "Tensors of the
 * main nodes" table gives attn.core's o [B, 16, 128] and attn.o_proj's
 * x [T, 2048]).
 *
 *   x        bf16 [B][K]   the attention output rows
 *   w        bf16 [N][K]   o_proj weight, row n = output feature n
 *   y_out    double [B][N] the exact (double) product, or NULL
 *   y_bits   bf16 [B][N]   y rounded once to bf16 (nearest-even), or NULL
 *
 * The sum over k runs in index order. Returns 0 or ORC_ERR_ARG. */
int oracle_o_proj(const uint16_t *x, const uint16_t *w, int B, int K, int N, double *y_out, uint16_t *y_bits)
{
    if (!x || !w || B < 1 || K < 1 || N < 1 || (!y_out && !y_bits))
        return ORC_ERR_ARG;
    for (int b = 0; b < B; ++b) {
        const uint16_t *xb = x + (size_t)b * K;
        for (int n = 0; n < N; ++n) {
            const uint16_t *wn = w + (size_t)n * K;
            double acc = 0.0;
            for (int k = 0; k < K; ++k) acc += oracle_bf16_to_f64(xb[k]) * oracle_bf16_to_f64(wn[k]);
            if (y_out) y_out[(size_t)b * N + n] = acc;
            if (y_bits) y_bits[(size_t)b * N + n] = oracle_f64_to_bf16_rne(acc);
        }
    }
    return 0;
}

/* ---- array forms of the conversions, for the tests ---------------------- */

void oracle_bf16_to_f64_array(const uint16_t *in, double *out, size_t n)
{
    for (size_t i = 0; i < n; ++i) out[i] = oracle_bf16_to_f64(in[i]);
}

void oracle_f64_to_bf16_rne_array(const double *in, uint16_t *out, size_t n)
{
    for (size_t i = 0; i < n; ++i) out[i] = oracle_f64_to_bf16_rne(in[i]);
}
