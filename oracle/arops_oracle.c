/*
 * Oracle for the per-token operators of autoregressive speech-model decode.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is a plain, slow, fp64 CPU statement of
 * what the GPU library computes.  Only the test suite, the smoke check and the
 * CPU-baseline leg of the benchmark may load it; the product path never does.
 * It shares no code, header, table or constant with the CUDA library.
 *
 * Every routine takes fp64 copies of the exact values the GPU receives and
 * returns fp64 results; rounding to the output dtype is a separate, explicit
 * step (oracle_round_bf16 / a C cast to float for fp32).
 *
 * Sources (page title, then section):
 *   - "Optimising autoregressive speech models" (research.convozen.ai), §09
 *     "LayerNorm -> RMSNorm": the RMSNorm equation gamma * x / sqrt(mean(x^2)+eps)
 *     and the module that computes it with eps = 1e-6 inside the root, the mean
 *     over the last dimension and a per-channel weight.
 *   - "Open Source: Triton-Kernel-Fusion ..." (news.hada.io topic 27742, de/fr/vi),
 *     section 3: the four fused operators RMSNorm, M-RoPE, Norm+Residual, SwiGLU
 *     (names only).
 *   - forpes.ru post 233929, "Stage 2: RoPE": positions are encoded into Q and K
 *     by a rotation in the complex plane.
 * The exact semantics of Norm+Residual, M-RoPE and SwiGLU are the plainest
 * reading of the workload definitions (rotate-half pairing, contiguous t/h/w
 * sections, textbook inverse frequencies theta^(-2j/D), silu(g) = g/(1+e^-g)).
 *
 * Pins: every routine here is checked by the CPU tests against closed forms,
 * invariants and textbook special cases (see tests/test_oracle_pins.py).
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fPIC -shared (no fast-math, no
 * contraction: each fp64 operation rounds once, in program order).
 * Compiling with -DORACLE_MUTANT=<n> plants one deliberate mistake; the tests use
 * that to show that the pins catch each kind of error.
 */
#include <math.h>
#include <stdint.h>

#ifndef ORACLE_MUTANT
#define ORACLE_MUTANT 0
#endif

/*
 * Row-parallel build.  Compiled with -fopenmp (liboracle_omp.so, the timed
 * multi-core baseline) the loops marked OMP_ROWS split their independent rows,
 * tokens or elements across the host's cores; in the plain build the mark
 * expands to nothing and every loop runs sequentially, exactly as written.
 * Nothing else differs between the two builds.
 */
#ifdef _OPENMP
#include <omp.h>
#define OMP_ROWS _Pragma("omp parallel for schedule(static)")
#else
#define OMP_ROWS
#endif

/* ------------------------------------------------------------------------- */
/* bf16 <-> fp64.                                                             */
/* bf16 is IEEE-754 binary32 with the low 16 mantissa bits removed: 1 sign    */
/* bit, 8 exponent bits (bias 127), 7 stored mantissa bits.                   */
/* ------------------------------------------------------------------------- */

/* Round half to even of a non-negative double to an integer-valued double. */
static double round_half_even(double q)
{
    double fl = floor(q);
    double diff = q - fl; /* exact: q and fl are within one unit of each other */
    if (diff > 0.5)
        return fl + 1.0;
    if (diff < 0.5)
        return fl;
    /* tie: pick the even neighbour */
    return (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
}

/* Round one fp64 value straight to bf16 (round to nearest, ties to even), with
 * no intermediate fp32 rounding.  Returns the 16-bit pattern. */
uint16_t oracle_round_bf16(double v)
{
    uint16_t sign = signbit(v) ? 0x8000u : 0u;
    if (isnan(v))
        return (uint16_t)(sign | 0x7FC0u);
    double a = fabs(v);
    if (a == 0.0)
        return sign;
    if (isinf(a))
        return (uint16_t)(sign | 0x7F80u);

    int e; /* a = m * 2^e with m in [0.5, 1): a lies in [2^(e-1), 2^e) */
    (void)frexp(a, &e);
    int unit_exp = (e - 1 < -126) ? -133 : (e - 1) - 7; /* log2 of one bf16 ulp */
#if ORACLE_MUTANT == 1
    unit_exp += 1; /* planted: one mantissa bit too few */
#endif
    double q = ldexp(a, -unit_exp); /* exact: scaling by a power of two */
    double r = round_half_even(q);

    uint32_t bits;
    if (e - 1 < -126) {
        /* subnormal range: the stored field is r itself; r == 128 carries into
         * the exponent and encodes the smallest normal number, as it should */
        bits = (uint32_t)r;
    } else {
        /* normal range: r in [128, 256]; r == 256 carries into the exponent */
        int32_t biased = (e - 1) + 127;
        bits = ((uint32_t)biased << 7) + ((uint32_t)r - 128u);
        if (bits >= 0x7F80u)
            bits = 0x7F80u; /* rounded past the largest finite value */
    }
    return (uint16_t)(sign | bits);
}

/* Exact value of a bf16 bit pattern. */
double oracle_bf16_value(uint16_t b)
{
    int s = (b >> 15) & 1;
    int ex = (b >> 7) & 0xFF;
    int mant = b & 0x7F;
    double v;
    if (ex == 0)
        v = ldexp((double)mant, -133);
    else if (ex == 0xFF)
        v = mant ? NAN : INFINITY;
    else
        v = ldexp(128.0 + (double)mant, ex - 127 - 7);
    return s ? -v : v;
}

void oracle_round_bf16_array(const double* v, uint16_t* out, int64_t n)
{
    OMP_ROWS
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_round_bf16(v[i]);
}

void oracle_bf16_value_array(const uint16_t* b, double* out, int64_t n)
{
    OMP_ROWS
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_bf16_value(b[i]);
}

/* Round each fp64 value to the activation dtype and back: dtype 0 = fp32,
 * dtype 1 = bf16. */
static double round_to_dtype(double v, int dtype)
{
    if (dtype == 1)
        return oracle_bf16_value(oracle_round_bf16(v));
    return (double)(float)v;
}

/* ------------------------------------------------------------------------- */
/* RMSNorm ("Optimising autoregressive speech models", §09, RMSNorm equation   */
/* and module): y = gamma * x / sqrt(mean(x^2) + eps), mean over the row.      */
/* ------------------------------------------------------------------------- */
void oracle_rmsnorm(const double* x, const double* gamma, double* y,
                    int64_t rows, int64_t hidden, double eps)
{
    OMP_ROWS
    for (int64_t r = 0; r < rows; ++r) {
        const double* xr = x + r * hidden;
        double* yr = y + r * hidden;
        double sumsq = 0.0;
        for (int64_t i = 0; i < hidden; ++i)
            sumsq += xr[i] * xr[i];
        double mean_sq = sumsq / (double)hidden;
#if ORACLE_MUTANT == 2
        double denom = sqrt(mean_sq) + eps; /* planted: eps outside the root */
#elif ORACLE_MUTANT == 3
        double denom = sqrt(sumsq + eps); /* planted: sum instead of mean */
#else
        double denom = sqrt(mean_sq + eps);
#endif
        for (int64_t i = 0; i < hidden; ++i) {
#if ORACLE_MUTANT == 4
            yr[i] = xr[i] / denom; /* planted: gamma dropped */
#else
            yr[i] = gamma[i] * xr[i] / denom;
#endif
        }
    }
}

/* ------------------------------------------------------------------------- */
/* Fused residual add + RMSNorm ("Norm+Residual" of the Triton fusion post,    */
/* section 3): s = x + residual; residual_out = s rounded to the activation    */
/* dtype; y = RMSNorm(residual_out).  That is "add, then norm" as two          */
/* operations on activation-dtype tensors.                                     */
/* ------------------------------------------------------------------------- */
void oracle_add_rmsnorm(const double* x, const double* residual, const double* gamma,
                        double* y, double* residual_out,
                        int64_t rows, int64_t hidden, double eps, int dtype)
{
    OMP_ROWS
    for (int64_t i = 0; i < rows * hidden; ++i) {
#if ORACLE_MUTANT == 5
        residual_out[i] = round_to_dtype(x[i] - residual[i], dtype); /* planted: sign */
#else
        residual_out[i] = round_to_dtype(x[i] + residual[i], dtype);
#endif
    }
#if ORACLE_MUTANT == 6
    oracle_rmsnorm(x, gamma, y, rows, hidden, eps); /* planted: norm of x, not of x+res */
#else
    oracle_rmsnorm(residual_out, gamma, y, rows, hidden, eps);
#endif
}

/* ------------------------------------------------------------------------- */
/* LayerNorm ("Optimising autoregressive speech models", §09, the LayerNorm     */
/* equation): y = gamma * (x - mean) / sqrt(variance + eps) + beta, with the    */
/* mean and the (population) variance taken over the row.                      */
/* ------------------------------------------------------------------------- */
void oracle_layernorm(const double* x, const double* gamma, const double* beta, double* y,
                      int64_t rows, int64_t hidden, double eps)
{
    OMP_ROWS
    for (int64_t r = 0; r < rows; ++r) {
        const double* xr = x + r * hidden;
        double* yr = y + r * hidden;
        double sum = 0.0;
        for (int64_t i = 0; i < hidden; ++i)
            sum += xr[i];
        double mean = sum / (double)hidden;
        double sq = 0.0;
        for (int64_t i = 0; i < hidden; ++i) {
            double d = xr[i] - mean;
            sq += d * d;
        }
#if ORACLE_MUTANT == 13
        double var = sq / (double)(hidden - 1); /* planted: unbiased variance */
#else
        double var = sq / (double)hidden;
#endif
        double denom = sqrt(var + eps);
        for (int64_t i = 0; i < hidden; ++i) {
#if ORACLE_MUTANT == 14
            yr[i] = gamma[i] * (xr[i] - mean) / denom; /* planted: beta dropped */
#else
            yr[i] = gamma[i] * (xr[i] - mean) / denom + beta[i];
#endif
        }
    }
}

/* Residual add + LayerNorm: the same "add, round to the dtype, then norm" as
 * oracle_add_rmsnorm, with LayerNorm as the norm. */
void oracle_add_layernorm(const double* x, const double* residual, const double* gamma,
                          const double* beta, double* y, double* residual_out,
                          int64_t rows, int64_t hidden, double eps, int dtype)
{
    OMP_ROWS
    for (int64_t i = 0; i < rows * hidden; ++i)
        residual_out[i] = round_to_dtype(x[i] + residual[i], dtype);
    oracle_layernorm(residual_out, gamma, beta, y, rows, hidden, eps);
}

/* ------------------------------------------------------------------------- */
/* Multi-section rotary embedding (M-RoPE) on q and k.                          */
/* Rotation of (x[j], x[j + D/2]) by the angle p * theta^(-2j/D), the textbook */
/* RoPE frequency, with the position p taken from row t, h or w of the         */
/* position ids according to which contiguous section the pair index j lies    */
/* in (sections[0] pairs from row t, then sections[1] from row h, then         */
/* sections[2] from row w).  The rotation is a multiplication of the complex   */
/* number x[j] + i*x[j+D/2] by e^(i*angle) (forpes.ru post 233929, Stage 2).   */
/*                                                                             */
/* q: [tokens][n_q_heads][head_dim], k: [tokens][n_k_heads][head_dim],         */
/* pos: [3][tokens] (int32), outputs have the input layouts.                    */
/* ------------------------------------------------------------------------- */
static int section_of(int j, const int32_t sections[3])
{
    if (j < sections[0])
        return 0;
    if (j < sections[0] + sections[1])
        return 1;
    return 2;
}

static void rotate_heads(const double* x, double* out, const int32_t* pos,
                         int64_t tokens, int64_t tok, int heads, int head_dim,
                         const int32_t sections[3], double theta)
{
    int half = head_dim / 2;
    for (int h = 0; h < heads; ++h) {
        const double* xh = x + (tok * heads + h) * (int64_t)head_dim;
        double* oh = out + (tok * heads + h) * (int64_t)head_dim;
        for (int j = 0; j < half; ++j) {
            int sec = section_of(j, sections);
#if ORACLE_MUTANT == 7
            sec = 0; /* planted: every pair takes row t */
#endif
            double p = (double)pos[(int64_t)sec * tokens + tok];
#if ORACLE_MUTANT == 8
            double inv_freq = pow(theta, -2.0 * (double)(j + 1) / (double)head_dim); /* planted: index off by one */
#else
            double inv_freq = pow(theta, -2.0 * (double)j / (double)head_dim);
#endif
            double angle = p * inv_freq;
            double c = cos(angle);
            double s = sin(angle);
            double a = xh[j];
#if ORACLE_MUTANT == 9
            double b = xh[(j + 1) % head_dim]; /* planted: interleaved partner */
#else
            double b = xh[j + half];
#endif
#if ORACLE_MUTANT == 10
            oh[j] = a * c + b * s; /* planted: rotation in the wrong direction */
            oh[j + half] = b * c - a * s;
#else
            oh[j] = a * c - b * s;
            oh[j + half] = b * c + a * s;
#endif
        }
    }
}

void oracle_mrope_qk(const double* q, const double* k, double* q_out, double* k_out,
                     const int32_t* pos, int64_t tokens, int n_q_heads, int n_k_heads,
                     int head_dim, const int32_t sections[3], double theta)
{
    OMP_ROWS
    for (int64_t t = 0; t < tokens; ++t) {
        rotate_heads(q, q_out, pos, tokens, t, n_q_heads, head_dim, sections, theta);
        rotate_heads(k, k_out, pos, tokens, t, n_k_heads, head_dim, sections, theta);
    }
}

/* ------------------------------------------------------------------------- */
/* M-RoPE fused with the KV-cache append ("Optimising autoregressive speech    */
/* models", "Custom Triton kernels", item 3: write the new K, V of a token into */
/* cache[head, position, :]).  q is rotated into q_out; k is rotated and        */
/* written, and v copied, into slot (cache_loc[0][t], cache_loc[1][t]) = (cache */
/* row b, position s) of caches laid out [cache_rows][n_kv_heads][max_seq][D].  */
/* Tokens whose (b, s) fall outside the cache leave it untouched.               */
/* ------------------------------------------------------------------------- */
void oracle_mrope_kv_append(const double* q, const double* k, const double* v, double* q_out,
                            double* k_cache, double* v_cache, const int32_t* pos,
                            const int32_t* cache_loc, int64_t tokens, int n_q_heads,
                            int n_kv_heads, int head_dim, int64_t cache_rows, int64_t max_seq,
                            const int32_t sections[3], double theta, double* k_rot /* T*Hk*D */)
{
    for (int64_t t = 0; t < tokens; ++t) {
        rotate_heads(q, q_out, pos, tokens, t, n_q_heads, head_dim, sections, theta);
        rotate_heads(k, k_rot, pos, tokens, t, n_kv_heads, head_dim, sections, theta);
    }
    for (int64_t t = 0; t < tokens; ++t) {
        int64_t b = cache_loc[t];
        int64_t slot = cache_loc[tokens + t];
#if ORACLE_MUTANT == 17
        int64_t tmp = b; /* planted: row and position swapped */
        b = slot;
        slot = tmp;
#endif
        if (b < 0 || b >= cache_rows || slot < 0 || slot >= max_seq)
            continue;
        for (int h = 0; h < n_kv_heads; ++h) {
            int64_t dst = ((b * n_kv_heads + h) * max_seq + slot) * head_dim;
            int64_t src = (t * n_kv_heads + h) * (int64_t)head_dim;
            for (int d = 0; d < head_dim; ++d) {
                k_cache[dst + d] = k_rot[src + d];
#if ORACLE_MUTANT == 18
                v_cache[dst + d] = k[src + d]; /* planted: k stored as v */
#else
                v_cache[dst + d] = v[src + d];
#endif
            }
        }
    }
}

/* ------------------------------------------------------------------------- */
/* SwiGLU (section 3 of the Triton fusion post, by name): out = silu(g) * u,   */
/* silu(g) = g * sigmoid(g) = g / (1 + e^-g).                                  */
/* ------------------------------------------------------------------------- */
void oracle_swiglu(const double* gate, const double* up, double* out, int64_t n)
{
    OMP_ROWS
    for (int64_t i = 0; i < n; ++i) {
        double g = gate[i];
#if ORACLE_MUTANT == 11
        double silu = g / (1.0 + exp(g)); /* planted: sign of the exponent */
#elif ORACLE_MUTANT == 12
        double silu = 1.0 / (1.0 + exp(-g)); /* planted: sigmoid without the g factor */
#else
        double silu = g / (1.0 + exp(-g));
#endif
        out[i] = silu * up[i];
    }
}

/* ------------------------------------------------------------------------- */
/* Fused softmax + top-k sampling ("Optimising autoregressive speech models",  */
/* "Custom Triton kernels", item 2: scale the logits by 1/temperature, softmax */
/* them and sample from the top k).                                            */
/*                                                                             */
/* Per row: candidates are the k largest logits, ordered by (logit desc, index */
/* asc), so ties go to the lower vocabulary index.  Rank j of that order gets  */
/* the caller's Gumbel(0,1) draw gumbel[row*k + j]; the sampled candidate is   */
/* the one with the largest score fl32(fl32(logit/T) + g) (ties to the lower   */
/* rank) -- Gumbel-max sampling from the top-k softmax.  The score is formed   */
/* with two correctly rounded fp32 operations, the precision the kernel takes  */
/* this integer decision in.  prob_out is the probability of the sampled token */
/* under softmax(logits/T) restricted to the k candidates, in fp64.            */
/* ------------------------------------------------------------------------- */
typedef struct {
    double v;
    int64_t idx;
} cand_t;

/* insertion into a list kept in (v desc, idx asc) order, at most k long */
static void cand_insert(cand_t* list, int* n, int k, double v, int64_t idx)
{
    int pos = *n;
    while (pos > 0 && (list[pos - 1].v < v || (list[pos - 1].v == v && list[pos - 1].idx > idx)))
        --pos;
    if (pos >= k)
        return;
    int last = (*n < k) ? *n : k - 1;
    for (int i = last; i > pos; --i)
        list[i] = list[i - 1];
    list[pos].v = v;
    list[pos].idx = idx;
    if (*n < k)
        ++*n;
}

void oracle_topk_sample(const double* logits, const float* gumbel, int32_t* token_out,
                        double* prob_out, int64_t rows, int64_t vocab, int k, float temperature,
                        cand_t* scratch /* k entries */)
{
    for (int64_t r = 0; r < rows; ++r) {
        const double* lr = logits + r * vocab;
        int n = 0;
        for (int64_t i = 0; i < vocab; ++i)
            cand_insert(scratch, &n, k, lr[i], i);
        /* decision in fp32, as fl(fl(l / T) + g) */
        int best = 0;
        float best_score = 0.0f;
        for (int j = 0; j < n; ++j) {
            volatile float q = (float)scratch[j].v / temperature;
#if ORACLE_MUTANT == 15
            volatile float score = q - gumbel[r * k + j]; /* planted: noise subtracted */
#else
            volatile float score = q + gumbel[r * k + j];
#endif
            if (j == 0 || score > best_score) {
                best = j;
                best_score = score;
            }
        }
        /* probability under the top-k softmax, fp64 */
        double zsum = 0.0;
        for (int j = 0; j < n; ++j)
            zsum += exp((scratch[j].v - scratch[0].v) / (double)temperature);
#if ORACLE_MUTANT == 16
        double p = exp(scratch[best].v - scratch[0].v) / zsum; /* planted: temperature dropped */
#else
        double p = exp((scratch[best].v - scratch[0].v) / (double)temperature) / zsum;
#endif
        token_out[r] = (int32_t)scratch[best].idx;
        prob_out[r] = p;
    }
}

/* Host threads the row-parallel loops use (1 in the plain build). */
int oracle_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Number of the planted mistake this build carries (0 = none). */
int oracle_mutant(void)
{
    return ORACLE_MUTANT;
}
