/*
 * CPU oracle for the pack -> attend -> unpack pipeline of
 * "Dispatch-Aware Ragged Attention for Pruned Vision Transformers".
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, fp64 statement of
 * what the pipeline computes.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load it; the product path never does.  It
 * shares no code, header, table or helper with the CUDA library: every step
 * (survivor bookkeeping, byte copies, format decoding, attention) is written
 * out here on its own.
 *
 * Sources, by page and section:
 *  - survivor bookkeeping and the packed layout: radpulse article, section
 *    "Integrated pack pipeline, 2.24x end-to-end" (cu_seqlens is computed
 *    first, survivors are copied into one contiguous flat tensor, the CLS
 *    token is extracted at the end), and its section on the FA2 dispatch
 *    ceiling (survivors packed into a contiguous ragged buffer, varlen API);
 *  - attention: abstract (bidirectional attention kernel over the ragged
 *    sequences) and the radpulse section "Bypassing the binding" (no causal
 *    mask, no KV cache): for each sequence b and head h,
 *        O = softmax(scale * Q K^T) V   over the L_b rows of sequence b.
 *    The softmax scale 1/sqrt(64) is the usual one; the pages do not print it;
 *  - keep-mask producers (Threshold-l2, score top-k): radpulse article,
 *    section "Integrated pack pipeline" (the pipeline serves any pruning
 *    method); their rules are readings, stated where they are defined below.
 *
 * Conventions (readings of the pages where they are silent):
 *  - index 0 (CLS) of every image is kept whatever the mask says;
 *  - any nonzero mask byte means "keep";
 *  - a packed sequence keeps ascending original token order, so CLS is the
 *    first row of every packed sequence;
 *  - scatter-unpack writes kept rows only and leaves dropped rows untouched.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -shared -fPIC -pthread ragged_oracle.c -lm
 * (no fast-math, no contraction into fused multiply-adds).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

enum { OR_F16 = 0, OR_BF16 = 1, OR_F32 = 2, OR_F64 = 3 };

/* ------------------------------------------------------------------------ */
/* Survivor bookkeeping: keep mask -> cu_seqlens and source rows.            */
/* ------------------------------------------------------------------------ */

static int is_kept(const uint8_t *keep, int64_t L_full, int64_t b, int64_t j)
{
    if (j == 0)
        return 1; /* CLS is always kept */
    return keep[b * L_full + j] != 0;
}

/* cu[0] = 0, cu[b+1] = cu[b] + (number of kept tokens of image b).
 * src_idx (optional) receives, for every packed row t, the flat dense row
 * b * L_full + j it comes from.  Returns T = cu[B]. */
int64_t oracle_seqlens(const uint8_t *keep, int64_t B, int64_t L_full,
                       int32_t *cu, int32_t *src_idx)
{
    int64_t t = 0;
    cu[0] = 0;
    for (int64_t b = 0; b < B; ++b) {
        for (int64_t j = 0; j < L_full; ++j) {
            if (is_kept(keep, L_full, b, j)) {
                if (src_idx)
                    src_idx[t] = (int32_t)(b * L_full + j);
                ++t;
            }
        }
        cu[b + 1] = (int32_t)t;
    }
    return t;
}

/* Pack: packed row t = dense row of the t-th survivor, bytes copied as is. */
int64_t oracle_pack(const uint8_t *dense, int64_t B, int64_t L_full, int64_t row_bytes,
                    const uint8_t *keep, uint8_t *packed, int32_t *cu)
{
    int64_t t = 0;
    cu[0] = 0;
    for (int64_t b = 0; b < B; ++b) {
        for (int64_t j = 0; j < L_full; ++j) {
            if (is_kept(keep, L_full, b, j)) {
                memcpy(packed + t * row_bytes, dense + (b * L_full + j) * row_bytes,
                       (size_t)row_bytes);
                ++t;
            }
        }
        cu[b + 1] = (int32_t)t;
    }
    return t;
}

/* CLS extraction: cls row b = packed row cu[b]. */
void oracle_unpack_cls(const uint8_t *packed, const int32_t *cu, int64_t B,
                       int64_t row_bytes, uint8_t *cls)
{
    for (int64_t b = 0; b < B; ++b)
        memcpy(cls + b * row_bytes, packed + (int64_t)cu[b] * row_bytes, (size_t)row_bytes);
}

/* Scatter back: dense_out[b, j] = packed row of survivor (b, j); rows of
 * dropped tokens are not written. */
void oracle_unpack(const uint8_t *packed, const uint8_t *keep, int64_t B, int64_t L_full,
                   int64_t row_bytes, uint8_t *dense_out)
{
    int64_t t = 0;
    for (int64_t b = 0; b < B; ++b) {
        for (int64_t j = 0; j < L_full; ++j) {
            if (is_kept(keep, L_full, b, j)) {
                memcpy(dense_out + (b * L_full + j) * row_bytes, packed + t * row_bytes,
                       (size_t)row_bytes);
                ++t;
            }
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Exact widening of the stored formats to double.                          */
/* ------------------------------------------------------------------------ */

/* IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
static double half_to_double(uint16_t h)
{
    int sign = h >> 15;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)f, -24);                 /* zero or subnormal: f * 2^-24 */
    else if (e == 31)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(0x400 | f), e - 25);    /* (1024 + f) * 2^(e - 15 - 10) */
    return sign ? -v : v;
}

/* bfloat16 is the upper half of an IEEE binary32. */
static double bfloat_to_double(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float x;
    memcpy(&x, &u, sizeof x);
    return (double)x;
}

static double load_elem(const void *base, int dtype, int64_t idx)
{
    switch (dtype) {
    case OR_F16: return half_to_double(((const uint16_t *)base)[idx]);
    case OR_BF16: return bfloat_to_double(((const uint16_t *)base)[idx]);
    case OR_F32: return (double)((const float *)base)[idx];
    default: return ((const double *)base)[idx];
    }
}

void oracle_decode(const void *src, int dtype, int64_t n, double *dst)
{
    for (int64_t i = 0; i < n; ++i)
        dst[i] = load_elem(src, dtype, i);
}

/* ------------------------------------------------------------------------ */
/* Attention over each packed sequence, in double.                          */
/* ------------------------------------------------------------------------ */

typedef struct {
    const void *q, *k, *v;
    int dtype;
    int64_t tok_stride, head_stride;     /* elements */
    const int32_t *cu;
    const int32_t *seqs;                 /* sequences to compute */
    int64_t n_seqs, H, d;
    double scale;
    double *out;                         /* [T, H, d] doubles */
    int64_t next;                        /* shared work counter */
    int failed;
} attn_job;

/* One (sequence, head): for every query row i,
 *   s_j = scale * <q_i, k_j>,  m = max_j s_j,
 *   p_j = exp(s_j - m) / sum_j' exp(s_j' - m),
 *   o_i = sum_j p_j v_j. */
static int attend_one(attn_job *J, int64_t b, int64_t h)
{
    const int64_t start = J->cu[b];
    const int64_t L = (int64_t)J->cu[b + 1] - start;
    const int64_t d = J->d;
    if (L <= 0)
        return 0;
    double *Q = malloc(sizeof(double) * (size_t)(L * d));
    double *K = malloc(sizeof(double) * (size_t)(L * d));
    double *V = malloc(sizeof(double) * (size_t)(L * d));
    double *s = malloc(sizeof(double) * (size_t)L);
    if (!Q || !K || !V || !s) {
        free(Q); free(K); free(V); free(s);
        return -1;
    }
    for (int64_t i = 0; i < L; ++i) {
        for (int64_t c = 0; c < d; ++c) {
            int64_t idx = (start + i) * J->tok_stride + h * J->head_stride + c;
            Q[i * d + c] = load_elem(J->q, J->dtype, idx);
            K[i * d + c] = load_elem(J->k, J->dtype, idx);
            V[i * d + c] = load_elem(J->v, J->dtype, idx);
        }
    }
    for (int64_t i = 0; i < L; ++i) {
        double m = -INFINITY;
        for (int64_t j = 0; j < L; ++j) {
            double dot = 0.0;
            for (int64_t c = 0; c < d; ++c)
                dot += Q[i * d + c] * K[j * d + c];
            s[j] = J->scale * dot;
            if (s[j] > m)
                m = s[j];
        }
        double l = 0.0;
        for (int64_t j = 0; j < L; ++j) {
            s[j] = exp(s[j] - m);
            l += s[j];
        }
        double *o = J->out + ((start + i) * J->H + h) * d;
        for (int64_t c = 0; c < d; ++c) {
            double acc = 0.0;
            for (int64_t j = 0; j < L; ++j)
                acc += s[j] * V[j * d + c];
            o[c] = acc / l;
        }
    }
    free(Q); free(K); free(V); free(s);
    return 0;
}

static void *attn_worker(void *arg)
{
    attn_job *J = (attn_job *)arg;
    for (;;) {
        int64_t item = __atomic_fetch_add(&J->next, 1, __ATOMIC_RELAXED);
        if (item >= J->n_seqs * J->H)
            break;
        int64_t b = J->seqs[item / J->H];
        int64_t h = item % J->H;
        if (attend_one(J, b, h) != 0)
            __atomic_store_n(&J->failed, 1, __ATOMIC_RELAXED);
    }
    return NULL;
}

int oracle_num_cores(void)
{
    long n = sysconf(_SC_NPROCESSORS_ONLN);
    return n > 0 ? (int)n : 1;
}

/* q, k, v: element pointers of the packed arrays (rows cu[b]..cu[b+1]-1 of
 * sequence b), token stride and head stride in elements, all three sharing the
 * same strides (separate arrays or views into one fused array).
 * seqs/n_seqs: the sequences to compute (NULL: all B); out rows of other
 * sequences are left untouched.  threads <= 0: one per online core.
 * Returns 0, or -1 if a buffer could not be allocated. */
int oracle_attention(const void *q, const void *k, const void *v, int dtype,
                     int64_t tok_stride, int64_t head_stride, const int32_t *cu, int64_t B,
                     int64_t H, int64_t d, double scale, const int32_t *seqs, int64_t n_seqs,
                     double *out, int threads)
{
    int32_t *all = NULL;
    if (!seqs) {
        all = malloc(sizeof(int32_t) * (size_t)(B > 0 ? B : 1));
        if (!all)
            return -1;
        for (int64_t b = 0; b < B; ++b)
            all[b] = (int32_t)b;
        seqs = all;
        n_seqs = B;
    }
    attn_job J = {q, k, v, dtype, tok_stride, head_stride, cu, seqs, n_seqs, H, d,
                  scale, out, 0, 0};
    if (threads <= 0)
        threads = oracle_num_cores();
    if (threads == 1) {
        attn_worker(&J);
    } else {
        pthread_t *tid = malloc(sizeof(pthread_t) * (size_t)threads);
        int started = 0;
        if (tid) {
            for (; started < threads - 1; ++started)
                if (pthread_create(&tid[started], NULL, attn_worker, &J) != 0)
                    break;
        }
        attn_worker(&J); /* the calling thread works too; finishes any leftovers */
        for (int i = 0; i < started; ++i)
            pthread_join(tid[i], NULL);
        free(tid);
    }
    free(all);
    return J.failed ? -1 : 0;
}


/* ------------------------------------------------------------------------ */
/* Keep-mask producers.  The radpulse article ("Integrated pack pipeline")   */
/* notes that the pipeline is independent of the pruning method and names    */
/* Threshold-l2 among the methods it serves; a score top-k is the other      */
/* common selector.  The pages give neither rule in detail; the readings are: */
/*  - Threshold-l2: token j of image b is kept when the Euclidean norm of its */
/*    feature vector is at least tau;                                        */
/*  - top-k: image b keeps its CLS token and the k_b - 1 other tokens with   */
/*    the highest scores, ties going to the lower index and NaN ranking      */
/*    below every number; k_b is clamped to [1, L_full].                     */
/* CLS (index 0) is always kept, as everywhere in the pipeline.              */
/* ------------------------------------------------------------------------ */

/* Does score a (token ia) rank before score b (token ib)? */
static int ranks_before(float a, int64_t ia, float b, int64_t ib)
{
    int na = isnan(a) != 0, nb = isnan(b) != 0;
    if (na != nb)
        return nb; /* every number ranks before NaN */
    if (!na && a != b)
        return a > b;
    return ia < ib;
}

/* keep [B, L_full] <- the top-k selection above; scores is [B, L_full]. */
void oracle_mask_topk(const float *scores, int64_t B, int64_t L_full, const int32_t *keep_count,
                      uint8_t *keep)
{
    int64_t *order = (int64_t *)malloc(sizeof(int64_t) * (size_t)(L_full > 0 ? L_full : 1));
    for (int64_t b = 0; b < B; ++b) {
        const float *s = scores + b * L_full;
        /* non-CLS tokens in rank order, by insertion */
        int64_t n = 0;
        for (int64_t j = 1; j < L_full; ++j) {
            int64_t pos = n;
            while (pos > 0 && ranks_before(s[j], j, s[order[pos - 1]], order[pos - 1])) {
                order[pos] = order[pos - 1];
                --pos;
            }
            order[pos] = j;
            ++n;
        }
        int64_t k = keep_count[b];
        if (k < 1)
            k = 1;
        if (k > L_full)
            k = L_full;
        memset(keep + b * L_full, 0, (size_t)L_full);
        keep[b * L_full] = 1;
        for (int64_t r = 0; r < k - 1; ++r)
            keep[b * L_full + order[r]] = 1;
    }
    free(order);
}

/* Threshold-l2 on exact values.  Every f16, bf16 and f32 value is an integer
 * multiple of 2^-149 (the smallest f32 subnormal), so every square, and every
 * sum of squares, is an integer multiple of 2^-298.  The sum of squares of a
 * token is therefore held exactly, as that integer, in a little-endian array
 * of 32-bit limbs; with at most 2^24 elements below 2^128 in magnitude it is
 * below 2^578, and 24 limbs (768 bits) hold it.  It is compared with tau^2,
 * also exact, so no rounding and no order of summation enters the decision:
 *     kept  <=>  j == 0  or  sqrt(sum of squares) >= tau.
 * A NaN element makes the norm NaN, which is not >= tau (dropped); an
 * infinite element without a NaN makes it infinite (kept). */
#define L2_UNIT 298  /* the sums count units of 2^-298 */
#define L2_LIMBS 24

/* |v| = m * 2^e with m odd (v finite and nonzero). */
static void odd_parts(double v, uint64_t *m, int *e)
{
    int k;
    const double f = frexp(fabs(v), &k);        /* |v| = f * 2^k, 0.5 <= f < 1 */
    uint64_t mm = (uint64_t)ldexp(f, 53);       /* exact: a double has 53 bits */
    int ee = k - 53;
    while ((mm & 1u) == 0) {
        mm >>= 1;
        ++ee;
    }
    *m = mm;
    *e = ee;
}

/* Bits lo .. lo + 31 of v (zeros outside 0 .. 127; lo may be negative). */
static uint32_t bits32(unsigned __int128 v, int lo)
{
    if (lo <= -32 || lo >= 128)
        return 0;
    if (lo < 0)
        return (uint32_t)(v << (-lo));
    return (uint32_t)(v >> lo);
}

/* acc += v * 2^shift (shift >= 0); the caller makes sure the sum fits. */
static void big_add(uint32_t *acc, unsigned __int128 v, int shift)
{
    uint64_t carry = 0;
    for (int i = 0; i < L2_LIMBS; ++i) {
        const uint64_t sum = (uint64_t)acc[i] + bits32(v, 32 * i - shift) + carry;
        acc[i] = (uint32_t)sum;
        carry = sum >> 32;
    }
}

static int bit_length(unsigned __int128 v)
{
    int n = 0;
    while (v != 0) {
        v >>= 1;
        ++n;
    }
    return n;
}

/* a >= b for two L2_LIMBS-limb integers. */
static int big_ge(const uint32_t *a, const uint32_t *b)
{
    for (int i = L2_LIMBS - 1; i >= 0; --i)
        if (a[i] != b[i])
            return a[i] > b[i];
    return 1;
}

/* Is S * 2^-298 >= tau^2, for tau > 0 finite and S the sum in units? */
static int sum_reaches(const uint32_t *S, double tau)
{
    uint64_t M;
    int E;
    odd_parts(tau, &M, &E);                      /* tau^2 = M^2 * 2^(2E) */
    const unsigned __int128 M2 = (unsigned __int128)M * M;
    const int shift = 2 * E + L2_UNIT;           /* tau^2 = M2 * 2^shift units */
    uint32_t T[L2_LIMBS];
    memset(T, 0, sizeof T);
    if (shift >= 0) {
        if (bit_length(M2) + shift > 32 * L2_LIMBS)
            return 0;                            /* tau^2 >= 2^768 units, above any sum */
        big_add(T, M2, shift);
    } else {
        /* S is a whole number of units: S >= M2 / 2^c  <=>  S >= ceil(M2 / 2^c) */
        const int c = -shift;
        unsigned __int128 q;
        if (c >= 128)
            q = 1;                               /* 0 < M2 / 2^c < 1 */
        else
            q = (M2 >> c) + ((M2 & ((((unsigned __int128)1) << c) - 1)) != 0);
        big_add(T, q, 0);
    }
    return big_ge(S, T);
}

/* keep [B, L_full] <- Threshold-l2 of the tokens of x: token (b, j) is the C
 * elements starting at element (b * L_full + j) * tok_stride. */
void oracle_mask_l2(const void *x, int dtype, int64_t B, int64_t L_full, int64_t C, int64_t tok_stride,
                    double tau, uint8_t *keep)
{
    for (int64_t t = 0; t < B * L_full; ++t) {
        uint32_t S[L2_LIMBS];
        memset(S, 0, sizeof S);
        int has_nan = 0, has_inf = 0;
        for (int64_t c = 0; c < C; ++c) {
            const double v = load_elem(x, dtype, t * tok_stride + c);
            if (isnan(v)) {
                has_nan = 1;
            } else if (isinf(v)) {
                has_inf = 1;
            } else if (v != 0.0) {
                uint64_t m;
                int e;
                odd_parts(v, &m, &e);            /* e >= -149 for every f32 value */
                if (2 * e + L2_UNIT < 0)
                    abort();                     /* not an f16 / bf16 / f32 value */
                big_add(S, (unsigned __int128)m * m, 2 * e + L2_UNIT);
            }
        }
        int kept;
        if (t % L_full == 0)
            kept = 1;                            /* CLS */
        else if (has_nan)
            kept = 0;
        else if (has_inf || !(tau > 0.0))
            kept = 1;                            /* an infinite norm, or tau <= 0 */
        else if (isinf(tau))
            kept = 0;
        else
            kept = sum_reaches(S, tau);
        keep[t] = (uint8_t)kept;
    }
}
