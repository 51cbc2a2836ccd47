/*
 * oracle/paged_decode_oracle.c -- plain, slow fp64 CPU oracle for single-token
 * decode attention over a paged bf16 KV cache.
 *
 * TEST INFRASTRUCTURE.  Only tests/, __graft_entry__.smoke() and the CPU
 * baseline / reference leg of bench.py may load this library.  It shares no
 * code, header, table or helper with the CUDA library, and the CUDA library
 * never calls it.
 *
 * What it computes, and where that comes from:
 *
 *  - AstrAI commit d565d44c, csrc/kernels/attn_paged_decode.cu (commit log):
 *    decode attention for one new query token per sequence, reading K/V through
 *    a per-sequence page table (entries on the scalar and MMA variants and on
 *    the page-table gather of the Python fallback); query heads share kv heads
 *    (grouped-query attention; the bindings require q_heads % kv_heads == 0);
 *    decode is causal, which for a single query token means it sees every
 *    stored position 0..L-1; split-KV workers each leave a partial output with
 *    its running max and sum (o_part / ml_part) and one combine kernel merges
 *    them.
 *  - The pages name scaled-dot-product attention and the online-softmax /
 *    split-combine scheme but never write them out, so this file writes the
 *    textbook definition they refer to:
 *        s_t  = scale * sum_d q[d] * k_t[d]                 (t < L)
 *        m    = max_t s_t,   w_t = exp(s_t - m),   l = sum_t w_t
 *        out  = sum_t w_t * v_t / l                          (L == 0 -> 0)
 *    and, for a partition of [0, L) into chunks c, the split form
 *        (m_c, l_c, acc_c) over the chunk,  M = max_c m_c over non-empty chunks
 *        out = sum_c e^{m_c - M} acc_c / sum_c e^{m_c - M} l_c.
 *    The split form is an exact re-association of the definition (up to
 *    rounding), which the tests check.
 *
 * Readings taken where the pages are silent (each one also listed in the
 * design notes):
 *  - KV cache logical layout [num_pages, page_size, kv_heads, head_dim] with
 *    free strides (HND storage arrives as a strided view).
 *  - q head h reads kv head floor(h / (Hq / Hkv)).
 *  - token t of sequence b lives in page page_table[b][t / P], slot t % P.
 *  - num_splits = S >= 1 splits sequence b into min(S, n_b) page-aligned chunks
 *    of c = ceil(n_b / min(S, n_b)) pages (n_b = ceil(L_b / P)); the last
 *    chunks may be short or empty.  num_splits = 0 ("auto", ejkernel
 *    PageAttentionConfig.num_splits) does not change the result.
 *
 * Arithmetic: bf16 inputs are widened to double exactly; every product of two
 * bf16 values is exact in double; sums, exp and the division are IEEE double
 * in program order.  No blocking, fusion or reordering beyond the formulas.
 * Rounding to bf16 (round-to-nearest-even) is a separate function.
 *
 * Pins (tests/test_oracle_pins.py): brute-force contiguous attention through a
 * library routine on tiny inputs, closed forms (L = 1, constant K, q = 0,
 * unique-max with a huge scale), a hand-derived golden example, page-table
 * permutation invariance, split/combine invariance, GQA == MHA with repeated
 * KV, and bf16 rounding examples.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct oracle_problem {
    const uint16_t* q;          /* bf16 bits, logical [B, Hq, D]              */
    int64_t q_stride[3];        /* element strides of q                        */
    const uint16_t* k;          /* bf16 bits, logical [NP, P, Hkv, D]         */
    const uint16_t* v;          /* same logical shape and strides as k        */
    int64_t kv_stride[4];       /* element strides: page, slot, head, dim      */
    const int32_t* page_table;  /* [B, MP]                                     */
    int64_t pt_stride[2];
    const int32_t* seq_lens;    /* [B]                                         */
    int32_t batch, num_q_heads, num_kv_heads, head_dim, page_size, num_pages, max_pages;
    double scale;
} oracle_problem;

enum { ORACLE_OK = 0, ORACLE_BAD_ARGS = 1, ORACLE_BAD_PAGE = 2, ORACLE_NO_MEMORY = 3 };

static double bf16_to_double(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Round a double to the nearest bf16 value, ties to even (8 significant bits,
 * 8 exponent bits).  Overflow goes to +-inf, NaN stays NaN, tiny values go to
 * bf16 subnormals / zero. */
uint16_t oracle_round_bf16(double x) {
    if (isnan(x)) return 0x7FC0u;
    uint16_t sign = signbit(x) ? 0x8000u : 0;
    double a = fabs(x);
    if (a == 0.0) return sign;
    /* a = f * 2^e with f in [0.5, 1). bf16 normal numbers: 2^-126 <= a;
     * spacing of the 8-bit significand at exponent e is 2^(e-8); subnormals
     * share the spacing 2^-133. */
    int e;
    frexp(a, &e);
    int spacing_exp = e - 8;
    if (spacing_exp < -133) spacing_exp = -133;
    double units = ldexp(a, -spacing_exp);     /* exact: scaling by a power of 2 */
    double r = nearbyint(units);               /* default mode: ties to even     */
    double y = ldexp(r, spacing_exp);
    if (y > 0x1.FEp127) return sign | 0x7F80u; /* beyond the largest finite bf16 */
    float f = (float)y;                        /* exact: y has <= 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(sign | ((u >> 16) & 0x7FFFu));
}

static int check_problem(const oracle_problem* p) {
    if (!p || !p->q || !p->k || !p->v || !p->page_table || !p->seq_lens) return ORACLE_BAD_ARGS;
    if (p->batch < 0 || p->num_q_heads <= 0 || p->num_kv_heads <= 0 || p->head_dim <= 0) return ORACLE_BAD_ARGS;
    if (p->page_size <= 0 || p->num_pages <= 0 || p->max_pages < 0) return ORACLE_BAD_ARGS;
    if (p->num_q_heads % p->num_kv_heads != 0) return ORACLE_BAD_ARGS;
    return ORACLE_OK;
}

/* address of element d of the K (or V) vector of token t of sequence b, kv head kvh */
static int token_base(const oracle_problem* p, int b, int64_t t, int kvh, int64_t* off) {
    int64_t j = t / p->page_size;
    int64_t slot = t % p->page_size;
    if (j >= p->max_pages) return ORACLE_BAD_PAGE;
    int32_t page = p->page_table[(int64_t)b * p->pt_stride[0] + j * p->pt_stride[1]];
    if (page < 0 || page >= p->num_pages) return ORACLE_BAD_PAGE;
    *off = (int64_t)page * p->kv_stride[0] + slot * p->kv_stride[1] + (int64_t)kvh * p->kv_stride[2];
    return ORACLE_OK;
}

static double logit(const oracle_problem* p, int b, int h, int64_t kbase) {
    double dot = 0.0;
    for (int d = 0; d < p->head_dim; ++d) {
        double qd = bf16_to_double(p->q[(int64_t)b * p->q_stride[0] + (int64_t)h * p->q_stride[1] + (int64_t)d * p->q_stride[2]]);
        double kd = bf16_to_double(p->k[kbase + (int64_t)d * p->kv_stride[3]]);
        dot += qd * kd;
    }
    return p->scale * dot;
}

/* The definition for one (b, h): out[0..D) in double. */
static int attend_definition(const oracle_problem* p, int b, int h, double* out) {
    const int D = p->head_dim;
    const int g = p->num_q_heads / p->num_kv_heads;
    const int kvh = h / g;
    const int64_t L = p->seq_lens[b];
    for (int d = 0; d < D; ++d) out[d] = 0.0;
    if (L <= 0) return ORACLE_OK;
    double* s = (double*)malloc(sizeof(double) * (size_t)L);
    int64_t* base = (int64_t*)malloc(sizeof(int64_t) * (size_t)L);
    if (!s || !base) { free(s); free(base); return ORACLE_NO_MEMORY; }
    int rc = ORACLE_OK;
    /* step 1: logits over every stored position t < L */
    for (int64_t t = 0; t < L && rc == ORACLE_OK; ++t) {
        rc = token_base(p, b, t, kvh, &base[t]);
        if (rc == ORACLE_OK) s[t] = logit(p, b, h, base[t]);
    }
    if (rc == ORACLE_OK) {
        /* step 2: softmax with the max subtracted */
        double m = -INFINITY;
        for (int64_t t = 0; t < L; ++t) m = s[t] > m ? s[t] : m;
        double l = 0.0;
        for (int64_t t = 0; t < L; ++t) { s[t] = exp(s[t] - m); l += s[t]; }
        /* step 3: weighted sum of V, divided by the sum of weights */
        for (int64_t t = 0; t < L; ++t)
            for (int d = 0; d < D; ++d)
                out[d] += s[t] * bf16_to_double(p->v[base[t] + (int64_t)d * p->kv_stride[3]]);
        for (int d = 0; d < D; ++d) out[d] /= l;
    }
    free(s);
    free(base);
    return rc;
}

/* Partial state over tokens [t0, t1) of (b, h): running max m, sum l of
 * exp(s - m), and acc = sum exp(s - m) v.  Empty range -> m = -inf, l = 0. */
static int attend_partial(const oracle_problem* p, int b, int h, int64_t t0, int64_t t1,
                          double* acc, double* m_out, double* l_out) {
    const int D = p->head_dim;
    const int g = p->num_q_heads / p->num_kv_heads;
    const int kvh = h / g;
    for (int d = 0; d < D; ++d) acc[d] = 0.0;
    *m_out = -INFINITY;
    *l_out = 0.0;
    if (t1 <= t0) return ORACLE_OK;
    double m = -INFINITY;
    int64_t off;
    for (int64_t t = t0; t < t1; ++t) {
        int rc = token_base(p, b, t, kvh, &off);
        if (rc) return rc;
        double st = logit(p, b, h, off);
        m = st > m ? st : m;
    }
    double l = 0.0;
    for (int64_t t = t0; t < t1; ++t) {
        token_base(p, b, t, kvh, &off);
        double w = exp(logit(p, b, h, off) - m);
        l += w;
        for (int d = 0; d < D; ++d) acc[d] += w * bf16_to_double(p->v[off + (int64_t)d * p->kv_stride[3]]);
    }
    *m_out = m;
    *l_out = l;
    return ORACLE_OK;
}

/* Combine chunk partials for one (b, h) over token boundaries
 * bounds[0] = 0 < ... < bounds[nb-1] = L (empty chunks allowed). */
static int attend_chunks(const oracle_problem* p, int b, int h, const int64_t* bounds, int nb, double* out) {
    const int D = p->head_dim;
    const int nchunks = nb - 1;
    double* acc = (double*)malloc(sizeof(double) * (size_t)D * (size_t)(nchunks > 0 ? nchunks : 1));
    double* ms = (double*)malloc(sizeof(double) * (size_t)(nchunks > 0 ? nchunks : 1));
    double* ls = (double*)malloc(sizeof(double) * (size_t)(nchunks > 0 ? nchunks : 1));
    if (!acc || !ms || !ls) { free(acc); free(ms); free(ls); return ORACLE_NO_MEMORY; }
    int rc = ORACLE_OK;
    for (int c = 0; c < nchunks && rc == ORACLE_OK; ++c)
        rc = attend_partial(p, b, h, bounds[c], bounds[c + 1], acc + (int64_t)c * D, &ms[c], &ls[c]);
    for (int d = 0; d < D; ++d) out[d] = 0.0;
    if (rc == ORACLE_OK) {
        double M = -INFINITY;
        for (int c = 0; c < nchunks; ++c)
            if (ls[c] > 0.0 && ms[c] > M) M = ms[c];
        if (M != -INFINITY) {
            double den = 0.0;
            for (int c = 0; c < nchunks; ++c) {
                if (ls[c] <= 0.0) continue;  /* an empty chunk adds nothing */
                double w = exp(ms[c] - M);
                den += w * ls[c];
                for (int d = 0; d < D; ++d) out[d] += w * acc[(int64_t)c * D + d];
            }
            for (int d = 0; d < D; ++d) out[d] /= den;
        }
    }
    free(acc);
    free(ms);
    free(ls);
    return rc;
}

static int run_rows(const oracle_problem* p, const int32_t* bh, int64_t nrows, double* out, int nthreads,
                    int mode, int num_splits) {
    int rc = check_problem(p);
    if (rc) return rc;
    const int D = p->head_dim;
    int err = ORACLE_OK;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
#endif
    for (int64_t r = 0; r < nrows; ++r) {
        int b, h;
        if (bh) { b = bh[2 * r]; h = bh[2 * r + 1]; }
        else { b = (int)(r / p->num_q_heads); h = (int)(r % p->num_q_heads); }
        int lrc = ORACLE_OK;
        if (b < 0 || b >= p->batch || h < 0 || h >= p->num_q_heads) {
            lrc = ORACLE_BAD_ARGS;
        } else if (mode == 0) {
            lrc = attend_definition(p, b, h, out + r * D);
        } else {
            /* uniform page-aligned split into min(S, n) chunks */
            int64_t L = p->seq_lens[b] > 0 ? p->seq_lens[b] : 0;
            int64_t n = (L + p->page_size - 1) / p->page_size;
            int64_t S = num_splits < 1 ? 1 : num_splits;
            if (S > n) S = n > 0 ? n : 1;
            int64_t c = n > 0 ? (n + S - 1) / S : 1;
            int64_t* bounds = (int64_t*)malloc(sizeof(int64_t) * (size_t)(S + 1));
            if (!bounds) {
                lrc = ORACLE_NO_MEMORY;
            } else {
                for (int64_t s = 0; s <= S; ++s) {
                    int64_t t = s * c * p->page_size;
                    bounds[s] = t < L ? t : L;
                }
                lrc = attend_chunks(p, b, h, bounds, (int)(S + 1), out + r * D);
                free(bounds);
            }
        }
        if (lrc) {
#ifdef _OPENMP
#pragma omp critical
#endif
            err = lrc;
        }
    }
    return err;
}

/* out: [B, Hq, D] doubles. nthreads <= 0 -> all OpenMP threads. */
int oracle_paged_decode(const oracle_problem* p, double* out, int nthreads) {
    return run_rows(p, NULL, (int64_t)p->batch * p->num_q_heads, out, nthreads, 0, 0);
}

/* Only the listed rows: bh = [(b0, h0), (b1, h1), ...]; out: [nrows, D]. */
int oracle_paged_decode_rows(const oracle_problem* p, const int32_t* bh, int64_t nrows, double* out, int nthreads) {
    return run_rows(p, bh, nrows, out, nthreads, 0, 0);
}

/* Split form with the uniform page-aligned rule; out: [B, Hq, D]. */
int oracle_paged_decode_split(const oracle_problem* p, int num_splits, double* out, int nthreads) {
    if (num_splits < 1) return ORACLE_BAD_ARGS;
    return run_rows(p, NULL, (int64_t)p->batch * p->num_q_heads, out, nthreads, 1, num_splits);
}

/* Split form over caller-given token boundaries for one (b, h). */
int oracle_paged_decode_chunks(const oracle_problem* p, int b, int h, const int64_t* bounds, int nbounds, double* out) {
    int rc = check_problem(p);
    if (rc) return rc;
    if (b < 0 || b >= p->batch || h < 0 || h >= p->num_q_heads || nbounds < 2) return ORACLE_BAD_ARGS;
    if (bounds[0] != 0 || bounds[nbounds - 1] != p->seq_lens[b]) return ORACLE_BAD_ARGS;
    for (int i = 1; i < nbounds; ++i)
        if (bounds[i] < bounds[i - 1]) return ORACLE_BAD_ARGS;
    return attend_chunks(p, b, h, bounds, nbounds, out);
}

/* Partial (m, l, acc) for tokens [t0, t1) of (b, h). */
int oracle_partial(const oracle_problem* p, int b, int h, int64_t t0, int64_t t1, double* acc, double* m, double* l) {
    int rc = check_problem(p);
    if (rc) return rc;
    if (b < 0 || b >= p->batch || h < 0 || h >= p->num_q_heads) return ORACLE_BAD_ARGS;
    return attend_partial(p, b, h, t0, t1, acc, m, l);
}

void oracle_round_bf16_array(const double* x, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_round_bf16(x[i]);
}

int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
