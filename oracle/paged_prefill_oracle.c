/*
 * oracle/paged_prefill_oracle.c -- plain fp64 CPU oracle for multi-query
 * (chunked prefill) attention over a paged bf16 KV cache.
 *
 * TEST INFRASTRUCTURE.  Only tests/, __graft_entry__.smoke() and bench.py's CPU
 * baseline may load this library.  It shares no code, header or helper with the
 * CUDA library.
 *
 * What it computes (AstrAI commit d565d44c, csrc/kernels/attn_paged_decode.cu,
 * commit log: prefill kernels templated on the paged KV policy; the unified
 * causal_offset, -1 = no causal mask, >= 0 = position of the first query; 2-D
 * [batch, kv_len] and 3-D [batch, q_len, kv_len] masks, which may be combined
 * with causal).  The page names these without writing them out; the readings:
 *
 *   query i (0 <= i < Lq) of sequence b, head h, kv head h / (Hq / Hkv), sees key
 *   t (0 <= t < L_b) when
 *       (causal_offset < 0 or t <= causal_offset + i)  and  (no mask, or mask != 0)
 *   with mask[b][t] (2-D) or mask[b][i][t] (3-D).  Over the visible keys:
 *       s_t = scale * <q, k_t>,  out = sum_t softmax(s)_t v_t;
 *   a query that sees no key gets zeros.
 *
 * K/V rows come through the page table exactly as in paged_decode_oracle.c (a
 * separate implementation).  Arithmetic: bf16 widened to double exactly, exact
 * products, IEEE double sums in index order, exp in double.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct prefill_problem {
    const uint16_t* q;          /* bf16 [B, Lq, Hq, D]                     */
    int64_t q_stride[4];
    const uint16_t* k;          /* bf16 [NP, P, Hkv, D]                    */
    const uint16_t* v;
    int64_t kv_stride[4];
    const int32_t* page_table;  /* [B, MP]                                 */
    int64_t pt_stride[2];
    const int32_t* seq_lens;    /* [B]                                     */
    const uint8_t* mask;        /* NULL, [B, kv_len] or [B, Lq, kv_len]    */
    int64_t mask_stride[3];     /* (b, i, t) strides; i-stride 0 for 2-D   */
    int64_t mask_kv_len;        /* the mask's last extent                  */
    int32_t batch, q_len, num_q_heads, num_kv_heads, head_dim, page_size, num_pages, max_pages;
    int32_t causal_offset;
    double scale;
} prefill_problem;

static double bf16d(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* offset of key/value row t of sequence b, kv head kvh; -1 when the page index
 * is outside the table or the pool */
static int64_t kv_row(const prefill_problem* p, int b, int64_t t, int kvh) {
    const int64_t j = t / p->page_size;
    if (j >= p->max_pages) return -1;
    const int32_t page = p->page_table[(int64_t)b * p->pt_stride[0] + j * p->pt_stride[1]];
    if (page < 0 || page >= p->num_pages) return -1;
    return (int64_t)page * p->kv_stride[0] + (t % p->page_size) * p->kv_stride[1] + (int64_t)kvh * p->kv_stride[2];
}

static int visible(const prefill_problem* p, int b, int i, int64_t t) {
    if (p->causal_offset >= 0 && t > (int64_t)p->causal_offset + i) return 0;
    if (p->mask) {
        if (t >= p->mask_kv_len) return 0;
        if (!p->mask[(int64_t)b * p->mask_stride[0] + (int64_t)i * p->mask_stride[1] + t * p->mask_stride[2]])
            return 0;
    }
    return 1;
}

/* One query row (b, i, h): out[0..D).  Returns 0, or 2 on a bad page. */
static int attend_row(const prefill_problem* p, int b, int i, int h, double* out, double* s, int64_t* rows) {
    const int D = p->head_dim;
    const int kvh = h / (p->num_q_heads / p->num_kv_heads);
    const int64_t L = p->seq_lens[b] > 0 ? p->seq_lens[b] : 0;
    const uint16_t* qrow = p->q + (int64_t)b * p->q_stride[0] + (int64_t)i * p->q_stride[1] + (int64_t)h * p->q_stride[2];
    for (int d = 0; d < D; ++d) out[d] = 0.0;
    int64_t n = 0;
    for (int64_t t = 0; t < L; ++t) {
        if (!visible(p, b, i, t)) continue;
        const int64_t off = kv_row(p, b, t, kvh);
        if (off < 0) return 2;
        double dot = 0.0;
        for (int d = 0; d < D; ++d) dot += bf16d(qrow[(int64_t)d * p->q_stride[3]]) * bf16d(p->k[off + (int64_t)d * p->kv_stride[3]]);
        s[n] = p->scale * dot;
        rows[n] = off;
        ++n;
    }
    if (n == 0) return 0; /* sees no key: zeros */
    double m = -INFINITY;
    for (int64_t j = 0; j < n; ++j) m = s[j] > m ? s[j] : m;
    double l = 0.0;
    for (int64_t j = 0; j < n; ++j) {
        s[j] = exp(s[j] - m);
        l += s[j];
    }
    for (int64_t j = 0; j < n; ++j)
        for (int d = 0; d < D; ++d) out[d] += s[j] * bf16d(p->v[rows[j] + (int64_t)d * p->kv_stride[3]]);
    for (int d = 0; d < D; ++d) out[d] /= l;
    return 0;
}

/* out: double [B, Lq, Hq, D] row-major.  Returns 0, 1 on bad arguments, 2 on a
 * page-table entry outside the pool, 3 when out of memory. */
int oracle_paged_prefill(const prefill_problem* p, double* out, int nthreads) {
    if (!p || !p->q || !p->k || !p->v || !p->page_table || !p->seq_lens || !out) return 1;
    if (p->batch < 0 || p->q_len < 0 || p->num_q_heads <= 0 || p->num_kv_heads <= 0 || p->head_dim <= 0 ||
        p->page_size <= 0 || p->num_q_heads % p->num_kv_heads)
        return 1;
    int64_t Lmax = 0;
    for (int b = 0; b < p->batch; ++b) Lmax = p->seq_lens[b] > Lmax ? p->seq_lens[b] : Lmax;
    const int64_t rows = (int64_t)p->batch * p->q_len * p->num_q_heads;
    const int D = p->head_dim;
    int err = 0;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel num_threads(nthreads)
#endif
    {
        double* s = (double*)malloc(sizeof(double) * (size_t)(Lmax > 0 ? Lmax : 1));
        int64_t* offs = (int64_t*)malloc(sizeof(int64_t) * (size_t)(Lmax > 0 ? Lmax : 1));
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
        for (int64_t r = 0; r < rows; ++r) {
            const int h = (int)(r % p->num_q_heads);
            const int i = (int)((r / p->num_q_heads) % p->q_len);
            const int b = (int)(r / ((int64_t)p->num_q_heads * p->q_len));
            int rc = (!s || !offs) ? 3 : attend_row(p, b, i, h, out + r * D, s, offs);
            if (rc) {
#ifdef _OPENMP
#pragma omp critical
#endif
                err = rc;
            }
        }
        free(s);
        free(offs);
    }
    return err;
}
