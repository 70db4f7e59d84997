/*
 * FP64 CPU oracle for sparse paged attention with an attention sink.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may link, load or
 * call this file: only the tests, the package's smoke check and the
 * benchmark's CPU-baseline leg use it. It shares no code, header, table or
 * helper with the CUDA library; it is a plain, slow, obviously correct
 * restatement of what the method computes.
 *
 * Sources (page title, then section):
 *  - "Roadmap item 24 - joint compressed/window attention with sink"
 *    (RL-Kernel PR #628), "Reuse and arithmetic": compressed KV, the full
 *    recent window and the sink share one softmax denominator; the sink has
 *    no V; O is BF16 and LSE is FP32 natural log. "Contracts and lifetime":
 *    logical request/position/kind keys, complete windows, C4/C128 group
 *    boundaries, canonical KV ordering. "MI300X validation": an FP64 O/LSE
 *    oracle. "Reuse and arithmetic": mixed FP8/BF16 cache with an explicit
 *    OCP format.
 *  - "test: add block-level DeepSeek-V4 attention test" (ROCm/ATOM PR
 *    #1723), opening section and "Validation": layer types ratio 0 / 4 / 128,
 *    per-token KV-set sizes, top-k truncation once ctx//4 > index_topk.
 *  - "[WS2] Add CP-aware Attention contract and dispatch metadata"
 *    (RL-Kernel PR #236), "Summary": deterministic (out, lse) merge.
 *  - "docs: Block AttnRes model + ROCm-first plan" (tessera PR #552),
 *    "Summary": attn-with-stats + softmax_merge and the merge lemma.
 *
 * Readings taken where the pages are silent (each is listed, with its reason,
 * in the design notes of the repository):
 *  - the window of a query at position p is the raw tokens
 *    max(0, p-W+1) .. p (the query's own token included);
 *  - compressed group g covers tokens r*g .. r*g+r-1 and is complete at
 *    position p iff r*(g+1) <= p+1, i.e. g < floor((p+1)/r);
 *  - a key is an int32: a compressed group index g, or WINDOW_TAG | t for
 *    raw token t (WINDOW_TAG = 1<<30); the canonical order of a set is the
 *    ascending order of its keys (so compressed groups come first);
 *  - top-k entries that are negative, not complete, or repeated are dropped
 *    (set semantics);
 *  - scale multiplies q.k only; the sink is a raw natural-log logit;
 *  - LSE = ln(e^sink + sum_j e^{s_j}) includes the sink;
 *  - FP8 decode: x = bf16_rne(float(e4m3(byte)) * scale), one FP32 multiply
 *    with one FP32 scale per 64 consecutive elements of a token row.
 *
 * Build: cc -O2 -std=c11 -ffp-contract=off -fPIC -shared -pthread -lm
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_WINDOW_TAG (1 << 30)

enum {
    ORACLE_OK = 0,
    ORACLE_BAD_ARG = 1,
    ORACLE_BAD_INDEX = 2,
    ORACLE_BAD_PAGE = 3,
    ORACLE_CAPACITY = 4,
    ORACLE_NO_MEMORY = 5,
};

/* ------------------------------------------------------------------------ */
/* Scalar conversions, written from the format definitions.                  */
/* ------------------------------------------------------------------------ */

/* A BF16 value is the top half of an IEEE binary32 value: widen exactly. */
double oracle_bf16_to_double(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Round a binary32 value to BF16, round-to-nearest-even on the 16 dropped
 * bits. NaN maps to a quiet NaN with the same sign. */
uint16_t oracle_float_to_bf16_rne(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu) != 0)
        return (uint16_t)(((u >> 16) & 0x8000u) | 0x7fc0u);
    uint32_t keep = u >> 16;
    uint32_t dropped = u & 0xffffu;
    if (dropped > 0x8000u || (dropped == 0x8000u && (keep & 1u)))
        keep += 1; /* may carry into the exponent: that is correct rounding */
    return (uint16_t)keep;
}

/* OCP 8-bit floating point, E4M3 variant: 1 sign bit, 4 exponent bits with
 * bias 7, 3 mantissa bits. Exponent field 0 encodes subnormals m * 2^-9.
 * S.1111.111 is NaN; there is no infinity, so S.1111.000 .. S.1111.110 are
 * finite and the largest magnitude is 1.75 * 2^8 = 448. */
double oracle_e4m3_to_double(uint8_t code)
{
    int sign = (code >> 7) & 1;
    int e = (code >> 3) & 0xf;
    int m = code & 0x7;
    double mag;
    if (e == 0xf && m == 0x7)
        return NAN;
    if (e == 0)
        mag = ldexp((double)m, -9);            /* (m/8) * 2^(1-7) */
    else
        mag = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -mag : mag;
}

/* E4M3 "FNUZ" variant (finite, no negative zero): the same three fields,
 * exponent bias 8; the code 1.0000.000 is the only NaN, every other code is
 * finite, so there is no -0 and the largest magnitude is 1.875 * 2^7 = 240.
 * Exponent field 0 encodes subnormals m * 2^-10. */
double oracle_e4m3fnuz_to_double(uint8_t code)
{
    int sign = (code >> 7) & 1;
    int e = (code >> 3) & 0xf;
    int m = code & 0x7;
    double mag;
    if (code == 0x80)
        return NAN;
    if (e == 0)
        mag = ldexp((double)m, -10);           /* (m/8) * 2^(1-8) */
    else
        mag = ldexp(1.0 + (double)m / 8.0, e - 8);
    return sign ? -mag : mag;
}

/* ------------------------------------------------------------------------ */
/* Per-token KV sets.                                                        */
/* ------------------------------------------------------------------------ */

static int cmp_i32(const void* a, const void* b)
{
    int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
    return (x > y) - (x < y);
}

/* Number of complete compressed groups at position p. */
static int64_t complete_groups(int64_t p, int32_t ratio)
{
    return ratio > 0 ? (p + 1) / ratio : 0;
}

/* Build the key set of one query into `out` (room for W + K or W + n_c
 * keys) as sort_ascending(Cset U Wset) with duplicates removed. Returns
 * the number of keys. */
static int64_t one_set(int64_t p, int32_t W, int32_t ratio, const int32_t* topk_row,
                       int32_t K, int32_t* out)
{
    int64_t n = 0;
    int64_t nc = complete_groups(p, ratio);
    if (ratio > 0) {
        if (topk_row == NULL) {
            for (int64_t g = 0; g < nc; ++g) out[n++] = (int32_t)g;
        } else {
            for (int32_t j = 0; j < K; ++j) {
                int32_t g = topk_row[j];
                if (g >= 0 && (int64_t)g < nc) out[n++] = g;
            }
        }
    }
    int64_t t0 = p - W + 1 > 0 ? p - W + 1 : 0;
    for (int64_t t = t0; t <= p; ++t) out[n++] = (int32_t)(ORACLE_WINDOW_TAG | t);
    qsort(out, (size_t)n, sizeof(int32_t), cmp_i32);
    int64_t u = 0;
    for (int64_t j = 0; j < n; ++j)
        if (u == 0 || out[j] != out[u - 1]) out[u++] = out[j];
    return u;
}

/* indptr[N+1] (exclusive prefix sum of set sizes) and indices[capacity].
 * topk is [N, K] row-major or NULL (all complete groups). */
int oracle_build_kv_sets(const int32_t* pos, int32_t N, int32_t W, int32_t ratio,
                         const int32_t* topk, int32_t K, int32_t* indptr,
                         int32_t* indices, int64_t capacity)
{
    if (N < 0 || W < 1 || (ratio != 0 && ratio != 4 && ratio != 128) || K < 0)
        return ORACLE_BAD_ARG;
    int64_t maxp = 0;
    for (int32_t i = 0; i < N; ++i) {
        if (pos[i] < 0 || pos[i] >= ORACLE_WINDOW_TAG) return ORACLE_BAD_INDEX;
        if (pos[i] > maxp) maxp = pos[i];
    }
    int64_t room = (int64_t)W + (topk ? K : complete_groups(maxp, ratio)) + 1;
    int32_t* buf = (int32_t*)malloc((size_t)room * sizeof(int32_t));
    if (!buf) return ORACLE_NO_MEMORY;
    int64_t off = 0;
    indptr[0] = 0;
    for (int32_t i = 0; i < N; ++i) {
        int64_t n = one_set(pos[i], W, ratio, topk ? topk + (int64_t)i * K : NULL, K, buf);
        if (off + n > capacity || off + n > INT32_MAX) { free(buf); return ORACLE_CAPACITY; }
        memcpy(indices + off, buf, (size_t)n * sizeof(int32_t));
        off += n;
        indptr[i + 1] = (int32_t)off;
    }
    free(buf);
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* FP8 page decode.                                                          */
/* ------------------------------------------------------------------------ */

/* src: [num_pages, page_size, d] bytes; scales: [num_pages, page_size, d/64]
 * FP32; the listed pages of dst ([num_pages, page_size, d] BF16 bits) get
 * bf16_rne(float(e4m3(byte)) * scale); other pages are left untouched.
 * fmt 0 reads the bytes as OCP E4M3, fmt 1 as E4M3 FNUZ. */
int oracle_dequant_fp8_pages_fmt(const uint8_t* src, const float* scales, int64_t num_pages,
                                 int32_t page_size, int32_t d, const int32_t* page_ids,
                                 int32_t n, int32_t fmt, uint16_t* dst)
{
    if (page_size < 1 || d < 64 || d % 64 != 0 || n < 0 || (fmt != 0 && fmt != 1)) return ORACLE_BAD_ARG;
    for (int32_t k = 0; k < n; ++k) {
        int64_t pg = page_ids[k];
        if (pg < 0 || pg >= num_pages) return ORACLE_BAD_PAGE;
        for (int64_t s = 0; s < page_size; ++s) {
            int64_t row = pg * page_size + s;
            for (int32_t e = 0; e < d; ++e) {
                uint8_t code = src[row * d + e];
                float value = (float)(fmt == 0 ? oracle_e4m3_to_double(code) : oracle_e4m3fnuz_to_double(code));
                float scale = scales[row * (d / 64) + e / 64];
                float product = value * scale; /* one binary32 multiply */
                dst[row * d + e] = oracle_float_to_bf16_rne(product);
            }
        }
    }
    return ORACLE_OK;
}

int oracle_dequant_fp8_pages(const uint8_t* src, const float* scales, int64_t num_pages,
                             int32_t page_size, int32_t d, const int32_t* page_ids,
                             int32_t n, uint16_t* dst)
{
    return oracle_dequant_fp8_pages_fmt(src, scales, num_pages, page_size, d, page_ids, n, 0, dst);
}

/* ------------------------------------------------------------------------ */
/* Packed D512 rows (584 bytes per token).                                   */
/* ------------------------------------------------------------------------ */

/* UE8M0 scale byte: 2^(byte - 127); 0xFF is NaN. */
double oracle_ue8m0_to_double(uint8_t b)
{
    if (b == 0xFF) return NAN;
    return ldexp(1.0, (int)b - 127);
}

/* The packed row of a 512-wide head, 584 bytes per token ("Roadmap item 24"
 * review: 584 bytes per token for head width 512, 576 of them data): 448
 * E4M3 codes (the first 448 elements), 64 BF16 values (the last 64
 * elements, 128 bytes), then 7 UE8M0 scale bytes (one per 64 codes) and one
 * unused byte. Element e < 448 decodes to bf16_rne(float(e4m3(code_e)) *
 * float(2^(scale_{e/64} - 127))), one binary32 multiply; e >= 448 is copied.
 * src: [num_pages, page_size, 584] bytes; dst: [num_pages, page_size, 512]
 * BF16 bits; only the listed pages are written. */
int oracle_unpack_d512_pages(const uint8_t* src, int64_t num_pages, int32_t page_size,
                             const int32_t* page_ids, int32_t n, uint16_t* dst)
{
    if (page_size < 1 || n < 0) return ORACLE_BAD_ARG;
    for (int32_t k = 0; k < n; ++k) {
        int64_t pg = page_ids[k];
        if (pg < 0 || pg >= num_pages) return ORACLE_BAD_PAGE;
        for (int64_t t = 0; t < page_size; ++t) {
            int64_t row = pg * page_size + t;
            const uint8_t* in = src + row * 584;
            uint16_t* out = dst + row * 512;
            for (int32_t e = 0; e < 448; ++e) {
                float value = (float)oracle_e4m3_to_double(in[e]);
                float scale = (float)oracle_ue8m0_to_double(in[576 + e / 64]);
                float product = value * scale; /* one binary32 multiply */
                out[e] = oracle_float_to_bf16_rne(product);
            }
            for (int32_t e = 0; e < 64; ++e)
                out[448 + e] = (uint16_t)(in[448 + 2 * e] | (in[448 + 2 * e + 1] << 8));
        }
    }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* Paged KV write.                                                           */
/* ------------------------------------------------------------------------ */

/* Token j (request req[j], position pos[j]) copies its d-element K and V
 * rows (BF16 bits) into row pt[req][pos / page_size] * page_size +
 * pos % page_size of the pools. A token whose request, position or page is
 * out of range is skipped; the return value ORs 2 (bad request/position)
 * and 1 (bad page) for the skipped ones, 0 when none was. */
int oracle_paged_kv_write(const uint16_t* k_new, const uint16_t* v_new, int32_t n, int32_t d,
                          const int32_t* req, const int32_t* pos, const int32_t* pt, int32_t pt_cols,
                          int32_t n_requests, int32_t page_size, int64_t num_pages,
                          uint16_t* k_pool, uint16_t* v_pool)
{
    int flags = 0;
    for (int32_t j = 0; j < n; ++j) {
        int32_t b = req[j], t = pos[j];
        if (b < 0 || b >= n_requests || t < 0 || t / page_size >= pt_cols) {
            flags |= 2;
            continue;
        }
        int64_t page = pt[(int64_t)b * pt_cols + t / page_size];
        if (page < 0 || page >= num_pages) {
            flags |= 1;
            continue;
        }
        int64_t row = page * page_size + t % page_size;
        memcpy(k_pool + row * d, k_new + (int64_t)j * d, (size_t)d * sizeof(uint16_t));
        memcpy(v_pool + row * d, v_new + (int64_t)j * d, (size_t)d * sizeof(uint16_t));
    }
    return flags;
}

/* ------------------------------------------------------------------------ */
/* Attention with an attention sink.                                         */
/* ------------------------------------------------------------------------ */

typedef struct {
    const uint16_t* q; int64_t q_stride_tok, q_stride_head;
    int32_t N, H, d;
    const uint16_t *k_raw, *v_raw; int64_t raw_pages; int32_t raw_ps;
    const int32_t* pt_raw; int32_t pt_raw_cols;
    const uint16_t *k_cmp, *v_cmp; int64_t cmp_pages; int32_t cmp_ps;
    const int32_t* pt_cmp; int32_t pt_cmp_cols;
    const int32_t* req; int32_t B;
    const int32_t* indptr; const int32_t* indices;
    const float* sink; double scale; int32_t include_sink;
    const int32_t* rows; int32_t n_rows;
    double* out; double* lse;
    int32_t next_row; pthread_mutex_t lock; int status;
} attn_job;

/* Find the K and V rows of one key through the page table of its kind. */
static int locate(const attn_job* J, int32_t b, int32_t key, const uint16_t** krow,
                  const uint16_t** vrow)
{
    int32_t ps, cols; int64_t pages; const int32_t* pt;
    const uint16_t *kp, *vp; int64_t logical;
    if (key < 0) return ORACLE_BAD_INDEX;
    if (key & ORACLE_WINDOW_TAG) {
        logical = key & (ORACLE_WINDOW_TAG - 1);
        ps = J->raw_ps; cols = J->pt_raw_cols; pages = J->raw_pages; pt = J->pt_raw;
        kp = J->k_raw; vp = J->v_raw;
    } else {
        logical = key;
        ps = J->cmp_ps; cols = J->pt_cmp_cols; pages = J->cmp_pages; pt = J->pt_cmp;
        kp = J->k_cmp; vp = J->v_cmp;
    }
    if (pt == NULL || logical / ps >= cols) return ORACLE_BAD_INDEX;
    int64_t page = pt[(int64_t)b * cols + logical / ps];
    if (page < 0 || page >= pages) return ORACLE_BAD_PAGE;
    int64_t row = page * ps + logical % ps;
    *krow = kp + row * J->d;
    *vrow = vp + row * J->d;
    return ORACLE_OK;
}

static int one_query(const attn_job* J, int32_t r, double* kbuf, double* vbuf, double* s)
{
    int32_t i = J->rows ? J->rows[r] : r;
    int32_t d = J->d, H = J->H;
    if (i < 0 || i >= J->N) return ORACLE_BAD_INDEX;
    int32_t b = J->req[i];
    if (b < 0 || b >= J->B) return ORACLE_BAD_INDEX;
    int32_t j0 = J->indptr[i], j1 = J->indptr[i + 1];
    int32_t n = j1 - j0;
    /* gather the set's K and V rows once; all heads share them */
    for (int32_t j = 0; j < n; ++j) {
        const uint16_t *kr, *vr;
        int st = locate(J, b, J->indices[j0 + j], &kr, &vr);
        if (st) return st;
        for (int32_t e = 0; e < d; ++e) {
            kbuf[(int64_t)j * d + e] = oracle_bf16_to_double(kr[e]);
            vbuf[(int64_t)j * d + e] = oracle_bf16_to_double(vr[e]);
        }
    }
    for (int32_t h = 0; h < H; ++h) {
        const uint16_t* qh = J->q + (int64_t)i * J->q_stride_tok + (int64_t)h * J->q_stride_head;
        double* o = J->out + ((int64_t)r * H + h) * d;
        double sink = J->include_sink ? (double)J->sink[h] : -INFINITY;
        /* logits s_j = scale * q . k_j */
        double m = sink;
        for (int32_t j = 0; j < n; ++j) {
            double acc = 0.0;
            for (int32_t e = 0; e < d; ++e)
                acc += oracle_bf16_to_double(qh[e]) * kbuf[(int64_t)j * d + e];
            s[j] = J->scale * acc;
            if (s[j] > m) m = s[j];
        }
        for (int32_t e = 0; e < d; ++e) o[e] = 0.0;
        if (m == -INFINITY) {               /* no sink and no keys */
            J->lse[(int64_t)r * H + h] = -INFINITY;
            continue;
        }
        /* denominator: the sink's term plus every key's term */
        double l = exp(sink - m);
        for (int32_t j = 0; j < n; ++j) {
            double w = exp(s[j] - m);
            l += w;
            for (int32_t e = 0; e < d; ++e) o[e] += w * vbuf[(int64_t)j * d + e];
        }
        for (int32_t e = 0; e < d; ++e) o[e] /= l;   /* the sink adds no V */
        J->lse[(int64_t)r * H + h] = m + log(l);
    }
    return ORACLE_OK;
}

static void* attn_worker(void* arg)
{
    attn_job* J = (attn_job*)arg;
    int32_t cap = 0;
    double *kbuf = NULL, *vbuf = NULL, *s = NULL;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        int32_t r = J->status ? J->n_rows : J->next_row++;
        pthread_mutex_unlock(&J->lock);
        if (r >= J->n_rows) break;
        int32_t i = J->rows ? J->rows[r] : r;
        int32_t n = (i >= 0 && i < J->N) ? J->indptr[i + 1] - J->indptr[i] : 0;
        if (n < 0) n = 0;
        if (n + 1 > cap) {
            cap = n + 1;
            free(kbuf); free(vbuf); free(s);
            kbuf = (double*)malloc((size_t)cap * J->d * sizeof(double));
            vbuf = (double*)malloc((size_t)cap * J->d * sizeof(double));
            s = (double*)malloc((size_t)cap * sizeof(double));
            if (!kbuf || !vbuf || !s) {
                pthread_mutex_lock(&J->lock); J->status = ORACLE_NO_MEMORY;
                pthread_mutex_unlock(&J->lock); break;
            }
        }
        int st = one_query(J, r, kbuf, vbuf, s);
        if (st) { pthread_mutex_lock(&J->lock); if (!J->status) J->status = st; pthread_mutex_unlock(&J->lock); }
    }
    free(kbuf); free(vbuf); free(s);
    return NULL;
}

/* O[r,h,:] and LSE[r,h] in FP64 for query tokens rows[0..n_rows) (all N
 * tokens in order when rows is NULL). q is BF16 bits [N,H,d] with the given
 * strides (elements); pools are BF16 bits [pages, page_size, d]; page tables
 * are int32 [B, cols]; indptr/indices are the CSR key sets. With
 * include_sink = 0 the sink is left out (a partial result over a subset). */
int oracle_sparse_sink_attn(
    const uint16_t* q, int64_t q_stride_tok, int64_t q_stride_head, int32_t N, int32_t H,
    int32_t d, const uint16_t* k_raw, const uint16_t* v_raw, int64_t raw_pages,
    int32_t raw_ps, const int32_t* pt_raw, int32_t pt_raw_cols, const uint16_t* k_cmp,
    const uint16_t* v_cmp, int64_t cmp_pages, int32_t cmp_ps, const int32_t* pt_cmp,
    int32_t pt_cmp_cols, const int32_t* req, int32_t B, const int32_t* indptr,
    const int32_t* indices, const float* sink, double scale, int32_t include_sink,
    const int32_t* rows, int32_t n_rows, double* out, double* lse, int32_t n_threads)
{
    if (N < 0 || H < 1 || d < 1 || raw_ps < 1 || (pt_cmp && cmp_ps < 1) || n_rows < 0)
        return ORACLE_BAD_ARG;
    attn_job J = {q, q_stride_tok, q_stride_head, N, H, d, k_raw, v_raw, raw_pages, raw_ps,
                  pt_raw, pt_raw_cols, k_cmp, v_cmp, cmp_pages, cmp_ps, pt_cmp, pt_cmp_cols,
                  req, B, indptr, indices, sink, scale, include_sink, rows, n_rows, out, lse,
                  0, PTHREAD_MUTEX_INITIALIZER, 0};
    if (n_threads < 1) n_threads = 1;
    if (n_threads > 256) n_threads = 256;
    pthread_t tid[256];
    int started = 0;
    for (int t = 1; t < n_threads; ++t)
        if (pthread_create(&tid[started], NULL, attn_worker, &J) == 0) ++started;
    attn_worker(&J);
    for (int t = 0; t < started; ++t) pthread_join(tid[t], NULL);
    return J.status;
}

/* ------------------------------------------------------------------------ */
/* Exact merge of partial results.                                           */
/* ------------------------------------------------------------------------ */

/* Merge n_parts partial results (O_s [d], LSE_s) of disjoint parts of one
 * (query, head)'s denominator into the whole: LSE = ln sum_s e^{LSE_s} and
 * O = sum_s e^{LSE_s - LSE} O_s. The sink is the part (O = 0, LSE = sink). */
void oracle_lse_merge(int32_t n_parts, const double* lse_parts, const double* o_parts,
                      int32_t d, double* o, double* lse)
{
    double m = -INFINITY;
    for (int32_t s = 0; s < n_parts; ++s)
        if (lse_parts[s] > m) m = lse_parts[s];
    for (int32_t e = 0; e < d; ++e) o[e] = 0.0;
    if (m == -INFINITY) { *lse = -INFINITY; return; }
    double l = 0.0;
    for (int32_t s = 0; s < n_parts; ++s) l += exp(lse_parts[s] - m);
    *lse = m + log(l);
    for (int32_t s = 0; s < n_parts; ++s) {
        double w = exp(lse_parts[s] - *lse);
        for (int32_t e = 0; e < d; ++e) o[e] += w * o_parts[(int64_t)s * d + e];
    }
}

/* ------------------------------------------------------------------------ */
/* Backward of the attention with sink.                                      */
/* ------------------------------------------------------------------------ */

/* Gradients of L = sum over (i, h, e) of dO[i,h,e] * O[i,h,e] for the query
 * tokens rows[0..n_rows) (all N when rows is NULL), in FP64, from the exact
 * forward of the same inputs, or, when o_saved / lse_saved are given
 * ([N, H, d] and [N, H], FP64), from those saved forward results: D then
 * takes O from o_saved and the probabilities take LSE from lse_saved, as a
 * backward that reads the forward's stored outputs does. "Roadmap item 24 - joint compressed/window
 * attention with sink" names the backward (dQ, dK/dV, d_sink) as its
 * follow-on item; the formulas are the chain rule through the forward
 * above. For one (i, h) with logits s_j = scale q.k_j and the sink c_h:
 *   p_j = e^{s_j - LSE}, p_c = e^{c_h - LSE}, O = sum_j p_j v_j,
 *   D = dO . O, dp_j = dO . v_j, ds_j = p_j (dp_j - D),
 *   dq = scale sum_j ds_j k_j, dk_j += scale ds_j q, dv_j += p_j dO,
 *   dsink_h += -p_c D (the sink's logit has no V, so its dp is 0).
 * dq is written ([n_rows, H, d]); dk/dv are ADDED into arrays shaped like
 * the pools ([pages * page_size, d]); dsink (may be NULL) is added into.
 * The per-query contributions to dk/dv/dsink are added in query order
 * whatever the thread count, so repeated calls give identical sums. */
typedef struct {
    attn_job A;
    const uint16_t* dout;            /* BF16 bits [N, H, d], contiguous */
    const double* o_saved;           /* [N, H, d] or NULL */
    const double* lse_saved;         /* [N, H] or NULL */
    double *dq, *dk_raw, *dv_raw, *dk_cmp, *dv_cmp, *dsink;
    int32_t next_commit;             /* the next row whose sums may be added */
    pthread_cond_t turn;
} bwd_job;

static int one_query_bwd(bwd_job* G, int32_t r, double* kbuf, double* vbuf, double* s,
                         double* dkb, double* dvb, int64_t* rowb, int* rawb, double* dsink_loc)
{
    const attn_job* J = &G->A;
    int32_t i = J->rows ? J->rows[r] : r;
    int32_t d = J->d, H = J->H;
    if (i < 0 || i >= J->N) return ORACLE_BAD_INDEX;
    int32_t b = J->req[i];
    if (b < 0 || b >= J->B) return ORACLE_BAD_INDEX;
    int32_t j0 = J->indptr[i], n = J->indptr[i + 1] - J->indptr[i];
    for (int32_t j = 0; j < n; ++j) {
        const uint16_t *kr, *vr;
        int32_t key = J->indices[j0 + j];
        int st = locate(J, b, key, &kr, &vr);
        if (st) return st;
        rawb[j] = (key & ORACLE_WINDOW_TAG) != 0;
        rowb[j] = (kr - (rawb[j] ? J->k_raw : J->k_cmp)) / d;
        for (int32_t e = 0; e < d; ++e) {
            kbuf[(int64_t)j * d + e] = oracle_bf16_to_double(kr[e]);
            vbuf[(int64_t)j * d + e] = oracle_bf16_to_double(vr[e]);
            dkb[(int64_t)j * d + e] = 0.0;
            dvb[(int64_t)j * d + e] = 0.0;
        }
    }
    double* p = s + n;               /* [n] */
    for (int32_t h = 0; h < H; ++h) {
        const uint16_t* qh = J->q + (int64_t)i * J->q_stride_tok + (int64_t)h * J->q_stride_head;
        const uint16_t* doh = G->dout + ((int64_t)i * H + h) * d;
        double* dq = G->dq + ((int64_t)r * H + h) * d;
        double sink = J->sink ? (double)J->sink[h] : -INFINITY;
        for (int32_t e = 0; e < d; ++e) dq[e] = 0.0;
        /* the forward: logits, max, denominator, LSE */
        double m = sink;
        for (int32_t j = 0; j < n; ++j) {
            double acc = 0.0;
            for (int32_t e = 0; e < d; ++e)
                acc += oracle_bf16_to_double(qh[e]) * kbuf[(int64_t)j * d + e];
            s[j] = J->scale * acc;
            if (s[j] > m) m = s[j];
        }
        if (m == -INFINITY) continue;            /* no keys, no sink: O = 0, no gradient */
        double l = exp(sink - m);
        for (int32_t j = 0; j < n; ++j) l += exp(s[j] - m);
        double lse = G->lse_saved ? G->lse_saved[(int64_t)i * H + h] : m + log(l);
        /* probabilities, O and D = dO . O */
        double D = 0.0;
        for (int32_t j = 0; j < n; ++j) p[j] = exp(s[j] - lse);
        for (int32_t e = 0; e < d; ++e) {
            double o = 0.0;
            if (G->o_saved) {
                o = G->o_saved[((int64_t)i * H + h) * d + e];
            } else {
                for (int32_t j = 0; j < n; ++j) o += p[j] * vbuf[(int64_t)j * d + e];
            }
            D += oracle_bf16_to_double(doh[e]) * o;
        }
        for (int32_t j = 0; j < n; ++j) {
            double dp = 0.0;
            for (int32_t e = 0; e < d; ++e)
                dp += oracle_bf16_to_double(doh[e]) * vbuf[(int64_t)j * d + e];
            double ds = p[j] * (dp - D);
            for (int32_t e = 0; e < d; ++e) {
                dq[e] += J->scale * ds * kbuf[(int64_t)j * d + e];
                dkb[(int64_t)j * d + e] += J->scale * ds * oracle_bf16_to_double(qh[e]);
                dvb[(int64_t)j * d + e] += p[j] * oracle_bf16_to_double(doh[e]);
            }
        }
        if (J->sink) dsink_loc[h] += -exp(sink - lse) * D;
    }
    return ORACLE_OK;
}

static void* bwd_worker(void* arg)
{
    bwd_job* G = (bwd_job*)arg;
    attn_job* J = &G->A;
    int32_t cap = 0, d = J->d;
    double *kbuf = NULL, *vbuf = NULL, *s = NULL, *dkb = NULL, *dvb = NULL;
    int64_t* rowb = NULL; int* rawb = NULL;
    double* dsink_loc = (double*)malloc((size_t)J->H * sizeof(double));   /* this query's dsink */
    if (!dsink_loc) {
        pthread_mutex_lock(&J->lock); J->status = ORACLE_NO_MEMORY;
        pthread_cond_broadcast(&G->turn); pthread_mutex_unlock(&J->lock); return NULL;
    }
    for (;;) {
        pthread_mutex_lock(&J->lock);
        int32_t r = J->status ? J->n_rows : J->next_row++;
        pthread_mutex_unlock(&J->lock);
        if (r >= J->n_rows) break;
        int32_t i = J->rows ? J->rows[r] : r;
        int32_t n = (i >= 0 && i < J->N) ? J->indptr[i + 1] - J->indptr[i] : 0;
        if (n < 0) n = 0;
        if (n + 1 > cap) {
            cap = n + 1;
            free(kbuf); free(vbuf); free(s); free(dkb); free(dvb); free(rowb); free(rawb);
            kbuf = (double*)malloc((size_t)cap * d * sizeof(double));
            vbuf = (double*)malloc((size_t)cap * d * sizeof(double));
            dkb = (double*)malloc((size_t)cap * d * sizeof(double));
            dvb = (double*)malloc((size_t)cap * d * sizeof(double));
            s = (double*)malloc((size_t)cap * 2 * sizeof(double));
            rowb = (int64_t*)malloc((size_t)cap * sizeof(int64_t));
            rawb = (int*)malloc((size_t)cap * sizeof(int));
            if (!kbuf || !vbuf || !s || !dkb || !dvb || !rowb || !rawb) {
                pthread_mutex_lock(&J->lock); J->status = ORACLE_NO_MEMORY;
                pthread_cond_broadcast(&G->turn); pthread_mutex_unlock(&J->lock); break;
            }
        }
        for (int32_t h = 0; h < J->H; ++h) dsink_loc[h] = 0.0;
        int st = one_query_bwd(G, r, kbuf, vbuf, s, dkb, dvb, rowb, rawb, dsink_loc);
        pthread_mutex_lock(&J->lock);
        if (st) {
            if (!J->status) J->status = st;
            pthread_cond_broadcast(&G->turn);
        } else {
            /* this query's key-row gradients into the pool-shaped sums, in
             * query order: wait until every earlier row has been added */
            while (G->next_commit != r && !J->status) pthread_cond_wait(&G->turn, &J->lock);
            if (!J->status) {
                for (int32_t j = 0; j < n; ++j) {
                    double* dk = (rawb[j] ? G->dk_raw : G->dk_cmp) + rowb[j] * d;
                    double* dv = (rawb[j] ? G->dv_raw : G->dv_cmp) + rowb[j] * d;
                    for (int32_t e = 0; e < d; ++e) {
                        dk[e] += dkb[(int64_t)j * d + e];
                        dv[e] += dvb[(int64_t)j * d + e];
                    }
                }
                if (G->dsink)
                    for (int32_t h = 0; h < J->H; ++h) G->dsink[h] += dsink_loc[h];
                ++G->next_commit;
                pthread_cond_broadcast(&G->turn);
            }
        }
        pthread_mutex_unlock(&J->lock);
    }
    free(kbuf); free(vbuf); free(s); free(dkb); free(dvb); free(rowb); free(rawb); free(dsink_loc);
    return NULL;
}

int oracle_sparse_sink_attn_bwd(
    const uint16_t* q, int64_t q_stride_tok, int64_t q_stride_head, int32_t N, int32_t H,
    int32_t d, const uint16_t* k_raw, const uint16_t* v_raw, int64_t raw_pages,
    int32_t raw_ps, const int32_t* pt_raw, int32_t pt_raw_cols, const uint16_t* k_cmp,
    const uint16_t* v_cmp, int64_t cmp_pages, int32_t cmp_ps, const int32_t* pt_cmp,
    int32_t pt_cmp_cols, const int32_t* req, int32_t B, const int32_t* indptr,
    const int32_t* indices, const float* sink, double scale, const uint16_t* dout,
    const double* o_saved, const double* lse_saved,
    const int32_t* rows, int32_t n_rows, double* dq, double* dk_raw, double* dv_raw,
    double* dk_cmp, double* dv_cmp, double* dsink, int32_t n_threads)
{
    if (N < 0 || H < 1 || d < 1 || raw_ps < 1 || (pt_cmp && cmp_ps < 1) || n_rows < 0 || !dout)
        return ORACLE_BAD_ARG;
    if (pt_cmp && (!dk_cmp || !dv_cmp)) return ORACLE_BAD_ARG;
    bwd_job G;
    attn_job A = {q, q_stride_tok, q_stride_head, N, H, d, k_raw, v_raw, raw_pages, raw_ps,
                  pt_raw, pt_raw_cols, k_cmp, v_cmp, cmp_pages, cmp_ps, pt_cmp, pt_cmp_cols,
                  req, B, indptr, indices, sink, scale, 1, rows, n_rows, NULL, NULL,
                  0, PTHREAD_MUTEX_INITIALIZER, 0};
    G.A = A;
    G.dout = dout; G.o_saved = o_saved; G.lse_saved = lse_saved; G.dq = dq; G.dk_raw = dk_raw; G.dv_raw = dv_raw;
    G.dk_cmp = dk_cmp; G.dv_cmp = dv_cmp; G.dsink = dsink;
    G.next_commit = 0;
    pthread_cond_init(&G.turn, NULL);
    if (n_threads < 1) n_threads = 1;
    if (n_threads > 256) n_threads = 256;
    pthread_t tid[256];
    int started = 0;
    for (int t = 1; t < n_threads; ++t)
        if (pthread_create(&tid[started], NULL, bwd_worker, &G) == 0) ++started;
    bwd_worker(&G);
    for (int t = 0; t < started; ++t) pthread_join(tid[t], NULL);
    pthread_cond_destroy(&G.turn);
    return G.A.status;
}
