/*
 * hi_ref.c - plain CPU oracle of the hierarchical index (HI) decode.
 *
 * TEST INFRASTRUCTURE, like ssa_ref.c next to it: only the test suite, the
 * smoke check and the benchmark's CPU legs may load it; it shares no code
 * with the CUDA library.
 *
 * What it computes: page 4 of the LoZA pages ("LongCat Sparse Attention:
 * Taming the Lightning via Streaming-aware Hierarchical Cross-Layer Indexing",
 * agihunt.info) describes an attention budget of fixed sink and window tokens
 * plus dynamically selected tokens, whose selection the hierarchical index
 * makes in two stages: a coarse pass over pages of 128 tokens recalls the top
 * pages (1,024 there), then only the tokens of those pages are scored one by
 * one, and the best tokens are kept (1,024 dynamic tokens there); the fixed
 * and the dynamic parts are attended separately and merged by their
 * log-sum-exp. The pages give neither the scoring function nor the page
 * representation; the readings taken (listed in the design notes) are:
 *   - the index score of a key is the dot product of a per-sequence index
 *     query q_I with the key's index key k_I (both supplied by the caller, as
 *     an indexer would produce them);
 *   - a page is represented by the mean of its 128 index keys; only whole
 *     pages (all 128 tokens at or before the query) that hold at least one
 *     token outside the fixed window are candidates;
 *   - the dynamic tokens are chosen among the tokens outside the fixed window,
 *     so the two parts are disjoint; ties go to the lower page / token index.
 * Because the scores decide a selection, they are computed here exactly as
 * the kernels compute them: fp32, one fused multiply-add per dimension in
 * index order starting from 0 (page sums: fp32 adds in token order, then
 * times 1/128). The attention itself is fp64, as in ssa_ref.c.
 *
 * Window membership (the fixed part): key t of query position i is in it iff
 * t <= i and (t < s*b or t >= lo(i)), lo(i) = max(0, (floor(i/b) - l + 1)*b);
 * l < 0 selects everything.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define HI_PAGE 128

static float bf16_to_f32(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

static int in_window(int64_t t, int64_t i, int b, int n_sink, int n_local) {
    if (t > i) return 0;
    if (n_local < 0) return 1;
    if (t < (int64_t)n_sink * b) return 1;
    int64_t lo = (i / b - n_local + 1) * (int64_t)b;
    if (lo < 0) lo = 0;
    return t >= lo;
}

/* Mean of the index keys of every whole page of every sequence:
 * page_keys[(n * pages_per_seq + p) * d + c]; pages past the sequence end are
 * left untouched. */
int hi_oracle_page_keys(const uint16_t *k_index, int64_t batch_stride, int64_t row_stride,
                        const int32_t *seqlens, int batch, int d, int64_t pages_per_seq, float *page_keys) {
    if (!k_index || !seqlens || !page_keys || batch < 1 || d < 1) return -1;
    for (int n = 0; n < batch; ++n) {
        const int64_t full = seqlens[n] / HI_PAGE;
        for (int64_t p = 0; p < full && p < pages_per_seq; ++p) {
            for (int c = 0; c < d; ++c) {
                float sum = 0.f;
                for (int r = 0; r < HI_PAGE; ++r)
                    sum += bf16_to_f32(k_index[n * batch_stride + (p * HI_PAGE + r) * row_stride + c]);
                page_keys[(n * pages_per_seq + p) * d + c] = sum * (1.0f / HI_PAGE);
            }
        }
    }
    return 0;
}

typedef struct {
    float score;
    int64_t index;
} scored;

/* higher score first, then the lower index (-0 and +0 compare equal) */
static int by_score(const void *a, const void *b) {
    const scored *x = (const scored *)a, *y = (const scored *)b;
    if (x->score > y->score) return -1;
    if (x->score < y->score) return 1;
    return (x->index > y->index) - (x->index < y->index);
}

static int by_index(const void *a, const void *b) {
    const int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
    return (x > y) - (x < y);
}

/* Tokens of each sequence chosen by the hierarchical index for its decode
 * query (position seqlens[n] - 1): selected[n * top_k + j], ascending, the
 * unused tail -1. */
int hi_oracle_select(const uint16_t *q_index, const uint16_t *k_index, int64_t batch_stride,
                     int64_t row_stride, const float *page_keys, int64_t pages_per_seq,
                     const int32_t *seqlens, int batch, int d, int block_size, int n_sink, int n_local,
                     int top_pages, int top_k, int32_t *selected) {
    if (!q_index || !k_index || !page_keys || !seqlens || !selected || batch < 1 || d < 1 || block_size < 1 ||
        top_pages < 0 || top_k < 0)
        return -1;
    for (int n = 0; n < batch; ++n) {
        const int64_t L = seqlens[n], i = L - 1;
        int32_t *out = selected + (int64_t)n * top_k;
        for (int j = 0; j < top_k; ++j) out[j] = -1;
        const int64_t full = L / HI_PAGE < pages_per_seq ? L / HI_PAGE : pages_per_seq;
        if (full <= 0 || top_k == 0 || top_pages == 0) continue;
        float *q = (float *)malloc(sizeof(float) * (size_t)d);
        for (int c = 0; c < d; ++c) q[c] = bf16_to_f32(q_index[(int64_t)n * d + c]);
        /* stage 1: whole pages with a token outside the window */
        scored *pages = (scored *)malloc(sizeof(scored) * (size_t)full);
        int64_t np = 0;
        for (int64_t p = 0; p < full; ++p) {
            int outside = 0;
            for (int r = 0; r < HI_PAGE && !outside; ++r)
                outside = !in_window(p * HI_PAGE + r, i, block_size, n_sink, n_local);
            if (!outside) continue;
            float s = 0.f;
            for (int c = 0; c < d; ++c) s = fmaf(q[c], page_keys[(n * pages_per_seq + p) * d + c], s);
            pages[np].score = s;
            pages[np].index = p;
            ++np;
        }
        qsort(pages, (size_t)np, sizeof(scored), by_score);
        const int64_t m = np < top_pages ? np : top_pages;
        /* stage 2: the tokens of those pages outside the window */
        scored *tok = (scored *)malloc(sizeof(scored) * (size_t)(m * HI_PAGE + 1));
        int64_t nt = 0;
        for (int64_t a = 0; a < m; ++a) {
            for (int r = 0; r < HI_PAGE; ++r) {
                const int64_t t = pages[a].index * HI_PAGE + r;
                if (in_window(t, i, block_size, n_sink, n_local)) continue;
                const uint16_t *kr = k_index + n * batch_stride + t * row_stride;
                float s = 0.f;
                for (int c = 0; c < d; ++c) s = fmaf(q[c], bf16_to_f32(kr[c]), s);
                tok[nt].score = s;
                tok[nt].index = t;
                ++nt;
            }
        }
        qsort(tok, (size_t)nt, sizeof(scored), by_score);
        const int64_t k = nt < top_k ? nt : top_k;
        for (int64_t j = 0; j < k; ++j) out[j] = (int32_t)tok[j].index;
        qsort(out, (size_t)k, sizeof(int32_t), by_index);
        free(tok);
        free(pages);
        free(q);
    }
    return 0;
}

static double widen(uint16_t bits) { return (double)bf16_to_f32(bits); }

/* Decode over the fixed window and the selected tokens (disjoint), all heads
 * reading one latent row per token (absorbed MLA: V = its first d_v columns):
 * fp64 softmax attention of position seqlens[n] - 1. */
int hi_oracle_decode(const uint16_t *q, const uint16_t *kv, int64_t batch_stride, int64_t row_stride,
                     const int32_t *seqlens, int batch, int n_heads, int d_qk, int d_v, int block_size,
                     int n_sink, int n_local, double scale, const int32_t *selected, int top_k, double *o,
                     double *lse) {
    if (!q || !kv || !seqlens || !o || !lse || batch < 1 || d_v > d_qk || top_k < 0) return -1;
    for (int n = 0; n < batch; ++n) {
        const int64_t L = seqlens[n], i = L - 1;
        int64_t *keys = (int64_t *)malloc(sizeof(int64_t) * (size_t)(L + top_k + 1));
        int64_t c = 0;
        for (int64_t t = 0; t <= i; ++t)
            if (in_window(t, i, block_size, n_sink, n_local)) keys[c++] = t;
        for (int j = 0; j < top_k; ++j)
            if (selected && selected[(int64_t)n * top_k + j] >= 0) keys[c++] = selected[(int64_t)n * top_k + j];
        double *z = (double *)malloc(sizeof(double) * (size_t)(c + 1));
        for (int h = 0; h < n_heads; ++h) {
            const uint16_t *qh = q + ((int64_t)n * n_heads + h) * d_qk;
            double mx = -INFINITY;
            for (int64_t a = 0; a < c; ++a) {
                const uint16_t *kr = kv + n * batch_stride + keys[a] * row_stride;
                double s = 0.0;
                for (int e = 0; e < d_qk; ++e) s += widen(qh[e]) * widen(kr[e]);
                z[a] = scale * s;
                if (z[a] > mx) mx = z[a];
            }
            double sum = 0.0;
            for (int64_t a = 0; a < c; ++a) sum += exp(z[a] - mx);
            const double l = mx + log(sum);
            double *oh = o + ((int64_t)n * n_heads + h) * d_v;
            for (int e = 0; e < d_v; ++e) oh[e] = 0.0;
            for (int64_t a = 0; a < c; ++a) {
                const double w = exp(z[a] - l);
                const uint16_t *vr = kv + n * batch_stride + keys[a] * row_stride;
                for (int e = 0; e < d_v; ++e) oh[e] += w * widen(vr[e]);
            }
            lse[(int64_t)n * n_heads + h] = l;
        }
        free(z);
        free(keys);
    }
    return 0;
}
