/*
 * ssa_ref.c - plain fp64 CPU oracle for LoZA streaming sparse attention (SSA).
 *
 * TEST INFRASTRUCTURE. This file is the slow, obviously-correct reference that
 * the CUDA library is checked against. Only the test suite, the smoke check and
 * the benchmark's CPU-baseline leg may load it. It shares no code, header or
 * table with the CUDA library and the library never calls it.
 *
 * What it computes (Efficient Context Scaling with LongCat ZigZag Attention):
 *   - Page 1 (163.com summary), section 01 (1) "calibration": the sparse branch
 *     of a sparsified MLA module is softmax attention over selected, blocked
 *     keys/values K*, V*, defined by the number of sink blocks s, the number of
 *     local blocks l and the block size b; the pattern is "streaming": every
 *     query sees a few sink blocks and its local blocks. The equation itself is
 *     lost in the page text; this oracle takes the plain scaled-dot-product
 *     softmax over exactly those keys.
 *   - Page 1, section 01 (2) "post-training": b = 128, s = 1, l = 7, a window of
 *     1,024 tokens. Page 2 (intelliparadigm blog) section 2.2 and page 5
 *     (QbitAI article) restate "1 + 7 blocks of 128 tokens"; page 2 section 2.2
 *     and page 5 give the cost as O(L*S) with S = 1024.
 *
 * Readings taken where the pages are silent (each listed in the design notes):
 *   - the local blocks include the query's own block: j-l+1 .. j, so 1 + 7
 *     blocks make exactly 1,024 tokens;
 *   - inside block j attention is token-causal (t <= i);
 *   - sink blocks are the first s blocks of each sequence; blocks restart at
 *     every sequence start of a packed batch; a short last block is allowed;
 *   - sink and local sets are united, so early query blocks see 0..j once;
 *   - LSE is the natural log of the sum of exp of the scaled logits.
 *
 * Per sequence n (rows cu[n] .. cu[n+1]-1, positions relative to cu[n]),
 * head h and query position i, with j = floor(i / b):
 *   1. Blocks(i) = {0 .. min(s, j+1)-1} U {max(0, j-l+1) .. j}
 *   2. A(i)      = { t : floor(t/b) in Blocks(i), t <= i }
 *   3. z_t       = scale * sum_d q[i,h,d] k[t,hk,d]               (t in A(i))
 *   4. LSE_i     = M + ln sum_t exp(z_t - M),  M = max_t z_t
 *   5. O_i       = sum_t exp(z_t - LSE_i) v[t,hk,:]
 *   Decode: the query is position L_n - 1 against cache rows 0 .. L_n - 1.
 *   Backward with upstream dO (same page 1, section 01 "training": the model is
 *   mid-trained with SSA in place, so SSA needs its gradients):
 *     D_i = dO_i . O_i ; P_it = exp(z_t - LSE_i) ; dP_it = dO_i . v_t ;
 *     dS_it = P_it (dP_it - D_i) ; dQ_i = scale sum_t dS_it k_t ;
 *     dK_t = scale sum_{i : t in A(i)} dS_it q_i ; dV_t = sum_{i : t in A(i)} P_it dO_i
 *
 * All inputs are bf16 bit patterns (uint16) widened exactly to double. n_local
 * < 0 means an unbounded local window (plain causal attention when n_sink = 0).
 * kv head hk = h / (n_heads / n_kv_heads).
 *
 * A second window, token-granular (ssa_oracle_forward_tokens_rows; page 4, the
 * LSA article's streaming-aware index of 16 sink tokens and a 1,024-token
 * sliding window), replaces steps 1-2 by
 *   A(i) = { t <= i : t < sink_tokens  or  i - t < window_tokens }
 * and keeps steps 3-5.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static double widen(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Step 1 as a predicate: is key block kb among Blocks(i) for query block j? */
static int block_selected(int64_t j, int64_t kb, int n_sink, int n_local) {
    if (kb > j) return 0;
    if (kb < n_sink) return 1;
    if (n_local < 0) return 1;
    return kb >= j - n_local + 1;
}

/* Steps 1-2: write A(i) into keys[] in increasing order of t; return |A(i)|.
 * keys[] must have room for i + 1 entries. */
static int64_t visible_keys(int64_t i, int b, int n_sink, int n_local, int64_t *keys) {
    const int64_t j = i / b;
    int64_t c = 0;
    for (int64_t kb = 0; kb <= j; ++kb) {
        if (!block_selected(j, kb, n_sink, n_local)) continue;
        for (int64_t t = kb * b; t < (kb + 1) * b && t <= i; ++t) keys[c++] = t;
    }
    return c;
}

/* The token-granular variant (page 4, the LSA article's streaming-aware
 * index: a fixed part of every query's key set made of the first sink tokens
 * and a sliding window of the most recent tokens, 16 + 1,024 there):
 *   A(i) = { t <= i : t < sink_tokens  or  i - t < window_tokens }.
 * Written into keys[] in increasing order of t; returns |A(i)|. */
static int64_t visible_tokens(int64_t i, int64_t sink_tokens, int64_t window_tokens, int64_t *keys) {
    int64_t c = 0;
    for (int64_t t = 0; t <= i; ++t)
        if (t < sink_tokens || i - t < window_tokens) keys[c++] = t;
    return c;
}

typedef struct {
    const uint16_t *q, *k, *v;   /* [T,H,dqk], [T,Hkv,dqk], [T,Hkv,dv] */
    int64_t total;
    int n_heads, n_kv_heads, d_qk, d_v;
    int b, n_sink, n_local;
    double scale;
    int64_t sink_tokens, window_tokens;  /* token-granular variant when window_tokens > 0 */
} problem;

/* Steps 3-5 for query position i of the sequence starting at global row base,
 * head h. keys[] and z[] need room for i + 1 entries; on return they hold A(i)
 * and the scaled logits. Writes o[d_v], returns LSE, sets *count = |A(i)|. */
static double row_forward(const problem *p, int64_t base, int64_t i, int h,
                          int64_t *keys, double *z, int64_t *count, double *o) {
    const int hk = h / (p->n_heads / p->n_kv_heads);
    const uint16_t *qi = p->q + ((base + i) * p->n_heads + h) * (int64_t)p->d_qk;
    const int64_t c = p->window_tokens > 0 ? visible_tokens(i, p->sink_tokens, p->window_tokens, keys)
                                           : visible_keys(i, p->b, p->n_sink, p->n_local, keys);
    double m = -INFINITY;
    for (int64_t a = 0; a < c; ++a) {
        const uint16_t *kt = p->k + ((base + keys[a]) * p->n_kv_heads + hk) * (int64_t)p->d_qk;
        double acc = 0.0;
        for (int d = 0; d < p->d_qk; ++d) acc += widen(qi[d]) * widen(kt[d]);
        z[a] = p->scale * acc;
        if (z[a] > m) m = z[a];
    }
    double sum = 0.0;
    for (int64_t a = 0; a < c; ++a) sum += exp(z[a] - m);
    const double lse = m + log(sum);
    for (int d = 0; d < p->d_v; ++d) o[d] = 0.0;
    for (int64_t a = 0; a < c; ++a) {
        const double pt = exp(z[a] - lse);
        const uint16_t *vt = p->v + ((base + keys[a]) * p->n_kv_heads + hk) * (int64_t)p->d_v;
        for (int d = 0; d < p->d_v; ++d) o[d] += pt * widen(vt[d]);
    }
    *count = c;
    return lse;
}

/* Locate the sequence that holds global row g. */
static int seq_of_row(const int32_t *cu, int batch, int64_t g) {
    int lo = 0, hi = batch - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) / 2;
        if (cu[mid] <= g) lo = mid; else hi = mid - 1;
    }
    return lo;
}

static int check_shape(const int32_t *cu, int batch, int n_heads, int n_kv_heads,
                       int d_qk, int d_v, int block_size) {
    if (batch < 1 || n_heads < 1 || n_kv_heads < 1 || n_heads % n_kv_heads) return -1;
    if (block_size < 1 || d_qk < 1 || d_v < 1) return -1;
    if (cu && cu[0] != 0) return -1;
    if (cu)
        for (int n = 0; n < batch; ++n)
            if (cu[n + 1] < cu[n]) return -1;
    return 0;
}

/* Steps 3-5 for a list of global query rows, all heads of each row. */
static int forward_rows(const problem *pp, const int32_t *cu_seqlens, int batch, const int64_t *rows,
                        int64_t n_rows, double *o_out, double *lse_out) {
    const problem p = *pp;
    const int n_heads = p.n_heads, d_v = p.d_v;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int64_t r = 0; r < n_rows * n_heads; ++r) {
        const int64_t ri = r / n_heads;
        const int h = (int)(r % n_heads);
        const int64_t g = rows[ri];
        if (g < 0 || g >= p.total) { bad |= 1; continue; }
        const int n = seq_of_row(cu_seqlens, batch, g);
        const int64_t base = cu_seqlens[n], i = g - base;
        int64_t *keys = (int64_t *)malloc(sizeof(int64_t) * (size_t)(i + 1));
        double *z = (double *)malloc(sizeof(double) * (size_t)(i + 1));
        int64_t c;
        lse_out[ri * n_heads + h] = row_forward(&p, base, i, h, keys, z, &c,
                                                o_out + (ri * n_heads + h) * (int64_t)d_v);
        free(keys);
        free(z);
    }
    return bad ? -1 : 0;
}

/*
 * Forward for a list of global query rows (all heads of each row).
 * rows: n_rows global row indices in [0, cu[batch]).
 * o_out [n_rows, H, d_v], lse_out [n_rows, H].
 */
int ssa_oracle_forward_rows(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                            const int32_t *cu_seqlens, int batch,
                            int n_heads, int n_kv_heads, int d_qk, int d_v,
                            int block_size, int n_sink, int n_local, double scale,
                            const int64_t *rows, int64_t n_rows,
                            double *o_out, double *lse_out) {
    if (!q || !k || !v || !cu_seqlens || !rows || !o_out || !lse_out) return -1;
    if (check_shape(cu_seqlens, batch, n_heads, n_kv_heads, d_qk, d_v, block_size)) return -1;
    problem p = {q, k, v, cu_seqlens[batch], n_heads, n_kv_heads, d_qk, d_v,
                 block_size, n_sink, n_local, scale, 0, 0};
    return forward_rows(&p, cu_seqlens, batch, rows, n_rows, o_out, lse_out);
}

/*
 * The same for the token-granular window (visible_tokens): sink_tokens >= 0,
 * window_tokens >= 1.
 */
int ssa_oracle_forward_tokens_rows(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                                   const int32_t *cu_seqlens, int batch,
                                   int n_heads, int n_kv_heads, int d_qk, int d_v,
                                   int64_t sink_tokens, int64_t window_tokens, double scale,
                                   const int64_t *rows, int64_t n_rows,
                                   double *o_out, double *lse_out) {
    if (!q || !k || !v || !cu_seqlens || !rows || !o_out || !lse_out) return -1;
    if (check_shape(cu_seqlens, batch, n_heads, n_kv_heads, d_qk, d_v, 1)) return -1;
    if (sink_tokens < 0 || window_tokens < 1) return -1;
    problem p = {q, k, v, cu_seqlens[batch], n_heads, n_kv_heads, d_qk, d_v,
                 1, 0, 0, scale, sink_tokens, window_tokens};
    return forward_rows(&p, cu_seqlens, batch, rows, n_rows, o_out, lse_out);
}

/*
 * Decode: sequence n's query q[n] (its last token, position L_n - 1) against
 * cache rows 0 .. L_n - 1 of that sequence (step 6 of the definition).
 * q [B,H,d_qk]; sequence n's cache row t lives at
 *   k_cache + ((n*cache_batch_rows + t)*Hkv + hk)*d_qk, and its value row at
 *   v_cache + (n*cache_batch_rows + t)*v_row_elems + hk*d_v
 * (v_row_elems = Hkv*d_v for a separate V cache; for an absorbed latent cache
 * v_cache = k_cache and v_row_elems = d_qk, so V is the first d_v columns).
 * o_out [B,H,d_v], lse_out [B,H].
 */
int ssa_oracle_decode(const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                      int64_t cache_batch_rows, int64_t v_row_elems, const int32_t *seqlens, int batch,
                      int n_heads, int n_kv_heads, int d_qk, int d_v,
                      int block_size, int n_sink, int n_local, double scale,
                      double *o_out, double *lse_out) {
    if (!q || !k_cache || !v_cache || !seqlens || !o_out || !lse_out) return -1;
    if (check_shape(NULL, batch, n_heads, n_kv_heads, d_qk, d_v, block_size)) return -1;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int64_t r = 0; r < (int64_t)batch * n_heads; ++r) {
        const int n = (int)(r / n_heads), h = (int)(r % n_heads);
        const int64_t L = seqlens[n];
        if (L < 1 || L > cache_batch_rows) { bad |= 1; continue; }
        /* the cache of sequence n, seen as a one-sequence problem whose query
         * row L-1 carries q[n] */
        const int hk = h / (n_heads / n_kv_heads);
        const int64_t i = L - 1;
        const uint16_t *qi = q + ((int64_t)n * n_heads + h) * d_qk;
        const uint16_t *kc = k_cache + (int64_t)n * cache_batch_rows * n_kv_heads * d_qk;
        const uint16_t *vc = v_cache + (int64_t)n * cache_batch_rows * v_row_elems;
        int64_t *keys = (int64_t *)malloc(sizeof(int64_t) * (size_t)L);
        double *z = (double *)malloc(sizeof(double) * (size_t)L);
        const int64_t c = visible_keys(i, block_size, n_sink, n_local, keys);
        double m = -INFINITY;
        for (int64_t a = 0; a < c; ++a) {
            const uint16_t *kt = kc + (keys[a] * n_kv_heads + hk) * (int64_t)d_qk;
            double acc = 0.0;
            for (int d = 0; d < d_qk; ++d) acc += widen(qi[d]) * widen(kt[d]);
            z[a] = scale * acc;
            if (z[a] > m) m = z[a];
        }
        double sum = 0.0;
        for (int64_t a = 0; a < c; ++a) sum += exp(z[a] - m);
        const double lse = m + log(sum);
        double *o = o_out + r * (int64_t)d_v;
        for (int d = 0; d < d_v; ++d) o[d] = 0.0;
        for (int64_t a = 0; a < c; ++a) {
            const double pt = exp(z[a] - lse);
            const uint16_t *vt = vc + keys[a] * v_row_elems + (int64_t)hk * d_v;
            for (int d = 0; d < d_v; ++d) o[d] += pt * widen(vt[d]);
        }
        lse_out[r] = lse;
        free(keys);
        free(z);
    }
    return bad ? -1 : 0;
}

/*
 * Backward on a sample: dQ for the listed query rows, dK/dV for the listed key
 * rows. Every query that a listed key row feeds is evaluated in full (its own
 * O, LSE and D), so each listed output is exact; nothing else is computed.
 * dout [T,H,d_v] bf16 bits. dq_out [n_q_rows,H,d_qk];
 * dk_out [n_k_rows,Hkv,d_qk]; dv_out [n_k_rows,Hkv,d_v].
 */
int ssa_oracle_backward_rows(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                             const uint16_t *dout, const int32_t *cu_seqlens, int batch,
                             int n_heads, int n_kv_heads, int d_qk, int d_v,
                             int block_size, int n_sink, int n_local, double scale,
                             const int64_t *q_rows, int64_t n_q_rows,
                             const int64_t *k_rows, int64_t n_k_rows,
                             double *dq_out, double *dk_out, double *dv_out) {
    if (!q || !k || !v || !dout || !cu_seqlens) return -1;
    if (n_q_rows > 0 && (!q_rows || !dq_out)) return -1;
    if (n_k_rows > 0 && (!k_rows || !dk_out || !dv_out)) return -1;
    if (check_shape(cu_seqlens, batch, n_heads, n_kv_heads, d_qk, d_v, block_size)) return -1;
    problem p = {q, k, v, cu_seqlens[batch], n_heads, n_kv_heads, d_qk, d_v,
                 block_size, n_sink, n_local, scale, 0, 0};
    const int group = n_heads / n_kv_heads;
    int bad = 0;

    /* dQ_i = scale * sum_{t in A(i)} dS_it k_t */
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int64_t r = 0; r < n_q_rows * n_heads; ++r) {
        const int64_t ri = r / n_heads;
        const int h = (int)(r % n_heads), hk = h / group;
        const int64_t g = q_rows[ri];
        if (g < 0 || g >= p.total) { bad |= 1; continue; }
        const int n = seq_of_row(cu_seqlens, batch, g);
        const int64_t base = cu_seqlens[n], i = g - base;
        int64_t *keys = (int64_t *)malloc(sizeof(int64_t) * (size_t)(i + 1));
        double *z = (double *)malloc(sizeof(double) * (size_t)(i + 1));
        double *o = (double *)malloc(sizeof(double) * (size_t)d_v);
        int64_t c;
        const double lse = row_forward(&p, base, i, h, keys, z, &c, o);
        const uint16_t *doi = dout + (g * n_heads + h) * (int64_t)d_v;
        double D = 0.0;
        for (int d = 0; d < d_v; ++d) D += widen(doi[d]) * o[d];
        double *dq = dq_out + (ri * n_heads + h) * (int64_t)d_qk;
        for (int d = 0; d < d_qk; ++d) dq[d] = 0.0;
        for (int64_t a = 0; a < c; ++a) {
            const int64_t t = keys[a];
            const double P = exp(z[a] - lse);
            const uint16_t *vt = v + ((base + t) * n_kv_heads + hk) * (int64_t)d_v;
            double dP = 0.0;
            for (int d = 0; d < d_v; ++d) dP += widen(doi[d]) * widen(vt[d]);
            const double dS = P * (dP - D);
            const uint16_t *kt = k + ((base + t) * n_kv_heads + hk) * (int64_t)d_qk;
            for (int d = 0; d < d_qk; ++d) dq[d] += scale * dS * widen(kt[d]);
        }
        free(keys);
        free(z);
        free(o);
    }

    /* dK_t, dV_t: sum over every (query i, head h of kv head hk) with t in A(i) */
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int64_t r = 0; r < n_k_rows * n_kv_heads; ++r) {
        const int64_t ri = r / n_kv_heads;
        const int hk = (int)(r % n_kv_heads);
        const int64_t g = k_rows[ri];
        if (g < 0 || g >= p.total) { bad |= 1; continue; }
        const int n = seq_of_row(cu_seqlens, batch, g);
        const int64_t base = cu_seqlens[n], t = g - base;
        const int64_t L = cu_seqlens[n + 1] - base;
        double *dk = dk_out + (ri * n_kv_heads + hk) * (int64_t)d_qk;
        double *dv = dv_out + (ri * n_kv_heads + hk) * (int64_t)d_v;
        for (int d = 0; d < d_qk; ++d) dk[d] = 0.0;
        for (int d = 0; d < d_v; ++d) dv[d] = 0.0;
        int64_t *keys = (int64_t *)malloc(sizeof(int64_t) * (size_t)L);
        double *z = (double *)malloc(sizeof(double) * (size_t)L);
        double *o = (double *)malloc(sizeof(double) * (size_t)d_v);
        const uint16_t *vt = v + (g * n_kv_heads + hk) * (int64_t)d_v;
        for (int64_t i = t; i < L; ++i) {
            if (!block_selected(i / block_size, t / block_size, n_sink, n_local)) continue;
            for (int h = hk * group; h < (hk + 1) * group; ++h) {
                int64_t c;
                const double lse = row_forward(&p, base, i, h, keys, z, &c, o);
                /* position of t inside A(i) (keys[] is increasing) */
                int64_t lo = 0, hi = c - 1;
                while (lo < hi) {
                    const int64_t mid = (lo + hi) / 2;
                    if (keys[mid] < t) lo = mid + 1; else hi = mid;
                }
                if (c == 0 || keys[lo] != t) { bad |= 2; continue; }
                const uint16_t *doi = dout + ((base + i) * n_heads + h) * (int64_t)d_v;
                const uint16_t *qi = q + ((base + i) * n_heads + h) * (int64_t)d_qk;
                double D = 0.0, dP = 0.0;
                for (int d = 0; d < d_v; ++d) D += widen(doi[d]) * o[d];
                for (int d = 0; d < d_v; ++d) dP += widen(doi[d]) * widen(vt[d]);
                const double P = exp(z[lo] - lse);
                const double dS = P * (dP - D);
                for (int d = 0; d < d_qk; ++d) dk[d] += scale * dS * widen(qi[d]);
                for (int d = 0; d < d_v; ++d) dv[d] += P * widen(doi[d]);
            }
        }
        free(keys);
        free(z);
        free(o);
    }
    return bad ? -1 : 0;
}

/* |A(i)| as the oracle's index map gives it (used by the pins). */
int64_t ssa_oracle_visible_count(int64_t i, int block_size, int n_sink, int n_local) {
    int64_t *keys = (int64_t *)malloc(sizeof(int64_t) * (size_t)(i + 1));
    const int64_t c = visible_keys(i, block_size, n_sink, n_local, keys);
    free(keys);
    return c;
}

/*
 * Combining two attention branches of one query (an adjacent step of the same
 * operator; page 1 section 01 (1) "calibration": during calibration an MLA
 * module's output is a weighted mix of its full-attention branch and its
 * sparse (SSA) branch; the formula is lost in the page text, and this oracle
 * takes the plain reading alpha * O_full + (1 - alpha) * O_ssa).
 *
 * ssa_oracle_merge: branches a and b are softmax attention of the same query
 * over two disjoint key sets A and B, given as (O, LSE); the result is
 * attention over A U B:
 *   LSE = ln(exp(LSE_a) + exp(LSE_b))
 *   O   = exp(LSE_a - LSE) O_a + exp(LSE_b - LSE) O_b
 * A branch with LSE = -inf has no keys and weight 0; if both have none the
 * result is O = 0, LSE = -inf. Rows are (token, head) pairs; O is [rows, d_v]
 * bf16 bits, LSE [rows] (fp32 values widened to double by the caller).
 *
 * ssa_oracle_mix: O = alpha * O_full + (1 - alpha) * O_ssa, elementwise.
 */
int ssa_oracle_merge(const uint16_t *o_a, const double *lse_a, const uint16_t *o_b, const double *lse_b,
                     int64_t rows, int d_v, double *o, double *lse) {
    if (rows < 0 || d_v < 1) return -1;
    for (int64_t r = 0; r < rows; ++r) {
        const double la = lse_a[r], lb = lse_b[r];
        double wa = 0.0, wb = 0.0, l = -INFINITY;
        if (la != -INFINITY || lb != -INFINITY) {
            const double m = la > lb ? la : lb;
            l = m + log(exp(la - m) + exp(lb - m));
            wa = exp(la - l);
            wb = exp(lb - l);
        }
        lse[r] = l;
        for (int d = 0; d < d_v; ++d)
            o[r * d_v + d] = wa * widen(o_a[r * d_v + d]) + wb * widen(o_b[r * d_v + d]);
    }
    return 0;
}

int ssa_oracle_mix(const uint16_t *o_full, const uint16_t *o_ssa, int64_t n, double alpha, double *o) {
    if (n < 0) return -1;
    for (int64_t i = 0; i < n; ++i) o[i] = alpha * widen(o_full[i]) + (1.0 - alpha) * widen(o_ssa[i]);
    return 0;
}
