/*
 * loza_ssa.h - C ABI of the B200 (sm_100a) streaming sparse attention library.
 *
 * Streaming sparse attention (SSA) is the sparse branch of LongCat ZigZag
 * Attention (Efficient Context Scaling with LongCat ZigZag Attention, page 1,
 * section 01 (1) "calibration"): every query token attends, by softmax
 * attention, only to selected and blocked keys/values K*, V*, defined by the
 * block size b, the number of sink blocks s and the number of local blocks l.
 * Page 1 section 01 (2) fixes b = 128, s = 1, l = 7, a 1,024-token window;
 * page 5 (QbitAI article) describes it as one global block and seven local
 * blocks of 128 tokens. With query position i in block j = floor(i/b), the keys
 * of a query are
 *     t <= i  with  floor(t/b) in {0 .. s-1} U {j-l+1 .. j}
 * i.e. the sink blocks, the l most recent blocks including its own, and
 * token-causal inside its own block (the "streaming" pattern). Blocks restart
 * at every sequence start of a packed batch; a sequence's last block may be
 * short.
 *
 * The operator runs inside MLA modules (page 1 section 01 (1); page 2 section
 * 1.2). Two layouts are supported:
 *   - per-head K/V ("non-absorbed" MLA, MHA): n_kv_heads == n_heads,
 *     (d_qk, d_v) in {(64, 64), (192, 128)};
 *   - one latent KV row shared by all heads ("absorbed" MLA): n_kv_heads == 1,
 *     d_qk = 576 (512 latent + 64 rope) and d_v = 512, where V is the first 512
 *     columns of the latent row (pass v == k).
 *
 * Conventions for every entry point:
 *   - All pointers named q, k, v, out, dout, dq, dk, dv, lse, workspace,
 *     cu_seqlens and seqlens are DEVICE pointers. bf16 tensors are raw bf16
 *     bit patterns. The caller owns and allocates every buffer; the library
 *     never allocates, frees or synchronises.
 *   - Calls are asynchronous on `stream` (0 = legacy default stream).
 *   - Validation errors return a negative status BEFORE anything is launched.
 *     A launch failure returns LOZA_ERR_CUDA. Kernels never trap; a kernel
 *     that gives up on a bounded wait records LOZA_ERR_TIMEOUT, which
 *     loza_device_status() reports.
 *   - Strides are in elements. Rows (tokens) may be strided; within a row,
 *     heads are contiguous with head stride = head dim.
 *   - Every row stride times 2 bytes and every base pointer must be 16-byte
 *     aligned (TMA requirement); otherwise LOZA_ERR_INVALID_ARG.
 *   - Window: block_size b a power of two from 1 to 65,536; n_sink >= 0,
 *     n_local >= 1 (n_sink * b and n_local * b at most 2^30), or n_local ==
 *     LOZA_UNBOUNDED for full causal attention (n_sink ignored). The keys of
 *     query position i are then {t <= i : t < n_sink * b or t >= lo(i)}, lo(i)
 *     = max(0, (floor(i / b) - n_local + 1) * b). b = 1 makes every token a
 *     block: {1, 16, 1024} is the fixed part of the streaming-aware index of
 *     page 4 ("LongCat Sparse Attention ...", agihunt.info), 16 sink tokens
 *     and a 1,024-token sliding window that includes the query. The prefill
 *     and decode entry points take any such window, and so does
 *     loza_ssa_backward (bounded windows only) and loza_ssa_prefill_host.
 *     Keys are read in tiles of 128 (64 in
 *     the half-block decode): the cache rows of positions below seqlens[n]
 *     that share a tile with a visible key are read and must hold finite
 *     values (they are the sequence's own context); rows at or past
 *     seqlens[n] never reach the result, whatever they hold.
 */
#ifndef LOZA_SSA_H
#define LOZA_SSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* cudaStream_t without the CUDA headers: the same opaque pointer. */
typedef struct CUstream_st *loza_stream_t;

/* Window parameters {b, s, l, scale}; the pages' configuration is
 * {128, 1, 7, scale}; {1, 16, 1024, scale} is page 4's token-granular sink
 * and sliding window. scale multiplies q.k before the softmax. */
typedef struct {
    int32_t block_size;
    int32_t n_sink;
    int32_t n_local;
    float scale;
} loza_ssa_params;

/* n_local value selecting full causal attention (the dense baseline). */
#define LOZA_UNBOUNDED (-1)

typedef enum {
    LOZA_OK = 0,
    LOZA_ERR_INVALID_ARG = -1,
    LOZA_ERR_UNSUPPORTED = -2,
    LOZA_ERR_WORKSPACE = -3,
    LOZA_ERR_CUDA = -4,
    LOZA_ERR_TIMEOUT = -5
} loza_status;

/* Operation codes for loza_ssa_workspace_size. */
#define LOZA_OP_PREFILL 0
#define LOZA_OP_DECODE 1
#define LOZA_OP_BACKWARD 2
#define LOZA_OP_PREFILL_HOST 3

/*
 * Bytes of device workspace the operation needs for this shape (0 if none).
 * batch: number of sequences; total_tokens: packed tokens (prefill/backward);
 * max_seqlen: longest sequence (decode: longest context). Returns 0 for an
 * unsupported shape as well; the entry point then reports the error.
 */
size_t loza_ssa_workspace_size(int op, int32_t batch, int64_t total_tokens, int32_t max_seqlen,
                               int32_t n_heads, int32_t n_kv_heads, int32_t d_qk, int32_t d_v,
                               loza_ssa_params p);

/*
 * Prefill / training forward over a packed variable-length batch.
 *   q   [T, n_heads, d_qk]     bf16, token stride q_row_stride (>= n_heads*d_qk)
 *   k   [T, n_kv_heads, d_qk]  bf16, token stride k_row_stride
 *   v   [T, n_kv_heads, d_v]   bf16, token stride v_row_stride (absorbed: v == k,
 *                              v_row_stride == k_row_stride, V = first d_v columns)
 *   cu_seqlens int32 [batch+1], cu_seqlens[0] = 0, non-decreasing,
 *               cu_seqlens[batch] == total_tokens (T)
 *   total_tokens T, the packed row count of q, k, v, out and lse (the bound the
 *               TMA descriptors are built with; rows past T read as zero)
 *   max_seqlen  >= every sequence length (sizes the launch grid)
 *   out [T, n_heads, d_v] bf16 contiguous; lse [T, n_heads] fp32, natural log of
 *   the sum of exp(scale * q.k) over the visible keys.
 *   workspace: optional. For the absorbed shapes (n_kv_heads 1, 576 / 512,
 *               even n_heads) with a bounded window of at most 32 blocks
 *               (n_sink + n_local <= 32), a workspace of at least
 *               loza_ssa_workspace_size(LOZA_OP_PREFILL, ...) bytes lets the
 *               kernel compute S once for both halves of the value dimension
 *               (it keeps P there between the two halves); with NULL or fewer
 *               bytes it recomputes S per half. Same results either way up to
 *               rounding order; the workspace is scratch owned by the caller
 *               and must not be used by other work running at the same time.
 * Definition: page 1 section 01 (1) and (2) of the LoZA pages (see above).
 */
loza_status loza_ssa_prefill(const void *q, const void *k, const void *v,
                             const int32_t *cu_seqlens, int32_t batch, int64_t total_tokens,
                             int32_t max_seqlen,
                             int32_t n_heads, int32_t n_kv_heads, int32_t d_qk, int32_t d_v,
                             int64_t q_row_stride, int64_t k_row_stride, int64_t v_row_stride,
                             loza_ssa_params p, void *out, float *lse,
                             void *workspace, size_t workspace_bytes, loza_stream_t stream);

/*
 * Prefill of a packed batch whose tensors live in host memory: the operation
 * and results of loza_ssa_prefill (same kernels; every output row is computed
 * exactly as in a device-resident call with the same cu_seqlens), with the
 * host-to-device copies of the inputs and the device-to-host copies of the
 * outputs inside the call. (The LoZA pages have no counterpart to this entry
 * point; it exists for callers whose activations are on the host.)
 *   q   [T, n_heads, d_qk]     bf16, contiguous rows
 *   k   [T, n_kv_heads, d_qk]  bf16, contiguous rows
 *   v   [T, n_kv_heads, d_v]   bf16, contiguous rows; absorbed MLA: v == k
 *                              (V = the first d_v columns of the latent row)
 *   out [T, n_heads, d_v] bf16 and lse [T, n_heads] fp32 (written)
 *   cu_seqlens: HOST int32 [batch+1], 0 = cu_seqlens[0] <= ... <=
 *               cu_seqlens[batch] = total_tokens (T); no sequence longer than
 *               max_seqlen; empty sequences are allowed
 * These five tensors may be host memory (page-locked memory lets the copies
 * run asynchronously and overlap; pageable memory gives the same results but
 * the copies serialise) or device memory; they are addressed through the
 * unified address space.
 * How it runs: each sequence's query rows are cut into chunks of whole units
 * of U = max(b, 128) rows (about 16 chunks per sequence, of 1,024 to 8,192
 * rows, at least as many as the prefix below; the unbounded window is one
 * chunk per sequence). A chunk's own rows [q0, q1) run as the local sequence
 * [sink rows | zero rows | rows q0-(l-1)b .. q0-1 | own rows] with zero query
 * rows before the own ones; the prefix is the smallest multiple of U that
 * holds the sink rows rounded up to whole 128-row tiles plus the (l-1)b halo
 * rows (exactly s + l - 1 blocks for b = 128). By the window rule (page 1
 * section 01 (1) of the LoZA pages) every own query then sees exactly its
 * keys of the whole sequence, each in the same place of its 128-row tile, so
 * the kernels read them in the same order. Up to three chunks are in flight: the
 * copy-in of one, the kernels of the next and the copy-out of a third
 * overlap, on two copy streams that the library creates on the first call per
 * device and keeps until exit. The call is asynchronous on `stream`: when
 * `stream` reaches this point of its work, out and lse hold the results.
 * Supported shapes are those of loza_ssa_prefill with n_kv_heads in
 * {1, n_heads}: (d_qk, d_v) in {(64, 64), (192, 128)} and the absorbed
 * (576, 512) with an even n_heads.
 *   workspace: device memory, 256-byte aligned, of at least
 *   loza_ssa_workspace_size(LOZA_OP_PREFILL_HOST, batch, T, max_seqlen, ...)
 *   bytes (chunk slots sized for the longest sequence, and the chunks' local
 *   cu_seqlens), owned by the caller and used by nothing else until `stream`
 *   has passed this call.
 *   Errors: LOZA_ERR_INVALID_ARG / LOZA_ERR_UNSUPPORTED / LOZA_ERR_WORKSPACE
 *   before anything is enqueued; LOZA_ERR_CUDA if enqueueing fails part way
 *   (synchronise `stream` before reusing any buffer in that case).
 */
loza_status loza_ssa_prefill_host(const void *q, const void *k, const void *v, const int32_t *cu_seqlens,
                                  int32_t batch, int64_t total_tokens, int32_t max_seqlen,
                                  int32_t n_heads, int32_t n_kv_heads, int32_t d_qk, int32_t d_v,
                                  loza_ssa_params p, void *out, float *lse,
                                  void *workspace, size_t workspace_bytes, loza_stream_t stream);

/*
 * Decode: one new query token per sequence against its KV cache.
 *   q        [batch, n_heads, d_qk] bf16 contiguous; the query of sequence n is
 *            its last token, position seqlens[n]-1, whose KV row is already in
 *            the cache (page 1 section 02: the streaming kernel in decode)
 *   k_cache  sequence n's row t at k_cache + (n*cache_batch_stride + t*cache_row_stride)
 *            elements, [n_kv_heads, d_qk] bf16 per row
 *   v_cache  absorbed MLA: NULL (or == k_cache): V is the first d_v columns of
 *            the latent row. Per-head K/V: a second cache whose strides are the
 *            K strides scaled by d_v / d_qk (both caches are [batch, Lcap,
 *            n_kv_heads, d] arrays with the same Lcap).
 *   The cache must hold at least max_seqlen rows per sequence
 *   (cache_batch_stride >= max_seqlen * cache_row_stride); rows at or past
 *   seqlens[n] are never used, whatever they contain.
 *   seqlens  int32 [batch], 1 <= seqlens[n] <= max_seqlen
 *   out [batch, n_heads, d_v] bf16; lse [batch, n_heads] fp32
 *   workspace: loza_ssa_workspace_size(LOZA_OP_DECODE, ...) bytes (split-KV
 *   partial results); contents on entry are ignored.
 * Compiled shapes: absorbed MLA (n_kv_heads == 1, 64 heads, (576, 512)) on
 * tensor cores, with split-KV partials merged in-kernel; per-head K/V
 * ((64, 64) or (192, 128)) on CUDA cores, which needs no workspace.
 */
loza_status loza_ssa_decode(const void *q, const void *k_cache, const void *v_cache,
                            const int32_t *seqlens, int32_t batch, int32_t max_seqlen,
                            int64_t cache_batch_stride, int64_t cache_row_stride,
                            int32_t n_heads, int32_t n_kv_heads, int32_t d_qk, int32_t d_v,
                            loza_ssa_params p, void *out, float *lse,
                            void *workspace, size_t workspace_bytes, loza_stream_t stream);

/*
 * Hierarchical index decode (page 4, "LongCat Sparse Attention: Taming the
 * Lightning via Streaming-aware Hierarchical Cross-Layer Indexing",
 * agihunt.info: its streaming-aware index gives every query fixed sink and
 * window tokens plus dynamically selected tokens, and its hierarchical index
 * selects those in two stages, top pages of 128 tokens first, then top tokens
 * within them). The fixed part is the SSA window `p` of this library; the
 * dynamic part is chosen among the tokens outside it, so the parts are
 * disjoint, and the query attends to both at once (one softmax over their
 * union, the same as merging the two parts by their log-sum-exp).
 * Scoring (the pages give none): the dot product of the sequence's index
 * query with a token's index key, both supplied by the caller (as an indexer
 * produces them); a page is scored by the mean of its 128 index keys. Scores
 * are fp32 fused multiply-adds over the index dimension in order, so the
 * selection is one exact set; ties go to the lower page / token index.
 * Common arguments:
 *   k_index   index keys: token t of sequence n at k_index + n *
 *             index_batch_stride + t * index_row_stride elements, d_index bf16
 *             each (d_index a multiple of 64, at most 512; 16-byte aligned;
 *             strides * 2 multiples of 16; index_batch_stride >= max_seqlen *
 *             index_row_stride)
 *   q_index   [batch, d_index] bf16 contiguous, one index query per sequence
 *   page_keys [batch, d_index, max_seqlen / 128] fp32, the page dimension
 *             innermost (from loza_hi_page_keys)
 *   seqlens   device int32 [batch], 1 <= seqlens[n] <= max_seqlen; the decode
 *             query is position seqlens[n] - 1, as in loza_ssa_decode
 *   p         the window: as loza_ssa_decode's, with at most 65,536 rows
 *             ((n_sink + n_local) * block_size); LOZA_UNBOUNDED leaves no
 *             token outside the window, so nothing is selected
 * Limits: max_seqlen / 128 <= 8192 pages; 1 <= top_k <= 2048; top_pages >= 1.
 *
 * loza_hi_page_keys: the mean index key of every whole page (tokens 128p ..
 * 128p+127 all below seqlens[n]): fp32 sums in token order times 1/128. Pages
 * past a sequence's end are not written. Maintained by the caller as its cache
 * fills (a page's mean never changes once the page is whole).
 */
loza_status loza_hi_page_keys(const void *k_index, int64_t index_batch_stride, int64_t index_row_stride,
                              const int32_t *seqlens, int32_t batch, int32_t max_seqlen, int32_t d_index,
                              float *page_keys, loza_stream_t stream);

/* Bytes of device workspace loza_hi_select and loza_hi_decode need (0 for an
 * unsupported request); loza_ssa_decode_selected needs the size for
 * top_pages = 1. */
size_t loza_hi_workspace_size(int32_t batch, int32_t max_seqlen, int32_t top_pages, int32_t top_k,
                              loza_ssa_params p);

/*
 * The tokens the hierarchical index selects for each sequence's decode query:
 * the top_pages whole pages holding a token outside the window, by page score,
 * then the top_k tokens outside the window in those pages, by token score.
 *   selected  device int32 [batch, top_k]: the tokens in ascending order, then
 *             -1 where fewer than top_k were available
 *   workspace loza_hi_workspace_size(...) bytes, 256-byte aligned
 */
loza_status loza_hi_select(const void *q_index, const void *k_index, int64_t index_batch_stride,
                           int64_t index_row_stride, const float *page_keys, const int32_t *seqlens, int32_t batch,
                           int32_t max_seqlen, int32_t d_index, loza_ssa_params p, int32_t top_pages, int32_t top_k,
                           int32_t *selected, void *workspace, size_t workspace_bytes, loza_stream_t stream);

/*
 * Softmax attention of each sequence's decode query (position seqlens[n] - 1)
 * over its window p and the tokens of a given selection (absorbed MLA: 64
 * heads, the 576-wide latent row as K, its first 512 columns as V): out
 * [batch, 64, 512] bf16, lse [batch, 64] fp32 (natural log). q [batch, 64,
 * 576] bf16 contiguous; the cache layout is loza_ssa_decode's.
 *   selected  device int32 [batch, top_k] (0 <= top_k <= 2048): entries that
 *             name a token before the query and outside the window are
 *             attended, every other entry (negative, past the query, inside
 *             the window) is ignored; the entries must be distinct
 *   workspace loza_hi_workspace_size(batch, max_seqlen, 1, top_k, p) bytes,
 *             256-byte aligned
 * The window rows and the selected rows are packed per sequence in the
 * workspace and attended by the tensor-core decode.
 */
loza_status loza_ssa_decode_selected(const void *q, const void *kv_cache, int64_t cache_batch_stride,
                                     int64_t cache_row_stride, const int32_t *seqlens, int32_t batch,
                                     int32_t max_seqlen, loza_ssa_params p, const int32_t *selected, int32_t top_k,
                                     void *out, float *lse, void *workspace, size_t workspace_bytes,
                                     loza_stream_t stream);

/*
 * The whole decode: loza_hi_select, then loza_ssa_decode_selected over the
 * window p and that selection, into out [batch, 64, 512] bf16 and lse
 * [batch, 64]. Same cache arguments as loza_ssa_decode (absorbed MLA, 64
 * heads, 576 / 512).
 *   workspace loza_hi_workspace_size(...) bytes, 256-byte aligned
 */
loza_status loza_hi_decode(const void *q, const void *kv_cache, int64_t cache_batch_stride, int64_t cache_row_stride,
                           const void *q_index, const void *k_index, int64_t index_batch_stride,
                           int64_t index_row_stride, const float *page_keys, const int32_t *seqlens, int32_t batch,
                           int32_t max_seqlen, int32_t d_index, loza_ssa_params p, int32_t top_pages, int32_t top_k,
                           void *out, float *lse, void *workspace, size_t workspace_bytes, loza_stream_t stream);

/*
 * Decode without any caller-provided device memory. (The LoZA pages have no
 * counterpart to this entry point; it exists for callers of this library.)
 *
 * Some callers cannot allocate device memory at the point where they decode:
 * a host application that owns the device allocator and gives plug-ins no
 * access to it, a serving runtime that has reserved all device memory for its
 * own KV-cache pool up front, or a latency-critical loop that must not pay
 * for cudaMalloc/cudaFree. For them this entry point takes the same arguments
 * as loza_ssa_decode minus the workspace. The absorbed decode needs scratch
 * only when a few sequences have long windows (more than 8 selected blocks
 * and batch * 16 <= number of SMs): its split-KV partial results then go to a
 * fixed 16 MiB array that is part of the library itself. Every other call
 * merges its partials on chip and needs none.
 *   - The library never allocates: every GPU that loads the library holds the
 *     16 MiB array until the process exits. With CUDA's lazy module loading
 *     (the default since CUDA 12.2) the array is placed on a device at the
 *     first call into this library on that device, whichever entry point it
 *     is; a runtime that reserves nearly all device memory for its own pool
 *     should make one call into the library on each device before it does so.
 *   - Limit: a call that needs scratch needs batch * nsplit * 132,096 bytes
 *     plus 256 for the counters, with nsplit = min(selected blocks,
 *     ceil(SMs / batch)), so it fits when batch * nsplit <= 127; e.g. with
 *     the unbounded window on a 148-SM B200, one sequence of up to 16,256
 *     tokens or four of up to 3,968 tokens. A larger call returns
 *     LOZA_ERR_WORKSPACE before anything is launched; use loza_ssa_decode with
 *     a workspace instead, or split the batch.
 *   - Every call that needs scratch looks up the array's device address on
 *     the current device (the first such call on a device also loads the
 *     library's device code there, if no earlier call did); make that first
 *     call before any stream capture on that device. After cudaDeviceReset
 *     the next call finds the array at its new address.
 *   - Every call uses the same array and leaves its last contents there; the
 *     arrival counters are cleared on the caller's stream at the start of each
 *     call. Two calls whose kernels can overlap on the GPU (different streams
 *     without ordering between them) race on the array and give wrong results.
 *   - Per-head K/V shapes need no scratch and behave exactly like
 *     loza_ssa_decode.
 */
loza_status loza_ssa_decode_noalloc(const void *q, const void *k_cache, const void *v_cache,
                                    const int32_t *seqlens, int32_t batch, int32_t max_seqlen,
                                    int64_t cache_batch_stride, int64_t cache_row_stride,
                                    int32_t n_heads, int32_t n_kv_heads, int32_t d_qk, int32_t d_v,
                                    loza_ssa_params p, void *out, float *lse, loza_stream_t stream);

/*
 * Training backward of loza_ssa_prefill (page 1 section 01 "training": the
 * model is mid-trained with SSA in place). Given q, k, v, the forward out and
 * lse, and the upstream gradient dout [T, n_heads, d_v] (bf16, contiguous),
 * writes dq [T, n_heads, d_qk], dk [T, n_kv_heads, d_qk], dv [T, n_kv_heads, d_v]
 * (bf16, contiguous); q, k, v, out and dout are contiguous [T, heads, dim]
 * tensors here. Gradients of a key block are owned by one CTA (no
 * atomics); the sink block, which every query block reads, is reduced from
 * fp32 partials in the workspace in a fixed order.
 * Only per-head K/V (n_kv_heads == n_heads) with (d_qk, d_v) in
 * {(64,64), (192,128)} is compiled for the backward.
 */
loza_status loza_ssa_backward(const void *q, const void *k, const void *v, const void *out,
                              const void *dout, const float *lse, const int32_t *cu_seqlens,
                              int32_t batch, int64_t total_tokens, int32_t max_seqlen,
                              int32_t n_heads,
                              int32_t n_kv_heads, int32_t d_qk, int32_t d_v,
                              loza_ssa_params p, void *dq, void *dk, void *dv,
                              void *workspace, size_t workspace_bytes, loza_stream_t stream);

/*
 * Absorbed decode (n_kv_heads 1, d_qk 576, d_v 512, n_heads 64) from a paged
 * latent cache: the pool holds num_pages pages of 128 rows (one 128-row tile
 * each), row r of page g at kv_pool + (g * 128 + r) * pool_row_stride
 * elements; logical block kb of sequence n (rows 128kb .. 128kb+127 of its
 * context) is page block_table[n * bt_stride + kb]. Every block the window
 * selects must have a page; other table entries are never read. Same
 * operation, outputs, workspace (loza_ssa_workspace_size(LOZA_OP_DECODE, ...)
 * with the same batch and max_seqlen) and errors as loza_ssa_decode; in
 * addition LOZA_ERR_INVALID_ARG if block_table is NULL, bt_stride <
 * ceil(max_seqlen / 128), num_pages < 1 or num_pages * 128 > INT32_MAX. A page
 * number outside [0, num_pages) reads zeros (it is not detected).
 *   block_table: device int32 [batch, bt_stride]; kv_pool: device bf16,
 *   16-byte aligned, pool_row_stride >= 576 and a multiple of 8.
 */
loza_status loza_ssa_decode_paged(const void *q, const void *kv_pool, int32_t num_pages, int64_t pool_row_stride,
                                  const int32_t *block_table, int32_t bt_stride, const int32_t *seqlens,
                                  int32_t batch, int32_t max_seqlen, int32_t n_heads, loza_ssa_params p,
                                  void *out, float *lse, void *workspace, size_t workspace_bytes,
                                  loza_stream_t stream);

/*
 * Combine two attention branches of the same (token, head) rows, each given
 * as O [rows, d_v] bf16 and LSE [rows] fp32 (natural log; -inf = a branch
 * without keys), where the branches attend to disjoint key sets (for example
 * SSA's sink + local blocks and a second set of selected blocks). Writes the
 * attention over the union of the two key sets:
 *     lse_out = ln(exp(lse_a) + exp(lse_b))
 *     out     = exp(lse_a - lse_out) o_a + exp(lse_b - lse_out) o_b
 * (both branches empty: out = 0, lse_out = -inf). This is the LSE combine of
 * the split-KV decode applied to two whole outputs.
 *   rows >= 0 (0 launches nothing); d_v a positive multiple of 8.
 *   o_a, o_b, out: device, 16-byte aligned, contiguous [rows, d_v] bf16;
 *   lse_a, lse_b, lse_out: device [rows] fp32. out may alias o_a or o_b
 *   (each element is read before it is written by the same thread).
 * Returns LOZA_ERR_INVALID_ARG for a bad size, alignment or null pointer.
 */
loza_status loza_ssa_merge(const void *o_a, const float *lse_a, const void *o_b, const float *lse_b,
                           int64_t rows, int32_t d_v, void *out, float *lse_out, loza_stream_t stream);

/*
 * Calibration mix of a module's full-attention and SSA outputs (page 1
 * section 01 (1) of the LoZA pages; the formula is lost in the page text, the
 * plain reading is used): out = alpha * o_full + (1 - alpha) * o_ssa,
 * elementwise over n bf16 values (n a multiple of 8; device pointers, 16-byte
 * aligned; out may alias either input).
 */
loza_status loza_ssa_mix(const void *o_full, const void *o_ssa, int64_t n, float alpha, void *out,
                         loza_stream_t stream);

/* Human-readable name of a status code (static string). */
const char *loza_status_string(loza_status s);

/*
 * Synchronises `stream`, then returns and clears the library's device-side
 * status word: LOZA_OK, or LOZA_ERR_TIMEOUT if a kernel gave up on a bounded
 * wait since the last call. LOZA_ERR_CUDA if the synchronisation failed.
 */
loza_status loza_device_status(loza_stream_t stream);

/* Number of kernel launches the library issued since load (all entry points). */
uint64_t loza_launch_count(void);

/*
 * Self-test of the bounded waits: launches one thread that waits on an
 * mbarrier nothing completes; after limit_us microseconds (1 ... 2,000,000)
 * it gives up and records a timeout exactly as a kernel's own wait would, so
 * the next loza_device_status returns LOZA_ERR_TIMEOUT and the context stays
 * usable. (Every wait in the library's kernels has the same bound, 2 s.)
 * LOZA_ERR_INVALID_ARG for a limit out of range.
 */
loza_status loza_wait_selftest(uint32_t limit_us, loza_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* LOZA_SSA_H */
