/*
 * hysparse.h -- C ABI of libhysparse.so, the B200 (sm_100a) hot path of the
 * HySparse hybrid block.
 *
 * Method (HySparse: A Hybrid Sparse Attention Architecture with Oracle Token
 * Selection and KV Cache Sharing, abstract; intelliparadigm write-up, sections
 * 2.1 "hybrid block", 2.2 "dual-branch sparse attention", 3.1 "cross-layer
 * sharing"): a full causal attention layer is followed by N sparse layers.
 * The full layer is the only writer of the KV cache and the "oracle" of token
 * importance; each sparse layer reuses its KV cache and its top-k key set and
 * mixes a global branch over those keys with a 128-token local window through
 * a sigmoid gate.
 *
 * Notation used below:
 *   B batch, Lq query rows, Lkv cache length, Hq query heads, Hkv KV heads,
 *   d head dim, G = Hq / Hkv (query head h reads KV head h / G),
 *   pos(i) = Lkv - Lq + i  (causal, bottom-right aligned: row i sees keys
 *   0 .. pos(i); decode is Lq = 1 with the new token at Lkv - 1, or at
 *   kv_len[b] - 1 in hysparse_block_varlen / hysparse_block_paged).
 *
 * Layouts (row-major, contiguous, every pointer 16-byte aligned):
 *   q, q_sparse[n], out, out_sparse[n]  [B][Lq][Hq][d]   (dtype of the shape)
 *   k, v                               [B][Lkv][Hkv][d]  (dtype of the shape)
 *   lse                                [B][Hq][Lq]        float, natural log
 *   scores (one row chunk)             [B][Hkv][row_count][ld_scores] float
 *   idx                                [B][Hkv][Lq][topk] int32
 *   gate_logit                         [B][Lq][Hq]        float
 *   k_win, v_win (own-window calls)    [B][lwin][Hkv][d]  (dtype of the shape),
 *                                      row r = cache position Lkv - lwin + r
 *
 * Conventions for every entry point:
 *   - All device buffers are owned by the caller (e.g. allocated by PyTorch).
 *     The library allocates no device or host memory and keeps no state
 *     between calls beyond one-time kernel attributes and each device's SM
 *     count (read once, to size grids); scratch lives in the caller's
 *     workspace `ws`.
 *   - Work is enqueued on `stream` and is asynchronous; nothing synchronises
 *     except hysparse_workspace_status.
 *   - Arguments are checked on the host before anything is launched; a
 *     non-zero return means nothing was launched and no output was touched.
 *     A failed launch returns HS_ERR_CUDA.
 *   - Supported: dtype HS_F32 with d in {64, 128}; dtype HS_BF16 with
 *     d = 128; Hq % Hkv == 0; 1 <= Hq / Hkv <= 32; Lq <= Lkv;
 *     1 <= topk <= 4096; 1 <= window <= 1024.
 *   - NaN or Inf inputs give undefined (but memory-safe) results.
 *   - One GPU per process: each kernel's one-time set-up (its shared-memory
 *     attribute) runs on the first call, on that call's device, and is not
 *     guarded against a concurrent first call; make the first call of each
 *     kind from one host thread.  Later calls may come from any thread.
 */
#ifndef HYSPARSE_H
#define HYSPARSE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t / CUstream; NULL is the legacy default stream. */
typedef struct CUstream_st *hs_stream_t;

typedef enum {
    HS_OK = 0,
    HS_ERR_INVALID_ARG = 1,   /* null or misaligned pointer, bad size, bad shape; (device) a
                                 cache length outside [1, Lkv] (mixed-length / paged decode) */
    HS_ERR_UNSUPPORTED = 2,   /* valid but not implemented (dtype/d combination) */
    HS_ERR_WORKSPACE = 3,     /* ws_bytes below hysparse_workspace_size() */
    HS_ERR_CUDA = 4,          /* a CUDA call or kernel launch failed */
    HS_ERR_INVALID_INDEX = 5, /* (device) an index list entry outside [-1, pos], or a block
                                 table entry outside the page pool (paged decode) */
    HS_ERR_TIMEOUT = 6        /* (device) a bounded wait inside a kernel gave up */
} hs_status;

typedef enum { HS_F32 = 0, HS_BF16 = 1 } hs_dtype;

typedef struct {
    int B, Lq, Lkv, Hq, Hkv, d;
    int dtype;    /* hs_dtype */
    float scale;  /* softmax scale on q.k; <= 0 selects 1/sqrt(d) */
} hs_shape;

/* Bytes of device workspace that hysparse_full_attn_scores,
 * hysparse_sparse_attn and hysparse_block need for this shape.  `row_chunk`
 * is the number of query rows hysparse_block scores at a time (<= 0: all Lq
 * rows); the other arguments are those of the calls.  Returns 0 for an
 * invalid shape.  The first 256 bytes of a workspace hold a status word (see
 * hysparse_workspace_status); zero them once before first use (the calls
 * only ever OR error bits into it). */
size_t hysparse_workspace_size(const hs_shape *shape, int topk, int window, int n_sparse,
                               int row_chunk);

/* The full attention layer of the hybrid block, restricted to the query rows
 * [row_begin, row_begin + row_count) of every batch element.
 *
 * Computes (HySparse abstract; write-up section 2.1, the full layer as the
 * token-importance oracle; the score is the group sum of the softmax
 * probabilities over the query heads that share a KV head):
 *   out[b,i,h]  = sum_{j <= pos(i)} softmax_j(scale * q[b,i,h].k[b,j,h/G]) v[b,j,h/G]
 *   lse[b,h,i]  = ln sum_{j <= pos(i)} exp(scale * q[b,i,h].k[b,j,h/G])
 *   scores[b,g,i-row_begin,j] = sum_{h : h/G = g} exp(scale * q.k_j - lse[b,h,i])
 *                              for j <= pos(i); entries j > pos(i) are left
 *                              unspecified and are never read by hysparse_topk.
 * `scores` may be NULL (forward pass only); otherwise ld_scores >= Lkv.
 * Only out/lse entries of the listed rows are written.  If a bounded wait
 * inside a kernel gives up (HS_ERR_TIMEOUT in the status word), the lse
 * entries of the rows and heads it could not finish are set to NaN and their
 * out and scores entries are undefined.
 * Decode (Lq == 1) uses split-K over the cache and needs `ws`.
 * Errors: HS_ERR_INVALID_ARG, HS_ERR_UNSUPPORTED, HS_ERR_WORKSPACE, HS_ERR_CUDA. */
int hysparse_full_attn_scores(const hs_shape *shape, const void *q, const void *k, const void *v,
                              void *out, float *lse, float *scores, long long ld_scores,
                              int row_begin, int row_count, void *ws, size_t ws_bytes,
                              hs_stream_t stream);

/* Per-row top-k over one chunk of importance rows (write-up section 2.2: the
 * global branch attends over the full layer's TopK indices; section 3.1: one
 * index set per row is shared by the following sparse layers).
 * For every (b, g, i) with i in [row_begin, row_begin + row_count): the
 * `topk` keys j <= pos(i) with the largest scores[b,g,i-row_begin,j], ties
 * going to the lower j.  A row with pos(i) + 1 <= topk takes all its keys.
 * The set is written to idx[b,g,i,:] in ascending key order, padded with -1.
 * Scores must be >= 0 (importance values are).  Exact and deterministic.
 * Errors: HS_ERR_INVALID_ARG, HS_ERR_CUDA. */
int hysparse_topk(const hs_shape *shape, const float *scores, long long ld_scores, int row_begin,
                  int row_count, int topk, int32_t *idx, hs_stream_t stream);

/* One sparse layer (write-up section 2.2, dual-branch sparse attention;
 * section 3.1, KV cache reuse: reads the full layer's k and v, writes no KV):
 *   Og = softmax attention of q[b,i,h] over { k_j : j in idx[b,h/G,i,:], j != -1 }
 *   Ol = softmax attention of q[b,i,h] over { k_j : max(0, pos(i)-window+1) <= j <= pos(i) }
 *   out = sigmoid(gate_logit[b,i,h]) * Og + (1 - sigmoid(gate_logit[b,i,h])) * Ol
 * The two branches may share keys; each has its own softmax.  An index list
 * with no valid entry gives Og = 0.  Index lists must hold distinct keys in
 * [0, pos(i)] (any order) padded with -1; entries outside [-1, pos(i)] are
 * skipped and reported as HS_ERR_INVALID_INDEX through the workspace status
 * word.  out_global / out_local (nullable) receive Og and Ol.
 * Decode (Lq == 1) uses split-K and needs `ws`.
 * Errors: HS_ERR_INVALID_ARG, HS_ERR_UNSUPPORTED, HS_ERR_WORKSPACE, HS_ERR_CUDA. */
int hysparse_sparse_attn(const hs_shape *shape, const void *q, const void *k, const void *v,
                         const int32_t *idx, int topk, const float *gate_logit, int window,
                         void *out, void *out_global, void *out_local, void *ws, size_t ws_bytes,
                         hs_stream_t stream);

/* One sparse layer whose local branch reads the layer's own window K/V
 * (write-up section 2.2: the global branch computes on the KV cache that the
 * full layer shares, while the local branch maintains its own 128-token
 * sliding window).  Same computation, arguments and errors as
 * hysparse_sparse_attn, except that the local branch's keys and values come
 * from k_win / v_win instead of k / v:
 *   Ol = softmax attention of q[b,i,h] over
 *        { k_win[b, j - (Lkv - lwin)] : max(0, pos(i)-window+1) <= j <= pos(i) }
 *   with values v_win at the same rows.
 * k_win, v_win  [B][lwin][Hkv][d] (dtype of the shape, caller-owned, 16-byte
 * aligned): the layer's window keys and values for cache positions
 * Lkv - lwin .. Lkv - 1 (lwin = Lkv for a prefill that projects every
 * position; lwin = window - 1 + Lq, or any length that reaches back far
 * enough, for decode against a ring of the last tokens laid out in position
 * order).  1 <= lwin <= Lkv and Lkv - lwin <= max(0, Lkv - Lq - window + 1)
 * (the buffer covers the first row's window), else HS_ERR_INVALID_ARG.
 * The global branch still reads k and v with idx.  Passing k_win = k,
 * v_win = v, lwin = Lkv gives hysparse_sparse_attn's result, bit for bit
 * when Hq / Hkv is even (with an odd ratio the plain call may choose a
 * kernel that this one does not, and the two agree to rounding). */
int hysparse_sparse_attn_own_window(const hs_shape *shape, const void *q, const void *k, const void *v,
                                    const void *k_win, const void *v_win, int lwin, const int32_t *idx, int topk,
                                    const float *gate_logit, int window, void *out, void *out_global,
                                    void *out_local, void *ws, size_t ws_bytes, hs_stream_t stream);

/* A whole hybrid block (HySparse abstract: one full layer interleaved with
 * several sparse layers; write-up section 3.1: index sharing and cache reuse):
 * the full layer over all rows (out_full, and its LSE into `lse` when not
 * NULL), its importance scores and top-k (scored `row_chunk` rows at a time
 * inside `ws`), then n_sparse sparse layers, each with its own queries and
 * gate logits, all reusing k, v and the one index set.
 * q_sparse, gate_logit and out_sparse are HOST arrays of n_sparse DEVICE
 * pointers.  idx_out (nullable) receives the index set [B][Hkv][Lq][topk];
 * when NULL it is kept in `ws`.  In decode (Lq == 1) the sparse layers run
 * as one gather launch per group of up to 16 (they share the index set and
 * the cache, so each row is read once per group); the outputs are those of
 * one hysparse_sparse_attn call per layer, bit for bit.
 * Errors: as the calls it makes. */
int hysparse_block(const hs_shape *shape, const void *q_full, const void *k, const void *v,
                   void *out_full, float *lse, int n_sparse, const void *const *q_sparse,
                   const float *const *gate_logit, void *const *out_sparse, int topk, int window,
                   int32_t *idx_out, int row_chunk, void *ws, size_t ws_bytes, hs_stream_t stream);

/* hysparse_block with every sparse layer reading its window branch from its
 * own window K/V (write-up section 2.2; the variant of
 * hysparse_sparse_attn_own_window): k_win and v_win are HOST arrays of
 * n_sparse DEVICE pointers, layer n's [B][lwin][Hkv][d] buffers for cache
 * positions Lkv - lwin .. Lkv - 1 (layouts and limits as in
 * hysparse_sparse_attn_own_window, the same lwin for every layer).  The full
 * layer, the index set and the global branches are hysparse_block's; the
 * outputs equal hysparse_sparse_attn_own_window per layer on the block's
 * index set.  Fixed-length caches only.  Errors: as hysparse_block, and
 * HS_ERR_INVALID_ARG for a missing, misaligned or too short window buffer. */
int hysparse_block_own_window(const hs_shape *shape, const void *q_full, const void *k, const void *v,
                              void *out_full, float *lse, int n_sparse, const void *const *q_sparse,
                              const float *const *gate_logit, const void *const *k_win, const void *const *v_win,
                              int lwin, void *const *out_sparse, int topk, int window, int32_t *idx_out,
                              int row_chunk, void *ws, size_t ws_bytes, hs_stream_t stream);

/* One decode step of the hybrid block over a batch whose sequences have
 * caches of different lengths (serving: every sequence decodes one token,
 * each at its own position).  Same computation, arguments and layouts as
 * hysparse_block with Lq == 1, plus
 *   kv_len  DEVICE array of B int32, 1 <= kv_len[b] <= Lkv: sequence b's
 *           cache is k[b, 0:kv_len[b]], v[b, 0:kv_len[b]] (the Lkv-row
 *           buffers hold it at their start; rows past it are never read)
 *           and its new query sits at position kv_len[b] - 1, so its full
 *           layer, scores, top-k and window branch see exactly those keys.
 * Requires Lq == 1 and the bf16, d = 128 path (else HS_ERR_UNSUPPORTED);
 * kv_len must be 4-byte aligned.  The lengths live on the device, so a value
 * outside [1, Lkv] is found there: it is clamped (nothing outside the cache
 * is read) and HS_ERR_INVALID_ARG is recorded in the workspace status word
 * (hysparse_workspace_status).  The whole batch is one row chunk.
 * Errors: as hysparse_block. */
int hysparse_block_varlen(const hs_shape *shape, const int32_t *kv_len, const void *q_full,
                          const void *k, const void *v, void *out_full, float *lse, int n_sparse,
                          const void *const *q_sparse, const float *const *gate_logit,
                          void *const *out_sparse, int topk, int window, int32_t *idx_out,
                          void *ws, size_t ws_bytes, hs_stream_t stream);

/* hysparse_block_varlen over paged caches: k_pages and v_pages are pools of
 * num_pages pages, each page_size rows of [Hkv][d] ([num_pages][page_size]
 * [Hkv][d], bf16), and sequence b's key j is row j % page_size of page
 * block_table[b * max_pages + j / page_size] (block_table: DEVICE int32,
 * B rows of max_pages entries, 4-byte aligned).  Only the entries that cover
 * keys 0 .. kv_len[b]-1 are read.  page_size is a power of two in
 * [1, 65536]; max_pages * page_size >= Lkv (shape->Lkv is the longest cache
 * any sequence may have) and num_pages * page_size < 2^31.  A table entry
 * outside [0, num_pages) is found on the device: the key is dropped and
 * HS_ERR_INVALID_INDEX recorded in the workspace status word.  The
 * workspace is the one hysparse_workspace_size gives for the shape.
 * Errors: as hysparse_block_varlen, HS_ERR_INVALID_ARG for the paging
 * arguments. */
int hysparse_block_paged(const hs_shape *shape, const int32_t *kv_len, const int32_t *block_table,
                         int page_size, int max_pages, int num_pages, const void *q_full,
                         const void *k_pages, const void *v_pages, void *out_full, float *lse,
                         int n_sparse, const void *const *q_sparse, const float *const *gate_logit,
                         void *const *out_sparse, int topk, int window, int32_t *idx_out, void *ws,
                         size_t ws_bytes, hs_stream_t stream);

/* Allocation-free variant of hysparse_full_attn_scores (the pages have no
 * counterpart; this is a deployment convenience).  Same computation,
 * arguments, layouts and errors, but no workspace: its scratch lives in a
 * fixed 16 MiB device array inside the library, so callers that may not
 * allocate device memory -- a serving process that has frozen its memory
 * pool, or a plug-in host that only lends input and output buffers -- can
 * still run the full layer.  Every GPU that loads the library holds that
 * array until the process exits.
 *   - Scratch needed: 256 bytes (status word) + 8*B*Hq*Lq bytes of per-row
 *     softmax statistics, rounded up to 256; decode-shaped calls (Lq == 1,
 *     bf16) also keep their split-K partials and logit stash there, a
 *     further 4*B*Hq*Lkv + 520*B*Hq*ceil(Lkv/1024) + 768 bytes rounded up
 *     to 256.  Shapes needing more than 16 MiB return HS_ERR_WORKSPACE
 *     before anything runs (score smaller row chunks, decode smaller
 *     batches, or use hysparse_full_attn_scores).
 *   - Calls no cudaMalloc/cudaFree and allocates nothing; the caller still
 *     provides q, k, v, out, lse and (optionally) scores.
 *   - The array's device address is looked up on the first call on each
 *     device (the current device, which `stream` must belong to) and kept
 *     for the life of the process; make that first call before any stream
 *     capture, and do not use this entry point after cudaDeviceReset in the
 *     same process (the array may move).
 *   - All calls share the one array and each zeroes its status word on
 *     `stream`: calls that can overlap on the GPU (other streams, other host
 *     threads without ordering) race on it and must be serialised by the
 *     caller.
 *   - The status word cannot be read through this API.  A bounded wait that
 *     gives up inside a tensor-core kernel (HS_ERR_TIMEOUT elsewhere) leaves
 *     NaN in the lse entries of the rows and heads it could not finish; the
 *     out and scores entries of those rows are then undefined. */
int hysparse_full_attn_scores_noalloc(const hs_shape *shape, const void *q, const void *k,
                                      const void *v, void *out, float *lse, float *scores,
                                      long long ld_scores, int row_begin, int row_count,
                                      hs_stream_t stream);

/* Synchronises `stream`, reads the workspace status word (HS_OK or the
 * lowest-numbered device error recorded since it was last cleared), clears
 * it and returns it.  Returns HS_ERR_CUDA if the synchronisation fails. */
int hysparse_workspace_status(void *ws, hs_stream_t stream);

/* Diagnostic (no counterpart on the pages): L2 read bandwidth probe, the
 * denominator for kernels whose reads are served from L2 (the prefill sparse
 * layers gather K/V rows from a cache that fits in L2).  Reads the DEVICE
 * buffer `buf` (`bytes`, a multiple of 256 and >= 4096, 256-byte aligned; the
 * caller makes it L2-resident, e.g. by one untimed call first) with `blocks`
 * CTAs of 512 threads on `stream`, using L2-only loads:
 *   mode 0: streaming 16-byte reads, `passes` times over the buffer;
 *   mode 1: whole 256-byte rows at hashed positions, passes * bytes / 256
 *           rows (the access pattern of the sparse layers' row gather).
 *   modes 2 and 3: as 0 and 1, but through cp.async into shared memory
 *           (one CTA of 7 warps per SM is the intended `blocks`: the path
 *           and occupancy of the row-gather kernel); bytes >= 65536.
 * Either way passes * bytes bytes are read; time the call with events on
 * `stream`.  `sink` is a DEVICE array of at least `blocks` 64-bit words that
 * receives an XOR of what each CTA read (it keeps the loads live).
 * Errors: HS_ERR_INVALID_ARG, HS_ERR_CUDA. */
int hysparse_probe_l2_read(const void *buf, size_t bytes, int passes, int mode, int blocks,
                           unsigned long long *sink, hs_stream_t stream);

/* Diagnostic: number of CUDA kernels this library has launched in this
 * process so far (counted on the host at each launch). */
unsigned long long hysparse_launch_count(void);

/* Static text for a status code. */
const char *hysparse_status_string(int status);

/* Library version, e.g. "hysparse-b200 0.1". */
const char *hysparse_version(void);

#ifdef __cplusplus
}
#endif

#endif /* HYSPARSE_H */
