// C-ABI entry points of libhysparse.so: argument checks on the host, the
// workspace layout, and dispatch to the kernels.  See include/hysparse.h for
// the contract of every call.
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "common.cuh"
#include "hysparse.h"
#include "internal.h"

namespace hs {
namespace {

constexpr int kMaxTopk = 4096;
constexpr int kMaxWindow = 1024;
constexpr int kMaxGroup = 32;
constexpr int kMaxLen = 1 << 24;

// Query rows below which the tensor-core full layer is not used (a 128-row
// tile would be mostly empty; decode takes the CUDA-core path).
constexpr int kTcMinRows = 64;

bool aligned16(const void *p) { return p != nullptr && ((uintptr_t)p & 15u) == 0; }

int resolve_shape(const hs_shape *in, Shape *out) {
    if (in == nullptr) return HS_ERR_INVALID_ARG;
    const hs_shape &s = *in;
    if (s.B < 1 || s.Lq < 1 || s.Lkv < 1 || s.Hq < 1 || s.Hkv < 1 || s.d < 1) return HS_ERR_INVALID_ARG;
    if (s.Lq > s.Lkv || s.Lkv > kMaxLen || s.Hq % s.Hkv != 0) return HS_ERR_INVALID_ARG;
    if (s.Hq / s.Hkv > kMaxGroup) return HS_ERR_UNSUPPORTED;
    if (s.dtype != HS_F32 && s.dtype != HS_BF16) return HS_ERR_INVALID_ARG;
    const bool ok = (s.dtype == HS_F32 && (s.d == 64 || s.d == 128)) || (s.dtype == HS_BF16 && s.d == 128);
    if (!ok) return HS_ERR_UNSUPPORTED;
    if (!(s.scale == s.scale) || isinf(s.scale)) return HS_ERR_INVALID_ARG;
    *out = Shape{s.B, s.Lq, s.Lkv, s.Hq, s.Hkv, s.d, s.dtype,
                 s.scale > 0.f ? s.scale : 1.0f / sqrtf((float)s.d)};
    return HS_OK;
}

// Workspace regions (byte offsets), all 256-byte aligned.
struct WsLayout {
    size_t status = 0;
    size_t stats = 0, stats_end = 0;          // full layer per-row statistics
    size_t dec = 0, full_end = 0;             // decode split-K partials + logit stash
    size_t selmask = 0, wl = 0, sparse_end = 0;  // dense-masked sparse layer: bitmask, window branch
    size_t block_scores = 0, block_lse = 0, block_idx = 0;
    size_t total = 0;
};

bool use_decode_path(const Shape &s) { return s.Lq == 1 && sparse_mma_supported(s); }

WsLayout ws_layout(const Shape &s, int topk, int row_chunk) {
    WsLayout L;
    size_t off = kStatusBytes;
    L.stats = off;
    off = align_up(off + (size_t)s.B * s.Hq * s.Lq * 2 * sizeof(float), 256);
    L.stats_end = off;
    L.dec = off;
    if (use_decode_path(s)) off = align_up(off + decode_ws_bytes(s), 256);
    L.full_end = off;
    L.selmask = off;
    if (sparse_dense_supported(s)) off = align_up(off + selmask_bytes(s), 256);
    L.wl = off;
    if (sparse_dense_supported(s) && sparse_pair_supported(s)) off = align_up(off + sparse_pair_wl_bytes(s), 256);
    L.sparse_end = off;
    const int chunk = (row_chunk <= 0 || row_chunk > s.Lq) ? s.Lq : row_chunk;
    L.block_scores = off;
    off = align_up(off + (size_t)s.B * s.Hkv * chunk * (size_t)s.Lkv * sizeof(float), 256);
    L.block_lse = off;
    off = align_up(off + (size_t)s.B * s.Hq * s.Lq * sizeof(float), 256);
    L.block_idx = off;
    off = align_up(off + (size_t)s.B * s.Hkv * s.Lq * (size_t)topk * sizeof(int32_t), 256);
    L.total = off;
    return L;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? HS_OK : HS_ERR_CUDA; }

int check_full_args(const Shape &s, const void *q, const void *k, const void *v, void *out,
                    float *lse, float *scores, long long ld, int row_begin, int row_count) {
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse))
        return HS_ERR_INVALID_ARG;
    if (row_begin < 0 || row_count < 1 || row_begin > s.Lq - row_count) return HS_ERR_INVALID_ARG;
    if (scores != nullptr && (!aligned16(scores) || ld < s.Lkv)) return HS_ERR_INVALID_ARG;
    return HS_OK;
}

int run_full(const Shape &s, const void *q, const void *k, const void *v, void *out, float *lse,
             float *scores, long long ld, int row_begin, int row_count, void *ws, cudaStream_t st) {
    if (use_decode_path(s)) {
        char *w = reinterpret_cast<char *>(ws);
        unsigned int *status = reinterpret_cast<unsigned int *>(ws);
        return cuda_status(decode_full_mma_launch(s, q, k, v, out, lse, scores, ld,
                                                  w + ws_layout(s, 1, row_count).dec, status, st));
    }
    if (full_attn_tc_supported(s) && s.Lq >= kTcMinRows) {
        char *w = reinterpret_cast<char *>(ws);
        float2 *stats = reinterpret_cast<float2 *>(w + ws_layout(s, 1, row_count).stats);
        unsigned int *status = reinterpret_cast<unsigned int *>(ws);
        return cuda_status(full_attn_scores_tc_launch(s, q, k, v, out, lse, scores, ld, row_begin,
                                                      row_count, stats, status, wait_limit_ns(), st));
    }
    return cuda_status(full_attn_scores_simt_launch(s, q, k, v, out, lse, scores, ld, row_begin,
                                                    row_count, st));
}

int run_topk(const Shape &s, const float *scores, long long ld, int row_begin, int row_count,
             int topk, int32_t *idx, cudaStream_t st, uint32_t *mask = nullptr, bool *mask_done = nullptr) {
    return cuda_status(topk_launch(s, scores, ld, row_begin, row_count, topk, idx, st, mask,
                                   mask ? selmask_words(s) : 0, mask_done));
}

// Which sparse-layer kernel to run.  Both compute the same two softmaxes;
// the estimate compares the dense-masked pass (every causal 128x128 tile of
// every query head on the tensor cores; kDenseTileCycles per tile on one SM,
// measured) with the gather (k_eff + w_eff K and V rows of 256 bytes per row
// and KV head at kGatherBytesPerS, measured).
// HYSPARSE_SPARSE_PATH=dense|gather overrides it.
constexpr double kDenseTileCycles = 4000.0;      // single-head kernel (odd G)
constexpr double kPairTileCycles = 2600.0;       // paired-head pipeline (even G), per head
constexpr double kGatherBytesPerS = 12.0e12;   // measured 11.9-15.6 TB/s of gathered rows (prefill)
bool prefer_dense_sparse(const Shape &s, int topk, int window) {
    if (!sparse_dense_supported(s)) return false;
    // own window K/V: only the paired-head pipeline reads the window pass from
    // a second buffer, and only one that spans the whole cache
    if (s.k_win != nullptr && (s.Lwin != s.Lkv || !sparse_pair_supported(s))) return false;
    const char *e = getenv("HYSPARSE_SPARSE_PATH");
    if (e && strcmp(e, "dense") == 0) return true;
    if (e && strcmp(e, "gather") == 0) return false;
    const double off = (double)(s.Lkv - s.Lq);
    double tiles = 0.0;                       // sum over 128-row tiles of causal key tiles
    const int n_rt = (s.Lq + 127) / 128;
    for (int t = 0; t < n_rt; ++t) {
        const double last = off + fmin((double)s.Lq, 128.0 * (t + 1)) - 1.0;
        tiles += floor(last / 128.0) + 1.0;
    }
    const double dense_s = tiles * s.Hq * s.B * (sparse_pair_supported(s) ? kPairTileCycles : kDenseTileCycles) /
                           (148.0 * 1.9e9);
    double keys = 0.0;                         // sum over rows of k_eff + w_eff
    for (int i = 0; i < s.Lq; i += 64) {
        const double n = off + i + 1.0;
        keys += 64.0 * (fmin(n, (double)topk) + fmin(n, (double)window));
    }
    const double gather_s = keys * s.Hkv * s.B * 512.0 / kGatherBytesPerS;
    return dense_s < gather_s;
}

// Which gather kernel runs the sparse layer: the tcgen05 row gather
// (sparse_gather_tc.cu) or the warp-MMA one (sparse_mma.cu).
// HYSPARSE_GATHER_KERNEL=tc|mma overrides the default.
bool use_gather_tc(const Shape &s) {
    if (!sparse_gather_tc_supported(s) || s.k_win != nullptr) return false;
    const char *e = getenv("HYSPARSE_GATHER_KERNEL");
    if (e && strcmp(e, "tc") == 0) return true;
    return false;
}

// Whether hysparse_block runs its sparse layers as one gather launch (the
// warp-MMA gather, several layers): by default for decode, where each layer
// reads its rows from HBM and a lone layer fills half the SMs; prefill's
// gather is served from L2 and bound by its instruction chains.
// HYSPARSE_LAYER_GROUP=0|1 turns it off or on for every shape.
bool group_sparse_layers(const Shape &s, int topk, int window, int n_sparse) {
    if (n_sparse < 2 || s.k_win != nullptr || !sparse_mma_supported(s)) return false;
    if (prefer_dense_sparse(s, topk, window) || use_gather_tc(s)) return false;
    const char *e = getenv("HYSPARSE_LAYER_GROUP");
    if (e && strcmp(e, "0") == 0) return false;
    if (e && strcmp(e, "1") == 0) return true;
    return s.Lq == 1;
}

// mask_ready: the dense path's selection bitmask in `ws` was already built
// from this very index set (hysparse_block builds it once for all its layers).
int run_sparse(const Shape &s, const void *q, const void *k, const void *v, const int32_t *idx,
               int topk, const float *gate, int window, void *out, void *og, void *ol, void *ws,
               cudaStream_t st, bool mask_ready = false) {
    unsigned int *status = reinterpret_cast<unsigned int *>(ws);
    if (prefer_dense_sparse(s, topk, window)) {
        const WsLayout L = ws_layout(s, topk, 1);
        uint32_t *mask = reinterpret_cast<uint32_t *>(reinterpret_cast<char *>(ws) + L.selmask);
        if (sparse_pair_supported(s)) {
            uint32_t *wl = reinterpret_cast<uint32_t *>(reinterpret_cast<char *>(ws) + L.wl);
            cudaError_t e = mask_ready ? cudaSuccess : selmask_build_launch(s, idx, topk, mask, status, st);
            if (e == cudaSuccess)
                e = sparse_pair_tc_launch(s, q, k, v, gate, window, out, og, ol, mask, selmask_words(s), wl, status,
                                          wait_limit_ns(), st);
            return cuda_status(e);
        }
        return cuda_status(sparse_dense_tc_launch(s, q, k, v, idx, topk, gate, window, out, og, ol, mask,
                                                  status, wait_limit_ns(), st));
    }
    if (use_gather_tc(s))
        return cuda_status(sparse_gather_tc_launch(s, q, k, v, idx, topk, gate, window, out, og, ol, status,
                                                   wait_limit_ns(), st));
    if (sparse_mma_supported(s))
        return cuda_status(sparse_attn_mma_launch(s, q, k, v, idx, topk, gate, window, out, og, ol, status,
                                                  wait_limit_ns(), st));
    return cuda_status(sparse_attn_simt_launch(s, q, k, v, idx, topk, gate, window, out, og, ol,
                                               status, st));
}

}  // namespace

static std::atomic<unsigned long long> g_launches{0};
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

unsigned long long wait_limit_ns() {
    // HYSPARSE_WAIT_LIMIT_NS lowers the bound on in-kernel waits; the tests
    // set it to 0 to drive the timeout path without hanging anything.
    const char *e = getenv("HYSPARSE_WAIT_LIMIT_NS");
    if (e && *e) return strtoull(e, nullptr, 10);
    return 1000000000ull;
}

}  // namespace hs

using namespace hs;

extern "C" {

size_t hysparse_workspace_size(const hs_shape *shape, int topk, int window, int n_sparse,
                               int row_chunk) {
    Shape s;
    if (resolve_shape(shape, &s) != HS_OK) return 0;
    if (topk < 1 || topk > kMaxTopk || window < 1 || window > kMaxWindow || n_sparse < 0) return 0;
    return ws_layout(s, topk, row_chunk).total;
}

int hysparse_full_attn_scores(const hs_shape *shape, const void *q, const void *k, const void *v,
                              void *out, float *lse, float *scores, long long ld_scores,
                              int row_begin, int row_count, void *ws, size_t ws_bytes,
                              hs_stream_t stream) {
    Shape s;
    int rc = resolve_shape(shape, &s);
    if (rc != HS_OK) return rc;
    rc = check_full_args(s, q, k, v, out, lse, scores, ld_scores, row_begin, row_count);
    if (rc != HS_OK) return rc;
    if (!aligned16(ws)) return HS_ERR_INVALID_ARG;
    if (ws_bytes < ws_layout(s, 1, row_count).full_end) return HS_ERR_WORKSPACE;
    return run_full(s, q, k, v, out, lse, scores, ld_scores, row_begin, row_count, ws,
                    (cudaStream_t)stream);
}

int hysparse_topk(const hs_shape *shape, const float *scores, long long ld_scores, int row_begin,
                  int row_count, int topk, int32_t *idx, hs_stream_t stream) {
    Shape s;
    int rc = resolve_shape(shape, &s);
    if (rc != HS_OK) return rc;
    if (!aligned16(scores) || !aligned16(idx) || ld_scores < s.Lkv) return HS_ERR_INVALID_ARG;
    if (row_begin < 0 || row_count < 1 || row_begin > s.Lq - row_count) return HS_ERR_INVALID_ARG;
    if (topk < 1 || topk > kMaxTopk) return HS_ERR_INVALID_ARG;
    return run_topk(s, scores, ld_scores, row_begin, row_count, topk, idx, (cudaStream_t)stream);
}

}  // extern "C"

namespace {
// Checks and runs one sparse layer for hysparse_sparse_attn and
// hysparse_sparse_attn_own_window (s carries the own window buffer, if any).
int sparse_attn_impl(const Shape &s, const void *q, const void *k, const void *v, const int32_t *idx, int topk,
                     const float *gate_logit, int window, void *out, void *out_global, void *out_local, void *ws,
                     size_t ws_bytes, cudaStream_t st) {
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(idx) || !aligned16(gate_logit) ||
        !aligned16(out))
        return HS_ERR_INVALID_ARG;
    if ((out_global && !aligned16(out_global)) || (out_local && !aligned16(out_local)))
        return HS_ERR_INVALID_ARG;
    if (topk < 1 || topk > kMaxTopk || window < 1 || window > kMaxWindow) return HS_ERR_INVALID_ARG;
    if (!aligned16(ws)) return HS_ERR_INVALID_ARG;
    if (ws_bytes < ws_layout(s, topk, 1).sparse_end) return HS_ERR_WORKSPACE;
    return run_sparse(s, q, k, v, idx, topk, gate_logit, window, out, out_global, out_local, ws, st);
}
}  // namespace

extern "C" {

int hysparse_sparse_attn(const hs_shape *shape, const void *q, const void *k, const void *v,
                         const int32_t *idx, int topk, const float *gate_logit, int window,
                         void *out, void *out_global, void *out_local, void *ws, size_t ws_bytes,
                         hs_stream_t stream) {
    Shape s;
    int rc = resolve_shape(shape, &s);
    if (rc != HS_OK) return rc;
    return sparse_attn_impl(s, q, k, v, idx, topk, gate_logit, window, out, out_global, out_local, ws, ws_bytes,
                            (cudaStream_t)stream);
}

int hysparse_sparse_attn_own_window(const hs_shape *shape, const void *q, const void *k, const void *v,
                                    const void *k_win, const void *v_win, int lwin, const int32_t *idx, int topk,
                                    const float *gate_logit, int window, void *out, void *out_global,
                                    void *out_local, void *ws, size_t ws_bytes, hs_stream_t stream) {
    Shape s;
    int rc = resolve_shape(shape, &s);
    if (rc != HS_OK) return rc;
    if (!aligned16(k_win) || !aligned16(v_win) || lwin < 1 || lwin > s.Lkv) return HS_ERR_INVALID_ARG;
    if (window < 1 || window > kMaxWindow) return HS_ERR_INVALID_ARG;
    // the buffer holds positions Lkv - lwin .. Lkv - 1 and must reach back to
    // the first key of the first query row's window
    const int first_key = s.Lkv - s.Lq - window + 1 > 0 ? s.Lkv - s.Lq - window + 1 : 0;
    if (s.Lkv - lwin > first_key) return HS_ERR_INVALID_ARG;
    s.k_win = k_win;
    s.v_win = v_win;
    s.Lwin = lwin;
    return sparse_attn_impl(s, q, k, v, idx, topk, gate_logit, window, out, out_global, out_local, ws, ws_bytes,
                            (cudaStream_t)stream);
}

namespace {
// Paged caches: where the pages are and how sequences map onto them.
struct Paging {
    const int32_t *table = nullptr;
    int page_size = 0, max_pages = 0, num_pages = 0;
};

// The sparse layers' own window K/V (hysparse_block_own_window): layer n
// reads k[n], v[n], lwin rows each.  k == NULL: the shared cache.
struct OwnWindows {
    const void *const *k = nullptr;
    const void *const *v = nullptr;
    int lwin = 0;
};

// hysparse_block; hysparse_block_varlen when kv_len is set; and
// hysparse_block_paged when the paging table is set too
int block_impl(const hs_shape *shape, const int32_t *kv_len, const Paging &pg, const void *q_full, const void *k,
               const void *v, void *out_full, float *lse, int n_sparse, const void *const *q_sparse,
               const float *const *gate_logit, void *const *out_sparse, int topk, int window,
               int32_t *idx_out, int row_chunk, void *ws, size_t ws_bytes, hs_stream_t stream,
               const OwnWindows &ow = OwnWindows{}) {
    Shape s;
    int rc = resolve_shape(shape, &s);
    if (rc != HS_OK) return rc;
    if (kv_len != nullptr) {
        // caches of different lengths: the bf16 decode path only
        if (s.Lq != 1 || !use_decode_path(s)) return HS_ERR_UNSUPPORTED;
        if ((reinterpret_cast<uintptr_t>(kv_len) & 3u) != 0) return HS_ERR_INVALID_ARG;
        s.kv_len = kv_len;
    }
    if (pg.table != nullptr) {
        if (kv_len == nullptr) return HS_ERR_INVALID_ARG;
        const int ps = pg.page_size;
        if (ps < 1 || ps > (1 << 16) || (ps & (ps - 1)) != 0) return HS_ERR_INVALID_ARG;
        if (pg.max_pages < 1 || pg.num_pages < 1) return HS_ERR_INVALID_ARG;
        if ((long long)pg.max_pages * ps < s.Lkv) return HS_ERR_INVALID_ARG;           // table too short
        if ((long long)pg.num_pages * ps > 0x7fffffffLL) return HS_ERR_INVALID_ARG;    // pool rows in int32
        if ((reinterpret_cast<uintptr_t>(pg.table) & 3u) != 0) return HS_ERR_INVALID_ARG;
        s.block_table = pg.table;
        s.page_shift = __builtin_ctz((unsigned)ps);
        s.max_pages = pg.max_pages;
        s.num_pages = pg.num_pages;
    }
    if (topk < 1 || topk > kMaxTopk || window < 1 || window > kMaxWindow || n_sparse < 0)
        return HS_ERR_INVALID_ARG;
    if (n_sparse > 0 && (q_sparse == nullptr || gate_logit == nullptr || out_sparse == nullptr))
        return HS_ERR_INVALID_ARG;
    if (!aligned16(q_full) || !aligned16(k) || !aligned16(v) || !aligned16(out_full))
        return HS_ERR_INVALID_ARG;
    if ((lse && !aligned16(lse)) || (idx_out && !aligned16(idx_out))) return HS_ERR_INVALID_ARG;
    for (int n = 0; n < n_sparse; ++n)
        if (!aligned16(q_sparse[n]) || !aligned16(gate_logit[n]) || !aligned16(out_sparse[n]))
            return HS_ERR_INVALID_ARG;
    if (ow.k != nullptr) {
        // own window buffers: fixed-length caches, every layer's buffer
        // reaching back to the first row's window
        if (kv_len != nullptr || ow.v == nullptr || ow.lwin < 1 || ow.lwin > s.Lkv) return HS_ERR_INVALID_ARG;
        const int first_key = s.Lkv - s.Lq - window + 1 > 0 ? s.Lkv - s.Lq - window + 1 : 0;
        if (s.Lkv - ow.lwin > first_key) return HS_ERR_INVALID_ARG;
        for (int n = 0; n < n_sparse; ++n)
            if (!aligned16(ow.k[n]) || !aligned16(ow.v[n])) return HS_ERR_INVALID_ARG;
    }
    if (!aligned16(ws)) return HS_ERR_INVALID_ARG;
    const int chunk = (row_chunk <= 0 || row_chunk > s.Lq) ? s.Lq : row_chunk;
    const WsLayout L = ws_layout(s, topk, chunk);
    if (ws_bytes < L.total) return HS_ERR_WORKSPACE;

    char *w = reinterpret_cast<char *>(ws);
    float *scores = reinterpret_cast<float *>(w + L.block_scores);
    float *lse_buf = lse ? lse : reinterpret_cast<float *>(w + L.block_lse);
    int32_t *idx = idx_out ? idx_out : reinterpret_cast<int32_t *>(w + L.block_idx);
    cudaStream_t st = (cudaStream_t)stream;
    // the index set is shared by every sparse layer of the block, and so is
    // the dense path's bitmask built from it: the top-k kernel writes it with
    // the indices where it can, else one pass over the index lists builds it
    const bool dense = n_sparse > 0 && prefer_dense_sparse(s, topk, window) && sparse_pair_supported(s);
    uint32_t *mask = dense ? reinterpret_cast<uint32_t *>(w + ws_layout(s, topk, 1).selmask) : nullptr;
    bool mask_all = dense;
    for (int r0 = 0; r0 < s.Lq; r0 += chunk) {
        const int rows = (s.Lq - r0 < chunk) ? s.Lq - r0 : chunk;
        rc = run_full(s, q_full, k, v, out_full, lse_buf, scores, s.Lkv, r0, rows, ws, st);
        if (rc != HS_OK) return rc;
        bool done = false;
        rc = run_topk(s, scores, s.Lkv, r0, rows, topk, idx, st, mask, &done);
        if (rc != HS_OK) return rc;
        mask_all = mask_all && done;
    }
    if (dense && !mask_all) {
        rc = cuda_status(selmask_build_launch(s, idx, topk, mask, reinterpret_cast<unsigned int *>(ws), st));
        if (rc != HS_OK) return rc;
    }
    const bool mask_ready = dense;
    if (ow.k != nullptr) {
        for (int n = 0; n < n_sparse; ++n) {
            Shape sl = s;
            sl.k_win = ow.k[n];
            sl.v_win = ow.v[n];
            sl.Lwin = ow.lwin;
            rc = run_sparse(sl, q_sparse[n], k, v, idx, topk, gate_logit[n], window, out_sparse[n], nullptr,
                            nullptr, ws, st, mask_ready);
            if (rc != HS_OK) return rc;
        }
        return HS_OK;
    }
    if (group_sparse_layers(s, topk, window, n_sparse)) {
        // the layers share the index set and the cache: one gather launch per
        // group of up to 16, so that each item's rows are read once per group
        for (int n0 = 0; n0 < n_sparse; n0 += 16) {
            const int n = n_sparse - n0 < 16 ? n_sparse - n0 : 16;
            rc = cuda_status(sparse_attn_mma_layers_launch(s, n, q_sparse + n0, k, v, idx, topk, gate_logit + n0,
                                                           window, out_sparse + n0,
                                                           reinterpret_cast<unsigned int *>(ws), wait_limit_ns(),
                                                           st));
            if (rc != HS_OK) return rc;
        }
        return HS_OK;
    }
    for (int n = 0; n < n_sparse; ++n) {
        rc = run_sparse(s, q_sparse[n], k, v, idx, topk, gate_logit[n], window, out_sparse[n],
                        nullptr, nullptr, ws, st, mask_ready);
        if (rc != HS_OK) return rc;
    }
    return HS_OK;
}
}  // namespace

int hysparse_block(const hs_shape *shape, const void *q_full, const void *k, const void *v,
                   void *out_full, float *lse, int n_sparse, const void *const *q_sparse,
                   const float *const *gate_logit, void *const *out_sparse, int topk, int window,
                   int32_t *idx_out, int row_chunk, void *ws, size_t ws_bytes,
                   hs_stream_t stream) {
    return block_impl(shape, nullptr, Paging{}, q_full, k, v, out_full, lse, n_sparse, q_sparse, gate_logit,
                      out_sparse, topk, window, idx_out, row_chunk, ws, ws_bytes, stream);
}

int hysparse_block_own_window(const hs_shape *shape, const void *q_full, const void *k, const void *v,
                              void *out_full, float *lse, int n_sparse, const void *const *q_sparse,
                              const float *const *gate_logit, const void *const *k_win, const void *const *v_win,
                              int lwin, void *const *out_sparse, int topk, int window, int32_t *idx_out,
                              int row_chunk, void *ws, size_t ws_bytes, hs_stream_t stream) {
    if (n_sparse > 0 && (k_win == nullptr || v_win == nullptr)) return HS_ERR_INVALID_ARG;
    OwnWindows ow;
    ow.k = n_sparse > 0 ? k_win : nullptr;
    ow.v = v_win;
    ow.lwin = lwin;
    return block_impl(shape, nullptr, Paging{}, q_full, k, v, out_full, lse, n_sparse, q_sparse, gate_logit,
                      out_sparse, topk, window, idx_out, row_chunk, ws, ws_bytes, stream, ow);
}

int hysparse_block_varlen(const hs_shape *shape, const int32_t *kv_len, const void *q_full, const void *k,
                          const void *v, void *out_full, float *lse, int n_sparse, const void *const *q_sparse,
                          const float *const *gate_logit, void *const *out_sparse, int topk, int window,
                          int32_t *idx_out, void *ws, size_t ws_bytes, hs_stream_t stream) {
    if (kv_len == nullptr) return HS_ERR_INVALID_ARG;
    return block_impl(shape, kv_len, Paging{}, q_full, k, v, out_full, lse, n_sparse, q_sparse, gate_logit,
                      out_sparse, topk, window, idx_out, 0, ws, ws_bytes, stream);
}

int hysparse_block_paged(const hs_shape *shape, const int32_t *kv_len, const int32_t *block_table, int page_size,
                         int max_pages, int num_pages, const void *q_full, const void *k_pages,
                         const void *v_pages, void *out_full, float *lse, int n_sparse,
                         const void *const *q_sparse, const float *const *gate_logit, void *const *out_sparse,
                         int topk, int window, int32_t *idx_out, void *ws, size_t ws_bytes, hs_stream_t stream) {
    if (kv_len == nullptr || block_table == nullptr) return HS_ERR_INVALID_ARG;
    Paging pg;
    pg.table = block_table;
    pg.page_size = page_size;
    pg.max_pages = max_pages;
    pg.num_pages = num_pages;
    return block_impl(shape, kv_len, pg, q_full, k_pages, v_pages, out_full, lse, n_sparse, q_sparse, gate_logit,
                      out_sparse, topk, window, idx_out, 0, ws, ws_bytes, stream);
}

int hysparse_workspace_status(void *ws, hs_stream_t stream) {
    if (!aligned16(ws)) return HS_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    unsigned int word = 0;
    if (cudaMemcpyAsync(&word, ws, sizeof(word), cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return HS_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return HS_ERR_CUDA;
    if (word == 0) return HS_OK;
    if (cudaMemsetAsync(ws, 0, sizeof(word), st) != cudaSuccess) return HS_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return HS_ERR_CUDA;
    for (int c = 1; c < 32; ++c)
        if (word & (1u << c)) return c;
    return HS_ERR_CUDA;
}

const char *hysparse_status_string(int status) {
    switch (status) {
        case HS_OK: return "ok";
        case HS_ERR_INVALID_ARG: return "invalid argument";
        case HS_ERR_UNSUPPORTED: return "unsupported shape or dtype";
        case HS_ERR_WORKSPACE: return "workspace too small";
        case HS_ERR_CUDA: return "CUDA error";
        case HS_ERR_INVALID_INDEX: return "index list entry outside [-1, pos]";
        case HS_ERR_TIMEOUT: return "bounded wait in a kernel timed out";
        default: return "unknown status";
    }
}

const char *hysparse_version(void) { return "hysparse-b200 0.1"; }

unsigned long long hysparse_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free variant of hysparse_full_attn_scores.
//
// Some callers cannot hand the library a workspace: code that runs after a
// serving process has fixed its device memory (every later cudaMalloc is
// refused or would break a memory budget the host framework enforces), and
// hosts that give a plug-in only its input and output buffers and no way to
// allocate.  For them this entry point keeps its scratch -- the status word
// and the full layer's per-row softmax statistics -- in the fixed array
// below, which every GPU that loads the library holds until the process
// exits.  Host code may not use the array's name as a device address; the
// address is looked up once per device with cudaGetSymbolAddress.
namespace hs {
namespace {

constexpr size_t kNoAllocScratchBytes = 16u << 20;  // 16 MiB
__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kNoAllocMaxDevices = 128;
void *g_noalloc_ptr[kNoAllocMaxDevices];
std::mutex g_noalloc_mu;

// Device address of g_noalloc_scratch on the current device (set up on the
// first call per device); nullptr and the CUDA error on failure.
void *noalloc_scratch(cudaError_t *err) {
    int dev = 0;
    *err = cudaGetDevice(&dev);
    if (*err != cudaSuccess) return nullptr;
    if (dev < 0 || dev >= kNoAllocMaxDevices) {
        *err = cudaErrorInvalidDevice;
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (g_noalloc_ptr[dev] == nullptr) {
        void *ptr = nullptr;
        *err = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
        if (*err != cudaSuccess) return nullptr;
        g_noalloc_ptr[dev] = ptr;
    }
    return g_noalloc_ptr[dev];
}

}  // namespace
}  // namespace hs

extern "C" int hysparse_full_attn_scores_noalloc(const hs_shape *shape, const void *q, const void *k,
                                                 const void *v, void *out, float *lse, float *scores,
                                                 long long ld_scores, int row_begin, int row_count,
                                                 hs_stream_t stream) {
    Shape s;
    int rc = resolve_shape(shape, &s);
    if (rc != HS_OK) return rc;
    rc = check_full_args(s, q, k, v, out, lse, scores, ld_scores, row_begin, row_count);
    if (rc != HS_OK) return rc;
    if (ws_layout(s, 1, row_count).full_end > kNoAllocScratchBytes) return HS_ERR_WORKSPACE;
    cudaError_t err = cudaSuccess;
    void *ws = noalloc_scratch(&err);
    if (ws == nullptr) return HS_ERR_CUDA;
    cudaStream_t st = (cudaStream_t)stream;
    // the status word must start at zero; the statistics are written before
    // they are read, so the rest of the array is left as the last call left it
    if (cudaMemsetAsync(ws, 0, kStatusBytes, st) != cudaSuccess) return HS_ERR_CUDA;
    return run_full(s, q, k, v, out, lse, scores, ld_scores, row_begin, row_count, ws, st);
}
