// Internal launcher interface between the C-ABI layer (hysparse_api.cu) and
// the kernel files.  Not installed, not part of the ABI.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "hysparse.h"

namespace hs {

// Number of kernels this library has launched (host-side count, exported for
// benchmarks through hysparse_launch_count).
void count_launch();

// A validated hs_shape (scale resolved).
struct Shape {
    int B, Lq, Lkv, Hq, Hkv, d;
    int dtype;
    float scale;
    // decode over caches of different lengths: kv_len[b] (device, int32) is
    // sequence b's cache length (its new token at position kv_len[b] - 1);
    // NULL = every sequence has Lkv.  Only the bf16 decode path reads it.
    const int32_t *kv_len = nullptr;
    // paged caches (decode): k and v are pools of num_pages pages of
    // 2^page_shift rows [page][row][Hkv][d]; key j of sequence b lives in page
    // block_table[b * max_pages + (j >> page_shift)] (device, int32).  NULL:
    // contiguous [B][Lkv][Hkv][d] caches.
    const int32_t *block_table = nullptr;
    int page_shift = 0, max_pages = 0, num_pages = 0;
    // a sparse layer's own window K/V (hysparse_sparse_attn_own_window):
    // [B][Lwin][Hkv][d] holding positions Lkv - Lwin .. Lkv - 1; the window
    // branch reads it instead of k, v.  NULL: the shared cache.
    const void *k_win = nullptr, *v_win = nullptr;
    int Lwin = 0;
    int G() const { return Hq / Hkv; }
};

// simt_attn.cu
cudaError_t full_attn_scores_simt_launch(const Shape &s, const void *q, const void *k,
                                         const void *v, void *out, float *lse, float *scores,
                                         long long ld, int row_begin, int row_count,
                                         cudaStream_t st);
cudaError_t sparse_attn_simt_launch(const Shape &s, const void *q, const void *k, const void *v,
                                    const int32_t *idx, int topk, const float *gate, int window,
                                    void *out, void *og, void *ol, unsigned int *status,
                                    cudaStream_t st);

// attn_tc.cu (bf16, d = 128, even group size)
bool full_attn_tc_supported(const Shape &s);
cudaError_t full_attn_scores_tc_launch(const Shape &s, const void *q, const void *k, const void *v,
                                       void *out, float *lse, float *scores, long long ld,
                                       int row_begin, int row_count, float2 *stats,
                                       unsigned int *status, unsigned long long wait_ns,
                                       cudaStream_t st);

// sparse_mma.cu (bf16, d = 128, G <= 16)
bool sparse_mma_supported(const Shape &s);
// n (<= 16) sparse layers over the same index set and cache in one gather
// launch (layer l: q[l], gate[l], out[l]; device pointers in host arrays)
cudaError_t sparse_attn_mma_layers_launch(const Shape &s, int n, const void *const *q, const void *k, const void *v,
                                          const int32_t *idx, int topk, const float *const *gate, int window,
                                          void *const *out, unsigned int *status, unsigned long long wait_ns,
                                          cudaStream_t st);
cudaError_t sparse_attn_mma_launch(const Shape &s, const void *q, const void *k, const void *v,
                                   const int32_t *idx, int topk, const float *gate, int window, void *out,
                                   void *og, void *ol, unsigned int *status, unsigned long long wait_ns,
                                   cudaStream_t st);

// sparse_gather_tc.cu (bf16, d = 128, G <= 16, contiguous caches): the
// sparse layer as a row gather on the tcgen05 tensor cores
bool sparse_gather_tc_supported(const Shape &s);
cudaError_t sparse_gather_tc_launch(const Shape &s, const void *q, const void *k, const void *v,
                                    const int32_t *idx, int topk, const float *gate, int window, void *out,
                                    void *og, void *ol, unsigned int *status, unsigned long long wait_ns,
                                    cudaStream_t st);

// sparse_mma.cu, decode full layer (bf16, d = 128, G <= 16, Lq == 1): split-K
// partials + logit stash in `ws` (decode_ws_bytes of it), then a combine.
size_t decode_ws_bytes(const Shape &s);
cudaError_t decode_full_mma_launch(const Shape &s, const void *q, const void *k, const void *v, void *out,
                                   float *lse, float *scores, long long ld, void *ws, unsigned int *status,
                                   cudaStream_t st);

// sparse_tc.cu: dense-masked sparse layer (bf16, d = 128, Lq >= 64); its
// selection bitmask (selmask_bytes) lives in the caller's workspace.
bool sparse_dense_supported(const Shape &s);
int selmask_words(const Shape &s);
size_t selmask_bytes(const Shape &s);
cudaError_t sparse_dense_tc_launch(const Shape &s, const void *q, const void *k, const void *v,
                                   const int32_t *idx, int topk, const float *gate, int window, void *out,
                                   void *og, void *ol, uint32_t *mask, unsigned int *status,
                                   unsigned long long wait_ns, cudaStream_t st);

cudaError_t selmask_build_launch(const Shape &s, const int32_t *idx, int topk, uint32_t *mask, unsigned int *status,
                                 cudaStream_t st);

// attn_tc.cu, dense-masked sparse layer on the paired-head pipeline of the
// full layer (even G): window branch into `wl` (bf16), then the masked global
// branch merged by the gate.
bool sparse_pair_supported(const Shape &s);
size_t sparse_pair_wl_bytes(const Shape &s);
cudaError_t sparse_pair_tc_launch(const Shape &s, const void *q, const void *k, const void *v, const float *gate,
                                  int window, void *out, void *og, void *ol, const uint32_t *mask, int W,
                                  uint32_t *wl, unsigned int *status, unsigned long long wait_ns, cudaStream_t st);

// Upper bound (ns) on any single barrier wait inside a kernel; after it the
// kernel records HS_ERR_TIMEOUT in the workspace status word and returns.
unsigned long long wait_limit_ns();

// topk.cu
// mask (optional, [B][Hkv][Lq][W] words): also write the rows' selection
// bitmask; *mask_done tells whether every row of the launch got one.
// Row lengths follow s.kv_len when it is set (decode over caches of
// different lengths).
cudaError_t topk_launch(const Shape &s, const float *scores, long long ld, int row_begin,
                        int row_count, int topk, int32_t *idx, cudaStream_t st, uint32_t *mask = nullptr,
                        int W = 0, bool *mask_done = nullptr);

}  // namespace hs
