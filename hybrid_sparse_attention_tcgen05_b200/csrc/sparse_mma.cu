// Sparse layer of the hybrid block on the tensor cores (bf16, d = 128):
// global branch over each row's top-k key set + causal 128-token window
// branch + sigmoid gate, reading the full layer's KV cache and writing no KV.
//
// Method: intelliparadigm write-up section 2.2 (dual-branch sparse attention:
// a global branch over the TopK indices of the preceding full layer, a local
// 128-token sliding window, out = gate*global + (1-gate)*local with a sigmoid
// gate) and section 3.1 (the sparse layers only read the full layer's cache).
//
// One warp owns one (KV head, batch, query row) item: the G query heads of
// that group share the item's key list.  Keys are gathered 32 at a time with
// cp.async 16-byte copies (each warp instruction moves two whole 256-byte K or
// V rows, so every L2 sector fetched is used) into a 3-stage shared-memory
// ring; rows are padded to 272 bytes so ldmatrix is conflict-free, and slots
// of invalid keys are zero-filled by the copy itself.  The maths runs on mma.sync m16n8k16 with the keys as M (so a
// small group of heads only pads N to 8 or 16): S^T = K Q^T, an online
// softmax per head column, then O^T += V^T P^T where movmatrix turns the
// S^T accumulator fragment into the B operand.  The window branch reuses the
// same pipeline over the contiguous key range; both branches are merged by
// the gate in registers and the G output rows are written once.
#include <cuda_bf16.h>
#include <stdlib.h>
#include <string.h>

#include "common.cuh"
#include "internal.h"
#include "tc_util.cuh"

namespace hs {
namespace tc {
namespace {

constexpr int RS = 256;           // row stride in shared memory (bytes): one K or V row

// Byte offset of 16-byte chunk c16 (0..15) of row r of a staged tile: the
// chunks of a row are XOR-permuted by r mod 8, so the eight rows an ldmatrix
// reads at one column fall in eight different bank groups (conflict-free at a
// 256-byte stride, without padding).
__device__ __forceinline__ uint32_t sw_off(int r, int c16) {
    return (uint32_t)r * RS + ((uint32_t)(c16 ^ (r & 7)) << 4);
}

// Per head-block count NB (heads padded to 8*NB) and keys per chunk CK (32;
// 16 measured slower): SW warps (items) per CTA, each with an ST-stage chunk
// ring.  A
// warp stages its query rows (and, at the end, its output rows) in the ring's
// last stage, which the pipeline only fills after the rows are in registers.
// Measured at the 64k-token, 16-head workload: 32-key chunks, two stages,
// and as many warps as shared memory holds (each warp is an independent
// gather stream; more of them keep more bytes in flight).
template <int NB, int CK>
struct SpSmem {
    static constexpr int ST = 2;
    static constexpr int SW = 7;
    static constexpr int STAGE_BYTES = 2 * CK * RS;
    static constexpr int WARP_BYTES = ST * STAGE_BYTES;
    static constexpr size_t bytes = (size_t)SW * WARP_BYTES;
    static_assert(8 * NB * RS <= STAGE_BYTES, "query / output staging fits one stage");
    static_assert(bytes <= 232448, "shared memory per CTA");
};

__device__ __forceinline__ float ex2f(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Online softmax + PV state of one branch for NB blocks of 8 heads.
template <int NB>
struct Branch {
    float m[NB][2], l[NB][2], o[NB][8][4];
    // l holds this lane's share of each head column's row sum until finish()
    // adds the eight lanes of the column (lanes with the same lane % 4)
    __device__ void finish() {
#pragma unroll
        for (int nb = 0; nb < NB; ++nb)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                float x = l[nb][e];
                x += __shfl_xor_sync(0xffffffffu, x, 4);
                x += __shfl_xor_sync(0xffffffffu, x, 8);
                x += __shfl_xor_sync(0xffffffffu, x, 16);
                l[nb][e] = x;
            }
    }
    __device__ void init() {
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
#pragma unroll
            for (int e = 0; e < 2; ++e) { m[nb][e] = -INFINITY; l[nb][e] = 0.f; }
#pragma unroll
            for (int md = 0; md < 8; ++md)
#pragma unroll
                for (int r = 0; r < 4; ++r) o[nb][md][r] = 0.f;
        }
    }
};

// Sparse layers one launch may run together (hysparse_block's layers share
// the index set and the cache).
constexpr int kMaxLayerGroup = 16;

struct SpParams {
    const __nv_bfloat16 *q, *k, *v;
    const int32_t *idx;
    const float *gate;
    __nv_bfloat16 *out, *out_g, *out_l;
    int B, Lq, Lkv, Hq, Hkv, G, topk, window;
    float scale_log2;
    unsigned int *status;
    unsigned long long wait_ns;
    const int32_t *kv_len;   // [B] cache lengths (decode over caches of different lengths) or NULL
    // paged caches (decode): k and v are pools of num_pages pages of 2^page_shift
    // rows; key j of sequence b is row j & (2^page_shift - 1) of page
    // block_table[b * max_pages + (j >> page_shift)].  NULL: contiguous caches.
    const int32_t *block_table;
    int page_shift, max_pages, num_pages;
    // the layer's own window K/V ([B][Lwin][Hkv][128], row 0 = position
    // Lkv - Lwin) read by the window branch, or NULL: the shared cache
    const __nv_bfloat16 *kw = nullptr, *vw = nullptr;
    int Lwin = 0;
    // n_layers > 1: that many sparse layers over the same index set and
    // cache in one launch, layer l with queries ql[l], gates gl[l], output
    // outl[l] (q, gate, out unused).  Warps take (item, layer) pairs, layer
    // fastest, so the warps of one item gather the same K/V rows at about the
    // same time and all but the first find them in L2.
    int n_layers = 1;
    const __nv_bfloat16 *ql[kMaxLayerGroup] = {};
    const float *gl[kMaxLayerGroup] = {};
    __nv_bfloat16 *outl[kMaxLayerGroup] = {};
};

// Cache length of sequence b: kv_len[b] when given (a value outside
// [1, Lkv] is reported and clamped, so no read leaves the cache), else Lkv.
__device__ __forceinline__ int seq_len(const SpParams &p, int b) {
    if (p.kv_len == nullptr) return p.Lkv;
    const int L = __ldg(p.kv_len + b);
    if (L < 1 || L > p.Lkv) {
        report(p.status, HS_ERR_INVALID_ARG);
        return L < 1 ? 1 : p.Lkv;
    }
    return L;
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Lane l's entry of chunk c (entry c*32 + l) as stored: the list entry, the
// window key, or -1 past the list.  Loaded one chunk before the chunk is
// issued, so that no warp waits on an index load it is about to use.
template <int CK>
__device__ __forceinline__ int chunk_entry(const int32_t *list, bool from_list, int lo, int n_list, int c, int lane) {
    const int t = c * CK + lane;
    if (lane >= CK || t >= n_list) return -1;
    return from_list ? __ldg(list + t) : lo + t;
}

// Gather the K and V rows of one chunk's 32 entries into `stage` and commit
// them as one cp.async group.  Lane l holds entry l (`entry`, as stored) and
// validates it here; the 32 rows are then copied two per instruction (16
// lanes x 16 bytes per 256-byte row).
template <int CK>
__device__ __forceinline__ void issue_chunk(const SpParams &p, int entry, int pos, const __nv_bfloat16 *kb,
                                            const __nv_bfloat16 *vb, uint8_t *stage, uint32_t &vmask, int lane,
                                            const int32_t *table) {
    int key = entry;
    if (key < -1 || key > pos) {
        report(p.status, HS_ERR_INVALID_INDEX);
        key = -1;
    }
    // row of the key in the cache (kb, vb): the key itself, or its row in the
    // page pool when the cache is paged (a page outside the pool is reported
    // and the key dropped, like an invalid index)
    if (table != nullptr && key >= 0) {
        const int page = __ldg(table + (key >> p.page_shift));
        if (page < 0 || page >= p.num_pages) {
            report(p.status, HS_ERR_INVALID_INDEX);
            key = -1;
        } else {
            key = (page << p.page_shift) | (key & ((1 << p.page_shift) - 1));
        }
    }
    vmask = __ballot_sync(0xffffffffu, key >= 0);
    const uint32_t sbase = smem_u32(stage);
    // four rows per instruction: lanes 8q .. 8q+7 copy row 4 r4 + q, lane s
    // its 16-byte chunk s in one instruction and chunk s + 8 in the next, so
    // each instruction reads four whole 128-byte halves of rows
    const int q = lane >> 3, sct = lane & 7;
#pragma unroll
    for (int r4 = 0; r4 < CK / 4; ++r4) {
        const int row = 4 * r4 + q;
        const int kr = __shfl_sync(0xffffffffu, key, row);
        const bool ok = kr >= 0;
        const size_t so = ok ? (size_t)kr * p.Hkv * 128 + sct * 8 : 0;
        const uint32_t d0 = sbase + sw_off(row, sct), d1 = sbase + sw_off(row, sct + 8);
        cp_async16(d0, kb + so, ok);
        cp_async16(d1, kb + so + 64, ok);
        cp_async16(d0 + CK * RS, vb + so, ok);
        cp_async16(d1 + CK * RS, vb + so + 64, ok);
    }
    cp_async_commit();
}

template <int NB, int CK>
__device__ __forceinline__ void compute_chunk(const uint8_t *stage, uint32_t vmask, const uint32_t (&bq)[NB][8][2],
                                              float c2, Branch<NB> &br, int lane, float *stash = nullptr,
                                              long long stash_ld = 0, int j0 = 0, int G = 0, int j_lim = 0) {
    const uint32_t ks_base = smem_u32(stage);
    constexpr int MT = CK / 16;   // 16-key MMA tiles per chunk
    const uint32_t vs_base = smem_u32(stage + CK * RS);
    float c[NB][MT][4];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int r = 0; r < 4; ++r) c[nb][mt][r] = 0.f;
    // S^T[CK keys x 8NB heads] = K Q^T
    const int arow = (lane & 7) + ((lane >> 3) & 1) * 8;
    const int acol = (lane >> 4) * 8;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            uint32_t a0, a1, a2, a3;
            ldsm_x4(ks_base + sw_off(16 * mt + arow, 2 * ks + (acol >> 3)), a0, a1, a2, a3);
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) mma16816(c[nb][mt], a0, a1, a2, a3, bq[nb][ks][0], bq[nb][ks][1]);
        }
    }
    // online softmax per head column (keys spread over lane/4 and the two row halves)
    bool kv[MT][2];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int rh = 0; rh < 2; ++rh) kv[mt][rh] = (vmask >> (16 * mt + (lane >> 2) + 8 * rh)) & 1u;
    uint32_t bp[NB][MT][2];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            float x[MT][2];
            float cm = -INFINITY;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int rh = 0; rh < 2; ++rh) {
                    x[mt][rh] = kv[mt][rh] ? c[nb][mt][2 * rh + e] * c2 : -INFINITY;
                    cm = fmaxf(cm, x[mt][rh]);
                    if (stash != nullptr) {
                        // every key of the range, -inf for one that was dropped (a page
                        // outside the pool), so that its score is 0 and no stale value
                        // is read back; rows past the range are not written
                        const int h = 8 * nb + 2 * (lane & 3) + e;
                        const int rr = 16 * mt + (lane >> 2) + 8 * rh;
                        if (h < G && rr < j_lim) stash[(long long)h * stash_ld + j0 + rr] = x[mt][rh];
                    }
                }
            cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, 4));
            cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, 8));
            cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, 16));
            const float mn = fmaxf(br.m[nb][e], cm);
            const float corr = (mn == -INFINITY) ? 1.f : ex2f(br.m[nb][e] - mn);
            float ps = 0.f;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int rh = 0; rh < 2; ++rh) {
                    const float pv = (mn == -INFINITY) ? 0.f : ex2f(x[mt][rh] - mn);
                    c[nb][mt][2 * rh + e] = pv;
                    ps += pv;
                }
            // each lane keeps its own share of the row sum (same reference m
            // across the head column); Branch::finish adds the shares up
            br.l[nb][e] = br.l[nb][e] * corr + ps;
            br.m[nb][e] = mn;
#pragma unroll
            for (int md = 0; md < 8; ++md) {
                br.o[nb][md][e] *= corr;
                br.o[nb][md][2 + e] *= corr;
            }
        }
        // P^T fragments (keys x heads) -> B operand (k = keys, n = heads)
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            bp[nb][mt][0] = movm_t(pack_bf16(c[nb][mt][0], c[nb][mt][1]));
            bp[nb][mt][1] = movm_t(pack_bf16(c[nb][mt][2], c[nb][mt][3]));
        }
    }
    // O^T[128 d x 8NB heads] += V^T P^T
    const int vrow = (lane & 7) + ((lane >> 4) & 1) * 8;
    const int vcol = ((lane >> 3) & 1) * 8;
#pragma unroll
    for (int md = 0; md < 8; ++md) {
#pragma unroll
        for (int kt = 0; kt < MT; ++kt) {
            uint32_t a0, a1, a2, a3;
            ldsm_x4_t(vs_base + sw_off(16 * kt + vrow, 2 * md + (vcol >> 3)), a0, a1, a2, a3);
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) mma16816(br.o[nb][md], a0, a1, a2, a3, bp[nb][kt][0], bp[nb][kt][1]);
        }
    }
}

// Everything one warp needs to run a branch's gather pipeline.
struct WarpCtx {
    const SpParams *p;
    const int32_t *list;
    const __nv_bfloat16 *kb, *vb;
    const int32_t *table = nullptr;   // this sequence's block table row (paged caches) or NULL
    uint8_t *wbase;
    int lo, pos, lane;
    float c2;
    float *stash = nullptr;   // decode full layer: scaled logits [G][stash_ld]
    long long stash_ld = 0;
    int G = 0;
};

__device__ __forceinline__ uint32_t pick4(int s, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    return s == 0 ? a : (s == 1 ? b : (s == 2 ? c : d));
}

// Run one branch (from_list: the top-k list, else the causal window) through
// the ST-stage cp.async pipeline.  One group is committed per iteration (an
// empty one past the end), so waiting for "at most ST-1 pending" always means
// the chunk about to be used has landed.
template <int NB, int CK>
__device__ __forceinline__ void run_branch(const WarpCtx &w, bool from_list, const uint32_t (&bq)[NB][8][2],
                                           Branch<NB> &br) {
    constexpr int ST = SpSmem<NB, CK>::ST;
    constexpr int STAGE_BYTES = SpSmem<NB, CK>::STAGE_BYTES;
    static_assert(ST >= 2 && ST <= 4, "pick4 holds two to four stages");
    const SpParams &p = *w.p;
    br.init();
    const int n_list = from_list ? p.topk : w.pos - w.lo + 1;
    const int nch = (n_list + CK - 1) / CK;
    uint32_t vm0 = 0, vm1 = 0, vm2 = 0, vm3 = 0;
    int entry = chunk_entry<CK>(w.list, from_list, w.lo, n_list, 0, w.lane);   // of the next chunk to issue
    auto issue = [&](int c) {
        const int s = c % ST;
        uint32_t vmask = 0;
        if (c < nch) {
            issue_chunk<CK>(p, entry, w.pos, w.kb, w.vb, w.wbase + s * STAGE_BYTES, vmask, w.lane, w.table);
            entry = chunk_entry<CK>(w.list, from_list, w.lo, n_list, c + 1, w.lane);
        } else {
            cp_async_commit();
        }
        if (s == 0) vm0 = vmask; else if (s == 1) vm1 = vmask; else if (s == 2) vm2 = vmask; else vm3 = vmask;
    };
    for (int c = 0; c < ST - 1; ++c) issue(c);
#pragma unroll 1
    for (int c = 0; c < nch; ++c) {
        __syncwarp();
        issue(c + ST - 1);
        cp_async_wait<ST - 1>();
        __syncwarp();
        const int s = c % ST;
        compute_chunk<NB, CK>(w.wbase + s * STAGE_BYTES, pick4(s, vm0, vm1, vm2, vm3), bq, w.c2, br, w.lane,
                              w.stash, w.stash_ld, w.lo + c * CK, w.G, n_list - c * CK);
    }
    cp_async_wait<0>();
    __syncwarp();
    br.finish();
}

template <int NB, int CK, bool LG>   // LG: a group of layers (n_layers > 1)
__global__ void __launch_bounds__(SpSmem<NB, CK>::SW * 32, 1) sparse_attn_mma(const SpParams p) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nl = LG ? p.n_layers : 1;
    long long item = (long long)blockIdx.x * SpSmem<NB, CK>::SW + warp;
    if (item >= (long long)p.B * p.Lq * p.Hkv * nl) return;   // whole warp leaves together
    const int layer = LG ? (int)(item % nl) : 0;
    if (LG) item /= nl;
    const __nv_bfloat16 *qp = LG ? p.ql[layer] : p.q;
    const float *gp = LG ? p.gl[layer] : p.gate;
    __nv_bfloat16 *outp = LG ? p.outl[layer] : p.out;
    // KV head slowest, then batch, then row: neighbouring warps gather from
    // the same KV head's cache (which stays in L2) and have similar row lengths
    const int i = (int)(item % p.Lq);
    const long long head_batch = item / p.Lq;
    const int b = (int)(head_batch % p.B);
    const int g = (int)(head_batch / p.B);
    const int G = p.G;
    const int pos = seq_len(p, b) - p.Lq + i;
    uint8_t *wbase = smem + warp * SpSmem<NB, CK>::WARP_BYTES;
    // query rows (and at the end the output rows) staged in the ring's last stage
    uint8_t *qs = wbase + (SpSmem<NB, CK>::ST - 1) * SpSmem<NB, CK>::STAGE_BYTES;
    // stage the group's query rows (zero rows pad the heads up to 8*NB)
    const size_t qrow = ((size_t)b * p.Lq + i) * p.Hq + (size_t)g * G;
    for (int e = lane; e < 8 * NB * 16; e += 32) {
        const int h = e >> 4, cc = e & 15;
        uint4 val = make_uint4(0, 0, 0, 0);
        if (h < G) val = __ldg(reinterpret_cast<const uint4 *>(qp + (qrow + h) * 128) + cc);
        *reinterpret_cast<uint4 *>(qs + sw_off(h, cc)) = val;
    }
    __syncwarp();
    uint32_t bq[NB][8][2];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
        for (int kp = 0; kp < 4; ++kp)
            ldsm_x4(smem_u32(qs + sw_off(8 * nb + (lane & 7), 4 * kp + (lane >> 3))),
                    bq[nb][2 * kp][0], bq[nb][2 * kp][1], bq[nb][2 * kp + 1][0], bq[nb][2 * kp + 1][1]);

    WarpCtx w;
    w.p = &p;
    if (p.block_table != nullptr) {   // paged: rows of the page pool, located through the table
        w.kb = p.k + (size_t)g * 128;
        w.vb = p.v + (size_t)g * 128;
        w.table = p.block_table + (size_t)b * p.max_pages;
    } else {
        w.kb = p.k + ((size_t)b * p.Lkv * p.Hkv + g) * 128;
        w.vb = p.v + ((size_t)b * p.Lkv * p.Hkv + g) * 128;
    }
    w.list = p.idx + (((size_t)b * p.Hkv + g) * p.Lq + i) * p.topk;
    w.wbase = wbase;
    w.lo = max(0, pos - p.window + 1);
    w.pos = pos;
    w.lane = lane;
    w.c2 = p.scale_log2;
    Branch<NB> bg, bl;
    run_branch<NB, CK>(w, true, bq, bg);
    if (p.kw != nullptr) {
        // the window branch over the layer's own window K/V: its keys are that
        // buffer's rows, position - (Lkv - Lwin)
        const int off = p.Lkv - p.Lwin;
        WarpCtx wl = w;
        wl.kb = p.kw + ((size_t)b * p.Lwin * p.Hkv + g) * 128;
        wl.vb = p.vw + ((size_t)b * p.Lwin * p.Hkv + g) * 128;
        wl.table = nullptr;
        wl.lo = w.lo - off;
        wl.pos = w.pos - off;
        run_branch<NB, CK>(wl, false, bq, bl);
    } else {
        run_branch<NB, CK>(w, false, bq, bl);
    }

    // gate merge, stage the G output rows in shared memory, write them once
    __syncwarp();
    const size_t orow = qrow * 128;
#pragma unroll 1
    for (int which = 0; which < 3; ++which) {
        __nv_bfloat16 *dst = which == 0 ? outp : (which == 1 ? p.out_g : p.out_l);
        if (dst == nullptr) continue;
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int h = 8 * nb + 2 * (lane & 3) + e;
                const float lg = bg.l[nb][e], ll = bl.l[nb][e];
                const float ig = lg > 0.f ? 1.f / lg : 0.f;
                const float il = ll > 0.f ? 1.f / ll : 0.f;
                float sg = 0.f;
                if (h < G) {
                    const float x = gp[((size_t)b * p.Lq + i) * p.Hq + (size_t)g * G + h];
                    sg = 1.0f / (1.0f + expf(-x));
                }
                const float wg = which == 0 ? sg * ig : (which == 1 ? ig : 0.f);
                const float wl = which == 0 ? (1.f - sg) * il : (which == 2 ? il : 0.f);
#pragma unroll
                for (int md = 0; md < 8; ++md)
#pragma unroll
                    for (int rh = 0; rh < 2; ++rh) {
                        const int d = 16 * md + (lane >> 2) + 8 * rh;
                        const float val = bg.o[nb][md][2 * rh + e] * wg + bl.o[nb][md][2 * rh + e] * wl;
                        *reinterpret_cast<__nv_bfloat16 *>(qs + sw_off(h, d >> 3) + (d & 7) * 2) =
                            __float2bfloat16_rn(val);
                    }
            }
        }
        __syncwarp();
        for (int e = lane; e < G * 16; e += 32) {
            const int h = e >> 4, cc = e & 15;
            reinterpret_cast<uint4 *>(dst + orow + (size_t)h * 128)[cc] =
                *reinterpret_cast<const uint4 *>(qs + sw_off(h, cc));
        }
        __syncwarp();
    }
}

// ------------------------------------------------------------ decode full layer
//
// One new query row per batch element (Lq = 1): the full layer is a stream
// over the whole cache, bound by HBM.  Split-K: one warp owns (batch, KV head,
// chunk of kDecChunk keys) and runs the contiguous-range pipeline above,
// writing its online-softmax partial (m, l, unnormalised O per head) and the
// scaled logits of every key (the stash).  decode_combine then merges the
// partials into O and LSE and turns the stash into the exact group-summed
// probabilities with the final per-head max and sum.

constexpr int kDecChunk = 1024;

struct DecParams {
    SpParams sp;
    float *part_o;      // [B][Hq][nchunk][128]
    float2 *part_ml;    // [B][Hq][nchunk]  (m in log2 units, l)
    float *stash;       // [B][Hq][Lkv]
    int nchunk;
};

template <int NB, int CK>
__global__ void __launch_bounds__(SpSmem<NB, CK>::SW * 32, 1) decode_full_mma(const DecParams dp) {
    extern __shared__ __align__(128) uint8_t smem[];
    const SpParams &p = dp.sp;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long item = (long long)blockIdx.x * SpSmem<NB, CK>::SW + warp;
    if (item >= (long long)p.B * p.Hkv * dp.nchunk) return;
    // KV head fastest: neighbouring warps read the same keys' adjacent
    // 256-byte head slices of each 2 KB K and V row
    const int g = (int)(item % p.Hkv);
    const long long rest = item / p.Hkv;
    const int ch = (int)(rest % dp.nchunk);
    const int b = (int)(rest / dp.nchunk);
    const int G = p.G;
    uint8_t *wbase = smem + warp * SpSmem<NB, CK>::WARP_BYTES;
    // query rows (and at the end the output rows) staged in the ring's last stage
    uint8_t *qs = wbase + (SpSmem<NB, CK>::ST - 1) * SpSmem<NB, CK>::STAGE_BYTES;
    const size_t qrow = (size_t)b * p.Hq + (size_t)g * G;      // Lq == 1
    for (int e = lane; e < 8 * NB * 16; e += 32) {
        const int h = e >> 4, cc = e & 15;
        uint4 val = make_uint4(0, 0, 0, 0);
        if (h < G) val = __ldg(reinterpret_cast<const uint4 *>(p.q + (qrow + h) * 128) + cc);
        *reinterpret_cast<uint4 *>(qs + sw_off(h, cc)) = val;
    }
    __syncwarp();
    uint32_t bq[NB][8][2];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
        for (int kp = 0; kp < 4; ++kp)
            ldsm_x4(smem_u32(qs + sw_off(8 * nb + (lane & 7), 4 * kp + (lane >> 3))),
                    bq[nb][2 * kp][0], bq[nb][2 * kp][1], bq[nb][2 * kp + 1][0], bq[nb][2 * kp + 1][1]);
    const int Lb = seq_len(p, b);
    const int lo = ch * kDecChunk;
    const int hi = min(Lb, lo + kDecChunk);
    WarpCtx w;
    w.p = &p;
    if (p.block_table != nullptr) {   // paged: rows of the page pool, located through the table
        w.kb = p.k + (size_t)g * 128;
        w.vb = p.v + (size_t)g * 128;
        w.table = p.block_table + (size_t)b * p.max_pages;
    } else {
        w.kb = p.k + ((size_t)b * p.Lkv * p.Hkv + g) * 128;
        w.vb = p.v + ((size_t)b * p.Lkv * p.Hkv + g) * 128;
    }
    w.list = nullptr;
    w.wbase = wbase;
    w.lo = lo;
    w.pos = hi - 1;            // the range [lo, hi) is read as a "window" ending at hi-1
    w.lane = lane;
    w.c2 = p.scale_log2;
    w.stash = dp.stash + qrow * (size_t)p.Lkv;
    w.stash_ld = p.Lkv;
    w.G = G;
    Branch<NB> br;
    if (lo < hi) run_branch<NB, CK>(w, false, bq, br);
    else br.init();   // a chunk past this sequence's cache: an empty partial (m = -inf, l = 0, O = 0)
#pragma unroll
    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int h = 8 * nb + 2 * (lane & 3) + e;
            if (h >= G) continue;
            const size_t pi = (qrow + h) * dp.nchunk + ch;
            if ((lane >> 2) == 0) dp.part_ml[pi] = make_float2(br.m[nb][e], br.l[nb][e]);
            float *po = dp.part_o + pi * 128;
#pragma unroll
            for (int md = 0; md < 8; ++md)
#pragma unroll
                for (int rh = 0; rh < 2; ++rh) po[16 * md + (lane >> 2) + 8 * rh] = br.o[nb][md][2 * rh + e];
        }
}

// One CTA per (batch, KV head): merge the split-K partials of the G heads
// into O and LSE, then write the importance row from the logit stash.
__global__ void __launch_bounds__(256, 4) decode_combine(const DecParams dp, float *lse, float *scores,
                                                      long long ld_scores) {
    const SpParams &p = dp.sp;
    const int g = blockIdx.x, b = blockIdx.y;
    const int G = p.G;
    __shared__ float s_m[32], s_il[32];
    const size_t qrow = (size_t)b * p.Hq + (size_t)g * G;
    for (int h = threadIdx.x >> 7; h < G; h += blockDim.x >> 7) {
        const int d = threadIdx.x & 127;
        const float2 *ml = dp.part_ml + (qrow + h) * dp.nchunk;
        float M = -INFINITY;
        for (int c = 0; c < dp.nchunk; ++c) M = fmaxf(M, ml[c].x);
        float L = 0.f, acc = 0.f;
        const float *po = dp.part_o + (qrow + h) * dp.nchunk * 128;
        for (int c = 0; c < dp.nchunk; ++c) {
            const float2 v = ml[c];
            const float f = v.x == -INFINITY ? 0.f : ex2f(v.x - M);
            L = fmaf(v.y, f, L);
            acc = fmaf(po[(size_t)c * 128 + d], f, acc);
        }
        p.out[(qrow + h) * 128 + d] = __float2bfloat16_rn(acc / L);
        if (d == 0) {
            lse[qrow + h] = (M + log2f(L)) * kLn2;
            s_m[h] = M;
            s_il[h] = 1.0f / L;
        }
    }
    __syncthreads();
    if (scores == nullptr) return;
    const float *st = dp.stash + qrow * (size_t)p.Lkv;
    float *srow = scores + ((size_t)b * p.Hkv + g) * ld_scores;
    const int Lb = seq_len(p, b);
    // four consecutive keys per thread through 16-byte loads and stores when
    // the rows allow it (more bytes in flight: the pass reads the whole
    // stash), the same arithmetic per key as the scalar loop for the rest
    int j_done = 0;
    if ((p.Lkv & 3) == 0 && (ld_scores & 3) == 0 && (reinterpret_cast<uintptr_t>(st) & 15u) == 0 &&
        (reinterpret_cast<uintptr_t>(srow) & 15u) == 0) {
        const int n4 = Lb >> 2;
#pragma unroll 2
        for (int j4 = threadIdx.x; j4 < n4; j4 += blockDim.x) {
            float4 sc = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int h = 0; h < G; ++h) {
                const float4 x = __ldg(reinterpret_cast<const float4 *>(st + (size_t)h * p.Lkv) + j4);
                const float m = s_m[h], il = s_il[h];
                sc.x = fmaf(ex2f(x.x - m), il, sc.x);
                sc.y = fmaf(ex2f(x.y - m), il, sc.y);
                sc.z = fmaf(ex2f(x.z - m), il, sc.z);
                sc.w = fmaf(ex2f(x.w - m), il, sc.w);
            }
            reinterpret_cast<float4 *>(srow)[j4] = sc;
        }
        j_done = 4 * n4;
    }
    for (int j = j_done + threadIdx.x; j < Lb; j += blockDim.x) {
        float sc = 0.f;
        for (int h = 0; h < G; ++h) sc = fmaf(ex2f(st[(size_t)h * p.Lkv + j] - s_m[h]), s_il[h], sc);
        srow[j] = sc;
    }
}

template <int NB, int CK>
cudaError_t launch_decode(const DecParams &dp, float *lse, float *scores, long long ld, cudaStream_t st) {
    using S = SpSmem<NB, CK>;
    static bool attr = false;
    if (!attr) {
        cudaError_t e = cudaFuncSetAttribute(decode_full_mma<NB, CK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)S::bytes);
        if (e != cudaSuccess) return e;
        attr = true;
    }
    const long long items = (long long)dp.sp.B * dp.sp.Hkv * dp.nchunk;
    const long long blocks = (items + S::SW - 1) / S::SW;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
    decode_full_mma<NB, CK><<<(unsigned)blocks, S::SW * 32, S::bytes, st>>>(dp); count_launch();
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    decode_combine<<<dim3(dp.sp.Hkv, dp.sp.B), 256, 0, st>>>(dp, lse, scores, ld); count_launch();
    return cudaGetLastError();
}

template <int NB, int CK, bool LG = false>
cudaError_t launch_nb(const SpParams &p, cudaStream_t st) {
    using S = SpSmem<NB, CK>;
    static bool attr = false;
    if (!attr) {
        cudaError_t e = cudaFuncSetAttribute(sparse_attn_mma<NB, CK, LG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)S::bytes);
        if (e != cudaSuccess) return e;
        attr = true;
    }
    const long long items = (long long)p.B * p.Lq * p.Hkv * (LG ? p.n_layers : 1);
    const long long blocks = (items + S::SW - 1) / S::SW;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
    sparse_attn_mma<NB, CK, LG><<<(unsigned)blocks, S::SW * 32, S::bytes, st>>>(p); count_launch();
    return cudaGetLastError();
}

}  // namespace
}  // namespace tc

bool sparse_mma_supported(const Shape &s) { return s.dtype == HS_BF16 && s.d == 128 && s.G() <= 16; }

cudaError_t sparse_attn_mma_launch(const Shape &s, const void *q, const void *k, const void *v,
                                   const int32_t *idx, int topk, const float *gate, int window, void *out,
                                   void *og, void *ol, unsigned int *status, unsigned long long wait_ns,
                                   cudaStream_t st) {
    tc::SpParams p{(const __nv_bfloat16 *)q, (const __nv_bfloat16 *)k, (const __nv_bfloat16 *)v, idx, gate,
                   (__nv_bfloat16 *)out, (__nv_bfloat16 *)og, (__nv_bfloat16 *)ol, s.B, s.Lq, s.Lkv, s.Hq,
                   s.Hkv, s.G(), topk, window, s.scale * kLog2e, status, wait_ns, s.kv_len,
                   s.block_table, s.page_shift, s.max_pages, s.num_pages};
    p.kw = (const __nv_bfloat16 *)s.k_win;
    p.vw = (const __nv_bfloat16 *)s.v_win;
    p.Lwin = s.Lwin;
    if (s.G() <= 8) return tc::launch_nb<1, 32>(p, st);
    return tc::launch_nb<2, 32>(p, st);
}

cudaError_t sparse_attn_mma_layers_launch(const Shape &s, int n, const void *const *q, const void *k, const void *v,
                                          const int32_t *idx, int topk, const float *const *gate, int window,
                                          void *const *out, unsigned int *status, unsigned long long wait_ns,
                                          cudaStream_t st) {
    if (n < 1 || n > tc::kMaxLayerGroup || s.k_win != nullptr) return cudaErrorInvalidValue;
    tc::SpParams p{(const __nv_bfloat16 *)q[0], (const __nv_bfloat16 *)k, (const __nv_bfloat16 *)v, idx, gate[0],
                   (__nv_bfloat16 *)out[0], nullptr, nullptr, s.B, s.Lq, s.Lkv, s.Hq, s.Hkv, s.G(), topk, window,
                   s.scale * kLog2e, status, wait_ns, s.kv_len, s.block_table, s.page_shift, s.max_pages,
                   s.num_pages};
    p.n_layers = n;
    for (int l = 0; l < n; ++l) {
        p.ql[l] = (const __nv_bfloat16 *)q[l];
        p.gl[l] = gate[l];
        p.outl[l] = (__nv_bfloat16 *)out[l];
    }
    if (s.G() <= 8) return tc::launch_nb<1, 32, true>(p, st);
    return tc::launch_nb<2, 32, true>(p, st);
}

size_t decode_ws_bytes(const Shape &s) {
    const size_t nchunk = (s.Lkv + tc::kDecChunk - 1) / tc::kDecChunk;
    const size_t rows = (size_t)s.B * s.Hq;
    return rows * nchunk * 128 * sizeof(float) + rows * nchunk * sizeof(float2) + rows * s.Lkv * sizeof(float) +
           3 * 256;
}

cudaError_t decode_full_mma_launch(const Shape &s, const void *q, const void *k, const void *v, void *out,
                                   float *lse, float *scores, long long ld, void *ws, unsigned int *status,
                                   cudaStream_t st) {
    const int nchunk = (s.Lkv + tc::kDecChunk - 1) / tc::kDecChunk;
    const size_t rows = (size_t)s.B * s.Hq;
    char *w = reinterpret_cast<char *>(ws);
    tc::DecParams dp;
    dp.sp = tc::SpParams{(const __nv_bfloat16 *)q, (const __nv_bfloat16 *)k, (const __nv_bfloat16 *)v, nullptr,
                         nullptr, (__nv_bfloat16 *)out, nullptr, nullptr, s.B, 1, s.Lkv, s.Hq, s.Hkv, s.G(),
                         1, 1, s.scale * kLog2e, status, 0, s.kv_len,
                         s.block_table, s.page_shift, s.max_pages, s.num_pages};
    dp.part_o = reinterpret_cast<float *>(w);
    w += align_up(rows * nchunk * 128 * sizeof(float), 256);
    dp.part_ml = reinterpret_cast<float2 *>(w);
    w += align_up(rows * nchunk * sizeof(float2), 256);
    dp.stash = reinterpret_cast<float *>(w);
    dp.nchunk = nchunk;
    if (s.G() <= 8) return tc::launch_decode<1, 32>(dp, lse, scores, ld, st);
    return tc::launch_decode<2, 32>(dp, lse, scores, ld, st);
}

}  // namespace hs
