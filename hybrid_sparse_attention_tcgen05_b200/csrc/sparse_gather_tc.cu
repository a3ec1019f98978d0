// Sparse layer of the hybrid block as a row gather on the tcgen05 tensor
// cores (bf16, d = 128, up to 16 query heads per KV head): the global branch
// over each row's top-k key set, the causal 128-token window branch, and the
// sigmoid gate, reading the full layer's KV cache and writing no KV.
//
// Method: intelliparadigm write-up section 2.2 (dual-branch sparse attention:
// a global branch over the TopK indices of the preceding full layer, a local
// sliding window, out = gate*global + (1-gate)*local with a sigmoid gate) and
// section 3.1 (the sparse layers only read the full layer's cache).
//
// Work item = (KV head, batch, query row): the G query heads of the group
// share the item's key list.  Its keys are processed in chunks of 128 (the
// top-k list, then the window), each chunk a "swap-AB" pair of MMAs with the
// keys as the M dimension so that a small head group fills the N side:
//   S^T[128 keys x 16 heads]  = K_chunk Q^T      (A = gathered K rows, B = Q)
//   O^T[128 d x 16 heads]    += V_chunk^T P      (A = gathered V rows read
//                                                 M-major, B = P^T in smem)
// Both accumulators live in TMEM (S double-buffered, one O per branch).
//
// CTA (persistent, two per SM, items strided over the grid KV head by KV
// head so that one head's K and V stay in L2):
//   warps 0-3  softmax: thread t owns key slot t of a chunk (TMEM lane t of
//              S^T) and, in the epilogue, output column d = t (lane t of O^T)
//   warp 4     producer: gathers the chunk's 128 K rows and 128 V rows with
//              TMA tile::gather4 loads (four 128-byte row halves per
//              instruction, 128-byte swizzled K-major as the MMA reads them),
//              plus the item's query rows with a tiled TMA load; a 3-slot ring
//              of 32 KB tiles in MMA order K0, K1, V0, K2, V1, ...
//   warp 5     MMA issuer (one thread)
// Per-head softmax statistics need a reduction over the keys, i.e. across
// TMEM lanes: each warp takes its 16 maxima with redux.sync.max.f32, and the
// warps agree through one barrier reduction whether any head's reference
// must move (only when a chunk's maximum exceeds it by more than 8 in log2
// units, so after the first chunk this is rare); only then do they exchange
// maxima through shared memory and rescale O in TMEM.  Row sums are kept per
// thread and reduced once per item.
#include <cuda_bf16.h>
#include <stddef.h>
#include <stdlib.h>
#include <string.h>

#include "common.cuh"
#include "internal.h"
#include "tc_attn.cuh"
#include "tc_util.cuh"

namespace hs {
namespace gtc {
namespace {

using namespace tc;

constexpr int CK = 128;              // keys per chunk (MMA M)
constexpr int NH = 16;               // heads per item (MMA N); groups of fewer heads are zero-padded
constexpr int NS_MAX = 6;            // most ring slots of any configuration
constexpr int TILE_B = CK * 256;     // one 128-row bf16 K or V tile: 32 KB
constexpr int HALF_B = TILE_B / 2;   // one 64-column swizzled half
constexpr int QP_B = NH * 256;       // Q or one P buffer: 16 rows x 128 bf16
constexpr int QP_HALF = QP_B / 2;
constexpr int SOFT_WARPS = 4, PROD_WARPS = 1, MMA_WARP = SOFT_WARPS + PROD_WARPS;
constexpr int KPL = 4;               // keys of a chunk per producer lane (rows 4 l .. 4 l + 3)
constexpr int THREADS = 32 * (MMA_WARP + 1);
constexpr uint32_t TMEM_COLS = 64;   // S0 | S1 | O_global | O_local, 16 columns each
constexpr float kLazy = 8.0f;        // log2 units a chunk maximum may exceed the reference by
constexpr uint64_t kDrainNs = 1000000000ull;

struct Bars {
    uint64_t kv_full[NS_MAX], kv_empty[NS_MAX];
    uint64_t q_empty;
    uint64_t s_full[2], s_free[2], p_full[2], pv_done[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
    alignas(16) float xmax[SOFT_WARPS][NH];   // per-warp chunk maxima (exchange; read as float4)
    float red[SOFT_WARPS][2 * NH];   // per-warp row-sum partials (epilogue)
    float wts[4][NH];                // epilogue weights: gate*1/l_g, (1-gate)*1/l_l, 1/l_g, 1/l_l
};

static_assert(offsetof(Bars, xmax) % 16 == 0, "xmax is read and written as float4");

// Ring depth NS and resident CTAs per SM: three 32 KB slots with two CTAs per
// SM, or six with one.
template <int NS>
struct Cfg {
    static constexpr int CTAS = NS <= 3 ? 2 : 1;
    static constexpr size_t kRing = (size_t)NS * TILE_B;
    static constexpr size_t kSmem = 1024 + kRing + QP_B + 2 * QP_B + ((sizeof(Bars) + 127) / 128) * 128;
    static_assert(NS <= NS_MAX, "ring barriers");
    static_assert(CTAS * (kSmem + 1024) <= 233472, "shared memory per SM");
};

struct Params {
    const __nv_bfloat16 *q, *k, *v;
    const int32_t *idx;
    const float *gate;
    __nv_bfloat16 *out, *out_g, *out_l;
    int B, Lq, Lkv, Hq, Hkv, G, topk, window;
    float scale_log2;
    unsigned int *status;
    unsigned long long wait_ns;
    const int32_t *kv_len;   // [B] cache lengths (decode over caches of different lengths) or NULL
    long long n_items;
};

struct Item {
    int b, i, g, pos, lo, n_g, n;
};

__device__ __forceinline__ int seq_len(const Params &p, int b) {
    if (p.kv_len == nullptr) return p.Lkv;
    const int L = __ldg(p.kv_len + b);
    if (L < 1 || L > p.Lkv) {
        report(p.status, HS_ERR_INVALID_ARG);
        return L < 1 ? 1 : p.Lkv;
    }
    return L;
}

// Items are (KV head slowest, batch, row fastest).  n_g = chunks of the top-k
// list, n = n_g + chunks of the window [lo, pos].
__device__ __forceinline__ Item item_of(const Params &p, long long it) {
    Item r;
    r.i = (int)(it % p.Lq);
    const long long hb = it / p.Lq;
    r.b = (int)(hb % p.B);
    r.g = (int)(hb / p.B);
    r.pos = seq_len(p, r.b) - p.Lq + r.i;
    r.lo = max(0, r.pos - p.window + 1);
    r.n_g = (p.topk + CK - 1) / CK;
    r.n = r.n_g + (r.pos - r.lo + CK) / CK;
    return r;
}

// Ring position (relative to the item's first tile) of K_j and V_j: the MMA
// issues S_{j+1} = K_{j+1} Q^T before O += V_j^T P_j.
__device__ __forceinline__ int seq_k(int j) { return j == 0 ? 0 : 2 * j - 1; }
__device__ __forceinline__ int seq_v(int j, int n) { return j + 1 < n ? 2 * j + 2 : 2 * j + 1; }

// TMA gather of four rows (tile::gather4, 2-D map, one-row box): the box's
// columns of rows r0..r3 land as four consecutive box rows at dst.  Signals
// `bar` with the bytes written.  No multicast.
__device__ __forceinline__ void tma_gather4(uint32_t dst, const CUtensorMap *m, uint32_t bar, int x, int r0, int r1,
                                            int r2, int r3) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(x), "r"(r0), "r"(r1), "r"(r2), "r"(r3)
        : "memory");
}

// 2-D tiled TMA load; signals `bar` with the bytes written.  No multicast.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *m, uint32_t bar, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(x), "r"(y)
        : "memory");
}

__device__ __forceinline__ float redux_max(float x) {
    float r;
    asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(x));
    return r;
}

// Bounded barrier wait (gives up after limit_ns or on abort, like mbar_wait)
// that polls with the non-blocking test_wait: a chunk's work between two
// hand-offs is short, and a suspended waiter wakes up late.
__device__ __forceinline__ bool test_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ bool wait_sleep(uint32_t bar, uint32_t parity, uint64_t limit_ns, volatile int *abort) {
    if (test_wait(bar, parity)) return true;
    if (limit_ns == 0) {   // zero budget: give up at the first unsatisfied poll
        *abort = 1;
        return false;
    }
    const uint64_t t0 = globaltimer();
    for (uint32_t it = 1;; ++it) {
        if (test_wait(bar, parity)) return true;
        if ((it & 255u) == 0) {
            if (*abort) return false;
            if (globaltimer() - t0 > limit_ns) {
                *abort = 1;
                return false;
            }
        }
    }
}

// Named barrier 1 over the softmax warpgroup (128 threads), with an OR
// reduction of a predicate: every thread gets the same answer.
__device__ __forceinline__ bool wg_any(bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, 1, 128, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ void wg_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Raw key of list entry / window slot t of chunk j: the list entry as
// stored (not yet checked), the window key, or -1 past the list or window.
// Loads are issued well ahead of their use and checked by key_checked at use,
// so that no warp stalls on an index load it does not need yet.
__device__ __forceinline__ int chunk_key_raw(const Params &p, const int32_t *list, const Item &it, int j, int t) {
    if (j < it.n_g) {
        const int e = j * CK + t;
        return e < p.topk ? __ldg(list + e) : -1;
    }
    const int key = it.lo + (j - it.n_g) * CK + t;
    return key <= it.pos ? key : -1;
}

// A raw key checked against the row's causal range: -1 for none; an entry
// outside [-1, pos] is dropped (and reported when report_bad).
__device__ __forceinline__ int key_checked(const Params &p, int key, int pos, bool report_bad) {
    if (key < -1 || key > pos) {
        if (report_bad) report(p.status, HS_ERR_INVALID_INDEX);
        return -1;
    }
    return key;
}

__device__ __forceinline__ const int32_t *list_of(const Params &p, const Item &it) {
    return p.idx + (((size_t)it.b * p.Hkv + it.g) * p.Lq + it.i) * p.topk;
}

// Registers per thread: two CTAs of THREADS threads share the SM's 65536.
template <int NS>
constexpr int max_regs() { return Cfg<NS>::CTAS == 2 ? (65536 / (2 * THREADS)) / 8 * 8 : 255; }

template <int NS>
__global__ void __launch_bounds__(THREADS) __maxnreg__(max_regs<NS>()) sparse_gather_tc(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                 const __grid_constant__ CUtensorMap tv, const Params p) {
    constexpr size_t kRing = Cfg<NS>::kRing;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *ring = smem;
    uint8_t *sq = smem + kRing;
    uint8_t *sp = sq + QP_B;                 // two P buffers
    Bars *bars = reinterpret_cast<Bars *>(sp + 2 * QP_B);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(smem_u32(&bars->kv_full[s]), 1);
            mbar_init(smem_u32(&bars->kv_empty[s]), 1);
        }
        mbar_init(smem_u32(&bars->q_empty), 1);
        for (int w = 0; w < 2; ++w) {
            mbar_init(smem_u32(&bars->s_full[w]), 1);
            mbar_init(smem_u32(&bars->s_free[w]), 128);
            mbar_init(smem_u32(&bars->p_full[w]), 128);
            mbar_init(smem_u32(&bars->pv_done[w]), 1);
        }
        mbar_init(smem_u32(&bars->drain), 1);
        bars->abort = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(&bars->tmem_base), TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    volatile int *abort = &bars->abort;
    const long long stride = gridDim.x;

    if (warp >= SOFT_WARPS && warp < MMA_WARP) {
        // ------------------------------------------------------ producer warp
        // Lane l fetches rows 4l .. 4l+3 of every tile with TMA gathers: one
        // tile::gather4 per 64-column half moves four whole 128-byte row halves,
        // 128-byte swizzled as the MMA reads them, and the TMA unit signals the
        // slot's full barrier with the bytes it wrote.
        if (lane == 0) {
            tma_prefetch(&tq);
            tma_prefetch(&tk);
            tma_prefetch(&tv);
        }
        int seq = 0, item_n = 0;
        bool ok = true;
        // look-ahead over the CTA's stream of chunks (items in order, their
        // chunks in order): the keys of the chunk two K tiles ahead are loaded
        // while the warp waits, across item boundaries too; they are checked
        // against the row's range only at use
        long long la_item = blockIdx.x;
        Item la = item_of(p, la_item);
        int la_j = 0;
        auto la_keys = [&](int (&dst)[KPL]) {
            const bool live = la_item < p.n_items;
#pragma unroll
            for (int u = 0; u < KPL; ++u)
                dst[u] = live ? chunk_key_raw(p, list_of(p, la), la, la_j, 4 * lane + u) : -1;
            if (live && ++la_j == la.n) {
                la_j = 0;
                la_item += stride;
                if (la_item < p.n_items) la = item_of(p, la_item);
            }
        };
        int ka[KPL], kp[KPL], kn[KPL], knn[KPL];
#pragma unroll
        for (int u = 0; u < KPL; ++u) ka[u] = kp[u] = -1;
        la_keys(kn);
        la_keys(knn);
        for (long long it_ = blockIdx.x; ok && it_ < p.n_items; it_ += stride, ++item_n) {
            const Item it = item_of(p, it_);
            const int row0 = it.b * p.Lkv;                    // key 0 of this sequence in the [B*Lkv] rows
            const int col0 = it.g * 128;                      // this KV head's columns
            const int qr = (it.b * p.Lq + it.i) * p.Hq + it.g * p.G;   // first query row of the group
            int jk = -1;
            for (int t = 0; t < 2 * it.n; ++t) {
                // production order: K0, then (K_{j+1}, V_j) pairs, then the last V
                int j, is_v;
                if (t == 0) { j = 0; is_v = 0; }
                else if (t == 2 * it.n - 1) { j = it.n - 1; is_v = 1; }
                else { is_v = (t & 1) == 0; j = is_v ? (t - 2) / 2 : (t + 1) / 2; }
                int key[KPL];
                if (!is_v) {
                    jk = j;
#pragma unroll
                    for (int u = 0; u < KPL; ++u) {
                        kp[u] = ka[u];
                        ka[u] = key_checked(p, kn[u], it.pos, true);   // loaded two K tiles ago
                        kn[u] = knn[u];
                        key[u] = ka[u];
                    }
                    la_keys(knn);
                } else {                   // the item's last V follows its own K; else V_{jk-1}
#pragma unroll
                    for (int u = 0; u < KPL; ++u) key[u] = j == jk ? ka[u] : kp[u];
                }
                const int slot = seq % NS, use = seq / NS;
                if (!(ok = __all_sync(0xffffffffu, wait_sleep(smem_u32(&bars->kv_empty[slot]), (use & 1) ^ 1,
                                                              p.wait_ns, abort))))
                    break;
                if (t == 0 && !(ok = __all_sync(0xffffffffu, wait_sleep(smem_u32(&bars->q_empty), (item_n & 1) ^ 1,
                                                                        p.wait_ns, abort))))
                    break;   // the previous item's last S = K Q^T must have read Q
                const uint32_t fb = smem_u32(&bars->kv_full[slot]);
                if (lane == 0) mbar_expect_tx(fb, TILE_B + (t == 0 ? QP_B : 0));
                __syncwarp();
                if (t == 0 && lane < 2)   // the group's query rows (rows past the tensor read as zeros)
                    tma_load_2d(smem_u32(sq) + lane * QP_HALF, &tq, fb, lane * 64, qr);
                // a key that is -1 (or was dropped) fetches key 0's row, which the
                // softmax masks out: every row written is finite data
                int r[KPL];
#pragma unroll
                for (int u = 0; u < KPL; ++u) r[u] = row0 + (key[u] >= 0 ? key[u] : 0);
                const CUtensorMap *m = is_v ? &tv : &tk;
                const uint32_t tb = smem_u32(ring + slot * TILE_B) + (uint32_t)lane * 4u * 128u;
                tma_gather4(tb, m, fb, col0, r[0], r[1], r[2], r[3]);
                tma_gather4(tb + HALF_B, m, fb, col0 + 64, r[0], r[1], r[2], r[3]);
                ++seq;
            }
        }
        if (lane == 0 && *abort) {
            // let our own copies land before the CTA goes away
            for (int s2 = seq > NS ? seq - NS : 0; s2 < seq; ++s2)
                mbar_drain(smem_u32(&bars->kv_full[s2 % NS]), (s2 / NS) & 1);
        }
    } else if (warp == MMA_WARP) {
        // ------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t I_S = idesc_bf16(CK, NH, false, false);
            constexpr uint32_t I_O = idesc_bf16(128, NH, true, false);
            const uint32_t qa = smem_u32(sq);
            int gc = 0, T = 0;
            bool ok = true;
            for (long long it_ = blockIdx.x; ok && it_ < p.n_items; it_ += stride) {
                const Item it = item_of(p, it_);
                auto issue_s = [&](int j) -> bool {
                    const int c = gc + j, tk = T + seq_k(j), slot = tk % NS;
                    if (!wait_sleep(smem_u32(&bars->kv_full[slot]), (tk / NS) & 1, p.wait_ns, abort)) return false;
                    if (!wait_sleep(smem_u32(&bars->s_free[c & 1]), ((c >> 1) & 1) ^ 1, p.wait_ns, abort))
                        return false;
                    tc_fence_after();
                    const uint32_t ka = smem_u32(ring + slot * TILE_B);
                    const uint32_t d = tmem + (uint32_t)((c & 1) * NH);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t o = (kk & 3) * 32;
                        mma_ss(d, sdesc_sw128(ka + (kk >> 2) * HALF_B + o, 16, 1024),
                               sdesc_sw128(qa + (kk >> 2) * QP_HALF + o, 16, 1024), I_S, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(smem_u32(&bars->s_full[c & 1]));
                    if (j == it.n - 1) mma_commit(smem_u32(&bars->q_empty));
                    mma_commit(smem_u32(&bars->kv_empty[slot]));
                    return true;
                };
                if (!(ok = issue_s(0))) break;
                for (int j = 0; j < it.n; ++j) {
                    if (j + 1 < it.n && !(ok = issue_s(j + 1))) break;
                    const int c = gc + j, tv_ = T + seq_v(j, it.n), slot = tv_ % NS;
                    if (!(ok = wait_sleep(smem_u32(&bars->kv_full[slot]), (tv_ / NS) & 1, p.wait_ns, abort))) break;
                    if (!(ok = wait_sleep(smem_u32(&bars->p_full[c & 1]), (c >> 1) & 1, p.wait_ns, abort))) break;
                    tc_fence_after();
                    const uint32_t va = smem_u32(ring + slot * TILE_B);
                    const uint32_t pa = smem_u32(sp + (c & 1) * QP_B);
                    const bool first = j == 0 || j == it.n_g;
                    const uint32_t d = tmem + (uint32_t)(2 * NH + (j < it.n_g ? 0 : NH));
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        mma_ss(d, sdesc_sw128(va + kk * 2048, HALF_B, 1024),
                               sdesc_sw128(pa + (kk >> 2) * QP_HALF + (kk & 3) * 32, 16, 1024), I_O,
                               (!first || kk > 0) ? 1u : 0u);
                    }
                    mma_commit(smem_u32(&bars->pv_done[c & 1]));
                    mma_commit(smem_u32(&bars->kv_empty[slot]));
                }
                gc += it.n;
                T += 2 * it.n;
            }
            mma_commit(smem_u32(&bars->drain));
            int dummy = 0;
            mbar_wait(smem_u32(&bars->drain), 0, kDrainNs, &dummy);
        }
    } else {
        // ------------------------------------------------------ softmax warpgroup
        const int t = threadIdx.x;                         // key slot / output column
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        const float c2 = p.scale_log2;
        bool bad = false;
        int gc = 0;
        for (long long it_ = blockIdx.x; it_ < p.n_items; it_ += stride) {
            if (wg_any(bad || *abort)) break;
            const Item it = item_of(p, it_);
            const int32_t *list = list_of(p, it);
            float m[NH], lp_g[NH], lp_l[NH];
#pragma unroll
            for (int h = 0; h < NH; ++h) { m[h] = -INFINITY; lp_g[h] = 0.f; lp_l[h] = 0.f; }
            int key_next = chunk_key_raw(p, list, it, 0, t);
            for (int j = 0; j < it.n; ++j) {
                const int c = gc + j;
                if (wg_any(bad || *abort)) break;
                const bool glob = j < it.n_g;
                const bool first = j == 0 || j == it.n_g;
                if (j == it.n_g) {
#pragma unroll
                    for (int h = 0; h < NH; ++h) m[h] = -INFINITY;   // the window branch starts afresh
                }
                const bool valid = key_checked(p, key_next, it.pos, false) >= 0;
                if (j + 1 < it.n) key_next = chunk_key_raw(p, list, it, j + 1, t);
                bad |= !__all_sync(0xffffffffu, wait_sleep(smem_u32(&bars->s_full[c & 1]), (c >> 1) & 1,
                                                          p.wait_ns, abort));
                tc_fence_after();
                float x[NH];
                {
                    uint32_t r[NH];
                    tmem_ld16(tmem + lane_off + (uint32_t)((c & 1) * NH), r);
                    tmem_wait_ld();
#pragma unroll
                    for (int h = 0; h < NH; ++h) x[h] = valid ? __uint_as_float(r[h]) * c2 : -INFINITY;
                }
                tc_fence_before();
                mbar_arrive(smem_u32(&bars->s_free[c & 1]));
                float wmax[NH];
                bool need = false;
#pragma unroll
                for (int h = 0; h < NH; ++h) {
                    wmax[h] = redux_max(x[h]);
                    need |= wmax[h] > m[h] + kLazy;
                }
                if (wg_any(need)) {
                    if (lane == 0) {
#pragma unroll
                        for (int h = 0; h < NH; h += 4)
                            *reinterpret_cast<float4 *>(&bars->xmax[warp][h]) =
                                make_float4(wmax[h], wmax[h + 1], wmax[h + 2], wmax[h + 3]);
                    }
                    wg_sync();
                    float corr[NH];
#pragma unroll
                    for (int h = 0; h < NH; h += 4) {
                        float4 a = *reinterpret_cast<const float4 *>(&bars->xmax[0][h]);
#pragma unroll
                        for (int w = 1; w < SOFT_WARPS; ++w) {
                            const float4 b4 = *reinterpret_cast<const float4 *>(&bars->xmax[w][h]);
                            a = make_float4(fmaxf(a.x, b4.x), fmaxf(a.y, b4.y), fmaxf(a.z, b4.z), fmaxf(a.w, b4.w));
                        }
                        const float cm[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float mn = fmaxf(m[h + e], cm[e]);
                            corr[h + e] = mn == -INFINITY ? 1.f : ex2(m[h + e] - mn);
                            m[h + e] = mn;
                        }
                    }
                    if (!first) {
                        // O of this branch must hold the previous chunk's product
                        // before it is rescaled in place
                        const int cp_ = c - 1;
                        bad |= !__all_sync(0xffffffffu, wait_sleep(smem_u32(&bars->pv_done[cp_ & 1]),
                                                                  (cp_ >> 1) & 1, p.wait_ns, abort));
                        tc_fence_after();
                        const uint32_t to = tmem + lane_off + (uint32_t)(2 * NH + (glob ? 0 : NH));
                        uint32_t o[NH];
                        tmem_ld16(to, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int h = 0; h < NH; ++h) o[h] = __float_as_uint(__uint_as_float(o[h]) * corr[h]);
                        tmem_st16(to, o);
                        tmem_wait_st();
                        tc_fence_before();
                    }
#pragma unroll
                    for (int h = 0; h < NH; ++h) {
                        lp_g[h] *= glob ? corr[h] : 1.f;
                        lp_l[h] *= glob ? 1.f : corr[h];
                    }
                }
                // P buffer c&1 was last read by PV(c-2)
                if (c >= 2)
                    bad |= !__all_sync(0xffffffffu, wait_sleep(smem_u32(&bars->pv_done[c & 1]), ((c - 2) >> 1) & 1,
                                                              p.wait_ns, abort));
                uint8_t *pb = sp + (c & 1) * QP_B + (t >> 6) * QP_HALF + ((t & 7) << 1);
                const int c8 = (t & 63) >> 3;
#pragma unroll
                for (int h = 0; h < NH; ++h) {
                    const float mref = m[h] == -INFINITY ? 0.f : m[h];
                    const float pv = ex2(x[h] - mref);
                    if (glob) lp_g[h] += pv; else lp_l[h] += pv;
                    *reinterpret_cast<__nv_bfloat16 *>(pb + h * 128 + ((c8 ^ (h & 7)) << 4)) = __float2bfloat16_rn(pv);
                }
                fence_proxy_async_smem();
                mbar_arrive(smem_u32(&bars->p_full[c & 1]));
            }
            const int c_last = gc + it.n - 1;
            gc += it.n;
            if (wg_any(bad || *abort)) break;
            // ---- epilogue: row sums, gate, the item's G output rows
            bad |= !__all_sync(0xffffffffu, wait_sleep(smem_u32(&bars->pv_done[c_last & 1]), (c_last >> 1) & 1,
                                                      p.wait_ns, abort));
            tc_fence_after();
            {
                // reduce the 32 per-thread partial sums over the warp: after the
                // transposed butterfly, lane l holds the sum of value l
                float v[2 * NH];
#pragma unroll
                for (int h = 0; h < NH; ++h) { v[h] = lp_g[h]; v[NH + h] = lp_l[h]; }
#pragma unroll
                for (int o = 16, n = 32; o >= 1; o >>= 1, n >>= 1) {
                    const bool upper = (lane & o) != 0;
#pragma unroll
                    for (int e = 0; e < n / 2; ++e) {
                        const float send = upper ? v[e] : v[e + n / 2];
                        const float keep = upper ? v[e + n / 2] : v[e];
                        v[e] = keep + __shfl_xor_sync(0xffffffffu, send, o);
                    }
                }
                bars->red[warp][lane] = v[0];
            }
            wg_sync();
            if (warp == 0) {
                const float l = bars->red[0][lane] + bars->red[1][lane] + bars->red[2][lane] + bars->red[3][lane];
                const float il = l > 0.f ? 1.0f / l : 0.f;    // an empty branch gives zero
                const int h = lane & (NH - 1);
                const float il_g = __shfl_sync(0xffffffffu, il, h);
                const float il_l = __shfl_sync(0xffffffffu, il, NH + h);
                if (lane < NH) {
                    float sg = 0.f;
                    if (h < p.G) {
                        const float gl = __ldg(p.gate + ((size_t)it.b * p.Lq + it.i) * p.Hq + (size_t)it.g * p.G + h);
                        sg = 1.0f / (1.0f + expf(-gl));
                    }
                    bars->wts[0][h] = sg * il_g;
                    bars->wts[1][h] = (1.f - sg) * il_l;
                    bars->wts[2][h] = il_g;
                    bars->wts[3][h] = il_l;
                }
            }
            wg_sync();
            float og[NH], ol[NH];
            {
                uint32_t r[NH];
                tmem_ld16(tmem + lane_off + (uint32_t)(2 * NH), r);
                tmem_wait_ld();
#pragma unroll
                for (int h = 0; h < NH; ++h) og[h] = __uint_as_float(r[h]);
                tmem_ld16(tmem + lane_off + (uint32_t)(3 * NH), r);
                tmem_wait_ld();
#pragma unroll
                for (int h = 0; h < NH; ++h) ol[h] = __uint_as_float(r[h]);
            }
            tc_fence_before();
            // stage [G][128] bf16 rows in the (now idle) P buffers, then write the
            // group's G contiguous output rows with 16-byte stores
            __nv_bfloat16 *stg = reinterpret_cast<__nv_bfloat16 *>(sp);
            const size_t orow = (((size_t)it.b * p.Lq + it.i) * p.Hq + (size_t)it.g * p.G) * 128;
#pragma unroll 1
            for (int which = 0; which < 3; ++which) {
                __nv_bfloat16 *dst = which == 0 ? p.out : (which == 1 ? p.out_g : p.out_l);
                if (dst == nullptr) continue;
#pragma unroll
                for (int h = 0; h < NH; ++h) {
                    const float a = which == 0 ? bars->wts[0][h] : (which == 1 ? bars->wts[2][h] : 0.f);
                    const float b = which == 0 ? bars->wts[1][h] : (which == 2 ? bars->wts[3][h] : 0.f);
                    stg[h * 128 + t] = __float2bfloat16_rn(og[h] * a + ol[h] * b);
                }
                wg_sync();
                for (int e = t; e < p.G * 16; e += 128)
                    reinterpret_cast<uint4 *>(dst + orow)[e] = reinterpret_cast<const uint4 *>(stg)[e];
                wg_sync();
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
    if (threadIdx.x == 0 && bars->abort) report(p.status, HS_ERR_TIMEOUT);
}

}  // namespace
}  // namespace gtc

bool sparse_gather_tc_supported(const Shape &s) {
    return s.dtype == HS_BF16 && s.d == 128 && s.G() <= gtc::NH && s.block_table == nullptr;
}

namespace {
// 2-D map over a bf16 matrix of `rows` rows of `cols` elements (row pitch
// `cols` elements), a {64, box_rows} box, 128-byte swizzle; rows past the end
// read as zeros.
bool make_map_2d(CUtensorMap *m, const void *base, long long cols, long long rows, int box_rows) {
    auto enc = tc::encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int NS>
cudaError_t launch_ns(const gtc::Params &p0, cudaStream_t st) {
    CUtensorMap mq, mk, mv;
    // K and V as [B*Lkv rows][Hkv*128] (one gathered row = one key's KV-head slice,
    // one-row box for tile::gather4); Q as [B*Lq*Hq rows][128] with a 16-row box
    if (!make_map_2d(&mk, p0.k, (long long)p0.Hkv * 128, (long long)p0.B * p0.Lkv, 1) ||
        !make_map_2d(&mv, p0.v, (long long)p0.Hkv * 128, (long long)p0.B * p0.Lkv, 1) ||
        !make_map_2d(&mq, p0.q, 128, (long long)p0.B * p0.Lq * p0.Hq, gtc::NH))
        return cudaErrorInvalidValue;
    using namespace gtc;
    static bool attr = false;
    if (!attr) {
        cudaError_t e = cudaFuncSetAttribute(sparse_gather_tc<NS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)Cfg<NS>::kSmem);
        if (e != cudaSuccess) return e;
        attr = true;
    }
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    // items are dealt round-robin over the resident CTAs, and the grid is
    // trimmed so that every CTA gets the same number of items (or one fewer)
    const long long slots = (long long)Cfg<NS>::CTAS * sms;
    const long long per = (p0.n_items + slots - 1) / slots;
    const long long grid = (p0.n_items + per - 1) / per;
    sparse_gather_tc<NS><<<(unsigned)grid, THREADS, Cfg<NS>::kSmem, st>>>(mq, mk, mv, p0);
    count_launch();
    return cudaGetLastError();
}
}  // namespace

cudaError_t sparse_gather_tc_launch(const Shape &s, const void *q, const void *k, const void *v, const int32_t *idx,
                                    int topk, const float *gate, int window, void *out, void *og, void *ol,
                                    unsigned int *status, unsigned long long wait_ns, cudaStream_t st) {
    using namespace gtc;
    Params p{(const __nv_bfloat16 *)q, (const __nv_bfloat16 *)k, (const __nv_bfloat16 *)v, idx, gate,
             (__nv_bfloat16 *)out, (__nv_bfloat16 *)og, (__nv_bfloat16 *)ol, s.B, s.Lq, s.Lkv, s.Hq, s.Hkv, s.G(),
             topk, window, s.scale * kLog2e, status, wait_ns, s.kv_len, (long long)s.B * s.Lq * s.Hkv};
    const char *e = getenv("HYSPARSE_GATHER_TC_SLOTS");
    if (e && strcmp(e, "6") == 0) return launch_ns<6>(p, st);
    return launch_ns<3>(p, st);
}

}  // namespace hs
