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
//   warps 4-5  producers: gather the chunk's 128 K rows and 128 V rows with
//              16-byte cp.async into 128-byte-swizzled K-major tiles (a key
//              that is -1 or out of range is zero-filled), plus the item's
//              query rows; a 3-slot ring of 32 KB tiles in MMA order
//              K0, K1, V0, K2, V1, ...
//   warp 6     MMA issuer (one thread)
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
constexpr int THREADS = 32 * (MMA_WARP + 1);
constexpr int PROD_THREADS = 32 * PROD_WARPS;
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

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
                 : "memory");
}
// Arrive on `bar` when every cp.async this thread has issued so far has
// completed; the arrival counts toward the barrier's expected count.
__device__ __forceinline__ void cp_async_arrive_noinc(uint32_t bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

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

// Key of list entry / window slot t of chunk j (-1: none or out of range).
__device__ __forceinline__ int chunk_key(const Params &p, const int32_t *list, const Item &it, int j, int t,
                                         bool report_bad) {
    if (j < it.n_g) {
        const int e = j * CK + t;
        if (e >= p.topk) return -1;
        int key = __ldg(list + e);
        if (key < -1 || key > it.pos) {
            if (report_bad) report(p.status, HS_ERR_INVALID_INDEX);
            key = -1;
        }
        return key;
    }
    const int key = it.lo + (j - it.n_g) * CK + t;
    return key <= it.pos ? key : -1;
}

__device__ __forceinline__ const int32_t *list_of(const Params &p, const Item &it) {
    return p.idx + (((size_t)it.b * p.Hkv + it.g) * p.Lq + it.i) * p.topk;
}

// Byte offset of 16-byte column chunk c16 (0..15) of row r in a K-major,
// 128-byte-swizzled tile whose two 64-column halves are `half_bytes` apart.
__device__ __forceinline__ uint32_t sw128(int r, int c16, uint32_t half_bytes) {
    return (uint32_t)(c16 >> 3) * half_bytes + (uint32_t)r * 128u + ((uint32_t)((c16 & 7) ^ (r & 7)) << 4);
}

template <int NS>
__global__ void __launch_bounds__(THREADS, Cfg<NS>::CTAS) sparse_gather_tc(const Params p) {
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
            mbar_init(smem_u32(&bars->kv_full[s]), PROD_THREADS);
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
        const int half = lane >> 4, part = lane & 15;
        int seq = 0, item_n = 0;
        bool ok = true;
        for (long long it_ = blockIdx.x; ok && it_ < p.n_items; it_ += stride, ++item_n) {
            const Item it = item_of(p, it_);
            const int32_t *list = list_of(p, it);
            const __nv_bfloat16 *kb = p.k + ((size_t)it.b * p.Lkv * p.Hkv + it.g) * 128;
            const __nv_bfloat16 *vb = p.v + ((size_t)it.b * p.Lkv * p.Hkv + it.g) * 128;
            const size_t qrow = ((size_t)it.b * p.Lq + it.i) * p.Hq + (size_t)it.g * p.G;
            // keys of this lane's four rows (lane + 32 u): ka of the latest K chunk
            // jk, kp of chunk jk - 1, kn of chunk jk + 1 (loaded one K tile ahead,
            // while the warp waits for a free slot)
            int jk = -1, ka[4], kp[4], kn[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                ka[u] = kp[u] = -1;
                kn[u] = chunk_key(p, list, it, 0, 32 * u + lane, true);
            }
            for (int t = 0; t < 2 * it.n; ++t) {
                // production order: K0, then (K_{j+1}, V_j) pairs, then the last V
                int j, is_v;
                if (t == 0) { j = 0; is_v = 0; }
                else if (t == 2 * it.n - 1) { j = it.n - 1; is_v = 1; }
                else { is_v = (t & 1) == 0; j = is_v ? (t - 2) / 2 : (t + 1) / 2; }
                int key[4];
                if (!is_v) {
                    jk = j;
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        kp[u] = ka[u];
                        ka[u] = kn[u];
                        key[u] = ka[u];
                    }
                    if (j + 1 < it.n) {
#pragma unroll
                        for (int u = 0; u < 4; ++u) kn[u] = chunk_key(p, list, it, j + 1, 32 * u + lane, true);
                    }
                } else {                   // the item's last V follows its own K; else V_{jk-1}
#pragma unroll
                    for (int u = 0; u < 4; ++u) key[u] = j == jk ? ka[u] : kp[u];
                }
                const int slot = seq % NS, use = seq / NS;
                // every lane takes part in the shuffles below: the warp agrees on the wait
                if (!(ok = __all_sync(0xffffffffu, wait_sleep(smem_u32(&bars->kv_empty[slot]), (use & 1) ^ 1,
                                                              p.wait_ns, abort))))
                    break;
                const uint32_t tb = smem_u32(ring + slot * TILE_B);
                if (t == 0) {
                    // the item's query rows travel in the same copy group as K0: the
                    // previous item's last S = K Q^T must have finished reading Q
                    if (!(ok = __all_sync(0xffffffffu, wait_sleep(smem_u32(&bars->q_empty), (item_n & 1) ^ 1,
                                                                  p.wait_ns, abort))))
                        break;
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const int e = lane * 8 + u;            // 0..255: head e/16, chunk e%16
                        const int h = e >> 4, c16 = e & 15;
                        const bool val = h < p.G;
                        cp_async16(smem_u32(sq) + sw128(h, c16, QP_HALF),
                                   p.q + (val ? (qrow + h) * 128 + c16 * 8 : 0), val);
                    }
                }
                const __nv_bfloat16 *src = (is_v ? vb : kb) + part * 8;
                const uint32_t dbase = tb + (uint32_t)(part >> 3) * HALF_B;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
#pragma unroll
                    for (int r2 = 0; r2 < 16; ++r2) {
                        // two rows per instruction: lanes 0-15 row 32 u + 2 r2, lanes 16-31 the next
                        const int rl = 2 * r2 + half, row = 32 * u + rl;
                        const int kr = __shfl_sync(0xffffffffu, key[u], rl);
                        const bool val = kr >= 0;
                        cp_async16(dbase + (uint32_t)row * 128u + ((uint32_t)((part & 7) ^ (row & 7)) << 4),
                                   src + (val ? (size_t)kr * p.Hkv * 128 : 0), val);
                    }
                }
                // the slot's full barrier counts this thread's arrival once all its
                // copies so far have landed
                cp_async_arrive_noinc(smem_u32(&bars->kv_full[slot]));
                ++seq;
            }
        }
        cp_async_wait_all();   // no copy of ours is still in flight when the CTA exits
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
                    fence_proxy_async_smem();   // copies landed through the generic proxy; the MMA reads async
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
                    const int c = gc + j, tv = T + seq_v(j, it.n), slot = tv % NS;
                    if (!(ok = wait_sleep(smem_u32(&bars->kv_full[slot]), (tv / NS) & 1, p.wait_ns, abort))) break;
                    fence_proxy_async_smem();
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
            int key_next = chunk_key(p, list, it, 0, t, false);
            for (int j = 0; j < it.n; ++j) {
                const int c = gc + j;
                if (wg_any(bad || *abort)) break;
                const bool glob = j < it.n_g;
                const bool first = j == 0 || j == it.n_g;
                if (j == it.n_g) {
#pragma unroll
                    for (int h = 0; h < NH; ++h) m[h] = -INFINITY;   // the window branch starts afresh
                }
                const bool valid = key_next >= 0;
                if (j + 1 < it.n) key_next = chunk_key(p, list, it, j + 1, t, false);
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
template <int NS>
cudaError_t launch_ns(const gtc::Params &p0, cudaStream_t st) {
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
    sparse_gather_tc<NS><<<(unsigned)grid, THREADS, Cfg<NS>::kSmem, st>>>(p0);
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
