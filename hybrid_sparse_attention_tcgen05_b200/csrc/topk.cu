// Per-row top-k over importance scores by radix selection on the fp32 bit
// patterns (write-up section 2.2: the global branch attends over the full
// layer's TopK indices; baidu article "Top-K selection").
//
// Importance scores are sums of probabilities, so they are >= 0: the sign
// bit is 0 and the 32-bit patterns, read as unsigned integers, sort in the
// same order as the values.  With M the row's largest pattern and m its
// smallest, every key has y = M - x in [0, M - m] < 2^L (L = bit length of
// M - m), and the k largest scores are the k smallest y.  Digit passes over
// y of at most 11 bits, most significant first (ceil(L / 11) passes: two for
// the nearly flat rows of attention, whose keys share the exponent and the
// leading mantissa bits), find the exact y_T of the k-th key and how many
// keys equal to it must be taken; an ordered compaction then emits every key
// above T = M - y_T and the lowest-indexed keys equal to T, which is exactly
// "largest scores, ties to the lower index", already in ascending key order.
// Integer work only: the result is exact and deterministic.
//
// Three kernels compute this same select:
//   topk_warp_kernel     one warp per (row, KV head), for launches with many
//                        rows (prefill);
//   topk_sampled_kernel  one 512-thread CTA per row that brackets the k-th key
//                        from a sample and settles it in one pass over the row
//                        (launches with few rows: decode), falling back in
//                        place to the exact CTA select below;
//   topk_radix_kernel    the exact CTA select on its own (when forced, or for
//                        few rows too long for the sampled kernel's shared
//                        memory).
// In the CTA select the max / min pass copies the row into shared memory
// when it is short enough to keep four CTAs on an SM; longer rows are
// re-read from global memory (L2) by every pass.  Keys are read four at a
// time (16 bytes); histogram bins take plain shared atomics.
#include <cstdlib>
#include <cstring>

#include "common.cuh"
#include "internal.h"

namespace hs {
namespace {

constexpr int NT = 512;
constexpr int NW = NT / 32;
constexpr unsigned int FULL = 0xffffffffu;
constexpr int kDigitBits = 11;
constexpr int kBins = 1 << kDigitBits;

// Rows of up to kSmemKeys keys are cached in shared memory (39 KB + 16 KB of
// histograms per CTA at the limit: four CTAs per SM).
constexpr int kSmemKeys = 9984;

// Launches with at least this many (row, KV head) items take the one-warp-
// per-row kernel; fewer, longer rows (decode) take one CTA per row.
constexpr long long kWarpMinItems = 4096;

// Keys of row i of batch b: the causal prefix of its cache, whose length is
// kv_len[b] when given (clamped to [1, Lkv]; the decode kernels report values
// outside it), else Lkv.
__device__ __forceinline__ int row_keys(const int32_t *kv_len, int b, int Lq, int Lkv, int i) {
    int L = Lkv;
    if (kv_len != nullptr) L = min(max(__ldg(kv_len + b), 1), Lkv);
    return L - Lq + i + 1;
}

struct TopkShared {
    unsigned int h[2][kBins];      // digit histograms (passes alternate)
    unsigned int wa[NW], wb[NW];   // per-warp partials
    unsigned int digit, remaining;
};

// Keys 4g .. 4g+3 of the row (all four inside it).
template <bool SMEM>
__device__ __forceinline__ uint4 load4(const unsigned int *u, int g, bool aligned) {
    if (SMEM) return reinterpret_cast<const uint4 *>(u)[g];
    if (aligned) return __ldg(reinterpret_cast<const uint4 *>(u) + g);
    const unsigned int *p = u + 4 * g;
    return make_uint4(__ldg(p), __ldg(p + 1), __ldg(p + 2), __ldg(p + 3));
}

template <bool SMEM>
__device__ __forceinline__ unsigned int load1(const unsigned int *u, int j) {
    return SMEM ? u[j] : __ldg(u + j);
}

// One digit pass: key x takes part when the already fixed high bits of
// y = M - x equal `pre` (y >> hs_ == pre; hs_ = 32: none fixed yet), and
// falls into bin (y >> s) & nbm1.
struct Digit {
    unsigned int M, pre;
    int hs_, s;
    unsigned int nbm1;
    __device__ __forceinline__ bool take(unsigned int x, unsigned int &bin) const {
        const unsigned int y = M - x;
        bin = (y >> s) & nbm1;
        return hs_ >= 32 || (y >> hs_) == pre;
    }
};

template <bool SMEM>
__device__ __forceinline__ void hist_pass(unsigned int *hist, const unsigned int *u, int n, bool aligned,
                                          const Digit &d, int tid) {
    const int n4 = n >> 2;
    for (int g = tid; g < n4; g += NT) {
        const uint4 v = load4<SMEM>(u, g, aligned);
        unsigned int b0, b1, b2, b3;
        const bool t0 = d.take(v.x, b0), t1 = d.take(v.y, b1), t2 = d.take(v.z, b2), t3 = d.take(v.w, b3);
        if (t0) atomicAdd(&hist[b0], 1u);
        if (t1) atomicAdd(&hist[b1], 1u);
        if (t2) atomicAdd(&hist[b2], 1u);
        if (t3) atomicAdd(&hist[b3], 1u);
    }
    if (tid < n - 4 * n4) {
        unsigned int bb;
        if (d.take(load1<SMEM>(u, 4 * n4 + tid), bb)) atomicAdd(&hist[bb], 1u);
    }
}

// Find the bin (ascending: smallest y first) in which the running count of
// keys first reaches `remaining`; thread t owns bins per*t .. per*t+per-1.
// Writes the bin and the count still needed inside it to sh.digit and
// sh.remaining; the caller synchronises before reading them.
__device__ __forceinline__ void find_bin(TopkShared &sh, const unsigned int *hist, unsigned int nb,
                                         unsigned int remaining, int tid) {
    const int lane = tid & 31, warp = tid >> 5;
    const int per = nb >= (unsigned)NT ? (int)nb / NT : 1;
    unsigned int c[kBins / NT];
    unsigned int tot = 0;
#pragma unroll
    for (int k = 0; k < kBins / NT; ++k) {
        const unsigned int bin = (unsigned)(per * tid + k);
        c[k] = (k < per && bin < nb) ? hist[bin] : 0u;
        tot += c[k];
    }
    unsigned int incl = tot;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const unsigned int y = __shfl_up_sync(FULL, incl, off);
        if (lane >= off) incl += y;
    }
    if (lane == 31) sh.wa[warp] = incl;
    __syncthreads();
    const unsigned int woff = __reduce_add_sync(FULL, lane < warp ? sh.wa[lane] : 0u);
    const unsigned int excl = woff + incl - tot;
    if (excl < remaining && remaining <= excl + tot) {
        unsigned int cum = excl;
#pragma unroll
        for (int k = 0; k < kBins / NT; ++k) {
            if (k < per && cum + c[k] >= remaining) {
                sh.digit = (unsigned)(per * tid + k);
                sh.remaining = remaining - cum;
                break;
            }
            cum += c[k];
        }
    }
}

// The exact select of one row by one CTA of NT threads (n > topk): a max /
// min pass (copying the row to row_cache when SMEM), digit passes, and the
// ordered compaction into o.  Every thread of the CTA calls it.
template <bool SMEM>
__device__ __forceinline__ void radix_select_row(TopkShared &sh, int *cnt_gt, int *cnt_eq, const unsigned int *gu,
                                                 unsigned int *row_cache, int n, int topk, int32_t *o, int tid) {
    const int lane = tid & 31, warp = tid >> 5;
    const bool aligned = (reinterpret_cast<uintptr_t>(gu) & 15u) == 0;
    for (int t = tid; t < 2 * kBins; t += NT) (&sh.h[0][0])[t] = 0u;

    // max / min bit pattern of the row (and its copy into shared memory)
    unsigned int mx = 0u, mn = FULL;
    const int n4 = n >> 2;
    if (aligned) {
        for (int q = tid; q < n4; q += NT) {
            const uint4 v = __ldg(reinterpret_cast<const uint4 *>(gu) + q);
            if (SMEM) reinterpret_cast<uint4 *>(row_cache)[q] = v;
            mx = max(mx, max(max(v.x, v.y), max(v.z, v.w)));
            mn = min(mn, min(min(v.x, v.y), min(v.z, v.w)));
        }
    } else {
        for (int j = tid; j < 4 * n4; j += NT) {
            const unsigned int x = __ldg(gu + j);
            if (SMEM) row_cache[j] = x;
            mx = max(mx, x);
            mn = min(mn, x);
        }
    }
    if (tid < n - 4 * n4) {
        const unsigned int x = __ldg(gu + 4 * n4 + tid);
        if (SMEM) row_cache[4 * n4 + tid] = x;
        mx = max(mx, x);
        mn = min(mn, x);
    }
    mx = __reduce_max_sync(FULL, mx);
    mn = __reduce_min_sync(FULL, mn);
    if (lane == 0) {
        sh.wa[warp] = mx;
        sh.wb[warp] = mn;
    }
    __syncthreads();
    const unsigned int M = __reduce_max_sync(FULL, lane < NW ? sh.wa[lane] : 0u);
    const unsigned int range = M - __reduce_min_sync(FULL, lane < NW ? sh.wb[lane] : FULL);
    const int L = range ? 32 - __clz(range) : 0;

    const unsigned int *u = SMEM ? row_cache : gu;
    const bool al = SMEM || aligned;

    // digit passes over y = M - x, most significant first: after the pass
    // covering bits [s, top), `pre` = y >> s of the k-th key
    unsigned int pre = 0u, remaining = (unsigned int)topk;
    int hs_ = 32, top = L, buf = 0;
    while (top > 0) {
        const int s = max(0, top - kDigitBits);
        const unsigned int nb = 1u << (top - s);
        const Digit d{M, pre, hs_, s, nb - 1u};
        hist_pass<SMEM>(sh.h[buf], u, n, al, d, tid);
        __syncthreads();
        find_bin(sh, sh.h[buf], nb, remaining, tid);
        __syncthreads();
        pre = (pre << (top - s)) | sh.digit;
        remaining = sh.remaining;
        for (int t = tid; t < (int)nb; t += NT) sh.h[buf][t] = 0u;   // read by nobody until two passes on
        hs_ = s;
        top = s;
        buf ^= 1;
    }
    const unsigned int T = M - pre;   // bit pattern of the k-th largest score
    const int rem = (int)remaining;   // keys equal to T to take (lowest indices first)

    // Ordered compaction: warp w owns the contiguous key range
    // [w*seg, (w+1)*seg), 128 keys (4 per lane) per step.  (A negative
    // input, which importance scores never are, could only make more keys
    // compare above T; the `at < topk` guard keeps writes in bounds.)
    const int seg = ((n + NW - 1) / NW + 127) & ~127;
    const int j_lo = warp * seg, j_hi = min(n, j_lo + seg);
    int cg = 0, ce = 0;
    for (int j = j_lo + 4 * lane; j < j_hi; j += 128) {
        if (j + 4 <= j_hi) {
            const uint4 v = load4<SMEM>(u, j >> 2, al);
            cg += (v.x > T) + (v.y > T) + (v.z > T) + (v.w > T);
            ce += (v.x == T) + (v.y == T) + (v.z == T) + (v.w == T);
        } else {
            for (int c = j; c < j_hi; ++c) {
                const unsigned int x = load1<SMEM>(u, c);
                cg += x > T;
                ce += x == T;
            }
        }
    }
    cg = (int)__reduce_add_sync(FULL, (unsigned int)cg);
    ce = (int)__reduce_add_sync(FULL, (unsigned int)ce);
    if (lane == 0) {
        cnt_gt[warp] = cg;
        cnt_eq[warp] = ce;
    }
    __syncthreads();
    int gt_base = (int)__reduce_add_sync(FULL, lane < warp ? (unsigned int)cnt_gt[lane] : 0u);
    int eq_base = (int)__reduce_add_sync(FULL, lane < warp ? (unsigned int)cnt_eq[lane] : 0u);
    for (int j0 = j_lo; j0 < j_hi; j0 += 128) {
        const int j = j0 + 4 * lane;
        const int nv = max(0, min(4, j_hi - j));
        unsigned int xv[4] = {0u, 0u, 0u, 0u};
        if (nv == 4) {
            const uint4 v = load4<SMEM>(u, j >> 2, al);
            xv[0] = v.x; xv[1] = v.y; xv[2] = v.z; xv[3] = v.w;
        } else {
#pragma unroll
            for (int c = 0; c < 4; ++c)
                if (c < nv) xv[c] = load1<SMEM>(u, j + c);
        }
        bool isg[4], ise[4];
        int ng = 0, ne = 0;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            isg[c] = c < nv && xv[c] > T;
            ise[c] = c < nv && xv[c] == T;
            ng += isg[c];
            ne += ise[c];
        }
        // exclusive lane prefix of (gt, eq) counts, packed 16:16 (<= 128 each)
        const unsigned int packed = ((unsigned int)ng << 16) | (unsigned int)ne;
        unsigned int incl = packed;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const unsigned int y = __shfl_up_sync(FULL, incl, off);
            if (lane >= off) incl += y;
        }
        const unsigned int tot = __shfl_sync(FULL, incl, 31);
        const unsigned int excl = incl - packed;
        int gb = gt_base + (int)(excl >> 16), eb = eq_base + (int)(excl & 0xffffu);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            if (isg[c] || (ise[c] && eb < rem)) {
                const int at = gb + min(eb, rem);
                if (at < topk) o[at] = j + c;
            }
            gb += isg[c];
            eb += ise[c];
        }
        gt_base += (int)(tot >> 16);
        eq_base += (int)(tot & 0xffffu);
    }
}

template <bool SMEM>
__global__ void __launch_bounds__(NT, 4)
topk_radix_kernel(const float *__restrict__ scores, long long ld, int Lq, int Lkv, int Hkv, int row_begin,
                  int row_count, int r_lo, int topk, int32_t *__restrict__ idx, const int32_t *__restrict__ kv_len) {
    extern __shared__ __align__(16) unsigned int row_cache[];
    __shared__ TopkShared sh;
    __shared__ int cnt_gt[NW], cnt_eq[NW];

    const int r = r_lo + blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x;
    const int i = row_begin + r;
    const int n = row_keys(kv_len, b, Lq, Lkv, i);
    const unsigned int *gu =
        reinterpret_cast<const unsigned int *>(scores + (((size_t)b * Hkv + g) * row_count + r) * ld);
    int32_t *o = idx + (((size_t)b * Hkv + g) * Lq + i) * (size_t)topk;

    if (n <= topk) {
        for (int t = tid; t < topk; t += NT) o[t] = t < n ? t : -1;
        return;
    }
    radix_select_row<SMEM>(sh, cnt_gt, cnt_eq, gu, row_cache, n, topk, o, tid);
}

// ------------------------------------------------------------ one warp per row
//
// For launches with many rows (prefill): one warp owns one (row, KV head)
// with a private 1024-bin histogram in shared memory, so the per-row fixed
// work (histogram scans, clears) is one warp's and no block barrier is
// needed; the compaction runs once over the row in key order (ballots give
// each selected key its output slot), with no separate counting pass.  The
// row is re-read from global memory (L1 / L2) by each of its passes: three
// (sampled first digit, second digit, compaction), or two for long rows,
// whose compaction also settles the k-th key's bin (select_with_candidates).

constexpr int WK_WARPS = 8;
constexpr int WK_BITS = 10;
constexpr int WK_BINS = 1 << WK_BITS;

template <bool AL>
__device__ __forceinline__ uint4 ld4(const unsigned int *u, int g) {
    if (AL) return __ldg(reinterpret_cast<const uint4 *>(u) + g);
    const unsigned int *p = u + 4 * g;
    return make_uint4(__ldg(p), __ldg(p + 1), __ldg(p + 2), __ldg(p + 3));
}

__device__ __forceinline__ void wk_zero(unsigned int *h, int lane) {
#pragma unroll
    for (int k = 0; k < WK_BINS / 128; ++k)
        reinterpret_cast<uint4 *>(h)[k * 32 + lane] = make_uint4(0u, 0u, 0u, 0u);
}

// Smallest bin b (ascending) whose running count reaches `remaining`;
// returns b, the count still needed inside it and the bin's own count.
__device__ __forceinline__ unsigned int wk_find(const unsigned int *h, unsigned int remaining, int lane,
                                                unsigned int &rem_out, unsigned int &cnt_out) {
    // lane l sums bins [32l, 32l+32), reading them in a rotated order so the
    // 32 lanes hit 32 different banks
    unsigned int tot = 0;
#pragma unroll 8
    for (int k = 0; k < 32; ++k) tot += h[32 * lane + ((k + lane) & 31)];
    unsigned int incl = tot;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const unsigned int y = __shfl_up_sync(FULL, incl, off);
        if (lane >= off) incl += y;
    }
    const int c = max(0, __ffs(__ballot_sync(FULL, incl >= remaining)) - 1);   // chunk holding the k-th key
    const unsigned int before = __shfl_sync(FULL, incl - tot, c);
    const unsigned int v = h[32 * c + lane];
    unsigned int in2 = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const unsigned int y = __shfl_up_sync(FULL, in2, off);
        if (lane >= off) in2 += y;
    }
    const int e = max(0, __ffs(__ballot_sync(FULL, before + in2 >= remaining)) - 1);
    rem_out = remaining - before - __shfl_sync(FULL, in2 - v, e);
    cnt_out = __shfl_sync(FULL, v, e);
    return (unsigned int)(32 * c + e);
}

// Once a digit pass has found the k-th key's bin, the keys above the bin
// ("definites") are final and the few keys inside it ("candidates") can be
// ranked among themselves: one pass over the row writes the definites in key
// order, as the plain compaction does, and lists the candidates in the
// warp's histogram space with their bits of y below the bin and the number
// of definites before them.  The `remaining` candidates with the smallest
// such bits (ties to the lower key) are then merged into the index list.
// This replaces a second digit pass and the compaction (two passes over the
// row) with one.
constexpr int WK_CAND = WK_BINS / 2;     // key index + packed word each
constexpr int WK_CAND_SHIFT = 19;        // bits of y below the bin kept per candidate
constexpr int WK_DEF_BITS = 13;          // definites before it (topk < 8192)
constexpr int WK_MOVE = 8;               // 32-entry chunks per batch of the final merge
constexpr int WK_CAND_MIN_ROW = 6;       // rows of at least this many times topk keys (the merge costs
                                         // about one pass over topk entries)
static_assert(WK_CAND_SHIFT + WK_DEF_BITS == 32, "candidate word");

template <bool AL>
__device__ __forceinline__ void select_with_candidates(const unsigned int *u, int n4, int nt, unsigned int M,
                                                       unsigned int pre, int sh, unsigned int R, int topk,
                                                       unsigned int *h, int32_t *o, uint32_t *mrow, int W,
                                                       int lane) {
    unsigned int *ck = h, *cw = h + WK_CAND;
    const unsigned int lt = (1u << lane) - 1u, lowm = (1u << sh) - 1u;
    int base = 0, cb = 0;
    for (int g0 = 0; g0 < n4 + 1; g0 += 32) {   // the extra step carries the tail keys
        const int g = g0 + lane;
        unsigned int x[4];
        bool ok[4];
        if (g < n4) {
            const uint4 v = ld4<AL>(u, g);
            x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
            ok[0] = ok[1] = ok[2] = ok[3] = true;
        } else {
            const int tail0 = 4 * n4 + 4 * (g - n4);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                ok[c] = g == n4 && c < nt;
                x[c] = ok[c] ? __ldg(u + tail0 + c) : 0u;
            }
        }
        // keys above M (a sampled maximum) lie above the bin
        bool df[4], cd[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const unsigned int hi = (M - x[c]) >> sh;
            df[c] = ok[c] && (x[c] > M || hi < pre);
            cd[c] = ok[c] && x[c] <= M && hi == pre;
        }
        int before = 0, tot = 0;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const unsigned int bb = __ballot_sync(FULL, df[c]);
            before += __popc(bb & lt);
            tot += __popc(bb);
        }
        int cbef = 0, ctot = 0;
        const bool any_cd = __any_sync(FULL, cd[0] || cd[1] || cd[2] || cd[3]);
        if (any_cd) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const unsigned int bb = __ballot_sync(FULL, cd[c]);
                cbef += __popc(bb & lt);
                ctot += __popc(bb);
            }
        }
        int at = base + before, ca = cb + cbef;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            if (df[c] && at < topk) o[at] = 4 * g + c;
            if (cd[c] && ca < WK_CAND) {
                ck[ca] = (unsigned int)(4 * g + c);
                cw[ca] = (((M - x[c]) & lowm) << WK_DEF_BITS) | (unsigned int)min(at, topk);
            }
            at += df[c];
            ca += cd[c];
        }
        base += tot;
        cb += ctot;
        if (mrow) {   // definites' bits; the chosen candidates' are OR-ed in below
            unsigned int wd = ((df[0] ? 1u : 0u) | (df[1] ? 2u : 0u) | (df[2] ? 4u : 0u) | (df[3] ? 8u : 0u))
                              << (4 * (lane & 7));
            wd |= __shfl_xor_sync(FULL, wd, 1);
            wd |= __shfl_xor_sync(FULL, wd, 2);
            wd |= __shfl_xor_sync(FULL, wd, 4);
            const int w = g0 / 8 + (lane >> 3);
            if ((lane & 7) == 0 && w < W) mrow[w] = wd;
        }
    }
    if (mrow)   // words past the row's causal end
        for (int w = 4 * ((n4 + 32) / 32) + lane; w < W; w += 32) mrow[w] = 0u;
    __syncwarp();

    // the R-th smallest candidate bits, bit by bit from the top: `ans` keeps
    // the largest value with fewer than R candidates below it
    const int C = min(cb, WK_CAND);
    unsigned int ans = 0;
    for (int bit = sh - 1; bit >= 0; --bit) {
        const unsigned int t = ans | (1u << bit);
        unsigned int c = 0;
        for (int j = lane; j < C; j += 32) c += (cw[j] >> WK_DEF_BITS) < t;
        if (__reduce_add_sync(FULL, c) < R) ans = t;
    }
    unsigned int nl = 0;
    for (int j = lane; j < C; j += 32) nl += (cw[j] >> WK_DEF_BITS) < ans;
    const int take_eq = (int)R - (int)__reduce_add_sync(FULL, nl);

    // keep the chosen candidates (in key order, in place): key, definites before it
    int sb = 0, eb = 0;
    for (int j0 = 0; j0 < C; j0 += 32) {
        const int j = j0 + lane;
        const bool v = j < C;
        const unsigned int key = v ? ck[j] : 0u, wv = v ? cw[j] : 0u;
        const unsigned int low = wv >> WK_DEF_BITS;
        const bool eq = v && low == ans;
        const unsigned int eqb = __ballot_sync(FULL, eq);
        const bool sel = v && (low < ans || (eq && eb + __popc(eqb & lt) < take_eq));
        eb += __popc(eqb);
        const unsigned int sbb = __ballot_sync(FULL, sel);
        __syncwarp();
        if (sel) {
            const int p = sb + __popc(sbb & lt);
            ck[p] = key;
            cw[p] = wv & ((1u << WK_DEF_BITS) - 1u);
            if (mrow) atomicOr(mrow + (key >> 5), 1u << (key & 31u));
        }
        sb += __popc(sbb);
        __syncwarp();
    }

    // definite d moves up by the number of chosen candidates with at most d
    // definites before them; from the top down, WK_MOVE chunks of 32 read
    // before any is written, so no entry is overwritten before it is read
    const int D = min(base, topk);
    int jh = sb;
    for (int t0 = (D - 1) & ~31; t0 >= 0 && jh > 0; t0 -= 32 * WK_MOVE) {
        int key[WK_MOVE], rs[WK_MOVE];
#pragma unroll
        for (int q = 0; q < WK_MOVE; ++q) {
            const int d0 = t0 - 32 * q, d = d0 + lane;
            rs[q] = 0;
            key[q] = 0;
            if (d0 < 0 || jh == 0) continue;
            while (jh > 0 && (int)cw[jh - 1] > d0 + 31) --jh;
            int k = jh, cnt = 0;
            while (k > 0) {
                const int db = (int)cw[k - 1];
                if (db < d0) break;
                cnt += db <= d;
                --k;
            }
            rs[q] = d < D ? k + cnt : 0;
            if (rs[q] > 0) key[q] = __ldcg(o + d);
            jh = k;
        }
        __syncwarp();
#pragma unroll
        for (int q = 0; q < WK_MOVE; ++q) {
            const int d = t0 - 32 * q + lane;
            if (rs[q] > 0 && d + rs[q] < topk) o[d + rs[q]] = key[q];
        }
    }
    __syncwarp();
    for (int j = lane; j < sb; j += 32) {
        const int p = j + (int)cw[j];
        if (p < topk) o[p] = (int)ck[j];
    }
}

template <bool AL>
__global__ void __launch_bounds__(WK_WARPS * 32, 5)
topk_warp_kernel(const float *__restrict__ scores, long long ld, int Lq, int Lkv, int Hkv, int row_begin,
                 int row_count, int topk, long long n_items, int32_t *__restrict__ idx, uint32_t *__restrict__ mask,
                 int W, const int32_t *__restrict__ kv_len) {
    __shared__ __align__(16) unsigned int hist_all[WK_WARPS][WK_BINS];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long item = (long long)blockIdx.x * WK_WARPS + warp;
    if (item >= n_items) return;
    // longest rows first; (batch, KV head) slowest
    const int r = row_count - 1 - (int)(item % row_count);
    const long long bg = item / row_count;
    const int i = row_begin + r;
    const int n = row_keys(kv_len, (int)(bg / Hkv), Lq, Lkv, i);
    const unsigned int *u = reinterpret_cast<const unsigned int *>(scores + ((size_t)bg * row_count + r) * ld);
    int32_t *o = idx + ((size_t)bg * Lq + i) * (size_t)topk;
    uint32_t *mrow = mask ? mask + ((size_t)bg * Lq + i) * (size_t)W : nullptr;
    if (n <= topk) {
        for (int t = lane; t < topk; t += 32) o[t] = t < n ? t : -1;
        if (mrow)
            for (int w = lane; w < W; w += 32) {
                const int lo = 32 * w;
                mrow[w] = lo + 32 <= n ? FULL : (lo < n ? (1u << (n - lo)) - 1u : 0u);
            }
        return;
    }
    unsigned int *h = hist_all[warp];
    wk_zero(h, lane);
    __syncwarp();

    const int n4 = n >> 2, nt = n - 4 * n4;
    const unsigned int xt = lane < nt ? __ldg(u + 4 * n4 + lane) : 0u;   // tail keys (< 4)
    unsigned int M = 0u, pre = 0u, remaining = (unsigned int)topk, cnt_eq = (unsigned int)n;
    int hs_ = 32, top = -1;
    if (n >= 1024) {
        // First digit without a separate max / min pass: the digit range comes
        // from 8 sampled 32-key lines (keys outside it are clamped into the
        // edge bins) while the same pass takes the row's exact max and min.
        // Only if the k-th key falls in a clamped edge bin is the pass redone
        // over the exact range.
        unsigned int xs[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) xs[q] = __ldg(u + (int)(((long long)(n - 32) * q) / 7) + lane);
        unsigned int smx = xs[0], smn = xs[0];
#pragma unroll
        for (int q = 1; q < 8; ++q) {
            smx = max(smx, xs[q]);
            smn = min(smn, xs[q]);
        }
        const unsigned int Ms = __reduce_max_sync(FULL, smx), ms = __reduce_min_sync(FULL, smn);
        if (Ms > ms) {
            const int tp = 32 - __clz(Ms - ms), s = max(0, tp - WK_BITS);
            const unsigned int nbm1 = (1u << (tp - s)) - 1u;
            unsigned int mx = lane < nt ? xt : 0u, mn = lane < nt ? xt : FULL;
            auto bin = [&](unsigned int x) { return x > Ms ? 0u : min(nbm1, (Ms - x) >> s); };
            for (int g = lane; g < n4; g += 32) {
                const uint4 v = ld4<AL>(u, g);
                mx = max(mx, max(max(v.x, v.y), max(v.z, v.w)));
                mn = min(mn, min(min(v.x, v.y), min(v.z, v.w)));
                atomicAdd(&h[bin(v.x)], 1u);
                atomicAdd(&h[bin(v.y)], 1u);
                atomicAdd(&h[bin(v.z)], 1u);
                atomicAdd(&h[bin(v.w)], 1u);
            }
            if (lane < nt) atomicAdd(&h[bin(xt)], 1u);
            const unsigned int Mx = __reduce_max_sync(FULL, mx), Mn = __reduce_min_sync(FULL, mn);
            __syncwarp();
            unsigned int rem2, cnt;
            const unsigned int dig = wk_find(h, remaining, lane, rem2, cnt);
            __syncwarp();
            wk_zero(h, lane);
            __syncwarp();
            const bool clamped = (dig == 0u && Mx > Ms) || (dig == nbm1 && ((Ms - Mn) >> s) > nbm1);
            if (!clamped) {
                M = Ms;
                pre = dig;
                remaining = rem2;
                cnt_eq = cnt;
                hs_ = s;
                top = s;
            } else {
                M = Mx;
                top = Mx > Mn ? 32 - __clz(Mx - Mn) : 0;
            }
        }
    }
    if (top < 0) {   // short or constant-looking sample: exact max / min first
        unsigned int mx = lane < nt ? xt : 0u, mn = lane < nt ? xt : FULL;
        for (int g = lane; g < n4; g += 32) {
            const uint4 v = ld4<AL>(u, g);
            mx = max(mx, max(max(v.x, v.y), max(v.z, v.w)));
            mn = min(mn, min(min(v.x, v.y), min(v.z, v.w)));
        }
        M = __reduce_max_sync(FULL, mx);
        const unsigned int range = M - __reduce_min_sync(FULL, mn);
        top = range ? 32 - __clz(range) : 0;
        __syncwarp();
    }

    while (top > 0) {
        // After a digit pass that left few keys in the k-th key's bin, settle
        // the rest from those keys alone (one more pass over the row, not two)
        if (hs_ < 32 && top <= WK_CAND_SHIFT && cnt_eq <= (unsigned int)WK_CAND && topk < (1 << WK_DEF_BITS) &&
            n >= WK_CAND_MIN_ROW * topk) {
            select_with_candidates<AL>(u, n4, nt, M, pre, hs_, remaining, topk, h, o, mrow, W, lane);
            return;
        }
        const int s = max(0, top - WK_BITS);
        const unsigned int msk = (1u << (top - s)) - 1u;
        if (hs_ >= 32) {
            for (int g = lane; g < n4; g += 32) {
                const uint4 v = ld4<AL>(u, g);
                atomicAdd(&h[(M - v.x) >> s], 1u);
                atomicAdd(&h[(M - v.y) >> s], 1u);
                atomicAdd(&h[(M - v.z) >> s], 1u);
                atomicAdd(&h[(M - v.w) >> s], 1u);
            }
            if (lane < nt) atomicAdd(&h[(M - xt) >> s], 1u);
        } else {
            for (int g = lane; g < n4; g += 32) {
                const uint4 v = ld4<AL>(u, g);
                const unsigned int y0 = M - v.x, y1 = M - v.y, y2 = M - v.z, y3 = M - v.w;
                if ((y0 >> hs_) == pre) atomicAdd(&h[(y0 >> s) & msk], 1u);
                if ((y1 >> hs_) == pre) atomicAdd(&h[(y1 >> s) & msk], 1u);
                if ((y2 >> hs_) == pre) atomicAdd(&h[(y2 >> s) & msk], 1u);
                if ((y3 >> hs_) == pre) atomicAdd(&h[(y3 >> s) & msk], 1u);
            }
            if (lane < nt && ((M - xt) >> hs_) == pre) atomicAdd(&h[((M - xt) >> s) & msk], 1u);
        }
        __syncwarp();
        unsigned int rem2, cnt;
        const unsigned int dig = wk_find(h, remaining, lane, rem2, cnt);
        __syncwarp();
        wk_zero(h, lane);
        __syncwarp();
        pre = (pre << (top - s)) | dig;
        remaining = rem2;
        cnt_eq = cnt;
        hs_ = s;
        top = s;
    }
    const unsigned int T = M - pre;            // bit pattern of the k-th largest score
    const bool take_all = remaining == cnt_eq; // every key equal to T is taken: no tie ranks needed
    const unsigned int lt = (1u << lane) - 1u;
    int base = 0, eq_base = 0;
    for (int g0 = 0; g0 < n4 + 1; g0 += 32) {   // the extra step carries the tail keys
        const int g = g0 + lane;
        unsigned int x[4];
        bool ok[4];
        if (g < n4) {
            const uint4 v = ld4<AL>(u, g);
            x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
            ok[0] = ok[1] = ok[2] = ok[3] = true;
        } else {
            const int tail0 = 4 * n4 + 4 * (g - n4);   // tail keys sit in group n4 only
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                ok[c] = g == n4 && c < nt;
                x[c] = ok[c] ? __ldg(u + tail0 + c) : 0u;
            }
        }
        bool sel[4];
        if (take_all) {
#pragma unroll
            for (int c = 0; c < 4; ++c) sel[c] = ok[c] && x[c] >= T;
        } else {
            bool eq[4];
            int eq_lane = 0;
            unsigned int eb_all = 0;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                eq[c] = ok[c] && x[c] == T;
                const unsigned int bb = __ballot_sync(FULL, eq[c]);
                eq_lane += __popc(bb & lt);
                eb_all += __popc(bb);
            }
            int er = eq_base + eq_lane;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                sel[c] = (ok[c] && x[c] > T) || (eq[c] && er < (int)remaining);
                er += eq[c];
            }
            eq_base += (int)eb_all;
        }
        int before = 0, tot = 0;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const unsigned int bb = __ballot_sync(FULL, sel[c]);
            before += __popc(bb & lt);
            tot += __popc(bb);
        }
        int at = base + before;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            if (sel[c] && at < topk) o[at] = 4 * g + c;
            at += sel[c];
        }
        base += tot;
        if (mrow) {
            // bitmask: lanes 8m .. 8m+7 hold keys 32m' .. 32m'+31 of word m' =
            // g0/8 + m; their 4-bit nibbles are OR-ed across the 8 lanes
            unsigned int wd = ((sel[0] ? 1u : 0u) | (sel[1] ? 2u : 0u) | (sel[2] ? 4u : 0u) | (sel[3] ? 8u : 0u))
                              << (4 * (lane & 7));
            wd |= __shfl_xor_sync(FULL, wd, 1);
            wd |= __shfl_xor_sync(FULL, wd, 2);
            wd |= __shfl_xor_sync(FULL, wd, 4);
            const int w = g0 / 8 + (lane >> 3);
            if ((lane & 7) == 0 && w < W) mrow[w] = wd;
        }
    }
    if (mrow)   // words past the row's causal end
        for (int w = 4 * ((n4 + 32) / 32) + lane; w < W; w += 32) mrow[w] = 0u;
}

// ------------------------------------------------ sampled single-pass select
//
// One CTA (NT threads) per (row, KV head), one pass over the row in the
// common case.  A sample of SP_SAMPLE keys (SP_LINES lines of 32 consecutive
// keys, evenly spaced over the row) brackets the k-th largest key: with
// p = topk / n, the number of sampled keys above the k-th key is binomial
// with mean SP_SAMPLE p and spread sigma = sqrt(SP_SAMPLE p (1 - p)), so the
// sample's ranks SP_SAMPLE p -/+ SP_Z sigma give an interval [yA, yB] of
// y = Ms - x (Ms: the sample's largest pattern) that holds the k-th key
// unless the sample is off by more than SP_Z sigma.  One pass over the row
// then sorts every key into: above the interval (taken: a bit in a shared-
// memory bitmask), inside it (a candidate: listed with y - yA, and counted
// in a 1024-bin histogram over the interval) or below it (not taken).  When
// fewer than topk keys were taken and the candidates reach topk, the k-th
// key is a candidate: the histogram names its bin, the few candidates in
// that bin give its exact pattern, and the candidates below it plus the
// lowest-indexed ones equal to it join the bitmask.  One compaction turns
// the bitmask into the ascending index list (and, when asked, the dense
// path's selection mask is the bitmask itself).  Otherwise (the interval
// missed the k-th key, the candidate list overflowed, or the k-th key's bin
// is crowded) the CTA runs the exact digit-pass select over the row.
// Integer work throughout: the result is the exact top-k with ties to the
// lower index, as every other select here computes it.
constexpr int SP_LINES = 32;
constexpr int SP_SAMPLE = SP_LINES * 32;
constexpr float SP_Z = 3.0f;
constexpr int SP_BINS = 1024;
constexpr int SP_VARS = 64;                // words of SpVars, rounded up
constexpr int SP_SMALL = SP_BINS / 2;      // candidates of the k-th key's bin held for the exact search
constexpr int SP_MIN_KEYS = 64;            // shorter rows take the exact select directly
constexpr int SP_UNROLL = 4;               // 16-byte loads in flight per thread in the pass

struct SpVars {
    unsigned int yA, yB, s1, ncand, nb, bstar, rb, fb, yT, keylim;
    unsigned int wa[NW], wb[NW];
};
static_assert(sizeof(SpVars) <= SP_VARS * 4, "SpVars");

// Shared-memory words before the bitmask: the histogram, the variables and
// the candidate list (key, y - yA), or the exact select's state.
__host__ __device__ constexpr int sp_region_words(int cap) {
    const int a = SP_BINS + SP_VARS + 2 * cap;
    const int b = (int)((sizeof(TopkShared) + 2 * NW * sizeof(int) + 3) / 4);
    return ((a > b ? a : b) + 3) & ~3;
}

// Exclusive prefix over the CTA of one value per thread (via V.wa).
__device__ __forceinline__ unsigned int sp_block_excl(SpVars &V, unsigned int v, int lane, int warp,
                                                      unsigned int &total) {
    unsigned int incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const unsigned int y = __shfl_up_sync(FULL, incl, off);
        if (lane >= off) incl += y;
    }
    if (lane == 31) V.wa[warp] = incl;
    __syncthreads();
    const unsigned int wv = lane < NW ? V.wa[lane] : 0u;
    const unsigned int woff = __reduce_add_sync(FULL, lane < warp ? wv : 0u);
    total = __reduce_add_sync(FULL, wv);
    return woff + incl - v;
}

template <bool AL>
__global__ void __launch_bounds__(NT, 2)
topk_sampled_kernel(const float *__restrict__ scores, long long ld, int Lq, int Lkv, int Hkv, int row_begin,
                    int row_count, int topk, int cap, int32_t *__restrict__ idx, uint32_t *__restrict__ mask,
                    int W, const int32_t *__restrict__ kv_len) {
    extern __shared__ __align__(16) unsigned int sp_smem[];
    unsigned int *hist = sp_smem;
    SpVars &V = *reinterpret_cast<SpVars *>(sp_smem + SP_BINS);
    unsigned int *ck = sp_smem + SP_BINS + SP_VARS, *cy = ck + cap;
    unsigned int *sel = sp_smem + sp_region_words(cap);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    // longest rows first; (batch, KV head) slowest
    const long long item = blockIdx.x;
    const int r = row_count - 1 - (int)(item % row_count);
    const long long bg = item / row_count;
    const int i = row_begin + r;
    const int n = row_keys(kv_len, (int)(bg / Hkv), Lq, Lkv, i);
    const unsigned int *u = reinterpret_cast<const unsigned int *>(scores + ((size_t)bg * row_count + r) * ld);
    int32_t *o = idx + ((size_t)bg * Lq + i) * (size_t)topk;
    uint32_t *mrow = mask ? mask + ((size_t)bg * Lq + i) * (size_t)W : nullptr;
    if (n <= topk) {
        for (int t = tid; t < topk; t += NT) o[t] = t < n ? t : -1;
        if (mrow)
            for (int w = tid; w < W; w += NT) {
                const int lo = 32 * w;
                mrow[w] = lo + 32 <= n ? FULL : (lo < n ? (1u << (n - lo)) - 1u : 0u);
            }
        return;
    }
    const int Wn = (n + 31) >> 5;
    for (int t = tid; t < SP_BINS; t += NT) hist[t] = 0u;
    for (int t = tid; t < Wn; t += NT) sel[t] = 0u;
    if (tid == 0) {
        V.ncand = 0u;
        V.nb = 0u;
    }

    // the sample: lines q and q + 16 (warp q), one key per lane each
    bool fb = n < SP_MIN_KEYS;
    unsigned int x0 = 0u, x1 = 0u;
    if (!fb) {
        const long long span = n - 32;
        x0 = __ldg(u + (int)(span * warp / (SP_LINES - 1)) + lane);
        x1 = __ldg(u + (int)(span * (warp + NW) / (SP_LINES - 1)) + lane);
    }
    {
        const unsigned int mx = __reduce_max_sync(FULL, max(x0, x1)), mn = __reduce_min_sync(FULL, min(x0, x1));
        if (lane == 0) {
            V.wa[warp] = mx;
            V.wb[warp] = mn;
        }
    }
    __syncthreads();
    const unsigned int Ms = __reduce_max_sync(FULL, lane < NW ? V.wa[lane] : 0u);
    const unsigned int ms = __reduce_min_sync(FULL, lane < NW ? V.wb[lane] : FULL);
    fb = fb || Ms == ms;
    const int s0 = max(0, (Ms > ms ? 32 - __clz(Ms - ms) : 0) - 10);
    if (!fb) {
        atomicAdd(&hist[(Ms - x0) >> s0], 1u);
        atomicAdd(&hist[(Ms - x1) >> s0], 1u);
    }
    __syncthreads();
    if (!fb && warp == 0) {
        const float p = (float)topk / (float)n;
        const float c = (float)SP_SAMPLE * p, sd = sqrtf((float)SP_SAMPLE * p * (1.f - p));
        const int rh = (int)floorf(c - SP_Z * sd), rl = (int)ceilf(c + SP_Z * sd);
        unsigned int yA = 0u, yB = FULL, rem, cnt;
        if (rh >= 1) yA = wk_find(hist, (unsigned int)rh, lane, rem, cnt) << s0;
        if (rl <= SP_SAMPLE) yB = ((wk_find(hist, (unsigned int)rl, lane, rem, cnt) + 1u) << s0) - 1u;
        const unsigned int span = min(yB, Ms) - yA;   // y = Ms - x never exceeds Ms
        if (lane == 0) {
            V.yA = yA;
            V.yB = yB;
            V.s1 = (unsigned int)max(0, (span ? 32 - __clz(span) : 0) - 10);
        }
    }
    __syncthreads();
    const unsigned int yA = V.yA, yB = V.yB;
    const int s1 = (int)V.s1;
    for (int t = tid; t < SP_BINS; t += NT) hist[t] = 0u;
    __syncthreads();

    // the pass: warp w takes 128-key groups w, w + NW, ... (lane l: keys
    // 4j .. 4j+3, j = 32 group + l), SP_UNROLL groups' loads in flight per
    // lane; the group after the last full one carries the n mod 4 tail keys
    if (!fb) {
        const int n4 = n >> 2, nt = n & 3;
        const unsigned int lt = (1u << lane) - 1u;
        for (int jb = warp * 32; jb < n4 + 1; jb += NT * SP_UNROLL) {
            uint4 vq[SP_UNROLL];
#pragma unroll
            for (int q = 0; q < SP_UNROLL; ++q) {
                const int j = jb + q * NT + lane;
                vq[q] = j < n4 ? ld4<AL>(u, j) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int q = 0; q < SP_UNROLL; ++q) {
                const int j0 = jb + q * NT;
                if (j0 >= n4 + 1) break;   // warp-uniform
                const int j = j0 + lane;
                unsigned int x[4];
                bool ok[4];
                if (j < n4) {
                    x[0] = vq[q].x; x[1] = vq[q].y; x[2] = vq[q].z; x[3] = vq[q].w;
                    ok[0] = ok[1] = ok[2] = ok[3] = true;
                } else {
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        ok[c] = j == n4 && c < nt;
                        x[c] = ok[c] ? __ldg(u + 4 * n4 + c) : 0u;
                    }
                }
                bool df[4], cd[4];
                unsigned int yv[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const unsigned int y = Ms - x[c];
                    df[c] = ok[c] && (x[c] > Ms || y < yA);
                    cd[c] = ok[c] && x[c] <= Ms && y >= yA && y <= yB;
                    yv[c] = y - yA;
                }
                // definites: word j >> 3 holds the nibbles of lanes 8m .. 8m+7
                unsigned int wd = ((df[0] ? 1u : 0u) | (df[1] ? 2u : 0u) | (df[2] ? 4u : 0u) | (df[3] ? 8u : 0u))
                                  << (4 * (lane & 7));
                wd |= __shfl_xor_sync(FULL, wd, 1);
                wd |= __shfl_xor_sync(FULL, wd, 2);
                wd |= __shfl_xor_sync(FULL, wd, 4);
                if ((lane & 7) == 0 && (j >> 3) < Wn) sel[j >> 3] = wd;
                if (__any_sync(FULL, cd[0] || cd[1] || cd[2] || cd[3])) {
                    int cbef = 0, ctot = 0;
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const unsigned int bb = __ballot_sync(FULL, cd[c]);
                        cbef += __popc(bb & lt);
                        ctot += __popc(bb);
                    }
                    unsigned int base = 0u;
                    if (lane == 0) base = atomicAdd(&V.ncand, (unsigned int)ctot);
                    unsigned int at = __shfl_sync(FULL, base, 0) + (unsigned int)cbef;
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        if (cd[c]) {
                            if (at < (unsigned int)cap) {
                                ck[at] = (unsigned int)(4 * j + c);
                                cy[at] = yv[c];
                            }
                            atomicAdd(&hist[yv[c] >> s1], 1u);
                            ++at;
                        }
                    }
                }
            }
        }
    }
    __syncthreads();

    // keys taken so far (D) and the rank of the k-th key among the candidates
    unsigned int dcnt = 0u;
    for (int t = tid; t < Wn; t += NT) dcnt += __popc(sel[t]);
    dcnt = __reduce_add_sync(FULL, dcnt);
    if (lane == 0) V.wa[warp] = dcnt;
    __syncthreads();
    const unsigned int D = __reduce_add_sync(FULL, lane < NW ? V.wa[lane] : 0u);
    const unsigned int ncand = V.ncand;
    fb = fb || D >= (unsigned int)topk || D + ncand < (unsigned int)topk || ncand > (unsigned int)cap;
    const unsigned int R = (unsigned int)topk - D;   // 1 .. ncand when !fb
    __syncthreads();
    if (!fb && warp == 0) {
        unsigned int rb, cnt;
        const unsigned int b = wk_find(hist, R, lane, rb, cnt);
        if (lane == 0) {
            V.bstar = b;
            V.rb = rb;
            V.fb = cnt > (unsigned int)SP_SMALL ? 1u : 0u;
        }
    }
    __syncthreads();
    fb = fb || V.fb != 0u;
    __syncthreads();   // every thread has read the flag before the fallback's state overlays it
    if (!fb) {
        // the k-th key's bin: its candidates, (key, low bits of y - yA), into
        // the histogram's space
        const unsigned int bstar = V.bstar, lowm = s1 ? (1u << s1) - 1u : 0u;
        for (int t = tid; t < (int)ncand; t += NT) {
            const unsigned int yc = cy[t];
            if ((yc >> s1) == bstar) {
                const unsigned int slot = atomicAdd(&V.nb, 1u);
                hist[2 * slot] = ck[t];
                hist[2 * slot + 1] = yc & lowm;
            }
        }
        __syncthreads();
        if (warp == 0) {
            // the rb-th smallest low bits, bit by bit from the top: `ans`
            // keeps the largest value with fewer than rb entries below it
            const int nb = (int)V.nb;
            const unsigned int rb = V.rb;
            unsigned int ans = 0u;
            for (int bit = s1 - 1; bit >= 0; --bit) {
                const unsigned int t = ans | (1u << bit);
                unsigned int c = 0u;
                for (int e = lane; e < nb; e += 32) c += hist[2 * e + 1] < t;
                if (__reduce_add_sync(FULL, c) < rb) ans = t;
            }
            unsigned int nl = 0u, ne = 0u;
            for (int e = lane; e < nb; e += 32) {
                nl += hist[2 * e + 1] < ans;
                ne += hist[2 * e + 1] == ans;
            }
            const unsigned int take_eq = rb - __reduce_add_sync(FULL, nl);
            ne = __reduce_add_sync(FULL, ne);
            unsigned int keylim = FULL;
            if (take_eq < ne) {
                // the take_eq-th smallest key among the entries equal to ans
                unsigned int kk = 0u;
                for (int bit = 31 - __clz((unsigned int)n); bit >= 0; --bit) {
                    const unsigned int t = kk | (1u << bit);
                    unsigned int c = 0u;
                    for (int e = lane; e < nb; e += 32) c += hist[2 * e + 1] == ans && hist[2 * e] < t;
                    if (__reduce_add_sync(FULL, c) < take_eq) kk = t;
                }
                keylim = kk;
            }
            if (lane == 0) {
                V.yT = (bstar << s1) | ans;
                V.keylim = keylim;
            }
        }
        __syncthreads();
        const unsigned int yT = V.yT, keylim = V.keylim;
        for (int t = tid; t < (int)ncand; t += NT) {
            const unsigned int yc = cy[t], key = ck[t];
            if (yc < yT || (yc == yT && key <= keylim)) atomicOr(&sel[key >> 5], 1u << (key & 31u));
        }
    } else {
        radix_select_row<false>(*reinterpret_cast<TopkShared *>(sp_smem),
                                reinterpret_cast<int *>(sp_smem) + sizeof(TopkShared) / 4,
                                reinterpret_cast<int *>(sp_smem) + sizeof(TopkShared) / 4 + NW, u, nullptr, n,
                                topk, o, tid);
        if (mrow == nullptr) return;
        __syncthreads();
        for (int t = tid; t < Wn; t += NT) sel[t] = 0u;
        __syncthreads();
        for (int t = tid; t < topk; t += NT) {
            const int key = o[t];
            atomicOr(&sel[key >> 5], 1u << (key & 31));
        }
    }
    __syncthreads();

    // ascending index list from the bitmask: thread t owns words
    // [t per, t per + per), its slots follow the exclusive prefix
    const int per = (Wn + NT - 1) / NT, w0 = tid * per;
    unsigned int cnt = 0u;
    for (int w = w0; w < min(w0 + per, Wn); ++w) cnt += __popc(sel[w]);
    unsigned int total;
    unsigned int pos = sp_block_excl(V, cnt, lane, warp, total);
    if (!fb)
        for (int w = w0; w < min(w0 + per, Wn); ++w) {
            unsigned int bits = sel[w];
            while (bits) {
                const int bb = __ffs(bits) - 1;
                if (pos < (unsigned int)topk) o[pos] = 32 * w + bb;
                ++pos;
                bits &= bits - 1u;
            }
        }
    if (mrow)
        for (int w = tid; w < W; w += NT) mrow[w] = w < Wn ? sel[w] : 0u;
}

}  // namespace

// Candidate-list capacity of the sampled select for rows of up to n_max keys
// (1.6 times the expected candidates of the longest row, plus the sample
// histogram's rounding) and its shared memory; 0 when it does not fit.
static int sp_capacity(long long n_max, int topk) {
    if (n_max <= topk) return 512;
    const double kk = topk, nn = (double)n_max;
    const double cand = 1.6 * 2.0 * SP_Z * sqrt(kk * (nn - kk) / SP_SAMPLE) + nn / 128.0 + 256.0;
    const long long cap = ((long long)cand + 255) & ~255ll;
    return (int)std::max(512ll, std::min(cap, 16384ll));
}
static size_t sp_smem_bytes(long long n_max, int cap) {
    const long long wsel = (((n_max + 31) >> 5) + 3) & ~3ll;
    return 4 * ((size_t)sp_region_words(cap) + (size_t)wsel);
}
constexpr size_t kSpMaxSmem = 160 * 1024;

cudaError_t topk_launch(const Shape &s, const float *scores, long long ld, int row_begin, int row_count,
                        int topk, int32_t *idx, cudaStream_t st, uint32_t *mask, int W, bool *mask_done) {
    if (mask_done) *mask_done = false;
    static bool attr = false;
    if (!attr) {
        cudaError_t e = cudaFuncSetAttribute(topk_radix_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kSmemKeys * 4);
        if (e != cudaSuccess) return e;
        attr = true;
    }
    const long long n_items = (long long)s.B * s.Hkv * row_count;
    const long long off = (long long)s.Lkv - s.Lq;
    const bool al = (reinterpret_cast<uintptr_t>(scores) & 15u) == 0 && (ld & 3) == 0;
    // HYSPARSE_TOPK_PATH=sampled|warp|block forces one kernel (the tests run
    // all three); the sampled single pass is the default where its shared
    // memory fits
    const char *force = getenv("HYSPARSE_TOPK_PATH");
    const bool f_warp = force && strcmp(force, "warp") == 0, f_block = force && strcmp(force, "block") == 0;
    const long long n_max = s.kv_len ? (long long)s.Lkv : off + row_begin + row_count;
    const int cap = sp_capacity(n_max, topk);
    const size_t sp_bytes = sp_smem_bytes(n_max, cap);
    // the sampled select for launches with few rows (decode).  With many
    // rows its fixed per-row work (serial phases of one warp while the CTA
    // waits at barriers, ~14 K warp instructions a row) costs more than the
    // one-warp-per-row kernel's extra passes: measured slower at 8 K to 64 K
    // keys per row.
    const bool f_sampled = force && strcmp(force, "sampled") == 0;
    const bool sampled = f_sampled || (!f_warp && !f_block && n_items < kWarpMinItems);
    if (sampled && sp_bytes <= kSpMaxSmem && n_items <= 0x7fffffffLL) {
        static size_t sp_attr = 0;
        if (sp_bytes > sp_attr) {
            cudaError_t e = cudaFuncSetAttribute(topk_sampled_kernel<true>,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSpMaxSmem);
            if (e == cudaSuccess)
                e = cudaFuncSetAttribute(topk_sampled_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSpMaxSmem);
            if (e != cudaSuccess) return e;
            sp_attr = kSpMaxSmem;
        }
        if (al)
            topk_sampled_kernel<true><<<(unsigned int)n_items, NT, sp_bytes, st>>>(
                scores, ld, s.Lq, s.Lkv, s.Hkv, row_begin, row_count, topk, cap, idx, mask, W, s.kv_len);
        else
            topk_sampled_kernel<false><<<(unsigned int)n_items, NT, sp_bytes, st>>>(
                scores, ld, s.Lq, s.Lkv, s.Hkv, row_begin, row_count, topk, cap, idx, mask, W, s.kv_len);
        count_launch();
        if (mask_done) *mask_done = mask != nullptr;
        return cudaGetLastError();
    }
    const bool many = f_warp || (!f_block && n_items >= kWarpMinItems);
    if (many) {
        const unsigned int grid = (unsigned int)((n_items + WK_WARPS - 1) / WK_WARPS);
        if (al)
            topk_warp_kernel<true><<<grid, WK_WARPS * 32, 0, st>>>(scores, ld, s.Lq, s.Lkv, s.Hkv, row_begin,
                                                                   row_count, topk, n_items, idx, mask, W, s.kv_len);
        else
            topk_warp_kernel<false><<<grid, WK_WARPS * 32, 0, st>>>(scores, ld, s.Lq, s.Lkv, s.Hkv, row_begin,
                                                                    row_count, topk, n_items, idx, mask, W, s.kv_len);
        count_launch();
        if (mask_done) *mask_done = mask != nullptr;
        return cudaGetLastError();
    }
    // Few rows (decode): one CTA per row.  Rows are ordered by causal length
    // n = off + row_begin + r + 1: those with n <= kSmemKeys run with the row
    // cached in shared memory (sized for the longest of them), the rest read
    // global memory.
    const long long split = max(0ll, min((long long)row_count, (long long)kSmemKeys - off - row_begin));
    if (split > 0) {
        const long long n_max = off + row_begin + split;
        topk_radix_kernel<true><<<dim3((unsigned)split, s.Hkv, s.B), NT, (size_t)n_max * 4, st>>>(
            scores, ld, s.Lq, s.Lkv, s.Hkv, row_begin, row_count, 0, topk, idx, s.kv_len); count_launch();
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (split < row_count) {
        topk_radix_kernel<false><<<dim3((unsigned)(row_count - split), s.Hkv, s.B), NT, 0, st>>>(
            scores, ld, s.Lq, s.Lkv, s.Hkv, row_begin, row_count, (int)split, topk, idx, s.kv_len); count_launch();
    }
    return cudaGetLastError();
}

}  // namespace hs
