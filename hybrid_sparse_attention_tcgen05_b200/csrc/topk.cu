// Per-row top-k over importance scores by radix selection on the fp32 bit
// patterns (write-up section 2.2: the global branch attends over the full
// layer's TopK indices; baidu article "Top-K selection").
//
// Importance scores are sums of probabilities, so they are >= 0: the sign
// bit is 0 and the other 31 bits, read as an unsigned integer, sort in the
// same order as the values.  Three digit passes (bits 30-20, 19-10, 9-0) find
// the exact bit pattern T of the k-th largest score and how many keys equal
// to T must be taken; an ordered compaction then emits every key above T and
// the lowest-indexed keys equal to T, which is exactly "largest scores, ties
// to the lower index", already in ascending key order.  Integer work only:
// the result is exact and deterministic.
//
// Rows whose causal length fits (kSmemKeys) are first copied into shared
// memory, so only that one read touches L2/HBM; longer rows are re-read from
// global memory each pass.  The bin holding the k-th key is found by a
// block-parallel scan over the bins (descending); the compaction uses
// per-warp ballot counts and one pass over warp totals.
#include "common.cuh"
#include "internal.h"

namespace hs {
namespace {

constexpr int NT = 512;
constexpr int NW = NT / 32;
constexpr int kSmemKeys = 24576;       // 96 KB of row cache
constexpr int kHistBins = 2048;

struct TopkShared {
    unsigned int hist[kHistBins];
    unsigned int sh_digit, sh_remaining;
    unsigned int wsum[NW], woff[NW];
    int cnt_gt[NW], cnt_eq[NW];
};

// Find the bin (scanning from the top) in which the running count of keys
// first reaches `remaining`; every thread owns nb / NT consecutive bins.
// Writes the bin and the count still needed inside it to shared memory.
__device__ __forceinline__ void find_bin(TopkShared &sh, unsigned int nb, unsigned int remaining, int tid) {
    const int lane = tid & 31, warp = tid >> 5;
    const int per = (int)nb / NT;
    unsigned int c[kHistBins / NT];
    unsigned int tot = 0;
#pragma unroll
    for (int k = 0; k < kHistBins / NT; ++k) {
        c[k] = k < per ? sh.hist[nb - 1 - (unsigned)(per * tid + k)] : 0u;
        tot += c[k];
    }
    unsigned int incl = tot;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const unsigned int y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
    }
    if (lane == 31) sh.wsum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        unsigned int v = lane < NW ? sh.wsum[lane] : 0u;
        unsigned int vi = v;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const unsigned int y = __shfl_up_sync(0xffffffffu, vi, off);
            if (lane >= off) vi += y;
        }
        if (lane < NW) sh.woff[lane] = vi - v;
    }
    __syncthreads();
    const unsigned int excl = sh.woff[warp] + incl - tot;
    if (excl < remaining && remaining <= excl + tot) {
        unsigned int cum = excl;
#pragma unroll
        for (int k = 0; k < kHistBins / NT; ++k) {
            if (k < per && cum + c[k] >= remaining) {
                sh.sh_digit = nb - 1 - (unsigned)(per * tid + k);
                sh.sh_remaining = remaining - cum;
                break;
            }
            cum += c[k];
        }
    }
}

template <bool SMEM>
__global__ void __launch_bounds__(NT)
topk_radix_kernel(const float *__restrict__ scores, long long ld, int Lq, int Lkv, int Hkv, int row_begin,
                  int row_count, int r_lo, int topk, int32_t *__restrict__ idx) {
    extern __shared__ unsigned int row_cache[];
    __shared__ TopkShared sh;

    const int r = r_lo + blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int i = row_begin + r;
    const int n = Lkv - Lq + i + 1;
    const unsigned int *gu =
        reinterpret_cast<const unsigned int *>(scores + (((size_t)b * Hkv + g) * row_count + r) * ld);
    int32_t *o = idx + (((size_t)b * Hkv + g) * Lq + i) * (size_t)topk;

    if (n <= topk) {
        for (int t = tid; t < topk; t += NT) o[t] = t < n ? t : -1;
        return;
    }
    const unsigned int *u = gu;
    if (SMEM) {
        for (int j = tid; j < n; j += NT) row_cache[j] = __ldg(gu + j);
        __syncthreads();
        u = row_cache;
    }

    unsigned int prefix = 0, mask = 0, remaining = (unsigned int)topk;
#pragma unroll
    for (int ps = 0; ps < 3; ++ps) {
        const int shift = ps == 0 ? 20 : (ps == 1 ? 10 : 0);
        const unsigned int nb = ps == 0 ? 2048u : 1024u;
        for (int t = tid; t < (int)nb; t += NT) sh.hist[t] = 0;
        __syncthreads();
        for (int j = tid; j < n; j += NT) {
            const unsigned int x = SMEM ? u[j] : __ldg(u + j);
            if ((x & mask) == prefix) atomicAdd(&sh.hist[(x >> shift) & (nb - 1u)], 1u);
        }
        __syncthreads();
        find_bin(sh, nb, remaining, tid);
        __syncthreads();
        prefix |= sh.sh_digit << shift;
        mask |= (nb - 1u) << shift;
        remaining = sh.sh_remaining;
        __syncthreads();
    }

    // prefix == the bit pattern of the k-th largest score.  Ordered
    // compaction: warp w owns the contiguous key range [w*seg, (w+1)*seg).
    // (A negative input, which importance scores never are, could only make
    // more keys compare above T; the `at < topk` guard keeps writes in bounds.)
    const unsigned int T = prefix;
    const int seg = ((n + NW - 1) / NW + 31) & ~31;
    const int j_lo = warp * seg, j_hi = min(n, j_lo + seg);
    int gt = 0, eq = 0;
    for (int j0 = j_lo; j0 < j_hi; j0 += 32) {
        const int j = j0 + lane;
        const unsigned int x = j < j_hi ? (SMEM ? u[j] : __ldg(u + j)) : 0u;
        gt += __popc(__ballot_sync(0xffffffffu, j < j_hi && x > T));
        eq += __popc(__ballot_sync(0xffffffffu, j < j_hi && x == T));
    }
    if (lane == 0) {
        sh.cnt_gt[warp] = gt;
        sh.cnt_eq[warp] = eq;
    }
    __syncthreads();
    int gt_base = 0, eq_base = 0;
    for (int w = 0; w < warp; ++w) {
        gt_base += sh.cnt_gt[w];
        eq_base += sh.cnt_eq[w];
    }
    const unsigned int lt_mask = (1u << lane) - 1u;
    for (int j0 = j_lo; j0 < j_hi; j0 += 32) {
        const int j = j0 + lane;
        const unsigned int x = j < j_hi ? (SMEM ? u[j] : __ldg(u + j)) : 0u;
        const unsigned int bg = __ballot_sync(0xffffffffu, j < j_hi && x > T);
        const unsigned int be = __ballot_sync(0xffffffffu, j < j_hi && x == T);
        const int gtb = gt_base + __popc(bg & lt_mask);
        const int eqb = eq_base + __popc(be & lt_mask);
        const bool is_gt = (bg >> lane) & 1u, is_eq = (be >> lane) & 1u;
        if (is_gt || (is_eq && eqb < (int)remaining)) {
            const int at = gtb + min(eqb, (int)remaining);
            if (at < topk) o[at] = j;
        }
        gt_base += __popc(bg);
        eq_base += __popc(be);
    }
}

}  // namespace

cudaError_t topk_launch(const Shape &s, const float *scores, long long ld, int row_begin, int row_count,
                        int topk, int32_t *idx, cudaStream_t st) {
    static bool attr = false;
    if (!attr) {
        cudaError_t e = cudaFuncSetAttribute(topk_radix_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kSmemKeys * 4);
        if (e != cudaSuccess) return e;
        attr = true;
    }
    // rows are ordered by causal length; those up to kSmemKeys keys run with
    // the row cached in shared memory, sized for the longest of them
    const int off = s.Lkv - s.Lq;
    const int n_first = off + row_begin + 1;
    int split = row_count;                                   // rows [0, split) fit
    if (n_first > kSmemKeys) split = 0;
    else if (off + row_begin + row_count > kSmemKeys) split = kSmemKeys - off - row_begin;
    if (split > 0) {
        const int n_max = off + row_begin + split;
        topk_radix_kernel<true><<<dim3(split, s.Hkv, s.B), NT, (size_t)n_max * 4, st>>>(
            scores, ld, s.Lq, s.Lkv, s.Hkv, row_begin, row_count, 0, topk, idx); count_launch();
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (split < row_count) {
        topk_radix_kernel<false><<<dim3(row_count - split, s.Hkv, s.B), NT, 0, st>>>(
            scores, ld, s.Lq, s.Lkv, s.Hkv, row_begin, row_count, split, topk, idx); count_launch();
    }
    return cudaGetLastError();
}

}  // namespace hs
