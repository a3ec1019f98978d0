// Per-row top-k over importance scores by radix selection on the fp32 bit
// patterns (write-up section 2.2: the global branch attends over the full
// layer's TopK indices; baidu article "Top-K selection").
//
// Importance scores are sums of probabilities, so they are >= 0 and their
// IEEE-754 bit patterns, read as uint32, sort in the same order as the
// values.  Four 8-bit digit passes find the exact bit pattern T of the k-th
// largest score and how many keys equal to T must be taken; a final pass in
// ascending key order emits every key above T and the lowest-indexed keys
// equal to T, which is exactly "largest scores, ties to the lower index",
// already in ascending order.  Integer work only: the result is exact and
// deterministic.
#include <cub/block/block_scan.cuh>

#include "common.cuh"
#include "internal.h"

namespace hs {
namespace {

template <int NT>
__global__ void __launch_bounds__(NT)
topk_radix_kernel(const float *__restrict__ scores, long long ld, int Lq, int Lkv, int Hkv,
                  int row_begin, int row_count, int topk, int32_t *__restrict__ idx) {
    using Scan = cub::BlockScan<int, NT>;
    __shared__ typename Scan::TempStorage scan_tmp;
    __shared__ unsigned int hist[256];
    __shared__ unsigned int sh_digit, sh_remaining;

    const int r = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x;
    const int i = row_begin + r;
    const int n = Lkv - Lq + i + 1;
    const unsigned int *u = reinterpret_cast<const unsigned int *>(
        scores + (((size_t)b * Hkv + g) * row_count + r) * ld);
    int32_t *o = idx + (((size_t)b * Hkv + g) * Lq + i) * (size_t)topk;

    if (n <= topk) {
        for (int t = tid; t < topk; t += NT) o[t] = t < n ? t : -1;
        return;
    }

    unsigned int prefix = 0, mask = 0, remaining = (unsigned int)topk;
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int t = tid; t < 256; t += NT) hist[t] = 0;
        __syncthreads();
        for (int j = tid; j < n; j += NT) {
            const unsigned int x = u[j];
            if ((x & mask) == prefix) atomicAdd(&hist[(x >> shift) & 255u], 1u);
        }
        __syncthreads();
        if (tid < 32) {
            // lane covers digits 255-8*lane .. 255-8*lane-7 (descending order)
            unsigned int c[8], tot = 0;
#pragma unroll
            for (int t = 0; t < 8; ++t) {
                c[t] = hist[255 - (8 * tid + t)];
                tot += c[t];
            }
            unsigned int incl = tot;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const unsigned int y = __shfl_up_sync(0xffffffffu, incl, off);
                if (tid >= off) incl += y;
            }
            const unsigned int excl = incl - tot;
            if (excl < remaining && remaining <= incl) {
                unsigned int cum = excl;
#pragma unroll
                for (int t = 0; t < 8; ++t) {
                    if (cum + c[t] >= remaining) {
                        sh_digit = 255u - (unsigned int)(8 * tid + t);
                        sh_remaining = remaining - cum;
                        break;
                    }
                    cum += c[t];
                }
            }
        }
        __syncthreads();
        prefix |= sh_digit << shift;
        mask |= 255u << shift;
        remaining = sh_remaining;
        __syncthreads();
    }

    // prefix == bit pattern of the k-th largest score; take every key above it
    // and the first `remaining` keys equal to it, in ascending key order.
    int base_sel = 0, base_eq = 0;
    for (int j0 = 0; j0 < n; j0 += NT) {
        const int j = j0 + tid;
        const bool valid = j < n;
        const unsigned int x = valid ? u[j] : 0u;
        const int is_eq = (valid && x == prefix) ? 1 : 0;
        int eq_rank, eq_total;
        Scan(scan_tmp).ExclusiveSum(is_eq, eq_rank, eq_total);
        __syncthreads();
        const int sel = (valid && (x > prefix || (is_eq && base_eq + eq_rank < (int)remaining))) ? 1 : 0;
        int sel_rank, sel_total;
        Scan(scan_tmp).ExclusiveSum(sel, sel_rank, sel_total);
        __syncthreads();
        if (sel && base_sel + sel_rank < topk) o[base_sel + sel_rank] = j;
        base_sel += sel_total;
        base_eq += eq_total;
        if (base_sel >= topk) break;
    }
}

}  // namespace

cudaError_t topk_launch(const Shape &s, const float *scores, long long ld, int row_begin,
                        int row_count, int topk, int32_t *idx, cudaStream_t st) {
    constexpr int NT = 512;
    dim3 grid(row_count, s.Hkv, s.B);
    topk_radix_kernel<NT><<<grid, NT, 0, st>>>(scores, ld, s.Lq, s.Lkv, s.Hkv, row_begin, row_count,
                                                topk, idx);
    return cudaGetLastError();
}

}  // namespace hs
