// L2 read-bandwidth probes, the denominator for kernels whose traffic is
// served from L2 rather than HBM (the prefill sparse layers gather their K/V
// rows from a cache that fits in L2: one KV head's K and V are tens of MB).
//
// Access patterns over a caller buffer that is already resident in L2:
//   mode 0  streaming: every thread reads consecutive 16-byte words, grid
//           stride, `passes` times over the buffer;
//   mode 1  row gather: every half-warp reads one whole 256-byte row at a
//           hashed position (the gather kernels' access pattern: one K or V
//           row of one KV head per 16 lanes), `passes` x (bytes / 256) rows;
//   modes 2 and 3: the same two patterns through cp.async into shared memory.
// Loads are L2-only (ld.global.cg / cp.async.cg) so that L1 hits do not
// inflate the figure.
// Each block folds what it read into one word of `sink` so nothing is dead.
#include <cuda_runtime.h>
#include <stdint.h>

#include "hysparse.h"
#include "internal.h"

namespace hs {
namespace {

constexpr int kProbeThreads = 512;

__device__ __forceinline__ uint32_t mix32(uint32_t x) {
    // integer finaliser (xor-shift-multiply), a cheap well-spread hash
    x ^= x >> 16;
    x *= 0x7feb352du;
    x ^= x >> 15;
    x *= 0x846ca68bu;
    x ^= x >> 16;
    return x;
}

// Each thread keeps kInFlight 16-byte loads outstanding (the loaded L2
// latency is microseconds, so a probe with few loads in flight measures
// latency, not bandwidth).
constexpr int kInFlight = 8;

__global__ void __launch_bounds__(kProbeThreads) l2_stream_probe(const uint4 *buf, size_t n16, int passes,
                                                                 unsigned long long *sink) {
    uint32_t acc = 0;
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    for (int p = 0; p < passes; ++p) {
        size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
        for (; i + (kInFlight - 1) * stride < n16; i += kInFlight * stride) {
            uint4 v[kInFlight];
#pragma unroll
            for (int u = 0; u < kInFlight; ++u) v[u] = __ldcg(buf + i + u * stride);
#pragma unroll
            for (int u = 0; u < kInFlight; ++u) acc ^= v[u].x ^ v[u].w;
        }
        for (; i < n16; i += stride) {
            const uint4 a = __ldcg(buf + i);
            acc ^= a.x ^ a.w;
        }
    }
    for (int o = 16; o > 0; o >>= 1) acc ^= __shfl_xor_sync(0xffffffffu, acc, o);
    if ((threadIdx.x & 31) == 0) atomicXor(sink + blockIdx.x, (unsigned long long)acc);
}

__global__ void __launch_bounds__(kProbeThreads) l2_gather_probe(const uint4 *buf, uint32_t nrows,
                                                                 long long rows_total, unsigned long long *sink) {
    uint32_t acc = 0;
    const int lane = threadIdx.x & 31, half = lane >> 4, part = lane & 15;
    const long long warp = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
    // each warp step reads 2 * kInFlight rows (two per instruction)
    for (long long r0 = warp * 2 * kInFlight; r0 < rows_total; r0 += nwarps * 2 * kInFlight) {
        uint4 v[kInFlight];
        const uint32_t base = (uint32_t)r0;
#pragma unroll
        for (int u = 0; u < kInFlight; ++u) {
            const uint32_t row = mix32((base + 2 * u + half) * 2654435761u + 12345u) % nrows;
            v[u] = __ldcg(buf + (size_t)row * 16 + part);
        }
#pragma unroll
        for (int u = 0; u < kInFlight; ++u) acc ^= v[u].x ^ v[u].w;
    }
    for (int o = 16; o > 0; o >>= 1) acc ^= __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) atomicXor(sink + blockIdx.x, (unsigned long long)acc);
}

// Modes 2 and 3: the same two patterns read with cp.async into a shared-
// memory ring, the path the row-gather kernels use: kCpWarps warps per CTA,
// each streaming 8 KB stages of 32 whole 256-byte rows, kCpStages - 1 in
// flight.
constexpr int kCpWarps = 7;
constexpr int kCpStages = 4;
constexpr int kCpStage = 8192;
constexpr int kCpSmem = kCpWarps * kCpStages * kCpStage;

__device__ __forceinline__ void cp16(uint32_t dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

__global__ void __launch_bounds__(kCpWarps * 32) l2_cp_probe(const uint8_t *buf, uint32_t nrows, long long steps,
                                                            int random, unsigned long long *sink) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, q = lane >> 3, sct = lane & 7;
    const long long gw = (long long)blockIdx.x * kCpWarps + warp, nw = (long long)gridDim.x * kCpWarps;
    uint8_t *ring = smem + warp * kCpStages * kCpStage;
    // warp step s reads 32 rows: rows [32 s', 32 s' + 32) mod nrows (stream) or
    // 32 hashed rows (random), s' = gw + s * nw; `steps` steps in all
    int k = 0;
    for (long long s0 = gw; s0 < steps; s0 += nw, ++k) {
        const uint32_t dst = (uint32_t)__cvta_generic_to_shared(ring + (k % kCpStages) * kCpStage);
        const uint32_t first = (uint32_t)((s0 * 32) % nrows);   // one 64-bit step per 32 rows
        // the row gather's copy pattern: four rows per instruction, lanes
        // 8q .. 8q+7 on row 4 r4 + q, lane s its 16-byte chunk s and then s + 8
#pragma unroll
        for (int r4 = 0; r4 < 8; ++r4) {
            const uint32_t rl = 4 * r4 + q;
            uint32_t row;
            if (random) {
                row = mix32(((uint32_t)s0 * 32u + rl) * 2654435761u + 12345u) % nrows;
            } else {
                row = first + rl;
                if (row >= nrows) row -= nrows;
            }
            cp16(dst + rl * 256 + sct * 16, buf + (size_t)row * 256 + sct * 16);
            cp16(dst + rl * 256 + (sct + 8) * 16, buf + (size_t)row * 256 + (sct + 8) * 16);
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
        asm volatile("cp.async.wait_group %0;" ::"n"(kCpStages - 1) : "memory");
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncwarp();
    const uint32_t v = *reinterpret_cast<const uint32_t *>(ring + lane * 4);
    if (lane == 0) atomicXor(sink + blockIdx.x, (unsigned long long)v);
}

}  // namespace
}  // namespace hs

extern "C" int hysparse_probe_l2_read(const void *buf, size_t bytes, int passes, int mode, int blocks,
                                      unsigned long long *sink, hs_stream_t stream) {
    if (buf == nullptr || sink == nullptr || ((uintptr_t)buf & 255u) != 0 || bytes < 4096 || (bytes & 255u) != 0)
        return HS_ERR_INVALID_ARG;
    if (passes < 1 || blocks < 1 || blocks > 65535 || mode < 0 || mode > 3) return HS_ERR_INVALID_ARG;
    if (bytes / 256 > 0xffffffffull || (mode >= 2 && bytes < 65536)) return HS_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    const uint4 *b = reinterpret_cast<const uint4 *>(buf);
    if (mode == 0) {
        hs::l2_stream_probe<<<blocks, hs::kProbeThreads, 0, st>>>(b, bytes / 16, passes, sink);
    } else if (mode == 1) {
        hs::l2_gather_probe<<<blocks, hs::kProbeThreads, 0, st>>>(b, (uint32_t)(bytes / 256),
                                                                  (long long)passes * (long long)(bytes / 256), sink);
    } else {
        static bool attr = false;
        if (!attr) {
            if (cudaFuncSetAttribute(hs::l2_cp_probe, cudaFuncAttributeMaxDynamicSharedMemorySize, hs::kCpSmem) !=
                cudaSuccess)
                return HS_ERR_CUDA;
            attr = true;
        }
        // passes * bytes in steps of 32 rows (8 KB); bytes is a multiple of 256
        const long long steps = (long long)passes * (long long)(bytes / 256) / 32;
        hs::l2_cp_probe<<<blocks, hs::kCpWarps * 32, hs::kCpSmem, st>>>(
            reinterpret_cast<const uint8_t *>(buf), (uint32_t)(bytes / 256), steps, mode == 3 ? 1 : 0, sink);
    }
    hs::count_launch();
    return cudaGetLastError() == cudaSuccess ? HS_OK : HS_ERR_CUDA;
}
