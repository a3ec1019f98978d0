// L2 read-bandwidth probes, the denominator for kernels whose traffic is
// served from L2 rather than HBM (the prefill sparse layers gather their K/V
// rows from a cache that fits in L2: one KV head's K and V are tens of MB).
//
// Two access patterns over a caller buffer that is already resident in L2:
//   mode 0  streaming: every thread reads consecutive 16-byte words, grid
//           stride, `passes` times over the buffer;
//   mode 1  row gather: every half-warp reads one whole 256-byte row at a
//           hashed position (the gather kernels' access pattern: one K or V
//           row of one KV head per 16 lanes), `passes` x (bytes / 256) rows.
// Loads are L2-only (ld.global.cg) so that L1 hits do not inflate the figure.
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

__global__ void __launch_bounds__(kProbeThreads) l2_stream_probe(const uint4 *buf, size_t n16, int passes,
                                                                 unsigned long long *sink) {
    uint32_t acc = 0;
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    for (int p = 0; p < passes; ++p) {
        size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
        for (; i + 3 * stride < n16; i += 4 * stride) {
            const uint4 a = __ldcg(buf + i), b = __ldcg(buf + i + stride);
            const uint4 c = __ldcg(buf + i + 2 * stride), d = __ldcg(buf + i + 3 * stride);
            acc ^= a.x ^ a.w ^ b.y ^ b.z ^ c.x ^ c.w ^ d.y ^ d.z;
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
    // each warp step reads 8 rows (two per instruction, four instructions in flight)
    for (long long r0 = warp * 8; r0 < rows_total; r0 += nwarps * 8) {
        uint4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const uint32_t row = mix32((uint32_t)(r0 + 2 * u + half) * 2654435761u + 12345u) % nrows;
            v[u] = __ldcg(buf + (size_t)row * 16 + part);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) acc ^= v[u].x ^ v[u].w;
    }
    for (int o = 16; o > 0; o >>= 1) acc ^= __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) atomicXor(sink + blockIdx.x, (unsigned long long)acc);
}

}  // namespace
}  // namespace hs

extern "C" int hysparse_probe_l2_read(const void *buf, size_t bytes, int passes, int mode, int blocks,
                                      unsigned long long *sink, hs_stream_t stream) {
    if (buf == nullptr || sink == nullptr || ((uintptr_t)buf & 255u) != 0 || bytes < 4096 || (bytes & 255u) != 0)
        return HS_ERR_INVALID_ARG;
    if (passes < 1 || blocks < 1 || blocks > 65535 || (mode != 0 && mode != 1)) return HS_ERR_INVALID_ARG;
    if (bytes / 256 > 0xffffffffull) return HS_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    const uint4 *b = reinterpret_cast<const uint4 *>(buf);
    if (mode == 0)
        hs::l2_stream_probe<<<blocks, hs::kProbeThreads, 0, st>>>(b, bytes / 16, passes, sink);
    else
        hs::l2_gather_probe<<<blocks, hs::kProbeThreads, 0, st>>>(b, (uint32_t)(bytes / 256),
                                                                  (long long)passes * (long long)(bytes / 256), sink);
    hs::count_launch();
    return cudaGetLastError() == cudaSuccess ? HS_OK : HS_ERR_CUDA;
}
