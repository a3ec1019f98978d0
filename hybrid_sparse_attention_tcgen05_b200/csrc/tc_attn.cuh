// Pieces shared by the tcgen05 attention kernels (full layer and the
// dense-masked sparse layer): tile geometry, the two MMA issue helpers and
// the TMA tensor maps over [B][L][H][128] bf16 tensors.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include "tc_util.cuh"

namespace hs {
namespace tc {

constexpr int BM = 128;                 // query rows per tile
constexpr int BN = 128;                 // keys per tile
constexpr int HD = 128;                 // head dim
constexpr int TILE = BM * HD * 2;       // one 128x128 bf16 tile: 32 KB
constexpr int HALF = TILE / 2;          // one 64-column swizzled half: 16 KB
constexpr int KV_STAGES = 4;
// Forward kernels: softmax warpgroups 0 and 1 (one query head each), then a
// third warpgroup whose warp 8 issues the TMA loads and warp 9 the MMAs
// (warps 10 and 11 only complete the warpgroup for the register hand-over).
constexpr int FWD_THREADS = 384;
// Registers per thread at launch (65536 / 384, rounded down to a multiple of
// 8) and after the hand-over: the control warpgroup drops to kFwdCtlRegs and
// the softmax warpgroups rise to kFwdSoftRegs.  The shares must add up to at
// most what the block was launched with, or the increase never completes.
constexpr int kFwdLaunchRegs = 168;
constexpr int kFwdCtlRegs = 104;
constexpr int kFwdSoftRegs = 200;
static_assert(128 * kFwdCtlRegs + 256 * kFwdSoftRegs <= FWD_THREADS * kFwdLaunchRegs, "register hand-over over budget");
static_assert(kFwdLaunchRegs * FWD_THREADS <= 65536, "launch registers");
constexpr uint64_t kDrainNs = 1000000000ull;

// Register hand-over between warpgroups (sm_100a setmaxnreg): every warp of
// the warpgroup executes the same instruction.
template <int N>
__device__ __forceinline__ void regs_release() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void regs_acquire() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Two fp32 fused multiply-adds in one packed f32x2 instruction (sm_100):
// each lane is rounded exactly as fmaf would round it.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}

// Two fp32 additions in one packed f32x2 instruction (sm_100).
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

// max(a, b, c) in one three-input instruction (sm_100); NaN inputs are
// ignored as by fmaxf.
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// Row-tile grids are launched as (heads, row tiles x batch): the hardware
// hands out blocks in linear order with x fastest, so the heaviest causal
// row tile of every head and batch is dispatched before any lighter one.
// When tiles x batch exceed the y limit the batch moves to z.
inline dim3 tile_grid(int heads, int n_tiles, int batch) {
    if ((long long)n_tiles * batch <= 65535) return dim3(heads, n_tiles * batch, 1);
    return dim3(heads, n_tiles, batch);
}

// This block's row tile (0 = first 128 rows) and batch under tile_grid.
__device__ __forceinline__ void tile_of_block(int n_tiles, int &tile, int &b) {
    const int nb_y = gridDim.y / n_tiles;   // batches folded into y (1 when z carries them)
    tile = n_tiles - 1 - (int)blockIdx.y / nb_y;
    b = (int)blockIdx.z + (int)blockIdx.y % nb_y;
}

__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Wait that ignores the abort flag: used only to drain our own in-flight
// copies / MMAs before the CTA exits.
__device__ __forceinline__ void mbar_drain(uint32_t bar, uint32_t parity) {
    int dummy = 0;
    mbar_wait(bar, parity, kDrainNs, &dummy);
}

// S = Q K^T for one 128x128 tile: 8 MMAs of K=16 along the head dim.  Both
// operands are K-major 128-byte-swizzled [128][64] halves 16 KB apart.
__device__ __forceinline__ void issue_qk(uint32_t d_tmem, uint32_t q_addr, uint32_t k_addr) {
    constexpr uint32_t I = idesc_bf16(128, 128, false, false);
#pragma unroll
    for (int kk = 0; kk < HD / 16; ++kk) {
        const uint32_t o = (kk >> 2) * HALF + (kk & 3) * 32;
        mma_ss(d_tmem, sdesc_sw128(q_addr + o, 16, 1024), sdesc_sw128(k_addr + o, 16, 1024), I,
               kk > 0 ? 1u : 0u);
    }
}

// O (+)= P V: P is 128x128 bf16 in TMEM (64 columns), V a [128 keys][128 d]
// tile stored as two [128][64] swizzled halves -> N(=d)-major B operand.
__device__ __forceinline__ void issue_pv(uint32_t d_tmem, uint32_t p_tmem, uint32_t v_addr,
                                         bool accumulate) {
    constexpr uint32_t I = idesc_bf16(128, 128, false, true);
#pragma unroll
    for (int kk = 0; kk < BN / 16; ++kk) {
        mma_ts(d_tmem, p_tmem + kk * 8, sdesc_sw128(v_addr + kk * 2048, HALF, 1024), I,
               (accumulate || kk > 0) ? 1u : 0u);
    }
}


inline PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (fn == nullptr) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

// [B][L][H][128] bf16 -> 4-D map (d, H, L, B) with a {64, 1, 128, 1} box,
// 128-byte swizzle; rows past L read as zeros.
inline bool make_map(CUtensorMap *m, const void *base, int H, int L, int B) {
    auto enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[4] = {(cuuint64_t)HD, (cuuint64_t)H, (cuuint64_t)L, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)HD * 2, (cuuint64_t)HD * 2 * H, (cuuint64_t)HD * 2 * H * L};
    cuuint32_t box[4] = {64, 1, (cuuint32_t)BM, 1};
    cuuint32_t es[4] = {1, 1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace tc
}  // namespace hs
