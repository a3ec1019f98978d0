// Sparse layer of the hybrid block as a dense-masked pass on tcgen05.
//
// Method: intelliparadigm write-up section 2.2 (global branch over the TopK
// keys of the preceding full layer, local 128-token window, out = gate*global
// + (1-gate)*local, gate = sigmoid) and section 3.1 (the sparse layers read
// the full layer's cache and write none).
//
// When a row's top-k set covers a sizeable fraction of its causal keys (the
// prefill shapes: k/(pos+1) of 3-25 %), touching every causal key tile on the
// tensor cores costs less than gathering k rows per (row, KV head) from L2:
// every 128x128 S tile is computed, and the softmax threads apply two masks,
// "key is in this row's top-k set" (a bitmask built from the index lists) and
// "key is in this row's window", keeping one online-softmax state per branch.
// The exact same two softmaxes as the gather kernel result; only the masked
// work differs.  The host picks this kernel or the gather kernel from a cost
// estimate.
//
// CTA = 128 query rows of one query head.  Warps 0-3: softmax (thread = row =
// TMEM lane); warp 4: TMA producer (Q once, then K_j, V_j through a 4-slot
// ring); warp 5: MMA issuer.  TMEM: S0 | S1 (double-buffered scores) | Og |
// Ol.  P for the global branch overwrites S columns 0-63, P for the window
// branch columns 64-127 (window tiles only); both feed PV MMAs from TMEM.
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "internal.h"
#include "tc_attn.cuh"

namespace hs {
namespace tc {
namespace {

constexpr int SD_THREADS = 192;
constexpr int SD_KV = 4;

struct SdBars {
    uint64_t q_full;
    uint64_t kv_full[SD_KV], kv_empty[SD_KV];
    uint64_t s_full[2];
    uint64_t p_full;
    uint64_t o_done;
    uint64_t o_final;
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

constexpr size_t kSdSmem = 1024 + TILE + SD_KV * TILE + sizeof(SdBars);

struct SdParams {
    int Lq, Lkv, Hq, Hkv, G, window, W;
    float scale_log2;
    const uint32_t *selmask;   // [B][Hkv][Lq][W]
    const float *gate;         // [B][Lq][Hq]
    __nv_bfloat16 *out, *out_g, *out_l;
    unsigned int *status;
    unsigned long long wait_ns;
};

// Rescale 128 columns of an accumulator row in TMEM by `corr` (per thread).
__device__ __forceinline__ void tmem_scale128(uint32_t t, float corr) {
#pragma unroll 1
    for (int c = 0; c < 8; ++c) {
        uint32_t o[16];
        tmem_ld16(t + 16 * c, o);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * corr);
        tmem_st16(t + 16 * c, o);
    }
    tmem_wait_st();
}

__global__ void __launch_bounds__(SD_THREADS, 1)
sparse_dense_tc(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                const __grid_constant__ CUtensorMap tv, const SdParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    uint8_t *sq = smem;
    uint8_t *skv = smem + TILE;
    SdBars *bars = reinterpret_cast<SdBars *>(smem + TILE + SD_KV * TILE);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int tile, b;
    tile_of_block((p.Lq + BM - 1) / BM, tile, b);   // heaviest row tiles first
    const int r0 = tile * BM;
    const int r_end = min(r0 + BM, p.Lq);
    const int h = blockIdx.x;
    const int g = h / p.G;
    const int off = p.Lkv - p.Lq;
    const int pos_first = off + r0;
    const int pos_last = off + r_end - 1;
    const int n_kv = pos_last / BN + 1;
    const int jw0 = max(0, pos_first - p.window + 1) / BN;   // first tile any row's window touches

    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bars->q_full), 1);
        for (int s = 0; s < SD_KV; ++s) {
            mbar_init(smem_u32(&bars->kv_full[s]), 1);
            mbar_init(smem_u32(&bars->kv_empty[s]), 1);
        }
        mbar_init(smem_u32(&bars->s_full[0]), 1);
        mbar_init(smem_u32(&bars->s_full[1]), 1);
        mbar_init(smem_u32(&bars->p_full), 128);
        mbar_init(smem_u32(&bars->o_done), 1);
        mbar_init(smem_u32(&bars->o_final), 1);
        mbar_init(smem_u32(&bars->drain), 1);
        bars->abort = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(&bars->tmem_base), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    volatile int *abort = &bars->abort;

    if (warp == 4) {
        if (lane == 0) {
            tma_prefetch(&tq);
            tma_prefetch(&tk);
            tma_prefetch(&tv);
            const uint32_t qb = smem_u32(&bars->q_full);
            mbar_expect_tx(qb, TILE);
            for (int hf = 0; hf < 2; ++hf) tma_load_4d(smem_u32(sq + hf * HALF), &tq, qb, hf * 64, h, r0, b);
            int issued = 0;
            for (int it = 0; it < 2 * n_kv; ++it) {
                const int slot = it % SD_KV, use = it / SD_KV;
                if (!mbar_wait(smem_u32(&bars->kv_empty[slot]), (use & 1) ^ 1, p.wait_ns, abort)) break;
                const uint32_t fb = smem_u32(&bars->kv_full[slot]);
                mbar_expect_tx(fb, TILE);
                const CUtensorMap *m = (it & 1) ? &tv : &tk;
                for (int hf = 0; hf < 2; ++hf)
                    tma_load_4d(smem_u32(skv + slot * TILE + hf * HALF), m, fb, hf * 64, g, (it >> 1) * BN, b);
                issued = it + 1;
            }
            if (*abort) {
                mbar_drain(qb, 0);
                for (int it = issued > SD_KV ? issued - SD_KV : 0; it < issued; ++it)
                    mbar_drain(smem_u32(&bars->kv_full[it % SD_KV]), (it / SD_KV) & 1);
            }
        }
    } else if (warp == 5) {
        if (lane == 0) {
            const uint32_t tS[2] = {tmem, tmem + 128};
            const uint32_t tOg = tmem + 256, tOl = tmem + 384;
            const uint32_t qa = smem_u32(sq);
            bool ok = mbar_wait(smem_u32(&bars->q_full), 0, p.wait_ns, abort);
            for (int jj = 0; ok && jj < min(2, n_kv); ++jj) {
                const int itK = 2 * jj, sk = itK % SD_KV;
                if (!(ok = mbar_wait(smem_u32(&bars->kv_full[sk]), (itK / SD_KV) & 1, p.wait_ns, abort))) break;
                tc_fence_after();
                issue_qk(tS[jj], qa, smem_u32(skv + sk * TILE));
                mma_commit(smem_u32(&bars->s_full[jj]));
                mma_commit(smem_u32(&bars->kv_empty[sk]));
            }
            for (int j = 0; ok && j < n_kv; ++j) {
                const int buf = j & 1;
                const int itV = 2 * j + 1, sv = itV % SD_KV;
                if (!(ok = mbar_wait(smem_u32(&bars->p_full), j & 1, p.wait_ns, abort))) break;
                if (!(ok = mbar_wait(smem_u32(&bars->kv_full[sv]), (itV / SD_KV) & 1, p.wait_ns, abort))) break;
                tc_fence_after();
                const uint32_t va = smem_u32(skv + sv * TILE);
                issue_pv(tOg, tS[buf], va, j > 0);
                if (j >= jw0) issue_pv(tOl, tS[buf] + 64, va, j > jw0);
                mma_commit(smem_u32(&bars->o_done));
                mma_commit(smem_u32(&bars->kv_empty[sv]));
                if (j == n_kv - 1) mma_commit(smem_u32(&bars->o_final));
                if (j + 2 < n_kv) {
                    const int itK = 2 * (j + 2), sk = itK % SD_KV;
                    if (!(ok = mbar_wait(smem_u32(&bars->kv_full[sk]), (itK / SD_KV) & 1, p.wait_ns, abort))) break;
                    tc_fence_after();
                    issue_qk(tS[buf], qa, smem_u32(skv + sk * TILE));
                    mma_commit(smem_u32(&bars->s_full[buf]));
                    mma_commit(smem_u32(&bars->kv_empty[sk]));
                }
            }
            mma_commit(smem_u32(&bars->drain));
            mbar_drain(smem_u32(&bars->drain), 0);
        }
    } else {
        const int tw = threadIdx.x;
        const int row = r0 + tw;
        const bool valid = row < r_end;
        const int rrow = min(row, r_end - 1);
        const int pos = off + rrow;
        const int lo_w = max(0, pos - p.window + 1);
        const uint32_t lane_off = (uint32_t)(tw & ~31) << 16;
        const uint32_t tOg = tmem + lane_off + 256u, tOl = tmem + lane_off + 384u;
        const uint4 *mrow = reinterpret_cast<const uint4 *>(p.selmask + (((size_t)b * p.Hkv + g) * p.Lq + rrow) * p.W);
        const float c2 = p.scale_log2;
        float mg = -INFINITY, lg = 0.f, cg = 0.f;
        float ml = -INFINITY, ll = 0.f, cl = 0.f;
        bool ok = true;
        uint4 mw = __ldg(mrow);
        for (int j = 0; j < n_kv; ++j) {
            const int buf = j & 1;
            const uint32_t tS = tmem + lane_off + (uint32_t)(buf * 128);
            const uint32_t mwords[4] = {mw.x, mw.y, mw.z, mw.w};
            if (j + 1 < n_kv) mw = __ldg(mrow + j + 1);   // prefetch the next tile's mask
            ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bars->s_full[buf]), (j >> 1) & 1, p.wait_ns, abort));
            if (!ok) break;
            tc_fence_after();
            float sv[128];
            {
                uint32_t r[4][32];
#pragma unroll
                for (int c = 0; c < 4; ++c) tmem_ld32(tS + 32 * c, r[c]);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 128; ++c) sv[c] = __uint_as_float(r[c >> 5][c & 31]);
            }
            const int j0 = j * BN;
            const bool wtile = j >= jw0;
            const bool diag = j0 + BN - 1 > pos_first;      // causal edge may cut this tile
            // PV of the previous tile must be done before O is touched
            if (j > 0) {
                ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bars->o_done), (j - 1) & 1, p.wait_ns, abort));
                if (!ok) break;
                tc_fence_after();
            }
            float sl0 = 0.f, sl1 = 0.f;
            if (wtile) {
                // window branch first, on the unmasked scores
                float w4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                for (int c = 0; c < 128; ++c)
                    if (j0 + c >= lo_w && j0 + c <= pos) w4[c & 3] = fmaxf(w4[c & 3], sv[c]);
                const float mxl2 = fmaxf(fmaxf(w4[0], w4[1]), fmaxf(w4[2], w4[3])) * c2;
                if (__any_sync(0xffffffffu, mxl2 > ml + 8.0f)) {
                    const float mn = fmaxf(ml, mxl2);
                    if (j > jw0) {
                        const float corr = (mn == -INFINITY || ml == -INFINITY) ? (mn == -INFINITY ? 1.f : 0.f) : ex2(ml - mn);
                        ll *= corr;
                        cl *= corr;
                        tmem_scale128(tOl, corr);
                    }
                    ml = mn;
                }
                const float mlx = ml == -INFINITY ? 0.f : ml;
#pragma unroll
                for (int qq = 0; qq < 4; ++qq) {
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const int c = qq * 32 + 2 * e;
                        const bool w0 = j0 + c >= lo_w && j0 + c <= pos;
                        const bool w1 = j0 + c + 1 >= lo_w && j0 + c + 1 <= pos;
                        const float a = w0 ? ex2(fmaf(sv[c], c2, -mlx)) : 0.f;
                        const float bb = w1 ? ex2(fmaf(sv[c + 1], c2, -mlx)) : 0.f;
                        sl0 += a;
                        sl1 += bb;
                        pk[e] = pack_bf16(a, bb);
                    }
                    tmem_st16(tS + 64 + 16 * qq, pk);
                }
            }
            // global branch: unselected keys become -inf in place (one select per key)
            float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
            if (diag) {
#pragma unroll
                for (int c = 0; c < 128; ++c) {
                    const bool sel = ((mwords[c >> 5] >> (c & 31)) & 1u) && (j0 + c <= pos);
                    sv[c] = sel ? sv[c] : -INFINITY;
                    m4[c & 3] = fmaxf(m4[c & 3], sv[c]);
                }
            } else {
#pragma unroll
                for (int c = 0; c < 128; ++c) {
                    sv[c] = ((mwords[c >> 5] >> (c & 31)) & 1u) ? sv[c] : -INFINITY;
                    m4[c & 3] = fmaxf(m4[c & 3], sv[c]);
                }
            }
            const float mxg2 = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * c2;
            if (__any_sync(0xffffffffu, mxg2 > mg + 8.0f)) {
                const float mn = fmaxf(mg, mxg2);
                if (j > 0) {
                    const float corr = (mn == -INFINITY || mg == -INFINITY) ? (mn == -INFINITY ? 1.f : 0.f) : ex2(mg - mn);
                    lg *= corr;
                    cg *= corr;
                    tmem_scale128(tOg, corr);
                }
                mg = mn;
            }
            // global P: masked keys are -inf, so 2^(-inf) = 0 needs no select
            const float mgx = mg == -INFINITY ? 0.f : mg;
            float a4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int c = qq * 32 + 2 * e;
                    const float a = ex2(fmaf(sv[c], c2, -mgx));
                    const float bb = ex2(fmaf(sv[c + 1], c2, -mgx));
                    a4[e & 1] += a;
                    a4[2 + (e & 1)] += bb;
                    pk[e] = pack_bf16(a, bb);
                }
                tmem_st16(tS + 16 * qq, pk);
            }
            const float sg0 = a4[0] + a4[2], sg1 = a4[1] + a4[3];
            tmem_wait_st();
            {
                const float y = (sg0 + sg1) - cg;
                const float t = lg + y;
                cg = (t - lg) - y;
                lg = t;
            }
            {
                const float y = (sl0 + sl1) - cl;
                const float t = ll + y;
                cl = (t - ll) - y;
                ll = t;
            }
            tc_fence_before();
            mbar_arrive(smem_u32(&bars->p_full));
        }
        const bool fin = __all_sync(0xffffffffu, ok && mbar_wait(smem_u32(&bars->o_final), 0, p.wait_ns, abort));
        if (fin) {
            tc_fence_after();
            const float ig = lg > 0.f ? 1.f / lg : 0.f;
            const float il = ll > 0.f ? 1.f / ll : 0.f;
            float sgate = 0.f;
            if (valid) {
                const float x = p.gate[((size_t)b * p.Lq + row) * p.Hq + h];
                sgate = 1.0f / (1.0f + expf(-x));
            }
            const size_t orow = (((size_t)b * p.Lq + row) * p.Hq + h) * HD;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t og[32], ol[32];
                tmem_ld32(tOg + 32 * c, og);
                tmem_ld32(tOl + 32 * c, ol);
                tmem_wait_ld();
                uint32_t po[16], pg[16], pl[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const float g0 = __uint_as_float(og[2 * e]) * ig, g1 = __uint_as_float(og[2 * e + 1]) * ig;
                    const float l0 = __uint_as_float(ol[2 * e]) * il, l1 = __uint_as_float(ol[2 * e + 1]) * il;
                    po[e] = pack_bf16(sgate * g0 + (1.f - sgate) * l0, sgate * g1 + (1.f - sgate) * l1);
                    pg[e] = pack_bf16(g0, g1);
                    pl[e] = pack_bf16(l0, l1);
                }
                if (valid) {
                    uint4 *d0 = reinterpret_cast<uint4 *>(p.out + orow + 32 * c);
#pragma unroll
                    for (int e = 0; e < 4; ++e) d0[e] = make_uint4(po[4 * e], po[4 * e + 1], po[4 * e + 2], po[4 * e + 3]);
                    if (p.out_g) {
                        uint4 *d1 = reinterpret_cast<uint4 *>(p.out_g + orow + 32 * c);
#pragma unroll
                        for (int e = 0; e < 4; ++e) d1[e] = make_uint4(pg[4 * e], pg[4 * e + 1], pg[4 * e + 2], pg[4 * e + 3]);
                    }
                    if (p.out_l) {
                        uint4 *d2 = reinterpret_cast<uint4 *>(p.out_l + orow + 32 * c);
#pragma unroll
                        for (int e = 0; e < 4; ++e) d2[e] = make_uint4(pl[4 * e], pl[4 * e + 1], pl[4 * e + 2], pl[4 * e + 3]);
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
    if (threadIdx.x == 0 && bars->abort) report(p.status, HS_ERR_TIMEOUT);
}

// One warp per (batch, KV head, row): the row's index list as a bitmask of W
// words (W = 4 * ceil(Lkv / 128)), built in shared memory, written once.
constexpr int SM_WARPS = 4;

__global__ void __launch_bounds__(SM_WARPS * 32)
build_selmask(const int32_t *__restrict__ idx, int topk, int Lq, int Lkv, int W, long long n_rows,
              uint32_t *__restrict__ mask, unsigned int *status) {
    extern __shared__ uint32_t words_all[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long r = (long long)blockIdx.x * SM_WARPS + warp;
    if (r >= n_rows) return;
    uint32_t *words = words_all + (size_t)warp * W;
    const int i = (int)(r % Lq);
    const int pos = Lkv - Lq + i;
    for (int t = lane; t < W; t += 32) words[t] = 0u;
    __syncwarp();
    const int32_t *lst = idx + r * topk;
    for (int t = lane; t < topk; t += 32) {
        const int j = __ldg(lst + t);
        if (j >= 0 && j <= pos)
            atomicOr(&words[j >> 5], 1u << (j & 31));
        else if (j != -1)
            report(status, HS_ERR_INVALID_INDEX);
    }
    __syncwarp();
    uint4 *dst = reinterpret_cast<uint4 *>(mask + r * W);
    for (int t = lane; t < W / 4; t += 32) dst[t] = reinterpret_cast<const uint4 *>(words)[t];
}

}  // namespace
}  // namespace tc

int selmask_words(const Shape &s) { return 4 * ((s.Lkv + tc::BN - 1) / tc::BN); }

size_t selmask_bytes(const Shape &s) {
    return (size_t)s.B * s.Hkv * s.Lq * (size_t)selmask_words(s) * sizeof(uint32_t);
}

bool sparse_dense_supported(const Shape &s) {
    return s.dtype == HS_BF16 && s.d == 128 && s.Lq >= 64 && selmask_words(s) * 4 * tc::SM_WARPS <= 96 * 1024;
}

cudaError_t selmask_build_launch(const Shape &s, const int32_t *idx, int topk, uint32_t *mask, unsigned int *status,
                                 cudaStream_t st) {
    using namespace tc;
    const int W = selmask_words(s);
    static bool attr = false;
    if (!attr) {
        cudaError_t e = cudaFuncSetAttribute(build_selmask, cudaFuncAttributeMaxDynamicSharedMemorySize, 96 * 1024);
        if (e != cudaSuccess) return e;
        attr = true;
    }
    const long long n_rows = (long long)s.B * s.Hkv * s.Lq;
    const long long mb = (n_rows + SM_WARPS - 1) / SM_WARPS;
    if (mb > 0x7fffffffLL) return cudaErrorInvalidValue;
    build_selmask<<<(unsigned)mb, SM_WARPS * 32, (size_t)SM_WARPS * W * 4, st>>>(idx, topk, s.Lq, s.Lkv, W, n_rows,
                                                                                mask, status); count_launch();
    return cudaGetLastError();
}

cudaError_t sparse_dense_tc_launch(const Shape &s, const void *q, const void *k, const void *v,
                                   const int32_t *idx, int topk, const float *gate, int window, void *out,
                                   void *og, void *ol, uint32_t *mask, unsigned int *status,
                                   unsigned long long wait_ns, cudaStream_t st) {
    using namespace tc;
    const int W = selmask_words(s);
    static bool attr = false;
    if (!attr) {
        cudaError_t e = cudaFuncSetAttribute(sparse_dense_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSdSmem);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(build_selmask, cudaFuncAttributeMaxDynamicSharedMemorySize, 96 * 1024);
        if (e != cudaSuccess) return e;
        attr = true;
    }
    const long long n_rows = (long long)s.B * s.Hkv * s.Lq;
    const long long mb = (n_rows + SM_WARPS - 1) / SM_WARPS;
    if (mb > 0x7fffffffLL) return cudaErrorInvalidValue;
    build_selmask<<<(unsigned)mb, SM_WARPS * 32, (size_t)SM_WARPS * W * 4, st>>>(idx, topk, s.Lq, s.Lkv, W, n_rows,
                                                                                mask, status); count_launch();
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, q, s.Hq, s.Lq, s.B) || !make_map(&mk, k, s.Hkv, s.Lkv, s.B) ||
        !make_map(&mv, v, s.Hkv, s.Lkv, s.B))
        return cudaErrorInvalidValue;
    SdParams p{s.Lq, s.Lkv, s.Hq, s.Hkv, s.G(), window, W, s.scale * kLog2e, mask, gate,
               (__nv_bfloat16 *)out, (__nv_bfloat16 *)og, (__nv_bfloat16 *)ol, status, wait_ns};
    const int n_tiles = (s.Lq + BM - 1) / BM;
    sparse_dense_tc<<<tile_grid(s.Hq, n_tiles, s.B), SD_THREADS, kSdSmem, st>>>(mq, mk, mv, p); count_launch();
    return cudaGetLastError();
}

}  // namespace hs
