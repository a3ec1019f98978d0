// Tensor-core (tcgen05 / TMEM / TMA) kernels for the full layer of the
// hybrid block, bf16 inputs, head dim 128:
//
//   attn_fwd_tc    : O and LSE (and per-row softmax statistics) of causal GQA
//                    attention, flash-style online softmax over 128-key tiles.
//   attn_scores_tc : the importance scores, a second pass over the keys that
//                    re-computes q.k on the tensor cores and turns it into
//                    exact probabilities with the saved statistics, summed
//                    over the query heads that share a KV head.
//
// Method: HySparse abstract (the full attention layer is the oracle that
// picks the tokens each following sparse layer attends to); the
// intelliparadigm write-up, section 2.1 (full layer as the hub that computes
// token importance) and section 3.1 (index sharing).  The tiling is the IO-
// aware exact attention the ultralytics glossary names (FlashAttention):
// online softmax, log-sum-exp saved for reuse.
//
// Forward kernel layout (one CTA = 128 query rows x 2 query heads of one KV
// group, so each K/V tile is loaded once for two Q tiles):
//   warps 0-3  softmax for Q tile 0 (thread t owns row t = TMEM lane t)
//   warps 4-7  softmax for Q tile 1
//   warp 8     TMA producer (Q tiles once, then K and V tiles through a
//              3-slot ring filled in the order the MMAs consume them)
//   warp 9     MMA issuer (one thread)
//   warps 10-11 idle; they complete the third warpgroup so that warps 8-11
//              can hand registers to the softmax warpgroups (setmaxnreg:
//              168 per thread at launch, then 104 for warps 8-11 and 200
//              for warps 0-7, which holds a row of S and its packed
//              f32x2 arithmetic without spills)
// TMEM (512 columns): S0 | S1 | O0 | O1, 128 f32 columns each.  P (bf16) goes
// to shared memory in the swizzled layout of a Q tile, so the softmax
// threads release S_j as soon as they have read it and S_{j+1} = Q K_{j+1}^T
// runs on the tensor cores while they are still turning S_j into P_j.
// The running max is only moved when it grows by more than 8 (log2 units);
// the final normalisation uses the same reference, so the result is exact.
#include <algorithm>
#include <cstring>

#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"
#include "tc_attn.cuh"
#include "tc_util.cuh"

namespace hs {
namespace tc {
namespace {

constexpr int FWD_KV = 3;   // K/V ring slots (shared memory also holds Q0, Q1, P0, P1)

struct FwdBars {
    uint64_t q_full;
    uint64_t kv_full[FWD_KV];
    uint64_t kv_empty[FWD_KV];
    uint64_t s_full[2];    // S_w holds Q_w K_j^T           (MMA commit)
    uint64_t s_free[2];    // softmax w has S_w in registers (128 arrivals)
    uint64_t p_full[2];    // P_w written to shared memory   (128 arrivals)
    uint64_t pv_done[2];   // O_w += P_w V_j completed; P_w buffer free (MMA commit)
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

constexpr size_t kFwdSmem = 1024 + 2 * TILE + FWD_KV * TILE + 2 * TILE + sizeof(FwdBars);
static_assert(kFwdSmem <= 232448, "forward kernel shared memory");

// What the pipeline computes.  FULL: causal attention of the full layer (O,
// LSE, statistics for the score pass).  WIN: the sparse layer's window
// branch (keys pos-window+1 .. pos), normalised into an fp32 buffer.  SEL:
// the sparse layer's global branch (keys in the row's top-k set), merged
// with the window branch by the gate into the layer output.
enum FwdMode { FWD_FULL = 0, FWD_WIN = 1, FWD_SEL = 2 };

struct FwdParams {
    int Lq, Lkv, Hq, Hkv, G;
    int row_begin, row_end;
    float scale_log2;
    __nv_bfloat16 *out;
    float *lse;
    float2 *stats;
    unsigned int *status;
    unsigned long long wait_ns;
    // sparse-layer modes
    int window, W;                   // window length; words per selection-mask row
    const uint32_t *selmask;         // [B][Hkv][Lq][W]
    uint32_t *wl;                    // [B][Lq][Hq][128] window branch, normalised, bf16 pairs
    const float *gate;               // [B][Lq][Hq]
    __nv_bfloat16 *out_g, *out_l;    // optional branch outputs
};

// O (+)= P V with P a 128x128 bf16 tile in shared memory (K-major, 128-byte
// swizzle, the layout of a Q tile) and V an N-major tile.
__device__ __forceinline__ void issue_pv_ss(uint32_t d_tmem, uint32_t p_addr, uint32_t v_addr, bool accumulate) {
    constexpr uint32_t I = idesc_bf16(128, 128, false, true);
#pragma unroll
    for (int kk = 0; kk < BN / 16; ++kk) {
        const uint32_t o = (kk >> 2) * HALF + (kk & 3) * 32;
        mma_ss(d_tmem, sdesc_sw128(p_addr + o, 16, 1024), sdesc_sw128(v_addr + kk * 2048, HALF, 1024), I,
               (accumulate || kk > 0) ? 1u : 0u);
    }
}

// KV ring order = MMA consumption order: K0, K1, V0, K2, V1, K3, V2, ...
// (S_{j+1} = Q K_{j+1}^T is issued before O += P_j V_j).
__device__ __forceinline__ int kv_seq_k(int j) { return j == 0 ? 0 : 2 * j - 1; }
__device__ __forceinline__ int kv_seq_v(int j, int n) { return j + 1 < n ? 2 * j + 2 : 2 * j + 1; }

template <int MODE>
__global__ void __launch_bounds__(FWD_THREADS, 1)
attn_fwd_tc(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
            const __grid_constant__ CUtensorMap tv, const FwdParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    uint8_t *sq = smem;
    uint8_t *skv = smem + 2 * TILE;
    uint8_t *sp = smem + 2 * TILE + FWD_KV * TILE;
    FwdBars *bars = reinterpret_cast<FwdBars *>(smem + 4 * TILE + FWD_KV * TILE);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int tile, b;
    tile_of_block((p.row_end - p.row_begin + BM - 1) / BM, tile, b);   // heaviest row tiles first
    const int r0 = p.row_begin + tile * BM;
    const int r_end = min(r0 + BM, p.row_end);
    const int h0 = 2 * blockIdx.x;
    const int g = h0 / p.G;
    const int off = p.Lkv - p.Lq;
    const int pos_first = off + r0;
    const int pos_last = off + r_end - 1;
    // key tiles j_begin .. j_begin + n_kv - 1 (the window mode skips tiles no
    // row's window reaches); loop counters below are relative to j_begin
    const int j_begin = MODE == FWD_WIN ? max(0, pos_first - p.window + 1) / BN : 0;
    const int n_kv = pos_last / BN + 1 - j_begin;

    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bars->q_full), 1);
        for (int s = 0; s < FWD_KV; ++s) {
            mbar_init(smem_u32(&bars->kv_full[s]), 1);
            mbar_init(smem_u32(&bars->kv_empty[s]), 1);
        }
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
        tmem_alloc(smem_u32(&bars->tmem_base), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    volatile int *abort = &bars->abort;
    if (warp >= 8) {
      regs_release<kFwdCtlRegs>();
      if (warp == 8) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch(&tq);
            tma_prefetch(&tk);
            tma_prefetch(&tv);
            const uint32_t qb = smem_u32(&bars->q_full);
            mbar_expect_tx(qb, 2 * TILE);
            for (int s = 0; s < 2; ++s)
                for (int hf = 0; hf < 2; ++hf)
                    tma_load_4d(smem_u32(sq + s * TILE + hf * HALF), &tq, qb, hf * 64, h0 + s, r0, b);
            int issued = 0;
            for (int it = 0; it < 2 * n_kv; ++it) {
                // sequence position -> which tile: 0 -> K0, then (K_{m+1}, V_m) pairs, last V_{n-1}
                int j, is_v;
                if (it == 0) { j = 0; is_v = 0; }
                else if (it == 2 * n_kv - 1) { j = n_kv - 1; is_v = 1; }
                else { is_v = (it & 1) == 0; j = is_v ? (it - 2) / 2 : (it + 1) / 2; }
                const int slot = it % FWD_KV, use = it / FWD_KV;
                if (!mbar_wait(smem_u32(&bars->kv_empty[slot]), (use & 1) ^ 1, p.wait_ns, abort)) break;
                const uint32_t fb = smem_u32(&bars->kv_full[slot]);
                mbar_expect_tx(fb, TILE);
                const CUtensorMap *m = is_v ? &tv : &tk;
                for (int hf = 0; hf < 2; ++hf)
                    tma_load_4d(smem_u32(skv + slot * TILE + hf * HALF), m, fb, hf * 64, g, (j_begin + j) * BN, b);
                issued = it + 1;
            }
            if (*abort) {  // let our own copies land before the CTA goes away
                mbar_drain(qb, 0);
                for (int it = issued > FWD_KV ? issued - FWD_KV : 0; it < issued; ++it)
                    mbar_drain(smem_u32(&bars->kv_full[it % FWD_KV]), (it / FWD_KV) & 1);
            }
        }
      } else if (warp == 9) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t tS[2] = {tmem, tmem + 128}, tO[2] = {tmem + 256, tmem + 384};
            const uint32_t qa[2] = {smem_u32(sq), smem_u32(sq + TILE)};
            const uint32_t pa[2] = {smem_u32(sp), smem_u32(sp + TILE)};
            bool ok = mbar_wait(smem_u32(&bars->q_full), 0, p.wait_ns, abort);
            if (ok) ok = mbar_wait(smem_u32(&bars->kv_full[0]), 0, p.wait_ns, abort);
            if (ok) {
                tc_fence_after();
                for (int w = 0; w < 2; ++w) {
                    issue_qk(tS[w], qa[w], smem_u32(skv));
                    mma_commit(smem_u32(&bars->s_full[w]));
                }
                mma_commit(smem_u32(&bars->kv_empty[0]));
            }
            for (int j = 0; ok && j < n_kv; ++j) {
                if (j + 1 < n_kv) {
                    const int itK = kv_seq_k(j + 1), sk = itK % FWD_KV;
                    if (!(ok = mbar_wait(smem_u32(&bars->kv_full[sk]), (itK / FWD_KV) & 1, p.wait_ns, abort))) break;
                    for (int w = 0; w < 2; ++w) {
                        if (!(ok = mbar_wait(smem_u32(&bars->s_free[w]), j & 1, p.wait_ns, abort))) break;
                        tc_fence_after();
                        issue_qk(tS[w], qa[w], smem_u32(skv + sk * TILE));
                        mma_commit(smem_u32(&bars->s_full[w]));
                    }
                    if (!ok) break;
                    mma_commit(smem_u32(&bars->kv_empty[sk]));
                }
                const int itV = kv_seq_v(j, n_kv), sv = itV % FWD_KV;
                if (!(ok = mbar_wait(smem_u32(&bars->kv_full[sv]), (itV / FWD_KV) & 1, p.wait_ns, abort))) break;
                for (int w = 0; w < 2; ++w) {
                    if (!(ok = mbar_wait(smem_u32(&bars->p_full[w]), j & 1, p.wait_ns, abort))) break;
                    tc_fence_after();
                    issue_pv_ss(tO[w], pa[w], smem_u32(skv + sv * TILE), j > 0);
                    mma_commit(smem_u32(&bars->pv_done[w]));
                }
                if (!ok) break;
                mma_commit(smem_u32(&bars->kv_empty[sv]));
            }
            // all MMAs this thread issued have completed before TMEM is freed
            mma_commit(smem_u32(&bars->drain));
            mbar_drain(smem_u32(&bars->drain), 0);
        }
      }
    } else {
        regs_acquire<kFwdSoftRegs>();
        // ------------------------------------------------ softmax warpgroups
        const int w = warp >> 2;
        const int tw = threadIdx.x - 128 * w;
        const int row = r0 + tw;
        const bool valid = row < r_end;
        const int pos = off + min(row, r_end - 1);
        const uint32_t lane_off = (uint32_t)(tw & ~31) << 16;
        const uint32_t tS = tmem + lane_off + (uint32_t)(w * 128);
        const uint32_t tO = tmem + lane_off + 256u + (uint32_t)(w * 128);
        uint8_t *prow = sp + w * TILE + tw * 128;      // this row of P (two 16 KB halves)
        const int sw = tw & 7;                          // 128-byte swizzle phase of the row
        const float c2 = p.scale_log2;
        const int lo_w = max(0, pos - p.window + 1);     // window mode: first key of the row's window
        const uint4 *mrow = nullptr;                      // select mode: the row's top-k bitmask
        uint4 mw = make_uint4(0, 0, 0, 0);
        if (MODE == FWD_SEL) {
            mrow = reinterpret_cast<const uint4 *>(p.selmask + (((size_t)b * p.Hkv + g) * p.Lq + (pos - off)) * p.W);
            mw = __ldg(mrow);
        }
        float m = -INFINITY, l = 0.f, lc = 0.f;
        bool ok = true;
        for (int j = 0; j < n_kv; ++j) {
            const int j0 = (j_begin + j) * BN;           // key index of column 0
            uint32_t mwords[4] = {mw.x, mw.y, mw.z, mw.w};
            if (MODE == FWD_SEL && j + 1 < n_kv) mw = __ldg(mrow + j + 1);
            ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bars->s_full[w]), j & 1, p.wait_ns, abort));
            if (!ok) break;
            tc_fence_after();
            float s[128];
            {
                uint32_t r[4][32];
#pragma unroll
                for (int c = 0; c < 4; ++c) tmem_ld32(tS + 32 * c, r[c]);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 128; ++c) s[c] = __uint_as_float(r[c >> 5][c & 31]);
            }
            tc_fence_before();
            mbar_arrive(smem_u32(&bars->s_free[w]));       // the MMA may now write S_{j+1}
            if (MODE == FWD_SEL) {
                if (j0 + BN - 1 > pos_first) {
#pragma unroll
                    for (int c = 0; c < 128; ++c)
                        if (!((mwords[c >> 5] >> (c & 31)) & 1u) || j0 + c > pos) s[c] = -INFINITY;
                } else {
#pragma unroll
                    for (int c = 0; c < 128; ++c)
                        if (!((mwords[c >> 5] >> (c & 31)) & 1u)) s[c] = -INFINITY;
                }
            } else if (MODE == FWD_WIN) {
#pragma unroll
                for (int c = 0; c < 128; ++c)
                    if (j0 + c > pos || j0 + c < lo_w) s[c] = -INFINITY;
            } else if (j0 + BN - 1 > pos_first) {
#pragma unroll
                for (int c = 0; c < 128; ++c)
                    if (j0 + c > pos) s[c] = -INFINITY;
            }
            float m4[4] = {s[0], s[1], s[2], s[3]};
#pragma unroll
            for (int c = 4; c < 128; c += 2) m4[(c >> 1) & 3] = fmax3(m4[(c >> 1) & 3], s[c], s[c + 1]);
            const float mx2 = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * c2;
            // PV of the previous tile done: O is stable and the P buffer is free
            if (j > 0) {
                ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bars->pv_done[w]), (j - 1) & 1, p.wait_ns, abort));
                if (!ok) break;
                tc_fence_after();
            }
            if (__any_sync(0xffffffffu, mx2 > m + 8.0f)) {
                const float m_new = fmaxf(m, mx2);
                if (j > 0) {
                    // a row with nothing visible yet has m = -inf and an all-zero O row
                    const float corr = m_new == -INFINITY ? 1.f : ex2(m - m_new);
                    l *= corr;
                    lc *= corr;
#pragma unroll 1
                    for (int c = 0; c < 8; ++c) {
                        uint32_t o[16];
                        tmem_ld16(tO + 16 * c, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * corr);
                        tmem_st16(tO + 16 * c, o);
                    }
                    tmem_wait_st();
                }
                m = m_new;
            }
            const float mref = m == -INFINITY ? 0.f : m;   // masked keys (-inf) give 2^-inf = 0
            const float2 c2v = make_float2(c2, c2), mv = make_float2(-mref, -mref);
            float2 ps01 = make_float2(0.f, 0.f), ps23 = make_float2(0.f, 0.f);
#pragma unroll
            for (int ch = 0; ch < 16; ++ch) {           // 16-byte chunks of 8 keys
                uint32_t pk[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int c = ch * 8 + 2 * e;
                    const float2 t = ffma2(make_float2(s[c], s[c + 1]), c2v, mv);
                    const float2 ab = make_float2(ex2(t.x), ex2(t.y));
                    if (e & 1) ps23 = fadd2(ps23, ab); else ps01 = fadd2(ps01, ab);
                    pk[e] = pack_bf16(ab.x, ab.y);
                }
                const int half = ch >> 3, c8 = ch & 7;
                *reinterpret_cast<uint4 *>(prow + half * HALF + ((c8 ^ sw) << 4)) =
                    make_uint4(pk[0], pk[1], pk[2], pk[3]);
            }
            fence_proxy_async_smem();
            mbar_arrive(smem_u32(&bars->p_full[w]));
            const float ts = (ps01.x + ps01.y) + (ps23.x + ps23.y);
            const float y = ts - lc;
            const float t = l + y;
            lc = (t - l) - y;
            l = t;
        }
        const bool fin = __all_sync(0xffffffffu, ok && mbar_wait(smem_u32(&bars->pv_done[w]), (n_kv - 1) & 1,
                                                                 p.wait_ns, abort));
        if (fin && MODE == FWD_FULL) {
            tc_fence_after();
            const int h = h0 + w;
            const float inv_l = 1.0f / l;
            __nv_bfloat16 *orow = p.out + (((size_t)b * p.Lq + row) * p.Hq + h) * HD;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t o[32];
                tmem_ld32(tO + 32 * c, o);
                tmem_wait_ld();
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    pk[e] = pack_bf16(__uint_as_float(o[2 * e]) * inv_l, __uint_as_float(o[2 * e + 1]) * inv_l);
                if (valid) {
                    uint4 *dst = reinterpret_cast<uint4 *>(orow + 32 * c);
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
                }
            }
            if (valid) {
                const size_t si = ((size_t)b * p.Hq + h) * p.Lq + row;
                p.lse[si] = (m + log2f(l)) * kLn2;
                if (p.stats) p.stats[si] = make_float2(m, inv_l);
            }
        }
        if (!fin && MODE == FWD_FULL && valid) {
            // a bounded wait gave up: mark the row's LSE, which callers own,
            // so that the timeout is visible without the workspace status word
            p.lse[((size_t)b * p.Hq + h0 + w) * p.Lq + row] = __int_as_float(0x7fc00000);
        }
        if (fin && MODE == FWD_WIN) {
            // normalised window branch, bf16 (the precision of the branch
            // output), for the select pass to merge
            tc_fence_after();
            const int h = h0 + w;
            const float inv_l = l > 0.f ? 1.0f / l : 0.f;
            uint4 *wrow = reinterpret_cast<uint4 *>(p.wl + (((size_t)b * p.Lq + row) * p.Hq + h) * (HD / 2));
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t o[32];
                tmem_ld32(tO + 32 * c, o);
                tmem_wait_ld();
                if (valid) {
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        wrow[4 * c + e] = make_uint4(
                            pack_bf16(__uint_as_float(o[8 * e]) * inv_l, __uint_as_float(o[8 * e + 1]) * inv_l),
                            pack_bf16(__uint_as_float(o[8 * e + 2]) * inv_l, __uint_as_float(o[8 * e + 3]) * inv_l),
                            pack_bf16(__uint_as_float(o[8 * e + 4]) * inv_l, __uint_as_float(o[8 * e + 5]) * inv_l),
                            pack_bf16(__uint_as_float(o[8 * e + 6]) * inv_l, __uint_as_float(o[8 * e + 7]) * inv_l));
                }
            }
        }
        if (fin && MODE == FWD_SEL) {
            // out = sigmoid(gate) * global + (1 - sigmoid(gate)) * window
            tc_fence_after();
            const int h = h0 + w;
            const float inv_l = l > 0.f ? 1.0f / l : 0.f;   // an empty top-k set gives a zero branch
            const size_t ro = ((size_t)b * p.Lq + row) * p.Hq + h;
            float sg = 0.f;
            if (valid) sg = 1.0f / (1.0f + expf(-p.gate[ro]));
            const uint4 *wrow = reinterpret_cast<const uint4 *>(p.wl + ro * (HD / 2));
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t o[32];
                tmem_ld32(tO + 32 * c, o);
                tmem_wait_ld();
                if (valid) {
                    uint32_t po[16], pg[16], pl[16];
                    uint32_t wq[16];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const uint4 t4 = wrow[4 * c + e];
                        wq[4 * e] = t4.x; wq[4 * e + 1] = t4.y; wq[4 * e + 2] = t4.z; wq[4 * e + 3] = t4.w;
                    }
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float4 wv = make_float4(__uint_as_float(wq[2 * e] << 16), __uint_as_float(wq[2 * e] & 0xffff0000u),
                                                      __uint_as_float(wq[2 * e + 1] << 16),
                                                      __uint_as_float(wq[2 * e + 1] & 0xffff0000u));
                        const float g0 = __uint_as_float(o[4 * e]) * inv_l, g1 = __uint_as_float(o[4 * e + 1]) * inv_l;
                        const float g2 = __uint_as_float(o[4 * e + 2]) * inv_l, g3 = __uint_as_float(o[4 * e + 3]) * inv_l;
                        po[2 * e] = pack_bf16(sg * g0 + (1.f - sg) * wv.x, sg * g1 + (1.f - sg) * wv.y);
                        po[2 * e + 1] = pack_bf16(sg * g2 + (1.f - sg) * wv.z, sg * g3 + (1.f - sg) * wv.w);
                        pg[2 * e] = pack_bf16(g0, g1);
                        pg[2 * e + 1] = pack_bf16(g2, g3);
                        pl[2 * e] = wq[2 * e];
                        pl[2 * e + 1] = wq[2 * e + 1];
                    }
                    uint4 *d0 = reinterpret_cast<uint4 *>(p.out + ro * HD + 32 * c);
#pragma unroll
                    for (int e = 0; e < 4; ++e) d0[e] = make_uint4(po[4 * e], po[4 * e + 1], po[4 * e + 2], po[4 * e + 3]);
                    if (p.out_g) {
                        uint4 *d1 = reinterpret_cast<uint4 *>(p.out_g + ro * HD + 32 * c);
#pragma unroll
                        for (int e = 0; e < 4; ++e) d1[e] = make_uint4(pg[4 * e], pg[4 * e + 1], pg[4 * e + 2], pg[4 * e + 3]);
                    }
                    if (p.out_l) {
                        uint4 *d2 = reinterpret_cast<uint4 *>(p.out_l + ro * HD + 32 * c);
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

// ------------------------------------------------------------------ scores

constexpr int SC_Q_STAGES = 4;   // Q slots: all G query tiles stay resident when G <= 4, else a ring
constexpr int SC_K_STAGES = 2;
constexpr int kScUnitsPerSm = 6;   // key-segment CTAs per SM a score launch aims for
constexpr int kScMinSeg = 8;       // fewest key tiles per CTA (its Q tiles are loaded once per CTA)
constexpr int SC_BUFS = 4;
// warps 0-15 scores (four per TMEM lane quarter, 32 columns each), 16 TMA, 17 MMA
constexpr int SC_SCORE_WARPS = 16;
constexpr int SC_TMA_WARP = SC_SCORE_WARPS, SC_MMA_WARP = SC_SCORE_WARPS + 1;
constexpr int SC_THREADS = 32 * (SC_SCORE_WARPS + 2);
// Score staging for the bulk tensor stores: per score warp one 2 KB buffer,
// a 32-row x 16-column fp32 box in the 64-byte swizzled layout.
constexpr int SC_STG_BYTES = 2048;
constexpr int SC_STG_TOTAL = SC_SCORE_WARPS * SC_STG_BYTES;

struct ScBars {
    uint64_t q_full[SC_Q_STAGES], q_empty[SC_Q_STAGES];
    uint64_t k_full[SC_K_STAGES], k_empty[SC_K_STAGES];
    uint64_t s_full[SC_BUFS], s_free[SC_BUFS];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

constexpr size_t kScSmem = 1024 + (SC_Q_STAGES + SC_K_STAGES) * TILE + SC_STG_TOTAL + sizeof(ScBars);

struct ScParams {
    int Lq, Lkv, Hq, Hkv, G;
    int row_begin, row_end, row_count;
    float scale_log2;
    const float2 *stats;
    float *scores;
    long long ld;
    unsigned int *status;
    unsigned long long wait_ns;
    float *lse;      // [B][Hq][Lq]: set to NaN for this tile's rows and heads if a wait gives up
    int tma_store;   // scores leave through `ts` (bulk tensor stores) rather than per-thread stores
    int kv_seg;      // key tiles per CTA: blockIdx.x = segment * Hkv + KV head
};

__global__ void __launch_bounds__(SC_THREADS, 1)
attn_scores_tc(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
               const __grid_constant__ CUtensorMap ts, const ScParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    uint8_t *sq = smem;
    uint8_t *sk = smem + SC_Q_STAGES * TILE;
    uint8_t *sst = smem + (SC_Q_STAGES + SC_K_STAGES) * TILE;
    ScBars *bars = reinterpret_cast<ScBars *>(sst + SC_STG_TOTAL);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int tile, b;
    tile_of_block((p.row_end - p.row_begin + BM - 1) / BM, tile, b);   // heaviest row tiles first
    const int r0 = p.row_begin + tile * BM;
    const int r_end = min(r0 + BM, p.row_end);
    // The scores of different keys are independent once the forward pass has
    // saved each row's statistics, so a row tile's causal key range is split
    // into segments of kv_seg tiles, one CTA each: the grid fills the SMs
    // even when a row chunk has few row tiles.
    const int g = blockIdx.x % p.Hkv;
    const int j_begin = (blockIdx.x / p.Hkv) * p.kv_seg;
    const int G = p.G;
    const bool resident = G <= SC_Q_STAGES;
    const int off = p.Lkv - p.Lq;
    const int pos_last = off + r_end - 1;
    if (j_begin > pos_last / BN) return;   // segment past this row tile's causal end: nothing set up yet
    const int n_kv = min(pos_last / BN + 1 - j_begin, p.kv_seg);   // key tiles j_begin .. j_begin + n_kv - 1

    if (threadIdx.x == 0) {
        for (int s = 0; s < SC_Q_STAGES; ++s) {
            mbar_init(smem_u32(&bars->q_full[s]), 1);
            mbar_init(smem_u32(&bars->q_empty[s]), 1);
        }
        for (int s = 0; s < SC_K_STAGES; ++s) {
            mbar_init(smem_u32(&bars->k_full[s]), 1);
            mbar_init(smem_u32(&bars->k_empty[s]), 1);
        }
        for (int s = 0; s < SC_BUFS; ++s) {
            mbar_init(smem_u32(&bars->s_full[s]), 1);
            mbar_init(smem_u32(&bars->s_free[s]), 32 * SC_SCORE_WARPS);
        }
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

    if (warp == SC_TMA_WARP) {
        if (lane == 0) {
            tma_prefetch(&tq);
            tma_prefetch(&tk);
            int k_issued = 0, q_issued = 0;
            bool ok = true;
            if (resident) {
                for (int hh = 0; hh < G; ++hh) {
                    const uint32_t qb = smem_u32(&bars->q_full[hh]);
                    mbar_expect_tx(qb, TILE);
                    for (int hf = 0; hf < 2; ++hf)
                        tma_load_4d(smem_u32(sq + hh * TILE + hf * HALF), &tq, qb, hf * 64, g * G + hh, r0, b);
                }
            }
            for (int j = 0; ok && j < n_kv; ++j) {
                const int sk_ = j % SC_K_STAGES;
                if (!(ok = mbar_wait(smem_u32(&bars->k_empty[sk_]), ((j / SC_K_STAGES) & 1) ^ 1, p.wait_ns, abort))) break;
                const uint32_t kb = smem_u32(&bars->k_full[sk_]);
                mbar_expect_tx(kb, TILE);
                for (int hf = 0; hf < 2; ++hf)
                    tma_load_4d(smem_u32(sk + sk_ * TILE + hf * HALF), &tk, kb, hf * 64, g, (j_begin + j) * BN, b);
                k_issued = j + 1;
                for (int hh = 0; !resident && hh < G; ++hh) {
                    const int it = j * G + hh, sq_ = it % SC_Q_STAGES;
                    if (!(ok = mbar_wait(smem_u32(&bars->q_empty[sq_]), ((it / SC_Q_STAGES) & 1) ^ 1, p.wait_ns, abort))) break;
                    const uint32_t qb = smem_u32(&bars->q_full[sq_]);
                    mbar_expect_tx(qb, TILE);
                    for (int hf = 0; hf < 2; ++hf)
                        tma_load_4d(smem_u32(sq + sq_ * TILE + hf * HALF), &tq, qb, hf * 64, g * G + hh, r0, b);
                    q_issued = it + 1;
                }
            }
            if (*abort) {
                for (int j = k_issued > SC_K_STAGES ? k_issued - SC_K_STAGES : 0; j < k_issued; ++j)
                    mbar_drain(smem_u32(&bars->k_full[j % SC_K_STAGES]), (j / SC_K_STAGES) & 1);
                if (resident)
                    for (int hh = 0; hh < G; ++hh) mbar_drain(smem_u32(&bars->q_full[hh]), 0);
                for (int it = q_issued > SC_Q_STAGES ? q_issued - SC_Q_STAGES : 0; it < q_issued; ++it)
                    mbar_drain(smem_u32(&bars->q_full[it % SC_Q_STAGES]), (it / SC_Q_STAGES) & 1);
            }
        }
    } else if (warp == SC_MMA_WARP) {
        if (lane == 0) {
            bool ok = true;
            for (int j = 0; ok && j < n_kv; ++j) {
                const int sk_ = j % SC_K_STAGES;
                if (!(ok = mbar_wait(smem_u32(&bars->k_full[sk_]), (j / SC_K_STAGES) & 1, p.wait_ns, abort))) break;
                const uint32_t ka = smem_u32(sk + sk_ * TILE);
                for (int hh = 0; hh < G; ++hh) {
                    const int it = j * G + hh, buf = it % SC_BUFS;
                    const int sq_ = resident ? hh : it % SC_Q_STAGES;
                    if (!resident || j == 0) {
                        const uint32_t par = resident ? 0u : (uint32_t)((it / SC_Q_STAGES) & 1);
                        if (!(ok = mbar_wait(smem_u32(&bars->q_full[sq_]), par, p.wait_ns, abort))) break;
                    }
                    if (!(ok = mbar_wait(smem_u32(&bars->s_free[buf]), ((it / SC_BUFS) & 1) ^ 1, p.wait_ns, abort))) break;
                    tc_fence_after();
                    issue_qk(tmem + (uint32_t)(buf * 128), smem_u32(sq + sq_ * TILE), ka);
                    mma_commit(smem_u32(&bars->s_full[buf]));
                    if (!resident) mma_commit(smem_u32(&bars->q_empty[sq_]));
                }
                if (ok) mma_commit(smem_u32(&bars->k_empty[sk_]));
            }
            mma_commit(smem_u32(&bars->drain));
            mbar_drain(smem_u32(&bars->drain), 0);
        }
    } else {
        // ------------------------------------------------ score warps
        // warp w serves TMEM lanes 32*(w%4) .. +31 and columns 32*(w/4) .. +31
        const int q4 = warp & 3, cq = warp >> 2;
        const int tw = 32 * q4 + lane;
        const int row = r0 + tw;
        const bool valid = row < r_end;
        const int pos = off + min(row, r_end - 1);
        const uint32_t lane_off = (uint32_t)(32 * q4) << 16;
        const uint32_t colq = (uint32_t)(32 * cq);
        const float c2 = p.scale_log2;
        float *srow = valid ? p.scores + (((size_t)b * p.Hkv + g) * p.row_count + (row - p.row_begin)) * p.ld
                            : nullptr;
        const bool vec4 = (p.ld & 3) == 0;
        uint8_t *stg = sst + warp * SC_STG_BYTES;
        const int srow0 = r0 - p.row_begin + 32 * q4;       // this warp's first row within the chunk
        const int zbg = b * p.Hkv + g;
        const int sw = (lane >> 1) & 3;                      // 64-byte swizzle phase of this thread's row
        // the per-(row, head) statistics are loaded one head ahead
        const size_t st0 = ((size_t)b * p.Hq + (size_t)g * G) * p.Lq + row;
        float2 st_next = valid ? p.stats[st0] : make_float2(0.f, 0.f);
        bool ok = true;
        for (int j = 0; ok && j < n_kv; ++j) {
            float acc[32];
#pragma unroll
            for (int c = 0; c < 32; ++c) acc[c] = 0.f;
            for (int hh = 0; hh < G; ++hh) {
                const int it = j * G + hh, buf = it % SC_BUFS;
                const float2 st = st_next;
                const int hn = hh + 1 < G ? hh + 1 : 0;
                if (valid) st_next = p.stats[st0 + (size_t)hn * p.Lq];
                ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bars->s_full[buf]), (it / SC_BUFS) & 1, p.wait_ns, abort));
                if (!ok) break;
                tc_fence_after();
                uint32_t r[32];
                tmem_ld32(tmem + lane_off + (uint32_t)(buf * 128) + colq, r);
                tmem_wait_ld();
                tc_fence_before();
                mbar_arrive(smem_u32(&bars->s_free[buf]));   // S is in registers; the MMA may reuse the buffer
                const float2 c2v = make_float2(c2, c2), mv = make_float2(-st.x, -st.x), lv = make_float2(st.y, st.y);
#pragma unroll
                for (int c = 0; c < 32; c += 2) {
                    const float2 t = ffma2(make_float2(__uint_as_float(r[c]), __uint_as_float(r[c + 1])), c2v, mv);
                    const float2 e = make_float2(ex2(t.x), ex2(t.y));
                    const float2 a2 = ffma2(e, lv, make_float2(acc[c], acc[c + 1]));
                    acc[c] = a2.x;
                    acc[c + 1] = a2.y;
                }
            }
            if (!ok) break;
            const int j0 = (j_begin + j) * BN + 32 * cq;
            const int keep = pos - j0 + 1;                  // causal columns of this row in the 32
            if (p.tma_store) {
                // 2 boxes of 32 rows x 16 columns through the staging buffer
#pragma unroll
                for (int rnd = 0; rnd < 2; ++rnd) {
                    if (lane == 0) bulk_wait_read<0>();     // the previous store has read the buffer
                    __syncwarp();
#pragma unroll
                    for (int c4 = 0; c4 < 4; ++c4) {
                        const int c = 16 * rnd + 4 * c4;
                        const float4 v4 = make_float4(c < keep ? acc[c] : 0.f, c + 1 < keep ? acc[c + 1] : 0.f,
                                                      c + 2 < keep ? acc[c + 2] : 0.f, c + 3 < keep ? acc[c + 3] : 0.f);
                        *reinterpret_cast<float4 *>(stg + lane * 64 + ((c4 ^ sw) << 4)) = v4;
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    const int x0 = j0 + 16 * rnd;
                    if (lane == 0 && x0 < p.Lkv && srow0 < p.row_count) {
                        tma_store_3d(&ts, smem_u32(stg), x0, srow0, zbg);
                        bulk_commit();
                    }
                }
            } else if (valid) {
                const int lim = min(32, p.Lkv - j0);      // columns inside the cache
                float *dst = srow + j0;
                if (lim > 0) {
                    if (vec4 && lim == 32) {
#pragma unroll
                        for (int c = 0; c < 32; c += 4) {
                            float4 v4 = make_float4(c < keep ? acc[c] : 0.f, c + 1 < keep ? acc[c + 1] : 0.f,
                                                    c + 2 < keep ? acc[c + 2] : 0.f, c + 3 < keep ? acc[c + 3] : 0.f);
                            *reinterpret_cast<float4 *>(dst + c) = v4;
                        }
                    } else {
#pragma unroll
                        for (int c = 0; c < 32; ++c)
                            if (c < lim) dst[c] = c < keep ? acc[c] : 0.f;
                    }
                }
            }
        }
        if (p.tma_store && lane == 0) bulk_wait_all();   // scores written before the CTA retires
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
    if (bars->abort) {
        // a bounded wait gave up: this tile's scores are undefined; mark the
        // LSE of its rows and heads (caller-owned) so that the timeout is visible
        for (int e = threadIdx.x; e < G * BM; e += blockDim.x) {
            const int row = r0 + (e & (BM - 1));
            if (row < r_end) p.lse[((size_t)b * p.Hq + g * G + (e >> 7)) * p.Lq + row] = __int_as_float(0x7fc00000);
        }
        if (threadIdx.x == 0) report(p.status, HS_ERR_TIMEOUT);
    }
}

// ----------------------------------------------------------------- host side

}  // namespace
}  // namespace tc

bool full_attn_tc_supported(const Shape &s) {
    return s.dtype == HS_BF16 && s.d == 128 && (s.G() % 2) == 0 && s.Lkv < (1 << 24);
}

// One-time set-up of a forward instantiation: its dynamic shared memory, and
// a check that it is launched with exactly the registers per thread that the
// in-kernel hand-over between warpgroups is sized for (with fewer, the
// softmax warpgroups' increase could never be satisfied).
template <int MODE>
static cudaError_t fwd_prepare() {
    using namespace tc;
    cudaError_t e = cudaFuncSetAttribute(attn_fwd_tc<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kFwdSmem);
    if (e != cudaSuccess) return e;
    cudaFuncAttributes a;
    e = cudaFuncGetAttributes(&a, attn_fwd_tc<MODE>);
    if (e != cudaSuccess) return e;
    return a.numRegs == kFwdLaunchRegs ? cudaSuccess : cudaErrorInvalidDeviceFunction;
}

// SMs of the current device, read once per device.
static int num_sms() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (cached[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cached[dev] = n;
    }
    return cached[dev];
}

cudaError_t full_attn_scores_tc_launch(const Shape &s, const void *q, const void *k, const void *v,
                                       void *out, float *lse, float *scores, long long ld,
                                       int row_begin, int row_count, float2 *stats,
                                       unsigned int *status, unsigned long long wait_ns,
                                       cudaStream_t st) {
    using namespace tc;
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, q, s.Hq, s.Lq, s.B) || !make_map(&mk, k, s.Hkv, s.Lkv, s.B) ||
        !make_map(&mv, v, s.Hkv, s.Lkv, s.B))
        return cudaErrorInvalidValue;
    static bool attr_done = false;
    if (!attr_done) {
        cudaError_t e = fwd_prepare<FWD_FULL>();
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(attn_scores_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kScSmem);
        if (e != cudaSuccess) return e;
        attr_done = true;
    }
    const int n_tiles = (row_count + BM - 1) / BM;
    FwdParams fp{};
    fp.Lq = s.Lq; fp.Lkv = s.Lkv; fp.Hq = s.Hq; fp.Hkv = s.Hkv; fp.G = s.G();
    fp.row_begin = row_begin; fp.row_end = row_begin + row_count;
    fp.scale_log2 = s.scale * kLog2e;
    fp.out = (__nv_bfloat16 *)out; fp.lse = lse; fp.stats = stats; fp.status = status; fp.wait_ns = wait_ns;
    attn_fwd_tc<FWD_FULL><<<tile_grid(s.Hq / 2, n_tiles, s.B), FWD_THREADS, kFwdSmem, st>>>(mq, mk, mv, fp); count_launch();
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || scores == nullptr) return e;
    ScParams sp{s.Lq, s.Lkv, s.Hq, s.Hkv, s.G(), row_begin, row_begin + row_count, row_count,
                s.scale * kLog2e, stats, scores, ld, status, wait_ns, lse, 0, 0};
    // One CTA per (row tile, KV head) while the heaviest row tile is well
    // under an SM's share of the chunk's causal (row tile, key tile) pairs;
    // otherwise key segments, about kScUnitsPerSm CTAs per SM of at least
    // kScMinSeg key tiles each (measured: splitting a grid that is already
    // balanced costs a few percent in Q reloads and CTA start-up).
    const long long off = (long long)s.Lkv - s.Lq;
    long long pairs = 0;
    for (int t = 0; t < n_tiles; ++t)
        pairs += (off + min(row_begin + (t + 1) * BM, row_begin + row_count) - 1) / BN + 1;
    const long long total = pairs * s.Hkv * s.B;
    const int n_kv_max = (int)((off + row_begin + row_count - 1) / BN + 1);
    sp.kv_seg = n_kv_max;
    if (3ll * n_kv_max * num_sms() > 2 * total) {
        const long long units = (long long)kScUnitsPerSm * num_sms();
        sp.kv_seg = (int)std::min<long long>(n_kv_max, std::max<long long>(kScMinSeg, (total + units - 1) / units));
    }
    const int n_seg = (n_kv_max + sp.kv_seg - 1) / sp.kv_seg;
    // scores [B][Hkv][row_count][ld] f32 as a 3-D map (key, row, batch*KV head)
    // with 16 x 32 boxes in the 64-byte swizzle; needs 16-byte aligned rows
    CUtensorMap ms;
    memset(&ms, 0, sizeof(ms));
    if ((ld & 3) == 0 && (reinterpret_cast<uintptr_t>(scores) & 15u) == 0) {
        auto enc = encode_fn();
        cuuint64_t dims[3] = {(cuuint64_t)s.Lkv, (cuuint64_t)row_count, (cuuint64_t)s.B * s.Hkv};
        cuuint64_t strides[2] = {(cuuint64_t)ld * 4, (cuuint64_t)ld * 4 * row_count};
        cuuint32_t box[3] = {16, 32, 1};
        cuuint32_t es[3] = {1, 1, 1};
        if (enc && enc(&ms, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, scores, dims, strides, box, es,
                       CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                       CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS)
            sp.tma_store = 1;
    }
    attn_scores_tc<<<tile_grid(s.Hkv * n_seg, n_tiles, s.B), SC_THREADS, kScSmem, st>>>(mq, mk, ms, sp); count_launch();
    return cudaGetLastError();
}

bool sparse_pair_supported(const Shape &s) {
    return s.dtype == HS_BF16 && s.d == 128 && (s.G() % 2) == 0 && s.Lq >= 64;
}

size_t sparse_pair_wl_bytes(const Shape &s) { return (size_t)s.B * s.Lq * s.Hq * 128 * sizeof(uint16_t); }

cudaError_t sparse_pair_tc_launch(const Shape &s, const void *q, const void *k, const void *v, const float *gate,
                                  int window, void *out, void *og, void *ol, const uint32_t *mask, int W,
                                  uint32_t *wl, unsigned int *status, unsigned long long wait_ns, cudaStream_t st) {
    using namespace tc;
    CUtensorMap mq, mk, mv, mkw, mvw;
    if (!make_map(&mq, q, s.Hq, s.Lq, s.B) || !make_map(&mk, k, s.Hkv, s.Lkv, s.B) ||
        !make_map(&mv, v, s.Hkv, s.Lkv, s.B))
        return cudaErrorInvalidValue;
    // a layer with its own window K/V (one row per cache position, so the
    // same [B][Lkv][Hkv][d] extent) reads the window pass from that buffer
    if (s.k_win != nullptr) {
        if (s.Lwin != s.Lkv || !make_map(&mkw, s.k_win, s.Hkv, s.Lkv, s.B) ||
            !make_map(&mvw, s.v_win, s.Hkv, s.Lkv, s.B))
            return cudaErrorInvalidValue;
    } else {
        mkw = mk;
        mvw = mv;
    }
    static bool attr_done = false;
    if (!attr_done) {
        cudaError_t e = fwd_prepare<FWD_WIN>();
        if (e != cudaSuccess) return e;
        e = fwd_prepare<FWD_SEL>();
        if (e != cudaSuccess) return e;
        attr_done = true;
    }
    FwdParams fp{};
    fp.Lq = s.Lq; fp.Lkv = s.Lkv; fp.Hq = s.Hq; fp.Hkv = s.Hkv; fp.G = s.G();
    fp.row_begin = 0; fp.row_end = s.Lq;
    fp.scale_log2 = s.scale * kLog2e;
    fp.out = (__nv_bfloat16 *)out; fp.status = status; fp.wait_ns = wait_ns;
    fp.window = window; fp.W = W; fp.selmask = mask; fp.wl = wl; fp.gate = gate;
    fp.out_g = (__nv_bfloat16 *)og; fp.out_l = (__nv_bfloat16 *)ol;
    const int n_tiles = (s.Lq + BM - 1) / BM;
    attn_fwd_tc<FWD_WIN><<<tile_grid(s.Hq / 2, n_tiles, s.B), FWD_THREADS, kFwdSmem, st>>>(mq, mkw, mvw, fp); count_launch();
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    attn_fwd_tc<FWD_SEL><<<tile_grid(s.Hq / 2, n_tiles, s.B), FWD_THREADS, kFwdSmem, st>>>(mq, mk, mv, fp); count_launch();
    return cudaGetLastError();
}


}  // namespace hs
