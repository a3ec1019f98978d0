// CUDA-core (SIMT) kernels for the full layer (O, LSE, importance scores)
// and the sparse layer (global top-k branch + causal window branch + gate).
//
// These are the fp32 path (exact fp32 FMA arithmetic, which tensor-core tf32
// could not match at a 1e-4 tolerance) and the general fallback for shapes
// the tensor-core kernels do not cover.  One CTA serves one query row and one
// KV head; its G warps are the G query heads of that group, so each staged
// key/value tile is read once for the whole group.
//
// Full layer: HySparse abstract and the intelliparadigm write-up section 2.1
// (the full layer is the oracle of token importance); the importance of key j
// for a row is the group sum of the softmax probabilities.  Sparse layer:
// write-up section 2.2 (global branch over the TopK indices, local 128-token
// window, out = gate*global + (1-gate)*local with gate = sigmoid(logit)).
#include "common.cuh"
#include "internal.h"

namespace hs {
namespace {

constexpr int KT = 32;  // keys per staged tile (one per lane)

template <typename T, int D>
struct SimtSmem {
    // Ks is padded to D+1 floats per row so lane j reading row j is conflict-free.
    static constexpr size_t ks = KT * (D + 1);
    static constexpr size_t vs = KT * D;
    static size_t bytes(int G) { return sizeof(float) * (ks + vs + (size_t)G * D + (size_t)G * KT); }
};

// Stage keys [key_of(t) for t in tile] of KV head g into shared memory as
// fp32; invalid slots (key < 0) are zero-filled.
template <typename T, int D>
__device__ inline void stage_tile(const T *__restrict__ kbase, const T *__restrict__ vbase,
                                  const int *keys, int Hkv, float *Ks, float *Vs) {
    constexpr int V8 = D / 8;
    for (int e = threadIdx.x; e < KT * V8; e += blockDim.x) {
        const int t = e / V8, c8 = (e % V8) * 8;
        const int j = keys[t];
        float kf[8], vf[8];
        if (j >= 0) {
            load8(kbase + (size_t)j * Hkv * D + c8, kf);
            load8(vbase + (size_t)j * Hkv * D + c8, vf);
        } else {
#pragma unroll
            for (int u = 0; u < 8; ++u) kf[u] = vf[u] = 0.f;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            Ks[t * (D + 1) + c8 + u] = kf[u];
            Vs[t * D + c8 + u] = vf[u];
        }
    }
}

// Lane-parallel dot: lane t returns q . K[t] (scaled to log2 units).
template <int D>
__device__ inline float tile_logit(const float *qs, const float *Ks, int lane, float scale_log2) {
    float acc = 0.f;
#pragma unroll 8
    for (int c = 0; c < D; ++c) acc = fmaf(qs[c], Ks[lane * (D + 1) + c], acc);
    return acc * scale_log2;
}

// Online-softmax state of one warp (one query head): running max m (log2
// units), running sum l, and D/32 output columns per lane.
template <int D>
struct Online {
    float m = -INFINITY, l = 0.f, acc[D / 32];
    __device__ Online() {
#pragma unroll
        for (int t = 0; t < D / 32; ++t) acc[t] = 0.f;
    }
    // x: this lane's key logit (log2 units), -inf when masked.
    __device__ void step(float x, const float *Vs, float *ps, int lane) {
        const float tmax = warp_max(x);
        const float mnew = fmaxf(m, tmax);
        if (mnew == -INFINITY) return;  // whole tile masked and nothing seen yet
        const float corr = exp2f(m - mnew);
        const float p = exp2f(x - mnew);
        l = l * corr + warp_sum(p);
        m = mnew;
        ps[lane] = p;
        __syncwarp();
#pragma unroll
        for (int t = 0; t < D / 32; ++t) acc[t] *= corr;
#pragma unroll 4
        for (int j = 0; j < KT; ++j) {
            const float pj = ps[j];
#pragma unroll
            for (int t = 0; t < D / 32; ++t) acc[t] = fmaf(pj, Vs[j * D + lane + 32 * t], acc[t]);
        }
        __syncwarp();
    }
};

template <typename T, int D>
__global__ void __launch_bounds__(1024)
full_attn_scores_simt(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                      T *__restrict__ out, float *__restrict__ lse, float *__restrict__ scores,
                      long long ld_scores, int Lq, int Lkv, int Hq, int Hkv, int row_begin,
                      int row_count, float scale_log2) {
    extern __shared__ float smem[];
    const int G = Hq / Hkv;
    float *Ks = smem;
    float *Vs = Ks + SimtSmem<T, D>::ks;
    float *qs_all = Vs + SimtSmem<T, D>::vs;
    float *ps_all = qs_all + G * D;
    __shared__ int keys[KT];

    const int r = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int i = row_begin + r;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = g * G + warp;
    const int n = Lkv - Lq + i + 1;  // keys 0 .. pos
    float *qs = qs_all + warp * D;
    float *ps = ps_all + warp * KT;

    const T *qrow = q + (((size_t)b * Lq + i) * Hq + h) * D;
    for (int c = lane; c < D; c += 32) qs[c] = Elem<T>::to_f(qrow[c]);
    const T *kbase = k + ((size_t)b * Lkv * Hkv + g) * D;
    const T *vbase = v + ((size_t)b * Lkv * Hkv + g) * D;

    Online<D> st;
    for (int j0 = 0; j0 < n; j0 += KT) {
        __syncthreads();
        if (threadIdx.x < KT) keys[threadIdx.x] = (j0 + (int)threadIdx.x < n) ? j0 + (int)threadIdx.x : -1;
        __syncthreads();
        stage_tile<T, D>(kbase, vbase, keys, Hkv, Ks, Vs);
        __syncthreads();
        const float x = (j0 + lane < n) ? tile_logit<D>(qs, Ks, lane, scale_log2) : -INFINITY;
        st.step(x, Vs, ps, lane);
    }
    const float inv_l = 1.0f / st.l;
    T *orow = out + (((size_t)b * Lq + i) * Hq + h) * D;
#pragma unroll
    for (int t = 0; t < D / 32; ++t) orow[lane + 32 * t] = Elem<T>::from_f(st.acc[t] * inv_l);
    if (lane == 0) lse[((size_t)b * Hq + h) * Lq + i] = (st.m + log2f(st.l)) * kLn2;
    if (scores == nullptr) return;

    // Score pass: P_hj = 2^(x_j - m) / l, summed over the G heads of the group.
    float *srow = scores + (((size_t)b * Hkv + g) * row_count + r) * ld_scores;
    for (int j0 = 0; j0 < n; j0 += KT) {
        __syncthreads();
        if (threadIdx.x < KT) keys[threadIdx.x] = (j0 + (int)threadIdx.x < n) ? j0 + (int)threadIdx.x : -1;
        __syncthreads();
        stage_tile<T, D>(kbase, vbase, keys, Hkv, Ks, Vs);
        __syncthreads();
        const float x = tile_logit<D>(qs, Ks, lane, scale_log2);
        ps[lane] = exp2f(x - st.m) * inv_l;
        __syncthreads();
        if (warp == 0 && j0 + lane < n) {
            float s = 0.f;
            for (int w = 0; w < G; ++w) s += ps_all[w * KT + lane];
            srow[j0 + lane] = s;
        }
    }
}

template <typename T, int D>
__device__ inline void attend_keys(const T *kbase, const T *vbase, int Hkv, const int *list,
                                   int nlist, bool from_list, int lo, int pos, const float *qs,
                                   float *Ks, float *Vs, float *ps, int *keys, float scale_log2,
                                   Online<D> &st, unsigned int *status) {
    const int lane = threadIdx.x & 31;
    for (int t0 = 0; t0 < nlist; t0 += KT) {
        __syncthreads();
        if (threadIdx.x < KT) {
            int j = -1;
            const int t = t0 + threadIdx.x;
            if (t < nlist) {
                j = from_list ? list[t] : lo + t;
                if (j < -1 || j > pos) {
                    report(status, HS_ERR_INVALID_INDEX);
                    j = -1;
                }
            }
            keys[threadIdx.x] = j;
        }
        __syncthreads();
        stage_tile<T, D>(kbase, vbase, keys, Hkv, Ks, Vs);
        __syncthreads();
        const float x = keys[lane] >= 0 ? tile_logit<D>(qs, Ks, lane, scale_log2) : -INFINITY;
        st.step(x, Vs, ps, lane);
    }
}

template <typename T, int D>
__global__ void __launch_bounds__(1024)
sparse_attn_simt(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                 const int32_t *__restrict__ idx, int topk, const float *__restrict__ gate,
                 int window, T *__restrict__ out, T *__restrict__ out_g, T *__restrict__ out_l,
                 int Lq, int Lkv, int Hq, int Hkv, float scale_log2, unsigned int *status,
                 const T *__restrict__ kw, const T *__restrict__ vw, int Lwin) {
    extern __shared__ float smem[];
    const int G = Hq / Hkv;
    float *Ks = smem;
    float *Vs = Ks + SimtSmem<T, D>::ks;
    float *qs_all = Vs + SimtSmem<T, D>::vs;
    float *ps_all = qs_all + G * D;
    __shared__ int keys[KT];

    const int i = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = g * G + warp;
    const int pos = Lkv - Lq + i;
    float *qs = qs_all + warp * D;
    float *ps = ps_all + warp * KT;
    const size_t orow_off = (((size_t)b * Lq + i) * Hq + h) * D;
    for (int c = lane; c < D; c += 32) qs[c] = Elem<T>::to_f(q[orow_off + c]);
    const T *kbase = k + ((size_t)b * Lkv * Hkv + g) * D;
    const T *vbase = v + ((size_t)b * Lkv * Hkv + g) * D;
    const int32_t *list = idx + (((size_t)b * Hkv + g) * Lq + i) * topk;

    Online<D> sg, sl;
    attend_keys<T, D>(kbase, vbase, Hkv, list, topk, true, 0, pos, qs, Ks, Vs, ps, keys,
                      scale_log2, sg, status);
    const int lo = max(0, pos - window + 1);
    // the window branch: the shared cache, or the layer's own window K/V whose
    // row 0 is position Lkv - Lwin (the keys are then that buffer's rows)
    const int woff = kw ? Lkv - Lwin : 0;
    const T *kwb = kw ? kw + ((size_t)b * Lwin * Hkv + g) * D : kbase;
    const T *vwb = kw ? vw + ((size_t)b * Lwin * Hkv + g) * D : vbase;
    attend_keys<T, D>(kwb, vwb, Hkv, nullptr, pos - lo + 1, false, lo - woff, pos - woff, qs, Ks, Vs, ps,
                      keys, scale_log2, sl, status);

    const float x = gate[((size_t)b * Lq + i) * Hq + h];
    const float gs = 1.0f / (1.0f + expf(-x));
    const float ig = sg.l > 0.f ? 1.0f / sg.l : 0.f;
    const float il = 1.0f / sl.l;
#pragma unroll
    for (int t = 0; t < D / 32; ++t) {
        const float og = sg.acc[t] * ig, ol = sl.acc[t] * il;
        const int c = lane + 32 * t;
        out[orow_off + c] = Elem<T>::from_f(gs * og + (1.0f - gs) * ol);
        if (out_g) out_g[orow_off + c] = Elem<T>::from_f(og);
        if (out_l) out_l[orow_off + c] = Elem<T>::from_f(ol);
    }
}

template <typename T, int D>
cudaError_t launch_full_simt(const Shape &s, const void *q, const void *k, const void *v, void *out,
                             float *lse, float *scores, long long ld, int row_begin, int row_count,
                             cudaStream_t st) {
    const int G = s.Hq / s.Hkv;
    const size_t sm = SimtSmem<T, D>::bytes(G);
    auto kern = full_attn_scores_simt<T, D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    dim3 grid(row_count, s.Hkv, s.B);
    kern<<<grid, 32 * G, sm, st>>>((const T *)q, (const T *)k, (const T *)v, (T *)out, lse, scores,
                                   ld, s.Lq, s.Lkv, s.Hq, s.Hkv, row_begin, row_count,
                                   s.scale * kLog2e); count_launch();
    return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_sparse_simt(const Shape &s, const void *q, const void *k, const void *v,
                               const int32_t *idx, int topk, const float *gate, int window,
                               void *out, void *og, void *ol, unsigned int *status,
                               cudaStream_t st) {
    const int G = s.Hq / s.Hkv;
    const size_t sm = SimtSmem<T, D>::bytes(G);
    auto kern = sparse_attn_simt<T, D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    dim3 grid(s.Lq, s.Hkv, s.B);
    kern<<<grid, 32 * G, sm, st>>>((const T *)q, (const T *)k, (const T *)v, idx, topk, gate,
                                   window, (T *)out, (T *)og, (T *)ol, s.Lq, s.Lkv, s.Hq, s.Hkv,
                                   s.scale * kLog2e, status, (const T *)s.k_win, (const T *)s.v_win,
                                   s.Lwin); count_launch();
    return cudaGetLastError();
}

}  // namespace

cudaError_t full_attn_scores_simt_launch(const Shape &s, const void *q, const void *k,
                                         const void *v, void *out, float *lse, float *scores,
                                         long long ld, int row_begin, int row_count,
                                         cudaStream_t st) {
    if (s.dtype == HS_F32 && s.d == 64)
        return launch_full_simt<float, 64>(s, q, k, v, out, lse, scores, ld, row_begin, row_count, st);
    if (s.dtype == HS_F32 && s.d == 128)
        return launch_full_simt<float, 128>(s, q, k, v, out, lse, scores, ld, row_begin, row_count, st);
    if (s.dtype == HS_BF16 && s.d == 128)
        return launch_full_simt<__nv_bfloat16, 128>(s, q, k, v, out, lse, scores, ld, row_begin,
                                                    row_count, st);
    return cudaErrorInvalidValue;
}

cudaError_t sparse_attn_simt_launch(const Shape &s, const void *q, const void *k, const void *v,
                                    const int32_t *idx, int topk, const float *gate, int window,
                                    void *out, void *og, void *ol, unsigned int *status,
                                    cudaStream_t st) {
    if (s.dtype == HS_F32 && s.d == 64)
        return launch_sparse_simt<float, 64>(s, q, k, v, idx, topk, gate, window, out, og, ol, status, st);
    if (s.dtype == HS_F32 && s.d == 128)
        return launch_sparse_simt<float, 128>(s, q, k, v, idx, topk, gate, window, out, og, ol, status, st);
    if (s.dtype == HS_BF16 && s.d == 128)
        return launch_sparse_simt<__nv_bfloat16, 128>(s, q, k, v, idx, topk, gate, window, out, og,
                                                      ol, status, st);
    return cudaErrorInvalidValue;
}

}  // namespace hs
