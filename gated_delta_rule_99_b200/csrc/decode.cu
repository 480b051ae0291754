// Recurrent decode: advance the per-(sequence, head) state token by token.
//
// The inference form of the same recurrence (jax-linear-attention 0.1.0,
// "FAQ": inference decodes with each layer's recurrent state).  For each
// token t of a short row (T is small, usually 1):
//
//   S <- a_t (S - b_t (S k_t) k_t^T) + b_t v_t k_t^T,   a_t = exp(g_t)
//   o_t = scale S q_t
//
// with S = state^T kept in fp32 (with GDN_FLAG_QK_L2NORM, q_t and k_t are first
// divided by their norms, as the pages' API option use_qk_l2norm does; the
// factors 1/|q_t| and 1/|k_t| are applied where q_t and k_t enter).  One CTA per
// (sequence, head); the state is read once and written once per call and
// lives in registers in between (two threads per row of S).  HBM bound: the
// state (2 d_k d_v 4 bytes per sequence and head) dominates the traffic.
#include "gdn_internal.cuh"

namespace gdn {
namespace {

template <typename T>
__device__ __forceinline__ float ldf(const T *p, int64_t i);
template <>
__device__ __forceinline__ float ldf<float>(const float *p, int64_t i) { return p[i]; }
template <>
__device__ __forceinline__ float ldf<__nv_bfloat16>(const __nv_bfloat16 *p, int64_t i) {
    return __bfloat162float(p[i]);
}
__device__ __forceinline__ void stf(float *p, int64_t i, float x) { p[i] = x; }
__device__ __forceinline__ void stf(__nv_bfloat16 *p, int64_t i, float x) {
    p[i] = __float2bfloat16_rn(x);
}

// 256 threads per (sequence, head): thread t owns half t / 128 of the keys
// (K / 2 entries) of state row v = t % 128, so a row's state lives in two
// threads' registers; the halves' dot products meet in shared memory, added in a
// fixed order.
template <typename T, int K>
__global__ void __launch_bounds__(256) decode_kernel(const T *q, const T *k, const T *v,
                                                     const float *g, const float *beta,
                                                     float *state, T *o, int Tn, int H, int V,
                                                     float scale, int l2n) {
    constexpr int KH = K / 2;
    __shared__ float qs[K], ks[K], red_k[2][128], red_o[2][128];
    const int bh = blockIdx.x, b = bh / H, h = bh % H, t = threadIdx.x;
    const int vi = t & 127, half = t >> 7, k0 = half * KH;
    const bool active = vi < V;
    float *st = state + (size_t)bh * K * V;
    float S[KH];
#pragma unroll
    for (int j = 0; j < KH; ++j) S[j] = active ? st[(size_t)(k0 + j) * V + vi] : 0.f;
    for (int tk = 0; tk < Tn; ++tk) {
        const int64_t row = ((int64_t)b * Tn + tk) * H + h;
        __syncthreads();  // the previous token's q, k and partial sums are no longer read
        for (int kk = t; kk < K; kk += 256) {
            qs[kk] = ldf(q, row * K + kk);
            ks[kk] = ldf(k, row * K + kk);
        }
        __syncthreads();
        const float a = expf(g[row]), bt = beta[row];
        const float vv = active ? ldf(v, row * V + vi) : 0.f;
        float iq = 1.f, ik = 1.f;  // 1/|q_t|, 1/|k_t| (zero rows stay zero)
        if (l2n) {
            float nq = 0.f, nk = 0.f;
#pragma unroll
            for (int kk = 0; kk < K; ++kk) {
                nq = fmaf(qs[kk], qs[kk], nq);
                nk = fmaf(ks[kk], ks[kk], nk);
            }
            iq = nq > 0.f ? 1.f / sqrtf(nq) : 0.f;
            ik = nk > 0.f ? 1.f / sqrtf(nk) : 0.f;
        }
        float sk0 = 0.f, sk1 = 0.f;
#pragma unroll
        for (int j = 0; j < KH; j += 2) {
            sk0 = fmaf(S[j], ks[k0 + j], sk0);
            sk1 = fmaf(S[j + 1], ks[k0 + j + 1], sk1);
        }
        red_k[half][vi] = sk0 + sk1;
        __syncthreads();
        const float sk = ik * (red_k[0][vi] + red_k[1][vi]);
        const float c1 = bt * sk * ik, c2 = bt * vv * ik;
        float o0 = 0.f, o1 = 0.f;
#pragma unroll
        for (int j = 0; j < KH; ++j) {
            const float kj = ks[k0 + j];
            S[j] = a * (S[j] - c1 * kj) + c2 * kj;
            if (j & 1) o1 = fmaf(S[j], qs[k0 + j], o1);
            else o0 = fmaf(S[j], qs[k0 + j], o0);
        }
        red_o[half][vi] = o0 + o1;
        __syncthreads();
        if (half == 0 && active)
            stf(o, row * V + vi, scale * iq * (red_o[0][vi] + red_o[1][vi]));
    }
    if (active) {
#pragma unroll
        for (int j = 0; j < KH; ++j) st[(size_t)(k0 + j) * V + vi] = S[j];
    }
}

template <typename T>
cudaError_t launch_typed(const gdn_desc *d, const void *q, const void *k, const void *v,
                         const float *g, const float *beta, float *state, void *o,
                         cudaStream_t s) {
    const int nbh = (int)(d->B * d->H), Tn = (int)d->T, H = (int)d->H, V = (int)d->dv;
    const int l2n = (d->flags & GDN_FLAG_QK_L2NORM) ? 1 : 0;
    if (d->dk == 128) {
        GDN_LAUNCH(kKDecode, s,
                   decode_kernel<T, 128><<<nbh, 256, 0, s>>>(
                       (const T *)q, (const T *)k, (const T *)v, g, beta, state, (T *)o, Tn, H,
                       V, d->scale, l2n));
    } else {
        GDN_LAUNCH(kKDecode, s,
                   decode_kernel<T, 64><<<nbh, 256, 0, s>>>(
                       (const T *)q, (const T *)k, (const T *)v, g, beta, state, (T *)o, Tn, H,
                       V, d->scale, l2n));
    }
    return cudaSuccess;
}

bool mis(const void *p) { return p && (reinterpret_cast<uintptr_t>(p) % 16) != 0; }

}  // namespace
}  // namespace gdn

extern "C" gdn_status gdn_decode(const gdn_desc *d, const void *q, const void *k, const void *v,
                                 const float *g, const float *beta, float *state, void *o,
                                 void *stream) {
    using namespace gdn;
    if (!d) return GDN_ERR_INVALID_ARG;
    if (d->B < 1 || d->T < 1 || d->H < 1 || d->n_seqs != 0) return GDN_ERR_INVALID_ARG;
    if (d->dtype != GDN_BF16 && d->dtype != GDN_FP32) return GDN_ERR_UNSUPPORTED;
    if ((d->dk != 64 && d->dk != 128) || (d->dv != 64 && d->dv != 128)) return GDN_ERR_UNSUPPORTED;
    // range checks before any product is formed (no signed overflow on huge inputs)
    constexpr int64_t kLim = int64_t(1) << 31;
    if (d->B >= kLim || d->T >= kLim || d->H >= kLim || d->H >= kLim / d->B ||
        d->T >= kLim / d->B)
        return GDN_ERR_INVALID_ARG;
    if (!(d->scale == d->scale)) return GDN_ERR_INVALID_ARG;
    if (d->reserved != 0 ||
        (d->flags & ~(GDN_FLAG_PIECE_SCAN | GDN_FLAG_QK_L2NORM | GDN_FLAG_VALUE_SLICES)))
        return GDN_ERR_INVALID_ARG;
    if (!q || !k || !v || !g || !beta || !state || !o) return GDN_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k, v, g, beta, state, o};
    for (const void *p : ptrs)
        if (mis(p)) return GDN_ERR_ALIGNMENT;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    arm_planted_failure();
    cudaError_t e = d->dtype == GDN_BF16
                        ? launch_typed<__nv_bfloat16>(d, q, k, v, g, beta, state, o, s)
                        : launch_typed<float>(d, q, k, v, g, beta, state, o, s);
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}
