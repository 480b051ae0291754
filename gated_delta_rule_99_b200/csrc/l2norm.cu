// q/k L2 normalisation passes of the paths whose kernels do not normalise their
// own tiles (fp32, and head dims other than 128).
//
// The layer's optional normalisation of q and k (jax-linear-attention 0.1.0,
// "Quick start": use_qk_l2norm=True): x^ = x / |x| for every row of d_k values
// (one token and head; a zero row stays zero), computed in fp32 and rounded to
// the input dtype.  In the backward the gradient with respect to x^ is carried
// back to the raw row: dx = (dx^ - x^ (x^ . dx^)) / |x|.  One warp per row; the
// lanes' partial sums meet in a fixed butterfly and lane 0's total is used by
// all, so the result does not depend on scheduling.
#include "gdn_internal.cuh"

namespace gdn {
namespace {

__device__ __forceinline__ float ldv(const float *p, int64_t i) { return p[i]; }
__device__ __forceinline__ float ldv(const __nv_bfloat16 *p, int64_t i) {
    return __bfloat162float(p[i]);
}
__device__ __forceinline__ void stv(float *p, int64_t i, float x) { p[i] = x; }
__device__ __forceinline__ void stv(__nv_bfloat16 *p, int64_t i, float x) {
    p[i] = __float2bfloat16_rn(x);
}

__device__ __forceinline__ float row_total(float s) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    return __shfl_sync(0xffffffffu, s, 0);
}

constexpr int kRowsPerBlock = 8;  // one warp per row

template <typename T>
__global__ void __launch_bounds__(32 * kRowsPerBlock)
    l2norm_rows_kernel(const T *x, T *xn, float *inv, int64_t rows, int K) {
    const int l = threadIdx.x & 31;
    for (int64_t row = (int64_t)blockIdx.x * kRowsPerBlock + (threadIdx.x >> 5); row < rows;
         row += (int64_t)gridDim.x * kRowsPerBlock) {
        const T *xr = x + row * K;
        float s = 0.f;
        for (int c = l; c < K; c += 32) {
            const float v = ldv(xr, c);
            s = fmaf(v, v, s);
        }
        s = row_total(s);
        const float r = s > 0.f ? 1.f / sqrtf(s) : 0.f;
        T *o = xn + row * K;
        for (int c = l; c < K; c += 32) stv(o, c, ldv(xr, c) * r);
        if (l == 0) inv[row] = r;
    }
}

template <typename T>
__global__ void __launch_bounds__(32 * kRowsPerBlock)
    l2norm_back_kernel(const T *xn, const float *inv, T *dx, int64_t rows, int K) {
    const int l = threadIdx.x & 31;
    for (int64_t row = (int64_t)blockIdx.x * kRowsPerBlock + (threadIdx.x >> 5); row < rows;
         row += (int64_t)gridDim.x * kRowsPerBlock) {
        const T *xr = xn + row * K;
        T *dr = dx + row * K;
        float s = 0.f;
        for (int c = l; c < K; c += 32) s = fmaf(ldv(xr, c), ldv(dr, c), s);
        s = row_total(s);
        const float r = inv[row];
        for (int c = l; c < K; c += 32) stv(dr, c, (ldv(dr, c) - ldv(xr, c) * s) * r);
    }
}

unsigned grid_for(int64_t rows) {
    const int64_t want = (rows + kRowsPerBlock - 1) / kRowsPerBlock, cap = 148 * 64;
    return (unsigned)(want < cap ? want : cap);
}

}  // namespace

cudaError_t launch_l2norm_rows(const void *x, void *xn, float *inv, int64_t rows, int K, bool bf16,
                               cudaStream_t stream) {
    if (rows <= 0) return cudaSuccess;
    const unsigned grid = grid_for(rows);
    if (bf16) {
        GDN_LAUNCH(kKL2Norm, stream,
                   l2norm_rows_kernel<__nv_bfloat16><<<grid, 32 * kRowsPerBlock, 0, stream>>>(
                       static_cast<const __nv_bfloat16 *>(x), static_cast<__nv_bfloat16 *>(xn),
                       inv, rows, K));
    } else {
        GDN_LAUNCH(kKL2Norm, stream,
                   l2norm_rows_kernel<float><<<grid, 32 * kRowsPerBlock, 0, stream>>>(
                       static_cast<const float *>(x), static_cast<float *>(xn), inv, rows, K));
    }
    return cudaSuccess;
}

cudaError_t launch_l2norm_back(const void *xn, const float *inv, void *dx, int64_t rows, int K,
                               bool bf16, cudaStream_t stream) {
    if (rows <= 0) return cudaSuccess;
    const unsigned grid = grid_for(rows);
    if (bf16) {
        GDN_LAUNCH(kKL2NormBack, stream,
                   l2norm_back_kernel<__nv_bfloat16><<<grid, 32 * kRowsPerBlock, 0, stream>>>(
                       static_cast<const __nv_bfloat16 *>(xn), inv,
                       static_cast<__nv_bfloat16 *>(dx), rows, K));
    } else {
        GDN_LAUNCH(kKL2NormBack, stream,
                   l2norm_back_kernel<float><<<grid, 32 * kRowsPerBlock, 0, stream>>>(
                       static_cast<const float *>(xn), inv, static_cast<float *>(dx), rows, K));
    }
    return cudaSuccess;
}

}  // namespace gdn
