// fp32 SIMT kernels of the chunkwise Gated DeltaNet forward and backward.
//
// This is the path of fp32 inputs (fp32 CUDA-core FMAs throughout; the bf16
// tensor-core path is a separate implementation of the same algebra, and both
// are checked against the fp64 oracle, not against each other).  It follows the
// chunkwise form of
// the recurrence S_t = a_t S_{t-1}(I - b_t k_t k_t^T) + b_t v_t k_t^T,
// o_t = scale S_t q_t (the pages name the method and its chunk-parallel
// form -- jax-linear-attention 0.1.0, "How it works" -- without printing it).
// Per chunk of 64 tokens, with H = S^T (dk x dv) the state entering it:
//
//   G = cumsum(g) ; gam_i = exp(G_i) ; Gam_ij = exp(G_i - G_j) (i >= j)
//   A = (I + strict_lower(diag(b) K K^T . Gam))^-1      forward substitution
//   W = A diag(b gam) K ; Ut = A diag(b) V               prep kernel
//   U = Ut - W H ; H <- gam_C H + (diag(e) K)^T U        state kernel (serial)
//   O = scale (diag(gam) Q H + lower(Q K^T . Gam) U)     output kernel
//
// and the backward is the reverse-mode of the same steps: a serial reverse
// pass carries dH across chunks, then a chunk-parallel kernel forms every
// gradient.  Rows past the end of a partial chunk are zero (k = v = q = do =
// 0, b = 0, g = 0), which leaves every product exact.
//
// Matrices of a chunk live in a per-CTA fp32 scratch slot in global memory
// (L1/L2 resident); all block-level products go through `bmm`.
#include "gdn_internal.cuh"

namespace gdn {
namespace {

constexpr int kThreads = 256;
constexpr int C = kChunk;

__device__ __forceinline__ float ld_in(const void *p, int64_t i, int bf16) {
    return bf16 ? __bfloat162float(static_cast<const __nv_bfloat16 *>(p)[i])
                : static_cast<const float *>(p)[i];
}

__device__ __forceinline__ void st_out(void *p, int64_t i, float x, int bf16) {
    if (bf16) static_cast<__nv_bfloat16 *>(p)[i] = __float2bfloat16_rn(x);
    else static_cast<float *>(p)[i] = x;
}

// C = alpha * A B + cbeta * C for an M x N result with inner size Kd.
// Element (i, j) of X sits at X[i * xr + j * xc].  Every thread of the block
// must call it; it ends with a block barrier.
template <int TM, int TN>
__device__ void bmm(float *Cm, int cr, int cc, const float *Am, int ar, int ac, const float *Bm,
                    int br, int bc, int M, int N, int Kd, float alpha, float cbeta) {
    const int tn = N / TN, tiles = (M / TM) * tn;
    for (int t = threadIdx.x; t < tiles; t += blockDim.x) {
        const int i0 = (t / tn) * TM, j0 = (t % tn) * TN;
        float acc[TM][TN];
#pragma unroll
        for (int i = 0; i < TM; ++i)
#pragma unroll
            for (int j = 0; j < TN; ++j) acc[i][j] = 0.f;
        for (int kk = 0; kk < Kd; ++kk) {
            float a[TM], b[TN];
#pragma unroll
            for (int i = 0; i < TM; ++i) a[i] = Am[(i0 + i) * ar + kk * ac];
#pragma unroll
            for (int j = 0; j < TN; ++j) b[j] = Bm[kk * br + (j0 + j) * bc];
#pragma unroll
            for (int i = 0; i < TM; ++i)
#pragma unroll
                for (int j = 0; j < TN; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
#pragma unroll
        for (int i = 0; i < TM; ++i)
#pragma unroll
            for (int j = 0; j < TN; ++j) {
                float *c = Cm + (i0 + i) * cr + (j0 + j) * cc;
                *c = cbeta != 0.f ? fmaf(alpha, acc[i][j], cbeta * *c) : alpha * acc[i][j];
            }
    }
    __syncthreads();
}

// Rows [0, 64) of a [tokens][H][D] tensor for one chunk and head, times `mul`;
// rows at or past `len` are zero.
__device__ void load_rows(float *dst, const void *src, int bf16, int64_t tok0, int len, int h,
                          int H, int D, float mul) {
    for (int e = threadIdx.x; e < C * D; e += blockDim.x) {
        const int r = e / D, d = e % D;
        dst[e] = r < len ? mul * ld_in(src, ((tok0 + r) * H + h) * (int64_t)D + d, bf16) : 0.f;
    }
}

// Per-chunk cumulative log-decay G (64 entries, zero gates past len) and the
// write strengths b (zero past len).  The gates are staged in parallel, then
// one thread sums them in token order so every kernel gets bit-identical G.
// Ends with a barrier.
__device__ void load_gate(float *G, float *bta, const Params &p, const ChunkInfo &ci, int h) {
    const int r = threadIdx.x;
    if (r < C) {
        const int64_t idx = (int64_t)(ci.tok0 + r) * p.H + h;
        G[r] = r < ci.len ? p.g[idx] : 0.f;
        if (bta) bta[r] = r < ci.len ? p.beta[idx] : 0.f;
    }
    __syncthreads();
    if (r == 0) {
        float s = 0.f;
        for (int i = 0; i < C; ++i) {
            s += G[i];
            G[i] = s;
        }
    }
    __syncthreads();
}

// A = (I + M)^-1 for a strictly lower M (64 x 64, row-major): row i of A is
// e_i - sum_{m<i} M[i][m] A[m], computed top to bottom.
__device__ void invert_unit_lower(float *A, const float *M) {
    for (int e = threadIdx.x; e < C * C; e += blockDim.x) A[e] = (e / C == e % C) ? 1.f : 0.f;
    __syncthreads();
    for (int i = 1; i < C; ++i) {
        const int j = threadIdx.x;
        if (j < i) {
            float s = 0.f;
            for (int m = j; m < i; ++m) s = fmaf(M[i * C + m], A[m * C + j], s);
            A[i * C + j] = -s;
        }
        __syncthreads();
    }
}

__device__ __forceinline__ float *slot(const Params &p) {
    return p.scratch + (size_t)blockIdx.x * simt_scratch_floats(simt_tile_width(p.K, p.V));
}

// ---------------------------------------------------------------- prep: A, W, Ut
__global__ void __launch_bounds__(kThreads) simt_prep_kernel(Params p) {
    if (p.hdr->status) return;
    const int K = p.K, V = p.V, H = p.H;
    const int TW = C * simt_tile_width(K, V);
    float *fk = slot(p), *fv = fk + TW, *bk = fv + TW, *bv = bk + TW;
    float *M = bv + TW, *G = M + C * C, *bta = G + C;
    for (int ch = blockIdx.x; ch < p.NC * H; ch += gridDim.x) {
        const int c = ch / H, h = ch % H;
        const ChunkInfo ci = chunk_at(p, c);
        load_rows(fk, p.k, p.bf16, ci.tok0, ci.len, h, H, K, 1.f);
        load_rows(fv, p.v, p.bf16, ci.tok0, ci.len, h, H, V, 1.f);
        load_gate(G, bta, p, ci, h);
        bmm<4, 4>(M, C, 1, fk, K, 1, fk, 1, K, C, C, K, 1.f, 0.f);  // K K^T
        for (int e = threadIdx.x; e < C * C; e += blockDim.x) {
            const int i = e / C, j = e % C;
            M[e] = i > j ? bta[i] * expf(G[i] - G[j]) * M[e] : 0.f;
        }
        __syncthreads();
        float *A = p.A + (size_t)ch * C * C;
        invert_unit_lower(A, M);
        for (int e = threadIdx.x; e < C * K; e += blockDim.x) {
            const int i = e / K;
            bk[e] = bta[i] * expf(G[i]) * fk[e];
        }
        for (int e = threadIdx.x; e < C * V; e += blockDim.x) bv[e] = bta[e / V] * fv[e];
        __syncthreads();
        bmm<4, 4>(p.W + (size_t)ch * C * K, K, 1, A, C, 1, bk, K, 1, C, K, C, 1.f, 0.f);
        bmm<4, 4>(p.Ut + (size_t)ch * C * V, V, 1, A, C, 1, bv, V, 1, C, V, C, 1.f, 0.f);
    }
}

// ------------------------------------------------- forward state pass (serial)
// One CTA per (sequence, head, 32 value columns).  Writes the state entering
// every chunk (Hs), the corrected values U, and the final state.
__global__ void __launch_bounds__(kThreads) simt_state_fwd_kernel(Params p) {
    if (p.hdr->status) return;
    extern __shared__ float sm[];
    const int K = p.K, V = p.V, H = p.H, nvs = V / kSimtVSlice;
    const int vs = blockIdx.x % nvs, h = (blockIdx.x / nvs) % H, n = blockIdx.x / (nvs * H);
    const int v0 = vs * kSimtVSlice, VS = kSimtVSlice;
    float *Hsl = sm, *Usl = Hsl + K * VS, *ek = Usl + C * VS, *G = ek + C * K;
    for (int e = threadIdx.x; e < K * VS; e += blockDim.x) {
        const int kk = e / VS, j = e % VS;
        Hsl[e] = p.h0 ? p.h0[(((int64_t)n * H + h) * K + kk) * V + v0 + j] : 0.f;
    }
    __syncthreads();
    const int c0 = seq_first_at(p, n), c1 = seq_first_at(p, n + 1);
    for (int c = c0; c < c1; ++c) {
        const ChunkInfo ci = chunk_at(p, c);
        const size_t ch = (size_t)c * H + h;
        load_gate(G, nullptr, p, ci, h);
        const float gC = expf(G[C - 1]);
        for (int e = threadIdx.x; e < C * K; e += blockDim.x) {
            const int i = e / K, kk = e % K;
            ek[e] = i < ci.len ? expf(G[C - 1] - G[i]) *
                                     ld_in(p.k, ((int64_t)(ci.tok0 + i) * H + h) * K + kk, p.bf16)
                               : 0.f;
        }
        for (int e = threadIdx.x; e < K * VS; e += blockDim.x) {
            const int kk = e / VS, j = e % VS;
            p.Hs[ch * K * V + (size_t)kk * V + v0 + j] = Hsl[e];
        }
        for (int e = threadIdx.x; e < C * VS; e += blockDim.x) {
            const int i = e / VS, j = e % VS;
            Usl[e] = p.Ut[ch * C * V + (size_t)i * V + v0 + j];
        }
        __syncthreads();
        bmm<2, 2>(Usl, VS, 1, p.W + ch * C * K, K, 1, Hsl, VS, 1, C, VS, K, -1.f, 1.f);
        for (int e = threadIdx.x; e < C * VS; e += blockDim.x) {
            const int i = e / VS, j = e % VS;
            p.U[ch * C * V + (size_t)i * V + v0 + j] = Usl[e];
        }
        bmm<2, 2>(Hsl, VS, 1, ek, 1, K, Usl, VS, 1, K, VS, C, 1.f, gC);
    }
    if (p.hT) {
        for (int e = threadIdx.x; e < K * VS; e += blockDim.x) {
            const int kk = e / VS, j = e % VS;
            p.hT[(((int64_t)n * H + h) * K + kk) * V + v0 + j] = Hsl[e];
        }
    }
}

// ------------------------------------------------------------- output
__global__ void __launch_bounds__(kThreads) simt_out_kernel(Params p) {
    if (p.hdr->status) return;
    const int K = p.K, V = p.V, H = p.H;
    const int TW = C * simt_tile_width(K, V);
    float *fq = slot(p), *fk = fq + TW, *O = fk + TW, *P = O + TW, *G = P + C * C;
    for (int ch = blockIdx.x; ch < p.NC * H; ch += gridDim.x) {
        const int c = ch / H, h = ch % H;
        const ChunkInfo ci = chunk_at(p, c);
        load_rows(fq, p.q, p.bf16, ci.tok0, ci.len, h, H, K, p.scale);
        load_rows(fk, p.k, p.bf16, ci.tok0, ci.len, h, H, K, 1.f);
        load_gate(G, nullptr, p, ci, h);
        bmm<4, 4>(P, C, 1, fq, K, 1, fk, 1, K, C, C, K, 1.f, 0.f);
        for (int e = threadIdx.x; e < C * C; e += blockDim.x) {
            const int i = e / C, j = e % C;
            P[e] = j <= i ? P[e] * expf(G[i] - G[j]) : 0.f;
        }
        for (int e = threadIdx.x; e < C * K; e += blockDim.x) fq[e] *= expf(G[e / K]);
        __syncthreads();
        bmm<4, 4>(O, V, 1, fq, K, 1, p.Hs + (size_t)ch * K * V, V, 1, C, V, K, 1.f, 0.f);
        bmm<4, 4>(O, V, 1, P, C, 1, p.U + (size_t)ch * C * V, V, 1, C, V, C, 1.f, 1.f);
        for (int e = threadIdx.x; e < C * V; e += blockDim.x) {
            const int i = e / V, d = e % V;
            if (i < ci.len) st_out(p.o, ((int64_t)(ci.tok0 + i) * H + h) * V + d, O[e], p.bf16);
        }
        __syncthreads();
    }
}

// ------------------------------------------- backward: chunk-local P^T dO
__global__ void __launch_bounds__(kThreads) simt_duloc_kernel(Params p) {
    if (p.hdr->status) return;
    const int K = p.K, V = p.V, H = p.H;
    const int TW = C * simt_tile_width(K, V);
    float *fq = slot(p), *fk = fq + TW, *fdo = fk + TW, *P = fdo + TW,
          *G = P + C * C;
    for (int ch = blockIdx.x; ch < p.NC * H; ch += gridDim.x) {
        const int c = ch / H, h = ch % H;
        const ChunkInfo ci = chunk_at(p, c);
        load_rows(fq, p.q, p.bf16, ci.tok0, ci.len, h, H, K, p.scale);
        load_rows(fk, p.k, p.bf16, ci.tok0, ci.len, h, H, K, 1.f);
        load_rows(fdo, p.do_, p.bf16, ci.tok0, ci.len, h, H, V, 1.f);
        load_gate(G, nullptr, p, ci, h);
        bmm<4, 4>(P, C, 1, fq, K, 1, fk, 1, K, C, C, K, 1.f, 0.f);
        for (int e = threadIdx.x; e < C * C; e += blockDim.x) {
            const int i = e / C, j = e % C;
            P[e] = j <= i ? P[e] * expf(G[i] - G[j]) : 0.f;
        }
        __syncthreads();
        bmm<4, 4>(p.dUloc + (size_t)ch * C * V, V, 1, P, 1, C, fdo, V, 1, C, V, C, 1.f, 0.f);
    }
}

// ---------------------------------------------- backward state pass (serial)
// Chunks in reverse.  dH enters as dhT; per chunk it records dH (the gradient
// of the state leaving the chunk) and dU, then steps to the state entering it:
//   dU = diag(e) K dH + P^T dO ;  dH <- gam_C dH + (diag(gam) Q')^T dO - W^T dU
__global__ void __launch_bounds__(kThreads) simt_state_bwd_kernel(Params p) {
    if (p.hdr->status) return;
    extern __shared__ float sm[];
    const int K = p.K, V = p.V, H = p.H, nvs = V / kSimtVSlice;
    const int vs = blockIdx.x % nvs, h = (blockIdx.x / nvs) % H, n = blockIdx.x / (nvs * H);
    const int v0 = vs * kSimtVSlice, VS = kSimtVSlice;
    float *dHsl = sm, *dUsl = dHsl + K * VS, *ek = dUsl + C * VS, *gq = ek + C * K,
          *dOs = gq + C * K, *G = dOs + C * VS;
    for (int e = threadIdx.x; e < K * VS; e += blockDim.x) {
        const int kk = e / VS, j = e % VS;
        dHsl[e] = p.dhT ? p.dhT[(((int64_t)n * H + h) * K + kk) * V + v0 + j] : 0.f;
    }
    __syncthreads();
    const int c0 = seq_first_at(p, n), c1 = seq_first_at(p, n + 1);
    for (int c = c1 - 1; c >= c0; --c) {
        const ChunkInfo ci = chunk_at(p, c);
        const size_t ch = (size_t)c * H + h;
        load_gate(G, nullptr, p, ci, h);
        const float gC = expf(G[C - 1]);
        for (int e = threadIdx.x; e < C * K; e += blockDim.x) {
            const int i = e / K, kk = e % K;
            const int64_t src = ((int64_t)(ci.tok0 + i) * H + h) * K + kk;
            const bool in = i < ci.len;
            ek[e] = in ? expf(G[C - 1] - G[i]) * ld_in(p.k, src, p.bf16) : 0.f;
            gq[e] = in ? p.scale * expf(G[i]) * ld_in(p.q, src, p.bf16) : 0.f;
        }
        for (int e = threadIdx.x; e < C * VS; e += blockDim.x) {
            const int i = e / VS, j = e % VS;
            dOs[e] = i < ci.len ? ld_in(p.do_, ((int64_t)(ci.tok0 + i) * H + h) * V + v0 + j, p.bf16)
                                : 0.f;
            dUsl[e] = p.dUloc[ch * C * V + (size_t)i * V + v0 + j];
        }
        for (int e = threadIdx.x; e < K * VS; e += blockDim.x) {
            const int kk = e / VS, j = e % VS;
            p.dHn[ch * K * V + (size_t)kk * V + v0 + j] = dHsl[e];
        }
        __syncthreads();
        bmm<2, 2>(dUsl, VS, 1, ek, K, 1, dHsl, VS, 1, C, VS, K, 1.f, 1.f);
        for (int e = threadIdx.x; e < C * VS; e += blockDim.x) {
            const int i = e / VS, j = e % VS;
            p.dU[ch * C * V + (size_t)i * V + v0 + j] = dUsl[e];
        }
        bmm<2, 2>(dHsl, VS, 1, gq, 1, K, dOs, VS, 1, K, VS, C, 1.f, gC);
        bmm<2, 2>(dHsl, VS, 1, p.W + ch * C * K, 1, K, dUsl, VS, 1, K, VS, C, -1.f, 1.f);
    }
    if (p.dh0) {
        for (int e = threadIdx.x; e < K * VS; e += blockDim.x) {
            const int kk = e / VS, j = e % VS;
            p.dh0[(((int64_t)n * H + h) * K + kk) * V + v0 + j] = dHsl[e];
        }
    }
}

// ------------------------------------------- backward: chunk-local gradients
__global__ void __launch_bounds__(kThreads) simt_grads_kernel(Params p) {
    if (p.hdr->status) return;
    const int K = p.K, V = p.V, H = p.H;
    const int T8 = C * simt_tile_width(K, V);
    constexpr int T4 = C * C;
    float *fq = slot(p), *fk = fq + T8, *fv = fk + T8, *fdo = fv + T8, *X1 = fdo + T8,
          *X2 = X1 + T8, *X3 = X2 + T8, *Z = X3 + T8, *AtdU = Z + T8, *bv = AtdU + T8,
          *bgk = bv + T8, *dQ = bgk + T8, *dK = dQ + T8;
    float *Gam = dK + T8, *P = Gam + T4, *KK = P + T4, *Lm = KK + T4, *dP = Lm + T4,
          *dA = dP + T4, *T1 = dA + T4, *dL = T1 + T4, *dS = dL + T4, *dLG = dS + T4;
    float *G = dLG + T4, *bta = G + C, *gam = bta + C, *e = gam + C, *dG = e + C, *red = dG + C;
    for (int ch = blockIdx.x; ch < p.NC * H; ch += gridDim.x) {
        const int c = ch / H, h = ch % H;
        const ChunkInfo ci = chunk_at(p, c);
        const float *Hs = p.Hs + (size_t)ch * K * V, *dHn = p.dHn + (size_t)ch * K * V;
        const float *U = p.U + (size_t)ch * C * V, *dU = p.dU + (size_t)ch * C * V;
        const float *A = p.A + (size_t)ch * C * C;
        load_rows(fq, p.q, p.bf16, ci.tok0, ci.len, h, H, K, p.scale);
        load_rows(fk, p.k, p.bf16, ci.tok0, ci.len, h, H, K, 1.f);
        load_rows(fv, p.v, p.bf16, ci.tok0, ci.len, h, H, V, 1.f);
        load_rows(fdo, p.do_, p.bf16, ci.tok0, ci.len, h, H, V, 1.f);
        load_gate(G, bta, p, ci, h);
        for (int i = threadIdx.x; i < C; i += blockDim.x) {
            gam[i] = expf(G[i]);
            e[i] = expf(G[C - 1] - G[i]);
        }
        for (int x = threadIdx.x; x < T4; x += blockDim.x) {
            const int i = x / C, j = x % C;
            Gam[x] = j <= i ? expf(G[i] - G[j]) : 0.f;
        }
        __syncthreads();
        bmm<4, 4>(KK, C, 1, fk, K, 1, fk, 1, K, C, C, K, 1.f, 0.f);
        bmm<4, 4>(P, C, 1, fq, K, 1, fk, 1, K, C, C, K, 1.f, 0.f);
        for (int x = threadIdx.x; x < T4; x += blockDim.x) {
            const int i = x / C, j = x % C;
            P[x] *= Gam[x];
            Lm[x] = i > j ? bta[i] * Gam[x] * KK[x] : 0.f;
        }
        __syncthreads();
        // products with the state entering (Hs) and the gradient leaving (dHn)
        bmm<4, 4>(X1, K, 1, fdo, V, 1, Hs, 1, V, C, K, V, 1.f, 0.f);  // dO Hs^T
        bmm<4, 4>(X2, K, 1, U, V, 1, dHn, 1, V, C, K, V, 1.f, 0.f);   // U dHn^T
        bmm<4, 4>(X3, K, 1, dU, V, 1, Hs, 1, V, C, K, V, 1.f, 0.f);   // dU Hs^T (= -dW)
        bmm<4, 4>(dP, C, 1, fdo, V, 1, U, 1, V, C, C, V, 1.f, 0.f);   // dO U^T
        bmm<4, 4>(AtdU, V, 1, A, 1, C, dU, V, 1, C, V, C, 1.f, 0.f);  // A^T dU
        for (int x = threadIdx.x; x < T4; x += blockDim.x) {
            const int i = x / C, j = x % C;
            if (j > i) dP[x] = 0.f;
        }
        for (int x = threadIdx.x; x < C * V; x += blockDim.x) bv[x] = bta[x / V] * fv[x];
        for (int x = threadIdx.x; x < C * K; x += blockDim.x) {
            const int i = x / K;
            bgk[x] = bta[i] * gam[i] * fk[x];
        }
        // <Hs, dHn> for the gradient of gam_C
        {
            float s = 0.f;
            for (int x = threadIdx.x; x < K * V; x += blockDim.x) s = fmaf(Hs[x], dHn[x], s);
            for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
            if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
        }
        __syncthreads();
        bmm<4, 4>(dA, C, 1, dU, V, 1, bv, 1, V, C, C, V, 1.f, 0.f);    // dU (bV)^T
        bmm<4, 4>(dA, C, 1, X3, K, 1, bgk, 1, K, C, C, K, -1.f, 1.f);  // + dW (bgK)^T
        bmm<4, 4>(Z, K, 1, A, 1, C, X3, K, 1, C, K, C, -1.f, 0.f);     // A^T dW
        bmm<4, 4>(T1, C, 1, A, 1, C, dA, C, 1, C, C, C, 1.f, 0.f);     // A^T dA
        bmm<4, 4>(dL, C, 1, T1, C, 1, A, 1, C, C, C, C, -1.f, 0.f);    // -A^T dA A^T
        for (int x = threadIdx.x; x < T4; x += blockDim.x) {
            const int i = x / C, j = x % C;
            if (j >= i) dL[x] = 0.f;
            dS[x] = dP[x] * Gam[x];
            dLG[x] = (j < i ? dL[x] : 0.f) * Gam[x];
        }
        __syncthreads();
        // per-row scalars: dbeta and the gradient of the cumulative gate G
        if (threadIdx.x < C) {
            const int i = threadIdx.x;
            float db = 0.f, kz = 0.f, qx = 0.f, kx = 0.f, dlgk = 0.f, pp = 0.f, ll = 0.f;
            for (int d = 0; d < V; ++d) db = fmaf(fv[i * V + d], AtdU[i * V + d], db);
            for (int d = 0; d < K; ++d) {
                kz = fmaf(fk[i * K + d], Z[i * K + d], kz);
                qx = fmaf(fq[i * K + d], X1[i * K + d], qx);
                kx = fmaf(fk[i * K + d], X2[i * K + d], kx);
            }
            for (int j = 0; j < C; ++j) {
                dlgk = fmaf(dLG[i * C + j], KK[i * C + j], dlgk);
                pp += dP[i * C + j] * P[i * C + j] - dP[j * C + i] * P[j * C + i];
                ll += dL[i * C + j] * Lm[i * C + j] - dL[j * C + i] * Lm[j * C + i];
            }
            dG[i] = -e[i] * kx + gam[i] * qx + pp + bta[i] * gam[i] * kz + ll;
            red[8 + i] = db + gam[i] * kz + dlgk;  // dbeta
            red[8 + C + i] = e[i] * kx;            // e_j k_j . dKd_j for the G_C term
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            float hd = 0.f, s = 0.f;
            for (int w = 0; w < kThreads / 32; ++w) hd += red[w];
            for (int j = 0; j < C; ++j) s += red[8 + C + j];
            dG[C - 1] += gam[C - 1] * hd + s;
            float acc = 0.f;
            for (int j = C - 1; j >= 0; --j) {  // dg = reverse cumsum of dG
                acc += dG[j];
                dG[j] = acc;
            }
        }
        __syncthreads();
        // dQ' = diag(gam) X1 + dS K ; dK = diag(e) X2 + dS^T Q' + diag(b gam) Z + ...
        for (int x = threadIdx.x; x < C * K; x += blockDim.x) {
            const int i = x / K;
            dQ[x] = gam[i] * X1[x];
            dK[x] = e[i] * X2[x] + bta[i] * gam[i] * Z[x];
        }
        __syncthreads();
        bmm<4, 4>(dQ, K, 1, dS, C, 1, fk, K, 1, C, K, C, 1.f, 1.f);
        bmm<4, 4>(dK, K, 1, dS, 1, C, fq, K, 1, C, K, C, 1.f, 1.f);
        bmm<4, 4>(X1, K, 1, dLG, C, 1, fk, K, 1, C, K, C, 1.f, 0.f);  // dLG K
        for (int x = threadIdx.x; x < T4; x += blockDim.x) dA[x] = bta[x / C] * dLG[x];
        for (int x = threadIdx.x; x < C * K; x += blockDim.x) dK[x] += bta[x / K] * X1[x];
        __syncthreads();
        bmm<4, 4>(dK, K, 1, dA, 1, C, fk, K, 1, C, K, C, 1.f, 1.f);  // (diag(b) dLG)^T K
        for (int x = threadIdx.x; x < C * K; x += blockDim.x) {
            const int i = x / K, d = x % K;
            if (i < ci.len) {
                const int64_t o = ((int64_t)(ci.tok0 + i) * H + h) * K + d;
                st_out(p.dq, o, p.scale * dQ[x], p.bf16);
                st_out(p.dk, o, dK[x], p.bf16);
            }
        }
        for (int x = threadIdx.x; x < C * V; x += blockDim.x) {
            const int i = x / V, d = x % V;
            if (i < ci.len)
                st_out(p.dv, ((int64_t)(ci.tok0 + i) * H + h) * V + d, bta[i] * AtdU[x], p.bf16);
        }
        if (threadIdx.x < ci.len) {
            const int64_t o = (int64_t)(ci.tok0 + threadIdx.x) * H + h;
            p.dg[o] = dG[threadIdx.x];
            p.dbeta[o] = red[8 + threadIdx.x];
        }
        __syncthreads();
    }
}

size_t state_smem(int K, bool bwd) {
    const int VS = kSimtVSlice;
    if (!bwd) return sizeof(float) * (K * VS + C * VS + C * K + C);
    return sizeof(float) * (K * VS + C * VS + 2 * C * K + C * VS + C);
}

int simt_grid(const Params &p) {
    const long long n = (long long)p.NC * p.H;
    return (int)(n < kSimtSlots ? (n > 0 ? n : 1) : kSimtSlots);
}

}  // namespace

cudaError_t launch_simt_fwd(const Params &p, cudaStream_t stream) {
    const int nstate = p.N * p.H * (p.V / kSimtVSlice);
    if (p.NC > 0)
        GDN_LAUNCH(kKSimtPrep, stream, simt_prep_kernel<<<simt_grid(p), kThreads, 0, stream>>>(p));
    if (nstate > 0) {
        const size_t sm = state_smem(p.K, false);
        cudaError_t e = cudaFuncSetAttribute(simt_state_fwd_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        if (e != cudaSuccess) return e;
        GDN_LAUNCH(kKSimtStateFwd, stream,
                   simt_state_fwd_kernel<<<nstate, kThreads, sm, stream>>>(p));
    }
    if (p.NC > 0)
        GDN_LAUNCH(kKSimtOut, stream, simt_out_kernel<<<simt_grid(p), kThreads, 0, stream>>>(p));
    return cudaSuccess;
}

cudaError_t launch_simt_bwd(const Params &p, cudaStream_t stream) {
    const int nstate = p.N * p.H * (p.V / kSimtVSlice);
    Params pf = p;
    pf.hT = nullptr;  // the recompute pass only needs the per-chunk states
    if (p.NC > 0)
        GDN_LAUNCH(kKSimtPrep, stream, simt_prep_kernel<<<simt_grid(p), kThreads, 0, stream>>>(p));
    if (nstate > 0) {
        const size_t sm = state_smem(p.K, false);
        cudaError_t e = cudaFuncSetAttribute(simt_state_fwd_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        if (e != cudaSuccess) return e;
        GDN_LAUNCH(kKSimtStateFwd, stream,
                   simt_state_fwd_kernel<<<nstate, kThreads, sm, stream>>>(pf));
    }
    if (p.NC > 0)
        GDN_LAUNCH(kKSimtDuloc, stream,
                   simt_duloc_kernel<<<simt_grid(p), kThreads, 0, stream>>>(p));
    if (nstate > 0) {
        const size_t sm = state_smem(p.K, true);
        cudaError_t e = cudaFuncSetAttribute(simt_state_bwd_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        if (e != cudaSuccess) return e;
        GDN_LAUNCH(kKSimtStateBwd, stream,
                   simt_state_bwd_kernel<<<nstate, kThreads, sm, stream>>>(p));
    }
    if (p.NC > 0)
        GDN_LAUNCH(kKSimtGrads, stream,
                   simt_grads_kernel<<<simt_grid(p), kThreads, 0, stream>>>(p));
    return cudaSuccess;
}

}  // namespace gdn
