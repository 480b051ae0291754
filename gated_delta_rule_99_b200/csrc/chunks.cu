// Chunk index build: cu_seqlens (or dense rows) -> per-chunk table.
//
// Chunks restart at every document start so that a packed row is computed
// exactly as its documents one by one (jax-linear-attention 0.1.0, "How it
// works": packed documents reset the state at every boundary).  Integer work
// only; the table is bit-exact by construction.
#include "gdn_internal.cuh"

namespace gdn {
namespace {

constexpr int kThreads = 1024;

__device__ __forceinline__ int64_t seq_start(const Params &p, int n) {
    return p.cu ? (int64_t)p.cu[n] : (int64_t)n * p.T;
}

__global__ void __launch_bounds__(kThreads) build_chunks_kernel(Params p) {
    __shared__ int32_t scan[kThreads];
    __shared__ int32_t carry, bad;
    const int tid = threadIdx.x;
    if (tid == 0) {
        carry = 0;
        bad = 0;
        if (seq_start(p, 0) != 0 || seq_start(p, p.N) != p.BT) bad = 1;
    }
    __syncthreads();
    for (int base = 0; base < p.N; base += kThreads) {
        const int n = base + tid;
        int cnt = 0;
        if (n < p.N) {
            const int64_t s0 = seq_start(p, n), s1 = seq_start(p, n + 1);
            if (s1 < s0) bad = 1;
            else cnt = (int)((s1 - s0 + kChunk - 1) / kChunk);
        }
        scan[tid] = cnt;
        __syncthreads();
        for (int off = 1; off < kThreads; off <<= 1) {
            const int add = tid >= off ? scan[tid - off] : 0;
            __syncthreads();
            scan[tid] += add;
            __syncthreads();
        }
        if (n < p.N) p.seq_first[n] = carry + scan[tid] - cnt;
        __syncthreads();
        if (tid == kThreads - 1) carry += scan[kThreads - 1];
        __syncthreads();
    }
    if (tid == 0 && carry != p.NC) bad = 1;
    __syncthreads();
    if (bad) {
        if (tid == 0) {
            p.hdr->status = kDevBadSeqlens;
            p.hdr->n_chunks = 0;
            p.hdr->where = 0;
        }
        return;
    }
    if (tid == 0) {
        p.seq_first[p.N] = carry;
        p.hdr->status = kDevOk;
        p.hdr->n_chunks = carry;
        p.hdr->where = 0;
    }
    for (int n = tid; n < p.N; n += kThreads) {
        const int64_t s0 = seq_start(p, n), s1 = seq_start(p, n + 1);
        const int first = p.seq_first[n];
        const int cnt = (int)((s1 - s0 + kChunk - 1) / kChunk);
        for (int j = 0; j < cnt; ++j) {
            ChunkInfo ci;
            ci.seq = n;
            ci.tok0 = (int32_t)(s0 + (int64_t)j * kChunk);
            ci.len = (int32_t)((s1 - ci.tok0) < kChunk ? (s1 - ci.tok0) : kChunk);
            ci.idx = j;
            p.chunks[first + j] = ci;
        }
    }
}

}  // namespace

cudaError_t launch_build_chunks(const Params &p, cudaStream_t stream) {
    GDN_LAUNCH(kKBuildChunks, stream, build_chunks_kernel<<<1, kThreads, 0, stream>>>(p));
    return cudaSuccess;
}

}  // namespace gdn
