// Shared helpers of the tensor-core kernels (forward in tc.cu, backward in
// tc_bwd.cu): tile loads into 128-byte-swizzled shared memory, per-chunk
// gates, bounded MMA waits, bf16 packing, TMEM addressing.
#pragma once

#include "gdn_internal.cuh"
#include "tc_ptx.cuh"

namespace gdn {
namespace tc {

using namespace ptx;
using bf16 = __nv_bfloat16;


constexpr int C = kChunk;      // 64
constexpr int D = 128;         // d_k = d_v
constexpr int NT = 128;        // threads per CTA

constexpr size_t kImg64 = (size_t)C * D * 2;   // 64 x 128 bf16 tile image (16 KB)
constexpr size_t kImg128 = (size_t)D * D * 2;  // 128 x 128 (32 KB)
constexpr size_t kImgUT = (size_t)D * C * 2;   // 128 x 64 (16 KB)

__device__ __forceinline__ uint8_t *align1k(uint8_t *p) {
    return (uint8_t *)(((uintptr_t)p + 1023) & ~(uintptr_t)1023);
}

__device__ __forceinline__ void record_timeout(const Params &p, int where) {
    atomicExch(&p.hdr->status, kDevTimeout);
    atomicExch(&p.hdr->where, where);
}

// Bounded wait on an MMA-completion barrier, decided uniformly by the CTA.
__device__ __forceinline__ bool cta_wait(uint64_t *mbar, uint32_t parity, const Params &p,
                                         int where) {
    const bool ok = mbar_wait(mbar, parity, p.wait_limit);
    const bool all_ok = __syncthreads_and(ok);
    if (!all_ok && threadIdx.x == 0) record_timeout(p, where);
    tc_fence_after();
    return all_ok;
}

// Barrier that orders generic smem writes (operands) before MMAs issued after it.
__device__ __forceinline__ void operands_ready() {
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
}

// Bytes one load_rows_tma call completes on its mbarrier (one 64 x 64 box per
// 64 columns of the source rows).
__device__ __forceinline__ uint32_t row_tile_bytes(int width) { return width == D ? 16384u : 8192u; }

// Rows [0, 64) of one chunk and head (tokens tok0..tok0+63 of head h) of a
// [tokens][H][width] bf16 tensor (width 64 or 128) into the first width/64
// column blocks of an SW128 tile with R rows, starting at row `row0` (0 or 64):
// one 64 x 64 box per block by the tensor engine, row_tile_bytes(width) on
// `bar`.  One thread issues it.  Tokens past the tensor arrive as zeros; the
// rows past the chunk's end and the columns past `width` are cleared by
// fix_rows once the copy has landed.
__device__ __forceinline__ void load_rows_tma(uint8_t *tile, int R, int row0,
                                              const CUtensorMap *map, int64_t tok0, int h,
                                              int width, uint64_t *bar) {
    const uint32_t base = smem_u32(tile) + (uint32_t)row0 * 128u;
    tma_load_3d(base, map, 0, h, (int)tok0, bar);
    if (width == D) tma_load_3d(base + (uint32_t)R * 128u, map, 64, h, (int)tok0, bar);
}

// Zeroes, in the tile block load_rows_tma filled, the rows at or past `len`
// (in a chunk shorter than 64 they hold the next sequence's tokens) and, for a
// head dim of 64, the second 64-column block (a head dim of 64 runs on the
// 128-wide tiles: the zero columns add nothing to any product, and the state's
// padded rows and columns stay zero).
__device__ __forceinline__ void fix_rows(uint8_t *tile, int R, int row0, int len, int width,
                                         int nthreads = NT) {
    if (len >= C && width == D) return;
    for (int t = threadIdx.x; t < C * 16; t += nthreads) {
        const int r = t >> 4, j = t & 15;
        if (r >= len || j * 8 >= width)
            *reinterpret_cast<uint4 *>(tile + sw128_chunk(R, row0 + r, j)) = make_uint4(0, 0, 0, 0);
    }
}

// Bounded wait for phase `parity` of `bar` (a CTA's input copies), decided by the
// whole CTA (a barrier); the caller must have made the mbarrier's init visible
// to every thread (a barrier after it) first.  On failure records `where` and
// waits once more, bounded, so that no copy is left in flight when the CTA
// gives up.
__device__ __forceinline__ bool copies_arrived(uint64_t *bar, const Params &p, int where,
                                               uint32_t parity = 0) {
    const bool ok = __syncthreads_and(mbar_wait(bar, parity, p.wait_limit));
    if (!ok && threadIdx.x == 0) {
        record_timeout(p, where);
        mbar_wait(bar, parity, kWaitLimit);
    }
    return ok;
}

// In-chunk cumulative log-decay (zero gates past len) and the write strengths.
// Threads 0-63 hold one token each: an inclusive shuffle scan inside each warp
// (five steps, each lane adding in the same fixed order), then the second warp
// adds the first warp's total.  Every kernel runs this same code, so all get
// bit-identical values.  Called by the whole CTA (it ends with a barrier).
__device__ __forceinline__ void chunk_gates(float *G, float *bta, const Params &p, const ChunkInfo &ci, int h) {
    const int r = threadIdx.x;
    if (r < C) {
        const int64_t idx = (int64_t)(ci.tok0 + r) * p.H + h;
        float x = r < ci.len ? p.g[idx] : 0.f;
        if (bta) bta[r] = r < ci.len ? p.beta[idx] : 0.f;
        const int l = r & 31;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, x, off);
            if (l >= off) x += y;
        }
        G[r] = x;
    }
    __syncthreads();
    if (r >= 32 && r < C) G[r] += G[31];
    __syncthreads();
}

__device__ __forceinline__ void unpack8(uint4 u, float *f) {
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 x = __bfloat1622float2(h[i]);
        f[2 * i] = x.x;
        f[2 * i + 1] = x.y;
    }
}

__device__ __forceinline__ uint4 pack8(const float *f) {
    uint4 u;
    u.x = pack_bf16(f[0], f[1]);
    u.y = pack_bf16(f[2], f[3]);
    u.z = pack_bf16(f[4], f[5]);
    u.w = pack_bf16(f[6], f[7]);
    return u;
}

// Writes x[0, 2 NW) as NW packed bf16 pairs (the lower element in the low half) to
// TMEM columns [0, NW) from taddr in this thread's lane: a row of a K-major A
// operand of the products (NW a multiple of 16).  Warp-collective.
template <int NW>
__device__ __forceinline__ void tmem_store_bf16(uint32_t taddr, const float *x) {
#pragma unroll
    for (int c = 0; c < NW; c += 16) {
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) w[i] = pack_bf16(x[2 * (c + i)], x[2 * (c + i) + 1]);
        tmem_st16(taddr + (uint32_t)c, w);
    }
}

// TMEM address of (lane base of this warp, column col).
__device__ __forceinline__ uint32_t tm(uint32_t tmem, int col) {
    return tmem + ((uint32_t)((threadIdx.x >> 5) * 32) << 16) + (uint32_t)col;
}

// TMEM address for CTAs of more than four warps: warp w reaches the lane
// quadrant w % 4 only.
__device__ __forceinline__ uint32_t tmq(uint32_t tmem, int col) {
    return tmem + ((uint32_t)(((threadIdx.x >> 5) & 3) * 32) << 16) + (uint32_t)col;
}

// Row of a 64-row (M = 64) accumulator held by this thread's lane, or -1.
__device__ __forceinline__ int m64_row() {
    const int l = threadIdx.x & 31;
    return l < 16 ? (int)(threadIdx.x >> 5) * 16 + l : -1;
}


template <typename Kern>
inline cudaError_t set_smem(Kern k, int bytes) {
    return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

// Grid of a persistent launch: `per_sm` CTAs on every SM of the current device, or
// one per unit if there are fewer units.
inline cudaError_t persistent_grid(int units, int per_sm, int &grid) {
    int dev = 0, nsm = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    grid = units < per_sm * nsm ? units : per_sm * nsm;
    return e;
}

// The layer's optional q/k normalisation inside a kernel (jax-linear-attention
// 0.1.0, "Quick start": use_qk_l2norm=True): rows [row0, row0 + 64) of a bf16
// SW128 tile with R rows and 128 columns are divided by their Euclidean norms
// (fp32 sums of squares in a fixed order; a zero row stays zero) and rounded
// back to bf16 in place; 1/|row| goes to inv[] when it is given.  Threads
// [tbase, tbase + 128) take two per row.  Every kernel that loads a q or k tile
// runs this same code, so all see bit-identical normalised rows.
__device__ __forceinline__ void l2norm_tile_rows(uint8_t *tile, int R, int row0, float *inv,
                                                 int tbase = 0) {
    const int t = (int)threadIdx.x - tbase;
    if (t < 0 || t >= 2 * C) return;
    const int r = t >> 1, half = t & 1;
    float s = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        float f[8];
        unpack8(*reinterpret_cast<const uint4 *>(tile + sw128_chunk(R, row0 + r, 8 * half + j)), f);
#pragma unroll
        for (int q = 0; q < 8; ++q) s = fmaf(f[q], f[q], s);
    }
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    const float rn = s > 0.f ? 1.f / sqrtf(s) : 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        uint4 *ch = reinterpret_cast<uint4 *>(tile + sw128_chunk(R, row0 + r, 8 * half + j));
        float f[8];
        unpack8(*ch, f);
#pragma unroll
        for (int q = 0; q < 8; ++q) f[q] *= rn;
        *ch = pack8(f);
    }
    if (inv && half == 0) inv[r] = rn;
}

// P = scale lower(Q K^T . Gam), diagonal included, from the M = 64 accumulator at
// TMEM column 0 into a 64 x 64 bf16 SW128 tile (CTAs of four warps).  The rows
// of a warp lie in one 16-block, so the blocks above it are written as zeros
// without evaluating their decays.
__device__ __forceinline__ void build_p_tile(uint32_t tmem, const float *G, float scale,
                                             uint8_t *Ps) {
    const int i = m64_row();
    float d[4][16];
#pragma unroll
    for (int cb = 0; cb < 4; ++cb) tmem_ld16(tm(tmem, 16 * cb), d[cb]);
    tmem_ld_wait();
    if (i < 0) return;
    const int ib = i >> 4;
    const float gi = G[i];
#pragma unroll
    for (int cb = 0; cb < 4; ++cb) {
        if (cb <= ib) {
#pragma unroll
            for (int q = 0; q < 16; ++q) {
                const int j = 16 * cb + q;
                d[cb][q] = j <= i ? scale * expf(gi - G[j]) * d[cb][q] : 0.f;
            }
        } else {
#pragma unroll
            for (int q = 0; q < 16; ++q) d[cb][q] = 0.f;
        }
        *reinterpret_cast<uint4 *>(Ps + sw128_chunk(C, i, 2 * cb)) = pack8(d[cb]);
        *reinterpret_cast<uint4 *>(Ps + sw128_chunk(C, i, 2 * cb + 1)) = pack8(d[cb] + 8);
    }
}

}  // namespace tc
}  // namespace gdn
