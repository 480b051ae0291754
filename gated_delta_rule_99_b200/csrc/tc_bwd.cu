// Tensor-core (tcgen05) backward of the bf16 layer, d_k = d_v = 128.
//
// Reverse-mode of the chunkwise forward (see tc.cu).  After the forward
// pieces are recomputed (tc_prep keeps A in fp32; tc_state_fwd rewrites the
// state entering every chunk and U^T), three kernels run:
//
//   tc_local      chunk-parallel: P = scale lower(Q K^T . Gam), the local
//                 dU^T = dO^T P, and Qg = scale diag(gam) Q (a tile image)
//   tc_state_bwd  serial over the chunks of a sequence, in reverse; thread v
//                 owns row v of dS = dH^T (fp32 registers); per chunk
//                   dU^T = dS Kd^T + (local dU^T)
//                   dS  <- gam_n dS + dO^T Qg - dU^T W
//                 and writes dS (the gradient of the state leaving the chunk)
//                 and dU^T as tile images
//   tc_grads      chunk-parallel: every chunk-local gradient (dq, dk, dv, dg,
//                 dbeta) from the recomputed and propagated pieces.
//
// Products run in transposed form wherever that lets the accumulator use all
// 128 TMEM lanes (M = 128 over the key or value dim); 64 x 64 products use the
// M = 64 form (row m in lane 32 (m / 16) + m % 16).
#include "tc_common.cuh"
#include "tc_prep.cuh"
#include "tc_state.cuh"

namespace gdn {


namespace {

using namespace tc;

// ============================================================ tc_local
struct LocalSmem {
    // P overwrites the Q half of the [Q; K] tile once Q K^T and Qg have consumed it
    static constexpr int kQK = 0, kDO = kQK + 32768, kP = kQK, kG = kDO + 16384, kEnd = kG + 256;
};
constexpr int kLocalSmem = LocalSmem::kEnd + 1024;

// Body of the local step for CTA `ch` (chunk ch / H, head ch % H).  It forms
// the chunk gates itself (the same code as tc_prep, so bit-identical), which
// makes it independent of tc_prep: the two share one launch.
__device__ __forceinline__ void local_body(const Params &p, int ch) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = align1k(smem_raw);
    __shared__ uint64_t mbar, lbar;
    __shared__ uint32_t tslot;
    if (p.hdr->status) return;
    const int H = p.H, c = ch / H, h = ch % H, tid = threadIdx.x;
    const ChunkInfo ci = chunk_at(p, c);
    uint8_t *QK = sm + LocalSmem::kQK, *DO = sm + LocalSmem::kDO, *Ps = sm + LocalSmem::kP;
    float *G = reinterpret_cast<float *>(sm + LocalSmem::kG);
    if (tid == 0) {  // q, k and dO rows by the tensor engine
        mbar_init(&mbar, 1);
        mbar_init(&lbar, 1);
        fence_mbar_init();
        mbar_arrive_expect_tx(&lbar, 2 * row_tile_bytes(p.K) + row_tile_bytes(p.V));
        load_rows_tma(QK, D, 0, &p.tm_q, ci.tok0, h, p.K, &lbar);
        load_rows_tma(QK, D, C, &p.tm_k, ci.tok0, h, p.K, &lbar);
        load_rows_tma(DO, C, 0, &p.tm_do, ci.tok0, h, p.V, &lbar);
    }
    if (tid < 32) {
        tmem_alloc(&tslot, 128);
        tmem_relinquish();
    }
    chunk_gates(G, nullptr, p, ci, h);  // its barriers also publish the mbarrier inits
    bool ok = copies_arrived(&lbar, p, 32);
    if (ok) {
        fix_rows(QK, D, 0, ci.len, p.K);
        fix_rows(QK, D, C, ci.len, p.K);
        fix_rows(DO, C, 0, ci.len, p.V);
    }
    operands_ready();
    if (ok && p.l2norm) {  // q and k rows divided by their norms
        l2norm_tile_rows(QK, D, 0, nullptr);
        l2norm_tile_rows(QK, D, C, nullptr);
        operands_ready();
    }
    const uint32_t tmem = tslot;
    if (ok && tid == 0) {  // Q K^T: M = 64, N = 64, K = 128
        const uint32_t qb = smem_u32(QK), kb = qb + C * 128, id = idesc_bf16(64, 64, 0, 0);
#pragma unroll
        for (int s = 0; s < D / 16; ++s)
            mma_bf16(tmem, desc_kmajor(qb, D, s), desc_kmajor(kb, D, s), id, s > 0);
        mma_commit(&mbar);
    }
    if (ok) {  // Qg = scale diag(gam) Q: an operand of the reverse state pass (tile image)
        uint8_t *img = static_cast<uint8_t *>(p.tQg) + (size_t)ch * kImg64;
        for (int t = tid; t < C * 16; t += NT) {
            const int r = t >> 4, j = t & 15;
            float f[8];
            unpack8(*reinterpret_cast<const uint4 *>(QK + sw128_chunk(D, r, j)), f);
            const float s = p.scale * expf(G[r]);
#pragma unroll
            for (int q = 0; q < 8; ++q) f[q] *= s;
            *reinterpret_cast<uint4 *>(img + sw128_chunk(C, r, j)) = pack8(f);
        }
    }
    if (ok) ok = cta_wait(&mbar, 0, p, 11);
    if (ok) {
        const int i = m64_row();
        for (int c0 = 0; c0 < C; c0 += 16) {
            float d[16];
            tmem_ld16(tm(tmem, c0), d);
            tmem_ld_wait();
            if (i >= 0) {
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    const int j = c0 + q;
                    d[q] = j <= i ? p.scale * expf(G[i] - G[j]) * d[q] : 0.f;
                }
                *reinterpret_cast<uint4 *>(Ps + sw128_chunk(C, i, c0 / 8)) = pack8(d);
                *reinterpret_cast<uint4 *>(Ps + sw128_chunk(C, i, c0 / 8 + 1)) = pack8(d + 8);
            }
        }
        operands_ready();
        if (tid == 0) {  // local dU^T[v][j] = sum_i dO[i][v] P[i][j]: M = 128, N = 64, K = 64
            const uint32_t db = smem_u32(DO), pb = smem_u32(Ps), id = idesc_bf16(128, 64, 1, 1);
#pragma unroll
            for (int s = 0; s < C / 16; ++s)
                mma_bf16(tmem + 64, desc_mnmajor(db, C, s), desc_mnmajor(pb, C, s), id, s > 0);
            mma_commit(&mbar);
        }
        ok = cta_wait(&mbar, 1, p, 12);
    }
    if (ok) {
        uint8_t *dul = static_cast<uint8_t *>(p.tdUL) + (size_t)ch * kImgUT;
        for (int c0 = 0; c0 < C; c0 += 16) {
            float d[16];
            tmem_ld16(tm(tmem, 64 + c0), d);
            tmem_ld_wait();
            *reinterpret_cast<uint4 *>(dul + sw128_chunk(D, tid, c0 / 8)) = pack8(d);
            *reinterpret_cast<uint4 *>(dul + sw128_chunk(D, tid, c0 / 8 + 1)) = pack8(d + 8);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (tid < 32) tmem_dealloc(tmem, 128);
}

// tc_prep (with A for the backward) on CTAs [0, NC*H) and tc_local on
// [NC*H, 2*NC*H): independent chunk-parallel steps in one launch.
__global__ void __launch_bounds__(NT, 4) tc_prep_local_kernel(const __grid_constant__ Params p) {
    const int nch = p.NC * p.H;
    if ((int)blockIdx.x < nch) prep_body(p, blockIdx.x, 1);
    else local_body(p, blockIdx.x - nch);
}

// ============================================================ tc_state_bwd
struct SbwdSmem {
    static constexpr int kdS = 0, kdU = kdS + 32768, kBuf = kdU + 16384;
    // per buffer: Kd image, W image, Qg image, dO tile, local dU^T rows, gates
    static constexpr int kKd = 0, kW = 16384, kQg = 32768, kDO = 49152, kDUL = 65536,
                         kG = 81920, kBufBytes = 81920 + 1024;
    static constexpr int kEnd = kBuf + 2 * kBufBytes;
};
constexpr int kSbwdSmem = SbwdSmem::kEnd + 1024;

// Chunk ch's Kd, W and Qg images, local dU^T image and gate row by bulk copies,
// its dO rows by the tensor engine (thread 0, all completing on `bar`).
__device__ __forceinline__ void sbwd_prefetch(uint8_t *sm, int buf, size_t ch,
                                              const ChunkInfo &ci, int h, const Params &p,
                                              uint64_t *bar) {
    uint8_t *b = sm + SbwdSmem::kBuf + buf * SbwdSmem::kBufBytes;
    if (threadIdx.x == 0) {
        mbar_arrive_expect_tx(bar, 3u * (uint32_t)kImg64 + (uint32_t)kImgUT + C * 4u +
                                       row_tile_bytes(p.V));
        bulk_load(smem_u32(b + SbwdSmem::kKd), static_cast<const uint8_t *>(p.tKd) + ch * kImg64,
                  kImg64, bar);
        bulk_load(smem_u32(b + SbwdSmem::kW), static_cast<const uint8_t *>(p.tW) + ch * kImg64,
                  kImg64, bar);
        bulk_load(smem_u32(b + SbwdSmem::kQg), static_cast<const uint8_t *>(p.tQg) + ch * kImg64,
                  kImg64, bar);
        bulk_load(smem_u32(b + SbwdSmem::kDUL),
                  static_cast<const uint8_t *>(p.tdUL) + ch * kImgUT, kImgUT, bar);
        bulk_load(smem_u32(b + SbwdSmem::kG), p.tG + ch * C, C * 4, bar);
        load_rows_tma(b + SbwdSmem::kDO, C, 0, &p.tm_do, ci.tok0, h, p.V, bar);
    }
}

// Body of the reverse state pass for CTA `blk` (sequence blk / H, head blk % H).
__device__ __forceinline__ void state_bwd_body(const Params &p, int blk) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = align1k(smem_raw);
    __shared__ uint64_t mbar, lbar[2];
    __shared__ uint32_t tslot;
    if (p.hdr->status) return;
    const int H = p.H, n = blk / H, h = blk % H, v = threadIdx.x;
    float S[D];  // dS row v (gradient of the state leaving the current chunk)
    if (p.dhT) {  // [K][V] blocks; rows and columns past them are zero
        const float *g0 = p.dhT + ((size_t)n * H + h) * p.K * p.V;
#pragma unroll
        for (int kk = 0; kk < D; ++kk) S[kk] = (kk < p.K && v < p.V) ? g0[kk * p.V + v] : 0.f;
    } else {
#pragma unroll
        for (int kk = 0; kk < D; ++kk) S[kk] = 0.f;
    }
    if (v == 0) {
        mbar_init(&mbar, 1);
        mbar_init(&lbar[0], 1);
        mbar_init(&lbar[1], 1);
        fence_mbar_init();
    }
    if (v < 32) {
        tmem_alloc(&tslot, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tslot;
    const int c0 = seq_first_at(p, n), c1 = seq_first_at(p, n + 1);
    uint32_t phase = 0;
    // per buffer b (bit b): bulk copies in flight, and the parity of their next completion
    uint32_t pend = 0, lpar = 0;
    if (c0 < c1) {
        sbwd_prefetch(sm, 0, (size_t)(c1 - 1) * H + h, chunk_in_seq(p, n, c0, c1 - 1), h, p,
                      &lbar[0]);
        pend = 1;
    }
    uint8_t *dSs = sm + SbwdSmem::kdS, *dUs = sm + SbwdSmem::kdU;
    const uint32_t id1 = idesc_bf16(128, 64, 0, 0), idx = idesc_bf16(128, 128, 1, 1),
                   idy = idesc_bf16(128, 128, 0, 1);
    for (int c = c1 - 1; c >= c0; --c) {
        const int buf = (c1 - 1 - c) & 1;
        const size_t ch = (size_t)c * H + h;
        if (c - 1 >= c0) {
            sbwd_prefetch(sm, buf ^ 1, ch - H, chunk_in_seq(p, n, c0, c - 1), h, p,
                          &lbar[buf ^ 1]);
            pend |= 2u >> buf;
        }
        const bool lok = mbar_wait(&lbar[buf], (lpar >> buf) & 1u, kWaitLimit);
        uint8_t *b = sm + SbwdSmem::kBuf + buf * SbwdSmem::kBufBytes;
        if (lok) fix_rows(b + SbwdSmem::kDO, C, 0, chunk_in_seq(p, n, c0, c).len, p.V);
#pragma unroll
        for (int j = 0; j < 16; ++j)
            *reinterpret_cast<uint4 *>(dSs + sw128_chunk(D, v, j)) = pack8(S + 8 * j);
        fence_async_smem();
        tc_fence_before();
        const bool all = __syncthreads_and(lok);
        tc_fence_after();
        if (!all) {
            if (v == 0) record_timeout(p, 45);
            break;
        }
        pend &= ~(1u << buf);
        lpar ^= 1u << buf;
        const float gC = expf(reinterpret_cast<const float *>(b + SbwdSmem::kG)[C - 1]);
        if (v == 0) {
            const uint32_t sb = smem_u32(dSs), kb = smem_u32(b + SbwdSmem::kKd),
                           qb = smem_u32(b + SbwdSmem::kQg), ob = smem_u32(b + SbwdSmem::kDO);
            // dS Kd^T: M = 128 (v), N = 64 tokens, K = 128 keys
#pragma unroll
            for (int s = 0; s < D / 16; ++s)
                mma_bf16(tmem, desc_kmajor(sb, D, s), desc_kmajor(kb, C, s), id1, s > 0);
            // dO^T Qg: M = 128 (v), N = 128 keys, K = 64 tokens
#pragma unroll
            for (int s = 0; s < C / 16; ++s)
                mma_bf16(tmem + 64, desc_mnmajor(ob, C, s), desc_mnmajor(qb, C, s), idx, s > 0);
            mma_commit(&mbar);
            bulk_store(static_cast<uint8_t *>(p.tdSn) + ch * kImg128, sb, (uint32_t)kImg128);
            bulk_commit();
        }
        if (!cta_wait(&mbar, phase, p, 13)) break;
        phase ^= 1;
        {  // dU^T = dS Kd^T + local dU^T: the next operand, and (bulk-stored) an image for tc_grads
            const uint8_t *dul = b + SbwdSmem::kDUL;  // local dU^T, swizzled rows
#pragma unroll
            for (int c16 = 0; c16 < C; c16 += 16) {
                float d[16], l[16];
                tmem_ld16(tm(tmem, c16), d);
                tmem_ld_wait();
                unpack8(*reinterpret_cast<const uint4 *>(dul + sw128_chunk(D, v, c16 / 8)), l);
                unpack8(*reinterpret_cast<const uint4 *>(dul + sw128_chunk(D, v, c16 / 8 + 1)),
                        l + 8);
#pragma unroll
                for (int q = 0; q < 16; ++q) d[q] += l[q];
                *reinterpret_cast<uint4 *>(dUs + sw128_chunk(D, v, c16 / 8)) = pack8(d);
                *reinterpret_cast<uint4 *>(dUs + sw128_chunk(D, v, c16 / 8 + 1)) = pack8(d + 8);
            }
        }
        operands_ready();
        if (v == 0) {  // + dU^T (-W): M = 128 (v), N = 128 keys, K = 64 tokens (W image negated)
            const uint32_t ub = smem_u32(dUs), wb = smem_u32(b + SbwdSmem::kW);
#pragma unroll
            for (int s = 0; s < C / 16; ++s)
                mma_bf16(tmem + 64, desc_kmajor(ub, D, s), desc_mnmajor(wb, C, s), idy, 1);
            mma_commit(&mbar);
            bulk_store(static_cast<uint8_t *>(p.tdUT) + ch * kImgUT, ub, (uint32_t)kImgUT);
            bulk_commit();
        }
        if (!cta_wait(&mbar, phase, p, 14)) break;
        phase ^= 1;
#pragma unroll
        for (int c32 = 0; c32 < D; c32 += 32) {
            float d[32];
            tmem_ld16(tm(tmem, 64 + c32), d);
            tmem_ld16(tm(tmem, 64 + c32 + 16), d + 16);
            tmem_ld_wait();
#pragma unroll
            for (int q = 0; q < 32; ++q) S[c32 + q] = fmaf(gC, S[c32 + q], d[q]);
        }
        if (v == 0) bulk_wait_read();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }
    if (v == 0) {  // copies still in flight after an early exit
        for (int q = 0; q < 2; ++q)
            if ((pend >> q) & 1u) mbar_wait(&lbar[q], (lpar >> q) & 1u, kWaitLimit);
        bulk_wait_all();
    }
    if (p.dh0) {
        float *g0 = p.dh0 + ((size_t)n * H + h) * p.K * p.V;
        if (v < p.V) {
#pragma unroll
            for (int kk = 0; kk < D; ++kk)
                if (kk < p.K) g0[kk * p.V + v] = S[kk];
        }
    }
    tc_fence_before();
    __syncthreads();
    if (v < 32) tmem_dealloc(tmem, 256);
}

// Both chains of the backward in one launch: CTAs [0, N*H) recompute the
// forward states (pf has no final-state output), CTAs [N*H, 2*N*H) run the
// reverse pass.  They are independent, so each gets its own SMs.
__global__ void __launch_bounds__(NT, 1) tc_chains_kernel(const __grid_constant__ Params pf,
                                                           const __grid_constant__ Params pb) {
    const int nh = pb.N * pb.H;
    if ((int)blockIdx.x < nh) state_fwd_body(pf, blockIdx.x);
    else state_bwd_body(pb, blockIdx.x - nh);
}

// ============================================================ tc_grads
// Four warpgroups (512 threads): warp w reaches TMEM lane quadrant w % 4, so
// for every 64-column accumulator warpgroup g handles columns [16 g, 16 g + 16).
constexpr int NG = 512;
constexpr int CW = 16;  // columns per warpgroup

struct GradSmem {
    static constexpr int kQK = 0, kDO = 32768, kV = 49152, kSC = 65536, kDSN = 98304,
                         kUT = 131072, kDUT = 147456, kAB = 163840, kX3 = 172032,
                         kDA = 188416, kT1 = 196608, kDPG = 204800, kDLG = 212992,
                         kVec = 221184, kEnd = kVec + 24 * 256;
    // reused once the first products have consumed the images there: fp32
    // 64 x 65 P (then dP.P + dL.L) and Gam.KK^T, per-warp partial column sums
    // [3][4][64], and the 64 x 64 decay matrix Gam (columns xor-swizzled by row)
    static constexpr int kPE = kSC, kKKG = kSC + 64 * 65 * 4, kRed = kDSN + 1024,
                         kGam = kDUT;
};
constexpr int kGradSmem = GradSmem::kEnd + 1024;
constexpr int LP = 65;  // padded row stride (floats) of the fp32 scratch

__device__ __forceinline__ int gidx(int i, int j) { return i * 64 + (j ^ (i & 31)); }

// Column c of an SW128 tile with R rows, read row by row: the swizzle term
// depends on the row only through row % 8, so it is computed once.
struct ColSw {
    const uint8_t *col;
    uint32_t x[8];
    __device__ __forceinline__ ColSw(const uint8_t *tile, int R, int c) {
        col = tile + (c >> 6) * R * 128 + (c & 7) * 2;
        const int cp = (c & 63) >> 3;
#pragma unroll
        for (int b = 0; b < 8; ++b) x[b] = (uint32_t)((cp ^ b) << 4);
    }
    // row i = i0 + q with i0 a multiple of 8 and q a compile-time constant
    __device__ __forceinline__ float at(int i0, int q) const {
        return __bfloat162float(
            *reinterpret_cast<const bf16 *>(col + (i0 + q) * 128 + x[q & 7]));
    }
};

// Copies rows [0, len) and columns [0, width) of a 64 x 128 bf16 staging tile
// (plain rows) to one chunk and head of a [tokens][H][width] tensor with
// 16-byte stores.
__device__ __forceinline__ void store_rows(bf16 *dst, const uint8_t *stage, int64_t tok0, int len,
                                           int h, int H, int width) {
    for (int t = threadIdx.x; t < C * 16; t += NG) {
        const int i = t >> 4, j = t & 15;
        if (i < len && j * 8 < width)
            *reinterpret_cast<uint4 *>(dst + ((tok0 + i) * H + h) * width + j * 8) =
                *reinterpret_cast<const uint4 *>(stage + i * 256 + j * 16);
    }
}


// Column sums over the 32 lanes of a warp of the CW = 16 values v[q] that each
// thread holds (lane l of the warp is row l of a 32-row slice; v[q] belongs to
// column cb + q): a butterfly that halves the values at every step leaves the
// sum of column cb + q(l) in lane l, q(l) = 8 b4 + 4 b3 + 2 b2 + b1 with b the
// lane's bits, written by the even lanes to wsum[w4][cb + q].
__device__ __forceinline__ void warp_colsum(float *v, float *wsum, int w4, int cb, int l) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const bool up = l & 16;
        const float send = up ? v[k] : v[k + 8], keep = up ? v[k + 8] : v[k];
        v[k] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const bool up = l & 8;
        const float send = up ? v[k] : v[k + 4], keep = up ? v[k + 4] : v[k];
        v[k] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const bool up = l & 4;
        const float send = up ? v[k] : v[k + 2], keep = up ? v[k + 2] : v[k];
        v[k] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
    }
    {
        const bool up = l & 2;
        const float send = up ? v[0] : v[1], keep = up ? v[1] : v[0];
        v[0] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
    }
    v[0] += __shfl_xor_sync(0xffffffffu, v[0], 1);
    const int q = ((l >> 4) & 1) * 8 + ((l >> 3) & 1) * 4 + ((l >> 2) & 1) * 2 + ((l >> 1) & 1);
    if (!(l & 1)) wsum[w4 * 64 + cb + q] = v[0];
}

// Backward of the optional row normalisation for this thread's column of 16
// tokens i = cb + q (x holds the gradient w.r.t. the normalised rows u):
// x <- (x - u (u . x)) / |row|, the dot products over the 128 columns summed by
// warp butterflies and four warp partials.  Called by every thread of the CTA.
__device__ __forceinline__ void project_rows(float *x, const ColSw &u, const float *inv,
                                             float *dot, float *wsum, int w4, int cb, int l) {
    float y[CW];
#pragma unroll
    for (int q = 0; q < CW; ++q) y[q] = u.at(cb, q) * x[q];
    warp_colsum(y, wsum, w4, cb, l);
    __syncthreads();
    if (threadIdx.x < C) {
        const int t = threadIdx.x;
        dot[t] = (wsum[t] + wsum[64 + t]) + (wsum[128 + t] + wsum[192 + t]);
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < CW; ++q) {
        const int i = cb + q;
        x[q] = (x[q] - u.at(cb, q) * dot[i]) * inv[i];
    }
}

// CW consecutive fp32 columns of this thread's TMEM lane (quadrant w % 4).
__device__ __forceinline__ void ldcw(uint32_t tmem, int col, float *d) {
    tmem_ld16(tmq(tmem, col), d);
    tmem_ld_wait();
}

__global__ void __launch_bounds__(NG, 1) tc_grads_kernel(const __grid_constant__ Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = align1k(smem_raw);
    __shared__ uint64_t mbar;
    __shared__ uint32_t tslot;
    __shared__ float s_hd;
    if (p.hdr->status) return;
    const int H = p.H, ch = blockIdx.x, c = ch / H, h = ch % H, tid = threadIdx.x;
    const int wg = tid >> 7, r = tid & 127, cb = CW * wg;
    const int l = tid & 31, i64 = l < 16 ? ((tid >> 5) & 3) * 16 + l : -1;  // M = 64 row
    const ChunkInfo ci = chunk_at(p, c);
    using S_ = GradSmem;
    uint8_t *QK = sm + S_::kQK, *DO = sm + S_::kDO, *VT = sm + S_::kV, *SC = sm + S_::kSC,
            *DSN = sm + S_::kDSN, *UT = sm + S_::kUT, *DUT = sm + S_::kDUT, *AB = sm + S_::kAB,
            *X3 = sm + S_::kX3, *DA = sm + S_::kDA, *T1 = sm + S_::kT1, *DPG = sm + S_::kDPG,
            *DLG = sm + S_::kDLG;
    float *vec = reinterpret_cast<float *>(sm + S_::kVec);
    float *G = vec, *bta = vec + 64, *gam = vec + 128, *e = vec + 192, *dB = vec + 256,
          *qx = vec + 320, *kx = vec + 384, *kz = vec + 448, *dG = vec + 512, *tmp = vec + 576,
          *dbl2 = vec + 640, *qinv = vec + 896, *kinv = vec + 960, *qdot = vec + 1024,
          *kdot = vec + 1088;
    float *wsum = reinterpret_cast<float *>(sm + S_::kRed);  // [3][4 warps][64 columns]
    const int w4 = (tid >> 5) & 3;
    float *PE = reinterpret_cast<float *>(sm + S_::kPE);
    float *KKG = reinterpret_cast<float *>(sm + S_::kKKG);
    float *Gam = reinterpret_cast<float *>(sm + S_::kGam);

    __shared__ uint64_t lbar;
    constexpr uint32_t kImgA = C * C * 2;
    if (tid == 0) {  // the tile images and A by bulk copies (one instruction each)
        mbar_init(&lbar, 1);
        fence_mbar_init();
        mbar_arrive_expect_tx(&lbar, 2 * kImg128 + 2 * kImgUT + kImgA + 2 * row_tile_bytes(p.K) +
                                         2 * row_tile_bytes(p.V));
        bulk_load(smem_u32(SC), static_cast<const uint8_t *>(p.tS) + (size_t)ch * kImg128,
                  kImg128, &lbar);
        bulk_load(smem_u32(DSN), static_cast<const uint8_t *>(p.tdSn) + (size_t)ch * kImg128,
                  kImg128, &lbar);
        bulk_load(smem_u32(UT), static_cast<const uint8_t *>(p.tUT) + (size_t)ch * kImgUT, kImgUT,
                  &lbar);
        bulk_load(smem_u32(DUT), static_cast<const uint8_t *>(p.tdUT) + (size_t)ch * kImgUT,
                  kImgUT, &lbar);
        bulk_load(smem_u32(AB), static_cast<const uint8_t *>(p.tA) + (size_t)ch * kImgA, kImgA,
                  &lbar);
        // q, k, dO, v rows by the tensor engine
        load_rows_tma(QK, D, 0, &p.tm_q, ci.tok0, h, p.K, &lbar);
        load_rows_tma(QK, D, C, &p.tm_k, ci.tok0, h, p.K, &lbar);
        load_rows_tma(DO, C, 0, &p.tm_do, ci.tok0, h, p.V, &lbar);
        load_rows_tma(VT, C, 0, &p.tm_v, ci.tok0, h, p.V, &lbar);
    }
    if (tid < C) {
        const int64_t idx = (int64_t)(ci.tok0 + tid) * H + h;
        G[tid] = p.tG[(size_t)ch * C + tid];
        bta[tid] = tid < ci.len ? p.beta[idx] : 0.f;
    }
    if (tid == 0) {
        mbar_init(&mbar, 1);
        fence_mbar_init();
    }
    if (tid < 32) {
        tmem_alloc(&tslot, 512);
        tmem_relinquish();
    }
    __syncthreads();
    if (tid < C) {
        gam[tid] = expf(G[tid]);
        e[tid] = expf(G[C - 1] - G[tid]);
    }
    if (!copies_arrived(&lbar, p, 20)) {  // (the barrier above published the inits)
        tc_fence_before();
        __syncthreads();
        if (tid < 32) tmem_dealloc(tslot, 512);
        return;
    }
    fix_rows(QK, D, 0, ci.len, p.K, NG);
    fix_rows(QK, D, C, ci.len, p.K, NG);
    fix_rows(DO, C, 0, ci.len, p.V, NG);
    fix_rows(VT, C, 0, ci.len, p.V, NG);
    operands_ready();
    if (p.l2norm) {  // q rows (threads 0-127) and k rows (128-255) divided by their norms
        l2norm_tile_rows(QK, D, 0, qinv, 0);
        l2norm_tile_rows(QK, D, C, kinv, 2 * C);
        operands_ready();
    }
    const uint32_t tmem = tslot;
    const uint32_t qkb = smem_u32(QK), kb = qkb + C * 128, dob = smem_u32(DO), vb = smem_u32(VT),
                   scb = smem_u32(SC), dsb = smem_u32(DSN), utb = smem_u32(UT),
                   dub = smem_u32(DUT), ab = smem_u32(AB), x3b = smem_u32(X3), dab = smem_u32(DA),
                   t1b = smem_u32(T1), dpb = smem_u32(DPG), dlb = smem_u32(DLG);
    // TMEM columns
    // (Y2 takes X3's columns once X3 is read, T1 then Y2's; dL takes Q K^T's once P is formed)
    constexpr int cQK = 0, cX1 = 64, cX2 = 128, cX3 = 192, cDP = 256, cAU = 320, cY1 = 384,
                  cY2 = 192, cZ = 448, cT1 = 192, cDL = 0, cDQ = 256, cDK = 320, cDKA = 384;
    uint32_t phase = 0;
    bool ok;
    float d[CW];
    if (tid == 0) {
        const uint32_t i128 = idesc_bf16(128, 64, 0, 0), i128mk = idesc_bf16(128, 64, 1, 0),
                       i128mm = idesc_bf16(128, 64, 1, 1), i128km = idesc_bf16(128, 64, 0, 1),
                       i64km = idesc_bf16(64, 64, 0, 1), i64mk = idesc_bf16(64, 64, 1, 0);
#pragma unroll
        for (int s = 0; s < 8; ++s)  // [Q;K] K^T: lanes 0-63 Q K^T, lanes 64-127 K K^T
            mma_bf16(tmem + cQK, desc_kmajor(qkb, D, s), desc_kmajor(kb, D, s), i128, s > 0);
#pragma unroll
        for (int s = 0; s < 8; ++s)  // X1^T = S^T dO^T  (over v)
            mma_bf16(tmem + cX1, desc_mnmajor(scb, D, s), desc_kmajor(dob, C, s), i128mk, s > 0);
#pragma unroll
        for (int s = 0; s < 8; ++s)  // X2^T = dSn^T U^T
            mma_bf16(tmem + cX2, desc_mnmajor(dsb, D, s), desc_mnmajor(utb, D, s), i128mm, s > 0);
#pragma unroll
        for (int s = 0; s < 8; ++s)  // X3^T = S^T dU^T
            mma_bf16(tmem + cX3, desc_mnmajor(scb, D, s), desc_mnmajor(dub, D, s), i128mm, s > 0);
#pragma unroll
        for (int s = 0; s < 8; ++s)  // dP = dO U^T (M = 64)
            mma_bf16(tmem + cDP, desc_kmajor(dob, C, s), desc_mnmajor(utb, D, s), i64km, s > 0);
#pragma unroll
        for (int s = 0; s < 4; ++s)  // (A^T dU)^T = dU^T A
            mma_bf16(tmem + cAU, desc_kmajor(dub, D, s), desc_mnmajor(ab, C, s), i128km, s > 0);
#pragma unroll
        for (int s = 0; s < 8; ++s)  // Y1 = dU V^T (M = 64)
            mma_bf16(tmem + cY1, desc_mnmajor(dub, D, s), desc_kmajor(vb, C, s), i64mk, s > 0);
        mma_commit(&mbar);
    }
    {  // <S, dSn> (elementwise over identically laid out images) while the products run
        float s = 0.f;
        for (int t = tid; t < D * D / 8; t += NG) {
            float a[8], b[8];
            unpack8(*reinterpret_cast<const uint4 *>(SC + t * 16), a);
            unpack8(*reinterpret_cast<const uint4 *>(DSN + t * 16), b);
#pragma unroll
            for (int q = 0; q < 8; ++q) s = fmaf(a[q], b[q], s);
        }
        for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        if (l == 0) tmp[tid >> 5] = s;
        __syncthreads();
        if (tid == 0) {
            float a = 0.f;
            for (int w = 0; w < NG / 32; ++w) a += tmp[w];
            s_hd = a;  // read after the barrier of the wait below
        }
    }
    ok = cta_wait(&mbar, phase, p, 21);
    phase ^= 1;
    if (!ok) goto done;
    // the decay matrix, once (the dU^T image there is consumed)
    for (int t = tid; t < C * C; t += NG) {
        const int i = t >> 6, j = t & 63;
        Gam[gidx(i, j)] = j <= i ? expf(G[i] - G[j]) : 0.f;
    }
    __syncthreads();
    ldcw(tmem, cX3 + cb, d);  // X3^T as an operand tile (row kk)
#pragma unroll
    for (int q = 0; q < CW / 8; ++q)
        *reinterpret_cast<uint4 *>(X3 + sw128_chunk(D, r, cb / 8 + q)) = pack8(d + 8 * q);
    operands_ready();
    if (tid == 0) {  // issued now; the SIMT work below runs while they execute
        const uint32_t i64mk = idesc_bf16(64, 64, 1, 0), i128km = idesc_bf16(128, 64, 0, 1);
#pragma unroll
        for (int s = 0; s < 8; ++s)  // Y2 = X3 K^T (M = 64)
            mma_bf16(tmem + cY2, desc_mnmajor(x3b, D, s), desc_kmajor(kb, D, s), i64mk, s > 0);
#pragma unroll
        for (int s = 0; s < 4; ++s)  // Zp^T = X3^T A   (Z = -Zp)
            mma_bf16(tmem + cZ, desc_kmajor(x3b, D, s), desc_mnmajor(ab, C, s), i128km, s > 0);
        mma_commit(&mbar);
    }
    // meanwhile: P, Gam . K K^T, dv and the column sums, dP
    // P (scaled, lower incl. diagonal) and Gam . K K^T (strictly lower), fp32
    ldcw(tmem, cQK + cb, d);
    if (r < 64) {
#pragma unroll
        for (int q = 0; q < CW; ++q) {
            const int j = cb + q;
            PE[r * LP + j] = j <= r ? p.scale * Gam[gidx(r, j)] * d[q] : 0.f;
        }
    } else {
        const int i = r - 64;
#pragma unroll
        for (int q = 0; q < CW; ++q) {
            const int j = cb + q;
            KKG[i * LP + j] = j < i ? Gam[gidx(i, j)] * d[q] : 0.f;
        }
    }
    {  // dv = diag(b) A^T dU (staged as rows in the consumed dO tile); partial v . (A^T dU)
        bf16 *stage = reinterpret_cast<bf16 *>(DO);
        const ColSw vcol(VT, C, r);
        ldcw(tmem, cAU + cb, d);
#pragma unroll
        for (int q = 0; q < CW; ++q) {
            const int i = cb + q;
            stage[i * D + r] = __float2bfloat16_rn(bta[i] * d[q]);
            d[q] *= vcol.at(cb, q);
        }
        warp_colsum(d, wsum, w4, cb, l);
    }
    {  // column readers of q and k are built where used (they cost 8 registers each)
        const ColSw qcol(QK, D, r), kcol(QK + C * 128, D, r);
        ldcw(tmem, cX1 + cb, d);  // partial q' . X1 (thread kk)
#pragma unroll
        for (int q = 0; q < CW; ++q) d[q] *= p.scale * qcol.at(cb, q);
        warp_colsum(d, wsum + 256, w4, cb, l);
        ldcw(tmem, cX2 + cb, d);  // partial k . X2
#pragma unroll
        for (int q = 0; q < CW; ++q) d[q] *= kcol.at(cb, q);
        warp_colsum(d, wsum + 512, w4, cb, l);
    }
    __syncthreads();
    if (tid < 3 * C) {
        const int k = tid >> 6, i = tid & 63;
        const float *w = wsum + k * 256 + i;
        (k == 0 ? dB : k == 1 ? qx : kx)[i] = (w[0] + w[64]) + (w[128] + w[192]);
    }
    __syncthreads();
    store_rows(static_cast<bf16 *>(p.dv), DO, ci.tok0, ci.len, h, H, p.V);
    ldcw(tmem, cDP + cb, d);  // dP: dPG = dP . Gam as an operand tile; PE <- dP . P
    if (i64 >= 0) {
#pragma unroll
        for (int q = 0; q < CW; ++q) {
            const int j = cb + q;
            const float dp = j <= i64 ? d[q] : 0.f;
            PE[i64 * LP + j] *= dp;
            d[q] = dp * Gam[gidx(i64, j)];
        }
#pragma unroll
        for (int q = 0; q < CW / 8; ++q)
            *reinterpret_cast<uint4 *>(DPG + sw128_chunk(C, i64, cb / 8 + q)) = pack8(d + 8 * q);
    }
    ok = cta_wait(&mbar, phase, p, 22);
    phase ^= 1;
    if (!ok) goto done;
    {  // dA = (dU V^T) diag(b) - (X3 K^T) diag(b gam)
        float y2[CW];
        tmem_ld16(tmq(tmem, cY1 + cb), d);
        tmem_ld16(tmq(tmem, cY2 + cb), y2);
        tmem_ld_wait();
        if (i64 >= 0) {
#pragma unroll
            for (int q = 0; q < CW; ++q) {
                const int m = cb + q;
                d[q] = bta[m] * d[q] - bta[m] * gam[m] * y2[q];
            }
#pragma unroll
            for (int q = 0; q < CW / 8; ++q)
                *reinterpret_cast<uint4 *>(DA + sw128_chunk(C, i64, cb / 8 + q)) = pack8(d + 8 * q);
        }
    }
    operands_ready();
    if (tid == 0) {  // T1 = A^T dA (M = 64)
        const uint32_t id = idesc_bf16(64, 64, 1, 1);
#pragma unroll
        for (int s = 0; s < 4; ++s)
            mma_bf16(tmem + cT1, desc_mnmajor(ab, C, s), desc_mnmajor(dab, C, s), id, s > 0);
        mma_commit(&mbar);
    }
    // meanwhile: k . Z
    {
        const ColSw kcol(QK + C * 128, D, r);
        ldcw(tmem, cZ + cb, d);  // partial k . Z = -k . Zp
#pragma unroll
        for (int q = 0; q < CW; ++q) d[q] *= -kcol.at(cb, q);
        warp_colsum(d, wsum, w4, cb, l);
    }
    __syncthreads();
    if (tid < C) kz[tid] = (wsum[tid] + wsum[64 + tid]) + (wsum[128 + tid] + wsum[192 + tid]);
    ok = cta_wait(&mbar, phase, p, 23);
    phase ^= 1;
    if (!ok) goto done;
    ldcw(tmem, cT1 + cb, d);
    if (i64 >= 0) {
#pragma unroll
        for (int q = 0; q < CW / 8; ++q)
            *reinterpret_cast<uint4 *>(T1 + sw128_chunk(C, i64, cb / 8 + q)) = pack8(d + 8 * q);
    }
    operands_ready();
    if (tid == 0) {  // T1 A^T = -dL (M = 64)
        const uint32_t id = idesc_bf16(64, 64, 0, 0);
#pragma unroll
        for (int s = 0; s < 4; ++s)
            mma_bf16(tmem + cDL, desc_kmajor(t1b, C, s), desc_kmajor(ab, C, s), id, s > 0);
        mma_commit(&mbar);
    }
    ok = cta_wait(&mbar, phase, p, 24);
    phase ^= 1;
    if (!ok) goto done;
    ldcw(tmem, cDL + cb, d);  // dL (strictly lower); diag(b) dL . Gam tile; PE += dL . L
    if (i64 >= 0) {
        float dbl = 0.f;
        const float bi = bta[i64];
#pragma unroll
        for (int q = 0; q < CW; ++q) {
            const int j = cb + q;
            const float dl = j < i64 ? -d[q] : 0.f;
            const float kkg = KKG[i64 * LP + j];
            PE[i64 * LP + j] += dl * bi * kkg;
            dbl = fmaf(dl, kkg, dbl);
            d[q] = bi * dl * Gam[gidx(i64, j)];
        }
#pragma unroll
        for (int q = 0; q < CW / 8; ++q)
            *reinterpret_cast<uint4 *>(DLG + sw128_chunk(C, i64, cb / 8 + q)) = pack8(d + 8 * q);
        dbl2[wg * 64 + i64] = dbl;
    }
    operands_ready();
    if (tid == 0) {
        const uint32_t imk = idesc_bf16(128, 64, 1, 0), imm = idesc_bf16(128, 64, 1, 1);
#pragma unroll
        for (int s = 0; s < 4; ++s)  // (dPG K)^T = K^T dPG^T
            mma_bf16(tmem + cDQ, desc_mnmajor(kb, D, s), desc_kmajor(dpb, C, s), imk, s > 0);
#pragma unroll
        for (int s = 0; s < 4; ++s)  // (dPG^T Q)^T = Q^T dPG
            mma_bf16(tmem + cDKA, desc_mnmajor(qkb, D, s), desc_mnmajor(dpb, C, s), imm, s > 0);
#pragma unroll
        for (int s = 0; s < 4; ++s)  // (diag(b) dLG K)^T
            mma_bf16(tmem + cDK, desc_mnmajor(kb, D, s), desc_kmajor(dlb, C, s), imk, s > 0);
#pragma unroll
        for (int s = 0; s < 4; ++s)  // ((diag(b) dLG)^T K)^T
            mma_bf16(tmem + cDK, desc_mnmajor(kb, D, s), desc_mnmajor(dlb, C, s), imm, 1);
        mma_commit(&mbar);
    }
    // meanwhile: dbeta and dG (rows), then dg = reverse cumulative sum of dG
    {  // row and column sums of PE: eight threads per token, eight entries each
        const int i = tid >> 3, part = tid & 7;
        float rs = 0.f, cs = 0.f;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            rs += PE[i * LP + part * 8 + t];
            cs += PE[(part * 8 + t) * LP + i];
        }
        float x = rs - cs;
#pragma unroll
        for (int off = 1; off < 8; off <<= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
        if (part == 0) {
            dG[i] = -e[i] * kx[i] + gam[i] * qx[i] + x + bta[i] * gam[i] * kz[i];
            dB[i] += (dbl2[i] + dbl2[64 + i]) + (dbl2[128 + i] + dbl2[192 + i]) + gam[i] * kz[i];
        }
    }
    __syncthreads();
    if (tid < 32) {  // dg = reverse cumulative sum of dG (+ the terms of the last token)
        const float a = dG[2 * l], b = dG[2 * l + 1];
        float s = e[2 * l] * kx[2 * l] + e[2 * l + 1] * kx[2 * l + 1];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        const float extra = gam[C - 1] * s_hd + s;
        float x = a + b;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float t = __shfl_down_sync(0xffffffffu, x, off);
            if (l + off < 32) x += t;
        }
        const int i0 = 2 * l;
        if (i0 < ci.len) {
            const int64_t o = (int64_t)(ci.tok0 + i0) * H + h;
            p.dg[o] = x + extra;
            p.dbeta[o] = dB[i0];
        }
        if (i0 + 1 < ci.len) {
            const int64_t o = (int64_t)(ci.tok0 + i0 + 1) * H + h;
            p.dg[o] = (x - a) + extra;
            p.dbeta[o] = dB[i0 + 1];
        }
    }
    ok = cta_wait(&mbar, phase, p, 25);
    phase ^= 1;
    if (!ok) goto done;
    {  // dq = scale (diag(gam) X1 + dPG K) ; dk = diag(e) X2 + diag(b gam) Z + dPG^T Q' + dL terms
        // staged as rows in the consumed dO and V tiles, then 16-byte stores
        bf16 *sq = reinterpret_cast<bf16 *>(DO), *sk = reinterpret_cast<bf16 *>(VT);
        const ColSw qcol(QK, D, r), kcol(QK + C * 128, D, r);
        float a[CW];
        tmem_ld16(tmq(tmem, cX1 + cb), d);
        tmem_ld16(tmq(tmem, cDQ + cb), a);
        tmem_ld_wait();
#pragma unroll
        for (int q = 0; q < CW; ++q) d[q] = p.scale * (gam[cb + q] * d[q] + a[q]);
        if (p.l2norm) project_rows(d, qcol, qinv, qdot, wsum, w4, cb, l);
#pragma unroll
        for (int q = 0; q < CW; ++q) sq[(cb + q) * D + r] = __float2bfloat16_rn(d[q]);
        tmem_ld16(tmq(tmem, cX2 + cb), d);
        tmem_ld16(tmq(tmem, cZ + cb), a);
        tmem_ld_wait();
#pragma unroll
        for (int q = 0; q < CW; ++q) d[q] = e[cb + q] * d[q] - bta[cb + q] * gam[cb + q] * a[q];
        ldcw(tmem, cDKA + cb, a);
#pragma unroll
        for (int q = 0; q < CW; ++q) d[q] += p.scale * a[q];
        ldcw(tmem, cDK + cb, a);
#pragma unroll
        for (int q = 0; q < CW; ++q) d[q] += a[q];
        if (p.l2norm) project_rows(d, kcol, kinv, kdot, wsum + 256, w4, cb, l);
#pragma unroll
        for (int q = 0; q < CW; ++q) sk[(cb + q) * D + r] = __float2bfloat16_rn(d[q]);
        __syncthreads();
        store_rows(static_cast<bf16 *>(p.dq), DO, ci.tok0, ci.len, h, H, p.K);
        store_rows(static_cast<bf16 *>(p.dk), VT, ci.tok0, ci.len, h, H, p.K);
    }
done:
    tc_fence_before();
    __syncthreads();
    if (tid < 32) tmem_dealloc(tmem, 512);
}

}  // namespace

cudaError_t launch_tc_bwd(const Params &p, const Problem &, cudaStream_t stream) {
    cudaError_t e;
    const int nch = p.NC * p.H, nseq = p.N * p.H;
    Params pf = p;
    pf.hT = nullptr;
    if (nch > 0) {
        const int sm = kLocalSmem > kPrepSmemRequest ? kLocalSmem : kPrepSmemRequest;
        if ((e = set_smem(tc_prep_local_kernel, sm))) return e;
        GDN_LAUNCH(kKTcLocal, stream,
                   tc_prep_local_kernel<<<2 * nch, NT, sm, stream>>>(p));
    }
    if (nseq > 0) {
        const int sm = kSbwdSmem > kStateSmem ? kSbwdSmem : kStateSmem;
        if ((e = set_smem(tc_chains_kernel, sm))) return e;
        GDN_LAUNCH(kKTcStateBwd, stream, tc_chains_kernel<<<2 * nseq, NT, sm, stream>>>(pf, p));
    }
    if (nch > 0) {
        if ((e = set_smem(tc_grads_kernel, kGradSmem))) return e;
        GDN_LAUNCH(kKTcGrads, stream, tc_grads_kernel<<<nch, NG, kGradSmem, stream>>>(p));
    }
    return cudaSuccess;
}

static_assert(kGradSmem <= 227 * 1024, "grads shared memory");
static_assert(kSbwdSmem <= 227 * 1024, "reverse state shared memory");

}  // namespace gdn
