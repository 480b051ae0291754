// Tensor-core (tcgen05) backward of the bf16 layer, d_k = d_v = 128.
//
// Reverse-mode of the chunkwise forward (see tc.cu).  After the forward
// pieces are recomputed (tc_prep keeps A in fp32; tc_state_fwd rewrites the
// state entering every chunk and U^T), three kernels run:
//
//   tc_prep_local chunk-parallel: the preparation step (tc_prep.cuh) with A
//                 written too, and the tile images P = scale lower(Q K^T . Gam)
//                 and Qg = scale diag(gam) Q
//   tc_state_bwd  serial over the chunks of a sequence, in reverse; thread v
//                 owns row v of dS = dH^T (fp32 registers); per chunk
//                   dU^T = dO^T P + dS Kd^T
//                   dS  <- gam_n dS + dO^T Qg - dU^T W
//                 and writes dS (the gradient of the state leaving the chunk)
//                 and dU^T as tile images
//   tc_grads      chunk-parallel: every chunk-local gradient (dq, dk, dv, dg,
//                 dbeta) from the recomputed and propagated pieces; one
//                 persistent CTA per SM walks its (chunk, head) units and
//                 fetches each input group of the next unit into the buffers
//                 the current one has finished with, so the copies run under
//                 the compute; dq and dk leave by tensor-map stores, dv by
//                 stores of every thread.
//
// The gradient of L takes two dependent products, not four: with
// M = diag(b) V - diag(b gam) K H, U = A M, and dA = dU M^T, so
// dL = -A^T dA A^T = -A^T dU (A M)^T = -A^T (dU U^T); and the gradient of W's
// K factor, A^T dW = -A^T dU H^T, is formed as (H (dU^T A))^T from the
// product dU^T A that dv needs anyway.
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

// ============================================================ tc_prep_local
// The preparation step with A also written (the backward's gradient kernel reads
// it); the same step writes the P and Qg images the reverse chain reads.
__global__ void __launch_bounds__(NT, 4) tc_prep_local_kernel(const __grid_constant__ Params p) {
    prep_body(p, blockIdx.x, 1);
}

// ============================================================ tc_state_bwd
struct SbwdSmem {
    // two dS images (the next chunk's is written while the current one may still be
    // read), dU^T, then per prefetch buffer: Kd image, W image, Qg image, dO tile,
    // P tile; the buffers' gate rows last
    static constexpr int kdS0 = 0, kdU = kdS0 + 2 * 32768, kBuf = kdU + 16384;
    static constexpr int kKd = 0, kW = 16384, kQg = 32768, kDO = 49152, kP = 65536,
                         kBufBytes = 73728;
    static constexpr int kGr = kBuf + 2 * kBufBytes, kEnd = kGr + 2 * 256;
};
constexpr int kSbwdSmem = SbwdSmem::kEnd + 1024;

// Chunk ch's Kd, W, Qg and P images and gate row by bulk copies,
// its dO rows by the tensor engine (thread 0, all completing on `bar`).
__device__ __forceinline__ void sbwd_prefetch(uint8_t *sm, int buf, size_t ch,
                                              const ChunkInfo &ci, int h, const Params &p,
                                              uint64_t *bar) {
    uint8_t *b = sm + SbwdSmem::kBuf + buf * SbwdSmem::kBufBytes;
    if (threadIdx.x == 0) {
        mbar_arrive_expect_tx(bar, 3u * (uint32_t)kImg64 + (uint32_t)(C * C * 2) + C * 4u +
                                       row_tile_bytes(p.V));
        bulk_load(smem_u32(b + SbwdSmem::kKd), static_cast<const uint8_t *>(p.tKd) + ch * kImg64,
                  kImg64, bar);
        bulk_load(smem_u32(b + SbwdSmem::kW), static_cast<const uint8_t *>(p.tW) + ch * kImg64,
                  kImg64, bar);
        bulk_load(smem_u32(b + SbwdSmem::kQg), static_cast<const uint8_t *>(p.tQg) + ch * kImg64,
                  kImg64, bar);
        bulk_load(smem_u32(b + SbwdSmem::kP),
                  static_cast<const uint8_t *>(p.tP) + ch * (size_t)(C * C * 2), C * C * 2, bar);
        bulk_load(smem_u32(sm + SbwdSmem::kGr + buf * 256), p.tG + ch * C, C * 4, bar);
        load_rows_tma(b + SbwdSmem::kDO, C, 0, &p.tm_do, ci.tok0, h, p.V, bar);
    }
}

// One run of the reverse chain over chunks [c0, c1) of one head, last chunk first.
struct ChainBwd {
    int n, h, c0, c1;    // sequence n (its first chunk gives the chunks' positions), range
    const float *init;   // dS leaving chunk c1 - 1 (fp32), or nullptr for zero
    int init_user;       // init is a caller's [K][V] block (else an internal [128][128] one)
    int init_identity;   // start from dS = I (the transition run of the piece scan)
    int zero_local;      // drop the dO terms (the transition run)
    int snapshots;       // write dS leaving every chunk and dU^T (tile images)
    float *final_out;    // dS entering chunk c0 (fp32), or nullptr
    int out_user;        // final_out is a caller's [K][V] block (else [128][128])
    int where;           // tag recorded if a bounded wait gives up
};

// The reverse chain: thread v owns row v of dS = dH^T (fp32 registers), the
// gradient of the state leaving the current chunk; per chunk
//   dU^T = dO^T P + dS Kd^T ;  dS <- gam_n dS + dO^T Qg - dU^T W.
__device__ __forceinline__ void chain_bwd(const Params &p, const ChainBwd &a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = align1k(smem_raw);
    __shared__ uint64_t mbar, lbar[2];
    __shared__ uint32_t tslot;
    if (p.hdr->status) return;
    const int H = p.H, n = a.n, h = a.h, v = threadIdx.x;
    const int sq0 = seq_first_at(p, n);  // the sequence's first chunk (chunk positions)
    float S[D];  // dS row v (gradient of the state leaving the current chunk)
    if (a.init) {  // [K][V] or [128][128] blocks; rows and columns past them are zero
        const int ik = a.init_user ? p.K : D, iv = a.init_user ? p.V : D;
#pragma unroll
        for (int kk = 0; kk < D; ++kk) S[kk] = (kk < ik && v < iv) ? a.init[kk * iv + v] : 0.f;
    } else {
#pragma unroll
        for (int kk = 0; kk < D; ++kk) S[kk] = (a.init_identity && kk == v) ? 1.f : 0.f;
    }
    if (v == 0) {
        mbar_init(&mbar, 1);
        mbar_init(&lbar[0], 1);
        mbar_init(&lbar[1], 1);
        fence_mbar_init();
    }
    if (v < 32) {
        tmem_alloc(&tslot, 512);
        tmem_relinquish();
    }
    if (a.snapshots) state_image(sm + SbwdSmem::kdS0, S, v);  // dS leaving the last chunk
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tslot;
    // TMEM columns: 0-63 dU^T, 64-191 the dS update, 256-319 the dS image and 320-351
    // the dU^T image (bf16 pairs: the A operands of the products that read them; the
    // shared-memory images are kept for the snapshots only)
    constexpr uint32_t cSI = 256, cUI = 320;
    tmem_store_bf16<64>(tm(tmem, cSI), S);
    tmem_st_wait();
    const int c0 = a.c0, c1 = a.c1;
    const bool local = !a.zero_local;
    uint32_t phase = 0;
    // per buffer b (bit b): bulk copies in flight, and the parity of their next completion
    uint32_t pend = 0, lpar = 0;
    if (c0 < c1) {
        sbwd_prefetch(sm, 0, (size_t)(c1 - 1) * H + h, chunk_in_seq(p, n, sq0, c1 - 1), h, p,
                      &lbar[0]);
        pend = 1;
    }
    uint8_t *dUs = sm + SbwdSmem::kdU;
    const uint32_t id1 = idesc_bf16(128, 64, 0, 0), idx = idesc_bf16(128, 128, 1, 1),
                   idy = idesc_bf16(128, 128, 0, 1), idp = idesc_bf16(128, 64, 1, 1);
    for (int c = c1 - 1; c >= c0; --c) {
        const int buf = (c1 - 1 - c) & 1;
        const size_t ch = (size_t)c * H + h;
        if (c - 1 >= c0) {
            sbwd_prefetch(sm, buf ^ 1, ch - H, chunk_in_seq(p, n, sq0, c - 1), h, p,
                          &lbar[buf ^ 1]);
            pend |= 2u >> buf;
        }
        const bool lok = mbar_wait(&lbar[buf], (lpar >> buf) & 1u, p.wait_limit);
        uint8_t *b = sm + SbwdSmem::kBuf + buf * SbwdSmem::kBufBytes;
        // the dS image this chunk reads (written by the previous chunk's update), and the
        // one this chunk's update writes
        uint8_t *dSs = sm + SbwdSmem::kdS0 + buf * 32768, *dSn = sm + SbwdSmem::kdS0 + (buf ^ 1) * 32768;
        const uint32_t sb = smem_u32(dSs), kb = smem_u32(b + SbwdSmem::kKd),
                       qb = smem_u32(b + SbwdSmem::kQg), ob = smem_u32(b + SbwdSmem::kDO),
                       pb = smem_u32(b + SbwdSmem::kP);
        // dO^T P (the local dU^T; M = 128 (v), N = 64, K = 64 tokens) and dO^T Qg (M = 128,
        // N = 128 keys, K = 64) do not depend on dS: on a full chunk (whose dO rows need no
        // clearing) thread 0 issues them as soon as its copies landed
        const int len = chunk_in_seq(p, n, sq0, c).len;
        const bool early = local && len == C && p.V == D;
        auto issue_local = [&]() {
#pragma unroll
            for (int s = 0; s < C / 16; ++s)
                mma_bf16(tmem, desc_mnmajor(ob, C, s), desc_mnmajor(pb, C, s), idp, s > 0);
#pragma unroll
            for (int s = 0; s < C / 16; ++s)
                mma_bf16(tmem + 64, desc_mnmajor(ob, C, s), desc_mnmajor(qb, C, s), idx, s > 0);
        };
        if (v == 0 && lok && early) issue_local();
        if (lok && local && !early) fix_rows(b + SbwdSmem::kDO, C, 0, len, p.V);
        fence_async_smem();
        tc_fence_before();
        const bool all = __syncthreads_and(lok);
        tc_fence_after();
        if (!all) {
            if (v == 0) record_timeout(p, a.where);
            break;
        }
        pend &= ~(1u << buf);
        lpar ^= 1u << buf;
        const float gC =
            expf(reinterpret_cast<const float *>(sm + SbwdSmem::kGr + buf * 256)[C - 1]);
        if (v == 0) {
            if (local && !early) issue_local();
            // + dS Kd^T: M = 128 (v), N = 64 tokens, K = 128 keys
#pragma unroll
            for (int s = 0; s < D / 16; ++s)
                mma_bf16_ta(tmem, tmem + cSI + 8 * s, desc_kmajor(kb, C, s), id1, local || s > 0);
            mma_commit(&mbar);
        }
        if (v == 0 && a.snapshots) {
            bulk_store(static_cast<uint8_t *>(p.tdSn) + ch * kImg128, sb, (uint32_t)kImg128);
            bulk_commit();
            // the previous chunk's stores (dU^T, and the dS image this chunk's update
            // rewrites) have read their sources
            bulk_wait_read_n<1>();
        }
        if (!cta_wait(&mbar, phase, p, a.where + 1)) break;
        phase ^= 1;
#pragma unroll
        for (int c32 = 0; c32 < C; c32 += 32) {  // dU^T: the next operand, and an image for tc_grads
            float d[32];
            tmem_ld16(tm(tmem, c32), d);
            tmem_ld16(tm(tmem, c32 + 16), d + 16);
            tmem_ld_wait();
            tmem_store_bf16<16>(tm(tmem, cUI + c32 / 2), d);
            if (a.snapshots) {
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    *reinterpret_cast<uint4 *>(dUs + sw128_chunk(D, v, c32 / 8 + q)) =
                        pack8(d + 8 * q);
            }
        }
        tmem_st_wait();
        operands_ready();
        if (v == 0) {  // + dU^T (-W): M = 128 (v), N = 128 keys, K = 64 tokens (W image negated)
            const uint32_t wb = smem_u32(b + SbwdSmem::kW);
#pragma unroll
            for (int s = 0; s < C / 16; ++s)
                mma_bf16_ta(tmem + 64, tmem + cUI + 8 * s, desc_mnmajor(wb, C, s), idy,
                            local || s > 0);
            mma_commit(&mbar);
        }
        if (v == 0 && a.snapshots) {
            bulk_store(static_cast<uint8_t *>(p.tdUT) + ch * kImgUT, smem_u32(dUs), (uint32_t)kImgUT);
            bulk_commit();
        }
        if (!cta_wait(&mbar, phase, p, a.where + 2)) break;
        phase ^= 1;
#pragma unroll
        for (int c32 = 0; c32 < D; c32 += 32) {
            float d[32];
            tmem_ld16(tm(tmem, 64 + c32), d);
            tmem_ld16(tm(tmem, 64 + c32 + 16), d + 16);
            tmem_ld_wait();
#pragma unroll
            for (int q = 0; q < 32; ++q) S[c32 + q] = fmaf(gC, S[c32 + q], d[q]);
            tmem_store_bf16<16>(tm(tmem, cSI + c32 / 2), S + c32);  // the next chunk's dS image
            if (a.snapshots) {
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    *reinterpret_cast<uint4 *>(dSn + sw128_chunk(D, v, c32 / 8 + q)) =
                        pack8(S + c32 + 8 * q);
            }
        }
        tmem_st_wait();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }
    if (v == 0) {  // copies still in flight after an early exit
        for (int q = 0; q < 2; ++q)
            if ((pend >> q) & 1u) mbar_wait(&lbar[q], (lpar >> q) & 1u, kWaitLimit);
        if (a.snapshots) bulk_wait_all();
    }
    if (a.final_out) {
        const int ok = a.out_user ? p.K : D, ov = a.out_user ? p.V : D;
        if (v < ov) {
#pragma unroll
            for (int kk = 0; kk < D; ++kk)
                if (kk < ok) a.final_out[kk * ov + v] = S[kk];
        }
    }
    tc_fence_before();
    __syncthreads();
    if (v < 32) tmem_dealloc(tmem, 512);
}

// Body of the reverse state pass for CTA `blk` (sequence blk / H, head blk % H):
// the whole sequence from dhT, writing the per-chunk snapshots and dh0.
__device__ __forceinline__ void state_bwd_body(const Params &p, int blk) {
    const int H = p.H, n = blk / H, h = blk % H;
    ChainBwd a;
    a.n = n;
    a.h = h;
    a.c0 = seq_first_at(p, n);
    a.c1 = seq_first_at(p, n + 1);
    a.init = p.dhT ? p.dhT + ((size_t)n * H + h) * p.K * p.V : nullptr;
    a.init_user = 1;
    a.init_identity = 0;
    a.zero_local = 0;
    a.snapshots = 1;
    a.final_out = p.dh0 ? p.dh0 + ((size_t)n * H + h) * p.K * p.V : nullptr;
    a.out_user = 1;
    a.where = 45;
    chain_bwd(p, a);
}

// ============================================================ piece scan (long rows)
// The backward's piece scan: the forward chain's roles of the forward piece scan
// (piece_a_fwd_role, piece_c_fwd_role, with snapshots for the gradient kernel
// and no final state), and the mirrored roles of the reverse chain, whose chunk
// map is affine in dS as well:
//   dS_prev = dS (gam_n I - Kd^T W) + dO^T (Qg - P W).
// Phase A: the last piece runs from dhT with snapshots (its result enters piece
// P - 2); every middle piece runs once from zero (-> its offset, tBr) and once
// from dS = I without its dO terms (-> its transition, tTr).
__device__ __forceinline__ void piece_a_bwd_role(const Params &p, int unit, int r) {
    const int n = unit / p.H, h = unit % p.H;
    const size_t u = (size_t)unit * p.P, DD = (size_t)D * D;
    ChainBwd a;
    a.n = n;
    a.h = h;
    a.where = 60;
    a.init_user = 1;  // dhT (the last piece); the middle pieces start from zero or the identity
    a.out_user = 0;   // tdHin, tBr, tTr are internal [128][128] blocks
    int piece;
    if (r == 0) {
        piece = p.P - 1;
        a.init = p.dhT ? p.dhT + (size_t)unit * DD : nullptr;
        a.init_identity = 0;
        a.zero_local = 0;
        a.snapshots = 1;
        a.final_out = p.tdHin + (u + p.P - 2) * DD;
    } else if (r & 1) {
        piece = (r + 1) / 2;
        a.init = nullptr;
        a.init_identity = 0;
        a.zero_local = 0;
        a.snapshots = 0;
        a.final_out = p.tBr + (u + piece) * DD;
    } else {
        piece = r / 2;
        a.init = nullptr;
        a.init_identity = 1;
        a.zero_local = 1;
        a.snapshots = 0;
        a.final_out = p.tTr + (u + piece) * DD;
    }
    piece_range(p, n, piece, &a.c0, &a.c1);
    chain_bwd(p, a);
}

// Phase C: piece `piece` <= P - 2 reruns the reverse chain from the dS leaving it
// (tdHin) with snapshots; piece 0 writes dh0.
__device__ __forceinline__ void piece_c_bwd_role(const Params &p, int unit, int piece) {
    const int n = unit / p.H, h = unit % p.H;
    const size_t DD = (size_t)D * D;
    ChainBwd a;
    a.n = n;
    a.h = h;
    a.where = 64;
    a.init_user = 0;
    a.out_user = 1;
    a.init = p.tdHin + ((size_t)unit * p.P + piece) * DD;
    a.init_identity = 0;
    a.zero_local = 0;
    a.snapshots = 1;
    a.final_out = (piece == 0 && p.dh0) ? p.dh0 + (size_t)unit * DD : nullptr;
    piece_range(p, n, piece, &a.c0, &a.c1);
    chain_bwd(p, a);
}

// One launch per phase for both chains: CTAs [0, units * roles) take the forward
// chain's roles (pf: no final state), the rest the reverse chain's.
__global__ void __launch_bounds__(NT, 1) tc_bwd_piece_a_kernel(const __grid_constant__ Params pf,
                                                                const __grid_constant__ Params p) {
    const int roles = 2 * p.P - 3, nf = p.N * p.H * roles, blk = blockIdx.x;
    if (blk < nf) piece_a_fwd_role(pf, blk / roles, blk % roles, 0);
    else piece_a_bwd_role(p, (blk - nf) / roles, (blk - nf) % roles);
}

__global__ void __launch_bounds__(NT, 1) tc_bwd_piece_scan_kernel(const __grid_constant__ Params p) {
    const int units = p.N * p.H;
    if ((int)blockIdx.x < units)  // H_in(q) = M_{q-1} H_in(q-1) + B_{q-1}, q = 2 .. P - 1
        piece_scan_body(p, blockIdx.x, p.tHin, p.tMp, p.tBp, 2, p.P - 1, 1, 33);
    else  // dS leaving piece q = dS leaving piece q + 1, times T_{q+1}, plus its offset
        piece_scan_body(p, blockIdx.x - units, p.tdHin, p.tTr, p.tBr, p.P - 3, 0, -1, 66);
}

__global__ void __launch_bounds__(NT, 1) tc_bwd_piece_c_kernel(const __grid_constant__ Params pf,
                                                                const __grid_constant__ Params p) {
    const int per = p.P - 1, nf = p.N * p.H * per, blk = blockIdx.x;
    if (blk < nf) piece_c_fwd_role(pf, blk / per, 1 + blk % per, 0);
    else piece_c_bwd_role(p, (blk - nf) / per, (blk - nf) % per);
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
    // q rows 0-63 and k rows 64-127 form one 128-row tile, dO and v another; then the
    // images S, dSn, U^T, dU^T, A; TA: the dU^T A operand tile, then dq's staged rows;
    // DKS: dv's staged rows, then dk's; the dPG tile; the dLG tile, which first holds
    // the Y = dU U^T operand tile
    static constexpr int kQK = 0, kDV = 32768, kSC = 65536, kDSN = 98304, kUT = 131072,
                         kDUT = 147456, kAB = 163840, kTA = 172032, kDKS = 188416,
                         kDPG = 204800, kDLG = 212992, kY = kDLG, kVec = 221184,
                         kVecFloats = 2432, kEnd = kVec + kVecFloats * 4;
};
constexpr int kGradSmem = GradSmem::kEnd + 1024;
static_assert(GradSmem::kDPG == GradSmem::kDKS + 2 * C * 128, "dv's and dk's staged rows: 16 KB");
static_assert(GradSmem::kAB == GradSmem::kDUT + 2 * C * 128 && GradSmem::kAB % 1024 == 0,
              "the 8 KB before A (the second half of dU^T) are the unused rows of A^T Y");

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

// Writes this thread's column (tokens cb + q, column `col`) into a 64-row SW128
// bf16 tile (the layout of the row loads and stores).
__device__ __forceinline__ void stage_col(uint8_t *tile, const float *x, int cb, int col) {
    uint8_t *c0 = tile + (col >> 6) * C * 128 + (col & 7) * 2;
    const int cp = (col & 63) >> 3;
#pragma unroll
    for (int q = 0; q < CW; ++q)  // row cb + q, whose swizzle term is q % 8 (cb is a multiple of 8)
        *reinterpret_cast<bf16 *>(c0 + (cb + q) * 128 + ((cp ^ (q & 7)) << 4)) =
            __float2bfloat16_rn(x[q]);
}

// Stores rows [0, len) and columns [0, width) of a staged 64-row SW128 tile to
// one chunk and head of a [tokens][H][width] bf16 tensor.  A full chunk goes
// out by tensor-map stores (one box per 64 columns) issued by thread 0 (which
// must wait for their reads before the tile is rewritten); a shorter chunk by
// 16-byte stores of every thread, so that no row past its end is written.  The
// staged rows must have been fenced for the async proxy and published by a
// barrier.
__device__ __forceinline__ void store_tile(const CUtensorMap *map, bf16 *dst, const uint8_t *tile,
                                           int64_t tok0, int len, int h, int H, int width) {
    if (len == C) {
        if (threadIdx.x == 0) {
            tma_store_3d(map, 0, h, (int)tok0, smem_u32(tile));
            if (width == D) tma_store_3d(map, 64, h, (int)tok0, smem_u32(tile) + C * 128);
            bulk_commit();
        }
        return;
    }
    for (int t = threadIdx.x; t < C * 16; t += NG) {
        const int i = t >> 4, j = t & 15;
        if (i < len && j * 8 < width)
            *reinterpret_cast<uint4 *>(dst + ((tok0 + i) * H + h) * width + j * 8) =
                *reinterpret_cast<const uint4 *>(tile + sw128_chunk(C, i, j));
    }
}

// Input groups of one tc_grads unit, each completing on its own mbarrier (bit b
// of a mask is group b): the state images with G and b, the dO and v rows, A,
// and the q and k rows.
enum : uint32_t { kGrpImg = 1, kGrpDV = 2, kGrpA = 4, kGrpQK = 8, kGrpAll = 15 };
constexpr int kGrpCount = 4;

// Issues (one thread) the copies of the groups in `mask` for unit u, whose
// chunk is cn; G and b land in [G | b] slot `gslot` of the vector area.
__device__ __forceinline__ void grads_fetch(const Params &p, uint8_t *sm, int u,
                                            const ChunkInfo &cn, uint32_t mask, int gslot,
                                            uint64_t *bars) {
    using S_ = GradSmem;
    constexpr uint32_t kImgA = C * C * 2;
    const int h = u % p.H;
    if (mask & kGrpImg) {
        uint64_t *bar = &bars[0];
        mbar_arrive_expect_tx(bar, 2 * kImg128 + 2 * kImgUT + 2 * C * 4);
        bulk_load(smem_u32(sm + S_::kSC), static_cast<const uint8_t *>(p.tS) + (size_t)u * kImg128,
                  kImg128, bar);
        bulk_load(smem_u32(sm + S_::kDSN),
                  static_cast<const uint8_t *>(p.tdSn) + (size_t)u * kImg128, kImg128, bar);
        bulk_load(smem_u32(sm + S_::kUT), static_cast<const uint8_t *>(p.tUT) + (size_t)u * kImgUT,
                  kImgUT, bar);
        bulk_load(smem_u32(sm + S_::kDUT),
                  static_cast<const uint8_t *>(p.tdUT) + (size_t)u * kImgUT, kImgUT, bar);
        float *gb = reinterpret_cast<float *>(sm + S_::kVec) + gslot * 128;
        bulk_load(smem_u32(gb), p.tG + (size_t)u * C, C * 4, bar);
        bulk_load(smem_u32(gb + C), p.tB + (size_t)u * C, C * 4, bar);
    }
    if (mask & kGrpDV) {
        uint64_t *bar = &bars[1];
        mbar_arrive_expect_tx(bar, 2 * row_tile_bytes(p.V));
        load_rows_tma(sm + S_::kDV, D, 0, &p.tm_do, cn.tok0, h, p.V, bar);
        load_rows_tma(sm + S_::kDV, D, C, &p.tm_v, cn.tok0, h, p.V, bar);
    }
    if (mask & kGrpA) {
        uint64_t *bar = &bars[2];
        mbar_arrive_expect_tx(bar, kImgA);
        bulk_load(smem_u32(sm + S_::kAB), static_cast<const uint8_t *>(p.tA) + (size_t)u * kImgA,
                  kImgA, bar);
    }
    if (mask & kGrpQK) {
        uint64_t *bar = &bars[3];
        mbar_arrive_expect_tx(bar, 2 * row_tile_bytes(p.K));
        load_rows_tma(sm + S_::kQK, D, 0, &p.tm_q, cn.tok0, h, p.K, bar);
        load_rows_tma(sm + S_::kQK, D, C, &p.tm_k, cn.tok0, h, p.K, bar);
    }
}

// Bounded wait of the whole CTA for the groups in `mask` to complete phase
// `parity`; records `where` on failure.
__device__ __forceinline__ bool groups_arrived(uint64_t *bars, uint32_t mask, uint32_t parity,
                                               const Params &p, int where) {
    bool ok = true;
    for (int g = 0; g < kGrpCount; ++g)
        if ((mask >> g) & 1) ok = ok && mbar_wait(&bars[g], parity, p.wait_limit);
    const bool all = __syncthreads_and(ok);
    if (!all && threadIdx.x == 0) record_timeout(p, where);
    return all;
}

// After a failed wait: one more bounded wait for the groups still in flight.
__device__ __forceinline__ void groups_drain(uint64_t *bars, uint32_t mask, uint32_t parity) {
    for (int g = 0; g < kGrpCount; ++g)
        if ((mask >> g) & 1) mbar_wait(&bars[g], parity, kWaitLimit);
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

// Bounded wait of one thread for an MMA-completion phase, after which it may
// read the products (the CTA decides on a failure at its next barrier).
__device__ __forceinline__ bool thread_wait(uint64_t *bar, uint32_t parity, uint32_t limit) {
    const bool ok = mbar_wait(bar, parity, limit);
    tc_fence_after();
    return ok;
}

// Shared-memory addresses of tc_grads' operand tiles, from the aligned base.
struct GradTiles {
    uint32_t qk, k, dv, sc, dsn, ut, dut, a, ta, y, dpg, dlg;
    __device__ __forceinline__ explicit GradTiles(uint32_t b)
        : qk(b + GradSmem::kQK), k(b + GradSmem::kQK + C * 128), dv(b + GradSmem::kDV),
          sc(b + GradSmem::kSC), dsn(b + GradSmem::kDSN), ut(b + GradSmem::kUT),
          dut(b + GradSmem::kDUT), a(b + GradSmem::kAB), ta(b + GradSmem::kTA), y(b + GradSmem::kY),
          dpg(b + GradSmem::kDPG), dlg(b + GradSmem::kDLG) {}
};

__global__ void __launch_bounds__(NG, 1) tc_grads_kernel(const __grid_constant__ Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = align1k(smem_raw);
    // MMA completions (one phase in flight on each): mbar_a Y and (A^T dU)^T; mbar
    // [Q;K] K^T and dP, then the last products; mbar_z -dL and Zp; mbar_c X1^T, X2^T
    __shared__ uint64_t mbar, mbar_a, mbar_c, mbar_z, ibar, lbar[kGrpCount];
    __shared__ uint32_t tslot;
    __shared__ float s_hd;
    if (p.hdr->status) return;
    const int H = p.H, nunits = p.NC * H, tid = threadIdx.x;
    const int wg = tid >> 7, r = tid & 127, cb = CW * wg, l = tid & 31, w4 = (tid >> 5) & 3;
    const int i64 = l < 16 ? w4 * 16 + l : -1;  // M = 64 row of this thread's lane
    using S_ = GradSmem;
    uint8_t *QK = sm + S_::kQK, *DV = sm + S_::kDV, *SC = sm + S_::kSC, *DSN = sm + S_::kDSN,
            *TA = sm + S_::kTA, *DKS = sm + S_::kDKS, *YT = sm + S_::kY, *DPG = sm + S_::kDPG,
            *DLG = sm + S_::kDLG;
    float *vec = reinterpret_cast<float *>(sm + S_::kVec);
    // vec + 0: two [G | b] slots of 128 floats, the current unit's and the prefetched one's
    float *gam = vec + 256, *e = vec + 320, *dB = vec + 384, *qx = vec + 448, *kx = vec + 512,
          *kz = vec + 576, *dG = vec + 640, *tmp = vec + 704, *dbl2 = vec + 768,
          *qinv = vec + 1024, *kinv = vec + 1088, *rowp = vec + 1152;
    // per-warp partial column sums, four sets of [4 warps][64 columns]
    float *wsum = vec + 1408;
    float *qdot = rowp, *kdot = rowp + 64;  // (the row partials are consumed before the epilogue)
    const uint32_t smb = smem_u32(sm);  // (the tiles' addresses are formed where issued)
    if (tid == 0) {
        for (int g = 0; g < kGrpCount; ++g) mbar_init(&lbar[g], 1);
        mbar_init(&mbar, 1);
        mbar_init(&mbar_a, 1);
        mbar_init(&mbar_c, 1);
        mbar_init(&mbar_z, 1);
        mbar_init(&ibar, 1);
        fence_mbar_init();
    }
    if (tid < 32) {
        tmem_alloc(&tslot, 512);
        tmem_relinquish();
    }
    __syncthreads();  // publishes the mbarrier inits and the TMEM address
    const uint32_t tmem = tslot;
    // The CTA runs units (chunk, head) blockIdx.x, + gridDim.x, ...  Each input
    // group of the next unit is fetched as soon as the current unit has
    // consumed that group's buffers, so the copies run under the compute.
    int unit = blockIdx.x;
    if (tid == 0 && unit < nunits) {
        const ChunkInfo cn = chunk_at(p, unit / H);
        grads_fetch(p, sm, unit, cn, kGrpAll, 0, lbar);
    }
    uint32_t pend = kGrpAll, ppar = 0;  // load groups in flight and the phase they complete
    uint32_t phase = 0;                 // MMA-completion barrier
    bool ok = true;
    for (int it = 0; unit < nunits; ++it, unit += gridDim.x) {
        const int c = unit / H, h = unit % H, next = unit + (int)gridDim.x;
        const bool more = next < nunits;
        const ChunkInfo ci = chunk_at(p, c);
        const float *G = vec + (it & 1) * 128, *bta = G + 64;
        // A full chunk with 128-wide heads and no normalisation needs no pass over its
        // rows: its q and k rows are then waited for by the thread that issues [Q;K] K^T
        // only, after the products that do not read them
        const bool late_qk = ci.len == C && p.K == D && p.V == D && !p.l2norm;
        const uint32_t first = late_qk ? (pend & ~uint32_t(kGrpQK)) : pend;
        ok = groups_arrived(lbar, first, ppar, p, 20);
        if (!ok) break;
        pend &= ~first;
        if (tid < C) {
            gam[tid] = expf(G[tid]);
            e[tid] = expf(G[C - 1] - G[tid]);
        }
        if (!late_qk) {
            fix_rows(QK, D, 0, ci.len, p.K, NG);
            fix_rows(QK, D, C, ci.len, p.K, NG);
            fix_rows(DV, D, 0, ci.len, p.V, NG);
            fix_rows(DV, D, C, ci.len, p.V, NG);
            operands_ready();
        }
        if (p.l2norm) {  // q rows (threads 0-127) and k rows (128-255) divided by their norms
            l2norm_tile_rows(QK, D, 0, qinv, 0);
            l2norm_tile_rows(QK, D, C, kinv, 2 * C);
            operands_ready();
        }
        // TMEM columns (64 each).  [Q;K] K^T stays to the dL phase (P on lanes 0-63, K K^T
        // on lanes 64-127).  Y = dU U^T (M = 64) is read into a tile, and its columns then
        // take A^T Y = -dL; (A^T dU)^T's take Zp^T = (A^T dU H^T)^T once read; dP's take
        // (dPG K)^T.
        constexpr int cQK = 0, cX1 = 64, cX2 = 128, cDK = 192, cDP = 256, cAU = 320, cY = 384,
                      cDKA = 448, cZ = cAU, cDL = cY, cDQ = cDP;
        float d[CW];
        bool qk_ok = true;
        if (tid == 0) {  // the products the SIMT work needs first
            const GradTiles t(smb);
            const uint32_t i64mm = idesc_bf16(64, 64, 1, 1), i128km = idesc_bf16(128, 64, 0, 1);
#pragma unroll
            for (int s = 0; s < 8; ++s)  // Y = dU U^T (M = 64, over v)
                mma_bf16(tmem + cY, desc_mnmajor(t.dut, D, s), desc_mnmajor(t.ut, D, s), i64mm, s > 0);
#pragma unroll
            for (int s = 0; s < 4; ++s)  // (A^T dU)^T = dU^T A
                mma_bf16(tmem + cAU, desc_kmajor(t.dut, D, s), desc_mnmajor(t.a, C, s), i128km, s > 0);
            mma_commit(&mbar_a);
            mbar_arrive(&ibar);  // the products of the P . dP phase go in after these
        } else if (tid == 32) {  // warp 1's leader: the products of the P . dP phase
            const GradTiles t(smb);
            const uint32_t i128 = idesc_bf16(128, 64, 0, 0), i128km = idesc_bf16(128, 64, 0, 1);
            qk_ok = mbar_wait(&ibar, it & 1, p.wait_limit);
            if (qk_ok) {
#pragma unroll
                for (int s = 0; s < 8; ++s)  // [dO; V] U^T: lanes 0-63 dP = dO U^T, next to P
                    mma_bf16(tmem + cDP, desc_kmajor(t.dv, D, s), desc_mnmajor(t.ut, D, s), i128km,
                             s > 0);
                qk_ok = !(pend & kGrpQK) || mbar_wait(&lbar[3], ppar, p.wait_limit);
            }
            if (qk_ok) {
#pragma unroll
                for (int s = 0; s < 8; ++s)  // [Q;K] K^T: lanes 0-63 Q K^T, lanes 64-127 K K^T
                    mma_bf16(tmem + cQK, desc_kmajor(t.qk, D, s), desc_kmajor(t.k, D, s), i128,
                             s > 0);
            }
            mma_commit(&mbar);
        } else if (tid >= 64) {  // <S, dSn> (identically laid out images) by warps 2-15
            float s = 0.f;
            for (int t = tid - 64; t < D * D / 8; t += NG - 64) {
                float a[8], b[8];
                unpack8(*reinterpret_cast<const uint4 *>(SC + t * 16), a);
                unpack8(*reinterpret_cast<const uint4 *>(DSN + t * 16), b);
#pragma unroll
                for (int q = 0; q < 8; ++q) s = fmaf(a[q], b[q], s);
            }
            for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
            if (l == 0) tmp[(tid >> 5) - 2] = s;
            bar_sync(1, NG - 64);
            if (tid == 64) {
                float a = 0.f;
                for (int w = 0; w < NG / 32 - 2; ++w) a += tmp[w];
                s_hd = a;  // read after later barriers
            }
        }
        if (tid == 0) bulk_wait_read();  // the previous unit's dq and dk rows staged in TA, DKS are out
        {
            const bool ok_a = mbar_wait(&mbar_a, it & 1, p.wait_limit);
            ok = __syncthreads_and(ok_a && qk_ok);  // (qk_ok: thread 32's wait for the q, k rows)
            tc_fence_after();
            if (!ok) {
                if (!ok_a) record_timeout(p, 26);
                if (!qk_ok) record_timeout(p, 20);
                break;
            }
        }
        pend &= ~uint32_t(kGrpQK);
        ldcw(tmem, cY + cb, d);  // Y as a 64 x 64 operand tile (rows of the M = 64 layout)
        if (i64 >= 0) {
#pragma unroll
            for (int q = 0; q < CW / 8; ++q)
                *reinterpret_cast<uint4 *>(YT + sw128_chunk(C, i64, cb / 8 + q)) = pack8(d + 8 * q);
        }
        {  // (A^T dU)^T = dU^T A (thread r holds row v = r): as an operand tile in TA;
           // dv = diag(b) A^T dU, staged in DKS (thread r holds column r); partial v . (A^T dU)
            ldcw(tmem, cAU + cb, d);
#pragma unroll
            for (int q = 0; q < CW / 8; ++q)
                *reinterpret_cast<uint4 *>(TA + sw128_chunk(D, r, cb / 8 + q)) = pack8(d + 8 * q);
            {
                float y[CW];
#pragma unroll
                for (int q = 0; q < CW; ++q) y[q] = bta[cb + q] * d[q];
                stage_col(DKS, y, cb, r);
            }
            {
                const ColSw vcol(DV + C * 128, D, r);
#pragma unroll
                for (int q = 0; q < CW; ++q) d[q] *= vcol.at(cb, q);
            }
            warp_colsum(d, wsum, w4, cb, l);
        }
        operands_ready();  // (also publishes the staged dv rows to the tensor-map store)
        store_tile(&p.tm_dv, static_cast<bf16 *>(p.dv), DKS, ci.tok0, ci.len, h, H, p.V);
        if (tid == 2 * 32) {  // warp 2 (rows 64-95) has no part in the P . dP phase below
            const GradTiles t(smb);
            const uint32_t i128mm = idesc_bf16(128, 64, 1, 1), i128mk = idesc_bf16(128, 64, 1, 0);
#pragma unroll
            for (int s = 0; s < 4; ++s)  // A^T Y = -dL on rows 64-127 (M = 128: rows 0-63 of
                                         // the A operand are the 8 KB before A, not used)
                mma_bf16(tmem + cDL, desc_mnmajor(t.a - C * 128, C, s), desc_mnmajor(t.y, C, s),
                         i128mm, s > 0);
#pragma unroll
            for (int s = 0; s < 8; ++s)  // Zp^T = S^T (dU^T A) = (A^T X3)^T, X3 = dU H^T
                mma_bf16(tmem + cZ, desc_mnmajor(t.sc, D, s), desc_mnmajor(t.ta, D, s), i128mm,
                         s > 0);
            mma_commit(&mbar_z);
#pragma unroll
            for (int s = 0; s < 8; ++s)  // X1^T = S^T dO^T  (over v)
                mma_bf16(tmem + cX1, desc_mnmajor(t.sc, D, s), desc_kmajor(t.dv, D, s), i128mk,
                         s > 0);
#pragma unroll
            for (int s = 0; s < 8; ++s)  // X2^T = dSn^T U^T
                mma_bf16(tmem + cX2, desc_mnmajor(t.dsn, D, s), desc_mnmajor(t.ut, D, s), i128mm,
                         s > 0);
            mma_commit(&mbar_c);
        }
        if (tid < C) {  // dbeta's share from Ut = A diag(b) V (the partials were published above)
            const float *w = wsum + tid;
            dB[tid] = (w[0] + w[64]) + (w[128] + w[192]);
        }
        // meanwhile, each thread waiting for what it reads itself (no barrier waits on the
        // issuing warp); the CTA decides on a failed wait at the barrier after them.  The
        // P . dP phase (rows on lanes 0-63) and the dL phase (lanes 64-127) run side by side
        bool fine = true;
        if (w4 < 2) fine = thread_wait(&mbar, phase, p.wait_limit);  // Q K^T and dP
        else  // K K^T, and -dL
            fine = thread_wait(&mbar, phase, p.wait_limit) && thread_wait(&mbar_z, it & 1, p.wait_limit);
        phase ^= 1;
        if (w4 < 2) {  // row i = r of P and dP: P . dP (row and column partials), dPG = dP . Gam
            float pq[CW];
            tmem_ld16(tmq(tmem, cQK + cb), pq);
            tmem_ld16(tmq(tmem, cDP + cb), d);
            tmem_ld_wait();
            const float gi = G[r];
            float rs = 0.f;
#pragma unroll
            for (int q = 0; q < CW; ++q) {
                const int j = cb + q;
                const float gm = __expf(j <= r ? gi - G[j] : -INFINITY);  // Gam (0 above diagonal)
                const float dp = j <= r ? d[q] : 0.f;
                pq[q] = (p.scale * gm * pq[q]) * dp;
                rs += pq[q];
                d[q] = dp * gm;
            }
            rowp[wg * 64 + r] = rs;
#pragma unroll
            for (int q = 0; q < CW / 8; ++q)
                *reinterpret_cast<uint4 *>(DPG + sw128_chunk(C, r, cb / 8 + q)) = pack8(d + 8 * q);
            warp_colsum(pq, wsum + 768, w4, cb, l);
        } else {  // row i = r - 64: dL (strictly lower), Gam . K K^T; dLG = diag(b) dL . Gam
            const int i = r - C;
            float kk[CW];
            tmem_ld16(tmq(tmem, cQK + cb), kk);
            tmem_ld16(tmq(tmem, cDL + cb), d);
            tmem_ld_wait();
            const float bi = bta[i], gi = G[i];
            float dbl = 0.f;
#pragma unroll
            for (int q = 0; q < CW; ++q) {
                const int j = cb + q;
                const float gm = __expf(j < i ? gi - G[j] : -INFINITY);
                const float dl = j < i ? -d[q] : 0.f;
                const float kkg = gm * kk[q];
                kk[q] = dl * bi * kkg;
                dbl = fmaf(dl, kkg, dbl);
                d[q] = bi * dl * gm;
            }
#pragma unroll
            for (int q = 0; q < CW / 8; ++q)
                *reinterpret_cast<uint4 *>(DLG + sw128_chunk(C, i, cb / 8 + q)) = pack8(d + 8 * q);
            dbl2[wg * 64 + i] = dbl;
            warp_colsum(kk, wsum + 768, w4, cb, l);
        }
        ok = __syncthreads_and(fine);
        if (!ok) {
            if (tid == 0) record_timeout(p, 21);
            break;
        }
        if (more) {  // A of the next unit (its last product is done)
            if (tid == 0) grads_fetch(p, sm, next, ci, kGrpA, 0, lbar);
            pend |= kGrpA;
        }
        fine = thread_wait(&mbar_c, it & 1, p.wait_limit);  // X1, X2
        {  // partial q' . X1 (thread kk); a column reader costs 8 registers: built where used
            const ColSw qcol(QK, D, r);
            ldcw(tmem, cX1 + cb, d);
#pragma unroll
            for (int q = 0; q < CW; ++q) d[q] *= p.scale * qcol.at(cb, q);
            warp_colsum(d, wsum + 256, w4, cb, l);
        }
        {  // partial k . X2, and k . Z = -k . Zp (its set of partials was consumed above)
            const ColSw kcol(QK + C * 128, D, r);
            float z[CW];
            tmem_ld16(tmq(tmem, cX2 + cb), d);
            tmem_ld16(tmq(tmem, cZ + cb), z);
            tmem_ld_wait();
#pragma unroll
            for (int q = 0; q < CW; ++q) {
                const float kv = kcol.at(cb, q);
                d[q] *= kv;
                z[q] *= -kv;
            }
            warp_colsum(d, wsum + 512, w4, cb, l);
            warp_colsum(z, wsum, w4, cb, l);
        }
        fence_async_smem();  // the dPG and dLG tiles are read by the products below
        tc_fence_before();
        ok = __syncthreads_and(fine);
        tc_fence_after();
        if (!ok) {
            if (tid == 0) record_timeout(p, 23);
            break;
        }
        if (more) {  // S, dSn, U^T, dU^T, G and b, and the dO and v rows of the next unit
                     // (every product reading them is complete: X2 was the last)
            if (tid == 0) {
                grads_fetch(p, sm, next, ci, kGrpImg, (it + 1) & 1, lbar);
                grads_fetch(p, sm, next, chunk_at(p, next / H), kGrpDV, 0, lbar);
            }
            pend |= kGrpImg | kGrpDV;
            ppar = (it + 1) & 1;
        }
        if (tid == 7 * 32) {  // warp 7 has no part in the sums and the scan below
            const GradTiles t(smb);
            const uint32_t imk = idesc_bf16(128, 64, 1, 0), imm = idesc_bf16(128, 64, 1, 1);
#pragma unroll
            for (int s = 0; s < 4; ++s)  // (dPG K)^T = K^T dPG^T
                mma_bf16(tmem + cDQ, desc_mnmajor(t.k, D, s), desc_kmajor(t.dpg, C, s), imk, s > 0);
#pragma unroll
            for (int s = 0; s < 4; ++s)  // (dPG^T Q)^T = Q^T dPG
                mma_bf16(tmem + cDKA, desc_mnmajor(t.qk, D, s), desc_mnmajor(t.dpg, C, s), imm, s > 0);
#pragma unroll
            for (int s = 0; s < 4; ++s)  // (diag(b) dLG K)^T
                mma_bf16(tmem + cDK, desc_mnmajor(t.k, D, s), desc_kmajor(t.dlg, C, s), imk, s > 0);
#pragma unroll
            for (int s = 0; s < 4; ++s)  // ((diag(b) dLG)^T K)^T
                mma_bf16(tmem + cDK, desc_mnmajor(t.k, D, s), desc_mnmajor(t.dlg, C, s), imm, 1);
            mma_commit(&mbar);
        }
        if (tid < 3 * C) {  // (warps 0-5)
            const int k = tid >> 6, i = tid & 63;
            const float *w = wsum + k * 256 + i;
            (k == 0 ? kz : k == 1 ? qx : kx)[i] = (w[0] + w[64]) + (w[128] + w[192]);
            bar_sync(2, 3 * C);
        }
        // meanwhile: dbeta and dG (rows), then dg = reverse cumulative sum of dG.  The
        // row sums of P . dP + dL . L are the row partials plus b times the dL rows'
        // sums; the column sums come from the last set of warp partials.
        if (tid < C) {
            const int i = tid;
            const float *w = wsum + 768 + i;
            const float dbs = (dbl2[i] + dbl2[64 + i]) + (dbl2[128 + i] + dbl2[192 + i]);
            const float rsum = ((rowp[i] + rowp[64 + i]) + (rowp[128 + i] + rowp[192 + i])) +
                               bta[i] * dbs;
            const float csum = (w[0] + w[64]) + (w[128] + w[192]);
            dG[i] = -e[i] * kx[i] + gam[i] * qx[i] + (rsum - csum) + bta[i] * gam[i] * kz[i];
            dB[i] += dbs + gam[i] * kz[i];
            bar_sync(3, C);  // (warps 0-1)
        }
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
        if (tid == 0) bulk_wait_read();  // the staged dv rows are out (dk's are staged next)
        ok = cta_wait(&mbar, phase, p, 25);
        phase ^= 1;
        if (!ok) break;
        if (more && !p.l2norm) {  // q and k rows of the next unit (the epilogue reads only TMEM)
            if (tid == 0) grads_fetch(p, sm, next, chunk_at(p, next / H), kGrpQK, 0, lbar);
            pend |= kGrpQK;
        }
        {  // dq = scale (diag(gam) X1 + dPG K); dk = diag(e) X2 + diag(b gam) Z + dPG^T Q'
           // + dL terms; staged (thread r holds column r): dq in TA, dk in DKS
            float a[CW];
            tmem_ld16(tmq(tmem, cX1 + cb), d);
            tmem_ld16(tmq(tmem, cDQ + cb), a);
            tmem_ld_wait();
#pragma unroll
            for (int q = 0; q < CW; ++q) d[q] = p.scale * (gam[cb + q] * d[q] + a[q]);
            if (p.l2norm) project_rows(d, ColSw(QK, D, r), qinv, qdot, wsum, w4, cb, l);
            stage_col(TA, d, cb, r);
            tmem_ld16(tmq(tmem, cX2 + cb), d);
            tmem_ld16(tmq(tmem, cZ + cb), a);
            tmem_ld_wait();
#pragma unroll
            for (int q = 0; q < CW; ++q) d[q] = e[cb + q] * d[q] - bta[cb + q] * gam[cb + q] * a[q];
            {
                float z[CW];
                tmem_ld16(tmq(tmem, cDKA + cb), a);
                tmem_ld16(tmq(tmem, cDK + cb), z);
                tmem_ld_wait();
#pragma unroll
                for (int q = 0; q < CW; ++q) d[q] += p.scale * a[q] + z[q];
            }
            if (p.l2norm)
                project_rows(d, ColSw(QK + C * 128, D, r), kinv, kdot, wsum + 256, w4, cb, l);
            stage_col(DKS, d, cb, r);
        }
        fence_async_smem();
        __syncthreads();  // the unit's reads are done and the staged rows are visible
        if (more && p.l2norm) {
            if (tid == 0) grads_fetch(p, sm, next, chunk_at(p, next / H), kGrpQK, 0, lbar);
            pend |= kGrpQK;
        }
        store_tile(&p.tm_dq, static_cast<bf16 *>(p.dq), TA, ci.tok0, ci.len, h, H, p.K);
        store_tile(&p.tm_dk, static_cast<bf16 *>(p.dk), DKS, ci.tok0, ci.len, h, H, p.K);
        if (ci.len < C) __syncthreads();  // (the next unit rewrites the tiles)
    }
    if (!ok && tid == 0) groups_drain(lbar, pend, ppar);  // leave no copy in flight
    if (tid == 0) bulk_wait_all();
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
        if ((e = set_smem(tc_prep_local_kernel, kPrepSmemRequest))) return e;
        GDN_LAUNCH(kKTcLocal, stream,
                   tc_prep_local_kernel<<<nch, NT, kPrepSmemRequest, stream>>>(p));
    }
    const int sm = kSbwdSmem > kStateSmem ? kSbwdSmem : kStateSmem;
    if (nseq > 0 && p.P > 1) {  // piece scan of long rows, for both chains
        pf.vslice = 0;
        const int roles = 2 * p.P - 3;
        if ((e = set_smem(tc_bwd_piece_a_kernel, sm))) return e;
        GDN_LAUNCH(kKTcPieceA, stream,
                   tc_bwd_piece_a_kernel<<<2 * nseq * roles, NT, sm, stream>>>(pf, p));
        if ((e = set_smem(tc_bwd_piece_scan_kernel, kScanSmem))) return e;
        GDN_LAUNCH(kKTcPieceScan, stream,
                   tc_bwd_piece_scan_kernel<<<2 * nseq, NT, kScanSmem, stream>>>(p));
        if ((e = set_smem(tc_bwd_piece_c_kernel, sm))) return e;
        GDN_LAUNCH(kKTcPieceC, stream,
                   tc_bwd_piece_c_kernel<<<2 * nseq * (p.P - 1), NT, sm, stream>>>(pf, p));
    } else if (nseq > 0) {
        if ((e = set_smem(tc_chains_kernel, sm))) return e;
        GDN_LAUNCH(kKTcStateBwd, stream, tc_chains_kernel<<<2 * nseq, NT, sm, stream>>>(pf, p));
    }
    if (nch > 0) {
        if ((e = set_smem(tc_grads_kernel, kGradSmem))) return e;
        int grid = 0;  // one persistent CTA per SM (or per unit, if fewer)
        if ((e = persistent_grid(nch, 1, grid))) return e;
        GDN_LAUNCH(kKTcGrads, stream, tc_grads_kernel<<<grid, NG, kGradSmem, stream>>>(p));
    }
    return cudaSuccess;
}

static_assert(kGradSmem <= 227 * 1024, "grads shared memory");
static_assert(kSbwdSmem <= 227 * 1024, "reverse state shared memory");

}  // namespace gdn
