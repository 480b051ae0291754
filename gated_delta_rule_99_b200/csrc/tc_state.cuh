// Forward state pass of the tensor-core path (shared by the forward launch
// and by the backward, which recomputes the per-chunk states concurrently
// with its reverse pass).
#pragma once

#include "tc_common.cuh"

namespace gdn {
namespace tc {

// ============================================================ tc_state_fwd
// One CTA per (sequence, head); thread v owns row v of S (fp32 registers).
struct StateSmem {
    // two images of the state (the next chunk's is written while the current one
    // may still be read), U^T, the 64 x 64 identity block that adds Ut^T inside
    // the first product, and per prefetch buffer the W, Kd and Ut images and gates
    static constexpr int kS0 = 0, kUT = kS0 + 2 * 32768, kI = kUT + 16384, kW0 = kI + 8192,
                         kKd0 = kW0 + 2 * 16384, kUt0 = kKd0 + 2 * 16384, kG0 = kUt0 + 2 * 16384,
                         kEnd = kG0 + 2 * 256;
};
constexpr int kStateSmem = StateSmem::kEnd + 1024;

// Bulk copies (thread 0) of chunk ch's W, Kd and Ut images (Ut unless the run
// takes it as zero) and its gate row into buffer `buf`, completing on `bar`.
// Thread kPrefetcher issues the chains' prefetch copies and snapshot stores, so that
// thread 0, which issues the products, is not held up by them.
constexpr int kPrefetcher = 64;

__device__ __forceinline__ void state_prefetch(uint8_t *sm, int buf, size_t ch, const Params &p,
                                               bool with_ut, uint64_t *bar) {
    if (threadIdx.x != kPrefetcher) return;
    mbar_arrive_expect_tx(bar, (with_ut ? 3u : 2u) * (uint32_t)kImg64 + C * 4u);
    bulk_load(smem_u32(sm + StateSmem::kW0 + buf * 16384),
              static_cast<const uint8_t *>(p.tW) + ch * kImg64, kImg64, bar);
    bulk_load(smem_u32(sm + StateSmem::kKd0 + buf * 16384),
              static_cast<const uint8_t *>(p.tKd) + ch * kImg64, kImg64, bar);
    if (with_ut)
        bulk_load(smem_u32(sm + StateSmem::kUt0 + buf * 16384),
                  static_cast<const uint8_t *>(p.tUt) + ch * kImg64, kImg64, bar);
    bulk_load(smem_u32(sm + StateSmem::kG0 + buf * 256), p.tG + ch * C, C * 4, bar);
}

// One run of the forward chain over chunks [c0, c1) of one head.
struct ChainFwd {
    int h, c0, c1;
    const float *init;   // state H entering chunk c0 (fp32), or nullptr for zero
    int init_user;       // init is a caller's [K][V] block (else an internal [128][128] one)
    int init_identity;   // start from H = I (the transition-matrix run of the piece scan)
    int zero_ut;         // take Ut as zero (the transition-matrix run)
    int snapshots;       // write the state entering every chunk and U^T (tile images)
    float *final_out;    // state leaving chunk c1 - 1 (fp32), or nullptr
    int out_user;        // final_out is a caller's [K][V] block (else [128][128])
    int where;           // tag recorded if a bounded wait gives up
    int slice;           // value columns [64 slice, 64 slice + 64) (chain_fwd_sliced only)
};

// Writes the 64 x 64 bf16 identity as an SW128 tile (all threads of the CTA).
__device__ __forceinline__ void identity_tile(uint8_t *tile) {
    for (int t = threadIdx.x; t < C * 8; t += NT) {
        const int r = t >> 3, j = t & 7;
        float f[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) f[q] = (r == 8 * j + q) ? 1.f : 0.f;
        *reinterpret_cast<uint4 *>(tile + sw128_chunk(C, r, j)) = pack8(f);
    }
}

// Row v of the state as bf16 operand row v of a 128 x 128 SW128 tile.
__device__ __forceinline__ void state_image(uint8_t *img, const float *S, int v) {
#pragma unroll
    for (int j = 0; j < 16; ++j)
        *reinterpret_cast<uint4 *>(img + sw128_chunk(D, v, j)) = pack8(S + 8 * j);
}

// The forward state chain: thread v owns row v of S = H^T (fp32 registers).
// Per chunk the first product adds Ut^T through an identity block, so U^T
// leaves the accumulator ready to be rounded; the state image of the next
// chunk is written into the other image while the state is updated.
__device__ __forceinline__ void chain_fwd(const Params &p, const ChainFwd &a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = align1k(smem_raw);
    __shared__ uint64_t mbar, lbar[2];
    __shared__ uint32_t tslot;
    if (p.hdr->status) return;
    const int H = p.H, h = a.h, v = threadIdx.x;
    float S[D];
    if (a.init) {
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
    const bool with_ut = !a.zero_ut;
    identity_tile(sm + StateSmem::kI);
    if (a.snapshots) state_image(sm + StateSmem::kS0, S, v);  // the state entering the first chunk
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tslot;
    // TMEM columns: 0-63 U^T, 64-191 the state update, 256-319 the state image and
    // 320-351 the U^T image (bf16 pairs: the A operands of the products that read them;
    // the shared-memory images are kept for the snapshots only)
    constexpr uint32_t cSI = 256, cUI = 320;
    tmem_store_bf16<64>(tm(tmem, cSI), S);
    tmem_st_wait();
    const int c0 = a.c0, c1 = a.c1;
    uint32_t phase = 0;
    // per buffer b (bit b): a copy in flight, and the parity of its next completion
    uint32_t pend = 0, lpar = 0;
    if (c0 < c1) {
        state_prefetch(sm, 0, (size_t)c0 * H + h, p, with_ut, &lbar[0]);
        pend = 1;
    }
    uint8_t *UTs = sm + StateSmem::kUT;
    const uint32_t id1 = idesc_bf16(128, 64, 0, 0), idu = idesc_bf16(128, 64, 1, 0),
                   id2 = idesc_bf16(128, 128, 0, 1), ib = smem_u32(sm + StateSmem::kI);
    for (int c = c0; c < c1; ++c) {
        const int buf = (c - c0) & 1;
        const size_t ch = (size_t)c * H + h;
        uint8_t *Ss = sm + StateSmem::kS0 + buf * 32768, *Sn = sm + StateSmem::kS0 + (buf ^ 1) * 32768;
        const bool lok = mbar_wait(&lbar[buf], (lpar >> buf) & 1u, p.wait_limit);
        fence_async_smem();  // the state image written by the previous chunk's update
        tc_fence_before();
        const bool all = __syncthreads_and(lok);
        tc_fence_after();
        if (!all) {
            if (v == 0) record_timeout(p, 40 + a.where);
            break;
        }
        pend &= ~(1u << buf);
        lpar ^= 1u << buf;
        // the other buffer's chunk was consumed by the previous chunk's products
        if (c + 1 < c1) {
            state_prefetch(sm, buf ^ 1, ch + H, p, with_ut, &lbar[buf ^ 1]);
            pend |= 2u >> buf;
        }
        const float gC =
            expf(reinterpret_cast<const float *>(sm + StateSmem::kG0 + buf * 256)[C - 1]);
        if (v == 0) {  // U^T = S (-W)^T + Ut^T I  (the W image is stored negated)
            const uint32_t wb = smem_u32(sm + StateSmem::kW0 + buf * 16384),
                           ub = smem_u32(sm + StateSmem::kUt0 + buf * 16384);
#pragma unroll
            for (int s = 0; s < D / 16; ++s)
                mma_bf16_ta(tmem, tmem + cSI + 8 * s, desc_kmajor(wb, C, s), id1, s > 0);
            if (with_ut) {
#pragma unroll
                for (int s = 0; s < C / 16; ++s)
                    mma_bf16(tmem, desc_mnmajor(ub, C, s), desc_kmajor(ib, C, s), idu, 1);
            }
            mma_commit(&mbar);
        }
        if (v == kPrefetcher && a.snapshots) {
            bulk_store(static_cast<uint8_t *>(p.tS) + ch * kImg128, smem_u32(Ss), (uint32_t)kImg128);
            bulk_commit();
            // the previous chunk's stores (U^T, and the state image that this chunk's
            // update rewrites) have read their sources
            bulk_wait_read_n<1>();
        }
        if (!cta_wait(&mbar, phase, p, a.where)) break;
        phase ^= 1;
#pragma unroll
        for (int c32 = 0; c32 < C; c32 += 32) {  // U^T as an operand (row v)
            float d[32];
            tmem_ld16(tm(tmem, c32), d);
            tmem_ld16(tm(tmem, c32 + 16), d + 16);
            tmem_ld_wait();
            tmem_store_bf16<16>(tm(tmem, cUI + c32 / 2), d);
            if (a.snapshots) {
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    *reinterpret_cast<uint4 *>(UTs + sw128_chunk(D, v, c32 / 8 + q)) =
                        pack8(d + 8 * q);
            }
        }
        tmem_st_wait();
        operands_ready();
        if (v == 0) {
            const uint32_t kb = smem_u32(sm + StateSmem::kKd0 + buf * 16384);
#pragma unroll
            for (int s = 0; s < C / 16; ++s)
                mma_bf16_ta(tmem + 64, tmem + cUI + 8 * s, desc_mnmajor(kb, C, s), id2, s > 0);
            mma_commit(&mbar);
        }
        if (v == kPrefetcher && a.snapshots) {
            bulk_store(static_cast<uint8_t *>(p.tUT) + ch * kImgUT, smem_u32(UTs), (uint32_t)kImgUT);
            bulk_commit();
        }
        if (!cta_wait(&mbar, phase, p, a.where + 1)) break;
        phase ^= 1;
#pragma unroll
        for (int c32 = 0; c32 < D; c32 += 32) {  // S <- gam_n S + U^T Kd, and the next image
            float d[32];
            tmem_ld16(tm(tmem, 64 + c32), d);
            tmem_ld16(tm(tmem, 64 + c32 + 16), d + 16);
            tmem_ld_wait();
#pragma unroll
            for (int q = 0; q < 32; ++q) S[c32 + q] = fmaf(gC, S[c32 + q], d[q]);
            tmem_store_bf16<16>(tm(tmem, cSI + c32 / 2), S + c32);
            if (a.snapshots) {
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    *reinterpret_cast<uint4 *>(Sn + sw128_chunk(D, v, c32 / 8 + q)) =
                        pack8(S + c32 + 8 * q);
            }
        }
        tmem_st_wait();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }
    if (v == kPrefetcher) {  // copies still in flight after an early exit
        for (int b = 0; b < 2; ++b)
            if ((pend >> b) & 1u) mbar_wait(&lbar[b], (lpar >> b) & 1u, kWaitLimit);
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

// ============================================================ chain with the output
// The forward pass's chain with the output formed in the same CTA.  Each chunk's
// state S and U^T are on the SM anyway, so
//   O^T = S Qg^T + U^T P^T    (M = 128 values, N = 64 tokens, K = 128 + 64)
// over tc_prep's Qg and P images gives the chunk's output without S or U^T
// leaving the SM.  The state and U^T operand images live in TMEM (bf16 pairs,
// the A operand of every product that reads them), so the products read only
// their B operands from shared memory.  Threads 0-127 (warpgroup 0) run the
// chain (thread v owns row v of S; thread 0 issues its products).  Threads
// 128-255 (warpgroup 1) form the output: their leader issues S Qg^T once the
// chain has issued the chunk's first product (m1bar) and U^T P^T once it has
// issued the second (m2bar), into one of two TMEM buffers; then the warpgroup
// reads the accumulator, stages it as token rows and stores them by the tensor
// engine.  The state image is double-buffered, so the chain writes the next
// chunk's while S Qg^T may still read the current one; it waits for obar (the
// previous chunk's output is complete) before rewriting the U^T image, the other
// state image or the previous chunk's prefetch slot.  Every wait is bounded.
struct OutChainSmem {
    // the identity block, two staging tiles of output rows, then per prefetch slot the
    // W, Kd, Ut and Qg images and the P tile; the slots' gate rows (the state and U^T
    // images are in TMEM)
    static constexpr int kI = 0, kStage = kI + 8192, kBuf = kStage + 2 * 16384;
    static constexpr int kW = 0, kKd = 16384, kUt = 32768, kQg = 49152, kP = 65536,
                         kBufBytes = 73728;
    static constexpr int kG0 = kBuf + 2 * kBufBytes, kEnd = kG0 + 2 * 256;
};
constexpr int kOutChainSmem = OutChainSmem::kEnd + 1024;
constexpr int kOutChainThreads = 256;

__device__ __forceinline__ void outchain_prefetch(uint8_t *sm, int buf, size_t ch, const Params &p,
                                                  uint64_t *bar) {
    uint8_t *b = sm + OutChainSmem::kBuf + buf * OutChainSmem::kBufBytes;
    mbar_arrive_expect_tx(bar, 4u * (uint32_t)kImg64 + (uint32_t)(C * C * 2) + C * 4u);
    bulk_load(smem_u32(b + OutChainSmem::kW), static_cast<const uint8_t *>(p.tW) + ch * kImg64,
              kImg64, bar);
    bulk_load(smem_u32(b + OutChainSmem::kKd), static_cast<const uint8_t *>(p.tKd) + ch * kImg64,
              kImg64, bar);
    bulk_load(smem_u32(b + OutChainSmem::kUt), static_cast<const uint8_t *>(p.tUt) + ch * kImg64,
              kImg64, bar);
    bulk_load(smem_u32(b + OutChainSmem::kQg), static_cast<const uint8_t *>(p.tQg) + ch * kImg64,
              kImg64, bar);
    bulk_load(smem_u32(b + OutChainSmem::kP),
              static_cast<const uint8_t *>(p.tP) + ch * (size_t)(C * C * 2), C * C * 2, bar);
    bulk_load(smem_u32(sm + OutChainSmem::kG0 + buf * 256), p.tG + ch * C, C * 4, bar);
}

// Bounded wait of one warpgroup (named barrier `id`, 128 threads) on an mbarrier
// phase, decided by the warpgroup.
__device__ __forceinline__ bool wg_wait(uint64_t *bar, uint32_t parity, const Params &p, int id,
                                        int where) {
    const bool ok = bar_and(id, NT, mbar_wait(bar, parity, p.wait_limit));
    if (!ok && (threadIdx.x & (NT - 1)) == 0) record_timeout(p, where);
    tc_fence_after();
    return ok;
}

// Body for CTA `blk` (sequence blk / H, head blk % H): the whole sequence from h0,
// writing o and hT.
__device__ __forceinline__ void state_fwd_out_body(const Params &p, int blk) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = align1k(smem_raw);
    __shared__ uint64_t mbar, m1bar, m2bar, lbar[2], obar[2];
    __shared__ uint32_t tslot;
    if (p.hdr->status) return;
    const int H = p.H, n = blk / H, h = blk % H, tid = threadIdx.x;
    const int c0 = seq_first_at(p, n), c1 = seq_first_at(p, n + 1);
    if (tid == 0) {
        mbar_init(&mbar, 1);
        mbar_init(&m1bar, 1);
        mbar_init(&m2bar, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&lbar[b], 1);
            mbar_init(&obar[b], 1);
        }
        fence_mbar_init();
    }
    if (tid < 32) {
        tmem_alloc(&tslot, 512);
        tmem_relinquish();
    }
    // TMEM columns: 0-63 U^T, 64-191 the state update, 256 + 64 b output buffer b, 384-415
    // the U^T image (the A operand of the update and U^T P^T), and two state images (bf16
    // pairs: the A operand of U^T and S Qg^T) at 192 and 448, the one of chunk it at
    // sI(it): the update writes the next chunk's into the other
    constexpr uint32_t cUI = 384;
    auto sI = [](int it) -> uint32_t { return (it & 1) ? 448u : 192u; };
    if (tid < NT) identity_tile(sm + OutChainSmem::kI);
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tslot;
    const uint32_t id1 = idesc_bf16(128, 64, 0, 0);
    if (tid < NT) {
        // ---------------------------------------------------------- warpgroup 0: the chain
        const int v = tid;
        float S[D];
        const float *init = p.h0 ? p.h0 + ((size_t)n * H + h) * p.K * p.V : nullptr;
#pragma unroll
        for (int kk = 0; kk < D; ++kk)
            S[kk] = (init && kk < p.K && v < p.V) ? init[kk * p.V + v] : 0.f;
        tmem_store_bf16<64>(tm(tmem, sI(0)), S);  // the state entering the first chunk
        tmem_st_wait();
        uint32_t phase = 0, pend = 0, lpar = 0;
        if (c0 < c1 && v == kPrefetcher) {
            outchain_prefetch(sm, 0, (size_t)c0 * H + h, p, &lbar[0]);
            pend = 1;
        }
        const uint32_t idu = idesc_bf16(128, 64, 1, 0), id2 = idesc_bf16(128, 128, 0, 1),
                       ib = smem_u32(sm + OutChainSmem::kI);
        bool ut_in = false;  // thread 0: the chunk's Ut^T I is already in the U^T accumulator
        for (int c = c0; c < c1; ++c) {
            const int it = c - c0, buf = it & 1;
            const size_t ch = (size_t)c * H + h;
            uint8_t *b = sm + OutChainSmem::kBuf + buf * OutChainSmem::kBufBytes;
            // the previous chunk's output is complete: its U^T image (rewritten below) and
            // its prefetch slot (refilled below) are free
            bool ok = it == 0 || mbar_wait(&obar[(it - 1) & 1], ((it - 1) >> 1) & 1, p.wait_limit);
            const bool lok = ok && mbar_wait(&lbar[buf], (lpar >> buf) & 1u, p.wait_limit);
            tc_fence_before();  // (the state image written by the previous chunk's update)
            const bool all = bar_and(1, NT, lok);
            tc_fence_after();
            if (!all) {
                if (v == 0) record_timeout(p, 50);
                break;
            }
            pend &= ~(1u << buf);
            lpar ^= 1u << buf;
            if (v == kPrefetcher && c + 1 < c1) {  // (while thread 0 issues the products)
                outchain_prefetch(sm, buf ^ 1, ch + H, p, &lbar[buf ^ 1]);
                pend |= 2u >> buf;
            }
            const float gC =
                expf(reinterpret_cast<const float *>(sm + OutChainSmem::kG0 + buf * 256)[C - 1]);
            if (v == 0) {  // U^T = Ut^T I + S (-W)^T  (the W image is stored negated)
                const uint32_t wb = smem_u32(b + OutChainSmem::kW),
                               ub = smem_u32(b + OutChainSmem::kUt);
                if (!ut_in) {
#pragma unroll
                    for (int s = 0; s < C / 16; ++s)
                        mma_bf16(tmem, desc_mnmajor(ub, C, s), desc_kmajor(ib, C, s), idu, s > 0);
                }
#pragma unroll
                for (int s = 0; s < D / 16; ++s)
                    mma_bf16_ta(tmem, tmem + sI(it) + 8 * s, desc_kmajor(wb, C, s), id1, 1);
                mma_commit(&mbar);
                mbar_arrive(&m1bar);  // the state image and the slot are ready for S Qg^T
            }
            if (!wg_wait(&mbar, phase, p, 1, 51)) break;
            phase ^= 1;
#pragma unroll
            for (int c32 = 0; c32 < C; c32 += 32) {  // U^T as an operand (row v)
                float d[32];
                tmem_ld16(tm(tmem, c32), d);
                tmem_ld16(tm(tmem, c32 + 16), d + 16);
                tmem_ld_wait();
                tmem_store_bf16<16>(tm(tmem, cUI + c32 / 2), d);
            }
            tmem_st_wait();
            tc_fence_before();
            bar_sync(1, NT);
            tc_fence_after();
            if (v == 0) {
                const uint32_t kb = smem_u32(b + OutChainSmem::kKd);
#pragma unroll
                for (int s = 0; s < C / 16; ++s)  // S <- gam_n S + U^T Kd
                    mma_bf16_ta(tmem + 64, tmem + cUI + 8 * s, desc_mnmajor(kb, C, s), id2, s > 0);
                mma_commit(&mbar);
                mbar_arrive(&m2bar);  // the U^T image is ready for U^T P^T
                // the next chunk's Ut^T I into the (read) U^T accumulator while the state
                // is updated, if that chunk's copies have landed already (no wait here)
                ut_in = c + 1 < c1 && mbar_test(&lbar[buf ^ 1], (lpar >> (buf ^ 1)) & 1u);
                if (ut_in) {
                    tc_fence_after();
                    const uint32_t un = smem_u32(sm + OutChainSmem::kBuf +
                                                 (buf ^ 1) * OutChainSmem::kBufBytes + OutChainSmem::kUt);
#pragma unroll
                    for (int s = 0; s < C / 16; ++s)
                        mma_bf16(tmem, desc_mnmajor(un, C, s), desc_kmajor(ib, C, s), idu, s > 0);
                }
            }
            if (!wg_wait(&mbar, phase, p, 1, 53)) break;
            phase ^= 1;
#pragma unroll
            for (int c32 = 0; c32 < D; c32 += 32) {  // S <- gam_n S + U^T Kd
                float d[32];
                tmem_ld16(tm(tmem, 64 + c32), d);
                tmem_ld16(tm(tmem, 64 + c32 + 16), d + 16);
                tmem_ld_wait();
#pragma unroll
                for (int q = 0; q < 32; ++q) S[c32 + q] = fmaf(gC, S[c32 + q], d[q]);
            }
            // the next chunk's image: its buffer was last read by the previous chunk's
            // S Qg^T, complete with that chunk's output (obar, waited for at this step's start)
            tmem_store_bf16<64>(tm(tmem, sI(it + 1)), S);
            tmem_st_wait();
            tc_fence_before();
            bar_sync(1, NT);
            tc_fence_after();
        }
        if (v == kPrefetcher) {  // copies still in flight after an early exit
            for (int b2 = 0; b2 < 2; ++b2)
                if ((pend >> b2) & 1u) mbar_wait(&lbar[b2], (lpar >> b2) & 1u, kWaitLimit);
        }
        if (p.hT && v < p.V) {
            float *out = p.hT + ((size_t)n * H + h) * p.K * p.V;
#pragma unroll
            for (int kk = 0; kk < D; ++kk)
                if (kk < p.K) out[kk * p.V + v] = S[kk];
        }
    } else {
        // ---------------------------------------------------------- warpgroup 1: the output
        const int r = tid - NT;  // row v = r of O^T (warp 4 + w reaches TMEM lane quadrant w)
        bf16 *o = static_cast<bf16 *>(p.o);
        for (int c = c0; c < c1; ++c) {
            const int it = c - c0, buf = it & 1;
            uint8_t *b = sm + OutChainSmem::kBuf + buf * OutChainSmem::kBufBytes;
            const uint32_t ob = tmem + 256 + 64 * buf;
            bool ok = true;
            if (r == 0) {  // the leader issues the chunk's output product in two parts
                ok = mbar_wait(&m1bar, it & 1, p.wait_limit);
                if (ok) {
                    tc_fence_after();
                    const uint32_t qg = smem_u32(b + OutChainSmem::kQg);
#pragma unroll
                    for (int s = 0; s < D / 16; ++s)
                        mma_bf16_ta(ob, tmem + sI(it) + 8 * s, desc_kmajor(qg, C, s), id1, s > 0);
                    ok = mbar_wait(&m2bar, it & 1, p.wait_limit);
                }
                if (ok) {
                    tc_fence_after();
                    const uint32_t pb = smem_u32(b + OutChainSmem::kP);
#pragma unroll
                    for (int s = 0; s < C / 16; ++s)
                        mma_bf16_ta(ob, tmem + cUI + 8 * s, desc_kmajor(pb, C, s), id1, 1);
                    mma_commit(&obar[buf]);
                } else {
                    record_timeout(p, 55);
                }
            }
            // staging tile `buf` held chunk it - 2's rows: their store has read it
            if (r == 0 && it >= 2) bulk_wait_read_n<1>();
            if (!bar_and(2, NT, ok)) break;
            if (!wg_wait(&obar[buf], (it >> 1) & 1, p, 2, 54)) break;
            // thread r holds row v = r of O^T, column v of the chunk's output rows: staged
            // as token rows, then stored by the tensor engine (a full chunk) or by 16-byte
            // stores of the warpgroup (rows past the chunk's end are not written)
            uint8_t *stg = sm + OutChainSmem::kStage + buf * 16384;
            for (int c16 = 0; c16 < C; c16 += 16) {
                float d[16];
                tmem_ld16(tmq(ob, c16), d);
                tmem_ld_wait();
                uint8_t *c0p = stg + (r >> 6) * C * 128 + (r & 7) * 2;
                const int cp = (r & 63) >> 3;
#pragma unroll
                for (int q = 0; q < 16; ++q)  // row c16 + q, whose swizzle term is q % 8
                    *reinterpret_cast<bf16 *>(c0p + (c16 + q) * 128 + ((cp ^ (q & 7)) << 4)) =
                        __float2bfloat16_rn(d[q]);
            }
            fence_async_smem();
            tc_fence_before();  // (buffer `buf` is read: the next barrier orders its reuse)
            bar_sync(2, NT);
            const ChunkInfo ci = chunk_in_seq(p, n, c0, c);
            if (ci.len == C) {
                if (r == 0) {
                    tma_store_3d(&p.tm_o, 0, h, (int)ci.tok0, smem_u32(stg));
                    if (p.V == D) tma_store_3d(&p.tm_o, 64, h, (int)ci.tok0, smem_u32(stg) + C * 128);
                    bulk_commit();
                }
            } else {
                for (int t = r; t < C * 16; t += NT) {
                    const int i = t >> 4, j = t & 15;
                    if (i < ci.len && j * 8 < p.V)
                        *reinterpret_cast<uint4 *>(o + ((int64_t)(ci.tok0 + i) * H + h) * p.V + j * 8) =
                            *reinterpret_cast<const uint4 *>(stg + sw128_chunk(C, i, j));
                }
                bar_sync(2, NT);  // the staging rows are read before the tile is rewritten
            }
        }
        if (r == 0) bulk_wait_all();  // (the stores read the staging tiles)
    }
    tc_fence_before();
    __syncthreads();
    if (tid < 32) tmem_dealloc(tmem, 512);
}

// ============================================================ chain by value slices
// The value columns of the state evolve independently given a chunk's W, Kd,
// gates and their own columns of Ut (rows of S = H^T do not mix), so a chain
// can be split over CTAs by value columns.  chain_fwd_sliced runs the columns
// [v0, v0 + 64) of one (sequence, head) in a CTA of its own, in the
// untransposed form: thread k owns row k of H_s = H[:, v0:v0+64] (64 fp32
// registers, half of chain_fwd's) and per chunk
//
//   U_s = Ut_s - W H_s          (M = 64 tokens, N = 64 values, K = 128 keys)
//   H_s <- gam_n H_s + Kd^T U_s  (M = 128 keys, N = 64 values, K = 64 tokens)
//
// With snapshots it writes the state entering each chunk as block `slice` of a
// 128 x 128 SW128 tile of H (rows = keys) and U_s as block `slice` of a
// 64 x 128 tile of U (rows = tokens): the layouts tc_out reads.
struct SliceSmem {
    static constexpr int kH = 0, kU = kH + 16384, kI = kU + 8192, kW0 = kI + 8192,
                         kKd0 = kW0 + 2 * 16384, kUt0 = kKd0 + 2 * 16384, kG0 = kUt0 + 2 * 8192,
                         kEnd = kG0 + 2 * 256;
};
constexpr int kSliceSmem = SliceSmem::kEnd + 1024;

// Bulk copies (thread 0) of chunk ch's W and Kd images, column block `sl` of
// its Ut image (unless the run takes Ut as zero) and its gate row into buffer
// `buf`, completing on `bar`.
__device__ __forceinline__ void slice_prefetch(uint8_t *sm, int buf, size_t ch, int sl,
                                               const Params &p, bool with_ut, uint64_t *bar) {
    if (threadIdx.x != 0) return;
    mbar_arrive_expect_tx(bar, 2u * (uint32_t)kImg64 + (with_ut ? 8192u : 0u) + C * 4u);
    bulk_load(smem_u32(sm + SliceSmem::kW0 + buf * 16384),
              static_cast<const uint8_t *>(p.tW) + ch * kImg64, kImg64, bar);
    bulk_load(smem_u32(sm + SliceSmem::kKd0 + buf * 16384),
              static_cast<const uint8_t *>(p.tKd) + ch * kImg64, kImg64, bar);
    if (with_ut)
        bulk_load(smem_u32(sm + SliceSmem::kUt0 + buf * 8192),
                  static_cast<const uint8_t *>(p.tUt) + ch * kImg64 + sl * 8192, 8192, bar);
    bulk_load(smem_u32(sm + SliceSmem::kG0 + buf * 256), p.tG + ch * C, C * 4, bar);
}

__device__ __forceinline__ void chain_fwd_sliced(const Params &p, const ChainFwd &a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = align1k(smem_raw);
    __shared__ uint64_t mbar, lbar[2];
    __shared__ uint32_t tslot;
    if (p.hdr->status) return;
    const int H = p.H, h = a.h, k = threadIdx.x, sl = a.slice, v0 = 64 * sl;
    float S[64];  // row k of H_s
    if (a.init) {
        const int ik = a.init_user ? p.K : D, iv = a.init_user ? p.V : D;
#pragma unroll
        for (int j = 0; j < 64; ++j)
            S[j] = (k < ik && v0 + j < iv) ? a.init[(size_t)k * iv + v0 + j] : 0.f;
    } else {
#pragma unroll
        for (int j = 0; j < 64; ++j) S[j] = (a.init_identity && k == v0 + j) ? 1.f : 0.f;
    }
    if (k == 0) {
        mbar_init(&mbar, 1);
        mbar_init(&lbar[0], 1);
        mbar_init(&lbar[1], 1);
        fence_mbar_init();
    }
    if (k < 32) {
        tmem_alloc(&tslot, 64);
        tmem_relinquish();
    }
    identity_tile(sm + SliceSmem::kI);
    tc_fence_before();
    fence_async_smem();
    __syncthreads();
    tc_fence_after();
    // 64 TMEM columns: the first product (M = 64) is read out before the second
    // (M = 128) overwrites the same columns
    const uint32_t tmem = tslot;
    const int c0 = a.c0, c1 = a.c1;
    const bool with_ut = !a.zero_ut;
    uint32_t phase = 0, pend = 0, lpar = 0;  // per buffer b (bit b): copy in flight, parity
    if (c0 < c1) {
        slice_prefetch(sm, 0, (size_t)c0 * H + h, sl, p, with_ut, &lbar[0]);
        pend = 1;
    }
    uint8_t *Hs = sm + SliceSmem::kH, *Us = sm + SliceSmem::kU;
    const uint32_t hb = smem_u32(Hs), ub = smem_u32(Us);
    const uint32_t id1 = idesc_bf16(64, 64, 0, 1), id2 = idesc_bf16(128, 64, 1, 1);
    for (int c = c0; c < c1; ++c) {
        const int buf = (c - c0) & 1;
        const size_t ch = (size_t)c * H + h;
        if (c + 1 < c1) {
            slice_prefetch(sm, buf ^ 1, ch + H, sl, p, with_ut, &lbar[buf ^ 1]);
            pend |= 2u >> buf;
        }
        const bool lok = mbar_wait(&lbar[buf], (lpar >> buf) & 1u, p.wait_limit);
        // the state entering this chunk: row k of the H_s operand tile (128 bytes)
#pragma unroll
        for (int j = 0; j < 8; ++j)
            *reinterpret_cast<uint4 *>(Hs + sw128_chunk(D, k, j)) = pack8(S + 8 * j);
        fence_async_smem();
        tc_fence_before();
        const bool all = __syncthreads_and(lok);
        tc_fence_after();
        if (!all) {
            if (k == 0) record_timeout(p, 40 + a.where);
            break;
        }
        pend &= ~(1u << buf);
        lpar ^= 1u << buf;
        const float gC =
            expf(reinterpret_cast<const float *>(sm + SliceSmem::kG0 + buf * 256)[C - 1]);
        if (k == 0) {  // U_s = -W H_s + I Ut_s (the W image is stored negated)
            const uint32_t wb = smem_u32(sm + SliceSmem::kW0 + buf * 16384),
                           utb = smem_u32(sm + SliceSmem::kUt0 + buf * 8192),
                           ib = smem_u32(sm + SliceSmem::kI);
#pragma unroll
            for (int s = 0; s < D / 16; ++s)
                mma_bf16(tmem, desc_kmajor(wb, C, s), desc_mnmajor(hb, D, s), id1, s > 0);
            if (with_ut) {
#pragma unroll
                for (int s = 0; s < C / 16; ++s)
                    mma_bf16(tmem, desc_kmajor(ib, C, s), desc_mnmajor(utb, C, s), id1, 1);
            }
            mma_commit(&mbar);
            if (a.snapshots) {
                bulk_store(static_cast<uint8_t *>(p.tS) + ch * kImg128 + sl * 16384, hb, 16384u);
                bulk_commit();
            }
        }
        if (!cta_wait(&mbar, phase, p, a.where)) break;
        phase ^= 1;
        {  // U_s as an operand tile: row i on the M = 64 lanes
            const int i = m64_row();
            float d[64];
#pragma unroll
            for (int q = 0; q < 4; ++q) tmem_ld16(tm(tmem, 16 * q), d + 16 * q);
            tmem_ld_wait();
            if (i >= 0) {
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    *reinterpret_cast<uint4 *>(Us + sw128_chunk(C, i, j)) = pack8(d + 8 * j);
            }
        }
        operands_ready();  // (also orders the TMEM reads above before the product below)
        if (k == 0) {  // Kd^T U_s
            const uint32_t kb = smem_u32(sm + SliceSmem::kKd0 + buf * 16384);
#pragma unroll
            for (int s = 0; s < C / 16; ++s)
                mma_bf16(tmem, desc_mnmajor(kb, C, s), desc_mnmajor(ub, C, s), id2, s > 0);
            mma_commit(&mbar);
            if (a.snapshots) {
                bulk_store(static_cast<uint8_t *>(p.tUT) + ch * kImgUT + sl * 8192, ub, 8192u);
                bulk_commit();
            }
        }
        if (!cta_wait(&mbar, phase, p, a.where + 1)) break;
        phase ^= 1;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            float d[16];
            tmem_ld16(tm(tmem, 16 * q), d);
            tmem_ld_wait();
#pragma unroll
            for (int x = 0; x < 16; ++x) S[16 * q + x] = fmaf(gC, S[16 * q + x], d[x]);
        }
        // the operand tiles are rewritten next chunk: their bulk stores must have read them
        if (k == 0 && a.snapshots) bulk_wait_read();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }
    if (k == 0) {  // copies still in flight after an early exit
        for (int b = 0; b < 2; ++b)
            if ((pend >> b) & 1u) mbar_wait(&lbar[b], (lpar >> b) & 1u, kWaitLimit);
        if (a.snapshots) bulk_wait_all();
    }
    if (a.final_out) {
        const int ok = a.out_user ? p.K : D, ov = a.out_user ? p.V : D;
        if (k < ok) {
#pragma unroll
            for (int j = 0; j < 64; ++j)
                if (v0 + j < ov) a.final_out[(size_t)k * ov + v0 + j] = S[j];
        }
    }
    tc_fence_before();
    __syncthreads();
    if (k < 32) tmem_dealloc(tmem, 64);
}

// Body of the forward state pass for CTA `blk` (sequence blk / H, head blk % H):
// the whole sequence from h0, writing the per-chunk snapshots and hT.
__device__ __forceinline__ void state_fwd_body(const Params &p, int blk) {
    const int H = p.H, n = blk / H, h = blk % H;
    ChainFwd a;
    a.h = h;
    a.c0 = seq_first_at(p, n);
    a.c1 = seq_first_at(p, n + 1);
    a.init = p.h0 ? p.h0 + ((size_t)n * H + h) * p.K * p.V : nullptr;
    a.init_user = 1;
    a.init_identity = 0;
    a.zero_ut = 0;
    a.snapshots = 1;
    a.final_out = p.hT ? p.hT + ((size_t)n * H + h) * p.K * p.V : nullptr;
    a.out_user = 1;
    a.where = 3;
    a.slice = 0;
    chain_fwd(p, a);
}

// Value slices of the forward chain's rows (64 value columns each).
__device__ __forceinline__ int value_slices(const Params &p) { return (p.V + 63) / 64; }

// The forward pass's state chain by value slices: CTA `blk` runs slice
// blk % value_slices of (sequence, head) blk / value_slices, the whole sequence
// from h0, writing the H and U snapshots tc_out reads and its columns of hT.
__device__ __forceinline__ void state_fwd_sliced_body(const Params &p, int blk) {
    const int nsl = value_slices(p), unit = blk / nsl, H = p.H, n = unit / H, h = unit % H;
    ChainFwd a;
    a.h = h;
    a.slice = blk % nsl;
    a.c0 = seq_first_at(p, n);
    a.c1 = seq_first_at(p, n + 1);
    a.init = p.h0 ? p.h0 + ((size_t)n * H + h) * p.K * p.V : nullptr;
    a.init_user = 1;
    a.init_identity = 0;
    a.zero_ut = 0;
    a.snapshots = 1;
    a.final_out = p.hT ? p.hT + ((size_t)n * H + h) * p.K * p.V : nullptr;
    a.out_user = 1;
    a.where = 3;
    chain_fwd_sliced(p, a);
}

// ============================================================ piece scan roles
constexpr int kScanSmem = 65536 + 1024;  // the scan's state and transition operand images

// The exact piece scan of long dense rows: each chunk maps the state affinely,
// H' = M_c H + B_c, so a row split into P pieces of p.L chunks is joined by
// composing every piece's (transition, offset) pair.

// Chunks [c0, c1) of piece `piece` of dense row n (pieces of p.L chunks; the
// last may be shorter or empty).
__device__ __forceinline__ void piece_range(const Params &p, int n, int piece, int *c0, int *c1) {
    const int end = seq_first_at(p, n + 1);
    int a = seq_first_at(p, n) + piece * p.L;
    a = a < end ? a : end;
    const int b = a + p.L < end ? a + p.L : end;
    *c0 = a;
    *c1 = b;
}

// Forward phase A, role r of (row, head) unit `unit`: r = 0 runs piece 0 from
// h0 with snapshots (its final state enters piece 1: tHin[1]); odd r runs middle
// piece (r + 1) / 2 from zero (-> its offset B, tBp); even r >= 2 runs middle
// piece r / 2 from the identity with Ut taken as zero (-> its transition M, tMp).
__device__ __forceinline__ void piece_a_fwd_role(const Params &p, int unit, int r, int slice) {
    const int n = unit / p.H, h = unit % p.H;
    const size_t u = (size_t)unit * p.P, DD = (size_t)D * D;
    ChainFwd a;
    a.h = h;
    a.slice = slice;
    a.where = 31;
    a.init_user = 1;  // h0 (piece 0); the middle pieces start from zero or the identity
    a.out_user = 0;   // tHin, tBp, tMp are internal [128][128] blocks
    int piece;
    if (r == 0) {
        piece = 0;
        a.init = p.h0 ? p.h0 + (size_t)unit * DD : nullptr;
        a.init_identity = 0;
        a.zero_ut = 0;
        a.snapshots = 1;
        a.final_out = p.tHin + (u + 1) * DD;
    } else if (r & 1) {
        piece = (r + 1) / 2;
        a.init = nullptr;
        a.init_identity = 0;
        a.zero_ut = 0;
        a.snapshots = 0;
        a.final_out = p.tBp + (u + piece) * DD;
    } else {
        piece = r / 2;
        a.init = nullptr;
        a.init_identity = 1;
        a.zero_ut = 1;
        a.snapshots = 0;
        a.final_out = p.tMp + (u + piece) * DD;
    }
    piece_range(p, n, piece, &a.c0, &a.c1);
    if (p.vslice) chain_fwd_sliced(p, a);
    else chain_fwd(p, a);
}

// Forward phase C: piece `piece` >= 1 of unit `unit` reruns its chain from its
// entering state (tHin) with snapshots; the last piece writes hT (if given).
__device__ __forceinline__ void piece_c_fwd_role(const Params &p, int unit, int piece, int slice) {
    const int n = unit / p.H, h = unit % p.H;
    const size_t DD = (size_t)D * D;
    ChainFwd a;
    a.h = h;
    a.slice = slice;
    a.where = 35;
    a.init_user = 0;  // tHin
    a.out_user = 1;   // hT
    a.init = p.tHin + ((size_t)unit * p.P + piece) * DD;
    a.init_identity = 0;
    a.zero_ut = 0;
    a.snapshots = 1;
    a.final_out = (piece == p.P - 1 && p.hT) ? p.hT + (size_t)unit * DD : nullptr;
    piece_range(p, n, piece, &a.c0, &a.c1);
    if (p.vslice) chain_fwd_sliced(p, a);
    else chain_fwd(p, a);
}

// Phase B for unit `unit`: X[q] = X[q - dir] * T[q - dir] + B[q - dir] for q from
// q_first to q_last in steps of dir (+1 for the forward, -1 for the reverse
// chain), one tensor-core product per piece.  X, T, B are [P][128][128] fp32
// blocks per unit with element [k][v]; in S form (thread v owns row v of S = X^T)
// the step is S <- S T^T + B^T, the transition read as a K-major operand with rows
// k.  (For the reverse chain the blocks hold dS^T from a run started at dS = I,
// and the step dS <- dS T + B reads them the same way.)
__device__ __forceinline__ void piece_scan_body(const Params &p, int unit, float *X, const float *T,
                                                const float *Bq, int q_first, int q_last, int dir,
                                                int where) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = align1k(smem_raw);
    __shared__ uint64_t mbar;
    __shared__ uint32_t tslot;
    if (p.hdr->status) return;
    const int v = threadIdx.x;
    const size_t u = (size_t)unit * p.P, DD = (size_t)D * D;
    uint8_t *Ss = sm, *Mt = sm + 32768;
    float S[D];
    const float *x0 = X + (u + q_first - dir) * DD;
#pragma unroll
    for (int kk = 0; kk < D; ++kk) S[kk] = x0[kk * D + v];
    if (v == 0) {
        mbar_init(&mbar, 1);
        fence_mbar_init();
    }
    if (v < 32) {
        tmem_alloc(&tslot, 128);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tslot, id = idesc_bf16(128, 128, 0, 0);
    uint32_t phase = 0;
    for (int q = q_first; dir > 0 ? q <= q_last : q >= q_last; q += dir) {
        const float *M = T + (u + q - dir) * DD, *Bm = Bq + (u + q - dir) * DD;
        for (int t = v; t < D * 16; t += NT) {  // the transition as a K-major operand: rows k
            const int r = t >> 4, j8 = t & 15;
            const float4 a0 = *reinterpret_cast<const float4 *>(M + r * D + j8 * 8);
            const float4 a1 = *reinterpret_cast<const float4 *>(M + r * D + j8 * 8 + 4);
            const float f[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            *reinterpret_cast<uint4 *>(Mt + sw128_chunk(D, r, j8)) = pack8(f);
        }
        state_image(Ss, S, v);
        operands_ready();
        if (v == 0) {
            const uint32_t sb = smem_u32(Ss), mb = smem_u32(Mt);
#pragma unroll
            for (int s = 0; s < D / 16; ++s)
                mma_bf16(tmem, desc_kmajor(sb, D, s), desc_kmajor(mb, D, s), id, s > 0);
            mma_commit(&mbar);
        }
        if (!cta_wait(&mbar, phase, p, where)) break;
        phase ^= 1;
        float *xq = X + (u + q) * DD;
#pragma unroll
        for (int c32 = 0; c32 < D; c32 += 32) {
            float d[32];
            tmem_ld16(tm(tmem, c32), d);
            tmem_ld16(tm(tmem, c32 + 16), d + 16);
            tmem_ld_wait();
#pragma unroll
            for (int x = 0; x < 32; ++x) {
                S[c32 + x] = d[x] + Bm[(c32 + x) * D + v];
                xq[(c32 + x) * D + v] = S[c32 + x];
            }
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }
    tc_fence_before();
    __syncthreads();
    if (v < 32) tmem_dealloc(tmem, 128);
}

}  // namespace tc
}  // namespace gdn
