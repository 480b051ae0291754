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
    static constexpr int kS = 0, kUT = kS + 32768, kW0 = kUT + 16384, kKd0 = kW0 + 2 * 16384,
                         kUt0 = kKd0 + 2 * 16384, kG0 = kUt0 + 2 * 16384, kEnd = kG0 + 2 * 256;
};
constexpr int kStateSmem = StateSmem::kEnd + 1024;

// Bulk copies (thread 0) of chunk ch's W and Kd images, its Ut rows (unless
// the run takes Ut as zero) and its gate row into buffer `buf`, completing
// on `bar`.
__device__ __forceinline__ void state_prefetch(uint8_t *sm, int buf, size_t ch, const Params &p,
                                               bool with_ut, uint64_t *bar) {
    if (threadIdx.x != 0) return;
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
};

// The forward state chain: thread v owns row v of S = H^T (fp32 registers).
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
        tmem_alloc(&tslot, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tslot;
    const int c0 = a.c0, c1 = a.c1;
    const bool with_ut = !a.zero_ut;
    uint32_t phase = 0;
    // per buffer b (bit b): a copy in flight, and the parity of its next completion
    uint32_t pend = 0, lpar = 0;
    if (c0 < c1) {
        state_prefetch(sm, 0, (size_t)c0 * H + h, p, with_ut, &lbar[0]);
        pend = 1;
    }
    uint8_t *Ss = sm + StateSmem::kS, *UTs = sm + StateSmem::kUT;
    const uint32_t id1 = idesc_bf16(128, 64, 0, 0), id2 = idesc_bf16(128, 128, 0, 1);
    for (int c = c0; c < c1; ++c) {
        const int buf = (c - c0) & 1;
        const size_t ch = (size_t)c * H + h;
        if (c + 1 < c1) {
            state_prefetch(sm, buf ^ 1, ch + H, p, with_ut, &lbar[buf ^ 1]);
            pend |= 2u >> buf;
        }
        const bool lok = mbar_wait(&lbar[buf], (lpar >> buf) & 1u, p.wait_limit);
        // the state entering this chunk, as bf16 operand rows
#pragma unroll
        for (int j = 0; j < 16; ++j)
            *reinterpret_cast<uint4 *>(Ss + sw128_chunk(D, v, j)) = pack8(S + 8 * j);
        fence_async_smem();
        tc_fence_before();
        const bool all = __syncthreads_and(lok);
        tc_fence_after();
        if (!all) {
            if (v == 0) record_timeout(p, 40 + a.where);
            break;
        }
        pend &= ~(1u << buf);
        lpar ^= 1u << buf;
        const float gC =
            expf(reinterpret_cast<const float *>(sm + StateSmem::kG0 + buf * 256)[C - 1]);
        if (v == 0) {
            const uint32_t sb = smem_u32(Ss), wb = smem_u32(sm + StateSmem::kW0 + buf * 16384);
#pragma unroll
            for (int s = 0; s < D / 16; ++s)
                mma_bf16(tmem, desc_kmajor(sb, D, s), desc_kmajor(wb, C, s), id1, s > 0);
            mma_commit(&mbar);
            if (a.snapshots) {
                bulk_store(static_cast<uint8_t *>(p.tS) + ch * kImg128, sb, (uint32_t)kImg128);
                bulk_commit();
            }
        }
        if (!cta_wait(&mbar, phase, p, a.where)) break;
        phase ^= 1;
        // U^T[v][i] = Ut[i][v] - (S W^T)[v][i]
        const bf16 *Ut = reinterpret_cast<const bf16 *>(sm + StateSmem::kUt0 + buf * 16384);
#pragma unroll
        for (int c32 = 0; c32 < C; c32 += 32) {
            float d[32];
            tmem_ld16(tm(tmem, c32), d);
            tmem_ld16(tm(tmem, c32 + 16), d + 16);
            tmem_ld_wait();
#pragma unroll
            for (int q = 0; q < 32; ++q)
                d[q] = (with_ut ? __bfloat162float(Ut[(c32 + q) * D + v]) : 0.f) + d[q];
#pragma unroll
            for (int q = 0; q < 4; ++q)
                *reinterpret_cast<uint4 *>(UTs + sw128_chunk(D, v, c32 / 8 + q)) = pack8(d + 8 * q);
        }
        operands_ready();
        if (v == 0) {
            const uint32_t ub = smem_u32(UTs), kb = smem_u32(sm + StateSmem::kKd0 + buf * 16384);
#pragma unroll
            for (int s = 0; s < C / 16; ++s)
                mma_bf16(tmem + 64, desc_kmajor(ub, D, s), desc_mnmajor(kb, C, s), id2, s > 0);
            mma_commit(&mbar);
            if (a.snapshots) {
                bulk_store(static_cast<uint8_t *>(p.tUT) + ch * kImgUT, ub, (uint32_t)kImgUT);
                bulk_commit();
            }
        }
        if (!cta_wait(&mbar, phase, p, a.where + 1)) break;
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
        // shared operands are rewritten next chunk: their bulk stores must have read them
        if (v == 0 && a.snapshots) bulk_wait_read();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }
    if (v == 0) {  // copies still in flight after an early exit
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
    if (v < 32) tmem_dealloc(tmem, 256);
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
    chain_fwd(p, a);
}

}  // namespace tc
}  // namespace gdn
