// Per-chunk preparation step of the tensor-core path (shared by the forward
// launch and by the backward, where it shares a launch with tc_local).
#pragma once

#include "tc_common.cuh"

namespace gdn {
namespace tc {

// ============================================================ tc_prep
// Per (chunk, head): gates, A = (I + L)^-1 (fp32, by 16 x 16 blocks), and the
// tile images W, Kd and Ut that the state chains consume, and the images of
// Qg = scale diag(gam) Q and P = scale lower(Q K^T . Gam) that the output and
// the reverse chain consume.  One M = 128 product [Q; K] K^T gives Q K^T on
// lanes 0-63 and K K^T on lanes 64-127, so P (threads 0-63) and L (threads
// 64-127) are built in the same phase.
constexpr int LS = 68;  // row stride (floats) of L: 16-byte aligned rows for vector loads

struct PrepSmem {
    // [Q; K] rows as one 128-row tile (Q rows 0-63, K rows 64-127); once Q is
    // consumed, the V rows are loaded into its place.  L (fp32 64 x 68) becomes A
    // in place; once A is read out, its bytes hold the two bf16 operand tiles
    // A diag(b gam) and A diag(b).  F: per-column decay factors exp(G_e - G_j) to
    // the end e of column j's 16-block; E: exp(G_j); EK: exp(G_n - G_j), n the
    // chunk's last token.
    static constexpr int kQK = 0, kL = kQK + 32768, kAb = kL, kAc = kL + 8192,
                         kG = kL + C * LS * 4, kB = kG + 256, kF = kB + 256, kE = kF + 256,
                         kEK = kE + 256, kEnd = kEK + 256;
};
constexpr int kPrepSmem = PrepSmem::kEnd + 1024 + 48;
constexpr int kPrepSmemRequest = 52 * 1024;  // four CTAs per SM (TMEM: 128 columns each)

// acc += a x (four columns)
__device__ __forceinline__ void fma4(float4 &acc, float a, const float4 x) {
    acc.x = fmaf(a, x.x, acc.x);
    acc.y = fmaf(a, x.y, acc.y);
    acc.z = fmaf(a, x.z, acc.z);
    acc.w = fmaf(a, x.w, acc.w);
}

// Byte offset, in a [Q; K] tile of 128 rows, of byte `off` of a 64-row tile image
// (block off / 8192, row and chunk position within it) taken from rows
// [row0, row0 + 64): the swizzle depends on the row only through row % 8.
__device__ __forceinline__ uint32_t qk_src(int off, int row0) {
    return (uint32_t)((off >> 13) * 16384 + row0 * 128 + (off & 8191));
}

// Byte offset, in the [Q; K] tile of 128 rows, of chunk j (0-15) of row i of a 64-row
// tile image staged in rows [row0, row0 + 64): 64-column block j / 8 of the image
// lies in the tile's block j / 8, so each block leaves by one contiguous copy.
__device__ __forceinline__ uint32_t qk_stage(int row0, int j, int i) {
    return (uint32_t)((j >> 3) * 2 * C * 128 + (row0 + i) * 128 + (((j & 7) ^ (i & 7)) << 4));
}

// Body of the prep step for CTA `ch` (chunk ch / H, head ch % H).
__device__ __forceinline__ void prep_body(const Params &p, int ch, int want_A) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = align1k(smem_raw);
    __shared__ uint64_t mbar, lbar, vbar;
    __shared__ uint32_t tslot;
    if (p.hdr->status) return;
    const int H = p.H, c = ch / H, h = ch % H;
    const ChunkInfo ci = chunk_at(p, c);
    uint8_t *QK = sm + PrepSmem::kQK;
    uint8_t *Ab = sm + PrepSmem::kAb, *Ac = sm + PrepSmem::kAc;
    float *L = reinterpret_cast<float *>(sm + PrepSmem::kL);
    float *G = reinterpret_cast<float *>(sm + PrepSmem::kG);
    float *bta = reinterpret_cast<float *>(sm + PrepSmem::kB);
    float *F = reinterpret_cast<float *>(sm + PrepSmem::kF);
    float *E = reinterpret_cast<float *>(sm + PrepSmem::kE);
    float *EK = reinterpret_cast<float *>(sm + PrepSmem::kEK);
    const int tid = threadIdx.x;
    const uint32_t qkb = smem_u32(QK), kb = qkb + C * 128;  // K rows: 64-127 of the tile

    // warp 3 sets up (the mbarriers, the Q and K copies, TMEM) while warps 0-1 load the
    // gates, the first global reads of the CTA
    if (tid == 3 * 32) {  // Q and K rows by the tensor engine (V comes once Q is consumed)
        mbar_init(&mbar, 1);
        mbar_init(&lbar, 1);
        mbar_init(&vbar, 1);
        fence_mbar_init();
        // (the planted stall of the tests: 16 bytes more than the copies bring, on the
        // first (chunk, head) only, so its bounded wait runs out after they have landed)
        const uint32_t planted = (p.test_hook == GDN_TEST_STALL_COPY && ch == 0) ? 16u : 0u;
        mbar_arrive_expect_tx(&lbar, 2 * row_tile_bytes(p.K) + planted);
        load_rows_tma(QK, D, 0, &p.tm_q, ci.tok0, h, p.K, &lbar);
        load_rows_tma(QK, D, C, &p.tm_k, ci.tok0, h, p.K, &lbar);
    }
    if (tid >= 3 * 32) {
        tmem_alloc(&tslot, 128);
        tmem_relinquish();
    }
    chunk_gates(G, bta, p, ci, h);  // its barriers also publish the mbarrier inits
    if (tid < C) {  // the decay factors, once (published by the barrier of the wait below)
        F[tid] = __expf(G[tid | 15] - G[tid]);
        E[tid] = __expf(G[tid]);
        EK[tid] = __expf(G[C - 1] - G[tid]);
    }
    bool ok = copies_arrived(&lbar, p, 31);
    if (ok) {
        fix_rows(QK, D, 0, ci.len, p.K);
        fix_rows(QK, D, C, ci.len, p.K);
    }
    operands_ready();
    if (ok && p.l2norm) {  // q and k rows divided by their norms
        l2norm_tile_rows(QK, D, 0, nullptr);
        l2norm_tile_rows(QK, D, C, nullptr);
        operands_ready();
    }
    const uint32_t tmem = tslot;
    uint32_t phase = 0;
    bool v_pending = false;  // the V copy is in flight and not yet waited for

    // [Q; K] K^T (M = 128 rows: Q K^T on lanes 0-63, K K^T on lanes 64-127; N = 64; K = 128)
    if (ok && tid == 0) {
        const uint32_t id = idesc_bf16(128, 64, 0, 0);
#pragma unroll
        for (int s = 0; s < D / 16; ++s)
            mma_bf16(tmem, desc_kmajor(qkb, D, s), desc_kmajor(kb, D, s), id, s > 0);
        mma_commit(&mbar);
    }
    // meanwhile: the Kd = diag(e) K and Qg = scale diag(gam) Q images, G and b
    if (ok) {
        uint8_t *kd = static_cast<uint8_t *>(p.tKd) + (size_t)ch * kImg64;
        uint8_t *qg = static_cast<uint8_t *>(p.tQg) + (size_t)ch * kImg64;
        for (int t = tid; t < C * 16; t += NT) {
            const int off = t * 16, r = (off & 8191) >> 7;
            float f[8], g[8];
            unpack8(*reinterpret_cast<const uint4 *>(QK + qk_src(off, C)), f);
            unpack8(*reinterpret_cast<const uint4 *>(QK + qk_src(off, 0)), g);
            const float e = EK[r], gq = p.scale * E[r];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                f[i] *= e;
                g[i] *= gq;
            }
            *reinterpret_cast<uint4 *>(kd + off) = pack8(f);
            *reinterpret_cast<uint4 *>(qg + off) = pack8(g);
        }
        if (tid < C) {
            p.tG[(size_t)ch * C + tid] = G[tid];
            if (p.tB) p.tB[(size_t)ch * C + tid] = bta[tid];
        }
    }
    if (ok) ok = cta_wait(&mbar, phase, p, 1);
    phase ^= 1;
    if (ok && tid == 0) {  // Q is consumed (the product and the Qg image): V rows in its place
        fence_async_smem();
        mbar_arrive_expect_tx(&vbar, row_tile_bytes(p.V));
        load_rows_tma(QK, D, 0, &p.tm_v, ci.tok0, h, p.V, &vbar);
    }
    v_pending = ok;
    if (ok) {
        // Rows of the [Q; K] K^T accumulator (M = 128: row = lane = thread).  Threads 0-63:
        // P = scale lower(Q K^T . Gam), diagonal included, as a 64 x 64 tile image.
        // Threads 64-127: L = strict_lower(diag(b) K K^T . Gam) into shared memory (fp32).
        // The 16 rows of a half-warp lie in one 16-block, so the cases are warp-uniform.
        // Gam_ij = exp(G_i - G_e) exp(G_e - G_j) below a row's diagonal block (e = the
        // block's last column, both factors <= 1), directly inside it (the fast
        // exponential: its relative error, a few units in the last place of fp32,
        // is far below the bf16 rounding every product operand gets).
        float d[4][16];
#pragma unroll
        for (int cb = 0; cb < 4; ++cb) tmem_ld16(tm(tmem, 16 * cb), d[cb]);
        tmem_ld_wait();
        const bool lrow = tid >= C;
        const int i = lrow ? tid - C : tid, ib = i >> 4;
        const float ci0 = lrow ? bta[i] : p.scale;
        uint8_t *Pimg = static_cast<uint8_t *>(p.tP) + (size_t)ch * (C * C * 2);
        float *Li = L + i * LS;
#pragma unroll
        for (int cb = 0; cb < 4; ++cb) {
            const int c0 = 16 * cb;
            float x[16];
            if (cb < ib) {
                const float ri = ci0 * __expf(G[i] - G[c0 + 15]);
#pragma unroll
                for (int q = 0; q < 16; ++q) x[q] = ri * F[c0 + q] * d[cb][q];
            } else if (cb == ib) {
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    const int j = c0 + q;
                    x[q] = (lrow ? j < i : j <= i) ? ci0 * __expf(G[i] - G[j]) * d[cb][q] : 0.f;
                }
            } else {
#pragma unroll
                for (int q = 0; q < 16; ++q) x[q] = 0.f;
            }
            if (lrow) {
#pragma unroll
                for (int q = 0; q < 16; q += 4)
                    *reinterpret_cast<float4 *>(Li + c0 + q) =
                        make_float4(x[q], x[q + 1], x[q + 2], x[q + 3]);
            } else {
                *reinterpret_cast<uint4 *>(Pimg + sw128_chunk(C, i, 2 * cb)) = pack8(x);
                *reinterpret_cast<uint4 *>(Pimg + sw128_chunk(C, i, 2 * cb + 1)) = pack8(x + 8);
            }
        }
        tc_fence_before();
        __syncthreads();
        // A = (I + L)^-1 in fp32 by 16 x 16 blocks, in place over L (stride LS):
        // the diagonal blocks by forward substitution (one thread per column), then
        // row block by row block  A_ij = -A_ii sum_{k=j}^{i-1} L_ik A_kj  (j < i),
        // each row block's products formed in registers before any of its L blocks
        // is overwritten.  Blocks above the diagonal stay zero.
        {
            float a[16];
            const int b = tid >> 4, jj = tid & 15;
            if (tid < C) {
                const float *Lb = L + 16 * b * LS + 16 * b;
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    float s0 = 0.f, s1 = 0.f;
#pragma unroll
                    for (int m = 0; m < r; m += 4) {
                        const float4 l4 = *reinterpret_cast<const float4 *>(Lb + r * LS + m);
                        s0 = fmaf(l4.x, a[m], s0);
                        if (m + 1 < r) s1 = fmaf(l4.y, a[m + 1], s1);
                        if (m + 2 < r) s0 = fmaf(l4.z, a[m + 2], s0);
                        if (m + 3 < r) s1 = fmaf(l4.w, a[m + 3], s1);
                    }
                    a[r] = r < jj ? 0.f : (r == jj ? 1.f : -(s0 + s1));
                }
            }
            __syncthreads();
            if (tid < C) {
                float *Lb = L + 16 * b * LS + 16 * b;
#pragma unroll
                for (int r = 0; r < 16; ++r) Lb[r * LS + jj] = a[r];
            }
            __syncthreads();
        }
        // Row blocks ib = 1..3: unit u of row block ib is block j = u / 64, row
        // r = (u / 4) % 16, columns c4 .. c4 + 3 (c4 = 4 (u % 4)); thread t takes unit t
        // and, for ib = 3, threads 64-127 also unit t + 64 (block j = 2, the shortest
        // sum).  A thread forms its four columns from float4 rows (the 32 units of a warp
        // share j, so the k loop bound is uniform; rows r of stride LS = 68 floats fall
        // in distinct banks).
#pragma unroll
        for (int ib = 1; ib < 4; ++ib) {
            float4 t[2];
#pragma unroll
            for (int n = 0; n < 2; ++n) {  // T_ij = sum_{k=j}^{ib-1} L_ik A_kj
                const int u = tid + 64 * n, j = u >> 6, r = (u >> 2) & 15, c4 = (u & 3) * 4;
                if (u >= 64 * ib || (n && tid < 64)) continue;
                const float *Lr = L + (16 * ib + r) * LS;
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
                for (int k = j; k < ib; ++k) {
                    const float *Ak = L + (16 * k) * LS + 16 * j + c4;
#pragma unroll
                    for (int m = 0; m < 16; m += 4) {
                        const float4 l4 = *reinterpret_cast<const float4 *>(Lr + 16 * k + m);
                        fma4(acc, l4.x, *reinterpret_cast<const float4 *>(Ak + m * LS));
                        fma4(acc, l4.y, *reinterpret_cast<const float4 *>(Ak + (m + 1) * LS));
                        fma4(acc, l4.z, *reinterpret_cast<const float4 *>(Ak + (m + 2) * LS));
                        fma4(acc, l4.w, *reinterpret_cast<const float4 *>(Ak + (m + 3) * LS));
                    }
                }
                t[n] = acc;
            }
            __syncthreads();  // every product of this row block has read its L blocks
#pragma unroll
            for (int n = 0; n < 2; ++n) {
                const int u = tid + 64 * n, j = u >> 6, r = (u >> 2) & 15, c4 = (u & 3) * 4;
                if (u >= 64 * ib || (n && tid < 64)) continue;
                *reinterpret_cast<float4 *>(L + (16 * ib + r) * LS + 16 * j + c4) = t[n];
            }
            __syncthreads();
#pragma unroll
            for (int n = 0; n < 2; ++n) {  // A_ij = -A_ii T_ij
                const int u = tid + 64 * n, j = u >> 6, r = (u >> 2) & 15, c4 = (u & 3) * 4;
                if (u >= 64 * ib || (n && tid < 64)) continue;
                const float *Ai = L + (16 * ib + r) * LS + 16 * ib;  // row r of A_ii
                const float *Tj = L + (16 * ib) * LS + 16 * j + c4;  // T_ij, columns c4 ..
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int m = 0; m < 16; m += 4) {
                    const float4 a4 = *reinterpret_cast<const float4 *>(Ai + m);
                    fma4(acc, a4.x, *reinterpret_cast<const float4 *>(Tj + m * LS));
                    fma4(acc, a4.y, *reinterpret_cast<const float4 *>(Tj + (m + 1) * LS));
                    fma4(acc, a4.z, *reinterpret_cast<const float4 *>(Tj + (m + 2) * LS));
                    fma4(acc, a4.w, *reinterpret_cast<const float4 *>(Tj + (m + 3) * LS));
                }
                t[n] = make_float4(-acc.x, -acc.y, -acc.z, -acc.w);
            }
            __syncthreads();
#pragma unroll
            for (int n = 0; n < 2; ++n) {
                const int u = tid + 64 * n, j = u >> 6, r = (u >> 2) & 15, c4 = (u & 3) * 4;
                if (u >= 64 * ib || (n && tid < 64)) continue;
                *reinterpret_cast<float4 *>(L + (16 * ib + r) * LS + 16 * j + c4) = t[n];
            }
            __syncthreads();
        }
        // the bf16 operand tiles A diag(b gam), A diag(b) (and A itself for the backward):
        // every thread reads its four 8-column pieces of A before the tiles overwrite L
        {
            float av[4][8];
#pragma unroll
            for (int n = 0; n < 4; ++n) {
                const int e = tid + NT * n, r = e >> 3, cc = e & 7;
                const float4 x0 = *reinterpret_cast<const float4 *>(L + r * LS + 8 * cc);
                const float4 x1 = *reinterpret_cast<const float4 *>(L + r * LS + 8 * cc + 4);
                av[n][0] = x0.x; av[n][1] = x0.y; av[n][2] = x0.z; av[n][3] = x0.w;
                av[n][4] = x1.x; av[n][5] = x1.y; av[n][6] = x1.z; av[n][7] = x1.w;
            }
            __syncthreads();  // L is dead from here: the operand tiles overwrite it
#pragma unroll
            for (int n = 0; n < 4; ++n) {
                const int e = tid + NT * n, r = e >> 3, cc = e & 7;
                float fb[8], fc[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const int c = 8 * cc + q;
                    fc[q] = av[n][q] * bta[c];
                    fb[q] = fc[q] * E[c];
                }
                *reinterpret_cast<uint4 *>(Ab + sw128_chunk(C, r, cc)) = pack8(fb);
                *reinterpret_cast<uint4 *>(Ac + sw128_chunk(C, r, cc)) = pack8(fc);
                if (want_A) {
                    uint8_t *Ag = reinterpret_cast<uint8_t *>(p.tA) + (size_t)ch * C * C * 2;
                    *reinterpret_cast<uint4 *>(Ag + sw128_chunk(C, r, cc)) = pack8(av[n]);
                }
            }
        }
        operands_ready();
        // W = (A diag(b gam)) K, then Ut = (A diag(b)) V: M = 64, N = 128, K = 64 tokens,
        // one after the other in the same 128 TMEM columns
        const uint32_t id = idesc_bf16(64, 128, 0, 1);
        if (tid == 0) {
            const uint32_t ab = smem_u32(Ab);
#pragma unroll
            for (int s = 0; s < C / 16; ++s)
                mma_bf16(tmem, desc_kmajor(ab, C, s), desc_mnmajor(kb, D, s), id, s > 0);
            mma_commit(&mbar);
        }
        ok = cta_wait(&mbar, phase, p, 2);
        phase ^= 1;
        if (ok) {
            // W, stored negated (both chains subtract W products), is staged in the K rows'
            // place (the product has read them) and leaves by two bulk copies
            const int i = m64_row();
            for (int c0 = 0; c0 < D; c0 += 32) {
                float w[32];
                tmem_ld16(tm(tmem, c0), w);
                tmem_ld16(tm(tmem, c0 + 16), w + 16);
                tmem_ld_wait();
                if (i >= 0) {
#pragma unroll
                    for (int q = 0; q < 32; ++q) w[q] = -w[q];
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        *reinterpret_cast<uint4 *>(QK + qk_stage(C, c0 / 8 + q, i)) = pack8(w + 8 * q);
                }
            }
            fence_async_smem();
            tc_fence_before();
            __syncthreads();
            tc_fence_after();
            if (tid == 0) {
                uint8_t *Wimg = static_cast<uint8_t *>(p.tW) + (size_t)ch * kImg64;
                bulk_store(Wimg, smem_u32(QK) + C * 128, (uint32_t)kImg64 / 2);
                bulk_store(Wimg + kImg64 / 2, smem_u32(QK) + 3 * C * 128, (uint32_t)kImg64 / 2);
                bulk_commit();
            }
            // the V rows (loaded into the Q rows' place after the first product)
            ok = copies_arrived(&vbar, p, 34);
            v_pending = false;
            if (ok) fix_rows(QK, D, 0, ci.len, p.V);
            operands_ready();
            if (ok && tid == 0) {
                const uint32_t ac = smem_u32(Ac);
#pragma unroll
                for (int s = 0; s < C / 16; ++s)
                    mma_bf16(tmem, desc_kmajor(ac, C, s), desc_mnmajor(qkb, D, s), id, s > 0);
                mma_commit(&mbar);
            }
            if (ok) ok = cta_wait(&mbar, phase, p, 2);
            phase ^= 1;
        }
    }
    if (v_pending && tid == 0) mbar_wait(&vbar, 0, kWaitLimit);  // leave no copy in flight
    if (ok) {  // Ut as a 64 x 128 tile image (rows = tokens): an operand of the chains'
               // first product, whose 64-column blocks are the two halves of the values;
               // staged in the V rows' place (the product has read them), two bulk copies
        const int i = m64_row();
        for (int c0 = 0; c0 < D; c0 += 32) {
            float u[32];
            tmem_ld16(tm(tmem, c0), u);
            tmem_ld16(tm(tmem, c0 + 16), u + 16);
            tmem_ld_wait();
            if (i >= 0) {
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    *reinterpret_cast<uint4 *>(QK + qk_stage(0, c0 / 8 + q, i)) = pack8(u + 8 * q);
            }
        }
        fence_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    if (ok && tid == 0) {
        uint8_t *Ut = static_cast<uint8_t *>(p.tUt) + (size_t)ch * kImg64;
        bulk_store(Ut, smem_u32(QK), (uint32_t)kImg64 / 2);
        bulk_store(Ut + kImg64 / 2, smem_u32(QK) + 2 * C * 128, (uint32_t)kImg64 / 2);
        bulk_commit();
    }
    if (tid == 0) bulk_wait_read();  // (the staged rows are read before the CTA exits)
    if (tid >= 3 * 32) tmem_dealloc(tmem, 128);
}

}  // namespace tc
}  // namespace gdn
