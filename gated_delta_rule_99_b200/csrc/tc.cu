// Tensor-core (tcgen05) path of the bf16 layer, d_k = d_v = 128.
//
// Same chunkwise algebra as the fp32 path (chunk of 64 tokens; H = S^T the
// state entering a chunk; G the in-chunk cumulative log-decay):
//
//   A = (I + strict_lower(diag(b) K K^T . Gam))^-1 ; W = A diag(b gam) K ; Ut = A diag(b) V
//   U = Ut - W H ;  H' = gam_n H + (diag(e) K)^T U ;  O = diag(gam) Q' H + lower(Q' K^T . Gam) U
//
// Every product runs on tcgen05 (bf16 operands in 128-byte-swizzled shared
// memory, fp32 accumulators in TMEM).  The state chain runs in transposed
// form so its accumulators use all 128 TMEM lanes: thread v of the state
// kernel owns row v of S = H^T in fp32 registers, and per chunk
//
//   U^T = Ut^T - S W^T        (M = 128 rows v, N = 64 tokens, K = 128)
//   S  <- gam_n S + U^T Kd    (M = 128 rows v, N = 128 keys,  K = 64 tokens)
//
// Kernels: tc_prep (chunk-parallel: gates, [Q; K] K^T, the blocked inverse A
// in fp32, W, Ut, Kd = diag(e) K, Qg = scale diag(gam) Q and P), tc_state_fwd
// (serial over the chunks of a sequence; one CTA per (sequence, head); writes
// the state entering every chunk and U^T as swizzled tile images), tc_out
// (chunk-parallel output: one product over the four images).
#include "tc_common.cuh"
#include "tc_prep.cuh"
#include "tc_state.cuh"

namespace gdn {
namespace {

using namespace tc;

// ============================================================ tc_prep
__global__ void __launch_bounds__(NT, 4) tc_prep_kernel(const __grid_constant__ Params p, int want_A) {
    prep_body(p, blockIdx.x, want_A);
}

// ============================================================ tc_state_fwd
// One CTA per (sequence, head), or per (sequence, head, value slice) with p.vslice.
__global__ void __launch_bounds__(NT, 1) tc_state_fwd_kernel(Params p) {
    if (p.vslice) state_fwd_sliced_body(p, blockIdx.x);
    else state_fwd_body(p, blockIdx.x);
}

// ============================================================ tc_state_fwd_out
// The forward chain with the output formed in the same CTA (the default forward
// of sequences that run without the piece scan or value slices).
__global__ void __launch_bounds__(kOutChainThreads, 1)
    tc_state_fwd_out_kernel(const __grid_constant__ Params p) {
    state_fwd_out_body(p, blockIdx.x);
}

// ============================================================ piece scan (long rows)
// Phase A: piece 0 of every (row, head) runs the ordinary chain from h0, every
// middle piece once from zero and once from the identity (piece_a_fwd_role);
// phase B joins them (piece_scan_body); phase C reruns every later piece from
// its entering state (piece_c_fwd_role).  With p.vslice each role runs as value
// slices.
__global__ void __launch_bounds__(NT, 1) tc_piece_a_kernel(Params p) {
    const int nsl = p.vslice ? value_slices(p) : 1, roles = 2 * p.P - 3, blk = blockIdx.x / nsl;
    piece_a_fwd_role(p, blk / roles, blk % roles, blockIdx.x % nsl);
}

__global__ void __launch_bounds__(NT, 1) tc_piece_scan_kernel(Params p) {
    // H_in(q) = M_{q-1} H_in(q-1) + B_{q-1} for q = 2 .. P - 1
    piece_scan_body(p, blockIdx.x, p.tHin, p.tMp, p.tBp, 2, p.P - 1, 1, 33);
}

__global__ void __launch_bounds__(NT, 1) tc_piece_c_kernel(Params p) {
    const int nsl = p.vslice ? value_slices(p) : 1, blk = blockIdx.x / nsl, per = p.P - 1;
    piece_c_fwd_role(p, blk / per, 1 + blk % per, blockIdx.x % nsl);
}

// ============================================================ tc_out
// O^T[v][i] = S[v][:] . (scale gam_i q_i) + sum_j U^T[v][j] P[i][j],
// P = scale lower(Q K^T . Gam).  One CTA per (chunk, head), one M = 128 product
// over four tile images: the chain's snapshots S and U^T (read K-major), or,
// from the chain by value slices (p.vslice), H = S^T (rows = keys) and U (rows =
// tokens) read MN-major, the same A operands; and tc_prep's Qg = scale diag(gam) Q
// and P.  73 KB of shared memory: three CTAs per SM.
struct OutSmem {
    static constexpr int kS = 0, kUT = kS + 32768, kQG = kUT + 16384, kP = kQG + 16384,
                         kEnd = kP + 8192;
};
constexpr int kOutSmem = OutSmem::kEnd + 1024;

__global__ void __launch_bounds__(NT) tc_out_kernel(const __grid_constant__ Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = align1k(smem_raw);
    __shared__ uint64_t mbar, lbar;
    __shared__ uint32_t tslot;
    if (p.hdr->status) return;
    const int H = p.H, ch = blockIdx.x, c = ch / H, h = ch % H, tid = threadIdx.x;
    const ChunkInfo ci = chunk_at(p, c);
    uint8_t *Ss = sm + OutSmem::kS, *UTs = sm + OutSmem::kUT, *QG = sm + OutSmem::kQG,
            *Ps = sm + OutSmem::kP;
    if (tid == 0) {  // the four images by bulk copies
        mbar_init(&mbar, 1);
        mbar_init(&lbar, 1);
        fence_mbar_init();
        mbar_arrive_expect_tx(&lbar, (uint32_t)(kImg128 + kImgUT + kImg64 + C * C * 2));
        bulk_load(smem_u32(Ss), static_cast<const uint8_t *>(p.tS) + (size_t)ch * kImg128,
                  (uint32_t)kImg128, &lbar);
        bulk_load(smem_u32(UTs), static_cast<const uint8_t *>(p.tUT) + (size_t)ch * kImgUT,
                  (uint32_t)kImgUT, &lbar);
        bulk_load(smem_u32(QG), static_cast<const uint8_t *>(p.tQg) + (size_t)ch * kImg64,
                  (uint32_t)kImg64, &lbar);
        bulk_load(smem_u32(Ps), static_cast<const uint8_t *>(p.tP) + (size_t)ch * (C * C * 2),
                  (uint32_t)(C * C * 2), &lbar);
    }
    if (tid < 32) {
        tmem_alloc(&tslot, 64);
        tmem_relinquish();
    }
    __syncthreads();  // thread 0's mbarrier inits are visible before any thread waits on them
    bool ok = copies_arrived(&lbar, p, 7);
    tc_fence_after();
    const uint32_t tmem = tslot;
    if (ok && tid == 0) {
        const uint32_t sb = smem_u32(Ss), qg = smem_u32(QG), ub = smem_u32(UTs), pb = smem_u32(Ps);
        if (!p.vslice) {
            const uint32_t id = idesc_bf16(128, 64, 0, 0);
#pragma unroll
            for (int s = 0; s < D / 16; ++s)
                mma_bf16(tmem, desc_kmajor(sb, D, s), desc_kmajor(qg, C, s), id, s > 0);
#pragma unroll
            for (int s = 0; s < C / 16; ++s)
                mma_bf16(tmem, desc_kmajor(ub, D, s), desc_kmajor(pb, C, s), id, 1);
        } else {
            const uint32_t id = idesc_bf16(128, 64, 1, 0);
#pragma unroll
            for (int s = 0; s < D / 16; ++s)
                mma_bf16(tmem, desc_mnmajor(sb, D, s), desc_kmajor(qg, C, s), id, s > 0);
#pragma unroll
            for (int s = 0; s < C / 16; ++s)
                mma_bf16(tmem, desc_mnmajor(ub, C, s), desc_kmajor(pb, C, s), id, 1);
        }
        mma_commit(&mbar);
    }
    if (ok) ok = cta_wait(&mbar, 0, p, 6);
    if (ok) {  // O^T column v -> rows of a staging tile over the consumed S image, 16-byte stores
        bf16 *stage = reinterpret_cast<bf16 *>(Ss);
        for (int c0 = 0; c0 < C; c0 += 16) {
            float d[16];
            tmem_ld16(tm(tmem, c0), d);
            tmem_ld_wait();
#pragma unroll
            for (int q = 0; q < 16; ++q) stage[(c0 + q) * D + tid] = __float2bfloat16_rn(d[q]);
        }
        __syncthreads();
        bf16 *o = static_cast<bf16 *>(p.o);
        for (int t = tid; t < C * 16; t += NT) {
            const int i = t >> 4, j = t & 15;
            if (i < ci.len && j * 8 < p.V)
                *reinterpret_cast<uint4 *>(o + ((int64_t)(ci.tok0 + i) * H + h) * p.V + j * 8) =
                    *reinterpret_cast<const uint4 *>(Ss + i * 256 + j * 16);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (tid < 32) tmem_dealloc(tmem, 64);
}


}  // namespace

// Head dims 64 run on the 128-wide tiles zero-padded in shared memory.
bool tc_supported(const Problem &pb) {
    return (pb.K == 64 || pb.K == 128) && (pb.V == 64 || pb.V == 128);
}

bool tc_bwd_ready() { return true; }

cudaError_t tc_launch_prep(const Params &p, int want_A, cudaStream_t stream) {
    const int nch = p.NC * p.H;
    if (nch == 0) return cudaSuccess;
    cudaError_t e = set_smem(tc_prep_kernel, kPrepSmemRequest);
    if (e != cudaSuccess) return e;
    GDN_LAUNCH(kKTcPrep, stream,
               tc_prep_kernel<<<nch, NT, kPrepSmemRequest, stream>>>(p, want_A));
    return cudaSuccess;
}

// CTAs per forward chain, and their shared memory: one per (sequence, head), or one
// per value slice with p.vslice.
static int chain_slices(const Params &p) { return p.vslice ? (p.V + 63) / 64 : 1; }
static int chain_smem(const Params &p) { return p.vslice ? kSliceSmem : kStateSmem; }

cudaError_t tc_launch_state_fwd(const Params &p, cudaStream_t stream) {
    const int nseq = p.N * p.H * chain_slices(p), sm = chain_smem(p);
    if (nseq == 0) return cudaSuccess;
    cudaError_t e = set_smem(tc_state_fwd_kernel, sm);
    if (e != cudaSuccess) return e;
    GDN_LAUNCH(kKTcStateFwd, stream, tc_state_fwd_kernel<<<nseq, NT, sm, stream>>>(p));
    return cudaSuccess;
}

cudaError_t launch_tc_fwd(const Params &p, const Problem &, cudaStream_t stream) {
    cudaError_t e;
    if ((e = tc_launch_prep(p, 0, stream))) return e;
    if (p.P == 1 && !p.vslice) {  // the chain writes the output itself
        const int nseq = p.N * p.H;
        if (nseq == 0) return cudaSuccess;
        if ((e = set_smem(tc_state_fwd_out_kernel, kOutChainSmem))) return e;
        GDN_LAUNCH(kKTcStateFwd, stream,
                   tc_state_fwd_out_kernel<<<nseq, kOutChainThreads, kOutChainSmem, stream>>>(p));
        return cudaSuccess;
    }
    if (p.P > 1 && p.N * p.H > 0) {  // piece scan of long rows
        const int units = p.N * p.H, nsl = chain_slices(p), sm = chain_smem(p);
        if ((e = set_smem(tc_piece_a_kernel, sm))) return e;
        GDN_LAUNCH(kKTcPieceA, stream,
                   tc_piece_a_kernel<<<units * (2 * p.P - 3) * nsl, NT, sm, stream>>>(p));
        if ((e = set_smem(tc_piece_scan_kernel, kScanSmem))) return e;
        GDN_LAUNCH(kKTcPieceScan, stream,
                   tc_piece_scan_kernel<<<units, NT, kScanSmem, stream>>>(p));
        if ((e = set_smem(tc_piece_c_kernel, sm))) return e;
        GDN_LAUNCH(kKTcPieceC, stream,
                   tc_piece_c_kernel<<<units * (p.P - 1) * nsl, NT, sm, stream>>>(p));
    } else if ((e = tc_launch_state_fwd(p, stream))) {
        return e;
    }
    const int nch = p.NC * p.H;
    if (nch > 0) {
        if ((e = set_smem(tc_out_kernel, kOutSmem))) return e;
        GDN_LAUNCH(kKTcOut, stream, tc_out_kernel<<<nch, NT, kOutSmem, stream>>>(p));
    }
    return cudaSuccess;
}

static_assert(kPrepSmem <= kPrepSmemRequest, "prep shared memory");
static_assert(kOutChainSmem <= 227 * 1024, "chain-with-output shared memory");

}  // namespace gdn
