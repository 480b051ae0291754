// Internal declarations shared by the C ABI (gdn_api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

#include "gdn.h"

namespace gdn {

constexpr int kChunk = 64;        // tokens per chunk (the chunkwise form's block length)
constexpr int kSimtSlots = 512;   // CTAs of the SIMT chunk-parallel kernels (each owns a scratch slot)
constexpr int kSimtVSlice = 32;   // value columns per CTA in the SIMT state passes
// Polls of a bounded mbarrier wait (about a second) unless gdn_set_wait_limit
// lowered it; the waits that drain copies still in flight after a failure
// always use this one.
constexpr uint32_t kWaitLimit = 1u << 23;

// One chunk of one sequence: tokens [tok0, tok0 + len) of the flattened B*T rows.
struct ChunkInfo {
    int32_t seq;  // sequence (dense row or packed document) index
    int32_t tok0; // first token (flattened over rows)
    int32_t len;  // 1..64
    int32_t idx;  // chunk index inside its sequence
};

// First 256 bytes of every workspace.
struct WsHeader {
    int32_t status;    // gdn_status recorded on the device (0 = ok)
    int32_t n_chunks;  // chunk count the device built
    int32_t where;     // diagnostic: which wait gave up (0 = none)
    int32_t pad[61];
};

// Everything a kernel needs; passed by value.
struct Params {
    // problem
    int32_t B, T, H, K, V, N, NC;  // N sequences, NC chunks (exact, from the host)
    int64_t BT;                    // tokens over all rows
    float scale;
    int32_t bf16;                  // 1: q/k/v/o/do/dq/dk/dv are bf16, 0: fp32
    int32_t l2norm;                // 1: q and k rows are divided by their norms first
    int32_t vslice;                // 1: the forward chains run by value slices (GDN_FLAG_VALUE_SLICES)
    uint32_t wait_limit;           // polls of a bounded mbarrier wait before it gives up
    int32_t test_hook;             // planted failure for the tests (GDN_TEST_*), 0 = none
    // inputs
    const void *q, *k, *v, *do_;
    const float *g, *beta, *h0, *dhT;
    const int32_t *cu;             // device cu_seqlens, or nullptr for dense rows
    // outputs
    void *o, *dq, *dk, *dv;
    float *hT, *dg, *dbeta, *dh0;
    // workspace
    WsHeader *hdr;
    ChunkInfo *chunks;
    int32_t *seq_first;            // N + 1 entries: first chunk of each sequence
    // fp32 per-(chunk, head) intermediates of the SIMT path
    float *W, *Ut, *A, *U, *Hs, *dUloc, *dU, *dHn;
    float *scratch;                // kSimtSlots slots of simt_scratch_floats(tile width)
    // bf16 tensor-core path intermediates, per (chunk, head): tile images
    // (128-byte-swizzled, as the MMAs read them) and plain rows
    void *tW, *tUt, *tKd;          // 64x128 W image, 64x128 Ut rows, 64x128 diag(e)K image
    void *tS, *tUT;                // 128x128 image of the state entering the chunk, 128x64 U^T image
    void *tQg, *tP, *tdSn, *tdUT;  // backward: scaled-q image, P tile, dS image, dU^T image
    float *tG;                     // 64 cumulative gates per (chunk, head)
    float *tB;                     // 64 write strengths per (chunk, head), 0 past its end
    void *tA;                      // 64x64 bf16 tile image of A (backward)
    // piece scan of long rows (forward): pieces per sequence, chunks per piece, and per
    // (sequence, head, piece) the entering state, the composed transition and offset
    int32_t P, L;
    float *tHin, *tMp, *tBp;
    // and, for the backward's reverse chain, per (sequence, head, piece) the dS
    // leaving the piece, the piece's transition and its offset
    float *tdHin, *tTr, *tBr;
    // tensor maps of the bf16 [tokens][H][d] inputs for the tensor-core path: a box is 64
    // tokens x 64 elements of one head, written to shared memory with the operand tiles'
    // 128-byte swizzle (encoded on the host for every call)
    CUtensorMap tm_q, tm_k, tm_v, tm_do, tm_dq, tm_dk, tm_dv, tm_o;
};

// Row width (floats) of the SIMT path's 64-row chunk tiles: 128, or 256 when a head
// dim is 256; and the per-CTA scratch floats of its chunk-parallel kernels.
__host__ __device__ constexpr int simt_tile_width(int K, int V) { return (K > 128 || V > 128) ? 256 : 128; }
__host__ __device__ constexpr size_t simt_scratch_floats(int D) {
    return (size_t)64 * D * 14 + 64 * 64 * 10 + 64 * 8;
}

// Chunk c of the call: from the table build_chunks writes for packed documents,
// or in closed form for dense rows (row c / n, chunk c % n of a row, n = ceil(T / 64)),
// which then need no table.
__device__ __forceinline__ ChunkInfo chunk_at(const Params &p, int c) {
    if (p.cu) return p.chunks[c];
    const int npr = (p.T + kChunk - 1) / kChunk, row = c / npr, j = c - row * npr;
    ChunkInfo ci;
    ci.seq = row;
    ci.tok0 = row * p.T + j * kChunk;
    ci.len = p.T - j * kChunk < kChunk ? p.T - j * kChunk : kChunk;
    ci.idx = j;
    return ci;
}
// Chunk c of sequence n whose first chunk is c0 (no division: for the loops
// that walk one sequence's chunks).
__device__ __forceinline__ ChunkInfo chunk_in_seq(const Params &p, int n, int c0, int c) {
    if (p.cu) return p.chunks[c];
    const int j = c - c0;
    ChunkInfo ci;
    ci.seq = n;
    ci.tok0 = n * p.T + j * kChunk;
    ci.len = p.T - j * kChunk < kChunk ? p.T - j * kChunk : kChunk;
    ci.idx = j;
    return ci;
}
// First chunk of sequence n (n = N gives the chunk count).
__device__ __forceinline__ int seq_first_at(const Params &p, int n) {
    return p.cu ? p.seq_first[n] : n * ((p.T + kChunk - 1) / kChunk);
}

// Host-side problem summary after validation.
struct Problem {
    int64_t B, T, H, K, V, N, BT;
    int64_t NCmax;  // capacity used for the workspace layout (depends only on the descriptor)
    int64_t NC;     // exact chunk count of this call
    int dtype;
    float scale;
    int64_t P, L;   // pieces per sequence (1 = no piece scan) and chunks per piece
    int l2norm;     // GDN_FLAG_QK_L2NORM
    int vslice;     // GDN_FLAG_VALUE_SLICES
};

// Workspace layout: offsets in bytes from the workspace base.
struct Layout {
    size_t chunks, seq_first;
    size_t W, Ut, A, U, Hs, dUloc, dU, dHn, scratch;
    size_t tW, tUt, tKd, tS, tUT, tQg, tP, tdSn, tdUT, tG, tB, tA, tHin, tMp, tBp;
    size_t tdHin, tTr, tBr;
    size_t qn, kn, qinv, kinv;  // normalised q, k copies and 1/|row| (passes of the fp32 path)
    size_t total;
};

Layout make_layout(const Problem &p, bool bwd);

// Kernel launchers (all asynchronous on `stream`; return the launch error).
cudaError_t launch_build_chunks(const Params &p, cudaStream_t stream);
cudaError_t launch_simt_fwd(const Params &p, cudaStream_t stream);
cudaError_t launch_simt_bwd(const Params &p, cudaStream_t stream);
bool tc_supported(const Problem &p);
// Normalisation pass: xn = x / |x| per row of K values (dtype of x), inv = 1/|x|.
cudaError_t launch_l2norm_rows(const void *x, void *xn, float *inv, int64_t rows, int K,
                               bool bf16, cudaStream_t stream);
// Projection pass, in place: dx <- (dx - xn (xn . dx)) * inv per row.
cudaError_t launch_l2norm_back(const void *xn, const float *inv, void *dx, int64_t rows, int K,
                               bool bf16, cudaStream_t stream);
bool tc_bwd_ready();
cudaError_t launch_tc_fwd(const Params &p, const Problem &pb, cudaStream_t stream);
// Encodes p.tm_q, tm_k, tm_v (and tm_do, tm_dq, tm_dk, tm_dv for the backward) from
// p.q, p.k, p.v, p.do_, p.dq, p.dk, p.dv.
bool encode_row_maps(Params &p, bool bwd);
cudaError_t launch_tc_bwd(const Params &p, const Problem &pb, cudaStream_t stream);

// Kernel ids recorded by the launch trace (gdn_trace_install).
enum KernelId : int32_t {
    kKBuildChunks = 0,
    kKSimtPrep,
    kKSimtStateFwd,
    kKSimtOut,
    kKSimtDuloc,
    kKSimtStateBwd,
    kKSimtGrads,
    kKTcPrep,
    kKTcStateFwd,
    kKTcOut,
    kKTcStateBwd,  // backward chains (forward recompute + reverse pass)
    kKTcGrads,
    kKTcLocal,
    kKDecode,
    kKTcPieceA,
    kKTcPieceScan,
    kKTcPieceC,
    kKL2Norm,
    kKL2NormBack,
    kKernelCount
};

// Brackets one launch with the installed trace's events (no-op when none).
void trace_before(int32_t id, cudaStream_t stream);
void trace_after(cudaStream_t stream);

// Per-host-thread settings of the testing hooks (gdn_set_wait_limit,
// gdn_set_test_hook): the wait limit and hook the next call's kernels get,
// arming the planted launch failure at the start of an ABI call, and taking it
// (true once per armed call) before a launch.
uint32_t call_wait_limit();
int32_t call_test_hook();
void arm_planted_failure();
bool take_planted_failure();

// Launches `...` (a kernel<<<>>>(...) expression) inside a trace bracket and
// returns its launch error from the enclosing function.
#define GDN_LAUNCH(id, stream, ...)                              \
    do {                                                         \
        if (::gdn::take_planted_failure()) return cudaErrorLaunchFailure; \
        ::gdn::trace_before((id), (stream));                     \
        __VA_ARGS__;                                             \
        ::gdn::trace_after((stream));                            \
        cudaError_t gdn_launch_err_ = cudaGetLastError();        \
        if (gdn_launch_err_ != cudaSuccess) return gdn_launch_err_; \
    } while (0)

// Device-side status codes written into WsHeader::status.
enum : int32_t { kDevOk = 0, kDevBadSeqlens = GDN_ERR_INVALID_ARG, kDevTimeout = GDN_ERR_TIMEOUT };

}  // namespace gdn
