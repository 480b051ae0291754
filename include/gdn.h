/*
 * gdn.h -- C ABI of the B200 (sm_100a) Gated DeltaNet layer: chunkwise
 * forward and backward of the gated delta rule.
 *
 * The operation (per sequence and head; S is d_v x d_k, state kept in fp32):
 *
 *     S_t = a_t * S_{t-1} * (I - b_t k_t k_t^T) + b_t v_t k_t^T,  a_t = exp(g_t)
 *     o_t = scale * S_t q_t
 *
 * g is the per-token log-decay and b ("beta") the write strength, both one
 * value per token and head (jax-linear-attention 0.1.0, "Quick start").  The
 * library computes it chunkwise in parallel with fp32 state and fp32
 * accumulation, exactly (no truncated history): packed documents reset the
 * state at every boundary so a packed row equals its documents run one by
 * one (same page, "How it works"), an optional initial state h0 is read and
 * an optional final state hT written (same page, "Quick start": the final
 * state comes back per row and head), and one long call equals chained calls
 * with the state carried over (same page, "Highlights").
 *
 * Layouts (all row-major, contiguous, "sequence first" as flash-linear-
 * attention switched to: hysenlabs review of flash-linear-attention):
 *   q, k, dq, dk      [B][T][H][dk]      dtype (bf16 or fp32)
 *   v, o, do_, dv     [B][T][H][dv]      dtype
 *   g, beta, dg, dbeta[B][T][H]          fp32
 *   h0, hT, dh0, dhT  [N][H][dk][dv]     fp32, element [i][j] = S[j][i]
 * N = B for dense rows (n_seqs == 0) or N = n_seqs for packed documents
 * (which requires B == 1; cu_seqlens[0] = 0, cu_seqlens[N] = T,
 * non-decreasing; empty documents are allowed and pass their state through).
 *
 * Pointers: q..dbeta, h0..dhT and cu_seqlens are DEVICE pointers on the
 * current device, 16-byte aligned; cu_seqlens_host is a HOST mirror of
 * cu_seqlens used for validation and grid sizing (if it is NULL while
 * cu_seqlens is set, the call copies cu_seqlens to the host and synchronises
 * the stream first).  The workspace is a device buffer of at least the size
 * the matching *_workspace_size function returns, 256-byte aligned.
 *
 * Ownership: the caller owns every buffer, the workspace and the stream
 * (passed as a cudaStream_t cast to void*, NULL = legacy default stream).
 * The library allocates no device memory and keeps no global state (the
 * optional launch trace below is per host thread); calls are reentrant, but
 * calls that share one workspace must not overlap on the GPU.
 *
 * Errors: argument, shape, alignment and workspace errors are returned
 * synchronously, before anything is launched.  Head dims other than 64 and
 * 128 return GDN_ERR_UNSUPPORTED (there is no fallback path).  A failure on
 * the device (a bounded wait that ran out) is recorded in the workspace and
 * read back by gdn_device_status.  All successful calls are asynchronous on
 * the given stream.
 */
#ifndef GDN_H
#define GDN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum gdn_status {
    GDN_OK = 0,
    GDN_ERR_INVALID_ARG = 1, /* bad shape, null pointer, bad cu_seqlens */
    GDN_ERR_UNSUPPORTED = 2, /* head dim not in {64, 128, 256} ({64, 128} for decode), unknown dtype */
    GDN_ERR_ALIGNMENT = 3,   /* a pointer is not 16-byte (workspace: 256-byte) aligned */
    GDN_ERR_WORKSPACE = 4,   /* workspace missing or too small */
    GDN_ERR_CUDA = 5,        /* a CUDA runtime call failed (launch, copy) */
    GDN_ERR_TIMEOUT = 6      /* a device-side bounded wait ran out */
} gdn_status;

typedef enum gdn_dtype {
    GDN_BF16 = 0, /* q, k, v, o, do_, dq, dk, dv in bfloat16 */
    GDN_FP32 = 1  /* ... in float32 */
} gdn_dtype;

typedef struct gdn_desc {
    int64_t B;      /* rows (must be 1 when n_seqs > 0) */
    int64_t T;      /* tokens per row; B * T < 2^31 */
    int64_t H;      /* heads */
    int64_t dk;     /* key/query head dim: 64, 128 or 256 (256: CUDA-core kernels; not decode) */
    int64_t dv;     /* value head dim: 64, 128 or 256 (256: CUDA-core kernels; not decode) */
    int64_t n_seqs; /* 0: B dense rows; > 0: packed documents given by cu_seqlens */
    int32_t dtype;  /* gdn_dtype */
    float scale;    /* output scale applied to q (1.0 for the plain recurrence) */
    int32_t flags;  /* GDN_FLAG_* options, 0 for the defaults */
    int32_t reserved; /* must be 0 */
} gdn_desc;

/* Forward option: split long dense rows into pieces that run in parallel and
 * are joined exactly.  Each chunk maps the state affinely, H' = M_c H + B_c
 * (no history is dropped), so every piece computes its composed (M, B) pair
 * from a zero and an identity start, a short scan over pieces gives every
 * piece its entering state, and each piece then reruns its chain from that
 * state.  It pays off when rows are long and (rows x heads) is small (the
 * pages' long single rows: jax-linear-attention 0.1.0, "Where we lose", which
 * splits them exactly; the FlashQLA article, "Skipping the warm-up", whose
 * split is approximate).  Results equal the default path up to the bf16
 * rounding of the transition matrices, so the default path's bitwise
 * one-call-equals-chained-calls property does not carry over.  In gdn_bwd both
 * chains are split: the recomputed forward chain as above, and the reverse
 * chain, whose chunk map is affine in dS too, by the mirrored scheme (pieces run
 * from a zero and an identity dS, a scan from the row's end, reruns).  Applies
 * to bf16 dense rows with d_k = d_v = 128 in gdn_fwd and gdn_bwd; ignored
 * elsewhere. */
#define GDN_FLAG_PIECE_SCAN 1

/* Option for gdn_fwd, gdn_fwd_noalloc, gdn_bwd and gdn_decode: the layer first
 * divides every q and k row (one token and head, d_k values) by its Euclidean
 * norm, in fp32, rounding the result to the input dtype (a zero row stays
 * zero); gdn_bwd then returns dq and dk with respect to the raw q and k,
 * dq = (dq^ - q^ (q^ . dq^)) / |q| with q^ the normalised row and dq^ the
 * gradient with respect to it.  The pages' API names the option
 * (jax-linear-attention 0.1.0, "Quick start": use_qk_l2norm=True) without a
 * formula; x / |x| is the reading taken.  On the bf16 d_k = d_v = 128 path the
 * kernels that load q and k normalise their tiles themselves; elsewhere a
 * normalisation pass runs first (and, in gdn_bwd, a projection pass last), with
 * the normalised copies in the workspace. */
#define GDN_FLAG_QK_L2NORM 2

/* Forward option: run the forward state chains by value slices.  The rows of
 * S (one per value column) evolve independently given a chunk's keys, write
 * strengths and gates, so each (sequence, head) chain can be split over CTAs
 * by value columns (the d_v slicing of the chunkwise form): two CTAs of 64
 * value columns each, in the untransposed form in which the key dimension is
 * the M = 128 side of the state update.  Same results up to the association
 * of the products inside the tensor cores; not bitwise equal to the default.
 * On a B200 it is not faster (a chain step is bound by the fixed latency of
 * its two dependent tensor-core products, which does not shrink with their
 * size), so it is off by default.  Applies to the bf16 forward with head dims
 * 64 or 128 (and the piece scan); ignored elsewhere, and by gdn_bwd and gdn_decode. */
#define GDN_FLAG_VALUE_SLICES 4

/* Library version (major * 10000 + minor * 100 + patch). */
int gdn_version(void);

/* Fixed chunk length of the chunkwise algorithm (tokens). */
int gdn_chunk_size(void);

/* Bytes of device workspace gdn_fwd / gdn_bwd need for this problem (0 on a
 * bad descriptor).  The size depends only on the descriptor. */
size_t gdn_fwd_workspace_size(const gdn_desc *desc);
size_t gdn_bwd_workspace_size(const gdn_desc *desc);

/* Forward: o (and hT when non-NULL) from q, k, v, g, beta and h0 (NULL means
 * a zero initial state).  cu_seqlens/cu_seqlens_host are NULL for dense rows. */
gdn_status gdn_fwd(const gdn_desc *desc, const void *q, const void *k, const void *v,
                   const float *g, const float *beta, const int32_t *cu_seqlens,
                   const int32_t *cu_seqlens_host, const float *h0, void *o, float *hT,
                   void *workspace, size_t workspace_bytes, void *stream);

/* Forward for callers that cannot allocate device memory (no counterpart in
 * the pages describing the method: it is a packaging variant of gdn_fwd).
 * A caller whose device memory is all owned elsewhere -- a serving process
 * that reserved HBM in a fixed pool at start-up and may not call cudaMalloc
 * while serving, or a plugin handed only its input and output buffers --
 * passes the same arguments as gdn_fwd minus the workspace.  The scratch is a
 * static device array of GDN_NOALLOC_MAX_WORKSPACE bytes inside the library;
 * every GPU that loads the library keeps it until the process exits.
 * Problems whose gdn_fwd_workspace_size exceeds that return
 * GDN_ERR_WORKSPACE (use gdn_fwd with your own workspace instead).  The first
 * call on each device looks up the array's device address with that device
 * current, so make the first call before any stream capture.  All calls share
 * the one array: calls that overlap on the GPU (other streams, other host
 * threads) race and corrupt each other's results, so serialise them.  The
 * device-side status of these calls lives in the array's header: read it with
 * gdn_fwd_noalloc_status.  No allocation of any kind is made. */
#define GDN_NOALLOC_MAX_WORKSPACE (64u * 1024u * 1024u)
gdn_status gdn_fwd_noalloc(const gdn_desc *desc, const void *q, const void *k, const void *v,
                           const float *g, const float *beta, const int32_t *cu_seqlens,
                           const int32_t *cu_seqlens_host, const float *h0, void *o, float *hT,
                           void *stream);

/* gdn_device_status for gdn_fwd_noalloc on the current device: synchronises
 * the stream, then returns and clears the device-side status the last
 * gdn_fwd_noalloc call on this device recorded in the library's static
 * scratch (GDN_OK, GDN_ERR_TIMEOUT, or GDN_ERR_INVALID_ARG when the device copy
 * of cu_seqlens disagreed with the host mirror).  GDN_OK if gdn_fwd_noalloc has
 * not run on this device yet; GDN_ERR_CUDA if the stream failed.  It copies a
 * few bytes between host and device and allocates nothing. */
gdn_status gdn_fwd_noalloc_status(void *stream);

/* Backward of (o, hT) given do_ and dhT (NULL means zero): writes dq, dk, dv,
 * dg, dbeta and dh0 (dh0 may be NULL to skip it).  The per-chunk states are
 * recomputed from the inputs, not read from a forward call. */
gdn_status gdn_bwd(const gdn_desc *desc, const void *q, const void *k, const void *v,
                   const float *g, const float *beta, const int32_t *cu_seqlens,
                   const int32_t *cu_seqlens_host, const float *h0, const void *do_,
                   const float *dhT, void *dq, void *dk, void *dv, float *dg, float *dbeta,
                   float *dh0, void *workspace, size_t workspace_bytes, void *stream);

/* Recurrent decode: advance each sequence's state through T tokens (usually
 * T = 1) with the token-by-token form of the same recurrence, for inference
 * with a cached per-layer state (jax-linear-attention 0.1.0, "FAQ": decode
 * runs with each layer's recurrent state).  desc: B sequences of T tokens,
 * n_seqs must be 0; q, k [B][T][H][dk], v, o [B][T][H][dv] in desc->dtype;
 * g, beta [B][T][H] fp32; state [B][H][dk][dv] fp32 (= S^T, the layout of
 * h0/hT), read and overwritten in place with the state after the last token.
 * Needs no workspace; asynchronous on the stream; argument errors return
 * before any launch. */
gdn_status gdn_decode(const gdn_desc *desc, const void *q, const void *k, const void *v,
                      const float *g, const float *beta, float *state, void *o, void *stream);

/* Synchronises the stream, then returns and clears the device-side status
 * that the last gdn_fwd/gdn_bwd on this workspace recorded (GDN_OK,
 * GDN_ERR_TIMEOUT, or GDN_ERR_INVALID_ARG when the device copy of cu_seqlens
 * disagreed with the host mirror).  GDN_ERR_CUDA if the stream failed. */
gdn_status gdn_device_status(void *workspace, void *stream);

/* Static English name of a status code. */
const char *gdn_status_string(gdn_status status);

/* Testing hooks, per host thread (they let the tests drive the failure paths
 * without faulting a GPU).  Both apply to every later call from the calling
 * thread until changed; the defaults are 0.
 *
 * gdn_set_wait_limit: every bounded device-side wait of the tensor-core
 * kernels gives up after `polls` polls of its mbarrier instead of the built-in
 * 2^23 (about a second); 0 restores the built-in limit.  A wait that gives up
 * records GDN_ERR_TIMEOUT, and the kernels of the call that start after it
 * return at once (read it with gdn_device_status).
 *
 * gdn_set_test_hook: plants one failure in each later call.
 *   GDN_TEST_STALL_COPY  the first (chunk, head) CTA of the call's tensor-core
 *                        preparation step arms its input-copy mbarrier for 16
 *                        bytes more than its copies bring: every copy lands,
 *                        the wait runs out, and the call records
 *                        GDN_ERR_TIMEOUT (outputs are then undefined).
 *   GDN_TEST_FAIL_LAUNCH the call's first kernel launch is skipped and treated
 *                        as a failed launch: the call returns GDN_ERR_CUDA.
 * 0 removes the hook. */
#define GDN_TEST_STALL_COPY 1
#define GDN_TEST_FAIL_LAUNCH 2
void gdn_set_wait_limit(uint32_t polls);
void gdn_set_test_hook(int32_t hook);

/* Optional launch tracing (profiling aid).  While a trace is installed on the
 * calling host thread, every kernel that gdn_fwd / gdn_bwd launch from that
 * thread is bracketed by a pair of caller-created CUDA events recorded on the
 * call's stream, so the caller can time each kernel with
 * cudaEventElapsedTime.  events holds 2 * capacity cudaEvent_t (cast to
 * void*); pair i is events[2i] (before) and events[2i+1] (after), and
 * kernel_ids[i] names the kernel (see gdn_kernel_name).  The library only
 * increments count; launches beyond capacity are counted in `dropped` and
 * not recorded.  The caller owns the struct and the events and must keep
 * them alive while installed.  NULL uninstalls.  No effect on results. */
typedef struct gdn_trace {
    int32_t capacity;
    int32_t count;
    int32_t dropped;
    int32_t pad;
    void **events;
    int32_t *kernel_ids;
} gdn_trace;

void gdn_trace_install(gdn_trace *trace);

/* Static name of a kernel id recorded in a trace ("?" if unknown). */
const char *gdn_kernel_name(int32_t id);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H */
