// C ABI of the Gated DeltaNet layer: validation, workspace layout and launch
// sequencing on the caller's stream.  Declared in include/gdn.h.
#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>
#include <vector>

#include "gdn_internal.cuh"

namespace gdn {

namespace {

constexpr size_t kAlign = 256;

size_t up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// Shape checks that need no pointers.  Fills everything but NC.
gdn_status describe(const gdn_desc *d, Problem *p) {
    if (!d) return GDN_ERR_INVALID_ARG;
    if (d->B < 1 || d->T < 0 || d->H < 1 || d->n_seqs < 0) return GDN_ERR_INVALID_ARG;
    if (d->dtype != GDN_BF16 && d->dtype != GDN_FP32) return GDN_ERR_UNSUPPORTED;
    // head dims 64 and 128 (both paths) and 256 (the fp32 CUDA-core kernels, either dtype)
    const auto dim_ok = [](int64_t x) { return x == 64 || x == 128 || x == 256; };
    if (!dim_ok(d->dk) || !dim_ok(d->dv)) return GDN_ERR_UNSUPPORTED;
    if (d->n_seqs > 0 && d->B != 1) return GDN_ERR_INVALID_ARG;
    // range checks before any product is formed (no signed overflow on huge inputs)
    constexpr int64_t kLim = int64_t(1) << 31;
    if (d->B >= kLim || d->T >= kLim || d->T >= kLim / d->B || d->H >= (1 << 16) ||
        d->n_seqs >= kLim)
        return GDN_ERR_INVALID_ARG;
    if (!(d->scale == d->scale)) return GDN_ERR_INVALID_ARG;  // NaN scale
    p->B = d->B;
    p->T = d->T;
    p->H = d->H;
    p->K = d->dk;
    p->V = d->dv;
    p->BT = d->B * d->T;
    p->N = d->n_seqs > 0 ? d->n_seqs : d->B;
    if (p->N >= (int64_t(1) << 30)) return GDN_ERR_INVALID_ARG;
    p->NCmax = d->n_seqs > 0 ? (d->T + kChunk - 1) / kChunk + d->n_seqs
                             : d->B * ((d->T + kChunk - 1) / kChunk);
    // grids of (chunk, head) and (sequence, head) CTAs are formed in int32
    if (p->NCmax * p->H >= (int64_t(1) << 30)) return GDN_ERR_INVALID_ARG;
    p->NC = 0;
    p->dtype = d->dtype;
    p->scale = d->scale;
    if (d->reserved != 0 ||
        (d->flags & ~(GDN_FLAG_PIECE_SCAN | GDN_FLAG_QK_L2NORM | GDN_FLAG_VALUE_SLICES)))
        return GDN_ERR_INVALID_ARG;
    p->l2norm = (d->flags & GDN_FLAG_QK_L2NORM) ? 1 : 0;
    p->vslice = (d->flags & GDN_FLAG_VALUE_SLICES) ? 1 : 0;
    p->P = 1;
    p->L = 0;
    if ((d->flags & GDN_FLAG_PIECE_SCAN) && d->n_seqs == 0 && d->dtype == GDN_BF16 &&
        p->K == 128 && p->V == 128) {
        // pieces per row: phase C (one CTA per later piece) fits one wave of the
        // 148 SMs, phase A (two runs per middle piece) at most two, and every
        // piece spans at least 16 chunks; fewer than 3 pieces gain nothing
        const int64_t units = p->B * p->H, npr = (p->T + kChunk - 1) / kChunk;
        int64_t P = 148 / units + 1;
        const int64_t pa = (2 * 148 / units + 3) / 2;
        if (pa < P) P = pa;
        if (npr / 16 < P) P = npr / 16;
        if (P >= 3) {
            p->P = P;
            p->L = (npr + P - 1) / P;
        }
    }
    return GDN_OK;
}

bool misaligned(const void *ptr, size_t a = 16) {
    return ptr && (reinterpret_cast<uintptr_t>(ptr) % a) != 0;
}

// Host-side check of cu_seqlens; fills p->NC.
gdn_status check_seqlens(const gdn_desc *d, const int32_t *cu_dev, const int32_t *cu_host,
                         cudaStream_t stream, Problem *p) {
    if (d->n_seqs == 0) {
        if (cu_dev || cu_host) return GDN_ERR_INVALID_ARG;
        p->NC = p->NCmax;
        return GDN_OK;
    }
    if (!cu_dev) return GDN_ERR_INVALID_ARG;
    if (misaligned(cu_dev, 4)) return GDN_ERR_ALIGNMENT;
    std::vector<int32_t> copy;
    if (!cu_host) {
        copy.resize((size_t)d->n_seqs + 1);
        if (cudaMemcpyAsync(copy.data(), cu_dev, sizeof(int32_t) * copy.size(),
                            cudaMemcpyDeviceToHost, stream) != cudaSuccess)
            return GDN_ERR_CUDA;
        if (cudaStreamSynchronize(stream) != cudaSuccess) return GDN_ERR_CUDA;
        cu_host = copy.data();
    }
    if (cu_host[0] != 0 || cu_host[d->n_seqs] != d->T) return GDN_ERR_INVALID_ARG;
    int64_t nc = 0;
    for (int64_t n = 0; n < d->n_seqs; ++n) {
        const int64_t len = (int64_t)cu_host[n + 1] - cu_host[n];
        if (len < 0) return GDN_ERR_INVALID_ARG;
        nc += (len + kChunk - 1) / kChunk;
    }
    if (nc > p->NCmax) return GDN_ERR_INVALID_ARG;
    p->NC = nc;
    return GDN_OK;
}

Params base_params(const Problem &pb, const gdn_desc *d, void *ws, const Layout &L,
                   const int32_t *cu_dev) {
    Params p;
    std::memset(&p, 0, sizeof(p));
    p.B = (int32_t)pb.B;
    p.T = (int32_t)pb.T;
    p.H = (int32_t)pb.H;
    p.K = (int32_t)pb.K;
    p.V = (int32_t)pb.V;
    p.N = (int32_t)pb.N;
    p.NC = (int32_t)pb.NC;
    p.BT = pb.BT;
    p.scale = d->scale;
    p.bf16 = d->dtype == GDN_BF16;
    p.l2norm = pb.l2norm;
    p.vslice = pb.vslice;
    p.wait_limit = call_wait_limit();
    p.test_hook = call_test_hook();
    p.cu = d->n_seqs > 0 ? cu_dev : nullptr;
    char *base = static_cast<char *>(ws);
    p.hdr = reinterpret_cast<WsHeader *>(base);
    p.chunks = reinterpret_cast<ChunkInfo *>(base + L.chunks);
    p.seq_first = reinterpret_cast<int32_t *>(base + L.seq_first);
    auto f = [&](size_t off) { return off ? reinterpret_cast<float *>(base + off) : nullptr; };
    p.W = f(L.W);
    p.Ut = f(L.Ut);
    p.A = f(L.A);
    p.U = f(L.U);
    p.Hs = f(L.Hs);
    p.dUloc = f(L.dUloc);
    p.dU = f(L.dU);
    p.dHn = f(L.dHn);
    p.scratch = f(L.scratch);
    auto b = [&](size_t off) { return off ? static_cast<void *>(base + off) : nullptr; };
    p.tW = b(L.tW);
    p.tUt = b(L.tUt);
    p.tKd = b(L.tKd);
    p.tS = b(L.tS);
    p.tUT = b(L.tUT);
    p.tQg = b(L.tQg);
    p.tP = b(L.tP);
    p.tdSn = b(L.tdSn);
    p.tdUT = b(L.tdUT);
    p.tG = f(L.tG);
    p.tB = f(L.tB);
    p.tA = b(L.tA);
    p.P = (int32_t)pb.P;
    p.L = (int32_t)pb.L;
    p.tHin = f(L.tHin);
    p.tMp = f(L.tMp);
    p.tBp = f(L.tBp);
    p.tdHin = f(L.tdHin);
    p.tTr = f(L.tTr);
    p.tBr = f(L.tBr);
    return p;
}

// The driver's tensor-map encoder, looked up once through the runtime.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000,
                                             cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
        else
            (void)cudaGetLastError();
    });
    return fn;
}

// [tokens][H][width] bf16 viewed as a 3-d tensor (element, head, token); a box is
// 64 elements x 1 head x 64 tokens (128-byte rows in the operand tiles' swizzle).
bool encode_rows(CUtensorMap *m, const void *ptr, int64_t BT, int64_t H, int64_t width) {
    PFN_cuTensorMapEncodeTiled_v12000 fn = tensor_map_encoder();
    if (!fn || !ptr) return false;
    cuuint64_t dims[3] = {(cuuint64_t)width, (cuuint64_t)H, (cuuint64_t)BT};
    cuuint64_t strides[2] = {(cuuint64_t)width * 2, (cuuint64_t)H * width * 2};
    cuuint32_t box[3] = {64, 1, 64};
    cuuint32_t estride[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box,
              estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Normalisation pass of the fp32 path: q and k rows divided by their norms into
// the workspace copies, which the kernels then read in place of q and k.
bool normalise_qk(const Problem &pb, const Layout &L, void *ws, Params *p, cudaStream_t s) {
    if (pb.BT == 0) return true;
    char *base = static_cast<char *>(ws);
    const int64_t rows = pb.BT * pb.H;
    if (launch_l2norm_rows(p->q, base + L.qn, reinterpret_cast<float *>(base + L.qinv), rows,
                           (int)pb.K, p->bf16, s) != cudaSuccess ||
        launch_l2norm_rows(p->k, base + L.kn, reinterpret_cast<float *>(base + L.kinv), rows,
                           (int)pb.K, p->bf16, s) != cudaSuccess)
        return false;
    p->q = base + L.qn;
    p->k = base + L.kn;
    return true;
}

// Packed documents: the chunk table, built and checked on the device (which also
// resets the workspace's status word).  Dense rows: no table (kernels use the
// closed form), only the status word reset.
cudaError_t start_call(const Params &p, const gdn_desc *d, cudaStream_t s) {
    if (d->n_seqs > 0) return launch_build_chunks(p, s);
    return cudaMemsetAsync(p.hdr, 0, 16, s);
}

bool use_tc(const Problem &pb, bool bwd) {
    return pb.dtype == GDN_BF16 && tc_supported(pb) && (!bwd || tc_bwd_ready());
}

}  // namespace

bool encode_row_maps(Params &p, bool bwd) {
    if (p.BT <= 0) return true;  // nothing is loaded
    return encode_rows(&p.tm_q, p.q, p.BT, p.H, p.K) && encode_rows(&p.tm_k, p.k, p.BT, p.H, p.K) &&
           encode_rows(&p.tm_v, p.v, p.BT, p.H, p.V) &&
           (bwd || !p.o || encode_rows(&p.tm_o, p.o, p.BT, p.H, p.V)) &&
           (!bwd || (encode_rows(&p.tm_do, p.do_, p.BT, p.H, p.V) &&
                     encode_rows(&p.tm_dq, p.dq, p.BT, p.H, p.K) &&
                     encode_rows(&p.tm_dk, p.dk, p.BT, p.H, p.K) &&
                     encode_rows(&p.tm_dv, p.dv, p.BT, p.H, p.V)));
}

// Workspace layout.  The SIMT path (fp32) keeps fp32 per-(chunk, head)
// intermediates; the tensor-core path (bf16) has its own region.
Layout make_layout(const Problem &pb, bool bwd) {
    Layout L;
    std::memset(&L, 0, sizeof(L));
    size_t off = kAlign;  // WsHeader
    L.chunks = off;
    off += up(sizeof(ChunkInfo) * (size_t)(pb.NCmax > 0 ? pb.NCmax : 1));
    L.seq_first = off;
    off += up(sizeof(int32_t) * (size_t)(pb.N + 1));
    const size_t nch = (size_t)pb.NCmax * pb.H, f = sizeof(float);
    auto take = [&](size_t bytes) {
        size_t o = off;
        off += up(bytes > 0 ? bytes : 1);
        return o;
    };
    if (use_tc(pb, bwd)) {
        // bf16 tile images per (chunk, head); d_k = d_v = 128
        const size_t img64 = (size_t)kChunk * 128 * 2, img128 = (size_t)128 * 128 * 2;
        L.tW = take(nch * img64);
        L.tUt = take(nch * img64);
        L.tKd = take(nch * img64);
        L.tG = take(nch * kChunk * f);
        L.tS = take(nch * img128);
        L.tUT = take(nch * img64);
        L.tQg = take(nch * img64);                   // bf16 tile image of scale diag(gam) Q
        L.tP = take(nch * kChunk * kChunk * 2);      // bf16 tile image of P
        if (pb.P > 1) {  // piece scan: each piece's entering state, transition and offset
            const size_t units = (size_t)pb.N * pb.H * pb.P, st = (size_t)128 * 128 * f;
            L.tHin = take(units * st);
            L.tMp = take(units * st);
            L.tBp = take(units * st);
            if (bwd) {  // the same for the reverse chain
                L.tdHin = take(units * st);
                L.tTr = take(units * st);
                L.tBr = take(units * st);
            }
        }
        if (bwd) {
            L.tA = take(nch * kChunk * kChunk * 2);  // bf16 tile image of A
            L.tB = take(nch * kChunk * f);
            L.tdSn = take(nch * img128);
            L.tdUT = take(nch * img64);
        }
    } else {
        L.W = take(nch * kChunk * pb.K * f);
        L.Ut = take(nch * kChunk * pb.V * f);
        L.A = take(nch * kChunk * kChunk * f);
        L.U = take(nch * kChunk * pb.V * f);
        L.Hs = take(nch * pb.K * pb.V * f);
        if (bwd) {
            L.dUloc = take(nch * kChunk * pb.V * f);
            L.dU = take(nch * kChunk * pb.V * f);
            L.dHn = take(nch * pb.K * pb.V * f);
        }
        // one scratch slot per CTA of the chunk-parallel kernels (grid = min(NC*H, kSimtSlots))
        const size_t slots = nch < (size_t)kSimtSlots ? (nch > 0 ? nch : 1) : (size_t)kSimtSlots;
        L.scratch = take(slots * simt_scratch_floats(simt_tile_width((int)pb.K, (int)pb.V)) * f);
        if (pb.l2norm) {  // normalised copies of q and k, and their inverse norms
            const size_t rows = (size_t)pb.BT * pb.H, es = pb.dtype == GDN_BF16 ? 2 : 4;
            L.qn = take(rows * pb.K * es);
            L.kn = take(rows * pb.K * es);
            L.qinv = take(rows * f);
            L.kinv = take(rows * f);
        }
    }
    L.total = off;
    return L;
}

}  // namespace gdn

using namespace gdn;

extern "C" {

int gdn_version(void) { return 101; }

int gdn_chunk_size(void) { return kChunk; }

size_t gdn_fwd_workspace_size(const gdn_desc *desc) {
    Problem pb;
    if (describe(desc, &pb) != GDN_OK) return 0;
    return make_layout(pb, false).total;
}

size_t gdn_bwd_workspace_size(const gdn_desc *desc) {
    Problem pb;
    if (describe(desc, &pb) != GDN_OK) return 0;
    return make_layout(pb, true).total;
}

gdn_status gdn_fwd(const gdn_desc *desc, const void *q, const void *k, const void *v,
                   const float *g, const float *beta, const int32_t *cu_seqlens,
                   const int32_t *cu_seqlens_host, const float *h0, void *o, float *hT,
                   void *workspace, size_t workspace_bytes, void *stream) {
    Problem pb;
    gdn_status st = describe(desc, &pb);
    if (st != GDN_OK) return st;
    if (pb.BT > 0 && (!q || !k || !v || !g || !beta || !o)) return GDN_ERR_INVALID_ARG;
    for (const void *ptr : {q, k, v, (const void *)g, (const void *)beta, (const void *)h0,
                            (const void *)o, (const void *)hT})
        if (misaligned(ptr)) return GDN_ERR_ALIGNMENT;
    if (!workspace) return GDN_ERR_WORKSPACE;
    if (misaligned(workspace, kAlign)) return GDN_ERR_ALIGNMENT;
    const Layout L = make_layout(pb, false);
    if (workspace_bytes < L.total) return GDN_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if ((st = check_seqlens(desc, cu_seqlens, cu_seqlens_host, s, &pb)) != GDN_OK) return st;

    Params p = base_params(pb, desc, workspace, L, cu_seqlens);
    p.q = q;
    p.k = k;
    p.v = v;
    p.g = g;
    p.beta = beta;
    p.h0 = h0;
    p.o = o;
    p.hT = hT;
    const bool tc = use_tc(pb, false);
    if (tc && !encode_row_maps(p, false)) return GDN_ERR_CUDA;
    arm_planted_failure();
    if (start_call(p, desc, s) != cudaSuccess) return GDN_ERR_CUDA;
    if (!tc && pb.l2norm && !normalise_qk(pb, L, workspace, &p, s)) return GDN_ERR_CUDA;
    cudaError_t e = tc ? launch_tc_fwd(p, pb, s) : launch_simt_fwd(p, s);
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

gdn_status gdn_bwd(const gdn_desc *desc, const void *q, const void *k, const void *v,
                   const float *g, const float *beta, const int32_t *cu_seqlens,
                   const int32_t *cu_seqlens_host, const float *h0, const void *do_,
                   const float *dhT, void *dq, void *dk, void *dv, float *dg, float *dbeta,
                   float *dh0, void *workspace, size_t workspace_bytes, void *stream) {
    Problem pb;
    gdn_status st = describe(desc, &pb);
    if (st != GDN_OK) return st;
    if (pb.BT > 0 && (!q || !k || !v || !g || !beta || !do_ || !dq || !dk || !dv || !dg || !dbeta))
        return GDN_ERR_INVALID_ARG;
    for (const void *ptr : {q, k, v, (const void *)g, (const void *)beta, (const void *)h0, do_,
                            (const void *)dhT, (const void *)dq, (const void *)dk, (const void *)dv,
                            (const void *)dg, (const void *)dbeta, (const void *)dh0})
        if (misaligned(ptr)) return GDN_ERR_ALIGNMENT;
    if (!workspace) return GDN_ERR_WORKSPACE;
    if (misaligned(workspace, kAlign)) return GDN_ERR_ALIGNMENT;
    const Layout L = make_layout(pb, true);
    if (workspace_bytes < L.total) return GDN_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if ((st = check_seqlens(desc, cu_seqlens, cu_seqlens_host, s, &pb)) != GDN_OK) return st;

    Params p = base_params(pb, desc, workspace, L, cu_seqlens);
    p.q = q;
    p.k = k;
    p.v = v;
    p.g = g;
    p.beta = beta;
    p.h0 = h0;
    p.do_ = do_;
    p.dhT = dhT;
    p.dq = dq;
    p.dk = dk;
    p.dv = dv;
    p.dg = dg;
    p.dbeta = dbeta;
    p.dh0 = dh0;
    const bool tc = use_tc(pb, true);
    if (tc && !encode_row_maps(p, true)) return GDN_ERR_CUDA;
    arm_planted_failure();
    if (start_call(p, desc, s) != cudaSuccess) return GDN_ERR_CUDA;
    const bool pre = !tc && pb.l2norm;
    if (pre && !normalise_qk(pb, L, workspace, &p, s)) return GDN_ERR_CUDA;
    cudaError_t e = tc ? launch_tc_bwd(p, pb, s) : launch_simt_bwd(p, s);
    if (e == cudaSuccess && pre && pb.BT > 0) {  // gradients w.r.t. the raw q and k
        char *base = static_cast<char *>(workspace);
        const int64_t rows = pb.BT * pb.H;
        e = launch_l2norm_back(base + L.qn, reinterpret_cast<float *>(base + L.qinv), dq, rows,
                               (int)pb.K, p.bf16, s);
        if (e == cudaSuccess)
            e = launch_l2norm_back(base + L.kn, reinterpret_cast<float *>(base + L.kinv), dk,
                                   rows, (int)pb.K, p.bf16, s);
    }
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

gdn_status gdn_device_status(void *workspace, void *stream) {
    if (!workspace) return GDN_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    WsHeader h;
    if (cudaStreamSynchronize(s) != cudaSuccess) return GDN_ERR_CUDA;
    if (cudaMemcpy(&h, workspace, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess)
        return GDN_ERR_CUDA;
    if (h.status != 0) {
        const int32_t zero = 0;
        if (cudaMemcpy(workspace, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
            return GDN_ERR_CUDA;
    }
    return h.status == 0 ? GDN_OK : static_cast<gdn_status>(h.status);
}

const char *gdn_status_string(gdn_status status) {
    switch (status) {
    case GDN_OK: return "ok";
    case GDN_ERR_INVALID_ARG: return "invalid argument";
    case GDN_ERR_UNSUPPORTED: return "unsupported configuration";
    case GDN_ERR_ALIGNMENT: return "misaligned pointer";
    case GDN_ERR_WORKSPACE: return "workspace missing or too small";
    case GDN_ERR_CUDA: return "CUDA runtime error";
    case GDN_ERR_TIMEOUT: return "device-side wait timed out";
    }
    return "unknown status";
}

}  // extern "C"
