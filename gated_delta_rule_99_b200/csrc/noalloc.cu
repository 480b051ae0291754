// gdn_fwd_noalloc: the forward for callers that cannot allocate device memory.
//
// Some callers own no allocator they may use at call time: a serving process
// that reserved all of HBM in a fixed pool at start-up and may not call
// cudaMalloc on the request path (an allocation there stalls the device and
// fragments the pool), or a plugin that is handed only its input and output
// buffers.  This entry point takes no workspace: its scratch is a fixed array
// compiled into the library, which every device that loads the library holds
// until the process exits.
#include <mutex>

#include "gdn_internal.cuh"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[GDN_NOALLOC_MAX_WORKSPACE];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_addr[kMaxDevices] = {};

}  // namespace

extern "C" gdn_status gdn_fwd_noalloc(const gdn_desc *desc, const void *q, const void *k,
                                      const void *v, const float *g, const float *beta,
                                      const int32_t *cu_seqlens, const int32_t *cu_seqlens_host,
                                      const float *h0, void *o, float *hT, void *stream) {
    const size_t need = gdn_fwd_workspace_size(desc);
    if (need == 0) {
        // same status gdn_fwd gives for this descriptor
        return gdn_fwd(desc, q, k, v, g, beta, cu_seqlens, cu_seqlens_host, h0, o, hT, nullptr,
                       0, stream);
    }
    if (need > (size_t)GDN_NOALLOC_MAX_WORKSPACE) return GDN_ERR_WORKSPACE;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return GDN_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return GDN_ERR_UNSUPPORTED;
    void *scratch = nullptr;
    {
        // First call on a device: look up the array's device address (host
        // code cannot use the symbol itself), with that device current.
        std::lock_guard<std::mutex> lock(g_mu);
        if (!g_scratch_addr[dev]) {
            void *addr = nullptr;
            if (cudaGetSymbolAddress(&addr, g_noalloc_scratch) != cudaSuccess || !addr)
                return GDN_ERR_CUDA;
            g_scratch_addr[dev] = addr;
        }
        scratch = g_scratch_addr[dev];
    }
    return gdn_fwd(desc, q, k, v, g, beta, cu_seqlens, cu_seqlens_host, h0, o, hT, scratch,
                   (size_t)GDN_NOALLOC_MAX_WORKSPACE, stream);
}

// The status word heads the scratch (it is gdn_fwd's workspace header there),
// so it is read and cleared through the symbol itself: no address lookup, and
// a device that never ran gdn_fwd_noalloc reads its zero-initialised word.
extern "C" gdn_status gdn_fwd_noalloc_status(void *stream) {
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return GDN_ERR_CUDA;
    int32_t status = 0;
    if (cudaMemcpyFromSymbol(&status, g_noalloc_scratch, sizeof(status)) != cudaSuccess)
        return GDN_ERR_CUDA;
    if (status != 0) {
        const int32_t zero = 0;
        if (cudaMemcpyToSymbol(g_noalloc_scratch, &zero, sizeof(zero)) != cudaSuccess)
            return GDN_ERR_CUDA;
    }
    return status == 0 ? GDN_OK : static_cast<gdn_status>(status);
}
