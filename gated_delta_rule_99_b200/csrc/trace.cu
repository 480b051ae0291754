// Optional per-launch CUDA-event tracing (see gdn_trace_install in gdn.h).
#include "gdn_internal.cuh"

namespace gdn {
namespace {
thread_local gdn_trace *g_trace = nullptr;
thread_local bool g_open = false;
// testing hooks (gdn_set_wait_limit, gdn_set_test_hook)
thread_local uint32_t g_wait_limit = 0;
thread_local int32_t g_hook = 0;
thread_local bool g_fail_armed = false;

const char *const kNames[kKernelCount] = {
    "build_chunks", "simt_prep", "simt_state_fwd", "simt_out", "simt_duloc", "simt_state_bwd",
    "simt_grads", "tc_prep", "tc_state_fwd", "tc_out", "tc_chains", "tc_grads", "tc_prep_local", "decode", "tc_piece_a", "tc_piece_scan", "tc_piece_c", "l2norm", "l2norm_back"};
}  // namespace

void trace_before(int32_t id, cudaStream_t stream) {
    gdn_trace *t = g_trace;
    g_open = false;
    if (!t) return;
    if (t->count >= t->capacity) {
        ++t->dropped;
        return;
    }
    t->kernel_ids[t->count] = id;
    if (cudaEventRecord(static_cast<cudaEvent_t>(t->events[2 * t->count]), stream) != cudaSuccess) {
        cudaGetLastError();  // a bad event must not look like a failed launch
        ++t->dropped;
        return;
    }
    g_open = true;
}

void trace_after(cudaStream_t stream) {
    gdn_trace *t = g_trace;
    if (!t || !g_open) return;
    if (cudaEventRecord(static_cast<cudaEvent_t>(t->events[2 * t->count + 1]), stream) !=
        cudaSuccess) {
        cudaGetLastError();
        ++t->dropped;
    } else {
        ++t->count;
    }
    g_open = false;
}

uint32_t call_wait_limit() { return g_wait_limit ? g_wait_limit : kWaitLimit; }

int32_t call_test_hook() { return g_hook; }

void arm_planted_failure() { g_fail_armed = g_hook == GDN_TEST_FAIL_LAUNCH; }

bool take_planted_failure() {
    const bool f = g_fail_armed;
    g_fail_armed = false;
    return f;
}

}  // namespace gdn

extern "C" {

void gdn_set_wait_limit(uint32_t polls) { gdn::g_wait_limit = polls; }

void gdn_set_test_hook(int32_t hook) {
    gdn::g_hook = hook;
    gdn::g_fail_armed = false;
}

void gdn_trace_install(gdn_trace *trace) {
    gdn::g_trace = trace;
    gdn::g_open = false;
}

const char *gdn_kernel_name(int32_t id) {
    return (id >= 0 && id < gdn::kKernelCount) ? gdn::kNames[id] : "?";
}

}  // extern "C"
