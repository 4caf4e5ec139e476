// fvattn_sparse_attn_noalloc: block-sparse attention for callers that
// cannot allocate device memory.
//
// fvattn_sparse_attn takes its scratch (the longest-first work list: per-head
// item order, head costs, head order and the item counter) from a workspace
// the caller allocates.  Some callers cannot do that: a plugin running inside
// a host framework whose allocator owns all device memory, a C program that
// links only this library and has no device allocator of its own, or code
// that must not call cudaMalloc (or fail on it) once it is running.  This
// entry point needs no workspace: its scratch is one file-scope device array
// of FVATTN_NOALLOC_SCRATCH_BYTES that every GPU loading the library holds
// until the process exits.
#include <mutex>

#include "common.cuh"

namespace fv {

// Work-list scratch shared by every call of the entry point on a device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[FVATTN_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch per device ordinal, looked up once
// per device (with that device current) on the first call.
constexpr int kMaxDevices = 64;
static void* g_scratch_ptr[kMaxDevices] = {nullptr};
static std::mutex g_scratch_mutex;

static int scratch_on_current_device(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FVATTN_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return FVATTN_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        // In host code g_noalloc_scratch names a host-side stand-in; the
        // device address must come from the runtime.
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return FVATTN_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return FVATTN_OK;
}

}  // namespace fv

using namespace fv;

extern "C" int fvattn_sparse_attn_noalloc(const fvattn_geom* gp, const void* q_t, const void* k_t, const void* v_t,
                                          const int32_t* kv_idx, const int32_t* kv_cnt, float scale, void* o_t,
                                          unsigned long long* sm_stats, fvattn_stream_t stream) {
    if (!gp) return FVATTN_ERR_INVALID;
    const size_t need = fvattn_attn_workspace_size(gp);
    if (need == 0 || need > static_cast<size_t>(FVATTN_NOALLOC_SCRATCH_BYTES)) return FVATTN_ERR_UNSUPPORTED;
    void* scratch = nullptr;
    const int rc = scratch_on_current_device(&scratch);
    if (rc != FVATTN_OK) return rc;
    // The work-list kernels rewrite every scratch byte the attention kernel
    // reads (item order, head costs, head order) and reset the item counter
    // to zero before each launch, so nothing from an earlier call is reused.
    return fvattn_sparse_attn(gp, q_t, k_t, v_t, kv_idx, kv_cnt, scale, o_t, sm_stats, scratch,
                              static_cast<size_t>(FVATTN_NOALLOC_SCRATCH_BYTES), stream);
}
