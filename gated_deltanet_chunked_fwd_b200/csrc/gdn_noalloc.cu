// gdn_noalloc.cu -- gdn_chunk_fwd_noalloc: the forward without a caller-provided
// workspace, for callers that cannot allocate device memory.
//
// Some callers have no way to call cudaMalloc: code that runs inside a framework
// plugin or an inference server whose memory is pooled and frozen after start-up,
// or a runtime that forbids allocation on the request path.  For them this entry
// point runs the CUDA-core forward (the portable kernels) with its scratch in a
// fixed, file-scope device array instead of a workspace argument.  The array is part of the library image: every GPU that
// loads libgdn.so holds it until the process exits.
#include <mutex>

#include "gdn_internal.cuh"

namespace gdn {
namespace {

constexpr size_t kNoAllocScratchBytes = GDN_NOALLOC_SCRATCH_BYTES;

// The scratch itself.  In host code `g_noalloc_scratch` names a host-side stand-in,
// not a device address: kernels must be given the address that
// cudaGetSymbolAddress reports for the current device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once per
// device (with that device current) and cached.
gdn_status scratch_for_current_device(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GDN_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_scratch_ptr[dev]) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return GDN_ERR_CUDA;
        g_scratch_ptr[dev] = ptr;
    }
    *out = g_scratch_ptr[dev];
    return GDN_OK;
}

}  // namespace
}  // namespace gdn

using namespace gdn;

extern "C" {

gdn_status gdn_chunk_fwd_noalloc(const gdn_fwd_args* args, void* stream) {
    if (!args) return GDN_ERR_INVALID_ARG;
    gdn_fwd_args a = *args;
    a.flags |= GDN_FLAG_PORTABLE;  // the CUDA-core kernels
    FwdPlan plan;
    gdn_status st = plan_fwd(&a, &plan);
    if (st) return st;
    if (plan.total > kNoAllocScratchBytes) return GDN_ERR_TOO_LARGE;
    void* scratch = nullptr;
    if ((st = scratch_for_current_device(&scratch))) return st;
    // The portable kernels write every scratch element before reading it, so
    // nothing has to be cleared between calls.
    return gdn_chunk_fwd(&a, scratch, kNoAllocScratchBytes, stream);
}

}  // extern "C"
