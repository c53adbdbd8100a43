// gdn_noalloc.cu -- gdn_chunk_fwd_noalloc: the forward without a caller-provided
// workspace, for callers that cannot allocate device memory.
//
// Some callers have no way to call cudaMalloc: code that runs inside a framework
// plugin or an inference server whose memory is pooled and frozen after start-up,
// or a runtime that forbids allocation on the request path.  For them this entry
// point runs the CUDA-core forward (the portable kernels) with its scratch in a
// fixed, file-scope device array instead of a workspace argument.  The array is part of the library image: every GPU that
// loads libgdn.so holds it until the process exits.
#include <cuda.h>

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

// Which CUDA context the cached address belongs to: the driver's per-process unique context
// id (a reset device gets a new primary context, and the array a new address).
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

bool current_context_id(unsigned long long* id) {
    static CtxGetCurrentFn get_cur = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static bool resolved = false;
    if (!resolved) {  // under g_mutex
        void* f1 = nullptr;
        void* f2 = nullptr;
        cudaDriverEntryPointQueryResult q1, q2;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1) == cudaSuccess &&
            q1 == cudaDriverEntryPointSuccess &&
            cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2) == cudaSuccess &&
            q2 == cudaDriverEntryPointSuccess) {
            get_cur = (CtxGetCurrentFn)f1;
            get_id = (CtxGetIdFn)f2;
        }
        resolved = true;
    }
    CUcontext ctx = nullptr;
    if (!get_cur || !get_id || get_cur(&ctx) != CUDA_SUCCESS || !ctx) return false;
    return get_id(ctx, id) == CUDA_SUCCESS;
}

struct ScratchEntry {
    void* ptr;
    unsigned long long ctx_id;
};
std::mutex g_mutex;
ScratchEntry g_scratch[kMaxDevices] = {};

// Device address of the scratch array on the current device.  It is looked up (with the
// device current) on the first call in each CUDA context of a device and cached; a call in a
// new context of that device (after cudaDeviceReset, say) looks it up again.
gdn_status scratch_for_current_device(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GDN_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mutex);
    unsigned long long id = 0;
    const bool have_id = current_context_id(&id);
    ScratchEntry& e = g_scratch[dev];
    if (!e.ptr || !have_id || e.ctx_id != id) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return GDN_ERR_CUDA;
        // the lookup made the device's primary context current if none was
        e.ptr = ptr;
        e.ctx_id = current_context_id(&id) ? id : 0;
    }
    *out = e.ptr;
    return GDN_OK;
}

}  // namespace
}  // namespace gdn

using namespace gdn;

extern "C" {

gdn_status gdn_chunk_fwd_noalloc(const gdn_fwd_args* args, void* stream) {
    // the caller's struct is read only after its declared size and version say it is whole
    if (!args || args->struct_size < sizeof(gdn_fwd_args) || args->abi_version != GDN_ABI_VERSION)
        return GDN_ERR_INVALID_ARG;
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
