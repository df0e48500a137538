// tbik_logprob_noalloc: the fused lm_head -> log-softmax -> target logprob
// (tensor-core mode) for callers that cannot allocate device memory.
//
// Some callers have no way to obtain a device workspace: code that must not
// call cudaMalloc (for instance because the process is in the middle of a
// stream capture, or runs under an allocator that forbids side allocations),
// or plain C callers that link this library without any device-memory
// allocator of their own.  This entry point runs the same kernels as
// tbik_logprob but carves its scratch out of a fixed, file-scope device array
// instead of a caller-provided workspace.  It never allocates or frees memory.
//
// Cost of the array: TBIK_NOALLOC_SCRATCH_BYTES (32 MiB) of device memory on
// every GPU that loads this library, held until the process exits.
#include <cuda_runtime.h>

#include <mutex>

#include "tbik.h"

// Defined in tbik_api.cu (library-internal): tbik_logprob's planning status for
// these arguments and, when TBIK_OK, its workspace bytes.
tbik_status tbik_logprob_plan_status(int M, int V, int H, int T, int leaf, unsigned mode, size_t* bytes);

namespace {

// The shared scratch area.  In host code this name is only a host-side stand-in
// for the device symbol; its device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_noalloc_scratch[TBIK_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Set-up, once per device, with that device current: look up the device
// address of the scratch array.  The address is kept for the life of the
// process; a cudaDeviceReset (which unloads the module and may place the array
// elsewhere when it is loaded again) makes it stale, so this entry point is not
// for use across a device reset.
tbik_status scratch_address(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TBIK_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return TBIK_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return TBIK_OK;
}

}  // namespace

extern "C" TBIK_API tbik_status tbik_logprob_noalloc(const uint16_t* hidden, const uint16_t* W_lm,
                                                     const int32_t* targets, float* out, int M, int V, int H, int T,
                                                     int leaf, unsigned mode, void* stream) {
    if (!(mode & TBIK_TC) || (mode & TBIK_EXACT)) return TBIK_ERR_ARG;
    size_t need = 0;
    tbik_status st = tbik_logprob_plan_status(M, V, H, T, leaf, mode, &need);
    if (st != TBIK_OK) return st;  // the code tbik_logprob would return
    if (need > (size_t)TBIK_NOALLOC_SCRATCH_BYTES) return TBIK_ERR_WORKSPACE;
    void* ws = nullptr;
    st = scratch_address(&ws);
    if (st != TBIK_OK) return st;
    // Every region of the scratch that the kernels read is written earlier in
    // the same call, so nothing has to be cleared between calls.
    return tbik_logprob(hidden, W_lm, targets, out, M, V, H, T, leaf, mode, ws, (size_t)TBIK_NOALLOC_SCRATCH_BYTES,
                        stream);
}
