// ssd_fwd_no_alloc: the SSD forward for callers that cannot allocate device
// memory. Some hosts own every device allocation themselves and hand a
// library nothing but the input and output buffers (plugin interfaces of
// inference engines, custom pool allocators the library cannot reach), and
// some call paths cannot afford cudaMalloc, which may synchronize the whole
// device. For them this entry point takes its scratch space from one
// file-scope device array instead of a caller-provided workspace.
//
// The array is fixed at kNoAllocScratchBytes; every GPU that loads the library
// reserves that much memory until the process exits. Shapes whose workspace
// (ssd_fwd_workspace_size) does not fit are rejected with SSD_ERR_UNSUPPORTED.
#include <cuda_runtime.h>

#include <cstdio>

#include "ssd.h"
#include "ssd_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;  // 64 MiB

// Device-side scratch shared by every ssd_fwd_no_alloc call on a device. In
// host code this name is only a stand-in for the symbol, never an address a
// kernel may be given: the device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_ssd_scratch[kNoAllocScratchBytes];

// The device address of the scratch array on the current device, looked up on
// every call (a host-side symbol lookup, nothing enqueued), so that it follows
// the current device and a context recreated after cudaDeviceReset. Returns
// nullptr (and a detail message) on failure.
void* scratch_for_current_device() {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_ssd_scratch);
    if (e != cudaSuccess || !p) {
        char msg[160];
        snprintf(msg, sizeof(msg), "ssd_fwd_no_alloc: cudaGetSymbolAddress failed: %s",
                 cudaGetErrorString(e));
        ssd::set_error_detail(msg);
        return nullptr;
    }
    return p;
}

}  // namespace

extern "C" ssd_status_t ssd_fwd_no_alloc(const ssd_shape_t* shape, const void* x, const float* dt,
                                         const float* A, const void* B, const void* C,
                                         const float* D, const float* initial_states, void* y,
                                         float* final_states, void* stream) {
    size_t need = 0;
    ssd_status_t st = ssd_fwd_workspace_size(shape, &need);
    if (st != SSD_OK) return st;
    if (need > kNoAllocScratchBytes) {
        char msg[200];
        snprintf(msg, sizeof(msg),
                 "ssd_fwd_no_alloc: this shape needs %zu bytes of scratch, more than the "
                 "%zu-byte static scratch array; use ssd_fwd with a workspace",
                 need, kNoAllocScratchBytes);
        ssd::set_error_detail(msg);
        return SSD_ERR_UNSUPPORTED;
    }
    void* scratch = scratch_for_current_device();
    if (!scratch) return SSD_ERR_CUDA;
    // ssd_fwd overwrites every workspace byte it reads before reading it, so
    // nothing left in the array by an earlier call needs clearing here.
    return ssd_fwd(shape, x, dt, A, B, C, D, initial_states, y, final_states, scratch,
                   kNoAllocScratchBytes, stream);
}

extern "C" ssd_status_t ssd_fwd_no_alloc_check(const ssd_shape_t* shape, void* stream) {
    void* scratch = scratch_for_current_device();
    if (!scratch) return SSD_ERR_CUDA;
    // the last ssd_fwd_no_alloc on this device left its status words where any
    // ssd_fwd call on a workspace leaves them: at the start of the scratch array
    return ssd_fwd_check(shape, scratch, kNoAllocScratchBytes, stream);
}
