// fa_static_workspace.cu -- fa_fwd_static_workspace: the key-split forward
// with its scratch in a fixed device array instead of a caller-owned
// workspace, so the call allocates nothing at all.
//
// The array is a file-scope __device__ variable of this translation unit
// (its own module): FA_STATIC_WORKSPACE_BYTES of device memory that comes
// with the module, not from an allocator.  Its address is looked up once per
// device with cudaGetSymbolAddress (the first call on that device, with the
// device current) and cached; every call on the device then passes that
// pointer to the split pass and the merge as their workspace.
//
// Nothing in the array has to start at zero: the split pass writes every
// (split, row) partial that the merge reads in the same call.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "fa.h"
#include "fa_internal.h"

namespace {

constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_scratch[FA_STATIC_WORKSPACE_BYTES];

std::mutex g_mu;
void *g_scratch_ptr[kMaxDevices] = {};

// Address of g_scratch on the current device (looked up on first use).
fa_status scratch_for_current_device(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || p == nullptr) {
            cudaGetLastError();  // clear the error so that it does not surface in a later call
            return FA_ERR_CUDA;
        }
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return FA_OK;
}

}  // namespace

extern "C" {

fa_status fa_fwd_static_workspace(const fa_fwd_params *p, void *stream) {
    // order: argument checks (no CUDA call), the size limit, the device, then
    // the array's address
    fa_status st = fa_detail::validate_args(p);
    if (st != FA_OK) return st;
    if ((long long)p->B * p->H * p->N == 0) return FA_OK;
    fa_fwd_params c = *p;
    c.workspace = nullptr;
    c.workspace_bytes = 0;
    if (c.num_splits > 1) {
        const size_t need = fa_fwd_workspace_bytes(&c);
        if (need > (size_t)FA_STATIC_WORKSPACE_BYTES) return FA_ERR_WORKSPACE_LIMIT;
        if ((st = fa_detail::probe_current_device()) != FA_OK) return st;
        void *ws = nullptr;
        if ((st = scratch_for_current_device(&ws)) != FA_OK) return st;
        c.workspace = ws;
        c.workspace_bytes = (size_t)FA_STATIC_WORKSPACE_BYTES;
    }
    return fa_fwd_ex(&c, stream);
}

}  // extern "C"
