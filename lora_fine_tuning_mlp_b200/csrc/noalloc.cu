// lora_mlp_forward_noalloc: the forward pass with its scratch workspace in a
// fixed device array owned by this library, for callers that cannot allocate
// device memory themselves (see include/lora_mlp.h for who and why).
//
// The array lives in this translation unit, so it belongs to a module of its
// own.  Under lazy module loading (CUDA_MODULE_LOADING=LAZY, the default)
// CUDA loads that module, and reserves the array on a device, only when this
// entry point is first used there; with CUDA_MODULE_LOADING=EAGER every
// context that loads the library reserves it.  It is kept until the process
// exits.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "lora_mlp.h"

namespace {

constexpr int kMaxDevices = 64;

// Every call on a device shares this one array; nothing here clears it.  The
// forward pass itself zeroes the part that must start at zero (its per-tile
// counters) at the start of every call.
static __device__ __align__(256) unsigned char g_noalloc_scratch[LORA_MLP_NOALLOC_SCRATCH_BYTES];

std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices];

// Device address of g_noalloc_scratch on the current device.  In host code the
// array's name only stands for the symbol; its device address has to be asked
// for, once per device, with that device current.
int scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LORA_MLP_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_scratch_ptr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return LORA_MLP_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return LORA_MLP_OK;
}

}  // namespace

extern "C" int lora_mlp_forward_noalloc(const lora_mlp_shape* shape, const lora_mlp_weights* w, const void* X,
                                        void* out, void* g, void* u, void* saved, void* stream) {
    size_t need = 0;
    const int rc = lora_mlp_sizes(shape, &need, nullptr, nullptr);
    if (rc != LORA_MLP_OK) return rc;
    if (need > LORA_MLP_NOALLOC_SCRATCH_BYTES) return LORA_MLP_ERR_WORKSPACE_TOO_SMALL;
    void* scratch = nullptr;
    const int rs = scratch_address(&scratch);
    if (rs != LORA_MLP_OK) return rs;
    return lora_mlp_forward(shape, w, X, out, g, u, saved, scratch, LORA_MLP_NOALLOC_SCRATCH_BYTES, stream);
}
