// noalloc.cu -- the forward pass for callers that cannot allocate device memory.
//
// lora_linear_fwd needs a caller-provided scratch workspace (split-K partials and
// arrival counters of the x.A^T prologue, and room for s.xa when it is not saved).
// Some callers have no way to provide one: a plugin running inside a host framework
// that owns every device allocation and hands out only the tensors of the op, or a
// service that pre-plans its whole device-memory budget at start-up and forbids
// allocation afterwards (cudaMalloc can synchronise the device and fragments the
// heap).  This file gives them lora_linear_fwd_noalloc, which takes the same inputs
// and outputs but no workspace: its scratch is a fixed 4 MiB array in device global
// memory that every GPU loading this library holds until the process exits.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/lora_linear.h"

namespace {

constexpr size_t kNoallocScratchBytes = size_t(4) << 20;

// The scratch itself.  In host code this name is only a host-side stand-in for the
// symbol; the device address comes from cudaGetSymbolAddress (once per device).
__device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

std::mutex g_noalloc_mu;
void *g_noalloc_addr[64] = {};

// Device address of the scratch on the current device, looked up on the first call
// made with that device current.
lora_status_t scratch_address(void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return LORA_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return LORA_ERR_CUDA;
        g_noalloc_addr[dev] = p;
    }
    *out = g_noalloc_addr[dev];
    return LORA_OK;
}

}  // namespace

extern "C" LORA_API lora_status_t lora_linear_fwd_noalloc(const uint16_t *x, const uint16_t *W,
                                                          const uint16_t *A, const uint16_t *B, uint16_t *h,
                                                          uint16_t *xa_save, int64_t M, int64_t d_in,
                                                          int64_t d_out, int r, float alpha, void *stream) {
    const size_t need = lora_linear_workspace_size(LORA_OP_FWD, M, d_in, d_out, r);
    if (need == 0) return LORA_ERR_INVALID_ARG;
    if (need > kNoallocScratchBytes) return LORA_ERR_WORKSPACE;  // problem too large for the fixed scratch
    void *scratch = nullptr;
    lora_status_t st = scratch_address(&scratch);
    if (st != LORA_OK) return st;
    // The scratch keeps whatever the previous call left; the counters and the error
    // word must start at zero, so clear the part this call uses.
    if (cudaMemsetAsync(scratch, 0, need, static_cast<cudaStream_t>(stream)) != cudaSuccess) return LORA_ERR_CUDA;
    return lora_linear_fwd(x, W, A, B, h, xa_save, M, d_in, d_out, r, alpha, scratch, kNoallocScratchBytes, stream);
}
