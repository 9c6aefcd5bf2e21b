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
//
// The scratch starts, like every workspace of this library, with the device error
// word (bytes 0..255); the kernels' arrival counters and partial sums follow.  Each
// call clears only what follows the error word, so a bounded wait that ran out in one
// call stays recorded until lora_linear_noalloc_check reads and clears it.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/lora_linear.h"

namespace {

constexpr size_t kNoallocScratchBytes = size_t(4) << 20;
constexpr size_t kErrBytes = 256;  // the error word's slot at the start of every workspace

// The scratch itself.  In host code this name is only a host-side stand-in for the
// symbol; the device address comes from cudaGetSymbolAddress, once per context.
__device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);

// The driver's cuCtxGetCurrent, looked up through the runtime (no link to libcuda).
CtxGetCurrentFn ctx_get_current() {
    static CtxGetCurrentFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(p);
    });
    return fn;
}

// Scratch addresses already looked up, keyed by CUDA context: the address of a
// __device__ array belongs to the context the module was loaded in, so a caller that
// switches between contexts of one device gets each context's own copy.
struct Entry {
    CUcontext ctx;
    void *addr;
};
constexpr int kMaxEntries = 64;
std::mutex g_noalloc_mu;
Entry g_entries[kMaxEntries];
int g_n_entries = 0;

// Device address of the scratch in the current context, looked up (and its error word
// cleared, on `stream`) on the first call made with that context current.
lora_status_t scratch_address(cudaStream_t stream, void **out) {
    CtxGetCurrentFn get = ctx_get_current();
    if (!get) return LORA_ERR_CUDA;
    CUcontext ctx = nullptr;
    if (get(&ctx) != CUDA_SUCCESS) return LORA_ERR_CUDA;
    void *p = nullptr;
    if (!ctx) {
        // No context current on this thread yet: the runtime call makes the current
        // device's primary context current (and resolves the address in it).
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return LORA_ERR_CUDA;
        if (get(&ctx) != CUDA_SUCCESS || !ctx) return LORA_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    for (int i = 0; i < g_n_entries; ++i)
        if (g_entries[i].ctx == ctx) {
            *out = g_entries[i].addr;
            return LORA_OK;
        }
    if (!p && (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p)) return LORA_ERR_CUDA;
    if (cudaMemsetAsync(p, 0, kErrBytes, stream) != cudaSuccess) return LORA_ERR_CUDA;
    if (g_n_entries < kMaxEntries) g_entries[g_n_entries++] = {ctx, p};
    *out = p;
    return LORA_OK;
}

}  // namespace

// In lora_linear.cu (same library, not exported).
extern "C" size_t lora_workspace_min(int op, int64_t M, int64_t d_in, int64_t d_out, int r);

extern "C" LORA_API lora_status_t lora_linear_fwd_noalloc(const uint16_t *x, const uint16_t *W,
                                                          const uint16_t *A, const uint16_t *B, uint16_t *h,
                                                          uint16_t *xa_save, int64_t M, int64_t d_in,
                                                          int64_t d_out, int r, float alpha, void *stream) {
    // the forward's smallest workspace: without room for the K-split hand-over buffer it
    // cuts a partial last wave along N, computing the same function
    const size_t need = lora_workspace_min(LORA_OP_FWD, M, d_in, d_out, r);
    if (need == 0) return LORA_ERR_INVALID_ARG;
    if (need > kNoallocScratchBytes) return LORA_ERR_WORKSPACE;  // problem too large for the fixed scratch
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    void *scratch = nullptr;
    lora_status_t s = scratch_address(st, &scratch);
    if (s != LORA_OK) return s;
    // The scratch keeps whatever the previous call left; the arrival counters must start
    // at zero, so clear the part this call uses, all but the error word.
    if (need > kErrBytes &&
        cudaMemsetAsync(static_cast<unsigned char *>(scratch) + kErrBytes, 0, need - kErrBytes, st) != cudaSuccess)
        return LORA_ERR_CUDA;
    return lora_linear_fwd(x, W, A, B, h, xa_save, M, d_in, d_out, r, alpha, scratch, kNoallocScratchBytes, stream);
}

extern "C" LORA_API lora_status_t lora_linear_noalloc_check(void *stream) {
    void *scratch = nullptr;
    lora_status_t s = scratch_address(static_cast<cudaStream_t>(stream), &scratch);
    if (s != LORA_OK) return s;
    return lora_linear_check(scratch, stream);
}

extern "C" LORA_API lora_status_t lora_linear_noalloc_selftest_timeout(uint32_t limit_us, void *stream) {
    void *scratch = nullptr;
    lora_status_t s = scratch_address(static_cast<cudaStream_t>(stream), &scratch);
    if (s != LORA_OK) return s;
    return lora_linear_selftest_timeout(scratch, kNoallocScratchBytes, limit_us, stream);
}
