/*
 * lora_linear.h -- C ABI of the fused LoRA linear layer for NVIDIA B200 (sm_100a).
 *
 * The layer (row-major, tokens are rows):
 *   forward   h  = x.W^T + s.(x.A^T).B^T                     s = alpha / r
 *   backward  dX = dY.W + s.(dY.B).A
 *             dB = s.dY^T.(x.A^T)          dA = s.(dY.B)^T.x
 * with a frozen weight W (no dW).  The forward is the low-rank update of a frozen
 * weight, h = W x + B (A x), of page "UnSloth加速库集成：编译级优化带来的性能飞跃",
 * section 为什么标准LoRA会慢？, written for row vectors with the scale s on the update.
 * The backward is its chain rule; page "ms-swift高效微调组合：LoRA+UnSloth提速实践",
 * section 1.2 (梯度计算绕过Autograd) prints the two weight gradients in a shortened
 * form, and page "Unsloth — 微调 2-5x 加速", section 核心要点 (数学化简反向公式) fixes
 * the association A.(B.dY) that never forms the d_out x d_in update.
 *
 * Shapes and layouts (all row-major, contiguous, element strides = the last dim):
 *   x [M, d_in]   W [d_out, d_in] (torch.nn.Linear.weight)   A [r, d_in] (lora_A)
 *   B [d_out, r] (lora_B)   h, dY [M, d_out]   dX [M, d_in]   dA [r, d_in]   dB [d_out, r]
 *   xa_save [M, r] holds bf16(s . x.A^T), written by the forward, read by the backward.
 * Element types: "bf16" arguments are bfloat16 values passed as their 16-bit patterns
 * (uint16_t); dA and dB are fp32.  The 4-bit weight of the *_q4 entry points is
 * Wq [d_out, d_in/2] (uint8, two codes per byte along d_in, low nibble = even index)
 * with Wscale [d_out, d_in/64] (bf16): w'[n,k] = (q[n,k] - 8) * Wscale[n, k/64] / 7.
 *
 * Conventions shared by every entry point:
 *   - Pointers are device pointers (cudaMalloc or equivalent) on the current device.
 *     The caller owns every buffer, including the workspace.  The library never
 *     allocates, frees or synchronises the stream; all work is enqueued on `stream`
 *     (a cudaStream_t passed as void*; NULL = the legacy default stream) and the
 *     call returns without waiting.
 *   - Outputs are overwritten, never accumulated into.  Inputs and outputs must not
 *     alias.  Calls on distinct streams with distinct workspaces may run concurrently.
 *   - Validation happens before any launch; on a validation error (INVALID_ARG,
 *     MISALIGNED, WORKSPACE, UNSUPPORTED) nothing is enqueued.  LORA_ERR_CUDA from a
 *     launch may leave the call's earlier kernels enqueued; their outputs are then
 *     undefined.
 *     Required: non-null required pointers; every pointer 16-byte aligned;
 *     1 <= M <= 2^30; d_in and d_out multiples of 8 in 8 .. 2^24, with
 *     ceil(M/128) * ceil(max(d_in, d_out)/128) <= 2^31 - 1 (32-bit tile counts: only
 *     an output of more than 2^45 elements reaches it); 1 <= r <= 256 with r % 8 == 0; alpha finite;
 *     for *_q4 and *_nf4 also d_in % 64 == 0; for *_fp8 d_in % 16 == 0.
 *   - The workspace must hold lora_linear_workspace_size(op, ...) bytes (the bf16
 *     forward also runs in less, down to the size without its K-split hand-over buffer,
 *     cutting its last wave along N instead: see lora_plan_t.fwd_tail), be 256-byte
 *     aligned, be zero-filled before its first use, and must not be used by two calls
 *     that may run at the same time.  Every call that completes leaves the workspace's
 *     arrival counters at zero again, so a workspace is zeroed once, not per call
 *     (after LORA_ERR_TIMEOUT the caller zero-fills it again).
 *   - Consecutive kernels are launched with programmatic dependent launch: each waits
 *     for its predecessor in the stream before touching global memory, so stream
 *     order is preserved; only launch latency and set-up overlap.
 *   - The device must be compute capability 10.0 (B200); otherwise
 *     LORA_ERR_UNSUPPORTED is returned and nothing runs.  The *_q4, *_fp8 and *_nf4
 *     entry points also need two-SM clusters (CTA pairs); without them they return
 *     LORA_ERR_UNSUPPORTED.
 *   - Device-side waits are bounded.  A wait that runs out sets an error word in the
 *     workspace and the kernels return early; lora_linear_check() reports it.
 *   - No C++ exception crosses this interface.
 *   - Two environment variables, read at each call, exist for measurement and tests:
 *     LORA_LINEAR_PAIR=0 runs the main GEMMs on single SMs instead of CTA pairs (the
 *     4-bit entry points then return LORA_ERR_UNSUPPORTED); LORA_LINEAR_PDL=0 launches
 *     without programmatic dependent launch.  Either way the results meet the same bounds.
 */
#ifndef LORA_LINEAR_H
#define LORA_LINEAR_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LORA_API __attribute__((visibility("default")))
#else
#define LORA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    LORA_OK = 0,
    LORA_ERR_INVALID_ARG = 1,  /* null pointer, bad shape, r or alpha out of range */
    LORA_ERR_MISALIGNED = 2,   /* a pointer is not 16-byte (workspace: 256-byte) aligned */
    LORA_ERR_UNSUPPORTED = 3,  /* no sm_100 device, or a shape this build does not cover */
    LORA_ERR_WORKSPACE = 4,    /* workspace missing or smaller than required */
    LORA_ERR_CUDA = 5,         /* a CUDA runtime/driver call failed (launch, tensor map) */
    LORA_ERR_TIMEOUT = 6       /* a device-side bounded wait ran out (see lora_linear_check) */
} lora_status_t;

typedef enum {
    LORA_OP_FWD = 0,
    LORA_OP_BWD = 1,
    LORA_OP_FWD_Q4 = 2,
    LORA_OP_BWD_Q4 = 3,
    LORA_OP_FWD_FP8 = 4,
    LORA_OP_BWD_FP8 = 5,
    LORA_OP_FWD_NF4 = 6,
    LORA_OP_BWD_NF4 = 7
} lora_op_t;

/*
 * Plans.  How a layer of a given shape splits its work: which kernels compute the
 * rank-r side products, how their CTAs are grouped, and how the main GEMMs end their
 * last wave.  The library chooses a plan per shape from fixed rules and a streaming
 * cost model; lora_linear_set_plan overrides any part of it for one shape, which is
 * how a tuner that times candidate plans on the device installs its choice (page
 * "UnSloth加速库集成：编译级优化带来的性能飞跃", section 技术三: probe the kernel
 * configuration per GPU, sequence length and rank, and cache the result).  Every
 * plan computes the same function; results differ only in the order of fp32 sums.
 * A field of 0 means "the library's choice".
 */
typedef struct {
    int32_t side_fwd;   /* s.xa: 1 the cluster-reduction side kernel (r <= 64), 2 the split-K kernel */
    int32_t side_bwd;   /* s.g with dB, then dA: 1 the side kernels (one pass over dY; r <= 32),
                           2 the split-K kernels (s.g, then dB and dA in one launch) */
    int32_t xa_cluster; /* side s.xa: CTAs per cluster, 1, 2 or 4 (they split d_in) */
    int32_t g_cluster;  /* side s.g + dB: CTAs per cluster, 1, 2 or 4 (they split d_out) */
    int32_t g_group;    /* side s.g + dB: 128-token blocks per round, 1..6, with g_group * r <= 64 */
    int32_t da_cluster; /* side dA: CTAs per cluster, 1, 2 or 4 (they split the tokens) */
    int32_t fwd_tail;   /* forward main GEMM: 1 a partial last wave is cut along N, 2 it is not,
                           3 (bf16 weight; the library's choice there) each of its tiles is cut
                           along K into two halves on two CTA pairs, the first handing its fp32
                           accumulator to the second through the workspace (a workspace below
                           lora_linear_workspace_size's figure but at least the rest cuts along N) */
    int32_t dx_overlap; /* backward: 1 dA (and dB) start beside the dX GEMM's last wave, whose tiles
                           stay whole (the library's choice); 2 they follow the dX GEMM, whose
                           last wave is cut along N where it can be; 3 (bf16 weight) they follow
                           it, its last wave cut along K as fwd_tail 3 describes */
    int32_t splitk[4];  /* split-K kernels: K splits (1 .. 64) of s.xa, s.g, dB and dA */
} lora_plan_t;

/* Install `plan` for every operation on layers of exactly this shape (M, d_in, d_out,
 * r), replacing any earlier one; NULL removes it.  Fields out of range, or a side kernel
 * asked for a rank it does not take, give LORA_ERR_INVALID_ARG / LORA_ERR_UNSUPPORTED
 * and change nothing.  The workspace size follows the plan: call
 * lora_linear_workspace_size again after changing it.  Host-only and thread-safe (at
 * most 256 shapes hold a plan); takes effect for calls made after it returns. */
LORA_API lora_status_t lora_linear_set_plan(int64_t M, int64_t d_in, int64_t d_out, int r, const lora_plan_t *plan);

/* The plan `op` uses for this shape: the override's fields and the library's choice for
 * the rest, filled in for the kernels the plan runs (fields of kernels it does not run,
 * e.g. the split-K splits when the side kernels take the products, are 0).  Host-only;
 * LORA_ERR_INVALID_ARG for invalid sizes or op. */
LORA_API lora_status_t lora_linear_get_plan(int op, int64_t M, int64_t d_in, int64_t d_out, int r,
                                            lora_plan_t *plan);

/* Bytes of workspace the given operation needs for these sizes (0 if the sizes are
 * invalid).  Pure host function; needs no device. */
LORA_API size_t lora_linear_workspace_size(int op, int64_t M, int64_t d_in, int64_t d_out, int r);

/*
 * Forward: h = x.W^T + s.(x.A^T).B^T, s = alpha / r
 * (page "UnSloth加速库集成：编译级优化带来的性能飞跃", section 为什么标准LoRA会慢？, and
 * the single fused Linear -> LoRA_A -> LoRA_B -> Add pass of page
 * "ms-swift高效微调组合：LoRA+UnSloth提速实践", section 1.2, 算子融合).
 *   x, W, A, B : inputs (bf16).            h : output [M, d_out] (bf16).
 *   xa_save    : optional output [M, r] (bf16) = bf16(s . x.A^T); pass it to
 *                lora_linear_bwd to skip recomputing x.A^T.  May be NULL.
 *   workspace  : scratch of lora_linear_workspace_size(LORA_OP_FWD, ...) bytes.
 */
LORA_API lora_status_t lora_linear_fwd(const uint16_t *x, const uint16_t *W, const uint16_t *A,
                              const uint16_t *B, uint16_t *h, uint16_t *xa_save,
                              int64_t M, int64_t d_in, int64_t d_out, int r, float alpha,
                              void *workspace, size_t workspace_bytes, void *stream);

/*
 * Backward: dX = dY.W + s.(dY.B).A, dB = s.dY^T.(x.A^T), dA = s.(dY.B)^T.x
 * (chain rule of the forward above; the gradient pair of page
 * "ms-swift高效微调组合：LoRA+UnSloth提速实践", section 1.2, 梯度计算绕过Autograd, in
 * complete form; association A.(B.dY) from page "Unsloth — 微调 2-5x 加速", section
 * 核心要点).  W is frozen: no dW.
 *   dY, x, W, A, B : inputs (bf16).
 *   xa_save        : bf16(s . x.A^T) from lora_linear_fwd, or NULL to recompute it.
 *   dX             : output [M, d_in] (bf16), or NULL to skip the input gradient.
 *   dA, dB         : outputs (fp32), overwritten.
 */
LORA_API lora_status_t lora_linear_bwd(const uint16_t *dY, const uint16_t *x, const uint16_t *W,
                              const uint16_t *A, const uint16_t *B, const uint16_t *xa_save,
                              uint16_t *dX, float *dA, float *dB,
                              int64_t M, int64_t d_in, int64_t d_out, int r, float alpha,
                              void *workspace, size_t workspace_bytes, void *stream);

/*
 * Forward with a 4-bit frozen weight, dequantised in shared memory inside the GEMM
 * and never written back as bf16 (page "Unsloth — 微调 2-5x 加速", section 核心要点:
 * 4-bit dequantisation fused into the matmul; page
 * "ms-swift框架下UnSloth与Liger-Kernel优化实战", section UnSloth：让LoRA真正“低秩”起来:
 * int4 storage restored on the fly).  As lora_linear_fwd with W replaced by
 * (Wq, Wscale); d_in % 64 == 0.
 */
LORA_API lora_status_t lora_linear_fwd_q4(const uint16_t *x, const uint8_t *Wq, const uint16_t *Wscale,
                                 const uint16_t *A, const uint16_t *B, uint16_t *h,
                                 uint16_t *xa_save, int64_t M, int64_t d_in, int64_t d_out,
                                 int r, float alpha, void *workspace, size_t workspace_bytes,
                                 void *stream);

/* Backward with the 4-bit frozen weight (same passages); as lora_linear_bwd with W
 * replaced by (Wq, Wscale). */
LORA_API lora_status_t lora_linear_bwd_q4(const uint16_t *dY, const uint16_t *x, const uint8_t *Wq,
                                 const uint16_t *Wscale, const uint16_t *A, const uint16_t *B,
                                 const uint16_t *xa_save, uint16_t *dX, float *dA, float *dB,
                                 int64_t M, int64_t d_in, int64_t d_out, int r, float alpha,
                                 void *workspace, size_t workspace_bytes, void *stream);

/*
 * Forward with an FP8 frozen weight: the weight is stored as E4M3 codes with one bf16
 * scale per output row and the layer computes in bf16 (page
 * "ms-swift高效微调组合：LoRA+UnSloth提速实践", section 3.2: FP8 storage of the
 * weights with BF16 computation).  The codes are decoded in shared memory inside the
 * GEMMs and never written back as bf16; each decoded weight is e4m3(q) * scale, formed
 * exactly in fp32 and rounded once to bf16 for the tensor cores.
 *   W8 [d_out, d_in] uint8, one E4M3 code per weight (sign, 4-bit exponent of bias 7,
 *   3-bit mantissa; 0x7F / 0xFF are NaN);  W8scale [d_out] bf16.
 * As lora_linear_fwd with W replaced by (W8, W8scale); d_in % 16 == 0; the workspace is
 * lora_linear_workspace_size(LORA_OP_FWD_FP8, ...). */
LORA_API lora_status_t lora_linear_fwd_fp8(const uint16_t *x, const uint8_t *W8, const uint16_t *W8scale,
                                           const uint16_t *A, const uint16_t *B, uint16_t *h,
                                           uint16_t *xa_save, int64_t M, int64_t d_in, int64_t d_out,
                                           int r, float alpha, void *workspace, size_t workspace_bytes,
                                           void *stream);

/* Backward with the FP8 frozen weight (same passage and layout); as lora_linear_bwd
 * with W replaced by (W8, W8scale); workspace of LORA_OP_BWD_FP8. */
LORA_API lora_status_t lora_linear_bwd_fp8(const uint16_t *dY, const uint16_t *x, const uint8_t *W8,
                                           const uint16_t *W8scale, const uint16_t *A, const uint16_t *B,
                                           const uint16_t *xa_save, uint16_t *dX, float *dA, float *dB,
                                           int64_t M, int64_t d_in, int64_t d_out, int r, float alpha,
                                           void *workspace, size_t workspace_bytes, void *stream);

/*
 * Forward with a 4-bit codebook weight, the BNB-style 4-bit format (page
 * "ms-swift框架下UnSloth与Liger-Kernel优化实战", section UnSloth：让LoRA真正“低秩”起来:
 * BNB 4-bit weights restored on the fly): each weight is a 4-bit index into a table of
 * 16 values, scaled by a bf16 absmax per 64 weights along d_in,
 *     w'[n, k] = codebook[q[n, k]] * Wscale[n, k / 64].
 * NF4 is the codebook of the 4-bit NormalFloat type (16 quantiles of a standard normal
 * scaled to [-1, 1], with an exact zero); any 16 finite values work.  Codes and scales
 * are laid out as in lora_linear_fwd_q4 (Wq [d_out, d_in/2], low nibble = even index;
 * Wscale [d_out, d_in/64]); `codebook` points to 16 floats in HOST memory, read during
 * the call.  The codes are decoded in shared memory inside the GEMMs: each table value
 * codebook[i] * scale is formed in fp32 and rounded once to bf16.  d_in % 64 == 0;
 * workspace of LORA_OP_FWD_NF4; a non-finite codebook value gives LORA_ERR_INVALID_ARG. */
LORA_API lora_status_t lora_linear_fwd_nf4(const uint16_t *x, const uint8_t *Wq, const uint16_t *Wscale,
                                           const float *codebook, const uint16_t *A, const uint16_t *B,
                                           uint16_t *h, uint16_t *xa_save, int64_t M, int64_t d_in,
                                           int64_t d_out, int r, float alpha, void *workspace,
                                           size_t workspace_bytes, void *stream);

/* Backward with the 4-bit codebook weight (same passage and layout); as lora_linear_bwd
 * with W replaced by (Wq, Wscale, codebook); workspace of LORA_OP_BWD_NF4. */
LORA_API lora_status_t lora_linear_bwd_nf4(const uint16_t *dY, const uint16_t *x, const uint8_t *Wq,
                                           const uint16_t *Wscale, const float *codebook, const uint16_t *A,
                                           const uint16_t *B, const uint16_t *xa_save, uint16_t *dX, float *dA,
                                           float *dB, int64_t M, int64_t d_in, int64_t d_out, int r,
                                           float alpha, void *workspace, size_t workspace_bytes, void *stream);

/*
 * Forward without a workspace, for callers that cannot allocate device memory: a
 * plugin inside a host framework that owns every device allocation and passes in
 * only the op's tensors, or a service that fixes its device-memory budget at start-up
 * and forbids allocation afterwards (cudaMalloc may synchronise the device and
 * fragments the heap).  The pages have no counterpart; this is an interface
 * convenience.  Same arguments and results as lora_linear_fwd, minus the workspace;
 * it runs the same kernels, so h and xa_save are bit for bit those of
 * lora_linear_fwd.
 *   - Scratch: a fixed 4 MiB array in device memory, held by every GPU that loads this
 *     library until the process exits.  Problems whose forward workspace
 *     (lora_linear_workspace_size(LORA_OP_FWD, ...)) exceeds 4 MiB are rejected with
 *     LORA_ERR_WORKSPACE before anything is enqueued (every r <= 16 workload of
 *     M <= 8192 fits; rank 128 at M = 16384 does not).
 *   - Allocates nothing: no cudaMalloc/cudaFree; it enqueues a memset that clears the
 *     part of the scratch the call uses (all but the error word), then the forward
 *     kernels.
 *   - The first call in a CUDA context (with that context current; the runtime's
 *     primary context of the current device when none is) looks up the scratch's
 *     device address in it (cudaGetSymbolAddress) and enqueues a clear of its error
 *     word; make that first call before any stream capture.  Each context has its own
 *     copy of the scratch.
 *   - Errors: a bounded device wait that runs out records its code in the scratch's
 *     error word, which later calls leave in place; lora_linear_noalloc_check reports
 *     it (LORA_ERR_TIMEOUT) and clears it.  lora_linear_check cannot see it.
 *   - All calls share the one scratch: calls that can overlap on the GPU (different
 *     streams, or host threads without ordering) race and give wrong results.
 */
LORA_API lora_status_t lora_linear_fwd_noalloc(const uint16_t *x, const uint16_t *W, const uint16_t *A,
                                               const uint16_t *B, uint16_t *h, uint16_t *xa_save,
                                               int64_t M, int64_t d_in, int64_t d_out, int r, float alpha,
                                               void *stream);

/* Companion of lora_linear_fwd_noalloc (no counterpart in the pages): waits for
 * `stream`, then reads and clears the error word of the workspace-free forward's
 * scratch in the current context.  LORA_OK, LORA_ERR_TIMEOUT (a bounded device wait of
 * an earlier call ran out; that call's h is undefined) or LORA_ERR_CUDA.
 * Synchronising: for tests and diagnostics, not for the hot path. */
LORA_API lora_status_t lora_linear_noalloc_check(void *stream);

/* Failure-path self-test of the workspace-free forward (no counterpart in the pages):
 * as lora_linear_selftest_timeout, on the error word of that forward's scratch in the
 * current context, so that lora_linear_noalloc_check then reports LORA_ERR_TIMEOUT.
 * limit_us in 1 .. 2000000. */
LORA_API lora_status_t lora_linear_noalloc_selftest_timeout(uint32_t limit_us, void *stream);

/* Waits for `stream`, then reads and clears the device error word kept in
 * `workspace` (NULL: only waits).  Returns LORA_OK, LORA_ERR_TIMEOUT (a bounded device
 * wait ran out) or LORA_ERR_CUDA (the stream reported an error).  Synchronising: for
 * tests and diagnostics, not for the hot path. */
LORA_API lora_status_t lora_linear_check(void *workspace, void *stream);

/* Static description of a status code; never NULL. */
LORA_API const char *lora_status_string(lora_status_t status);

/*
 * Merge the adapter into the frozen weight for deployment:
 *     W_out = W + s * B . A,   s = alpha / r
 * (page "ms-swift框架下UnSloth与Liger-Kernel优化实战", section 设计权衡与最佳实践, item 4:
 * the model is exported in the standard format, adapter merged, before inference).
 *   W, W_out  bf16 [d_out, d_in] row-major; W_out may equal W (in place) but must not
 *             otherwise overlap it.
 *   A [r, d_in], B [d_out, r]  bf16 row-major.  Every pointer 16-byte aligned.
 * Per element: w + s * sum_j B[n, j] * A[j, k], the sum formed on the tensor cores in
 * fp32 (the bf16 products are exact), the weight added in fp32, rounded once to bf16.
 * A persistent TMA-fed kernel streams 128 x 128 tiles (bounded waits; see
 * lora_linear_merge_check).  Requires 8 <= d_in <= 2^24 with
 * d_in % 8 == 0, 1 <= d_out <= 2^24, 1 <= r <= 256, r % 8 == 0, finite alpha; otherwise
 * LORA_ERR_INVALID_ARG / LORA_ERR_MISALIGNED before any launch.  Stream-ordered,
 * allocates nothing, needs no workspace.
 */
LORA_API lora_status_t lora_linear_merge(const uint16_t *W, const uint16_t *A, const uint16_t *B, uint16_t *W_out,
                                         int64_t d_in, int64_t d_out, int r, float alpha, void *stream);

/* The same from the 4-bit weight (codes Wq [d_out, d_in/2], bf16 scales [d_out,
 * d_in/64], layout as lora_linear_fwd_q4; d_in % 64 == 0; Wscale non-null and 16-byte
 * aligned like the other pointers):
 *     W_out = (q - 8) * scale / 7 + s * B . A
 * with the decoded weight formed in fp32 as in the 4-bit GEMMs, rounded once to bf16. */
LORA_API lora_status_t lora_linear_merge_q4(const uint8_t *Wq, const uint16_t *Wscale, const uint16_t *A,
                                            const uint16_t *B, uint16_t *W_out, int64_t d_in, int64_t d_out, int r,
                                            float alpha, void *stream);

/* The same from the FP8 (E4M3) weight (codes W8 [d_out, d_in] uint8, one bf16 scale per
 * row W8scale [d_out], layout as lora_linear_fwd_fp8; d_in % 16 == 0):
 *     W_out = e4m3(q) * scale + s * B . A
 * with the decoded weight exact in fp32, rounded once to bf16 with the update. */
LORA_API lora_status_t lora_linear_merge_fp8(const uint8_t *W8, const uint16_t *W8scale, const uint16_t *A,
                                             const uint16_t *B, uint16_t *W_out, int64_t d_in, int64_t d_out, int r,
                                             float alpha, void *stream);

/* The same from the 4-bit codebook weight (Wq, Wscale and `codebook`, 16 floats in HOST
 * memory read during the call, as lora_linear_fwd_nf4; d_in % 64 == 0):
 *     W_out = codebook[q] * scale + s * B . A
 * with codebook[q] * scale formed in fp32; a non-finite codebook value gives
 * LORA_ERR_INVALID_ARG. */
LORA_API lora_status_t lora_linear_merge_nf4(const uint8_t *Wq, const uint16_t *Wscale, const float *codebook,
                                             const uint16_t *A, const uint16_t *B, uint16_t *W_out, int64_t d_in,
                                             int64_t d_out, int r, float alpha, void *stream);

/* Waits for `stream`, then reads and clears the merge kernels' device error word
 * (their pipeline waits are bounded like the layer's).  LORA_OK, LORA_ERR_TIMEOUT, or
 * LORA_ERR_CUDA.  Synchronising: for tests and diagnostics. */
LORA_API lora_status_t lora_linear_merge_check(void *stream);

/* Failure-path self-test (no counterpart in the pages: it tests this library's
 * bounded waits).  Enqueues on `stream` a one-warp kernel that waits, through the same
 * bounded-wait routine the layer's kernels use, on a barrier nothing arrives on; after
 * `limit_us` microseconds (1 .. 2000000) the wait gives up and records its code in the
 * error word of `workspace` (any workspace from lora_linear_workspace_size, 256-byte
 * aligned), exactly as a stalled pipeline stage would, and the kernel returns: the GPU
 * is neither hung nor faulted.  A following lora_linear_check(workspace, stream)
 * then returns LORA_ERR_TIMEOUT and clears the word.  Returns LORA_OK once enqueued,
 * LORA_ERR_WORKSPACE / LORA_ERR_MISALIGNED / LORA_ERR_INVALID_ARG for bad arguments,
 * LORA_ERR_UNSUPPORTED off sm_100, LORA_ERR_CUDA if the launch fails. */
LORA_API lora_status_t lora_linear_selftest_timeout(void *workspace, size_t ws_bytes, uint32_t limit_us,
                                                    void *stream);

/* ---- measurement hooks (no effect on results) ---------------------------------
 * Kernel kinds, in the order a forward + backward launches them. */
typedef enum {
    LORA_K_XA = 0,       /* forward prologue: bf16(s . x.A^T), split over d_in      */
    LORA_K_FWD_MAIN = 1, /* forward main GEMM: [x | s.xa].[W | B]^T                 */
    LORA_K_G = 2,        /* backward prologue: bf16(s . dY.B), split over d_out     */
    LORA_K_DX_MAIN = 3,  /* backward main GEMM: [dY | s.g].[W ; A]                  */
    LORA_K_DADB = 4,     /* dB = dY^T.(s.xa) and dA = (s.g)^T.x in one launch, each
                            split over tokens; runs beside the dX GEMM's last wave  */
    LORA_K_COUNT = 5
} lora_kernel_kind_t;

/* Total kernels this library has launched since it was loaded. */
LORA_API int64_t lora_linear_launch_count(void);

/* When enabled, every launch is bracketed by CUDA events recorded on its stream.
 * lora_linear_timing_read() waits for the recorded events and returns, per kernel
 * kind, the summed device time in ms and the number of launches, then clears the
 * record.  Returns LORA_OK, or LORA_ERR_CUDA if an event failed. */
LORA_API lora_status_t lora_linear_timing_enable(int enable);
LORA_API lora_status_t lora_linear_timing_read(double *ms_per_kind, int64_t *launches_per_kind,
                                      int kinds);

/* Per-CTA timestamp trace for diagnostics.  With a device buffer set, every launch of
 * kernel kind k writes, for each of its CTAs c, 32 uint64 words at word offset
 * k * (bytes / 8 / LORA_K_COUNT) + 32 * c: globaltimer ns at entry, after set-up, at
 * the end of the TMA producer, of the MMA issuer and of the epilogue, at exit; the SM
 * id; the tile count; the epilogue completion time of the CTA's first 8 tiles
 * (words 8-15); for the main GEMMs the total ns the producer waited for free stages
 * (16), the ns the MMA issuer waited for a drained accumulator (18) and the K blocks
 * it consumed (19); the SM cycle counter after set-up (20) and at exit (21), which
 * with the two ns stamps give the SM clock.  The CTA-pair main GEMMs add, in SM
 * cycles: the MMA issuer's waits for A tiles (22) and for decoded B tiles (23, 4-bit
 * weight), and the first dequant warp's waits for packed codes (24), its code reads
 * and scale preparation (25), decode + stores + publish (26), waits for a free B tile
 * (27) and code-fetch issue (28), summed over its K blocks.
 * Launches whose grid does not fit their share of the buffer are not traced.  Pass
 * NULL to switch tracing off.  Returns LORA_OK or LORA_ERR_MISALIGNED (8 bytes). */
LORA_API lora_status_t lora_linear_trace_enable(void *device_buffer, size_t bytes);

#ifdef __cplusplus
}
#endif

#endif /* LORA_LINEAR_H */
