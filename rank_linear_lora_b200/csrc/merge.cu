// merge.cu -- fold the adapter into the frozen weight for deployment:
//     W' = W + s * B . A,   s = alpha / r,   W, W' [d_out, d_in] bf16
// (page "ms-swift框架下UnSloth与Liger-Kernel优化实战", section 设计权衡与最佳实践, item 4:
// before inference the model is exported in the standard format, the adapter merged
// into the weight; the merged weight follows from h = W x + B (A x) of page
// "UnSloth加速库集成：编译级优化带来的性能飞跃", section 为什么标准LoRA会慢？).  The
// 4-bit variant starts from the decoded code, w = (q - 8) * scale / 7.
//
// The work is one read of W and one write of W' (HBM-bound).  Up to r = 64 the rank-r
// update runs on the tensor cores (k_merge_tc: a tcgen05 contraction over the ranks into
// TMEM, the weight added in the epilogue, TMA in and out); wider ranks take k_merge, a
// CUDA-core kernel whose threads accumulate 4-row x 8-column micro-tiles in fp32.  Both
// add the weight in fp32 and round once to bf16 (bf16 products are exact in fp32).  W'
// may be W itself (in place): a tile is read before it is written, and tiles are
// disjoint.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/lora_linear.h"
#include "tc_gemm.cuh"  // bounded mbarrier waits, TMA and mbarrier wrappers
#include "tmap.h"

namespace {

constexpr int MT = 32;        // rows per CTA tile
constexpr int NT = 256;       // columns per CTA tile
constexpr int RCH = 64;       // ranks staged per pass
constexpr int THREADS = 256;  // 8 warps; warp w owns rows 4w .. 4w+3, lane owns 8 columns

__device__ __forceinline__ float bf16_to_f32(uint16_t b) { return __uint_as_float(static_cast<uint32_t>(b) << 16); }

// Decoded 4-bit weight, 8 consecutive columns from one 32-bit word of codes (low nibble
// = even column), in fp32: (q - 8) * (scale / 7), the rule of the main GEMMs' decode.
__device__ __forceinline__ void decode8_f32(uint32_t word, float s7, float (&w)[8]) {
#pragma unroll
    for (int e = 0; e < 8; ++e) w[e] = static_cast<float>(static_cast<int>((word >> (4 * e)) & 0xFu) - 8) * s7;
}

template <bool Q4>
__global__ void __launch_bounds__(THREADS) k_merge(const uint16_t *W, const uint8_t *Wq,  // may alias Wout
                                                   const uint16_t *__restrict__ Wscale, const uint16_t *__restrict__ A,
                                                   const uint16_t *__restrict__ B, uint16_t *Wout, int64_t d_in,
                                                   int64_t d_out, int r, float s) {
    __shared__ __align__(16) uint16_t sA[RCH][NT];  // A[j0 + jj][col0 + c]
    __shared__ __align__(16) uint16_t sB[MT][RCH];  // B[row0 + i][j0 + jj]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // Tiles in row-major order (column tile fastest), so the CTAs resident at one time
    // read whole rows of W together rather than one 512-byte piece of many rows.
    const int64_t col_tiles = (d_in + NT - 1) / NT;
    const int64_t row0 = (static_cast<int64_t>(blockIdx.x) / col_tiles) * MT;
    const int64_t col0 = (static_cast<int64_t>(blockIdx.x) % col_tiles) * NT;
    const int64_t col = col0 + lane * 8;  // this thread's 8 columns
    const bool col_ok = col < d_in;       // d_in % 8 == 0, so a group is all in or all out

    // This thread's weight (4 rows x 8 columns) is loaded first, so its DRAM latency
    // overlaps the staging and the FMAs below; every load precedes every store, which
    // keeps W' = W (in place) correct.
    uint4 wv[4];     // bf16 weight
    uint32_t qw[4];  // 4-bit weight: one word of codes per row
    uint16_t sc[4];  //               and its group scale
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int64_t row = row0 + warp * 4 + i;
        wv[i] = make_uint4(0, 0, 0, 0);
        qw[i] = 0;
        sc[i] = 0;
        if (col_ok && row < d_out) {
            if (Q4) {
                qw[i] = *reinterpret_cast<const uint32_t *>(Wq + row * (d_in / 2) + col / 2);
                sc[i] = Wscale[row * (d_in / 64) + col / 64];
            } else {
                wv[i] = *reinterpret_cast<const uint4 *>(W + row * d_in + col);
            }
        }
    }

    float acc[4][8];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[i][e] = 0.f;

    for (int j0 = 0; j0 < r; j0 += RCH) {
        const int rc = min(RCH, r - j0);
        __syncthreads();  // the previous chunk's readers are done
        // A panel: rc rows x 256 columns, 16 bytes per load (zero past d_in)
        for (int v = threadIdx.x; v < rc * (NT / 8); v += THREADS) {
            const int jj = v / (NT / 8), c8 = (v % (NT / 8)) * 8;
            uint4 val = make_uint4(0, 0, 0, 0);
            if (col0 + c8 < d_in) val = *reinterpret_cast<const uint4 *>(A + (j0 + jj) * d_in + col0 + c8);
            *reinterpret_cast<uint4 *>(&sA[jj][c8]) = val;
        }
        // B rows: 32 rows x rc ranks (zero past d_out)
        for (int v = threadIdx.x; v < MT * rc; v += THREADS) {
            const int i = v / rc, jj = v % rc;
            sB[i][jj] = (row0 + i < d_out) ? B[(row0 + i) * r + j0 + jj] : uint16_t(0);
        }
        __syncthreads();
        for (int jj = 0; jj < rc; ++jj) {
            const uint4 av = *reinterpret_cast<const uint4 *>(&sA[jj][lane * 8]);
            const uint32_t aw[4] = {av.x, av.y, av.z, av.w};
            float a[8];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                a[2 * q] = __uint_as_float(aw[q] << 16);
                a[2 * q + 1] = __uint_as_float(aw[q] & 0xFFFF0000u);
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float b = bf16_to_f32(sB[warp * 4 + i][jj]);
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[i][e] = fmaf(b, a[e], acc[i][e]);
            }
        }
    }
    if (!col_ok) return;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int64_t row = row0 + warp * 4 + i;
        if (row >= d_out) break;
        float w[8];
        if (Q4) {
            decode8_f32(qw[i], bf16_to_f32(sc[i]) / 7.0f, w);
        } else {
            const uint32_t ww[4] = {wv[i].x, wv[i].y, wv[i].z, wv[i].w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                w[2 * q] = __uint_as_float(ww[q] << 16);
                w[2 * q + 1] = __uint_as_float(ww[q] & 0xFFFF0000u);
            }
        }
        uint32_t out[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            __nv_bfloat162 b2 = __floats2bfloat162_rn(fmaf(s, acc[i][2 * q], w[2 * q]),
                                                      fmaf(s, acc[i][2 * q + 1], w[2 * q + 1]));
            out[q] = *reinterpret_cast<uint32_t *>(&b2);
        }
        *reinterpret_cast<uint4 *>(Wout + row * d_in + col) = make_uint4(out[0], out[1], out[2], out[3]);
    }
}

// ---------------------------------------------------------------- tensor cores (r <= 64)
// The kernel above spends ~14 instructions per element on the rank-r update (shared-memory
// operand loads, widening, r FMAs) and is issue-bound at less than half the HBM bandwidth.
// Here the update s * B . A of a 128-row x 128-column tile is one to four tcgen05 MMAs
// (M = 128, N = 128, K = 16 ranks each) into an fp32 TMEM accumulator, and the epilogue
// only adds the weight: tcgen05.ld of 32 columns, the weight from the TMA-staged tile in
// shared memory, one fp32 FMA and one rounding per element, the result written over the
// staged tile (bf16 weight) or into a staging tile (4-bit weight), then TMA-stored.
// Roles as in the layer's kernels: warp 0 the TMA producer, warp 1 TMEM and the
// single-thread MMA issue, warps 2..5 the epilogue (one accumulator row each thread);
// three stages of operands, two TMEM accumulators.  Persistent, one CTA per SM, tiles in
// row-major order.  128 columns rather than 256: a 4096 x 4096 weight is 1024 tiles, 6.9
// per SM, where 256-column tiles would leave 14% of the SMs' time on a partial last wave.
// Every wait is bounded (2 s); a timeout sets g_merge_err (lora_linear_merge_check).
constexpr int TC_M = 128, TC_N = 128, TC_STAGES = 3, TC_ACC = 2, TC_THREADS = 192;
constexpr int TC_CHUNKS = TC_N / 64;              // 64-column chunks (one 128B-swizzle box each)
constexpr int TC_W_BYTES = TC_M * TC_N * 2;       // bf16 weight tile, or an output staging tile
constexpr int TC_Q_BYTES = TC_M * TC_N / 2;       // 4-bit codes of the tile
constexpr int TC_B_BYTES = TC_M * 64 * 2;         // B rows [128 x 64 ranks], K-major, 128B swizzle
constexpr int TC_A_BYTES = TC_CHUNKS * 64 * 128;  // A panel: 64-column chunks x 64 ranks, MN-major

__device__ int g_merge_err;

struct MergeArgs {
    CUtensorMap tmW;    // bf16 W [d_out][d_in] box {64, 128}, 128B swizzle; or codes uint8 [d_out][d_in/2] box {64, 128}
    CUtensorMap tmOut;  // bf16 W' [d_out][d_in] box {64, 128}, 128B swizzle
    CUtensorMap tmA;    // bf16 A [r][d_in] box {64, kr}, 128B swizzle (the MMA's MN-major B operand)
    CUtensorMap tmB;    // bf16 B [d_out][r] box {64, 128}, 128B swizzle (the MMA's K-major A operand)
    const uint16_t *Wscale;  // 4-bit weight: bf16 [d_out][d_in/64]
    int64_t d_in, d_out, col_tiles, tiles;
    int kr;             // r rounded up to 16 (the MMAs' K); ranks past r are zero-filled by TMA
    float s;
    int *err;
};

template <bool Q4>
struct MergeCfg {
    static constexpr int WSTAGE = Q4 ? TC_Q_BYTES : TC_W_BYTES;
    static constexpr int STAGE_BYTES = WSTAGE + TC_B_BYTES + TC_A_BYTES;
    static constexpr int STAGING = Q4 ? 2 * TC_W_BYTES : 0;  // 4-bit weight: output tiles staged apart
    static constexpr int SMEM_BYTES = 1024 + TC_STAGES * STAGE_BYTES + STAGING + 256;
    static_assert(STAGE_BYTES % 1024 == 0, "stages keep the 1024-byte alignment of the swizzled boxes");
    static_assert(SMEM_BYTES <= 232448, "at most 227 KB of shared memory per CTA");
};

template <bool Q4>
__global__ void __launch_bounds__(TC_THREADS, 1) k_merge_tc(const __grid_constant__ MergeArgs p) {
    using Cfg = MergeCfg<Q4>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *staging = smem + TC_STAGES * Cfg::STAGE_BYTES;
    uint64_t *bars = reinterpret_cast<uint64_t *>(staging + Cfg::STAGING);
    uint64_t *full_bar = bars;                      // [stages] the tile's operands landed
    uint64_t *empty_bar = bars + TC_STAGES;         // [stages] the stage (and its store) is done with
    uint64_t *tfull_bar = bars + 2 * TC_STAGES;     // [acc] accumulator ready
    uint64_t *tempty_bar = tfull_bar + TC_ACC;      // [acc] accumulator drained
    uint64_t *drain_bar = tempty_bar + TC_ACC;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain_bar + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    volatile int *epi_ok = reinterpret_cast<volatile int *>(tmem_slot + 2);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int b = 0; b < TC_STAGES; ++b) {
            lora::mbar_init(lora::smem_u32(&full_bar[b]), 1);
            lora::mbar_init(lora::smem_u32(&empty_bar[b]), 1);
        }
        for (int b = 0; b < TC_ACC; ++b) {
            lora::mbar_init(lora::smem_u32(&tfull_bar[b]), 1);
            lora::mbar_init(lora::smem_u32(&tempty_bar[b]), 4);
        }
        lora::mbar_init(lora::smem_u32(drain_bar), 1);
        *abort_flag = 0;
        lora::fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        lora::tma_prefetch_desc(&p.tmW);
        lora::tma_prefetch_desc(&p.tmOut);
        lora::tma_prefetch_desc(&p.tmA);
        lora::tma_prefetch_desc(&p.tmB);
    }
    if (warp == 1) {
        lora::tmem_alloc(lora::smem_u32(tmem_slot), TC_ACC * TC_N);
        lora::tmem_relinquish();
    }
    lora::tc_fence_before();
    __syncthreads();
    lora::tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t issued = 0, issued_phase = 0;
            int k = 0;
            for (int64_t t = blockIdx.x; t < p.tiles; t += gridDim.x, ++k) {
                const int st = k % TC_STAGES;
                const uint32_t ph = static_cast<uint32_t>(k / TC_STAGES) & 1u;
                if (!lora::wait_bounded(lora::smem_u32(&empty_bar[st]), ph ^ 1u, abort_flag, p.err,
                                        lora::DERR_WAIT_EMPTY))
                    break;
                const int row0 = static_cast<int>((t / p.col_tiles) * TC_M);
                const int col0 = static_cast<int>((t % p.col_tiles) * TC_N);
                uint8_t *base = smem + st * Cfg::STAGE_BYTES;
                const uint32_t fb = lora::smem_u32(&full_bar[st]);
                lora::mbar_arrive_expect_tx(
                    fb, Cfg::WSTAGE + TC_B_BYTES + static_cast<uint32_t>(TC_CHUNKS * 128 * p.kr));
                if (Q4) {
                    lora::tma_load_2d(lora::smem_u32(base), &p.tmW, fb, col0 / 2, row0);
                } else {
                    for (int j = 0; j < TC_CHUNKS; ++j)
                        lora::tma_load_2d(lora::smem_u32(base + j * 16384), &p.tmW, fb, col0 + 64 * j, row0);
                }
                lora::tma_load_2d(lora::smem_u32(base + Cfg::WSTAGE), &p.tmB, fb, 0, row0);
                for (int j = 0; j < TC_CHUNKS; ++j)
                    lora::tma_load_2d(lora::smem_u32(base + Cfg::WSTAGE + TC_B_BYTES + j * 8192), &p.tmA, fb,
                                      col0 + 64 * j, 0);
                issued |= 1u << st;
                issued_phase = (issued_phase & ~(1u << st)) | (ph << st);
            }
            // copies still in flight (only after a failed wait) land before the CTA exits
            for (int st = 0; st < TC_STAGES; ++st)
                if (issued & (1u << st)) {
                    volatile int never = 0;
                    lora::wait_bounded(lora::smem_u32(&full_bar[st]), (issued_phase >> st) & 1u, &never, p.err,
                                       lora::DERR_WAIT_DRAIN);
                }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            // acc [128 rows x 128 columns] = B rows (K-major) . A panel (MN-major), K = kr ranks
            constexpr uint32_t idesc = lora::idesc_bf16(TC_M, TC_N, false, true);
            int k = 0;
            for (int64_t t = blockIdx.x; t < p.tiles; t += gridDim.x, ++k) {
                const int st = k % TC_STAGES, buf = k % TC_ACC;
                if (!lora::wait_bounded(lora::smem_u32(&tempty_bar[buf]), (static_cast<uint32_t>(k / TC_ACC) & 1u) ^ 1u,
                                        abort_flag, p.err, lora::DERR_WAIT_TMEM_EMPTY))
                    break;
                if (!lora::wait_bounded(lora::smem_u32(&full_bar[st]), static_cast<uint32_t>(k / TC_STAGES) & 1u,
                                        abort_flag, p.err, lora::DERR_WAIT_FULL))
                    break;
                lora::tc_fence_after();
                const uint32_t bsm = lora::smem_u32(smem + st * Cfg::STAGE_BYTES + Cfg::WSTAGE);
                // K-major 128B swizzle: 8-row groups 1024 bytes apart, a K step of 16 = 32 bytes
                const uint64_t ad = lora::sdesc_sw128(bsm, 16, 1024);
                // MN-major 128B swizzle: 64-column chunks 8192 bytes apart (LBO), 8-rank
                // groups 1024 bytes apart (SBO), a K step of 16 ranks = 2048 bytes
                const uint64_t bd = lora::sdesc_sw128(bsm + TC_B_BYTES, 8192, 1024);
                for (int kk = 0; kk < p.kr / 16; ++kk)
                    lora::tc_mma_bf16(tmem_base + static_cast<uint32_t>(buf * TC_N), ad + (kk * 32 >> 4),
                                      bd + (kk * 2048 >> 4), idesc, kk > 0 ? 1u : 0u);
                lora::tc_commit(lora::smem_u32(&tfull_bar[buf]));
            }
            lora::tc_commit(lora::smem_u32(drain_bar));
            volatile int never = 0;
            lora::wait_bounded(lora::smem_u32(drain_bar), 0, &never, p.err, lora::DERR_WAIT_DRAIN);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;  // warps 2..5 -> TMEM lane quarters 2, 3, 0, 1
        const int lr = q * 32 + lane;  // accumulator row = tile row
        const int et = threadIdx.x - 64;
        int k = 0, prev_st = -1;
        for (int64_t t = blockIdx.x; t < p.tiles; t += gridDim.x, ++k) {
            const int st = k % TC_STAGES, buf = k % TC_ACC;
            const uint32_t sph = static_cast<uint32_t>(k / TC_STAGES) & 1u;
            if (et == 0)
                epi_ok[0] = lora::wait_bounded(lora::smem_u32(&tfull_bar[buf]), static_cast<uint32_t>(k / TC_ACC) & 1u,
                                               abort_flag, p.err, lora::DERR_WAIT_TMEM_FULL)
                                ? 1
                                : 0;
            lora::named_bar_sync(1, 128);
            const bool ok = epi_ok[0] != 0;
            lora::named_bar_sync(1, 128);
            if (!ok) break;
            // the stage's operands landed before the MMA ran, so this returns at once; it
            // makes the weight tile's TMA writes visible to this thread
            lora::wait_bounded(lora::smem_u32(&full_bar[st]), sph, abort_flag, p.err, lora::DERR_WAIT_FULL);
            lora::tc_fence_after();
            const int64_t row = (t / p.col_tiles) * TC_M + lr;
            const int64_t col0 = (t % p.col_tiles) * TC_N;
            uint8_t *wst = smem + st * Cfg::STAGE_BYTES;
            uint8_t *out = Q4 ? staging + (k & 1) * TC_W_BYTES : wst;  // 64-column chunks, 128B swizzle
            const uint32_t t_row =
                tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(buf * TC_N);
#pragma unroll 1
            for (int c = 0; c < TC_CHUNKS; ++c) {
                uint32_t v0[32], v1[32];
                lora::tmem_ld_32x32b_x32(t_row + c * 64, v0);
                lora::tmem_ld_32x32b_x32(t_row + c * 64 + 32, v1);
                lora::tc_wait_ld();
                if (c == TC_CHUNKS - 1) {
                    lora::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) lora::mbar_arrive(lora::smem_u32(&tempty_bar[buf]));
                }
                float w[64];
                if (Q4) {
                    // 64 codes of this row (32 bytes, low nibble = even column) and their scale
                    const uint4 *qp = reinterpret_cast<const uint4 *>(wst + lr * (TC_N / 2) + c * 32);
                    const uint4 q0 = qp[0], q1 = qp[1];
                    const uint32_t words[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
                    const int64_t gcol = col0 + c * 64;
                    const float s7 = (row < p.d_out && gcol < p.d_in)
                                         ? bf16_to_f32(p.Wscale[row * (p.d_in / 64) + gcol / 64]) / 7.0f
                                         : 0.f;
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        float d8[8];
                        decode8_f32(words[j], s7, d8);
#pragma unroll
                        for (int e = 0; e < 8; ++e) w[j * 8 + e] = d8[e];
                    }
                } else {
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch) {
                        const uint4 wv =
                            *reinterpret_cast<const uint4 *>(wst + c * 16384 + lr * 128 + ((ch ^ (lr & 7)) * 16));
                        const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            w[ch * 8 + 2 * e] = __uint_as_float(ww[e] << 16);
                            w[ch * 8 + 2 * e + 1] = __uint_as_float(ww[e] & 0xFFFF0000u);
                        }
                    }
                }
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    uint32_t o[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int col = ch * 8 + 2 * e;
                        const float a0 = __uint_as_float(col < 32 ? v0[col] : v1[col - 32]);
                        const float a1 = __uint_as_float(col + 1 < 32 ? v0[col + 1] : v1[col + 1 - 32]);
                        __nv_bfloat162 b2 = __floats2bfloat162_rn(fmaf(p.s, a0, w[col]), fmaf(p.s, a1, w[col + 1]));
                        o[e] = *reinterpret_cast<uint32_t *>(&b2);
                    }
                    *reinterpret_cast<uint4 *>(out + c * 16384 + lr * 128 + ((ch ^ (lr & 7)) * 16)) =
                        make_uint4(o[0], o[1], o[2], o[3]);
                }
            }
            lora::fence_proxy_async_smem();
            lora::named_bar_sync(1, 128);
            if (et == 0) {
                for (int c = 0; c < TC_CHUNKS; ++c)
                    if (col0 + 64 * c < p.d_in)  // a chunk wholly past d_in has nothing to store
                        lora::tma_store_2d(&p.tmOut, lora::smem_u32(out + c * 16384),
                                           static_cast<int32_t>(col0 + 64 * c),
                                           static_cast<int32_t>((t / p.col_tiles) * TC_M));
                lora::bulk_commit_group();
                if (Q4) {
                    // the codes are in registers already; the other staging tile's store
                    // has read it before the next tile writes there
                    lora::mbar_arrive(lora::smem_u32(&empty_bar[st]));
                    lora::bulk_wait_group_read<1>();
                } else {
                    // the stage holds this tile's output until its store has read it: free
                    // the previous tile's stage once that store (one group back) has
                    lora::bulk_wait_group_read<1>();
                    if (prev_st >= 0) lora::mbar_arrive(lora::smem_u32(&empty_bar[prev_st]));
                }
            }
            lora::named_bar_sync(1, 128);
            prev_st = st;
        }
        if (et == 0) lora::bulk_wait_group<0>();
    }

    // ---------------------------------------------------------------- teardown
    __syncwarp();
    lora::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        lora::tc_fence_after();
        lora::tmem_dealloc(tmem_base, TC_ACC * TC_N);
    }
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Every pointer 16-byte aligned, as for the layer: the ring kernel reads W (or the codes),
// A and B by TMA and the other kernel reads W and A in 16-byte vectors.
lora_status_t merge_checks(const void *w0, const void *scale, const void *A, const void *B, const void *Wout,
                           int64_t d_in, int64_t d_out, int r, float alpha, bool q4) {
    if (!w0 || !A || !B || !Wout || (q4 && !scale)) return LORA_ERR_INVALID_ARG;
    if (d_in < 8 || d_out < 1 || d_in % 8 || (q4 && d_in % 64)) return LORA_ERR_INVALID_ARG;
    if (d_in > (int64_t(1) << 24) || d_out > (int64_t(1) << 24)) return LORA_ERR_INVALID_ARG;
    if (((d_out + MT - 1) / MT) * ((d_in + NT - 1) / NT) > 0x7FFFFFFF) return LORA_ERR_INVALID_ARG;
    if (r < 1 || r > 256 || r % 8) return LORA_ERR_INVALID_ARG;
    if (!(alpha == alpha) || alpha > 3.4e38f || alpha < -3.4e38f) return LORA_ERR_INVALID_ARG;
    if (!aligned16(w0) || !aligned16(A) || !aligned16(B) || !aligned16(Wout) || (q4 && !aligned16(scale)))
        return LORA_ERR_MISALIGNED;
    return LORA_OK;
}

// ------------------------------------------------------------------ host
std::mutex g_err_mu;
int *g_err_addr[64] = {};

int *merge_err_word(int dev) {
    std::lock_guard<std::mutex> lk(g_err_mu);
    if (!g_err_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_merge_err) != cudaSuccess) return nullptr;
        g_err_addr[dev] = static_cast<int *>(p);
    }
    return g_err_addr[dev];
}

lora_status_t merge_launch(bool q4, const uint16_t *W, const uint8_t *Wq, const uint16_t *Wscale, const uint16_t *A,
                           const uint16_t *B, uint16_t *Wout, int64_t d_in, int64_t d_out, int r, float alpha,
                           void *stream) {
    int dev = 0, major = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return LORA_ERR_CUDA;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return LORA_ERR_CUDA;
    if (major != 10) return LORA_ERR_UNSUPPORTED;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return LORA_ERR_CUDA;
    const float s = alpha / static_cast<float>(r);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int64_t col_tiles = (d_in + NT - 1) / NT, tiles = ((d_out + MT - 1) / MT) * col_tiles;

    if (r <= 64) {
        int *err = merge_err_word(dev);
        if (!err) return LORA_ERR_CUDA;
        MergeArgs a;
        std::memset(&a, 0, sizeof(a));
        a.kr = (r + 15) / 16 * 16;
        const bool maps =
            (q4 ? lora_host::tmap_2d(&a.tmW, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, Wq, d_in / 2, d_out, TC_N / 2, TC_M,
                                     CU_TENSOR_MAP_SWIZZLE_NONE)
                : lora_host::tmap_2d(&a.tmW, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, W, d_in, d_out, 64, TC_M,
                                     CU_TENSOR_MAP_SWIZZLE_128B)) &&
            lora_host::tmap_2d(&a.tmOut, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Wout, d_in, d_out, 64, TC_M,
                               CU_TENSOR_MAP_SWIZZLE_128B) &&
            lora_host::tmap_2d(&a.tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, A, d_in, r, 64, a.kr,
                               CU_TENSOR_MAP_SWIZZLE_128B) &&
            lora_host::tmap_2d(&a.tmB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, B, r, d_out, 64, TC_M,
                               CU_TENSOR_MAP_SWIZZLE_128B);
        if (!maps) return LORA_ERR_CUDA;
        const int64_t tc_col_tiles = (d_in + TC_N - 1) / TC_N;
        a.Wscale = Wscale;
        a.d_in = d_in;
        a.d_out = d_out;
        a.col_tiles = tc_col_tiles;
        a.tiles = ((d_out + TC_M - 1) / TC_M) * tc_col_tiles;
        a.s = s;
        a.err = err;
        auto kern = q4 ? k_merge_tc<true> : k_merge_tc<false>;
        const int smem = q4 ? MergeCfg<true>::SMEM_BYTES : MergeCfg<false>::SMEM_BYTES;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
            return LORA_ERR_CUDA;
        const unsigned grid = static_cast<unsigned>(std::min<int64_t>(a.tiles, sms));
        kern<<<grid, TC_THREADS, smem, st>>>(a);
        return cudaGetLastError() == cudaSuccess ? LORA_OK : LORA_ERR_CUDA;
    }
    // r > 64: the CUDA-core kernel, one tile per CTA
    const dim3 grid(static_cast<unsigned>(tiles));
    if (q4)
        k_merge<true><<<grid, THREADS, 0, st>>>(nullptr, Wq, Wscale, A, B, Wout, d_in, d_out, r, s);
    else
        k_merge<false><<<grid, THREADS, 0, st>>>(W, nullptr, nullptr, A, B, Wout, d_in, d_out, r, s);
    return cudaGetLastError() == cudaSuccess ? LORA_OK : LORA_ERR_CUDA;
}

}  // namespace

extern "C" LORA_API lora_status_t lora_linear_merge(const uint16_t *W, const uint16_t *A, const uint16_t *B,
                                                    uint16_t *W_out, int64_t d_in, int64_t d_out, int r, float alpha,
                                                    void *stream) {
    const lora_status_t st = merge_checks(W, nullptr, A, B, W_out, d_in, d_out, r, alpha, false);
    if (st != LORA_OK) return st;
    return merge_launch(false, W, nullptr, nullptr, A, B, W_out, d_in, d_out, r, alpha, stream);
}

extern "C" LORA_API lora_status_t lora_linear_merge_q4(const uint8_t *Wq, const uint16_t *Wscale, const uint16_t *A,
                                                       const uint16_t *B, uint16_t *W_out, int64_t d_in, int64_t d_out,
                                                       int r, float alpha, void *stream) {
    const lora_status_t st = merge_checks(Wq, Wscale, A, B, W_out, d_in, d_out, r, alpha, true);
    if (st != LORA_OK) return st;
    return merge_launch(true, nullptr, Wq, Wscale, A, B, W_out, d_in, d_out, r, alpha, stream);
}

extern "C" LORA_API lora_status_t lora_linear_merge_check(void *stream) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return LORA_ERR_CUDA;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return LORA_ERR_CUDA;
    int *err = merge_err_word(dev);
    if (!err) return LORA_ERR_CUDA;
    int word = 0;
    if (cudaMemcpy(&word, err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return LORA_ERR_CUDA;
    if (word != 0) {
        cudaMemset(err, 0, sizeof(int));
        return LORA_ERR_TIMEOUT;
    }
    return LORA_OK;
}
