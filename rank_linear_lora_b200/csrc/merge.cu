// merge.cu -- fold the adapter into the frozen weight for deployment:
//     W' = W + s * B . A,   s = alpha / r,   W, W' [d_out, d_in] bf16
// (page "ms-swift框架下UnSloth与Liger-Kernel优化实战", section 设计权衡与最佳实践, item 4:
// before inference the model is exported in the standard format, the adapter merged
// into the weight; the merged weight follows from h = W x + B (A x) of page
// "UnSloth加速库集成：编译级优化带来的性能飞跃", section 为什么标准LoRA会慢？).  The
// 4-bit variant starts from the decoded code, w = (q - 8) * scale / 7.
//
// The work is one read of W and one write of W' (HBM-bound); the rank-r update costs r
// FMAs per element.  One CTA of 256 threads owns a 32-row x 256-column tile: it stages
// its 32 rows of B and the 256-column panel of A in shared memory, 64 ranks at a time,
// and each thread accumulates a 4-row x 8-column micro-tile in fp32 (bf16 products are
// exact in fp32), adds the weight in fp32 and rounds once to bf16.  Every global access
// is a 16-byte vector of 8 consecutive columns; a warp covers 256 columns of one row
// (coalesced).  W' may be W itself (in place): a CTA reads each element of its tile
// before it writes it, and tiles are disjoint.
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

// ---------------------------------------------------------------- TMA-fed ring (r <= 64)
// The simple kernel above keeps only ~48 KB in flight per SM (three resident CTAs, a
// 16 KB tile each), which at the loaded DRAM latency holds it near 2.5 TB/s.  Here one
// persistent CTA per SM runs a ring of stages: a producer thread TMA-loads each tile's
// weight (bf16 16 KB, or 4 KB of codes), its A panel (r x 256) and its 32 rows of B
// into a free stage, ~100 KB ahead of its eight consumer warps (two CTAs per SM), which compute from
// shared memory exactly as the simple kernel does and store W'.  All waits are bounded
// (2 s); a timeout sets g_merge_err, read by lora_linear_merge_check.
constexpr int CONSUMERS = 8;
constexpr int THREADS_TMA = 32 * (CONSUMERS + 1);
constexpr int MAX_STAGES = 8;
constexpr int RING_SMEM = 110 * 1024;  // per CTA; two CTAs (16 consumer warps) per SM

__device__ int g_merge_err;

struct MergeArgs {
    CUtensorMap tmW;  // bf16 W [d_out][d_in] box {256, 32}, or codes uint8 [d_out][d_in/2] box {128, 32}
    CUtensorMap tmA;  // bf16 A [r][d_in], box {256, r}
    CUtensorMap tmB;  // bf16 B [d_out][r], box {r, 32}
    const uint16_t *Wscale;
    uint16_t *Wout;
    int64_t d_in, d_out, col_tiles, tiles;
    int r, stages;
    uint32_t w_bytes, a_bytes, stage_bytes;
    float s;
    int *err;
};

template <bool Q4>
__global__ void __launch_bounds__(THREADS_TMA, 2) k_merge_ring(const __grid_constant__ MergeArgs p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full_bar = reinterpret_cast<uint64_t *>(smem + p.stages * p.stage_bytes);  // [stages]
    uint64_t *empty_bar = full_bar + MAX_STAGES;                                        // [stages]
    volatile int *abort_flag = reinterpret_cast<volatile int *>(empty_bar + MAX_STAGES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int st = 0; st < p.stages; ++st) {
            lora::mbar_init(lora::smem_u32(&full_bar[st]), 1);
            lora::mbar_init(lora::smem_u32(&empty_bar[st]), CONSUMERS);
        }
        *abort_flag = 0;
        lora::fence_mbar_init();
    }
    __syncthreads();

    if (warp == CONSUMERS) {
        // ---------------------------------------------------------------- producer
        if (lane == 0) {
            lora::tma_prefetch_desc(&p.tmW);
            lora::tma_prefetch_desc(&p.tmA);
            lora::tma_prefetch_desc(&p.tmB);
            int k = 0;
            for (int64_t t = blockIdx.x; t < p.tiles; t += gridDim.x, ++k) {
                const int st = k % p.stages;
                const uint32_t ph = static_cast<uint32_t>(k / p.stages) & 1u;
                if (!lora::wait_bounded(lora::smem_u32(&empty_bar[st]), ph ^ 1u, abort_flag, p.err,
                                        lora::DERR_WAIT_EMPTY))
                    break;
                const int row0 = static_cast<int>((t / p.col_tiles) * MT);
                const int col0 = static_cast<int>((t % p.col_tiles) * NT);
                uint8_t *base = smem + st * p.stage_bytes;
                const uint32_t fb = lora::smem_u32(&full_bar[st]);
                lora::mbar_arrive_expect_tx(fb, p.stage_bytes);
                lora::tma_load_2d(lora::smem_u32(base), &p.tmW, fb, Q4 ? col0 / 2 : col0, row0);
                lora::tma_load_2d(lora::smem_u32(base + p.w_bytes), &p.tmA, fb, col0, 0);
                lora::tma_load_2d(lora::smem_u32(base + p.w_bytes + p.a_bytes), &p.tmB, fb, 0, row0);
            }
            // copies still in flight (only after a failed wait) land before the CTA exits
            for (int j = k > p.stages ? k - p.stages : 0; j < k; ++j) {
                volatile int never = 0;
                lora::wait_bounded(lora::smem_u32(&full_bar[j % p.stages]),
                                   static_cast<uint32_t>(j / p.stages) & 1u, &never, p.err, lora::DERR_WAIT_DRAIN);
            }
        }
        return;
    }

    // -------------------------------------------------------------------- consumers
    const int r = p.r;
    int k = 0;
    // scale words of the next tile (4-bit), fetched one tile ahead
    auto scales_of = [&](int64_t t, uint16_t (&sc)[4]) {
#pragma unroll
        for (int i = 0; i < 4; ++i) sc[i] = 0;
        if (!Q4 || t >= p.tiles) return;
        const int64_t row = (t / p.col_tiles) * MT + warp * 4, col = (t % p.col_tiles) * NT + lane * 8;
        if (col >= p.d_in) return;
#pragma unroll
        for (int i = 0; i < 4; ++i)
            if (row + i < p.d_out) sc[i] = p.Wscale[(row + i) * (p.d_in / 64) + col / 64];
    };
    uint16_t sc_next[4];
    scales_of(blockIdx.x, sc_next);
    for (int64_t t = blockIdx.x; t < p.tiles; t += gridDim.x, ++k) {
        uint16_t sc[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) sc[i] = sc_next[i];
        scales_of(t + gridDim.x, sc_next);
        const int st = k % p.stages;
        const uint32_t ph = static_cast<uint32_t>(k / p.stages) & 1u;
        if (!__all_sync(0xffffffffu, lora::wait_bounded(lora::smem_u32(&full_bar[st]), ph, abort_flag, p.err,
                                                        lora::DERR_WAIT_FULL)))
            break;
        const uint8_t *base = smem + st * p.stage_bytes;
        const uint16_t *sA = reinterpret_cast<const uint16_t *>(base + p.w_bytes);            // [r][256]
        const uint16_t *sB = reinterpret_cast<const uint16_t *>(base + p.w_bytes + p.a_bytes);  // [32][r]
        float acc[4][8];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[i][e] = 0.f;
#pragma unroll 4
        for (int jj = 0; jj < r; ++jj) {
            const uint4 av = *reinterpret_cast<const uint4 *>(sA + jj * NT + lane * 8);
            const uint32_t aw[4] = {av.x, av.y, av.z, av.w};
            float a[8];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                a[2 * q] = __uint_as_float(aw[q] << 16);
                a[2 * q + 1] = __uint_as_float(aw[q] & 0xFFFF0000u);
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float b = bf16_to_f32(sB[(warp * 4 + i) * r + jj]);
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[i][e] = fmaf(b, a[e], acc[i][e]);
            }
        }
        const int64_t row0 = (t / p.col_tiles) * MT, col = (t % p.col_tiles) * NT + lane * 8;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int lr = warp * 4 + i;
            const int64_t row = row0 + lr;
            float w[8];
            if (Q4) {
                decode8_f32(*reinterpret_cast<const uint32_t *>(base + lr * (NT / 2) + lane * 4),
                            bf16_to_f32(sc[i]) / 7.0f, w);
            } else {
                const uint4 wv = *reinterpret_cast<const uint4 *>(base + (lr * NT + lane * 8) * 2);
                const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    w[2 * q] = __uint_as_float(ww[q] << 16);
                    w[2 * q + 1] = __uint_as_float(ww[q] & 0xFFFF0000u);
                }
            }
            if (row < p.d_out && col < p.d_in) {
                uint32_t out[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    __nv_bfloat162 b2 = __floats2bfloat162_rn(fmaf(p.s, acc[i][2 * q], w[2 * q]),
                                                              fmaf(p.s, acc[i][2 * q + 1], w[2 * q + 1]));
                    out[q] = *reinterpret_cast<uint32_t *>(&b2);
                }
                *reinterpret_cast<uint4 *>(p.Wout + row * p.d_in + col) = make_uint4(out[0], out[1], out[2], out[3]);
            }
        }
        __syncwarp();  // every lane is done with this stage
        if (lane == 0) lora::mbar_arrive(lora::smem_u32(&empty_bar[st]));
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
// Row-major 2D tensor [rows][cols] of `esize`-byte elements, box {box_cols, box_rows},
// no swizzle (threads read the tiles), zero fill outside.
bool tmap_plain(CUtensorMap *m, CUtensorMapDataType type, int esize, const void *base, uint64_t cols, uint64_t rows,
                uint32_t box_cols, uint32_t box_rows) {
    return lora_host::tmap_2d(m, type, esize, base, cols, rows, box_cols, box_rows, CU_TENSOR_MAP_SWIZZLE_NONE);
}

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

    MergeArgs a;
    std::memset(&a, 0, sizeof(a));
    a.w_bytes = q4 ? MT * NT / 2 : MT * NT * 2;
    a.a_bytes = static_cast<uint32_t>(r) * NT * 2;
    a.stage_bytes = a.w_bytes + a.a_bytes + static_cast<uint32_t>(MT * r * 2);
    a.stages = static_cast<int>(std::min<int64_t>(MAX_STAGES, RING_SMEM / a.stage_bytes));
    if (r <= 64 && a.stages >= 2) {
        int *err = merge_err_word(dev);
        if (!err) return LORA_ERR_CUDA;
        const bool maps = (q4 ? tmap_plain(&a.tmW, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, Wq, d_in / 2, d_out, NT / 2, MT)
                              : tmap_plain(&a.tmW, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, W, d_in, d_out, NT, MT)) &&
                          tmap_plain(&a.tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, A, d_in, r, NT, r) &&
                          tmap_plain(&a.tmB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, B, r, d_out, r, MT);
        if (!maps) return LORA_ERR_CUDA;
        a.Wscale = Wscale;
        a.Wout = Wout;
        a.d_in = d_in;
        a.d_out = d_out;
        a.col_tiles = col_tiles;
        a.tiles = tiles;
        a.r = r;
        a.s = s;
        a.err = err;
        const int smem = 1024 + a.stages * static_cast<int>(a.stage_bytes) + 2 * MAX_STAGES * 8 + 16;
        auto kern = q4 ? k_merge_ring<true> : k_merge_ring<false>;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
            return LORA_ERR_CUDA;
        const unsigned grid = static_cast<unsigned>(std::min<int64_t>(tiles, 2 * sms));
        kern<<<grid, THREADS_TMA, smem, st>>>(a);
        return cudaGetLastError() == cudaSuccess ? LORA_OK : LORA_ERR_CUDA;
    }
    // r > 64: the A panel does not fit a multi-stage ring; one tile per CTA
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
