// merge.cu -- fold the adapter into the frozen weight for deployment:
//     W' = W + s * B . A,   s = alpha / r,   W, W' [d_out, d_in] bf16
// (page "ms-swift框架下UnSloth与Liger-Kernel优化实战", section 设计权衡与最佳实践, item 4:
// before inference the model is exported in the standard format, the adapter merged
// into the weight; the merged weight follows from h = W x + B (A x) of page
// "UnSloth加速库集成：编译级优化带来的性能飞跃", section 为什么标准LoRA会慢？).  A stored
// weight in one of the layer's coded formats is decoded first: the 4-bit code
// (q - 8) * scale / 7, the FP8 (E4M3) code e4m3(q) * row scale, or the 4-bit codebook
// (NF4) codebook[q] * scale.
//
// The work is one read of W and one write of W' (HBM-bound).  The rank-r update of a
// 128-row x 128-column tile is a tcgen05 contraction over the ranks (M = 128, N = 128,
// K = 16 per instruction) into an fp32 TMEM accumulator; the epilogue adds the decoded
// weight in fp32 and rounds once to bf16 (bf16 products are exact in fp32).  W' may be
// W itself (in place): a tile is read before it is written, and tiles are disjoint.
//
// Roles: warp 0 the TMA producer, warp 1 TMEM and the single-thread MMA issue, warps
// 2..9 the epilogue in two groups of four that take alternate tiles (four TMEM
// accumulators, so both groups and the MMA stay busy).  Each epilogue warp drains its
// TMEM lane quarter (32 rows of the tile), adds the weight and TMA-stores its own 32-row
// boxes: no barrier spans warps, so the per-tile latency of one warp (TMEM load,
// shared-memory reads, arithmetic, store) overlaps the others'.  Two rings in shared
// memory: weight tiles (deep, since the stream needs ~100 KB of reads in flight per SM)
// and rank chunks (up to 64 ranks of B's 128 rows and of A's 128 columns each; narrow
// swizzles for r <= 32 so they take little room).  A bf16 weight tile is overwritten by
// its result and stored from there; a coded tile is decoded into its group's bf16
// staging tile.  The coded formats' scales are loaded one tile ahead.  Persistent, one
// CTA per SM, tiles in row-major order.  Every wait is bounded (2 s); a timeout sets
// g_merge_err, which lora_linear_merge_check reads.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "../../include/lora_linear.h"
#include "tc_gemm.cuh"  // bounded mbarrier waits, TMA, mbarrier and tcgen05 wrappers
#include "tmap.h"

namespace {

enum MergeFmt { MF_BF16 = 0, MF_Q4 = 1, MF_FP8 = 2, MF_CB = 3 };

constexpr int TM = 128, TN = 128;         // tile rows, columns
constexpr int EPI_WARPS = 8, THREADS = 64 + 32 * EPI_WARPS;
constexpr int MAX_WS = 8, MAX_OS = 4;     // ring depths (barrier arrays)
constexpr int ACC = 4;                    // TMEM accumulators of TN columns (all 512 columns)
constexpr int OUT_BYTES = TM * TN * 2;    // one bf16 tile (two 64-column boxes, 128B swizzle)
constexpr int SMEM_LIMIT = 232448;        // 227 KB per CTA
constexpr int SMEM_RESERVED = 1024 + 512; // alignment slack; barriers, codebook, TMEM slot (~310 B)

__device__ int g_merge_err;

// Bytes of one stored weight tile in each format.
__host__ __device__ constexpr int w_tile_bytes(int wf) {
    return wf == MF_BF16 ? OUT_BYTES : wf == MF_FP8 ? TM * TN : TM * TN / 2;
}

struct MergeArgs {
    CUtensorMap tmW;    // bf16 W: box {64, 128}, 128B swizzle; FP8 codes: {128 B, 128}, 128B swizzle;
                        // 4-bit codes [d_out][d_in/2]: {64 B, 128}, 64B swizzle
    CUtensorMap tmOut;  // bf16 W' box {64, 32} (one warp's rows), 128B swizzle
    CUtensorMap tmA;    // bf16 A [r][d_in] box {64, cr}, 128B swizzle (the MMA's MN-major B operand)
    CUtensorMap tmB;    // bf16 B [d_out][r] box {nb, 128}, swizzle span nb * 2 bytes (K-major A operand)
    const uint16_t *Wscale;  // bf16: 4-bit formats [d_out][d_in/64]; FP8 [d_out]
    float cb[16];            // codebook format: the 16 values
    int64_t d_in, d_out, col_tiles, tiles;
    int n_chunks;       // rank chunks per tile
    int cr;             // ranks per chunk (a multiple of 16, <= 64)
    int kr_last;        // MMA K of the last chunk (ranks past r are zero-filled by TMA)
    int nb;             // B box width: 16, 32 or 64 ranks
    int n_ws, n_os;     // ring depths
    int w_stage, o_stage, b_bytes;  // bytes
    float s;
    int *err;
};

__device__ __forceinline__ float bf16f(uint16_t b) { return __uint_as_float(static_cast<uint32_t>(b) << 16); }

// Two E4M3 codes (element 0 in the low byte) to fp32, exactly (E4M3 -> f16 -> f32).
__device__ __forceinline__ void e4m3x2_f32(uint32_t two, float &lo, float &hi) {
    asm("{\n\t.reg .b16 c, hl, hh;\n\t.reg .b32 h;\n\t"
        "cvt.u16.u32 c, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 h, c;\n\t"
        "mov.b32 {hl, hh}, h;\n\t"
        "cvt.f32.f16 %0, hl;\n\t"
        "cvt.f32.f16 %1, hh;\n\t}"
        : "=f"(lo), "=f"(hi)
        : "r"(two));
}

// Packed fp32 pairs (Blackwell's f32x2 arithmetic: two fp32 lanes per instruction, each
// rounded as its scalar form).
__device__ __forceinline__ uint64_t pack2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
// bf16x2 of (s * acc + w) for two adjacent columns: one fp32 FMA each, one rounding to bf16.
__device__ __forceinline__ uint32_t fma_bf16x2(uint32_t acc_lo, uint32_t acc_hi, uint64_t s2, uint64_t w2) {
    uint32_t out;
    asm("{\n\t.reg .b64 a, d;\n\t.reg .b32 e, o;\n\t"
        "mov.b64 a, {%1, %2};\n\t"
        "fma.rn.f32x2 d, a, %3, %4;\n\t"
        "mov.b64 {e, o}, d;\n\t"
        "cvt.rn.bf16x2.f32 %0, o, e;\n\t}"
        : "=r"(out)
        : "r"(acc_lo), "r"(acc_hi), "l"(s2), "l"(w2));
    return out;
}

// The decoded weight of this thread's row over one 64-column half c of the tile, in
// fp32, as 32 packed pairs (columns 2i, 2i + 1).  wst: the weight tile in shared
// memory, in its format's TMA layout; sc: the scale that applies (coded formats).
template <int WF>
__device__ __forceinline__ void load_w64(const uint8_t *wst, const float *cbs, int lr, int c, float sc,
                                         uint64_t (&w)[32]) {
    if (WF == MF_BF16) {
        // box c: 128 rows of 128 bytes, 16-byte piece j of row lr at (j ^ (lr & 7)) * 16
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint4 v = *reinterpret_cast<const uint4 *>(wst + c * 16384 + lr * 128 + ((j ^ (lr & 7)) << 4));
            const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e)
                w[4 * j + e] = pack2(__uint_as_float(u[e] << 16), __uint_as_float(u[e] & 0xFFFF0000u));
        }
    } else if (WF == MF_FP8) {
        // 128 rows of 128 code bytes (128B swizzle); this half is pieces 4c .. 4c+3; sc: the
        // row's scale; e4m3(q) * sc is exact in fp32
        const uint64_t sc2 = pack2(sc, sc);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint4 v = *reinterpret_cast<const uint4 *>(wst + lr * 128 + (((4 * c + j) ^ (lr & 7)) << 4));
            const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                float f0, f1, f2, f3;
                e4m3x2_f32(u[e] & 0xFFFFu, f0, f1);
                e4m3x2_f32(u[e] >> 16, f2, f3);
                w[8 * j + 2 * e] = mul2(pack2(f0, f1), sc2);
                w[8 * j + 2 * e + 1] = mul2(pack2(f2, f3), sc2);
            }
        }
    } else {
        // 128 rows of 64 code bytes (64B swizzle: piece j of row lr at (j ^ ((lr >> 1) & 3)) * 16);
        // this half is pieces 2c, 2c+1; a byte holds columns 2i (low nibble) and 2i + 1;
        // sc: the half's 64-column scale
        const uint64_t s2 = WF == MF_Q4 ? pack2(sc / 7.0f, sc / 7.0f) : pack2(sc, sc);
        constexpr uint64_t kMinus2p23p8x2 = 0xCB000008CB000008ull;  // -(2^23 + 8) in both halves
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const uint4 v =
                *reinterpret_cast<const uint4 *>(wst + lr * 64 + (((2 * c + j) ^ ((lr >> 1) & 3)) << 4));
            const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const uint32_t lo = u[e] & 0x0F0F0F0Fu, hi = (u[e] >> 4) & 0x0F0F0F0Fu;
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    uint64_t f;
                    if (WF == MF_Q4) {
                        // 2^23 + q exactly (the code under the exponent of 2^23), then q - 8
                        // exactly, then one rounding: (q - 8) * (scale / 7)
                        uint64_t t = pack2(__uint_as_float(__byte_perm(lo, 0x4B000000u, 0x7650 + b)),
                                           __uint_as_float(__byte_perm(hi, 0x4B000000u, 0x7650 + b)));
                        asm("add.rn.f32x2 %0, %1, %2;" : "=l"(f) : "l"(t), "l"(kMinus2p23p8x2));
                    } else {
                        f = pack2(cbs[(lo >> (8 * b)) & 0xFu], cbs[(hi >> (8 * b)) & 0xFu]);
                    }
                    w[16 * j + 4 * e + b] = mul2(f, s2);
                }
            }
        }
    }
}

template <int WF>
__global__ void __launch_bounds__(THREADS, 1) k_merge_tc(const __grid_constant__ MergeArgs p) {
    constexpr bool kInPlace = WF == MF_BF16;  // the result overwrites the staged weight tile
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *wring = smem;                          // n_ws weight tiles
    uint8_t *oring = wring + p.n_ws * p.w_stage;    // n_os rank chunks: [B rows | A panel]
    uint8_t *staging = oring + p.n_os * p.o_stage;  // coded formats: one bf16 output tile per group
    uint64_t *bars = reinterpret_cast<uint64_t *>(staging + (kInPlace ? 0 : 2 * OUT_BYTES));
    uint64_t *wfull = bars, *wempty = bars + MAX_WS;
    uint64_t *ofull = bars + 2 * MAX_WS, *oempty = ofull + MAX_OS;
    uint64_t *tfull = oempty + MAX_OS, *tempty = tfull + ACC;
    uint64_t *drain = tempty + ACC;
    float *cbs = reinterpret_cast<float *>(drain + 1);  // [16]
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(cbs + 16);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int b = 0; b < MAX_WS; ++b) {
            lora::mbar_init(lora::smem_u32(&wfull[b]), 1);
            lora::mbar_init(lora::smem_u32(&wempty[b]), 4);  // the 4 warps of the tile's group
        }
        for (int b = 0; b < MAX_OS; ++b) {
            lora::mbar_init(lora::smem_u32(&ofull[b]), 1);
            lora::mbar_init(lora::smem_u32(&oempty[b]), 1);
        }
        for (int b = 0; b < ACC; ++b) {
            lora::mbar_init(lora::smem_u32(&tfull[b]), 1);
            lora::mbar_init(lora::smem_u32(&tempty[b]), 4);
        }
        lora::mbar_init(lora::smem_u32(drain), 1);
        *abort_flag = 0;
        lora::fence_mbar_init();
    }
    if (threadIdx.x < 16) cbs[threadIdx.x] = p.cb[threadIdx.x];
    if (warp == 0 && lane == 0) {
        lora::tma_prefetch_desc(&p.tmW);
        lora::tma_prefetch_desc(&p.tmOut);
        lora::tma_prefetch_desc(&p.tmA);
        lora::tma_prefetch_desc(&p.tmB);
    }
    if (warp == 1) {
        lora::tmem_alloc(lora::smem_u32(tmem_slot), ACC * TN);
        lora::tmem_relinquish();
    }
    lora::tc_fence_before();
    __syncthreads();
    lora::tc_fence_after();
    // set-up above overlaps the previous kernel's tail (programmatic dependent launch);
    // nothing below touches global memory before that kernel has completed
    lora::grid_dep_wait();
    lora::grid_dep_launch_dependents();
    const uint32_t tmem_base = *tmem_slot;
    const uint32_t a_box_bytes = static_cast<uint32_t>(p.cr) * 128u;  // one 64-column box of A

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t w_issued = 0, w_ph = 0, o_issued = 0, o_ph = 0;
            int k = 0, oc = 0;
            bool ok = true;
            for (int64_t t = blockIdx.x; ok && t < p.tiles; t += gridDim.x, ++k) {
                const int row0 = static_cast<int>((t / p.col_tiles) * TM);
                const int col0 = static_cast<int>((t % p.col_tiles) * TN);
                const int ws = k % p.n_ws;
                const uint32_t wph = static_cast<uint32_t>(k / p.n_ws) & 1u;
                if (!lora::wait_bounded(lora::smem_u32(&wempty[ws]), wph ^ 1u, abort_flag, p.err,
                                        lora::DERR_WAIT_EMPTY))
                    break;
                uint8_t *wdst = wring + ws * p.w_stage;
                const uint32_t wb = lora::smem_u32(&wfull[ws]);
                lora::mbar_arrive_expect_tx(wb, static_cast<uint32_t>(p.w_stage));
                if (WF == MF_BF16) {
                    lora::tma_load_2d(lora::smem_u32(wdst), &p.tmW, wb, col0, row0);
                    lora::tma_load_2d(lora::smem_u32(wdst + 16384), &p.tmW, wb, col0 + 64, row0);
                } else if (WF == MF_FP8) {
                    lora::tma_load_2d(lora::smem_u32(wdst), &p.tmW, wb, col0, row0);
                } else {
                    lora::tma_load_2d(lora::smem_u32(wdst), &p.tmW, wb, col0 / 2, row0);
                }
                w_issued |= 1u << ws;
                w_ph = (w_ph & ~(1u << ws)) | (wph << ws);
                for (int ch = 0; ch < p.n_chunks; ++ch, ++oc) {
                    const int os = oc % p.n_os;
                    const uint32_t oph = static_cast<uint32_t>(oc / p.n_os) & 1u;
                    if (!lora::wait_bounded(lora::smem_u32(&oempty[os]), oph ^ 1u, abort_flag, p.err,
                                            lora::DERR_WAIT_EMPTY)) {
                        ok = false;
                        break;
                    }
                    uint8_t *odst = oring + os * p.o_stage;
                    const uint32_t ob = lora::smem_u32(&ofull[os]);
                    lora::mbar_arrive_expect_tx(ob, static_cast<uint32_t>(p.b_bytes) + 2u * a_box_bytes);
                    lora::tma_load_2d(lora::smem_u32(odst), &p.tmB, ob, 64 * ch, row0);
                    lora::tma_load_2d(lora::smem_u32(odst + p.b_bytes), &p.tmA, ob, col0, 64 * ch);
                    lora::tma_load_2d(lora::smem_u32(odst + p.b_bytes + a_box_bytes), &p.tmA, ob, col0 + 64,
                                      64 * ch);
                    o_issued |= 1u << os;
                    o_ph = (o_ph & ~(1u << os)) | (oph << os);
                }
            }
            // copies still in flight (only after a failed wait) land before the CTA exits
            volatile int never = 0;
            for (int b = 0; b < p.n_ws; ++b)
                if (w_issued & (1u << b))
                    lora::wait_bounded(lora::smem_u32(&wfull[b]), (w_ph >> b) & 1u, &never, p.err,
                                       lora::DERR_WAIT_DRAIN);
            for (int b = 0; b < p.n_os; ++b)
                if (o_issued & (1u << b))
                    lora::wait_bounded(lora::smem_u32(&ofull[b]), (o_ph >> b) & 1u, &never, p.err,
                                       lora::DERR_WAIT_DRAIN);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            // acc [128 rows x 128 columns] += B rows (K-major) . A panel (MN-major), chunk by chunk
            constexpr uint32_t idesc = lora::idesc_bf16(TM, TN, false, true);
            const uint32_t b_layout =
                p.nb == 16 ? lora::SDESC_SW32 : (p.nb == 32 ? lora::SDESC_SW64 : lora::SDESC_SW128);
            int k = 0, oc = 0;
            bool ok = true;
            for (int64_t t = blockIdx.x; ok && t < p.tiles; t += gridDim.x, ++k) {
                const int buf = k % ACC;
                if (!lora::wait_bounded(lora::smem_u32(&tempty[buf]), (static_cast<uint32_t>(k / ACC) & 1u) ^ 1u,
                                        abort_flag, p.err, lora::DERR_WAIT_TMEM_EMPTY))
                    break;
                lora::tc_fence_after();
                for (int ch = 0; ch < p.n_chunks; ++ch, ++oc) {
                    const int os = oc % p.n_os;
                    if (!lora::wait_bounded(lora::smem_u32(&ofull[os]), static_cast<uint32_t>(oc / p.n_os) & 1u,
                                            abort_flag, p.err, lora::DERR_WAIT_FULL)) {
                        ok = false;
                        break;
                    }
                    lora::tc_fence_after();
                    const uint32_t bsm = lora::smem_u32(oring + os * p.o_stage);
                    // B rows: rows of nb ranks, 8-row swizzle atoms nb * 16 bytes apart; a K
                    // step of 16 ranks is 32 bytes along the row
                    const uint64_t ad = lora::sdesc(bsm, 16, static_cast<uint32_t>(p.nb) * 16u, b_layout);
                    // A panel: two 64-column boxes (LBO apart), 8-rank atoms 1024 bytes apart;
                    // a K step of 16 ranks is 2048 bytes
                    const uint64_t bd = lora::sdesc_sw128(bsm + p.b_bytes, a_box_bytes, 1024);
                    const int ksteps = (ch == p.n_chunks - 1 ? p.kr_last : p.cr) / 16;
                    for (int kk = 0; kk < ksteps; ++kk)
                        lora::tc_mma_bf16(tmem_base + static_cast<uint32_t>(buf * TN), ad + (kk * 32 >> 4),
                                          bd + (kk * 2048 >> 4), idesc, (ch > 0 || kk > 0) ? 1u : 0u);
                    lora::tc_commit(lora::smem_u32(&oempty[os]));
                }
                if (!ok) break;
                lora::tc_commit(lora::smem_u32(&tfull[buf]));
            }
            lora::tc_commit(lora::smem_u32(drain));
            volatile int never = 0;
            lora::wait_bounded(lora::smem_u32(drain), 0, &never, p.err, lora::DERR_WAIT_DRAIN);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        // Every warp works on its own: warp group g = (warp - 2) / 4 takes the CTA's tiles
        // k = g, g + 2, ...; within a tile, warp w drains TMEM lane quarter w % 4 (32 rows,
        // all 128 columns) and stores its own 32-row boxes, so no barrier spans warps.
        const int q = warp & 3;          // TMEM lane quarter (warps 2..9 -> 2, 3, 0, 1, 2, 3, 0, 1)
        const int g = (warp - 2) >> 2;   // warp group
        const int lr = q * 32 + lane;    // accumulator row = tile row
        const uint64_t s2 = pack2(p.s, p.s);
        uint8_t *const stage_out = staging + g * OUT_BYTES;  // coded formats: this group's output tile
        // scales of tile t for this thread's row: FP8 one per row; 4-bit one per 64 columns
        auto load_scales = [&](int64_t t, float &s0, float &s1) {
            s0 = s1 = 0.f;
            if (WF == MF_BF16 || t >= p.tiles) return;
            const int64_t row = (t / p.col_tiles) * TM + lr, col0 = (t % p.col_tiles) * TN;
            if (row >= p.d_out) return;
            if (WF == MF_FP8) {
                s0 = s1 = bf16f(p.Wscale[row]);
            } else {
                const uint16_t *sr = p.Wscale + row * (p.d_in / 64) + col0 / 64;
                s0 = bf16f(sr[0]);
                if (col0 + 64 < p.d_in) s1 = bf16f(sr[1]);
            }
        };
        float sc0, sc1;
        load_scales(blockIdx.x + static_cast<int64_t>(g) * gridDim.x, sc0, sc1);
        for (int k = g;; k += 2) {
            const int64_t t = blockIdx.x + static_cast<int64_t>(k) * gridDim.x;
            if (t >= p.tiles) break;
            const int buf = k % ACC, ws = k % p.n_ws;
            const uint32_t wph = static_cast<uint32_t>(k / p.n_ws) & 1u;
            // the next tile's scales load while this one is processed (DRAM latency off the path)
            float nx0, nx1;
            load_scales(t + 2 * static_cast<int64_t>(gridDim.x), nx0, nx1);
            const bool ok = lora::wait_bounded(lora::smem_u32(&tfull[buf]), static_cast<uint32_t>(k / ACC) & 1u,
                                               abort_flag, p.err, lora::DERR_WAIT_TMEM_FULL) &&
                            lora::wait_bounded(lora::smem_u32(&wfull[ws]), wph, abort_flag, p.err,
                                               lora::DERR_WAIT_FULL);
            if (!__all_sync(0xFFFFFFFFu, ok)) break;  // the warp leaves together
            lora::tc_fence_after();
            const int64_t row0 = (t / p.col_tiles) * TM;
            const int64_t col0 = (t % p.col_tiles) * TN;
            const uint8_t *wst = wring + ws * p.w_stage;
            uint8_t *out = kInPlace ? wring + ws * p.w_stage : stage_out;
            if (!kInPlace) {
                // this warp's rows of the group's output tile: its previous store has read them
                if (lane == 0) lora::bulk_wait_group_read<0>();
                __syncwarp();
            }
            const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(buf * TN);
#pragma unroll 1
            for (int c = 0; c < 2; ++c) {
                uint32_t v0[32], v1[32];
                lora::tmem_ld_32x32b_x32(t_row + c * 64, v0);
                lora::tmem_ld_32x32b_x32(t_row + c * 64 + 32, v1);
                uint64_t w[32];
                load_w64<WF>(wst, cbs, lr, c, c == 0 ? sc0 : sc1, w);
                lora::tc_wait_ld();
                if (c == 1) {
                    lora::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) lora::mbar_arrive(lora::smem_u32(&tempty[buf]));
                }
                // (in place, a thread overwrites exactly the 64 weights of its row it has just read)
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    uint32_t o[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int col = 8 * j + 2 * e;  // even: the pair never straddles v0 / v1
                        o[e] = col < 32 ? fma_bf16x2(v0[col], v0[col + 1], s2, w[4 * j + e])
                                        : fma_bf16x2(v1[col - 32], v1[col - 31], s2, w[4 * j + e]);
                    }
                    *reinterpret_cast<uint4 *>(out + c * 16384 + lr * 128 + ((j ^ (lr & 7)) << 4)) =
                        make_uint4(o[0], o[1], o[2], o[3]);
                }
            }
            lora::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                if (!kInPlace) lora::mbar_arrive(lora::smem_u32(&wempty[ws]));  // the codes are decoded
                // this warp's 32 rows: two boxes of 64 columns (the 128B swizzle repeats every
                // 8 rows, so a 32-row box at row 32q of the tile has the tile's layout)
                if (row0 + 32 * q < p.d_out)
                    for (int cc = 0; cc < 2; ++cc)
                        if (col0 + 64 * cc < p.d_in)  // a box wholly past the weight has nothing to store
                            lora::tma_store_2d(&p.tmOut, lora::smem_u32(out + cc * 16384 + q * 32 * 128),
                                               static_cast<int32_t>(col0 + 64 * cc),
                                               static_cast<int32_t>(row0 + 32 * q));
                lora::bulk_commit_group();
                if (kInPlace) {
                    // the stage holds the output until the store has read it
                    lora::bulk_wait_group_read<0>();
                    lora::mbar_arrive(lora::smem_u32(&wempty[ws]));
                }
            }
            __syncwarp();
            sc0 = nx0;
            sc1 = nx1;
        }
        if (lane == 0) lora::bulk_wait_group<0>();
    }

    // ---------------------------------------------------------------- teardown
    __syncwarp();
    lora::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        lora::tc_fence_after();
        lora::tmem_dealloc(tmem_base, ACC * TN);
    }
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The weight as the caller stores it.
struct MergeWeight {
    int wf = MF_BF16;
    const void *w = nullptr;          // bf16 W, or the codes
    const uint16_t *scale = nullptr;  // coded formats
    const float *codebook = nullptr;  // MF_CB: 16 values (host)
};

// Every pointer 16-byte aligned (TMA), sizes within the tensor maps' ranges.
lora_status_t merge_checks(const MergeWeight &mw, const void *A, const void *B, const void *Wout, int64_t d_in,
                           int64_t d_out, int r, float alpha) {
    const bool coded = mw.wf != MF_BF16;
    if (!mw.w || !A || !B || !Wout || (coded && !mw.scale) || (mw.wf == MF_CB && !mw.codebook))
        return LORA_ERR_INVALID_ARG;
    if (d_in < 8 || d_out < 1 || d_in % 8) return LORA_ERR_INVALID_ARG;
    if ((mw.wf == MF_Q4 || mw.wf == MF_CB) && d_in % 64) return LORA_ERR_INVALID_ARG;
    if (mw.wf == MF_FP8 && d_in % 16) return LORA_ERR_INVALID_ARG;
    if (d_in > (int64_t(1) << 24) || d_out > (int64_t(1) << 24)) return LORA_ERR_INVALID_ARG;
    if (r < 1 || r > 256 || r % 8) return LORA_ERR_INVALID_ARG;
    if (!(alpha == alpha) || alpha > 3.4e38f || alpha < -3.4e38f) return LORA_ERR_INVALID_ARG;
    if (mw.wf == MF_CB)
        for (int i = 0; i < 16; ++i)
            if (!std::isfinite(mw.codebook[i])) return LORA_ERR_INVALID_ARG;
    if (!aligned16(mw.w) || !aligned16(A) || !aligned16(B) || !aligned16(Wout) || (coded && !aligned16(mw.scale)))
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

// Ring depths: the rank-chunk ring gets about 64 KB (2 to 4 chunks), the weight ring
// the rest, up to 8 tiles.
void merge_rings(int wf, int o_stage, int &n_ws, int &n_os) {
    n_os = std::max(2, std::min(MAX_OS, 65536 / o_stage));
    const int staging = wf == MF_BF16 ? 0 : 2 * OUT_BYTES;
    const int avail = SMEM_LIMIT - SMEM_RESERVED - staging - n_os * o_stage;
    n_ws = std::min(MAX_WS, avail / w_tile_bytes(wf));
}

// Programmatic dependent launch, as for the layer's kernels (LORA_LINEAR_PDL=0 turns it
// off, for measurement): merges of a model's layers run back to back, and each one's
// launch and set-up overlap the previous one's last tiles.
bool merge_pdl_enabled() {
    const char *v = std::getenv("LORA_LINEAR_PDL");
    return !(v && v[0] == '0');
}

template <int WF>
cudaError_t merge_kernel_launch(const MergeArgs &a, int grid, cudaStream_t st) {
    const int smem = SMEM_RESERVED + a.n_ws * a.w_stage + a.n_os * a.o_stage + (WF == MF_BF16 ? 0 : 2 * OUT_BYTES);
    cudaError_t e = cudaFuncSetAttribute(k_merge_tc<WF>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = merge_pdl_enabled() ? 1 : 0;
    e = cudaLaunchKernelEx(&cfg, k_merge_tc<WF>, a);
    return e == cudaSuccess ? cudaGetLastError() : e;
}

lora_status_t merge_launch(const MergeWeight &mw, const uint16_t *A, const uint16_t *B, uint16_t *Wout, int64_t d_in,
                           int64_t d_out, int r, float alpha, void *stream) {
    int dev = 0, major = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return LORA_ERR_CUDA;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return LORA_ERR_CUDA;
    if (major != 10) return LORA_ERR_UNSUPPORTED;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return LORA_ERR_CUDA;
    int *err = merge_err_word(dev);
    if (!err) return LORA_ERR_CUDA;

    MergeArgs a;
    std::memset(&a, 0, sizeof(a));
    const int kr = (r + 15) / 16 * 16;
    a.n_chunks = (kr + 63) / 64;
    a.cr = std::min(kr, 64);
    a.kr_last = kr - 64 * (a.n_chunks - 1);
    a.nb = kr <= 16 ? 16 : (kr <= 32 ? 32 : 64);
    a.b_bytes = TM * a.nb * 2;
    a.o_stage = a.b_bytes + 2 * a.cr * 128;
    a.w_stage = w_tile_bytes(mw.wf);
    merge_rings(mw.wf, a.o_stage, a.n_ws, a.n_os);
    const CUtensorMapSwizzle b_swz = a.nb == 16   ? CU_TENSOR_MAP_SWIZZLE_32B
                                     : a.nb == 32 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                  : CU_TENSOR_MAP_SWIZZLE_128B;
    bool maps = true;
    switch (mw.wf) {
        case MF_BF16:
            maps = lora_host::tmap_2d(&a.tmW, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, mw.w, d_in, d_out, 64, TM,
                                      CU_TENSOR_MAP_SWIZZLE_128B);
            break;
        case MF_FP8:
            maps = lora_host::tmap_2d(&a.tmW, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, mw.w, d_in, d_out, TN, TM,
                                      CU_TENSOR_MAP_SWIZZLE_128B);
            break;
        default:
            maps = lora_host::tmap_2d(&a.tmW, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, mw.w, d_in / 2, d_out, TN / 2, TM,
                                      CU_TENSOR_MAP_SWIZZLE_64B);
    }
    maps = maps &&
           lora_host::tmap_2d(&a.tmOut, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Wout, d_in, d_out, 64, 32,
                              CU_TENSOR_MAP_SWIZZLE_128B) &&
           lora_host::tmap_2d(&a.tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, A, d_in, r, 64, a.cr,
                              CU_TENSOR_MAP_SWIZZLE_128B) &&
           lora_host::tmap_2d(&a.tmB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, B, r, d_out, a.nb, TM, b_swz);
    if (!maps) return LORA_ERR_CUDA;
    a.Wscale = mw.scale;
    if (mw.wf == MF_CB)
        for (int i = 0; i < 16; ++i) a.cb[i] = mw.codebook[i];
    a.d_in = d_in;
    a.d_out = d_out;
    a.col_tiles = (d_in + TN - 1) / TN;
    a.tiles = ((d_out + TM - 1) / TM) * a.col_tiles;
    a.s = alpha / static_cast<float>(r);
    a.err = err;
    const int grid = static_cast<int>(std::min<int64_t>(a.tiles, sms));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaSuccess;
    switch (mw.wf) {
        case MF_BF16: e = merge_kernel_launch<MF_BF16>(a, grid, st); break;
        case MF_Q4: e = merge_kernel_launch<MF_Q4>(a, grid, st); break;
        case MF_FP8: e = merge_kernel_launch<MF_FP8>(a, grid, st); break;
        default: e = merge_kernel_launch<MF_CB>(a, grid, st);
    }
    return e == cudaSuccess ? LORA_OK : LORA_ERR_CUDA;
}

lora_status_t merge(const MergeWeight &mw, const uint16_t *A, const uint16_t *B, uint16_t *W_out, int64_t d_in,
                    int64_t d_out, int r, float alpha, void *stream) {
    const lora_status_t st = merge_checks(mw, A, B, W_out, d_in, d_out, r, alpha);
    if (st != LORA_OK) return st;
    return merge_launch(mw, A, B, W_out, d_in, d_out, r, alpha, stream);
}

}  // namespace

extern "C" LORA_API lora_status_t lora_linear_merge(const uint16_t *W, const uint16_t *A, const uint16_t *B,
                                                    uint16_t *W_out, int64_t d_in, int64_t d_out, int r, float alpha,
                                                    void *stream) {
    MergeWeight mw;
    mw.w = W;
    return merge(mw, A, B, W_out, d_in, d_out, r, alpha, stream);
}

extern "C" LORA_API lora_status_t lora_linear_merge_q4(const uint8_t *Wq, const uint16_t *Wscale, const uint16_t *A,
                                                       const uint16_t *B, uint16_t *W_out, int64_t d_in, int64_t d_out,
                                                       int r, float alpha, void *stream) {
    MergeWeight mw;
    mw.wf = MF_Q4;
    mw.w = Wq;
    mw.scale = Wscale;
    return merge(mw, A, B, W_out, d_in, d_out, r, alpha, stream);
}

extern "C" LORA_API lora_status_t lora_linear_merge_fp8(const uint8_t *W8, const uint16_t *W8scale, const uint16_t *A,
                                                        const uint16_t *B, uint16_t *W_out, int64_t d_in,
                                                        int64_t d_out, int r, float alpha, void *stream) {
    MergeWeight mw;
    mw.wf = MF_FP8;
    mw.w = W8;
    mw.scale = W8scale;
    return merge(mw, A, B, W_out, d_in, d_out, r, alpha, stream);
}

extern "C" LORA_API lora_status_t lora_linear_merge_nf4(const uint8_t *Wq, const uint16_t *Wscale,
                                                        const float *codebook, const uint16_t *A, const uint16_t *B,
                                                        uint16_t *W_out, int64_t d_in, int64_t d_out, int r,
                                                        float alpha, void *stream) {
    MergeWeight mw;
    mw.wf = MF_CB;
    mw.w = Wq;
    mw.scale = Wscale;
    mw.codebook = codebook;
    return merge(mw, A, B, W_out, d_in, d_out, r, alpha, stream);
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
