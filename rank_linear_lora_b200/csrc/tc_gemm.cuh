// tc_gemm.cuh -- the tcgen05 contraction engine behind every step of the layer.
//
// One persistent, warp-specialised kernel template computes 128 x BN output tiles
//     D = sum over K-segments  A_seg . B_seg^T
// with bf16 operands staged by TMA into 128-byte-swizzled shared memory and fp32
// accumulators in tensor memory:
//   warp 0      TMA producer (one elected lane), STAGES-deep smem ring
//   warp 1      TMEM allocator and single-thread tcgen05.mma issuer
//   warps 2..5  epilogue: tcgen05.ld of their 32-lane TMEM quarter
// Two accumulators alternate in TMEM so the epilogue of one work item overlaps the
// K loop of the next.
//
// K-segments: segment 0 is the frozen-weight contraction (K = d_in or d_out);
// segment 1, when present, is the rank-r side product appended to the same K loop
// (K = r), so the low-rank term is added by the tensor cores inside the same
// accumulator instead of by a separate pass.  Operands may be K-major (the K index
// contiguous in memory) or MN-major (the M/N index contiguous), so W is read in
// place for both x.W^T and dY.W.
//
// Work items and epilogues:
//   EPI_STORE  (h, dX) whole tiles in grouped raster order, `dp_waves` per CTA; when
//              the tile count leaves a partial last wave of `tail_tiles` tiles, each of
//              them is cut along N into `tail_split` narrower tiles (128 x 128 or
//              128 x 64, full K) taken by one CTA each, so the last wave is shorter and
//              every output element is still produced by one accumulator.  Stores go
//              through 128B-swizzled smem staging and TMA.
//   EPI_SPLITK (s.xa, s.g, dB, dA) skinny outputs, K split over CTAs; the last split
//              to finish a tile sums the fp32 partials in split order and writes bf16
//              rows, fp32 rows or fp32 columns (dA, written transposed).
//
// Launch: programmatic dependent launch is honoured -- set-up (barrier init, TMEM
// allocation, descriptor prefetch) runs before griddepcontrol.wait; every global
// memory access comes after it.
//
// Every wait is bounded (globaltimer); on expiry the kernel records an error code,
// drains its outstanding copies and MMAs, frees TMEM and returns.
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"

namespace lora {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int NUM_THREADS = 192;
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;  // 2 s per wait

enum EpiMode { EPI_STORE = 0, EPI_SPLITK = 1 };
enum OutMode { OUT_BF16_ROWS = 0, OUT_F32_ROWS = 1, OUT_F32_COLS = 2 };

// Error codes written to the workspace error word (first writer wins).
enum DevErr {
    DERR_NONE = 0,
    DERR_WAIT_EMPTY = 0x101,
    DERR_WAIT_FULL = 0x102,
    DERR_WAIT_TMEM_EMPTY = 0x103,
    DERR_WAIT_TMEM_FULL = 0x104,
    DERR_WAIT_DRAIN = 0x105,
    DERR_WAIT_PARTIAL = 0x106,  // a K-split tail tile's first half never published its partial
};

// One skinny split-K problem: output [rows_valid, n_valid] over K = kb0 * 64.
struct SkinnyJob {
    int m_tiles;             // 128-row output tiles
    int kb0;                 // 64-wide K blocks
    int splits;              // K splits (each a CTA tile)
    int kb_per_split;
    int num_tiles;           // m_tiles * splits
    int rows_valid;          // valid output rows
    int n_valid;             // valid output columns (r)
    int out_mode;            // OutMode
    float out_scale;
    float *part;             // fp32 partials [splits][m_tiles*BM][n_valid]
    int *counters;           // per-tile arrival counters (zero on entry, zero on exit)
    void *out;
    int64_t out_ld;          // OUT_F32_COLS: row stride of the transposed output
};

struct GemmArgs {
    CUtensorMap tmA0, tmB0;  // segment 0
    CUtensorMap tmA1, tmB1;  // segment 1 (rank-r tail), used when kb1 > 0
    CUtensorMap tmC;         // EPI_STORE output (bf16, box 64 x 32, 128B swizzle)
    CUtensorMap tmB0n, tmB1n;  // K-major B with box rows BN / tail_split (narrow tail tiles); see b3d
    CUtensorMap tmQ;           // 4-bit frozen weight: packed codes (uint8), no swizzle
    int m_tiles, n_tiles;
    int kb0, kb1;            // 64-wide K blocks per segment
    int mma_last1;           // K=16 MMAs in the last block of segment 1 (1..4)
    int num_tiles;
    // EPI_SPLITK: one or two independent skinny problems in one launch; job 0 reads
    // tmA0/tmB0, job 1 tmA1/tmB1.  Tiles of job 0 come first.
    int n_jobs;
    SkinnyJob job[2];
    // EPI_STORE
    int group_m;             // rasterisation: M tiles per group
    int dp_tiles;            // tiles done whole (raster order 0 .. dp_tiles-1)
    int dp_waves;            // whole tiles per CTA (at most)
    int tail_tiles;          // last-wave tiles cut along N (raster dp_tiles ..)
    int tail_split;          // 1 (none), 2 or 4 narrow tiles per tail tile
    // 4-bit frozen weight: bf16 scales [scale_rows][scale_ld], one per 64 codes along d_in
    const uint16_t *wscale;
    int scale_ld;
    int scale_rows;
    float cb[16];            // 4-bit codebook weight: the 16 values of the code
    int *err;                // device error word
    unsigned long long *trace;  // optional per-CTA timestamps (TRACE_WORDS each), or null
    // 1: this kernel reads nothing its stream predecessor writes, so it starts its work
    // without waiting and waits for the predecessor only before it exits; its own
    // completion then still implies the predecessor's (stream order is kept).
    int defer_dep_wait;
    // CTA-pair GEMM, bf16 weight: 1 cuts each last-wave tile along K into two items on
    // two clusters; the first hands its fp32 accumulator over through ks_part and raises
    // its flag in ks_flag (zero on entry, cleared by the reader), the second adds it.
    int tail_ksplit;
    float *ks_part;          // [tail tile][CTA rank][chunk (4)][16-byte column group (16)][row (128)] float4
    int *ks_flag;            // [tail tile][CTA rank]
    // CTA-pair GEMM, MN-major bf16 weight: 1 when tmB0 is the 3D column-chunk map, so a
    // CTA's 128 weight columns of a K block come in one copy instead of two; tmB0n is
    // then the weight's 2D map {64, 64}, for the 64-column halves of split tail tiles.
    int b3d;
};

// Release / acquire of a global int at GPU scope (the K-split tail's hand-over).
__device__ __forceinline__ void st_release_gpu(int *p, int v) {
    asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ int ld_acquire_gpu(const int *p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Trace record of one CTA (globaltimer ns unless noted).
enum TraceField {
    TR_ENTRY = 0, TR_SETUP = 1, TR_PROD_END = 2, TR_MMA_END = 3, TR_EPI_END = 4, TR_EXIT = 5,
    TR_SMID = 6, TR_TILES = 7, TR_TILE_DONE0 = 8,  // epilogue completion of the first 8 items
    TR_WAIT_EMPTY = 16,  // total ns the producer waited for free stages
    TR_WAIT_TEMPTY = 18, // total ns the MMA issuer waited for a drained accumulator
    TR_KBLOCKS = 19,     // K blocks consumed by the MMA issuer
    TR_CLK_SETUP = 20,   // SM cycle counter after set-up
    TR_CLK_EXIT = 21,    // SM cycle counter at exit (with TR_SETUP/TR_EXIT gives the SM clock)
    // CTA-pair kernel, SM cycles: the MMA issuer's waits for A tiles (full) and, 4-bit
    // weight, for decoded B tiles (B-ready); the first dequant warp's waits for packed
    // codes, its code reads and scale preparation (DECODE), decode + stores + publish
    // (PUBLISH), waits for a free B tile (SLOT) and code-fetch issue (ISSUE).
    TR_MMA_WAIT_A = 22, TR_MMA_WAIT_B = 23, TR_DQ_WAIT = 24, TR_DQ_DECODE = 25, TR_DQ_PUBLISH = 26,
    TR_DQ_SLOT = 27, TR_DQ_ISSUE = 28,
    TRACE_WORDS = 32
};

template <int BN, bool A_MN, bool B_MN, int EPI, int STAGES>
struct GemmCfg {
    static constexpr int A_BYTES = BM * BK * 2;   // 16 KB
    static constexpr int B_BYTES = BN * BK * 2;   // BN rows (or BN/64 chunks) x 128 B
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int EPI_BYTES = (EPI == EPI_STORE) ? 4 * 2 * 32 * 128 : 0;
    static constexpr int TMEM_COLS = (2 * BN < 32) ? 32 : 2 * BN;
    static constexpr int BAR_BYTES = 256;
    static constexpr int SMEM_BYTES = 1024 /*align slack*/ + STAGES * STAGE_BYTES + EPI_BYTES + BAR_BYTES;
    static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N for M=128 is 16..256 step 16");
    static_assert(!B_MN || BN % 64 == 0, "MN-major B uses 64-wide swizzle chunks");
    static_assert(B_BYTES % 1024 == 0, "stage tiles must stay 1024-byte aligned");
    static_assert((TMEM_COLS & (TMEM_COLS - 1)) == 0 && TMEM_COLS <= 512, "TMEM alloc is a power of 2");
    static_assert(EPI != EPI_STORE || BN % 64 == 0, "store epilogue works in 64-column chunks");
    static_assert(SMEM_BYTES <= 232448, "at most 227 KB of shared memory per CTA");
};

// Bounded mbarrier wait.  Returns false (and raises the abort flag and the error
// word) if the barrier does not reach `parity` within `limit_ns` (WAIT_LIMIT_NS unless
// a self-test shortens it), or if another role already aborted.
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                             int *err, int code, uint64_t limit_ns = WAIT_LIMIT_NS) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 31u) == 0) {
            if (*abort_flag) return false;
            if (globaltimer_ns() - t0 > limit_ns) {
                *abort_flag = 1;
                atomicCAS(err, 0, code);
                return false;
            }
        }
    }
}

// Bounded wait until a monotonic shared-memory counter reaches `target` (acquire);
// false on timeout or abort, as wait_bounded.  Polls with a short sleep so that a
// waiting thread takes little shared-memory bandwidth from the tensor core.
__device__ __forceinline__ bool wait_count_bounded(uint32_t addr, uint32_t target, volatile int *abort_flag,
                                                   int *err, int code) {
    if (ld_acquire_shared(addr) >= target) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t i = 1;; ++i) {
        __nanosleep(32);
        if (ld_acquire_shared(addr) >= target) return true;
        if ((i & 31u) == 0) {
            if (*abort_flag) return false;
            if (globaltimer_ns() - t0 > WAIT_LIMIT_NS) {
                *abort_flag = 1;
                atomicCAS(err, 0, code);
                return false;
            }
        }
    }
}

// Bounded wait until a global flag is nonzero (acquire at GPU scope); false on timeout
// (recording `code`) or abort, as wait_bounded.
__device__ __forceinline__ bool wait_flag_bounded(const int *flag, volatile int *abort_flag, int *err, int code) {
    if (ld_acquire_gpu(flag) != 0) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t i = 1;; ++i) {
        __nanosleep(64);
        if (ld_acquire_gpu(flag) != 0) return true;
        if ((i & 31u) == 0) {
            if (*abort_flag) return false;
            if (globaltimer_ns() - t0 > WAIT_LIMIT_NS) {
                *abort_flag = 1;
                atomicCAS(err, 0, code);
                return false;
            }
        }
    }
}

// One unit of work of a CTA: output tile (m, n), K blocks [kb_lo, kb_hi) of the
// concatenated segments, and how its result is finished.
struct WorkItem {
    int m, n;
    int kb_lo, kb_hi;
    int job;     // EPI_SPLITK: which problem
    int piece;   // EPI_SPLITK: split index
    int col0;    // EPI_STORE: first output column
    int nsplit;  // EPI_STORE: 1 for a whole tile, else tail_split (width BN / nsplit)
};

__device__ __forceinline__ void raster(const GemmArgs &p, int t, int &m, int &n) {
    // Grouped rasterisation: group_m M-tiles share each B (weight) tile in L2.
    const int group = p.group_m * p.n_tiles;
    const int g = t / group, idx = t % group;
    const int m0 = g * p.group_m;
    const int gm = min(p.group_m, p.m_tiles - m0);
    m = m0 + idx % gm;
    n = idx / gm;
}

// Item i (0, 1, ...) of this CTA; false when the CTA has no more work.
template <int BN, int EPI>
__device__ __forceinline__ bool get_item(const GemmArgs &p, int i, WorkItem &w) {
    const int G = gridDim.x, c = blockIdx.x;
    if (EPI == EPI_SPLITK) {
        int t = c + i * G;
        w.job = 0;
        if (t >= p.job[0].num_tiles) {
            t -= p.job[0].num_tiles;
            w.job = 1;
            if (p.n_jobs < 2 || t >= p.job[1].num_tiles) return false;
        }
        const SkinnyJob &J = p.job[w.job];
        w.piece = t % J.splits;
        const int mt = t / J.splits;
        w.m = mt % J.m_tiles;
        w.n = 0;
        w.kb_lo = w.piece * J.kb_per_split;
        w.kb_hi = min(J.kb0, w.kb_lo + J.kb_per_split);
        w.col0 = 0;
        w.nsplit = 1;
        return true;
    }
    w.job = 0;
    w.kb_lo = 0;
    w.kb_hi = p.kb0 + p.kb1;
    w.piece = 0;
    if (i < p.dp_waves) {
        const int t = c + i * G;
        if (t >= p.dp_tiles) return false;
        raster(p, t, w.m, w.n);
        w.nsplit = 1;
        w.col0 = w.n * BN;
        return true;
    }
    if (i == p.dp_waves && p.tail_split > 1 && c < p.tail_tiles * p.tail_split) {
        const int tt = c / p.tail_split, h = c % p.tail_split;
        raster(p, p.dp_tiles + tt, w.m, w.n);
        w.nsplit = p.tail_split;
        w.col0 = w.n * BN + h * (BN / p.tail_split);
        return true;
    }
    return false;
}

// Pack 64 fp32 columns of one accumulator row to bf16 and write them into row `lane`
// of a 32 x 64 staging box with the 128-byte swizzle TMA expects (16-byte chunk cc of
// row r lands at chunk cc ^ (r % 8)).
__device__ __forceinline__ void stage_row64(uint8_t *sbuf, int lane, const uint32_t (&v0)[32],
                                            const uint32_t (&v1)[32]) {
    uint32_t packed[32];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        __nv_bfloat162 lo2 = __floats2bfloat162_rn(__uint_as_float(v0[2 * j]), __uint_as_float(v0[2 * j + 1]));
        __nv_bfloat162 hi2 = __floats2bfloat162_rn(__uint_as_float(v1[2 * j]), __uint_as_float(v1[2 * j + 1]));
        packed[j] = *reinterpret_cast<uint32_t *>(&lo2);
        packed[16 + j] = *reinterpret_cast<uint32_t *>(&hi2);
    }
    uint8_t *row_ptr = sbuf + lane * 128;
#pragma unroll
    for (int cc = 0; cc < 8; ++cc) {
        uint4 w = make_uint4(packed[4 * cc], packed[4 * cc + 1], packed[4 * cc + 2], packed[4 * cc + 3]);
        *reinterpret_cast<uint4 *>(row_ptr + ((cc ^ (lane & 7)) * 16)) = w;
    }
}

// Half of stage_row64: 32 fp32 columns (half 0: columns 0..31, half 1: 32..63) of one
// accumulator row into their four swizzled 16-byte chunks; for kernels short of registers.
__device__ __forceinline__ void stage_row32(uint8_t *sbuf, int lane, int half, const uint32_t (&v)[32]) {
    uint8_t *row_ptr = sbuf + lane * 128;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(v[8 * q + 2 * e]), __uint_as_float(v[8 * q + 2 * e + 1]));
            w[e] = *reinterpret_cast<uint32_t *>(&b2);
        }
        const int cc = half * 4 + q;
        *reinterpret_cast<uint4 *>(row_ptr + ((cc ^ (lane & 7)) * 16)) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

template <int BN, bool A_MN, bool B_MN, int EPI, int STAGES>
__global__ void __launch_bounds__(NUM_THREADS, 1) k_tc_gemm(const __grid_constant__ GemmArgs p) {
    using Cfg = GemmCfg<BN, A_MN, B_MN, EPI, STAGES>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem;
    uint8_t *sB = smem + STAGES * Cfg::A_BYTES;
    uint8_t *sEpi = smem + STAGES * Cfg::STAGE_BYTES;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sEpi + Cfg::EPI_BYTES);
    uint64_t *full_bar = bars;                    // [STAGES]
    uint64_t *empty_bar = bars + STAGES;          // [STAGES]
    uint64_t *tfull_bar = bars + 2 * STAGES;      // [2]
    uint64_t *tempty_bar = bars + 2 * STAGES + 2; // [2]
    uint64_t *drain_bar = bars + 2 * STAGES + 4;  // [1]
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * STAGES + 5);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    volatile int *last_flag = reinterpret_cast<volatile int *>(tmem_slot + 2);
    volatile int *epi_ok = reinterpret_cast<volatile int *>(tmem_slot + 3);  // [2]

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    unsigned long long *trace = p.trace ? p.trace + static_cast<size_t>(blockIdx.x) * TRACE_WORDS : nullptr;
    if (trace && threadIdx.x == 0) {
        uint32_t smid;
        asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
        trace[TR_ENTRY] = globaltimer_ns();
        trace[TR_SMID] = smid;
    }

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_u32(&full_bar[s]), 1);
            mbar_init(smem_u32(&empty_bar[s]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&tfull_bar[b]), 1);
            mbar_init(smem_u32(&tempty_bar[b]), 4);
        }
        mbar_init(smem_u32(drain_bar), 1);
        *abort_flag = 0;
        *last_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&p.tmA0);
        tma_prefetch_desc(&p.tmB0);
        if (p.kb1 > 0 || p.n_jobs > 1) {
            tma_prefetch_desc(&p.tmA1);
            tma_prefetch_desc(&p.tmB1);
        }
        if (EPI == EPI_STORE) tma_prefetch_desc(&p.tmC);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), Cfg::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // Everything above touched no global memory; from here on we may read what the
    // previous kernel in the stream wrote and overwrite what it read (unless this kernel
    // is independent of it, see defer_dep_wait).
    if (!p.defer_dep_wait) grid_dep_wait();
    grid_dep_launch_dependents();
    if (trace && threadIdx.x == 0) {
        trace[TR_SETUP] = globaltimer_ns();
        trace[TR_CLK_SETUP] = clock64();
    }

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued_mask = 0, issued_phase = 0;  // per stage: issued?, parity of last issue
            bool ok = true;
            WorkItem w;
            for (int i = 0; ok && get_item<BN, EPI>(p, i, w); ++i) {
                for (int kb = w.kb_lo; kb < w.kb_hi; ++kb) {
                    if (!wait_bounded(smem_u32(&empty_bar[stage]), phase ^ 1u, abort_flag, p.err,
                                      DERR_WAIT_EMPTY)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = smem_u32(&full_bar[stage]);
                    const int bn = BN / w.nsplit;  // columns of B this item loads
                    mbar_arrive_expect_tx(fb, Cfg::A_BYTES + bn * BK * 2);
                    issued_mask |= 1u << stage;
                    issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
                    // Second map pair: the rank-r K segment (EPI_STORE) or job 1 (EPI_SPLITK).
                    const bool seg1 = (EPI == EPI_SPLITK) ? (w.job == 1) : (kb >= p.kb0);
                    const CUtensorMap *ta = seg1 ? &p.tmA1 : &p.tmA0;
                    const CUtensorMap *tb = seg1 ? &p.tmB1 : &p.tmB0;
                    const int k0 = ((EPI == EPI_STORE && seg1) ? kb - p.kb0 : kb) * BK;
                    const uint32_t a_dst = smem_u32(sA + stage * Cfg::A_BYTES);
                    const uint32_t b_dst = smem_u32(sB + stage * Cfg::B_BYTES);
                    if (A_MN) {
                        tma_load_2d(a_dst, ta, fb, w.m * BM, k0);
                        tma_load_2d(a_dst + 64 * 128, ta, fb, w.m * BM + 64, k0);
                    } else {
                        tma_load_2d(a_dst, ta, fb, k0, w.m * BM);
                    }
                    if (B_MN) {
                        for (int j = 0; j < bn / 64; ++j)
                            tma_load_2d(b_dst + j * 64 * 128, tb, fb, w.col0 + 64 * j, k0);
                    } else if (w.nsplit == 1) {
                        tma_load_2d(b_dst, tb, fb, k0, w.col0);
                    } else {
                        tma_load_2d(b_dst, seg1 ? &p.tmB1n : &p.tmB0n, fb, k0, w.col0);
                    }
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // Drain: every issued copy must have landed before the CTA exits.
            for (int s = 0; s < STAGES; ++s)
                if (issued_mask & (1u << s)) {
                    volatile int never = 0;
                    wait_bounded(smem_u32(&full_bar[s]), (issued_phase >> s) & 1u, &never, p.err,
                                 DERR_WAIT_DRAIN);
                }
            if (trace) trace[TR_PROD_END] = globaltimer_ns();
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_full = idesc_bf16(BM, BN, A_MN, B_MN);
            constexpr uint32_t idesc_half = idesc_bf16(BM, BN >= 128 ? BN / 2 : BN, A_MN, B_MN);
            constexpr uint32_t idesc_quarter = idesc_bf16(BM, BN >= 256 ? BN / 4 : BN, A_MN, B_MN);
            // Descriptor fields advance in 16-byte units: K step of 16 elements is +32 B
            // along a K-major row, +16 rows (2 swizzle atoms) in an MN-major tile.
            constexpr uint64_t a_kstep = (A_MN ? 2048u : 32u) >> 4;
            constexpr uint64_t b_kstep = (B_MN ? 2048u : 32u) >> 4;
            constexpr uint32_t a_lbo = A_MN ? 64u * 128u : 16u;
            constexpr uint32_t b_lbo = B_MN ? 64u * 128u : 16u;
            const uint64_t ad_base = sdesc_sw128(smem_u32(sA), a_lbo, 1024);
            const uint64_t bd_base = sdesc_sw128(smem_u32(sB), b_lbo, 1024);
            const int kb_last = p.kb0 + p.kb1 - 1;
            int stage = 0;
            uint32_t phase = 0;
            int it = 0;
            bool ok = true;
            WorkItem w;
            for (; ok && get_item<BN, EPI>(p, it, w); ++it) {
                const int buf = it & 1;
                const uint32_t aphase = (it >> 1) & 1;
                if (!wait_bounded(smem_u32(&tempty_bar[buf]), aphase ^ 1u, abort_flag, p.err,
                                  DERR_WAIT_TMEM_EMPTY)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * BN);
                const uint32_t idesc = w.nsplit == 1 ? idesc_full : (w.nsplit == 2 ? idesc_half : idesc_quarter);
                // Lean K loop: one try_wait on the fast path, constant-offset descriptors,
                // unrolled MMAs; the issue rate must keep pace with the tensor pipe.
                for (int kb = w.kb_lo; kb < w.kb_hi; ++kb) {
                    const uint32_t fb = smem_u32(&full_bar[stage]);
                    if (!mbar_try_wait(fb, phase) &&
                        !wait_bounded(fb, phase, abort_flag, p.err, DERR_WAIT_FULL)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t ad = ad_base + static_cast<uint64_t>((stage * Cfg::A_BYTES) >> 4);
                    const uint64_t bd = bd_base + static_cast<uint64_t>((stage * Cfg::B_BYTES) >> 4);
                    const uint32_t acc0 = kb > w.kb_lo ? 1u : 0u;
                    if (kb != kb_last || p.kb1 == 0) {
                        tc_mma_bf16(d_tmem, ad, bd, idesc, acc0);
                        tc_mma_bf16(d_tmem, ad + a_kstep, bd + b_kstep, idesc, 1u);
                        tc_mma_bf16(d_tmem, ad + 2 * a_kstep, bd + 2 * b_kstep, idesc, 1u);
                        tc_mma_bf16(d_tmem, ad + 3 * a_kstep, bd + 3 * b_kstep, idesc, 1u);
                    } else {
                        // last block of the rank-r segment: only ceil(r_tail / 16) MMAs
                        for (int kk = 0; kk < p.mma_last1; ++kk)
                            tc_mma_bf16(d_tmem, ad + kk * a_kstep, bd + kk * b_kstep, idesc, (acc0 | kk) ? 1u : 0u);
                    }
                    tc_commit(smem_u32(&empty_bar[stage]));
                    stage = stage + 1 == STAGES ? 0 : stage + 1;
                    phase = stage == 0 ? phase ^ 1u : phase;
                }
                if (!ok) break;
                tc_commit(smem_u32(&tfull_bar[buf]));
            }
            // Drain: all MMAs issued by this thread complete before TMEM is freed.
            tc_commit(smem_u32(drain_bar));
            volatile int never = 0;
            wait_bounded(smem_u32(drain_bar), 0, &never, p.err, DERR_WAIT_DRAIN);
            if (trace) {
                trace[TR_MMA_END] = globaltimer_ns();
                trace[TR_TILES] = static_cast<unsigned long long>(it);
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;                 // TMEM lane quarter of this warp
        const int row_local = q * 32 + lane;    // accumulator row of this thread
        const int epi_tid = threadIdx.x - 64;   // 0..127
        int it = 0;
        WorkItem w;
        for (; get_item<BN, EPI>(p, it, w); ++it) {
            const int buf = it & 1;
            const uint32_t aphase = (it >> 1) & 1;
            // One thread waits; the outcome is broadcast so all four warps take the
            // same path (the fixups below use named barriers).
            if (epi_tid == 0)
                epi_ok[it & 1] = wait_bounded(smem_u32(&tfull_bar[buf]), aphase, abort_flag, p.err,
                                              DERR_WAIT_TMEM_FULL) ? 1 : 0;
            named_bar_sync(1, 128);
            if (!epi_ok[it & 1]) break;
            tc_fence_after();
            const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                   static_cast<uint32_t>(buf * BN);
            if constexpr (EPI == EPI_STORE) {
                // TMEM -> bf16 -> swizzled smem -> TMA store, 64 columns at a time.
                uint8_t *stage_base = sEpi + (q * 2) * (32 * 128);
                const int nch = (BN / 64) / w.nsplit;
#pragma unroll 1
                for (int ch = 0; ch < nch; ++ch) {
                    uint32_t v0[32], v1[32];
                    tmem_ld_32x32b_x32(t_row + ch * 64, v0);
                    tmem_ld_32x32b_x32(t_row + ch * 64 + 32, v1);
                    tc_wait_ld();
                    if (ch == nch - 1) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(smem_u32(&tempty_bar[buf]));
                    }
                    uint8_t *sbuf = stage_base + (ch & 1) * (32 * 128);
                    // The TMA store that used this buffer two chunks ago must have read it.
                    if (lane == 0) bulk_wait_group_read<1>();
                    __syncwarp();
                    stage_row64(sbuf, lane, v0, v1);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(&p.tmC, smem_u32(sbuf), w.col0 + ch * 64, w.m * BM + q * 32);
                        bulk_commit_group();
                    }
                }
            } else {
                // fp32 partial of this K split -> workspace.
                const SkinnyJob &J = p.job[w.job];
                const int64_t rows_total = static_cast<int64_t>(J.m_tiles) * BM;
                const int64_t grow = static_cast<int64_t>(w.m) * BM + row_local;
                float *my_part = J.part + ((static_cast<int64_t>(w.piece) * rows_total + grow) * J.n_valid);
                for (int c0 = 0; c0 < J.n_valid; c0 += 8) {
                    uint32_t v[8];
                    tmem_ld_32x32b_x8(t_row + c0, v);
                    tc_wait_ld();
                    float4 *dst = reinterpret_cast<float4 *>(my_part + c0);
                    dst[0] = make_float4(__uint_as_float(v[0]), __uint_as_float(v[1]), __uint_as_float(v[2]),
                                         __uint_as_float(v[3]));
                    dst[1] = make_float4(__uint_as_float(v[4]), __uint_as_float(v[5]), __uint_as_float(v[6]),
                                         __uint_as_float(v[7]));
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&tempty_bar[buf]));
                __threadfence();
                named_bar_sync(1, 128);
                const int ctr = w.m;
                if (epi_tid == 0) *last_flag = (atomicAdd(&J.counters[ctr], 1) == J.splits - 1) ? 1 : 0;
                named_bar_sync(1, 128);
                const bool last = *last_flag != 0;
                named_bar_sync(1, 128);  // everyone has read last_flag before it is reused
                if (last) {
                    __threadfence();
                    if (grow < J.rows_valid) {
                        const float *prow = J.part + grow * J.n_valid;
                        const int64_t split_stride = rows_total * J.n_valid;
                        for (int c0 = 0; c0 < J.n_valid; c0 += 4) {
                            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
                            // Eight splits' loads in flight at a time, summed in split order.
                            for (int s0 = 0; s0 < J.splits; s0 += 8) {
                                float4 v[8];
#pragma unroll
                                for (int u = 0; u < 8; ++u)
                                    v[u] = (s0 + u < J.splits)
                                               ? __ldcg(reinterpret_cast<const float4 *>(
                                                     prow + (s0 + u) * split_stride + c0))
                                               : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                                for (int u = 0; u < 8; ++u) {
                                    if (s0 + u < J.splits) {
                                        acc.x += v[u].x;
                                        acc.y += v[u].y;
                                        acc.z += v[u].z;
                                        acc.w += v[u].w;
                                    }
                                }
                            }
                            acc.x *= J.out_scale;
                            acc.y *= J.out_scale;
                            acc.z *= J.out_scale;
                            acc.w *= J.out_scale;
                            if (J.out_mode == OUT_BF16_ROWS) {
                                __nv_bfloat162 a = __floats2bfloat162_rn(acc.x, acc.y);
                                __nv_bfloat162 b = __floats2bfloat162_rn(acc.z, acc.w);
                                uint2 u2 = make_uint2(*reinterpret_cast<uint32_t *>(&a), *reinterpret_cast<uint32_t *>(&b));
                                *reinterpret_cast<uint2 *>(static_cast<__nv_bfloat16 *>(J.out) + grow * J.n_valid + c0) = u2;
                            } else if (J.out_mode == OUT_F32_ROWS) {
                                *reinterpret_cast<float4 *>(static_cast<float *>(J.out) + grow * J.n_valid + c0) = acc;
                            } else {
                                float *o = static_cast<float *>(J.out);
                                o[(c0 + 0) * J.out_ld + grow] = acc.x;
                                o[(c0 + 1) * J.out_ld + grow] = acc.y;
                                o[(c0 + 2) * J.out_ld + grow] = acc.z;
                                o[(c0 + 3) * J.out_ld + grow] = acc.w;
                            }
                        }
                    }
                    if (epi_tid == 0) J.counters[ctr] = 0;  // ready for the next call
                }
            }
            if (trace && epi_tid == 0 && it < 8) trace[TR_TILE_DONE0 + it] = globaltimer_ns();
        }
        if (trace && epi_tid == 0) trace[TR_EPI_END] = globaltimer_ns();
        if constexpr (EPI == EPI_STORE) {
            if (lane == 0) bulk_wait_group<0>();
        }
    }

    // ---------------------------------------------------------------- teardown
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
    }
    if (p.defer_dep_wait) grid_dep_wait();
    if (trace && threadIdx.x == 0) {
        trace[TR_EXIT] = globaltimer_ns();
        trace[TR_CLK_EXIT] = clock64();
    }
}

}  // namespace lora
