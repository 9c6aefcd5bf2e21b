// tc_gemm2.cuh -- the main K-concatenated GEMMs on CTA pairs (tcgen05 cta_group::2).
//
// A cluster of two CTAs on two SMs computes one 256 x 256 output tile with
// 256 x N x 16 tcgen05 MMAs: each CTA stages its own 128 rows of A and its own half
// (128 rows of N) of B, so per K block a CTA loads 32 KB for the work a single-SM
// 128 x 256 tile would need 48 KB for, and six stages fit in shared memory.
//
//   warp 0      TMA producer in both CTAs (no multicast: each CTA loads its halves);
//               every copy of the pair completes on the leader CTA's full barrier
//   warp 1      TMEM allocation in both CTAs (collective); in the leader CTA the
//               single-thread tcgen05.mma.cta_group::2 issuer; its commits arrive on
//               both CTAs' barriers (stage free / accumulator ready)
//   warps 2..5  epilogue in both CTAs: each drains its own 128 accumulator rows from
//               TMEM, reports to the leader's accumulator-empty barrier, and stores
//               bf16 through 128B-swizzled smem staging with TMA
//   warps 6..   (4-bit or FP8 frozen weight) dequant warps in both CTAs, none on warp
//               1's scheduler: fetch the weight's codes by TMA, decode them to bf16
//               straight into the B tile of the weight K segment and report to the
//               leader's B-ready barrier; the producer then loads only A for those
//               blocks (and A + B for the rank-r tail blocks, as in the bf16 case)
//
// Schedule: whole pair tiles in grouped raster order, `dp_waves` per cluster; a
// partial last wave of `tail_tiles` tiles is cut along N into two 256 x 128 tiles,
// one per cluster, when they fit in one wave.  Every output element comes from one
// accumulator; no partial sums, deterministic.
//
// Programmatic dependent launch, bounded waits and the error word work as in
// tc_gemm.cuh.  A cluster barrier at set-up (barriers initialised, TMEM allocated in
// both CTAs) and at teardown (no CTA leaves while its partner may still signal it)
// brackets the work.
#pragma once

#include "tc_gemm.cuh"

namespace lora {

constexpr int PAIR_BM = 256;      // output rows per pair tile (128 per CTA)
constexpr int PAIR_BN = 256;      // output columns per pair tile
constexpr int CTA_BN = PAIR_BN / 2;  // B rows (N) staged per CTA
constexpr int DQ_WARPS = 12;         // coded weight: dequant warps per CTA (3 idle warps besides)
constexpr int DQ_QDEPTH = 1;         // packed-code slots per dequant warp (own K blocks in flight)

// Frozen-weight formats of the pair GEMM: bf16, the linear 4-bit code, FP8 E4M3, and a
// 4-bit code decoded through a 16-value codebook (e.g. NF4).
enum WeightFmt { WF_BF16 = 0, WF_Q4 = 1, WF_FP8 = 2, WF_CB = 3 };
// Bytes of codes per run of 64 weights: two 4-bit codes per byte, or one E4M3 code per byte.
__host__ __device__ constexpr int dq_run_bytes(int wf) { return wf == WF_FP8 ? 64 : 32; }
// Runs of 64 codes a thread decodes per K block: two for the 4-bit codes (the per-block
// fixed cost, the codebook table included, paid once per two runs); one for FP8, whose
// halved code slots leave room for a fifth pipeline stage.
__host__ __device__ constexpr int dq_runs(int wf) { return wf == WF_FP8 ? 1 : 2; }
__host__ __device__ constexpr int dq_group_warps(int wf) { return 4 / dq_runs(wf); }  // warps per 128-run B tile
__host__ __device__ constexpr int dq_groups(int wf) { return DQ_WARPS / dq_group_warps(wf); }  // take K blocks in turn
__host__ __device__ constexpr int dq_qrows(int wf) { return 32 * dq_runs(wf); }  // runs fetched per warp and K block
// One packed-code slot of a dequant warp: dq_qrows runs.
__host__ __device__ constexpr int dq_qslot(int wf) { return dq_qrows(wf) * dq_run_bytes(wf); }

// A warp's scheduler (SM sub-partition) is its id mod 4.  The single-thread MMA issuer
// (warp 1) must issue each tcgen05.mma as soon as the tensor core takes the previous one
// (its queue is about one MMA deep), so no dequant warp shares its sub-partition: warp
// ids >= 6 that are 1 mod 4 stay idle and the dequant warps take the others in order
// (measured on the 4-bit up projection: the main GEMMs 1.93 -> 1.72 ms).
__host__ __device__ constexpr bool dq_idle_warp(int w) { return w >= 6 && w % 4 == 1; }
// Warp ids from 6 on that host n dequant warps; dequant index of (non-idle) warp w.
__host__ __device__ constexpr int dq_warp_span(int n) {
    int w = 6, got = 0;
    while (got < n) got += dq_idle_warp(w++) ? 0 : 1;
    return w - 6;
}
__host__ __device__ constexpr int dq_index(int w) {
    int i = 0;
    for (int v = 6; v < w; ++v) i += dq_idle_warp(v) ? 0 : 1;
    return i;
}

template <bool B_MN, int WF, int STAGES>
struct PairCfg {
    static constexpr bool DQ = WF != WF_BF16;         // the weight's B tiles are decoded in shared memory
    static constexpr int A_BYTES = 128 * BK * 2;      // 16 KB: this CTA's 128 rows of A
    static constexpr int B_BYTES = CTA_BN * BK * 2;   // 16 KB: this CTA's 128 rows of B
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int Q_BYTES = DQ ? DQ_WARPS * DQ_QDEPTH * dq_qslot(WF) : 0;  // per-warp packed-code rings
    static constexpr int EPI_BUFS = 2;  // output staging per epilogue warp: 32 rows x 64 columns, double-buffered
    static constexpr int EPI_BYTES = 4 * EPI_BUFS * 32 * 128;
    static constexpr int TMEM_COLS = 2 * PAIR_BN;     // two 256-column accumulators
    static constexpr int BAR_BYTES = DQ ? 1024 : 512;
    static constexpr int THREADS = DQ ? NUM_THREADS + 32 * dq_warp_span(DQ_WARPS) : NUM_THREADS;  // + dequant warps
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + Q_BYTES + EPI_BYTES + BAR_BYTES;
    static_assert(STAGES <= 32, "per-stage phase bits are kept in one 32-bit mask");
    static_assert(SMEM_BYTES <= 232448, "at most 227 KB of shared memory per CTA");
};

// Two codes, each given as the fp32 bit pattern of 2^23 + q, to the bf16 pair
// ((q_even - 8) * s7, (q_odd - 8) * s7), even element in the low half.  The packed
// fp32 add is exact (it leaves q - 8), the packed multiply rounds once in fp32 and the
// conversion rounds once more to bf16.
__device__ __forceinline__ uint32_t q4_pair(uint32_t f_even, uint32_t f_odd, uint64_t s7x2) {
    constexpr uint64_t kMinus2p23p8x2 = 0xCB000008CB000008ull;  // -(2^23 + 8) in both fp32 halves
    uint32_t out;
    asm("{\n\t.reg .b64 v;\n\t.reg .b32 e, o;\n\t"
        "mov.b64 v, {%1, %2};\n\t"
        "add.rn.f32x2 v, v, %3;\n\t"
        "mul.rn.f32x2 v, v, %4;\n\t"
        "mov.b64 {e, o}, v;\n\t"
        "cvt.rn.bf16x2.f32 %0, o, e;\n\t}"
        : "=r"(out)
        : "r"(f_even), "r"(f_odd), "l"(kMinus2p23p8x2), "l"(s7x2));
    return out;
}

// Decode one 32-bit word of 4-bit codes (8 consecutive elements, element i in bits
// 4i..4i+3: low nibble of each byte = even index) into 8 bf16 values (q - 8) * s7.
// A byte permute places each nibble under the exponent of 2^23.
__device__ __forceinline__ uint4 q4_decode8(uint32_t word, uint64_t s7x2) {
    const uint32_t lo = word & 0x0F0F0F0Fu, hi = (word >> 4) & 0x0F0F0F0Fu;
    constexpr uint32_t kExp = 0x4B000000u;  // 2^23
    uint4 r;
    r.x = q4_pair(__byte_perm(lo, kExp, 0x7540), __byte_perm(hi, kExp, 0x7540), s7x2);
    r.y = q4_pair(__byte_perm(lo, kExp, 0x7541), __byte_perm(hi, kExp, 0x7541), s7x2);
    r.z = q4_pair(__byte_perm(lo, kExp, 0x7542), __byte_perm(hi, kExp, 0x7542), s7x2);
    r.w = q4_pair(__byte_perm(lo, kExp, 0x7543), __byte_perm(hi, kExp, 0x7543), s7x2);
    return r;
}

// Eight E4M3 codes (two 32-bit words, element i in byte i) to eight bf16 values
// e4m3(q) * scale, four codes at a time: each code pair converts exactly to f16x2, each
// half widens exactly to fp32, the packed fp32 product with the bf16 scale is exact
// (4 + 8 significant bits), and the conversion to bf16x2 is the one rounding (NaN codes
// stay NaN).  `scx2` is the fp32 scale in both halves.
__device__ __forceinline__ void fp8_quad(uint32_t w, uint64_t scx2, uint32_t &p01, uint32_t &p23) {
    asm("{\n\t.reg .b16 c0, c1, a0, a1, a2, a3;\n\t.reg .b32 h0, h1;\n\t.reg .f32 f0, f1, f2, f3;\n\t"
        ".reg .b64 v0, v1;\n\t"
        "mov.b32 {c0, c1}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 h0, c0;\n\t"
        "cvt.rn.f16x2.e4m3x2 h1, c1;\n\t"
        "mov.b32 {a0, a1}, h0;\n\t"
        "mov.b32 {a2, a3}, h1;\n\t"
        "cvt.f32.f16 f0, a0;\n\t"
        "cvt.f32.f16 f1, a1;\n\t"
        "cvt.f32.f16 f2, a2;\n\t"
        "cvt.f32.f16 f3, a3;\n\t"
        "mov.b64 v0, {f0, f1};\n\t"
        "mov.b64 v1, {f2, f3};\n\t"
        "mul.rn.f32x2 v0, v0, %3;\n\t"
        "mul.rn.f32x2 v1, v1, %3;\n\t"
        "mov.b64 {f0, f1}, v0;\n\t"
        "mov.b64 {f2, f3}, v1;\n\t"
        "cvt.rn.bf16x2.f32 %0, f1, f0;\n\t"
        "cvt.rn.bf16x2.f32 %1, f3, f2;\n\t}"
        : "=r"(p01), "=r"(p23)
        : "r"(w), "l"(scx2));
}
__device__ __forceinline__ uint4 fp8_decode8(uint32_t w0, uint32_t w1, uint64_t scx2) {
    uint4 r;
    fp8_quad(w0, scx2, r.x, r.y);
    fp8_quad(w1, scx2, r.z, r.w);
    return r;
}

// 4-bit codebook decode.  The 16 values of a run's table, codebook[i] * scale rounded
// once to bf16, are held as byte tables: lo[t] / hi[t] hold the low / high bytes of
// entries 4t .. 4t+3.  A prmt picks 4 bytes from 8 by 3-bit selectors, so entries 0-7
// and 8-15 are looked up separately and bit 3 of each code chooses between them.
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}
struct CbTable {
    uint32_t lo[4], hi[4];
};
__device__ __forceinline__ CbTable cb_table(const float (&cb)[16], float sc) {
    CbTable t;
#pragma unroll
    for (int q = 0; q < 4; ++q) {  // entries 4q .. 4q+3
        uint32_t w0, w1;           // bf16x2 (entry 4q+1 : 4q), (4q+3 : 4q+2)
        asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(w0) : "f"(cb[4 * q + 1] * sc), "f"(cb[4 * q] * sc));
        asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(w1) : "f"(cb[4 * q + 3] * sc), "f"(cb[4 * q + 2] * sc));
        t.lo[q] = prmt(w0, w1, 0x6420);
        t.hi[q] = prmt(w0, w1, 0x7531);
    }
    return t;
}
// Codes c0..c3 in the low nibbles of the bytes of v -> the low (L) and high (H) bytes of
// their four bf16 table values, byte i for code i.
__device__ __forceinline__ void cb_look4(const CbTable &t, uint32_t v, uint32_t &L, uint32_t &H) {
    const uint32_t x = v & 0x07070707u;
    const uint32_t sel = prmt(x | (x >> 4), 0u, 0x4420);  // nibble i = c_i & 7
    const uint32_t m = prmt(v << 4, 0u, 0xBA98);          // byte i = 0xFF where c_i >= 8
    const uint32_t l0 = prmt(t.lo[0], t.lo[1], sel), l1 = prmt(t.lo[2], t.lo[3], sel);
    const uint32_t h0 = prmt(t.hi[0], t.hi[1], sel), h1 = prmt(t.hi[2], t.hi[3], sel);
    L = (l0 & ~m) | (l1 & m);
    H = (h0 & ~m) | (h1 & m);
}
// One 32-bit word of 4-bit codes (element i in bits 4i..4i+3) to 8 bf16 table values.
__device__ __forceinline__ uint4 cb_decode8(const CbTable &t, uint32_t word) {
    uint32_t Le, He, Lo, Ho;
    cb_look4(t, word & 0x0F0F0F0Fu, Le, He);          // elements 0, 2, 4, 6
    cb_look4(t, (word >> 4) & 0x0F0F0F0Fu, Lo, Ho);   // elements 1, 3, 5, 7
    const uint32_t ev01 = prmt(Le, He, 0x5140), od01 = prmt(Lo, Ho, 0x5140);  // {e0, e2}, {e1, e3}
    const uint32_t ev23 = prmt(Le, He, 0x7362), od23 = prmt(Lo, Ho, 0x7362);  // {e4, e6}, {e5, e7}
    uint4 r;
    r.x = prmt(ev01, od01, 0x5410);
    r.y = prmt(ev01, od01, 0x7632);
    r.z = prmt(ev23, od23, 0x5410);
    r.w = prmt(ev23, od23, 0x7632);
    return r;
}

// Item i of this cluster: pair tile (m, n), its first output column and width split.
__device__ __forceinline__ bool get_pair_item(const GemmArgs &p, int cluster, int n_clusters, int i, WorkItem &w) {
    w.kb_lo = 0;
    w.kb_hi = p.kb0 + p.kb1;
    w.piece = 0;
    w.nsplit = 1;
    if (p.tail_ksplit) {
        // Last-wave tile tt cut along K into two halves, the FIRST items of clusters 2tt and
        // 2tt + 1: the first half hands its fp32 partial over, the second (with the rank-r
        // tail) adds it; both hand-overs overlap the clusters' later tiles, and every
        // cluster ends after its whole tiles (W + 1/2 tiles on clusters 0 .. 2R-1).
        const int tt = cluster >> 1;
        if (tt < p.tail_tiles) {
            if (i == 0) {
                const int kb_all = p.kb0 + p.kb1, kb_mid = kb_all / 2;
                raster(p, p.dp_tiles + tt, w.m, w.n);
                w.kb_lo = (cluster & 1) ? kb_mid : 0;
                w.kb_hi = (cluster & 1) ? kb_all : kb_mid;
                w.piece = 1 + (cluster & 1);
                w.job = tt;
                w.col0 = w.n * PAIR_BN;
                return true;
            }
            --i;
        }
        if (i < p.dp_waves) {
            const int t = cluster + i * n_clusters;
            if (t >= p.dp_tiles) return false;
            raster(p, t, w.m, w.n);
            w.col0 = w.n * PAIR_BN;
            return true;
        }
        return false;
    }
    if (i < p.dp_waves) {
        const int t = cluster + i * n_clusters;
        if (t >= p.dp_tiles) return false;
        raster(p, t, w.m, w.n);
        w.col0 = w.n * PAIR_BN;
        return true;
    }
    if (i == p.dp_waves && p.tail_split > 1 && cluster < p.tail_tiles * p.tail_split) {
        const int tt = cluster / p.tail_split, h = cluster % p.tail_split;
        raster(p, p.dp_tiles + tt, w.m, w.n);
        w.nsplit = p.tail_split;
        w.col0 = w.n * PAIR_BN + h * (PAIR_BN / p.tail_split);
        return true;
    }
    return false;
}

template <bool B_MN, int WF, int STAGES>
__global__ void __launch_bounds__(PairCfg<B_MN, WF, STAGES>::THREADS, 1)
    k_tc_gemm_pair(const __grid_constant__ GemmArgs p) {
    using Cfg = PairCfg<B_MN, WF, STAGES>;
    constexpr bool DQ = Cfg::DQ;  // the weight's B tiles are decoded (4-bit or FP8 codes)
    constexpr int QSLOT = dq_qslot(WF);
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem;
    uint8_t *sB = smem + STAGES * Cfg::A_BYTES;
    uint8_t *sQ = smem + STAGES * Cfg::STAGE_BYTES;  // decoded weight: packed-code rings of the dequant warps
    uint8_t *sEpi = sQ + Cfg::Q_BYTES;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sEpi + Cfg::EPI_BYTES);
    uint64_t *full_bar = bars;                    // [STAGES] (leader's counts the pair's A (and B) bytes)
    uint64_t *empty_bar = bars + STAGES;          // [STAGES]
    uint64_t *tfull_bar = bars + 2 * STAGES;      // [2]
    uint64_t *tempty_bar = bars + 2 * STAGES + 2; // [2] (leader's: 8 epilogue warps of the pair)
    uint64_t *drain_bar = bars + 2 * STAGES + 4;  // [1]
    uint64_t *bready_bar = bars + 2 * STAGES + 5; // [STAGES] DQ, leader: both CTAs' decoded B tiles written
    uint64_t *qfull_bar = bars + 3 * STAGES + 5;  // [DQ_WARPS][DQ_QDEPTH] Q4: a warp's packed codes landed
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(qfull_bar + (DQ ? DQ_WARPS * DQ_QDEPTH : 0));
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    volatile int *epi_ok = reinterpret_cast<volatile int *>(tmem_slot + 3);  // [2]
    // decoded weight: K blocks (in the CTA's sequence) whose stage the producer has seen released by
    // the MMA, i.e. whose B tile the dequant warps may write.  A monotonic count: the
    // dequant groups run ahead of the MMA by different amounts, so a parity wait on the
    // stage's empty barrier could match a later phase than the one meant.
    uint32_t *bfree = tmem_slot + 5;
    volatile int *ks_ok = reinterpret_cast<volatile int *>(tmem_slot + 6);  // K-split tail: the partial is there

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int cluster = blockIdx.x >> 1;
    const int n_clusters = gridDim.x >> 1;
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
            mbar_init(smem_u32(&tempty_bar[b]), 8);
        }
        mbar_init(smem_u32(drain_bar), 1);
        if (DQ) {
            for (int s = 0; s < STAGES; ++s) mbar_init(smem_u32(&bready_bar[s]), 2 * dq_group_warps(WF));
            for (int q = 0; q < DQ_WARPS * DQ_QDEPTH; ++q) mbar_init(smem_u32(&qfull_bar[q]), 1);
        }
        *abort_flag = 0;
        *bfree = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        if (DQ) tma_prefetch_desc(&p.tmQ);
        tma_prefetch_desc(&p.tmA0);
        tma_prefetch_desc(&p.tmB0);
        if (p.kb1 > 0) {
            tma_prefetch_desc(&p.tmA1);
            tma_prefetch_desc(&p.tmB1);
        }
        tma_prefetch_desc(&p.tmC);
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_u32(tmem_slot), Cfg::TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // both CTAs' barriers initialised and TMEM allocated
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    grid_dep_wait();
    grid_dep_launch_dependents();
    if (trace && threadIdx.x == 0) {
        trace[TR_SETUP] = globaltimer_ns();
        trace[TR_CLK_SETUP] = clock64();
    }

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer (both CTAs)
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued_mask = 0, issued_phase = 0;  // leader's full barriers
            bool ok = true;
            uint64_t wait_empty_ns = 0;
            uint32_t flat = 0;  // K blocks of the CTA's sequence handled so far
            WorkItem w;
            for (int i = 0; ok && get_pair_item(p, cluster, n_clusters, i, w); ++i) {
                const int bn_cta = (PAIR_BN / w.nsplit) / 2;  // B rows this CTA stages
                const int a_row = w.m * PAIR_BM + static_cast<int>(rank) * 128;
                const int b_row = w.col0 + static_cast<int>(rank) * bn_cta;
                for (int kb = w.kb_lo; kb < w.kb_hi; ++kb) {
                    // decoded weight: the weight segment's B tiles are written by the dequant warps, so the
                    // leader's full barrier then counts A only; rank-r tail B tiles come by TMA.
                    const bool seg1 = kb >= p.kb0;
                    const bool b_tma = !DQ || seg1;
                    const uint32_t tx = 2u * static_cast<uint32_t>(Cfg::A_BYTES + (b_tma ? bn_cta * BK * 2 : 0));
                    const uint64_t tw = trace ? globaltimer_ns() : 0;
                    if (!wait_bounded(smem_u32(&empty_bar[stage]), phase ^ 1u, abort_flag, p.err,
                                      DERR_WAIT_EMPTY)) {
                        ok = false;
                        break;
                    }
                    if (trace) wait_empty_ns += globaltimer_ns() - tw;
                    if (DQ) st_release_shared(smem_u32(bfree), ++flat);
                    const uint32_t fb_local = smem_u32(&full_bar[stage]);
                    const uint32_t fb_leader = mapa_shared(fb_local, 0);
                    if (leader) {
                        mbar_arrive_expect_tx(fb_local, tx);
                        issued_mask |= 1u << stage;
                        issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
                    }
                    const int k0 = (seg1 ? kb - p.kb0 : kb) * BK;
                    const uint32_t a_dst = smem_u32(sA + stage * Cfg::A_BYTES);
                    const uint32_t b_dst = smem_u32(sB + stage * Cfg::B_BYTES);
                    tma_load_2d_pair(a_dst, seg1 ? &p.tmA1 : &p.tmA0, fb_leader, k0, a_row);
                    if (!b_tma) {
                    } else if (B_MN) {
                        // the weight's 128 columns in one 3D copy (two 64-column chunks), else
                        // one 2D copy per 64-column chunk (with the 3D map in tmB0, the
                        // weight's 2D map is tmB0n: a 2D copy must name a 2D map)
                        if (p.b3d && !seg1 && bn_cta == 128) {
                            tma_load_3d_pair(b_dst, &p.tmB0, fb_leader, 0, k0, b_row / 64);
                        } else {
                            const CUtensorMap *tb = seg1 ? &p.tmB1 : p.b3d ? &p.tmB0n : &p.tmB0;
                            for (int j = 0; j < bn_cta / 64; ++j)
                                tma_load_2d_pair(b_dst + j * 64 * 128, tb, fb_leader, b_row + 64 * j, k0);
                        }
                    } else {
                        const CUtensorMap *tb = w.nsplit == 1 ? (seg1 ? &p.tmB1 : &p.tmB0)
                                                              : (seg1 ? &p.tmB1n : &p.tmB0n);
                        tma_load_2d_pair(b_dst, tb, fb_leader, k0, b_row);
                    }
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // Drain (leader): every copy of the pair has landed before either CTA leaves
            // (the teardown cluster barrier orders the partner's exit after this).
            if (leader)
                for (int s = 0; s < STAGES; ++s)
                    if (issued_mask & (1u << s)) {
                        volatile int never = 0;
                        wait_bounded(smem_u32(&full_bar[s]), (issued_phase >> s) & 1u, &never, p.err,
                                     DERR_WAIT_DRAIN);
                    }
            if (trace) {
                trace[TR_PROD_END] = globaltimer_ns();
                trace[TR_WAIT_EMPTY] = wait_empty_ns;
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (leader)
        if (lane == 0 && leader) {
            constexpr uint32_t idesc_full = idesc_bf16(PAIR_BM, PAIR_BN, false, B_MN);
            constexpr uint32_t idesc_half = idesc_bf16(PAIR_BM, PAIR_BN / 2, false, B_MN);
            // Descriptor fields advance in 16-byte units: K step of 16 elements is +32 B
            // along a K-major row, +16 rows (2 swizzle atoms) in an MN-major tile.
            constexpr uint64_t a_kstep = 32u >> 4;
            constexpr uint64_t b_kstep = (B_MN ? 2048u : 32u) >> 4;
            constexpr uint32_t b_lbo = B_MN ? 64u * 128u : 16u;
            const uint64_t ad_base = sdesc_sw128(smem_u32(sA), 16u, 1024);
            const uint64_t bd_base = sdesc_sw128(smem_u32(sB), b_lbo, 1024);
            const int kb_last = p.kb0 + p.kb1 - 1;
            int stage = 0;
            uint32_t phase = 0;
            int it = 0;
            bool ok = true;
            uint64_t wait_tempty_ns = 0, kblocks = 0;
            long long wait_a_cyc = 0, wait_b_cyc = 0;
            uint32_t bready_phase = 0;  // decoded weight: bit s = parity of the next B-ready completion of stage s
            WorkItem w;
            for (; ok && get_pair_item(p, cluster, n_clusters, it, w); ++it) {
                const int buf = it & 1;
                const uint32_t aphase = (it >> 1) & 1;
                const uint64_t tt = trace ? globaltimer_ns() : 0;
                if (!wait_bounded(smem_u32(&tempty_bar[buf]), aphase ^ 1u, abort_flag, p.err, DERR_WAIT_TMEM_EMPTY)) {
                    ok = false;
                    break;
                }
                if (trace) wait_tempty_ns += globaltimer_ns() - tt;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * PAIR_BN);
                const uint32_t idesc = w.nsplit == 1 ? idesc_full : idesc_half;
                // Lean K loop: one try_wait on the fast path, constant-offset descriptors,
                // unrolled MMAs; the issue rate must keep pace with the tensor pipe.
                for (int kb = w.kb_lo; kb < w.kb_hi; ++kb) {
                    const uint32_t fb = smem_u32(&full_bar[stage]);
                    if (!mbar_try_wait(fb, phase)) {
                        const long long c0 = trace ? clock64() : 0;
                        if (!wait_bounded(fb, phase, abort_flag, p.err, DERR_WAIT_FULL)) {
                            ok = false;
                            break;
                        }
                        if (trace) wait_a_cyc += clock64() - c0;
                    }
                    if (DQ && kb < p.kb0) {
                        // B-ready completes only for weight K blocks (rank-r tail blocks come
                        // by TMA), so its phase per stage is tracked apart from the ring's.
                        const uint32_t rb = smem_u32(&bready_bar[stage]);
                        const uint32_t bp = (bready_phase >> stage) & 1u;
                        bready_phase ^= 1u << stage;
                        if (!mbar_try_wait(rb, bp)) {
                            const long long c0 = trace ? clock64() : 0;
                            if (!wait_bounded(rb, bp, abort_flag, p.err, DERR_WAIT_FULL)) {
                                ok = false;
                                break;
                            }
                            if (trace) wait_b_cyc += clock64() - c0;
                        }
                    }
                    tc_fence_after();
                    const uint64_t ad = ad_base + static_cast<uint64_t>((stage * Cfg::A_BYTES) >> 4);
                    const uint64_t bd = bd_base + static_cast<uint64_t>((stage * Cfg::B_BYTES) >> 4);
                    const uint32_t acc0 = kb > w.kb_lo ? 1u : 0u;
                    if (kb != kb_last || p.kb1 == 0) {
                        tc_mma_bf16_pair(d_tmem, ad, bd, idesc, acc0);
                        tc_mma_bf16_pair(d_tmem, ad + a_kstep, bd + b_kstep, idesc, 1u);
                        tc_mma_bf16_pair(d_tmem, ad + 2 * a_kstep, bd + 2 * b_kstep, idesc, 1u);
                        tc_mma_bf16_pair(d_tmem, ad + 3 * a_kstep, bd + 3 * b_kstep, idesc, 1u);
                    } else {
                        // last block of the rank-r segment: only ceil(r_tail / 16) MMAs
                        for (int kk = 0; kk < p.mma_last1; ++kk)
                            tc_mma_bf16_pair(d_tmem, ad + kk * a_kstep, bd + kk * b_kstep, idesc,
                                             (acc0 | kk) ? 1u : 0u);
                    }
                    tc_commit_pair_mc(smem_u32(&empty_bar[stage]), 0x3);
                    stage = stage + 1 == STAGES ? 0 : stage + 1;
                    phase = stage == 0 ? phase ^ 1u : phase;
                }
                if (!ok) break;
                kblocks += static_cast<uint64_t>(w.kb_hi - w.kb_lo);
                tc_commit_pair_mc(smem_u32(&tfull_bar[buf]), 0x3);
            }
            tc_commit_pair_mc(smem_u32(drain_bar), 0x1);
            volatile int never = 0;
            wait_bounded(smem_u32(drain_bar), 0, &never, p.err, DERR_WAIT_DRAIN);
            if (trace) {
                trace[TR_MMA_END] = globaltimer_ns();
                trace[TR_TILES] = static_cast<unsigned long long>(it);
                trace[TR_WAIT_TEMPTY] = wait_tempty_ns;
                trace[TR_KBLOCKS] = kblocks;
                trace[TR_MMA_WAIT_A] = static_cast<unsigned long long>(wait_a_cyc);
                trace[TR_MMA_WAIT_B] = static_cast<unsigned long long>(wait_b_cyc);
            }
        }
    } else if (DQ && warp >= 6 && dq_idle_warp(warp)) {
        // idle: keeps the MMA issuer's sub-partition free of decode work
    } else if (DQ && warp >= 6) {
        // ------------------------------------------------------------ dequant warps (both CTAs, 4-bit or FP8 weight)
        // The weight segment's B tiles are decoded here from 4-bit codes.  Warps form
        // DQ_GROUPS groups of DQ_GROUP_WARPS; group g takes the weight K blocks g,
        // g + DQ_GROUPS, ... of the CTA's sequence (the rank-r tail blocks come by TMA and
        // are not touched).  A thread owns DQ_RUNS 32-byte runs of codes (64 elements
        // each): K-major, weight row rn of the tile; MN-major, K row rn of 64-column chunk
        // jc.  Each warp fetches its own DQ_QROWS runs by TMA into a private DQ_QDEPTH-slot
        // ring, DQ_QDEPTH own blocks ahead, so code loads never wait for a stage.  Per
        // block: wait for the codes, wait until the MMA has released the stage's B tile,
        // decode straight into the 128B-swizzled layout the MMA reads, fence to the async
        // proxy, and arrive (one arrival per warp) on the leader's B-ready barrier.  The
        // per-block cost outside the decode (waits, scale fetch, addressing, the
        // cluster-scope release) is paid once per DQ_RUNS runs, and one block takes a
        // group microseconds end to end, so DQ_GROUPS blocks are in flight at once.
        constexpr int DQ_RUNS = dq_runs(WF), DQ_GROUP_WARPS = dq_group_warps(WF), DQ_GROUPS = dq_groups(WF),
                      DQ_QROWS = dq_qrows(WF);
        static_assert(DQ_RUNS == 1 || DQ_RUNS == 2, "a warp's runs stay inside one 64-run chunk");
        const int dw = dq_index(warp);                       // dequant warp 0 .. DQ_WARPS-1
        const int grp = dw / DQ_GROUP_WARPS, wg = dw % DQ_GROUP_WARPS;
        const int r0 = wg * DQ_QROWS;                  // the warp's first run; lane owns r0 + lane + 32 i
        uint8_t *qring = sQ + dw * (DQ_QDEPTH * QSLOT);
        uint64_t *qbar = qfull_bar + dw * DQ_QDEPTH;
        const uint32_t bready_leader0 = mapa_shared(smem_u32(&bready_bar[0]), 0);
        const int kb_all = p.kb0 + p.kb1;
        // Own block j is weight K block kb of work item `item`, with flat weight index
        // grp + j * DQ_GROUPS.  Cursors step from one own block to the next without
        // divisions; the item's geometry is recomputed only when a cursor enters a new item.
        struct Cursor {
            int j, item, kb, b_row;
            bool valid;
        };
        auto enter_item = [&](Cursor &c) {
            WorkItem wi;
            c.valid = get_pair_item(p, cluster, n_clusters, c.item, wi);
            c.b_row = c.valid ? wi.col0 + static_cast<int>(rank) * ((PAIR_BN / wi.nsplit) / 2) : 0;
        };
        auto seek = [&](Cursor &c, int j) {
            const int wit = grp + j * DQ_GROUPS;
            c.j = j;
            c.item = wit / p.kb0;
            c.kb = wit - c.item * p.kb0;
            enter_item(c);
        };
        auto step = [&](Cursor &c) {
            ++c.j;
            c.kb += DQ_GROUPS;
            if (c.kb >= p.kb0) {
                const int adv = c.kb / p.kb0;
                c.kb -= adv * p.kb0;
                c.item += adv;
                enter_item(c);
            }
        };
        // Lane 0: TMA of this warp's DQ_QROWS runs of own block c.j into slot c.j % DQ_QDEPTH.
        auto issue = [&](const Cursor &c) {
            const uint32_t bar = smem_u32(&qbar[c.j % DQ_QDEPTH]);
            const uint32_t dst = smem_u32(qring + (c.j % DQ_QDEPTH) * QSLOT);
            mbar_arrive_expect_tx(bar, static_cast<uint32_t>(QSLOT));
            constexpr int RB = dq_run_bytes(WF);  // bytes of codes per 64 weights
            if (B_MN)  // K rows kb*64 + (r0 % 64) .., bytes of d_in columns b_row + 64*(r0 / 64) ..
                tma_load_2d(dst, &p.tmQ, bar, (c.b_row + 64 * (r0 >> 6)) * RB / 64, c.kb * BK + (r0 & 63));
            else       // weight rows b_row + r0 .., bytes of K columns kb*64 ..
                tma_load_2d(dst, &p.tmQ, bar, c.kb * RB, c.b_row + r0);
        };
        // Raw bf16 bits of the group scale of this thread's run i in own block c.j (0
        // outside the weight).  K-major: weight row rn; MN-major: K row rn, chunk jc.
        auto scale_bits = [&](const Cursor &c, int i) -> uint32_t {
            const int run = r0 + lane + 32 * i;
            const int rn = B_MN ? (run & 63) : run, jc = B_MN ? (run >> 6) : 0;
            if (!c.valid) return 0u;
            const int srow = B_MN ? c.kb * BK + rn : c.b_row + rn;
            // 4-bit: one scale per 64 weights of a row; FP8: one per row
            const int scol = WF == WF_FP8 ? 0 : B_MN ? (c.b_row + 64 * jc) / 64 : c.kb;
            if (srow >= p.scale_rows || scol >= p.scale_ld) return 0u;
            return static_cast<uint32_t>(__ldg(p.wscale + static_cast<int64_t>(srow) * p.scale_ld + scol));
        };
        const bool tr_dq = trace != nullptr && dw == 0 && lane == 0;
        long long dq_wait = 0, dq_decode = 0, dq_slot = 0, dq_publish = 0, dq_issue = 0;
        Cursor cur, ahead;  // own block being decoded; the next one whose codes to fetch
        seek(cur, 0);
        seek(ahead, 0);
        int issued = 0;  // own blocks whose codes were requested
        while (issued < DQ_QDEPTH && ahead.valid) {
            if (lane == 0) issue(ahead);
            ++issued;
            step(ahead);
        }
        uint32_t sc[DQ_RUNS];  // fetched one own block ahead (at the end of the previous one)
#pragma unroll
        for (int i = 0; i < DQ_RUNS; ++i) sc[i] = scale_bits(cur, i);
        while (cur.valid) {
            const int j = cur.j;
            const int flat = cur.item * kb_all + cur.kb;
            const int stage = flat % STAGES;
            const int slot = j % DQ_QDEPTH;
            const long long c0 = tr_dq ? clock64() : 0;
            if (!__all_sync(0xffffffffu, wait_bounded(smem_u32(&qbar[slot]), static_cast<uint32_t>(j / DQ_QDEPTH) & 1u,
                                                      abort_flag, p.err, DERR_WAIT_FULL)))
                break;
            const long long c1 = tr_dq ? clock64() : 0;
            const long long c2 = tr_dq ? clock64() : 0;
            // The stage's B tile is free once the producer has seen the MMA release it.
            // Lane 0 polls; the warp barrier passes its acquire on to the other lanes.
            bool granted = true;
            if (lane == 0)
                granted = wait_count_bounded(smem_u32(bfree), static_cast<uint32_t>(flat) + 1u, abort_flag, p.err,
                                             DERR_WAIT_EMPTY);
            __syncwarp();
            if (!__shfl_sync(0xffffffffu, granted, 0)) break;
            const long long c3 = tr_dq ? clock64() : 0;
#pragma unroll
            for (int i = 0; i < DQ_RUNS; ++i) {
                const int run = r0 + lane + 32 * i;
                const int rn = B_MN ? (run & 63) : run, jc = B_MN ? (run >> 6) : 0;
                // the slot holds the runs in rows of RB bytes, swizzled by the TMA: chunk t
                // of row lr sits at t ^ ((lr >> 1) & 3) (64-byte rows) or t ^ ((lr >> 2) & 1)
                // (32-byte rows), the slot being 1024-byte-aligned
                const int lr = lane + 32 * i;
                const uint4 *src = reinterpret_cast<const uint4 *>(qring + slot * QSLOT + lr * dq_run_bytes(WF));
                const int sw = dq_run_bytes(WF) == 64 ? ((lr >> 1) & 3) : ((lr >> 2) & 1);
                uint8_t *row =
                    sB + stage * Cfg::B_BYTES + (B_MN ? jc * 64 * 128 : 0) + (rn >> 3) * 1024 + (rn & 7) * 128;
                if constexpr (WF == WF_FP8) {
                    // 64 codes: 16-byte chunk c of the bf16 row holds codes 8c .. 8c+7
                    const uint64_t scx2 = (static_cast<uint64_t>(sc[i] << 16) << 32) | (sc[i] << 16);
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        const uint4 v = src[h ^ sw];
                        *reinterpret_cast<uint4 *>(row + (((2 * h) ^ (rn & 7)) * 16)) = fp8_decode8(v.x, v.y, scx2);
                        *reinterpret_cast<uint4 *>(row + (((2 * h + 1) ^ (rn & 7)) * 16)) = fp8_decode8(v.z, v.w, scx2);
                    }
                } else if constexpr (WF == WF_CB) {
                    const CbTable tb = cb_table(p.cb, __uint_as_float(sc[i] << 16));
                    const uint4 v0 = src[sw], v1 = src[1 ^ sw];
                    const uint32_t wds[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        *reinterpret_cast<uint4 *>(row + ((c ^ (rn & 7)) * 16)) = cb_decode8(tb, wds[c]);
                } else {
                    const uint4 v0 = src[sw], v1 = src[1 ^ sw];
                    const float s7 = __uint_as_float(sc[i] << 16) / 7.0f;
                    const uint64_t s7x2 = (static_cast<uint64_t>(__float_as_uint(s7)) << 32) | __float_as_uint(s7);
                    const uint32_t wds[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        *reinterpret_cast<uint4 *>(row + ((c ^ (rn & 7)) * 16)) = q4_decode8(wds[c], s7x2);
                }
            }
            // Orders the B-tile stores (and this slot's code reads, whose values are used
            // above) before the tensor core's reads and the slot's next TMA write.
            fence_proxy_async_smem();
            __syncwarp();
            long long c4 = 0;
            if (lane == 0) {
                mbar_arrive_cluster(bready_leader0 + static_cast<uint32_t>(stage * 8));
                if (tr_dq) c4 = clock64();
            }
            if (ahead.valid) {  // the slot just read is free: fetch own block j + DQ_QDEPTH
                if (lane == 0) issue(ahead);
                ++issued;
                step(ahead);
            }
            step(cur);
#pragma unroll
            for (int i = 0; i < DQ_RUNS; ++i) sc[i] = scale_bits(cur, i);
            if (tr_dq) {
                const long long c5 = clock64();
                dq_wait += c1 - c0;
                dq_decode += c2 - c1;
                dq_slot += c3 - c2;
                dq_publish += c4 - c3;
                dq_issue += c5 - c4;
            }
        }
        const int j = cur.j;
        // Copies still in flight (only after a failed wait): let them land before exit.
        if (lane == 0)
            for (int jj = j; jj < issued; ++jj) {
                volatile int never = 0;
                wait_bounded(smem_u32(&qbar[jj % DQ_QDEPTH]), static_cast<uint32_t>(jj / DQ_QDEPTH) & 1u, &never,
                             p.err, DERR_WAIT_DRAIN);
            }
        if (tr_dq) {
            trace[TR_DQ_WAIT] = static_cast<unsigned long long>(dq_wait);
            trace[TR_DQ_DECODE] = static_cast<unsigned long long>(dq_decode);
            trace[TR_DQ_SLOT] = static_cast<unsigned long long>(dq_slot);
            trace[TR_DQ_PUBLISH] = static_cast<unsigned long long>(dq_publish);
            trace[TR_DQ_ISSUE] = static_cast<unsigned long long>(dq_issue);
        }
    } else {
        // ------------------------------------------------------------ epilogue (both CTAs)
        const int q = warp & 3;
        const int epi_tid = threadIdx.x - 64;
        const uint32_t tempty_leader0 = mapa_shared(smem_u32(&tempty_bar[0]), 0);
        const uint32_t tempty_leader1 = mapa_shared(smem_u32(&tempty_bar[1]), 0);
        int it = 0;
        WorkItem w;
        for (; get_pair_item(p, cluster, n_clusters, it, w); ++it) {
            const int buf = it & 1;
            const uint32_t aphase = (it >> 1) & 1;
            if (epi_tid == 0)
                epi_ok[it & 1] = wait_bounded(smem_u32(&tfull_bar[buf]), aphase, abort_flag, p.err,
                                              DERR_WAIT_TMEM_FULL) ? 1 : 0;
            named_bar_sync(1, 128);
            if (!epi_ok[it & 1]) break;
            tc_fence_after();
            if (!DQ && w.piece > 0) {
                // Last-wave tile cut along K (both halves are their clusters' first items; the
                // MMAs of the next tile run in the other TMEM accumulator meanwhile).  The first
                // half (piece 1) hands this CTA's 128 rows of its fp32 accumulator to the
                // workspace from registers and raises its flag; the second (piece 2) reads them,
                // adds them to its own accumulator and stores the tile.  Hand-over layout,
                // 128 KB per CTA: float4 [chunk (4)][16-byte column group (16)][row (128)], so a
                // warp's accesses are 512 contiguous bytes.
                constexpr uint32_t KS_BYTES = 4 * 16 * 128 * 16;
                const int slot = w.job * 2 + static_cast<int>(rank);
                float4 *part = reinterpret_cast<float4 *>(p.ks_part) + static_cast<size_t>(slot) * (KS_BYTES / 16);
                const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                       static_cast<uint32_t>(buf * PAIR_BN);
                if (w.piece == 1) {
#pragma unroll 1
                    for (int ch = 0; ch < 4; ++ch) {
                        uint32_t v0[32], v1[32];
                        tmem_ld_32x32b_x32(t_row + ch * 64, v0);
                        tmem_ld_32x32b_x32(t_row + ch * 64 + 32, v1);
                        tc_wait_ld();
                        if (ch == 3) {
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0) mbar_arrive_cluster(buf ? tempty_leader1 : tempty_leader0);
                        }
#pragma unroll
                        for (int g = 0; g < 16; ++g) {
                            const uint32_t *src = g < 8 ? &v0[4 * g] : &v1[4 * (g - 8)];
                            __stcg(part + (ch * 16 + g) * 128 + q * 32 + lane,
                                   make_float4(__uint_as_float(src[0]), __uint_as_float(src[1]),
                                               __uint_as_float(src[2]), __uint_as_float(src[3])));
                        }
                    }
                    __threadfence();
                    named_bar_sync(1, 128);
                    if (epi_tid == 0) st_release_gpu(p.ks_flag + slot, 1);
                    if (trace && epi_tid == 0 && it < 8) trace[TR_TILE_DONE0 + it] = globaltimer_ns();
                    continue;
                }
                // piece 2: the first half's partial, once its flag is up (both halves are their
                // clusters' first items, so this wait overlaps this cluster's next tile; bounded).
                // Its own flag slot: the epilogue's epi_ok slots are reused by the next items.
                if (epi_tid == 0) {
                    const bool ok = wait_flag_bounded(p.ks_flag + slot, abort_flag, p.err, DERR_WAIT_PARTIAL);
                    if (ok) p.ks_flag[slot] = 0;  // zero again for the next call
                    *ks_ok = ok ? 1 : 0;
                }
                named_bar_sync(1, 128);
                if (!*ks_ok) break;
                uint8_t *stage_base = sEpi + (q * Cfg::EPI_BUFS) * (32 * 128);
                const int out_row = w.m * PAIR_BM + static_cast<int>(rank) * 128 + q * 32;
#pragma unroll 1
                for (int ch = 0; ch < 4; ++ch) {
                    uint8_t *sbuf = stage_base + (ch % Cfg::EPI_BUFS) * (32 * 128);
                    float4 o[16];
#pragma unroll
                    for (int g = 0; g < 16; ++g) o[g] = __ldcg(part + (ch * 16 + g) * 128 + q * 32 + lane);
                    uint32_t v0[32], v1[32];
                    tmem_ld_32x32b_x32(t_row + ch * 64, v0);
                    tmem_ld_32x32b_x32(t_row + ch * 64 + 32, v1);
                    tc_wait_ld();
                    if (ch == 3) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive_cluster(buf ? tempty_leader1 : tempty_leader0);
                    }
                    // own accumulator + the first half's (two terms: the order does not change the sum)
#pragma unroll
                    for (int g = 0; g < 16; ++g) {
                        uint32_t *dst = g < 8 ? &v0[4 * g] : &v1[4 * (g - 8)];
                        dst[0] = __float_as_uint(__uint_as_float(dst[0]) + o[g].x);
                        dst[1] = __float_as_uint(__uint_as_float(dst[1]) + o[g].y);
                        dst[2] = __float_as_uint(__uint_as_float(dst[2]) + o[g].z);
                        dst[3] = __float_as_uint(__uint_as_float(dst[3]) + o[g].w);
                    }
                    if (lane == 0) bulk_wait_group_read<Cfg::EPI_BUFS - 1>();
                    __syncwarp();
                    stage_row64(sbuf, lane, v0, v1);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(&p.tmC, smem_u32(sbuf), w.col0 + ch * 64, out_row);
                        bulk_commit_group();
                    }
                }
                if (trace && epi_tid == 0 && it < 8) trace[TR_TILE_DONE0 + it] = globaltimer_ns();
                continue;
            }
            const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                   static_cast<uint32_t>(buf * PAIR_BN);
            uint8_t *stage_base = sEpi + (q * Cfg::EPI_BUFS) * (32 * 128);
            const int nch = (PAIR_BN / 64) / w.nsplit;
            const int out_row = w.m * PAIR_BM + static_cast<int>(rank) * 128 + q * 32;
#pragma unroll 1
            for (int ch = 0; ch < nch; ++ch) {
                uint8_t *sbuf = stage_base + (ch % Cfg::EPI_BUFS) * (32 * 128);
                if (DQ) {
                    // 32 columns at a time: the dequant warps leave fewer registers per thread
                    if (lane == 0) bulk_wait_group_read<Cfg::EPI_BUFS - 1>();
                    __syncwarp();
#pragma unroll 1
                    for (int half = 0; half < 2; ++half) {
                        uint32_t v[32];
                        tmem_ld_32x32b_x32(t_row + ch * 64 + 32 * half, v);
                        tc_wait_ld();
                        if (half == 1 && ch == nch - 1) {
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0) mbar_arrive_cluster(buf ? tempty_leader1 : tempty_leader0);
                        }
                        stage_row32(sbuf, lane, half, v);
                    }
                } else {
                    uint32_t v0[32], v1[32];
                    tmem_ld_32x32b_x32(t_row + ch * 64, v0);
                    tmem_ld_32x32b_x32(t_row + ch * 64 + 32, v1);
                    tc_wait_ld();
                    if (ch == nch - 1) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive_cluster(buf ? tempty_leader1 : tempty_leader0);
                    }
                    if (lane == 0) bulk_wait_group_read<Cfg::EPI_BUFS - 1>();
                    __syncwarp();
                    stage_row64(sbuf, lane, v0, v1);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_2d(&p.tmC, smem_u32(sbuf), w.col0 + ch * 64, out_row);
                    bulk_commit_group();
                }
            }
            if (trace && epi_tid == 0 && it < 8) trace[TR_TILE_DONE0 + it] = globaltimer_ns();
        }
        if (trace && epi_tid == 0) trace[TR_EPI_END] = globaltimer_ns();
        if (lane == 0) bulk_wait_group<0>();
    }

    // ---------------------------------------------------------------- teardown
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // neither CTA leaves while its partner may still signal or read it
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, Cfg::TMEM_COLS);
    }
    if (trace && threadIdx.x == 0) {
        trace[TR_EXIT] = globaltimer_ns();
        trace[TR_CLK_EXIT] = clock64();
    }
}

}  // namespace lora
