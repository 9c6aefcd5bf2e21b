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

template <bool B_MN, bool Q4, int STAGES>
struct PairCfg {
    static constexpr int A_BYTES = 128 * BK * 2;      // 16 KB: this CTA's 128 rows of A
    static constexpr int B_BYTES = CTA_BN * BK * 2;   // 16 KB: this CTA's 128 rows of B
    static constexpr int Q_BYTES = Q4 ? CTA_BN * BK / 2 : 0;  // 4 KB of packed 4-bit codes
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + Q_BYTES;
    static constexpr int EPI_BYTES = 4 * 2 * 32 * 128;
    static constexpr int TMEM_COLS = 2 * PAIR_BN;     // two 256-column accumulators
    static constexpr int BAR_BYTES = 512;
    static constexpr int THREADS = Q4 ? NUM_THREADS + 128 : NUM_THREADS;  // + dequant warpgroup
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + EPI_BYTES + BAR_BYTES;
};

// Decode one 32-bit word of 4-bit codes (8 consecutive elements, element i in bits
// 4i..4i+3: low nibble of each byte = even index) into 8 bf16 values
// w' = (q - 8) * s7, computed in fp32 (q - 8 exact) and rounded once to bf16.
__device__ __forceinline__ uint4 q4_decode8(uint32_t word, float s7) {
    uint32_t out[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t q0 = (word >> (8 * j)) & 0xFu;
        const uint32_t q1 = (word >> (8 * j + 4)) & 0xFu;
        // 2^23 + q as a float, minus 2^23 + 8: exactly q - 8.
        const float f0 = (__uint_as_float(0x4B000000u | q0) - 8388616.0f) * s7;
        const float f1 = (__uint_as_float(0x4B000000u | q1) - 8388616.0f) * s7;
        __nv_bfloat162 b = __floats2bfloat162_rn(f0, f1);
        out[j] = *reinterpret_cast<uint32_t *>(&b);
    }
    return make_uint4(out[0], out[1], out[2], out[3]);
}

// Item i of this cluster: pair tile (m, n), its first output column and width split.
__device__ __forceinline__ bool get_pair_item(const GemmArgs &p, int cluster, int n_clusters, int i, WorkItem &w) {
    w.kb_lo = 0;
    w.kb_hi = p.kb0 + p.kb1;
    w.piece = 0;
    if (i < p.dp_waves) {
        const int t = cluster + i * n_clusters;
        if (t >= p.dp_tiles) return false;
        raster(p, t, w.m, w.n);
        w.nsplit = 1;
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

template <bool B_MN, bool Q4, int STAGES>
__global__ void __launch_bounds__(PairCfg<B_MN, Q4, STAGES>::THREADS, 1)
    k_tc_gemm_pair(const __grid_constant__ GemmArgs p) {
    using Cfg = PairCfg<B_MN, Q4, STAGES>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem;
    uint8_t *sB = smem + STAGES * Cfg::A_BYTES;
    uint8_t *sQ = smem + STAGES * (Cfg::A_BYTES + Cfg::B_BYTES);  // packed codes (Q4)
    uint8_t *sEpi = smem + STAGES * Cfg::STAGE_BYTES;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sEpi + Cfg::EPI_BYTES);
    uint64_t *full_bar = bars;                    // [STAGES] (leader's counts the pair's A (and B) bytes)
    uint64_t *empty_bar = bars + STAGES;          // [STAGES]
    uint64_t *tfull_bar = bars + 2 * STAGES;      // [2]
    uint64_t *tempty_bar = bars + 2 * STAGES + 2; // [2] (leader's: 8 epilogue warps of the pair)
    uint64_t *drain_bar = bars + 2 * STAGES + 4;  // [1]
    uint64_t *pfull_bar = bars + 2 * STAGES + 5;  // [STAGES] Q4: this CTA's packed codes (or bf16 tail B) landed
    uint64_t *bready_bar = bars + 3 * STAGES + 5; // [STAGES] Q4, leader: both CTAs' bf16 B tiles written
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 4 * STAGES + 5);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    volatile int *epi_ok = reinterpret_cast<volatile int *>(tmem_slot + 3);  // [2]
    volatile int *dq_ok = reinterpret_cast<volatile int *>(tmem_slot + 5);   // [2]

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
        if (Q4)
            for (int s = 0; s < STAGES; ++s) {
                mbar_init(smem_u32(&pfull_bar[s]), 1);
                mbar_init(smem_u32(&bready_bar[s]), 2);
            }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        if (Q4) tma_prefetch_desc(&p.tmQ);
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
            uint32_t issued_mask = 0, issued_phase = 0;    // leader's full barriers
            uint32_t qissued_mask = 0, qissued_phase = 0;  // Q4: this CTA's packed-code barriers
            bool ok = true;
            uint64_t wait_empty_ns = 0;
            WorkItem w;
            for (int i = 0; ok && get_pair_item(p, cluster, n_clusters, i, w); ++i) {
                const int bn_cta = (PAIR_BN / w.nsplit) / 2;  // B rows this CTA stages
                const int a_row = w.m * PAIR_BM + static_cast<int>(rank) * 128;
                const int b_row = w.col0 + static_cast<int>(rank) * bn_cta;
                // Q4: B reaches this CTA's smem as packed codes (main K segment) or bf16 (rank-r
                // tail), completing on its own barrier; the leader's full barrier counts A only.
                const uint32_t tx = Q4 ? 2u * static_cast<uint32_t>(Cfg::A_BYTES)
                                       : 2u * static_cast<uint32_t>(Cfg::A_BYTES + bn_cta * BK * 2);
                for (int kb = w.kb_lo; kb < w.kb_hi; ++kb) {
                    const uint64_t tw = trace ? globaltimer_ns() : 0;
                    if (!wait_bounded(smem_u32(&empty_bar[stage]), phase ^ 1u, abort_flag, p.err,
                                      DERR_WAIT_EMPTY)) {
                        ok = false;
                        break;
                    }
                    if (trace) wait_empty_ns += globaltimer_ns() - tw;
                    const uint32_t fb_local = smem_u32(&full_bar[stage]);
                    const uint32_t fb_leader = mapa_shared(fb_local, 0);
                    if (leader) {
                        mbar_arrive_expect_tx(fb_local, tx);
                        issued_mask |= 1u << stage;
                        issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
                    }
                    const bool seg1 = kb >= p.kb0;
                    const int k0 = (seg1 ? kb - p.kb0 : kb) * BK;
                    const uint32_t a_dst = smem_u32(sA + stage * Cfg::A_BYTES);
                    const uint32_t b_dst = smem_u32(sB + stage * Cfg::B_BYTES);
                    tma_load_2d_pair(a_dst, seg1 ? &p.tmA1 : &p.tmA0, fb_leader, k0, a_row);
                    if (Q4) {
                        const uint32_t pb = smem_u32(&pfull_bar[stage]);
                        qissued_mask |= 1u << stage;
                        qissued_phase = (qissued_phase & ~(1u << stage)) | (phase << stage);
                        if (!seg1) {
                            mbar_arrive_expect_tx(pb, static_cast<uint32_t>(Cfg::Q_BYTES));
                            const uint32_t q_dst = smem_u32(sQ + stage * Cfg::Q_BYTES);
                            if (B_MN)  // K rows k0.., bytes of d_in columns b_row..b_row+127
                                tma_load_2d(q_dst, &p.tmQ, pb, b_row / 2, k0);
                            else       // N rows b_row.., bytes of K columns k0..k0+63
                                tma_load_2d(q_dst, &p.tmQ, pb, k0 / 2, b_row);
                        } else {
                            mbar_arrive_expect_tx(pb, static_cast<uint32_t>(bn_cta * BK * 2));
                            if (B_MN) {
                                for (int j = 0; j < bn_cta / 64; ++j)
                                    tma_load_2d(b_dst + j * 64 * 128, &p.tmB1, pb, b_row + 64 * j, k0);
                            } else {
                                tma_load_2d(b_dst, &p.tmB1, pb, k0, b_row);
                            }
                        }
                    } else if (B_MN) {
                        const CUtensorMap *tb = seg1 ? &p.tmB1 : &p.tmB0;
                        for (int j = 0; j < bn_cta / 64; ++j)
                            tma_load_2d_pair(b_dst + j * 64 * 128, tb, fb_leader, b_row + 64 * j, k0);
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
            if (Q4)
                for (int s = 0; s < STAGES; ++s)
                    if (qissued_mask & (1u << s)) {
                        volatile int never = 0;
                        wait_bounded(smem_u32(&pfull_bar[s]), (qissued_phase >> s) & 1u, &never, p.err,
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
                    if (!mbar_try_wait(fb, phase) &&
                        !wait_bounded(fb, phase, abort_flag, p.err, DERR_WAIT_FULL)) {
                        ok = false;
                        break;
                    }
                    if (Q4) {
                        const uint32_t rb = smem_u32(&bready_bar[stage]);
                        if (!mbar_try_wait(rb, phase) &&
                            !wait_bounded(rb, phase, abort_flag, p.err, DERR_WAIT_FULL)) {
                            ok = false;
                            break;
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
            }
        }
    } else if (Q4 && warp >= 6) {
        // ------------------------------------------------------------ dequant warpgroup (both CTAs, Q4)
        // Each K block of the weight segment: wait for this CTA's packed codes, decode
        // them to bf16 into the swizzled B tile the MMA reads, make the generic-proxy
        // stores visible to the tensor core, then report to the leader's B-ready barrier.
        // Rank-r tail blocks arrive as bf16 already and are only reported.
        const int dq = threadIdx.x - 192;  // 0..127
        const uint32_t bready_leader0 = mapa_shared(smem_u32(&bready_bar[0]), 0);
        int stage = 0;
        uint32_t phase = 0;
        int it = 0;
        WorkItem w;
        bool ok = true;
        for (int i = 0; ok && get_pair_item(p, cluster, n_clusters, i, w); ++i) {
            const int bn_cta = (PAIR_BN / w.nsplit) / 2;
            const int b_row = w.col0 + static_cast<int>(rank) * bn_cta;
            for (int kb = w.kb_lo; kb < w.kb_hi; ++kb, ++it) {
                const bool seg1 = kb >= p.kb0;
                const int k0 = kb * BK;
                // this thread's row (K-major: weight row n) or K row and 64-column chunk (MN-major)
                int srow, scol;
                if (B_MN) {
                    srow = k0 + (dq & 63);
                    scol = (b_row + 64 * (dq >> 6)) / 64;
                } else {
                    srow = b_row + dq;
                    scol = kb;
                }
                float s7 = 0.f;
                if (!seg1 && srow < p.scale_rows && scol < p.scale_ld &&
                    (B_MN ? (dq >> 6) < bn_cta / 64 : dq < bn_cta)) {
                    const uint16_t sb = __ldg(p.wscale + static_cast<int64_t>(srow) * p.scale_ld + scol);
                    s7 = __uint_as_float(static_cast<uint32_t>(sb) << 16) / 7.0f;
                }
                if (dq == 0)
                    dq_ok[it & 1] = wait_bounded(smem_u32(&pfull_bar[stage]), phase, abort_flag, p.err,
                                                 DERR_WAIT_FULL) ? 1 : 0;
                named_bar_sync(2, 128);
                if (!dq_ok[it & 1]) {
                    ok = false;
                    break;
                }
                if (!seg1) {
                    const uint8_t *qsrc = sQ + stage * Cfg::Q_BYTES;
                    uint8_t *bdst = sB + stage * Cfg::B_BYTES;
                    if (B_MN) {
                        const int k = dq & 63, j = dq >> 6;
                        if (j < bn_cta / 64) {
                            const uint4 *src = reinterpret_cast<const uint4 *>(qsrc + k * (bn_cta / 2) + j * 32);
                            uint8_t *row = bdst + j * 64 * 128 + (k >> 3) * 1024 + (k & 7) * 128;
#pragma unroll
                            for (int h2 = 0; h2 < 2; ++h2) {
                                const uint4 v = src[h2];
                                const uint32_t wds[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    const int c = h2 * 4 + e;
                                    *reinterpret_cast<uint4 *>(row + ((c ^ (k & 7)) * 16)) = q4_decode8(wds[e], s7);
                                }
                            }
                        }
                    } else if (dq < bn_cta) {
                        const int n = dq;
                        const uint4 *src = reinterpret_cast<const uint4 *>(qsrc + n * 32);
                        uint8_t *row = bdst + (n >> 3) * 1024 + (n & 7) * 128;
#pragma unroll
                        for (int h2 = 0; h2 < 2; ++h2) {
                            const uint4 v = src[h2];
                            const uint32_t wds[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int c = h2 * 4 + e;
                                *reinterpret_cast<uint4 *>(row + ((c ^ (n & 7)) * 16)) = q4_decode8(wds[e], s7);
                            }
                        }
                    }
                    fence_proxy_async_smem();
                }
                named_bar_sync(2, 128);
                if (dq == 0) mbar_arrive_cluster(bready_leader0 + static_cast<uint32_t>(stage * 8));
                stage = stage + 1 == STAGES ? 0 : stage + 1;
                phase = stage == 0 ? phase ^ 1u : phase;
            }
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
            const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                   static_cast<uint32_t>(buf * PAIR_BN);
            uint8_t *stage_base = sEpi + (q * 2) * (32 * 128);
            const int nch = (PAIR_BN / 64) / w.nsplit;
            const int out_row = w.m * PAIR_BM + static_cast<int>(rank) * 128 + q * 32;
#pragma unroll 1
            for (int ch = 0; ch < nch; ++ch) {
                uint32_t v0[32], v1[32];
                tmem_ld_32x32b_x32(t_row + ch * 64, v0);
                tmem_ld_32x32b_x32(t_row + ch * 64 + 32, v1);
                tc_wait_ld();
                if (ch == nch - 1) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(buf ? tempty_leader1 : tempty_leader0);
                }
                uint8_t *sbuf = stage_base + (ch & 1) * (32 * 128);
                if (lane == 0) bulk_wait_group_read<1>();
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
