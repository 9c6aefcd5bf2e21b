// side.cuh -- the rank-r side products of the layer, streamed once from HBM on tcgen05.
//
// Three products share one persistent, warp-specialised kernel.  Each streams one
// large bf16 operand (x or dY) through a TMA ring in shared memory, exactly once, and
// contracts it on the tensor cores against small operands that stay in L2:
//
//   SIDE_XA   s.xa = bf16(s . x.A^T)              [M, r]       reduction over d_in
//   SIDE_GDB  s.g  = bf16(s . dY.B)               [M, r]       reduction over d_out
//             dB   = dY^T.(s.xa)  (partials)      [d_out, r]   reduction over tokens
//   SIDE_DA   dA   = (s.g)^T.x   (written [r, d_in])           reduction over tokens
//             dB   = sum of the SIDE_GDB partials, in order (finishing job)
//
// SIDE_GDB is the single pass over dY of the backward: every 128-token x 128-column dY
// tile in shared memory feeds two MMAs, dY.B (the tile K-major) and dY^T.(s.xa) (the
// same tile read MN-major), so dY is read from HBM once for both.
//
// Work split.  The outputs come in blocks of 128 rows (tokens for s.xa and s.g,
// columns of d_in for dA).  A cluster of C CTAs takes `group` output blocks per round
// and splits the reduction dimension among its CTAs; at the end of the round each CTA
// leaves its fp32 partial in its own shared memory, and after a cluster barrier the
// partials are summed across the cluster over distributed shared memory, in CTA-rank
// order (deterministic), and stored.  No global partials, counters or atomics are
// needed for s.xa, s.g or dA.  dB's reduction runs over tokens, which the rounds split,
// so SIDE_GDB leaves one fp32 partial per round; SIDE_DA, which runs later beside the
// dX GEMM, sums them.
//
// Roles: warp 0 TMA producer (one lane), warp 1 TMEM allocation and single-thread MMA
// issue, warps 2..5 epilogue (one TMEM lane = one output row each).  Every mbarrier
// wait is bounded; on expiry the kernel records an error code, skips the remaining
// work (but still takes every cluster barrier its peers take), drains its copies and
// MMAs, frees TMEM and returns.
#pragma once

#include "tc_gemm.cuh"

namespace lora {

enum SideMode { SIDE_XA = 0, SIDE_GDB = 1, SIDE_DA = 2 };

constexpr int SIDE_THREADS = 192;
constexpr int SIDE_MAX_R = 64;   // widest rank the side kernels take (MN-major operands are 64 wide)
constexpr int SIDE_RED_BYTES = 128 * SIDE_MAX_R * 4;  // reduction landing area: group * 128 * r fp32 at most
constexpr int SIDE_MAX_R_NARROW = 32;  // s.g + dB and dA: r <= 32, their narrow operands N = 16 or 32

struct SideArgs {
    CUtensorMap tmX;   // the streamed operand: x (XA, DA) or dY (GDB); bf16, box {64, 128}, 128B swizzle
    CUtensorMap tmS0;  // XA: A [r, d_in] box {64, nr}, 128B swizzle; GDB: B [d_out, r], DA: s.g [M, r],
                       // box {nb, 128} with the 32B (nb = 16) or 64B (nb = 32) swizzle
    CUtensorMap tmS1;  // GDB: s.xa [M, r], as tmS0
    int r;             // rank (multiple of 8, <= SIDE_MAX_R)
    int nr;            // XA: MMA N = r rounded up to 16
    int nb;            // GDB, DA: MMA N of the narrow operands (B, s.xa, s.g): 16 (r <= 16) or 32
    int n_out;         // 128-row output blocks: ceil(M/128) (XA, GDB) or ceil(d_in/128) (DA)
    int rows_valid;    // output rows: M (XA, GDB) or d_in (DA)
    int n_red;         // reduction blocks: ceil(d_in/64) (XA), ceil(d_out/128) (GDB), ceil(M/128) (DA)
    int per_cta;       // reduction blocks per CTA of a cluster
    int group;         // output blocks per round (GDB; 1 otherwise)
    int n_rounds;      // ceil(n_out / group)
    float scale;       // XA and GDB's g: s, applied in fp32 before the bf16 rounding
    uint16_t *out_bf16;  // XA: s.xa [M, r]; GDB: s.g [M, r]
    float *out_f32;      // DA: dA [r, d_in] (the transposed product is stored transposed)
    float *db_part;      // GDB: writes, DA: reads the dB partials [n_rounds of GDB][d_out][r]
    int d_out;
    float *dB;           // DA: dB [d_out, r] (finishing job), or null
    int db_rounds;       // DA: partial count
    int *err;
    int defer_dep_wait;  // see GemmArgs::defer_dep_wait
    unsigned long long *trace;
};

template <int MODE, int STAGES>
struct SideCfg {
    // streamed tile: XA 128 rows x 64 (16 KB); GDB and DA 128 rows x 128 as two 64-wide
    // 128B-swizzled chunks of 128 rows each (32 KB)
    static constexpr int X_BYTES = (MODE == SIDE_XA) ? 128 * 64 * 2 : 2 * 128 * 64 * 2;
    // small operands: XA the A tile [nr <= 64 rows x 64] K-major; GDB the B tile [128
    // K rows x nb] and the s.xa tile [128 K rows x nb], both MN-major; DA the s.g tile
    static constexpr int S0_BYTES = (MODE == SIDE_XA) ? 64 * 64 * 2 : 128 * SIDE_MAX_R_NARROW * 2;
    static constexpr int S1_BYTES = (MODE == SIDE_GDB) ? 128 * SIDE_MAX_R_NARROW * 2 : 0;
    static constexpr int STAGE_BYTES = X_BYTES + S0_BYTES + S1_BYTES;
    // the cluster reduction's landing area: C slots of each owned row, group * 128 * r
    // fp32 in all (XA: one block of r <= 64; GDB: group * r <= 64; DA: one block of r <= 32)
    static constexpr int RED_BYTES = (MODE == SIDE_DA) ? 128 * SIDE_MAX_R_NARROW * 4 : SIDE_RED_BYTES;
    static constexpr int BAR_BYTES = 256;
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + RED_BYTES + BAR_BYTES;
    static_assert(SMEM_BYTES <= 232448, "at most 227 KB of shared memory per CTA");
    static_assert(STAGE_BYTES % 1024 == 0, "stage tiles stay 1024-byte aligned");
};

// dB accumulators of the s.g + dB kernel: the epilogue drains one per 128-column block
// while the MMA fills the others, so its drain latency stays off the stream.
constexpr int SIDE_NDB = 4;

// TMEM columns a side kernel allocates: XA one accumulator of nr <= 64 columns, DA one
// of nb; GDB `group` g accumulators and SIDE_NDB dB accumulators of nb columns each.
__host__ __device__ constexpr int side_tmem_cols(int mode, int group, int nb) {
    const int need = mode == SIDE_GDB ? (group + SIDE_NDB) * nb : mode == SIDE_DA ? nb : 64;
    return need <= 32 ? 32 : need <= 64 ? 64 : need <= 128 ? 128 : need <= 256 ? 256 : 512;
}

__device__ __forceinline__ uint32_t cluster_nctarank() {
    uint32_t n;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(n));
    return n;
}

// Split cluster barrier: arrive without ordering (this CTA has started), wait with
// acquire; every thread alternates the two.
__device__ __forceinline__ void cluster_arrive_relaxed() {
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.aligned;" ::: "memory"); }

__device__ __forceinline__ void st_shared_cluster_f4(uint32_t addr, float4 v) {
    asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(v.x), "f"(v.y), "f"(v.z),
                 "f"(v.w)
                 : "memory");
}

template <int MODE, int STAGES>
__global__ void __launch_bounds__(SIDE_THREADS, 1) k_side(const __grid_constant__ SideArgs p) {
    using Cfg = SideCfg<MODE, STAGES>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *ring = smem;
    // Cluster reduction: the output rows of a round are split into C contiguous chunks,
    // chunk c owned by CTA rank c; every CTA stores its fp32 partial of each row into the
    // owner's landing area, slot [its rank][row in chunk][r], over distributed shared
    // memory, so the owner then sums local shared memory only.
    float *red = reinterpret_cast<float *>(smem + STAGES * Cfg::STAGE_BYTES);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + STAGES * Cfg::STAGE_BYTES + Cfg::RED_BYTES);
    uint64_t *full_bar = bars;                 // [STAGES]
    uint64_t *empty_bar = bars + STAGES;       // [STAGES]
    uint64_t *acc_bar = bars + 2 * STAGES;     // [1] the round's accumulators are complete
    uint64_t *dbf_bar = bars + 2 * STAGES + 1;             // [SIDE_NDB] GDB: a dB accumulator is complete
    uint64_t *dbe_bar = dbf_bar + SIDE_NDB;                // [SIDE_NDB] GDB: a dB accumulator has been drained
    uint64_t *drain_bar = dbe_bar + SIDE_NDB;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain_bar + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    volatile int *epi_ok = reinterpret_cast<volatile int *>(tmem_slot + 2);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int C = static_cast<int>(cluster_nctarank());
    const int q = static_cast<int>(cluster_ctarank());
    const int cl = static_cast<int>(blockIdx.x) / C;
    const int n_clusters = static_cast<int>(gridDim.x) / C;
    const int tmem_cols = side_tmem_cols(MODE, p.group, p.nb);
    const int nb = p.nb;
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
        mbar_init(smem_u32(acc_bar), 1);
        for (int b = 0; b < SIDE_NDB; ++b) {
            mbar_init(smem_u32(&dbf_bar[b]), 1);
            mbar_init(smem_u32(&dbe_bar[b]), 4);
        }
        mbar_init(smem_u32(drain_bar), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&p.tmX);
        tma_prefetch_desc(&p.tmS0);
        if (MODE == SIDE_GDB) tma_prefetch_desc(&p.tmS1);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), static_cast<uint32_t>(tmem_cols));
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // Peers store into this CTA's shared memory only after they have seen every CTA of
    // the cluster start: the matching wait comes just before the first remote store.
    cluster_arrive_relaxed();
    if (!p.defer_dep_wait) grid_dep_wait();
    grid_dep_launch_dependents();
    if (trace && threadIdx.x == 0) trace[TR_SETUP] = globaltimer_ns();

    // This CTA's share of the reduction dimension (possibly empty).
    const int kb_lo = q * p.per_cta;
    const int kb_hi = min(p.n_red, kb_lo + p.per_cta);
    const bool has_work = kb_hi > kb_lo;
    const int r = p.r;

    // --------------------------------------------------------------- DA: finish dB
    // dB = sum over GDB's rounds of its partials, in round order; the rows are split
    // over the whole grid.  The partials were written by a kernel that completed before
    // this one's stream predecessor started (see the host's launch order).
    if (MODE == SIDE_DA && p.dB != nullptr && warp >= 2) {
        const int et = threadIdx.x - 64;
        const int64_t n4 = static_cast<int64_t>(p.d_out) * r / 4;
        const int64_t per = (n4 + gridDim.x - 1) / gridDim.x;
        const int64_t lo = per * blockIdx.x, hi = min(n4, lo + per);
        const int64_t stride4 = n4;  // one partial, in float4 units
        const float4 *part = reinterpret_cast<const float4 *>(p.db_part);
        // 16 rounds' loads in flight at a time (one after another they cost ~9 us at
        // 32 rounds, a third of that in batches), summed in round order all the same
        for (int64_t i = lo + et; i < hi; i += 128) {
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            int t = 0;
            for (; t + 16 <= p.db_rounds; t += 16) {
                float4 v[16];
#pragma unroll
                for (int u = 0; u < 16; ++u) v[u] = __ldcg(part + (t + u) * stride4 + i);
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    acc.x += v[u].x;
                    acc.y += v[u].y;
                    acc.z += v[u].z;
                    acc.w += v[u].w;
                }
            }
            for (; t < p.db_rounds; ++t) {
                const float4 v = __ldcg(part + t * stride4 + i);
                acc.x += v.x;
                acc.y += v.y;
                acc.z += v.z;
                acc.w += v.w;
            }
            reinterpret_cast<float4 *>(p.dB)[i] = acc;
        }
    }

    // Pipeline state, carried across rounds.
    int p_stage = 0;
    uint32_t p_phase = 0;
    uint32_t issued_mask = 0, issued_phase = 0;  // producer: stages with a copy issued, parity of the last
    int m_stage = 0;
    uint32_t m_phase = 0;
    int db_use = 0;  // GDB: dB accumulator uses so far (MMA and epilogue count alike)
    int round_i = 0;

    for (int t = cl; t < p.n_rounds; t += n_clusters, ++round_i) {
        const int o_lo = t * p.group;
        const int o_n = min(p.group, p.n_out - o_lo);

        if (warp == 0) {
            // ----------------------------------------------------------- TMA producer
            if (lane == 0 && has_work && !*abort_flag) {
                bool ok = true;
                for (int kb = kb_lo; ok && kb < kb_hi; ++kb) {
                    for (int i = 0; i < o_n; ++i) {
                        if (!wait_bounded(smem_u32(&empty_bar[p_stage]), p_phase ^ 1u, abort_flag, p.err,
                                          DERR_WAIT_EMPTY)) {
                            ok = false;
                            break;
                        }
                        const uint32_t fb = smem_u32(&full_bar[p_stage]);
                        uint8_t *st = ring + p_stage * Cfg::STAGE_BYTES;
                        const uint32_t xs = smem_u32(st), s0 = smem_u32(st + Cfg::X_BYTES),
                                       s1 = smem_u32(st + Cfg::X_BYTES + Cfg::S0_BYTES);
                        const int o = o_lo + i;
                        if (MODE == SIDE_XA) {
                            mbar_arrive_expect_tx(fb, Cfg::X_BYTES + p.nr * 128);
                            tma_load_2d(xs, &p.tmX, fb, kb * 64, o * 128);
                            tma_load_2d(s0, &p.tmS0, fb, kb * 64, 0);
                        } else if (MODE == SIDE_GDB) {
                            // dY [128 tokens of block o][128 columns of block kb] as two chunks,
                            // B rows of block kb, s.xa rows of block o
                            mbar_arrive_expect_tx(fb, Cfg::X_BYTES + 2 * 128 * nb * 2);
                            tma_load_2d(xs, &p.tmX, fb, kb * 128, o * 128);
                            tma_load_2d(xs + 16384, &p.tmX, fb, kb * 128 + 64, o * 128);
                            tma_load_2d(s0, &p.tmS0, fb, 0, kb * 128);
                            tma_load_2d(s1, &p.tmS1, fb, 0, o * 128);
                        } else {
                            // x [128 tokens of block kb][128 columns of d_in block o] as two
                            // chunks, s.g rows of token block kb
                            mbar_arrive_expect_tx(fb, Cfg::X_BYTES + 128 * nb * 2);
                            tma_load_2d(xs, &p.tmX, fb, o * 128, kb * 128);
                            tma_load_2d(xs + 16384, &p.tmX, fb, o * 128 + 64, kb * 128);
                            tma_load_2d(s0, &p.tmS0, fb, 0, kb * 128);
                        }
                        issued_mask |= 1u << p_stage;
                        issued_phase = (issued_phase & ~(1u << p_stage)) | (p_phase << p_stage);
                        if (++p_stage == STAGES) {
                            p_stage = 0;
                            p_phase ^= 1u;
                        }
                    }
                }
                if (trace) trace[TR_PROD_END] = globaltimer_ns();
            }
            __syncwarp();
            if (round_i == 0) cluster_wait();
        } else if (warp == 1) {
            // ----------------------------------------------------------- MMA issuer
            if (lane == 0) {
                bool ok = has_work && !*abort_flag;
                for (int kb = kb_lo; ok && kb < kb_hi; ++kb) {
                    uint32_t db_tmem = 0;
                    if (MODE == SIDE_GDB) {
                        // the dB accumulator of this column block: free once drained
                        const int b = db_use % SIDE_NDB;
                        if (!wait_bounded(smem_u32(&dbe_bar[b]), ((db_use / SIDE_NDB) & 1) ^ 1u, abort_flag, p.err,
                                          DERR_WAIT_TMEM_EMPTY)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        db_tmem = tmem_base + static_cast<uint32_t>((p.group + b) * nb);
                    }
                    for (int i = 0; i < o_n; ++i) {
                        const uint32_t fb = smem_u32(&full_bar[m_stage]);
                        if (!wait_bounded(fb, m_phase, abort_flag, p.err, DERR_WAIT_FULL)) {
                            ok = false;
                            break;
                        }
                        if (trace && kb == kb_lo && i == 0 && round_i == 0) trace[TR_TILE_DONE0] = globaltimer_ns();
                        tc_fence_after();
                        const uint32_t xs = smem_u32(ring + m_stage * Cfg::STAGE_BYTES);
                        const uint32_t s0 = xs + Cfg::X_BYTES, s1 = s0 + Cfg::S0_BYTES;
                        if (MODE == SIDE_XA) {
                            // acc [128 tokens x nr] += x tile (K-major) . A tile^T (K-major)
                            const uint32_t idesc = idesc_bf16(128, p.nr, false, false);
                            const uint64_t ad = sdesc_sw128(xs, 16, 1024), bd = sdesc_sw128(s0, 16, 1024);
                            for (int kk = 0; kk < 4; ++kk)
                                tc_mma_bf16(tmem_base, ad + (kk * 32 >> 4), bd + (kk * 32 >> 4), idesc,
                                            (kb > kb_lo || kk > 0) ? 1u : 0u);
                        } else if (MODE == SIDE_GDB) {
                            // g acc of block i [128 tokens x nb] += dY tile (K-major, K = 128 columns) . B
                            const uint32_t idesc_g = idesc_bf16(128, nb, false, true);
                            const uint32_t g_tmem = tmem_base + static_cast<uint32_t>(i * nb);
                            const uint64_t bd = sdesc_mn_narrow(s0, nb);
                            const uint32_t bstep = static_cast<uint32_t>(nb) * 32u >> 4;  // 16 K rows
                            for (int kk = 0; kk < 8; ++kk) {
                                const uint64_t ad = sdesc_sw128(xs + (kk >> 2) * 16384, 16, 1024) + ((kk & 3) * 32 >> 4);
                                tc_mma_bf16(g_tmem, ad, bd + kk * bstep, idesc_g, (kb > kb_lo || kk > 0) ? 1u : 0u);
                            }
                            // dB acc [128 columns x nb] += dY tile^T (MN-major, K = 128 tokens) . s.xa
                            const uint32_t idesc_b = idesc_bf16(128, nb, true, true);
                            const uint64_t ad2 = sdesc_sw128(xs, 16384, 1024), bd2 = sdesc_mn_narrow(s1, nb);
                            for (int kk = 0; kk < 8; ++kk)
                                tc_mma_bf16(db_tmem, ad2 + (kk * 2048 >> 4), bd2 + kk * bstep, idesc_b,
                                            (i > 0 || kk > 0) ? 1u : 0u);
                        } else {
                            // dA^T acc [128 columns of d_in x nb] += x tile^T (MN-major, K = 128 tokens) . s.g
                            const uint32_t idesc_a = idesc_bf16(128, nb, true, true);
                            const uint64_t ad = sdesc_sw128(xs, 16384, 1024), bd = sdesc_mn_narrow(s0, nb);
                            const uint32_t bstep = static_cast<uint32_t>(nb) * 32u >> 4;  // 16 K rows
                            for (int kk = 0; kk < 8; ++kk)
                                tc_mma_bf16(tmem_base, ad + (kk * 2048 >> 4), bd + kk * bstep, idesc_a,
                                            (kb > kb_lo || kk > 0) ? 1u : 0u);
                        }
                        tc_commit(smem_u32(&empty_bar[m_stage]));
                        if (++m_stage == STAGES) {
                            m_stage = 0;
                            m_phase ^= 1u;
                        }
                    }
                    if (MODE == SIDE_GDB && ok) {
                        tc_commit(smem_u32(&dbf_bar[db_use % SIDE_NDB]));
                        ++db_use;
                    }
                }
                // the round's accumulators (s.xa, s.g or dA) are complete once every MMA is
                tc_commit(smem_u32(acc_bar));
                if (trace) trace[TR_MMA_END] = globaltimer_ns();
            }
            __syncwarp();
            if (round_i == 0) cluster_wait();
        } else {
            // ----------------------------------------------------------- epilogue
            const int qd = warp & 3;
            const int row = qd * 32 + lane;  // TMEM lane = row of the 128-row block
            const int et = threadIdx.x - 64;
            const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(qd * 32) << 16);
            if (MODE == SIDE_GDB && has_work) {
                // dB partial of each column block of this CTA, for this round's tokens
                // Each warp drains its own 32 rows on its own (its lanes wait, the warp votes),
                // with one TMEM load of all nb columns: no barrier spans warps, so the drain's
                // latency overlaps the MMAs into the other dB accumulators.
                for (int kb = kb_lo; kb < kb_hi; ++kb) {
                    const int b = db_use % SIDE_NDB;
                    const bool okk = !*abort_flag && wait_bounded(smem_u32(&dbf_bar[b]), (db_use / SIDE_NDB) & 1u,
                                                                  abort_flag, p.err, DERR_WAIT_TMEM_FULL);
                    if (!__all_sync(0xFFFFFFFFu, okk)) break;
                    tc_fence_after();
                    const int n = kb * 128 + row;
                    float *dst = p.db_part + (static_cast<int64_t>(t) * p.d_out + n) * r;
                    uint32_t v[32];
                    const uint32_t taddr = lane_base + static_cast<uint32_t>((p.group + b) * nb);
                    if (nb == 16) {
                        uint32_t (&v16)[16] = *reinterpret_cast<uint32_t(*)[16]>(v);
                        tmem_ld_32x32b_x16(taddr, v16);
                    } else {
                        tmem_ld_32x32b_x32(taddr, v);
                    }
                    tc_wait_ld();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(smem_u32(&dbe_bar[b]));
                    if (n < p.d_out) {
#pragma unroll
                        for (int c0 = 0; c0 < 32; c0 += 4)  // constant indices keep v in registers
                            if (c0 < r)
                                *reinterpret_cast<float4 *>(dst + c0) =
                                    make_float4(__uint_as_float(v[c0]), __uint_as_float(v[c0 + 1]),
                                                __uint_as_float(v[c0 + 2]), __uint_as_float(v[c0 + 3]));
                    }
                    ++db_use;
                }
            }
            // this CTA's partial of each of the round's output rows -> the owner's landing area
            if (et == 0)
                epi_ok[1] = (!*abort_flag && wait_bounded(smem_u32(acc_bar), static_cast<uint32_t>(round_i) & 1u,
                                                          abort_flag, p.err, DERR_WAIT_TMEM_FULL))
                                ? 1
                                : 0;
            named_bar_sync(1, 128);
            const bool acc_ok = epi_ok[1] != 0;
            tc_fence_after();
            const int chunk = (o_n * 128 + C - 1) / C;
            if (round_i == 0) cluster_wait();  // every CTA of the cluster has started
            for (int i = 0; i < o_n; ++i) {
                const int idx = i * 128 + row;
                const uint32_t owner = static_cast<uint32_t>(idx / chunk);
                const uint32_t dst = mapa_shared(
                    smem_u32(red) + static_cast<uint32_t>(((q * chunk + idx % chunk) * r) * 4), owner);
                for (int c0 = 0; c0 < r; c0 += 8) {
                    float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
                    if (acc_ok && has_work) {
                        uint32_t v[8];
                        tmem_ld_32x32b_x8(lane_base + static_cast<uint32_t>(i * (MODE == SIDE_XA ? 64 : nb) + c0), v);
                        tc_wait_ld();
                        a = make_float4(__uint_as_float(v[0]), __uint_as_float(v[1]), __uint_as_float(v[2]),
                                        __uint_as_float(v[3]));
                        b = make_float4(__uint_as_float(v[4]), __uint_as_float(v[5]), __uint_as_float(v[6]),
                                        __uint_as_float(v[7]));
                    }
                    st_shared_cluster_f4(dst + static_cast<uint32_t>(c0 * 4), a);
                    st_shared_cluster_f4(dst + static_cast<uint32_t>(c0 * 4 + 16), b);
                }
            }
            tc_fence_before();
        }

        // ------------------------------------------------------------- cluster reduction
        // Every thread of every CTA of the cluster takes the same barriers, in every round,
        // whatever happened before, so no CTA waits for a peer that left.
        __syncthreads();
        cluster_sync();  // every partial has landed in its owner's shared memory
        if (trace && threadIdx.x == 0) trace[TR_TILE_DONE0 + 1] = globaltimer_ns();
        if (warp >= 2) {
            const int et = threadIdx.x - 64;
            const int rows = o_n * 128;
            const int chunk = (rows + C - 1) / C;
            const int lo = q * chunk, hi = min(rows, lo + chunk);
            const int r4 = r / 4;
            // one (row, 4 columns) item per thread and step, summed over the C slots in rank order
            for (int it = et; it < (hi - lo) * r4; it += 128) {
                const int lr = it / r4, c0 = (it - lr * r4) * 4;
                const int orow = o_lo * 128 + lo + lr;  // output row (token, or column of d_in)
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
                for (int c = 0; c < C; ++c) {
                    const float4 v = *reinterpret_cast<const float4 *>(red + (c * chunk + lr) * r + c0);
                    acc.x += v.x;
                    acc.y += v.y;
                    acc.z += v.z;
                    acc.w += v.w;
                }
                if (orow >= p.rows_valid || *abort_flag) continue;
                if (MODE == SIDE_DA) {
                    float *o = p.out_f32;
                    o[static_cast<int64_t>(c0 + 0) * p.rows_valid + orow] = acc.x;
                    o[static_cast<int64_t>(c0 + 1) * p.rows_valid + orow] = acc.y;
                    o[static_cast<int64_t>(c0 + 2) * p.rows_valid + orow] = acc.z;
                    o[static_cast<int64_t>(c0 + 3) * p.rows_valid + orow] = acc.w;
                } else {
                    __nv_bfloat162 lo2 = __floats2bfloat162_rn(acc.x * p.scale, acc.y * p.scale);
                    __nv_bfloat162 hi2 = __floats2bfloat162_rn(acc.z * p.scale, acc.w * p.scale);
                    *reinterpret_cast<uint2 *>(p.out_bf16 + static_cast<int64_t>(orow) * r + c0) =
                        make_uint2(*reinterpret_cast<uint32_t *>(&lo2), *reinterpret_cast<uint32_t *>(&hi2));
                }
            }
        }
        // Before the next round's partials land here, every owner has read this round's
        // (the peers store nothing after the barrier above, so the last round needs none).
        if (t + n_clusters < p.n_rounds) {
            __syncthreads();
            cluster_sync();
        }
    }
    if (round_i == 0) cluster_wait();  // no round: close the start-up barrier phase
    if (trace && threadIdx.x == 0) trace[TR_EPI_END] = globaltimer_ns();

    // ---------------------------------------------------------------- teardown
    if (warp == 0 && lane == 0) {
        // copies issued and never consumed (only after a failed wait) land before exit
        for (int s = 0; s < STAGES; ++s)
            if (issued_mask & (1u << s)) {
                volatile int never = 0;
                wait_bounded(smem_u32(&full_bar[s]), (issued_phase >> s) & 1u, &never, p.err, DERR_WAIT_DRAIN);
            }
    }
    if (warp == 1 && lane == 0) {
        tc_commit(smem_u32(drain_bar));
        volatile int never = 0;
        wait_bounded(smem_u32(drain_bar), 0, &never, p.err, DERR_WAIT_DRAIN);
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, static_cast<uint32_t>(tmem_cols));
    }
    if (p.defer_dep_wait) grid_dep_wait();
    if (trace && threadIdx.x == 0) trace[TR_EXIT] = globaltimer_ns();
}

}  // namespace lora
