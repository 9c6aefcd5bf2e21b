// lora_linear.cu -- host side of the C ABI declared in include/lora_linear.h.
//
// Validates arguments, carves the caller's workspace, encodes TMA tensor maps and
// enqueues the tcgen05 kernels of tc_gemm.cuh on the caller's stream:
//
//   forward   xa  : s.xa = bf16(s . x.A^T)                      reduction over d_in
//             fwd : h = [x | s.xa] . [W | B]^T                  K = d_in + r, one accumulator
//   backward  xa  : (only when no saved s.xa)
//             g   : s.g = bf16(s . dY.B), and dB's partials     one pass over dY
//             dx  : dX = [dY | s.g] . [W ; A]                   K = d_out + r, W and A MN-major
//             dadb: dA = (s.g)^T . x (written as [r, d_in]), and dB summed from its
//                   partials, overlapping the dX GEMM's last wave
//
// For r <= 64 the rank-r products run on the cluster-reduction side kernels of
// side.cuh; wider ranks use the split-K kernels of tc_gemm.cuh (s.xa, s.g, then dB and
// dA in one launch, each split over its reduction dimension with a fixed-order fix-up).
//
// No allocation, no synchronisation, no exceptions across the ABI.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/lora_linear.h"
#include "side.cuh"
#include "tc_gemm.cuh"
#include "tc_gemm2.cuh"
#include "tmap.h"

using namespace lora;

namespace {

// ------------------------------------------------------------------ kernel configs
constexpr int MAIN_BN = 256;
constexpr int MAIN_STAGES = 4;
constexpr int SKINNY_SMEM_BUDGET = 196 * 1024;

template <int BN>
constexpr int skinny_stages() {
    constexpr int stage = BM * BK * 2 + BN * BK * 2;
    constexpr int s = SKINNY_SMEM_BUDGET / stage;
    return s > 8 ? 8 : s;
}

// ------------------------------------------------------------------ device info
struct DevInfo {
    bool probed = false;
    bool supported = false;
    int sms = 0;
    uint64_t attr_set = 0;  // bit per kernel instantiation whose smem attribute is set
};
std::mutex g_mu;
DevInfo g_dev[64];

bool device_info(int *dev_out, DevInfo **info) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
    std::lock_guard<std::mutex> lk(g_mu);
    DevInfo &d = g_dev[dev];
    if (!d.probed) {
        int major = 0, minor = 0, sms = 0;
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        d.supported = (major == 10 && minor == 0);
        d.sms = sms;
        d.probed = true;
    }
    *dev_out = dev;
    *info = &d;
    return true;
}

// ------------------------------------------------------------------ tensor maps
// Row-major 2D bf16 tensor [rows][cols] (cols contiguous), tile box {box_cols, box_rows},
// 128-byte swizzle (the tensor cores' operand layout), zero fill outside the tensor.
bool tmap_bf16(CUtensorMap *m, const void *base, uint64_t cols, uint64_t rows, uint32_t box_cols,
               uint32_t box_rows) {
    return lora_host::tmap_2d(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, cols, rows, box_cols, box_rows,
                              CU_TENSOR_MAP_SWIZZLE_128B);
}

// Row-major 2D uint8 tensor [rows][cols_bytes], box {box_bytes, box_rows} of 32- or 64-byte
// rows (the packed codes, read by threads rather than by the tensor cores), with the
// swizzle of the row's width: it moves each row's 16-byte chunks so that the 32 lanes of
// a warp, each reading one row, spread over all the shared-memory banks.
bool tmap_u8(CUtensorMap *m, const void *base, uint64_t cols_bytes, uint64_t rows, uint32_t box_bytes,
             uint32_t box_rows) {
    const CUtensorMapSwizzle swz = box_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
    return lora_host::tmap_2d(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, base, cols_bytes, rows, box_bytes, box_rows, swz);
}

// ------------------------------------------------------------------ timing hooks
std::atomic<int64_t> g_launches{0};
std::atomic<int> g_timing{0};
struct TimedLaunch {
    int kind;
    cudaEvent_t a, b;
};
std::mutex g_tmu;
std::vector<TimedLaunch> g_timed;
std::vector<cudaEvent_t> g_event_pool;

cudaEvent_t pool_event() {
    if (!g_event_pool.empty()) {
        cudaEvent_t e = g_event_pool.back();
        g_event_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}

// Optional device trace buffer: kind k writes its CTAs' records at k * trace_stride words.
std::atomic<unsigned long long *> g_trace{nullptr};
std::atomic<size_t> g_trace_stride{0};

// Programmatic dependent launch between consecutive kernels (LORA_LINEAR_PDL=0 turns
// it off, for measurement).
bool pdl_enabled() {
    const char *v = std::getenv("LORA_LINEAR_PDL");
    return !(v && v[0] == '0');
}

// Main GEMMs on CTA pairs (tcgen05 cta_group::2); LORA_LINEAR_PAIR=0 selects the
// single-SM kernel instead, for measurement.
bool pair_enabled() {
    const char *v = std::getenv("LORA_LINEAR_PAIR");
    return !(v && v[0] == '0');
}

// Rank-r products (r <= 64) on the cluster-reduction side kernels; LORA_LINEAR_SIDE=0
// selects the split-K kernels instead, for measurement.  Read when a plan is made
// (the workspace size follows it).
bool side_enabled() {
    const char *v = std::getenv("LORA_LINEAR_SIDE");
    return !(v && v[0] == '0');
}

// ------------------------------------------------------------------ launch helpers
template <int BN, bool A_MN, bool B_MN, int EPI, int STAGES>
cudaError_t launch_gemm(const GemmArgs &args, int grid, cudaStream_t st, DevInfo *dev, int attr_bit, int kind) {
    using Cfg = GemmCfg<BN, A_MN, B_MN, EPI, STAGES>;
    auto kern = k_tc_gemm<BN, A_MN, B_MN, EPI, STAGES>;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!(dev->attr_set & (1ull << attr_bit))) {
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES);
            if (e != cudaSuccess) return e;
            dev->attr_set |= 1ull << attr_bit;
        }
    }
    cudaEvent_t ea = nullptr, eb = nullptr;
    const bool timed = g_timing.load() != 0;
    if (timed) {
        std::lock_guard<std::mutex> lk(g_tmu);
        ea = pool_event();
        eb = pool_event();
        if (ea) cudaEventRecord(ea, st);
    }
    GemmArgs a2 = args;
    unsigned long long *tr = g_trace.load();
    const size_t stride = g_trace_stride.load();
    if (tr && static_cast<size_t>(grid) * TRACE_WORDS <= stride) a2.trace = tr + static_cast<size_t>(kind) * stride;
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(NUM_THREADS);
    cfg.dynamicSmemBytes = Cfg::SMEM_BYTES;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 1 : 0;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, a2);
    if (e == cudaSuccess) e = cudaGetLastError();
    g_launches.fetch_add(1);
    if (timed && ea && eb) {
        cudaEventRecord(eb, st);
        std::lock_guard<std::mutex> lk(g_tmu);
        g_timed.push_back({kind, ea, eb});
    }
    return e;
}

constexpr int PAIR_STAGES = 6;
constexpr int PAIR_STAGES_Q4 = 5;
constexpr int PAIR_STAGES_FP8 = 5;  // with one run per thread, the FP8 code slots take what the 4-bit ones do

template <int WF>
constexpr int pair_stages() {
    return (WF == WF_Q4 || WF == WF_CB) ? PAIR_STAGES_Q4 : WF == WF_FP8 ? PAIR_STAGES_FP8 : PAIR_STAGES;
}

template <bool B_MN, int WF>
cudaError_t launch_pair(const GemmArgs &args, int grid, cudaStream_t st, DevInfo *dev, int attr_bit, int kind) {
    constexpr int S = pair_stages<WF>();
    using Cfg = PairCfg<B_MN, WF, S>;
    auto kern = k_tc_gemm_pair<B_MN, WF, S>;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!(dev->attr_set & (1ull << attr_bit))) {
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES);
            if (e != cudaSuccess) return e;
            dev->attr_set |= 1ull << attr_bit;
        }
    }
    cudaEvent_t ea = nullptr, eb = nullptr;
    const bool timed = g_timing.load() != 0;
    if (timed) {
        std::lock_guard<std::mutex> lk(g_tmu);
        ea = pool_event();
        eb = pool_event();
        if (ea) cudaEventRecord(ea, st);
    }
    GemmArgs a2 = args;
    unsigned long long *tr = g_trace.load();
    const size_t stride = g_trace_stride.load();
    if (tr && static_cast<size_t>(grid) * TRACE_WORDS <= stride) a2.trace = tr + static_cast<size_t>(kind) * stride;
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(Cfg::THREADS);
    cfg.dynamicSmemBytes = Cfg::SMEM_BYTES;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 2 : 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, a2);
    if (e == cudaSuccess) e = cudaGetLastError();
    g_launches.fetch_add(1);
    if (timed && ea && eb) {
        cudaEventRecord(eb, st);
        std::lock_guard<std::mutex> lk(g_tmu);
        g_timed.push_back({kind, ea, eb});
    }
    return e;
}

// Side kernels: clusters of C CTAs (1, 2 or 4), programmatic dependent launch.  The
// grid is `clusters` clusters, capped at the clusters the device keeps resident at once
// (the rounds are then spread over fewer clusters; results do not depend on the grid).
template <int MODE, int STAGES>
cudaError_t launch_side(const SideArgs &args, int clusters, int C, cudaStream_t st, DevInfo *dev, int attr_bit,
                        int kind) {
    using Cfg = SideCfg<MODE, STAGES>;
    auto kern = k_side<MODE, STAGES>;
    static int resident[64][4] = {};  // [device][log2 C]: clusters resident at once (0: not probed)
    int d = 0;
    cudaGetDevice(&d);
    const int lc = C >= 4 ? 2 : C >= 2 ? 1 : 0;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!(dev->attr_set & (1ull << attr_bit))) {
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES);
            if (e != cudaSuccess) return e;
            dev->attr_set |= 1ull << attr_bit;
        }
        if (d >= 0 && d < 64 && resident[d][lc] == 0) {
            cudaLaunchConfig_t oc;
            std::memset(&oc, 0, sizeof(oc));
            oc.gridDim = dim3(static_cast<unsigned>(C * std::max(1, dev->sms / C)));
            oc.blockDim = dim3(SIDE_THREADS);
            oc.dynamicSmemBytes = Cfg::SMEM_BYTES;
            cudaLaunchAttribute ca[1];
            ca[0].id = cudaLaunchAttributeClusterDimension;
            ca[0].val.clusterDim.x = C;
            ca[0].val.clusterDim.y = 1;
            ca[0].val.clusterDim.z = 1;
            oc.attrs = ca;
            oc.numAttrs = 1;
            int n = 0;
            if (cudaOccupancyMaxActiveClusters(&n, kern, &oc) != cudaSuccess || n < 1) {
                cudaGetLastError();
                n = -1;  // unknown: no cap
            }
            resident[d][lc] = n;
        }
        if (d >= 0 && d < 64 && resident[d][lc] > 0) clusters = std::min(clusters, resident[d][lc]);
    }
    const int grid = clusters * C;
    cudaEvent_t ea = nullptr, eb = nullptr;
    const bool timed = g_timing.load() != 0;
    if (timed) {
        std::lock_guard<std::mutex> lk(g_tmu);
        ea = pool_event();
        eb = pool_event();
        if (ea) cudaEventRecord(ea, st);
    }
    SideArgs a2 = args;
    unsigned long long *tr = g_trace.load();
    const size_t stride = g_trace_stride.load();
    if (tr && static_cast<size_t>(grid) * TRACE_WORDS <= stride) a2.trace = tr + static_cast<size_t>(kind) * stride;
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(SIDE_THREADS);
    cfg.dynamicSmemBytes = Cfg::SMEM_BYTES;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 2 : 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, a2);
    if (e == cudaSuccess) e = cudaGetLastError();
    g_launches.fetch_add(1);
    if (timed && ea && eb) {
        cudaEventRecord(eb, st);
        std::lock_guard<std::mutex> lk(g_tmu);
        g_timed.push_back({kind, ea, eb});
    }
    return e;
}

template <bool B_MN, int WF>
int probe_pair_clusters(const DevInfo *dev) {
    constexpr int S = pair_stages<WF>();
    using Cfg = PairCfg<B_MN, WF, S>;
    auto kern = k_tc_gemm_pair<B_MN, WF, S>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(2 * (dev->sms / 2));
    cfg.blockDim = dim3(Cfg::THREADS);
    cfg.dynamicSmemBytes = Cfg::SMEM_BYTES;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
        cudaGetLastError();
        n = 0;
    }
    return n;
}

// Clusters of two CTAs of the pair kernel that can be resident at once (0 if none).
int pair_clusters(DevInfo *dev, bool b_mn, int wf) {
    static int cached[64][8] = {};
    static bool probed[64][8] = {};
    int d = 0;
    cudaGetDevice(&d);
    std::lock_guard<std::mutex> lk(g_mu);
    if (d < 0 || d >= 64) return 0;
    const int v = (b_mn ? 1 : 0) + 2 * wf;
    if (!probed[d][v]) {
        probed[d][v] = true;
        switch (v) {
            case 0: cached[d][v] = probe_pair_clusters<false, WF_BF16>(dev); break;
            case 1: cached[d][v] = probe_pair_clusters<true, WF_BF16>(dev); break;
            case 2: cached[d][v] = probe_pair_clusters<false, WF_Q4>(dev); break;
            case 3: cached[d][v] = probe_pair_clusters<true, WF_Q4>(dev); break;
            case 4: cached[d][v] = probe_pair_clusters<false, WF_FP8>(dev); break;
            case 5: cached[d][v] = probe_pair_clusters<true, WF_FP8>(dev); break;
            case 6: cached[d][v] = probe_pair_clusters<false, WF_CB>(dev); break;
            default: cached[d][v] = probe_pair_clusters<true, WF_CB>(dev); break;
        }
    }
    return cached[d][v];
}

// Attribute bits of the instantiations (one per template combination).
enum {
    AB_FWD = 0,
    AB_DX = 1,
    AB_XA16 = 2, AB_XA64, AB_XA128, AB_XA256,
    AB_G64 = 6, AB_G128, AB_G256,
    AB_T64 = 9, AB_T128, AB_T256,
    AB_PAIR_K = 12, AB_PAIR_MN = 13, AB_PAIR_K_Q4 = 14, AB_PAIR_MN_Q4 = 15,
    AB_SIDE_XA = 16, AB_SIDE_GDB = 17, AB_SIDE_DA = 18,
    AB_PAIR_K_FP8 = 19, AB_PAIR_MN_FP8 = 20, AB_PAIR_K_CB = 21, AB_PAIR_MN_CB = 22,
};

int bn_class_kmajor(int r) { return r <= 16 ? 16 : r <= 64 ? 64 : r <= 128 ? 128 : 256; }
int bn_class_mnmajor(int r) { return r <= 64 ? 64 : r <= 128 ? 128 : 256; }

// ------------------------------------------------------------------ workspace plan
int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }
size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

struct Split {
    int splits = 1, per = 1;
};

// Splits of K (in 64-wide blocks) for a skinny kernel with `mt` output tiles.  Each
// CTA should stream one long contiguous K range (the per-tile epilogue and split-K
// fixup cost about as much as a few blocks of loads), so the split count is the
// largest that still gives every SM at most one tile, keeping >= 4 blocks per split.
Split choose_split(int64_t mt, int64_t kb, int sms) {
    Split sp;
    int64_t s = std::max<int64_t>(1, sms / std::max<int64_t>(1, mt));
    s = std::min<int64_t>(s, std::max<int64_t>(1, kb / 4));
    s = std::min<int64_t>(s, 64);
    const int64_t per = cdiv(kb, s);
    sp.per = static_cast<int>(per);
    sp.splits = static_cast<int>(cdiv(kb, per));
    return sp;
}

constexpr int PLAN_SMS = 148;  // SMs a launch uses at most (sizes splits and the workspace)
constexpr int KSPLIT_MIN_KB = 32;  // K blocks of 64 below which the forward's tail is not cut along K

// Main-GEMM schedule: whole 128 x 256 tiles in waves over G CTAs; a partial last
// wave of R tiles is cut along N into 2 or 4 narrower tiles (one per CTA) when they
// fit in one wave, so the last wave lasts a half or a quarter tile.
struct MainSched {
    int tiles = 0, dp_tiles = 0, dp_waves = 0, tail_tiles = 0, tail_split = 1;
};

MainSched main_sched(int64_t M, int64_t N, int G) {
    MainSched s;
    const int64_t T = cdiv(M, BM) * cdiv(N, MAIN_BN);
    s.tiles = static_cast<int>(T);
    const int64_t W = T / G, R = T % G;
    const int split = (R > 0 && 4 * R <= G) ? 4 : (R > 0 && 2 * R <= G) ? 2 : 1;
    if (W >= 1 && split > 1) {
        s.dp_tiles = static_cast<int>(W * G);
        s.dp_waves = static_cast<int>(W);
        s.tail_tiles = static_cast<int>(R);
        s.tail_split = split;
    } else {
        s.dp_tiles = static_cast<int>(T);
        s.dp_waves = static_cast<int>(cdiv(T, G));
    }
    return s;
}

// Side-kernel plan (r <= 64): a cluster of C CTAs takes `group` 128-row output blocks
// per round and splits the n_red reduction blocks among its CTAs.
struct SidePlan {
    int C = 1, clusters = 0, group = 1, rounds = 0, per_cta = 0, n_out = 0, n_red = 0;
};

constexpr int SIDE_XA_STAGES = 8;   // 24 KB stages: 128 KB of x in flight
constexpr int SIDE_GDB_STAGES = 4;  // 48 KB stages: 128 KB of dY in flight
constexpr int SIDE_DA_STAGES = 5;   // 40 KB stages: 160 KB of x in flight

// Cluster sizes of the side kernels.  A cluster's CTAs (one per SM: each holds ~225 KB
// of shared memory) must fit in one GPC together; clusters of 8 did not all fit at once
// on B200 and ran in two waves, clusters of 4 did.  dA, when it starts on the SMs the dX
// GEMM's CTA pairs leave as they finish, takes pairs.
constexpr int SIDE_MAX_C = 4;
constexpr int SIDE_MAX_C_DA = 2;

// One output block per round; C the largest power of two <= max_c that keeps one round
// of every output block within `sms` CTAs and gives each CTA some reduction work.
SidePlan side_plan(int64_t n_out, int64_t n_red, int sms, int max_c, int force_c = 0) {
    SidePlan sp;
    int C = 1;
    while (C < max_c && n_out * 2 * C <= sms && 2 * C <= n_red) C *= 2;
    if (force_c > 0) C = force_c;
    sp.C = C;
    sp.n_out = static_cast<int>(n_out);
    sp.n_red = static_cast<int>(n_red);
    sp.group = 1;
    sp.rounds = static_cast<int>(n_out);
    sp.clusters = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(n_out, sms / C)));
    sp.per_cta = static_cast<int>(cdiv(n_red, C));
    return sp;
}

// Streaming cost model of the plans below: HBM bandwidth shared by the CTAs that
// stream, up to what one SM's copy engine sustains on its own (both measured on B200).
constexpr double SIDE_HBM_GBS = 6100.0;
constexpr double SIDE_SM_GBS = 55.0;

double side_stream_us(double bytes_per_cta, int ctas) {
    const double bw = std::min(SIDE_HBM_GBS / std::max(1, ctas), SIDE_SM_GBS);
    return bytes_per_cta / (bw * 1e3);
}

// s.g and dB in one pass over dY: `group` token blocks per round (their g accumulators
// stay in tensor memory while the round's CTAs sweep d_out), C CTAs split d_out.  Each
// round leaves one fp32 dB partial [d_out, r]; the choice weighs the streaming time of
// the busiest CTA against writing those partials.
SidePlan side_plan_gdb(int64_t M, int64_t d_out, int r, int sms, int force_c = 0, int force_a = 0) {
    const int64_t n_out = cdiv(M, BM), n_red = cdiv(d_out, 128);
    SidePlan best;
    double best_cost = 1e300;
    for (int a = 1; a <= 6; ++a) {
        if (static_cast<int64_t>(a) * 128 * r * 4 > SIDE_RED_BYTES) break;  // the round's partials fit
        if (force_a > 0 && a != force_a) continue;
        for (int C = 1; C <= SIDE_MAX_C; C *= 2) {
            if (force_c > 0 ? C != force_c : C > n_red) continue;
            const int64_t need = cdiv(n_out, a);
            const int64_t clusters = std::min<int64_t>(need, sms / C);
            if (clusters < 1) continue;
            const int64_t rounds_max = cdiv(need, clusters);
            const int64_t per_cta = cdiv(n_red, C);
            const double us = side_stream_us(double(rounds_max * a * per_cta) * 32768.0, static_cast<int>(clusters * C)) +
                              double(need) * double(d_out) * r * 4.0 / (SIDE_HBM_GBS * 1e3);
            if (us < best_cost * 0.999) {
                best_cost = us;
                best.C = C;
                best.group = a;
                best.n_out = static_cast<int>(n_out);
                best.n_red = static_cast<int>(n_red);
                best.rounds = static_cast<int>(need);
                best.clusters = static_cast<int>(clusters);
                best.per_cta = static_cast<int>(per_cta);
            }
        }
    }
    return best;
}

// The one-pass backward (s.g with dB's partials, then dA) writes one fp32 dB partial per
// round of `group` token blocks: r / (64 * group) of the dY stream's bytes, with group
// at most 64 / r (the landing area), and dA reads them back.  The library takes it up to
// r = 16 (at most an eighth of the stream; at r = 32 the stacked gate + up layer wrote
// 90 MB of partials and ran 41 us slower per step than on the split-K kernels); a plan
// can ask for it up to r = 32, the widest its narrow operands take.
constexpr int SIDE_MAX_R_BWD = SIDE_MAX_R_NARROW;
constexpr int SIDE_DEFAULT_R_BWD = 16;

struct Plan {
    size_t err = 0, ctr = 0, xa = 0, g = 0, part_xa = 0, part_g = 0, part_db = 0, part_da = 0;
    size_t total = 0;
    int64_t n_ctr = 0;
    Split s_xa, s_g, s_db, s_da;
    bool side = false;          // s.xa on the side kernels (r <= 64)
    bool side_bwd = false;      // s.g + dB and dA on the side kernels (r <= 32)
    SidePlan sx, sg, sd;        // s.xa, s.g + dB partials, dA + dB
    bool fwd_tail = true;       // forward main GEMM: cut a partial last wave (along N, or along K below)
    bool fwd_ksplit = false;    // bf16 forward: cut it along K instead, tiles handed over in fp32
    bool dx_ksplit = false;     // bf16 backward: the dX GEMM's last wave cut along K, dA + dB after it
    size_t ks_part = 0, ks_flag = 0;  // K-split hand-over buffers (the end of the workspace)
    int ks_tiles = 0;           // tail tiles they hold
    size_t total_min = 0;       // the workspace without them (the forward then cuts along N)
    int dx_mode = 0;            // 0: dA beside the dX GEMM's last wave unless that wave can be cut
                                // along N (then dA follows); 1: always beside; 2: always after
    int da_force_c = 0;         // dA's cluster size if the plan fixes it
};

// ------------------------------------------------------------------ plan overrides
struct PlanOverride {
    int64_t M, d_in, d_out;
    int r;
    lora_plan_t p;
};
std::mutex g_plan_mu;
std::vector<PlanOverride> g_overrides;
constexpr size_t MAX_OVERRIDES = 256;

bool find_override(int64_t M, int64_t d_in, int64_t d_out, int r, lora_plan_t *out) {
    std::lock_guard<std::mutex> lk(g_plan_mu);
    for (const PlanOverride &o : g_overrides)
        if (o.M == M && o.d_in == d_in && o.d_out == d_out && o.r == r) {
            *out = o.p;
            return true;
        }
    return false;
}

// Split of kb K blocks into `splits` (as even as whole blocks allow).
Split forced_split(int64_t kb, int splits) {
    Split sp;
    const int64_t per = cdiv(kb, std::min<int64_t>(splits, kb));
    sp.per = static_cast<int>(per);
    sp.splits = static_cast<int>(cdiv(kb, per));
    return sp;
}

bool make_plan(int op, int64_t M, int64_t d_in, int64_t d_out, int r, int sms, Plan *pl) {
    const bool bwd = (op == LORA_OP_BWD || op == LORA_OP_BWD_Q4 || op == LORA_OP_BWD_FP8 || op == LORA_OP_BWD_NF4);
    const int64_t mt_tok = cdiv(M, BM), mt_in = cdiv(d_in, BM), mt_out = cdiv(d_out, BM);
    lora_plan_t ov;
    std::memset(&ov, 0, sizeof(ov));
    find_override(M, d_in, d_out, r, &ov);  // all zero (the library's choice) without one
    size_t off = 0;
    pl->err = off;
    off += 256;
    pl->side = ov.side_fwd ? ov.side_fwd == 1 : (r <= SIDE_MAX_R && side_enabled());
    pl->side_bwd = bwd && (ov.side_bwd ? ov.side_bwd == 1 : (r <= SIDE_DEFAULT_R_BWD && side_enabled()));
    pl->fwd_tail = ov.fwd_tail != 2;
    pl->fwd_ksplit = op == LORA_OP_FWD && (ov.fwd_tail == 0 || ov.fwd_tail == 3);
    pl->dx_mode = ov.dx_overlap;
    pl->da_force_c = ov.da_cluster;
    // split-K counters and partials (every s.xa when not on the side kernels; the
    // backward's s.g, dB and dA when not on the side kernels)
    const bool sk_xa = !pl->side, sk_bwd = bwd && !pl->side_bwd;
    pl->s_xa = ov.splitk[0] ? forced_split(cdiv(d_in, BK), ov.splitk[0]) : choose_split(mt_tok, cdiv(d_in, BK), sms);
    pl->s_g = ov.splitk[1] ? forced_split(cdiv(d_out, BK), ov.splitk[1]) : choose_split(mt_tok, cdiv(d_out, BK), sms);
    pl->s_db = ov.splitk[2] ? forced_split(cdiv(M, BK), ov.splitk[2]) : choose_split(mt_out, cdiv(M, BK), sms);
    pl->s_da = ov.splitk[3] ? forced_split(cdiv(M, BK), ov.splitk[3]) : choose_split(mt_in, cdiv(M, BK), sms);
    if (pl->side) pl->sx = side_plan(mt_tok, cdiv(d_in, BK), sms, SIDE_MAX_C, ov.xa_cluster);
    if (pl->side_bwd) {
        pl->sg = side_plan_gdb(M, d_out, r, sms, ov.g_cluster, ov.g_group);
        pl->sd = side_plan(mt_in, mt_tok, sms, SIDE_MAX_C_DA, ov.da_cluster);
    }
    pl->ctr = off;
    pl->n_ctr = (sk_xa || sk_bwd) ? mt_tok * 2 + mt_in + mt_out : 0;
    off = align256(off + pl->n_ctr * sizeof(int));
    pl->xa = off;
    off = align256(off + M * r * 2);
    if (sk_xa) {
        pl->part_xa = off;
        off = align256(off + static_cast<size_t>(pl->s_xa.splits) * mt_tok * BM * r * 4);
    }
    if (bwd) {
        pl->g = off;
        off = align256(off + M * r * 2);
        if (pl->side_bwd) {
            pl->part_db = off;
            off = align256(off + static_cast<size_t>(pl->sg.rounds) * d_out * r * 4);
        } else {
            pl->part_g = off;
            off = align256(off + static_cast<size_t>(pl->s_g.splits) * mt_tok * BM * r * 4);
            pl->part_db = off;
            off = align256(off + static_cast<size_t>(pl->s_db.splits) * mt_out * BM * r * 4);
            pl->part_da = off;
            off = align256(off + static_cast<size_t>(pl->s_da.splits) * mt_in * BM * r * 4);
        }
    }
    pl->total_min = off;
    pl->dx_ksplit = op == LORA_OP_BWD && ov.dx_overlap == 3;
    if (pl->fwd_ksplit || pl->dx_ksplit) {
        // the last wave of the CTA-pair GEMM (256 x 256 tiles on PLAN_SMS / 2 clusters; the
        // forward's N = d_out, K = d_in, dX's N = d_in, K = d_out): K-split when it holds at
        // most half as many tiles as there are clusters and K + r is at least KSPLIT_MIN_KB
        // blocks (half a tile must outweigh the hand-over)
        const int64_t N = pl->fwd_ksplit ? d_out : d_in, K = pl->fwd_ksplit ? d_in : d_out;
        const int64_t C = PLAN_SMS / 2, T = cdiv(M, 256) * cdiv(N, 256), R = T % C;
        if (T >= C && R > 0 && 2 * R <= C && cdiv(K, BK) + cdiv(r, BK) >= KSPLIT_MIN_KB) {
            pl->ks_tiles = static_cast<int>(R);
            pl->ks_flag = off;
            off = align256(off + static_cast<size_t>(R) * 4 * sizeof(int));
            pl->ks_part = off;
            off = align256(off + static_cast<size_t>(R) * 256 * 256 * 4);
        } else {
            pl->fwd_ksplit = pl->dx_ksplit = false;
        }
    }
    pl->total = off;
    return true;
}

// The backward's dA placement: beside the dX GEMM's last wave (true) or after it.  The
// library's choice is beside: cutting the dX GEMM's last wave along N saves half a tile,
// but dA after it then pays a whole launch, ramp and reduction on the critical path
// (measured at the attention projection on one B200: 250 us per fwd+bwd against 234-242
// us with dA hidden in the whole last wave).
bool dx_overlaps(const Plan &pl, int64_t M, int64_t d_in, int pair_clusters, bool coded) {
    (void)M;
    (void)d_in;
    (void)pair_clusters;
    (void)coded;
    return pl.dx_mode != 2 && !pl.dx_ksplit;
}

// ------------------------------------------------------------------ validation
bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// wf: the frozen weight's format (WF_BF16, WF_Q4, WF_FP8).
lora_status_t check_shapes(int64_t M, int64_t d_in, int64_t d_out, int r, float alpha, int wf) {
    if (M < 1 || M > (int64_t(1) << 30)) return LORA_ERR_INVALID_ARG;
    if (d_in < 8 || d_out < 8 || d_in % 8 || d_out % 8) return LORA_ERR_INVALID_ARG;
    if (d_in > (int64_t(1) << 24) || d_out > (int64_t(1) << 24)) return LORA_ERR_INVALID_ARG;
    // Tile counts are 32-bit: bound the 128 x 128 tiles of the larger output (past this
    // bound the larger output alone holds more than 2^45 elements).
    if (((M + 127) / 128) * ((std::max(d_in, d_out) + 127) / 128) > INT32_MAX) return LORA_ERR_INVALID_ARG;
    if (r < 1 || r > 256 || r % 8) return LORA_ERR_INVALID_ARG;
    if (!std::isfinite(alpha)) return LORA_ERR_INVALID_ARG;
    if ((wf == WF_Q4 || wf == WF_CB) && d_in % 64) return LORA_ERR_INVALID_ARG;  // one scale per 64 codes
    if (wf == WF_FP8 && d_in % 16) return LORA_ERR_INVALID_ARG;  // code rows of whole 16-byte units
    return LORA_OK;
}

struct Ctx {
    int dev = 0;
    DevInfo *info = nullptr;
    Plan plan;
    uint8_t *ws = nullptr;
    cudaStream_t st = nullptr;
};

lora_status_t prepare(int op, int64_t M, int64_t d_in, int64_t d_out, int r, void *ws, size_t ws_bytes,
                      void *stream, Ctx *c) {
    if (!device_info(&c->dev, &c->info)) return LORA_ERR_CUDA;
    if (!c->info->supported) return LORA_ERR_UNSUPPORTED;
    make_plan(op, M, d_in, d_out, r, PLAN_SMS, &c->plan);
    if (!ws) return LORA_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(ws) & 255u) return LORA_ERR_MISALIGNED;
    if (ws_bytes < c->plan.total_min) return LORA_ERR_WORKSPACE;
    if (ws_bytes < c->plan.total) c->plan.fwd_ksplit = c->plan.dx_ksplit = false;  // no room for the hand-over
    c->ws = static_cast<uint8_t *>(ws);
    c->st = static_cast<cudaStream_t>(stream);
    return LORA_OK;
}

// ------------------------------------------------------------------ step launchers
GemmArgs base_args(const Ctx &c) {
    GemmArgs a;
    std::memset(&a, 0, sizeof(a));
    a.err = reinterpret_cast<int *>(c.ws + c.plan.err);
    a.group_m = 1;
    return a;
}

// One skinny split-K problem: D [rows, r] over K = kdim, split as `sp`.
SkinnyJob make_job(int r, int64_t rows, int64_t kdim, const Split &sp, float *part, int *ctr, void *out,
                   int out_mode, int64_t out_ld, float scale) {
    SkinnyJob j;
    std::memset(&j, 0, sizeof(j));
    j.m_tiles = static_cast<int>(cdiv(rows, BM));
    j.kb0 = static_cast<int>(cdiv(kdim, BK));
    j.splits = sp.splits;
    j.kb_per_split = sp.per;
    j.num_tiles = j.m_tiles * sp.splits;
    j.rows_valid = static_cast<int>(rows);
    j.n_valid = r;
    j.out_mode = out_mode;
    j.out_scale = scale;
    j.part = part;
    j.counters = ctr;
    j.out = out;
    j.out_ld = out_ld;
    return j;
}

// Launch the skinny split-K kernel over a.job[0 .. a.n_jobs) (tensor maps already set)
// on at most `grid_cap` CTAs.  a_mn / b_mn select the operand majorness.
template <bool A_MN, bool B_MN>
lora_status_t launch_skinny(const Ctx &c, GemmArgs &a, int r, int grid_cap, int kind) {
    a.kb1 = 0;
    a.num_tiles = a.job[0].num_tiles + (a.n_jobs > 1 ? a.job[1].num_tiles : 0);
    const int grid = std::max(1, std::min({a.num_tiles, c.info->sms, grid_cap}));
    cudaError_t e;
    if (!A_MN && !B_MN) {
        switch (bn_class_kmajor(r)) {
            case 16: e = launch_gemm<16, false, false, EPI_SPLITK, skinny_stages<16>()>(a, grid, c.st, c.info, AB_XA16, kind); break;
            case 64: e = launch_gemm<64, false, false, EPI_SPLITK, skinny_stages<64>()>(a, grid, c.st, c.info, AB_XA64, kind); break;
            case 128: e = launch_gemm<128, false, false, EPI_SPLITK, skinny_stages<128>()>(a, grid, c.st, c.info, AB_XA128, kind); break;
            default: e = launch_gemm<256, false, false, EPI_SPLITK, skinny_stages<256>()>(a, grid, c.st, c.info, AB_XA256, kind); break;
        }
    } else if (!A_MN && B_MN) {
        switch (bn_class_mnmajor(r)) {
            case 64: e = launch_gemm<64, false, true, EPI_SPLITK, skinny_stages<64>()>(a, grid, c.st, c.info, AB_G64, kind); break;
            case 128: e = launch_gemm<128, false, true, EPI_SPLITK, skinny_stages<128>()>(a, grid, c.st, c.info, AB_G128, kind); break;
            default: e = launch_gemm<256, false, true, EPI_SPLITK, skinny_stages<256>()>(a, grid, c.st, c.info, AB_G256, kind); break;
        }
    } else {
        switch (bn_class_mnmajor(r)) {
            case 64: e = launch_gemm<64, true, true, EPI_SPLITK, skinny_stages<64>()>(a, grid, c.st, c.info, AB_T64, kind); break;
            case 128: e = launch_gemm<128, true, true, EPI_SPLITK, skinny_stages<128>()>(a, grid, c.st, c.info, AB_T128, kind); break;
            default: e = launch_gemm<256, true, true, EPI_SPLITK, skinny_stages<256>()>(a, grid, c.st, c.info, AB_T256, kind); break;
        }
    }
    return e == cudaSuccess ? LORA_OK : LORA_ERR_CUDA;
}

int *counters_at(const Ctx &c, int64_t offset_tiles) {
    return reinterpret_cast<int *>(c.ws + c.plan.ctr) + offset_tiles;
}

// s.xa = bf16(s . x.A^T) -> dst [M, r]
lora_status_t step_xa(const Ctx &c, const uint16_t *x, const uint16_t *A, uint16_t *dst, int64_t M, int64_t d_in,
                      int r, float s) {
    GemmArgs a = base_args(c);
    const int bn = bn_class_kmajor(r);
    if (!tmap_bf16(&a.tmA0, x, d_in, M, 64, 128)) return LORA_ERR_CUDA;
    if (!tmap_bf16(&a.tmB0, A, d_in, r, 64, bn)) return LORA_ERR_CUDA;
    a.n_jobs = 1;
    a.job[0] = make_job(r, M, d_in, c.plan.s_xa, reinterpret_cast<float *>(c.ws + c.plan.part_xa), counters_at(c, 0),
                        dst, OUT_BF16_ROWS, 0, s);
    return launch_skinny<false, false>(c, a, r, PLAN_SMS, LORA_K_XA);
}

// s.g = bf16(s . dY.B) -> ws g [M, r]; B [d_out, r] is read MN-major (r contiguous).
lora_status_t step_g(const Ctx &c, const uint16_t *dY, const uint16_t *B, int64_t M, int64_t d_out, int r, float s) {
    GemmArgs a = base_args(c);
    if (!tmap_bf16(&a.tmA0, dY, d_out, M, 64, 128)) return LORA_ERR_CUDA;
    if (!tmap_bf16(&a.tmB0, B, r, d_out, 64, 64)) return LORA_ERR_CUDA;
    a.n_jobs = 1;
    a.job[0] = make_job(r, M, d_out, c.plan.s_g, reinterpret_cast<float *>(c.ws + c.plan.part_g),
                        counters_at(c, cdiv(M, BM)), c.ws + c.plan.g, OUT_BF16_ROWS, 0, s);
    return launch_skinny<false, true>(c, a, r, PLAN_SMS, LORA_K_G);
}

// The two weight gradients in one launch, both split over tokens with MN-major operands:
//   job 0: dB [d_out, r] = dY^T . (s.xa)
//   job 1: dA [r, d_in]  = (s.g)^T . x, computed as its transpose (M-dim = d_in), stored transposed.
// `defer`: launched right after the dX GEMM, whose outputs it does not read, so it may
// run on the SMs that GEMM's last wave leaves idle (`grid_cap` CTAs).
lora_status_t step_dadb(const Ctx &c, const uint16_t *dY, const uint16_t *x, const uint16_t *sxa,
                        const uint16_t *sg, float *dA, float *dB, int64_t M, int64_t d_in, int64_t d_out, int r,
                        bool defer, int grid_cap) {
    GemmArgs a = base_args(c);
    a.defer_dep_wait = defer ? 1 : 0;
    if (!tmap_bf16(&a.tmA0, dY, d_out, M, 64, 64)) return LORA_ERR_CUDA;
    if (!tmap_bf16(&a.tmB0, sxa, r, M, 64, 64)) return LORA_ERR_CUDA;
    if (!tmap_bf16(&a.tmA1, x, d_in, M, 64, 64)) return LORA_ERR_CUDA;
    if (!tmap_bf16(&a.tmB1, sg, r, M, 64, 64)) return LORA_ERR_CUDA;
    a.n_jobs = 2;
    a.job[0] = make_job(r, d_out, M, c.plan.s_db, reinterpret_cast<float *>(c.ws + c.plan.part_db),
                        counters_at(c, 2 * cdiv(M, BM)), dB, OUT_F32_ROWS, 0, 1.0f);
    a.job[1] = make_job(r, d_in, M, c.plan.s_da, reinterpret_cast<float *>(c.ws + c.plan.part_da),
                        counters_at(c, 2 * cdiv(M, BM) + cdiv(d_out, BM)), dA, OUT_F32_COLS, d_in, 1.0f);
    return launch_skinny<true, true>(c, a, r, grid_cap, LORA_K_DADB);
}

// ------------------------------------------------------------------ side kernels (r <= 64)
SideArgs side_args(const Ctx &c) {
    SideArgs a;
    std::memset(&a, 0, sizeof(a));
    a.err = reinterpret_cast<int *>(c.ws + c.plan.err);
    a.group = 1;
    return a;
}

void side_fill(SideArgs &a, const SidePlan &sp, int r) {
    a.r = r;
    a.n_out = sp.n_out;
    a.n_red = sp.n_red;
    a.per_cta = sp.per_cta;
    a.group = sp.group;
    a.n_rounds = sp.rounds;
}

// s.xa = bf16(s . x.A^T) -> dst [M, r]
lora_status_t side_xa(const Ctx &c, const uint16_t *x, const uint16_t *A, uint16_t *dst, int64_t M, int64_t d_in,
                      int r, float s) {
    const SidePlan &sp = c.plan.sx;
    SideArgs a = side_args(c);
    side_fill(a, sp, r);
    a.nr = (r + 15) / 16 * 16;
    if (!tmap_bf16(&a.tmX, x, d_in, M, 64, 128)) return LORA_ERR_CUDA;
    if (!tmap_bf16(&a.tmS0, A, d_in, r, 64, a.nr)) return LORA_ERR_CUDA;
    a.rows_valid = static_cast<int>(M);
    a.scale = s;
    a.out_bf16 = dst;
    const cudaError_t e =
        launch_side<SIDE_XA, SIDE_XA_STAGES>(a, sp.clusters, sp.C, c.st, c.info, AB_SIDE_XA, LORA_K_XA);
    return e == cudaSuccess ? LORA_OK : LORA_ERR_CUDA;
}

// MN-major narrow operand [rows][r] of the s.g + dB and dA kernels: box {nb, 128} with
// the swizzle whose span is nb bf16 (32 bytes for nb = 16, 64 bytes for nb = 32).
bool tmap_narrow(CUtensorMap *m, const void *base, int r, int64_t rows, int nb) {
    return lora_host::tmap_2d(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, r, rows, nb, 128,
                              nb == 16 ? CU_TENSOR_MAP_SWIZZLE_32B : CU_TENSOR_MAP_SWIZZLE_64B);
}
int narrow_n(int r) { return r <= 16 ? 16 : 32; }

// One pass over dY: s.g = bf16(s . dY.B) -> ws g [M, r], and dB's partials over each
// round's tokens -> ws [rounds][d_out][r].  B [d_out, r] and s.xa [M, r] are read MN-major.
lora_status_t side_gdb(const Ctx &c, const uint16_t *dY, const uint16_t *B, const uint16_t *sxa, int64_t M,
                       int64_t d_out, int r, float s) {
    const SidePlan &sp = c.plan.sg;
    SideArgs a = side_args(c);
    side_fill(a, sp, r);
    a.nb = narrow_n(r);
    if (!tmap_bf16(&a.tmX, dY, d_out, M, 64, 128)) return LORA_ERR_CUDA;
    if (!tmap_narrow(&a.tmS0, B, r, d_out, a.nb)) return LORA_ERR_CUDA;
    if (!tmap_narrow(&a.tmS1, sxa, r, M, a.nb)) return LORA_ERR_CUDA;
    a.rows_valid = static_cast<int>(M);
    a.scale = s;
    a.out_bf16 = reinterpret_cast<uint16_t *>(c.ws + c.plan.g);
    a.db_part = reinterpret_cast<float *>(c.ws + c.plan.part_db);
    a.d_out = static_cast<int>(d_out);
    const cudaError_t e =
        launch_side<SIDE_GDB, SIDE_GDB_STAGES>(a, sp.clusters, sp.C, c.st, c.info, AB_SIDE_GDB, LORA_K_G);
    return e == cudaSuccess ? LORA_OK : LORA_ERR_CUDA;
}

// dA [r, d_in] = ((s.g)^T . x), and dB [d_out, r] = the sum of the partials.  `defer`:
// launched right after the dX GEMM, whose outputs it does not read, so it starts on the
// SMs that GEMM's last wave leaves idle; `grid_cap` bounds its CTAs.
lora_status_t side_da(const Ctx &c, const uint16_t *x, const uint16_t *sg, float *dA, float *dB, int64_t M,
                      int64_t d_in, int64_t d_out, int r, bool defer, int grid_cap, int max_c) {
    const SidePlan sp = side_plan(c.plan.sd.n_out, c.plan.sd.n_red, PLAN_SMS, max_c, c.plan.da_force_c);
    SideArgs a = side_args(c);
    side_fill(a, sp, r);
    a.defer_dep_wait = defer ? 1 : 0;
    a.nb = narrow_n(r);
    if (!tmap_bf16(&a.tmX, x, d_in, M, 64, 128)) return LORA_ERR_CUDA;
    if (!tmap_narrow(&a.tmS0, sg, r, M, a.nb)) return LORA_ERR_CUDA;
    a.rows_valid = static_cast<int>(d_in);
    a.out_f32 = dA;
    a.db_part = reinterpret_cast<float *>(c.ws + c.plan.part_db);
    a.d_out = static_cast<int>(d_out);
    a.dB = dB;
    a.db_rounds = c.plan.sg.rounds;
    const int clusters = std::max(1, std::min(sp.clusters, grid_cap / sp.C));
    const cudaError_t e =
        launch_side<SIDE_DA, SIDE_DA_STAGES>(a, clusters, sp.C, c.st, c.info, AB_SIDE_DA, LORA_K_DADB);
    return e == cudaSuccess ? LORA_OK : LORA_ERR_CUDA;
}

// Main K-concatenated GEMM: out [M, N] = A0 . B0^T (K0) + A1 . B1^T (K1 = r).
//   A0 [M, K0], A1 [M, r]: K-major bf16.
//   B0, B1: K-major [N, K] (forward: W, B) or MN-major [K, N] (dX: W, A).
struct MainOperands {
    const void *A0, *B0, *A1, *B1;
    void *C;
    const uint8_t *Wq = nullptr;       // 4-bit or FP8 frozen weight's codes (B0 is then unused)
    const uint16_t *Wscale = nullptr;  // its bf16 scales: [d_out, d_in / 64] (4-bit) or [d_out] (FP8)
    int64_t q_rows = 0, q_cols = 0;    // W shape [d_out, d_in]
    int wf = WF_BF16;
    const float *codebook = nullptr;   // 4-bit codebook weight: its 16 values (host)
};

// `idle_sms` (optional) receives how many SMs the last wave leaves without work.
// `ksplit`: cut a partial last wave along K (bf16 weight, workspace permitting) rather
// than along N.
lora_status_t step_main(const Ctx &c, const MainOperands &o, int64_t M, int64_t N, int64_t K0, int r, bool b_mn,
                        int kind, bool allow_tail_split, int *idle_sms = nullptr, bool ksplit = false) {
    GemmArgs a = base_args(c);
    a.kb0 = static_cast<int>(cdiv(K0, BK));
    a.kb1 = static_cast<int>(cdiv(r, BK));
    a.mma_last1 = static_cast<int>(cdiv(r - (a.kb1 - 1) * BK, 16));
    if (!tmap_bf16(&a.tmA0, o.A0, K0, M, 64, 128)) return LORA_ERR_CUDA;
    if (!tmap_bf16(&a.tmA1, o.A1, r, M, 64, 128)) return LORA_ERR_CUDA;
    if (!tmap_bf16(&a.tmC, o.C, N, M, 64, 32)) return LORA_ERR_CUDA;
    const bool q4 = o.wf != WF_BF16;  // codes decoded in shared memory (4-bit or FP8)
    const int pair_C = pair_enabled() ? std::min(pair_clusters(c.info, b_mn, o.wf), PLAN_SMS / 2) : 0;
    if (q4 && pair_C == 0) return LORA_ERR_UNSUPPORTED;  // decoded weights run on CTA pairs only
    if (q4) {
        a.wscale = o.Wscale;
        a.scale_ld = o.wf == WF_FP8 ? 1 : static_cast<int>(o.q_cols / 64);
        if (o.wf == WF_CB)
            for (int i = 0; i < 16; ++i) a.cb[i] = o.codebook[i];
        a.scale_rows = static_cast<int>(o.q_rows);
        // codes [d_out][d_in / 2] (4-bit) or [d_out][d_in] (FP8) bytes; each dequant warp
        // fetches dq_qrows rows x the bytes of 64 codes at a time
        const int rb = dq_run_bytes(o.wf);
        if (!tmap_u8(&a.tmQ, o.Wq, o.q_cols * rb / 64, o.q_rows, rb, dq_qrows(o.wf))) return LORA_ERR_CUDA;
        allow_tail_split = false;
    }
    if (pair_C > 0) {
        // CTA pairs: 256 x 256 tiles, each CTA stages 128 rows of B.
        const int64_t T = cdiv(M, PAIR_BM) * cdiv(N, PAIR_BN);
        a.m_tiles = static_cast<int>(cdiv(M, PAIR_BM));
        a.n_tiles = static_cast<int>(cdiv(N, PAIR_BN));
        a.num_tiles = static_cast<int>(T);
        a.group_m = std::min(a.m_tiles, 8);
        const int64_t W = T / pair_C, R = T % pair_C;
        const bool kcut = ksplit && !q4 && W >= 1 && R > 0 && 2 * R <= pair_C && R <= c.plan.ks_tiles;
        const bool split = !kcut && allow_tail_split && W >= 1 && R > 0 && 2 * R <= pair_C;
        a.dp_tiles = static_cast<int>(split || kcut ? W * pair_C : T);
        a.dp_waves = static_cast<int>(split || kcut ? W : cdiv(T, pair_C));
        a.tail_tiles = static_cast<int>(split || kcut ? R : 0);
        a.tail_split = split ? 2 : 1;
        if (kcut) {
            a.tail_ksplit = 1;
            a.ks_part = reinterpret_cast<float *>(c.ws + c.plan.ks_part);
            a.ks_flag = reinterpret_cast<int *>(c.ws + c.plan.ks_flag);
        }
        if (b_mn) {
            // bf16 weight: the 3D column-chunk map when N is a multiple of 64 (one copy per
            // CTA and K block; two 2D copies cost ~7% of the dX GEMM at 4096 x 4096)
            a.b3d = !q4 && N % 64 == 0 ? 1 : 0;
            if (a.b3d) {
                // 3D map for whole tiles, 2D map for the 64-column halves of split tail tiles
                if (!lora_host::tmap_mn_chunks(&a.tmB0, o.B0, N, K0)) return LORA_ERR_CUDA;
                if (!tmap_bf16(&a.tmB0n, o.B0, N, K0, 64, 64)) return LORA_ERR_CUDA;
            } else if (!q4 && !tmap_bf16(&a.tmB0, o.B0, N, K0, 64, 64)) {
                return LORA_ERR_CUDA;
            }
            if (!tmap_bf16(&a.tmB1, o.B1, N, r, 64, 64)) return LORA_ERR_CUDA;
        } else {
            if (!q4 && !tmap_bf16(&a.tmB0, o.B0, K0, N, 64, CTA_BN)) return LORA_ERR_CUDA;
            if (!tmap_bf16(&a.tmB1, o.B1, r, N, 64, CTA_BN)) return LORA_ERR_CUDA;
            if (split) {
                if (!tmap_bf16(&a.tmB0n, o.B0, K0, N, 64, CTA_BN / 2)) return LORA_ERR_CUDA;
                if (!tmap_bf16(&a.tmB1n, o.B1, r, N, 64, CTA_BN / 2)) return LORA_ERR_CUDA;
            }
        }
        const int clusters = split || kcut ? pair_C : static_cast<int>(std::min<int64_t>(T, pair_C));
        if (idle_sms) *idle_sms = (!split && R > 0 && W >= 1) ? c.info->sms - static_cast<int>(2 * R) : 0;
        cudaError_t e;
        if (o.wf == WF_Q4)
            e = b_mn ? launch_pair<true, WF_Q4>(a, 2 * clusters, c.st, c.info, AB_PAIR_MN_Q4, kind)
                     : launch_pair<false, WF_Q4>(a, 2 * clusters, c.st, c.info, AB_PAIR_K_Q4, kind);
        else if (o.wf == WF_FP8)
            e = b_mn ? launch_pair<true, WF_FP8>(a, 2 * clusters, c.st, c.info, AB_PAIR_MN_FP8, kind)
                     : launch_pair<false, WF_FP8>(a, 2 * clusters, c.st, c.info, AB_PAIR_K_FP8, kind);
        else if (o.wf == WF_CB)
            e = b_mn ? launch_pair<true, WF_CB>(a, 2 * clusters, c.st, c.info, AB_PAIR_MN_CB, kind)
                     : launch_pair<false, WF_CB>(a, 2 * clusters, c.st, c.info, AB_PAIR_K_CB, kind);
        else
            e = b_mn ? launch_pair<true, WF_BF16>(a, 2 * clusters, c.st, c.info, AB_PAIR_MN, kind)
                     : launch_pair<false, WF_BF16>(a, 2 * clusters, c.st, c.info, AB_PAIR_K, kind);
        return e == cudaSuccess ? LORA_OK : LORA_ERR_CUDA;
    }
    // Single-SM kernel: 128 x 256 tiles.
    a.m_tiles = static_cast<int>(cdiv(M, BM));
    a.n_tiles = static_cast<int>(cdiv(N, MAIN_BN));
    a.num_tiles = a.m_tiles * a.n_tiles;
    a.group_m = std::min(a.m_tiles, 16);
    const int G = std::min(c.info->sms, PLAN_SMS);
    MainSched ms = main_sched(M, N, G);
    if (!allow_tail_split && ms.tail_split > 1) {
        ms.dp_tiles = ms.tiles;
        ms.dp_waves = static_cast<int>(cdiv(ms.tiles, G));
        ms.tail_tiles = 0;
        ms.tail_split = 1;
    }
    a.dp_tiles = ms.dp_tiles;
    a.dp_waves = ms.dp_waves;
    a.tail_tiles = ms.tail_tiles;
    a.tail_split = ms.tail_split;
    if (b_mn) {
        if (!tmap_bf16(&a.tmB0, o.B0, N, K0, 64, 64)) return LORA_ERR_CUDA;
        if (!tmap_bf16(&a.tmB1, o.B1, N, r, 64, 64)) return LORA_ERR_CUDA;
    } else {
        if (!tmap_bf16(&a.tmB0, o.B0, K0, N, 64, MAIN_BN)) return LORA_ERR_CUDA;
        if (!tmap_bf16(&a.tmB1, o.B1, r, N, 64, MAIN_BN)) return LORA_ERR_CUDA;
        if (ms.tail_split > 1) {
            const uint32_t rows = MAIN_BN / ms.tail_split;
            if (!tmap_bf16(&a.tmB0n, o.B0, K0, N, 64, rows)) return LORA_ERR_CUDA;
            if (!tmap_bf16(&a.tmB1n, o.B1, r, N, 64, rows)) return LORA_ERR_CUDA;
        }
    }
    const int grid = ms.tail_split > 1 ? G : std::min(a.num_tiles, G);
    if (idle_sms) {
        const int rem = ms.tiles % G;
        *idle_sms = (ms.tail_split == 1 && rem > 0 && ms.tiles >= G) ? c.info->sms - rem : 0;
    }
    cudaError_t e;
    if (b_mn)
        e = launch_gemm<MAIN_BN, false, true, EPI_STORE, MAIN_STAGES>(a, grid, c.st, c.info, AB_DX, kind);
    else
        e = launch_gemm<MAIN_BN, false, false, EPI_STORE, MAIN_STAGES>(a, grid, c.st, c.info, AB_FWD, kind);
    return e == cudaSuccess ? LORA_OK : LORA_ERR_CUDA;
}

#define LORA_TRY(x)                          \
    do {                                     \
        lora_status_t _s = (x);              \
        if (_s != LORA_OK) return _s;        \
    } while (0)

// The frozen weight: bf16 W [d_out, d_in], or 4-bit codes Wq [d_out, d_in / 2] with bf16
// scales Wscale [d_out, d_in / 64] (dequantised in shared memory inside the GEMMs).
struct Weight {
    const uint16_t *W = nullptr;
    const uint8_t *Wq = nullptr;       // 4-bit or FP8 codes
    const uint16_t *Wscale = nullptr;
    int wf = WF_BF16;
    const float *codebook = nullptr;   // WF_CB: 16 values (host memory)
    bool coded() const { return wf != WF_BF16; }
    bool present() const { return coded() ? (Wq && Wscale && (wf != WF_CB || codebook)) : W != nullptr; }
    bool aligned() const { return coded() ? (aligned16(Wq) && aligned16(Wscale)) : aligned16(W); }
    int op_fwd() const {
        return wf == WF_Q4 ? LORA_OP_FWD_Q4 : wf == WF_FP8 ? LORA_OP_FWD_FP8 : wf == WF_CB ? LORA_OP_FWD_NF4 : LORA_OP_FWD;
    }
    int op_bwd() const {
        return wf == WF_Q4 ? LORA_OP_BWD_Q4 : wf == WF_FP8 ? LORA_OP_BWD_FP8 : wf == WF_CB ? LORA_OP_BWD_NF4 : LORA_OP_BWD;
    }
};

MainOperands main_operands(const Weight &wt, const void *A0, const void *A1, const void *B1, void *C,
                           int64_t d_out, int64_t d_in) {
    MainOperands o{A0, wt.W, A1, B1, C};
    if (wt.coded()) {
        o.Wq = wt.Wq;
        o.Wscale = wt.Wscale;
        o.wf = wt.wf;
        o.codebook = wt.codebook;
        o.q_rows = d_out;
        o.q_cols = d_in;
    }
    return o;
}

lora_status_t fwd_impl(const uint16_t *x, const Weight &wt, const uint16_t *A, const uint16_t *B, uint16_t *h,
                       uint16_t *xa_save, int64_t M, int64_t d_in, int64_t d_out, int r, float alpha, void *ws,
                       size_t ws_bytes, void *stream) {
    LORA_TRY(check_shapes(M, d_in, d_out, r, alpha, wt.wf));
    if (!x || !wt.present() || !A || !B || !h) return LORA_ERR_INVALID_ARG;
    if (wt.wf == WF_CB)
        for (int i = 0; i < 16; ++i)
            if (!std::isfinite(wt.codebook[i])) return LORA_ERR_INVALID_ARG;
    if (!aligned16(x) || !wt.aligned() || !aligned16(A) || !aligned16(B) || !aligned16(h) ||
        (xa_save && !aligned16(xa_save)))
        return LORA_ERR_MISALIGNED;
    Ctx c;
    LORA_TRY(prepare(wt.op_fwd(), M, d_in, d_out, r, ws, ws_bytes, stream, &c));
    const float s = alpha / static_cast<float>(r);
    uint16_t *sxa = xa_save ? xa_save : reinterpret_cast<uint16_t *>(c.ws + c.plan.xa);
    LORA_TRY(c.plan.side ? side_xa(c, x, A, sxa, M, d_in, r, s) : step_xa(c, x, A, sxa, M, d_in, r, s));
    const MainOperands o = main_operands(wt, x, sxa, B, h, d_out, d_in);
    return step_main(c, o, M, d_out, d_in, r, false, LORA_K_FWD_MAIN, c.plan.fwd_tail, nullptr, c.plan.fwd_ksplit);
}

lora_status_t bwd_impl(const uint16_t *dY, const uint16_t *x, const Weight &wt, const uint16_t *A,
                       const uint16_t *B, const uint16_t *xa_save, uint16_t *dX, float *dA, float *dB, int64_t M,
                       int64_t d_in, int64_t d_out, int r, float alpha, void *ws, size_t ws_bytes, void *stream) {
    LORA_TRY(check_shapes(M, d_in, d_out, r, alpha, wt.wf));
    if (!dY || !x || !wt.present() || !A || !B || !dA || !dB) return LORA_ERR_INVALID_ARG;
    if (wt.wf == WF_CB)
        for (int i = 0; i < 16; ++i)
            if (!std::isfinite(wt.codebook[i])) return LORA_ERR_INVALID_ARG;
    if (!aligned16(dY) || !aligned16(x) || !wt.aligned() || !aligned16(A) || !aligned16(B) || !aligned16(dA) ||
        !aligned16(dB) || (xa_save && !aligned16(xa_save)) || (dX && !aligned16(dX)))
        return LORA_ERR_MISALIGNED;
    Ctx c;
    LORA_TRY(prepare(wt.op_bwd(), M, d_in, d_out, r, ws, ws_bytes, stream, &c));
    const float s = alpha / static_cast<float>(r);
    const uint16_t *sxa = xa_save;
    if (!sxa) {
        uint16_t *tmp = reinterpret_cast<uint16_t *>(c.ws + c.plan.xa);
        LORA_TRY(c.plan.side ? side_xa(c, x, A, tmp, M, d_in, r, s) : step_xa(c, x, A, tmp, M, d_in, r, s));
        sxa = tmp;
    }
    if (c.plan.side_bwd)
        LORA_TRY(side_gdb(c, dY, B, sxa, M, d_out, r, s));
    else
        LORA_TRY(step_g(c, dY, B, M, d_out, r, s));
    const uint16_t *sg = reinterpret_cast<const uint16_t *>(c.ws + c.plan.g);
    // dA (and dB) read nothing the dX GEMM writes: launched after it (programmatic
    // dependent launch), they start on the SMs its last wave leaves idle and wait for
    // it only before they exit.  The dX tail is then left whole (no narrow tiles) so
    // those SMs free up early.
    const int dx_pairs = dX ? std::min(pair_clusters(c.info, true, wt.wf), PLAN_SMS / 2) : 0;
    const bool overlap = dX != nullptr && pdl_enabled() && dx_overlaps(c.plan, M, d_in, dx_pairs, wt.coded());
    int idle = 0;
    if (dX) {
        // W [d_out, d_in] (or its codes) and A [r, d_in] are read MN-major (d_in contiguous).
        const MainOperands o = main_operands(wt, dY, sg, A, dX, d_out, d_in);
        LORA_TRY(step_main(c, o, M, d_in, d_out, r, true, LORA_K_DX_MAIN, !overlap, &idle, c.plan.dx_ksplit));
    }
    if (c.plan.side_bwd) {
        // dA reads nothing the dX GEMM writes, so it waits for that GEMM only before it
        // exits and its CTAs take SMs as they free up.  Beside a whole last wave: pairs on
        // that wave's idle SMs when there are enough of them to be worth a cluster grid;
        // otherwise (and after a last wave cut along N) every SM, in clusters of up to 4.
        const bool defer = dX != nullptr && pdl_enabled();
        const int cap = (overlap && idle >= 32) ? idle : PLAN_SMS;
        LORA_TRY(side_da(c, x, sg, dA, dB, M, d_in, d_out, r, defer, cap, overlap ? SIDE_MAX_C_DA : SIDE_MAX_C));
        return LORA_OK;
    }
    // Grid: the idle SMs when they can take all the dB / dA split tiles within about
    // four each (they then finish close to the dX GEMM); otherwise every SM, the rest of
    // the CTAs starting as the dX CTAs exit (at M = 16384 only 24 SMs are idle, and 256
    // tiles on 24 CTAs took 255 us where the full grid takes 72 us).
    const int64_t dadb_tiles = cdiv(d_out, BM) * c.plan.s_db.splits + cdiv(d_in, BM) * c.plan.s_da.splits;
    const bool few = overlap && idle >= 16 && dadb_tiles <= 4 * static_cast<int64_t>(idle);
    LORA_TRY(step_dadb(c, dY, x, sxa, sg, dA, dB, M, d_in, d_out, r, overlap, few ? idle : PLAN_SMS));
    return LORA_OK;
}

}  // namespace

// ====================================================================== C ABI
extern "C" {

// The smallest workspace the operation runs in (the bf16 forward without its K-split
// hand-over buffer); 0 for invalid arguments.  Used by the workspace-free forward.
size_t lora_workspace_min(int op, int64_t M, int64_t d_in, int64_t d_out, int r) {
    if (op < LORA_OP_FWD || op > LORA_OP_BWD_NF4) return 0;
    const int wf = op >= LORA_OP_FWD_NF4 ? WF_CB : op >= LORA_OP_FWD_FP8 ? WF_FP8 : op >= LORA_OP_FWD_Q4 ? WF_Q4 : WF_BF16;
    if (check_shapes(M, d_in, d_out, r, 1.0f, wf) != LORA_OK) return 0;
    Plan pl;
    make_plan(op, M, d_in, d_out, r, PLAN_SMS, &pl);
    return pl.total_min;
}

size_t lora_linear_workspace_size(int op, int64_t M, int64_t d_in, int64_t d_out, int r) {
    if (op < LORA_OP_FWD || op > LORA_OP_BWD_NF4) return 0;
    const int wf = op >= LORA_OP_FWD_NF4 ? WF_CB : op >= LORA_OP_FWD_FP8 ? WF_FP8 : op >= LORA_OP_FWD_Q4 ? WF_Q4 : WF_BF16;
    if (check_shapes(M, d_in, d_out, r, 1.0f, wf) != LORA_OK) return 0;
    Plan pl;
    make_plan(op, M, d_in, d_out, r, PLAN_SMS, &pl);
    return pl.total;
}

lora_status_t lora_linear_fwd(const uint16_t *x, const uint16_t *W, const uint16_t *A, const uint16_t *B, uint16_t *h,
                              uint16_t *xa_save, int64_t M, int64_t d_in, int64_t d_out, int r, float alpha,
                              void *workspace, size_t workspace_bytes, void *stream) {
    Weight wt;
    wt.W = W;
    return fwd_impl(x, wt, A, B, h, xa_save, M, d_in, d_out, r, alpha, workspace, workspace_bytes, stream);
}

lora_status_t lora_linear_bwd(const uint16_t *dY, const uint16_t *x, const uint16_t *W, const uint16_t *A,
                              const uint16_t *B, const uint16_t *xa_save, uint16_t *dX, float *dA, float *dB,
                              int64_t M, int64_t d_in, int64_t d_out, int r, float alpha, void *workspace,
                              size_t workspace_bytes, void *stream) {
    Weight wt;
    wt.W = W;
    return bwd_impl(dY, x, wt, A, B, xa_save, dX, dA, dB, M, d_in, d_out, r, alpha, workspace, workspace_bytes,
                    stream);
}

lora_status_t lora_linear_fwd_q4(const uint16_t *x, const uint8_t *Wq, const uint16_t *Wscale, const uint16_t *A,
                                 const uint16_t *B, uint16_t *h, uint16_t *xa_save, int64_t M, int64_t d_in,
                                 int64_t d_out, int r, float alpha, void *workspace, size_t workspace_bytes,
                                 void *stream) {
    Weight wt;
    wt.Wq = Wq;
    wt.Wscale = Wscale;
    wt.wf = WF_Q4;
    if (!Wq || !Wscale) return LORA_ERR_INVALID_ARG;
    return fwd_impl(x, wt, A, B, h, xa_save, M, d_in, d_out, r, alpha, workspace, workspace_bytes, stream);
}

lora_status_t lora_linear_bwd_q4(const uint16_t *dY, const uint16_t *x, const uint8_t *Wq, const uint16_t *Wscale,
                                 const uint16_t *A, const uint16_t *B, const uint16_t *xa_save, uint16_t *dX,
                                 float *dA, float *dB, int64_t M, int64_t d_in, int64_t d_out, int r, float alpha,
                                 void *workspace, size_t workspace_bytes, void *stream) {
    Weight wt;
    wt.Wq = Wq;
    wt.Wscale = Wscale;
    wt.wf = WF_Q4;
    if (!Wq || !Wscale) return LORA_ERR_INVALID_ARG;
    return bwd_impl(dY, x, wt, A, B, xa_save, dX, dA, dB, M, d_in, d_out, r, alpha, workspace, workspace_bytes,
                    stream);
}

lora_status_t lora_linear_fwd_fp8(const uint16_t *x, const uint8_t *W8, const uint16_t *W8scale, const uint16_t *A,
                                  const uint16_t *B, uint16_t *h, uint16_t *xa_save, int64_t M, int64_t d_in,
                                  int64_t d_out, int r, float alpha, void *workspace, size_t workspace_bytes,
                                  void *stream) {
    Weight wt;
    wt.Wq = W8;
    wt.Wscale = W8scale;
    wt.wf = WF_FP8;
    if (!W8 || !W8scale) return LORA_ERR_INVALID_ARG;
    return fwd_impl(x, wt, A, B, h, xa_save, M, d_in, d_out, r, alpha, workspace, workspace_bytes, stream);
}

lora_status_t lora_linear_bwd_fp8(const uint16_t *dY, const uint16_t *x, const uint8_t *W8, const uint16_t *W8scale,
                                  const uint16_t *A, const uint16_t *B, const uint16_t *xa_save, uint16_t *dX,
                                  float *dA, float *dB, int64_t M, int64_t d_in, int64_t d_out, int r, float alpha,
                                  void *workspace, size_t workspace_bytes, void *stream) {
    Weight wt;
    wt.Wq = W8;
    wt.Wscale = W8scale;
    wt.wf = WF_FP8;
    if (!W8 || !W8scale) return LORA_ERR_INVALID_ARG;
    return bwd_impl(dY, x, wt, A, B, xa_save, dX, dA, dB, M, d_in, d_out, r, alpha, workspace, workspace_bytes,
                    stream);
}

lora_status_t lora_linear_set_plan(int64_t M, int64_t d_in, int64_t d_out, int r, const lora_plan_t *plan) {
    if (check_shapes(M, d_in, d_out, r, 1.0f, WF_BF16) != LORA_OK) return LORA_ERR_INVALID_ARG;
    if (plan) {
        const lora_plan_t &q = *plan;
        auto in = [](int32_t v, std::initializer_list<int32_t> ok) {
            for (int32_t o : ok)
                if (v == o) return true;
            return false;
        };
        if (!in(q.side_fwd, {0, 1, 2}) || !in(q.side_bwd, {0, 1, 2}) || !in(q.xa_cluster, {0, 1, 2, 4}) ||
            !in(q.g_cluster, {0, 1, 2, 4}) || q.g_group < 0 || q.g_group > 6 || !in(q.da_cluster, {0, 1, 2, 4}) ||
            !in(q.fwd_tail, {0, 1, 2, 3}) || !in(q.dx_overlap, {0, 1, 2, 3}))
            return LORA_ERR_INVALID_ARG;
        for (int i = 0; i < 4; ++i)
            if (q.splitk[i] < 0 || q.splitk[i] > 64) return LORA_ERR_INVALID_ARG;
        if (q.side_fwd == 1 && r > SIDE_MAX_R) return LORA_ERR_UNSUPPORTED;
        if (q.side_bwd == 1 && r > SIDE_MAX_R_BWD) return LORA_ERR_UNSUPPORTED;
        if (q.g_group > 0 && q.g_group * r > SIDE_RED_BYTES / (128 * 4)) return LORA_ERR_UNSUPPORTED;
    }
    std::lock_guard<std::mutex> lk(g_plan_mu);
    for (size_t i = 0; i < g_overrides.size(); ++i)
        if (g_overrides[i].M == M && g_overrides[i].d_in == d_in && g_overrides[i].d_out == d_out &&
            g_overrides[i].r == r) {
            if (plan)
                g_overrides[i].p = *plan;
            else
                g_overrides.erase(g_overrides.begin() + static_cast<std::ptrdiff_t>(i));
            return LORA_OK;
        }
    if (!plan) return LORA_OK;
    if (g_overrides.size() >= MAX_OVERRIDES) return LORA_ERR_UNSUPPORTED;
    g_overrides.push_back({M, d_in, d_out, r, *plan});
    return LORA_OK;
}

lora_status_t lora_linear_get_plan(int op, int64_t M, int64_t d_in, int64_t d_out, int r, lora_plan_t *plan) {
    if (!plan || op < LORA_OP_FWD || op > LORA_OP_BWD_NF4) return LORA_ERR_INVALID_ARG;
    const int wf = op >= LORA_OP_FWD_NF4 ? WF_CB : op >= LORA_OP_FWD_FP8 ? WF_FP8 : op >= LORA_OP_FWD_Q4 ? WF_Q4 : WF_BF16;
    if (check_shapes(M, d_in, d_out, r, 1.0f, wf) != LORA_OK) return LORA_ERR_INVALID_ARG;
    Plan pl;
    make_plan(op, M, d_in, d_out, r, PLAN_SMS, &pl);
    std::memset(plan, 0, sizeof(*plan));
    const bool bwd = (op == LORA_OP_BWD || op == LORA_OP_BWD_Q4 || op == LORA_OP_BWD_FP8 || op == LORA_OP_BWD_NF4);
    plan->side_fwd = pl.side ? 1 : 2;
    plan->side_bwd = bwd ? (pl.side_bwd ? 1 : 2) : 0;
    plan->xa_cluster = pl.side ? pl.sx.C : 0;
    plan->g_cluster = pl.side_bwd ? pl.sg.C : 0;
    plan->g_group = pl.side_bwd ? pl.sg.group : 0;
    const bool coded = wf != WF_BF16;
    const bool overlap = dx_overlaps(pl, M, d_in, PLAN_SMS / 2, coded);
    plan->da_cluster = pl.side_bwd ? side_plan(pl.sd.n_out, pl.sd.n_red, PLAN_SMS,
                                               overlap ? SIDE_MAX_C_DA : SIDE_MAX_C, pl.da_force_c).C
                                   : 0;
    Plan fp;  // the forward of the same weight format (a backward plan reports the forward's tail)
    make_plan(op & ~1, M, d_in, d_out, r, PLAN_SMS, &fp);
    plan->fwd_tail = !fp.fwd_tail ? 2 : fp.fwd_ksplit ? 3 : 1;
    plan->dx_overlap = bwd ? (pl.dx_ksplit ? 3 : overlap ? 1 : 2) : 0;
    const bool sk_bwd = bwd && !pl.side_bwd;
    plan->splitk[0] = pl.side ? 0 : pl.s_xa.splits;
    plan->splitk[1] = sk_bwd ? pl.s_g.splits : 0;
    plan->splitk[2] = sk_bwd ? pl.s_db.splits : 0;
    plan->splitk[3] = sk_bwd ? pl.s_da.splits : 0;
    return LORA_OK;
}

lora_status_t lora_linear_fwd_nf4(const uint16_t *x, const uint8_t *Wq, const uint16_t *Wscale, const float *codebook,
                                  const uint16_t *A, const uint16_t *B, uint16_t *h, uint16_t *xa_save, int64_t M,
                                  int64_t d_in, int64_t d_out, int r, float alpha, void *workspace,
                                  size_t workspace_bytes, void *stream) {
    Weight wt;
    wt.Wq = Wq;
    wt.Wscale = Wscale;
    wt.codebook = codebook;
    wt.wf = WF_CB;
    if (!Wq || !Wscale || !codebook) return LORA_ERR_INVALID_ARG;
    return fwd_impl(x, wt, A, B, h, xa_save, M, d_in, d_out, r, alpha, workspace, workspace_bytes, stream);
}

lora_status_t lora_linear_bwd_nf4(const uint16_t *dY, const uint16_t *x, const uint8_t *Wq, const uint16_t *Wscale,
                                  const float *codebook, const uint16_t *A, const uint16_t *B,
                                  const uint16_t *xa_save, uint16_t *dX, float *dA, float *dB, int64_t M,
                                  int64_t d_in, int64_t d_out, int r, float alpha, void *workspace,
                                  size_t workspace_bytes, void *stream) {
    Weight wt;
    wt.Wq = Wq;
    wt.Wscale = Wscale;
    wt.codebook = codebook;
    wt.wf = WF_CB;
    if (!Wq || !Wscale || !codebook) return LORA_ERR_INVALID_ARG;
    return bwd_impl(dY, x, wt, A, B, xa_save, dX, dA, dB, M, d_in, d_out, r, alpha, workspace, workspace_bytes,
                    stream);
}

lora_status_t lora_linear_check(void *workspace, void *stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return LORA_ERR_CUDA;
    if (!workspace) return LORA_OK;
    int word = 0;
    if (cudaMemcpy(&word, workspace, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return LORA_ERR_CUDA;
    if (word != 0) {
        cudaMemset(workspace, 0, sizeof(int));
        return LORA_ERR_TIMEOUT;
    }
    return LORA_OK;
}

// Failure-path self-test: one warp waits, through the kernels' own bounded wait, on an
// mbarrier that nothing ever arrives on; the wait runs out after `limit_ns` and records
// its code in the error word, as a stalled pipeline stage in the layer's kernels would.
__global__ void k_wait_selftest(int *err, uint64_t limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ volatile int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncwarp();
    if (threadIdx.x == 0) wait_bounded(smem_u32(&bar), 0, &abort_flag, err, DERR_WAIT_FULL, limit_ns);
}

lora_status_t lora_linear_selftest_timeout(void *workspace, size_t ws_bytes, uint32_t limit_us, void *stream) {
    if (!workspace || ws_bytes < sizeof(int)) return LORA_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return LORA_ERR_MISALIGNED;
    if (limit_us == 0 || limit_us > 2000000u) return LORA_ERR_INVALID_ARG;
    int dev = 0;
    DevInfo *info = nullptr;
    if (!device_info(&dev, &info)) return LORA_ERR_CUDA;
    if (!info->supported) return LORA_ERR_UNSUPPORTED;
    k_wait_selftest<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<int *>(workspace),
                                                                     uint64_t(limit_us) * 1000u);
    return cudaGetLastError() == cudaSuccess ? LORA_OK : LORA_ERR_CUDA;
}

const char *lora_status_string(lora_status_t status) {
    switch (status) {
        case LORA_OK: return "ok";
        case LORA_ERR_INVALID_ARG: return "invalid argument (null pointer, shape, r or alpha)";
        case LORA_ERR_MISALIGNED: return "misaligned pointer (16 B; workspace 256 B)";
        case LORA_ERR_UNSUPPORTED: return "unsupported (needs an sm_100 device / covered shape)";
        case LORA_ERR_WORKSPACE: return "workspace missing or too small";
        case LORA_ERR_CUDA: return "CUDA error";
        case LORA_ERR_TIMEOUT: return "device wait timed out";
    }
    return "unknown status";
}

int64_t lora_linear_launch_count(void) { return g_launches.load(); }

lora_status_t lora_linear_trace_enable(void *device_buffer, size_t bytes) {
    if (!device_buffer || bytes < LORA_K_COUNT * 8) {
        g_trace.store(nullptr);
        g_trace_stride.store(0);
        return LORA_OK;
    }
    if (reinterpret_cast<uintptr_t>(device_buffer) & 7u) return LORA_ERR_MISALIGNED;
    g_trace_stride.store(bytes / 8 / LORA_K_COUNT);
    g_trace.store(static_cast<unsigned long long *>(device_buffer));
    return LORA_OK;
}

lora_status_t lora_linear_timing_enable(int enable) {
    g_timing.store(enable ? 1 : 0);
    return LORA_OK;
}

lora_status_t lora_linear_timing_read(double *ms_per_kind, int64_t *launches_per_kind, int kinds) {
    std::vector<TimedLaunch> rec;
    {
        std::lock_guard<std::mutex> lk(g_tmu);
        rec.swap(g_timed);
    }
    for (int k = 0; k < kinds; ++k) {
        if (ms_per_kind) ms_per_kind[k] = 0.0;
        if (launches_per_kind) launches_per_kind[k] = 0;
    }
    lora_status_t st = LORA_OK;
    for (const TimedLaunch &t : rec) {
        float ms = 0.f;
        if (cudaEventSynchronize(t.b) != cudaSuccess || cudaEventElapsedTime(&ms, t.a, t.b) != cudaSuccess)
            st = LORA_ERR_CUDA;
        else if (t.kind >= 0 && t.kind < kinds) {
            if (ms_per_kind) ms_per_kind[t.kind] += ms;
            if (launches_per_kind) launches_per_kind[t.kind] += 1;
        }
    }
    std::lock_guard<std::mutex> lk(g_tmu);
    for (const TimedLaunch &t : rec) {
        g_event_pool.push_back(t.a);
        g_event_pool.push_back(t.b);
    }
    return st;
}

}  // extern "C"
