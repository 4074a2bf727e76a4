// C-ABI entry points of liblb.so (declared and documented in include/lb.h).
// Host code only validates arguments, computes launch shapes and launches;
// every step of the decision path runs in the kernels included below.
#include <cudaTypedefs.h>

#include <algorithm>
#include <climits>
#include <cmath>
#include <cstdio>
#include <mutex>

#include "assign.cuh"
#include "common.cuh"
#include "count.cuh"
#include "decide.cuh"
#include "gate_topk.cuh"
#include "plan.cuh"
#include "solve.cuh"
#include "swaps.cuh"
#include "split_variants.cuh"
#include "split.cuh"

namespace {

using namespace lb;

int g_tune_stages = 0;
int g_tune_split = 0;
int g_tune_persistent = 0;   // 0 automatic, 1/2/4 = persistent with that many CTAs per SM, -1 never
int g_tune_kbox = 0;         // boxes per stage of the persistent kernel (0 automatic)
int g_tune_mp = 0;           // token tiles per work unit of the persistent kernel (0 automatic, 1 or 2)
int g_tune_max_ctas = 0;     // cap on the persistent kernel's grid (0: every SM's share)

inline bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Text of the last CUDA error a call of this thread returned LB_ECUDA for.
thread_local char g_last_error[256] = "";

inline int cuda_fail(cudaError_t e, const char *where) {
    std::snprintf(g_last_error, sizeof g_last_error, "%s: %s (%d)", where, cudaGetErrorString(e),
                  static_cast<int>(e));
    return LB_ECUDA;
}

inline int launched(const char *where = "launch") {
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? LB_OK : cuda_fail(e, where);
}

// Launch options (lb_launch_options): programmatic dependent launch, on by
// default; the largest block of the integer kernels (prep and scatter pick
// up to 1024 threads).
int g_pdl = 1;
int g_max_threads = 1024;

// Launch of a kernel without clusters, with programmatic stream
// serialization when enabled: the kernel may be scheduled while the previous
// kernel on the stream is still running, and waits for it in pdl_begin().
template <typename... KArgs, typename... Args>
int launch_kernel(const char *where, void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                  Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = g_pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
    if (e != cudaSuccess) return cuda_fail(e, where);
    return launched(where);
}

int device_sms() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
    return n;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 3-D bf16 tensor map [d2][d1][d0] (d0 innermost), box {64, box1, 1},
// 128-byte swizzle, out-of-range elements read as zero.
bool make_map(CUtensorMap *map, const void *base, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t box1) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
    cuuint32_t box[3] = {static_cast<cuuint32_t>(gate::BK), box1, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

constexpr int kMaxDevices = 256;

// Ordinal of the current device, or -1 (with the error recorded).
int current_device() {
    int dev = 0;
    const cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        cuda_fail(e, "cudaGetDevice");
        return -1;
    }
    if (dev < 0 || dev >= kMaxDevices) {
        std::snprintf(g_last_error, sizeof g_last_error, "device ordinal %d out of range", dev);
        return -1;
    }
    return dev;
}

// Raise a kernel's dynamic shared-memory limit to at least `bytes` (the
// limit plus the kernel's static shared memory must stay within the
// per-block opt-in maximum, so it is raised only as far as needed).  Kernel
// attributes belong to a device, so the record is kept per device ordinal.
struct SmemLimit {
    std::mutex mu;
    size_t current[kMaxDevices] = {};
    bool cluster_set[kMaxDevices] = {};
};

template <typename F>
bool allow_smem(F *kernel, SmemLimit &lim, size_t bytes, bool cluster16) {
    const int dev = current_device();
    if (dev < 0) return false;
    std::lock_guard<std::mutex> lock(lim.mu);
    if (bytes > lim.current[dev]) {
        const cudaError_t e =
            cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
        if (e != cudaSuccess) {
            cuda_fail(e, "cudaFuncSetAttribute(max dynamic shared memory)");
            return false;
        }
        lim.current[dev] = bytes;
    }
    if (cluster16 && !lim.cluster_set[dev]) {
        const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) {
            cuda_fail(e, "cudaFuncSetAttribute(non-portable cluster size)");
            return false;
        }
        lim.cluster_set[dev] = true;
    }
    return true;
}

// One limit record per kernel that several entry points launch.
SmemLimit g_lim_plan, g_lim_split, g_lim_prep, g_lim_scatter;

template <int KMAX, bool SPLITK, bool SPLITN = false>
int launch_gate(const CUtensorMap &ma, const CUtensorMap &mb, const gate::Params &p, int mtiles, int nbatch,
                size_t smem, cudaStream_t s) {
    auto kern = gate::gate_topk_kernel<KMAX, SPLITK, SPLITN>;
    static SmemLimit lim;
    if (!allow_smem(kern, lim, smem, SPLITK || SPLITN)) return LB_ECUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(mtiles * p.split, nbatch, 1);
    cfg.blockDim = dim3(gate::THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    if (SPLITK || SPLITN) {
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = p.split;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
    } else {
        // (programmatic dependent launch only for launches without clusters)
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = g_pdl ? 1 : 0;
    }
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, ma, mb, p);
    if (e != cudaSuccess) return cuda_fail(e, "cudaLaunchKernelEx(gate_topk)");
    return launched("gate_topk");
}

template <int KMAX, int ES, int MP>
int launch_gate_persistent(const CUtensorMap &ma, const CUtensorMap &mb, const gate::Params &p, int units,
                           int nunits, int grid, size_t smem, cudaStream_t s) {
    auto kern = gate::gate_topk_persistent<KMAX, ES, MP>;
    static SmemLimit lim;
    if (!allow_smem(kern, lim, smem, false)) return LB_ECUDA;
    return launch_kernel("gate_topk_persistent", kern, dim3(grid), dim3(gate::Shape<ES>::THREADS), smem, s, ma, mb, p,
                         units, nunits);
}

// (sixteen epilogue warps only for k <= 8: the hand-over lists of k <= 16
// would not fit the static shared memory)
template <int ES, int MP>
int launch_gate_persistent_es(int k, const CUtensorMap &ma, const CUtensorMap &mb, const gate::Params &p,
                              int units, int nunits, int grid, size_t smem, cudaStream_t s) {
    if (k <= 2) return launch_gate_persistent<2, ES, MP>(ma, mb, p, units, nunits, grid, smem, s);
    if (k <= 4) return launch_gate_persistent<4, ES, MP>(ma, mb, p, units, nunits, grid, smem, s);
    if (k <= 8) return launch_gate_persistent<8, ES, MP>(ma, mb, p, units, nunits, grid, smem, s);
    if constexpr (ES == 2) return launch_gate_persistent<16, 2, MP>(ma, mb, p, units, nunits, grid, smem, s);
    return LB_EINVAL;
}

template <int KMAX, int ES, int MP>
size_t static_smem_of() {
    cudaFuncAttributes a{};
    return cudaFuncGetAttributes(&a, gate::gate_topk_persistent<KMAX, ES, MP>) == cudaSuccess ? a.sharedSizeBytes
                                                                                             : 64 * 1024;
}

// Static shared memory of the persistent kernel instance a launch will use.
template <int ES, int MP>
size_t persistent_static_smem(int k) {
    if (k <= 2) return static_smem_of<2, ES, MP>();
    if (k <= 4) return static_smem_of<4, ES, MP>();
    if (k <= 8) return static_smem_of<8, ES, MP>();
    if constexpr (ES == 2) return static_smem_of<16, 2, MP>();
    return 64 * 1024;
}

template <int KMAX, int MP>
size_t static_smem_pair_of() {
    cudaFuncAttributes a{};
    return cudaFuncGetAttributes(&a, gate::gate_topk_persistent<KMAX, 4, MP, true>) == cudaSuccess
               ? a.sharedSizeBytes
               : 64 * 1024;
}

size_t persistent_static_smem_pair(int k, int mp) {
    if (mp == 2) {
        if (k <= 2) return static_smem_pair_of<2, 2>();
        if (k <= 4) return static_smem_pair_of<4, 2>();
        return static_smem_pair_of<8, 2>();
    }
    if (k <= 2) return static_smem_pair_of<2, 1>();
    if (k <= 4) return static_smem_pair_of<4, 1>();
    return static_smem_pair_of<8, 1>();
}

size_t persistent_static_smem(int k, int es, int mp) {
    if (es == 4) return mp == 2 ? persistent_static_smem<4, 2>(k) : persistent_static_smem<4, 1>(k);
    return mp == 2 ? persistent_static_smem<2, 2>(k) : persistent_static_smem<2, 1>(k);
}

// CTA-pair launch of the persistent gate (clusters of two CTAs sharing one
// MMA of M = 256; sixteen epilogue warps, k <= 8).
template <int KMAX, int MP>
int launch_gate_pair(const CUtensorMap &ma, const CUtensorMap &mb, const gate::Params &p, int units, int nunits,
                     int grid, size_t smem, cudaStream_t s) {
    auto kern = gate::gate_topk_persistent<KMAX, 4, MP, true>;
    static SmemLimit lim;
    if (!allow_smem(kern, lim, smem, false)) return LB_ECUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(gate::Shape<4>::THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, ma, mb, p, units, nunits);
    if (e != cudaSuccess) return cuda_fail(e, "cudaLaunchKernelEx(gate_topk pair)");
    return launched("gate_topk pair");
}

// Persistent gate over CTA pairs: work units of 256 tokens (one 128-token
// tile per CTA), each CTA loading half of the N = Epad B rows, so the map
// `mb` has boxes of Epad/2 rows.  One CTA per SM; TMEM holds two
// accumulators of Epad columns.
int run_pair(gate::Params &p, const void *h, int nprob, const CUtensorMap &mb, int sms, cudaStream_t s) {
    if (p.k > 8 || p.Epad % 16 != 0 || p.Epad < 16 || p.Epad > 256) return LB_EINVAL;
    // work units of one pair tile (256 tokens), or two sharing every W box
    // (tuning: two tiles per unit; single-buffered accumulator when two
    // double-buffered pairs of accumulators would not fit TMEM)
    const int mp = g_tune_mp == 2 ? 2 : 1;
    int nbuf = 2;
    uint32_t need = 2u * mp * static_cast<uint32_t>(p.Epad);
    if (need > 512u) {
        nbuf = 1;
        need = static_cast<uint32_t>(mp) * static_cast<uint32_t>(p.Epad);
    }
    uint32_t pcols = 32;
    while (pcols < need) pcols <<= 1;
    if (pcols > 512) return LB_EINVAL;
    p.tmem_cols = pcols;
    p.nbuf = nbuf;
    p.split = 1;
    const size_t stat = persistent_static_smem_pair(p.k, mp);
    const size_t room = 227 * 1024 - stat - 2048;
    const size_t box_bytes = 16384 * static_cast<size_t>(mp) + static_cast<size_t>(p.Epad / 2) * 128;
    p.kbox = g_tune_kbox ? g_tune_kbox : (mp == 2 ? 1 : 2);
    if (p.kbox * box_bytes * 2 + 1024 > std::min<size_t>(224 * 1024, room + 1024)) p.kbox = 1;
    const size_t stage_bytes = box_bytes * p.kbox;
    const size_t fit = std::min<size_t>(224 * 1024 - 1024, room) / stage_bytes;
    int stages = static_cast<int>(std::min<size_t>(gate::MAX_STAGES, fit));
    if (g_tune_stages) stages = std::min(stages, g_tune_stages);
    if (stages < 2) return LB_EINVAL;
    // at least half the SM's shared memory: one CTA per SM (TMEM)
    size_t smem = std::max(stages * stage_bytes + 1024, static_cast<size_t>(115 * 1024));
    if (smem > std::min<size_t>(224 * 1024, room + 1024)) return LB_EINVAL;
    p.stages = stages;
    CUtensorMap ma;
    if (!make_map(&ma, h, static_cast<uint64_t>(p.H), static_cast<uint64_t>(p.T), static_cast<uint64_t>(nprob),
                  gate::BM)) {
        std::snprintf(g_last_error, sizeof g_last_error, "cuTensorMapEncodeTiled failed for h");
        return LB_ECUDA;
    }
    const int units = (p.T + 2 * gate::BM * mp - 1) / (2 * gate::BM * mp);
    const long long nunits = static_cast<long long>(units) * nprob;
    long long cap = sms / 2;
    if (g_tune_max_ctas > 0) cap = std::min<long long>(cap, g_tune_max_ctas / 2);
    if (nunits < 1 || cap < 1 || nunits > INT_MAX) return LB_EINVAL;
    const long long rounds = (nunits + cap - 1) / cap;
    const int grid = 2 * static_cast<int>((nunits + rounds - 1) / rounds);
    const int nu = static_cast<int>(nunits);
    if (mp == 2) {
        if (p.k <= 2) return launch_gate_pair<2, 2>(ma, mb, p, units, nu, grid, smem, s);
        if (p.k <= 4) return launch_gate_pair<4, 2>(ma, mb, p, units, nu, grid, smem, s);
        return launch_gate_pair<8, 2>(ma, mb, p, units, nu, grid, smem, s);
    }
    if (p.k <= 2) return launch_gate_pair<2, 1>(ma, mb, p, units, nu, grid, smem, s);
    if (p.k <= 4) return launch_gate_pair<4, 1>(ma, mb, p, units, nu, grid, smem, s);
    return launch_gate_pair<8, 1>(ma, mb, p, units, nu, grid, smem, s);
}

// CTA pairs with H split in two: one 256-token unit per cluster of four
// (two pairs), the second pair's partial accumulators added by the first.
// One shared-memory limit record per instantiation of the pair split-H
// gate (its launch and the occupancy query below both raise the limit).
template <int KMAX, int KS>
SmemLimit &pairk_lim() {
    static SmemLimit lim;
    return lim;
}

// Clusters of 2 KS CTAs of the pair split-H gate (one CTA per SM) that are
// resident on the current device at once; 0 if the query fails.  Cached per
// device.
template <int KS>
int pairk_max_clusters() {
    static int cached[kMaxDevices] = {};   // 0 not asked yet, -1 failed
    const int dev = current_device();
    if (dev < 0) return 0;
    if (cached[dev] != 0) return std::max(cached[dev], 0);
    auto kern = gate::gate_topk_pairk<8, KS>;
    const size_t smem = 115 * 1024;   // one CTA per SM whatever the pipeline's size
    int n = 0;
    if (allow_smem(kern, pairk_lim<8, KS>(), smem, false)) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * KS * 64, 1, 1);
        cfg.blockDim = dim3(gate::Shape<4>::THREADS, 1, 1);
        cfg.dynamicSmemBytes = smem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2 * KS;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
            cudaGetLastError();
            n = 0;
        }
    }
    cached[dev] = n > 0 ? n : -1;
    return std::max(n, 0);
}

template <int KMAX, int KS>
int launch_gate_pairk(const CUtensorMap &ma, const CUtensorMap &mb, const gate::Params &p, int units, int nbatch,
                      size_t smem, cudaStream_t s) {
    auto kern = gate::gate_topk_pairk<KMAX, KS>;
    if (!allow_smem(kern, pairk_lim<KMAX, KS>(), smem, false)) return LB_ECUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * KS * units, nbatch, 1);
    cfg.blockDim = dim3(gate::Shape<4>::THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2 * KS;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    // (the kernel waits for its predecessor before it touches global memory)
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = g_pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, ma, mb, p);
    if (e != cudaSuccess) return cuda_fail(e, "cudaLaunchKernelEx(gate_topk pair, split H)");
    return launched("gate_topk pair, split H");
}

// CTA pairs with H split over ks pairs (2, 3 or 4): TMEM columns, boxes per
// stage, stages, and shared memory for the larger of the pipeline and the
// epilogue's staged partial plus the slices it receives.
int run_pairk(gate::Params &p, const void *h, const void *w, int nbatch, int ks, cudaStream_t s) {
    if (p.k > 8 || p.Epad % 16 != 0 || p.Epad < 16 || p.Epad > 256) return LB_EINVAL;
    if (ks < 2 || ks > 4) return LB_EINVAL;
    // every pair needs at least one k-block of H
    if ((ks - 1) * ((p.nkb + ks - 1) / ks) >= p.nkb) return LB_EINVAL;
    uint32_t pcols = 32;
    while (pcols < static_cast<uint32_t>(p.Epad)) pcols <<= 1;
    p.tmem_cols = pcols;
    p.nbuf = 1;
    p.split = 1;
    p.kbox = g_tune_kbox ? g_tune_kbox : 2;
    const size_t box_bytes = 16384 + static_cast<size_t>(p.Epad / 2) * 128;
    const size_t sr = static_cast<size_t>((p.Epad + 31) & ~31);
    const size_t rmax = static_cast<size_t>(((gate::BM + ks - 1) / ks + 7) & ~7);   // largest row slice
    const size_t epi_bytes = (gate::BM + static_cast<size_t>(ks - 1) * rmax) * sr * 4;
    const size_t room = 200 * 1024;
    if (2 * box_bytes * p.kbox > room) p.kbox = 1;
    const size_t stage_bytes = box_bytes * p.kbox;
    int stages = static_cast<int>(std::min<size_t>(gate::MAX_STAGES, room / stage_bytes));
    if (g_tune_stages) stages = std::min(stages, g_tune_stages);
    if (stages < 2) return LB_EINVAL;
    // one CTA per SM (TMEM); the epilogue reuses the pipeline buffers
    const size_t smem = std::max({stages * stage_bytes + 1024, epi_bytes + 1024, static_cast<size_t>(115 * 1024)});
    if (smem > 225 * 1024) return LB_EINVAL;
    p.stages = stages;
    CUtensorMap ma, mb;
    if (!make_map(&ma, h, static_cast<uint64_t>(p.H), static_cast<uint64_t>(p.T), static_cast<uint64_t>(nbatch),
                  gate::BM) ||
        !make_map(&mb, w, static_cast<uint64_t>(p.H), static_cast<uint64_t>(p.E), static_cast<uint64_t>(nbatch),
                  static_cast<uint32_t>(p.Epad / 2))) {
        std::snprintf(g_last_error, sizeof g_last_error, "cuTensorMapEncodeTiled failed");
        return LB_ECUDA;
    }
    const int units = (p.T + 2 * gate::BM - 1) / (2 * gate::BM);
    if (ks == 2) {
        if (p.k <= 2) return launch_gate_pairk<2, 2>(ma, mb, p, units, nbatch, smem, s);
        if (p.k <= 4) return launch_gate_pairk<4, 2>(ma, mb, p, units, nbatch, smem, s);
        return launch_gate_pairk<8, 2>(ma, mb, p, units, nbatch, smem, s);
    }
    if (ks == 3) {
        if (p.k <= 2) return launch_gate_pairk<2, 3>(ma, mb, p, units, nbatch, smem, s);
        if (p.k <= 4) return launch_gate_pairk<4, 3>(ma, mb, p, units, nbatch, smem, s);
        return launch_gate_pairk<8, 3>(ma, mb, p, units, nbatch, smem, s);
    }
    if (p.k <= 2) return launch_gate_pairk<2, 4>(ma, mb, p, units, nbatch, smem, s);
    if (p.k <= 4) return launch_gate_pairk<4, 4>(ma, mb, p, units, nbatch, smem, s);
    return launch_gate_pairk<8, 4>(ma, mb, p, units, nbatch, smem, s);
}

// Persistent gate launch shared by lb_predict_topk and lb_predict_topk_chain:
// TMEM columns for two accumulators of p.Epad, boxes per stage, stages, and
// shared memory padded so that at most per_sm CTAs share an SM.  The h map
// covers nprob problems of [T, H].
int run_persistent(gate::Params &p, const void *h, int nprob, const CUtensorMap &mb, int per_sm, int mtiles,
                   long long ntiles, int sms, cudaStream_t s) {
    // Work units of MP tiles sharing every W box: two when the MMA's N makes
    // W's L2 traffic comparable to h's (N >= 128) or when asked.
    int mp = g_tune_mp ? g_tune_mp : 1;   // measured: two tiles per unit gained nothing on the benchmark shapes
    if (mp == 2 && mtiles < 2) mp = 1;
    // epilogue sets: 16 warps at one CTA per SM (k <= 8), else 8; chain mode
    // with two tiles per unit needs the 16
    int es = (per_sm == 1 && p.k <= 8) ? 4 : 2;
    if (p.chain && mp == 2) {
        if (p.k > 8) mp = 1;
        else {
            es = 4;
            per_sm = 1;
        }
    }
    if (es == 4 && per_sm > 1) per_sm = 1;
    // TMEM: MP accumulators of Epad columns, double-buffered when they fit
    int nbuf = 2;
    uint32_t need = 2u * mp * static_cast<uint32_t>(p.Epad);
    if (need > 512u / per_sm) {
        nbuf = 1;
        need = static_cast<uint32_t>(mp) * static_cast<uint32_t>(p.Epad);
    }
    uint32_t pcols = 32;
    while (pcols < need) pcols <<= 1;
    if (pcols > 512 || static_cast<uint32_t>(per_sm) * pcols > 512) return LB_EINVAL;
    p.tmem_cols = pcols;
    p.nbuf = nbuf;
    p.split = 1;
    // boxes per stage (measured): two for N <= 64 and for N >= 256, one between
    const size_t stat = persistent_static_smem(p.k, es, mp);
    const size_t room = 227 * 1024 - stat - 2048;   // dynamic shared memory the CTA can still take
    const size_t box_bytes = 16384 * static_cast<size_t>(mp) + static_cast<size_t>(p.Epad) * 128;
    p.kbox = g_tune_kbox ? g_tune_kbox : ((p.Epad <= 64 || p.Epad >= 256) ? 2 : 1);
    // (automatic choice: back to one box per stage when two stages of two
    // boxes would not fit, e.g. two tiles per unit at N = 256)
    if (!g_tune_kbox && p.kbox == 2 && 4 * box_bytes + 1024 > std::min<size_t>(224 * 1024, room + 1024)) p.kbox = 1;
    const size_t stage_bytes = box_bytes * p.kbox;
    // per CTA when per_sm CTAs share the SM's 228 KB (static memory and the
    // 1 KB the driver reserves per CTA included)
    const size_t share = 228 * 1024 / per_sm - stat - 3 * 1024;
    // a requested stage count is clamped to what the CTA's shared memory holds
    const size_t fit = std::min<size_t>(224 * 1024 - 1024, room) / stage_bytes;
    int stages = g_tune_stages ? static_cast<int>(std::min<size_t>(g_tune_stages, fit))
                               : static_cast<int>(std::max<size_t>(
                                     2, std::min<size_t>(gate::MAX_STAGES,
                                                         std::min<size_t>(std::min<size_t>(96 * 1024 * 2 / per_sm,
                                                                                           share), room) /
                                                             stage_bytes)));
    if (stages < 2) return LB_EINVAL;
    size_t smem = stages * stage_bytes + 1024;
    smem = std::max(smem, static_cast<size_t>(228 * 1024) / (per_sm + 1) + 1);   // at most per_sm CTAs per SM
    if (smem > std::min<size_t>(224 * 1024, room + 1024)) return LB_EINVAL;
    p.stages = stages;
    CUtensorMap ma;
    if (!make_map(&ma, h, static_cast<uint64_t>(p.H), static_cast<uint64_t>(p.T), static_cast<uint64_t>(nprob),
                  gate::BM)) {
        std::snprintf(g_last_error, sizeof g_last_error, "cuTensorMapEncodeTiled failed for h");
        return LB_ECUDA;
    }
    const int units = (mtiles + mp - 1) / mp;
    const long long nunits = static_cast<long long>(units) * nprob;
    long long cap = static_cast<long long>(sms) * per_sm;
    if (g_tune_max_ctas > 0) cap = std::min<long long>(cap, g_tune_max_ctas);
    if (nunits < 1 || cap < 1) return LB_EINVAL;
    // the fewest CTAs that take the units in the same number of rounds: no
    // CTA does more units than with the full grid, and the slots left over
    // stay free for kernels on other streams
    const long long rounds = (nunits + cap - 1) / cap;
    const int grid = static_cast<int>((nunits + rounds - 1) / rounds);
    if (es == 4)
        return mp == 2 ? launch_gate_persistent_es<4, 2>(p.k, ma, mb, p, units, static_cast<int>(nunits), grid, smem, s)
                       : launch_gate_persistent_es<4, 1>(p.k, ma, mb, p, units, static_cast<int>(nunits), grid, smem, s);
    return mp == 2 ? launch_gate_persistent_es<2, 2>(p.k, ma, mb, p, units, static_cast<int>(nunits), grid, smem, s)
                   : launch_gate_persistent_es<2, 1>(p.k, ma, mb, p, units, static_cast<int>(nunits), grid, smem, s);
}

template <bool SPLITK, bool SPLITN = false>
int launch_gate_k(int k, const CUtensorMap &ma, const CUtensorMap &mb, const gate::Params &p, int mtiles,
                  int nbatch, size_t smem, cudaStream_t s) {
    if (k <= 2) return launch_gate<2, SPLITK, SPLITN>(ma, mb, p, mtiles, nbatch, smem, s);
    if (k <= 4) return launch_gate<4, SPLITK, SPLITN>(ma, mb, p, mtiles, nbatch, smem, s);
    if (k <= 8) return launch_gate<8, SPLITK, SPLITN>(ma, mb, p, mtiles, nbatch, smem, s);
    return launch_gate<16, SPLITK, SPLITN>(ma, mb, p, mtiles, nbatch, smem, s);
}

// Split of N across a cluster of S CTAs per token tile (each CTA Epad/S
// experts of the tile, lists merged over distributed shared memory).
int run_splitn(gate::Params &p, const void *h, const void *w, int nbatch, int mtiles, int S, cudaStream_t s) {
    const int Nc = p.Epad / S;
    if (S < 2 || S > 8 || p.Epad % (16 * S) != 0 || Nc < 16) return LB_EINVAL;
    uint32_t cols = 32;
    while (cols < static_cast<uint32_t>(Nc)) cols <<= 1;
    p.tmem_cols = cols;
    p.split = S;
    const size_t stage_bytes = 16384 + static_cast<size_t>(Nc) * 128;
    int stages = g_tune_stages ? g_tune_stages
                               : static_cast<int>(std::min<size_t>(gate::MAX_STAGES, (200 * 1024) / stage_bytes));
    size_t smem = stages * stage_bytes + 1024;
    if (smem > 224 * 1024) {
        stages = static_cast<int>((224 * 1024 - 1024) / stage_bytes);
        smem = stages * stage_bytes + 1024;
    }
    if (stages < 2) return LB_EINVAL;
    smem = std::max(smem, static_cast<size_t>(gate::BM) * LB_MAX_K_GATE * 4 + 1024);   // the hand-over lists
    {
        // no more CTAs per SM than TMEM serves (a cluster's CTA blocked in
        // tcgen05.alloc behind a sibling waiting at the cluster barrier
        // would never proceed)
        const size_t max_ctas = 512 / p.tmem_cols;
        smem = std::max(smem, static_cast<size_t>(228 * 1024) / (max_ctas + 1) + 1);
        if (smem > 224 * 1024) return LB_EINVAL;
    }
    p.stages = stages;
    CUtensorMap ma, mb;
    if (!make_map(&ma, h, static_cast<uint64_t>(p.H), static_cast<uint64_t>(p.T), static_cast<uint64_t>(nbatch),
                  gate::BM)) {
        std::snprintf(g_last_error, sizeof g_last_error, "cuTensorMapEncodeTiled failed for h");
        return LB_ECUDA;
    }
    if (!make_map(&mb, w, static_cast<uint64_t>(p.H), static_cast<uint64_t>(p.E), static_cast<uint64_t>(nbatch),
                  static_cast<uint32_t>(Nc))) {
        std::snprintf(g_last_error, sizeof g_last_error, "cuTensorMapEncodeTiled failed for w");
        return LB_ECUDA;
    }
    return launch_gate_k<false, true>(p.k, ma, mb, p, mtiles, nbatch, smem, s);
}

// CTAs per source rank for the count: a cluster of up to 8 (rows of at
// least 256 tokens each) while the problem's ranks alone underfill the GPU
// (one Qwen3-235B-shaped problem: G = 8 ranks of 4096 tokens).
int count_split(int nbatch, int T, int G) {
    const long long ctas = static_cast<long long>(G) * nbatch;
    const long long sms = device_sms();
    int S = 1;
    while (S < 8 && ctas * S * 2 <= sms && (T / G) / (S * 2) >= 256) S *= 2;
    return S;
}

template <int K, bool VEC>
int launch_count(const int32_t *ids, int nbatch, int T, int k, int E, int G, int32_t *cnt, cudaStream_t s) {
    const int S = count_split(nbatch, T, G);
    if (S == 1)
        return launch_kernel("count", count::count_kernel<K, VEC>, dim3(G, nbatch), dim3(count::THREADS),
                             E * sizeof(int), s, ids, T, k, E, G, cnt);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(G * S, nbatch, 1);
    cfg.blockDim = dim3(count::THREADS, 1, 1);
    cfg.dynamicSmemBytes = E * sizeof(int);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = S;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, count::count_kernel_cluster<K, VEC>, ids, T, k, E, G, S, cnt);
    if (e != cudaSuccess) return cuda_fail(e, "cudaLaunchKernelEx(count, cluster)");
    return launched("count (cluster)");
}

template <int K>
int launch_count_v(bool vec, const int32_t *ids, int nbatch, int T, int k, int E, int G, int32_t *cnt,
                   cudaStream_t s) {
    return vec ? launch_count<K, true>(ids, nbatch, T, k, E, G, cnt, s)
               : launch_count<K, false>(ids, nbatch, T, k, E, G, cnt, s);
}

// Scatter CTAs per problem: one per source block, or one per SC_WARPS small
// blocks (one block per warp).
int scatter_grid_x(int T, int k, int G, int nw = assign::SC_WARPS, int slices = 1, bool cta_blocks = false) {
    const long long nitems = static_cast<long long>(T / G) * k;
    return nitems <= assign::WARP_BLOCK_MAX && !cta_blocks ? (G + nw - 1) / nw : G * slices;
}

// Scatter CTAs per large source block: when one CTA per block leaves most
// SMs idle (one problem's latency: G = 8 blocks of 4096 tokens take 8 SMs),
// token-aligned slices of at least 256 tokens, as many as keep the CTAs
// within one wave; each slice's CTA first counts its block's earlier slices.
// (Qwen3-235B-shaped problem, one launch of lb_assign, T = 32768, G = 8.)
int scatter_slices(int nbatch, int T, int k, int G) {
    if (T <= 0 || static_cast<long long>(T / G) * k <= assign::WARP_BLOCK_MAX) return 1;
    const long long ctas = static_cast<long long>(G) * nbatch;
    const long long sms = device_sms();
    int S = 1;
    while (ctas * S * 2 <= sms && (T / G) / (S * 2) >= 256) S *= 2;
    return S;
}

// The assign's prep for one problem's latency on a cluster of 8 CTAs (each
// owning G/8 ranks of the (rank, expert) key table) when the table is large
// and the problems' clusters all fit the device at once (on a B200 about 15
// clusters of 8 whole-SM CTAs): at the decode shape (64 x 256 keys) one CTA was
// instruction-bound for about 34 us.  Otherwise one CTA per problem.
SmemLimit g_lim_prep_cluster;

// Clusters of 8 prep CTAs of nt threads that the device holds at once
// (cached per device and block size; 0 if the query fails), asked with the
// largest shared memory the prep may take.
int prep_max_clusters(int nt) {
    static int cached[kMaxDevices][3] = {};   // 0 not asked yet, -1 none or failed
    const int dev = current_device();
    const int t = nt >= 1024 ? 2 : nt >= 512 ? 1 : 0;
    if (dev < 0) return 0;
    if (cached[dev][t] != 0) return std::max(cached[dev][t], 0);
    const size_t smem = 224 * 1024;
    int n = 0;
    if (allow_smem(assign::prep_kernel_cluster, g_lim_prep_cluster, smem, false)) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(8, 64, 1);
        cfg.blockDim = dim3(nt, 1, 1);
        cfg.dynamicSmemBytes = smem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 8;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaOccupancyMaxActiveClusters(&n, assign::prep_kernel_cluster, &cfg) != cudaSuccess) {
            cudaGetLastError();
            n = 0;
        }
    }
    cached[dev][t] = n > 0 ? n : -1;
    return std::max(n, 0);
}

int launch_prep(const assign::Args &a, int nbatch, size_t smem, cudaStream_t s, const char *what) {
    const int nt = std::min(assign::PREP_THREADS, g_max_threads);
    // the cluster form only when every problem's cluster runs at once
    const bool cl = static_cast<long long>(a.G) * a.E >= 8192 && a.G % 8 == 0 && nbatch <= prep_max_clusters(nt);
    if (!cl) {
        if (!allow_smem(assign::prep_kernel, g_lim_prep, smem, false)) return LB_ECUDA;
        return launch_kernel(what, assign::prep_kernel, dim3(nbatch), dim3(nt), smem, s, a);
    }
    if (!allow_smem(assign::prep_kernel_cluster, g_lim_prep_cluster, smem, false)) return LB_ECUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(8, nbatch, 1);
    cfg.blockDim = dim3(nt, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 8;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = g_pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, assign::prep_kernel_cluster, a);
    if (e != cudaSuccess) return cuda_fail(e, "cudaLaunchKernelEx(assign prep, cluster)");
    return launched(what);
}

// Warps per scatter CTA for sliced blocks: one chunk of 32 tokens per warp
// covers the slice (at least 8 warps: the prefix counts use a row of the
// per-warp table).
int slice_warps(int T, int G, int S) {
    const int tps = (T / G + S - 1) / S;
    int nw = 8;
    while (nw < assign::SC_WARPS && nw * 32 < tps) nw <<= 1;
    return nw;
}

// Warps per scatter CTA: 32 while the problems' CTAs leave SMs free (one
// problem's latency), 16 once they fill the GPU twice over (throughput: two
// CTAs per SM); fewer if the per-warp tables would not fit shared memory.
// Small source blocks (one warp each) go in CTAs of 8 warps while those fit
// one wave, so that one problem's blocks spread over more SMs (decode shape,
// G=64, one problem: lb_assign 80.0 against 93.6 us at T=8192 and 69.6
// against 77.5 us at T=4096 with 32 warps per CTA; 4, 2 or 1 were slower).
int scatter_warps(int nbatch, int T, int k, int G, int E, int N) {
    if (static_cast<long long>(T / G) * k <= assign::WARP_BLOCK_MAX &&
        static_cast<long long>(scatter_grid_x(T, k, G, 8)) * nbatch <= device_sms())
        return 8;
    const long long ctas = static_cast<long long>(scatter_grid_x(T, k, G, 16)) * nbatch;
    int nw = ctas >= 2LL * device_sms() ? 16 : assign::SC_WARPS;
    nw = std::min(nw, g_max_threads / 32);
    while (nw > 8 && assign::scatter_smem_bytes(G, E, N, nw) > 224 * 1024) nw >>= 1;
    return nw;
}

// Launch shape of the scatter for a.T, a.k, a.G, a.E, a.N over nbatch
// problems: sets a.slices and a.cta_blocks, returns the warps per CTA (grid:
// scatter_grid_x).  Small source blocks whose CTAs all fit one wave go one
// block per CTA down the CTA path (token ranks from per-warp masks) rather
// than one block per warp: one decode-shaped problem (G = 64 blocks of 128
// tokens x top-8) otherwise keeps 8 SMs busy for most of the launch.
int scatter_shape(assign::Args &a, int nbatch) {
    const int T = a.T, k = a.k, G = a.G, E = a.E, N = a.N;
    a.slices = scatter_slices(nbatch, T, k, G);
    a.cta_blocks = 0;
    if (T == 0) return assign::SC_WARPS;
    if (a.slices > 1) return std::min(slice_warps(T, G, a.slices), g_max_threads / 32);
    if (static_cast<long long>(T / G) * k <= assign::WARP_BLOCK_MAX &&
        static_cast<long long>(G) * nbatch <= device_sms()) {
        int nw = std::min(slice_warps(T, G, 1), g_max_threads / 32);
        while (nw > 8 && assign::scatter_smem_bytes(G, E, N, nw) > 224 * 1024) nw >>= 1;
        if (assign::scatter_smem_bytes(G, E, N, nw) <= 224 * 1024) {
            a.cta_blocks = 1;
            return nw;
        }
    }
    return scatter_warps(nbatch, T, k, G, E, N);
}

bool plan_shape_ok(int G, int E, int N, int L) {
    if (G < 1 || G > LB_MAX_G || E < 1 || E > LB_MAX_E || E % G != 0) return false;
    if (N < 0 || N > LB_MAX_N || N > E - E / G || L < 0 || L > N) return false;
    // the planner stages the counts in shared memory; the split its tables
    if (plan::smem_bytes(G, E, N) > 224 * 1024 || split::smem_bytes(G, E, N) > 224 * 1024) return false;
    return true;
}

}  // namespace

extern "C" {

int lb_version(void) { return 100; }

int lb_swaps_capacity(int E) { return E < 2 ? 1 : E / 2; }

const char *lb_strerror(int code) {
    switch (code) {
        case LB_OK: return "ok";
        case LB_EINVAL: return "invalid argument";
        case LB_ECUDA: return "CUDA error";
        case LB_EDATA: return "bad data seen on the device";
        case LB_ENOSPACE: return "workspace too small";
        default: return "unknown error";
    }
}

int lb_get_status(int32_t *flags, int clear) {
    if (!flags) return LB_EINVAL;
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
    int v = 0;
    e = cudaMemcpyFromSymbol(&v, lb::g_status, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e, "read status word");
    *flags = v;
    if (clear) {
        const int z = 0;
        e = cudaMemcpyToSymbol(lb::g_status, &z, sizeof(int));
        if (e != cudaSuccess) return cuda_fail(e, "clear status word");
    }
    return v ? LB_EDATA : LB_OK;
}

const char *lb_last_error(void) { return g_last_error; }

#ifdef LB_TIMING
int lb_debug_ticks(long long *out, int n) {
    if (!out || n < 1 || n > 64 + 1024) return LB_EINVAL;
    if (cudaDeviceSynchronize() != cudaSuccess) return LB_ECUDA;
    return cudaMemcpyFromSymbol(out, lb::g_ticks, sizeof(long long) * n) == cudaSuccess ? LB_OK : LB_ECUDA;
}
#endif

int lb_launch_options(int programmatic_dependent_launch, int max_block_threads) {
    if (programmatic_dependent_launch != 0 && programmatic_dependent_launch != 1) return LB_EINVAL;
    if (max_block_threads != 0 && max_block_threads != 256 && max_block_threads != 512 && max_block_threads != 1024)
        return LB_EINVAL;
    g_pdl = programmatic_dependent_launch;
    g_max_threads = max_block_threads ? max_block_threads : 1024;
    return LB_OK;
}

int lb_gate_tuning(int stages, int split, int persistent, int kbox, int tiles_per_unit, int max_ctas) {
    if (tiles_per_unit != 0 && tiles_per_unit != 1 && tiles_per_unit != 2) return LB_EINVAL;
    if (max_ctas < 0) return LB_EINVAL;
    if (kbox != 0 && kbox != 1 && kbox != 2 && kbox != 4) return LB_EINVAL;
    if (stages != 0 && (stages < 2 || stages > gate::MAX_STAGES)) return LB_EINVAL;
    if (split != 0 && split != 1 && split != 2 && split != 4 && split != 8 && split != 16 && split != -2 &&
        split != -4 && split != -8)
        return LB_EINVAL;
    if (persistent != -1 && persistent != 0 && persistent != 1 && persistent != 2 && persistent != 3 &&
        persistent != 4 && persistent != 5 && persistent != 6 && persistent != 7)
        return LB_EINVAL;
    g_tune_stages = stages;
    g_tune_split = split;
    g_tune_persistent = persistent;
    g_tune_kbox = kbox;
    g_tune_mp = tiles_per_unit;
    g_tune_max_ctas = max_ctas;
    return LB_OK;
}

int lb_predict_topk(const void *h, const void *w, const float *bias, int nbatch, int T, int H, int E, int k,
                    int32_t *ids, float *logits, void *stream) {
    if (nbatch < 1 || nbatch > 65535 || T < 0 || H < 8 || H % 8 != 0 || E < 1 || E > LB_MAX_E_GATE || k < 1 ||
        k > E || k > LB_MAX_K_GATE)
        return LB_EINVAL;
    if (!h || !w || !ids || !aligned(h, 16) || !aligned(w, 16) || !aligned(ids, 4)) return LB_EINVAL;
    if (bias && !aligned(bias, 4)) return LB_EINVAL;
    if (logits && !aligned(logits, 4)) return LB_EINVAL;
    if (static_cast<long long>(T) * nbatch * std::max(k, E) >= INT_MAX) return LB_EINVAL;
    if (T == 0) return LB_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    gate::Params p{};
    p.bias = bias;
    p.ids = ids;
    p.logits = logits;
    p.T = T;
    p.H = H;
    p.E = E;
    p.Epad = (E + 15) / 16 * 16;
    p.k = k;
    p.nkb = (H + gate::BK - 1) / gate::BK;
    p.kbox = 1;
    uint32_t cols = 32;
    while (cols < static_cast<uint32_t>(p.Epad)) cols <<= 1;
    p.tmem_cols = cols;
    const int mtiles = (T + gate::BM - 1) / gate::BM;
    const int sms = device_sms();
    const long long ntiles = static_cast<long long>(mtiles) * nbatch;

    // enough tiles for every SM: the persistent kernel (one CTA per SM)
    // Automatic choice (measured on the benchmark shapes): with at least two
    // tiles per SM, a persistent kernel with two CTAs per SM while two
    // double-buffered accumulators fit in TMEM (E <= 128); otherwise one CTA
    // per tile.
    int per_sm = g_tune_persistent;
    if (per_sm == 0 && g_tune_split <= 1 && ntiles >= 2LL * sms && p.Epad <= 128) per_sm = 2;
    // CTA pairs with H split over the most pairs (four, three, two) whose
    // clusters (8, 6 or 4 CTAs per 256-token unit) fit in one wave.
    // Measured (H=7168, E=256): T=2048 24.8 us with four pairs against
    // 53.0 us for a cluster split of H per tile, T=4096 30.3 us with three
    // (34.5 with two, 47.2 with four in two waves), T=8192 36.3 against
    // 65.4 us with two; the same order at H=4096, E=128 and H=2048, E=64
    // from 2048 to 8192 tokens.
    // Four pairs below 2048 tokens only at E > 128 (at E <= 128 no faster
    // there); two pairs in two waves only at E > 128 (T=12288: 68 against
    // 96 us at E=256; at E <= 128 slower than the split per tile); never
    // when a pair would get fewer than eight k-blocks.
    if (per_sm == 0 && g_tune_split == 0 && k <= 8 && p.Epad >= 64 && p.nkb >= 32) {
        const long long units = static_cast<long long>((T + 2 * gate::BM - 1) / (2 * gate::BM)) * nbatch;
        const long long c2 = pairk_max_clusters<2>();
        if (units <= pairk_max_clusters<4>() && (units >= 8 || p.Epad > 128))
            per_sm = 6;
        else if (units >= 8 && units <= pairk_max_clusters<3>())
            per_sm = 7;
        else if (units >= 16 && (units <= c2 || (p.Epad > 128 && units <= 2 * c2)))
            per_sm = 5;
    }
    if (per_sm >= 5) return run_pairk(p, h, w, nbatch, per_sm == 5 ? 2 : per_sm == 6 ? 4 : 3, s);
    if (per_sm == 3) {
        CUtensorMap mb;
        if (p.Epad % 16 != 0 ||
            !make_map(&mb, w, static_cast<uint64_t>(H), static_cast<uint64_t>(E), static_cast<uint64_t>(nbatch),
                      static_cast<uint32_t>(p.Epad / 2))) {
            std::snprintf(g_last_error, sizeof g_last_error, "cuTensorMapEncodeTiled failed for w");
            return LB_ECUDA;
        }
        return run_pair(p, h, nbatch, mb, sms, s);
    }
    if (per_sm > 0) {
        CUtensorMap mb;
        if (!make_map(&mb, w, static_cast<uint64_t>(H), static_cast<uint64_t>(E), static_cast<uint64_t>(nbatch),
                      static_cast<uint32_t>(p.Epad))) {
            std::snprintf(g_last_error, sizeof g_last_error, "cuTensorMapEncodeTiled failed for w");
            return LB_ECUDA;
        }
        return run_persistent(p, h, nbatch, mb, per_sm, mtiles, ntiles, sms, s);
    }

    // Split across a cluster when the token tiles alone underfill the GPU.
    // Automatic (measured at H=7168, E=256; the CTAs stream their operands
    // from L2, so the split that moves the fewest bytes per CTA within one
    // wave wins): split H over the most CTAs per tile that still fit one wave
    // (decode shape T=4096: 4 per tile, 35 us, against 80 us for 8 in two waves); where
    // that is two or fewer, split N in two instead (T=8192: 57 us, against
    // 67 us for H in two).  A negative tuning value splits N.
    if (g_tune_split < 0) return run_splitn(p, h, w, nbatch, mtiles, -g_tune_split, s);
    int S = 1;
    if (g_tune_split) {
        S = g_tune_split;
    } else {
        // (sixteen only for one or two tiles: at T=1024, eight tiles, eight per
        // tile took 26.7 us against 43.7 us for sixteen)
        const int smax = ntiles <= 2 ? 16 : 8;
        while (static_cast<long long>(mtiles) * nbatch * S * 2 <= sms && S * 2 <= smax && S * 2 <= p.nkb / 2 &&
               p.Epad % (4 * S * 2) == 0)
            S *= 2;
        if (S <= 2 && ntiles * 2 <= sms && ntiles < sms && p.Epad % 32 == 0 && p.Epad / 2 >= 32)
            return run_splitn(p, h, w, nbatch, mtiles, 2, s);
    }
    // each of the S CTAs of a cluster reduces Epad/S columns per row with
    // 16-byte shared-memory loads, so Epad/S must be a multiple of 4
    if (S > p.nkb || p.Epad % (4 * S) != 0 || gate::BM % S != 0) return LB_EINVAL;
    p.split = S;

    const size_t stage_bytes = 16384 + static_cast<size_t>(p.Epad) * 128;
    int stages = g_tune_stages;
    if (!stages)
        stages = (ntiles * S >= sms)
                     ? 2
                     : static_cast<int>(std::min<size_t>(8, std::max<size_t>(2, (110 * 1024 - 1024) / stage_bytes)));
    size_t smem = stages * stage_bytes + 1024;
    if (S > 1) smem = std::max(smem, static_cast<size_t>(gate::BM) * (p.Epad + 4) * 4 + 1024);
    if (smem > 224 * 1024) {
        stages = static_cast<int>((224 * 1024 - 1024) / stage_bytes);
        smem = stages * stage_bytes + 1024;
        if (S > 1) smem = std::max(smem, static_cast<size_t>(gate::BM) * (p.Epad + 4) * 4 + 1024);
        if (stages < 2 || smem > 224 * 1024) return LB_EINVAL;
    }
    p.stages = stages;
    // Never let more CTAs share an SM than its 512 TMEM columns can serve at
    // once: pad the shared-memory request so the extra CTA does not fit.  (In
    // a cluster, a CTA blocked in tcgen05.alloc behind a sibling that waits at
    // the cluster barrier would never proceed.)
    {
        const size_t sm_per_sm = 228 * 1024;
        const size_t max_ctas = 512 / p.tmem_cols;
        smem = std::max(smem, sm_per_sm / (max_ctas + 1) + 1);
        if (smem > 224 * 1024) return LB_EINVAL;
    }

    CUtensorMap ma, mb;
    if (!make_map(&ma, h, static_cast<uint64_t>(H), static_cast<uint64_t>(T), static_cast<uint64_t>(nbatch),
                  gate::BM)) {
        std::snprintf(g_last_error, sizeof g_last_error, "cuTensorMapEncodeTiled failed for h");
        return LB_ECUDA;
    }
    if (!make_map(&mb, w, static_cast<uint64_t>(H), static_cast<uint64_t>(E), static_cast<uint64_t>(nbatch),
                  static_cast<uint32_t>(p.Epad))) {
        std::snprintf(g_last_error, sizeof g_last_error, "cuTensorMapEncodeTiled failed for w");
        return LB_ECUDA;
    }
    return S > 1 ? launch_gate_k<true>(k, ma, mb, p, mtiles, nbatch, smem, s)
                 : launch_gate_k<false>(k, ma, mb, p, mtiles, nbatch, smem, s);
}

int lb_predict_topk_chain(const void *h, const void *w, const float *bias, int L, int T, int H, int E, int k,
                          int32_t *ids_pred, int32_t *ids_act, float *logits_pred, float *logits_act,
                          void *stream) {
    if (L < 1 || L > 65534 || T < 0 || H < 8 || H % 8 != 0 || E < 16 || E % 16 != 0 || 2 * E > 256 || k < 1 ||
        k > E || k > LB_MAX_K_GATE)
        return LB_EINVAL;
    if (!h || !w || !ids_pred || !ids_act || !aligned(h, 16) || !aligned(w, 16) || !aligned(ids_pred, 4) ||
        !aligned(ids_act, 4))
        return LB_EINVAL;
    if ((bias && !aligned(bias, 4)) || (logits_pred && !aligned(logits_pred, 4)) ||
        (logits_act && !aligned(logits_act, 4)))
        return LB_EINVAL;
    if (static_cast<long long>(T) * (L + 1) * std::max(k, E) >= INT_MAX ||
        static_cast<long long>(L) * E * H * 2 >= (1LL << 40))
        return LB_EINVAL;
    if (T == 0) return LB_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    gate::Params p{};
    p.bias = bias;
    p.ids = ids_act;
    p.logits = logits_act;
    p.ids2 = ids_pred;
    p.logits2 = logits_pred;
    p.chain = 1;
    p.L = L;
    p.T = T;
    p.H = H;
    p.E = E;
    p.Epad = 2 * E;   // the MMA's N: W_{b-1} and W_b side by side
    p.k = k;
    p.nkb = (H + gate::BK - 1) / gate::BK;
    const int mtiles = (T + gate::BM - 1) / gate::BM;
    const int sms = device_sms();
    const long long ntiles = static_cast<long long>(mtiles) * (L + 1);
    uint32_t pcols = 32;
    while (pcols < 4u * static_cast<uint32_t>(E)) pcols <<= 1;
    // (the per-layer modes 5 to 7, pairs with a split of H, do not apply to the chain)
    const int tune = g_tune_persistent >= 5 ? 0 : g_tune_persistent;
    int per_sm = tune > 0 ? tune : std::max(1, std::min(2, static_cast<int>(512 / pcols)));
    // Automatic: CTA pairs when the two gates fill the MMA's N = 256 (E = 128;
    // measured: Qwen3-235B-shaped chain 964 against 1124 us for 16 layers,
    // Qwen3-30B-shaped 293 against 332 us), where one CTA would stream a
    // weight box twice the size of its h box; one CTA per tile below that
    // (OLMoE-shaped, N = 128: 62 against 72 us).
    if (tune == 0 && 2 * E >= 256 && k <= 8) per_sm = 3;
    if (per_sm == 3) {
        // CTA pairs: each CTA loads one gate, a box of E rows starting at row
        // (b-1)E (CTA 0) or bE (CTA 1)
        CUtensorMap mb;
        if (!make_map(&mb, w, static_cast<uint64_t>(H), static_cast<uint64_t>(L) * E, 1, static_cast<uint32_t>(E))) {
            std::snprintf(g_last_error, sizeof g_last_error, "cuTensorMapEncodeTiled failed for w");
            return LB_ECUDA;
        }
        return run_pair(p, h, L + 1, mb, sms, s);
    }
    // the stack of gates as one [L*E, H] matrix; a box of 2E rows starting
    // at row (b-1)E (negative for b = 0, past the end for b = L: zeros)
    CUtensorMap mb;
    if (!make_map(&mb, w, static_cast<uint64_t>(H), static_cast<uint64_t>(L) * E, 1, static_cast<uint32_t>(2 * E))) {
        std::snprintf(g_last_error, sizeof g_last_error, "cuTensorMapEncodeTiled failed for w");
        return LB_ECUDA;
    }
    return run_persistent(p, h, L + 1, mb, per_sm, mtiles, ntiles, sms, s);
}

int lb_plan_swaps(const int32_t *cnt, const int32_t *placement, int nbatch, int G, int E, double gamma, double tau,
                  double alpha, double beta, double expert_bytes, double budget, double link_budget,
                  int32_t *placement_out, int32_t *swaps_out, int32_t *n_swaps, int32_t *loads, void *stream) {
    if (nbatch < 1 || nbatch > 65535 || G < 1 || G > LB_MAX_G || E < 1 || E > LB_MAX_E || E % G != 0)
        return LB_EINVAL;
    if (!cnt || !placement_out || !swaps_out || !n_swaps || !loads) return LB_EINVAL;
    if (!aligned(cnt, 4) || !aligned(placement_out, 4) || !aligned(swaps_out, 4) || !aligned(n_swaps, 4) ||
        !aligned(loads, 4) || (placement && !aligned(placement, 4)))
        return LB_EINVAL;
    // finite or +inf parameters in range (NaN fails every comparison)
    if (!(gamma >= 0.0) || !(tau >= 0.0) || !(alpha >= 0.0) || !(beta > 0.0) || !(expert_bytes >= 0.0) ||
        !(budget >= 0.0) || !(link_budget >= 0.0) || !(gamma < HUGE_VAL) || !(alpha < HUGE_VAL) ||
        !(expert_bytes < HUGE_VAL))
        return LB_EINVAL;
    const size_t smem = swaps::smem_bytes(G, E);
    if (smem > 224 * 1024) return LB_EINVAL;
    swaps::Params p;
    p.cnt = cnt;
    p.pi_in = placement;
    p.G = G;
    p.E = E;
    p.gamma = gamma;
    p.tau = tau;
    p.cost = alpha + (expert_bytes + expert_bytes) / beta;   // eq. 9 with S(e) = expert_bytes for every expert
    p.budget = budget;
    p.link_budget = link_budget;
    p.pi_out = placement_out;
    p.swaps = swaps_out;
    p.n_swaps = n_swaps;
    p.loads = loads;
    p.max_swaps = lb_swaps_capacity(E);
    static SmemLimit lim;
    if (!allow_smem(swaps::swaps_kernel, lim, smem, false)) return LB_ECUDA;
    return launch_kernel("plan swaps", swaps::swaps_kernel, dim3(nbatch), dim3(swaps::THREADS), smem,
                         static_cast<cudaStream_t>(stream), p);
}

int lb_split_variant(const int32_t *cnt, const void *plan, int nbatch, int G, int E, int N, int passes, int variant,
                     int32_t *tok, int32_t *mass, int32_t *loads, int32_t *passes_run, void *stream) {
    if (nbatch < 1 || nbatch > 65535 || !plan_shape_ok(G, E, N, 0) || passes < 0 || passes > 4096 || variant < 0 ||
        variant >= splitv::COUNT)
        return LB_EINVAL;
    if (!cnt || !plan || !loads || !passes_run || !aligned(cnt, 4) || !aligned(plan, 256) || !aligned(loads, 4) ||
        !aligned(passes_run, 4))
        return LB_EINVAL;
    if (G * N > 0 && (!tok || !mass || !aligned(tok, 4) || !aligned(mass, 4))) return LB_EINVAL;
    const size_t smem = splitv::smem_bytes(G, E, N);
    if (smem > 224 * 1024) return LB_EINVAL;
    splitv::Params p;
    p.cnt = cnt;
    p.plan = static_cast<const uint8_t *>(plan);
    p.plan_stride = plan::layout(G, E, N).total;
    p.G = G;
    p.E = E;
    p.N = N;
    p.passes = passes;
    p.variant = variant;
    p.tok = tok;
    p.mass = mass;
    p.loads = loads;
    p.passes_run = passes_run;
    static SmemLimit lim;
    if (!allow_smem(splitv::split_variant_kernel, lim, smem, false)) return LB_ECUDA;
    return launch_kernel("split variant", splitv::split_variant_kernel, dim3(nbatch), dim3(splitv::THREADS), smem,
                         static_cast<cudaStream_t>(stream), p);
}

int lb_count(const int32_t *ids, int nbatch, int T, int k, int E, int G, int32_t *cnt, void *stream) {
    if (nbatch < 1 || nbatch > 65535 || T < 0 || G < 1 || G > LB_MAX_G || T % G != 0 || E < 1 || E > LB_MAX_E ||
        k < 1 || k > LB_MAX_K)
        return LB_EINVAL;
    if (!cnt || (T > 0 && !ids) || !aligned(cnt, 4) || (ids && !aligned(ids, 4))) return LB_EINVAL;
    if (static_cast<long long>(T) * k * nbatch >= INT_MAX) return LB_EINVAL;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool vec = ids && aligned(ids, 16);
    if (k <= 2) return launch_count_v<2>(vec, ids, nbatch, T, k, E, G, cnt, s);
    if (k <= 4) return launch_count_v<4>(vec, ids, nbatch, T, k, E, G, cnt, s);
    if (k <= 8) return launch_count_v<8>(vec, ids, nbatch, T, k, E, G, cnt, s);
    if (k <= 16) return launch_count_v<16>(vec, ids, nbatch, T, k, E, G, cnt, s);
    return launch_count_v<32>(vec, ids, nbatch, T, k, E, G, cnt, s);
}

size_t lb_plan_bytes(int G, int E, int N) {
    if (G < 1 || E < 1 || N < 0) return 0;
    return plan::layout(G, E, N).total;
}

int lb_plan_layout_of(int G, int E, int N, lb_plan_layout *out) {
    if (!out || G < 1 || E < 1 || N < 0) return LB_EINVAL;
    const plan::Layout L = plan::layout(G, E, N);
    out->hdr = L.hdr;
    out->used = L.used;
    out->slots = L.slots;
    out->slot_phase = L.slot_phase;
    out->plan_load = L.plan_load;
    out->edge_u = L.edge_u;
    out->edge_v = L.edge_v;
    out->edge_e = L.edge_e;
    out->edge_round = L.edge_round;
    out->round_ptr = L.round_ptr;
    out->rep_ptr = L.rep_ptr;
    out->rep_edge = L.rep_edge;
    out->holds = L.holds;
    out->total = L.total;
    return LB_OK;
}

int lb_plan_replicas(const int32_t *cnt, int nbatch, int G, int E, int N, int L, void *plan, void *stream) {
    if (nbatch < 1 || !plan_shape_ok(G, E, N, L) || !cnt || !plan || !aligned(plan, 256) || !aligned(cnt, 4))
        return LB_EINVAL;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t smem = plan::smem_bytes(G, E, N);
    if (smem > 224 * 1024) return LB_EINVAL;
    if (!allow_smem(plan::plan_kernel, g_lim_plan, smem, false)) return LB_ECUDA;
    return launch_kernel("plan", plan::plan_kernel, dim3(nbatch), dim3(plan::THREADS), smem, s, cnt, G, E, N, L,
                         static_cast<uint8_t *>(plan), plan::layout(G, E, N).total);
}

int lb_split(const int32_t *cnt, const void *plan, int nbatch, int G, int E, int N, int passes, int32_t *tok,
             int32_t *mass, int32_t *loads, int32_t *passes_run, void *stream) {
    if (nbatch < 1 || !plan_shape_ok(G, E, N, 0) || passes < 0 || passes > 4096) return LB_EINVAL;
    if (!cnt || !plan || !loads || !passes_run || !aligned(plan, 256)) return LB_EINVAL;
    if (G * N > 0 && (!tok || !mass)) return LB_EINVAL;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t smem = split::smem_bytes(G, E, N);
    if (!allow_smem(split::split_kernel, g_lim_split, smem, false)) return LB_ECUDA;
    return launch_kernel("split", split::split_kernel, dim3(nbatch), dim3(split::THREADS), smem, s, cnt,
                         static_cast<const uint8_t *>(plan), plan::layout(G, E, N).total, G, E, N, passes, tok, mass,
                         loads, passes_run);
}

size_t lb_assign_workspace_bytes(int nbatch, int T, int k, int G, int E, int N) {
    (void)T;
    (void)k;
    if (nbatch < 1 || G < 1 || E < 1 || N < 0) return 0;
    return static_cast<size_t>(nbatch) * assign::ws_words(G, E, N) * 4;
}

int lb_assign(const int32_t *ids, const int32_t *cnt, const void *plan, const int32_t *tok, const int32_t *mass,
              int nbatch, int T, int k, int G, int E, int N, int32_t *dest, int32_t *perm, int32_t *offs,
              void *workspace, size_t workspace_bytes, void *stream) {
    // (G is range-checked by plan_shape_ok before T % G is taken)
    if (nbatch < 1 || nbatch > 65535 || T < 0 || k < 1 || k > LB_MAX_K || !plan_shape_ok(G, E, N, 0) || T % G != 0)
        return LB_EINVAL;
    if (!cnt || !plan || !offs || !workspace || !aligned(plan, 256) || !aligned(workspace, 256)) return LB_EINVAL;
    if (G * N > 0 && (!tok || !mass)) return LB_EINVAL;
    if (T > 0 && (!ids || !dest || !perm)) return LB_EINVAL;
    if (static_cast<long long>(T) * k * nbatch >= INT_MAX) return LB_EINVAL;
    if (assign::scatter_smem_bytes(G, E, N, 8) > 224 * 1024 || assign::prep_smem_bytes(G, E, N) > 224 * 1024)
        return LB_EINVAL;
    if (workspace_bytes < lb_assign_workspace_bytes(nbatch, T, k, G, E, N)) return LB_ENOSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    assign::Args a;
    a.ids = ids;
    a.cnt = cnt;
    a.tok = tok;
    a.mass = mass;
    a.plan = static_cast<const uint8_t *>(plan);
    a.plan_stride = plan::layout(G, E, N).total;
    a.T = T;
    a.k = k;
    a.G = G;
    a.E = E;
    a.N = N;
    a.dest = dest;
    a.perm = perm;
    a.offs = offs;
    a.ws = static_cast<int32_t *>(workspace);
    a.ws_stride = assign::ws_words(G, E, N);
    const int nw = scatter_shape(a, nbatch);
    const size_t sm1 = assign::prep_smem_bytes(G, E, N), sm2 = assign::scatter_smem_bytes(G, E, N, nw);
    if (!allow_smem(assign::scatter_kernel, g_lim_scatter, sm2, false)) return LB_ECUDA;
    if (launch_prep(a, nbatch, sm1, s, "assign prep") != LB_OK) return LB_ECUDA;
    if (T == 0) return LB_OK;
    return launch_kernel("assign scatter", assign::scatter_kernel, dim3(scatter_grid_x(T, k, G, nw, a.slices, a.cta_blocks != 0), nbatch),
                         dim3(nw * 32), assign::scatter_smem_bytes(G, E, N, nw), s, a);
}

int lb_decide(const int32_t *cnt_pred, const int32_t *cnt, const int32_t *ids, void *plan, int nbatch, int T,
              int k, int G, int E, int N, int L, int passes, int32_t *tok, int32_t *mass, int32_t *loads,
              int32_t *passes_run, int32_t *dest, int32_t *perm, int32_t *offs, void *workspace,
              size_t workspace_bytes, void *stream) {
    const bool with_plan = cnt_pred != nullptr;
    if (nbatch < 1 || nbatch > 65535 || T < 0 || k < 1 || k > LB_MAX_K ||
        !plan_shape_ok(G, E, N, with_plan ? L : 0) || T % G != 0 || passes < 0 || passes > 4096)
        return LB_EINVAL;
    if (!cnt || !plan || !loads || !passes_run || !offs || !workspace || !aligned(plan, 256) ||
        !aligned(workspace, 256) || (with_plan && !aligned(cnt_pred, 4)))
        return LB_EINVAL;
    if (G * N > 0 && (!tok || !mass)) return LB_EINVAL;
    if (T > 0 && (!ids || !dest || !perm)) return LB_EINVAL;
    if (static_cast<long long>(T) * k * nbatch >= INT_MAX) return LB_EINVAL;
    const size_t sm1 = decide::smem_bytes(G, E, N, with_plan);
    if (assign::scatter_smem_bytes(G, E, N, 8) > 224 * 1024 || sm1 > 224 * 1024) return LB_EINVAL;
    if (workspace_bytes < lb_assign_workspace_bytes(nbatch, T, k, G, E, N)) return LB_ENOSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    assign::Args a;
    a.ids = ids;
    a.cnt = cnt;
    a.tok = tok;
    a.mass = mass;
    a.plan = static_cast<const uint8_t *>(plan);
    a.plan_stride = plan::layout(G, E, N).total;
    a.T = T;
    a.k = k;
    a.G = G;
    a.E = E;
    a.N = N;
    a.dest = dest;
    a.perm = perm;
    a.offs = offs;
    a.ws = static_cast<int32_t *>(workspace);
    a.ws_stride = assign::ws_words(G, E, N);
    const int nw = scatter_shape(a, nbatch);
    const size_t sm2 = assign::scatter_smem_bytes(G, E, N, nw);
    static SmemLimit lim0, lim1;
    if (!allow_smem(assign::scatter_kernel, g_lim_scatter, sm2, false)) return LB_ECUDA;
    int rc;
    if (decide::fused_for(G, E)) {
        if (with_plan) {
            if (!allow_smem(decide::decide_kernel<true>, lim1, sm1, false)) return LB_ECUDA;
            rc = launch_kernel("decide (plan, split, tables)", decide::decide_kernel<true>, dim3(nbatch),
                               dim3(decide::THREADS), sm1, s, cnt_pred, L, a, passes, loads, passes_run);
        } else {
            if (!allow_smem(decide::decide_kernel<false>, lim0, sm1, false)) return LB_ECUDA;
            rc = launch_kernel("decide (split, tables)", decide::decide_kernel<false>, dim3(nbatch),
                               dim3(decide::THREADS), sm1, s, cnt_pred, L, a, passes, loads, passes_run);
        }
    } else {
        // large count tables: plan, split and tables as separate launches
        const size_t stride = plan::layout(G, E, N).total;
        const size_t smp = plan::smem_bytes(G, E, N), sms = split::smem_bytes(G, E, N),
                     smt = assign::prep_smem_bytes(G, E, N);
        if ((with_plan && !allow_smem(plan::plan_kernel, g_lim_plan, smp, false)) ||
            !allow_smem(split::split_kernel, g_lim_split, sms, false))
            return LB_ECUDA;
        rc = LB_OK;
        if (with_plan)
            rc = launch_kernel("plan", plan::plan_kernel, dim3(nbatch), dim3(plan::THREADS), smp, s, cnt_pred, G, E,
                               N, L, static_cast<uint8_t *>(plan), stride);
        if (rc == LB_OK)
            rc = launch_kernel("split", split::split_kernel, dim3(nbatch), dim3(split::THREADS), sms, s, cnt,
                               static_cast<const uint8_t *>(plan), stride, G, E, N, passes, tok, mass, loads,
                               passes_run);
        if (rc == LB_OK) rc = launch_prep(a, nbatch, smt, s, "assign prep");
    }
    if (rc != LB_OK || T == 0) return rc;
    return launch_kernel("assign scatter", assign::scatter_kernel, dim3(scatter_grid_x(T, k, G, nw, a.slices, a.cta_blocks != 0), nbatch),
                         dim3(nw * 32), sm2, s, a);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Fused count + split + assign (one cluster launch per batch of problems).
namespace {

// CTAs per problem: about one per 4096 assignments, a power of two up to 16
// that divides G or that G divides (so slices are whole blocks or equal parts
// of one), and 1 when nothing fits.
int solve_cluster(int T, int k, int G, int sms, int nbatch) {
    long long items = static_cast<long long>(T) * k;
    int C = 1;
    while (C < 16 && items / (2LL * C) >= 4096 && static_cast<long long>(nbatch) * C * 2 <= 2LL * sms) C *= 2;
    while (C > 1 && !((C <= G && G % C == 0) || (C > G && C % G == 0))) C >>= 1;
    return C;
}

}  // namespace

extern "C" int lb_solve(const int32_t *ids, const void *plan, int nbatch, int T, int k, int G, int E, int N,
                        int passes, int32_t *cnt, int32_t *tok, int32_t *mass, int32_t *loads,
                        int32_t *passes_run, int32_t *dest, int32_t *perm, int32_t *offs, void *workspace,
                        size_t workspace_bytes, void *stream) {
    if (nbatch < 1 || nbatch > 65535 || T < 0 || k < 1 || k > LB_MAX_K || !plan_shape_ok(G, E, N, 0) ||
        T % G != 0 || passes < 0 || passes > 4096)
        return LB_EINVAL;
    if (!plan || !cnt || !offs || !loads || !passes_run || !workspace || !aligned(plan, 256) ||
        !aligned(workspace, 256))
        return LB_EINVAL;
    if (G * N > 0 && (!tok || !mass)) return LB_EINVAL;
    if (T > 0 && (!ids || !dest || !perm)) return LB_EINVAL;
    if (static_cast<long long>(T) * k * nbatch >= INT_MAX) return LB_EINVAL;
    if (workspace_bytes < lb_assign_workspace_bytes(nbatch, T, k, G, E, N)) return LB_ENOSPACE;
    int C = solve_cluster(T, k, G, device_sms(), nbatch);
    // a larger cluster keeps fewer source blocks' counts per CTA
    while (solve::smem_bytes(G, E, N, C) > 224 * 1024 && C < 16 && G % (2 * C) == 0) C *= 2;
    const size_t smem = solve::smem_bytes(G, E, N, C);
    if (smem > 224 * 1024) {
        // does not fit one SM: the same work as three launches
        int rc = lb_count(ids, nbatch, T, k, E, G, cnt, stream);
        if (rc == LB_OK) rc = lb_split(cnt, plan, nbatch, G, E, N, passes, tok, mass, loads, passes_run, stream);
        if (rc == LB_OK)
            rc = lb_assign(ids, cnt, plan, tok, mass, nbatch, T, k, G, E, N, dest, perm, offs, workspace,
                           workspace_bytes, stream);
        return rc;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    assign::Args a;
    a.ids = ids;
    a.cnt = cnt;
    a.tok = tok;
    a.mass = mass;
    a.plan = static_cast<const uint8_t *>(plan);
    a.plan_stride = plan::layout(G, E, N).total;
    a.T = T;
    a.k = k;
    a.G = G;
    a.E = E;
    a.N = N;
    a.dest = dest;
    a.perm = perm;
    a.offs = offs;
    a.ws = static_cast<int32_t *>(workspace);
    a.ws_stride = assign::ws_words(G, E, N);
    static SmemLimit lim;
    if (!allow_smem(solve::solve_kernel, lim, smem, true)) return LB_ECUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(C, nbatch, 1);
    cfg.blockDim = dim3(solve::THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, solve::solve_kernel, a, passes, loads, passes_run);
    if (e != cudaSuccess) return cuda_fail(e, "cudaLaunchKernelEx(solve)");
    return launched("solve");
}

// ---------------------------------------------------------------------------
// Allocation-free variant of lb_assign.
//
// Some callers cannot hand this library a device workspace: a serving
// runtime that gave all device memory to its own arena at start-up, or a
// plain-C host loop with no device allocator of its own (and cudaMalloc
// would synchronize the device in the middle of a step).  For them the
// scratch lives in a file-scope device array of fixed size instead.  Every
// GPU that loads this library holds that array (LB_NOALLOC_SCRATCH_BYTES)
// until the process exits.
namespace {

constexpr size_t kNoAllocScratchBytes = LB_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) int32_t g_noalloc_scratch[kNoAllocScratchBytes / sizeof(int32_t)];

std::mutex g_noalloc_mu;
int32_t *g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (the array's
// name in host code is only a host-side stand-in).  Looked up once per
// device, with that device current.
int32_t *noalloc_scratch() {
    const int dev = current_device();
    if (dev < 0) return nullptr;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (g_noalloc_ptr[dev] == nullptr) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) {
            cuda_fail(e, "cudaGetSymbolAddress(scratch)");
            return nullptr;
        }
        g_noalloc_ptr[dev] = static_cast<int32_t *>(p);
    }
    return g_noalloc_ptr[dev];
}

}  // namespace

extern "C" int lb_assign_noalloc(const int32_t *ids, const int32_t *cnt, const void *plan, const int32_t *tok,
                                 const int32_t *mass, int nbatch, int T, int k, int G, int E, int N,
                                 int32_t *dest, int32_t *perm, int32_t *offs, void *stream) {
    // (G is range-checked by plan_shape_ok before T % G is taken)
    if (nbatch < 1 || nbatch > 65535 || T < 0 || k < 1 || k > LB_MAX_K || !plan_shape_ok(G, E, N, 0) || T % G != 0)
        return LB_EINVAL;
    if (!cnt || !plan || !offs || !aligned(plan, 256)) return LB_EINVAL;
    if (G * N > 0 && (!tok || !mass)) return LB_EINVAL;
    if (T > 0 && (!ids || !dest || !perm)) return LB_EINVAL;
    if (static_cast<long long>(T) * k * nbatch >= INT_MAX) return LB_EINVAL;
    if (assign::scatter_smem_bytes(G, E, N, 8) > 224 * 1024 || assign::prep_smem_bytes(G, E, N) > 224 * 1024)
        return LB_EINVAL;
    const size_t need = lb_assign_workspace_bytes(nbatch, T, k, G, E, N);
    if (need > kNoAllocScratchBytes) {
        std::snprintf(g_last_error, sizeof g_last_error,
                      "lb_assign_noalloc needs %zu bytes of scratch, more than its fixed %zu; use lb_assign", need,
                      kNoAllocScratchBytes);
        return LB_ENOSPACE;
    }
    int32_t *scratch = noalloc_scratch();
    if (scratch == nullptr) return LB_ECUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    assign::Args a;
    a.ids = ids;
    a.cnt = cnt;
    a.tok = tok;
    a.mass = mass;
    a.plan = static_cast<const uint8_t *>(plan);
    a.plan_stride = plan::layout(G, E, N).total;
    a.T = T;
    a.k = k;
    a.G = G;
    a.E = E;
    a.N = N;
    a.dest = dest;
    a.perm = perm;
    a.offs = offs;
    a.ws = scratch;
    a.ws_stride = assign::ws_words(G, E, N);
    const int nw = scatter_shape(a, nbatch);
    if (!allow_smem(assign::scatter_kernel, g_lim_scatter, assign::scatter_smem_bytes(G, E, N, nw), false))
        return LB_ECUDA;
    if (launch_prep(a, nbatch, assign::prep_smem_bytes(G, E, N), s, "assign prep (noalloc)") != LB_OK)
        return LB_ECUDA;
    if (T == 0) return LB_OK;
    return launch_kernel("assign scatter (noalloc)", assign::scatter_kernel, dim3(scatter_grid_x(T, k, G, nw, a.slices, a.cta_blocks != 0), nbatch),
                         dim3(nw * 32), assign::scatter_smem_bytes(G, E, N, nw), s, a);
}
