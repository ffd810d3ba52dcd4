// spec_verify.cu -- host side of libspecverify.so: argument checks, the
// piece plan and workspace layout, launches of K1 (row statistics), K2a
// (acceptance scan) and K2b (final draw), and the extern "C" entry points
// declared in include/spec_verify.h.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>

#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include "spec_verify.h"
#include "sv_common.cuh"
#include "sv_row_stats.cuh"
#include "sv_verify_scan.cuh"
#include "sv_verify_draw.cuh"
#include "sv_verify_cluster.cuh"

namespace sv {
namespace {

constexpr int kTmaConsumerWarps = SV_TMA_CONSUMER_WARPS;
constexpr int kTmaStages = SV_TMA_STAGES;
constexpr int kLdgThreads = 256;
// Share of the pieces the bulk-copy row-statistics kernel splits statically
// (the rest is handed out piece by piece).
#ifndef SV_STATIC_PCT
#define SV_STATIC_PCT 50
#endif
constexpr int kMaxDevices = 64;
constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;

struct DeviceInfo {
    int sm_count = 0;
    int max_smem_optin = 0;
    bool ready = false;
};

DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mutex;

// Fixed scratch of spec_verify_static_scratch (see the header): one array per
// device, holding the workspace of the same kernels.  Host code may only use
// the device address looked up with cudaGetSymbolAddress (with the device
// current), cached per device together with the unique id of the context it
// was looked up in: when the device's context is replaced (cudaDeviceReset
// and a new context), the id changes and the address is looked up again.
static __device__ __align__(256) unsigned char g_static_scratch[SV_STATIC_SCRATCH_BYTES];

struct ScratchAddr {
    void* addr = nullptr;
    unsigned long long ctx_id = 0;
};
ScratchAddr g_static_scratch_addr[kMaxDevices];

// Unique id of the calling thread's current context (driver entry points
// looked up through the runtime, so the library needs no link to the driver
// library); 0 when there is none or the driver cannot tell.
unsigned long long current_context_id() {
    using GetCurrent = int (*)(void**);
    using GetId = int (*)(void*, unsigned long long*);
    static GetCurrent get_current = nullptr;
    static GetId get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<GetCurrent>(f);
        f = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<GetId>(f);
    });
    if (!get_current || !get_id) return 0;
    void* ctx = nullptr;
    unsigned long long id = 0;
    if (get_current(&ctx) != 0 || !ctx || get_id(ctx, &id) != 0) return 0;
    return id;
}

cudaError_t static_scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    const unsigned long long id = current_context_id();
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    ScratchAddr& c = g_static_scratch_addr[dev];
    if (!c.addr || id == 0 || c.ctx_id != id) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_static_scratch);  // with device `dev` current
        if (e != cudaSuccess) return e;
        c.addr = p;
        c.ctx_id = current_context_id();                 // the context the lookup made current
    }
    *out = c.addr;
    return cudaSuccess;
}

cudaError_t device_info(DeviceInfo** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    DeviceInfo& d = g_dev[dev];
    if (!d.ready) {
        e = cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        e = cudaDeviceGetAttribute(&d.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        if (e != cudaSuccess) return e;
        d.ready = true;
    }
    *out = &d;
    return cudaSuccess;
}

// Launch setup of a kernel, done once per context and kernel (later calls
// find it in small tables): the kernel asks for the largest shared-memory
// carveout -- so consecutive kernels find the SMs in the same L1 /
// shared-memory split and a dependent grid's CTAs can move in while the
// previous grid drains -- and opts into the largest dynamic shared memory
// any call has needed so far (the attribute only grows, so every earlier
// size still launches); *per_sm (if given) receives the resident blocks per
// SM for this size and block size.  Without a context id (the driver cannot
// tell) nothing is cached.
struct SetupKey {
    unsigned long long ctx;
    const void* kernel;
    size_t smem;
    int threads;
    bool operator<(const SetupKey& o) const {
        return std::tie(ctx, kernel, smem, threads) < std::tie(o.ctx, o.kernel, o.smem, o.threads);
    }
};
std::map<std::pair<unsigned long long, const void*>, size_t> g_smem_set;  // largest opt-in set per kernel
std::map<SetupKey, int> g_resident;                                        // resident blocks per SM
std::mutex g_setup_mutex;
constexpr size_t kMaxSetupEntries = 4096;

template <typename Kernel>
cudaError_t kernel_setup(Kernel k, size_t smem, int threads, int* per_sm) {
    const SetupKey key{current_context_id(), reinterpret_cast<const void*>(k), smem, threads};
    const auto kk = std::make_pair(key.ctx, key.kernel);
    bool attrs_ok = false;
    int n = -1;
    if (key.ctx != 0) {
        std::lock_guard<std::mutex> lock(g_setup_mutex);
        const auto a = g_smem_set.find(kk);
        attrs_ok = a != g_smem_set.end() && a->second >= smem;
        const auto it = g_resident.find(key);
        if (it != g_resident.end()) n = it->second;
    }
    cudaError_t e = cudaSuccess;
    if (!attrs_ok) {
        e = cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
        if (e == cudaSuccess) e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        if (e != cudaSuccess) return e;
    }
    if (n < 0 && (e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k, threads, smem)) != cudaSuccess) return e;
    if (key.ctx != 0) {
        std::lock_guard<std::mutex> lock(g_setup_mutex);
        if (g_resident.size() >= kMaxSetupEntries) g_resident.clear();
        g_resident[key] = n;
        if (!attrs_ok) {
            size_t& m = g_smem_set[kk];
            if (smem > m) m = smem;
        }
    }
    if (per_sm) *per_sm = n;
    return cudaSuccess;
}

struct Plan {
    int P = 1;       // pieces per row
    int PE = 4096;   // elements per piece
    int es = 4;      // element size
    int64_t stride = 0;
};

// Rows are cut into pieces of kPieceBytes (the last one ragged); a piece
// starts on a 16-byte boundary of an aligned row.
Plan make_plan(const sv_shape& s) {
    Plan p;
    p.es = s.dtype == SV_BF16 ? 2 : 4;
    p.stride = s.row_stride ? s.row_stride : s.V;
    p.PE = kPieceBytes / p.es;
    p.P = static_cast<int>((int64_t(s.V) + p.PE - 1) / p.PE);
    return p;
}

bool shape_ok(const sv_shape* s, sv_status* why) {
    if (!s) { *why = SV_EINVAL; return false; }
    if (s->B < 0 || s->k_max < 0 || s->V < 1) { *why = SV_EINVAL; return false; }
    if (s->dtype != SV_F32 && s->dtype != SV_BF16) { *why = SV_EUNSUPPORTED; return false; }
    if (s->k_max > SV_MAX_K || s->V > SV_MAX_V) { *why = SV_EUNSUPPORTED; return false; }
    const int64_t stride = s->row_stride ? s->row_stride : s->V;
    if (stride < s->V) { *why = SV_EINVAL; return false; }
    return true;
}

size_t align256(size_t n) { return (n + 255) & ~size_t(255); }

// Control words, zeroed (zero_ctrl_kernel) before every call: [0] residual
// draws queued, [1] one-piece draws queued, [2 + l] the pieces the l-th
// row-statistics launch (up to 4096 requests each) has handed out.
int64_t stats_launches(const sv_shape& s) {
    return (int64_t(s.B) + kMaxRequestsPerLaunch - 1) / kMaxRequestsPerLaunch;
}
int64_t ctrl_ints(const sv_shape& s) { return 2 + stats_launches(s); }

// Workspace: the row-statistics partials, the control words, then the draw
// queue the scan kernel fills and the draw kernel drains.
struct WsLayout {
    size_t partials, ctrl, res_req, one_req, res_lost, seg, total;
};

WsLayout ws_layout(const sv_shape& s, const Plan& p) {
    const size_t B = size_t(s.B);
    WsLayout l{};
    size_t off = 0;
    l.partials = off; off += align256(B * size_t(2 * s.k_max + 1) * size_t(p.P) * sizeof(float2));
    l.ctrl = off;     off += align256(ctrl_ints(s) * sizeof(int32_t));
    l.res_req = off;  off += align256(B * sizeof(DrawReq));
    l.one_req = off;  off += align256(B * sizeof(DrawReq));
    l.res_lost = off; off += align256(B * sizeof(int32_t));
    l.seg = off;      off += align256(B * size_t(p.P) * kSegsPerPiece * sizeof(float));
    l.total = off;
    return l;
}

size_t workspace_bytes_for(const sv_shape& s, const Plan& p) { return ws_layout(s, p).total; }

bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

// NVTX range around the launches of one kernel (header-only NVTX: a no-op
// unless a profiler is attached), so timelines name the phases of a call.
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
};

// Zeroes the control words.  It is itself a programmatic dependent of
// whatever precedes the call on the stream (the previous call's last kernel
// lets it in early), so it first waits for that work to complete; then it
// lets the row-statistics kernel launch (as its programmatic dependent: that
// kernel waits for this grid only before its first ticket, so its prologue
// and first copies overlap this one) and zeroes the words.
__global__ void zero_ctrl_kernel(int32_t* ctrl, int n) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");
    for (int i = threadIdx.x; i < n; i += blockDim.x) ctrl[i] = 0;
}

template <typename T, bool kGreedy>
cudaError_t launch_stats(const StatsParams& base, int B, int variant, const DeviceInfo& dev, cudaStream_t st) {
    for (int b0 = 0; b0 < B; b0 += kMaxRequestsPerLaunch) {
        StatsParams prm = base;
        prm.b0 = b0;
        prm.dyn_ticket = base.dyn_ticket + b0 / kMaxRequestsPerLaunch;
        prm.nB = B - b0 < kMaxRequestsPerLaunch ? B - b0 : kMaxRequestsPerLaunch;
        const int rows_max = prm.use_draft ? 2 * prm.k_max + 1 : prm.k_max + 1;
        const int64_t items_upper = int64_t(prm.nB) * rows_max * prm.P;
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.stream = st;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        cudaError_t e;
        if (variant == SV_STATS_TMA) {
            auto k = row_stats_tma_kernel<T, kGreedy, kTmaConsumerWarps, kTmaStages>;
            const size_t smem = TmaSmem<kTmaConsumerWarps, kTmaStages>::bytes(prm.nB);
            // one wave of resident CTAs (a long request list can make the
            // row prefix in shared memory lower the occupancy)
            int per_sm = 0;
            if ((e = kernel_setup(k, smem, (kTmaConsumerWarps + 1) * 32, &per_sm)) != cudaSuccess) return e;
            per_sm = per_sm < 1 ? 1 : (per_sm > TmaCtasPerSm<T>::value ? TmaCtasPerSm<T>::value : per_sm);
            const int64_t cap = int64_t(dev.sm_count) * per_sm;
            const int64_t grid = items_upper < cap ? items_upper : cap;
            cfg.gridDim = dim3(static_cast<unsigned>(grid));
            cfg.blockDim = dim3((kTmaConsumerWarps + 1) * 32);
            cfg.dynamicSmemBytes = smem;
            e = cudaLaunchKernelEx(&cfg, k, prm);
        } else {
            auto k = variant == SV_STATS_VEC16 ? row_stats_ldg_kernel<T, kGreedy, true, kLdgThreads>
                                               : row_stats_ldg_kernel<T, kGreedy, false, kLdgThreads>;
            const size_t smem = 4 * size_t(prm.nB + 1);
            int per_sm = 0;
            if ((e = kernel_setup(k, smem, kLdgThreads, &per_sm)) != cudaSuccess) return e;
            if (per_sm < 1) per_sm = 1;
            const int64_t cap = int64_t(dev.sm_count) * per_sm;
            const int64_t grid = items_upper < cap ? items_upper : cap;
            cfg.gridDim = dim3(static_cast<unsigned>(grid));
            cfg.blockDim = dim3(kLdgThreads);
            cfg.dynamicSmemBytes = smem;
            e = cudaLaunchKernelEx(&cfg, k, prm);
        }
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

// K2a (one CTA per request), then for sampling K2b (persistent, one wave) and,
// with draft logits, K2c (one warp per possible residual draw), each a
// programmatic dependent of the kernel before it.
// Largest cluster size the cluster kernel uses with `smem` bytes of dynamic
// shared memory: 16 when the device can place at least one such cluster
// (non-portable size, opted into here), else the portable 8.  Cached per
// context and size.
std::map<std::pair<unsigned long long, size_t>, int> g_cluster_max;

template <typename T>
cudaError_t cluster_max_ctas(size_t smem, int* cmax) {
    auto k = verify_cluster_kernel<T>;
    const auto key = std::make_pair(current_context_id(), smem);
    if (key.first != 0) {
        std::lock_guard<std::mutex> lock(g_setup_mutex);
        const auto it = g_cluster_max.find(key);
        if (it != g_cluster_max.end()) {
            *cmax = it->second;
            return cudaSuccess;
        }
    }
    // the kernel's shared-memory attributes first: the query below uses them
    if (const cudaError_t e = kernel_setup(k, smem, kScanThreads, nullptr); e != cudaSuccess) return e;
    int result = kClusterPortableCtas;
    if (cudaFuncSetAttribute(k, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess) {
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = kClusterMaxCtas;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(kClusterMaxCtas);
        cfg.blockDim = dim3(kScanThreads);
        cfg.dynamicSmemBytes = smem;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, k, &cfg) == cudaSuccess && n > 0) result = kClusterMaxCtas;
    }
    (void)cudaGetLastError();  // a refused query leaves no error behind
    if (key.first != 0) {
        std::lock_guard<std::mutex> lock(g_setup_mutex);
        g_cluster_max[key] = result;
    }
    *cmax = result;
    return cudaSuccess;
}

// AUTO's choice: the cluster path when the batch's CTAs fit in half of one
// resident wave of the cluster kernel (clusters are placed whole, inside one
// GPC), so every request's cluster starts at once.
template <typename T>
cudaError_t cluster_fits(int B, int k_max, int P, const DeviceInfo& dev, bool* fits) {
    int per_sm = 0, cmax = 0;
    const size_t smem = cluster_smem_bytes(k_max, P);
    cudaError_t e = kernel_setup(verify_cluster_kernel<T>, smem, kScanThreads, &per_sm);
    if (e == cudaSuccess) e = cluster_max_ctas<T>(smem, &cmax);
    if (e != cudaSuccess) return e;
    *fits = int64_t(B) * cluster_ctas(P, cmax) * 2 <= int64_t(per_sm) * dev.sm_count;
    return cudaSuccess;
}

// The cluster path for a sampling call: one cluster of cluster_ctas(P) CTAs
// per request, as a programmatic dependent of the row statistics.  AUTO
// takes it when the batch's CTAs fit in half of one resident wave (clusters
// are placed whole, inside one GPC).
template <typename T>
cudaError_t launch_cluster(const ScanParams& sp, const DrawParams& dp, int B, int path, const DeviceInfo& dev,
                           cudaStream_t st, bool* launched) {
    *launched = false;
    if (path == SV_DRAW_QUEUE) return cudaSuccess;
    auto k = verify_cluster_kernel<T>;
    const size_t smem = cluster_smem_bytes(dp.k_max, dp.P);
    int cmax = 0;
    if (const cudaError_t e = cluster_max_ctas<T>(smem, &cmax); e != cudaSuccess) return e;
    const int C = cluster_ctas(dp.P, cmax);
    if (path == SV_DRAW_AUTO) {
        bool fits = false;
        const cudaError_t e = cluster_fits<T>(B, dp.k_max, dp.P, dev, &fits);
        if (e != cudaSuccess || !fits) return e;
    } else if (const cudaError_t e = kernel_setup(k, smem, kScanThreads, nullptr); e != cudaSuccess) {
        return e;
    }
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = static_cast<unsigned>(C);
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(int64_t(B) * C));
    cfg.blockDim = dim3(kScanThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, k, sp, dp);
    if (e != cudaSuccess) return e;
    *launched = true;
    return cudaSuccess;
}

template <typename T>
cudaError_t launch_scan_draw(const ScanParams& sp, const DrawParams& dp, const SelectParams& cp, int B, bool draw,
                             int path, const DeviceInfo& dev, cudaStream_t st) {
    if (draw) {
        bool launched = false;
        const cudaError_t e = launch_cluster<T>(sp, dp, B, path, dev, st, &launched);
        if (e != cudaSuccess || launched) return e;
    }
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    {
        auto k = verify_scan_kernel<T>;
        const size_t smem = scan_smem_bytes(sp.k_max, sp.P);
        cudaError_t e = kernel_setup(k, smem, kScanThreads, nullptr);
        if (e != cudaSuccess) return e;
        cfg.gridDim = dim3(static_cast<unsigned>(B));
        cfg.blockDim = dim3(kScanThreads);
        cfg.dynamicSmemBytes = smem;
        if ((e = cudaLaunchKernelEx(&cfg, k, sp)) != cudaSuccess) return e;
    }
    if (!draw) return cudaSuccess;
    {
        auto k = verify_draw_kernel<T>;
        // persistent: at most one wave of resident CTAs, and no more than the
        // largest possible number of tasks
        int per_sm = 0;
        cudaError_t e = kernel_setup(k, kDrawSmemBytes, kDrawThreads, &per_sm);
        if (e != cudaSuccess) return e;
        per_sm = per_sm < 1 ? 1 : (per_sm > kDrawCtasPerSm ? kDrawCtasPerSm : per_sm);
        const int64_t cap = int64_t(dev.sm_count) * per_sm;
        const int64_t max_tasks = int64_t(B) * (dp.P + 1);
        cfg.gridDim = dim3(static_cast<unsigned>(max_tasks < cap ? max_tasks : cap));
        cfg.blockDim = dim3(kDrawThreads);
        cfg.dynamicSmemBytes = kDrawSmemBytes;
        if ((e = cudaLaunchKernelEx(&cfg, k, dp)) != cudaSuccess) return e;
    }
    // residual draws need draft logits: with one-hot q the queue holds none
    if (cp.draft == nullptr) return cudaSuccess;
    auto k = verify_select_kernel<T>;
    if (cudaError_t e = kernel_setup(k, 0, kSelectThreads, nullptr); e != cudaSuccess) return e;
    cfg.gridDim = dim3(static_cast<unsigned>((int64_t(B) + kSelectWarps - 1) / kSelectWarps));
    cfg.blockDim = dim3(kSelectThreads);
    cfg.dynamicSmemBytes = 0;
    return cudaLaunchKernelEx(&cfg, k, cp);
}

struct Call {
    const sv_shape* shape;
    const void* target;
    const void* draft;
    const int32_t* tokens;
    const int32_t* lens;
    const float* uniforms;
    float temperature;
    int greedy;
    int32_t* out_len;
    int32_t* out_tokens;
    float* out_lse_t;
    float* out_lse_d;
    float* out_p;
    float* out_q;
    void* workspace;
    size_t workspace_bytes;
    cudaStream_t stream;
    const sv_options* opts;
    bool stats_only;
    // acceptance simulation (stats_only with the acceptance outputs)
    bool accept_sim = false;
    float decay = 0.f;
    float* out_accept_prob = nullptr;
    float* out_expected_len = nullptr;
    int32_t* out_first_reject = nullptr;
    float* out_weights = nullptr;
};

template <typename T>
sv_status run_typed(const Call& a, const Plan& plan, const DeviceInfo& dev, int variant, bool rows_aligned) {
    const sv_shape& s = *a.shape;
    const bool greedy = a.greedy && !a.stats_only;
    const WsLayout wl = ws_layout(s, plan);
    unsigned char* ws = static_cast<unsigned char*>(a.workspace);
    int32_t* ctrl = reinterpret_cast<int32_t*>(ws + wl.ctrl);
    const float scale = greedy ? 1.f : static_cast<float>(kLog2e / static_cast<double>(a.temperature));

    ScanParams cp{};
    cp.target = static_cast<const unsigned char*>(a.target);
    cp.draft = greedy ? nullptr : static_cast<const unsigned char*>(a.draft);
    cp.tokens = a.tokens;
    cp.lens = a.lens;
    cp.uniforms = a.uniforms;
    cp.partials = reinterpret_cast<float2*>(ws + wl.partials);
    cp.out_len = a.out_len;
    cp.out_tokens = a.out_tokens;
    cp.out_lse_t = a.out_lse_t;
    cp.out_lse_d = a.out_lse_d;
    cp.out_p = a.out_p;
    cp.out_q = a.out_q;
    cp.out_accept_prob = a.out_accept_prob;
    cp.out_expected_len = a.out_expected_len;
    cp.out_first_reject = a.out_first_reject;
    cp.out_weights = a.out_weights;
    cp.decay = a.decay;
    cp.ctrl = ctrl;
    cp.res_req = reinterpret_cast<DrawReq*>(ws + wl.res_req);
    cp.one_req = reinterpret_cast<DrawReq*>(ws + wl.one_req);
    cp.res_lost = reinterpret_cast<int32_t*>(ws + wl.res_lost);
    cp.k_max = s.k_max;
    cp.V = s.V;
    cp.row_stride = plan.stride;
    cp.P = plan.P;
    cp.PE = plan.PE;
    cp.scale = scale;
    cp.greedy = greedy ? 1 : 0;
    cp.stats_only = a.stats_only ? 1 : 0;

    StatsParams sp{};
    sp.target = static_cast<const unsigned char*>(a.target);
    sp.draft = static_cast<const unsigned char*>(a.draft);
    sp.lens = a.lens;
    sp.partials = reinterpret_cast<float2*>(ws + wl.partials);
    sp.dyn_ticket = ctrl + 2;
    sp.static_pct = SV_STATIC_PCT;
    sp.k_max = s.k_max;
    sp.V = s.V;
    sp.row_stride = plan.stride;
    sp.P = plan.P;
    sp.PE = plan.PE;
    sp.scale = scale;
    sp.use_draft = (a.draft != nullptr && !greedy) ? 1 : 0;
    const int tmo = a.opts ? a.opts->wait_timeout_us : 0;
    sp.timeout_ns = tmo > 0 ? uint64_t(tmo) * 1000ull : kDefaultTimeoutNs;
    const int lost = a.opts ? a.opts->lost_copy_request : 0;
    sp.lost_copy_partial = lost > 0 ? int64_t(lost - 1) * (2 * s.k_max + 1) * plan.P : -1;

    cudaError_t e = kernel_setup(zero_ctrl_kernel, 0, 32, nullptr);
    if (e != cudaSuccess) return SV_ECUDA;
    {
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(1);
        cfg.blockDim = dim3(32);
        cfg.stream = a.stream;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if ((e = cudaLaunchKernelEx(&cfg, zero_ctrl_kernel, ctrl, static_cast<int>(ctrl_ints(s)))) != cudaSuccess)
            return SV_ECUDA;
    }
    if (a.opts && a.opts->event_stats_begin)
        if ((e = cudaEventRecord(static_cast<cudaEvent_t>(a.opts->event_stats_begin), a.stream)) != cudaSuccess)
            return SV_ECUDA;
    {
        NvtxRange range("spec_verify: row statistics");
        e = greedy ? launch_stats<T, true>(sp, s.B, variant, dev, a.stream)
                   : launch_stats<T, false>(sp, s.B, variant, dev, a.stream);
    }
    if (e != cudaSuccess) return SV_ECUDA;
    if (a.opts && a.opts->event_stats_end)
        if ((e = cudaEventRecord(static_cast<cudaEvent_t>(a.opts->event_stats_end), a.stream)) != cudaSuccess)
            return SV_ECUDA;

    DrawParams dp{};
    dp.B = s.B;
    dp.target = sp.target;
    dp.draft = cp.draft;
    dp.partials = sp.partials;
    dp.ctrl = ctrl;
    dp.res_req = cp.res_req;
    dp.one_req = cp.one_req;
    dp.res_lost = cp.res_lost;
    dp.seg = reinterpret_cast<float*>(ws + wl.seg);
    dp.out_len = a.out_len;
    dp.out_tokens = a.out_tokens;
    dp.k_max = s.k_max;
    dp.V = s.V;
    dp.row_stride = plan.stride;
    dp.P = plan.P;
    dp.PE = plan.PE;
    dp.scale = scale;
    dp.rows_aligned = rows_aligned ? 1 : 0;
    dp.timeout_ns = sp.timeout_ns;
    const int lost_draw = a.opts ? a.opts->lost_draw_request : 0;
    dp.lost_draw_b = lost_draw > 0 ? lost_draw - 1 : -1;
    SelectParams xp{};
    xp.B = s.B;
    xp.target = dp.target;
    xp.draft = dp.draft;
    xp.partials = dp.partials;
    xp.ctrl = ctrl;
    xp.res_req = dp.res_req;
    xp.seg = dp.seg;
    xp.res_lost = dp.res_lost;
    xp.out_len = a.out_len;
    xp.out_tokens = a.out_tokens;
    xp.k_max = s.k_max;
    xp.V = s.V;
    xp.row_stride = plan.stride;
    xp.P = plan.P;
    xp.PE = plan.PE;
    xp.scale = scale;
    xp.rows_aligned = dp.rows_aligned;
    {
        NvtxRange range("spec_verify: scan, draw, selection");
        e = launch_scan_draw<T>(cp, dp, xp, s.B, !greedy && !a.stats_only, a.opts ? a.opts->draw_path : SV_DRAW_AUTO,
                                dev, a.stream);
    }
    return e == cudaSuccess ? SV_OK : SV_ECUDA;
}

sv_status run(const Call& a) {
    sv_status why = SV_OK;
    if (!shape_ok(a.shape, &why)) return why;
    const sv_shape& s = *a.shape;
    if (a.opts) {
        for (int i = 0; i < 5; ++i)
            if (a.opts->reserved[i] != 0) return SV_EINVAL;
        if (a.opts->draw_path < SV_DRAW_AUTO || a.opts->draw_path > SV_DRAW_CLUSTER) return SV_EINVAL;
        if (a.opts->lost_copy_request < 0 || a.opts->lost_copy_request > s.B) return SV_EINVAL;
        if (a.opts->lost_draw_request < 0 || a.opts->lost_draw_request > s.B) return SV_EINVAL;
        if (a.opts->stats_kernel < SV_STATS_AUTO || a.opts->stats_kernel > SV_STATS_SCALAR) return SV_EINVAL;
        if (a.opts->wait_timeout_us < 0) return SV_EINVAL;
    }
    if (s.B == 0) return SV_OK;
    const bool greedy = a.greedy && !a.stats_only;
    if (!a.target) return SV_EINVAL;
    if (s.k_max > 0 && !a.tokens) return SV_EINVAL;
    if (a.accept_sim) {
        if (!a.out_accept_prob || !a.out_expected_len) return SV_EINVAL;
        if ((a.out_first_reject || a.out_weights) && !a.uniforms) return SV_EINVAL;
        if (!(a.decay >= 0.f && a.decay <= 1.f)) return SV_EINVAL;
    } else if (a.stats_only) {
        if (!a.out_lse_t) return SV_EINVAL;
    } else {
        if (!a.out_len || !a.out_tokens) return SV_EINVAL;
    }
    if (!greedy) {
        if (!(a.temperature > 0.f) || !std::isfinite(a.temperature)) return SV_EINVAL;
        if (!a.stats_only && !a.uniforms) return SV_EINVAL;
    }
    const Plan plan = make_plan(s);
    if (!a.workspace || a.workspace_bytes < workspace_bytes_for(s, plan)) return SV_EINVAL;
    if (!aligned16(a.workspace)) return SV_EINVAL;

    DeviceInfo* dev = nullptr;
    if (device_info(&dev) != cudaSuccess) return SV_ECUDA;

    // Kernel choice: the bulk-copy and vector paths need every row start on a
    // 16-byte boundary.
    const bool rows_aligned = aligned16(a.target) && (a.draft == nullptr || greedy || aligned16(a.draft)) &&
                              ((plan.stride * plan.es) % 16 == 0);
    int variant = a.opts ? a.opts->stats_kernel : SV_STATS_AUTO;
    if (variant == SV_STATS_AUTO) variant = rows_aligned ? SV_STATS_TMA : SV_STATS_SCALAR;
    if ((variant == SV_STATS_TMA || variant == SV_STATS_VEC16) && !rows_aligned) return SV_EINVAL;
    if (a.opts && a.opts->lost_copy_request != 0 && variant != SV_STATS_TMA) return SV_EUNSUPPORTED;

    return s.dtype == SV_BF16 ? run_typed<bf16_bits>(a, plan, *dev, variant, rows_aligned)
                              : run_typed<float>(a, plan, *dev, variant, rows_aligned);
}

struct HostLayout {
    size_t target, draft, tokens, lens, uniforms, out_len, out_tokens, total;
};

HostLayout host_layout(const sv_shape& s, bool has_draft, bool has_lens) {
    const Plan plan = make_plan(s);
    HostLayout h{};
    const size_t B = size_t(s.B), K = size_t(s.k_max), es = size_t(plan.es), st = size_t(plan.stride);
    size_t off = 0;
    h.target = off; off += align256(B * (K + 1) * st * es);
    h.draft = off; off += has_draft ? align256(B * K * st * es) : 0;
    h.tokens = off; off += align256(B * K * 4);
    h.lens = off; off += has_lens ? align256(B * 4) : 0;
    h.uniforms = off; off += align256(B * (K + 1) * 4);
    h.out_len = off; off += align256(B * 4);
    h.out_tokens = off; off += align256(B * (K + 1) * 4);
    h.total = off;
    return h;
}

}  // namespace
}  // namespace sv

extern "C" {

size_t spec_verify_workspace_bytes(const sv_shape* shape) {
    sv_status why;
    if (!sv::shape_ok(shape, &why)) return 0;
    return sv::workspace_bytes_for(*shape, sv::make_plan(*shape));
}

sv_status spec_verify_ex(const sv_shape* shape, const void* target_logits, const void* draft_logits,
                         const int32_t* draft_tokens, const int32_t* draft_lens, const float* uniforms,
                         float temperature, int32_t greedy, int32_t* out_accept_len, int32_t* out_tokens,
                         void* workspace, size_t workspace_bytes, void* stream, const sv_options* opts) {
    sv::Call a{shape,      target_logits, draft_logits, draft_tokens,   draft_lens,
               uniforms,   temperature,   greedy != 0,  out_accept_len, out_tokens,
               nullptr,    nullptr,       nullptr,      nullptr,        workspace,
               workspace_bytes, static_cast<cudaStream_t>(stream), opts, false};
    return sv::run(a);
}

sv_status spec_verify(const sv_shape* shape, const void* target_logits, const void* draft_logits,
                      const int32_t* draft_tokens, const int32_t* draft_lens, const float* uniforms,
                      float temperature, int32_t greedy, int32_t* out_accept_len, int32_t* out_tokens,
                      void* workspace, size_t workspace_bytes, void* stream) {
    return spec_verify_ex(shape, target_logits, draft_logits, draft_tokens, draft_lens, uniforms, temperature,
                          greedy, out_accept_len, out_tokens, workspace, workspace_bytes, stream, nullptr);
}

sv_status spec_verify_stats(const sv_shape* shape, const void* target_logits, const void* draft_logits,
                            const int32_t* draft_tokens, const int32_t* draft_lens, float temperature,
                            float* out_lse_target, float* out_lse_draft, float* out_p, float* out_q,
                            void* workspace, size_t workspace_bytes, void* stream, const sv_options* opts) {
    sv::Call a{shape,          target_logits, draft_logits, draft_tokens, draft_lens,
               nullptr,        temperature,   false,        nullptr,      nullptr,
               out_lse_target, out_lse_draft, out_p,        out_q,        workspace,
               workspace_bytes, static_cast<cudaStream_t>(stream), opts, true};
    return sv::run(a);
}

sv_status spec_verify_accept_sim(const sv_shape* shape, const void* target_logits, const void* draft_logits,
                                 const int32_t* draft_tokens, const int32_t* draft_lens, const float* uniforms,
                                 float temperature, float decay, float* out_accept_prob, float* out_expected_len,
                                 int32_t* out_first_reject, float* out_weights, void* workspace,
                                 size_t workspace_bytes, void* stream) {
    sv::Call a{shape,    target_logits, draft_logits, draft_tokens, draft_lens,
               uniforms, temperature,   false,        nullptr,      nullptr,
               nullptr,  nullptr,       nullptr,      nullptr,      workspace,
               workspace_bytes, static_cast<cudaStream_t>(stream), nullptr, true};
    a.accept_sim = true;
    a.decay = decay;
    a.out_accept_prob = out_accept_prob;
    a.out_expected_len = out_expected_len;
    a.out_first_reject = out_first_reject;
    a.out_weights = out_weights;
    return sv::run(a);
}

size_t spec_verify_host_staging_bytes(const sv_shape* shape, int32_t has_draft, int32_t has_lens) {
    sv_status why;
    if (!sv::shape_ok(shape, &why)) return 0;
    return sv::host_layout(*shape, has_draft != 0, has_lens != 0).total;
}

sv_status spec_verify_host(const sv_shape* shape, const void* h_target_logits, const void* h_draft_logits,
                           const int32_t* h_draft_tokens, const int32_t* h_draft_lens, const float* h_uniforms,
                           float temperature, int32_t greedy, int32_t* h_out_accept_len, int32_t* h_out_tokens,
                           void* device_staging, size_t staging_bytes, void* workspace, size_t workspace_bytes,
                           void* stream) {
    sv_status why;
    if (!sv::shape_ok(shape, &why)) return why;
    const sv_shape& s = *shape;
    if (s.B == 0) return SV_OK;
    const bool has_draft = h_draft_logits != nullptr && !greedy;
    const bool has_lens = h_draft_lens != nullptr;
    const sv::HostLayout h = sv::host_layout(s, has_draft, has_lens);
    if (!device_staging || staging_bytes < h.total || !sv::aligned16(device_staging)) return SV_EINVAL;
    if (!h_target_logits || !h_out_accept_len || !h_out_tokens) return SV_EINVAL;
    if (s.k_max > 0 && !h_draft_tokens) return SV_EINVAL;
    if (!greedy && !h_uniforms) return SV_EINVAL;
    const sv::Plan plan = sv::make_plan(s);
    const size_t B = size_t(s.B), K = size_t(s.k_max), es = size_t(plan.es), st = size_t(plan.stride);
    unsigned char* base = static_cast<unsigned char*>(device_staging);
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    auto h2d = [&](size_t off, const void* src, size_t n) {
        return n ? cudaMemcpyAsync(base + off, src, n, cudaMemcpyHostToDevice, cs) : cudaSuccess;
    };
    // Logits: only the rows the kernels read -- target rows 0..L_b and draft
    // rows 0..L_b-1 of request b, L_b clamped to [0, k_max] as the
    // row-statistics kernel clamps it -- one copy per contiguous run (the
    // rows of consecutive requests with L_b = k_max join up).  Without
    // draft_lens every row is read.  Staging rows that are not copied keep
    // whatever they held; no kernel reads them.
    const size_t trow = st * es;
    cudaError_t e = cudaSuccess;
    if (!has_lens) {
        e = h2d(h.target, h_target_logits, B * (K + 1) * trow);
        if (e == cudaSuccess && has_draft) e = h2d(h.draft, h_draft_logits, B * K * trow);
    } else {
        // run-length merge of [offset, offset + n) ranges of one tensor
        struct Run {
            size_t off = 0, n = 0;
        };
        auto flush = [&](Run& r, size_t dst_base, const void* src_base) {
            cudaError_t err = cudaSuccess;
            if (r.n) err = h2d(dst_base + r.off, static_cast<const unsigned char*>(src_base) + r.off, r.n);
            r = Run{};
            return err;
        };
        auto add = [&](Run& r, size_t off, size_t n, size_t dst_base, const void* src_base) {
            if (n == 0) return cudaSuccess;
            if (r.n && r.off + r.n == off) {
                r.n += n;
                return cudaSuccess;
            }
            const cudaError_t err = flush(r, dst_base, src_base);
            r.off = off;
            r.n = n;
            return err;
        };
        Run rt, rd;
        for (size_t b = 0; b < B && e == cudaSuccess; ++b) {
            const int32_t l = h_draft_lens[b];
            const size_t L = l < 0 ? 0 : (size_t(l) > K ? K : size_t(l));
            e = add(rt, b * (K + 1) * trow, (L + 1) * trow, h.target, h_target_logits);
            if (e == cudaSuccess && has_draft) e = add(rd, b * K * trow, L * trow, h.draft, h_draft_logits);
        }
        if (e == cudaSuccess) e = flush(rt, h.target, h_target_logits);
        if (e == cudaSuccess && has_draft) e = flush(rd, h.draft, h_draft_logits);
    }
    if (e == cudaSuccess && K) e = h2d(h.tokens, h_draft_tokens, B * K * 4);
    if (e == cudaSuccess && has_lens) e = h2d(h.lens, h_draft_lens, B * 4);
    if (e == cudaSuccess && !greedy) e = h2d(h.uniforms, h_uniforms, B * (K + 1) * 4);
    if (e != cudaSuccess) return SV_ECUDA;
    sv_status r = spec_verify(shape, base + h.target, has_draft ? base + h.draft : nullptr,
                              reinterpret_cast<const int32_t*>(base + h.tokens),
                              has_lens ? reinterpret_cast<const int32_t*>(base + h.lens) : nullptr,
                              greedy ? nullptr : reinterpret_cast<const float*>(base + h.uniforms), temperature,
                              greedy, reinterpret_cast<int32_t*>(base + h.out_len),
                              reinterpret_cast<int32_t*>(base + h.out_tokens), workspace, workspace_bytes, stream);
    if (r != SV_OK) return r;
    e = cudaMemcpyAsync(h_out_accept_len, base + h.out_len, B * 4, cudaMemcpyDeviceToHost, cs);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(h_out_tokens, base + h.out_tokens, B * (K + 1) * 4, cudaMemcpyDeviceToHost, cs);
    return e == cudaSuccess ? SV_OK : SV_ECUDA;
}

sv_status spec_verify_static_scratch(const sv_shape* shape, const void* target_logits, const void* draft_logits,
                                     const int32_t* draft_tokens, const int32_t* draft_lens, const float* uniforms,
                                     float temperature, int32_t greedy, int32_t* out_accept_len,
                                     int32_t* out_tokens, void* stream) {
    sv_status why;
    if (!sv::shape_ok(shape, &why)) return why;
    if (sv::workspace_bytes_for(*shape, sv::make_plan(*shape)) > SV_STATIC_SCRATCH_BYTES) return SV_ESCRATCH;
    void* scratch = nullptr;
    if (sv::static_scratch_address(&scratch) != cudaSuccess) return SV_ECUDA;
    return spec_verify_ex(shape, target_logits, draft_logits, draft_tokens, draft_lens, uniforms, temperature,
                          greedy, out_accept_len, out_tokens, scratch, SV_STATIC_SCRATCH_BYTES, stream, nullptr);
}

const char* spec_verify_status_string(sv_status status) {
    switch (status) {
        case SV_OK: return "ok";
        case SV_EINVAL: return "invalid argument";
        case SV_ECUDA: return "CUDA error";
        case SV_EUNSUPPORTED: return "unsupported shape or dtype";
        case SV_ESCRATCH: return "problem larger than the static scratch area (use spec_verify with a workspace)";
    }
    return "unknown status";
}

int32_t spec_verify_abi_version(void) { return SV_ABI_VERSION; }

int32_t spec_verify_auto_draw_path(const sv_shape* shape) {
    sv_status why;
    if (!sv::shape_ok(shape, &why)) return -1;
    sv::DeviceInfo* dev = nullptr;
    if (sv::device_info(&dev) != cudaSuccess) return -1;
    const sv::Plan plan = sv::make_plan(*shape);
    bool fits = false;
    const cudaError_t e = shape->dtype == SV_BF16
                              ? sv::cluster_fits<sv::bf16_bits>(shape->B, shape->k_max, plan.P, *dev, &fits)
                              : sv::cluster_fits<float>(shape->B, shape->k_max, plan.P, *dev, &fits);
    if (e != cudaSuccess) return -1;
    return fits ? SV_DRAW_CLUSTER : SV_DRAW_QUEUE;
}

}  // extern "C"
