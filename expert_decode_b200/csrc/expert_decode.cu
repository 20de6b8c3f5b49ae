// expert_decode.cu -- the C ABI (include/expert_decode.h): host-side
// validation, the workspace layout, path dispatch and kernel launches.
// Every kernel of the library is compiled into this one translation unit.

#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <cstdlib>
#include <mutex>

#include "../../include/expert_decode.h"
#include "common.cuh"
#include "router.cuh"
#include "streaming.cuh"
#include "grouped.cuh"
#include "decode_tc.cuh"
#include "ep.cuh"
#include "router_tc.cuh"
#include "decode_fp4.cuh"

namespace {

thread_local char t_error[512] = "";
thread_local int32_t t_launches = 0;
thread_local void *const *t_prof_events = nullptr;
thread_local int32_t t_prof_n = 0;

// Per-kernel timing hook (ep_profile_events): events around launch j.
struct KernelBracket {
    cudaStream_t st;
    int j;
    KernelBracket(cudaStream_t s, int index) : st(s), j(index) {
        if (t_prof_events != nullptr && 2 * j + 1 < t_prof_n)
            cudaEventRecord(static_cast<cudaEvent_t>(t_prof_events[2 * j]), st);
    }
    ~KernelBracket() {
        if (t_prof_events != nullptr && 2 * j + 1 < t_prof_n)
            cudaEventRecord(static_cast<cudaEvent_t>(t_prof_events[2 * j + 1]), st);
    }
};
std::atomic<int> g_dispatch{EP_DISPATCH_AUTO};
std::atomic<int> g_router{EP_ROUTER_AUTO};

ep_status fail(ep_status s, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(t_error, sizeof t_error, fmt, ap);
    va_end(ap);
    return s;
}

ep_status ok() {
    t_error[0] = '\0';
    return EP_OK;
}

#define EP_CUDA_CHECK(call)                                                                    \
    do {                                                                                       \
        cudaError_t err_ = (call);                                                             \
        if (err_ != cudaSuccess)                                                               \
            return fail(EP_ECUDA, "%s failed: %s", #call, cudaGetErrorString(err_));           \
    } while (0)

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Programmatic dependent launch: the kernel may start while the previous
// kernel on the stream is still running; it reads that kernel's outputs only
// after griddepcontrol.wait.  EXPERT_DECODE_NO_PDL=1 turns it off.
bool pdl_enabled() {
    static const bool on = [] {
        const char *v = getenv("EXPERT_DECODE_NO_PDL");
        return !(v != nullptr && v[0] == '1');
    }();
    return on;
}

template <typename... KArgs, typename... Args>
cudaError_t launch_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                           cudaStream_t st, unsigned cluster_x, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    int n = 0;
    if (pdl_enabled()) {
        attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[n].val.programmaticStreamSerializationAllowed = 1;
        ++n;
    }
    if (cluster_x > 0) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = cluster_x;
        attr[n].val.clusterDim.y = 1;
        attr[n].val.clusterDim.z = 1;
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

template <typename... KArgs, typename... Args>
cudaError_t launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                   Args... args) {
    return launch_cluster(kernel, grid, block, smem, st, 0u, args...);
}

struct DeviceInfo {
    bool ready = false;
    int sm_count = 0;
    int smem_optin = 0;
};

constexpr int kMaxDevices = 64;
std::mutex g_device_mu;
DeviceInfo g_devices[kMaxDevices];

// Per device, once: SM count, shared-memory limit, kernel attributes.
ep_status device_info(const DeviceInfo **out) {
    int dev = 0;
    EP_CUDA_CHECK(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kMaxDevices)
        return fail(EP_ECUDA, "device ordinal %d out of range", dev);
    std::lock_guard<std::mutex> lock(g_device_mu);
    DeviceInfo &d = g_devices[dev];
    if (!d.ready) {
        int major = 0;
        EP_CUDA_CHECK(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev));
        if (major != 10)
            return fail(EP_ECUDA, "device %d has compute capability %d.x; this library is built "
                                  "for sm_100a (B200)", dev, major);
        EP_CUDA_CHECK(cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev));
        EP_CUDA_CHECK(
            cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev));
        const int m = d.smem_optin;
#define EPK_RT_ATTR(XF, TMV, SG)                                                             \
    EP_CUDA_CHECK(cudaFuncSetAttribute(epk::router_tiled_kernel<XF, TMV, SG>,                \
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, m))
        for (int sg = 0; sg < 2; ++sg) {
            if (sg) {
                EPK_RT_ATTR(false, 1, true); EPK_RT_ATTR(false, 2, true); EPK_RT_ATTR(false, 4, true);
                EPK_RT_ATTR(true, 1, true); EPK_RT_ATTR(true, 2, true); EPK_RT_ATTR(true, 4, true);
            } else {
                EPK_RT_ATTR(false, 1, false); EPK_RT_ATTR(false, 2, false);
                EPK_RT_ATTR(false, 4, false); EPK_RT_ATTR(true, 1, false);
                EPK_RT_ATTR(true, 2, false); EPK_RT_ATTR(true, 4, false);
            }
        }
#undef EPK_RT_ATTR
#define EPK_RD_ATTR(XF, TBV, SG)                                                             \
    EP_CUDA_CHECK(cudaFuncSetAttribute(epk::router_dot2_kernel<XF, TBV, SG>,                 \
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, m))
        EPK_RD_ATTR(false, 1, false); EPK_RD_ATTR(false, 2, false);
        EPK_RD_ATTR(true, 1, false); EPK_RD_ATTR(true, 2, false);
        EPK_RD_ATTR(false, 1, true); EPK_RD_ATTR(false, 2, true);
        EPK_RD_ATTR(true, 1, true); EPK_RD_ATTR(true, 2, true);
#undef EPK_RD_ATTR
        EP_CUDA_CHECK(cudaFuncSetAttribute(epk::stream_gate_up_fp4_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, m));
        EP_CUDA_CHECK(cudaFuncSetAttribute(epk::stream_down_fp4_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, m));
        EP_CUDA_CHECK(cudaFuncSetAttribute(epk::router_tc_kernel<false>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, m));
        EP_CUDA_CHECK(cudaFuncSetAttribute(epk::router_tc_kernel<true>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, m));
        EP_CUDA_CHECK(cudaFuncSetAttribute(epk::stream_gate_up_kernel<false, false>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, m));
        EP_CUDA_CHECK(cudaFuncSetAttribute(epk::stream_gate_up_kernel<false, true>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, m));
        EP_CUDA_CHECK(cudaFuncSetAttribute(epk::stream_gate_up_kernel<true, true>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, m));
        EP_CUDA_CHECK(cudaFuncSetAttribute(epk::stream_down_fold_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, m));
        EP_CUDA_CHECK(cudaFuncSetAttribute(epk::stream_gate_up_tc_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, m));
        EP_CUDA_CHECK(cudaFuncSetAttribute(epk::stream_down_tc_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, m));
        ep_status s = epk::grouped_set_attributes(m);
        if (s != EP_OK)
            return fail(s, "setting the grouped GEMM kernel attributes failed");
        d.ready = true;
    }
    *out = &d;
    return EP_OK;
}

constexpr int64_t kMaxT = 65536;
constexpr int64_t kMaxPairs = 1 << 20;
constexpr int64_t kMaxH = 16384;
constexpr int64_t kMaxE = 1024;
constexpr int64_t kMaxI = 16384;
constexpr int kMaxTopK = 16;
// the decode path's gate/up runs on the tensor cores from this many tokens
constexpr int64_t kTcMinT = 2;


// moe_route computes every logit by Dot2 up to this many tokens
constexpr int64_t kRouterDot2MaxT = 32;
// Shared memory the streaming kernels may take, leaving the rest of the
// SM's unified L1 for the activations they read through the cache.
constexpr size_t kStreamSmemBudget = 200 * 1024;

size_t align256(size_t v) { return (v + 255) / 256 * 256; }

// ---------------------------------------------------------- workspace layout
struct Workspace {
    // streaming path (T <= 8): fp32 h for the CUDA-core down projection, bf16
    // hi/lo rows ([2 T k + 16][I], [16][I_s]) for the tensor-core one
    size_t h_routed = 0, h_shared = 0, hb_routed = 0, hb_shared = 0;
    size_t grp_done = 0;  // per-group completion words between the decode kernels
    // tensor path
    epk::GroupedWorkspace grouped;
    size_t total = 0;
};

// A call's number for the decode kernels' group completion words: 1 .. 2^48 - 1,
// never twice in a row on the same workspace.
unsigned long long next_epoch() {
    static std::atomic<unsigned long long> counter{0};
    unsigned long long e = 0;
    while (e == 0)
        e = (counter.fetch_add(1) + 1) & ((1ull << 48) - 1);
    return e;
}

Workspace workspace_layout(int64_t T, int64_t H, int64_t E, int64_t k, int64_t I, int64_t I_s) {
    Workspace w;
    size_t o = 0;
    if (T <= epk::kStreamMaxT) {
        w.h_routed = o;
        o = align256(o + (size_t)T * k * I * 4);
        w.h_shared = o;
        o = align256(o + (size_t)T * I_s * 4);
        w.hb_routed = o;
        o = align256(o + (size_t)(2 * T * k + 2 * epk::kTcSlice) * I * 2);
        w.hb_shared = o;
        o = align256(o + (size_t)2 * epk::kTcSlice * I_s * 2);
        w.grp_done = o;
        o = align256(o + (size_t)8 * epk::kTcMaxGroups);
    }
    w.grouped = epk::grouped_workspace_layout(o, T, H, E, k, I, I_s);
    o = align256(w.grouped.end);
    w.total = o;
    return w;
}

// --------------------------------------------------------- streaming path fit
struct StreamingPlan {
    bool fits = false;
    int down_rw = 1;  // down-projection rows per consumer warp per slot
    size_t down_h_arena = 0;  // bytes of the down kernel's h arena
    bool xs_f32 = false;  // gate/up keeps x as fp32 in shared memory
    int gu_slots = 0, down_slots = 0, down_grid = 0, down_rows_max = 0;
    size_t gu_smem = 0, down_smem = 0;
};

StreamingPlan streaming_fit(const DeviceInfo &d, int64_t T, int64_t H, int xb, int64_t k,
                            int64_t I, int64_t I_s) {
    StreamingPlan p;
    if (T < 1 || T > epk::kStreamMaxT || k > epk::kStreamMaxK)
        return p;
    const size_t budget = std::min<size_t>(kStreamSmemBudget, (size_t)d.smem_optin);
    // fp32 activations in shared memory skip the per-use unpacking; bf16 x
    // is widened when it takes at most 64 KB
    p.xs_f32 = xb == 4 || T * H * 4 <= 64 * 1024;
    const int xsb = p.xs_f32 ? 4 : 2;
    // The gate/up kernel keeps x in shared memory and reads nothing else
    // through L1, so its ring may take all the shared memory there is.  Each
    // slot has a single consumer warp: the slot count is the largest that
    // fits and has at least six consumers (12: six, 16: eight), else the
    // largest that fits with its most consumers (gate_up_consumers).
    const size_t gu_budget = (size_t)d.smem_optin;
    int slots = epk::kGUMaxSlots;
    while (slots >= 2 && epk::gate_up_smem_layout((int)T, (int)H, xsb, slots).total > gu_budget)
        --slots;
    if (slots < 2)
        return p;
    for (int s = slots; s >= 6; --s)
        if (epk::gate_up_consumers(s) >= 6) {
            slots = s;
            break;
        }
    p.gu_slots = slots;
    p.gu_smem = epk::gate_up_smem_layout((int)T, (int)H, xsb, slots).total;
    const int64_t I_max = std::max(I, I_s);
    p.down_grid = (int)std::max<int64_t>(1, std::min<int64_t>(d.sm_count, H / 8));
    p.down_rows_max = (int)((H + p.down_grid - 1) / p.down_grid);
    // two rows per warp per slot when three such slots still fit
    const size_t h_min = (size_t)T * I_max * 4;  // one group of every token
    for (int rw = epk::kDownMaxRowsPerWarp; rw >= 1; --rw) {
        slots = epk::kDownMaxSlots;
        while (slots >= 2 && epk::down_smem_layout((int)T, (int)I_max, slots, p.down_rows_max,
                                                   rw, h_min).total > budget)
            --slots;
        if (slots >= (rw > 1 ? 3 : 2)) {
            p.down_rw = rw;
            p.down_slots = slots;
            break;
        }
    }
    if (p.down_slots < 2)
        return p;
    // the h arena takes whatever the weight ring leaves of the budget
    const size_t rest = budget - epk::down_smem_layout((int)T, (int)I_max, p.down_slots,
                                                       p.down_rows_max, p.down_rw, 0).total;
    p.down_h_arena = std::max(h_min, rest / 128 * 128);
    p.down_smem = epk::down_smem_layout((int)T, (int)I_max, p.down_slots, p.down_rows_max,
                                        p.down_rw, p.down_h_arena).total;
    p.fits = true;
    return p;
}

}  // namespace

// =========================================================================== ABI

extern "C" ep_status ep_plan(int32_t num_experts, int32_t bands, ep_plan_t *out) {
    if (out == nullptr)
        return fail(EP_EINVAL, "ep_plan: out is NULL");
    if (num_experts < 1)
        return fail(EP_EINVAL, "ep_plan: num_experts = %d < 1", num_experts);
    if (bands < 1 || bands > num_experts || bands > EP_MAX_BANDS)
        return fail(EP_EINVAL, "ep_plan: bands = %d must be in [1, min(num_experts = %d, %d)]",
                    bands, num_experts, EP_MAX_BANDS);
    ep_plan_t p;
    memset(&p, 0, sizeof p);
    p.num_experts = num_experts;
    p.bands = bands;
    const int32_t base = num_experts / bands, extra = num_experts % bands;
    p.band_start[0] = 0;
    for (int32_t r = 0; r < bands; ++r)
        p.band_start[r + 1] = p.band_start[r] + base + (r < extra ? 1 : 0);
    *out = p;
    return ok();
}

extern "C" ep_status ep_set_dispatch(ep_dispatch mode) {
    if ((int)mode < (int)EP_DISPATCH_AUTO || (int)mode > (int)EP_DISPATCH_STREAMING_SIMT)
        return fail(EP_EINVAL, "ep_set_dispatch: unknown mode %d", (int)mode);
    g_dispatch.store((int)mode);
    return ok();
}

extern "C" ep_status ep_set_router(ep_router_mode mode) {
    if ((int)mode < (int)EP_ROUTER_AUTO || (int)mode > (int)EP_ROUTER_TENSOR)
        return fail(EP_EINVAL, "ep_set_router: unknown mode %d", (int)mode);
    g_router.store((int)mode);
    return ok();
}

extern "C" const char *ep_last_error(void) { return t_error; }

extern "C" int32_t ep_last_launch_count(void) { return t_launches; }

extern "C" ep_status ep_profile_events(void *const *events, int32_t n_events) {
    if (n_events < 0)
        return fail(EP_EINVAL, "ep_profile_events: n_events = %d < 0", n_events);
    t_prof_events = n_events > 0 ? events : nullptr;
    t_prof_n = events != nullptr ? n_events : 0;
    return ok();
}

extern "C" ep_status ep_check_status(void *stream) {
    EP_CUDA_CHECK(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
    unsigned int v = 0, zero = 0;
    EP_CUDA_CHECK(cudaMemcpyFromSymbol(&v, epk::g_status, sizeof v));
    EP_CUDA_CHECK(cudaMemcpyToSymbol(epk::g_status, &zero, sizeof zero));
    if (v & epk::kStatusTimeout)
        return fail(EP_ETIMEOUT, "a device-side wait ran out of time");
    if (v & epk::kStatusBadId)
        return fail(EP_EBADID, "an expert id outside [0, E) was skipped on the device");
    return ok();
}

namespace {

// Clusters of `csize` CTAs of `fn` with `smem` bytes that can be resident at
// once on this device (cudaOccupancyMaxActiveClusters), cached; 0 if none.
int max_active_clusters(const void *fn, int csize, uint32_t smem) {
    struct Entry {
        const void *fn;
        int dev, csize;
        uint32_t smem;
        int value;
    };
    static std::mutex mu;
    static Entry cache[128];
    static int n_cache = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return 0;
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < n_cache; ++i)
        if (cache[i].fn == fn && cache[i].dev == dev && cache[i].csize == csize &&
            cache[i].smem == smem)
            return cache[i].value;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)csize, 1, 1);
    cfg.blockDim = dim3((unsigned)epk::kRtThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = (unsigned)csize;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, fn, &cfg) != cudaSuccess) {
        (void)cudaGetLastError();
        n = 0;
    }
    if (n_cache < 128)
        cache[n_cache++] = Entry{fn, dev, csize, smem, n};
    return n;
}

// The tensor-core router takes batches of more than 32 tokens with bf16
// activations, at most 256 experts and at least two 64-wide blocks of H (so
// that every CTA of its cluster has a slice); the tiled fp32 router the rest.
bool tc_router_fits(const DeviceInfo &d, ep_dtype x_dtype, int64_t H, int64_t E) {
    if (x_dtype != EP_BF16 || E > epk::kRcMaxE || H < 2 * epk::kGemmBK)
        return false;
    const int MT = (int)((E + epk::kGemmBM - 1) / epk::kGemmBM);
    return epk::rc_smem_layout(MT, (int)E, epk::kRcMinCK).alloc <= (uint32_t)d.smem_optin &&
           epk::tensor_map_encoder() != nullptr;
}

// Both routers: sig selects the sigmoid variant (normalize, scale used only
// there); `who` names the entry point in error messages.
ep_status route_impl(const char *who, bool sig, const void *x, ep_dtype x_dtype, int64_t T,
                     int64_t H, const void *w_router, const float *bias, int64_t E,
                     int32_t top_k, int32_t normalize, float scale, int32_t *ids,
                     float *weights, void *stream, float *dump_logit = nullptr,
                     float *dump_bound = nullptr) {
    if (x_dtype != EP_BF16 && x_dtype != EP_F32)
        return fail(EP_EINVAL, "%s: unknown x dtype %d", who, (int)x_dtype);
    if (T < 0 || T > kMaxT)
        return fail(EP_EINVAL, "%s: T = %lld outside [0, %lld]", who, (long long)T,
                    (long long)kMaxT);
    if (H < 8 || H > kMaxH || H % 8 != 0)
        return fail(EP_EINVAL, "%s: H = %lld must be a multiple of 8 in [8, %lld]", who,
                    (long long)H, (long long)kMaxH);
    if (E < 1 || E > kMaxE)
        return fail(EP_EINVAL, "%s: E = %lld outside [1, %lld]", who, (long long)E,
                    (long long)kMaxE);
    if (top_k < 1 || top_k > kMaxTopK || top_k > E)
        return fail(EP_EINVAL, "%s: top_k = %d outside [1, min(E, %d)]", who, top_k, kMaxTopK);
    if (T == 0) {
        t_launches = 0;
        return ok();
    }
    const bool dump = dump_logit != nullptr;
    if (x == nullptr || w_router == nullptr || (!dump && (ids == nullptr || weights == nullptr)) ||
        (dump && dump_bound == nullptr))
        return fail(EP_EINVAL, "%s: NULL x, w_router, ids or weights", who);
    if (!aligned(x, 16) || !aligned(w_router, 16) || !aligned(ids, 4) || !aligned(weights, 4) ||
        (bias != nullptr && !aligned(bias, 4)) || !aligned(dump_logit, 4) ||
        !aligned(dump_bound, 4))
        return fail(EP_EINVAL, "%s: misaligned pointer (x, w_router need 16 bytes)", who);
    const DeviceInfo *d = nullptr;
    ep_status s = device_info(&d);
    if (s != EP_OK)
        return s;
    const int router_mode = g_router.load();
    if (router_mode == EP_ROUTER_TENSOR && T > kRouterDot2MaxT &&
        !tc_router_fits(*d, x_dtype, H, E))
        return fail(EP_EINVAL, "%s: the tensor-core router takes bf16 x, E <= %d and H >= %d",
                    who, epk::kRcMaxE, 2 * epk::kGemmBK);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const uint16_t *wr = static_cast<const uint16_t *>(w_router);
    KernelBracket kb0(st, 0);
    if (T <= kRouterDot2MaxT && !dump) {
        // small batches: every logit by Dot2, one cluster per token while
        // the clusters fit on the SMs at once, else two tokens per cluster
        const int64_t max_clusters = std::max(1, d->sm_count / epk::kRouterCluster);
        const int tb = T <= max_clusters ? 1 : epk::kRdMaxTB;
        const epk::RdSmem L = epk::rd_smem_layout(tb, (int)H, (int)E);
        if ((int)L.total > d->smem_optin)
            return fail(EP_EINVAL, "%s: H = %lld, E = %lld need %u bytes of shared memory", who,
                        (long long)H, (long long)E, L.total);
        const int64_t nblk = (T + tb - 1) / tb;
        const dim3 grid((unsigned)(nblk * epk::kRouterCluster));
        cudaError_t e;
#define EPK_RD(XF, TBV, SG)                                                                    \
    e = launch(epk::router_dot2_kernel<XF, TBV, SG>, grid, epk::kRdThreads, L.total, st, x, T,  \
               (int)H, wr, bias, (int)E, top_k, ids, weights, normalize, scale)
        const bool f32 = x_dtype == EP_F32;
        if (sig) {
            if (f32) { if (tb == 1) EPK_RD(true, 1, true); else EPK_RD(true, 2, true); }
            else { if (tb == 1) EPK_RD(false, 1, true); else EPK_RD(false, 2, true); }
        } else {
            if (f32) { if (tb == 1) EPK_RD(true, 1, false); else EPK_RD(true, 2, false); }
            else { if (tb == 1) EPK_RD(false, 1, false); else EPK_RD(false, 2, false); }
        }
#undef EPK_RD
        EP_CUDA_CHECK(e);
    } else if (router_mode != EP_ROUTER_TILED && tc_router_fits(*d, x_dtype, H, E)) {
        // larger batches of bf16 activations: logits on the tensor cores, a
        // cluster of CK CTAs per 64 tokens, Dot2 for the candidates
        const int MT = (int)((E + epk::kGemmBM - 1) / epk::kGemmBM);
        const int64_t tiles = (T + epk::kRcNT - 1) / epk::kRcNT;
        const int nkb = (int)((H + epk::kGemmBK - 1) / epk::kGemmBK);
        int CK = (int)std::max<int64_t>(epk::kRcMinCK,
                                        std::min<int64_t>(epk::kRcMaxCK, d->sm_count / tiles));
        CK = std::min(CK, nkb);
        const epk::RcSmem L = epk::rc_smem_layout(MT, (int)E, CK);
        epk::RcMaps maps;
        memset(&maps, 0, sizeof maps);
        if (!epk::map_2d(&maps.w, w_router, (uint64_t)H, (uint64_t)E, epk::kGemmBM) ||
            !epk::map_2d(&maps.x, x, (uint64_t)H, (uint64_t)T, epk::kRcNT))
            return fail(EP_ECUDA, "%s: encoding the router's tensor maps failed", who);
        const dim3 grid((unsigned)CK, (unsigned)tiles);
        const uint16_t *xb = static_cast<const uint16_t *>(x);
        const cudaError_t e =
            sig ? launch_cluster(epk::router_tc_kernel<true>, grid, epk::kRcThreads, L.alloc, st,
                                 (unsigned)CK, maps, xb, T, (int)H, wr, bias, (int)E, top_k, ids,
                                 weights, CK, normalize, scale, dump_logit, dump_bound)
                : launch_cluster(epk::router_tc_kernel<false>, grid, epk::kRcThreads, L.alloc, st,
                                 (unsigned)CK, maps, xb, T, (int)H, wr, bias, (int)E, top_k, ids,
                                 weights, CK, normalize, scale, dump_logit, dump_bound);
        EP_CUDA_CHECK(e);
    } else {
        // larger batches: register-tiled fp32 logits, Dot2 for the candidates
        const int BT = epk::rt_block_tokens((int)E);
        const epk::RtSmem L = epk::rt_smem_layout(BT, (int)E);
        if ((int)L.total > d->smem_optin)
            return fail(EP_EINVAL, "%s: E = %lld needs %u bytes of shared memory", who,
                        (long long)E, L.total);
        // the kernel for this activation type, block size and router
        using TiledFn = void (*)(const void *, int64_t, int, const uint16_t *, const float *, int,
                                 int, int32_t *, float *, int, int, int, float, float *, float *);
        TiledFn fn;
        {
            const bool f = x_dtype == EP_F32;
#define EPK_RT_FN(TMV)                                                                         \
    (sig ? (f ? epk::router_tiled_kernel<true, TMV, true> : epk::router_tiled_kernel<false, TMV, true>) \
         : (f ? epk::router_tiled_kernel<true, TMV, false> : epk::router_tiled_kernel<false, TMV, false>))
            fn = BT == 32 ? EPK_RT_FN(4) : (BT == 16 ? EPK_RT_FN(2) : EPK_RT_FN(1));
#undef EPK_RT_FN
        }
        // A cluster of CE expert slices x CK slices of H (at most 8 CTAs).
        // Splitting H shortens every CTA's main loop but makes the clusters
        // larger, and larger clusters fit fewer at a time on the GPCs; CK is
        // chosen for the least (waves) x (main loop / CK + the fixed tail),
        // the tail taken as a tenth of an unsplit main loop.
        const int CE = (int)((E + epk::kRtBE - 1) / epk::kRtBE);
        const int nkt = (int)((H + epk::kRtBK - 1) / epk::kRtBK);
        const int64_t blocks = (T + BT - 1) / BT;
        const int ck_max = std::max(1, std::min(epk::kRouterCluster / CE, nkt));
        int CK = 1;
        bool have = false;
        double best = 0.0;
        for (int ck = 1; ck <= ck_max; ++ck) {
            const int fit = max_active_clusters(reinterpret_cast<const void *>(fn), CE * ck,
                                                L.total);
            if (fit < 1)
                continue;
            const double waves = (double)((blocks + fit - 1) / fit);
            const double cost = waves * (1.0 / ck + 0.1);
            if (!have || cost < best) {
                have = true;
                best = cost;
                CK = ck;
            }
        }
        const dim3 grid((unsigned)(CE * CK), (unsigned)blocks);
        const cudaError_t e = launch_cluster(fn, grid, epk::kRtThreads, L.total, st,
                                             (unsigned)(CE * CK), x, T, (int)H, wr, bias, (int)E,
                                             top_k, ids, weights, CE, CK, normalize, scale,
                                             dump_logit, dump_bound);
        EP_CUDA_CHECK(e);
    }
    t_launches = 1;
    return ok();
}

}  // namespace

extern "C" ep_status moe_route(const void *x, ep_dtype x_dtype, int64_t T, int64_t H,
                               const void *w_router, const float *bias, int64_t E,
                               int32_t top_k, int32_t *ids, float *weights, void *stream) {
    return route_impl("moe_route", false, x, x_dtype, T, H, w_router, bias, E, top_k, 0, 1.0f,
                      ids, weights, stream);
}

extern "C" ep_status moe_route_logits(const void *x, ep_dtype x_dtype, int64_t T, int64_t H,
                                      const void *w_router, const float *bias, int64_t E,
                                      float *logits, float *bounds, void *stream) {
    if (logits == nullptr || bounds == nullptr)
        return fail(EP_EINVAL, "moe_route_logits: NULL logits or bounds");
    return route_impl("moe_route_logits", false, x, x_dtype, T, H, w_router, bias, E,
                      (int32_t)std::min<int64_t>(E, 1), 0, 1.0f, nullptr, nullptr, stream,
                      logits, bounds);
}

extern "C" ep_status moe_route_sigmoid(const void *x, ep_dtype x_dtype, int64_t T, int64_t H,
                                       const void *w_router, const float *bias, int64_t E,
                                       int32_t top_k, int32_t normalize, float scale,
                                       int32_t *ids, float *weights, void *stream) {
    if (normalize != 0 && normalize != 1)
        return fail(EP_EINVAL, "moe_route_sigmoid: normalize = %d must be 0 or 1", normalize);
    if (!(scale > 0.0f) || !std::isfinite(scale))
        return fail(EP_EINVAL, "moe_route_sigmoid: scale must be finite and positive");
    return route_impl("moe_route_sigmoid", true, x, x_dtype, T, H, w_router, bias, E, top_k,
                      normalize, scale, ids, weights, stream);
}

extern "C" size_t moe_ffn_workspace_size(int64_t T, int64_t H, int64_t E, int32_t top_k,
                                         int64_t I, int64_t I_s) {
    if (T <= 0 || H <= 0 || E <= 0 || top_k <= 0 || I <= 0 || I_s < 0)
        return 0;
    return workspace_layout(T, H, E, top_k, I, I_s).total;
}

extern "C" ep_status moe_ffn_workspace_layout(int64_t T, int64_t H, int64_t E, int32_t top_k,
                                             int64_t I, int64_t I_s, ep_workspace_layout_t *out) {
    if (out == nullptr)
        return fail(EP_EINVAL, "moe_ffn_workspace_layout: out is NULL");
    if (T < 0 || T > kMaxT || T * (int64_t)std::max(top_k, 1) > kMaxPairs || H < 8 ||
        H > kMaxH || H % 8 != 0 || E < 1 || E > kMaxE || top_k < 1 || top_k > kMaxTopK ||
        top_k > E || I < 8 || I > kMaxI || I % 8 != 0 ||
        (I_s != 0 && (I_s < 8 || I_s > kMaxI || I_s % 8 != 0)))
        return fail(EP_EINVAL, "moe_ffn_workspace_layout: sizes out of range");
    ep_workspace_layout_t l;
    memset(&l, 0, sizeof l);
    if (T > 0) {
        const Workspace W = workspace_layout(T, H, E, top_k, I, I_s);
        l.bytes = W.total;
        l.contrib_offset = W.grouped.c;
        l.shared_offset = W.grouped.s;
        l.group_offset_offset = W.grouped.group_offset;
        l.perm_offset = W.grouped.perm_pair;
    }
    *out = l;
    return ok();
}

namespace {

// moe_ffn_forward's body.  band_call: a band partial (moe_ffn_partial), whose
// picks may outnumber the band's experts (they span bands), so top_k is not
// bounded by E there.
ep_status ffn_forward_impl(bool band_call, const void *x, ep_dtype x_dtype, int64_t T, int64_t H,
                           const int32_t *ids, const float *weights, int32_t top_k,
                           const void *w_gate, const void *w_up, const void *w_down, int64_t E,
                           int64_t I, const void *ws_gate, const void *ws_up,
                           const void *ws_down, int64_t I_s, const ep_plan_t *plan, float *y,
                           void *workspace, size_t workspace_bytes, void *stream) {
    // ---- validation: nothing is launched and nothing written on failure
    if (plan == nullptr)
        return fail(EP_EINVAL, "moe_ffn_forward: plan is NULL");
    if (plan->num_experts != E)
        return fail(EP_EDIM, "moe_ffn_forward: plan covers %d experts, E = %lld",
                    plan->num_experts, (long long)E);
    if (plan->bands < 1 || plan->bands > EP_MAX_BANDS || plan->bands > E ||
        plan->band_start[0] != 0 || plan->band_start[plan->bands] != E)
        return fail(EP_EINVAL, "moe_ffn_forward: plan is not a partition of [0, E)");
    for (int r = 0; r < plan->bands; ++r)
        if (plan->band_start[r + 1] <= plan->band_start[r])
            return fail(EP_EINVAL, "moe_ffn_forward: band %d of the plan is empty or reversed", r);
    if (x_dtype != EP_BF16 && x_dtype != EP_F32)
        return fail(EP_EINVAL, "moe_ffn_forward: unknown x dtype %d", (int)x_dtype);
    if (T < 0 || T > kMaxT || T * (int64_t)std::max(top_k, 1) > kMaxPairs)
        return fail(EP_EINVAL, "moe_ffn_forward: T = %lld out of range", (long long)T);
    if (H < 8 || H > kMaxH || H % 8 != 0)
        return fail(EP_EINVAL, "moe_ffn_forward: H = %lld must be a multiple of 8 in [8, %lld]",
                    (long long)H, (long long)kMaxH);
    if (E < 1 || E > kMaxE)
        return fail(EP_EINVAL, "moe_ffn_forward: E = %lld outside [1, %lld]", (long long)E,
                    (long long)kMaxE);
    if (top_k < 1 || top_k > kMaxTopK || (!band_call && top_k > E))
        return fail(EP_EINVAL, "moe_ffn_forward: top_k = %d outside [1, min(E, %d)]", top_k,
                    kMaxTopK);
    if (I < 8 || I > kMaxI || I % 8 != 0)
        return fail(EP_EINVAL, "moe_ffn_forward: I = %lld must be a multiple of 8 in [8, %lld]",
                    (long long)I, (long long)kMaxI);
    if (I_s != 0 && (I_s < 8 || I_s > kMaxI || I_s % 8 != 0))
        return fail(EP_EINVAL, "moe_ffn_forward: I_s = %lld must be 0 or a multiple of 8 in "
                               "[8, %lld]", (long long)I_s, (long long)kMaxI);
    if (T == 0) {
        t_launches = 0;
        return ok();
    }
    if (x == nullptr || ids == nullptr || weights == nullptr || w_gate == nullptr ||
        w_up == nullptr || w_down == nullptr || y == nullptr)
        return fail(EP_EINVAL, "moe_ffn_forward: a required pointer is NULL");
    if ((I_s > 0) != (ws_gate != nullptr) || (I_s > 0) != (ws_up != nullptr) ||
        (I_s > 0) != (ws_down != nullptr))
        return fail(EP_EINVAL, "moe_ffn_forward: shared-expert pointers must all be set iff "
                               "I_s > 0");
    const void *al16[] = {x, w_gate, w_up, w_down, y, ws_gate, ws_up, ws_down};
    for (const void *p : al16)
        if (p != nullptr && !aligned(p, 16))
            return fail(EP_EINVAL, "moe_ffn_forward: a tensor is not 16-byte aligned");
    if (!aligned(ids, 4) || !aligned(weights, 4))
        return fail(EP_EINVAL, "moe_ffn_forward: ids / weights not 4-byte aligned");
    const Workspace W = workspace_layout(T, H, E, top_k, I, I_s);
    if (workspace == nullptr || workspace_bytes < W.total)
        return fail(EP_ENOMEM, "moe_ffn_forward: workspace of %zu bytes, %zu needed",
                    workspace_bytes, W.total);
    if (!aligned(workspace, 256))
        return fail(EP_EINVAL, "moe_ffn_forward: workspace not 256-byte aligned");
    const DeviceInfo *d = nullptr;
    ep_status s = device_info(&d);
    if (s != EP_OK)
        return s;

    const int xb = x_dtype == EP_F32 ? 4 : 2;
    const StreamingPlan sp = streaming_fit(*d, T, H, xb, top_k, I, I_s);
    const int mode = g_dispatch.load();
    bool use_streaming;
    if (mode == EP_DISPATCH_STREAMING || mode == EP_DISPATCH_STREAMING_TC ||
        mode == EP_DISPATCH_STREAMING_SIMT) {
        if (!sp.fits)
            return fail(EP_EINVAL, "moe_ffn_forward: the streaming path does not fit these sizes");
        use_streaming = true;
    } else if (mode == EP_DISPATCH_TENSOR) {
        use_streaming = false;
    } else {
        use_streaming = sp.fits;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);

    if (use_streaming) {
        epk::StreamGateUpArgs ga;
        ga.x = x;
        ga.T = (int)T; ga.H = (int)H; ga.E = (int)E; ga.I = (int)I; ga.I_s = (int)I_s;
        ga.top_k = top_k; ga.n_slots = sp.gu_slots;
        ga.w_gate = static_cast<const uint16_t *>(w_gate);
        ga.w_up = static_cast<const uint16_t *>(w_up);
        ga.ws_gate = static_cast<const uint16_t *>(ws_gate);
        ga.ws_up = static_cast<const uint16_t *>(ws_up);
        ga.ids = ids;
        ga.weights = weights;
        ga.h_routed = reinterpret_cast<float *>(ws + W.h_routed);
        ga.h_shared = reinterpret_cast<float *>(ws + W.h_shared);
        const dim3 gu_grid((unsigned)d->sm_count);
        // gate/up on the tensor cores needs bf16 activations and the tensor
        // maps; by default it takes over from 2 tokens on
        epk::TcMaps tm;
        memset(&tm, 0, sizeof tm);
        bool tc_ok = x_dtype == EP_BF16 && epk::TcSmem::alloc <= (uint32_t)d->smem_optin &&
                     epk::tensor_map_encoder() != nullptr;
        if (tc_ok && mode != EP_DISPATCH_STREAMING_SIMT &&
            (mode == EP_DISPATCH_STREAMING_TC || T >= kTcMinT)) {
            tc_ok = epk::map_3d(&tm.wg, w_gate, H, I, E, epk::kGateUpRows) &&
                    epk::map_3d(&tm.wu, w_up, H, I, E, epk::kGateUpRows) &&
                    epk::map_2d(&tm.x, x, H, T, epk::kTcN);
            if (I_s > 0)
                tc_ok = tc_ok && epk::map_2d(&tm.sg, ws_gate, H, I_s, epk::kGateUpRows) &&
                        epk::map_2d(&tm.su, ws_up, H, I_s, epk::kGateUpRows);
        }
        bool use_tc;
        if (mode == EP_DISPATCH_STREAMING_TC) {
            if (!tc_ok)
                return fail(EP_EINVAL, "moe_ffn_forward: tensor-core gate/up needs bf16 x");
            use_tc = true;
        } else {
            use_tc = tc_ok && mode != EP_DISPATCH_STREAMING_SIMT && T >= kTcMinT;
        }
        if (use_tc) {
            epk::TcArgs ta;
            ta.T = (int)T; ta.H = (int)H; ta.E = (int)E; ta.I = (int)I; ta.I_s = (int)I_s;
            ta.top_k = top_k;
            ta.ids = ids;
            ta.weights = weights;
            ta.h_routed = ga.h_routed;
            ta.h_shared = ga.h_shared;
            ta.hb_routed = reinterpret_cast<uint16_t *>(ws + W.hb_routed);
            ta.hb_shared = I_s > 0 ? reinterpret_cast<uint16_t *>(ws + W.hb_shared) : nullptr;
            ta.grp_done = reinterpret_cast<unsigned long long *>(ws + W.grp_done);
            ta.epoch = next_epoch();
            ta.pf[0] = ws_gate;
            ta.pf[1] = ws_up;
            ta.pf[2] = ws_down;
            for (int i = 0; i < 3; ++i)
                ta.pf_bytes[i] = I_s > 0 ? (size_t)I_s * H * 2 : 0;

            // the down projection on the tensor cores too: W_down rows against
            // the bf16 hi/lo slices of h, then the fold in combine_kernel
            epk::DtMaps dm;
            memset(&dm, 0, sizeof dm);
            bool dm_ok = epk::DtSmem::alloc <= (uint32_t)d->smem_optin &&
                         epk::map_3d(&dm.wd, w_down, I, H, E, epk::kGemmBM) &&
                         epk::map_2d(&dm.hr, ta.hb_routed, I,
                                     (uint64_t)(2 * T * top_k + 2 * epk::kTcSlice),
                                     2 * epk::kTcSlice);
            if (I_s > 0)
                dm_ok = dm_ok && epk::map_2d(&dm.sd, ws_down, I_s, H, epk::kGemmBM) &&
                        epk::map_2d(&dm.hs, ta.hb_shared, I_s, 2 * epk::kTcSlice,
                                    2 * epk::kTcSlice);
            if (!dm_ok)
                return fail(EP_ECUDA, "moe_ffn_forward: encoding a down tensor map failed");
            {
                KernelBracket kb0(st, 0);
                EP_CUDA_CHECK(launch(epk::stream_gate_up_tc_kernel, gu_grid, epk::kTcThreads,
                                     epk::TcSmem::alloc, st, tm, ta));
            }
            epk::DtArgs dta;
            dta.T = (int)T; dta.H = (int)H; dta.E = (int)E; dta.I = (int)I; dta.I_s = (int)I_s;
            dta.top_k = top_k;
            dta.ids = ids;
            dta.weights = weights;
            dta.c = reinterpret_cast<float *>(ws + W.grouped.c);
            dta.s = reinterpret_cast<float *>(ws + W.grouped.s);
            dta.grp_done = ta.grp_done;
            dta.epoch = ta.epoch;
            {
                KernelBracket kb1(st, 1);
                EP_CUDA_CHECK(launch(epk::stream_down_tc_kernel, gu_grid, epk::kTcThreads,
                                     epk::DtSmem::alloc, st, dm, dta));
            }
            {
                KernelBracket kb2(st, 2);
                // 64-thread blocks: a few tokens still spread over most SMs
                const dim3 cgrid((unsigned)T, (unsigned)((H / 4 + 63) / 64));
                EP_CUDA_CHECK(launch(epk::combine_kernel, cgrid, 64, 0, st,
                                     (const float *)dta.c,
                                     (const float *)(I_s > 0 ? dta.s : nullptr), ids, (int64_t)T,
                                     (int)H, (int)top_k, (int)E, y));
            }
            t_launches = 3;
            return ok();
        } else {
            KernelBracket kb0(st, 0);
            if (x_dtype == EP_F32)
                EP_CUDA_CHECK(launch(epk::stream_gate_up_kernel<true, true>, gu_grid,
                                     epk::kGUThreads, sp.gu_smem, st, ga));
            else if (sp.xs_f32)
                EP_CUDA_CHECK(launch(epk::stream_gate_up_kernel<false, true>, gu_grid,
                                     epk::kGUThreads, sp.gu_smem, st, ga));
            else
                EP_CUDA_CHECK(launch(epk::stream_gate_up_kernel<false, false>, gu_grid,
                                     epk::kGUThreads, sp.gu_smem, st, ga));
        }

        epk::StreamDownArgs da;
        da.T = (int)T; da.H = (int)H; da.E = (int)E; da.I = (int)I; da.I_s = (int)I_s;
        da.top_k = top_k; da.n_slots = sp.down_slots; da.rows_max = sp.down_rows_max;
        da.rw = sp.down_rw;
        da.h_arena = (int)sp.down_h_arena;
        da.w_down = static_cast<const uint16_t *>(w_down);
        da.ws_down = static_cast<const uint16_t *>(ws_down);
        da.ids = ids;
        da.weights = weights;
        da.h_routed = ga.h_routed;
        da.h_shared = ga.h_shared;
        da.y = y;
        {
            KernelBracket kb1(st, 1);
            EP_CUDA_CHECK(launch(epk::stream_down_fold_kernel, dim3((unsigned)sp.down_grid),
                                 epk::kDownThreads, sp.down_smem, st, da));
        }
        t_launches = 2;
        return ok();
    }

    epk::GroupedArgs g;
    g.x = x; g.x_f32 = x_dtype == EP_F32;
    g.T = T; g.H = H; g.E = E; g.I = I; g.I_s = I_s; g.top_k = top_k;
    g.ids = ids; g.weights = weights;
    g.w_gate = w_gate; g.w_up = w_up; g.w_down = w_down;
    g.ws_gate = ws_gate; g.ws_up = ws_up; g.ws_down = ws_down;
    g.y = y;
    g.sm_count = d->sm_count;
    g.smem_optin = d->smem_optin;
    g.pdl = pdl_enabled();
    int launches = 0;
    char why[256] = "";
    s = epk::grouped_forward(g, W.grouped, ws, st, &launches, why, sizeof why,
                             t_prof_events, t_prof_n);
    if (s != EP_OK)
        return fail(s, "moe_ffn_forward: %s", why);
    t_launches = launches;
    return ok();
}

}  // namespace

extern "C" ep_status moe_ffn_forward(const void *x, ep_dtype x_dtype, int64_t T, int64_t H,
                                     const int32_t *ids, const float *weights, int32_t top_k,
                                     const void *w_gate, const void *w_up, const void *w_down,
                                     int64_t E, int64_t I, const void *ws_gate,
                                     const void *ws_up, const void *ws_down, int64_t I_s,
                                     const ep_plan_t *plan, float *y, void *workspace,
                                     size_t workspace_bytes, void *stream) {
    return ffn_forward_impl(false, x, x_dtype, T, H, ids, weights, top_k, w_gate, w_up, w_down,
                            E, I, ws_gate, ws_up, ws_down, I_s, plan, y, workspace,
                            workspace_bytes, stream);
}

// ============================================================ NVFP4 decode
namespace {

struct Fp4Workspace {
    size_t x16 = 0, hb = 0, hs = 0, c = 0, s = 0, total = 0;
};

Fp4Workspace fp4_workspace_layout(int64_t T, int64_t H, int64_t k, int64_t I, int64_t I_s) {
    Fp4Workspace w;
    size_t o = 0;
    w.x16 = o; o = align256(o + (size_t)T * H * 2);
    w.hb = o;  o = align256(o + (size_t)(2 * T * k + 2 * epk::kTcSlice) * I * 2);
    w.hs = o;  o = align256(o + (size_t)2 * epk::kTcSlice * std::max<int64_t>(I_s, 64) * 2);
    w.c = o;   o = align256(o + (size_t)T * k * H * 4);
    w.s = o;   o = align256(o + (size_t)T * H * 4);
    w.total = o;
    return w;
}

bool fp4_mat_ok(const ep_nvfp4_t *m) {
    return m != nullptr && m->codes != nullptr && m->scales != nullptr && aligned(m->codes, 16) &&
           aligned(m->scales, 4) && std::isfinite(m->tensor_scale);
}

}  // namespace

extern "C" size_t moe_ffn_nvfp4_workspace_size(int64_t T, int64_t H, int64_t E, int32_t top_k,
                                               int64_t I, int64_t I_s) {
    if (T <= 0 || H <= 0 || E <= 0 || top_k <= 0 || I <= 0 || I_s < 0)
        return 0;
    return fp4_workspace_layout(T, H, top_k, I, I_s).total;
}

extern "C" ep_status moe_ffn_forward_nvfp4(const void *x, int64_t T, int64_t H,
                                           const int32_t *ids, const float *weights,
                                           int32_t top_k, const ep_nvfp4_t *w_gate,
                                           const ep_nvfp4_t *w_up, const ep_nvfp4_t *w_down,
                                           int64_t E, int64_t I, const ep_nvfp4_t *ws_gate,
                                           const ep_nvfp4_t *ws_up, const ep_nvfp4_t *ws_down,
                                           int64_t I_s, const ep_plan_t *plan, float *y,
                                           void *workspace, size_t workspace_bytes,
                                           void *stream) {
    const char *who = "moe_ffn_forward_nvfp4";
    if (plan == nullptr)
        return fail(EP_EINVAL, "%s: plan is NULL", who);
    if (plan->num_experts != E)
        return fail(EP_EDIM, "%s: plan covers %d experts, E = %lld", who, plan->num_experts,
                    (long long)E);
    if (plan->bands < 1 || plan->bands > EP_MAX_BANDS || plan->bands > E ||
        plan->band_start[0] != 0 || plan->band_start[plan->bands] != E)
        return fail(EP_EINVAL, "%s: plan is not a partition of [0, E)", who);
    for (int r = 0; r < plan->bands; ++r)
        if (plan->band_start[r + 1] <= plan->band_start[r])
            return fail(EP_EINVAL, "%s: band %d of the plan is empty or reversed", who, r);
    if (T < 0 || T > epk::kStreamMaxT)
        return fail(EP_EINVAL, "%s: T = %lld outside [0, %d]", who, (long long)T,
                    epk::kStreamMaxT);
    auto dim_ok = [](int64_t v) { return v >= 64 && v <= kMaxH && v % 64 == 0; };
    if (!dim_ok(H) || !dim_ok(I) || (I_s != 0 && !dim_ok(I_s)))
        return fail(EP_EINVAL, "%s: H, I and I_s must be multiples of 64 in [64, %lld]", who,
                    (long long)kMaxH);
    if (E < 1 || E > kMaxE)
        return fail(EP_EINVAL, "%s: E = %lld outside [1, %lld]", who, (long long)E,
                    (long long)kMaxE);
    if (top_k < 1 || top_k > kMaxTopK || top_k > E)
        return fail(EP_EINVAL, "%s: top_k = %d outside [1, min(E, %d)]", who, top_k, kMaxTopK);
    if (T == 0) {
        t_launches = 0;
        return ok();
    }
    if (x == nullptr || ids == nullptr || weights == nullptr || y == nullptr ||
        !fp4_mat_ok(w_gate) || !fp4_mat_ok(w_up) || !fp4_mat_ok(w_down))
        return fail(EP_EINVAL, "%s: a required pointer is NULL or misaligned", who);
    if ((I_s > 0) != (ws_gate != nullptr) || (I_s > 0) != (ws_up != nullptr) ||
        (I_s > 0) != (ws_down != nullptr) ||
        (I_s > 0 && (!fp4_mat_ok(ws_gate) || !fp4_mat_ok(ws_up) || !fp4_mat_ok(ws_down))))
        return fail(EP_EINVAL, "%s: shared-expert matrices must all be given iff I_s > 0", who);
    if (!aligned(x, 16) || !aligned(y, 16) || !aligned(ids, 4) || !aligned(weights, 4))
        return fail(EP_EINVAL, "%s: misaligned x, y, ids or weights", who);
    const Fp4Workspace W = fp4_workspace_layout(T, H, top_k, I, I_s);
    if (workspace == nullptr || workspace_bytes < W.total)
        return fail(EP_ENOMEM, "%s: workspace of %zu bytes, %zu needed", who, workspace_bytes,
                    W.total);
    if (!aligned(workspace, 256))
        return fail(EP_EINVAL, "%s: workspace not 256-byte aligned", who);
    const DeviceInfo *d = nullptr;
    ep_status s = device_info(&d);
    if (s != EP_OK)
        return s;
    if (epk::F4Smem::alloc > (uint32_t)d->smem_optin ||
        epk::F4DnSmem::alloc > (uint32_t)d->smem_optin || epk::tensor_map_encoder() == nullptr)
        return fail(EP_ECUDA, "%s: this device cannot run the NVFP4 kernels", who);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    uint16_t *x16 = reinterpret_cast<uint16_t *>(ws + W.x16);
    uint16_t *hb = reinterpret_cast<uint16_t *>(ws + W.hb);
    uint16_t *hs = reinterpret_cast<uint16_t *>(ws + W.hs);
    float *c = reinterpret_cast<float *>(ws + W.c);
    float *sh = reinterpret_cast<float *>(ws + W.s);

    epk::F4GuMaps gm;
    memset(&gm, 0, sizeof gm);
    bool okm = epk::map_codes(&gm.cg, w_gate->codes, H, I, E, epk::kGateUpRows) &&
               epk::map_codes(&gm.cu, w_up->codes, H, I, E, epk::kGateUpRows) &&
               epk::map_f16(&gm.x, x16, H, T, epk::kTcN);
    if (I_s > 0)
        okm = okm && epk::map_codes(&gm.sg, ws_gate->codes, H, I_s, 1, epk::kGateUpRows) &&
              epk::map_codes(&gm.su, ws_up->codes, H, I_s, 1, epk::kGateUpRows);
    epk::F4DnMaps dm;
    memset(&dm, 0, sizeof dm);
    okm = okm && epk::map_codes(&dm.cd, w_down->codes, I, H, E, epk::kGemmBM) &&
          epk::map_f16(&dm.hr, hb, I, (uint64_t)(2 * T * top_k + 2 * epk::kTcSlice),
                       2 * epk::kTcSlice);
    if (I_s > 0)
        okm = okm && epk::map_codes(&dm.sd, ws_down->codes, I_s, H, 1, epk::kGemmBM) &&
              epk::map_f16(&dm.hs, hs, I_s, 2 * epk::kTcSlice, 2 * epk::kTcSlice);
    if (!okm)
        return fail(EP_ECUDA, "%s: encoding a tensor map failed", who);

    auto mat = [](const ep_nvfp4_t *m, int64_t rows, int64_t cols) {
        epk::F4Mat f;
        f.scales = m == nullptr ? nullptr : static_cast<const uint8_t *>(m->scales);
        f.ts = m == nullptr ? 0.f : m->tensor_scale;
        f.rows = rows;
        f.cols = cols;
        return f;
    };
    const dim3 grid((unsigned)d->sm_count);
    {
        KernelBracket kb0(st, 0);
        const int64_t n = T * H;
        EP_CUDA_CHECK(launch(epk::to_f16_kernel, dim3((unsigned)((n + 255) / 256)), 256, 0, st,
                             static_cast<const uint16_t *>(x), n, x16));
    }
    epk::F4GuArgs ga;
    ga.T = (int)T; ga.H = (int)H; ga.E = (int)E; ga.I = (int)I; ga.I_s = (int)I_s;
    ga.top_k = top_k; ga.ids = ids; ga.weights = weights;
    ga.wg = mat(w_gate, I, H); ga.wu = mat(w_up, I, H);
    ga.sg = mat(ws_gate, I_s, H); ga.su = mat(ws_up, I_s, H);
    ga.hb_routed = hb; ga.hb_shared = I_s > 0 ? hs : nullptr;
    {
        KernelBracket kb1(st, 1);
        EP_CUDA_CHECK(launch(epk::stream_gate_up_fp4_kernel, grid, epk::kF4Threads,
                             epk::F4Smem::alloc, st, gm, ga));
    }
    epk::F4DnArgs da;
    da.T = (int)T; da.H = (int)H; da.E = (int)E; da.I = (int)I; da.I_s = (int)I_s;
    da.top_k = top_k; da.ids = ids; da.weights = weights;
    da.wd = mat(w_down, H, I); da.sd = mat(ws_down, H, I_s);
    da.c = c; da.s = sh;
    {
        KernelBracket kb2(st, 2);
        EP_CUDA_CHECK(launch(epk::stream_down_fp4_kernel, grid, epk::kF4Threads,
                             epk::F4DnSmem::alloc, st, dm, da));
    }
    {
        KernelBracket kb3(st, 3);
        const dim3 cgrid((unsigned)T, (unsigned)((H / 4 + 63) / 64));
        EP_CUDA_CHECK(launch(epk::combine_kernel, cgrid, 64, 0, st, (const float *)c,
                             (const float *)(I_s > 0 ? sh : nullptr), ids, (int64_t)T, (int)H,
                             (int)top_k, (int)E, y));
    }
    t_launches = 4;
    return ok();
}

// ======================================================== expert parallel
// One rank's band partial and the rank-order combine of all partials.

namespace {

size_t partial_ids_offset(int64_t T, int64_t H, int64_t E_band, int64_t k, int64_t I) {
    return align256(workspace_layout(T, H, E_band, k, I, 0).total);
}

}  // namespace

extern "C" size_t moe_ffn_partial_workspace_size(int64_t T, int64_t H, int64_t E_band,
                                                 int32_t top_k, int64_t I) {
    if (T <= 0 || H <= 0 || E_band <= 0 || top_k <= 0 || I <= 0)
        return 0;
    return partial_ids_offset(T, H, E_band, top_k, I) + align256((size_t)T * top_k * 4);
}

extern "C" ep_status moe_ffn_partial(const void *x, ep_dtype x_dtype, int64_t T, int64_t H,
                                     const int32_t *ids, const float *weights, int32_t top_k,
                                     const void *w_gate, const void *w_up, const void *w_down,
                                     int64_t I, const ep_plan_t *plan, int32_t rank,
                                     float *partial, void *workspace, size_t workspace_bytes,
                                     void *stream) {
    if (plan == nullptr)
        return fail(EP_EINVAL, "moe_ffn_partial: plan is NULL");
    const int64_t E = plan->num_experts;
    if (E < 1 || E > kMaxE || plan->bands < 1 || plan->bands > EP_MAX_BANDS ||
        plan->bands > E || plan->band_start[0] != 0 || plan->band_start[plan->bands] != E)
        return fail(EP_EINVAL, "moe_ffn_partial: plan is not a partition of [0, E)");
    for (int r = 0; r < plan->bands; ++r)
        if (plan->band_start[r + 1] <= plan->band_start[r])
            return fail(EP_EINVAL, "moe_ffn_partial: band %d of the plan is empty or reversed", r);
    if (rank < 0 || rank >= plan->bands)
        return fail(EP_EINVAL, "moe_ffn_partial: rank %d outside [0, %d)", rank, plan->bands);
    if (T < 0 || T > kMaxT || T * (int64_t)std::max(top_k, 1) > kMaxPairs)
        return fail(EP_EINVAL, "moe_ffn_partial: T = %lld out of range", (long long)T);
    if (top_k < 1 || top_k > kMaxTopK || top_k > E)
        return fail(EP_EINVAL, "moe_ffn_partial: top_k = %d outside [1, min(E, %d)]", top_k,
                    kMaxTopK);
    if (T == 0) {
        t_launches = 0;
        return ok();
    }
    if (ids == nullptr || partial == nullptr)
        return fail(EP_EINVAL, "moe_ffn_partial: a required pointer is NULL");
    if (!aligned(ids, 4))
        return fail(EP_EINVAL, "moe_ffn_partial: ids not 4-byte aligned");
    const int32_t e_lo = plan->band_start[rank], e_hi = plan->band_start[rank + 1];
    const int64_t E_band = e_hi - e_lo;
    const size_t need = moe_ffn_partial_workspace_size(T, H, E_band, top_k, I);
    if (workspace == nullptr || workspace_bytes < need || need == 0)
        return fail(EP_ENOMEM, "moe_ffn_partial: workspace of %zu bytes, %zu needed",
                    workspace_bytes, need);
    if (!aligned(workspace, 256))
        return fail(EP_EINVAL, "moe_ffn_partial: workspace not 256-byte aligned");
    const size_t ids_off = partial_ids_offset(T, H, E_band, top_k, I);
    int32_t *local = reinterpret_cast<int32_t *>(static_cast<uint8_t *>(workspace) + ids_off);
    const DeviceInfo *d = nullptr;
    ep_status s = device_info(&d);
    if (s != EP_OK)
        return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int64_t n = T * top_k;
    {
        const unsigned blocks = (unsigned)std::min<int64_t>((n + 255) / 256, (int64_t)d->sm_count * 4);
        EP_CUDA_CHECK(launch(epk::ep_band_ids_kernel, dim3(blocks), 256, 0, st, ids, n, (int32_t)E,
                             e_lo, e_hi, local));
    }
    // the band's picks through the single-band forward, without the shared expert
    ep_plan_t band;
    memset(&band, 0, sizeof band);
    band.num_experts = (int32_t)E_band;
    band.bands = 1;
    band.band_start[0] = 0;
    band.band_start[1] = (int32_t)E_band;
    s = ffn_forward_impl(true, x, x_dtype, T, H, local, weights, top_k, w_gate, w_up, w_down,
                         E_band, I, nullptr, nullptr, nullptr, 0, &band, partial, workspace,
                         ids_off, stream);
    if (s != EP_OK)
        return s;
    t_launches += 1;
    return ok();
}

extern "C" ep_status moe_ep_combine(const float *partials, int64_t T, int64_t H,
                                    const int32_t *ids, int32_t top_k, const ep_plan_t *plan,
                                    const float *shared, float *y, void *stream) {
    if (plan == nullptr)
        return fail(EP_EINVAL, "moe_ep_combine: plan is NULL");
    const int64_t E = plan->num_experts;
    if (E < 1 || plan->bands < 1 || plan->bands > EP_MAX_BANDS || plan->bands > E ||
        plan->band_start[0] != 0 || plan->band_start[plan->bands] != E)
        return fail(EP_EINVAL, "moe_ep_combine: plan is not a partition of [0, E)");
    for (int r = 0; r < plan->bands; ++r)
        if (plan->band_start[r + 1] <= plan->band_start[r])
            return fail(EP_EINVAL, "moe_ep_combine: band %d of the plan is empty or reversed", r);
    if (T < 0 || T > kMaxT || H < 1 || H > kMaxH || top_k < 1 || top_k > kMaxTopK)
        return fail(EP_EINVAL, "moe_ep_combine: T = %lld, H = %lld or top_k = %d out of range",
                    (long long)T, (long long)H, top_k);
    if (T == 0) {
        t_launches = 0;
        return ok();
    }
    if (partials == nullptr || ids == nullptr || y == nullptr)
        return fail(EP_EINVAL, "moe_ep_combine: a required pointer is NULL");
    if (!aligned(partials, 4) || !aligned(ids, 4) || !aligned(y, 4) ||
        (shared != nullptr && !aligned(shared, 4)))
        return fail(EP_EINVAL, "moe_ep_combine: misaligned pointer");
    const DeviceInfo *d = nullptr;
    const ep_status s = device_info(&d);
    if (s != EP_OK)
        return s;
    epk::EpBands bands;
    memset(&bands, 0, sizeof bands);
    for (int r = 0; r <= plan->bands; ++r)
        bands.start[r] = plan->band_start[r];
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const dim3 grid((unsigned)((H + epk::kEpCombineThreads - 1) / epk::kEpCombineThreads),
                    (unsigned)T);
    EP_CUDA_CHECK(launch(epk::ep_combine_kernel, grid, epk::kEpCombineThreads, 0, st, partials, T,
                         (int)H, ids, top_k, (int)E, bands, plan->bands, shared, y));
    t_launches = 1;
    return ok();
}

// ============================================================ no-alloc variant
// A fixed scratch area that lives in this library's own device memory (one
// copy per device, created when the CUDA runtime loads the library's kernels
// onto it), for callers that must not allocate.
static __device__ __align__(256) unsigned char ep_static_scratch[EP_STATIC_SCRATCH_BYTES];

namespace {

void *g_static_scratch[kMaxDevices];  // per device, guarded by g_device_mu

// Address of the current device's copy of ep_static_scratch, looked up once
// per device with that device current.
ep_status static_scratch(void **out) {
    int dev = 0;
    EP_CUDA_CHECK(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kMaxDevices)
        return fail(EP_ECUDA, "device ordinal %d out of range", dev);
    std::lock_guard<std::mutex> lock(g_device_mu);
    if (g_static_scratch[dev] == nullptr) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, ep_static_scratch);
        if (e != cudaSuccess || p == nullptr)
            return fail(EP_ECUDA, "moe_ffn_forward_noalloc: looking up the static scratch on "
                                  "device %d failed: %s", dev, cudaGetErrorString(e));
        g_static_scratch[dev] = p;
    }
    *out = g_static_scratch[dev];
    return EP_OK;
}

}  // namespace

extern "C" ep_status moe_ffn_forward_noalloc(const void *x, ep_dtype x_dtype, int64_t T,
                                             int64_t H, const int32_t *ids,
                                             const float *weights, int32_t top_k,
                                             const void *w_gate, const void *w_up,
                                             const void *w_down, int64_t E, int64_t I,
                                             const void *ws_gate, const void *ws_up,
                                             const void *ws_down, int64_t I_s,
                                             const ep_plan_t *plan, float *y, void *stream) {
    // sizes beyond the scratch are refused before anything else happens
    const size_t need = moe_ffn_workspace_size(T, H, E, top_k, I, I_s);
    if (need > (size_t)EP_STATIC_SCRATCH_BYTES)
        return fail(EP_ENOMEM, "moe_ffn_forward_noalloc: these sizes need %zu bytes of scratch, "
                               "more than the %zu bytes of its static scratch; call "
                               "moe_ffn_forward with a workspace instead",
                    need, (size_t)EP_STATIC_SCRATCH_BYTES);
    void *scratch = nullptr;
    const ep_status s = static_scratch(&scratch);
    if (s != EP_OK)
        return s;
    // Nothing in the scratch has to start at zero: every byte that either
    // path reads is written earlier in the same call, as with a caller's
    // workspace.
    return moe_ffn_forward(x, x_dtype, T, H, ids, weights, top_k, w_gate, w_up, w_down, E, I,
                           ws_gate, ws_up, ws_down, I_s, plan, y, scratch,
                           (size_t)EP_STATIC_SCRATCH_BYTES, stream);
}
