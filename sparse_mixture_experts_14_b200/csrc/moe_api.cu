// C ABI of the MoE layer: argument checks, workspace, launch orchestration.
// Every step of the layer runs in this library's kernels; nothing here
// computes on the host.  See include/moe.h for the contract of each call.
#include <climits>
#include <cstdlib>
#include <mutex>

#include <nvtx3/nvToolsExt.h>

#include "moe_common.cuh"
#include "ptx_sm100.cuh"

namespace moe {

// NVTX ranges around the layer's host-side stages, nested in one range per
// call, so a profiler timeline (Nsight Systems) or an ncu --nvtx filter can
// tell the stages apart.  Without a tool attached every call is a no-op.
class NvtxStages {
   public:
    NvtxStages(const char* call, const char* const* names, int n) : names_(names), n_(n) { nvtxRangePushA(call); }
    ~NvtxStages() {
        if (open_) nvtxRangePop();
        nvtxRangePop();
    }
    // close the current stage's range and open stage i's (i == n closes only)
    void next(int i) {
        if (open_) nvtxRangePop();
        open_ = i >= 0 && i < n_;
        if (open_) nvtxRangePushA(names_[i]);
    }

   private:
    const char* const* names_;
    int n_;
    bool open_ = false;
};

const char* const kFwdStageNames[MOE_NUM_STAGES] = {"moe.route", "moe.dispatch", "moe.gather",
                                                    "moe.expert1", "moe.expert2", "moe.combine"};
const char* const kBwdStageNames[MOE_BWD_NUM_STAGES] = {"moe.bwd.scatter", "moe.bwd.dgrad_h", "moe.bwd.swiglu",
                                                        "moe.bwd.dgrad_x", "moe.bwd.wgrad2", "moe.bwd.wgrad13",
                                                        "moe.bwd.router"};

__device__ int g_status;   // per-device sticky fault word (first fault wins)

namespace {

constexpr int kMaxDevices = 64;
// Chunks of the host entry point's pipelined path: a short first chunk (its copy in is the only
// one the layer waits for), a short last one (its copy out is the only one that follows the
// layer) and middle chunks in between.  Every chunk streams all touched expert weights once and
// pads each expert's rows to whole tiles, so the middle chunks stay few and large; the first
// chunk's layer has to last about as long as the copy in of the first middle chunk, which is why
// large batches take a longer first chunk (measured at the 8x22B shape, 16384 tokens: 1024-token
// edges around two 7168-token middles 17.6 ms per call, 2560-token edges around one 11264-token
// middle 16.9 ms).  Batches below kHostSplit3 run as two halves.
constexpr int kHostChunkMin = 4096;   // smaller batches run in one piece
constexpr int kHostSplit3 = 8192;
constexpr int kHostEdge = 1024;       // kHostSplit3 <= T < kHostLarge
constexpr int kHostMid = 7168;
constexpr int kHostLarge = 12288;
constexpr int kHostEdgeL = 2560;      // T >= kHostLarge
constexpr int kHostMidL = 11264;
constexpr int kMaxHostChunks = 64;     // at most this many chunks (larger batches take larger middle chunks)

std::mutex g_mu;
cudaMemPool_t g_pools[kMaxDevices] = {};
int* g_status_ptr[kMaxDevices] = {};
int g_num_sms[kMaxDevices] = {};

long long wait_limit_ns() {
    static long long v = [] {
        const char* s = std::getenv("MOE_WAIT_LIMIT_MS");
        long long ms = s ? std::atoll(s) : 1000;
        if (ms < 1) ms = 1;
        return ms * 1000000LL;
    }();
    return v;
}

struct DeviceState {
    cudaMemPool_t pool;
    int* status;
    int num_sms;
};

bool device_state(int dev, DeviceState* st) {
    if (dev < 0 || dev >= kMaxDevices) return false;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_pools[dev]) {
        cudaMemPoolProps props = {};
        props.allocType = cudaMemAllocationTypePinned;
        props.location.type = cudaMemLocationTypeDevice;
        props.location.id = dev;
        cudaMemPool_t pool;
        if (cudaMemPoolCreate(&pool, &props) != cudaSuccess) return false;
        uint64_t thr = UINT64_MAX;
        cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &thr);
        void* sp = nullptr;
        if (cudaGetSymbolAddress(&sp, g_status) != cudaSuccess) return false;
        int n = 0;
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        g_status_ptr[dev] = static_cast<int*>(sp);
        g_num_sms[dev] = n;
        g_pools[dev] = pool;
    }
    st->pool = g_pools[dev];
    st->status = g_status_ptr[dev];
    st->num_sms = g_num_sms[dev];
    return true;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Sizes every entry point shares.
moe_status check_sizes(int T, int d, int E, int k) {
    if (T < 0 || d <= 0 || E <= 0 || k <= 0 || k > E) return MOE_ERR_INVALID_ARG;
    if (E > kMaxExperts) return MOE_ERR_UNSUPPORTED;
    if ((long long)T * k + (long long)E * kSegRows >= INT_MAX) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

moe_status check_layer(const void* x, const void* Wg, const void* W1, const void* W3, const void* W2, const void* out,
                       int T, int d, int F, int E, int k, int dtype) {
    moe_status st = check_sizes(T, d, E, k);
    if (st != MOE_OK) return st;
    if (F <= 0) return MOE_ERR_INVALID_ARG;
    if (dtype == MOE_DTYPE_BF16) {
        if (d % 64 != 0 || F % 128 != 0) return MOE_ERR_UNSUPPORTED;
    } else if (dtype == MOE_DTYPE_F32) {
        if (d % 4 != 0) return MOE_ERR_UNSUPPORTED;
    } else {
        return MOE_ERR_INVALID_ARG;
    }
    if (T == 0) return MOE_OK;
    const void* ptrs[6] = {x, Wg, W1, W3, W2, out};
    for (const void* p : ptrs)
        if (!p || !aligned16(p)) return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

struct Plan {
    size_t idx, w, blk, meta, perm, inv, xp, h, y;
    size_t rstd, logits, bal;   // block form only (see make_plan's `block`)
    size_t keep_a, keep_b;      // training path, bf16: GEMM1's a and b, fp32 [slots][F]
    size_t tlogits;             // training path: the router scores, fp32 [T][E]
    size_t total;
    size_t slots;
};

// Workspace layout.  The block form adds each row's norm factor [T], the fp32
// scores [T][E] and the load-balance partial sums.
Plan make_plan(int T, int d, int F, int E, int k, int dtype, bool block = false, bool train = false) {
    Plan p{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = align_up(off + (bytes ? bytes : 1), 256);
        return o;
    };
    const size_t es = dtype == MOE_DTYPE_BF16 ? 2 : 4;
    const size_t tk = (size_t)T * k;
    p.slots = slots_capacity(T, E, k);
    p.idx = take(tk * 4);
    p.w = take(tk * 4);
    p.blk = take((size_t)dispatch_blocks(T) * E * 4);
    p.meta = take(sizeof(Meta));
    p.perm = take(p.slots * 4);
    p.inv = take(tk * 4);
    p.xp = take(p.slots * (size_t)d * es);
    p.h = take(p.slots * (size_t)F * es);
    p.y = take(p.slots * (size_t)d * 4);
    if (train && dtype == MOE_DTYPE_BF16) {
        p.keep_a = take(p.slots * (size_t)F * 4);
        p.keep_b = take(p.slots * (size_t)F * 4);
    }
    if (train) p.tlogits = take((size_t)T * E * 4);
    if (block) {
        p.rstd = take((size_t)T * 4);
        p.logits = take((size_t)T * E * 4);
        p.bal = take(balance_part_bytes(T, E));
    }
    p.total = off;
    return p;
}

// The block form's extra operands and outputs (null for the plain layer).
struct BlockArgs {
    const void* gamma;
    float eps;
    float alpha;
    float* stats;   // [2E + 1] or null
};

moe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

#define MOE_TRY(call)                                  \
    do {                                               \
        cudaError_t _e = (call);                       \
        if (_e != cudaSuccess) return MOE_ERR_CUDA;    \
    } while (0)

moe_status run_layer(const void* x, const void* Wg, const void* W1, const void* W3, const void* W2, void* out, int T,
                     int d, int F, int E, int k, int dtype, int path, uint8_t* ws, const DeviceState& dev,
                     cudaStream_t s, cudaEvent_t* ev = nullptr, int* launches = nullptr,
                     const BlockArgs* bo = nullptr) {
    const bool train = path == MOE_PATH_TRAIN;
    const Plan p = make_plan(T, d, F, E, k, dtype, bo != nullptr, train);
    RouteExtras ex;
    ex.status = dev.status;
    ex.wait_ns = wait_limit_ns();
    GatherNorm nm;
    if (bo) {
        ex.gamma = bo->gamma;
        ex.eps = bo->eps;
        ex.rstd = reinterpret_cast<float*>(ws + p.rstd);
        if (bo->stats) ex.logits = reinterpret_cast<float*>(ws + p.logits);
        nm.gamma = bo->gamma;
        nm.rstd = ex.rstd;
    }
    const void* resid = bo ? x : nullptr;
    if (train) ex.logits = reinterpret_cast<float*>(ws + p.tlogits);   // kept for the load-balance gradient
    int32_t* idx = reinterpret_cast<int32_t*>(ws + p.idx);
    float* w = reinterpret_cast<float*>(ws + p.w);
    int32_t* blk = reinterpret_cast<int32_t*>(ws + p.blk);
    Meta* meta = reinterpret_cast<Meta*>(ws + p.meta);
    int32_t* perm = reinterpret_cast<int32_t*>(ws + p.perm);
    int32_t* inv = reinterpret_cast<int32_t*>(ws + p.inv);
    void* xp = ws + p.xp;
    void* h = ws + p.h;
    float* y = reinterpret_cast<float*>(ws + p.y);

    NvtxStages nvtx(bo ? "moe.block_forward" : "moe.forward", kFwdStageNames, MOE_NUM_STAGES);
    auto mark = [&](int stage) -> cudaError_t {
        nvtx.next(stage);
        return ev ? cudaEventRecord(ev[stage], s) : cudaSuccess;
    };
    int n = 0;
    MOE_TRY(mark(MOE_STAGE_ROUTE));
    if (dtype == MOE_DTYPE_BF16) {
        MOE_TRY(launch_router_bf16(x, Wg, T, d, E, k, idx, w, dev.num_sms, s, ex));
    } else {
        MOE_TRY(launch_router_f32(static_cast<const float*>(x), static_cast<const float*>(Wg), T, d, E, k, idx, w,
                                  dev.num_sms, s, ex));
    }
    n += 1;
    if (bo && bo->stats) {
        MOE_TRY(launch_balance(ex.logits, idx, T, E, k, bo->alpha, ws + p.bal, bo->stats, s));
        n += 2;
    }
    MOE_TRY(mark(MOE_STAGE_DISPATCH));
    const size_t es = dtype == MOE_DTYPE_BF16 ? 2 : 4;
    if (dtype == MOE_DTYPE_BF16 && T <= kDecodeMaxTokens &&
        (path == MOE_PATH_DECODE || path == MOE_PATH_AUTO)) {
        // decode path: one launch sorts and gathers the token rows (the gather stage is empty)
        MOE_TRY(launch_dispatch_gather_small(idx, T, E, k, x, es, d, meta, perm, inv, xp, p.slots, dev.status, s, nm));
        n += 1;
        MOE_TRY(mark(MOE_STAGE_GATHER));
    } else {
        MOE_TRY(launch_dispatch(idx, T, E, k, blk, meta, perm, inv, dev.status, s));
        n += dispatch_launches(T);
        MOE_TRY(mark(MOE_STAGE_GATHER));
        MOE_TRY(launch_gather(x, es, T, d, E, k, meta, perm, xp, p.slots, dev.status, s, nm));
        n += 1;
    }
    if (dtype == MOE_DTYPE_BF16) {
        TcGemmArgs a{xp, W1, W3, W2, h, y, meta, E, d, F, p.slots, dev.num_sms, dev.status, wait_limit_ns()};
        const bool decode = path == MOE_PATH_DECODE || (path == MOE_PATH_AUTO && T <= kDecodeMaxTokens);
        MOE_TRY(mark(MOE_STAGE_EXPERT1));
        if (train) {
            MOE_TRY(launch_tc_gemm1_train(a, reinterpret_cast<float*>(ws + p.keep_a),
                                          reinterpret_cast<float*>(ws + p.keep_b), s));
        } else {
            MOE_TRY(decode ? launch_decode(a, 1, s) : launch_tc_gemm1(a, s));
        }
        MOE_TRY(mark(MOE_STAGE_EXPERT2));
        MOE_TRY(decode ? launch_decode(a, 2, s) : launch_tc_gemm2(a, s));
        MOE_TRY(mark(MOE_STAGE_COMBINE));
        MOE_TRY(launch_combine_bf16(y, w, inv, T, d, k, p.slots, dev.status, out, s, resid));
    } else {
        MOE_TRY(mark(MOE_STAGE_EXPERT1));
        MOE_TRY(launch_simt_gemm1_f32(static_cast<const float*>(xp), static_cast<const float*>(W1),
                                      static_cast<const float*>(W3), meta, E, d, F, static_cast<float*>(h), p.slots,
                                      s));
        MOE_TRY(mark(MOE_STAGE_EXPERT2));
        MOE_TRY(launch_simt_gemm2_f32(static_cast<const float*>(h), static_cast<const float*>(W2), meta, E, d, F, y,
                                      p.slots, s));
        MOE_TRY(mark(MOE_STAGE_COMBINE));
        MOE_TRY(launch_combine_f32(y, w, inv, T, d, k, p.slots, dev.status, static_cast<float*>(out), s,
                                   static_cast<const float*>(resid)));
    }
    n += 3;
    MOE_TRY(mark(MOE_NUM_STAGES));
    if (launches) *launches = n;
    return MOE_OK;
}

moe_status forward_pooled(const void* x, const void* Wg, const void* W1, const void* W3, const void* W2, void* out,
                          int T, int d, int F, int E, int k, int dtype, cudaStream_t s) {
    moe_status st = check_layer(x, Wg, W1, W3, W2, out, T, d, F, E, k, dtype);
    if (st != MOE_OK || T == 0) return st;
    DeviceState dev;
    const DeviceScope scope(x, false);
    if (!device_state(scope.device(), &dev)) return MOE_ERR_CUDA;
    const Plan p = make_plan(T, d, F, E, k, dtype);
    void* ws = nullptr;
    if (cudaMallocFromPoolAsync(&ws, p.total, dev.pool, s) != cudaSuccess) return MOE_ERR_WORKSPACE;
    st = run_layer(x, Wg, W1, W3, W2, out, T, d, F, E, k, dtype, MOE_PATH_AUTO, static_cast<uint8_t*>(ws), dev, s);
    if (cudaFreeAsync(ws, s) != cudaSuccess && st == MOE_OK) st = MOE_ERR_CUDA;
    return st;
}

// Checks of the block form's extra arguments (after check_layer).
moe_status check_block(const void* h, const void* gamma, float eps, float alpha, const float* stats, const void* out,
                       int T, int d, int dtype) {
    if (!(eps >= 0.f) || !(eps <= 3.4e38f) || !(alpha == alpha) || !(alpha - alpha == 0.f)) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!gamma || !aligned16(gamma)) return MOE_ERR_INVALID_ARG;
    if (stats && (reinterpret_cast<uintptr_t>(stats) & 3u) != 0) return MOE_ERR_INVALID_ARG;
    // out may be h itself (each element reads its h before writing it), no other overlap
    const size_t row = (size_t)d * (dtype == MOE_DTYPE_BF16 ? 2 : 4);
    const uintptr_t hb = reinterpret_cast<uintptr_t>(h), ob = reinterpret_cast<uintptr_t>(out);
    const uintptr_t he = hb + row * (size_t)T, oe = ob + row * (size_t)T;
    if (ob != hb && ob < he && hb < oe) return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

moe_status block_pooled(const void* h, const void* gamma, float eps, const void* Wg, const void* W1, const void* W3,
                        const void* W2, void* out, int T, int d, int F, int E, int k, float alpha, float* stats,
                        int dtype, cudaStream_t s) {
    moe_status st = check_layer(h, Wg, W1, W3, W2, out, T, d, F, E, k, dtype);
    if (st == MOE_OK) st = check_block(h, gamma, eps, alpha, stats, out, T, d, dtype);
    if (st != MOE_OK || T == 0) return st;
    DeviceState dev;
    const DeviceScope scope(h, false);
    if (!device_state(scope.device(), &dev)) return MOE_ERR_CUDA;
    const Plan p = make_plan(T, d, F, E, k, dtype, true);
    void* ws = nullptr;
    if (cudaMallocFromPoolAsync(&ws, p.total, dev.pool, s) != cudaSuccess) return MOE_ERR_WORKSPACE;
    const BlockArgs bo{gamma, eps, alpha, stats};
    st = run_layer(h, Wg, W1, W3, W2, out, T, d, F, E, k, dtype, MOE_PATH_AUTO, static_cast<uint8_t*>(ws), dev, s,
                   nullptr, nullptr, &bo);
    if (cudaFreeAsync(ws, s) != cudaSuccess && st == MOE_OK) st = MOE_ERR_CUDA;
    return st;
}

moe_status route_stats(const void* x, const void* Wg, int T, int d, int E, int k, float alpha, int32_t* idx,
                       float* w, float* stats, int dtype, cudaStream_t s) {
    moe_status st = check_sizes(T, d, E, k);
    if (st != MOE_OK) return st;
    if (d % (dtype == MOE_DTYPE_BF16 ? 8 : 4) != 0) return MOE_ERR_UNSUPPORTED;
    if (!(alpha == alpha) || !(alpha - alpha == 0.f)) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!x || !Wg || !idx || !w || !stats || !aligned16(x) || !aligned16(Wg)) return MOE_ERR_INVALID_ARG;
    DeviceState dev;
    const DeviceScope scope(x, false);
    if (!device_state(scope.device(), &dev)) return MOE_ERR_CUDA;
    const size_t lbytes = align_up((size_t)T * E * 4, 256);
    void* scratch = nullptr;
    if (cudaMallocFromPoolAsync(&scratch, lbytes + balance_part_bytes(T, E), dev.pool, s) != cudaSuccess)
        return MOE_ERR_WORKSPACE;
    RouteExtras ex;
    ex.logits = static_cast<float*>(scratch);
    ex.status = dev.status;
    ex.wait_ns = wait_limit_ns();
    cudaError_t e = dtype == MOE_DTYPE_BF16
                        ? launch_router_bf16(x, Wg, T, d, E, k, idx, w, dev.num_sms, s, ex)
                        : launch_router_f32(static_cast<const float*>(x), static_cast<const float*>(Wg), T, d, E, k,
                                            idx, w, dev.num_sms, s, ex);
    if (e == cudaSuccess)
        e = launch_balance(ex.logits, idx, T, E, k, alpha, static_cast<uint8_t*>(scratch) + lbytes, stats, s);
    cudaError_t f = cudaFreeAsync(scratch, s);
    return (e == cudaSuccess && f == cudaSuccess) ? MOE_OK : MOE_ERR_CUDA;
}

// Backward workspace layout (on top of the forward's workspace, which it reads).
struct BwdPlan {
    size_t dy, dg, ds, dh, dab, dxp, dwg, dgam, total;
};

BwdPlan make_bwd_plan(int T, int d, int F, int E, int k, int dtype, bool block = false) {
    BwdPlan b{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = align_up(off + (bytes ? bytes : 1), 256);
        return o;
    };
    const size_t es = dtype == MOE_DTYPE_BF16 ? 2 : 4;
    const size_t S = slots_capacity(T, E, k);
    b.dy = take(S * d * es);
    b.dg = take((size_t)T * k * 4);
    b.ds = take((size_t)T * E * 4);
    b.dh = take(dtype == MOE_DTYPE_BF16 ? 0 : S * F * 4);   // the bf16 path never stores dH
    b.dab = take(S * 2 * (size_t)F * es);
    b.dxp = take(S * d * 4);
    b.dwg = take(dwg_part_bytes(T, E, d));
    if (block) b.dgam = take(block_dgamma_part_bytes(T, d));
    b.total = off;
    return b;
}

moe_status run_backward(const void* x, const void* Wg, const void* W1, const void* W3, const void* W2,
                        const void* dout, void* dx, float* dWg, void* dW1, void* dW3, void* dW2, float* dlogits,
                        float alpha, int wgrad_dtype, int T, int d, int F, int E, int k, int dtype, const uint8_t* fws,
                        uint8_t* bws,
                        const DeviceState& dev, cudaStream_t s, cudaEvent_t* ev, int* launches,
                        const void* gamma = nullptr, float* dgamma = nullptr) {
    const bool block = gamma != nullptr;
    const Plan p = make_plan(T, d, F, E, k, dtype, block, true);
    const BwdPlan b = make_bwd_plan(T, d, F, E, k, dtype, block);
    uint8_t* fw = const_cast<uint8_t*>(fws);
    BwdArgs a{};
    a.bf16 = dtype == MOE_DTYPE_BF16;
    a.x = x;
    a.Wg = Wg;
    a.W1 = W1;
    a.W3 = W3;
    a.W2 = W2;
    a.dout = dout;
    a.idx = reinterpret_cast<const int32_t*>(fw + p.idx);
    a.w = reinterpret_cast<const float*>(fw + p.w);
    a.meta = reinterpret_cast<Meta*>(fw + p.meta);
    a.perm = reinterpret_cast<const int32_t*>(fw + p.perm);
    a.inv = reinterpret_cast<const int32_t*>(fw + p.inv);
    a.xp = fw + p.xp;
    a.H = fw + p.h;
    a.Y = reinterpret_cast<const float*>(fw + p.y);
    a.logits = reinterpret_cast<const float*>(fw + p.tlogits);
    a.alpha = alpha;
    if (dtype == MOE_DTYPE_BF16) {
        a.keep_a = reinterpret_cast<const float*>(fw + p.keep_a);
        a.keep_b = reinterpret_cast<const float*>(fw + p.keep_b);
    }
    a.dy = bws + b.dy;
    a.dg = reinterpret_cast<float*>(bws + b.dg);
    a.ds = dlogits ? dlogits : reinterpret_cast<float*>(bws + b.ds);
    a.dh = reinterpret_cast<float*>(bws + b.dh);
    a.dab = bws + b.dab;
    a.dxp = reinterpret_cast<float*>(bws + b.dxp);
    a.dwg_part = reinterpret_cast<float*>(bws + b.dwg);
    if (block) {
        a.gamma = gamma;
        a.rstd = reinterpret_cast<const float*>(fw + p.rstd);
        a.dgamma = dgamma;
        a.dgamma_part = reinterpret_cast<float*>(bws + b.dgam);
    }
    a.dx = dx;
    a.dWg = dWg;
    a.dW1 = static_cast<float*>(dW1);   // the CUDA-core (fp32) path: fp32 gradients only
    a.dW3 = static_cast<float*>(dW3);
    a.dW2 = static_cast<float*>(dW2);
    a.T = T;
    a.d = d;
    a.F = F;
    a.E = E;
    a.k = k;
    a.slots = p.slots;
    a.status = dev.status;

    NvtxStages nvtx("moe.backward", kBwdStageNames, MOE_BWD_NUM_STAGES);
    auto mark = [&](int stage) -> cudaError_t {
        nvtx.next(stage);
        return ev ? cudaEventRecord(ev[stage], s) : cudaSuccess;
    };
    int n = 0;
    MOE_TRY(mark(MOE_BWD_STAGE_SCATTER));
    MOE_TRY(launch_bwd_scatter(a, s));
    MOE_TRY(launch_router_bwd(a, s));
    n += 2;
    if (a.bf16) {
        TcBwdArgs t{};
        t.xp = a.xp;
        t.W1 = W1;
        t.W3 = W3;
        t.W2 = W2;
        t.H = a.H;
        t.keep_a = a.keep_a;
        t.keep_b = a.keep_b;
        t.dy = a.dy;
        t.dab = a.dab;
        t.dxp = a.dxp;
        t.dW1 = dW1;
        t.dW3 = dW3;
        t.dW2 = dW2;
        t.wgrad_bf16 = wgrad_dtype == MOE_DTYPE_BF16;
        t.meta = a.meta;
        t.E = E;
        t.d = d;
        t.F = F;
        t.slots = p.slots;
        t.num_sms = dev.num_sms;
        t.status = dev.status;
        t.wait_ns = wait_limit_ns();
        MOE_TRY(mark(MOE_BWD_STAGE_DGRAD_H));
        MOE_TRY(launch_tc_dgrad_h(t, s));   // SwiGLU backward fused into its epilogue
        MOE_TRY(mark(MOE_BWD_STAGE_SWIGLU));
        MOE_TRY(mark(MOE_BWD_STAGE_DGRAD_X));
        MOE_TRY(launch_tc_dgrad_x(t, s));
        MOE_TRY(mark(MOE_BWD_STAGE_WGRAD2));
        MOE_TRY(launch_tc_wgrad2(t, s));
        MOE_TRY(mark(MOE_BWD_STAGE_WGRAD13));
        MOE_TRY(launch_tc_wgrad13(t, s));
        n += 4;
    } else {
        MOE_TRY(mark(MOE_BWD_STAGE_DGRAD_H));
        MOE_TRY(mark(MOE_BWD_STAGE_SWIGLU));
        MOE_TRY(mark(MOE_BWD_STAGE_DGRAD_X));
        MOE_TRY(mark(MOE_BWD_STAGE_WGRAD2));
        MOE_TRY(launch_simt_bwd_gemms(a, s));
        MOE_TRY(mark(MOE_BWD_STAGE_WGRAD13));
        n += 5;
    }
    MOE_TRY(mark(MOE_BWD_STAGE_ROUTER));
    MOE_TRY(launch_dwg(a, s));
    MOE_TRY(launch_dx_combine(a, s));
    n += block ? 4 : 3;
    MOE_TRY(mark(MOE_BWD_NUM_STAGES));
    if (launches) *launches = n;
    return MOE_OK;
}

__global__ void wait_selftest_kernel(int* status, long long limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        ptx::mbar_init(&bar, 1);   // nothing ever arrives on this barrier
        abort_flag = 0;
        ptx::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const ptx::WaitCtl wc{&abort_flag, status, (uint64_t)limit_ns};
        ptx::mbar_wait(&bar, 0, wc);
    }
    __syncthreads();
}

}  // namespace

// Address of the status word on device `dev` (current), resolved once; creates no memory pool.
int* status_word(int dev) {
    static std::mutex mu;
    static int* ptrs[kMaxDevices] = {};
    if (dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lk(mu);
    if (!ptrs[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess) return nullptr;
        ptrs[dev] = static_cast<int*>(p);
    }
    return ptrs[dev];
}

// Two copy streams per device for the host entry point (host-to-device, device-to-host), created
// on first use, non-blocking (they never wait for the legacy default stream).
bool copy_streams(int dev, cudaStream_t* h2d, cudaStream_t* d2h) {
    static std::mutex mu;
    static cudaStream_t streams[kMaxDevices][2] = {};
    if (dev < 0 || dev >= kMaxDevices) return false;
    std::lock_guard<std::mutex> lk(mu);
    for (int i = 0; i < 2; ++i)
        if (!streams[dev][i] && cudaStreamCreateWithFlags(&streams[dev][i], cudaStreamNonBlocking) != cudaSuccess) {
            streams[dev][i] = nullptr;
            cudaGetLastError();
            return false;
        }
    *h2d = streams[dev][0];
    *d2h = streams[dev][1];
    return true;
}

// The library's stream-ordered pool on device `dev` (current), created on first use; null on failure.
cudaMemPool_t library_pool(int dev) {
    DeviceState st;
    return device_state(dev, &st) ? st.pool : nullptr;
}

// SM count of device `dev` (0 if unknown: launchers then assume 148).
int device_sms(int dev) {
    DeviceState st;
    return device_state(dev, &st) ? st.num_sms : 0;
}

// Time limit of one pipeline wait (MOE_WAIT_LIMIT_MS, default 1 s).
long long pipeline_wait_ns() { return wait_limit_ns(); }

}  // namespace moe

using namespace moe;

extern "C" {

moe_status moe_pool_stats(int device, size_t* reserved, size_t* used) {
    if (!reserved || !used || device < 0 || device >= kMaxDevices) return MOE_ERR_INVALID_ARG;
    *reserved = 0;
    *used = 0;
    cudaMemPool_t pool;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        pool = g_pools[device];
    }
    if (!pool) return MOE_OK;
    uint64_t r = 0, u = 0;
    if (cudaMemPoolGetAttribute(pool, cudaMemPoolAttrReservedMemCurrent, &r) != cudaSuccess ||
        cudaMemPoolGetAttribute(pool, cudaMemPoolAttrUsedMemCurrent, &u) != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    *reserved = (size_t)r;
    *used = (size_t)u;
    return MOE_OK;
}

moe_status moe_route(const void* x, const void* Wg, int T, int d, int E, int k, int32_t* topk_idx, float* topk_w,
                     cudaStream_t stream) {
    moe_status st = check_sizes(T, d, E, k);
    if (st != MOE_OK) return st;
    if (d % 8 != 0) return MOE_ERR_UNSUPPORTED;
    if (T == 0) return MOE_OK;
    if (!x || !Wg || !topk_idx || !topk_w || !aligned16(x) || !aligned16(Wg)) return MOE_ERR_INVALID_ARG;
    DeviceState dev;
    const DeviceScope scope(x, false);
    if (!device_state(scope.device(), &dev)) return MOE_ERR_CUDA;
    RouteExtras ex;
    ex.status = dev.status;
    ex.wait_ns = wait_limit_ns();
    return cuda_status(launch_router_bf16(x, Wg, T, d, E, k, topk_idx, topk_w, dev.num_sms, stream, ex));
}

moe_status moe_route_f32(const float* x, const float* Wg, int T, int d, int E, int k, int32_t* topk_idx,
                         float* topk_w, cudaStream_t stream) {
    moe_status st = check_sizes(T, d, E, k);
    if (st != MOE_OK) return st;
    if (d % 4 != 0) return MOE_ERR_UNSUPPORTED;
    if (T == 0) return MOE_OK;
    if (!x || !Wg || !topk_idx || !topk_w || !aligned16(x) || !aligned16(Wg)) return MOE_ERR_INVALID_ARG;
    DeviceState dev;
    const DeviceScope scope(x, false);
    if (!device_state(scope.device(), &dev)) return MOE_ERR_CUDA;
    return cuda_status(launch_router_f32(x, Wg, T, d, E, k, topk_idx, topk_w, dev.num_sms, stream));
}

size_t moe_slots_capacity(int T, int E, int k) {
    if (check_sizes(T, 1, E, k) != MOE_OK) return 0;
    return slots_capacity(T, E, k);
}

moe_status moe_dispatch(const int32_t* topk_idx, int T, int E, int k, int32_t* counts, int32_t* offsets,
                        int32_t* perm, int32_t* inv, cudaStream_t stream) {
    moe_status st = check_sizes(T, 1, E, k);
    if (st != MOE_OK) return st;
    if (!counts || !offsets || (T > 0 && (!topk_idx || !perm || !inv))) return MOE_ERR_INVALID_ARG;
    DeviceState dev;
    const DeviceScope scope(counts, false);
    if (!device_state(scope.device(), &dev)) return MOE_ERR_CUDA;
    const size_t blk_bytes = align_up((size_t)dispatch_blocks(T) * E * 4 + 1, 256);
    void* scratch = nullptr;
    if (cudaMallocFromPoolAsync(&scratch, blk_bytes + sizeof(Meta), dev.pool, stream) != cudaSuccess)
        return MOE_ERR_WORKSPACE;
    int32_t* blk = static_cast<int32_t*>(scratch);
    Meta* meta = reinterpret_cast<Meta*>(static_cast<uint8_t*>(scratch) + blk_bytes);
    cudaError_t e = cudaSuccess;
    if (T == 0) {
        e = cudaMemsetAsync(meta, 0, sizeof(Meta), stream);
    } else {
        e = launch_dispatch(topk_idx, T, E, k, blk, meta, perm, inv, dev.status, stream);
    }
    if (e == cudaSuccess) e = cudaMemcpyAsync(counts, meta->counts, E * 4, cudaMemcpyDeviceToDevice, stream);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(offsets, meta->offsets, (E + 1) * 4, cudaMemcpyDeviceToDevice, stream);
    cudaError_t f = cudaFreeAsync(scratch, stream);
    return (e == cudaSuccess && f == cudaSuccess) ? MOE_OK : MOE_ERR_CUDA;
}

moe_status moe_forward(const void* x, const void* Wg, const void* W1, const void* W3, const void* W2, void* out, int T,
                       int d, int ffn, int E, int k, cudaStream_t stream) {
    return forward_pooled(x, Wg, W1, W3, W2, out, T, d, ffn, E, k, MOE_DTYPE_BF16, stream);
}

moe_status moe_forward_f32(const float* x, const float* Wg, const float* W1, const float* W3, const float* W2,
                           float* out, int T, int d, int ffn, int E, int k, cudaStream_t stream) {
    return forward_pooled(x, Wg, W1, W3, W2, out, T, d, ffn, E, k, MOE_DTYPE_F32, stream);
}

size_t moe_workspace_size(int T, int d, int ffn, int E, int k, int dtype) {
    if (check_sizes(T, d, E, k) != MOE_OK || ffn <= 0) return 0;
    if (dtype != MOE_DTYPE_BF16 && dtype != MOE_DTYPE_F32) return 0;
    return make_plan(T, d, ffn, E, k, dtype).total;
}

moe_status moe_forward_ws(const void* x, const void* Wg, const void* W1, const void* W3, const void* W2, void* out,
                          int T, int d, int ffn, int E, int k, int dtype, int path, void* workspace,
                          size_t workspace_bytes, cudaStream_t stream) {
    moe_status st = check_layer(x, Wg, W1, W3, W2, out, T, d, ffn, E, k, dtype);
    if (st != MOE_OK) return st;
    if (path != MOE_PATH_AUTO && path != MOE_PATH_PREFILL && path != MOE_PATH_DECODE && path != MOE_PATH_TRAIN)
        return MOE_ERR_INVALID_ARG;
    if (path == MOE_PATH_DECODE && (dtype != MOE_DTYPE_BF16 || T > kDecodeMaxTokens)) return MOE_ERR_UNSUPPORTED;
    if (T == 0) return MOE_OK;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MOE_ERR_WORKSPACE;
    if (workspace_bytes < make_plan(T, d, ffn, E, k, dtype, false, path == MOE_PATH_TRAIN).total)
        return MOE_ERR_WORKSPACE;
    DeviceState dev;
    const DeviceScope scope(x, false);
    if (!device_state(scope.device(), &dev)) return MOE_ERR_CUDA;
    return run_layer(x, Wg, W1, W3, W2, out, T, d, ffn, E, k, dtype, path, static_cast<uint8_t*>(workspace), dev,
                     stream);
}

moe_status moe_forward_profiled(const void* x, const void* Wg, const void* W1, const void* W3, const void* W2,
                                void* out, int T, int d, int ffn, int E, int k, int dtype, int path, void* workspace,
                                size_t workspace_bytes, cudaEvent_t* stage_events, int* launches,
                                cudaStream_t stream) {
    if (launches) *launches = 0;
    moe_status st = check_layer(x, Wg, W1, W3, W2, out, T, d, ffn, E, k, dtype);
    if (st != MOE_OK) return st;
    if (path != MOE_PATH_AUTO && path != MOE_PATH_PREFILL && path != MOE_PATH_DECODE && path != MOE_PATH_TRAIN)
        return MOE_ERR_INVALID_ARG;
    if (path == MOE_PATH_DECODE && (dtype != MOE_DTYPE_BF16 || T > kDecodeMaxTokens)) return MOE_ERR_UNSUPPORTED;
    if (T == 0) return MOE_OK;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MOE_ERR_WORKSPACE;
    if (workspace_bytes < make_plan(T, d, ffn, E, k, dtype, false, path == MOE_PATH_TRAIN).total)
        return MOE_ERR_WORKSPACE;
    DeviceState dev;
    const DeviceScope scope(x, false);
    if (!device_state(scope.device(), &dev)) return MOE_ERR_CUDA;
    return run_layer(x, Wg, W1, W3, W2, out, T, d, ffn, E, k, dtype, path, static_cast<uint8_t*>(workspace), dev,
                     stream, stage_events, launches);
}

// Every chunk of a split batch holds at least kHostEdge tokens, so every chunk takes the
// prefill kernels (the decode path would give its tokens other bits than one call does).
int moe_host_chunk_plan(int T, int* starts, int max_chunks) {
    if (T < 0 || !starts || max_chunks < 1) return 0;
    int n = 1;
    if (T >= kHostSplit3) {
        // an edge-token first and last chunk around near-equal middle ones of up to mid_max
        // tokens (more middle tokens per chunk once the chunk count is at its cap)
        const int edge = T >= kHostLarge ? kHostEdgeL : kHostEdge;
        const int mid_max = T >= kHostLarge ? kHostMidL : kHostMid;
        const int mid = T - 2 * edge;
        const int nmid = min((mid + mid_max - 1) / mid_max, kMaxHostChunks - 2);
        n = nmid + 2;
        if (n > max_chunks) return 0;
        starts[1] = edge;
        for (int c = 0; c < nmid; ++c) starts[2 + c] = starts[1 + c] + mid / nmid + (c < mid % nmid ? 1 : 0);
    } else if (T >= kHostChunkMin) {
        n = 2;   // two halves
        if (n > max_chunks) return 0;
        starts[1] = T / 2;
    }
    starts[0] = 0;
    starts[n] = T;
    return n;
}

moe_status moe_forward_host(const void* x_host, const void* Wg, const void* W1, const void* W3, const void* W2,
                            void* out_host, int T, int d, int ffn, int E, int k, cudaStream_t stream) {
    moe_status st = check_layer(x_host, Wg, W1, W3, W2, out_host, T, d, ffn, E, k, MOE_DTYPE_BF16);
    if (st != MOE_OK || T == 0) return st;
    DeviceState dev;
    const DeviceScope scope(Wg, false);
    if (!device_state(scope.device(), &dev)) return MOE_ERR_CUDA;
    const size_t row = (size_t)d * 2;
    const size_t act = (size_t)T * row;
    const size_t act_al = align_up(act, 256);
    // Batches of 4096 tokens or more run in chunks, so that each chunk's copies overlap
    // another chunk's layer.  Tokens are independent and every kernel of the chunked path gives a
    // token the bits it gets in one call (the tensor-core router adds its K chunks in the same
    // order for any batch; a GEMM row's arithmetic does not depend on its place in a tile), so
    // the result equals the unchunked call bit for bit.
    int cstart[kMaxHostChunks + 1];
    const int nch = moe_host_chunk_plan(T, cstart, kMaxHostChunks);
    if (nch < 1) return MOE_ERR_INVALID_ARG;
    int tc = 0;   // the largest chunk sizes the workspace
    for (int c = 0; c < nch; ++c) tc = max(tc, cstart[c + 1] - cstart[c]);
    const Plan p = make_plan(tc, d, ffn, E, k, MOE_DTYPE_BF16);
    void* buf = nullptr;
    if (cudaMallocFromPoolAsync(&buf, 2 * act_al + p.total, dev.pool, stream) != cudaSuccess)
        return MOE_ERR_WORKSPACE;
    uint8_t* xd = static_cast<uint8_t*>(buf);
    uint8_t* od = xd + act_al;
    uint8_t* ws = od + act_al;
    cudaError_t e = cudaSuccess;
    if (nch == 1) {
        e = cudaMemcpyAsync(xd, x_host, act, cudaMemcpyHostToDevice, stream);
        if (e == cudaSuccess) {
            st = run_layer(xd, Wg, W1, W3, W2, od, T, d, ffn, E, k, MOE_DTYPE_BF16, MOE_PATH_AUTO, ws, dev, stream);
            if (st == MOE_OK) e = cudaMemcpyAsync(out_host, od, act, cudaMemcpyDeviceToHost, stream);
        }
    } else {
        cudaStream_t h2d = nullptr, d2h = nullptr;
        if (!copy_streams(scope.device(), &h2d, &d2h)) e = cudaErrorUnknown;
        // events: [0] the buffer exists; then per chunk "copied in" and "computed"; last "copied out"
        cudaEvent_t ev[2 * kMaxHostChunks + 2] = {};
        const int nev = 2 * nch + 2;
        for (int i = 0; i < nev && e == cudaSuccess; ++i) e = cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventRecord(ev[0], stream);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(h2d, ev[0], 0);
        for (int c = 0; c < nch && e == cudaSuccess; ++c) {
            const size_t t0 = (size_t)cstart[c], n = (size_t)(cstart[c + 1] - cstart[c]);
            e = cudaMemcpyAsync(xd + t0 * row, static_cast<const uint8_t*>(x_host) + t0 * row, n * row,
                                cudaMemcpyHostToDevice, h2d);
            if (e == cudaSuccess) e = cudaEventRecord(ev[1 + c], h2d);
        }
        for (int c = 0; c < nch && e == cudaSuccess && st == MOE_OK; ++c) {
            const size_t t0 = (size_t)cstart[c];
            const int n = cstart[c + 1] - cstart[c];
            e = cudaStreamWaitEvent(stream, ev[1 + c], 0);
            if (e != cudaSuccess) break;
            st = run_layer(xd + t0 * row, Wg, W1, W3, W2, od + t0 * row, n, d, ffn, E, k, MOE_DTYPE_BF16,
                           MOE_PATH_AUTO, ws, dev, stream);
            if (st != MOE_OK) break;
            e = cudaEventRecord(ev[1 + nch + c], stream);
            if (e == cudaSuccess) e = cudaStreamWaitEvent(d2h, ev[1 + nch + c], 0);
            if (e == cudaSuccess)
                e = cudaMemcpyAsync(static_cast<uint8_t*>(out_host) + t0 * row, od + t0 * row, (size_t)n * row,
                                    cudaMemcpyDeviceToHost, d2h);
        }
        // the buffer goes back to the pool only after the last copy out
        if (ev[nev - 1]) {
            if (cudaEventRecord(ev[nev - 1], d2h) == cudaSuccess) cudaStreamWaitEvent(stream, ev[nev - 1], 0);
            else cudaStreamSynchronize(d2h);
        }
        if (h2d) cudaStreamSynchronize(h2d);
        for (int i = 0; i < nev; ++i)
            if (ev[i]) cudaEventDestroy(ev[i]);
    }
    cudaError_t f = cudaFreeAsync(buf, stream);
    cudaError_t g = cudaStreamSynchronize(stream);
    if (st != MOE_OK) return st;
    return (e == cudaSuccess && f == cudaSuccess && g == cudaSuccess) ? MOE_OK : MOE_ERR_CUDA;
}

moe_status moe_get_device_status(cudaStream_t stream) {
    if (cudaStreamSynchronize(stream) != cudaSuccess) return MOE_ERR_CUDA;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
    DeviceState st;
    if (!device_state(dev, &st)) return MOE_ERR_CUDA;
    int v = 0;
    if (cudaMemcpy(&v, st.status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
    const int zero = 0;
    if (cudaMemcpy(st.status, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return MOE_ERR_CUDA;
    return static_cast<moe_status>(v);
}

moe_status moe_selftest_wait_timeout(long long limit_ns, cudaStream_t stream) {
    if (limit_ns < 1000 || limit_ns > 10000000000LL) return MOE_ERR_INVALID_ARG;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
    DeviceState st;
    if (!device_state(dev, &st)) return MOE_ERR_CUDA;
    wait_selftest_kernel<<<1, 32, 0, stream>>>(st.status, limit_ns);
    return cuda_status(cudaGetLastError());
}

const char* moe_status_string(moe_status status) {
    switch (status) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument";
        case MOE_ERR_UNSUPPORTED: return "unsupported size";
        case MOE_ERR_CUDA: return "CUDA runtime error";
        case MOE_ERR_TIMEOUT: return "device wait timed out";
        case MOE_ERR_WORKSPACE: return "workspace missing or too small";
        case MOE_ERR_DEVICE: return "device-side input check failed";
    }
    return "unknown status";
}

int moe_decode_max_tokens(void) { return kDecodeMaxTokens; }

size_t moe_block_workspace_size(int T, int d, int ffn, int E, int k, int dtype) {
    if (check_sizes(T, d, E, k) != MOE_OK || ffn <= 0) return 0;
    if (dtype != MOE_DTYPE_BF16 && dtype != MOE_DTYPE_F32) return 0;
    return make_plan(T, d, ffn, E, k, dtype, true).total;
}

moe_status moe_block_forward(const void* h, const void* gamma, float eps, const void* Wg, const void* W1,
                             const void* W3, const void* W2, void* out, int T, int d, int ffn, int E, int k,
                             float alpha, float* stats, cudaStream_t stream) {
    return block_pooled(h, gamma, eps, Wg, W1, W3, W2, out, T, d, ffn, E, k, alpha, stats, MOE_DTYPE_BF16, stream);
}

moe_status moe_block_forward_f32(const float* h, const float* gamma, float eps, const float* Wg, const float* W1,
                                 const float* W3, const float* W2, float* out, int T, int d, int ffn, int E, int k,
                                 float alpha, float* stats, cudaStream_t stream) {
    return block_pooled(h, gamma, eps, Wg, W1, W3, W2, out, T, d, ffn, E, k, alpha, stats, MOE_DTYPE_F32, stream);
}

moe_status moe_block_forward_ws(const void* h, const void* gamma, float eps, const void* Wg, const void* W1,
                                const void* W3, const void* W2, void* out, int T, int d, int ffn, int E, int k,
                                float alpha, float* stats, int dtype, int path, void* workspace,
                                size_t workspace_bytes, cudaEvent_t* stage_events, int* launches,
                                cudaStream_t stream) {
    if (launches) *launches = 0;
    moe_status st = check_layer(h, Wg, W1, W3, W2, out, T, d, ffn, E, k, dtype);
    if (st == MOE_OK) st = check_block(h, gamma, eps, alpha, stats, out, T, d, dtype);
    if (st != MOE_OK) return st;
    if (path != MOE_PATH_AUTO && path != MOE_PATH_PREFILL && path != MOE_PATH_DECODE && path != MOE_PATH_TRAIN)
        return MOE_ERR_INVALID_ARG;
    if (path == MOE_PATH_DECODE && (dtype != MOE_DTYPE_BF16 || T > kDecodeMaxTokens)) return MOE_ERR_UNSUPPORTED;
    if (T == 0) return MOE_OK;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MOE_ERR_WORKSPACE;
    if (workspace_bytes < make_plan(T, d, ffn, E, k, dtype, true, path == MOE_PATH_TRAIN).total)
        return MOE_ERR_WORKSPACE;
    DeviceState dev;
    const DeviceScope scope(h, false);
    if (!device_state(scope.device(), &dev)) return MOE_ERR_CUDA;
    const BlockArgs bo{gamma, eps, alpha, stats};
    return run_layer(h, Wg, W1, W3, W2, out, T, d, ffn, E, k, dtype, path, static_cast<uint8_t*>(workspace), dev,
                     stream, stage_events, launches, &bo);
}

size_t moe_train_workspace_size(int T, int d, int ffn, int E, int k, int dtype) {
    if (check_sizes(T, d, E, k) != MOE_OK || ffn <= 0) return 0;
    if (dtype != MOE_DTYPE_BF16 && dtype != MOE_DTYPE_F32) return 0;
    return make_plan(T, d, ffn, E, k, dtype, false, true).total;
}

size_t moe_backward_workspace_size(int T, int d, int ffn, int E, int k, int dtype) {
    if (check_sizes(T, d, E, k) != MOE_OK || ffn <= 0) return 0;
    if (dtype != MOE_DTYPE_BF16 && dtype != MOE_DTYPE_F32) return 0;
    return make_bwd_plan(T, d, ffn, E, k, dtype).total;
}

moe_status moe_backward_ws(const void* x, const void* Wg, const void* W1, const void* W3, const void* W2,
                           const void* dout, void* dx, float* dWg, void* dW1, void* dW3, void* dW2, float* dlogits,
                           float alpha, int wgrad_dtype, int T, int d, int ffn, int E, int k, int dtype,
                           const void* fwd_workspace,
                           size_t fwd_workspace_bytes, void* workspace, size_t workspace_bytes,
                           cudaEvent_t* stage_events, int* launches, cudaStream_t stream) {
    if (launches) *launches = 0;
    moe_status st = check_layer(x, Wg, W1, W3, W2, dx, T, d, ffn, E, k, dtype);
    if (st != MOE_OK) return st;
    if (T == 0) return MOE_OK;
    const void* ptrs[5] = {dout, dWg, dW1, dW3, dW2};
    for (const void* q : ptrs)
        if (!q || !aligned16(q)) return MOE_ERR_INVALID_ARG;
    if (dlogits && (reinterpret_cast<uintptr_t>(dlogits) & 3u) != 0) return MOE_ERR_INVALID_ARG;
    if (!(alpha == alpha) || !(alpha - alpha == 0.f)) return MOE_ERR_INVALID_ARG;
    if (wgrad_dtype != MOE_DTYPE_F32 && wgrad_dtype != MOE_DTYPE_BF16) return MOE_ERR_INVALID_ARG;
    if (wgrad_dtype == MOE_DTYPE_BF16 && dtype != MOE_DTYPE_BF16) return MOE_ERR_UNSUPPORTED;
    if (!fwd_workspace || (reinterpret_cast<uintptr_t>(fwd_workspace) & 255u) != 0) return MOE_ERR_WORKSPACE;
    if (fwd_workspace_bytes < make_plan(T, d, ffn, E, k, dtype, false, true).total) return MOE_ERR_WORKSPACE;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MOE_ERR_WORKSPACE;
    if (workspace_bytes < make_bwd_plan(T, d, ffn, E, k, dtype).total) return MOE_ERR_WORKSPACE;
    DeviceState dev;
    const DeviceScope scope(x, false);
    if (!device_state(scope.device(), &dev)) return MOE_ERR_CUDA;
    return run_backward(x, Wg, W1, W3, W2, dout, dx, dWg, dW1, dW3, dW2, dlogits, alpha, wgrad_dtype, T, d, ffn, E,
                        k, dtype,
                        static_cast<const uint8_t*>(fwd_workspace), static_cast<uint8_t*>(workspace), dev, stream,
                        stage_events, launches);
}

size_t moe_block_train_workspace_size(int T, int d, int ffn, int E, int k, int dtype) {
    if (check_sizes(T, d, E, k) != MOE_OK || ffn <= 0) return 0;
    if (dtype != MOE_DTYPE_BF16 && dtype != MOE_DTYPE_F32) return 0;
    return make_plan(T, d, ffn, E, k, dtype, true, true).total;
}

size_t moe_block_backward_workspace_size(int T, int d, int ffn, int E, int k, int dtype) {
    if (check_sizes(T, d, E, k) != MOE_OK || ffn <= 0) return 0;
    if (dtype != MOE_DTYPE_BF16 && dtype != MOE_DTYPE_F32) return 0;
    return make_bwd_plan(T, d, ffn, E, k, dtype, true).total;
}

moe_status moe_block_backward_ws(const void* h, const void* gamma, const void* Wg, const void* W1, const void* W3,
                                 const void* W2, const void* dout, void* dh, float* dgamma, float* dWg, void* dW1,
                                 void* dW3, void* dW2, float* dlogits, float alpha, int wgrad_dtype, int T, int d,
                                 int ffn, int E, int k, int dtype, const void* fwd_workspace,
                                 size_t fwd_workspace_bytes, void* workspace, size_t workspace_bytes,
                                 cudaEvent_t* stage_events, int* launches, cudaStream_t stream) {
    if (launches) *launches = 0;
    moe_status st = check_layer(h, Wg, W1, W3, W2, dh, T, d, ffn, E, k, dtype);
    if (st != MOE_OK) return st;
    if (d > 8192) return MOE_ERR_UNSUPPORTED;   // the dh pass holds a row of du in one block's registers
    if (T == 0) return MOE_OK;
    const void* ptrs[7] = {dout, dWg, dW1, dW3, dW2, gamma, dgamma};
    for (const void* q : ptrs)
        if (!q || !aligned16(q)) return MOE_ERR_INVALID_ARG;
    if (dlogits && (reinterpret_cast<uintptr_t>(dlogits) & 3u) != 0) return MOE_ERR_INVALID_ARG;
    if (!(alpha == alpha) || !(alpha - alpha == 0.f)) return MOE_ERR_INVALID_ARG;
    if (wgrad_dtype != MOE_DTYPE_F32 && wgrad_dtype != MOE_DTYPE_BF16) return MOE_ERR_INVALID_ARG;
    if (wgrad_dtype == MOE_DTYPE_BF16 && dtype != MOE_DTYPE_BF16) return MOE_ERR_UNSUPPORTED;
    // dh is written row by row while dout and h of the same row are read: no overlap with either
    const size_t row = (size_t)d * (dtype == MOE_DTYPE_BF16 ? 2 : 4);
    const uintptr_t ob = reinterpret_cast<uintptr_t>(dh), oe = ob + row * (size_t)T;
    for (const void* q : {h, dout}) {
        const uintptr_t b = reinterpret_cast<uintptr_t>(q), e = b + row * (size_t)T;
        if (ob < e && b < oe) return MOE_ERR_INVALID_ARG;
    }
    if (!fwd_workspace || (reinterpret_cast<uintptr_t>(fwd_workspace) & 255u) != 0) return MOE_ERR_WORKSPACE;
    if (fwd_workspace_bytes < make_plan(T, d, ffn, E, k, dtype, true, true).total) return MOE_ERR_WORKSPACE;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MOE_ERR_WORKSPACE;
    if (workspace_bytes < make_bwd_plan(T, d, ffn, E, k, dtype, true).total) return MOE_ERR_WORKSPACE;
    DeviceState dev;
    const DeviceScope scope(h, false);
    if (!device_state(scope.device(), &dev)) return MOE_ERR_CUDA;
    return run_backward(h, Wg, W1, W3, W2, dout, dh, dWg, dW1, dW3, dW2, dlogits, alpha, wgrad_dtype, T, d, ffn, E,
                        k, dtype, static_cast<const uint8_t*>(fwd_workspace), static_cast<uint8_t*>(workspace), dev,
                        stream, stage_events, launches, gamma, dgamma);
}

moe_status moe_route_stats(const void* x, const void* Wg, int T, int d, int E, int k, float alpha,
                           int32_t* topk_idx, float* topk_w, float* stats, cudaStream_t stream) {
    return route_stats(x, Wg, T, d, E, k, alpha, topk_idx, topk_w, stats, MOE_DTYPE_BF16, stream);
}

moe_status moe_route_stats_f32(const float* x, const float* Wg, int T, int d, int E, int k, float alpha,
                               int32_t* topk_idx, float* topk_w, float* stats, cudaStream_t stream) {
    return route_stats(x, Wg, T, d, E, k, alpha, topk_idx, topk_w, stats, MOE_DTYPE_F32, stream);
}

}  // extern "C"
