// Host-side definitions shared by the MoE layer's translation units: device
// selection and per-device set-up, the launch helper, buffer sizes and the
// launcher declarations.  Device code lives in moe_device.cuh (included here),
// so edits to these host declarations leave every kernel's device code as it is.
#pragma once

#include <atomic>

#include "moe_device.cuh"

namespace moe {
inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// For the length of one library call: the device that owns p is made current,
// and the caller's current device is restored on exit.  For a pointer that is
// not device (or managed) memory, device() is -1 when strict, else the
// caller's current device.
class DeviceScope {
   public:
    DeviceScope(const void* p, bool strict) {
        if (cudaGetDevice(&prev_) != cudaSuccess) {
            cudaGetLastError();
            prev_ = -1;
        }
        cudaPointerAttributes at;
        if (p && cudaPointerGetAttributes(&at, p) == cudaSuccess &&
            (at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged)) {
            if (at.device != prev_ && cudaSetDevice(at.device) != cudaSuccess) {
                cudaGetLastError();
                return;
            }
            dev_ = at.device;
        } else {
            cudaGetLastError();
            if (!strict) dev_ = prev_;
        }
    }
    ~DeviceScope() {
        if (prev_ >= 0 && dev_ >= 0 && dev_ != prev_) cudaSetDevice(prev_);
    }
    DeviceScope(const DeviceScope&) = delete;
    DeviceScope& operator=(const DeviceScope&) = delete;
    int device() const { return dev_; }

   private:
    int prev_ = -1;
    int dev_ = -1;
};

// Set-up that CUDA keeps per device (function attributes, occupancy facts):
// run f once on each device that is current when it is needed.  Concurrent
// first calls may both run f, which must therefore be idempotent.
class PerDeviceOnce {
   public:
    template <typename F>
    cudaError_t run(F&& f) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kSlots) return f();
        if (done_[dev].load(std::memory_order_acquire)) return cudaSuccess;
        const cudaError_t e = f();
        if (e == cudaSuccess) done_[dev].store(1, std::memory_order_release);
        return e;
    }

   private:
    static constexpr int kSlots = 64;
    std::atomic<int> done_[kSlots] = {};
};

// A per-device integer computed once (e.g. an occupancy limit).
class PerDeviceInt {
   public:
    template <typename F>
    int get(F&& f) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kSlots) return f();
        int v = val_[dev].load(std::memory_order_acquire);
        if (v < 0) {
            v = f();
            val_[dev].store(v, std::memory_order_release);
        }
        return v;
    }
    PerDeviceInt() {
        for (auto& x : val_) x.store(-1);
    }

   private:
    static constexpr int kSlots = 64;
    std::atomic<int> val_[kSlots];
};

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
    return e != cudaSuccess ? e : cudaGetLastError();
}

// Rows of the padded expert-contiguous buffers.
inline size_t slots_capacity(int T, int E, int k) {
    return align_up((size_t)T * k + (size_t)E * (kSegRows - 1), kSegRows);
}

inline int dispatch_blocks(int T) { return (T + kDispatchTokens - 1) / kDispatchTokens; }

// ---- kernel launchers (one per translation unit) ----
// Extra work of the router pass, all optional.  With gamma set, the pass
// routes RMSNorm(x) = gamma * x / sqrt(mean(x^2) + eps) instead of x and
// writes each row's 1/sqrt(mean(x^2) + eps) to rstd[T].  With logits set it
// also writes every fp32 score, [T][E], for the load-balance statistics.
struct RouteExtras {
    const void* gamma = nullptr;   // [d], same element type as x
    float eps = 0.f;
    float* rstd = nullptr;
    float* logits = nullptr;
    int* status = nullptr;                 // device status word (bounded pipeline waits record here)
    long long wait_ns = 1000000000LL;      // limit of one pipeline wait
};

cudaError_t launch_router_bf16(const void* x, const void* Wg, int T, int d, int E, int k, int32_t* idx,
                               float* w, int num_sms, cudaStream_t s, const RouteExtras& ex = RouteExtras());
cudaError_t launch_router_f32(const float* x, const float* Wg, int T, int d, int E, int k, int32_t* idx,
                              float* w, int num_sms, cudaStream_t s, const RouteExtras& ex = RouteExtras());

// Load-balance statistics from the router's scores and selections:
// stats[0..E) = f, stats[E..2E) = p, stats[2E] = alpha * E * sum f p.
// part holds balance_part_bytes(T, E) bytes of scratch.  Launches 2 kernels.
size_t balance_part_bytes(int T, int E);
cudaError_t launch_balance(const float* logits, const int32_t* idx, int T, int E, int k, float alpha, void* part,
                           float* stats, cudaStream_t s);

// Launches 1 kernel when T <= kDispatchTokens, else 3.
inline int dispatch_launches(int T) { return T <= kDispatchTokens ? 1 : 3; }
cudaError_t launch_dispatch(const int32_t* idx, int T, int E, int k, int32_t* blk_counts, Meta* meta,
                            int32_t* perm, int32_t* inv, int* status, cudaStream_t s);
// T <= 64: dispatch and gather fused in one launch (same results as the two separately).
// Row normalisation applied while gathering: row t becomes
// gamma * x_t * rstd[t], rounded to the row type.  gamma == nullptr copies rows unchanged.
struct GatherNorm {
    const void* gamma = nullptr;
    const float* rstd = nullptr;
};

cudaError_t launch_dispatch_gather_small(const int32_t* idx, int T, int E, int k, const void* x, size_t elem_bytes,
                                         int d, Meta* meta, int32_t* perm, int32_t* inv, void* xp, size_t slots,
                                         int* status, cudaStream_t s, const GatherNorm& nm = GatherNorm());
cudaError_t launch_gather(const void* x, size_t elem_bytes, int T, int d, int E, int k, const Meta* meta,
                          const int32_t* perm, void* xp, size_t slots, int* status, cudaStream_t s,
                          const GatherNorm& nm = GatherNorm());

// resid (nullable, [T][d] in the output type) is added after the gate-weighted sum.
cudaError_t launch_combine_bf16(const float* Y, const float* w, const int32_t* inv, int T, int d, int k,
                                size_t slots, int* status, void* out, cudaStream_t s, const void* resid = nullptr);
cudaError_t launch_combine_f32(const float* Y, const float* w, const int32_t* inv, int T, int d, int k,
                               size_t slots, int* status, float* out, cudaStream_t s, const float* resid = nullptr);

cudaError_t launch_simt_gemm1_f32(const float* xp, const float* W1, const float* W3, const Meta* meta, int E,
                                  int d, int F, float* H, size_t slots, cudaStream_t s);
cudaError_t launch_simt_gemm2_f32(const float* H, const float* W2, const Meta* meta, int E, int d, int F,
                                  float* Y, size_t slots, cudaStream_t s);

struct TcGemmArgs {
    const void* xp;     // [slots][d] bf16, expert-contiguous
    const void* W1;
    const void* W3;
    const void* W2;
    void* H;            // [slots][F] bf16
    float* Y;           // [slots][d] fp32
    const Meta* meta;
    int E, d, F;
    size_t slots;
    int num_sms;
    int* status;
    long long wait_ns;
};
cudaError_t launch_tc_gemm1(const TcGemmArgs& a, cudaStream_t s);
// GEMM1 of the training forward: also keeps a = Xp W1^T and b = Xp W3^T, fp32 [slots][F] each.
cudaError_t launch_tc_gemm1_train(const TcGemmArgs& a, float* keep_a, float* keep_b, cudaStream_t s);
cudaError_t launch_tc_gemm2(const TcGemmArgs& a, cudaStream_t s);

// Backward GEMMs on the same CTA-pair kernel (bf16 operands, fp32 accumulate).
struct TcBwdArgs {
    const void* xp;     // forward: [slots][d] bf16 gathered rows (padding rows zero)
    const void* W1;     // [E][F][d]
    const void* W3;
    const void* W2;     // [E][d][F]
    const void* H;      // forward: [slots][F] bf16
    const float* keep_a;  // forward (training path): a, b [slots][F] fp32
    const float* keep_b;
    const void* dy;     // [slots][d] bf16: g * dout scattered to the slots (padding rows zero)
    void* dab;          // [slots][2F] bf16: dA | dB
    float* dxp;         // [slots][d] fp32
    void* dW1;          // [E][F][d] fp32, or bf16 when wgrad_bf16
    void* dW3;
    void* dW2;          // [E][d][F] fp32, or bf16 when wgrad_bf16
    bool wgrad_bf16;    // weight gradients rounded once to bf16 in the epilogue
    Meta* meta;
    int E, d, F;
    size_t slots;
    int num_sms;
    int* status;
    long long wait_ns;
};
// Operands and buffers of one backward call (backward.cu); pointers are device
// memory, the *_f32 path uses float where bf16 is noted.
struct BwdArgs {
    bool bf16;
    const void* x;          // [T][d]
    const void* Wg;         // [E][d]
    const void* W1;
    const void* W3;
    const void* W2;
    const void* dout;       // [T][d]
    // forward state
    const int32_t* idx;     // [T][k]
    const float* w;         // [T][k] gates
    Meta* meta;
    const int32_t* perm;    // [slots]
    const int32_t* inv;     // [T][k]
    const void* xp;         // [slots][d]
    const void* H;          // [slots][F]
    const float* Y;         // [slots][d]
    const float* keep_a;    // [slots][F] fp32 (bf16 training path), else null
    const float* keep_b;
    const float* logits;    // [T][E] fp32 router scores kept by the training forward
    float alpha;            // load-balance loss coefficient (0: output-path gradient only)
    // backward buffers
    void* dy;               // [slots][d]
    float* dg;              // [T][k]
    float* ds;              // [T][E]
    float* dh;              // [slots][F]
    void* dab;              // [slots][2F]
    float* dxp;             // [slots][d]
    float* dwg_part;        // dwg_part_bytes(T, E, d)
    // outputs
    void* dx;               // [T][d]
    float* dWg;             // [E][d]
    float* dW1;             // [E][F][d]
    float* dW3;
    float* dW2;             // [E][d][F]
    int T, d, F, E, k;
    size_t slots;
    int* status;            // device status word (debug builds record index faults in it)
    // block form (out = h + MoE(RMSNorm(h))): x is h, dx receives dh; null gamma = the plain layer
    const void* gamma;      // [d]
    const float* rstd;      // [T] the forward's row factors r
    float* dgamma;          // [d] fp32
    float* dgamma_part;     // block_dgamma_part_bytes(T, d)
};
size_t dwg_part_bytes(int T, int E, int d);
size_t block_dgamma_part_bytes(int T, int d);
cudaError_t launch_bwd_scatter(const BwdArgs& a, cudaStream_t s);      // dY and dg (1 launch)
cudaError_t launch_router_bwd(const BwdArgs& a, cudaStream_t s);       // ds (1 launch)
cudaError_t launch_dwg(const BwdArgs& a, cudaStream_t s);              // dWg (2 launches)
cudaError_t launch_dx_combine(const BwdArgs& a, cudaStream_t s);       // dx (1 launch; block form: dh, dgamma: 2)
cudaError_t launch_simt_bwd_gemms(const BwdArgs& a, cudaStream_t s);   // fp32 expert GEMMs (5 launches)

cudaError_t launch_tc_dgrad_h(const TcBwdArgs& a, cudaStream_t s);      // dH = dY W2_e -> dA, dB
cudaError_t launch_tc_dgrad_x(const TcBwdArgs& a, cudaStream_t s);      // dXp = dA W1_e + dB W3_e
cudaError_t launch_tc_wgrad2(const TcBwdArgs& a, cudaStream_t s);       // dW2_e = dY_e^T H_e
cudaError_t launch_tc_wgrad13(const TcBwdArgs& a, cudaStream_t s);      // [dW1_e; dW3_e] = [dA dB]_e^T Xp_e
// Decode path: stage 1 (W1/W3 -> H) or stage 2 (W2 -> Y); at most 64 tokens per expert.
constexpr int kDecodeMaxTokens = 64;
cudaError_t launch_decode(const TcGemmArgs& a, int stage, cudaStream_t s);

cudaError_t launch_wait_selftest(int* status, long long limit_ns, cudaStream_t s);

}  // namespace moe
