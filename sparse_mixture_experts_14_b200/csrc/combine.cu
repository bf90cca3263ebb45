// Combine: out[t] = sum_{j=0}^{k-1} g[t][j] * Y[inv[t][j]], j ascending, in fp32,
// rounded once to the output type.  This is the output equation of
// subsection "Top-2ゲーティングの定式化" ("Mistral/Mixtral architecture" page),
// in the page code's order (slot 0 first, then slot 1, ...).  No atomics:
// each output element is owned by one thread, so the result is the same on
// every run.  Bound by HBM (k fp32 rows in, one row out per token).
//
// Block form: the residual row of the MoE sub-layer (section "Mixtral 8x7B —
// Sparse MoEの導入", subsection "Mixtralのアーキテクチャ") is added to the fp32
// sum before the single rounding: out[t] = h[t] + sum_j g[t][j] * Y[...].
#include "moe_common.cuh"

namespace moe {
namespace {

// Work unit: one warp, one token, 32 x U float4 columns of its row (U per
// lane, all of a slot's loads issued before its FMAs, so every lane keeps U
// 16-byte loads of Y in flight).  The units (T x ceil(d / (128 U))) are spread
// over a grid of a few blocks per SM, so the work stays balanced when T is
// not a multiple of the warp count.  Each element is still summed by one
// thread, slot 0 first: the arithmetic is the plain per-element loop's.
constexpr int kCombineU = 8;

template <bool BF16_OUT, bool RESID>
__global__ void __launch_bounds__(256) combine_kernel(const float* __restrict__ Y, const float* __restrict__ w,
                                                      const int32_t* __restrict__ inv, int T, int d, int k,
                                                      size_t slots, int* status, void* __restrict__ out,
                                                      const void* __restrict__ resid) {
    pdl_trigger();
    pdl_wait();
    constexpr int U = kCombineU;
    const int lane = threadIdx.x & 31;
    const int q = d / 4;   // float4 columns per row
    const int chunks = (q + 32 * U - 1) / (32 * U);
    const size_t units = (size_t)T * chunks;
    const size_t nwarps = (size_t)gridDim.x * (blockDim.x >> 5);
    const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
    for (size_t u = (size_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); u < units; u += nwarps) {
        const int t = (int)(u / chunks);
        const int c0 = (int)(u - (size_t)t * chunks) * 32 * U + lane;
        int my_slot = -1;
        float my_g = 0.f;
        if (lane < k) {
            my_slot = __ldg(inv + (size_t)t * k + lane);
            my_g = __ldg(w + (size_t)t * k + lane);
        }
        float4 acc[U];
#pragma unroll
        for (int i = 0; i < U; ++i) acc[i] = zero;
        for (int j = 0; j < k; ++j) {
            const int slot = __shfl_sync(0xffffffffu, my_slot, j);
            const float g = __shfl_sync(0xffffffffu, my_g, j);
            if (slot < 0 || !debug_check((size_t)slot < slots, status)) continue;
            const float4* yr = reinterpret_cast<const float4*>(Y + (size_t)slot * d);
            float4 y[U];
#pragma unroll
            for (int i = 0; i < U; ++i) {
                const int c = c0 + 32 * i;
                y[i] = c < q ? __ldcs(yr + c) : zero;
            }
#pragma unroll
            for (int i = 0; i < U; ++i) {
                acc[i].x = fmaf(g, y[i].x, acc[i].x);
                acc[i].y = fmaf(g, y[i].y, acc[i].y);
                acc[i].z = fmaf(g, y[i].z, acc[i].z);
                acc[i].w = fmaf(g, y[i].w, acc[i].w);
            }
        }
#pragma unroll
        for (int i = 0; i < U; ++i) {
            const int c = c0 + 32 * i;
            if (c >= q) break;
            float4 a = acc[i];
            if (RESID) {
                if (BF16_OUT) {
                    const uint2 h = __ldg(reinterpret_cast<const uint2*>(static_cast<const uint8_t*>(resid) +
                                                                         (size_t)t * d * 2) + c);
                    a.x += bf16_lo(h.x);
                    a.y += bf16_hi(h.x);
                    a.z += bf16_lo(h.y);
                    a.w += bf16_hi(h.y);
                } else {
                    const float4 h = __ldg(reinterpret_cast<const float4*>(static_cast<const float*>(resid) +
                                                                           (size_t)t * d) + c);
                    a.x += h.x;
                    a.y += h.y;
                    a.z += h.z;
                    a.w += h.w;
                }
            }
            if (BF16_OUT) {
                uint2 o;
                o.x = pack_bf16x2(a.x, a.y);
                o.y = pack_bf16x2(a.z, a.w);
                reinterpret_cast<uint2*>(static_cast<uint8_t*>(out) + (size_t)t * d * 2)[c] = o;
            } else {
                reinterpret_cast<float4*>(static_cast<float*>(out) + (size_t)t * d)[c] = a;
            }
        }
    }
}

template <bool BF16_OUT>
cudaError_t launch_combine_t(const float* Y, const float* w, const int32_t* inv, int T, int d, int k, size_t slots,
                             int* status, void* out, cudaStream_t s, const void* resid) {
    const int q = d / 4;
    const size_t units = (size_t)T * ((q + 32 * kCombineU - 1) / (32 * kCombineU));
    auto kern = resid ? combine_kernel<BF16_OUT, true> : combine_kernel<BF16_OUT, false>;
    // one wave of resident blocks (every SM full), no more blocks than units of 8 warps
    static PerDeviceInt resident_blocks[2];   // with and without the residual
    const int resident = resident_blocks[resid ? 1 : 0].get([kern] {
        int per_sm = 0, dev = 0, sms = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 256, 0) != cudaSuccess || per_sm < 1) {
            cudaGetLastError();
            return 148 * 4;
        }
        return sms * per_sm;
    });
    size_t blocks = (units + 7) / 8;   // 8 warps per block
    if (blocks > (size_t)resident) blocks = (size_t)resident;
    if (blocks < 1) blocks = 1;
    return launch_pdl(kern, dim3((unsigned)blocks), dim3(256), 0, s, Y, w, inv, T, d, k, slots, status, out, resid);
}

}  // namespace

cudaError_t launch_combine_bf16(const float* Y, const float* w, const int32_t* inv, int T, int d, int k, size_t slots,
                                int* status, void* out, cudaStream_t s, const void* resid) {
    return launch_combine_t<true>(Y, w, inv, T, d, k, slots, status, out, s, resid);
}

cudaError_t launch_combine_f32(const float* Y, const float* w, const int32_t* inv, int T, int d, int k, size_t slots,
                               int* status, float* out, cudaStream_t s, const float* resid) {
    return launch_combine_t<false>(Y, w, inv, T, d, k, slots, status, out, s, resid);
}

}  // namespace moe
