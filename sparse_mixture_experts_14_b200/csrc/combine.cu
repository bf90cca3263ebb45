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

template <bool BF16_OUT, bool RESID>
__global__ void __launch_bounds__(256) combine_kernel(const float* __restrict__ Y, const float* __restrict__ w,
                                                      const int32_t* __restrict__ inv, int T, int d, int k,
                                                      size_t slots, int* status, void* __restrict__ out,
                                                      const void* __restrict__ resid) {
    pdl_trigger();
    pdl_wait();
    const int q = d / 4;   // float4 columns per row
    const size_t n = (size_t)T * q;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        const int t = (int)(i / q);
        const int c = (int)(i - (size_t)t * q);
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int j = 0; j < k; ++j) {
            const int slot = __ldg(inv + (size_t)t * k + j);
            if (slot < 0 || !debug_check((size_t)slot < slots, status)) continue;
            const float g = __ldg(w + (size_t)t * k + j);
            const float4 y = __ldg(reinterpret_cast<const float4*>(Y + (size_t)slot * d) + c);
            acc.x = fmaf(g, y.x, acc.x);
            acc.y = fmaf(g, y.y, acc.y);
            acc.z = fmaf(g, y.z, acc.z);
            acc.w = fmaf(g, y.w, acc.w);
        }
        if (RESID) {
            if (BF16_OUT) {
                const uint2 h = __ldg(reinterpret_cast<const uint2*>(static_cast<const uint8_t*>(resid) +
                                                                     (size_t)t * d * 2) + c);
                acc.x += bf16_lo(h.x);
                acc.y += bf16_hi(h.x);
                acc.z += bf16_lo(h.y);
                acc.w += bf16_hi(h.y);
            } else {
                const float4 h = __ldg(reinterpret_cast<const float4*>(static_cast<const float*>(resid) +
                                                                       (size_t)t * d) + c);
                acc.x += h.x;
                acc.y += h.y;
                acc.z += h.z;
                acc.w += h.w;
            }
        }
        if (BF16_OUT) {
            uint2 o;
            o.x = pack_bf16x2(acc.x, acc.y);
            o.y = pack_bf16x2(acc.z, acc.w);
            reinterpret_cast<uint2*>(static_cast<uint8_t*>(out) + (size_t)t * d * 2)[c] = o;
        } else {
            reinterpret_cast<float4*>(static_cast<float*>(out) + (size_t)t * d)[c] = acc;
        }
    }
}

template <bool BF16_OUT>
cudaError_t launch_combine_t(const float* Y, const float* w, const int32_t* inv, int T, int d, int k, size_t slots,
                             int* status, void* out, cudaStream_t s, const void* resid) {
    const size_t n = (size_t)T * (d / 4);
    size_t blocks = (n + 255) / 256;
    if (blocks > 148 * 32) blocks = 148 * 32;
    if (blocks < 1) blocks = 1;
    auto kern = resid ? combine_kernel<BF16_OUT, true> : combine_kernel<BF16_OUT, false>;
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
