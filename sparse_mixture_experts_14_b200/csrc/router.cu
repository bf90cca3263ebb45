// Router: scores s = Wg x, top-k with lowest-index tie-break, softmax over the
// selected k -- subsection "Top-2ゲーティングの定式化" of the
// "Mistral/Mixtral architecture" page (score, Top-2 and gate equations) and its
// MoERouter.forward in "簡易MoEルーターの実装", fused into one pass over x.
//
// One warp owns TPW tokens.  Lanes stride over 16-byte chunks of the rows;
// each Wg chunk loaded once is applied to all TPW tokens.  Partial sums are
// reduced with a fixed xor-butterfly, so every lane ends with the same,
// run-to-run identical fp32 scores.  Scores are never rounded to bf16.
// The pass is bound by reading x once from HBM.
#include "moe_common.cuh"

namespace moe {
namespace {

template <typename In>
struct Chunk;

template <>
struct Chunk<__nv_bfloat16> {
    static constexpr int N = 8;
    __device__ __forceinline__ static void load(const __nv_bfloat16* p, float (&v)[8]) {
        uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
        v[0] = bf16_lo(u.x); v[1] = bf16_hi(u.x);
        v[2] = bf16_lo(u.y); v[3] = bf16_hi(u.y);
        v[4] = bf16_lo(u.z); v[5] = bf16_hi(u.z);
        v[6] = bf16_lo(u.w); v[7] = bf16_hi(u.w);
    }
};

template <>
struct Chunk<float> {
    static constexpr int N = 4;
    __device__ __forceinline__ static void load(const float* p, float (&v)[4]) {
        float4 u = __ldg(reinterpret_cast<const float4*>(p));
        v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w;
    }
};

// Top-k of s[0..E) (descending; equal scores -> lower index first) and the
// softmax of the selected scores, written to idx[0..k) / w[0..k).
template <int EB>
__device__ __forceinline__ void select_and_gate(const float (&s)[EB], int E, int k, int32_t* idx, float* w) {
    uint32_t chosen = 0;
    float sel[EB];
    for (int j = 0; j < k; ++j) {
        int best = -1;
        float bv = 0.f;
#pragma unroll
        for (int e = 0; e < EB; ++e) {
            if (e < E && !((chosen >> e) & 1u)) {
                if (best < 0 || s[e] > bv) {
                    best = e;
                    bv = s[e];
                }
            }
        }
        chosen |= 1u << best;
        idx[j] = best;
        sel[j] = bv;
    }
    float denom = 0.f;
    for (int j = 0; j < k; ++j) denom += expf(sel[j] - sel[0]);
    for (int j = 0; j < k; ++j) w[j] = expf(sel[j] - sel[0]) / denom;
}

template <typename In, int EB, int TPW>
__global__ void __launch_bounds__(256) router_kernel(const In* __restrict__ x, const In* __restrict__ Wg, int T,
                                                     int d, int E, int k, int32_t* __restrict__ idx,
                                                     float* __restrict__ w) {
    constexpr int CN = Chunk<In>::N;
    const int lane = threadIdx.x & 31;
    const int warps_per_block = blockDim.x >> 5;
    const int gwarp = blockIdx.x * warps_per_block + (threadIdx.x >> 5);
    const int nwarps = gridDim.x * warps_per_block;
    const int nchunks = d / CN;

    for (int t0 = gwarp * TPW; t0 < T; t0 += nwarps * TPW) {
        float acc[TPW][EB];
#pragma unroll
        for (int t = 0; t < TPW; ++t)
#pragma unroll
            for (int e = 0; e < EB; ++e) acc[t][e] = 0.f;

        for (int c = lane; c < nchunks; c += 32) {
            float xv[TPW][CN];
#pragma unroll
            for (int t = 0; t < TPW; ++t) {
                if (t0 + t < T) {
                    Chunk<In>::load(x + (size_t)(t0 + t) * d + (size_t)c * CN, xv[t]);
                } else {
#pragma unroll
                    for (int i = 0; i < CN; ++i) xv[t][i] = 0.f;
                }
            }
#pragma unroll
            for (int e = 0; e < EB; ++e) {
                if (e < E) {
                    float wv[CN];
                    Chunk<In>::load(Wg + (size_t)e * d + (size_t)c * CN, wv);
#pragma unroll
                    for (int t = 0; t < TPW; ++t)
#pragma unroll
                        for (int i = 0; i < CN; ++i) acc[t][e] = fmaf(xv[t][i], wv[i], acc[t][e]);
                }
            }
        }
#pragma unroll
        for (int t = 0; t < TPW; ++t)
#pragma unroll
            for (int e = 0; e < EB; ++e)
#pragma unroll
                for (int m = 16; m >= 1; m >>= 1) acc[t][e] += __shfl_xor_sync(0xffffffffu, acc[t][e], m);

#pragma unroll
        for (int t = 0; t < TPW; ++t) {
            if (lane == t && t0 + t < T) {
                select_and_gate<EB>(acc[t], E, k, idx + (size_t)(t0 + t) * k, w + (size_t)(t0 + t) * k);
            }
        }
    }
}

template <typename In, int EB, int TPW>
cudaError_t launch_router_t(const In* x, const In* Wg, int T, int d, int E, int k, int32_t* idx, float* w,
                            int num_sms, cudaStream_t s) {
    const int warps = (T + TPW - 1) / TPW;
    int blocks = (warps + 7) / 8;
    const int cap = num_sms * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    router_kernel<In, EB, TPW><<<blocks, 256, 0, s>>>(x, Wg, T, d, E, k, idx, w);
    return cudaGetLastError();
}

template <typename In>
cudaError_t launch_router_any(const In* x, const In* Wg, int T, int d, int E, int k, int32_t* idx, float* w,
                              int num_sms, cudaStream_t s) {
    if (E <= 8) return launch_router_t<In, 8, 4>(x, Wg, T, d, E, k, idx, w, num_sms, s);
    if (E <= 16) return launch_router_t<In, 16, 2>(x, Wg, T, d, E, k, idx, w, num_sms, s);
    return launch_router_t<In, 32, 1>(x, Wg, T, d, E, k, idx, w, num_sms, s);
}

}  // namespace

cudaError_t launch_router_bf16(const void* x, const void* Wg, int T, int d, int E, int k, int32_t* idx, float* w,
                               int num_sms, cudaStream_t s) {
    return launch_router_any<__nv_bfloat16>(static_cast<const __nv_bfloat16*>(x),
                                            static_cast<const __nv_bfloat16*>(Wg), T, d, E, k, idx, w, num_sms,
                                            s);
}

cudaError_t launch_router_f32(const float* x, const float* Wg, int T, int d, int E, int k, int32_t* idx, float* w,
                              int num_sms, cudaStream_t s) {
    return launch_router_any<float>(x, Wg, T, d, E, k, idx, w, num_sms, s);
}

}  // namespace moe
