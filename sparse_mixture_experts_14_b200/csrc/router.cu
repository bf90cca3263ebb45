// Router: scores s = Wg x, top-k with lowest-index tie-break, softmax over the
// selected k -- subsection "Top-2ゲーティングの定式化" of the
// "Mistral/Mixtral architecture" page (score, Top-2 and gate equations) and its
// MoERouter.forward in "簡易MoEルーターの実装", fused into one pass over x.
//
// Large batches: one warp owns TPW tokens and each Wg chunk it loads serves
// all of them.  Small batches: one block per token, its warps split the row.
// Partial sums are reduced in a fixed order (xor-butterfly, then warp order),
// so the fp32 scores are identical run to run for a given batch size; they
// are never rounded to bf16.  The pass is bound by reading x once from HBM.
#include "moe_common.cuh"

namespace moe {
namespace {

template <typename In>
struct Chunk;

template <>
struct Chunk<__nv_bfloat16> {
    static constexpr int N = 8;
    using Raw = uint4;
    __device__ __forceinline__ static Raw load(const __nv_bfloat16* p) {
        return __ldg(reinterpret_cast<const uint4*>(p));
    }
    __device__ __forceinline__ static Raw zero() { return make_uint4(0, 0, 0, 0); }
    __device__ __forceinline__ static void widen(const Raw& u, float (&v)[8]) {
        v[0] = bf16_lo(u.x); v[1] = bf16_hi(u.x);
        v[2] = bf16_lo(u.y); v[3] = bf16_hi(u.y);
        v[4] = bf16_lo(u.z); v[5] = bf16_hi(u.z);
        v[6] = bf16_lo(u.w); v[7] = bf16_hi(u.w);
    }
};

template <>
struct Chunk<float> {
    static constexpr int N = 4;
    using Raw = float4;
    __device__ __forceinline__ static Raw load(const float* p) { return __ldg(reinterpret_cast<const float4*>(p)); }
    __device__ __forceinline__ static Raw zero() { return make_float4(0.f, 0.f, 0.f, 0.f); }
    __device__ __forceinline__ static void widen(const Raw& u, float (&v)[4]) {
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

// acc[t][e] += x_t[chunk] . Wg_e[chunk] for one 16-byte chunk; rows of Wg
// past E alias row E-1 (their sums are never read), so every load is
// unconditional and issues before the arithmetic.
template <typename In, int EB, int TPW>
__device__ __forceinline__ void chunk_dot(const typename Chunk<In>::Raw (&xr)[TPW], const In* __restrict__ Wg, int d,
                                          int E, int c, float (&acc)[TPW][EB]) {
    constexpr int CN = Chunk<In>::N;
    typename Chunk<In>::Raw wr[EB];
#pragma unroll
    for (int e = 0; e < EB; ++e) wr[e] = Chunk<In>::load(Wg + (size_t)(e < E ? e : E - 1) * d + (size_t)c * CN);
    float xv[TPW][CN];
#pragma unroll
    for (int t = 0; t < TPW; ++t) Chunk<In>::widen(xr[t], xv[t]);
#pragma unroll
    for (int e = 0; e < EB; ++e) {
        float wv[CN];
        Chunk<In>::widen(wr[e], wv);
#pragma unroll
        for (int t = 0; t < TPW; ++t)
#pragma unroll
            for (int i = 0; i < CN; ++i) acc[t][e] = fmaf(xv[t][i], wv[i], acc[t][e]);
    }
}

// Large T: one warp owns TPW tokens, lanes stride over the chunks of the rows
// (the next x chunks are fetched while the current ones are used); a fixed
// xor-butterfly reduces the lanes' partial sums.
template <typename In, int EB, int TPW>
__global__ void __launch_bounds__(256) router_warp_kernel(const In* __restrict__ x, const In* __restrict__ Wg, int T,
                                                          int d, int E, int k, int32_t* __restrict__ idx,
                                                          float* __restrict__ w) {
    using Raw = typename Chunk<In>::Raw;
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
        Raw xn[TPW];
#pragma unroll
        for (int t = 0; t < TPW; ++t)
            xn[t] = (lane < nchunks && t0 + t < T) ? Chunk<In>::load(x + (size_t)(t0 + t) * d + (size_t)lane * CN)
                                                   : Chunk<In>::zero();
        for (int c = lane; c < nchunks; c += 32) {
            Raw xc[TPW];
#pragma unroll
            for (int t = 0; t < TPW; ++t) xc[t] = xn[t];
            const int cn = c + 32;
#pragma unroll
            for (int t = 0; t < TPW; ++t)
                if (cn < nchunks && t0 + t < T) xn[t] = Chunk<In>::load(x + (size_t)(t0 + t) * d + (size_t)cn * CN);
            chunk_dot<In, EB, TPW>(xc, Wg, d, E, c, acc);
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

// Small T: one block per token, its 8 warps split the row; warp sums meet in
// shared memory and are added in warp order.
template <typename In, int EB>
__global__ void __launch_bounds__(256) router_split_kernel(const In* __restrict__ x, const In* __restrict__ Wg, int T,
                                                           int d, int E, int k, int32_t* __restrict__ idx,
                                                           float* __restrict__ w) {
    using Raw = typename Chunk<In>::Raw;
    constexpr int CN = Chunk<In>::N;
    __shared__ float part[8][EB];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nchunks = d / CN;
    for (int t = blockIdx.x; t < T; t += gridDim.x) {
        float acc[1][EB];
#pragma unroll
        for (int e = 0; e < EB; ++e) acc[0][e] = 0.f;
        for (int c = threadIdx.x; c < nchunks; c += 256) {
            Raw xr[1] = {Chunk<In>::load(x + (size_t)t * d + (size_t)c * CN)};
            chunk_dot<In, EB, 1>(xr, Wg, d, E, c, acc);
        }
#pragma unroll
        for (int e = 0; e < EB; ++e)
#pragma unroll
            for (int m = 16; m >= 1; m >>= 1) acc[0][e] += __shfl_xor_sync(0xffffffffu, acc[0][e], m);
        if (lane == 0) {
#pragma unroll
            for (int e = 0; e < EB; ++e) part[warp][e] = acc[0][e];
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            float s[EB];
#pragma unroll
            for (int e = 0; e < EB; ++e) {
                float v = 0.f;
#pragma unroll
                for (int q = 0; q < 8; ++q) v += part[q][e];
                s[e] = v;
            }
            select_and_gate<EB>(s, E, k, idx + (size_t)t * k, w + (size_t)t * k);
        }
        __syncthreads();
    }
}

// Tokens at or below which one block handles one token.
constexpr int kSplitMaxTokens = 512;

template <typename In, int EB, int TPW>
cudaError_t launch_router_t(const In* x, const In* Wg, int T, int d, int E, int k, int32_t* idx, float* w,
                            int num_sms, cudaStream_t s) {
    if (T <= kSplitMaxTokens) {
        router_split_kernel<In, EB><<<T, 256, 0, s>>>(x, Wg, T, d, E, k, idx, w);
        return cudaGetLastError();
    }
    const int warps = (T + TPW - 1) / TPW;
    int blocks = (warps + 7) / 8;
    const int cap = num_sms * 16;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    router_warp_kernel<In, EB, TPW><<<blocks, 256, 0, s>>>(x, Wg, T, d, E, k, idx, w);
    return cudaGetLastError();
}

template <typename In>
cudaError_t launch_router_any(const In* x, const In* Wg, int T, int d, int E, int k, int32_t* idx, float* w,
                              int num_sms, cudaStream_t s) {
    if (E <= 8) return launch_router_t<In, 8, 2>(x, Wg, T, d, E, k, idx, w, num_sms, s);
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
