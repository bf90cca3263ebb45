// Load-balance statistics of one batch's routing: subsection "ロードバランス損失"
// of the "Mistral/Mixtral architecture" page (f, p and loss equations).
//     f_e = (1/T) #{(t, j) : idx[t][j] == e}         (all k selections count)
//     p_e = (1/T) sum_t softmax(s_t)_e               (softmax over all E scores)
//     L   = alpha * E * sum_e f_e p_e
// The scores s are the router pass's fp32 scores (scaled by the row's norm
// factor in the block form).  Two launches, no atomics on floats: partial
// sums per 256-token block in a fixed order (xor-butterfly in each warp, then
// warp order), then one block adds the partials in block order, so the
// result is the same on every run.  Selection counts are integers (shared
// memory atomics on ints are exact in any order).
#include "moe_common.cuh"

namespace moe {
namespace {

constexpr int kBalanceTokens = 256;

// part layout: psum [NB][E] floats, then counts [NB][E] ints
__global__ void __launch_bounds__(kBalanceTokens) balance_part_kernel(const float* __restrict__ logits,
                                                                       const int32_t* __restrict__ idx, int T, int E,
                                                                       int k, float* __restrict__ psum,
                                                                       int32_t* __restrict__ pcnt) {
    pdl_trigger();
    pdl_wait();
    __shared__ float warp_sum[kBalanceTokens / 32][kMaxExperts];
    __shared__ int cnt[kMaxExperts];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (threadIdx.x < kMaxExperts) cnt[threadIdx.x] = 0;
    __syncthreads();
    const int t = blockIdx.x * kBalanceTokens + threadIdx.x;
    const bool live = t < T;
    const float* s = logits + (size_t)(live ? t : 0) * E;
    float mx = -INFINITY, den = 0.f;
    if (live) {
        for (int e = 0; e < E; ++e) mx = fmaxf(mx, s[e]);
        for (int e = 0; e < E; ++e) den += expf(s[e] - mx);
        for (int j = 0; j < k; ++j) {
            const int e = idx[(size_t)t * k + j];
            if (e >= 0 && e < E) atomicAdd(&cnt[e], 1);
        }
    }
    for (int e = 0; e < E; ++e) {
        float v = live ? expf(s[e] - mx) / den : 0.f;
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) v += __shfl_xor_sync(0xffffffffu, v, m);
        if (lane == 0) warp_sum[warp][e] = v;
    }
    __syncthreads();
    if (threadIdx.x < E) {
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < kBalanceTokens / 32; ++w) v += warp_sum[w][threadIdx.x];
        psum[(size_t)blockIdx.x * E + threadIdx.x] = v;
        pcnt[(size_t)blockIdx.x * E + threadIdx.x] = cnt[threadIdx.x];
    }
}

__global__ void __launch_bounds__(32) balance_final_kernel(const float* __restrict__ psum,
                                                           const int32_t* __restrict__ pcnt, int NB, int T, int E,
                                                           float alpha, float* __restrict__ stats) {
    pdl_trigger();
    pdl_wait();
    __shared__ float fp[kMaxExperts];
    const int e = threadIdx.x;
    if (e < E) {
        float p = 0.f;
        long long c = 0;
        for (int b = 0; b < NB; ++b) {
            p += psum[(size_t)b * E + e];
            c += pcnt[(size_t)b * E + e];
        }
        const float f = (float)c / (float)T;
        p = p / (float)T;
        stats[e] = f;
        stats[E + e] = p;
        fp[e] = f * p;
    }
    __syncwarp();
    if (e == 0) {
        float acc = 0.f;
        for (int i = 0; i < E; ++i) acc += fp[i];
        stats[2 * E] = alpha * (float)E * acc;
    }
}

int balance_blocks(int T) { return (T + kBalanceTokens - 1) / kBalanceTokens; }

}  // namespace

size_t balance_part_bytes(int T, int E) {
    const size_t nb = (size_t)(T > 0 ? balance_blocks(T) : 1);
    return nb * (size_t)E * 8;
}

cudaError_t launch_balance(const float* logits, const int32_t* idx, int T, int E, int k, float alpha, void* part,
                           float* stats, cudaStream_t s) {
    if (T <= 0 || E > kMaxExperts) return cudaErrorInvalidValue;
    const int NB = balance_blocks(T);
    float* psum = static_cast<float*>(part);
    int32_t* pcnt = reinterpret_cast<int32_t*>(psum + (size_t)NB * E);
    cudaError_t e = launch_pdl(balance_part_kernel, dim3(NB), dim3(kBalanceTokens), 0, s, logits, idx, T, E, k, psum,
                               pcnt);
    if (e != cudaSuccess) return e;
    return launch_pdl(balance_final_kernel, dim3(1), dim3(32), 0, s, static_cast<const float*>(psum),
                      static_cast<const int32_t*>(pcnt), NB, T, E, alpha, stats);
}

}  // namespace moe
