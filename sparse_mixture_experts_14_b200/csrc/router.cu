// Router: scores s = Wg x, top-k with lowest-index tie-break, softmax over the
// selected k -- subsection "Top-2ゲーティングの定式化" of the
// "Mistral/Mixtral architecture" page (score, Top-2 and gate equations) and its
// MoERouter.forward in "簡易MoEルーターの実装", fused into one pass over x.
//
// Large bf16 batches: scores on the tensor cores (router_mma_kernel, 16
// tokens per block, warps split d).  Small batches and fp32 inputs: CUDA-core
// dot products (router_kernel, one block per token or per few tokens, every
// 16-byte chunk a thread needs in flight before the arithmetic; rows longer
// than 1024 chunks loop, router_loop_kernel).  Partial sums are reduced in a
// fixed order (xor-butterfly or MMA accumulation, then warp order), so the
// fp32 scores are identical run to run for a given batch size; they are
// never rounded to bf16.  The pass is bound by reading x once from HBM.
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

// Rows longer than 1024 chunks: one block per token, its threads loop over
// the row; warp sums meet in shared memory and are added in warp order.
template <typename In, int EB>
__global__ void __launch_bounds__(256) router_loop_kernel(const In* __restrict__ x, const In* __restrict__ Wg, int T,
                                                           int d, int E, int k, int32_t* __restrict__ idx,
                                                           float* __restrict__ w) {
    pdl_trigger();
    pdl_wait();
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

// One block (8 warps) owns TB consecutive tokens; thread i covers chunks i,
// i + 256, ... of the row (at most RMAX of them).  Every x chunk a thread
// needs is requested before any arithmetic, so a block has TB rows in flight
// at once; each Wg chunk it loads serves all TB tokens.  Lane partial sums
// are reduced by a fixed xor-butterfly, the 8 warp sums in warp order.
template <typename In, int EB, int TB, int RMAX>
__global__ void __launch_bounds__(256) router_kernel(const In* __restrict__ x, const In* __restrict__ Wg, int T, int d,
                                                     int E, int k, int32_t* __restrict__ idx,
                                                     float* __restrict__ w) {
    pdl_trigger();
    pdl_wait();
    using Raw = typename Chunk<In>::Raw;
    constexpr int CN = Chunk<In>::N;
    __shared__ float part[8][TB][EB];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nchunks = d / CN;
    for (int t0 = blockIdx.x * TB; t0 < T; t0 += gridDim.x * TB) {
        Raw xr[RMAX][TB];
#pragma unroll
        for (int r = 0; r < RMAX; ++r) {
            const int c = threadIdx.x + r * 256;
#pragma unroll
            for (int t = 0; t < TB; ++t)
                xr[r][t] = (c < nchunks && t0 + t < T) ? Chunk<In>::load(x + (size_t)(t0 + t) * d + (size_t)c * CN)
                                                       : Chunk<In>::zero();
        }
        float acc[TB][EB];
#pragma unroll
        for (int t = 0; t < TB; ++t)
#pragma unroll
            for (int e = 0; e < EB; ++e) acc[t][e] = 0.f;
#pragma unroll
        for (int r = 0; r < RMAX; ++r) {
            const int c = threadIdx.x + r * 256;
            if (c < nchunks) chunk_dot<In, EB, TB>(xr[r], Wg, d, E, c, acc);
        }
#pragma unroll
        for (int t = 0; t < TB; ++t)
#pragma unroll
            for (int e = 0; e < EB; ++e)
#pragma unroll
                for (int m = 16; m >= 1; m >>= 1) acc[t][e] += __shfl_xor_sync(0xffffffffu, acc[t][e], m);
        if (lane == 0) {
#pragma unroll
            for (int t = 0; t < TB; ++t)
#pragma unroll
                for (int e = 0; e < EB; ++e) part[warp][t][e] = acc[t][e];
        }
        __syncthreads();
        if (threadIdx.x < TB && t0 + (int)threadIdx.x < T) {
            const int t = threadIdx.x;
            float sc[EB];
#pragma unroll
            for (int e = 0; e < EB; ++e) {
                float v = 0.f;
#pragma unroll
                for (int q = 0; q < 8; ++q) v += part[q][t][e];
                sc[e] = v;
            }
            select_and_gate<EB>(sc, E, k, idx + (size_t)(t0 + t) * k, w + (size_t)(t0 + t) * k);
        }
        __syncthreads();
    }
}

// bf16 scores on the tensor cores (mma.sync m16n8k16, bf16 x bf16 -> fp32).
// The score matrix is the contraction x [T][d] . Wg^T [d][E]; with E <= 8 one
// n8 tile holds all experts.  A block takes 16 tokens and its 8 warps split d
// into 32-wide steps (warp w: steps w, w+8, ...).  Thread (g, q) of a warp
// loads 16 bytes of rows g and g+8 of x and of row g of Wg at k0 + 8q and
// feeds them to two MMAs: the MMA's k slots are a fixed permutation of the 32
// physical k of the step, the same for A and B, so the dot product is
// unchanged.  Each warp adds its MMA accumulator into fp32 registers every 16
// MMAs (K = 256), bounding the accumulation inside the tensor core; the 8 warp
// sums are added in warp order.  Products of bf16 values are exact in fp32.
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <int NT>
__global__ void __launch_bounds__(256) router_mma_kernel(const __nv_bfloat16* __restrict__ x,
                                                         const __nv_bfloat16* __restrict__ Wg, int T, int d, int E,
                                                         int k, int32_t* __restrict__ idx, float* __restrict__ w) {
    pdl_trigger();
    pdl_wait();
    constexpr int EB = 8 * NT;
    __shared__ float part[8][16][EB + 1];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, q = lane & 3;
    const int nsteps = d / 32;
    const uint4 zero = make_uint4(0, 0, 0, 0);
    for (int t0 = blockIdx.x * 16; t0 < T; t0 += gridDim.x * 16) {
        const int r0 = t0 + g, r1 = t0 + g + 8;
        const uint4* xr0 = reinterpret_cast<const uint4*>(x + (size_t)(r0 < T ? r0 : 0) * d);
        const uint4* xr1 = reinterpret_cast<const uint4*>(x + (size_t)(r1 < T ? r1 : 0) * d);
        float tot[NT][4], acc[NT][4];
#pragma unroll
        for (int n = 0; n < NT; ++n)
#pragma unroll
            for (int i = 0; i < 4; ++i) tot[n][i] = acc[n][i] = 0.f;
        int since_flush = 0;
#pragma unroll 4
        for (int st = warp; st < nsteps; st += 8) {
            const int c = st * 4 + q;   // 16-byte chunk index of k0 + 8q
            const uint4 xa = r0 < T ? __ldg(xr0 + c) : zero;
            const uint4 xb = r1 < T ? __ldg(xr1 + c) : zero;
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                const int e = n * 8 + g;
                const uint4 wv = e < E ? __ldg(reinterpret_cast<const uint4*>(Wg + (size_t)e * d) + c) : zero;
                mma_bf16_16816(acc[n], xa.x, xb.x, xa.y, xb.y, wv.x, wv.y);
                mma_bf16_16816(acc[n], xa.z, xb.z, xa.w, xb.w, wv.z, wv.w);
            }
            if (++since_flush == 8) {
                since_flush = 0;
#pragma unroll
                for (int n = 0; n < NT; ++n)
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        tot[n][i] += acc[n][i];
                        acc[n][i] = 0.f;
                    }
            }
        }
#pragma unroll
        for (int n = 0; n < NT; ++n) {
#pragma unroll
            for (int i = 0; i < 4; ++i) tot[n][i] += acc[n][i];
            // c0, c1: token g, experts 2q, 2q+1; c2, c3: token g + 8
            part[warp][g][n * 8 + 2 * q] = tot[n][0];
            part[warp][g][n * 8 + 2 * q + 1] = tot[n][1];
            part[warp][g + 8][n * 8 + 2 * q] = tot[n][2];
            part[warp][g + 8][n * 8 + 2 * q + 1] = tot[n][3];
        }
        __syncthreads();
        if (threadIdx.x < 16 && t0 + (int)threadIdx.x < T) {
            const int t = threadIdx.x;
            float sc[EB];
#pragma unroll
            for (int e = 0; e < EB; ++e) {
                float v = 0.f;
#pragma unroll
                for (int ww = 0; ww < 8; ++ww) v += part[ww][t][e];
                sc[e] = v;
            }
            select_and_gate<EB>(sc, E, k, idx + (size_t)(t0 + t) * k, w + (size_t)(t0 + t) * k);
        }
        __syncthreads();
    }
}

// Chunks per thread the kernels are compiled for: 16-byte chunks x 256 threads x RMAX
// cover d <= 8192 (bf16) / 4096 (fp32) with RMAX = 4; longer rows take the looping form.
template <typename In, int EB, int TB>
cudaError_t launch_router_t(const In* x, const In* Wg, int T, int d, int E, int k, int32_t* idx, float* w,
                            int num_sms, cudaStream_t s) {
    const int nchunks = d / Chunk<In>::N;
    // small batches: one token per block, so every SM gets work
    const bool small = T <= 4 * num_sms;
    const int tb = small ? 1 : TB;
    int blocks = (T + tb - 1) / tb;
    if (blocks < 1) blocks = 1;
    if (nchunks <= 256) {
        if (small) return launch_pdl(router_kernel<In, EB, 1, 1>, dim3(blocks), dim3(256), 0, s, x, Wg, T, d, E, k, idx, w);
        else return launch_pdl(router_kernel<In, EB, TB, 1>, dim3(blocks), dim3(256), 0, s, x, Wg, T, d, E, k, idx, w);
    } else if (nchunks <= 512) {
        if (small) return launch_pdl(router_kernel<In, EB, 1, 2>, dim3(blocks), dim3(256), 0, s, x, Wg, T, d, E, k, idx, w);
        else return launch_pdl(router_kernel<In, EB, TB, 2>, dim3(blocks), dim3(256), 0, s, x, Wg, T, d, E, k, idx, w);
    } else if (nchunks <= 1024) {
        if (small) return launch_pdl(router_kernel<In, EB, 1, 4>, dim3(blocks), dim3(256), 0, s, x, Wg, T, d, E, k, idx, w);
        else return launch_pdl(router_kernel<In, EB, TB, 4>, dim3(blocks), dim3(256), 0, s, x, Wg, T, d, E, k, idx, w);
    } else {
        const int g = T < 65535 ? T : 65535;
        return launch_pdl(router_loop_kernel<In, EB>, dim3(g), dim3(256), 0, s, x, Wg, T, d, E, k, idx, w);
    }
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
    // tensor-core scores for large batches; small batches spread one token per block instead
    if (d % 32 == 0 && T > 4 * num_sms) {
        const int tiles = (T + 15) / 16;
        int grid = tiles < num_sms * 16 ? tiles : num_sms * 16;
        if (grid < 1) grid = 1;
        const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
        const __nv_bfloat16* wb = static_cast<const __nv_bfloat16*>(Wg);
        if (E <= 8) return launch_pdl(router_mma_kernel<1>, dim3(grid), dim3(256), 0, s, xb, wb, T, d, E, k, idx, w);
        if (E <= 16) return launch_pdl(router_mma_kernel<2>, dim3(grid), dim3(256), 0, s, xb, wb, T, d, E, k, idx, w);
        return launch_pdl(router_mma_kernel<4>, dim3(grid), dim3(256), 0, s, xb, wb, T, d, E, k, idx, w);
    }
    return launch_router_any<__nv_bfloat16>(static_cast<const __nv_bfloat16*>(x),
                                            static_cast<const __nv_bfloat16*>(Wg), T, d, E, k, idx, w, num_sms,
                                            s);
}

cudaError_t launch_router_f32(const float* x, const float* Wg, int T, int d, int E, int k, int32_t* idx, float* w,
                              int num_sms, cudaStream_t s) {
    return launch_router_any<float>(x, Wg, T, d, E, k, idx, w, num_sms, s);
}

}  // namespace moe
