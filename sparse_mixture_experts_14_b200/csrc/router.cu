// Router: scores s = Wg x, top-k with lowest-index tie-break, softmax over the
// selected k -- subsection "Top-2ゲーティングの定式化" of the
// "Mistral/Mixtral architecture" page (score, Top-2 and gate equations) and its
// MoERouter.forward in "簡易MoEルーターの実装", fused into one pass over x.
//
// One block (8 warps) owns a few consecutive tokens (one per block for small
// batches); its threads split each row into 16-byte chunks, and every chunk a
// thread needs is in flight before the arithmetic starts.  Partial sums are
// reduced in a fixed order (xor-butterfly, then warp order), so the fp32
// scores are identical run to run for a given batch size; they are never
// rounded to bf16.  The pass is bound by reading x once from HBM.
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

// (bf16 pair) -> (f32, f32) in one 64-bit register: element 0 low, element 1 high
__device__ __forceinline__ unsigned long long bf16x2_to_f32x2(uint32_t w) {
    unsigned long long r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(w << 16), "r"(w & 0xffff0000u));
    return r;
}
// acc.lo += a.lo * b.lo, acc.hi += a.hi * b.hi (one instruction, round to nearest)
__device__ __forceinline__ void ffma2(unsigned long long& acc, unsigned long long a, unsigned long long b) {
    asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(a), "l"(b));
}
__device__ __forceinline__ float sum_f32x2(unsigned long long v) {
    uint32_t lo, hi;
    asm("mov.b64 {%0, %1}, %2;" : "=r"(lo), "=r"(hi) : "l"(v));
    return __uint_as_float(lo) + __uint_as_float(hi);
}

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                     static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst))),
                 "l"(gmem_src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

// Large batches: persistent blocks that keep Wg in shared memory and walk
// groups of TB tokens, the next group's rows streaming into the other half of
// a double buffer (cp.async) while the current group is reduced.  HBM sees x
// once and Wg once per SM.  The arithmetic is packed: each f32x2 FMA handles
// an (even k, odd k) pair, so every thread keeps two partial sums per (token,
// expert), added at the end; a reduce-scatter butterfly then leaves one
// (token, expert) sum per lane, and the 8 warp sums are added in warp order.
// The order is fixed, so the scores are identical run to run.
template <int EB, int TB>
__global__ void __launch_bounds__(256) router_smem_kernel(const __nv_bfloat16* __restrict__ x,
                                                          const __nv_bfloat16* __restrict__ Wg, int T, int d, int E,
                                                          int k, int32_t* __restrict__ idx, float* __restrict__ w) {
    pdl_trigger();
    pdl_wait();
    extern __shared__ uint4 sm[];
    using Raw = uint4;
    const int nchunks = d / 8;
    uint4* sWg = sm;                                   // [E][nchunks]
    uint4* sx = sm + (size_t)E * nchunks;              // [2][TB][nchunks]
    static_assert(TB * EB == 32, "one reduced value per lane");
    __shared__ float part_flat[8][32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int ngroups = (T + TB - 1) / TB;

    const uint4* gW = reinterpret_cast<const uint4*>(Wg);
    for (int i = threadIdx.x; i < E * nchunks; i += 256) cp_async16(sWg + i, gW + i);
    auto issue = [&](int g, int buf) {
        if (g < ngroups) {
            for (int i = threadIdx.x; i < TB * nchunks; i += 256) {
                const int t = g * TB + i / nchunks;
                const int c = i - (i / nchunks) * nchunks;
                if (t < T) cp_async16(sx + ((size_t)buf * TB * nchunks + i), reinterpret_cast<const uint4*>(x + (size_t)t * d) + c);
            }
        }
        cp_async_commit();
    };
    int buf = 0;
    issue(blockIdx.x, 0);
    for (int g = blockIdx.x; g < ngroups; g += gridDim.x) {
        issue(g + gridDim.x, buf ^ 1);
        cp_async_wait1();
        __syncthreads();
        const int t0 = g * TB;
        // acc[t][e] holds two partial sums (even and odd k) in one f32x2 register
        unsigned long long acc[TB][EB];
#pragma unroll
        for (int t = 0; t < TB; ++t)
#pragma unroll
            for (int e = 0; e < EB; ++e) acc[t][e] = 0ull;
        const uint4* xb = sx + (size_t)buf * TB * nchunks;
        for (int c = threadIdx.x; c < nchunks; c += 256) {
            unsigned long long xv[TB][4];
#pragma unroll
            for (int t = 0; t < TB; ++t) {
                const uint4 r = (t0 + t < T) ? xb[t * nchunks + c] : make_uint4(0, 0, 0, 0);
                xv[t][0] = bf16x2_to_f32x2(r.x);
                xv[t][1] = bf16x2_to_f32x2(r.y);
                xv[t][2] = bf16x2_to_f32x2(r.z);
                xv[t][3] = bf16x2_to_f32x2(r.w);
            }
#pragma unroll
            for (int e = 0; e < EB; ++e) {
                const uint4 r = sWg[(size_t)(e < E ? e : E - 1) * nchunks + c];
                const unsigned long long w0 = bf16x2_to_f32x2(r.x), w1 = bf16x2_to_f32x2(r.y);
                const unsigned long long w2 = bf16x2_to_f32x2(r.z), w3 = bf16x2_to_f32x2(r.w);
#pragma unroll
                for (int t = 0; t < TB; ++t) {
                    ffma2(acc[t][e], xv[t][0], w0);
                    ffma2(acc[t][e], xv[t][1], w1);
                    ffma2(acc[t][e], xv[t][2], w2);
                    ffma2(acc[t][e], xv[t][3], w3);
                }
            }
        }
        // even + odd partials, then a reduce-scatter butterfly: lane L ends with
        // the warp's sum of value L = t * EB + e
        float v[TB * EB];
#pragma unroll
        for (int t = 0; t < TB; ++t)
#pragma unroll
            for (int e = 0; e < EB; ++e) v[t * EB + e] = sum_f32x2(acc[t][e]);
#pragma unroll
        for (int m = 16, n = 16; m >= 1; m >>= 1, n >>= 1) {
            const bool upper = (lane & m) != 0;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                if (i < n) {
                    const float send = upper ? v[i] : v[i + n];
                    const float keep = upper ? v[i + n] : v[i];
                    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
                }
            }
        }
        part_flat[warp][lane] = v[0];
        __syncthreads();
        if (threadIdx.x < TB && t0 + (int)threadIdx.x < T) {
            const int t = threadIdx.x;
            float sc[EB];
#pragma unroll
            for (int e = 0; e < EB; ++e) {
                float acc_e = 0.f;
#pragma unroll
                for (int q = 0; q < 8; ++q) acc_e += part_flat[q][t * EB + e];
                sc[e] = acc_e;
            }
            select_and_gate<EB>(sc, E, k, idx + (size_t)(t0 + t) * k, w + (size_t)(t0 + t) * k);
        }
        buf ^= 1;
        __syncthreads();
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
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

constexpr int kSmemRouterTB = 4;
constexpr size_t kSmemRouterMax = 200 * 1024;

// Shared memory the persistent bf16 router needs, or 0 when it does not fit.
size_t router_smem_bytes(int d, int E) {
    const size_t b = ((size_t)E + 2 * kSmemRouterTB) * (size_t)d * 2;
    return b <= kSmemRouterMax ? b : 0;
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
    const size_t smem = router_smem_bytes(d, E);
    if (E <= 8 && smem > 0 && T > 4 * num_sms) {
        static PerDeviceOnce attr;
        cudaError_t e = attr.run([] {
            return cudaFuncSetAttribute(router_smem_kernel<8, kSmemRouterTB>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemRouterMax);
        });
        if (e != cudaSuccess) return e;
        const int groups = (T + kSmemRouterTB - 1) / kSmemRouterTB;
        const int per_sm = smem <= 110 * 1024 ? 2 : 1;
        int grid = num_sms * per_sm;
        if (grid > groups) grid = groups;
        return launch_pdl(router_smem_kernel<8, kSmemRouterTB>, dim3(grid), dim3(256), smem, s,
                          static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(Wg), T, d, E, k,
                          idx, w);
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
