// Router: scores s = Wg x, top-k with lowest-index tie-break, softmax over the
// selected k -- subsection "Top-2ゲーティングの定式化" of the
// "Mistral/Mixtral architecture" page (score, Top-2 and gate equations) and its
// MoERouter.forward in "簡易MoEルーターの実装", fused into one pass over x.
//
// Large bf16 batches (plain layer, E a multiple of 8): router_tc_kernel, the
// scores as a tcgen05 GEMM of 128-token tiles against Wg (N = E rounded up to
// 16), operands streamed by TMA, one tile per CTA; when there are fewer tiles
// than SMs the CTAs of a cluster split d and rank 0 adds their partial scores
// in rank order through distributed shared memory.  Block form and other E:
// router_mma_kernel (mma.sync, 16 tokens per block, warps split d).  Small batches and fp32 inputs: CUDA-core
// dot products (router_kernel, one block per token or per few tokens, every
// 16-byte chunk a thread needs in flight before the arithmetic; rows longer
// than 1024 chunks loop, router_loop_kernel).  Partial sums are reduced in a
// fixed order (xor-butterfly or MMA accumulation, then warp order), so the
// fp32 scores are identical run to run for a given batch size; they are
// never rounded to bf16.  The pass is bound by reading x once from HBM.
//
// Block form (the MoE sub-layer's pre-norm, section "Mixtral 8x7B — Sparse
// MoEの導入", subsection "Mixtralのアーキテクチャ"): the same pass routes
// u = RMSNorm(x) = gamma * x * r with r = 1/sqrt(mean(x^2) + eps).  Since r is
// one positive number per row, s = r * (Wg (gamma * x)): the pass sums the
// squares of x beside the dot products and scales the scores by r at the end.
// gamma * x is exact in fp32 for bf16 operands; on the tensor cores it enters
// as two bf16 operands, hi = bf16(gamma x) and lo = gamma x - hi, which are
// exact too, so the scores see the unrounded normalised row.
#include <cuda.h>

#include "moe_common.cuh"
#include "ptx_sm100.cuh"
#include "tma_map.cuh"

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

// Where a router pass writes its results (see RouteExtras for the optional ones).
template <typename In>
struct RouterIO {
    int32_t* idx;
    float* w;
    const In* gamma;   // non-null exactly when the kernel is instantiated with NORM
    float eps;
    float* rstd;
    float* logits;
};

// Per-token end of the pass: apply the row's norm factor, dump the scores if
// asked, select and gate.  ss = sum of x^2 over the row (NORM only).
template <typename In, int EB, bool NORM>
__device__ __forceinline__ void finish_token(float (&sc)[EB], float ss, int t, int d, int E, int k,
                                             const RouterIO<In>& io) {
    if (NORM) {
        const float r = 1.0f / sqrtf(ss / (float)d + io.eps);
#pragma unroll
        for (int e = 0; e < EB; ++e) sc[e] *= r;
        io.rstd[t] = r;
    }
    if (io.logits) {
        for (int e = 0; e < E; ++e) io.logits[(size_t)t * E + e] = sc[e];
    }
    select_and_gate<EB>(sc, E, k, io.idx + (size_t)t * k, io.w + (size_t)t * k);
}

// acc[t][e] += x_t[chunk] . Wg_e[chunk] for one 16-byte chunk; rows of Wg
// past E alias row E-1 (their sums are never read), so every load is
// unconditional and issues before the arithmetic.  NORM: x is multiplied by
// gamma first and ss[t] collects the squares of x.
template <typename In, int EB, int TPW, bool NORM>
__device__ __forceinline__ void chunk_dot(const typename Chunk<In>::Raw (&xr)[TPW], const In* __restrict__ Wg,
                                          const In* __restrict__ gamma, int d, int E, int c, float (&acc)[TPW][EB],
                                          float (&ss)[TPW]) {
    constexpr int CN = Chunk<In>::N;
    typename Chunk<In>::Raw wr[EB];
#pragma unroll
    for (int e = 0; e < EB; ++e) wr[e] = Chunk<In>::load(Wg + (size_t)(e < E ? e : E - 1) * d + (size_t)c * CN);
    float xv[TPW][CN];
#pragma unroll
    for (int t = 0; t < TPW; ++t) Chunk<In>::widen(xr[t], xv[t]);
    if (NORM) {
        float gv[CN];
        Chunk<In>::widen(Chunk<In>::load(gamma + (size_t)c * CN), gv);
#pragma unroll
        for (int t = 0; t < TPW; ++t)
#pragma unroll
            for (int i = 0; i < CN; ++i) {
                ss[t] = fmaf(xv[t][i], xv[t][i], ss[t]);
                xv[t][i] *= gv[i];
            }
    }
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
template <typename In, int EB, bool NORM>
__global__ void __launch_bounds__(256) router_loop_kernel(const In* __restrict__ x, const In* __restrict__ Wg, int T,
                                                           int d, int E, int k, RouterIO<In> io) {
    pdl_trigger();
    pdl_wait();
    using Raw = typename Chunk<In>::Raw;
    constexpr int CN = Chunk<In>::N;
    __shared__ float part[8][EB + 1];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nchunks = d / CN;
    for (int t = blockIdx.x; t < T; t += gridDim.x) {
        float acc[1][EB];
        float ss[1] = {0.f};
#pragma unroll
        for (int e = 0; e < EB; ++e) acc[0][e] = 0.f;
        for (int c = threadIdx.x; c < nchunks; c += 256) {
            Raw xr[1] = {Chunk<In>::load(x + (size_t)t * d + (size_t)c * CN)};
            chunk_dot<In, EB, 1, NORM>(xr, Wg, io.gamma, d, E, c, acc, ss);
        }
#pragma unroll
        for (int e = 0; e < EB; ++e)
#pragma unroll
            for (int m = 16; m >= 1; m >>= 1) acc[0][e] += __shfl_xor_sync(0xffffffffu, acc[0][e], m);
        if (NORM) {
#pragma unroll
            for (int m = 16; m >= 1; m >>= 1) ss[0] += __shfl_xor_sync(0xffffffffu, ss[0], m);
        }
        if (lane == 0) {
#pragma unroll
            for (int e = 0; e < EB; ++e) part[warp][e] = acc[0][e];
            part[warp][EB] = ss[0];
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            float s[EB];
            float sq = 0.f;
#pragma unroll
            for (int e = 0; e < EB; ++e) {
                float v = 0.f;
#pragma unroll
                for (int q = 0; q < 8; ++q) v += part[q][e];
                s[e] = v;
            }
#pragma unroll
            for (int q = 0; q < 8; ++q) sq += part[q][EB];
            finish_token<In, EB, NORM>(s, sq, t, d, E, k, io);
        }
        __syncthreads();
    }
}

// One block (8 warps) owns TB consecutive tokens; thread i covers chunks i,
// i + 256, ... of the row (at most RMAX of them).  Every x chunk a thread
// needs is requested before any arithmetic, so a block has TB rows in flight
// at once; each Wg chunk it loads serves all TB tokens.  Lane partial sums
// are reduced by a fixed xor-butterfly, the 8 warp sums in warp order.
template <typename In, int EB, int TB, int RMAX, bool NORM>
__global__ void __launch_bounds__(256) router_kernel(const In* __restrict__ x, const In* __restrict__ Wg, int T, int d,
                                                     int E, int k, RouterIO<In> io) {
    pdl_trigger();
    pdl_wait();
    using Raw = typename Chunk<In>::Raw;
    constexpr int CN = Chunk<In>::N;
    __shared__ float part[8][TB][EB + 1];
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
        float ss[TB];
#pragma unroll
        for (int t = 0; t < TB; ++t) {
            ss[t] = 0.f;
#pragma unroll
            for (int e = 0; e < EB; ++e) acc[t][e] = 0.f;
        }
#pragma unroll
        for (int r = 0; r < RMAX; ++r) {
            const int c = threadIdx.x + r * 256;
            if (c < nchunks) chunk_dot<In, EB, TB, NORM>(xr[r], Wg, io.gamma, d, E, c, acc, ss);
        }
#pragma unroll
        for (int t = 0; t < TB; ++t) {
#pragma unroll
            for (int e = 0; e < EB; ++e)
#pragma unroll
                for (int m = 16; m >= 1; m >>= 1) acc[t][e] += __shfl_xor_sync(0xffffffffu, acc[t][e], m);
            if (NORM) {
#pragma unroll
                for (int m = 16; m >= 1; m >>= 1) ss[t] += __shfl_xor_sync(0xffffffffu, ss[t], m);
            }
        }
        if (lane == 0) {
#pragma unroll
            for (int t = 0; t < TB; ++t) {
#pragma unroll
                for (int e = 0; e < EB; ++e) part[warp][t][e] = acc[t][e];
                part[warp][t][EB] = ss[t];
            }
        }
        __syncthreads();
        if (threadIdx.x < TB && t0 + (int)threadIdx.x < T) {
            const int t = threadIdx.x;
            float sc[EB];
            float sq = 0.f;
#pragma unroll
            for (int e = 0; e < EB; ++e) {
                float v = 0.f;
#pragma unroll
                for (int q = 0; q < 8; ++q) v += part[q][t][e];
                sc[e] = v;
            }
#pragma unroll
            for (int q = 0; q < 8; ++q) sq += part[q][t][EB];
            finish_token<In, EB, NORM>(sc, sq, t0 + t, d, E, k, io);
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

// gamma * x for the bf16 pair xv (x) and gv (gamma), split into bf16 parts
// hi + lo that sum to the fp32 product exactly; ss collects x^2.
__device__ __forceinline__ void scaled_pair(uint32_t xv, uint32_t gv, uint32_t& hi, uint32_t& lo, float& ss) {
    const float x0 = bf16_lo(xv), x1 = bf16_hi(xv);
    ss = fmaf(x0, x0, ss);
    ss = fmaf(x1, x1, ss);
    const float p0 = x0 * bf16_lo(gv), p1 = x1 * bf16_hi(gv);
    hi = pack_bf16x2(p0, p1);
    lo = pack_bf16x2(p0 - bf16_lo(hi), p1 - bf16_hi(hi));
}

// NORM: the A operand is gamma * x as hi + lo (four MMAs per step instead of
// two, so the accumulator is flushed every 4 steps to keep 16 MMAs per flush).
template <int NT, bool NORM>
__global__ void __launch_bounds__(256) router_mma_kernel(const __nv_bfloat16* __restrict__ x,
                                                         const __nv_bfloat16* __restrict__ Wg, int T, int d, int E,
                                                         int k, RouterIO<__nv_bfloat16> io) {
    pdl_trigger();
    pdl_wait();
    constexpr int EB = 8 * NT;
    constexpr int FLUSH = NORM ? 4 : 8;
    __shared__ float part[8][16][EB + 1];
    __shared__ float sqp[8][16];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, q = lane & 3;
    const int nsteps = d / 32;
    const uint4 zero = make_uint4(0, 0, 0, 0);
    const uint4* gam = reinterpret_cast<const uint4*>(io.gamma);
    for (int t0 = blockIdx.x * 16; t0 < T; t0 += gridDim.x * 16) {
        const int r0 = t0 + g, r1 = t0 + g + 8;
        const uint4* xr0 = reinterpret_cast<const uint4*>(x + (size_t)(r0 < T ? r0 : 0) * d);
        const uint4* xr1 = reinterpret_cast<const uint4*>(x + (size_t)(r1 < T ? r1 : 0) * d);
        float tot[NT][4], acc[NT][4];
        float ss0 = 0.f, ss1 = 0.f;
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
            if (NORM) {
                const uint4 gv = __ldg(gam + c);
                uint4 ah, al, bh, bl;
                scaled_pair(xa.x, gv.x, ah.x, al.x, ss0);
                scaled_pair(xa.y, gv.y, ah.y, al.y, ss0);
                scaled_pair(xa.z, gv.z, ah.z, al.z, ss0);
                scaled_pair(xa.w, gv.w, ah.w, al.w, ss0);
                scaled_pair(xb.x, gv.x, bh.x, bl.x, ss1);
                scaled_pair(xb.y, gv.y, bh.y, bl.y, ss1);
                scaled_pair(xb.z, gv.z, bh.z, bl.z, ss1);
                scaled_pair(xb.w, gv.w, bh.w, bl.w, ss1);
#pragma unroll
                for (int n = 0; n < NT; ++n) {
                    const int e = n * 8 + g;
                    const uint4 wv = e < E ? __ldg(reinterpret_cast<const uint4*>(Wg + (size_t)e * d) + c) : zero;
                    mma_bf16_16816(acc[n], ah.x, bh.x, ah.y, bh.y, wv.x, wv.y);
                    mma_bf16_16816(acc[n], ah.z, bh.z, ah.w, bh.w, wv.z, wv.w);
                    mma_bf16_16816(acc[n], al.x, bl.x, al.y, bl.y, wv.x, wv.y);
                    mma_bf16_16816(acc[n], al.z, bl.z, al.w, bl.w, wv.z, wv.w);
                }
            } else {
#pragma unroll
                for (int n = 0; n < NT; ++n) {
                    const int e = n * 8 + g;
                    const uint4 wv = e < E ? __ldg(reinterpret_cast<const uint4*>(Wg + (size_t)e * d) + c) : zero;
                    mma_bf16_16816(acc[n], xa.x, xb.x, xa.y, xb.y, wv.x, wv.y);
                    mma_bf16_16816(acc[n], xa.z, xb.z, xa.w, xb.w, wv.z, wv.w);
                }
            }
            if (++since_flush == FLUSH) {
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
        if (NORM) {
            // the 4 lanes of a group hold the row's chunks q = 0..3
#pragma unroll
            for (int m = 1; m <= 2; m <<= 1) {
                ss0 += __shfl_xor_sync(0xffffffffu, ss0, m);
                ss1 += __shfl_xor_sync(0xffffffffu, ss1, m);
            }
            if (q == 0) {
                sqp[warp][g] = ss0;
                sqp[warp][g + 8] = ss1;
            }
        }
        __syncthreads();
        if (threadIdx.x < 16 && t0 + (int)threadIdx.x < T) {
            const int t = threadIdx.x;
            float sc[EB];
            float sq = 0.f;
#pragma unroll
            for (int e = 0; e < EB; ++e) {
                float v = 0.f;
#pragma unroll
                for (int ww = 0; ww < 8; ++ww) v += part[ww][t][e];
                sc[e] = v;
            }
            if (NORM) {
#pragma unroll
                for (int ww = 0; ww < 8; ++ww) sq += sqp[ww][t];
            }
            finish_token<__nv_bfloat16, EB, NORM>(sc, sq, t0 + t, d, E, k, io);
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------- tcgen05 router

constexpr int RT_M = 128;                          // tokens per tile (MMA M, TMEM lanes)
constexpr int RT_BK = 64;                          // K per stage (one 128-byte swizzle row)
constexpr int RT_A_BYTES = RT_M * RT_BK * 2;       // 16 KiB of x
constexpr int RT_MAX_STAGES = 10;
// Ring of one kernel instance: A (x) and B (EP rows of Wg) per stage, about 180 KiB of x in
// flight per SM (the only CTA on it), enough to keep HBM busy from 128 SMs.
template <int EP>
struct RtRing {
    static constexpr int STAGE_BYTES = RT_A_BYTES + EP * RT_BK * 2;   // 18 or 20 KiB, 1 KiB aligned
    static constexpr int STAGES = EP == 16 ? 10 : 9;
};
constexpr int RT_CHUNK_KB = 4;                     // stages per fp32 flush (K = 256)
constexpr int RT_THREADS = 128;

struct RtCtrl {
    uint64_t full[RT_MAX_STAGES];
    uint64_t empty[RT_MAX_STAGES];
    uint64_t done;
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

template <int EP>
constexpr int rt_smem_bytes() {
    return RtRing<EP>::STAGES * RtRing<EP>::STAGE_BYTES + (int)sizeof(RtCtrl) + 1024;
}

// One 128-token tile per CTA (cluster rank = the K split it reads).  Warp 0
// lane 0 streams x (128 rows x 64) and Wg (EL rows x 64, EL = E) into a
// 9- or 10-stage ring; warp 1 lane 0 issues tcgen05.mma M = 128, N = EP (E rounded up
// to 16; the B rows past E hold zeros), accumulating every 256 of K into its
// own TMEM column block, so no accumulation inside the tensor core runs longer
// than K = 256; then all four warps read their 32 rows, add the blocks in
// order in fp32 and, with one split, finish the token (scores, top-k, gates).
// With several splits each CTA leaves the values of each of its 256-wide K
// chunks in shared memory (the ring, idle by then) and rank 0 adds all chunks in
// global K order.  Every split count therefore adds the same chunk values in the
// same order: the scores, and so the routing, of a token do not depend on the
// batch it comes in (for every T this kernel serves).
template <int EP>
__global__ void __launch_bounds__(RT_THREADS, 1)
    router_tc_kernel(const __grid_constant__ CUtensorMap mapX, const __grid_constant__ CUtensorMap mapW, int T,
                     int d, int E, int k, int tmem_cols, RouterIO<__nv_bfloat16> io, int* status,
                     long long wait_ns) {
    constexpr int RT_STAGES = RtRing<EP>::STAGES;
    constexpr int RT_STAGE_BYTES = RtRing<EP>::STAGE_BYTES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    // after the main loop the ring holds each chunk's scores for the cluster reduction: [chunk][row][EP + 1]
    float* part = reinterpret_cast<float*>(smem);
    RtCtrl* ctrl = reinterpret_cast<RtCtrl*>(smem + RT_STAGES * RT_STAGE_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint32_t nsplit;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(nsplit));
    const uint32_t split = ptx::cluster_ctarank();
    const int m0 = (int)(blockIdx.x / nsplit) * RT_M;
    const int nkb = d / RT_BK / (int)nsplit;            // stages of this CTA's K range
    const int kb0 = (int)split * nkb;
    const int chunks = (nkb + RT_CHUNK_KB - 1) / RT_CHUNK_KB;
    const int EL = E;                                    // Wg rows loaded (E % 8 == 0)
    const uint32_t tx = RT_A_BYTES + (uint32_t)EL * RT_BK * 2;

    pdl_trigger();
    if (threadIdx.x == 0) {
        for (int st = 0; st < RT_STAGES; ++st) {
            ptx::mbar_init(&ctrl->full[st], 1);
            ptx::mbar_init(&ctrl->empty[st], 1);
        }
        ptx::mbar_init(&ctrl->done, 1);
        ptx::mbar_init(&ctrl->drain, 1);
        ctrl->abort = 0;
        ptx::fence_mbar_init();
    }
    // B rows past E are never written by TMA: zero them once, so the MMA columns past E hold zeros
    if (EP > EL) {
        for (int st = 0; st < RT_STAGES; ++st) {
            uint32_t* b = reinterpret_cast<uint32_t*>(smem + st * RT_STAGE_BYTES + RT_A_BYTES + EL * RT_BK * 2);
            for (int i = threadIdx.x; i < (EP - EL) * RT_BK / 2; i += blockDim.x) b[i] = 0u;
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // visible to the tensor core
    }
    if (warp == 0 && lane == 0) {
        ptx::tma_prefetch_desc(&mapX);
        ptx::tma_prefetch_desc(&mapW);
    }
    if (warp == 1) {
        ptx::tmem_alloc(&ctrl->tmem_base, (uint32_t)tmem_cols);
        ptx::tmem_relinquish();
    }
    pdl_wait();   // global memory only after the previous kernel has completed
    ptx::tc_fence_before_sync();
    __syncthreads();
    ptx::tc_fence_after_sync();
    const uint32_t tmem_base = ctrl->tmem_base;
    const ptx::WaitCtl wc{&ctrl->abort, status, (uint64_t)wait_ns};

    if (warp == 0) {
        if (lane == 0) {
            const uint64_t pol_x = ptx::policy_evict_first();   // x is read once
            const uint64_t pol_w = ptx::policy_evict_last();    // Wg is read by every tile
            bool armed[RT_STAGES];
            uint32_t armed_phase[RT_STAGES];
#pragma unroll
            for (int st = 0; st < RT_STAGES; ++st) {
                armed[st] = false;
                armed_phase[st] = 0;
            }
            int stage = 0;
            uint32_t phase = 0;
            bool aborted = false;
            for (int kb = 0; kb < nkb; ++kb) {
                if (!ptx::mbar_wait(&ctrl->empty[stage], phase ^ 1u, wc)) {
                    aborted = true;
                    break;
                }
                uint8_t* sa = smem + stage * RT_STAGE_BYTES;
                ptx::mbar_arrive_expect_tx(&ctrl->full[stage], tx);
                ptx::tma_load_2d(sa, &mapX, &ctrl->full[stage], (kb0 + kb) * RT_BK, m0, pol_x);
                ptx::tma_load_2d(sa + RT_A_BYTES, &mapW, &ctrl->full[stage], (kb0 + kb) * RT_BK, 0, pol_w);
#pragma unroll
                for (int st = 0; st < RT_STAGES; ++st)
                    if (st == stage) {
                        armed[st] = true;
                        armed_phase[st] = phase;
                    }
                if (++stage == RT_STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (aborted || ctrl->abort) {
#pragma unroll
                for (int st = 0; st < RT_STAGES; ++st)
                    if (armed[st]) ptx::mbar_wait_drain(&ctrl->full[st], armed_phase[st], 100000000ull);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t IDESC = ptx::idesc_bf16_f32(RT_M, EP);
            int stage = 0;
            uint32_t phase = 0;
            bool issued = false, aborted = false;
            for (int kb = 0; kb < nkb; ++kb) {
                if (!ptx::mbar_wait(&ctrl->full[stage], phase, wc)) {
                    aborted = true;
                    break;
                }
                ptx::tc_fence_after_sync();
                const uint32_t a0 = ptx::smem_addr(smem + stage * RT_STAGE_BYTES);
                const uint32_t b0 = a0 + RT_A_BYTES;
                const uint32_t dcol = tmem_base + (uint32_t)((kb / RT_CHUNK_KB) * EP);
#pragma unroll
                for (int kk = 0; kk < RT_BK / 16; ++kk)
                    ptx::tc_mma_bf16(dcol, ptx::desc_kmajor_sw128(a0 + kk * 32), ptx::desc_kmajor_sw128(b0 + kk * 32),
                                     IDESC, ((kb % RT_CHUNK_KB) | kk) != 0);
                ptx::tc_commit(&ctrl->empty[stage]);
                issued = true;
                if (++stage == RT_STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (!aborted) {
                ptx::tc_commit(&ctrl->done);
            } else if (issued) {
                ptx::tc_commit(&ctrl->drain);
                ptx::mbar_wait_drain(&ctrl->drain, 0, 100000000ull);
            }
        }
    }
    __syncwarp();

    // epilogue: every warp reads its 32 TMEM lanes (rows m0 + 32 warp + lane)
    bool ok = ptx::mbar_wait(&ctrl->done, 0, wc);
    ok = __all_sync(0xffffffffu, ok);
    const int row = warp * 32 + lane;
    float sc[EP];
#pragma unroll
    for (int e = 0; e < EP; ++e) sc[e] = 0.f;
    if (ok) {
        ptx::tc_fence_after_sync();
        const uint32_t taddr = tmem_base + ((uint32_t)(warp * 32) << 16);
        for (int c = 0; c < chunks; ++c) {
            uint32_t r[EP];
            if constexpr (EP == 16) {
                ptx::tmem_ld_32x32b_x16(taddr + (uint32_t)(c * EP), r);
            } else {
                ptx::tmem_ld_32x32b_x32(taddr + (uint32_t)(c * EP), r);
            }
            ptx::tmem_ld_wait();
            if (nsplit > 1) {
                float* dst = part + ((size_t)c * RT_M + row) * (EP + 1);
#pragma unroll
                for (int e = 0; e < EP; ++e) dst[e] = __uint_as_float(r[e]);
            } else {
#pragma unroll
                for (int e = 0; e < EP; ++e) sc[e] += __uint_as_float(r[e]);
            }
        }
    }
    ptx::tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after_sync();
        ptx::tmem_dealloc(tmem_base, (uint32_t)tmem_cols);
    }
    if (nsplit > 1) {
        ptx::cluster_sync();   // every split's chunk scores are in its shared memory
        if (split == 0) {
            // all chunks in global K order: split r holds chunks r * chunks .. (r + 1) * chunks - 1
            for (uint32_t r = 0; r < nsplit; ++r) {
                for (int c = 0; c < chunks; ++c) {
                    const uint32_t peer =
                        ptx::map_to_rank(ptx::smem_addr(part + ((size_t)c * RT_M + row) * (EP + 1)), r);
#pragma unroll
                    for (int e = 0; e < EP; ++e) {
                        float v;
                        asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(peer + 4u * e) : "memory");
                        sc[e] += v;
                    }
                }
            }
        }
        ptx::cluster_sync();   // no CTA leaves while rank 0 still reads its chunks
        if (split != 0) return;
    }
    if (!ok || m0 + row >= T) return;
    finish_token<__nv_bfloat16, EP, false>(sc, 0.f, m0 + row, d, E, k, io);
}

template <int EP>
cudaError_t launch_router_tc_t(const __nv_bfloat16* x, const __nv_bfloat16* Wg, int T, int d, int E, int k,
                               const RouterIO<__nv_bfloat16>& io, int num_sms, int* status, long long wait_ns,
                               cudaStream_t s) {
    static PerDeviceOnce attr;
    cudaError_t e = attr.run([] {
        return cudaFuncSetAttribute(router_tc_kernel<EP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    rt_smem_bytes<EP>());
    });
    if (e != cudaSuccess) return e;
    const int tiles = (T + RT_M - 1) / RT_M;
    const int kbs = d / RT_BK;
    // A split count is usable when it divides d's K steps into whole 256-wide chunks per CTA (so
    // every split count adds the same chunks in the same order), the CTA's chunks fit the 512 TMEM
    // columns and, with a cluster, its chunk scores fit the idle ring.  Take the largest usable one
    // that keeps one CTA per SM, else the smallest usable one.
    const long long ring = (long long)RtRing<EP>::STAGES * RtRing<EP>::STAGE_BYTES;
    auto usable = [&](int sp) {
        if (kbs % sp != 0) return false;
        const int per = kbs / sp;
        if (sp > 1 && per % RT_CHUNK_KB != 0) return false;
        const int ch = (per + RT_CHUNK_KB - 1) / RT_CHUNK_KB;
        if (ch * EP > 512) return false;
        return sp == 1 || (long long)ch * RT_M * (EP + 1) * 4 <= ring;
    };
    int splits = 0;
    for (int sp = 8; sp >= 1 && !splits; sp /= 2)
        if (usable(sp) && (long long)tiles * sp <= num_sms) splits = sp;
    for (int sp = 1; sp <= 8 && !splits; sp *= 2)
        if (usable(sp)) splits = sp;
    if (!splits) return cudaErrorNotSupported;   // the caller takes the mma.sync router
    const int chunks = (kbs / splits + RT_CHUNK_KB - 1) / RT_CHUNK_KB;
    int cols = 32;
    while (cols < chunks * EP) cols *= 2;
    CUtensorMap mx, mw;
    if (!map_matrix(&mx, x, (size_t)T, d, RT_BK, RT_M) || !map_matrix(&mw, Wg, (size_t)E, d, RT_BK, E))
        return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(tiles * splits), 1, 1);
    cfg.blockDim = dim3(RT_THREADS, 1, 1);
    cfg.dynamicSmemBytes = rt_smem_bytes<EP>();
    cfg.stream = s;
    cudaLaunchAttribute attr2[2];
    attr2[0].id = cudaLaunchAttributeClusterDimension;
    attr2[0].val.clusterDim.x = (unsigned)splits;
    attr2[0].val.clusterDim.y = 1;
    attr2[0].val.clusterDim.z = 1;
    attr2[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr2[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr2;
    cfg.numAttrs = 2;
    e = cudaLaunchKernelEx(&cfg, router_tc_kernel<EP>, mx, mw, T, d, E, k, cols, io, status, wait_ns);
    return e != cudaSuccess ? e : cudaGetLastError();
}

// Chunks per thread the kernels are compiled for: 16-byte chunks x 256 threads x RMAX
// cover d <= 8192 (bf16) / 4096 (fp32) with RMAX = 4; longer rows take the looping form.
template <typename In, int EB, int TB, bool NORM>
cudaError_t launch_router_t(const In* x, const In* Wg, int T, int d, int E, int k, const RouterIO<In>& io,
                            int num_sms, cudaStream_t s) {
    const int nchunks = d / Chunk<In>::N;
    // small batches: one token per block, so every SM gets work
    const bool small = T <= 4 * num_sms;
    const int tb = small ? 1 : TB;
    int blocks = (T + tb - 1) / tb;
    if (blocks < 1) blocks = 1;
    const dim3 grid(blocks), block(256);
    if (nchunks <= 256) {
        if (small) return launch_pdl(router_kernel<In, EB, 1, 1, NORM>, grid, block, 0, s, x, Wg, T, d, E, k, io);
        return launch_pdl(router_kernel<In, EB, TB, 1, NORM>, grid, block, 0, s, x, Wg, T, d, E, k, io);
    } else if (nchunks <= 512) {
        if (small) return launch_pdl(router_kernel<In, EB, 1, 2, NORM>, grid, block, 0, s, x, Wg, T, d, E, k, io);
        return launch_pdl(router_kernel<In, EB, TB, 2, NORM>, grid, block, 0, s, x, Wg, T, d, E, k, io);
    } else if (nchunks <= 1024) {
        if (small) return launch_pdl(router_kernel<In, EB, 1, 4, NORM>, grid, block, 0, s, x, Wg, T, d, E, k, io);
        return launch_pdl(router_kernel<In, EB, TB, 4, NORM>, grid, block, 0, s, x, Wg, T, d, E, k, io);
    }
    const int g = T < 65535 ? T : 65535;
    return launch_pdl(router_loop_kernel<In, EB, NORM>, dim3(g), block, 0, s, x, Wg, T, d, E, k, io);
}

template <typename In, bool NORM>
cudaError_t launch_router_any(const In* x, const In* Wg, int T, int d, int E, int k, const RouterIO<In>& io,
                              int num_sms, cudaStream_t s) {
    if (E <= 8) return launch_router_t<In, 8, 4, NORM>(x, Wg, T, d, E, k, io, num_sms, s);
    if (E <= 16) return launch_router_t<In, 16, 2, NORM>(x, Wg, T, d, E, k, io, num_sms, s);
    return launch_router_t<In, 32, 1, NORM>(x, Wg, T, d, E, k, io, num_sms, s);
}

template <bool NORM>
cudaError_t launch_router_mma(const __nv_bfloat16* x, const __nv_bfloat16* Wg, int T, int d, int E, int k,
                              const RouterIO<__nv_bfloat16>& io, int num_sms, cudaStream_t s) {
    const int tiles = (T + 15) / 16;
    int grid = tiles < num_sms * 16 ? tiles : num_sms * 16;
    if (grid < 1) grid = 1;
    if (E <= 8) return launch_pdl(router_mma_kernel<1, NORM>, dim3(grid), dim3(256), 0, s, x, Wg, T, d, E, k, io);
    if (E <= 16) return launch_pdl(router_mma_kernel<2, NORM>, dim3(grid), dim3(256), 0, s, x, Wg, T, d, E, k, io);
    return launch_pdl(router_mma_kernel<4, NORM>, dim3(grid), dim3(256), 0, s, x, Wg, T, d, E, k, io);
}

template <typename In>
RouterIO<In> make_io(int32_t* idx, float* w, const RouteExtras& ex) {
    return RouterIO<In>{idx, w, static_cast<const In*>(ex.gamma), ex.eps, ex.rstd, ex.logits};
}

}  // namespace

cudaError_t launch_router_bf16(const void* x, const void* Wg, int T, int d, int E, int k, int32_t* idx, float* w,
                               int num_sms, cudaStream_t s, const RouteExtras& ex) {
    const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
    const __nv_bfloat16* wb = static_cast<const __nv_bfloat16*>(Wg);
    const RouterIO<__nv_bfloat16> io = make_io<__nv_bfloat16>(idx, w, ex);
    // tensor-core scores for large batches; small batches spread one token per block instead
    if (!ex.gamma && E % 8 == 0 && d % RT_BK == 0 && T > 4 * num_sms) {
        const cudaError_t e = E <= 16 ? launch_router_tc_t<16>(xb, wb, T, d, E, k, io, num_sms, ex.status, ex.wait_ns, s)
                                      : launch_router_tc_t<32>(xb, wb, T, d, E, k, io, num_sms, ex.status, ex.wait_ns, s);
        if (e != cudaErrorNotSupported) return e;   // else: no usable split of d, the mma.sync router below
    }
    if (d % 32 == 0 && T > 4 * num_sms) {
        return ex.gamma ? launch_router_mma<true>(xb, wb, T, d, E, k, io, num_sms, s)
                        : launch_router_mma<false>(xb, wb, T, d, E, k, io, num_sms, s);
    }
    return ex.gamma ? launch_router_any<__nv_bfloat16, true>(xb, wb, T, d, E, k, io, num_sms, s)
                    : launch_router_any<__nv_bfloat16, false>(xb, wb, T, d, E, k, io, num_sms, s);
}

cudaError_t launch_router_f32(const float* x, const float* Wg, int T, int d, int E, int k, int32_t* idx, float* w,
                              int num_sms, cudaStream_t s, const RouteExtras& ex) {
    const RouterIO<float> io = make_io<float>(idx, w, ex);
    return ex.gamma ? launch_router_any<float, true>(x, Wg, T, d, E, k, io, num_sms, s)
                    : launch_router_any<float, false>(x, Wg, T, d, E, k, io, num_sms, s);
}

}  // namespace moe
