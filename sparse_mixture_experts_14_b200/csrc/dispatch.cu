// Dispatch: a deterministic, stable counting sort of the routed assignments
// into expert-contiguous segments, then a gather of token rows into them.
//
// This is the per-expert batching of the page's "MoEレイヤー全体の実装" code
// (one mask per expert, x[mask] for the tokens that chose it), done in one
// integer-only pass instead of E masked passes.  Assignment (t, j) of a token
// that chose expert e lands in row
//     offsets[e] + #{t' < t : e is among the experts t' chose}
// so rows inside a segment follow token order.  Segments are padded to 128
// rows (one tensor-core tile); padding rows carry perm = -1 and zero inputs.
//
// Kernels: up to 1024 tokens, one block does it all; above that, histogram
// (per 1024-token block), scan (one block: totals, padded offsets, per-block
// bases) and scatter (per-block stable ranks by warp ballots).  Then gather
// (one warp per row, 16-byte copies).
//
// Block form: the gather also applies the pre-norm of the MoE sub-layer
// (section "Mixtral 8x7B — Sparse MoEの導入", subsection "Mixtralのアーキテクチャ"),
// writing (gamma * x) * r, r = the row's 1/sqrt(mean(x^2) + eps) from the
// router pass, rounded once to the row type.  NORM selects the row type:
// 0 = plain copy, 1 = bf16, 2 = fp32.
#include "moe_common.cuh"

namespace moe {
namespace {

// One 16-byte vector of a row after the optional normalisation.
template <int NORM>
__device__ __forceinline__ uint4 norm_vec(uint4 v, uint4 g, float r) {
    if (NORM == 1) {
        uint4 o;
        o.x = pack_bf16x2(bf16_lo(v.x) * bf16_lo(g.x) * r, bf16_hi(v.x) * bf16_hi(g.x) * r);
        o.y = pack_bf16x2(bf16_lo(v.y) * bf16_lo(g.y) * r, bf16_hi(v.y) * bf16_hi(g.y) * r);
        o.z = pack_bf16x2(bf16_lo(v.z) * bf16_lo(g.z) * r, bf16_hi(v.z) * bf16_hi(g.z) * r);
        o.w = pack_bf16x2(bf16_lo(v.w) * bf16_lo(g.w) * r, bf16_hi(v.w) * bf16_hi(g.w) * r);
        return o;
    }
    if (NORM == 2) {
        uint4 o;
        o.x = __float_as_uint(__uint_as_float(v.x) * __uint_as_float(g.x) * r);
        o.y = __float_as_uint(__uint_as_float(v.y) * __uint_as_float(g.y) * r);
        o.z = __float_as_uint(__uint_as_float(v.z) * __uint_as_float(g.z) * r);
        o.w = __float_as_uint(__uint_as_float(v.w) * __uint_as_float(g.w) * r);
        return o;
    }
    return v;
}

// Copy one row of nvec 16-byte vectors with this warp, 8 loads in flight per
// lane before their stores; NORM != 0 normalises with gamma and r.
template <int NORM>
__device__ __forceinline__ void copy_row(const uint4* __restrict__ src, uint4* __restrict__ dst, size_t nvec,
                                         int lane, const uint4* __restrict__ gam, float r) {
    for (size_t v0 = lane; v0 < nvec; v0 += 32 * 8) {
        uint4 buf[8], gb[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const size_t v = v0 + (size_t)u * 32;
            if (v < nvec) {
                buf[u] = __ldg(src + v);
                if (NORM) gb[u] = __ldg(gam + v);
            }
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const size_t v = v0 + (size_t)u * 32;
            if (v < nvec) dst[v] = NORM ? norm_vec<NORM>(buf[u], gb[u], r) : buf[u];
        }
    }
}

__global__ void __launch_bounds__(kDispatchTokens) hist_kernel(const int32_t* __restrict__ idx, int T, int E, int k,
                                                               int32_t* __restrict__ blk_counts, int* status) {
    pdl_trigger();
    pdl_wait();
    __shared__ int cnt[kMaxExperts];
    if (threadIdx.x < kMaxExperts) cnt[threadIdx.x] = 0;
    __syncthreads();
    const int t = blockIdx.x * kDispatchTokens + threadIdx.x;
    if (t < T) {
        uint32_t mask = 0;
        for (int j = 0; j < k; ++j) {
            const int e = idx[(size_t)t * k + j];
            if (e < 0 || e >= E || ((mask >> e) & 1u)) {
                record_status(status, MOE_ERR_DEVICE);   // out of range or chosen twice: dropped
                continue;
            }
            mask |= 1u << e;
            atomicAdd(&cnt[e], 1);
        }
    }
    __syncthreads();
    if (threadIdx.x < E) blk_counts[(size_t)blockIdx.x * E + threadIdx.x] = cnt[threadIdx.x];
}

// One block of 32 warps; warp e owns expert e.  In place: blk_counts[b][e]
// becomes the first row of block b's assignments to expert e.
__global__ void __launch_bounds__(1024) scan_kernel(int32_t* __restrict__ blk, int NB, int E, Meta* __restrict__ meta,
                                                    int32_t* __restrict__ perm, size_t slots, int* status) {
    pdl_trigger();
    pdl_wait();
    __shared__ int tot[kMaxExperts];
    __shared__ int offs[kMaxExperts + 1];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp < E) {
        int s = 0;
        for (int b = lane; b < NB; b += 32) s += blk[(size_t)b * E + warp];
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) s += __shfl_xor_sync(0xffffffffu, s, m);
        if (lane == 0) tot[warp] = s;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        offs[0] = 0;
        for (int e = 0; e < E; ++e) offs[e + 1] = offs[e] + (tot[e] + kSegRows - 1) / kSegRows * kSegRows;
        if ((size_t)offs[E] > slots) record_status(status, MOE_ERR_DEVICE);
        for (int e = 0; e < E; ++e) meta->counts[e] = tot[e];
        for (int e = 0; e <= E; ++e) meta->offsets[e] = offs[e];
        for (int i = 0; i < kWaveSlots; ++i) meta->waves[i] = 0;
    }
    __syncthreads();
    if (warp < E) {
        int carry = offs[warp];
        for (int b0 = 0; b0 < NB; b0 += 32) {
            const int b = b0 + lane;
            const int v = (b < NB) ? blk[(size_t)b * E + warp] : 0;
            int incl = v;
#pragma unroll
            for (int m = 1; m < 32; m <<= 1) {
                const int o = __shfl_up_sync(0xffffffffu, incl, m);
                if (lane >= m) incl += o;
            }
            if (b < NB) blk[(size_t)b * E + warp] = carry + incl - v;
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
    }
    // padding rows of every segment
    for (int e = 0; e < E; ++e) {
        const int beg = offs[e] + tot[e], end = offs[e + 1];
        for (int r = beg + threadIdx.x; r < end; r += blockDim.x)
            if ((size_t)r < slots) perm[r] = -1;
    }
}

__global__ void __launch_bounds__(kDispatchTokens) scatter_kernel(const int32_t* __restrict__ idx, int T, int E, int k,
                                                                  const int32_t* __restrict__ blk_base,
                                                                  int32_t* __restrict__ perm, int32_t* __restrict__ inv,
                                                                  size_t slots, int* status) {
    pdl_trigger();
    pdl_wait();
    __shared__ int wcnt[32][kMaxExperts + 1];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * kDispatchTokens + threadIdx.x;
    uint32_t mask = 0;
    if (t < T) {
        for (int j = 0; j < k; ++j) {
            const int e = idx[(size_t)t * k + j];
            if (e >= 0 && e < E) mask |= 1u << e;
        }
    }
    const uint32_t lt = (1u << lane) - 1u;
    int rank[kMaxExperts];   // in-warp rank of this token among the warp's tokens that chose e
    for (int e = 0; e < E; ++e) {
        const uint32_t bal = __ballot_sync(0xffffffffu, (mask >> e) & 1u);
        rank[e] = __popc(bal & lt);
        if (lane == 0) wcnt[warp][e] = __popc(bal);
    }
    __syncthreads();
    if (threadIdx.x < E) {
        const int e = threadIdx.x;
        int run = 0;
        for (int w = 0; w < 32; ++w) {
            const int c = wcnt[w][e];
            wcnt[w][e] = run;
            run += c;
        }
    }
    __syncthreads();
    if (t < T) {
        uint32_t seen = 0;
        for (int j = 0; j < k; ++j) {
            const int a = t * k + j;
            const int e = idx[a];
            if (e < 0 || e >= E || ((seen >> e) & 1u)) {
                inv[a] = -1;
                continue;
            }
            seen |= 1u << e;
            const int slot = blk_base[(size_t)blockIdx.x * E + e] + wcnt[warp][e] + rank[e];
            if (slot < 0 || (size_t)slot >= slots) {
                record_status(status, MOE_ERR_DEVICE);
                inv[a] = -1;
                continue;
            }
            perm[slot] = a;
            inv[a] = slot;
        }
    }
}

// Whole dispatch in one block when every token fits one 1024-thread block:
// histogram, padded offsets and stable ranks without global scratch.
__global__ void __launch_bounds__(kDispatchTokens) dispatch_single_kernel(const int32_t* __restrict__ idx, int T,
                                                                          int E, int k, Meta* __restrict__ meta,
                                                                          int32_t* __restrict__ perm,
                                                                          int32_t* __restrict__ inv, size_t slots,
                                                                          int* status) {
    pdl_trigger();
    pdl_wait();
    __shared__ int wcnt[32][kMaxExperts + 1];
    __shared__ int offs[kMaxExperts + 1];
    __shared__ int tot[kMaxExperts];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = threadIdx.x;
    uint32_t mask = 0;
    if (t < T) {
        for (int j = 0; j < k; ++j) {
            const int e = idx[(size_t)t * k + j];
            if (e < 0 || e >= E || ((mask >> e) & 1u)) {
                record_status(status, MOE_ERR_DEVICE);
                continue;
            }
            mask |= 1u << e;
        }
    }
    const uint32_t lt = (1u << lane) - 1u;
    int rank[kMaxExperts];
    for (int e = 0; e < E; ++e) {
        const uint32_t bal = __ballot_sync(0xffffffffu, (mask >> e) & 1u);
        rank[e] = __popc(bal & lt);
        if (lane == 0) wcnt[warp][e] = __popc(bal);
    }
    __syncthreads();
    if (threadIdx.x < E) {
        const int e = threadIdx.x;
        int run = 0;
        for (int w = 0; w < 32; ++w) {
            const int c = wcnt[w][e];
            wcnt[w][e] = run;
            run += c;
        }
        tot[e] = run;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        offs[0] = 0;
        for (int e = 0; e < E; ++e) offs[e + 1] = offs[e] + (tot[e] + kSegRows - 1) / kSegRows * kSegRows;
        if ((size_t)offs[E] > slots) record_status(status, MOE_ERR_DEVICE);
        for (int e = 0; e < E; ++e) meta->counts[e] = tot[e];
        for (int e = 0; e <= E; ++e) meta->offsets[e] = offs[e];
        for (int i = 0; i < kWaveSlots; ++i) meta->waves[i] = 0;
    }
    __syncthreads();
    if (t < T) {
        uint32_t seen = 0;
        for (int j = 0; j < k; ++j) {
            const int a = t * k + j;
            const int e = idx[a];
            if (e < 0 || e >= E || ((seen >> e) & 1u)) {
                inv[a] = -1;
                continue;
            }
            seen |= 1u << e;
            const int slot = offs[e] + wcnt[warp][e] + rank[e];
            if ((size_t)slot >= slots) {
                inv[a] = -1;
                continue;
            }
            perm[slot] = a;
            inv[a] = slot;
        }
    }
    for (int e = 0; e < E; ++e) {
        const int beg = offs[e] + tot[e], end = offs[e + 1];
        for (int r = beg + threadIdx.x; r < end; r += blockDim.x)
            if ((size_t)r < slots) perm[r] = -1;
    }
}

// Few tokens (T <= 64, the decode path): dispatch and gather in one launch.
// Every block recomputes the (tiny) stable counting sort in shared memory, so
// the blocks need no communication; block 0 publishes the segment table, perm
// and inv, and all blocks copy their share of token rows into the segments.
constexpr int kSmallTokens = 64;
constexpr int kSmallMaxRows = kSmallTokens * kMaxExperts + kMaxExperts * kSegRows;

template <int NORM>
__global__ void __launch_bounds__(256) dispatch_gather_small_kernel(const int32_t* __restrict__ idx, int T, int E,
                                                                    int k, const uint8_t* __restrict__ x,
                                                                    size_t row_bytes, Meta* __restrict__ meta,
                                                                    int32_t* __restrict__ perm,
                                                                    int32_t* __restrict__ inv,
                                                                    uint8_t* __restrict__ xp, size_t slots,
                                                                    int* status, const uint4* __restrict__ gam,
                                                                    const float* __restrict__ rstd) {
    pdl_trigger();
    pdl_wait();
    __shared__ int offs[kMaxExperts + 1];
    __shared__ int cnt[kMaxExperts];
    __shared__ int sidx[kSmallTokens * kMaxExperts];     // the assignments
    __shared__ int row_of[kSmallTokens * kMaxExperts];   // slot of assignment (t, j), -1 if dropped
    __shared__ int owner[kSmallMaxRows];                  // assignment held by each row, -1 on padding
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int a = tid; a < T * k; a += blockDim.x) {
        sidx[a] = idx[a];
        row_of[a] = -1;
    }
    __syncthreads();
    // warp 0: stable counting sort; lane owns tokens lane and lane + 32
    if (warp == 0) {
        uint32_t mask[2] = {0u, 0u};
        for (int h = 0; h < 2; ++h) {
            const int t = lane + 32 * h;
            if (t < T) {
                for (int j = 0; j < k; ++j) {
                    const int e = sidx[t * k + j];
                    if (e < 0 || e >= E || ((mask[h] >> e) & 1u)) {
                        if (blockIdx.x == 0) record_status(status, MOE_ERR_DEVICE);
                        continue;
                    }
                    mask[h] |= 1u << e;
                }
            }
        }
        const uint32_t lt = (1u << lane) - 1u;
        int base = 0;
        for (int e = 0; e < E; ++e) {
            const uint32_t b0 = __ballot_sync(0xffffffffu, (mask[0] >> e) & 1u);
            const uint32_t b1 = __ballot_sync(0xffffffffu, (mask[1] >> e) & 1u);
            const int n = __popc(b0) + __popc(b1);
            for (int h = 0; h < 2; ++h) {
                if ((mask[h] >> e) & 1u) {
                    const int t = lane + 32 * h;
                    const int r = h == 0 ? __popc(b0 & lt) : __popc(b0) + __popc(b1 & lt);
                    for (int j = 0; j < k; ++j)
                        if (sidx[t * k + j] == e) {
                            row_of[t * k + j] = base + r;   // first occurrence; duplicates stay dropped
                            break;
                        }
                }
            }
            if (lane == 0) {
                cnt[e] = n;
                offs[e] = base;
            }
            base += (n + kSegRows - 1) / kSegRows * kSegRows;
        }
        if (lane == 0) offs[E] = base;
    }
    __syncthreads();
    const int total = offs[E];
    for (int r = tid; r < total; r += blockDim.x) owner[r] = -1;
    __syncthreads();
    for (int a = tid; a < T * k; a += blockDim.x)
        if (row_of[a] >= 0) owner[row_of[a]] = a;
    __syncthreads();
    if (blockIdx.x == 0) {
        if (tid == 0) {
            if ((size_t)total > slots) record_status(status, MOE_ERR_DEVICE);
            for (int e = 0; e < E; ++e) meta->counts[e] = cnt[e];
            for (int e = 0; e <= E; ++e) meta->offsets[e] = offs[e];
            for (int i = 0; i < kWaveSlots; ++i) meta->waves[i] = 0;
        }
        for (int a = tid; a < T * k; a += blockDim.x) inv[a] = row_of[a];
        for (int r = tid; r < total; r += blockDim.x)
            if ((size_t)r < slots) perm[r] = owner[r];
    }
    // gather: one warp per assignment, strided over all blocks.  Only rows that
    // hold a token are written: the decode kernels read at most the first 64
    // rows of a segment and discard the MMA columns of rows past the expert's
    // token count, so padding rows are never used on this path.
    const size_t nvec = row_bytes / 16;
    const int gw = blockIdx.x * (blockDim.x >> 5) + warp;
    const int nw = gridDim.x * (blockDim.x >> 5);
    for (int a = gw; a < T * k; a += nw) {
        const int r = row_of[a];
        if (r < 0 || (size_t)r >= slots) continue;
        const int t = a / k;
        copy_row<NORM>(reinterpret_cast<const uint4*>(x + (size_t)t * row_bytes),
                       reinterpret_cast<uint4*>(xp + (size_t)r * row_bytes), nvec, lane, gam,
                       NORM ? rstd[t] : 0.f);
    }
}

// One warp per row of the padded buffer; rows past offsets[E] are left alone.
template <int NORM>
__global__ void __launch_bounds__(256) gather_kernel(const uint8_t* __restrict__ x, size_t row_bytes, int T, int k,
                                                     const Meta* __restrict__ meta, int E,
                                                     const int32_t* __restrict__ perm, uint8_t* __restrict__ xp,
                                                     size_t slots, int* status, const uint4* __restrict__ gam,
                                                     const float* __restrict__ rstd) {
    pdl_trigger();
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const size_t warps = (size_t)gridDim.x * (blockDim.x >> 5);
    const size_t total = (size_t)meta->offsets[E];
    debug_check(total <= slots, status);
    const size_t nvec = row_bytes / 16;
    const long long TK = (long long)T * k;
    for (size_t r = (size_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < total && r < slots;
         r += warps) {
        const int a = perm[r];
        uint4* dst = reinterpret_cast<uint4*>(xp + r * row_bytes);
        debug_check(a >= -1 && a < TK, status);   // -1 marks a padding row
        if (a >= 0 && a < TK) {
            const int t = a / k;
            copy_row<NORM>(reinterpret_cast<const uint4*>(x + (size_t)t * row_bytes), dst, nvec, lane, gam,
                           NORM ? rstd[t] : 0.f);
        } else {
            const uint4 z = make_uint4(0, 0, 0, 0);
            for (size_t v = lane; v < nvec; v += 32) dst[v] = z;
        }
    }
}

}  // namespace

cudaError_t launch_dispatch(const int32_t* idx, int T, int E, int k, int32_t* blk_counts, Meta* meta, int32_t* perm,
                            int32_t* inv, int* status, cudaStream_t s) {
    const int NB = dispatch_blocks(T);
    const size_t slots = slots_capacity(T, E, k);
    if (NB == 1) {
        return launch_pdl(dispatch_single_kernel, dim3(1), dim3(kDispatchTokens), 0, s, idx, T, E, k, meta, perm, inv,
                          slots, status);
    }
    cudaError_t e = launch_pdl(hist_kernel, dim3(NB), dim3(kDispatchTokens), 0, s, idx, T, E, k, blk_counts, status);
    if (e == cudaSuccess) e = launch_pdl(scan_kernel, dim3(1), dim3(1024), 0, s, blk_counts, NB, E, meta, perm, slots, status);
    if (e == cudaSuccess)
        e = launch_pdl(scatter_kernel, dim3(NB), dim3(kDispatchTokens), 0, s, idx, T, E, k, blk_counts, perm, inv, slots,
                       status);
    return e;
}

cudaError_t launch_dispatch_gather_small(const int32_t* idx, int T, int E, int k, const void* x, size_t elem_bytes,
                                         int d, Meta* meta, int32_t* perm, int32_t* inv, void* xp, size_t slots,
                                         int* status, cudaStream_t s, const GatherNorm& nm) {
    if (T > kSmallTokens) return cudaErrorInvalidValue;
    const int rows = T * k;
    int blocks = (rows + 7) / 8;   // about one row per warp
    if (blocks < 1) blocks = 1;
    if (blocks > 64) blocks = 64;
    const uint8_t* xb = static_cast<const uint8_t*>(x);
    uint8_t* xpb = static_cast<uint8_t*>(xp);
    const uint4* gam = static_cast<const uint4*>(nm.gamma);
    const size_t rb = (size_t)d * elem_bytes;
    auto kern = !nm.gamma ? dispatch_gather_small_kernel<0>
                          : (elem_bytes == 2 ? dispatch_gather_small_kernel<1> : dispatch_gather_small_kernel<2>);
    return launch_pdl(kern, dim3(blocks), dim3(256), 0, s, idx, T, E, k, xb, rb, meta, perm, inv, xpb, slots, status,
                      gam, nm.rstd);
}

cudaError_t launch_gather(const void* x, size_t elem_bytes, int T, int d, int E, int k, const Meta* meta,
                          const int32_t* perm, void* xp, size_t slots, int* status, cudaStream_t s,
                          const GatherNorm& nm) {
    const size_t rows_per_block = 8;
    size_t blocks = (slots + rows_per_block - 1) / rows_per_block;
    if (blocks > 65535 * 4) blocks = 65535 * 4;
    const uint4* gam = static_cast<const uint4*>(nm.gamma);
    auto kern = !nm.gamma ? gather_kernel<0> : (elem_bytes == 2 ? gather_kernel<1> : gather_kernel<2>);
    return launch_pdl(kern, dim3((unsigned)blocks), dim3(256), 0, s, static_cast<const uint8_t*>(x),
                      (size_t)d * elem_bytes, T, k, meta, E, perm, static_cast<uint8_t*>(xp), slots, status, gam,
                      nm.rstd);
}

}  // namespace moe
