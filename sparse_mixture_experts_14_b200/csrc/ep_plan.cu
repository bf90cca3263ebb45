// Expert-parallel dispatch plan (host code): which rows each rank sends to and
// receives from every other rank, and where the received rows land in its own
// expert segments.
//
// The summary page ("Mixtral of Experts", its limitations lists) names expert
// parallelism: experts spread over GPUs, each token's rows sent to the GPU that
// holds its chosen experts and the outputs sent back (an all-to-all each way).
// Experts are split into R contiguous groups, rank s owning [s E / R, (s+1) E / R).
//
// Send order on rank r: its assignments sorted by expert, stable in token order
// (the dispatch's counting sort without segment padding), so the rows for rank s
// are one contiguous run holding experts lo(s)..hi(s)-1 in order.  Receive order
// on rank s: by source rank, each source's run as sent.  In rank s's expert
// segments (padded to 128 rows, as the single-GPU dispatch pads them), local
// expert e holds the rows from source 0, then source 1, ...; within a source, in
// that source's token order.  With tokens numbered source-major (rank 0's
// tokens first), every segment is exactly the single-GPU dispatch's segment of
// the concatenated batch: the grouped GEMMs see the same rows in the same order.
#include <climits>

#include "moe_common.cuh"

using namespace moe;

extern "C" moe_status moe_ep_plan(const int32_t* counts_all, int R, int E, int rank, int32_t* send_counts,
                                  int32_t* send_offsets, int32_t* recv_counts, int32_t* recv_offsets,
                                  int32_t* expert_range, int32_t* seg_counts, int32_t* seg_offsets,
                                  int32_t* block_recv, int32_t* block_seg) {
    if (!counts_all || !send_counts || !send_offsets || !recv_counts || !recv_offsets || !expert_range ||
        !seg_counts || !seg_offsets || !block_recv || !block_seg)
        return MOE_ERR_INVALID_ARG;
    if (R <= 0 || E <= 0 || rank < 0 || rank >= R) return MOE_ERR_INVALID_ARG;
    if (E > kMaxExperts) return MOE_ERR_UNSUPPORTED;
    long long total = 0;
    for (long long i = 0; i < (long long)R * E; ++i) {
        if (counts_all[i] < 0) return MOE_ERR_INVALID_ARG;
        total += counts_all[i];
    }
    if (total + (long long)E * kSegRows >= INT_MAX) return MOE_ERR_UNSUPPORTED;
    auto lo = [&](int s) { return (int)((long long)s * E / R); };
    const int* me = counts_all + (size_t)rank * E;
    // rows to each rank: this rank's assignments to that rank's experts
    send_offsets[0] = 0;
    for (int s = 0; s < R; ++s) {
        int n = 0;
        for (int e = lo(s); e < lo(s + 1); ++e) n += me[e];
        send_counts[s] = n;
        send_offsets[s + 1] = send_offsets[s] + n;
    }
    const int e0 = lo(rank), e1 = lo(rank + 1), EL = e1 - e0;
    expert_range[0] = e0;
    expert_range[1] = e1;
    // rows from each rank: that rank's assignments to this rank's experts
    recv_offsets[0] = 0;
    for (int s = 0; s < R; ++s) {
        int n = 0;
        for (int e = e0; e < e1; ++e) n += counts_all[(size_t)s * E + e];
        recv_counts[s] = n;
        recv_offsets[s + 1] = recv_offsets[s] + n;
    }
    // local expert segments, padded to kSegRows rows each
    seg_offsets[0] = 0;
    for (int l = 0; l < EL; ++l) {
        int n = 0;
        for (int s = 0; s < R; ++s) n += counts_all[(size_t)s * E + e0 + l];
        seg_counts[l] = n;
        seg_offsets[l + 1] = seg_offsets[l] + (n + kSegRows - 1) / kSegRows * kSegRows;
    }
    // block (source s, local expert l): start in the receive buffer and in the segments
    for (int s = 0; s < R; ++s) {
        int at = recv_offsets[s];
        for (int l = 0; l < EL; ++l) {
            int before = 0;   // rows of expert e0 + l from sources before s
            for (int q = 0; q < s; ++q) before += counts_all[(size_t)q * E + e0 + l];
            block_recv[(size_t)s * EL + l] = at;
            block_seg[(size_t)s * EL + l] = seg_offsets[l] + before;
            at += counts_all[(size_t)s * E + e0 + l];
        }
    }
    return MOE_OK;
}

// ---------------------------------------------------------------- data plane (device)
//
// One rank's share of the layer under expert parallelism, between its two
// all-to-alls (which the caller runs, e.g. NCCL's through torch.distributed):
//   moe_ep_dispatch  route-side: the counting sort of its assignments, then its
//                    token rows copied into send order (one row per assignment)
//   moe_ep_experts   expert-side: received rows into its padded expert segments,
//                    the grouped GEMMs on its experts, outputs back in receive order
//   moe_ep_combine   route-side: the gate-weighted sum of each token's returned
//                    rows, slot 0 first, the single-GPU combine's arithmetic
// With every rank's rows numbered source-major, each expert segment equals the
// single-GPU dispatch's, so every output equals the single-GPU layer's bit for bit.

namespace moe {
namespace {

// Send row of assignment a = (t, j): the assignments before it in send order are
// those of lower experts, then those of its own expert in lower segment rows.
__global__ void __launch_bounds__(256) ep_pack_kernel(const uint8_t* __restrict__ x, size_t row_bytes,
                                                      const int32_t* __restrict__ idx, const int32_t* __restrict__ inv,
                                                      const Meta* __restrict__ meta, int T, int E, int k,
                                                      uint8_t* __restrict__ send, int32_t* __restrict__ send_pos,
                                                      int* status) {
    pdl_trigger();
    pdl_wait();
    __shared__ int cum[kMaxExperts + 1];
    if (threadIdx.x == 0) {
        cum[0] = 0;
        for (int e = 0; e < E; ++e) cum[e + 1] = cum[e] + meta->counts[e];
    }
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const long long TK = (long long)T * k;
    const size_t nvec = row_bytes / 16;
    for (long long a = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); a < TK;
         a += (long long)gridDim.x * (blockDim.x >> 5)) {
        const int e = idx[a], r = inv[a];
        if (e < 0 || e >= E || r < 0) {   // dropped by the dispatch (its own check recorded the fault)
            if (lane == 0) send_pos[a] = -1;
            continue;
        }
        const int p = cum[e] + (r - meta->offsets[e]);
        if (!debug_check(p >= cum[e] && p < cum[e + 1], status)) continue;
        if (lane == 0) send_pos[a] = p;
        const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)(a / k) * row_bytes);
        uint4* dst = reinterpret_cast<uint4*>(send + (size_t)p * row_bytes);
        for (size_t v = lane; v < nvec; v += 32) dst[v] = __ldg(src + v);
    }
}

// One block of (source s, local expert l) per CTA: rows [recv0, recv0 + n) of the
// receive buffer <-> rows [seg0, seg0 + n) of the segments; TO_SEG picks the
// direction.  With TO_SEG, CTA index nblocks + l also zeroes segment l's padding.
template <bool TO_SEG>
__global__ void __launch_bounds__(256) ep_move_kernel(const uint8_t* __restrict__ src, uint8_t* __restrict__ dst,
                                                      size_t row_bytes, const int32_t* __restrict__ tab, int nblocks,
                                                      int EL) {
    pdl_trigger();
    pdl_wait();
    const int b = blockIdx.x;
    const size_t nvec = row_bytes / 16;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    if (b < nblocks) {
        const int recv0 = tab[3 * b], seg0 = tab[3 * b + 1], n = tab[3 * b + 2];
        for (int i = warp; i < n; i += nw) {
            const size_t from = (size_t)(TO_SEG ? recv0 + i : seg0 + i), to = (size_t)(TO_SEG ? seg0 + i : recv0 + i);
            const uint4* s = reinterpret_cast<const uint4*>(src + from * row_bytes);
            uint4* d = reinterpret_cast<uint4*>(dst + to * row_bytes);
            for (size_t v = lane; v < nvec; v += 32) d[v] = __ldg(s + v);
        }
    } else if (TO_SEG && b < nblocks + EL) {
        // padding rows of segment l: table entries after the blocks hold (pad0, pad1) per segment
        const int l = b - nblocks;
        const int pad0 = tab[3 * nblocks + 2 * l], pad1 = tab[3 * nblocks + 2 * l + 1];
        const uint4 z = make_uint4(0, 0, 0, 0);
        for (int r = pad0 + warp; r < pad1; r += nw) {
            uint4* d = reinterpret_cast<uint4*>(dst + (size_t)r * row_bytes);
            for (size_t v = lane; v < nvec; v += 32) d[v] = z;
        }
    }
}

}  // namespace

moe_status ep_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

}  // namespace moe

namespace moe {
int* status_word(int dev);   // moe_api.cu: the device status word (no allocation)
cudaMemPool_t library_pool(int dev);   // moe_api.cu: the library's stream-ordered pool (created on first use)
int device_sms(int dev);
long long pipeline_wait_ns();
}

extern "C" moe_status moe_ep_dispatch(const void* x, const int32_t* topk_idx, int T, int d, int E, int k,
                                      void* send, int32_t* send_pos, int32_t* counts_host, cudaStream_t stream) {
    if (T < 0 || d <= 0 || E <= 0 || k <= 0 || k > E) return MOE_ERR_INVALID_ARG;
    if (E > kMaxExperts) return MOE_ERR_UNSUPPORTED;
    if (d % 64 != 0) return MOE_ERR_UNSUPPORTED;
    if ((long long)T * k + (long long)E * kSegRows >= INT_MAX) return MOE_ERR_UNSUPPORTED;
    if (!counts_host) return MOE_ERR_INVALID_ARG;
    if (T == 0) {
        for (int e = 0; e < E; ++e) counts_host[e] = 0;
        return MOE_OK;
    }
    if (!x || !topk_idx || !send || !send_pos) return MOE_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(send)) & 15u) return MOE_ERR_INVALID_ARG;
    const DeviceScope scope(x, false);
    const int dev = scope.device();
    cudaMemPool_t pool = library_pool(dev);
    int* status = status_word(dev);
    if (!pool || !status) return MOE_ERR_CUDA;
    const size_t slots = slots_capacity(T, E, k);
    const size_t blk_bytes = align_up((size_t)dispatch_blocks(T) * E * 4 + 1, 256);
    const size_t meta_off = blk_bytes;
    const size_t perm_off = align_up(meta_off + sizeof(Meta), 256);
    const size_t inv_off = align_up(perm_off + slots * 4, 256);
    const size_t total = inv_off + (size_t)T * k * 4;
    void* scratch = nullptr;
    if (cudaMallocFromPoolAsync(&scratch, total, pool, stream) != cudaSuccess) return MOE_ERR_WORKSPACE;
    uint8_t* ws = static_cast<uint8_t*>(scratch);
    Meta* meta = reinterpret_cast<Meta*>(ws + meta_off);
    int32_t* perm = reinterpret_cast<int32_t*>(ws + perm_off);
    int32_t* inv = reinterpret_cast<int32_t*>(ws + inv_off);
    cudaError_t e = launch_dispatch(topk_idx, T, E, k, reinterpret_cast<int32_t*>(ws), meta, perm, inv, status, stream);
    const long long TK = (long long)T * k;
    long long blocks = (TK + 7) / 8;
    if (blocks > 148 * 16) blocks = 148 * 16;
    if (e == cudaSuccess)
        e = launch_pdl(ep_pack_kernel, dim3((unsigned)blocks), dim3(256), 0, stream,
                       static_cast<const uint8_t*>(x), (size_t)d * 2, topk_idx, inv, meta, T, E, k,
                       static_cast<uint8_t*>(send), send_pos, status);
    if (e == cudaSuccess) e = cudaMemcpyAsync(counts_host, meta->counts, E * 4, cudaMemcpyDeviceToHost, stream);
    cudaError_t f = cudaFreeAsync(scratch, stream);
    cudaError_t g = cudaStreamSynchronize(stream);   // the counts are needed on the host for the exchange
    return (e == cudaSuccess && f == cudaSuccess && g == cudaSuccess) ? MOE_OK : MOE_ERR_CUDA;
}

extern "C" moe_status moe_ep_experts(const void* recv, const int32_t* counts_all, int R, int E, int rank,
                                     const void* W1, const void* W3, const void* W2, int d, int ffn, float* yrecv,
                                     cudaStream_t stream) {
    if (!counts_all || R <= 0 || E <= 0 || rank < 0 || rank >= R || d <= 0 || ffn <= 0) return MOE_ERR_INVALID_ARG;
    if (E > kMaxExperts) return MOE_ERR_UNSUPPORTED;
    if (d % 64 != 0 || ffn % 128 != 0) return MOE_ERR_UNSUPPORTED;
    int32_t send_counts[64], send_offsets[65], recv_counts[64], recv_offsets[65], range[2];
    int32_t seg_counts[kMaxExperts], seg_offsets[kMaxExperts + 1];
    if (R > 64) return MOE_ERR_UNSUPPORTED;
    int32_t* block_recv = static_cast<int32_t*>(malloc(sizeof(int32_t) * (size_t)R * E));
    int32_t* block_seg = static_cast<int32_t*>(malloc(sizeof(int32_t) * (size_t)R * E));
    if (!block_recv || !block_seg) {
        free(block_recv);
        free(block_seg);
        return MOE_ERR_WORKSPACE;
    }
    moe_status st = moe_ep_plan(counts_all, R, E, rank, send_counts, send_offsets, recv_counts, recv_offsets, range,
                                seg_counts, seg_offsets, block_recv, block_seg);
    const int lo = range[0], EL = range[1] - range[0];
    const int rows = recv_offsets[R];
    if (st != MOE_OK || EL == 0 || rows == 0) {
        free(block_recv);
        free(block_seg);
        return st;
    }
    if (!recv || !W1 || !W3 || !W2 || !yrecv) {
        free(block_recv);
        free(block_seg);
        return MOE_ERR_INVALID_ARG;
    }
    // host tables: (recv0, seg0, n) per (source, local expert), then (pad0, pad1) per segment; and the segment table
    const int nblocks = R * EL;
    const size_t tab_n = 3 * (size_t)nblocks + 2 * (size_t)EL;
    int32_t* tab = static_cast<int32_t*>(malloc(sizeof(int32_t) * tab_n));
    if (!tab) {
        free(block_recv);
        free(block_seg);
        return MOE_ERR_WORKSPACE;
    }
    for (int s = 0; s < R; ++s)
        for (int l = 0; l < EL; ++l) {
            const int b = s * EL + l;
            tab[3 * b] = block_recv[b];
            tab[3 * b + 1] = block_seg[b];
            tab[3 * b + 2] = counts_all[(size_t)s * E + lo + l];
        }
    for (int l = 0; l < EL; ++l) {
        tab[3 * nblocks + 2 * l] = seg_offsets[l] + seg_counts[l];
        tab[3 * nblocks + 2 * l + 1] = seg_offsets[l + 1];
    }
    free(block_recv);
    free(block_seg);
    Meta hmeta = {};
    for (int l = 0; l < EL; ++l) hmeta.counts[l] = seg_counts[l];
    for (int l = 0; l <= EL; ++l) hmeta.offsets[l] = seg_offsets[l];
    const size_t S = (size_t)seg_offsets[EL];
    const DeviceScope scope(W1, false);
    const int dev = scope.device();
    cudaMemPool_t pool = library_pool(dev);
    int* status = status_word(dev);
    if (!pool || !status) {
        free(tab);
        return MOE_ERR_CUDA;
    }
    const size_t meta_off = 0;
    const size_t tab_off = align_up(sizeof(Meta), 256);
    const size_t xp_off = align_up(tab_off + tab_n * 4, 256);
    const size_t h_off = align_up(xp_off + S * d * 2, 256);
    const size_t y_off = align_up(h_off + S * (size_t)ffn * 2, 256);
    const size_t total = y_off + S * d * 4;
    void* scratch = nullptr;
    if (cudaMallocFromPoolAsync(&scratch, total, pool, stream) != cudaSuccess) {
        free(tab);
        return MOE_ERR_WORKSPACE;
    }
    uint8_t* ws = static_cast<uint8_t*>(scratch);
    Meta* meta = reinterpret_cast<Meta*>(ws + meta_off);
    int32_t* dtab = reinterpret_cast<int32_t*>(ws + tab_off);
    cudaError_t e = cudaMemcpyAsync(meta, &hmeta, sizeof(Meta), cudaMemcpyHostToDevice, stream);
    if (e == cudaSuccess) e = cudaMemcpyAsync(dtab, tab, tab_n * 4, cudaMemcpyHostToDevice, stream);
    // the copies above read pageable host memory: they have been staged when they return
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    free(tab);
    if (e == cudaSuccess)
        e = launch_pdl(ep_move_kernel<true>, dim3((unsigned)(nblocks + EL)), dim3(256), 0, stream,
                       static_cast<const uint8_t*>(recv), ws + xp_off, (size_t)d * 2,
                       static_cast<const int32_t*>(dtab), nblocks, EL);
    TcGemmArgs a{ws + xp_off, W1, W3, W2, ws + h_off, reinterpret_cast<float*>(ws + y_off), meta, EL, d, ffn, S,
                 device_sms(dev), status, pipeline_wait_ns()};
    if (e == cudaSuccess) e = launch_tc_gemm1(a, stream);
    if (e == cudaSuccess) e = launch_tc_gemm2(a, stream);
    if (e == cudaSuccess)
        e = launch_pdl(ep_move_kernel<false>, dim3((unsigned)nblocks), dim3(256), 0, stream,
                       static_cast<const uint8_t*>(ws + y_off), reinterpret_cast<uint8_t*>(yrecv), (size_t)d * 4,
                       static_cast<const int32_t*>(dtab), nblocks, EL);
    cudaError_t f = cudaFreeAsync(scratch, stream);
    return (e == cudaSuccess && f == cudaSuccess) ? MOE_OK : MOE_ERR_CUDA;
}

extern "C" moe_status moe_ep_combine(const float* ysend, const float* topk_w, const int32_t* send_pos, int T, int d,
                                     int k, void* out, cudaStream_t stream) {
    if (T < 0 || d <= 0 || k <= 0) return MOE_ERR_INVALID_ARG;
    if (d % 64 != 0) return MOE_ERR_UNSUPPORTED;
    if (T == 0) return MOE_OK;
    if (!ysend || !topk_w || !send_pos || !out) return MOE_ERR_INVALID_ARG;
    const DeviceScope scope(out, false);
    int* status = status_word(scope.device());
    if (!status) return MOE_ERR_CUDA;
    return ep_status(launch_combine_bf16(ysend, topk_w, send_pos, T, d, k, (size_t)T * k, status, out, stream));
}
