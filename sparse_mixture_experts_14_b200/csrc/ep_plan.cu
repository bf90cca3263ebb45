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
