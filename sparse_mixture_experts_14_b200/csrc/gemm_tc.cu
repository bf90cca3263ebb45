// Tensor-core grouped GEMMs of the experts (bf16 in, fp32 accumulate in tensor
// memory), sm_100a: tcgen05.mma on CTA pairs, fed by TMA, accumulators in TMEM.
//
// Subsection "各エキスパートの構造" of the "Mistral/Mixtral architecture" page:
//     E_i(x) = W2_i (SiLU(W1_i x) * W3_i x)
// computed per expert over its expert-contiguous rows Xp_e (from dispatch):
//     GEMM1  acc = Xp_e [W1_e ; W3_e]^T,   H = SiLU(acc[:, :128]) * acc[:, 128:]  -> bf16
//     GEMM2  Y   = H_e W2_e^T                                              -> fp32
//
// A cluster of two CTAs (one SM pair) computes a 256 x 256 accumulator tile
// with tcgen05.mma.cta_group::2: each CTA holds 128 of the 256 rows (one
// 128-row m-tile of the expert) and 128 of the 256 B rows, so each SM moves
// 32 KiB of operands per 64-deep K step instead of 48 KiB for a 1-SM tile of
// the same per-SM work.  In GEMM1 the leader's B half is a 128-row block of
// W1_e and the peer's the same block of W3_e: the pair MMA gives each CTA
// both halves of the SwiGLU for its rows, and the gating runs in the epilogue
// straight out of TMEM.
//
// Persistent kernel, one CTA per SM, 6 warps per CTA:
//   warp 0     TMA producer (one thread per CTA): own A rows and own B half
//              into a 7-stage ring; completion bytes of both CTAs are counted
//              on the leader's barrier
//   warp 1     leader: MMA issuer (one thread); commits arrive on both CTAs'
//              barriers (multicast).  Both CTAs: TMEM owner (512 columns =
//              two 128 x 256 fp32 accumulators, so the epilogue of one tile
//              overlaps the MMAs of the next)
//   warps 2-5  epilogue of the CTA's own rows: tcgen05.ld of their 32-lane
//              quarter, gating / fp32 stores; then one arrival per warp on the
//              leader's "accumulator free" barrier
// Pair tiles are (expert, n-block, m-tile pair) with pairs fastest, so the
// CTAs at work share one block of expert weights through L2.  When an expert
// has an odd number of m-tiles, the peer of its last pair computes rows past
// the expert's segment and stores nothing.  The tile list is derived on the
// device from the dispatch offsets: no host synchronisation.
#include <cuda.h>

#include "moe_common.cuh"
#include "ptx_sm100.cuh"
#include "tma_map.cuh"

namespace moe {
namespace {

constexpr int BM = 128;                        // rows per CTA (256 per pair)
constexpr int BK = 64;                         // K per stage (one 128-byte swizzle row)
constexpr int BN = 256;                        // accumulator columns of the pair MMA
constexpr int BNH = BN / 2;                    // B rows held by each CTA
constexpr int STAGES = 7;
constexpr int A_BYTES = BM * BK * 2;           // 16 KiB
constexpr int B_BYTES = BNH * BK * 2;          // 16 KiB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr uint32_t PAIR_TX_BYTES = 2 * STAGE_BYTES;
constexpr int TMEM_COLS = 2 * BN;
constexpr int NUM_THREADS = 192;
constexpr int NUM_EPI_WARPS = 4;
constexpr uint32_t IDESC = ptx::idesc_bf16_f32(2 * BM, BN);

struct Ctrl {
    uint64_t full[STAGES];      // leader: both CTAs' bytes of a stage landed
    uint64_t empty[STAGES];     // each CTA: the pair MMAs reading a stage are done
    uint64_t tfull[2];          // each CTA: accumulator b holds a finished tile
    uint64_t tempty[2];         // leader: both CTAs' epilogues released accumulator b
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
    int total;
    int tile_base[kMaxExperts + 1];
    int mt[kMaxExperts];        // 128-row m-tiles of expert e
    int pt[kMaxExperts];        // pairs of m-tiles of expert e
    int row0[kMaxExperts];
};

constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + (int)sizeof(Ctrl) + 1024;

__device__ __forceinline__ void decode_tile(const Ctrl* c, int tile, int& e, int& pair, int& n_blk) {
    e = 0;
    while (tile >= c->tile_base[e + 1]) ++e;
    const int local = tile - c->tile_base[e];
    n_blk = local / c->pt[e];
    pair = local - n_blk * c->pt[e];
}

// Soft per-wave alignment of the clusters.  CTA pairs that share a block of
// expert weights run tiles of the same wave; if the clusters drift apart over
// many waves, a shared block leaves L2 between its first and last reader and
// is fetched from HBM again.  Each leader announces the start of its wave on a
// device counter and waits, for at most 20 us, until every cluster with a
// tile in that wave has announced it.  The wait is only a hint: on expiry the
// cluster goes on, so nothing can deadlock on it.
__device__ __forceinline__ void wave_sync(int* counter, int target) {
    atomicAdd(counter, 1);
    const uint64_t t0 = global_timer_ns();
    while (true) {
        int v;
        asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(counter) : "memory");
        if (v >= target || global_timer_ns() - t0 > 20000ull) break;
    }
}

// SWIGLU: GEMM1 (B halves = 128-row blocks of W1 and W3, out = H bf16 [slots][N]).
// !SWIGLU: GEMM2 (B halves = the two 128-row halves of a 256-row W2 block, out = Y fp32 [slots][N]).
template <bool SWIGLU>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB1,
                   const __grid_constant__ CUtensorMap mapB3, Meta* __restrict__ meta, int E, int K, int N,
                   size_t slots, void* __restrict__ out, int* status, long long wait_ns) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Ctrl* ctrl = reinterpret_cast<Ctrl*>(smem + STAGES * STAGE_BYTES);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = ptx::cluster_ctarank();
    const bool leader = rank == 0;
    const int cluster = blockIdx.x >> 1;
    const int nclusters = gridDim.x >> 1;
    constexpr int N_PER_TILE = SWIGLU ? BNH : BN;   // output columns per tile

    pdl_trigger();
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            ptx::mbar_init(&ctrl->full[s], 1);
            ptx::mbar_init(&ctrl->empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(&ctrl->tfull[b], 1);
            ptx::mbar_init(&ctrl->tempty[b], 2 * NUM_EPI_WARPS);
        }
        ptx::mbar_init(&ctrl->drain, 1);
        ctrl->abort = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        ptx::tma_prefetch_desc(&mapA);
        ptx::tma_prefetch_desc(&mapB1);
        if (SWIGLU) ptx::tma_prefetch_desc(&mapB3);
    }
    if (warp == 1) {
        ptx::tmem_alloc_pair(&ctrl->tmem_base, TMEM_COLS);
        ptx::tmem_relinquish_pair();
    }
    // everything above overlaps the previous kernel; global memory only after this
    pdl_wait();
    if (threadIdx.x == 0) {
        const int ntn = (N + N_PER_TILE - 1) / N_PER_TILE;
        ctrl->tile_base[0] = 0;
        bool ok = true;
        for (int e = 0; e < E; ++e) {
            const int r0 = meta->offsets[e], r1 = meta->offsets[e + 1];
            if (r1 < r0 || (r1 - r0) % BM != 0 || (size_t)r1 > slots) ok = false;
            const int mt = ok ? (r1 - r0) / BM : 0;
            ctrl->mt[e] = mt;
            ctrl->pt[e] = (mt + 1) / 2;
            ctrl->row0[e] = r0;
            ctrl->tile_base[e + 1] = ctrl->tile_base[e] + ctrl->pt[e] * ntn;
        }
        ctrl->total = ok ? ctrl->tile_base[E] : 0;
        if (!ok) record_status(status, MOE_ERR_DEVICE);
    }
    ptx::tc_fence_before_sync();
    ptx::cluster_sync();
    ptx::tc_fence_after_sync();

    const uint32_t tmem_base = ctrl->tmem_base;
    const int total = ctrl->total;
    const int nk = (K + BK - 1) / BK;
    const ptx::WaitCtl wc{&ctrl->abort, status, (uint64_t)wait_ns};

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA producer (both CTAs)
        if (lane == 0) {
            const uint64_t pol = ptx::policy_evict_normal();
            int stage = 0;
            uint32_t phase = 0;
            bool armed[STAGES];
            uint32_t armed_phase[STAGES];
#pragma unroll
            for (int s = 0; s < STAGES; ++s) {
                armed[s] = false;
                armed_phase[s] = 0;
            }
            bool aborted = false;
            int wave = 0;
            for (int tile = cluster; tile < total && !aborted; tile += nclusters, ++wave) {
                int e, pair, n_blk;
                decode_tile(ctrl, tile, e, pair, n_blk);
                const int rowA = ctrl->row0[e] + (2 * pair + (int)rank) * BM;
                if (leader) wave_sync(&meta->waves[SWIGLU ? 0 : 1], min(total, (wave + 1) * nclusters));
                const CUtensorMap* mapB = (SWIGLU && !leader) ? &mapB3 : &mapB1;
                const int rowB = SWIGLU ? n_blk * BNH : n_blk * BN + (int)rank * BNH;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!ptx::mbar_wait(&ctrl->empty[stage], phase ^ 1u, wc)) {
                        aborted = true;
                        break;
                    }
                    uint8_t* sa = smem + stage * STAGE_BYTES;
                    uint8_t* sb = sa + A_BYTES;
                    const uint32_t full_leader = ptx::map_to_rank(ptx::smem_addr(&ctrl->full[stage]), 0);
                    if (leader) ptx::mbar_arrive_expect_tx(&ctrl->full[stage], PAIR_TX_BYTES);
                    ptx::tma_load_2d_pair(sa, &mapA, full_leader, kb * BK, rowA, pol);
                    ptx::tma_load_3d_pair(sb, mapB, full_leader, kb * BK, rowB, e, pol);
#pragma unroll
                    for (int s = 0; s < STAGES; ++s)
                        if (s == stage) {
                            armed[s] = true;
                            armed_phase[s] = phase;
                        }
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (leader && (aborted || ctrl->abort)) {
                // let copies still in flight land before shared memory is released
#pragma unroll
                for (int s = 0; s < STAGES; ++s)
                    if (armed[s]) ptx::mbar_wait_drain(&ctrl->full[s], armed_phase[s], 100000000ull);
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer (leader)
        if (lane == 0 && leader) {
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool issued = false, aborted = false;
            for (int tile = cluster; tile < total && !aborted; tile += nclusters) {
                if (!ptx::mbar_wait(&ctrl->tempty[acc], acc_phase ^ 1u, wc)) {
                    aborted = true;
                    break;
                }
                ptx::tc_fence_after_sync();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
                for (int kb = 0; kb < nk; ++kb) {
                    if (!ptx::mbar_wait(&ctrl->full[stage], phase, wc)) {
                        aborted = true;
                        break;
                    }
                    ptx::tc_fence_after_sync();
                    const uint32_t a0 = ptx::smem_addr(smem + stage * STAGE_BYTES);
                    const uint32_t b0 = a0 + A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        ptx::tc_mma_bf16_pair(d_tmem, ptx::desc_kmajor_sw128(a0 + kk * 32),
                                              ptx::desc_kmajor_sw128(b0 + kk * 32), IDESC, (kb | kk) != 0);
                    }
                    ptx::tc_commit_pair_multicast(&ctrl->empty[stage], 0x3);
                    issued = true;
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (aborted) break;
                ptx::tc_commit_pair_multicast(&ctrl->tfull[acc], 0x3);
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1u;
            }
            if ((aborted || ctrl->abort) && issued) {
                ptx::tc_commit_pair(&ctrl->drain);
                ptx::mbar_wait_drain(&ctrl->drain, 0, 100000000ull);
            }
        }
    } else {
        // ---------------------------------------------------------------- epilogue (both CTAs)
        const int q = warp & 3;   // TMEM lane quarter this warp may access
        const uint64_t pol_out = ptx::policy_evict_first();
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = cluster; tile < total; tile += nclusters) {
            int e, pair, n_blk;
            decode_tile(ctrl, tile, e, pair, n_blk);
            const int m_tile = 2 * pair + (int)rank;
            bool ok = ptx::mbar_wait(&ctrl->tfull[acc], acc_phase, wc);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            ptx::tc_fence_after_sync();
            if (m_tile < ctrl->mt[e]) {
                const size_t row = (size_t)ctrl->row0[e] + (size_t)m_tile * BM + q * 32 + lane;
                const uint32_t taddr = tmem_base + (uint32_t)(acc * BN) + ((uint32_t)(q * 32) << 16);
                if (SWIGLU) {
                    __nv_bfloat16* H = static_cast<__nv_bfloat16*>(out);
#pragma unroll 1
                    for (int c = 0; c < BNH; c += 32) {
                        uint32_t ra[32], rb[32];
                        ptx::tmem_ld_32x32b_x32(taddr + c, ra);
                        ptx::tmem_ld_32x32b_x32(taddr + BNH + c, rb);
                        ptx::tmem_ld_wait();
                        uint32_t hp[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const float h0 = silu_mul(__uint_as_float(ra[2 * i]), __uint_as_float(rb[2 * i]));
                            const float h1 = silu_mul(__uint_as_float(ra[2 * i + 1]), __uint_as_float(rb[2 * i + 1]));
                            hp[i] = pack_bf16x2(h0, h1);
                        }
                        uint8_t* dst = reinterpret_cast<uint8_t*>(H + row * (size_t)N + n_blk * BNH + c);
#pragma unroll
                        for (int v = 0; v < 4; ++v)
                            ptx::st_global_v4_hint(dst + 16 * v, hp[4 * v], hp[4 * v + 1], hp[4 * v + 2], hp[4 * v + 3],
                                                   pol_out);
                    }
                } else {
                    float* Y = static_cast<float*>(out);
#pragma unroll 1
                    for (int c = 0; c < BN; c += 32) {
                        uint32_t r[32];
                        ptx::tmem_ld_32x32b_x32(taddr + c, r);
                        ptx::tmem_ld_wait();
                        const int col = n_blk * BN + c;
                        if (col < N) {
                            uint8_t* dst = reinterpret_cast<uint8_t*>(Y + row * (size_t)N + col);
#pragma unroll
                            for (int v = 0; v < 8; ++v)
                                ptx::st_global_v4_hint(dst + 16 * v, r[4 * v], r[4 * v + 1], r[4 * v + 2], r[4 * v + 3],
                                                       pol_out);
                        }
                    }
                }
            }
            ptx::tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive_cluster(ptx::map_to_rank(ptx::smem_addr(&ctrl->tempty[acc]), 0));
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1u;
        }
    }

    ptx::tc_fence_before_sync();
    __syncwarp();
    ptx::cluster_sync();
    if (warp == 1) {
        ptx::tc_fence_after_sync();
        ptx::tmem_dealloc_pair(tmem_base, TMEM_COLS);
    }
}

// ---------------------------------------------------------------- host side

// rows x K matrix, K contiguous: box 64 x box_rows
bool map_rows(CUtensorMap* m, const void* base, size_t rows, int K, int box_rows) {
    return map_matrix(m, base, rows, K, BK, box_rows);
}

// E x R x K weights, K contiguous: box 64 x box_rows x 1
bool map_weights(CUtensorMap* m, const void* base, int E, int R, int K, int box_rows) {
    return map_expert_weights(m, base, E, R, K, BK, box_rows);
}

template <bool SWIGLU>
cudaError_t ensure_smem_attr() {
    static PerDeviceOnce once;
    return once.run([] {
        return cudaFuncSetAttribute(tc_gemm_kernel<SWIGLU>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    });
}

// Persistent grid: as many CTA pairs as fit at once, no more than there are pair tiles.
template <bool SWIGLU>
int grid_for(size_t slots, int n_tiles_per_m, int num_sms) {
    static PerDeviceInt clusters_per_device;
    const int max_clusters = clusters_per_device.get([num_sms] {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * 74, 1, 1);
        cfg.blockDim = dim3(NUM_THREADS, 1, 1);
        cfg.dynamicSmemBytes = SMEM_BYTES;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, tc_gemm_kernel<SWIGLU>, &cfg) != cudaSuccess || n <= 0) {
            cudaGetLastError();
            n = (num_sms > 0 ? num_sms : 148) / 2;
        }
        return n;
    });
    const size_t pair_rows = (slots / BM + 1) / 2;
    const size_t upper = pair_rows * (size_t)n_tiles_per_m;
    size_t clusters = (size_t)max_clusters;
    if (clusters > upper) clusters = upper;
    if (clusters < 1) clusters = 1;
    return (int)(2 * clusters);
}

template <bool SWIGLU>
cudaError_t launch_pair(int grid, const CUtensorMap& mA, const CUtensorMap& mB1, const CUtensorMap& mB3,
                        const TcGemmArgs& a, int K, int N, void* out, cudaStream_t s) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(NUM_THREADS, 1, 1);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, tc_gemm_kernel<SWIGLU>, mA, mB1, mB3, const_cast<Meta*>(a.meta), a.E, K, N,
                              a.slots, out, a.status, a.wait_ns);
}

}  // namespace

cudaError_t launch_tc_gemm1(const TcGemmArgs& a, cudaStream_t s) {
    CUtensorMap mA, mB1, mB3;
    if (!map_rows(&mA, a.xp, a.slots, a.d, BM) || !map_weights(&mB1, a.W1, a.E, a.F, a.d, BNH) ||
        !map_weights(&mB3, a.W3, a.E, a.F, a.d, BNH))
        return cudaErrorInvalidValue;
    cudaError_t e = ensure_smem_attr<true>();
    if (e != cudaSuccess) return e;
    const int grid = grid_for<true>(a.slots, (a.F + BNH - 1) / BNH, a.num_sms);
    e = launch_pair<true>(grid, mA, mB1, mB3, a, a.d, a.F, a.H, s);
    return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_tc_gemm2(const TcGemmArgs& a, cudaStream_t s) {
    CUtensorMap mA, mB;
    if (!map_rows(&mA, a.H, a.slots, a.F, BM) || !map_weights(&mB, a.W2, a.E, a.d, a.F, BNH))
        return cudaErrorInvalidValue;
    cudaError_t e = ensure_smem_attr<false>();
    if (e != cudaSuccess) return e;
    const int grid = grid_for<false>(a.slots, (a.d + BN - 1) / BN, a.num_sms);
    e = launch_pair<false>(grid, mA, mB, mB, a, a.F, a.d, a.Y, s);
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace moe
