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
// Wide tiles (the forward GEMMs when K >= 5120): 256 x 512, each CTA holding
// 256 B rows and issuing two N = 256 MMAs per K = 16 slice on one A stage, a
// 4-stage ring of 48 KiB, one accumulator in all 512 TMEM columns and 8
// epilogue warps (one per lane quarter and accumulator half).
// Pair tiles are (expert, n-block, m-tile pair) with pairs fastest, so the
// CTAs at work share one block of expert weights through L2.  When an expert
// has an odd number of m-tiles, the peer of its last pair computes rows past
// the expert's segment and stores nothing.  The tile list is derived on the
// device from the dispatch offsets: no host synchronisation.
//
// The same kernel runs the layer's backward GEMMs (gradients of the expert
// equations, the training the page's "ロードバランス損失" subsection closes with):
//     dH    = dY_e W2_e                  W2 read MN-major (no transpose); the
//                                        epilogue turns dH into dA, dB with the
//                                        a = Xp W1^T, b = Xp W3^T that the training
//                                        forward's GEMM1 epilogue kept (fp32)
//     dXp   = dA_e W1_e + dB_e W3_e      W1 / W3 read MN-major, K = 2F
//     dW2_e = dY_e^T H_e                 both operands MN-major, K = the
//     dW1_e|dW3_e = [dA dB]_e^T Xp_e     expert's rows (grouped by K)
// MN-major tiles come in as two 64-wide TMA boxes (128-byte swizzle) and are
// described to tcgen05.mma as MN-major, so no operand is ever transposed in HBM.
#include <cuda.h>

#include <cstdlib>

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
constexpr int TMEM_COLS = 2 * BN;
constexpr int NUM_EPI_WARPS = 4;                 // epilogue warps of the row-grouped modes (one per lane quarter)
constexpr int MN_BOX = 64;                     // MN-major operands: two 64-wide boxes per 128 rows
constexpr uint32_t MN_LBO = MN_BOX * BK * 2;   // bytes between the two boxes (atoms along M/N)
constexpr uint32_t MN_SBO = 1024;              // bytes between 8-row groups along K
constexpr int OUT_PITCH = 32;                  // floats per staged 32 x 32 chunk row (8 float4 slots, swizzled)

// What one instantiation computes.
enum : int {
    kFwd1 = 0,       // H = SiLU(Xp W1^T) * (Xp W3^T)              -> bf16 [slots][N]
    kFwd2 = 1,       // C = A B_e^T, B K-major                     -> fp32 [slots][N]
    kFwd1Train = 2,  // kFwd1, and a = Xp W1^T, b = Xp W3^T kept    -> + fp32 [slots][N] x 2
    kDgradH = 3,     // dH = dY W2_e (W2 MN-major), SwiGLU backward -> dA | dB bf16 [slots][2N]
    kDgradX = 4,     // dXp = dA W1_e + dB W3_e (MN-major, K = 2F)   -> fp32 [slots][N]
    kWgrad = 5,      // dW_e = A_e^T B_e over the expert's rows       -> fp32 [E][M][N]
    kWgrad16 = 6,    // kWgrad rounded once to bf16                   -> bf16 [E][M][N]
    kFwd1W = 7,      // kFwd1 on 256 x 512 tiles (two N = 256 MMAs per A stage)
    kFwd2W = 8,      // kFwd2 on 256 x 512 tiles
    kDgradXW = 9,    // kDgradX on 256 x 512 tiles
};



// Scalar arguments of one launch.
struct GemmParams {
    Meta* meta;
    int E;
    int M;           // kWgrad: output rows per expert
    int N;           // output columns (kDgradH: F; its output rows hold dA | dB, 2N)
    int K;           // reduction length of the row-grouped modes
    int split;       // kWgrad: output rows m >= split go to out_hi, row m - split
    int kb_split;    // kDgradX: K blocks from mapB3 start here
    int wave_slot;
    size_t slots;
    void* out;
    void* out_hi;
    float* keep_a;      // kFwd1Train: a and b [slots][N] fp32
    float* keep_b;
    const float* aux_a; // kDgradH: the kept a and b [slots][N] fp32
    const float* aux_b;
    int* status;
    long long wait_ns;
};

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
    int row0[kMaxExperts];      // first row of expert e's segment
    int nkb[kMaxExperts];       // K blocks of expert e (grouped-by-K tiles)
    int ntn;                    // n-blocks per expert
    int n_fast;                 // tile order (decode_tile)
};

template <int MODE>
struct ModeT {
    // Wide tiles: the pair tile is 256 x 512, two N = 256 MMAs per K = 16 slice on one A stage,
    // so each CTA moves 48 KiB per 64-deep K step for twice the work of a 32 KiB step (a quarter
    // fewer operand bytes per MMA).  The accumulator takes all 512 TMEM columns (one buffer: the
    // epilogue of a tile is not overlapped with the next tile's MMAs, so it gets two warps per
    // TMEM lane quarter, one per 256-column half) and the ring has 4 stages.
    static constexpr bool WIDE = MODE == kFwd1W || MODE == kFwd2W || MODE == kDgradXW;
    static constexpr int BASE = MODE == kFwd1W    ? kFwd1
                                : MODE == kFwd2W  ? kFwd2
                                : MODE == kDgradXW ? kDgradX
                                                   : MODE;   // what it computes
    static constexpr int NW = WIDE ? 2 : 1;             // N = 256 MMAs per K = 16 slice
    static constexpr int ACCS = WIDE ? 1 : 2;           // accumulator buffers in the 512 TMEM columns
    static constexpr int B_ROWS = NW * BNH;             // B rows each CTA holds per stage
    static constexpr int STAGE_B = B_ROWS * BK * 2;
    static constexpr int STAGE = A_BYTES + STAGE_B;     // bytes per stage per CTA
    static constexpr uint32_t PAIR_TX = 2u * STAGE;
    static constexpr bool GATED = BASE == kFwd1 || BASE == kFwd1Train;   // B halves = W1 / W3 blocks
    static constexpr bool A_MN = MODE == kWgrad || MODE == kWgrad16;
    static constexpr bool B_MN = MODE == kDgradH || BASE == kDgradX || MODE == kWgrad || MODE == kWgrad16;
    static constexpr bool KGROUP = MODE == kWgrad || MODE == kWgrad16;   // tiles grouped by K, not by rows
    static constexpr bool OUT16 = MODE == kWgrad16;
    static constexpr int N_PER_TILE = GATED ? NW * BNH : NW * BN;
    static constexpr uint32_t IDESC = ptx::idesc_bf16_f32(2 * BM, BN, A_MN, B_MN);
    // An epilogue lane owns one accumulator row, so a lane's 16-byte global access touches
    // its own 128-byte line and a warp instruction 32 lines.  Epilogues that move several
    // times the output tile's bytes pass their fp32 chunks (32 rows x 32 columns) through
    // shared memory instead, and global memory sees 128-byte row segments (8 lanes each):
    //  * grouped-by-K tiles (K = one expert's rows, so short tiles): the fp32 gradient;
    //    they also get two epilogue warps per TMEM lane quarter, each taking half the columns;
    //  * the training forward's kept a, b (written) and the SwiGLU backward's (read), with
    //    the backward's dA | dB written the same way.
    // The space comes from the ring, which gives up one stage: each warp's 32 x 32 fp32 chunk
    // (4 KiB, two of them in the SwiGLU modes) is stored unpadded with its 16-byte slots
    // XOR-swizzled by row (stage_slot), so both the row-per-lane and the 8-lanes-per-row
    // accesses run at one 128-byte wavefront per 8 lanes without padding.
    static constexpr bool STAGED_OUT = KGROUP;
    static constexpr bool STAGED_AB = MODE == kFwd1Train || MODE == kDgradH;
    static constexpr int EPI_WARPS = STAGED_OUT || WIDE ? 2 * NUM_EPI_WARPS : NUM_EPI_WARPS;
    static constexpr int THREADS = 32 * (2 + EPI_WARPS);
    static constexpr int STAGES_M = WIDE ? 4 : STAGED_OUT || STAGED_AB ? STAGES - 1 : STAGES;
    static constexpr int STAGE_OUT_BYTES = (STAGED_OUT ? 1 : STAGED_AB ? 2 : 0) * EPI_WARPS * 32 * OUT_PITCH * 4;
    static constexpr int SMEM = STAGES_M * STAGE + STAGE_OUT_BYTES + (int)sizeof(Ctrl) + 1024;
};


// Tile order inside an expert: m-tile pairs fastest (the CTAs at work share one
// block of B), or with n_fast the n-blocks fastest (they share one block of A;
// for gradients whose A operand is the large one).
__device__ __forceinline__ void decode_tile(const Ctrl* c, int tile, int& e, int& pair, int& n_blk) {
    e = 0;
    while (tile >= c->tile_base[e + 1]) ++e;
    const int local = tile - c->tile_base[e];
    if (c->n_fast) {
        pair = local / c->ntn;
        n_blk = local - pair * c->ntn;
    } else {
        n_blk = local / c->pt[e];
        pair = local - n_blk * c->pt[e];
    }
}

// Float4 slot j (0..7) of row r of a staged 32 x 32 fp32 chunk: rows are 128 bytes with no
// padding and the slots of row r are permuted by j ^ (r & 7), so that 8 lanes writing slot j of
// 8 consecutive rows, or 8 lanes reading the 8 slots of one row, touch 8 different bank groups.
__device__ __forceinline__ float* stage_slot(float* buf, int r, int j) {
    return buf + r * OUT_PITCH + 4 * (j ^ (r & 7));
}

// Soft per-wave alignment of the clusters.  CTA pairs that share a block of
// expert weights run tiles of the same wave; if the clusters drift apart over
// many waves, a shared block leaves L2 between its first and last reader and
// is fetched from HBM again.  Each leader announces the start of its wave on a
// device counter and waits, for at most 50 us, until every cluster with a
// tile in that wave has announced it.  The wait is only a hint: on expiry the
// cluster goes on, so nothing can deadlock on it.  (At the 8x22B shape a 50 us
// limit measured 1.4% faster per layer than 20 us; 8 us was slower, 100 us no better.)
__device__ __forceinline__ void wave_sync(int* counter, int target) {
    atomicAdd(counter, 1);
    const uint64_t t0 = global_timer_ns();
    while (true) {
        int v;
        asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(counter) : "memory");
        if (v >= target || global_timer_ns() - t0 > 50000ull) break;
    }
}

template <int MODE>
__global__ void __launch_bounds__(ModeT<MODE>::THREADS, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB1,
                   const __grid_constant__ CUtensorMap mapB3, const GemmParams p) {
    using MT = ModeT<MODE>;
    constexpr int NST = MT::STAGES_M;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float* stage_out = reinterpret_cast<float*>(smem + NST * MT::STAGE);
    Ctrl* ctrl = reinterpret_cast<Ctrl*>(smem + NST * MT::STAGE + MT::STAGE_OUT_BYTES);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = ptx::cluster_ctarank();
    const bool leader = rank == 0;
    const int cluster = blockIdx.x >> 1;
    const int nclusters = gridDim.x >> 1;
    constexpr int N_PER_TILE = MT::N_PER_TILE;   // output columns per tile
    Meta* meta = p.meta;
    const int E = p.E, N = p.N;

    pdl_trigger();
    if (threadIdx.x == 0) {
        for (int s = 0; s < NST; ++s) {
            ptx::mbar_init(&ctrl->full[s], 1);
            ptx::mbar_init(&ctrl->empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(&ctrl->tfull[b], 1);
            ptx::mbar_init(&ctrl->tempty[b], 2 * MT::EPI_WARPS);
        }
        ptx::mbar_init(&ctrl->drain, 1);
        ctrl->abort = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        ptx::tma_prefetch_desc(&mapA);
        ptx::tma_prefetch_desc(&mapB1);
        if (MT::GATED || MT::BASE == kDgradX) ptx::tma_prefetch_desc(&mapB3);
    }
    if (warp == 1) {
        ptx::tmem_alloc_pair(&ctrl->tmem_base, TMEM_COLS);
        ptx::tmem_relinquish_pair();
    }
    // everything above overlaps the previous kernel; global memory only after this
    pdl_wait();
    if (threadIdx.x == 0) {
        const int ntn = (N + N_PER_TILE - 1) / N_PER_TILE;
        ctrl->ntn = ntn;
        ctrl->n_fast = MT::KGROUP && p.M > N;
        ctrl->tile_base[0] = 0;
        bool ok = true;
        for (int e = 0; e < E; ++e) {
            const int r0 = meta->offsets[e], r1 = meta->offsets[e + 1];
            if (r1 < r0 || (r1 - r0) % BM != 0 || (size_t)r1 > p.slots) ok = false;
            const int rows = ok ? r1 - r0 : 0;
            if (MT::KGROUP) {
                // every expert has the same output tiles; K = its rows (zero rows: zero gradient)
                const int mt = (p.M + BM - 1) / BM;
                ctrl->mt[e] = mt;
                ctrl->pt[e] = (mt + 1) / 2;
                ctrl->nkb[e] = rows / BK;
            } else {
                const int mt = rows / BM;
                ctrl->mt[e] = mt;
                ctrl->pt[e] = (mt + 1) / 2;
                ctrl->nkb[e] = (p.K + BK - 1) / BK;
            }
            ctrl->row0[e] = r0;
            ctrl->tile_base[e + 1] = ctrl->tile_base[e] + ctrl->pt[e] * ntn;
        }
        ctrl->total = ok ? ctrl->tile_base[E] : 0;
        if (!ok) record_status(p.status, MOE_ERR_DEVICE);
    }
    ptx::tc_fence_before_sync();
    ptx::cluster_sync();
    ptx::tc_fence_after_sync();

    const uint32_t tmem_base = ctrl->tmem_base;
    const int total = ctrl->total;
    const ptx::WaitCtl wc{&ctrl->abort, p.status, (uint64_t)p.wait_ns};

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA producer (both CTAs)
        if (lane == 0) {
            const uint64_t pol = ptx::policy_evict_normal();
            // GEMM1: an expert's gathered rows (A) are read once per n-block, its W1 / W3 blocks (B)
            // once per wave.  When the rows outgrow what L2 keeps across waves (workload 5: 50 MB
            // of rows per expert), streaming weights pushed them out and every wave read them
            // from HBM again (11.6 GB per launch for 4.7 GB of operands).  Weights evict-first,
            // rows evict-last: 5.6 GB, and GEMM1 4-6% faster at T >= 8192, neutral at T = 4096.
            const uint64_t polA = MT::GATED ? ptx::policy_evict_last() : pol;
            const uint64_t polB = MT::GATED ? ptx::policy_evict_first() : pol;
            int stage = 0;
            uint32_t phase = 0;
            bool armed[NST];
            uint32_t armed_phase[NST];
#pragma unroll
            for (int s = 0; s < NST; ++s) {
                armed[s] = false;
                armed_phase[s] = 0;
            }
            bool aborted = false;
            int wave = 0;
            for (int tile = cluster; tile < total && !aborted; tile += nclusters, ++wave) {
                int e, pair, n_blk;
                decode_tile(ctrl, tile, e, pair, n_blk);
                const int m_tile = 2 * pair + (int)rank;
                const int rowA = ctrl->row0[e] + m_tile * BM;            // row-grouped: A rows
                // this CTA's B rows (non-gated): for MMA h, rows n_blk * NW * BN + h * BN + rank * BNH
                const int n0 = n_blk * MT::NW * BN + (int)rank * BNH;
                const int nkb = ctrl->nkb[e];
                // grouped-by-K tiles are short and their operand blocks stay in L2 across a few
                // waves of drift: no alignment (it would hold every cluster to the slowest tile)
                if (leader && !MT::KGROUP) wave_sync(&meta->waves[p.wave_slot], min(total, (wave + 1) * nclusters));
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!ptx::mbar_wait(&ctrl->empty[stage], phase ^ 1u, wc)) {
                        aborted = true;
                        break;
                    }
                    uint8_t* sa = smem + stage * MT::STAGE;
                    uint8_t* sb = sa + A_BYTES;
                    const uint32_t full_leader = ptx::map_to_rank(ptx::smem_addr(&ctrl->full[stage]), 0);
                    if (leader) ptx::mbar_arrive_expect_tx(&ctrl->full[stage], MT::PAIR_TX);
                    if (MT::KGROUP) {
                        // A^T and B^T tiles of the expert's rows: [64 k][64 m] boxes, m / n contiguous
                        const int krow = ctrl->row0[e] + kb * BK;
                        const int m0 = m_tile * BM;
                        ptx::tma_load_2d_pair(sa, &mapA, full_leader, m0, krow, pol);
                        ptx::tma_load_2d_pair(sa + MN_LBO, &mapA, full_leader, m0 + MN_BOX, krow, pol);
                        ptx::tma_load_2d_pair(sb, &mapB1, full_leader, n0, krow, pol);
                        ptx::tma_load_2d_pair(sb + MN_LBO, &mapB1, full_leader, n0 + MN_BOX, krow, pol);
                    } else {
                        ptx::tma_load_2d_pair(sa, &mapA, full_leader, kb * BK, rowA, polA);
                        if (MT::B_MN) {
                            // weights [E][K][N], N contiguous: [64 k][64 n] boxes
                            const bool hi = MT::BASE == kDgradX && kb >= p.kb_split;
                            const CUtensorMap* mapB = hi ? &mapB3 : &mapB1;
                            const int kk = (hi ? kb - p.kb_split : kb) * BK;
#pragma unroll
                            for (int h = 0; h < MT::NW; ++h) {
                                ptx::tma_load_3d_pair(sb + h * B_BYTES, mapB, full_leader, n0 + h * BN, kk, e, pol);
                                ptx::tma_load_3d_pair(sb + h * B_BYTES + MN_LBO, mapB, full_leader, n0 + h * BN + MN_BOX,
                                                      kk, e, pol);
                            }
                        } else {
                            // 128-row blocks h = 0 .. NW-1 of this CTA's B rows (gated: features
                            // n_blk * NW * 128 + h * 128 of W1 in the leader, of W3 in the peer)
                            const CUtensorMap* mapB = (MT::GATED && !leader) ? &mapB3 : &mapB1;
#pragma unroll
                            for (int h = 0; h < MT::NW; ++h) {
                                const int rowB = MT::GATED ? (n_blk * MT::NW + h) * BNH : n0 + h * BN;
                                ptx::tma_load_3d_pair(sb + h * B_BYTES, mapB, full_leader, kb * BK, rowB, e, polB);
                            }
                        }
                    }
#pragma unroll
                    for (int s = 0; s < NST; ++s)
                        if (s == stage) {
                            armed[s] = true;
                            armed_phase[s] = phase;
                        }
                    if (++stage == NST) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (leader && (aborted || ctrl->abort)) {
                // let copies still in flight land before shared memory is released
#pragma unroll
                for (int s = 0; s < NST; ++s)
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
                int e, pair, n_blk;
                decode_tile(ctrl, tile, e, pair, n_blk);
                const int nkb = ctrl->nkb[e];
                if (!ptx::mbar_wait(&ctrl->tempty[acc], acc_phase ^ 1u, wc)) {
                    aborted = true;
                    break;
                }
                ptx::tc_fence_after_sync();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!ptx::mbar_wait(&ctrl->full[stage], phase, wc)) {
                        aborted = true;
                        break;
                    }
                    ptx::tc_fence_after_sync();
                    const uint32_t a0 = ptx::smem_addr(smem + stage * MT::STAGE);
                    const uint32_t b0 = a0 + A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        // one K = 16 slice: 32 bytes into each K-major row, or 16 rows of an MN-major tile
                        const uint64_t da = MT::A_MN ? ptx::desc_mnmajor_sw128(a0 + kk * 2048, MN_LBO, MN_SBO)
                                                     : ptx::desc_kmajor_sw128(a0 + kk * 32);
                        const uint64_t db = MT::B_MN ? ptx::desc_mnmajor_sw128(b0 + kk * 2048, MN_LBO, MN_SBO)
                                                     : ptx::desc_kmajor_sw128(b0 + kk * 32);
                        ptx::tc_mma_bf16_pair(d_tmem, da, db, MT::IDESC, (kb | kk) != 0);
                        if (MT::WIDE) {   // B rows 128-255 of each CTA: accumulator columns 256-511
                            const uint64_t db2 = MT::B_MN
                                                     ? ptx::desc_mnmajor_sw128(b0 + B_BYTES + kk * 2048, MN_LBO, MN_SBO)
                                                     : ptx::desc_kmajor_sw128(b0 + B_BYTES + kk * 32);
                            ptx::tc_mma_bf16_pair(d_tmem + BN, da, db2, MT::IDESC, (kb | kk) != 0);
                        }
                    }
                    ptx::tc_commit_pair_multicast(&ctrl->empty[stage], 0x3);
                    issued = true;
                    if (++stage == NST) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (aborted) break;
                ptx::tc_commit_pair_multicast(&ctrl->tfull[acc], 0x3);
                if (++acc == MT::ACCS) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
            }
            if ((aborted || ctrl->abort) && issued) {
                ptx::tc_commit_pair(&ctrl->drain);
                ptx::mbar_wait_drain(&ctrl->drain, 0, 100000000ull);
            }
        }
    } else {
        // ---------------------------------------------------------------- epilogue (both CTAs)
        const int q = warp & 3;   // TMEM lane quarter this warp may access
        const int ew = warp - 2;  // epilogue warp index; with 8 of them, ew / 4 picks a column half
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
            const bool live = MT::KGROUP ? m_tile * BM < p.M : m_tile < ctrl->mt[e];
            if (live) {
                const uint32_t taddr = tmem_base + (uint32_t)(acc * BN) + ((uint32_t)(q * 32) << 16);
                constexpr int HALVES = MT::EPI_WARPS / NUM_EPI_WARPS;   // warps per TMEM lane quarter
                const int half = ew / NUM_EPI_WARPS;
                if (MT::BASE == kFwd1 || MODE == kFwd1Train) {
                    const size_t row = (size_t)ctrl->row0[e] + (size_t)m_tile * BM + q * 32 + lane;
                    __nv_bfloat16* H = static_cast<__nv_bfloat16*>(p.out);
                    // (wide tiles: warp half h takes accumulator half h; otherwise one warp, every column)
                    // accumulator columns h * 256 + [0, 128) / [128, 256) hold W1 / W3 of features
                    // (n_blk * NW + h) * 128 + [0, 128) (h = 0 unless the tile is wide)
#pragma unroll 1
                    for (int ch = half * (MT::NW * BNH / HALVES); ch < (half + 1) * (MT::NW * BNH / HALVES); ch += 32) {
                        const int h = ch / BNH, c = ch % BNH;
                        const int fcol = (n_blk * MT::NW + h) * BNH + c;
                        if (fcol >= N) break;
                        uint32_t ra[32], rb[32];
                        ptx::tmem_ld_32x32b_x32(taddr + h * BN + c, ra);
                        ptx::tmem_ld_32x32b_x32(taddr + h * BN + BNH + c, rb);
                        ptx::tmem_ld_wait();
                        uint32_t hp[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const float h0 = silu_mul(__uint_as_float(ra[2 * i]), __uint_as_float(rb[2 * i]));
                            const float h1 = silu_mul(__uint_as_float(ra[2 * i + 1]), __uint_as_float(rb[2 * i + 1]));
                            hp[i] = pack_bf16x2(h0, h1);
                        }
                        uint8_t* dst = reinterpret_cast<uint8_t*>(H + row * (size_t)N + fcol);
#pragma unroll
                        for (int v = 0; v < 4; ++v)
                            ptx::st_global_v4_hint(dst + 16 * v, hp[4 * v], hp[4 * v + 1], hp[4 * v + 2], hp[4 * v + 3],
                                                   pol_out);
                        if (MODE == kFwd1Train) {
                            // keep the pre-activations for the backward: the 32 x 32 chunks of a
                            // and b through shared memory, then 128-byte row segments
                            float* sa = stage_out + ew * 2 * 32 * OUT_PITCH;
                            float* sb = sa + 32 * OUT_PITCH;
#pragma unroll
                            for (int v = 0; v < 8; ++v) {
                                *reinterpret_cast<uint4*>(stage_slot(sa, lane, v)) =
                                    make_uint4(ra[4 * v], ra[4 * v + 1], ra[4 * v + 2], ra[4 * v + 3]);
                                *reinterpret_cast<uint4*>(stage_slot(sb, lane, v)) =
                                    make_uint4(rb[4 * v], rb[4 * v + 1], rb[4 * v + 2], rb[4 * v + 3]);
                            }
                            __syncwarp();
                            const size_t row0w = (size_t)ctrl->row0[e] + (size_t)m_tile * BM + q * 32;
                            const int cc = (lane & 7) * 4;
#pragma unroll
                            for (int it = 0; it < 8; ++it) {
                                const int rr = it * 4 + (lane >> 3);
                                const size_t g = (row0w + rr) * (size_t)N + fcol + cc;
                                const uint4 va = *reinterpret_cast<const uint4*>(stage_slot(sa, rr, lane & 7));
                                const uint4 vb = *reinterpret_cast<const uint4*>(stage_slot(sb, rr, lane & 7));
                                ptx::st_global_v4_hint(p.keep_a + g, va.x, va.y, va.z, va.w, pol_out);
                                ptx::st_global_v4_hint(p.keep_b + g, vb.x, vb.y, vb.z, vb.w, pol_out);
                            }
                            __syncwarp();   // the next chunk reuses the buffers
                        }
                    }
                } else if (MODE == kDgradH) {
                    // dH tile (TMEM) -> SwiGLU backward with the kept a, b:
                    //     dA = dH b SiLU'(a),  dB = dH SiLU(a)   -> bf16 [slots][2N], dA | dB
                    // a, b come in and dA | dB go out as 128-byte row segments through shared memory
                    const size_t row0w = (size_t)ctrl->row0[e] + (size_t)m_tile * BM + q * 32;
                    __nv_bfloat16* dAB = static_cast<__nv_bfloat16*>(p.out);
                    float* sa = stage_out + ew * 2 * 32 * OUT_PITCH;
                    float* sb = sa + 32 * OUT_PITCH;
                    const int cc = (lane & 7) * 4;
                    constexpr int CW = BN / HALVES;
#pragma unroll 1
                    for (int c = half * CW; c < (half + 1) * CW; c += 32) {
                        const int col = n_blk * BN + c;
                        if (col >= N) break;
                        float4 ta[8], tb[8];
#pragma unroll
                        for (int it = 0; it < 8; ++it) {
                            const size_t g = (row0w + it * 4 + (lane >> 3)) * (size_t)N + col + cc;
                            ta[it] = __ldg(reinterpret_cast<const float4*>(p.aux_a + g));
                            tb[it] = __ldg(reinterpret_cast<const float4*>(p.aux_b + g));
                        }
#pragma unroll
                        for (int it = 0; it < 8; ++it) {
                            const int rr = it * 4 + (lane >> 3);
                            *reinterpret_cast<float4*>(stage_slot(sa, rr, lane & 7)) = ta[it];
                            *reinterpret_cast<float4*>(stage_slot(sb, rr, lane & 7)) = tb[it];
                        }
                        __syncwarp();
                        float av[32], bv[32];
#pragma unroll
                        for (int v = 0; v < 8; ++v) {
                            const float4 xa = *reinterpret_cast<const float4*>(stage_slot(sa, lane, v));
                            const float4 xb = *reinterpret_cast<const float4*>(stage_slot(sb, lane, v));
                            av[4 * v] = xa.x;
                            av[4 * v + 1] = xa.y;
                            av[4 * v + 2] = xa.z;
                            av[4 * v + 3] = xa.w;
                            bv[4 * v] = xb.x;
                            bv[4 * v + 1] = xb.y;
                            bv[4 * v + 2] = xb.z;
                            bv[4 * v + 3] = xb.w;
                        }
                        uint32_t r[32];
                        ptx::tmem_ld_32x32b_x32(taddr + c, r);
                        ptx::tmem_ld_wait();
                        uint32_t pa[16], pb[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            float da[2], dbv[2];
#pragma unroll
                            for (int u = 0; u < 2; ++u)
                                silu_bwd(av[2 * i + u], bv[2 * i + u], __uint_as_float(r[2 * i + u]), da[u], dbv[u]);
                            pa[i] = pack_bf16x2(da[0], da[1]);
                            pb[i] = pack_bf16x2(dbv[0], dbv[1]);
                        }
                        __syncwarp();   // every lane has its row of a, b: the buffer takes dA | dB
#pragma unroll
                        for (int v = 0; v < 4; ++v) {
                            *reinterpret_cast<uint4*>(stage_slot(sa, lane, v)) =
                                make_uint4(pa[4 * v], pa[4 * v + 1], pa[4 * v + 2], pa[4 * v + 3]);
                            *reinterpret_cast<uint4*>(stage_slot(sa, lane, 4 + v)) =
                                make_uint4(pb[4 * v], pb[4 * v + 1], pb[4 * v + 2], pb[4 * v + 3]);
                        }
                        __syncwarp();
                        // words 0-15 of a staged row are dA's 32 columns, words 16-31 dB's
                        const int part = cc >> 4;
                        const int ecol = col + 2 * (cc & 15);
#pragma unroll
                        for (int it = 0; it < 8; ++it) {
                            const int rr = it * 4 + (lane >> 3);
                            const uint4 v = *reinterpret_cast<const uint4*>(stage_slot(sa, rr, lane & 7));
                            __nv_bfloat16* dst = dAB + (row0w + rr) * (size_t)(2 * N) + (size_t)part * N + ecol;
                            ptx::st_global_v4_hint(dst, v.x, v.y, v.z, v.w, pol_out);
                        }
                        __syncwarp();   // the next chunk reuses the buffers
                    }
                } else if (MT::STAGED_OUT) {
                    // fp32 gradient tile of expert e, rows m of [M][N] (rows >= split to out_hi):
                    // each 32 x 32 chunk goes through shared memory so that the stores run along
                    // rows (8 lanes per 128-byte row segment) instead of one row per lane
                    float* stg = stage_out + ew * 32 * OUT_PITCH;
                    const bool zero = ctrl->nkb[e] == 0;   // no rows: the accumulator was never written
                    const int mbase = m_tile * BM + q * 32;
                    constexpr int CW = BN / HALVES;   // columns per warp
                    const int c0 = half * CW;
#pragma unroll 1
                    for (int c = c0; c < c0 + CW; c += 32) {
                        uint32_t r[32];
                        ptx::tmem_ld_32x32b_x32(taddr + c, r);
                        ptx::tmem_ld_wait();
                        const int col = n_blk * BN + c;
                        if (col >= N) continue;
#pragma unroll
                        for (int v = 0; v < 8; ++v)
                            *reinterpret_cast<float4*>(stage_slot(stg, lane, v)) =
                                zero ? make_float4(0.f, 0.f, 0.f, 0.f)
                                     : make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                                                   __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3]));
                        __syncwarp();
#pragma unroll
                        for (int it = 0; it < 8; ++it) {
                            const int rr = it * 4 + (lane >> 3);
                            const int cc = (lane & 7) * 4;
                            const int m = mbase + rr;
                            if (m < p.M) {
                                const float4 v = *reinterpret_cast<const float4*>(stage_slot(stg, rr, lane & 7));
                                const size_t orow = m < p.split ? (size_t)e * p.split + m
                                                                : (size_t)e * (p.M - p.split) + (m - p.split);
                                void* base = m < p.split ? p.out : p.out_hi;
                                if (MT::OUT16) {
                                    uint2 o;
                                    o.x = pack_bf16x2(v.x, v.y);
                                    o.y = pack_bf16x2(v.z, v.w);
                                    *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(base) + orow * (size_t)N +
                                                              col + cc) = o;
                                } else {
                                    float* dst = static_cast<float*>(base) + orow * (size_t)N;
                                    ptx::st_global_v4_hint(dst + col + cc, __float_as_uint(v.x), __float_as_uint(v.y),
                                                           __float_as_uint(v.z), __float_as_uint(v.w), pol_out);
                                }
                            }
                        }
                        __syncwarp();
                    }
                } else {
                    // fp32 tile (kFwd2, kDgradX; grouped-by-K tiles take the staged branch): row r of [slots][N]
                    const size_t row = (size_t)ctrl->row0[e] + (size_t)m_tile * BM + q * 32 + lane;
                    float* dst_row = static_cast<float*>(p.out) + row * (size_t)N;
#pragma unroll 1
                    for (int c = half * (MT::NW * BN / HALVES); c < (half + 1) * (MT::NW * BN / HALVES); c += 32) {
                        uint32_t r[32];
                        ptx::tmem_ld_32x32b_x32(taddr + c, r);
                        ptx::tmem_ld_wait();
                        const int col = n_blk * MT::NW * BN + c;
                        if (col < N) {
                            uint8_t* dst = reinterpret_cast<uint8_t*>(dst_row + col);
#pragma unroll
                            for (int v = 0; v < 8; ++v)
                                ptx::st_global_v4_hint(dst + 16 * v, r[4 * v], r[4 * v + 1], r[4 * v + 2], r[4 * v + 3],
                                                       pol_out);
                        }
                    }
                }
            }
            // accumulator b is free once every lane's tcgen05.ld has completed (tmem_ld_wait above);
            // the epilogue's global stores need not be visible to the MMA thread, so the arrive
            // is relaxed and does not wait for them to drain
            ptx::tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive_cluster_relaxed(ptx::map_to_rank(ptx::smem_addr(&ctrl->tempty[acc]), 0));
            if (++acc == MT::ACCS) {
                acc = 0;
                acc_phase ^= 1u;
            }
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

// [rows][inner] bf16 matrix read as MN-major 64 x 64 boxes (inner contiguous)
bool map_mn_rows(CUtensorMap* m, const void* base, size_t rows, int inner) {
    return map_matrix(m, base, rows, inner, MN_BOX, BK);
}

// [E][K][N] bf16 weights read as MN-major 64 (n) x 64 (k) x 1 boxes
bool map_mn_weights(CUtensorMap* m, const void* base, int E, int K, int N) {
    return map_expert_weights(m, base, E, K, N, MN_BOX, BK);
}

template <int MODE>
cudaError_t ensure_smem_attr() {
    static PerDeviceOnce once;
    return once.run([] {
        return cudaFuncSetAttribute(tc_gemm_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    ModeT<MODE>::SMEM);
    });
}

// Persistent grid: as many CTA pairs as fit at once, no more than there are pair tiles.
template <int MODE>
int grid_for(size_t pair_tiles, int num_sms) {
    static PerDeviceInt clusters_per_device;
    const int max_clusters = clusters_per_device.get([num_sms] {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * 74, 1, 1);
        cfg.blockDim = dim3(ModeT<MODE>::THREADS, 1, 1);
        cfg.dynamicSmemBytes = ModeT<MODE>::SMEM;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, tc_gemm_kernel<MODE>, &cfg) != cudaSuccess || n <= 0) {
            cudaGetLastError();
            n = (num_sms > 0 ? num_sms : 148) / 2;
        }
        return n;
    });
    size_t clusters = (size_t)max_clusters;
    if (clusters > pair_tiles) clusters = pair_tiles;
    if (clusters < 1) clusters = 1;
    return (int)(2 * clusters);
}

// Upper bound of the row-grouped pair tiles: every expert may add one half-empty pair.
size_t row_pair_tiles(size_t slots, int E, int n_tiles) {
    return ((slots / BM + (size_t)E) / 2 + 1) * (size_t)n_tiles;
}

template <int MODE>
cudaError_t launch_pair(size_t pair_tiles, int num_sms, const CUtensorMap& mA, const CUtensorMap& mB1,
                        const CUtensorMap& mB3, const GemmParams& gp, cudaStream_t s) {
    cudaError_t e = ensure_smem_attr<MODE>();
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid_for<MODE>(pair_tiles, num_sms), 1, 1);
    cfg.blockDim = dim3(ModeT<MODE>::THREADS, 1, 1);
    cfg.dynamicSmemBytes = ModeT<MODE>::SMEM;
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
    e = cudaLaunchKernelEx(&cfg, tc_gemm_kernel<MODE>, mA, mB1, mB3, gp);
    return e != cudaSuccess ? e : cudaGetLastError();
}

GemmParams params(Meta* meta, int E, int N, int K, int wave_slot, size_t slots, void* out, int* status,
                  long long wait_ns) {
    GemmParams gp = {};
    gp.meta = meta;
    gp.E = E;
    gp.N = N;
    gp.K = K;
    gp.wave_slot = wave_slot;
    gp.slots = slots;
    gp.out = out;
    gp.status = status;
    gp.wait_ns = wait_ns;
    return gp;
}

}  // namespace

// Wide (256 x 512) tiles when the reduction is long enough to hide their unoverlapped epilogue:
// measured A/B (one box, libraries alternating), GEMM2 (K = ffn = 14336 / 16384) ran 5-7% faster
// at every workload, GEMM1 4% faster at K = d = 6144 and 2% slower at K = 4096.  The environment
// variable MOE_WIDE_MIN_K (read once per process) moves the threshold; a value past every K keeps
// all tiles 256 x 256, which gives the same output bits (each output element sees the same MMAs
// in the same K order).
int wide_min_k() {
    static const int v = [] {
        const char* s = std::getenv("MOE_WIDE_MIN_K");
        return s && *s ? std::atoi(s) : 5120;
    }();
    return v;
}

cudaError_t launch_tc_gemm1(const TcGemmArgs& a, cudaStream_t s) {
    CUtensorMap mA, mB1, mB3;
    if (!map_rows(&mA, a.xp, a.slots, a.d, BM) || !map_weights(&mB1, a.W1, a.E, a.F, a.d, BNH) ||
        !map_weights(&mB3, a.W3, a.E, a.F, a.d, BNH))
        return cudaErrorInvalidValue;
    const GemmParams gp = params(const_cast<Meta*>(a.meta), a.E, a.F, a.d, kWaveFwd1, a.slots, a.H, a.status,
                                 a.wait_ns);
    if (a.d >= wide_min_k())
        return launch_pair<kFwd1W>(row_pair_tiles(a.slots, a.E, (a.F + 2 * BNH - 1) / (2 * BNH)), a.num_sms, mA, mB1,
                                   mB3, gp, s);
    return launch_pair<kFwd1>(row_pair_tiles(a.slots, a.E, (a.F + BNH - 1) / BNH), a.num_sms, mA, mB1, mB3, gp, s);
}

cudaError_t launch_tc_gemm1_train(const TcGemmArgs& a, float* keep_a, float* keep_b, cudaStream_t s) {
    CUtensorMap mA, mB1, mB3;
    if (!map_rows(&mA, a.xp, a.slots, a.d, BM) || !map_weights(&mB1, a.W1, a.E, a.F, a.d, BNH) ||
        !map_weights(&mB3, a.W3, a.E, a.F, a.d, BNH))
        return cudaErrorInvalidValue;
    GemmParams gp = params(const_cast<Meta*>(a.meta), a.E, a.F, a.d, kWaveFwd1, a.slots, a.H, a.status, a.wait_ns);
    gp.keep_a = keep_a;
    gp.keep_b = keep_b;
    return launch_pair<kFwd1Train>(row_pair_tiles(a.slots, a.E, (a.F + BNH - 1) / BNH), a.num_sms, mA, mB1, mB3, gp,
                                   s);
}

cudaError_t launch_tc_gemm2(const TcGemmArgs& a, cudaStream_t s) {
    CUtensorMap mA, mB;
    if (!map_rows(&mA, a.H, a.slots, a.F, BM) || !map_weights(&mB, a.W2, a.E, a.d, a.F, BNH))
        return cudaErrorInvalidValue;
    const GemmParams gp = params(const_cast<Meta*>(a.meta), a.E, a.d, a.F, kWaveFwd2, a.slots, a.Y, a.status,
                                 a.wait_ns);
    if (a.F >= wide_min_k())
        return launch_pair<kFwd2W>(row_pair_tiles(a.slots, a.E, (a.d + 2 * BN - 1) / (2 * BN)), a.num_sms, mA, mB, mB,
                                   gp, s);
    return launch_pair<kFwd2>(row_pair_tiles(a.slots, a.E, (a.d + BN - 1) / BN), a.num_sms, mA, mB, mB, gp, s);
}

cudaError_t launch_tc_dgrad_h(const TcBwdArgs& a, cudaStream_t s) {
    // dH [slots][F] = dY [slots][d] . W2_e [d][F] (B[n = f][k = i] is W2 read MN-major), turned into
    // dA | dB [slots][2F] in the epilogue with the kept a, b
    CUtensorMap mA, mB;
    if (!map_rows(&mA, a.dy, a.slots, a.d, BM) || !map_mn_weights(&mB, a.W2, a.E, a.d, a.F))
        return cudaErrorInvalidValue;
    GemmParams gp = params(a.meta, a.E, a.F, a.d, kWaveDgradH, a.slots, a.dab, a.status, a.wait_ns);
    gp.aux_a = a.keep_a;
    gp.aux_b = a.keep_b;
    return launch_pair<kDgradH>(row_pair_tiles(a.slots, a.E, (a.F + BN - 1) / BN), a.num_sms, mA, mB, mB, gp, s);
}

cudaError_t launch_tc_dgrad_x(const TcBwdArgs& a, cudaStream_t s) {
    // dXp [slots][d] = [dA dB] [slots][2F] . [W1_e ; W3_e] [2F][d]: W1 / W3 read MN-major
    CUtensorMap mA, mB1, mB3;
    if (!map_rows(&mA, a.dab, a.slots, 2 * a.F, BM) || !map_mn_weights(&mB1, a.W1, a.E, a.F, a.d) ||
        !map_mn_weights(&mB3, a.W3, a.E, a.F, a.d))
        return cudaErrorInvalidValue;
    GemmParams gp = params(a.meta, a.E, a.d, 2 * a.F, kWaveDgradX, a.slots, a.dxp, a.status, a.wait_ns);
    gp.kb_split = a.F / BK;
    if (2 * a.F >= wide_min_k())
        return launch_pair<kDgradXW>(row_pair_tiles(a.slots, a.E, (a.d + 2 * BN - 1) / (2 * BN)), a.num_sms, mA, mB1,
                                     mB3, gp, s);
    return launch_pair<kDgradX>(row_pair_tiles(a.slots, a.E, (a.d + BN - 1) / BN), a.num_sms, mA, mB1, mB3, gp,
                                s);
}

cudaError_t launch_tc_wgrad2(const TcBwdArgs& a, cudaStream_t s) {
    // dW2_e [d][F] = dY_e^T . H_e over the expert's rows: both read MN-major
    CUtensorMap mA, mB;
    if (!map_mn_rows(&mA, a.dy, a.slots, a.d) || !map_mn_rows(&mB, a.H, a.slots, a.F)) return cudaErrorInvalidValue;
    GemmParams gp = params(a.meta, a.E, a.F, 0, kWaveWgrad2, a.slots, a.dW2, a.status, a.wait_ns);
    gp.M = a.d;
    gp.split = a.d;
    gp.out_hi = a.dW2;
    const size_t tiles = (size_t)a.E * (((a.d + BM - 1) / BM + 1) / 2) * ((a.F + BN - 1) / BN);
    return a.wgrad_bf16 ? launch_pair<kWgrad16>(tiles, a.num_sms, mA, mB, mB, gp, s)
                        : launch_pair<kWgrad>(tiles, a.num_sms, mA, mB, mB, gp, s);
}

cudaError_t launch_tc_wgrad13(const TcBwdArgs& a, cudaStream_t s) {
    // [dW1_e ; dW3_e] [2F][d] = [dA dB]_e^T . Xp_e over the expert's rows: both read MN-major
    CUtensorMap mA, mB;
    if (!map_mn_rows(&mA, a.dab, a.slots, 2 * a.F) || !map_mn_rows(&mB, a.xp, a.slots, a.d))
        return cudaErrorInvalidValue;
    GemmParams gp = params(a.meta, a.E, a.d, 0, kWaveWgrad13, a.slots, a.dW1, a.status, a.wait_ns);
    gp.M = 2 * a.F;
    gp.split = a.F;
    gp.out_hi = a.dW3;
    const size_t tiles = (size_t)a.E * (((2 * a.F + BM - 1) / BM + 1) / 2) * ((a.d + BN - 1) / BN);
    return a.wgrad_bf16 ? launch_pair<kWgrad16>(tiles, a.num_sms, mA, mB, mB, gp, s)
                        : launch_pair<kWgrad>(tiles, a.num_sms, mA, mB, mB, gp, s);
}

}  // namespace moe
