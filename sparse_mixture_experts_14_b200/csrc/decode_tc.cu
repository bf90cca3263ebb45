// Decode path (few tokens): expert-weight streaming on the tensor cores.
//
// Same mathematics as the grouped GEMMs (subsection "各エキスパートの構造" of the
// "Mistral/Mixtral architecture" page, E_i(x) = W2_i (SiLU(W1_i x) * W3_i x)),
// arranged for the case where each expert sees a handful of tokens and the
// cost is reading its weights once from HBM: the weights are the M side of
// the MMA and the tokens the N side ("swap AB"),
//     stage 1   D1 = W1_e[f0:f0+128] Xp_e^T,  D3 = W3_e[f0:f0+128] Xp_e^T,
//               H[slot][f] = SiLU(D1[f][t]) * D3[f][t]          (bf16)
//     stage 2   D  = W2_e[r0:r0+128] H_e^T,   Y[slot][r] = D[r][t]  (fp32)
// Only experts with at least one token are read (the "Mixtral of Experts"
// summary page lists, among its limitations, that small-batch inference
// benefits from the small active parameter count while a large batch makes
// every expert active).  N = the expert's token
// count rounded up to 16 (at most 64), set per tile in the MMA instruction
// descriptor; TMA streams 128-row x 64-column weight boxes through a ring of
// 5 (stage 1) or 8 (stage 2) steps, 128-160 KiB of weights in flight per SM,
// with an evict-first L2 policy, since every weight byte is used once.
//
// One CTA per SM, 6 warps: warp 0 TMA producer, warp 1 MMA issuer + TMEM
// owner (256 columns: two accumulator sets of 2 x 64), warps 2-5 epilogue
// (thread = weight row; for each token the warp's 32 lanes store 32
// consecutive H or Y elements).
#include <cuda.h>

#include "moe_common.cuh"
#include "ptx_sm100.cuh"
#include "tma_map.cuh"

namespace moe {
namespace {

constexpr int DM = 128;                     // weight rows per tile (MMA M)
constexpr int DK = 64;                      // K per stage
constexpr int DNMAX = 64;                   // tokens per expert on this path (MMA N <= 64)
constexpr int W_BYTES = DM * DK * 2;        // 16 KiB
constexpr int X_BYTES = DNMAX * DK * 2;     // 8 KiB
constexpr int DSTAGES_MAX = 8;

// Ring geometry per stage kind: stage 1 streams two weight boxes (W1, W3) per
// step in 5 x 40 KiB, stage 2 one box (W2) in 8 x 24 KiB; both keep 128-160 KiB
// of weights in flight per SM.
template <bool GATE>
struct Ring {
    static constexpr int STAGES = GATE ? 5 : 8;
    static constexpr int W_BOXES = GATE ? 2 : 1;
    static constexpr int STAGE_BYTES = W_BOXES * W_BYTES + X_BYTES;
    static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES;
};
constexpr int DTMEM_COLS = 256;
constexpr int DTHREADS = 192;

struct DCtrl {
    uint64_t full[DSTAGES_MAX];
    uint64_t empty[DSTAGES_MAX];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
    int total;
    int tile_base[kMaxExperts + 1];
    int ntok[kMaxExperts];
    int row0[kMaxExperts];
};

template <bool GATE>
constexpr int dsmem_bytes() { return Ring<GATE>::SMEM_BYTES + (int)sizeof(DCtrl) + 1024; }

// GATE: stage 1 (mapWa = W1, mapWb = W3, mapX = Xp, out = H bf16 [slots][R]).
// !GATE: stage 2 (mapWa = W2, mapX = H, out = Y fp32 [slots][R]).
// R = weight rows per expert (F in stage 1, d in stage 2), K = reduction length.
template <bool GATE>
__global__ void __launch_bounds__(DTHREADS, 1)
    decode_kernel(const __grid_constant__ CUtensorMap mapWa, const __grid_constant__ CUtensorMap mapWb,
                  const __grid_constant__ CUtensorMap mapX, const Meta* __restrict__ meta, int E, int K, int R,
                  size_t slots, void* __restrict__ out, int* status, long long wait_ns) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    constexpr int DSTAGES = Ring<GATE>::STAGES;
    constexpr int DSTAGE_BYTES = Ring<GATE>::STAGE_BYTES;
    constexpr int X_OFF = Ring<GATE>::W_BOXES * W_BYTES;
    DCtrl* ctrl = reinterpret_cast<DCtrl*>(smem + Ring<GATE>::SMEM_BYTES);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    constexpr uint32_t STAGE_TX = (uint32_t)DSTAGE_BYTES;

    pdl_trigger();
    if (threadIdx.x == 0) {
        for (int s = 0; s < DSTAGES; ++s) {
            ptx::mbar_init(&ctrl->full[s], 1);
            ptx::mbar_init(&ctrl->empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(&ctrl->tfull[b], 1);
            ptx::mbar_init(&ctrl->tempty[b], 4);
        }
        ptx::mbar_init(&ctrl->drain, 1);
        ctrl->abort = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        ptx::tma_prefetch_desc(&mapWa);
        if (GATE) ptx::tma_prefetch_desc(&mapWb);
        ptx::tma_prefetch_desc(&mapX);
    }
    if (warp == 1) {
        ptx::tmem_alloc(&ctrl->tmem_base, DTMEM_COLS);
        ptx::tmem_relinquish();
    }
    // everything above overlaps the previous kernel; global memory only after this
    pdl_wait();
    if (threadIdx.x == 0) {
        const int blocks = (R + DM - 1) / DM;
        ctrl->tile_base[0] = 0;
        bool ok = true;
        for (int e = 0; e < E; ++e) {
            const int n = meta->counts[e];
            if (n < 0 || n > DNMAX) ok = false;
            if (!debug_check(n <= 0 || (meta->offsets[e] >= 0 && (size_t)meta->offsets[e] + n <= slots), nullptr))
                ok = false;   // the segment's rows must lie inside the buffers the epilogue writes
            ctrl->ntok[e] = n;
            ctrl->row0[e] = meta->offsets[e];
            ctrl->tile_base[e + 1] = ctrl->tile_base[e] + (n > 0 ? blocks : 0);
        }
        ctrl->total = ok ? ctrl->tile_base[E] : 0;
        if (!ok) record_status(status, MOE_ERR_DEVICE);
    }
    ptx::tc_fence_before_sync();
    __syncthreads();
    ptx::tc_fence_after_sync();

    const uint32_t tmem_base = ctrl->tmem_base;
    const int total = ctrl->total;
    const int nk = (K + DK - 1) / DK;
    const ptx::WaitCtl wc{&ctrl->abort, status, (uint64_t)wait_ns};

    auto decode_tile = [&](int tile, int& e, int& blk) {
        e = 0;
        while (tile >= ctrl->tile_base[e + 1]) ++e;
        blk = tile - ctrl->tile_base[e];
    };

    if (warp == 0) {
        if (lane == 0) {
            const uint64_t pol_w = ptx::policy_evict_first();
            const uint64_t pol_x = ptx::policy_evict_last();
            int stage = 0;
            uint32_t phase = 0;
            bool armed[DSTAGES];
            uint32_t armed_phase[DSTAGES];
#pragma unroll
            for (int s = 0; s < DSTAGES; ++s) {
                armed[s] = false;
                armed_phase[s] = 0;
            }
            bool aborted = false;
            for (int tile = blockIdx.x; tile < total && !aborted; tile += gridDim.x) {
                int e, blk;
                decode_tile(tile, e, blk);
                for (int kb = 0; kb < nk; ++kb) {
                    if (!ptx::mbar_wait(&ctrl->empty[stage], phase ^ 1u, wc)) {
                        aborted = true;
                        break;
                    }
                    uint8_t* sw = smem + stage * DSTAGE_BYTES;
                    ptx::mbar_arrive_expect_tx(&ctrl->full[stage], STAGE_TX);
                    ptx::tma_load_3d(sw, &mapWa, &ctrl->full[stage], kb * DK, blk * DM, e, pol_w);
                    if (GATE) ptx::tma_load_3d(sw + W_BYTES, &mapWb, &ctrl->full[stage], kb * DK, blk * DM, e, pol_w);
                    ptx::tma_load_2d(sw + X_OFF, &mapX, &ctrl->full[stage], kb * DK, ctrl->row0[e], pol_x);
#pragma unroll
                    for (int s = 0; s < DSTAGES; ++s)
                        if (s == stage) {
                            armed[s] = true;
                            armed_phase[s] = phase;
                        }
                    if (++stage == DSTAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (aborted || ctrl->abort) {
#pragma unroll
                for (int s = 0; s < DSTAGES; ++s)
                    if (armed[s]) ptx::mbar_wait_drain(&ctrl->full[s], armed_phase[s], 100000000ull);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool issued = false, aborted = false;
            for (int tile = blockIdx.x; tile < total && !aborted; tile += gridDim.x) {
                int e, blk;
                decode_tile(tile, e, blk);
                const int nn = (ctrl->ntok[e] + 15) / 16 * 16;
                const uint32_t idesc = ptx::idesc_bf16_f32(DM, nn);
                if (!ptx::mbar_wait(&ctrl->tempty[acc], acc_phase ^ 1u, wc)) {
                    aborted = true;
                    break;
                }
                ptx::tc_fence_after_sync();
                const uint32_t d1 = tmem_base + (uint32_t)(acc * 128);
                for (int kb = 0; kb < nk; ++kb) {
                    if (!ptx::mbar_wait(&ctrl->full[stage], phase, wc)) {
                        aborted = true;
                        break;
                    }
                    ptx::tc_fence_after_sync();
                    const uint32_t w0 = ptx::smem_addr(smem + stage * DSTAGE_BYTES);
                    const uint32_t x0 = w0 + X_OFF;
#pragma unroll
                    for (int kk = 0; kk < DK / 16; ++kk) {
                        const uint64_t bx = ptx::desc_kmajor_sw128(x0 + kk * 32);
                        ptx::tc_mma_bf16(d1, ptx::desc_kmajor_sw128(w0 + kk * 32), bx, idesc, (kb | kk) != 0);
                        if (GATE)
                            ptx::tc_mma_bf16(d1 + 64, ptx::desc_kmajor_sw128(w0 + W_BYTES + kk * 32), bx, idesc,
                                             (kb | kk) != 0);
                    }
                    ptx::tc_commit(&ctrl->empty[stage]);
                    issued = true;
                    if (++stage == DSTAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (aborted) break;
                ptx::tc_commit(&ctrl->tfull[acc]);
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1u;
            }
            if ((aborted || ctrl->abort) && issued) {
                ptx::tc_commit(&ctrl->drain);
                ptx::mbar_wait_drain(&ctrl->drain, 0, 100000000ull);
            }
        }
    } else {
        const int q = warp & 3;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
            int e, blk;
            decode_tile(tile, e, blk);
            const int n = ctrl->ntok[e];
            bool ok = ptx::mbar_wait(&ctrl->tfull[acc], acc_phase, wc);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            ptx::tc_fence_after_sync();
            const int r = blk * DM + q * 32 + lane;      // weight row = output column
            const size_t row0 = (size_t)ctrl->row0[e];
            const uint32_t taddr = tmem_base + (uint32_t)(acc * 128) + ((uint32_t)(q * 32) << 16);
            for (int t0 = 0; t0 < n; t0 += 16) {
                uint32_t a[16];
                ptx::tmem_ld_32x32b_x16(taddr + t0, a);
                if (GATE) {
                    uint32_t b[16];
                    ptx::tmem_ld_32x32b_x16(taddr + 64 + t0, b);
                    ptx::tmem_ld_wait();
                    __nv_bfloat16* H = static_cast<__nv_bfloat16*>(out);
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        if (t0 + i < n && r < R)
                            H[(row0 + t0 + i) * (size_t)R + r] =
                                __float2bfloat16_rn(silu_mul(__uint_as_float(a[i]), __uint_as_float(b[i])));
                    }
                } else {
                    ptx::tmem_ld_wait();
                    float* Y = static_cast<float*>(out);
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        if (t0 + i < n && r < R) Y[(row0 + t0 + i) * (size_t)R + r] = __uint_as_float(a[i]);
                    }
                }
            }
            ptx::tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&ctrl->tempty[acc]);
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1u;
        }
    }

    ptx::tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after_sync();
        ptx::tmem_dealloc(tmem_base, DTMEM_COLS);
    }
}

// E x R x K weights, K contiguous, box 64 x 128 x 1
bool map_w(CUtensorMap* m, const void* base, int E, int R, int K) {
    return map_expert_weights(m, base, E, R, K, DK, DM);
}

// rows x K token matrix, box 64 x 64
bool map_x(CUtensorMap* m, const void* base, size_t rows, int K) { return map_matrix(m, base, rows, K, DK, DNMAX); }

template <bool GATE>
cudaError_t launch_stage(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& x, const TcGemmArgs& g, int K,
                         int R, void* out, cudaStream_t s) {
    static PerDeviceOnce attr;
    cudaError_t e = attr.run([] {
        return cudaFuncSetAttribute(decode_kernel<GATE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    dsmem_bytes<GATE>());
    });
    if (e != cudaSuccess) return e;
    // As many waves as one CTA per SM needs, then as few CTAs as cover the tiles in that many
    // waves: every CTA gets the same number of tiles, so no short last wave leaves most SMs idle
    // while a few stream alone (896 tiles of stage 1 at E = 8: 7 waves on 128 CTAs, not 6 and a
    // tail of 8 on 148).  The tile count assumes every expert has tokens, as at decode sizes.
    const int sms = g.num_sms > 0 ? g.num_sms : 148;
    const int upper = g.E * ((R + DM - 1) / DM);
    const int waves = (upper + sms - 1) / sms;
    int grid = (upper + waves - 1) / waves;
    if (grid > sms) grid = sms;
    if (grid < 1) grid = 1;
    return launch_pdl(decode_kernel<GATE>, dim3(grid), dim3(DTHREADS), dsmem_bytes<GATE>(), s, a, b, x, g.meta, g.E, K, R,
                      g.slots, out, g.status, g.wait_ns);
}

}  // namespace

cudaError_t launch_decode(const TcGemmArgs& g, int stage, cudaStream_t s) {
    if (stage == 1) {
        CUtensorMap w1, w3, xp;
        if (!map_w(&w1, g.W1, g.E, g.F, g.d) || !map_w(&w3, g.W3, g.E, g.F, g.d) || !map_x(&xp, g.xp, g.slots, g.d))
            return cudaErrorInvalidValue;
        return launch_stage<true>(w1, w3, xp, g, g.d, g.F, g.H, s);
    }
    CUtensorMap w2, h;
    if (!map_w(&w2, g.W2, g.E, g.d, g.F) || !map_x(&h, g.H, g.slots, g.F)) return cudaErrorInvalidValue;
    return launch_stage<false>(w2, w2, h, g, g.F, g.d, g.Y, s);
}

}  // namespace moe
