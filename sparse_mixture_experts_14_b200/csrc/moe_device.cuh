// Device-side definitions shared by the MoE layer's kernels (sm_100a): the
// segment table every kernel reads, status and debug checks, bf16 and SwiGLU
// helpers, and programmatic dependent launch.  Host-only declarations live in
// moe_common.cuh.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

// Rows per expert segment granule: every expert's rows are padded to this, so
// a 128-row tensor-core tile never straddles two experts.
constexpr int kSegRows = 128;
constexpr int kMaxExperts = 32;
// wave counters in Meta: forward GEMM1, GEMM2, then the backward GEMMs (dH,
// SwiGLU backward, dX, dW2, dW1/dW3)
constexpr int kWaveSlots = 8;
enum WaveSlot : int { kWaveFwd1 = 0, kWaveFwd2 = 1, kWaveDgradH = 2, kWaveSwigluBwd = 3, kWaveDgradX = 4,
                      kWaveWgrad2 = 5, kWaveWgrad13 = 6 };
// Tokens handled by one dispatch block (histogram / scatter).
constexpr int kDispatchTokens = 1024;

// Small per-call table written by the dispatch scan, read by every later kernel.
struct Meta {
    int32_t counts[kMaxExperts];        // assignments per expert
    int32_t offsets[kMaxExperts + 1];   // padded segment start rows; offsets[E] = padded total
    int32_t waves[kWaveSlots];          // wave counters of the expert GEMMs (zeroed by dispatch / backward)
};

// Per-device sticky status word (first fault wins).
__device__ __forceinline__ void record_status(int* status, int code) {
    if (status) atomicCAS(status, 0, code);
}

#ifndef MOE_DEBUG
#define MOE_DEBUG 0
#endif
// Debug builds (nvcc -DMOE_DEBUG=1, libmoe_debug.so) check the indices a kernel
// reads from another kernel's output (segment rows, assignment slots, segment
// offsets, tile rows) against the buffer they address: a failed check records
// MOE_ERR_DEVICE and returns false, and the caller skips the access.  Release
// builds compile the check away (it is always true): those indices are in
// range by construction of the dispatch.
__device__ __forceinline__ bool debug_check(bool ok, int* status) {
#if MOE_DEBUG
    if (!ok) record_status(status, MOE_ERR_DEVICE);
    return ok;
#else
    (void)ok;
    (void)status;
    return true;
#endif
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

// SiLU(a) * b with SiLU(a) = a / (1 + e^-a).  For a < -88 the denominator is
// +inf and the fast division gives the correct limit 0.
__device__ __forceinline__ float silu_mul(float a, float b) {
    return __fdividef(a, 1.0f + __expf(-a)) * b;
}

// Backward of h = SiLU(a) b for the upstream gradient dh:
//     da = dh b SiLU'(a),  db = dh SiLU(a),  SiLU'(a) = s (1 + a (1 - s)),  s = 1 / (1 + e^-a).
// For a < -88, e^-a is +inf, s is 0 and both gradients are 0.
__device__ __forceinline__ void silu_bwd(float a, float b, float dh, float& da, float& db) {
    const float s = __fdividef(1.0f, 1.0f + __expf(-a));
    db = dh * a * s;
    da = dh * b * s * (1.0f + a * (1.0f - s));
}

// Programmatic dependent launch.  Every kernel of the layer is launched with
// programmatic stream serialisation: it lets the next kernel in the stream be
// scheduled once all of its own CTAs have started (pdl_trigger at entry),
// and it does no global-memory access before pdl_wait, which returns once
// the previous grid in the stream has completed and its writes are visible.
// The next kernel's launch latency and prologue (barrier set-up, tensor
// memory allocation) thereby overlap the tail of the current one.
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

}  // namespace moe
