// Backward pass of the layer: gradients of a loss L given dout = dL/dout.
//
// The layer is trained by gradient descent on the language-model loss plus
// the load-balance loss (subsection "ロードバランス損失" of the
// "Mistral/Mixtral architecture" page); this file holds everything of the
// backward except the tensor-core GEMMs (gemm_tc.cu).  Differentiating the
// output equation of subsection "Top-2ゲーティングの定式化" and the expert
// equation of subsection "各エキスパートの構造", with the top-k choice fixed
// (it is piecewise constant), per assignment (t, j) of expert e in slot r:
//     dY[r]  = g_tj dout_t                 dg_tj = <dout_t, Y[r]>
//     ds_te  = g_tj (dg_tj - sum_m g_tm dg_tm)       (softmax over the k)
//     dH     = dY W2_e,  dA, dB = SwiGLU backward,  dXp = dA W1_e + dB W3_e
//     dW2_e  = dY_e^T H_e,  dW1_e = dA_e^T Xp_e,  dW3_e = dB_e^T Xp_e
//     dWg    = ds^T x,      dx_t = sum_j dXp[slot(t, j)] + ds_t Wg
// With alpha != 0 the loss also holds alpha L_balance (f = counts / T held
// fixed, p_t = softmax(s_t) over all E): every score of token t gets
//     ds_te += (alpha E / T) p_te (f_e - sum_m p_tm f_m)
// Every sum runs in a fixed order (no float atomics), so the gradients are
// the same bits on every run.
//
// Kernels here: the gate-scaled scatter of dout into the expert segments
// (with dg), the router-score gradient ds, dWg (per-chunk partial sums, then
// one ordered pass), the dx combine, and the fp32 entry points' grouped GEMMs
// on the CUDA cores (operands read through strides, so none is transposed).
#include "moe_common.cuh"

namespace moe {
namespace {

template <typename T>
struct Elt;
template <>
struct Elt<float> {
    __device__ __forceinline__ static float get(const float* p, size_t i) { return __ldg(p + i); }
    __device__ __forceinline__ static void put(float* p, size_t i, float v) { p[i] = v; }
};
template <>
struct Elt<__nv_bfloat16> {
    __device__ __forceinline__ static float get(const __nv_bfloat16* p, size_t i) { return __bfloat162float(p[i]); }
    __device__ __forceinline__ static void put(__nv_bfloat16* p, size_t i, float v) { p[i] = __float2bfloat16_rn(v); }
};

// One warp per padded row r < offsets[E]: dY[r] = g dout_t rounded to the
// operand type (zero on padding rows) and dg[t][j] = <dout_t, Y[r]> (lane
// partial sums in column order, then a fixed butterfly).  Block 0 also
// zeroes the backward GEMMs' wave counters.
template <typename T>
__global__ void __launch_bounds__(256) bwd_scatter_kernel(const T* __restrict__ dout, const float* __restrict__ w,
                                                          const float* __restrict__ Y, Meta* __restrict__ meta,
                                                          const int32_t* __restrict__ perm, int E, int T_, int k,
                                                          int d, size_t slots, T* __restrict__ dY,
                                                          float* __restrict__ dg, int* status) {
    pdl_trigger();
    pdl_wait();
    if (blockIdx.x == 0 && threadIdx.x >= kWaveDgradH && threadIdx.x < kWaveSlots) meta->waves[threadIdx.x] = 0;
    const int lane = threadIdx.x & 31;
    const size_t total = (size_t)meta->offsets[E];
    const size_t warps = (size_t)gridDim.x * (blockDim.x >> 5);
    const long long TK = (long long)T_ * k;
    for (size_t r = (size_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < total && r < slots; r += warps) {
        const int a = perm[r];
        T* dst = dY + r * (size_t)d;
        debug_check(a >= -1 && a < TK, status);   // -1 marks a padding row
        if (a >= 0 && a < TK) {
            const int t = a / k;
            const float g = w[a];
            const T* src = dout + (size_t)t * d;
            const float* y = Y + r * (size_t)d;
            float acc = 0.f;
            if (sizeof(T) == 2) {
                // 8 elements per lane and step (d % 64 == 0 on the bf16 path)
                for (int v = lane; v < d / 8; v += 32) {
                    const uint4 u = __ldg(reinterpret_cast<const uint4*>(src) + v);
                    const float4 y0 = __ldg(reinterpret_cast<const float4*>(y) + 2 * v);
                    const float4 y1 = __ldg(reinterpret_cast<const float4*>(y) + 2 * v + 1);
                    const float go[8] = {bf16_lo(u.x), bf16_hi(u.x), bf16_lo(u.y), bf16_hi(u.y),
                                         bf16_lo(u.z), bf16_hi(u.z), bf16_lo(u.w), bf16_hi(u.w)};
                    const float yv[8] = {y0.x, y0.y, y0.z, y0.w, y1.x, y1.y, y1.z, y1.w};
#pragma unroll
                    for (int i = 0; i < 8; ++i) acc = fmaf(go[i], yv[i], acc);
                    uint4 o;
                    o.x = pack_bf16x2(g * go[0], g * go[1]);
                    o.y = pack_bf16x2(g * go[2], g * go[3]);
                    o.z = pack_bf16x2(g * go[4], g * go[5]);
                    o.w = pack_bf16x2(g * go[6], g * go[7]);
                    reinterpret_cast<uint4*>(dst)[v] = o;
                }
            } else {
                for (int i = lane; i < d; i += 32) {
                    const float go = Elt<T>::get(src, i);
                    Elt<T>::put(dst, i, g * go);
                    acc = fmaf(go, y[i], acc);
                }
            }
#pragma unroll
            for (int m = 16; m >= 1; m >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m);
            if (lane == 0) dg[a] = acc;
        } else {
            for (int i = lane; i < d; i += 32) Elt<T>::put(dst, i, 0.f);
        }
    }
}

// ds[t][e]: the gradient of the router scores (output path: zero for unselected
// experts; with alpha != 0 plus the load-balance part on every expert).
__global__ void __launch_bounds__(256) router_bwd_kernel(const int32_t* __restrict__ idx, const float* __restrict__ w,
                                                         const float* __restrict__ dg, const float* __restrict__ logits,
                                                         const Meta* __restrict__ meta, float alpha, int T_, int E,
                                                         int k, float* __restrict__ ds) {
    pdl_trigger();
    pdl_wait();
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= T_) return;
    float gdg = 0.f;
    for (int j = 0; j < k; ++j) gdg = fmaf(w[(size_t)t * k + j], dg[(size_t)t * k + j], gdg);
    float* row = ds + (size_t)t * E;
    for (int e = 0; e < E; ++e) row[e] = 0.f;
    for (int j = 0; j < k; ++j) {
        const int e = idx[(size_t)t * k + j];
        if (e >= 0 && e < E) row[e] = w[(size_t)t * k + j] * (dg[(size_t)t * k + j] - gdg);
    }
    if (alpha != 0.f) {
        const float* s = logits + (size_t)t * E;
        float mx = -INFINITY, den = 0.f, pf = 0.f;
        for (int e = 0; e < E; ++e) mx = fmaxf(mx, s[e]);
        for (int e = 0; e < E; ++e) den += expf(s[e] - mx);
        const float invT = 1.0f / (float)T_;
        for (int e = 0; e < E; ++e) pf += expf(s[e] - mx) / den * ((float)meta->counts[e] * invT);
        const float c = alpha * (float)E * invT;
        for (int e = 0; e < E; ++e) {
            const float p = expf(s[e] - mx) / den;
            row[e] += c * p * ((float)meta->counts[e] * invT - pf);
        }
    }
}

constexpr int kWgChunk = 64;    // tokens per dWg partial sum

// part[c][e][j] = sum over tokens t of chunk c (ascending) of ds[t][e] x[t][j].
// NORM (the block form): the router's input is the normalised row
// u[t][j] = (h[t][j] gamma[j]) r[t], formed here in fp32 from h (passed as x),
// gamma and the forward's row factors r.
template <typename T, int EB, bool NORM>
__global__ void __launch_bounds__(256) dwg_part_kernel(const T* __restrict__ x, const float* __restrict__ ds, int T_,
                                                       int d, int E, float* __restrict__ part,
                                                       const T* __restrict__ gamma, const float* __restrict__ rstd) {
    pdl_trigger();
    pdl_wait();
    __shared__ float sds[kWgChunk][EB];
    __shared__ float srow[kWgChunk];
    const int c = blockIdx.y;
    const int t0 = c * kWgChunk;
    const int nt = min(kWgChunk, T_ - t0);
    for (int i = threadIdx.x; i < nt * EB; i += blockDim.x) {
        const int t = i / EB, e = i - t * EB;
        sds[t][e] = e < E ? ds[(size_t)(t0 + t) * E + e] : 0.f;
    }
    if (NORM)
        for (int i = threadIdx.x; i < nt; i += blockDim.x) srow[i] = rstd[t0 + i];
    __syncthreads();
    const int j = blockIdx.x * blockDim.x + threadIdx.x;
    if (j >= d) return;
    const float gj = NORM ? Elt<T>::get(gamma, j) : 1.f;
    float acc[EB];
#pragma unroll
    for (int e = 0; e < EB; ++e) acc[e] = 0.f;
    int t = 0;
    for (; t + 8 <= nt; t += 8) {
        float xv[8];   // eight rows in flight before the arithmetic
#pragma unroll
        for (int u = 0; u < 8; ++u) xv[u] = Elt<T>::get(x, (size_t)(t0 + t + u) * d + j);
        if (NORM) {
#pragma unroll
            for (int u = 0; u < 8; ++u) xv[u] = (xv[u] * gj) * srow[t + u];
        }
#pragma unroll
        for (int u = 0; u < 8; ++u)
#pragma unroll
            for (int e = 0; e < EB; ++e) acc[e] = fmaf(sds[t + u][e], xv[u], acc[e]);
    }
    for (; t < nt; ++t) {
        float xv = Elt<T>::get(x, (size_t)(t0 + t) * d + j);
        if (NORM) xv = (xv * gj) * srow[t];
#pragma unroll
        for (int e = 0; e < EB; ++e) acc[e] = fmaf(sds[t][e], xv, acc[e]);
    }
#pragma unroll
    for (int e = 0; e < EB; ++e)
        if (e < E) part[((size_t)c * E + e) * d + j] = acc[e];
}

__global__ void __launch_bounds__(256) dwg_final_kernel(const float* __restrict__ part, int chunks, int E, int d,
                                                        float* __restrict__ dWg) {
    pdl_trigger();
    pdl_wait();
    const size_t n = (size_t)E * d;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        float v = 0.f;
        for (int c = 0; c < chunks; ++c) v += part[(size_t)c * n + i];
        dWg[i] = v;
    }
}

// dx[t] = sum_j dXp[inv[t][j]] (j ascending) + sum_e ds[t][e] Wg[e] (e ascending, nonzero ds only),
// in fp32, rounded once; four columns per thread (d % 4 == 0 on both paths).
template <typename T>
__global__ void __launch_bounds__(256) dx_combine_kernel(const float* __restrict__ dXp, const int32_t* __restrict__ inv,
                                                         const float* __restrict__ ds, const T* __restrict__ Wg, int T_,
                                                         int d, int E, int k, size_t slots, int* status,
                                                         T* __restrict__ dx) {
    pdl_trigger();
    pdl_wait();
    const unsigned q = (unsigned)d / 4;
    const size_t n = (size_t)T_ * q;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        const unsigned t = (unsigned)(i / q);
        const unsigned c = (unsigned)(i - (size_t)t * q);
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int j = 0; j < k; ++j) {
            const int slot = inv[(size_t)t * k + j];
            if (slot < 0 || !debug_check((size_t)slot < slots, status)) continue;
            const float4 v = __ldg(reinterpret_cast<const float4*>(dXp + (size_t)slot * d) + c);
            acc.x += v.x;
            acc.y += v.y;
            acc.z += v.z;
            acc.w += v.w;
        }
        for (int e = 0; e < E; ++e) {
            const float s = ds[(size_t)t * E + e];
            if (s == 0.f) continue;
            float w[4];
            if (sizeof(T) == 2) {
                const uint2 u = __ldg(reinterpret_cast<const uint2*>(Wg + (size_t)e * d) + c);
                w[0] = bf16_lo(u.x);
                w[1] = bf16_hi(u.x);
                w[2] = bf16_lo(u.y);
                w[3] = bf16_hi(u.y);
            } else {
                const float4 u = __ldg(reinterpret_cast<const float4*>(Wg + (size_t)e * d) + c);
                w[0] = u.x;
                w[1] = u.y;
                w[2] = u.z;
                w[3] = u.w;
            }
            acc.x = fmaf(s, w[0], acc.x);
            acc.y = fmaf(s, w[1], acc.y);
            acc.z = fmaf(s, w[2], acc.z);
            acc.w = fmaf(s, w[3], acc.w);
        }
        T* out = dx + (size_t)t * d + 4 * c;
        if (sizeof(T) == 2) {
            uint2 o;
            o.x = pack_bf16x2(acc.x, acc.y);
            o.y = pack_bf16x2(acc.z, acc.w);
            *reinterpret_cast<uint2*>(out) = o;
        } else {
            *reinterpret_cast<float4*>(out) = acc;
        }
    }
}

// Block form: the MoE layer's input is u = RMSNorm(h), u[t][j] = gamma[j] h[t][j] r[t] with
// r[t] = (mean_i h[t][i]^2 + eps)^(-1/2) (section "Mixtral 8x7B — Sparse MoEの導入",
// subsection "Mixtralのアーキテクチャ": RMSNorm, the MoE layer, then the residual add).  With
// du = dL/du (the MoE backward's input gradient: expert rows in selection order, then the router
// term over experts in ascending order, the dx_combine sum) and dr/dh_i = -r^3 h_i / d:
//     dh[t][i]    = dout[t][i] + r gamma[i] du[t][i] - (r^3 / d) h[t][i] <du[t], gamma . h[t]>
//     dgamma[j]   = sum_t du[t][j] h[t][j] r[t]
// (the residual passes dout to h unchanged).  One block per chunk of kBlkChunk tokens, taken in
// token order, its threads spanning the row (VPT float4 columns each), the chunk's slots and score
// gradients staged in shared memory first, so a token's row loads all go out at once:
// per token the block holds du's row in registers, reduces the projection in a fixed order
// (thread columns ascending, warp butterfly, warp order), writes dh rounded once, and adds
// du h r to its per-column dgamma partial, written once per chunk.  dgamma = the chunk partials
// summed in chunk order (dwg_final_kernel with one row).
constexpr int kBlkChunk = 8;

// Four consecutive elements of a row as one vector load, widened to fp32.
template <typename T>
struct V4;
template <>
struct V4<float> {
    using Raw = float4;
    __device__ __forceinline__ static Raw load(const float* p) { return __ldg(reinterpret_cast<const float4*>(p)); }
    __device__ __forceinline__ static float4 widen(const Raw& r) { return r; }
};
template <>
struct V4<__nv_bfloat16> {
    using Raw = uint2;
    __device__ __forceinline__ static Raw load(const __nv_bfloat16* p) {
        return __ldg(reinterpret_cast<const uint2*>(p));
    }
    __device__ __forceinline__ static float4 widen(const Raw& r) {
        return make_float4(bf16_lo(r.x), bf16_hi(r.x), bf16_lo(r.y), bf16_hi(r.y));
    }
};

template <typename T, int VPT>
__global__ void __launch_bounds__(512, 2) block_dx_kernel(const float* __restrict__ dXp, const int32_t* __restrict__ inv,
                                                          const float* __restrict__ ds, const T* __restrict__ Wg,
                                                          const T* __restrict__ h, const T* __restrict__ gamma,
                                                          const float* __restrict__ rstd, const T* __restrict__ dout,
                                                          int T_, int d, int E, int k, size_t slots, int* status,
                                                          T* __restrict__ dh, float* __restrict__ dgam_part) {
    pdl_trigger();
    pdl_wait();
    __shared__ float red[2][32];
    __shared__ int sslot[kBlkChunk][kMaxExperts];    // the chunk's assignment slots (k <= E <= 32)
    __shared__ float sds[kBlkChunk][kMaxExperts];     // and its score gradients
    const int q = d / 4;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    const int t0 = blockIdx.x * kBlkChunk;
    const int t1 = min(T_, t0 + kBlkChunk);
    for (int i = threadIdx.x; i < (t1 - t0) * kMaxExperts; i += blockDim.x) {
        const int tt = i / kMaxExperts, j = i - tt * kMaxExperts;
        sslot[tt][j] = j < k ? __ldg(inv + (size_t)(t0 + tt) * k + j) : -1;
        sds[tt][j] = j < E ? __ldg(ds + (size_t)(t0 + tt) * E + j) : 0.f;
    }
    __syncthreads();
    float4 dgp[VPT];
#pragma unroll
    for (int v = 0; v < VPT; ++v) dgp[v] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int t = t0; t < t1; ++t) {
        const int tt = t - t0;
        const int buf = tt & 1;
        float4 du[VPT];
        float proj = 0.f;
#pragma unroll
        for (int v = 0; v < VPT; ++v) {
            const int c = threadIdx.x + v * blockDim.x;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            if (c < q) {
                const size_t o = (size_t)t * d + 4 * (size_t)c;
                // the token's loads go out before the arithmetic that needs them
                const typename V4<T>::Raw hr = V4<T>::load(h + o);
                const typename V4<T>::Raw gr = V4<T>::load(gamma + 4 * (size_t)c);
                // expert rows in selection order
                for (int j = 0; j < k; ++j) {
                    const int slot = sslot[tt][j];
                    if (slot < 0 || !debug_check((size_t)slot < slots, status)) continue;
                    const float4 x4 = __ldg(reinterpret_cast<const float4*>(dXp + (size_t)slot * d) + c);
                    acc.x += x4.x;
                    acc.y += x4.y;
                    acc.z += x4.z;
                    acc.w += x4.w;
                }
                // then the router term in expert order, nonzero gradients only (dx_combine's sum);
                // the Wg columns of 8 experts are loaded before their FMAs
#pragma unroll 1
                for (int e0 = 0; e0 < E; e0 += 8) {
                    typename V4<T>::Raw wr[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u)
                        if (e0 + u < E && sds[tt][e0 + u] != 0.f)
                            wr[u] = V4<T>::load(Wg + (size_t)(e0 + u) * d + 4 * (size_t)c);
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const float sv = e0 + u < E ? sds[tt][e0 + u] : 0.f;
                        if (sv == 0.f) continue;
                        const float4 w4 = V4<T>::widen(wr[u]);
                        acc.x = fmaf(sv, w4.x, acc.x);
                        acc.y = fmaf(sv, w4.y, acc.y);
                        acc.z = fmaf(sv, w4.z, acc.z);
                        acc.w = fmaf(sv, w4.w, acc.w);
                    }
                }
                const float4 hv = V4<T>::widen(hr), gv = V4<T>::widen(gr);
                proj = fmaf(acc.x, gv.x * hv.x, proj);
                proj = fmaf(acc.y, gv.y * hv.y, proj);
                proj = fmaf(acc.z, gv.z * hv.z, proj);
                proj = fmaf(acc.w, gv.w * hv.w, proj);
            }
            du[v] = acc;
        }
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) proj += __shfl_xor_sync(0xffffffffu, proj, m);
        if (lane == 0) red[buf][warp] = proj;
        // one barrier per token: the buffers alternate, so a token's partials are written only after
        // every thread has passed the previous token's barrier and read the buffer of two tokens back
        __syncthreads();
        float tot = 0.f;
        for (int w = 0; w < nwarps; ++w) tot += red[buf][w];
        const float r = __ldg(rstd + t);
        const float c3 = r * r * r / (float)d * tot;
#pragma unroll
        for (int v = 0; v < VPT; ++v) {
            const int c = threadIdx.x + v * blockDim.x;
            if (c >= q) continue;
            const size_t o = (size_t)t * d + 4 * (size_t)c;
            // h, gamma and dout again: the row was just read, so these come from L1
            const float4 hv = V4<T>::widen(V4<T>::load(h + o));
            const float4 gv = V4<T>::widen(V4<T>::load(gamma + 4 * (size_t)c));
            const float4 go = V4<T>::widen(V4<T>::load(dout + o));
            float outv[4];
            outv[0] = go.x + r * gv.x * du[v].x - c3 * hv.x;
            outv[1] = go.y + r * gv.y * du[v].y - c3 * hv.y;
            outv[2] = go.z + r * gv.z * du[v].z - c3 * hv.z;
            outv[3] = go.w + r * gv.w * du[v].w - c3 * hv.w;
            if (sizeof(T) == 2) {
                uint2 pk;
                pk.x = pack_bf16x2(outv[0], outv[1]);
                pk.y = pack_bf16x2(outv[2], outv[3]);
                *reinterpret_cast<uint2*>(dh + o) = pk;
            } else {
                *reinterpret_cast<float4*>(reinterpret_cast<float*>(dh) + o) =
                    make_float4(outv[0], outv[1], outv[2], outv[3]);
            }
            dgp[v].x = fmaf(du[v].x * hv.x, r, dgp[v].x);
            dgp[v].y = fmaf(du[v].y * hv.y, r, dgp[v].y);
            dgp[v].z = fmaf(du[v].z * hv.z, r, dgp[v].z);
            dgp[v].w = fmaf(du[v].w * hv.w, r, dgp[v].w);
        }
    }
#pragma unroll
    for (int v = 0; v < VPT; ++v) {
        const int c = threadIdx.x + v * blockDim.x;
        if (c < q) reinterpret_cast<float4*>(dgam_part + (size_t)blockIdx.x * d)[c] = dgp[v];
    }
}

// ---------------------------------------------------------------- fp32 grouped GEMMs (CUDA cores)

// Strided view of one operand: element (row, k) of expert e is
// base[e * es + row * sr + k * sk]; a second base takes over for k >= ksplit.
struct View {
    const float* base;
    const float* base2;
    size_t es, sr, sk;
    int ksplit;
    __device__ __forceinline__ float at(int e, int row, int k) const {
        const float* b = base;
        if (k >= ksplit) {
            b = base2;
            k -= ksplit;
        }
        return __ldg(b + (size_t)e * es + (size_t)row * sr + (size_t)k * sk);
    }
};

constexpr int GT = 64, GK = 16;

// Row-grouped (ROWS): C[r][n] = sum_k A(r, k) B_e(n, k) over the rows r of
// expert e's segment, K = K.  Grouped by K (!ROWS): C_e[m][n] = sum over the
// expert's rows r of A(r, m) B(r, n).  SWIGLU_BWD: B and B3 give a and b of
// the row; the output row is dA | dB from dh.  Sums run over k ascending.
template <bool ROWS, bool SWIGLU_BWD>
__global__ void __launch_bounds__(256) simt_gemm_bwd_kernel(View A, View B, View B3, const Meta* __restrict__ meta,
                                                            int E, int M, int N, int K, const float* __restrict__ dh,
                                                            float* __restrict__ C, float* __restrict__ C_hi,
                                                            int split) {
    pdl_trigger();
    pdl_wait();
    __shared__ float As[GK][GT + 4];
    __shared__ float Bs[GK][GT + 4];
    __shared__ float B3s[SWIGLU_BWD ? GK : 1][GT + 4];
    int e, m0, k0, k1;
    if (ROWS) {
        m0 = blockIdx.x * GT;
        const int total = meta->offsets[E];
        if (m0 >= total) return;
        e = 0;
        while (e + 1 < E && m0 >= meta->offsets[e + 1]) ++e;
        k0 = 0;
        k1 = K;
    } else {
        e = blockIdx.z;
        m0 = blockIdx.x * GT;
        if (m0 >= M) return;
        k0 = meta->offsets[e];
        k1 = meta->offsets[e + 1];
    }
    const int n0 = blockIdx.y * GT;
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    float acc[4][4], acc3[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = acc3[i][j] = 0.f;
    for (int kk = k0; kk < k1; kk += GK) {
        for (int l = threadIdx.x; l < GT * GK; l += 256) {
            const int r = l / GK, c = l % GK;
            const int k = kk + c;
            const bool kin = k < k1;
            const int m = m0 + r, n = n0 + r;
            if (ROWS) {
                As[c][r] = kin ? A.at(0, m, k) : 0.f;
                Bs[c][r] = (kin && n < N) ? B.at(e, n, k) : 0.f;
                if (SWIGLU_BWD) B3s[c][r] = (kin && n < N) ? B3.at(e, n, k) : 0.f;
            } else {
                As[c][r] = (kin && m < M) ? A.at(0, k, m) : 0.f;
                Bs[c][r] = (kin && n < N) ? B.at(0, k, n) : 0.f;
            }
        }
        __syncthreads();
#pragma unroll
        for (int c = 0; c < GK; ++c) {
            float a[4], b[4], b3[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = As[c][ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                b[j] = Bs[c][tx * 4 + j];
                if (SWIGLU_BWD) b3[j] = B3s[c][tx * 4 + j];
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
                    if (SWIGLU_BWD) acc3[i][j] = fmaf(a[i], b3[j], acc3[i][j]);
                }
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int m = m0 + ty * 4 + i;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = n0 + tx * 4 + j;
            if (n >= N) continue;
            if (SWIGLU_BWD) {
                const float av = acc[i][j], bv = acc3[i][j], g = dh[(size_t)m * N + n];
                const float s = 1.0f / (1.0f + expf(-av));
                C[(size_t)m * (2 * N) + n] = g * bv * s * (1.0f + av * (1.0f - s));
                C[(size_t)m * (2 * N) + N + n] = g * av * s;
            } else if (ROWS) {
                C[(size_t)m * N + n] = acc[i][j];
            } else if (m < M) {
                float* dst = m < split ? C + ((size_t)e * split + m) * N
                                       : C_hi + ((size_t)e * (M - split) + (m - split)) * N;
                dst[n] = acc[i][j];
            }
        }
    }
}

View view(const float* base, size_t es, size_t sr, size_t sk, const float* base2 = nullptr, int ksplit = INT32_MAX) {
    return View{base, base2 ? base2 : base, es, sr, sk, ksplit};
}

template <typename T>
cudaError_t launch_scatter(const BwdArgs& a, cudaStream_t s) {
    size_t blocks = (a.slots + 7) / 8;
    if (blocks > 65535 * 4) blocks = 65535 * 4;
    if (blocks < 1) blocks = 1;
    return launch_pdl(bwd_scatter_kernel<T>, dim3((unsigned)blocks), dim3(256), 0, s,
                      static_cast<const T*>(a.dout), a.w, a.Y, a.meta, a.perm, a.E, a.T, a.k, a.d, a.slots,
                      static_cast<T*>(a.dy), a.dg, a.status);
}

template <typename T, bool NORM>
cudaError_t launch_dwg_part(const BwdArgs& a, cudaStream_t s, dim3 grid) {
    const T* x = static_cast<const T*>(a.x);
    const T* g = static_cast<const T*>(a.gamma);
    if (a.E <= 8)
        return launch_pdl(dwg_part_kernel<T, 8, NORM>, grid, dim3(256), 0, s, x, a.ds, a.T, a.d, a.E, a.dwg_part, g,
                          a.rstd);
    if (a.E <= 16)
        return launch_pdl(dwg_part_kernel<T, 16, NORM>, grid, dim3(256), 0, s, x, a.ds, a.T, a.d, a.E, a.dwg_part, g,
                          a.rstd);
    return launch_pdl(dwg_part_kernel<T, 32, NORM>, grid, dim3(256), 0, s, x, a.ds, a.T, a.d, a.E, a.dwg_part, g,
                      a.rstd);
}

template <typename T>
cudaError_t launch_dwg(const BwdArgs& a, cudaStream_t s) {
    const int chunks = (a.T + kWgChunk - 1) / kWgChunk;
    const dim3 grid((a.d + 255) / 256, chunks);
    cudaError_t e = a.gamma ? launch_dwg_part<T, true>(a, s, grid) : launch_dwg_part<T, false>(a, s, grid);
    if (e != cudaSuccess) return e;
    size_t blocks = ((size_t)a.E * a.d + 255) / 256;
    if (blocks > 148 * 8) blocks = 148 * 8;
    return launch_pdl(dwg_final_kernel, dim3((unsigned)blocks), dim3(256), 0, s, static_cast<const float*>(a.dwg_part),
                      chunks, a.E, a.d, a.dWg);
}

template <typename T>
cudaError_t launch_block_dx(const BwdArgs& a, cudaStream_t s) {
    const int chunks = (a.T + kBlkChunk - 1) / kBlkChunk;
    const int q = a.d / 4;
    const float* dxp = static_cast<const float*>(a.dxp);
    const T* Wg = static_cast<const T*>(a.Wg);
    const T* h = static_cast<const T*>(a.x);
    const T* g = static_cast<const T*>(a.gamma);
    const T* dout = static_cast<const T*>(a.dout);
    T* dh = static_cast<T*>(a.dx);
    cudaError_t e;
    // threads span the row, at most 512 per block (two blocks per SM): one float4 column each up to
    // d = 2048, two up to d = 4096, four up to d = 8192
    auto go = [&](auto kern, int vpt) {
        const unsigned nt = (unsigned)(((q + vpt - 1) / vpt + 31) / 32 * 32);
        return launch_pdl(kern, dim3(chunks), dim3(nt), 0, s, dxp, a.inv, a.ds, Wg, h, g, a.rstd, dout, a.T, a.d,
                          a.E, a.k, a.slots, a.status, dh, a.dgamma_part);
    };
    if (q > 2048) return cudaErrorInvalidValue;   // rows longer than 8192: refused by the entry point
    if (q <= 512) {
        e = go(block_dx_kernel<T, 1>, 1);
    } else if (q <= 1024) {
        e = go(block_dx_kernel<T, 2>, 2);
    } else {
        e = go(block_dx_kernel<T, 4>, 4);
    }
    if (e != cudaSuccess) return e;
    size_t blocks = ((size_t)a.d + 255) / 256;
    if (blocks > 148 * 8) blocks = 148 * 8;
    return launch_pdl(dwg_final_kernel, dim3((unsigned)blocks), dim3(256), 0, s,
                      static_cast<const float*>(a.dgamma_part), chunks, 1, a.d, a.dgamma);
}

template <typename T>
cudaError_t launch_dx(const BwdArgs& a, cudaStream_t s) {
    size_t blocks = ((size_t)a.T * (a.d / 4) + 255) / 256;
    if (blocks > 148 * 32) blocks = 148 * 32;
    if (blocks < 1) blocks = 1;
    return launch_pdl(dx_combine_kernel<T>, dim3((unsigned)blocks), dim3(256), 0, s, static_cast<const float*>(a.dxp),
                      a.inv, static_cast<const float*>(a.ds), static_cast<const T*>(a.Wg), a.T, a.d, a.E, a.k,
                      a.slots, a.status, static_cast<T*>(a.dx));
}

}  // namespace

size_t dwg_part_bytes(int T, int E, int d) {
    const size_t chunks = (size_t)(T > 0 ? (T + kWgChunk - 1) / kWgChunk : 1);
    return chunks * (size_t)E * d * 4;
}

cudaError_t launch_bwd_scatter(const BwdArgs& a, cudaStream_t s) {
    return a.bf16 ? launch_scatter<__nv_bfloat16>(a, s) : launch_scatter<float>(a, s);
}

cudaError_t launch_router_bwd(const BwdArgs& a, cudaStream_t s) {
    return launch_pdl(router_bwd_kernel, dim3((a.T + 255) / 256), dim3(256), 0, s, a.idx, a.w,
                      static_cast<const float*>(a.dg), a.logits, static_cast<const Meta*>(a.meta), a.alpha, a.T, a.E,
                      a.k, a.ds);
}

cudaError_t launch_dwg(const BwdArgs& a, cudaStream_t s) {
    return a.bf16 ? launch_dwg<__nv_bfloat16>(a, s) : launch_dwg<float>(a, s);
}

cudaError_t launch_dx_combine(const BwdArgs& a, cudaStream_t s) {
    if (a.gamma) return a.bf16 ? launch_block_dx<__nv_bfloat16>(a, s) : launch_block_dx<float>(a, s);
    return a.bf16 ? launch_dx<__nv_bfloat16>(a, s) : launch_dx<float>(a, s);
}

size_t block_dgamma_part_bytes(int T, int d) {
    const size_t chunks = (size_t)(T > 0 ? (T + kBlkChunk - 1) / kBlkChunk : 1);
    return chunks * (size_t)d * 4;
}

cudaError_t launch_simt_bwd_gemms(const BwdArgs& a, cudaStream_t s) {
    const int E = a.E, d = a.d, F = a.F;
    const size_t S = a.slots;
    const float* xp = static_cast<const float*>(a.xp);
    const float* W1 = static_cast<const float*>(a.W1);
    const float* W3 = static_cast<const float*>(a.W3);
    const float* W2 = static_cast<const float*>(a.W2);
    const float* H = static_cast<const float*>(a.H);
    const float* dy = static_cast<const float*>(a.dy);
    float* dab = static_cast<float*>(a.dab);
    const View none = view(nullptr, 0, 0, 0);
    const dim3 blk(256);
    // dH [S][F] = dY . W2_e : B(n = f, k = i) = W2[e][i][f]
    cudaError_t e = launch_pdl(simt_gemm_bwd_kernel<true, false>, dim3((unsigned)(S / GT), (F + GT - 1) / GT), blk, 0, s,
                               view(dy, 0, d, 1), view(W2, (size_t)d * F, 1, F), none, a.meta, E, 0, F, d,
                               static_cast<const float*>(nullptr), a.dh, static_cast<float*>(nullptr), 0);
    // dA | dB [S][2F] from a = Xp W1_e^T, b = Xp W3_e^T and dH
    if (e == cudaSuccess)
        e = launch_pdl(simt_gemm_bwd_kernel<true, true>, dim3((unsigned)(S / GT), (F + GT - 1) / GT), blk, 0, s,
                       view(xp, 0, d, 1), view(W1, (size_t)F * d, d, 1), view(W3, (size_t)F * d, d, 1), a.meta, E, 0,
                       F, d, static_cast<const float*>(a.dh), dab, static_cast<float*>(nullptr), 0);
    // dXp [S][d] = [dA dB] . [W1_e ; W3_e] : B(n = j, k = f) = W1[e][f][j], then W3 for k >= F
    if (e == cudaSuccess)
        e = launch_pdl(simt_gemm_bwd_kernel<true, false>, dim3((unsigned)(S / GT), (d + GT - 1) / GT), blk, 0, s,
                       view(dab, 0, 2 * F, 1), view(W1, (size_t)F * d, 1, d, W3, F), none, a.meta, E, 0, d, 2 * F,
                       static_cast<const float*>(nullptr), static_cast<float*>(a.dxp), static_cast<float*>(nullptr),
                       0);
    // dW2_e [d][F] = dY_e^T H_e
    if (e == cudaSuccess)
        e = launch_pdl(simt_gemm_bwd_kernel<false, false>, dim3((d + GT - 1) / GT, (F + GT - 1) / GT, E), blk, 0, s,
                       view(dy, 0, d, 1), view(H, 0, F, 1), none, a.meta, E, d, F, 0,
                       static_cast<const float*>(nullptr), a.dW2, a.dW2, d);
    // [dW1_e ; dW3_e] [2F][d] = [dA dB]_e^T Xp_e
    if (e == cudaSuccess)
        e = launch_pdl(simt_gemm_bwd_kernel<false, false>, dim3((2 * F + GT - 1) / GT, (d + GT - 1) / GT, E), blk, 0, s,
                       view(dab, 0, 2 * F, 1), view(xp, 0, d, 1), none, a.meta, E, 2 * F, d, 0,
                       static_cast<const float*>(nullptr), a.dW1, a.dW3, F);
    return e;
}

}  // namespace moe
