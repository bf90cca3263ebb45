// fp32 expert GEMMs on the CUDA cores (the fp32 entry points' path; no TF32,
// whose 10-bit mantissa would miss a 1e-5 relative tolerance).
//
// Subsection "各エキスパートの構造" of the "Mistral/Mixtral architecture" page:
// per expert e and each of its rows (tokens) x,
//     GEMM1: H = SiLU(x W1_e^T) * (x W3_e^T)        [rows][F]
//     GEMM2: Y = H W2_e^T                           [rows][d]
// Rows are the expert-contiguous, 128-padded segments written by dispatch.
// A block computes a 64 x 64 output tile; each thread 4 x 4 outputs (two
// accumulator sets in GEMM1).  Sums run over K in ascending order.
#include "moe_common.cuh"

namespace moe {
namespace {

constexpr int TM = 64, TN = 64, TK = 16;

// Which expert owns padded row r (offsets non-decreasing, r < offsets[E]).
__device__ __forceinline__ int owner(const Meta* meta, int E, int r) {
    int e = 0;
    while (e + 1 < E && r >= meta->offsets[e + 1]) ++e;
    return e;
}

// C[m][n] over K for A [rows][K] (row stride K) and B [N][K] (row stride K).
template <bool SWIGLU>
__global__ void __launch_bounds__(256) simt_gemm_kernel(const float* __restrict__ A, const float* __restrict__ B1,
                                                        const float* __restrict__ B3, const Meta* __restrict__ meta,
                                                        int E, int K, int N, size_t b_expert_stride,
                                                        float* __restrict__ C) {
    pdl_trigger();
    pdl_wait();
    __shared__ float As[TK][TM + 4];
    __shared__ float B1s[TK][TN + 4];
    __shared__ float B3s[SWIGLU ? TK : 1][TN + 4];
    const int row0 = blockIdx.x * TM;
    const int total = meta->offsets[E];
    if (row0 >= total) return;
    const int e = owner(meta, E, row0);
    const int n0 = blockIdx.y * TN;
    const float* b1 = B1 + (size_t)e * b_expert_stride;
    const float* b3 = SWIGLU ? B3 + (size_t)e * b_expert_stride : nullptr;
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;

    float acc1[4][4], acc3[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc1[i][j] = acc3[i][j] = 0.f;

    for (int k0 = 0; k0 < K; k0 += TK) {
        // 64 x 16 tiles: 1024 elements, 4 per thread
        for (int l = threadIdx.x; l < TM * TK; l += 256) {
            const int r = l / TK, c = l % TK;
            const int kk = k0 + c;
            As[c][r] = (kk < K) ? A[(size_t)(row0 + r) * K + kk] : 0.f;
            const int n = n0 + r;
            const bool ok = (kk < K) && (n < N);
            B1s[c][r] = ok ? b1[(size_t)n * K + kk] : 0.f;
            if (SWIGLU) B3s[c][r] = ok ? b3[(size_t)n * K + kk] : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int c = 0; c < TK; ++c) {
            float a[4], b[4], bb[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = As[c][ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                b[j] = B1s[c][tx * 4 + j];
                if (SWIGLU) bb[j] = B3s[c][tx * 4 + j];
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    acc1[i][j] = fmaf(a[i], b[j], acc1[i][j]);
                    if (SWIGLU) acc3[i][j] = fmaf(a[i], bb[j], acc3[i][j]);
                }
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = row0 + ty * 4 + i;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = n0 + tx * 4 + j;
            if (n < N) {
                const float v = SWIGLU ? acc1[i][j] / (1.0f + expf(-acc1[i][j])) * acc3[i][j] : acc1[i][j];
                C[(size_t)r * N + n] = v;
            }
        }
    }
}

}  // namespace

cudaError_t launch_simt_gemm1_f32(const float* xp, const float* W1, const float* W3, const Meta* meta, int E, int d,
                                  int F, float* H, size_t slots, cudaStream_t s) {
    dim3 grid((unsigned)(slots / TM), (unsigned)((F + TN - 1) / TN));
    return launch_pdl(simt_gemm_kernel<true>, grid, dim3(256), 0, s, xp, W1, W3, meta, E, d, F, (size_t)F * d, H);
}

cudaError_t launch_simt_gemm2_f32(const float* H, const float* W2, const Meta* meta, int E, int d, int F, float* Y,
                                  size_t slots, cudaStream_t s) {
    dim3 grid((unsigned)(slots / TM), (unsigned)((d + TN - 1) / TN));
    return launch_pdl(simt_gemm_kernel<false>, grid, dim3(256), 0, s, H, W2, static_cast<const float*>(nullptr), meta,
                      E, F, d, (size_t)d * F, Y);
}

}  // namespace moe
