/*
 * moe.h -- C ABI of the B200 (sm_100a) sparse mixture-of-experts feed-forward layer.
 *
 * The layer is the Mixtral-style top-k MoE FFN described on the page
 * "Mistral/Mixtralのアーキテクチャ — Sliding Window AttentionとMoEの融合"
 * (disassemble-channel.com/mistral-mixtral-architecture), section
 * "MoEの数学 — ルーターとゲーティング機構".  Per token x (a row of length d):
 *
 *   s   = Wg x                      router scores, Wg in R^{E x d}, no bias
 *                                   (subsection "Top-2ゲーティングの定式化")
 *   i_1..i_k = the k largest scores, s_i1 >= s_i2 >= ...; equal scores go to
 *                                   the lower expert index
 *   g_j = exp(s_ij) / sum_m exp(s_im)   softmax over the selected k only
 *   E_i(x) = W2_i (SiLU(W1_i x) * W3_i x),  SiLU(a) = a sigmoid(a)
 *                                   (subsection "各エキスパートの構造")
 *   out = g_1 E_i1(x) + ... + g_k E_ik(x), summed in that order
 *
 * Layouts (row-major, the nn.Linear weight convention of the page's
 * "MoEレイヤー全体の実装" code; every GEMM operand is contiguous along its
 * reduction axis):
 *   x   [T][d]          Wg [E][d]
 *   W1  [E][F][d]       W3 [E][F][d]       W2 [E][d][F]      (F = ffn)
 *   out [T][d]
 *   topk_idx [T][k] int32, topk_w [T][k] float   (slot j = j-th largest score)
 *
 * Element types: the plain entry points take bfloat16 tensors (bit patterns,
 * IEEE bfloat16, passed as void*), accumulate in fp32 and round the output to
 * bfloat16 (round to nearest even).  The *_f32 entry points take and return
 * float and compute in fp32 throughout (no TF32).
 *
 * Pointers: "device" means memory the current CUDA device can address
 * (cudaMalloc, cudaMallocAsync, torch CUDA tensors); "host" means ordinary or
 * pinned host memory.  Every pointer must be 16-byte aligned.  The caller owns
 * every buffer; the library keeps no pointer past the call.  Outputs are fully
 * overwritten, never accumulated into.  A call runs on the device that owns its
 * first device buffer (the current device for the host entry points), and
 * leaves the calling thread's current device as it found it.
 *
 * Streams: every call is stream-ordered on `stream` (0 = legacy default
 * stream) and returns without synchronising, except moe_forward_host and
 * moe_get_device_status, which synchronise `stream`.  Calls are reentrant;
 * calls on different streams may run concurrently, each with its own
 * workspace.
 *
 * Errors: argument checks run on the host before anything is launched and
 * return MOE_ERR_INVALID_ARG / MOE_ERR_UNSUPPORTED with nothing launched.  A
 * failed launch or allocation returns MOE_ERR_CUDA / MOE_ERR_WORKSPACE.  Faults
 * found on the device while kernels run (an expert index out of range, a
 * pipeline wait that ran past its time limit) do not trap: the kernel records
 * the first one in a per-device status word, stops its own work, releases what
 * it holds and returns; read the word with moe_get_device_status.  Outputs of a
 * call that recorded a device fault are unspecified.  Inputs are assumed
 * finite: the layer's definition says nothing about NaN or Inf.
 *
 * Supported sizes: 1 <= k <= E <= 32, T >= 0 (T == 0 is a no-op returning
 * MOE_OK).  bfloat16 entry points: d % 64 == 0, F % 128 == 0.  fp32 entry
 * points: d % 4 == 0, F >= 1.  T * k must stay below 2^31.
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,  /* null pointer, negative size, k > E, misaligned pointer */
    MOE_ERR_UNSUPPORTED = 2,  /* valid layer, but a size this library does not handle */
    MOE_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed */
    MOE_ERR_TIMEOUT = 4,      /* device: a pipeline wait ran past its time limit */
    MOE_ERR_WORKSPACE = 5,    /* workspace missing or smaller than moe_workspace_size() */
    MOE_ERR_DEVICE = 6        /* device: an input failed a kernel's own check (index range) */
} moe_status;

/* path selection for moe_forward_ws */
enum {
    MOE_PATH_AUTO = 0,    /* decode path when T <= moe_decode_max_tokens(), else grouped GEMMs */
    MOE_PATH_PREFILL = 1, /* gather + tensor-core grouped GEMMs (CTA pairs, 256-row tiles) */
    MOE_PATH_DECODE = 2,  /* expert-weight streaming, weights as the MMA's M side
                             (bfloat16 only, T <= moe_decode_max_tokens()) */
    MOE_PATH_TRAIN = 3    /* the grouped-GEMM path, and the workspace keeps what
                             moe_backward_ws needs (bfloat16: GEMM1's a = W1 x and
                             b = W3 x in fp32); workspace of moe_train_workspace_size() */
};

enum { MOE_DTYPE_F32 = 0, MOE_DTYPE_BF16 = 1 };

/*
 * Routing alone (router scores, top-k, softmax over the selected k): steps
 * "s = Wg x", "Top-2(s)" and the gate equation of subsection
 * "Top-2ゲーティングの定式化"; the page's MoERouter.forward in
 * "簡易MoEルーターの実装" returns the same (weights, indices) pair.
 *   x [T][d] bf16 (device), Wg [E][d] bf16 (device)
 *   topk_idx [T][k] int32 (device, out), topk_w [T][k] float (device, out)
 * Scores are accumulated in fp32 and never rounded to bf16.
 */
MOE_API moe_status moe_route(const void* x, const void* Wg, int T, int d, int E, int k,
                     int32_t* topk_idx, float* topk_w, cudaStream_t stream);

/* moe_route for float x [T][d] and Wg [E][d] (device). */
MOE_API moe_status moe_route_f32(const float* x, const float* Wg, int T, int d, int E, int k,
                         int32_t* topk_idx, float* topk_w, cudaStream_t stream);

/*
 * Number of rows of the expert-contiguous buffers that moe_dispatch fills:
 * each expert's segment is padded up to a multiple of 128 rows, so this is
 * T*k + E*127 rounded up to a multiple of 128.
 */
MOE_API size_t moe_slots_capacity(int T, int E, int k);

/*
 * Counting-sort dispatch of the routed tokens: the per-expert batching that
 * the page's "MoEレイヤー全体の実装" code does with one mask per expert
 * (x[mask] for the tokens that chose expert i), done as one stable pass.
 *   topk_idx [T][k] int32 (device, in): expert ids in [0, E)
 *   counts   [E]   int32 (device, out): assignments per expert
 *   offsets  [E+1] int32 (device, out): start row of each expert's segment;
 *                  offsets[e+1] - offsets[e] = counts[e] rounded up to 128
 *   perm     [moe_slots_capacity(T,E,k)] int32 (device, out): for each row of
 *                  a segment, the assignment t*k + j it holds, or -1 on a
 *                  padding row; rows past offsets[E] are left untouched
 *   inv      [T][k] int32 (device, out): the row that assignment (t, j) went to
 * Within a segment, rows are in increasing token order (stable).  Scratch
 * memory comes from the library's stream-ordered pool on `stream`.  An
 * expert id out of range records MOE_ERR_DEVICE in the status word.
 */
MOE_API moe_status moe_dispatch(const int32_t* topk_idx, int T, int E, int k, int32_t* counts,
                        int32_t* offsets, int32_t* perm, int32_t* inv, cudaStream_t stream);

/*
 * moe_dispatch for callers that cannot allocate device memory (no
 * counterpart on the pages: an interface addition of this library).
 *
 * Some callers may not request device memory at call time: a plugin inside
 * an inference runtime that is handed fixed buffers and forbidden to
 * allocate, or a service that reserves all its memory at start-up.
 * moe_dispatch takes its scratch from the library's memory pool, and creating
 * or growing that pool allocates; this call never allocates.  Arguments,
 * outputs and results are those of moe_dispatch, bit for bit.
 *
 * Scratch: one 16 KiB array compiled into the library, on every device that
 * loads it, held until the process exits.  Limit: ceil(T / 1024) * E <= 3968
 * (for example T <= 507,904 with E = 8, T <= 126,976 with E = 32); above it
 * the call returns MOE_ERR_UNSUPPORTED and launches nothing.  Every call
 * shares that array and finds the previous call's contents in it (each call
 * writes every entry before reading it); calls whose kernels overlap on the
 * GPU (other streams, other host threads) race on it.  The first call on a
 * device, with that device current, looks up the array's device address
 * once; make that call before any stream capture begins.
 *
 * One check is stricter than moe_dispatch's: `counts` must be device memory
 * (it picks the device whose copy of the array is used).  A host or
 * unregistered `counts` returns MOE_ERR_INVALID_ARG with nothing launched,
 * where moe_dispatch would launch on the current device and fail later.
 */
MOE_API moe_status moe_dispatch_noalloc(const int32_t* topk_idx, int T, int E, int k, int32_t* counts,
                                        int32_t* offsets, int32_t* perm, int32_t* inv, cudaStream_t stream);

/*
 * Bytes the library's stream-ordered memory pool on `device` holds
 * (reserved) and has handed out (used) at this moment, as the CUDA pool
 * attributes report them; both 0 if no call has created that pool yet.  An
 * observability call (no counterpart on the pages): it launches and
 * synchronises nothing, so allocations still queued on a stream may not be
 * counted yet.  reserved, used: host (out).  MOE_ERR_INVALID_ARG for a null
 * pointer or a device index outside [0, 64).
 */
MOE_API moe_status moe_pool_stats(int device, size_t* reserved, size_t* used);

/*
 * The whole layer (route, dispatch, experts, combine) with bfloat16 tensors
 * (all device): x [T][d], Wg [E][d], W1/W3 [E][F][d], W2 [E][d][F], out [T][d].
 * The workspace comes from the library's stream-ordered pool on `stream`
 * (cudaMallocAsync semantics: no host synchronisation).
 */
MOE_API moe_status moe_forward(const void* x, const void* Wg, const void* W1, const void* W3,
                       const void* W2, void* out, int T, int d, int ffn, int E, int k,
                       cudaStream_t stream);

/* moe_forward with float tensors (all device), fp32 arithmetic throughout. */
MOE_API moe_status moe_forward_f32(const float* x, const float* Wg, const float* W1, const float* W3,
                           const float* W2, float* out, int T, int d, int ffn, int E, int k,
                           cudaStream_t stream);

/* Bytes of workspace moe_forward_ws needs for this layer (dtype: MOE_DTYPE_*). */
MOE_API size_t moe_workspace_size(int T, int d, int ffn, int E, int k, int dtype);

/*
 * moe_forward / moe_forward_f32 with a caller-provided device workspace of
 * at least moe_workspace_size() bytes (256-byte aligned), and an explicit
 * path (MOE_PATH_*; the decode path needs dtype == MOE_DTYPE_BF16).  The
 * workspace must not be in use by another call in flight.  After one call on
 * a device, calls can be captured into a CUDA graph (stream capture) and the
 * graph replayed with the same operands and workspace.
 */
MOE_API moe_status moe_forward_ws(const void* x, const void* Wg, const void* W1, const void* W3,
                          const void* W2, void* out, int T, int d, int ffn, int E, int k,
                          int dtype, int path, void* workspace, size_t workspace_bytes,
                          cudaStream_t stream);

/* Workspace bytes of moe_forward_ws / moe_forward_profiled with MOE_PATH_TRAIN. */
MOE_API size_t moe_train_workspace_size(int T, int d, int ffn, int E, int k, int dtype);

/* Stages of one layer call, in launch order (moe_forward_profiled). */
enum {
    MOE_STAGE_ROUTE = 0,    /* scores, top-k, gates */
    MOE_STAGE_DISPATCH = 1, /* histogram, scan, stable scatter */
    MOE_STAGE_GATHER = 2,   /* token rows into expert segments */
    MOE_STAGE_EXPERT1 = 3,  /* W1/W3 GEMM with SwiGLU (or the decode pass over W1/W3) */
    MOE_STAGE_EXPERT2 = 4,  /* W2 GEMM (or the decode pass over W2) */
    MOE_STAGE_COMBINE = 5,  /* gate-weighted sum */
    MOE_NUM_STAGES = 6
};

/*
 * moe_forward_ws that also records stage_events[i] (cudaEvent_t, created by
 * the caller with timing enabled, device-side only) on `stream` just before
 * stage i is launched, and stage_events[MOE_NUM_STAGES] after the last stage,
 * so cudaEventElapsedTime of consecutive events gives each stage's device
 * time.  stage_events may be NULL.  If `launches` is not NULL it receives the
 * number of kernels the call launched.
 */
MOE_API moe_status moe_forward_profiled(const void* x, const void* Wg, const void* W1, const void* W3,
                                        const void* W2, void* out, int T, int d, int ffn, int E, int k,
                                        int dtype, int path, void* workspace, size_t workspace_bytes,
                                        cudaEvent_t* stage_events, int* launches, cudaStream_t stream);

/*
 * End-to-end call from host memory: copies x_host [T][d] (host, bf16) to the
 * device, runs moe_forward with the device-resident weights (device), copies
 * the result back into out_host [T][d] (host, bf16) and synchronises
 * `stream`.  Pinned host buffers give full copy bandwidth; pageable ones work.
 * From 4096 tokens on the batch runs in chunks on two library-owned copy
 * streams, so that copies overlap the layer (moe_host_chunk_plan gives them).
 * The result is bit for bit that of one call on the whole batch.
 */
MOE_API moe_status moe_forward_host(const void* x_host, const void* Wg, const void* W1, const void* W3,
                            const void* W2, void* out_host, int T, int d, int ffn, int E, int k,
                            cudaStream_t stream);

/*
 * The chunk plan moe_forward_host uses for a batch of T tokens (host only, no
 * device needed): writes the first token of each chunk to starts[0..n-1] and T
 * to starts[n] (starts: host, max_chunks + 1 ints, caller-owned) and returns
 * the chunk count n: 1 below 4096 tokens, 2 (halves) below 8192, then a
 * 1024-token first and last chunk around near-equal middle ones of up to 7168
 * tokens below 12288, else 2560-token first and last chunks around middle
 * ones of up to 11264 (at most 64 chunks in all; past that the middle ones
 * grow).  Returns
 * 0 with nothing written if T < 0, starts is NULL or n would exceed
 * max_chunks.  Chunks are runs of consecutive tokens; tokens are independent
 * (each token's routing and expert rows depend on that token alone, per the
 * Top-2 gating and expert equations of the Mistral/Mixtral page), which is why
 * the chunked call returns the bits of one call.
 */
MOE_API int moe_host_chunk_plan(int T, int* starts, int max_chunks);

/*
 * Synchronises `stream`, then returns and clears the current device's status
 * word: MOE_OK, MOE_ERR_TIMEOUT or MOE_ERR_DEVICE (the first fault recorded
 * since the last read), or MOE_ERR_CUDA if the synchronisation itself failed.
 */
MOE_API moe_status moe_get_device_status(cudaStream_t stream);

/*
 * Self-test of the device fault path: launches one CTA that waits on a
 * shared-memory barrier that nothing ever arrives at, with a time limit of
 * limit_ns nanoseconds (1e3 <= limit_ns <= 1e10).  The wait gives up, records
 * MOE_ERR_TIMEOUT in the status word and the kernel returns normally; read
 * the result with moe_get_device_status.  Nothing faults or hangs.
 */
MOE_API moe_status moe_selftest_wait_timeout(long long limit_ns, cudaStream_t stream);

/* Static description of a status code. */
MOE_API const char* moe_status_string(moe_status status);

/* Token count at or below which MOE_PATH_AUTO takes the decode path. */
MOE_API int moe_decode_max_tokens(void);

/* ------------------------------------------------------------------------
 * Block form: the MoE sub-layer of a Mixtral Transformer block, section
 * "Mixtral 8x7B — Sparse MoEの導入", subsection "Mixtralのアーキテクチャ" of the
 * same page (RMSNorm, then the MoE layer, then the residual connection):
 *
 *   u   = RMSNorm(h),  u_j = gamma_j h_j / sqrt((1/d) sum_i h_i^2 + eps)
 *   out = h + MoE(u)                    MoE as defined at the top of this file
 *
 * The page names RMSNorm without printing it; this is its usual definition,
 * with a per-channel gain gamma [d] and the caller's eps (>= 0; Mixtral-style
 * models use 1e-5).  Precision: each row's factor 1/sqrt(mean(h^2) + eps) is
 * computed in fp32; the router scores see the unrounded normalised row (they
 * are r * (Wg (gamma * h)) with exact fp32 products); the experts see u
 * rounded once to the operand type; the residual is added to the fp32
 * gate-weighted sum before the output is rounded once.  eps == 0 with an
 * all-zero row gives NaN, as the definition does.
 *
 * Load-balance statistics (optional, `stats`; subsection "ロードバランス損失"):
 *   f_e = (1/T) #{(t, j): topk_idx[t][j] == e}   (every one of the k selections)
 *   p_e = (1/T) sum_t softmax(s_t)_e             (softmax over all E scores)
 *   L   = alpha * E * sum_e f_e p_e
 * written as stats[0..E) = f, stats[E..2E) = p, stats[2E] = L (device, float,
 * 2E + 1 values).  The page's formula carries alpha and its code does not;
 * alpha = 1 gives the code's value.  Sums run in a fixed order: the same
 * inputs give the same bits on every run.
 *
 * h, out: [T][d] (device); gamma: [d] (device), same element type as h.
 * out may be h itself (the update is then in place); it must not overlap h in
 * any other way.  stats may be NULL (nothing is computed for it).
 * ------------------------------------------------------------------------ */

/* Workspace bytes moe_block_forward_ws needs (0 for invalid sizes or dtype). */
MOE_API size_t moe_block_workspace_size(int T, int d, int ffn, int E, int k, int dtype);

/* bfloat16 block; the workspace comes from a stream-ordered pool as in moe_forward. */
MOE_API moe_status moe_block_forward(const void* h, const void* gamma, float eps, const void* Wg,
                                     const void* W1, const void* W3, const void* W2, void* out, int T,
                                     int d, int ffn, int E, int k, float alpha, float* stats,
                                     cudaStream_t stream);

/* fp32 block (fp32 throughout). */
MOE_API moe_status moe_block_forward_f32(const float* h, const float* gamma, float eps, const float* Wg,
                                         const float* W1, const float* W3, const float* W2, float* out,
                                         int T, int d, int ffn, int E, int k, float alpha, float* stats,
                                         cudaStream_t stream);

/*
 * Block with a caller-provided workspace of at least moe_block_workspace_size()
 * bytes (device, 256-byte aligned, not in use by another call in flight), an
 * explicit path and dtype, and the optional stage events and launch count of
 * moe_forward_profiled (the statistics, when asked for, run in the route stage).
 * MOE_PATH_TRAIN also keeps what moe_block_backward_ws needs (the row factors,
 * the router scores and, bfloat16, GEMM1's a and b); it then needs
 * moe_block_train_workspace_size() bytes.
 */
MOE_API moe_status moe_block_forward_ws(const void* h, const void* gamma, float eps, const void* Wg,
                                        const void* W1, const void* W3, const void* W2, void* out, int T,
                                        int d, int ffn, int E, int k, float alpha, float* stats, int dtype,
                                        int path, void* workspace, size_t workspace_bytes,
                                        cudaEvent_t* stage_events, int* launches, cudaStream_t stream);

/*
 * moe_route (bfloat16) / moe_route_f32 plus the load-balance statistics of
 * that routing into stats (device, 2E + 1 floats, required).  Scratch comes
 * from the stream-ordered pool.
 */
MOE_API moe_status moe_route_stats(const void* x, const void* Wg, int T, int d, int E, int k, float alpha,
                                   int32_t* topk_idx, float* topk_w, float* stats, cudaStream_t stream);
MOE_API moe_status moe_route_stats_f32(const float* x, const float* Wg, int T, int d, int E, int k,
                                       float alpha, int32_t* topk_idx, float* topk_w, float* stats,
                                       cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Backward pass: gradients of a scalar loss L through the layer, given
 * dout = dL/dout [T][d].  The page trains the layer by gradient descent on
 * the language-model loss plus the load-balance loss (subsection
 * "ロードバランス損失"); these are the gradients of the equations at the top of
 * this file, with the top-k choice held fixed (it is piecewise constant):
 *
 *   dy_j = g_j dout,  dg_j = <dout, E_ij(x)>,  ds = g_j (dg_j - sum_m g_m dg_m)
 *   dh = W2^T dy,  da = dh * b * SiLU'(a),  db = dh * SiLU(a)   (a = W1 x, b = W3 x)
 *   dx = sum_j (W1^T da + W3^T db) + Wg^T ds
 *   dW2 += dy h^T,  dW1 += da x^T,  dW3 += db x^T,  dWg += ds x^T
 *
 * With alpha != 0 the loss also holds the load-balance loss alpha E sum f p
 * of the forward's routing (the page's total loss L_LM + L_balance): f is
 * piecewise constant, so every score of token t gets
 *   ds_te += (alpha E / T) softmax(s_t)_e (f_e - sum_m softmax(s_t)_m f_m)
 * before ds reaches dx and dWg.  alpha = 0 gives the output path alone.
 *
 * Use: run moe_forward_ws (or moe_forward_profiled) with MOE_PATH_TRAIN and
 * a workspace of moe_train_workspace_size() bytes on the same operands, then
 * pass that workspace here unchanged as fwd_workspace (device, read only).
 * The bfloat16 backward reads GEMM1's kept a and b instead of recomputing
 * them; the fp32 backward recomputes them.  workspace: at least
 * moe_backward_workspace_size() bytes (device, 256-byte aligned).
 * Outputs (device, overwritten): dx [T][d] in the layer's element type;
 * dWg [E][d] in float; dW1 [E][F][d], dW3 [E][F][d] and dW2 [E][d][F] in
 * wgrad_dtype: MOE_DTYPE_F32, or MOE_DTYPE_BF16 for a bfloat16 layer (the fp32
 * sums rounded once, half the bytes to write); dlogits [T][E] float
 * (optional, NULL allowed): the gradient of the router scores (zero for
 * unselected experts when alpha = 0).  Every sum runs in a fixed order (no
 * float atomics), so results are bitwise repeatable.  stage_events
 * (optional) receives MOE_BWD_NUM_STAGES + 1 events as in
 * moe_forward_profiled; launches (optional) the number of kernels launched.
 * ------------------------------------------------------------------------ */
enum {
    MOE_BWD_STAGE_SCATTER = 0,  /* dy = g dout into the expert segments, dg, ds */
    MOE_BWD_STAGE_DGRAD_H = 1,  /* dH = dY W2 (bfloat16: with the SwiGLU backward fused) */
    MOE_BWD_STAGE_SWIGLU = 2,   /* dA and dB (fp32 path: GEMM1 recomputed; bfloat16: empty) */
    MOE_BWD_STAGE_DGRAD_X = 3,  /* dXp = dA W1 + dB W3 */
    MOE_BWD_STAGE_WGRAD2 = 4,   /* dW2 */
    MOE_BWD_STAGE_WGRAD13 = 5,  /* dW1, dW3 */
    MOE_BWD_STAGE_ROUTER = 6,   /* dWg and the dx combine */
    MOE_BWD_NUM_STAGES = 7
};

MOE_API size_t moe_backward_workspace_size(int T, int d, int ffn, int E, int k, int dtype);

MOE_API moe_status moe_backward_ws(const void* x, const void* Wg, const void* W1, const void* W3,
                                   const void* W2, const void* dout, void* dx, float* dWg, void* dW1,
                                   void* dW3, void* dW2, float* dlogits, float alpha, int wgrad_dtype, int T,
                                   int d, int ffn, int E, int k, int dtype, const void* fwd_workspace,
                                   size_t fwd_workspace_bytes,
                                   void* workspace, size_t workspace_bytes, cudaEvent_t* stage_events,
                                   int* launches, cudaStream_t stream);

/*
 * Backward of the block form out = h + MoE(u), u = RMSNorm(h) (section
 * "Mixtral 8x7B — Sparse MoEの導入", subsection "Mixtralのアーキテクチャ", with
 * the training loss of subsection "ロードバランス損失").  With du = dL/du (the
 * layer backward above at x = u) and r = (mean_i h_i^2 + eps)^(-1/2) per row:
 *
 *   dh_i     = dout_i + r gamma_i du_i - (r^3 / d) h_i sum_j du_j gamma_j h_j
 *   dgamma_j = sum_t du_tj h_tj r_t
 *   dWg      = sum_t ds_t u_t^T   (u unrounded, as the router saw it)
 *
 * and dW1, dW3, dW2 as above with the experts' input u (rounded once to the
 * operand type, as the forward's experts saw it).  The residual passes dout to
 * h unchanged.  Use: moe_block_forward_ws with MOE_PATH_TRAIN and a workspace
 * of moe_block_train_workspace_size() bytes, then pass that workspace here as
 * fwd_workspace with the same h, gamma and weights.  Outputs (device,
 * overwritten): dh [T][d] in the layer's element type (must not overlap h or
 * dout), dgamma [d] float, the weight gradients and dlogits as in
 * moe_backward_ws.  d <= 8192 (MOE_ERR_UNSUPPORTED above: the dh pass keeps
 * one row of du in a thread block's registers).  Fixed-order sums throughout:
 * bitwise repeatable.  workspace: moe_block_backward_workspace_size() bytes.
 */
MOE_API size_t moe_block_train_workspace_size(int T, int d, int ffn, int E, int k, int dtype);
MOE_API size_t moe_block_backward_workspace_size(int T, int d, int ffn, int E, int k, int dtype);
MOE_API moe_status moe_block_backward_ws(const void* h, const void* gamma, const void* Wg, const void* W1,
                                         const void* W3, const void* W2, const void* dout, void* dh,
                                         float* dgamma, float* dWg, void* dW1, void* dW3, void* dW2,
                                         float* dlogits, float alpha, int wgrad_dtype, int T, int d, int ffn,
                                         int E, int k, int dtype, const void* fwd_workspace,
                                         size_t fwd_workspace_bytes, void* workspace, size_t workspace_bytes,
                                         cudaEvent_t* stage_events, int* launches, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Expert parallelism, the dispatch plan (host).  The summary page ("Mixtral of
 * Experts", its limitations lists) names expert parallelism: experts spread
 * over GPUs, each token's rows sent to the GPU that holds its chosen experts
 * and the outputs sent back, one all-to-all each way.  Experts are split into
 * R contiguous groups: rank s owns experts [s E / R, (s+1) E / R).
 *
 * counts_all [R][E] int32 (host, in): every rank's assignments per expert
 *   (each rank's moe_dispatch counts, gathered).
 * For rank `rank` (host, out; the caller owns every array):
 *   send_counts [R], send_offsets [R+1]: rows it sends to each rank, in its
 *     send order = its assignments sorted by expert, stable in token order
 *     (moe_dispatch's order without segment padding);
 *   recv_counts [R], recv_offsets [R+1]: rows it receives from each rank, the
 *     receive buffer ordered by source rank, each source's run as sent;
 *   expert_range [2]: its experts [lo, hi); with EL = hi - lo,
 *   seg_counts [EL], seg_offsets [EL+1]: its expert segments, padded to 128
 *     rows each (arrays of E and E+1 entries are always large enough);
 *   block_recv [R][EL], block_seg [R][EL]: the rows of source s for local
 *     expert l start at block_recv[s][l] in the receive buffer and at
 *     block_seg[s][l] in the segments; there are counts_all[s][lo + l] of them
 *     (arrays of R x E entries are always large enough).
 * Segment l holds source 0's rows, then source 1's, ...: with tokens numbered
 * source-major, each segment equals the single-GPU dispatch's segment of the
 * concatenated batch.  MOE_ERR_INVALID_ARG for a null pointer, R or E <= 0, a
 * rank outside [0, R) or a negative count; MOE_ERR_UNSUPPORTED for E > 32 or
 * more than 2^31 rows.
 * ------------------------------------------------------------------------ */
MOE_API moe_status moe_ep_plan(const int32_t* counts_all, int R, int E, int rank, int32_t* send_counts,
                               int32_t* send_offsets, int32_t* recv_counts, int32_t* recv_offsets,
                               int32_t* expert_range, int32_t* seg_counts, int32_t* seg_offsets,
                               int32_t* block_recv, int32_t* block_seg);

/*
 * Expert parallelism, the data plane (bfloat16): one rank's share of the layer
 * between its two all-to-alls, which the caller runs (NCCL through
 * torch.distributed, say) with the counts of moe_ep_plan.
 *
 * moe_ep_dispatch (route side, after moe_route): the counting sort of this
 * rank's assignments and its token rows copied into send order.
 *   x [T][d] bf16, topk_idx [T][k] int32 (device, in);
 *   send [T*k][d] bf16 (device, out): row p = the token row of the p-th
 *     assignment in send order (assignments sorted by expert, stable in token
 *     order; the rows for rank s are send[send_offsets[s] .. send_offsets[s+1]));
 *   send_pos [T][k] int32 (device, out): the send row of assignment (t, j);
 *   counts_host [E] int32 (host, out): assignments per expert, this rank's row
 *     of counts_all.  The call synchronises `stream` to return them.
 * moe_ep_experts (expert side): recv [recv_rows][d] bf16 (device, in) holds the
 *   rows this rank received, in the plan's receive order (recv_rows =
 *   recv_offsets[R]); counts_all [R][E] (host); W1, W3 [EL][F][d] and W2
 *   [EL][d][F] (device) are the weights of this rank's experts [lo, hi) only.
 *   The rows go into padded expert segments (each equal to the single-GPU
 *   dispatch's segment of the concatenated batch), the tensor-core grouped
 *   GEMMs run on them, and yrecv [recv_rows][d] float (device, out) receives
 *   each row's expert output in the receive order, ready to be sent back.
 *   Scratch comes from the library's pool; the call synchronises `stream` once
 *   (its small block tables are copied from host memory).
 * moe_ep_combine (route side, after the return all-to-all): ysend
 *   [T*k][d] float (device) in send order; out[t] = sum_j topk_w[t][j] *
 *   ysend[send_pos[t][j]], j ascending, in fp32, rounded once to bf16 (device,
 *   out [T][d]): the single-GPU combine's arithmetic.
 * Every output equals the single-GPU layer's bit for bit.  Sizes as the
 * bfloat16 layer: d % 64 == 0, ffn % 128 == 0, E <= 32; R <= 64.  The pages
 * describe the scheme (the summary page's limitations lists) without code.
 */
MOE_API moe_status moe_ep_dispatch(const void* x, const int32_t* topk_idx, int T, int d, int E, int k, void* send,
                                   int32_t* send_pos, int32_t* counts_host, cudaStream_t stream);
MOE_API moe_status moe_ep_experts(const void* recv, const int32_t* counts_all, int R, int E, int rank,
                                  const void* W1, const void* W3, const void* W2, int d, int ffn, float* yrecv,
                                  cudaStream_t stream);
MOE_API moe_status moe_ep_combine(const float* ysend, const float* topk_w, const int32_t* send_pos, int T, int d,
                                  int k, void* out, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H_ */
