// moe_dispatch_noalloc: the counting-sort dispatch with its scratch in a
// fixed array compiled into this library, for callers that cannot allocate
// device memory.
//
// Who needs it: code that runs where device memory belongs to someone else
// and must not be requested at call time, e.g. a plugin inside an inference
// runtime that hands it fixed buffers and forbids allocation, or a service
// that reserves all its memory at start-up and must never allocate on the hot
// path.  moe_dispatch takes its small scratch (per-block histogram and the
// segment table) from the library's stream-ordered pool, and creating or
// growing that pool allocates; this entry point never does.
//
// The scratch is one static __device__ array of kNoAllocScratchBytes (16 KiB)
// on every device that loads the library, held until the process exits.  It
// holds the segment table (first 512 bytes) and the per-block histogram
// (ceil(T / 1024) x E int32 after it), so the entry point accepts
// ceil(T / 1024) * E <= 3968 and returns MOE_ERR_UNSUPPORTED above that.
// Every call reuses the same array and keeps the previous call's contents;
// nothing in it has to start at zero, because every call writes each entry
// before reading it.  Two calls whose kernels overlap on the GPU (different
// streams, or different host threads) use the same array and race.
//
// In host code the array's name is not a device address: the first call on a
// device, with that device current, resolves the address once with
// cudaGetSymbolAddress and caches it.  Make that first call before any stream
// capture begins.
#include <climits>
#include <mutex>

#include "moe_common.cuh"

namespace moe {

int* status_word(int dev);   // moe_api.cu: address of the device status word (no allocation)

namespace {

constexpr size_t kNoAllocScratchBytes = 16384;
constexpr size_t kNoAllocMetaBytes = 512;
constexpr size_t kNoAllocHistInts = (kNoAllocScratchBytes - kNoAllocMetaBytes) / sizeof(int32_t);
static_assert(sizeof(Meta) <= kNoAllocMetaBytes, "segment table must fit its slot");

static __device__ __align__(256) unsigned char g_dispatch_scratch[kNoAllocScratchBytes];

constexpr int kMaxNoAllocDevices = 64;
std::mutex g_noalloc_mu;
unsigned char* g_noalloc_ptr[kMaxNoAllocDevices] = {};

// Device address of g_dispatch_scratch on device `dev` (which is current).
unsigned char* scratch_on(int dev) {
    if (dev < 0 || dev >= kMaxNoAllocDevices) return nullptr;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        unsigned char* p = nullptr;
        if (cudaGetSymbolAddress((void**)&p, g_dispatch_scratch) != cudaSuccess) return nullptr;
        g_noalloc_ptr[dev] = p;
    }
    return g_noalloc_ptr[dev];
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" moe_status moe_dispatch_noalloc(const int32_t* topk_idx, int T, int E, int k, int32_t* counts,
                                           int32_t* offsets, int32_t* perm, int32_t* inv, cudaStream_t stream) {
    if (T < 0 || E <= 0 || k <= 0 || k > E) return MOE_ERR_INVALID_ARG;
    if (E > kMaxExperts) return MOE_ERR_UNSUPPORTED;
    if ((long long)T * k + (long long)E * kSegRows >= INT_MAX) return MOE_ERR_UNSUPPORTED;
    if ((size_t)dispatch_blocks(T) * (size_t)E > kNoAllocHistInts) return MOE_ERR_UNSUPPORTED;
    if (!counts || !offsets || (T > 0 && (!topk_idx || !perm || !inv))) return MOE_ERR_INVALID_ARG;
    const DeviceScope scope(counts, true);
    const int dev = scope.device();
    if (dev < 0) return MOE_ERR_INVALID_ARG;
    unsigned char* scratch = scratch_on(dev);
    int* status = status_word(dev);
    if (!scratch || !status) return MOE_ERR_CUDA;
    Meta* meta = reinterpret_cast<Meta*>(scratch);
    int32_t* blk = reinterpret_cast<int32_t*>(scratch + kNoAllocMetaBytes);
    cudaError_t e = cudaSuccess;
    if (T == 0) {
        e = cudaMemsetAsync(meta, 0, sizeof(Meta), stream);
    } else {
        e = launch_dispatch(topk_idx, T, E, k, blk, meta, perm, inv, status, stream);
    }
    if (e == cudaSuccess) e = cudaMemcpyAsync(counts, meta->counts, E * 4, cudaMemcpyDeviceToDevice, stream);
    if (e == cudaSuccess) e = cudaMemcpyAsync(offsets, meta->offsets, (E + 1) * 4, cudaMemcpyDeviceToDevice, stream);
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
