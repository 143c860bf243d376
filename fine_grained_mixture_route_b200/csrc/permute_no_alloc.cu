// moe_permute_no_alloc: the per-expert grouping of moe_permute for callers that cannot
// allocate device memory at all.
//
// Who needs it: moe_permute takes its scratch (a per-block histogram table) from a
// caller-provided workspace.  Some callers have no way to provide one: a process whose
// framework has already handed every byte of device memory to its own caching allocator, a
// plug-in that is given raw input and output pointers but no allocator handle, or a
// latency-critical path that must not call cudaMalloc (which can synchronise the whole
// device).  This entry point keeps the scratch in a fixed-size array that is part of the
// library image, so the call itself allocates nothing.
//
// The array is MOE_PERMUTE_NO_ALLOC_SCRATCH_BYTES (1 MiB) of every GPU that loads the
// library, held until the process exits.  Host code must not pass the array's name to a
// kernel (on the host it is only a stand-in symbol); its device address is looked up with
// cudaGetSymbolAddress, with the device current, on the first call made in each CUDA context
// (each device's primary context, and again after cudaDeviceReset or in a context the caller
// created), and kept under that context's process-unique id.
#include <cuda.h>

#include <mutex>

#include "abi_checks.h"
#include "common.cuh"
#include "launch.h"

#define MOE_EXPORT __attribute__((visibility("default")))

namespace moe {
namespace {

constexpr size_t kScratchBytes = MOE_PERMUTE_NO_ALLOC_SCRATCH_BYTES;

// The scratch: one int32 per (histogram block, expert).  Nothing in it has to start at zero:
// the histogram kernel of every call overwrites each entry that the scan and scatter kernels
// of the same call later read.  Calls that overlap on the GPU (on different streams, or on
// the same device from different threads without ordering) share this array and race.
static __device__ __align__(256) int32_t g_permute_scratch[kScratchBytes / sizeof(int32_t)];

std::mutex g_mutex;

// Context ids (cuCtxGetId: unique for the life of the process, never reused) with the scratch
// address that was looked up in that context.  A context that is destroyed and replaced (for
// instance by cudaDeviceReset) gets a new id, so a stale address is never handed out.
constexpr int kMaxContexts = 64;
struct CachedAddress {
    unsigned long long ctx_id;
    int32_t* ptr;
};
CachedAddress g_cache[kMaxContexts] = {};
int g_cached = 0;

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Id of the calling thread's current context; false when it has none yet or the driver
// cannot tell.
bool current_context_id(unsigned long long* id) {
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static bool resolved = false;
    if (!resolved) {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = (CtxGetCurrentFn)f;
        f = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = (CtxGetIdFn)f;
        resolved = true;
    }
    if (!get_current || !get_id) return false;
    CUcontext ctx = nullptr;
    if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return false;
    return get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of the scratch in the current context (looked up on the first call there).
moe_status_t scratch_for_current_context(int32_t** out) {
    std::lock_guard<std::mutex> lock(g_mutex);
    unsigned long long id = 0;
    const bool have_id = current_context_id(&id);
    if (have_id)
        for (int i = 0; i < g_cached; ++i)
            if (g_cache[i].ctx_id == id) {
                *out = g_cache[i].ptr;
                return MOE_OK;
            }
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_permute_scratch) != cudaSuccess || !p) return MOE_ERR_CUDA;
    // the lookup makes the device's primary context current if no context was
    unsigned long long id2 = 0;
    if (current_context_id(&id2)) {
        if (g_cached == kMaxContexts) g_cached = 0;       // many contexts: start the table over
        g_cache[g_cached].ctx_id = id2;
        g_cache[g_cached].ptr = static_cast<int32_t*>(p);
        ++g_cached;
    }
    *out = static_cast<int32_t*>(p);
    return MOE_OK;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" MOE_EXPORT moe_status_t moe_permute_no_alloc(const moe_shape_t* s, const int32_t* topk_idx,
                                                        const float* topk_gate, int32_t* counts, int32_t* offsets,
                                                        int32_t* sorted_token, float* sorted_gate, int32_t* slot_of,
                                                        moe_stream_t stream) {
    Dims D = {};
    moe_status_t st = to_dims(s, &D);                     // the shape rules of moe_permute
    if (st != MOE_OK) return st;
    if (!counts || !offsets || (D.T > 0 && (!topk_idx || !topk_gate || !sorted_token || !sorted_gate || !slot_of)))
        return MOE_ERR_INVALID_ARG;
    const long long nblk = permute_blocks(D);
    const long long need = (nblk > 0 ? nblk : 1) * (long long)D.E * (long long)sizeof(int32_t);
    if (need > (long long)kScratchBytes) return MOE_ERR_UNSUPPORTED;   // beyond the fixed scratch
    st = check_device();
    if (st != MOE_OK) return st;
    int32_t* scratch = nullptr;
    st = scratch_for_current_context(&scratch);
    if (st != MOE_OK) return st;
    cudaGetLastError();
    if (launch_permute(D, topk_idx, topk_gate, counts, offsets, sorted_token, sorted_gate, slot_of, scratch, nullptr,
                       (cudaStream_t)stream) != cudaSuccess)
        return MOE_ERR_CUDA;
    return MOE_OK;
}
