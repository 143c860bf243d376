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
// kernel (on the host it is only a stand-in symbol); its device address is looked up once
// per device with cudaGetSymbolAddress, with that device current, on the first call made
// on that device.
#include <mutex>

#include "common.cuh"
#include "launch.h"

#define MOE_EXPORT __attribute__((visibility("default")))

namespace moe {
namespace {

constexpr size_t kScratchBytes = MOE_PERMUTE_NO_ALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

// The scratch: one int32 per (histogram block, expert).  Nothing in it has to start at zero:
// the histogram kernel of every call overwrites each entry that the scan and scatter kernels
// of the same call later read.  Calls that overlap on the GPU (on different streams, or on
// the same device from different threads without ordering) share this array and race.
static __device__ __align__(256) int32_t g_permute_scratch[kScratchBytes / sizeof(int32_t)];

std::mutex g_mutex;
int32_t* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch on the current device (looked up once per device).
moe_status_t scratch_for_current_device(int32_t** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_permute_scratch) != cudaSuccess || !p) return MOE_ERR_CUDA;
        g_scratch_ptr[dev] = static_cast<int32_t*>(p);
    }
    *out = g_scratch_ptr[dev];
    return MOE_OK;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" MOE_EXPORT moe_status_t moe_permute_no_alloc(const moe_shape_t* s, const int32_t* topk_idx,
                                                        const float* topk_gate, int32_t* counts, int32_t* offsets,
                                                        int32_t* sorted_token, float* sorted_gate, int32_t* slot_of,
                                                        moe_stream_t stream) {
    if (!s || (s->dtype != MOE_F32 && s->dtype != MOE_BF16)) return MOE_ERR_INVALID_ARG;
    if (s->T < 0 || s->n_experts < 1 || s->top_k < 1 || s->top_k > s->n_experts) return MOE_ERR_INVALID_ARG;
    if (s->n_experts > 1024 || s->top_k > 32 || (long long)s->T * s->top_k >= (1LL << 31)) return MOE_ERR_UNSUPPORTED;
    if (!counts || !offsets || (s->T > 0 && (!topk_idx || !topk_gate || !sorted_token || !sorted_gate || !slot_of)))
        return MOE_ERR_INVALID_ARG;
    Dims D = {};
    D.T = s->T; D.d = s->d; D.E = s->n_experts; D.I = s->inter; D.k = s->top_k;
    D.Ks = 0; D.Is = 0; D.bias = false; D.bf16 = s->dtype == MOE_BF16;
    const long long nblk = permute_blocks(D);
    const long long need = (nblk > 0 ? nblk : 1) * (long long)D.E * (long long)sizeof(int32_t);
    if (need > (long long)kScratchBytes) return MOE_ERR_UNSUPPORTED;   // beyond the fixed scratch
    int32_t* scratch = nullptr;
    moe_status_t st = scratch_for_current_device(&scratch);
    if (st != MOE_OK) return st;
    cudaGetLastError();
    if (launch_permute(D, topk_idx, topk_gate, counts, offsets, sorted_token, sorted_gate, slot_of, scratch, nullptr,
                       (cudaStream_t)stream) != cudaSuccess)
        return MOE_ERR_CUDA;
    return MOE_OK;
}
