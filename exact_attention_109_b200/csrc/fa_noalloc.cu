// fa_noalloc.cu -- fa_bwd_noalloc: the backward pass for callers that cannot
// allocate device memory.
//
// fa_bwd needs a caller-provided workspace (an fp32 dQ accumulator plus two
// fp32 row vectors).  Some callers have no way to provide one: a plugin loaded
// by a host application that owns every byte of device memory through its
// own pool and hands extensions no allocator, or a latency-critical serving
// path that forbids cudaMalloc after start-up because the call can
// synchronise the device and take driver locks.  For them this entry point
// uses a fixed scratch array that lives in the library's device image
// instead.  The array is reserved on every GPU that loads the library and is
// held until the process exits, so its size is kept modest
// (FA_BWD_NOALLOC_MAX_WORKSPACE_BYTES).
#include <cuda_runtime.h>

#include <mutex>

#include "fa.h"

namespace {

constexpr size_t kScratchBytes = FA_BWD_NOALLOC_MAX_WORKSPACE_BYTES;
constexpr int kMaxDevices = 64;

// The workspace shared by every fa_bwd_noalloc call on a device.  In host code
// this name is only a stand-in for the device object; its device address comes
// from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

// Device address of the array, per device; null until a lookup succeeds.
// Only a successful lookup is cached: a failed one (for instance a first call
// made while a stream was being captured, or a sticky error from earlier
// work) is reported to that caller, and the next call tries again.
std::mutex g_scratch_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

}  // namespace

extern "C" fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                                    const float* lse, const void* dO, void* dq, void* dk,
                                    void* dv, int B, int H, int N, int d, int causal,
                                    float scale, void* stream) {
    // Size checks first: nothing is touched for a problem the scratch cannot hold.
    if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
    const size_t need = fa_bwd_workspace_size(B, H, N, d);
    if (need == 0 || need > kScratchBytes) return FA_ERR_INVALID_ARG;

    // One-time set-up per device, with that device current: look up the
    // scratch array's device address (this also loads the library's device
    // image on the device if it is not loaded yet).
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FA_ERR_CUDA;
    void* scratch = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_scratch_mutex);
        if (g_scratch_ptr[dev] == nullptr) {
            void* ptr = nullptr;
            if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) {
                (void)cudaGetLastError();  // do not leave the lookup's error behind
                return FA_ERR_CUDA;
            }
            g_scratch_ptr[dev] = ptr;
        }
        scratch = g_scratch_ptr[dev];
    }

    // The existing backward pass, pointed at the scratch array.  Its first
    // stage rewrites every workspace word it later reads (it zeroes the dQ
    // accumulator and refills the row vectors), so leftovers from an earlier
    // call never leak into this one.
    return fa_bwd(q, k, v, o, lse, dO, dq, dk, dv, B, H, N, d, causal, scale, scratch,
                  kScratchBytes, stream);
}
