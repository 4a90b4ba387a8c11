// per_tensor_noalloc.cu -- fp8q_cast_per_tensor_noalloc: the per-tensor cast
// for callers that cannot allocate device memory.
//
// The ordinary per-tensor cast needs a small scratch buffer for the per-CTA
// partial maxima of its amax pass, and asks the caller for it.  Some callers
// cannot provide one: code that runs under an allocator owning all of the
// GPU's memory (a serving process that reserves HBM up front and forbids any
// other allocation), or code that must not call cudaMalloc because that call
// can synchronise the whole device.  For them this entry point keeps the
// scratch in a file-scope __device__ array that exists, once per GPU, from the
// moment the library is loaded until the process exits.
//
// In host code the array's name is only a host-side stand-in, never a device
// address; its device address is fetched with cudaGetSymbolAddress, once per
// device, with that device current, on the first call made on that device.
// The cached address belongs to the device's primary context: after
// cudaDeviceReset the context is rebuilt and the array may sit elsewhere, so
// this entry point must not be called again in that process.
#include <mutex>

#include "fp8q.h"
#include "fp8q_internal.h"

namespace fp8q {
namespace {

// room for kMaxPartials per-CTA maxima: 2048 x 4 bytes = 8 KiB per GPU.  The
// amax pass clamps its grid to kMaxPartials CTAs (one partial each), so every
// launch fits the array whatever the tensor's size or the device's SM count.
constexpr int kNoAllocPartials = kMaxPartials;
static_assert(kNoAllocPartials >= kMaxPartials, "the amax pass may write kMaxPartials partials");
static __device__ __align__(256) uint32_t g_noalloc_partials[kNoAllocPartials];

constexpr int kMaxDevices = 128;
std::mutex g_setup_mu;
uint32_t* g_scratch[kMaxDevices];  // device address of g_noalloc_partials, per device

// Device address of the scratch array on the current device.  The first call
// on a device looks it up (a runtime query, no allocation); later calls reuse
// the cached address.
fp8q_status scratch_on_current_device(uint32_t** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FP8Q_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_setup_mu);
    if (g_scratch[dev] == nullptr) {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_partials);
        if (e != cudaSuccess || p == nullptr) return FP8Q_ERR_CUDA;
        g_scratch[dev] = static_cast<uint32_t*>(p);
    }
    *out = g_scratch[dev];
    return FP8Q_OK;
}

bool fmt_ok(int f) { return f == FP8Q_E4M3FN || f == FP8Q_E5M2; }
bool dtype_ok(int t) { return t == FP8Q_F32 || t == FP8Q_F16 || t == FP8Q_BF16; }

}  // namespace
}  // namespace fp8q

using namespace fp8q;

extern "C" fp8q_status fp8q_cast_per_tensor_noalloc(const void* x, fp8q_dtype xt, int64_t numel,
                                                    fp8q_format fmt, uint8_t* q, float* scale_inv,
                                                    fp8q_stream_t stream) {
    if (!dtype_ok(xt)) return FP8Q_ERR_BAD_DTYPE;
    if (!fmt_ok(fmt)) return FP8Q_ERR_BAD_FORMAT;
    const int es = xt == FP8Q_F32 ? 4 : 2;
    if (numel < 0 || numel > INT64_MAX / es) return FP8Q_ERR_BAD_SHAPE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (!scale_inv) return FP8Q_ERR_NULL_POINTER;
    if ((uintptr_t)scale_inv % 4) return FP8Q_ERR_MISALIGNED;
    if (numel == 0) return launch_fill(scale_inv, 1, 1.0f, s);
    if (!x || !q) return FP8Q_ERR_NULL_POINTER;
    if ((uintptr_t)x % es) return FP8Q_ERR_MISALIGNED;
    uint32_t* scratch = nullptr;
    const fp8q_status st = scratch_on_current_device(&scratch);
    if (st != FP8Q_OK) return st;
    // Every slot the cast pass reads is written by the amax pass of the same
    // call, so nothing left over from an earlier call needs clearing.
    return launch_per_tensor(x, xt, numel, fmt, q, scale_inv, scratch, FP8Q_SCALE_IEEE, s);
}
