// moe_combine_noalloc: moe_combine for callers that cannot allocate device
// memory.
//
// Some callers of this library may not call cudaMalloc (or any allocator) on
// the path where they run the layer: a plugin inside an inference engine or
// framework that owns and pre-plans every byte of device memory, code that
// runs under a fixed memory budget, or code that must not trigger the device
// synchronisation an allocation can cause.  moe_combine needs an fp32
// accumulator of T*d floats for bf16 outputs, which such a caller cannot
// provide.  This entry point keeps that accumulator in a fixed-size array of
// static device memory instead, so it needs nothing from the caller beyond its
// inputs and outputs, and it calls no allocating routine itself.
//
// Costs and rules of the static array:
//  - every GPU that loads the library holds it (kNoAllocAccFloats floats,
//    16 MiB) until the process exits;
//  - it bounds the call: T * d (T * k * d for the ordered combine, whose slot
//    rows it then holds) must not exceed kNoAllocAccFloats;
//  - every call on a device shares it, and its contents are undefined
//    between calls; each call clears the part it uses before accumulating,
//    and calls whose executions overlap on the GPU (different streams, no
//    ordering) race on it and produce wrong results.
#include <mutex>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr size_t kNoAllocAccFloats = MOE_NOALLOC_MAX_ACC_FLOATS;

// The accumulator.  In host code this name is only a stand-in for the symbol,
// not a device address: kernels get the address from cudaGetSymbolAddress.
static __device__ __align__(256) float g_noalloc_acc[kNoAllocAccFloats];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
float *g_acc_ptr[kMaxDevices];

// Device address of g_noalloc_acc on the current device, looked up once per
// device (with that device current).  Returns nullptr on failure.
float *acc_ptr() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_acc_ptr[dev]) {
        float *p = nullptr;
        if (cudaGetSymbolAddress(reinterpret_cast<void **>(&p), g_noalloc_acc) != cudaSuccess) return nullptr;
        g_acc_ptr[dev] = p;
    }
    return g_acc_ptr[dev];
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" moe_status moe_combine_noalloc(const moe_config *c, const void *act, const void *w_down,
                                          const int32_t *offsets, const int32_t *sorted_rows, const float *gates,
                                          void *y, void *stream) {
    moe_status st = moe_validate(c);
    if (st != MOE_OK) return st;
    if (c->T == 0) return MOE_OK;
    if (!act || !w_down || !offsets || !sorted_rows || !gates || !y) return MOE_ERR_INVALID_ARG;
    const size_t need = combine_scratch_floats(*c);
    if (need > kNoAllocAccFloats) return MOE_ERR_WORKSPACE;
    uint32_t *err = device_error_word();
    float *buf = need ? acc_ptr() : nullptr;
    if (!err || (need && !buf)) return MOE_ERR_CUDA;
    const cudaError_t e = launch_combine(*c, act, w_down, offsets, sorted_rows, gates, y, buf,
                                         static_cast<cudaStream_t>(stream), err);
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
