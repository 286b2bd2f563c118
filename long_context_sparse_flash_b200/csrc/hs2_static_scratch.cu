// hs2_static_scratch.cu -- hs2_full_attn_select_static: the full-attention +
// selection layer for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocating routine) at the point
// where they run this layer: code that runs inside a host process whose
// device memory is owned by a pre-sized pool it may not grow, plugin or
// embedded runtimes that hand out only the input and output buffers, and
// steps that must not synchronise the device (cudaMalloc and cudaFree can).
// hs2_full_attn_select needs a caller-provided workspace for the selection
// pass; this entry point instead uses one fixed scratch array that lives in
// this file as a static __device__ array.
#include <mutex>

#include "hs2_kernels.h"

namespace hs2 {
namespace {

// The scratch: the 256-byte error-word header followed by the selection
// scores.  Every GPU that loads this library holds these bytes until exit.
constexpr size_t kStaticScratchBytes = size_t(HS2_STATIC_SCRATCH_BYTES);
__device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_static_scratch on the current device.  In host code the
// array's name is only a host-side stand-in, so the address comes from
// cudaGetSymbolAddress, once per device, with that device current.
hs2_status scratch_address(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return HS2_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_scratch_ptr[dev] == nullptr) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_static_scratch) != cudaSuccess || ptr == nullptr) return HS2_ERR_CUDA;
        g_scratch_ptr[dev] = ptr;
    }
    *out = g_scratch_ptr[dev];
    return HS2_OK;
}

}  // namespace
}  // namespace hs2

extern "C" hs2_status hs2_full_attn_select_static(const hs2_shape* shape, const void* q, const void* k,
                                                  const void* v, void* out, float* lse, int32_t* idx,
                                                  hs2_stream_t stream) {
    const size_t need = hs2_workspace_size(shape, HS2_ENTRY_FULL_SELECT);
    if (need == 0) {
        // an invalid shape: let the allocating entry point report which check failed
        return hs2_full_attn_select(shape, q, k, v, out, lse, idx, nullptr, 0, stream);
    }
    if (need > hs2::kStaticScratchBytes) return HS2_ERR_WORKSPACE;
    void* scratch = nullptr;
    const hs2_status s = hs2::scratch_address(&scratch);
    if (s != HS2_OK) return s;
    // the array keeps the previous call's contents: the error word must start at zero
    if (cudaMemsetAsync(scratch, 0, sizeof(hs2::WsHeader), reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
        return HS2_ERR_CUDA;
    return hs2_full_attn_select(shape, q, k, v, out, lse, idx, scratch, hs2::kStaticScratchBytes, stream);
}

extern "C" size_t hs2_static_scratch_bytes(void) { return hs2::kStaticScratchBytes; }

// The error word of the static array: what the last hs2_full_attn_select_static
// call on this device reported (the next call clears it first).  Synchronises
// the stream; copies the word to host memory on the stack and clears it;
// allocates nothing.
extern "C" hs2_status hs2_static_scratch_status(hs2_stream_t stream, uint32_t* info) {
    void* scratch = nullptr;
    const hs2_status s = hs2::scratch_address(&scratch);
    if (s != HS2_OK) return s;
    return hs2_get_device_status(scratch, stream, info);
}
