// Allocation-free variant of m2rnn_backward.
//
// Some callers cannot allocate device memory at the point where they need
// gradients: real-time or embedded services that forbid allocator calls after
// start-up (an allocation can synchronise the device or fail under memory
// pressure), or hosts that hand this library only the tensors they already
// own.  m2rnn_backward needs
// a caller-allocated workspace for its scratch (the device status word, the
// per-(b, h) dW partials and the per-CTA recompute buffer); this entry point
// takes that scratch from a fixed array compiled into the library instead, so
// it allocates nothing.
//
// Costs and limits:
//  * every GPU that loads the library reserves kNoAllocScratchBytes (32 MiB)
//    for the array until the process exits, whether the entry point is used
//    or not;
//  * problems whose workspace (m2rnn_workspace_size(d, 1)) exceeds that size
//    are rejected with M2RNN_ERR_WORKSPACE before anything is launched;
//  * all calls share the one array, so calls whose kernels overlap on the GPU
//    (different streams, or different host threads without ordering between
//    their streams) race on it and produce garbage;
//  * the first call on a device looks up the array's device address (a CUDA
//    runtime query, no allocation); make that first call before any stream
//    capture begins.  The address is cached per device for the life of the
//    process, so the entry point must not be used across a device reset;
//  * a device-side wait that runs out is recorded in the array's status word,
//    which this entry point clears at the start of each call and does not
//    report (m2rnn_backward with your own workspace does).
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/m2rnn.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;
constexpr size_t kStatusBytes = 256;   // leading status word, as in the caller-provided workspace
constexpr int kMaxDevices = 64;

// The scratch lives in global memory of every device that loads the library.
// In host code `g_noalloc_scratch` names a host-side stand-in, never a device
// address: the device address is obtained with cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_mu;
void* g_addr[kMaxDevices] = {};

// Device address of the array on the current device (looked up once per device).
cudaError_t scratch_address(void** out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_addr[dev] == nullptr) {
        void* ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_addr[dev] = ptr;
    }
    *out = g_addr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" m2rnn_status m2rnn_backward_noalloc(const m2rnn_dims* d, const void* k, const void* v, const void* q,
                                               const float* f, const void* W, const float* ckpt, const void* dy,
                                               const float* dHT, float* dk, float* dv, float* dq, float* df,
                                               float* dW, float* dH0, m2rnn_stream_t stream) {
    const size_t need = m2rnn_workspace_size(d, 1);
    if (need == 0)   // invalid dims: let m2rnn_backward name the problem (it checks dims first)
        return m2rnn_backward(d, k, v, q, f, W, ckpt, dy, dHT, dk, dv, dq, df, dW, dH0, nullptr, 0, stream);
    if (need > kNoAllocScratchBytes) return M2RNN_ERR_WORKSPACE;
    void* ws = nullptr;
    if (scratch_address(&ws) != cudaSuccess) return M2RNN_ERR_CUDA;
    // The status word must start at zero; everything else the kernels write
    // before they read it.
    if (cudaMemsetAsync(ws, 0, kStatusBytes, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
        return M2RNN_ERR_CUDA;
    return m2rnn_backward(d, k, v, q, f, W, ckpt, dy, dHT, dk, dv, dq, df, dW, dH0, ws, need, stream);
}
