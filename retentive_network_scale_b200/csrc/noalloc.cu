// noalloc.cu -- ret_chunkwise_gate_static: the chunkwise forward with the
// GroupNorm + swish gate (Y only) for callers that may not allocate device
// memory at call time.  Its scratch is a fixed device array owned by this
// library instead of a caller-provided workspace.
//
// The scratch holds the fp32 O that the CUDA-core chunkwise kernel writes
// and the gate kernel normalises (the path taken for shapes the tensor-core
// kernel does not cover); the tensor-core path needs none.  Every element
// the kernels read from it is written earlier in the same call, so nothing
// needs clearing; it keeps the last call's contents.  All calls on one
// device share the array, so calls that overlap on the GPU (other streams,
// other threads) race on it.
#include <mutex>

#include "launch.h"
#include "retention.h"

namespace {

constexpr size_t kScratchFloats = RET_STATIC_SCRATCH_FLOATS;  // 16 MiB of fp32
constexpr int kMaxDevices = 64;

// Host code must not take this symbol's address as a device pointer: its
// device address comes from cudaGetSymbolAddress, once per device.
__device__ __align__(256) float g_chunkwise_scratch[kScratchFloats];

std::mutex g_setup_mu[kMaxDevices];
void *g_scratch_ptr[kMaxDevices];  // NULL until a lookup on that device succeeded

// Device address of the scratch on the current device, looked up on first
// use with that device current.  Only a successful lookup is kept; after a
// failure (for instance a first call made inside a stream capture) the
// CUDA error is cleared, so that it is not reported by a later, unrelated
// launch, and the next call tries again.
ret_status scratch_on_current_device(void **ptr) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return RET_ERR_UNSUPPORTED;
    }
    std::lock_guard<std::mutex> lock(g_setup_mu[dev]);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_chunkwise_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            return RET_ERR_CUDA;
        }
        g_scratch_ptr[dev] = p;
    }
    *ptr = g_scratch_ptr[dev];
    return RET_OK;
}

}  // namespace

extern "C" ret_status ret_chunkwise_gate_static(const ret_desc *desc, int chunk, const void *Q,
                                                const void *K, const void *V,
                                                const float *state_in, float *state_out,
                                                const void *G, float gn_eps, void *Y,
                                                void *stream) {
    // The description, the chunk and the G / Y pair are checked first, so
    // that these errors are the ones ret_chunkwise would report; then the
    // scratch this call needs against the array.
    ret_status s = ret::validate_desc(desc);
    if (s != RET_OK) return s;
    if (chunk < 1) return RET_ERR_ARG;
    if ((long long)desc->B * desc->L > 0 && (!G || !Y)) return RET_ERR_NULL;
    const size_t need = ret_workspace_size(desc, chunk, 0, 1);
    if (need > kScratchFloats * sizeof(float)) return RET_ERR_WORKSPACE;
    if (need == 0) {
        // Either the tensor-core path (no scratch) or arguments ret_chunkwise
        // rejects: it reports which.
        return ret_chunkwise(desc, chunk, Q, K, V, state_in, state_out, nullptr, G, gn_eps, Y,
                             nullptr, 0, stream);
    }
    void *scratch = nullptr;
    s = scratch_on_current_device(&scratch);
    if (s != RET_OK) return s;
    return ret_chunkwise(desc, chunk, Q, K, V, state_in, state_out, nullptr, G, gn_eps, Y, scratch,
                         kScratchFloats * sizeof(float), stream);
}
