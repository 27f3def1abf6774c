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

std::once_flag g_setup_once[kMaxDevices];
void *g_scratch_ptr[kMaxDevices];
cudaError_t g_setup_err[kMaxDevices];

// Device address of the scratch on the current device (set up on first use).
ret_status scratch_on_current_device(void **ptr) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return RET_ERR_UNSUPPORTED;
    }
    std::call_once(g_setup_once[dev], [dev] {
        void *p = nullptr;
        g_setup_err[dev] = cudaGetSymbolAddress(&p, g_chunkwise_scratch);
        g_scratch_ptr[dev] = p;
    });
    if (g_setup_err[dev] != cudaSuccess || !g_scratch_ptr[dev]) return RET_ERR_CUDA;
    *ptr = g_scratch_ptr[dev];
    return RET_OK;
}

}  // namespace

extern "C" ret_status ret_chunkwise_gate_static(const ret_desc *desc, int chunk, const void *Q,
                                                const void *K, const void *V,
                                                const float *state_in, float *state_out,
                                                const void *G, float gn_eps, void *Y,
                                                void *stream) {
    // Same argument checks as ret_chunkwise; then the scratch it would need.
    const size_t need = ret_workspace_size(desc, chunk, 0, 1);
    if (need > kScratchFloats * sizeof(float)) return RET_ERR_WORKSPACE;
    if (need == 0) {
        // Either the tensor-core path (no scratch) or arguments ret_chunkwise
        // rejects: it reports which.
        return ret_chunkwise(desc, chunk, Q, K, V, state_in, state_out, nullptr, G, gn_eps, Y,
                             nullptr, 0, stream);
    }
    void *scratch = nullptr;
    ret_status s = scratch_on_current_device(&scratch);
    if (s != RET_OK) return s;
    return ret_chunkwise(desc, chunk, Q, K, V, state_in, state_out, nullptr, G, gn_eps, Y, scratch,
                         kScratchFloats * sizeof(float), stream);
}
