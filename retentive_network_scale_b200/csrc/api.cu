// api.cu -- the C ABI declared in include/retention.h: argument checks,
// parameter set-up and dispatch to the kernels.  Every check runs before
// any CUDA call, so a rejected call touches no device state.
#include <atomic>
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>

#include "common.cuh"
#include "launch.h"
#include "retention.h"

// Device status word latched by bounded waits inside kernels
// (RET_ERR_TIMEOUT); read and cleared by ret_last_device_status.
__device__ int g_ret_device_status = 0;

namespace ret {

static std::atomic<unsigned long long> g_launches{0};

void note_launches(int n) { g_launches.fetch_add((unsigned long long)n, std::memory_order_relaxed); }

int *device_status_word() {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_ret_device_status) != cudaSuccess) return nullptr;
    return static_cast<int *>(p);
}

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool valid_dtype(int d) { return d == RET_F32 || d == RET_BF16; }

ret_status check_desc(const ret_desc *d) {
    if (!d || !d->gamma) return RET_ERR_NULL;
    if (d->B < 0 || d->L < 0 || d->H < 1 || d->H > RET_MAX_HEADS) return RET_ERR_SHAPE;
    if (d->d_k < 1 || d->d_k > kMaxDk || d->d_v < 1 || d->d_v > kMaxDv || (d->d_v % 4) != 0)
        return RET_ERR_SHAPE;
    if (!valid_dtype(d->in_dtype) || !valid_dtype(d->out_dtype)) return RET_ERR_DTYPE;
    if (d->rotate != 0 && d->rotate != 1) return RET_ERR_ARG;
    if (d->rotate && ((d->d_k & 1) || !(d->theta_base > 0.0) || !std::isfinite(d->theta_base)))
        return RET_ERR_ARG;
    if (d->pos_offset < 0) return RET_ERR_ARG;
    for (int h = 0; h < d->H; ++h) {
        double g = d->gamma[h];
        if (!(g >= 0.0 && g <= 1.0)) return RET_ERR_ARG;  // also rejects NaN
    }
    return RET_OK;
}

ret_status check_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return RET_ERR_UNSUPPORTED;
    }
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
        cudaGetLastError();
        return RET_ERR_UNSUPPORTED;
    }
    return (major == 10 && minor == 0) ? RET_OK : RET_ERR_UNSUPPORTED;
}

void make_params(const ret_desc *d, Params *p) {
    std::memset(p, 0, sizeof(*p));
    p->B = d->B; p->H = d->H; p->L = d->L; p->dk = d->d_k; p->dv = d->d_v;
    p->rotate = d->rotate;
    p->pos_offset = d->pos_offset;
    p->seg_heads = 1;
    p->reverse = 0;
    p->seg_len = 0;
    for (int h = 0; h < d->H; ++h)
        p->log2g[h] = d->gamma[h] > 0.0 ? (float)std::log2(d->gamma[h]) : -INFINITY;
    if (d->rotate)
        for (int j = 0; j < d->d_k / 2; ++j)
            p->theta[j] = std::pow(d->theta_base, -2.0 * (double)j / (double)d->d_k);
}

ret_status from_cuda(cudaError_t e) { return e == cudaSuccess ? RET_OK : RET_ERR_CUDA; }

}  // namespace

ret_status validate_desc(const ret_desc *d) { return check_desc(d); }
void params_from_desc(const ret_desc *d, Params *p) { make_params(d, p); }

}  // namespace ret

using namespace ret;

extern "C" {

ret_status ret_msr_gammas(int H, double *gamma) {
    if (H < 1 || H > RET_MAX_HEADS) return RET_ERR_SHAPE;
    if (!gamma) return RET_ERR_NULL;
    for (int h = 0; h < H; ++h) gamma[h] = 1.0 - std::ldexp(1.0, -5 - h);
    return RET_OK;
}

const char *ret_status_string(ret_status s) {
    switch (s) {
        case RET_OK: return "ok";
        case RET_ERR_NULL: return "a required pointer is NULL";
        case RET_ERR_SHAPE: return "a size is negative or beyond the supported limits";
        case RET_ERR_DTYPE: return "unknown dtype code";
        case RET_ERR_ALIGN: return "a device pointer is not 16-byte aligned";
        case RET_ERR_ARG: return "invalid argument (gamma, chunk, rotation, eps or position)";
        case RET_ERR_WORKSPACE: return "workspace missing or too small";
        case RET_ERR_UNSUPPORTED: return "no sm_100 device is current";
        case RET_ERR_CUDA: return "a CUDA call or kernel launch failed";
        case RET_ERR_TIMEOUT: return "a bounded device wait gave up";
    }
    return "unknown status";
}

size_t ret_parallel_workspace_size(const ret_desc *desc) {
    if (check_desc(desc) != RET_OK) return 0;
    Params p;
    make_params(desc, &p);
    return parallel_tc_supported(p, desc->in_dtype == RET_BF16) ? parallel_tc_workspace(p) : 0;
}

ret_status ret_parallel(const ret_desc *desc, const void *Q, const void *K, const void *V,
                        void *O, void *workspace, size_t workspace_bytes, void *stream) {
    ret_status s = check_desc(desc);
    if (s != RET_OK) return s;
    const bool empty = (long long)desc->B * desc->L == 0;
    if (!empty && (!Q || !K || !V || !O)) return RET_ERR_NULL;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(workspace))
        return RET_ERR_ALIGN;
    const size_t need = empty ? 0 : ret_parallel_workspace_size(desc);
    if (need > 0 && (!workspace || workspace_bytes < need)) return RET_ERR_WORKSPACE;
    if ((s = check_device()) != RET_OK) return s;
    if (empty) return RET_OK;
    Params p;
    make_params(desc, &p);
    const bool in_bf16 = desc->in_dtype == RET_BF16, out_bf16 = desc->out_dtype == RET_BF16;
    if (parallel_tc_supported(p, in_bf16)) {
        int *status = device_status_word();
        if (!status) return RET_ERR_CUDA;
        return from_cuda(launch_parallel_tc(p, out_bf16, Q, K, V, O, workspace, status,
                                            (cudaStream_t)stream));
    }
    return from_cuda(launch_parallel_simt(p, in_bf16, out_bf16, Q, K, V, O, (cudaStream_t)stream));
}

size_t ret_workspace_size(const ret_desc *desc, int chunk, int want_O, int want_Y) {
    if (check_desc(desc) != RET_OK || chunk < 1) return 0;
    // The tensor-core kernel normalises in its epilogue; some of its shapes
    // need the streaming pass's workspace when rotated.  The CUDA-core
    // chunkwise path needs an fp32 O to normalise when only Y is requested.
    Params p;
    make_params(desc, &p);
    if (chunkwise_tc_supported(p, chunk, desc->in_dtype == RET_BF16))
        return chunkwise_tc_needs_prep(p, chunk) ? chunkwise_prep_bytes(p) : 0;
    if (want_Y && !want_O) return sizeof(float) * (size_t)desc->B * desc->H * desc->L * desc->d_v;
    return 0;
}

namespace {
// The chunk loop's CTAs (one per head and 128 value columns) would leave most
// of the 148 SMs idle.
bool few_heads(const ret::Params &p) { return (long long)p.B * p.H * ((p.dv + 127) / 128) < 64; }
}  // namespace

size_t ret_chunkwise_fast_size(const ret_desc *desc, int chunk) {
    if (check_desc(desc) != RET_OK || chunk < 1 || (long long)desc->B * desc->L == 0) return 0;
    Params p;
    make_params(desc, &p);
    if (!chunkwise_tc_supported(p, chunk, desc->in_dtype == RET_BF16)) return 0;
    const int S = auto_segments(p, chunk);
    size_t bytes = S > 1 ? segmented_bytes(p, S) : chunkwise_prep_bytes(p);
    // few heads on the one-launch shapes: room for its block sums too (a call
    // with a carried state takes the segments or the loop instead)
    if (few_heads(p) && onepass_supported(p, true, false)) bytes = std::max(bytes, onepass_bytes(p));
    return bytes;
}

size_t ret_chunkwise_prep_size(const ret_desc *desc, int chunk) {
    if (check_desc(desc) != RET_OK || chunk < 1) return 0;
    Params p;
    make_params(desc, &p);
    return chunkwise_tc_supported(p, chunk, desc->in_dtype == RET_BF16) ? chunkwise_prep_bytes(p)
                                                                        : 0;
}

ret_status ret_chunkwise_prepare(const ret_desc *desc, int chunk, const void *Q, const void *K,
                                 void *workspace, size_t workspace_bytes, void *stream) {
    ret_status s = check_desc(desc);
    if (s != RET_OK) return s;
    if (chunk < 1) return RET_ERR_ARG;
    const size_t need = ret_chunkwise_prep_size(desc, chunk);
    if (need == 0 && (long long)desc->B * desc->L > 0) return RET_ERR_SHAPE;
    if (need == 0) return RET_OK;  // empty problem
    if (!Q || !K || !workspace) return RET_ERR_NULL;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(workspace)) return RET_ERR_ALIGN;
    if (workspace_bytes < need) return RET_ERR_WORKSPACE;
    if ((s = check_device()) != RET_OK) return s;
    Params p;
    make_params(desc, &p);
    const void *q_used = nullptr, *k_used = nullptr;
    // the weights follow the 128-row blocks the tensor-core loop works in
    return from_cuda(launch_chunkwise_prep(p, kChunkBlock, Q, K, workspace, &q_used, &k_used,
                                           (cudaStream_t)stream));
}

ret_status ret_chunkwise_prepared(const ret_desc *desc, int chunk, const void *Qh, const void *Kt,
                                  const void *V, const float *state_in, float *state_out,
                                  void *O, const void *G, float gn_eps, void *Y, void *stream) {
    ret_status s = check_desc(desc);
    if (s != RET_OK) return s;
    if (chunk < 1) return RET_ERR_ARG;
    if ((long long)desc->B * desc->L == 0) return RET_ERR_SHAPE;  // nothing was prepared
    Params p;
    make_params(desc, &p);
    if (!chunkwise_tc_supported(p, chunk, desc->in_dtype == RET_BF16)) return RET_ERR_SHAPE;
    if ((G == nullptr) != (Y == nullptr) || (!O && !Y) || !Qh || !Kt || !V) return RET_ERR_NULL;
    if (Y && !(gn_eps >= 0.0f && std::isfinite(gn_eps))) return RET_ERR_ARG;
    if (!aligned16(Qh) || !aligned16(Kt) || !aligned16(V) || !aligned16(O) || !aligned16(G) ||
        !aligned16(Y) || !aligned16(state_in) || !aligned16(state_out))
        return RET_ERR_ALIGN;
    if ((s = check_device()) != RET_OK) return s;
    int *status = device_status_word();
    if (!status) return RET_ERR_CUDA;
    return from_cuda(launch_chunkwise_tc_rows(p, desc->out_dtype == RET_BF16, Qh, Kt, V, state_in,
                                              state_out, O, G, Y, gn_eps, status,
                                              (cudaStream_t)stream));
}

ret_status ret_chunkwise(const ret_desc *desc, int chunk, const void *Q, const void *K,
                         const void *V, const float *state_in, float *state_out, void *O,
                         const void *G, float gn_eps, void *Y, void *workspace,
                         size_t workspace_bytes, void *stream) {
    ret_status s = check_desc(desc);
    if (s != RET_OK) return s;
    if (chunk < 1) return RET_ERR_ARG;
    const bool empty = (long long)desc->B * desc->L == 0;
    const bool want_Y = Y != nullptr, want_O = O != nullptr;
    if (!empty) {
        // (an empty problem may come with NULL buffers: nothing is read or written)
        if ((G == nullptr) != (Y == nullptr)) return RET_ERR_NULL;
        if (!want_Y && !want_O) return RET_ERR_NULL;
        if (!Q || !K || !V) return RET_ERR_NULL;
    }
    if (want_Y && !(gn_eps >= 0.0f && std::isfinite(gn_eps))) return RET_ERR_ARG;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(G) ||
        !aligned16(Y) || !aligned16(state_in) || !aligned16(state_out) || !aligned16(workspace))
        return RET_ERR_ALIGN;
    const size_t need = ret_workspace_size(desc, chunk, want_O, want_Y);
    if (need > 0 && (!workspace || workspace_bytes < need)) return RET_ERR_WORKSPACE;
    if ((s = check_device()) != RET_OK) return s;

    cudaStream_t st = (cudaStream_t)stream;
    const size_t state_bytes = sizeof(float) * (size_t)desc->B * desc->H * desc->d_k * desc->d_v;
    if (desc->L == 0 || desc->B == 0) {
        // Nothing to absorb: the state passes through unchanged.
        if (state_out && state_out != state_in && state_bytes) {
            cudaError_t e = state_in ? cudaMemcpyAsync(state_out, state_in, state_bytes,
                                                       cudaMemcpyDeviceToDevice, st)
                                     : cudaMemsetAsync(state_out, 0, state_bytes, st);
            return from_cuda(e);
        }
        return RET_OK;
    }
    Params p;
    make_params(desc, &p);
    const bool in_bf16 = desc->in_dtype == RET_BF16, out_bf16 = desc->out_dtype == RET_BF16;
    void *o_buf = want_O ? O : workspace;
    const bool o_bf16 = want_O ? out_bf16 : false;
    if (chunkwise_tc_supported(p, chunk, in_bf16)) {
        int *status = device_status_word();
        if (!status) return RET_ERR_CUDA;
        // few (b, h) heads: every block of every sequence at once in one
        // launch (the one-launch shapes, no carried state, room for the block
        // sums), else every sequence cut into segments that run at once
        if (few_heads(p) && onepass_supported(p, in_bf16, state_in || state_out) && workspace &&
            workspace_bytes >= onepass_bytes(p))
            return from_cuda(launch_onepass(p, out_bf16, Q, K, V, O, G, Y, gn_eps, workspace, status,
                                            st));
        const int S = auto_segments(p, chunk);
        if (S > 1 && workspace && workspace_bytes >= segmented_bytes(p, S))
            return from_cuda(launch_segmented(p, S, out_bf16, Q, K, V, state_in, state_out, O, G,
                                              Y, gn_eps, workspace, status, st));
        // a workspace of ret_chunkwise_prep_size bytes holds the prepared rows
        void *prep = workspace && workspace_bytes >= chunkwise_prep_bytes(p) ? workspace : nullptr;
        return from_cuda(launch_chunkwise_tc(p, out_bf16, Q, K, V, state_in, state_out, O, G, Y,
                                             gn_eps, prep, status, st));
    }
    cudaError_t e = launch_chunkwise_simt(p, chunk, in_bf16, o_bf16, Q, K, V, state_in, state_out,
                                          o_buf, st);
    if (e == cudaSuccess && want_Y)
        e = launch_gate_norm(desc->B, desc->L, desc->H, desc->d_v, o_bf16, o_buf, in_bf16, G,
                             gn_eps, out_bf16, Y, st);
    return from_cuda(e);
}

ret_status ret_recurrent_step(const ret_desc *desc, const void *q, const void *k, const void *v,
                              float *state, void *o, void *stream) {
    ret_status s = check_desc(desc);
    if (s != RET_OK) return s;
    if (desc->L < 1 || desc->L > RET_MAX_DECODE_STEPS) return RET_ERR_SHAPE;
    const bool empty = desc->B == 0;
    if (!empty && (!q || !k || !v || !state || !o)) return RET_ERR_NULL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(state) || !aligned16(o))
        return RET_ERR_ALIGN;
    if ((s = check_device()) != RET_OK) return s;
    if (empty) return RET_OK;
    Params p;
    make_params(desc, &p);
    return from_cuda(launch_recurrent_step(p, desc->in_dtype == RET_BF16,
                                           desc->out_dtype == RET_BF16, q, k, v, state, o,
                                           (cudaStream_t)stream));
}

ret_status ret_gate_norm(int B, int L, int H, int d_v, int o_dtype, const void *O, int g_dtype,
                         const void *G, float eps, int y_dtype, void *Y, void *stream) {
    if (B < 0 || L < 0 || H < 1 || H > RET_MAX_HEADS || d_v < 1 || d_v > kMaxDv || d_v % 4)
        return RET_ERR_SHAPE;
    if (!valid_dtype(o_dtype) || !valid_dtype(g_dtype) || !valid_dtype(y_dtype))
        return RET_ERR_DTYPE;
    if (!(eps >= 0.0f && std::isfinite(eps))) return RET_ERR_ARG;
    const bool empty = (long long)B * L == 0;
    if (!empty && (!O || !G || !Y)) return RET_ERR_NULL;
    if (!aligned16(O) || !aligned16(G) || !aligned16(Y)) return RET_ERR_ALIGN;
    ret_status s = check_device();
    if (s != RET_OK) return s;
    if (empty) return RET_OK;
    return from_cuda(launch_gate_norm(B, L, H, d_v, o_dtype == RET_BF16, O, g_dtype == RET_BF16, G,
                                      eps, y_dtype == RET_BF16, Y, (cudaStream_t)stream));
}

ret_status ret_gate_norm_backward(int B, int L, int H, int d_v, int o_dtype, const void *O,
                                  int g_dtype, const void *G, const void *dY, float eps, void *dO,
                                  void *dG, void *stream) {
    if (B < 0 || L < 0 || H < 1 || H > RET_MAX_HEADS || d_v < 1 || d_v > kMaxDv || d_v % 4)
        return RET_ERR_SHAPE;
    if (!valid_dtype(o_dtype) || !valid_dtype(g_dtype)) return RET_ERR_DTYPE;
    if (!(eps >= 0.0f && std::isfinite(eps))) return RET_ERR_ARG;
    const bool empty = (long long)B * L == 0;
    if (!empty && (!O || !G || !dY || !dO || !dG)) return RET_ERR_NULL;
    if (!aligned16(O) || !aligned16(G) || !aligned16(dY) || !aligned16(dO) || !aligned16(dG))
        return RET_ERR_ALIGN;
    ret_status s = check_device();
    if (s != RET_OK) return s;
    if (empty) return RET_OK;
    return from_cuda(launch_gate_norm_backward(B, L, H, d_v, o_dtype == RET_BF16, O,
                                               g_dtype == RET_BF16, G, dY, eps, dO, dG,
                                               (cudaStream_t)stream));
}

unsigned long long ret_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

ret_status ret_last_device_status(void *stream) {
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return RET_ERR_CUDA;
    int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_ret_device_status, sizeof(int)) != cudaSuccess) return RET_ERR_CUDA;
    if (v != 0 && cudaMemcpyToSymbol(g_ret_device_status, &zero, sizeof(int)) != cudaSuccess)
        return RET_ERR_CUDA;
    return v == 0 ? RET_OK : (ret_status)v;
}

}  // extern "C"
