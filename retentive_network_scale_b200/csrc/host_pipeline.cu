// host_pipeline.cu -- ret_chunkwise_host: the chunkwise forward (with the
// optional GroupNorm + swish gate) from host buffers to host buffers.
//
// No counterpart in the paper: it is the end-to-end form of ret_chunkwise
// for callers whose Q, K, V, G live in host memory.  The batch is cut into
// slices (every (b, h) is independent, so the slices are separate
// problems) and the slices flow through a three-stream pipeline over two
// device slots: the host-to-device copies of slice i, the compute of slice
// i-1 and the device-to-host copy of slice i-2 run at the same time.  Each
// copy is one cudaMemcpyAsync of a contiguous range (a batch slice of every
// tensor is contiguous in the documented layouts).
#include <algorithm>

#include "launch.h"
#include "retention.h"

namespace {

constexpr size_t kAlign = 256;

size_t round_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }
size_t dtype_bytes(int d) { return d == RET_BF16 ? 2 : 4; }

// Byte sizes of one batch element of every tensor, and the device slot for
// `bs` batch elements (inputs, outputs, then ret_chunkwise's own workspace).
struct Slot {
    size_t q, k, v, g, y, o, ws;
    size_t off_q, off_k, off_v, off_g, off_y, off_o, off_ws, bytes;
};

Slot slot_layout(const ret_desc *d, int chunk, int bs, bool want_O, bool want_Y) {
    const size_t in = dtype_bytes(d->in_dtype), out = dtype_bytes(d->out_dtype);
    const size_t rows = (size_t)d->H * d->L;
    Slot s{};
    s.q = (size_t)bs * rows * d->d_k * in;
    s.k = s.q;
    s.v = (size_t)bs * rows * d->d_v * in;
    s.g = want_Y ? (size_t)bs * rows * d->d_v * in : 0;
    s.y = want_Y ? (size_t)bs * rows * d->d_v * out : 0;
    s.o = want_O ? (size_t)bs * rows * d->d_v * out : 0;
    ret_desc ds = *d;
    ds.B = bs;
    s.ws = std::max(ret_workspace_size(&ds, chunk, want_O, want_Y), ret_chunkwise_prep_size(&ds, chunk));
    s.off_q = 0;
    s.off_k = s.off_q + round_up(s.q);
    s.off_v = s.off_k + round_up(s.k);
    s.off_g = s.off_v + round_up(s.v);
    s.off_y = s.off_g + round_up(s.g);
    s.off_o = s.off_y + round_up(s.y);
    s.off_ws = s.off_o + round_up(s.o);
    s.bytes = s.off_ws + round_up(s.ws);
    return s;
}

int slice_rows(const ret_desc *d, int slices) {  // batch elements per slice
    const int n = std::max(1, std::min(slices, d->B));
    return (d->B + n - 1) / n;
}

}  // namespace

extern "C" {

size_t ret_chunkwise_host_workspace_size(const ret_desc *desc, int chunk, int want_O, int want_Y,
                                         int slices) {
    if (ret::validate_desc(desc) != RET_OK || chunk < 1 || slices < 1 || (!want_O && !want_Y))
        return 0;
    if ((long long)desc->B * desc->L == 0) return 0;
    const int bs = slice_rows(desc, slices);
    const int nslices = (desc->B + bs - 1) / bs;
    const Slot s = slot_layout(desc, chunk, bs, want_O != 0, want_Y != 0);
    return (nslices > 1 ? 2 : 1) * s.bytes;
}

ret_status ret_chunkwise_host(const ret_desc *desc, int chunk, const void *Q, const void *K,
                              const void *V, void *O, const void *G, float gn_eps, void *Y,
                              int slices, void *dev_workspace, size_t dev_workspace_bytes,
                              void *stream) {
    ret_status st = ret::validate_desc(desc);
    if (st != RET_OK) return st;
    if (chunk < 1 || slices < 1) return RET_ERR_ARG;
    const bool want_O = O != nullptr, want_Y = Y != nullptr;
    if ((G == nullptr) != (Y == nullptr)) return RET_ERR_NULL;
    if ((long long)desc->B * desc->L == 0) return RET_OK;  // nothing to copy or compute
    if (!want_O && !want_Y) return RET_ERR_NULL;
    if (!Q || !K || !V) return RET_ERR_NULL;
    if (want_Y && !(gn_eps >= 0.0f && gn_eps < 3.0e38f)) return RET_ERR_ARG;
    const size_t need = ret_chunkwise_host_workspace_size(desc, chunk, want_O, want_Y, slices);
    if (!dev_workspace || dev_workspace_bytes < need) return RET_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(dev_workspace) & (kAlign - 1)) != 0) return RET_ERR_ALIGN;

    const int bs = slice_rows(desc, slices);
    const int n = (desc->B + bs - 1) / bs;
    const Slot sl = slot_layout(desc, chunk, bs, want_O, want_Y);
    const size_t in = dtype_bytes(desc->in_dtype), out = dtype_bytes(desc->out_dtype);
    const size_t per_b_qk = (size_t)desc->H * desc->L * desc->d_k * in;
    const size_t per_b_v = (size_t)desc->H * desc->L * desc->d_v * in;
    const size_t per_b_out = (size_t)desc->H * desc->L * desc->d_v * out;

    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    cudaStream_t up = nullptr, down = nullptr;
    cudaEvent_t start = nullptr, ev[3][2] = {};  // [h2d, compute, d2h][slot]
    ret_status result = RET_OK;
    auto fail = [&](cudaError_t e) {
        if (e != cudaSuccess && result == RET_OK) result = RET_ERR_CUDA;
        return e != cudaSuccess;
    };
    do {
        if (fail(cudaStreamCreateWithFlags(&up, cudaStreamNonBlocking)) ||
            fail(cudaStreamCreateWithFlags(&down, cudaStreamNonBlocking)) ||
            fail(cudaEventCreateWithFlags(&start, cudaEventDisableTiming)))
            break;
        bool ok = true;
        for (int a = 0; a < 3 && ok; ++a)
            for (int b = 0; b < 2 && ok; ++b)
                ok = !fail(cudaEventCreateWithFlags(&ev[a][b], cudaEventDisableTiming));
        if (!ok) break;
        // the pipeline starts after the work already queued on the caller's stream
        if (fail(cudaEventRecord(start, cs)) || fail(cudaStreamWaitEvent(up, start, 0)) ||
            fail(cudaStreamWaitEvent(down, start, 0)))
            break;
        uint8_t *ws = static_cast<uint8_t *>(dev_workspace);
        for (int i = 0; i < n && result == RET_OK; ++i) {
            const int slot = i & 1;
            const int b0 = i * bs, nb = std::min(bs, desc->B - b0);
            uint8_t *base = ws + slot * sl.bytes;
            // inputs: the slot's previous compute (slice i-2) has read them
            if (i >= 2 && fail(cudaStreamWaitEvent(up, ev[1][slot], 0))) break;
            const auto *q = static_cast<const uint8_t *>(Q), *k = static_cast<const uint8_t *>(K);
            const auto *v = static_cast<const uint8_t *>(V), *g = static_cast<const uint8_t *>(G);
            if (fail(cudaMemcpyAsync(base + sl.off_q, q + b0 * per_b_qk, nb * per_b_qk, cudaMemcpyHostToDevice, up)) ||
                fail(cudaMemcpyAsync(base + sl.off_k, k + b0 * per_b_qk, nb * per_b_qk, cudaMemcpyHostToDevice, up)) ||
                fail(cudaMemcpyAsync(base + sl.off_v, v + b0 * per_b_v, nb * per_b_v, cudaMemcpyHostToDevice, up)))
                break;
            if (want_Y &&
                fail(cudaMemcpyAsync(base + sl.off_g, g + b0 * per_b_v, nb * per_b_v, cudaMemcpyHostToDevice, up)))
                break;
            if (fail(cudaEventRecord(ev[0][slot], up))) break;
            // compute: inputs landed, and the slot's outputs of slice i-2 are copied out
            if (fail(cudaStreamWaitEvent(cs, ev[0][slot], 0))) break;
            if (i >= 2 && fail(cudaStreamWaitEvent(cs, ev[2][slot], 0))) break;
            ret_desc ds = *desc;
            ds.B = nb;
            const ret_status s = ret_chunkwise(
                &ds, chunk, base + sl.off_q, base + sl.off_k, base + sl.off_v, nullptr, nullptr,
                want_O ? base + sl.off_o : nullptr, want_Y ? base + sl.off_g : nullptr, gn_eps,
                want_Y ? base + sl.off_y : nullptr, base + sl.off_ws, sl.ws, cs);
            if (s != RET_OK) {
                result = s;
                break;
            }
            if (fail(cudaEventRecord(ev[1][slot], cs)) || fail(cudaStreamWaitEvent(down, ev[1][slot], 0)))
                break;
            if (want_Y && fail(cudaMemcpyAsync(static_cast<uint8_t *>(Y) + b0 * per_b_out, base + sl.off_y,
                                               nb * per_b_out, cudaMemcpyDeviceToHost, down)))
                break;
            if (want_O && fail(cudaMemcpyAsync(static_cast<uint8_t *>(O) + b0 * per_b_out, base + sl.off_o,
                                               nb * per_b_out, cudaMemcpyDeviceToHost, down)))
                break;
            if (fail(cudaEventRecord(ev[2][slot], down))) break;
        }
        // the caller's stream resumes once every copy back has finished
        if (fail(cudaEventRecord(start, down))) break;
        fail(cudaStreamWaitEvent(cs, start, 0));
    } while (false);
    // after a failure, let whatever was queued finish before returning
    if (result != RET_OK) {
        if (up) cudaStreamSynchronize(up);
        if (down) cudaStreamSynchronize(down);
        cudaGetLastError();
    }
    // release (deferred by the runtime until the queued work has finished)
    for (auto &row : ev)
        for (auto &e : row)
            if (e) cudaEventDestroy(e);
    if (start) cudaEventDestroy(start);
    if (up) cudaStreamDestroy(up);
    if (down) cudaStreamDestroy(down);
    return result;
}

}  // extern "C"
