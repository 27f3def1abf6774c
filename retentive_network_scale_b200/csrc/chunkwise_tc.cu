// chunkwise_tc.cu -- the host side of chunkwise retention on the sm_100a
// tensor cores: which shapes the tensor-core path takes, and how a call is
// laid out over the streaming pass (prep.cu) and the warp-specialised chunk
// loop (chunkwise_ws.cu).
//
// "Retentive Network" paper summary, section 2.1, chunkwise recurrent form
// (3): parallel inside a chunk, a decayed state carried between chunks.  The
// loop evaluates it in the rescaled form described in chunkwise_ws.cu; all
// its factors stay in range while gamma^128 >= 2^-60, and other decays use
// the CUDA-core kernel (simt.cu).
//
// With room in the workspace the turned Q^ and the weighted K~ are written
// once by the streaming pass and the loop only loads them; without it the
// loop turns the landed tiles itself (d_k 128 and 256) or, without
// rotation, weights the value rows itself.  A call whose loop needs more
// than one wave of CTAs is cut into batch slices so that the streaming pass
// of the next slice runs beside the loop of the current one.
#include <algorithm>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "launch.h"

namespace ret {
namespace {

constexpr int kC = 128;       // rows per block of the loop (MMA M)
constexpr int kTV = 128;      // value columns per CTA
constexpr int kMaxCluster = kMaxDv / kTV;
constexpr float kMinLog2GammaTimesC = -60.f;  // gamma^C >= 2^-60

}  // namespace

// The loop works in blocks of kC rows whatever the chunk: a chunk of
// kC * m rows is m consecutive blocks, and a chunk of 64 rows pairs up two
// chunks per block.  The chunkwise recurrence holds exactly at any row
// boundary (the state carried between blocks is the exact state after
// those rows), so either is the same computation; only the rounding
// differs.  With rotation, d_k 64 needs the streaming pass's workspace
// (chunkwise_tc_needs_prep): the loop turns tiles of d_k 128 and 256 only.
bool chunkwise_tc_supported(const Params &p, int chunk, bool in_bf16) {
    const bool dk_ok = p.dk == 64 || p.dk == 128 || p.dk == 256;
    const bool dv_ok = p.dv == 64 || (p.dv % kTV == 0 && p.dv / kTV <= kMaxCluster);
    if (!in_bf16 || chunk % 64 != 0 || !dk_ok || !dv_ok || p.L < 1 || p.B * p.H < 1 ||
        (long long)p.B * p.H > 65535)
        return false;
    for (int h = 0; h < p.H; ++h)
        if (!(p.log2g[h] * kC >= kMinLog2GammaTimesC)) return false;  // also rejects gamma = 0
    return true;
}

bool chunkwise_tc_needs_prep(const Params &p, int chunk) {
    (void)chunk;  // the loop works in blocks of 128 rows for every chunk it takes
    return p.rotate && p.dk == 64;  // the loop turns tiles of d_k 128 and 256 itself
}

namespace {

// The chunk loop on rows that are ready (`pre`: prepared by the streaming
// pass, the key rows carrying their weight) or raw: then the loop turns the
// landed tiles itself when rotating (d_k 128 or 256) or weights the value
// rows itself when not.
cudaError_t launch_tc_rows(const Params &p, bool out_bf16, const void *Q, const void *K,
                           const void *V, const float *s_in, float *s_out, void *O, const void *G,
                           void *Y, float eps, int pre, int *status, cudaStream_t st) {
    const bool rot = !pre && p.rotate;
    if (rot && (p.dk == 64 || p.seg_heads != 1)) return cudaErrorInvalidValue;
    const RowLayout hm = bhld_layout(p, p.dk), vl = bhld_layout(p, p.dv);
    // G [B][L][H d_v] of the real heads (segment heads: H = real heads x
    // seg_heads, L = rows of one segment; the batch stride is the same)
    const RowLayout gl{(long long)(p.H / p.seg_heads) * p.dv, 0, (long long)p.L * p.H * p.dv};
    return launch_chunkwise_ws(p, out_bf16, Q, hm, K, hm, V, vl, true, s_in, s_out, O, G, gl, Y, eps,
                               !pre && !rot, rot, status, st);
}

// A second stream per device on which the streaming pass of the next batch
// slice runs while the chunk loop of the current one holds the SMs, and the
// two events that join it to the caller's stream.  Made once; the lock
// keeps the enqueue sequences of concurrent callers apart.
struct SideStream {
    std::mutex mu;
    bool made = false, ok = false;
    cudaStream_t s = nullptr;
    cudaEvent_t start = nullptr, ready = nullptr;
    cudaEvent_t aux[kSideAuxEvents] = {};  // for other users of the stream
    int sms = 0;
};
constexpr int kMaxDevices = 64;
SideStream g_side[kMaxDevices];

SideStream *side_stream() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return nullptr;
    }
    SideStream &ss = g_side[dev];
    std::lock_guard<std::mutex> lock(ss.mu);
    if (!ss.made) {
        ss.made = true;
        // the lowest priority: the loop's CTAs take the SMs first, the pass
        // fills those left over
        int least = 0, greatest = 0;
        ss.ok = cudaDeviceGetStreamPriorityRange(&least, &greatest) == cudaSuccess &&
                cudaStreamCreateWithPriority(&ss.s, cudaStreamNonBlocking, least) == cudaSuccess &&
                cudaEventCreateWithFlags(&ss.start, cudaEventDisableTiming) == cudaSuccess &&
                cudaEventCreateWithFlags(&ss.ready, cudaEventDisableTiming) == cudaSuccess &&
                cudaDeviceGetAttribute(&ss.sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess &&
                ss.sms > 0;
        for (int i = 0; i < kSideAuxEvents && ss.ok; ++i)
            ss.ok = cudaEventCreateWithFlags(&ss.aux[i], cudaEventDisableTiming) == cudaSuccess;
        if (!ss.ok) cudaGetLastError();
    }
    return ss.ok ? &ss : nullptr;
}

}  // namespace

bool side_stream_ref(SideStreamRef *r) {
    SideStream *ss = side_stream();
    if (!ss) return false;
    r->mu = &ss->mu;
    r->s = ss->s;
    r->start = ss->start;
    r->ready = ss->ready;
    for (int i = 0; i < kSideAuxEvents; ++i) r->aux[i] = ss->aux[i];
    r->sms = ss->sms;
    return true;
}

// With room for them, the turned Q^ and scaled K~ are written once by a
// streaming pass and the kernel only loads them.  When the chunk loop needs
// more than one wave of CTAs (one per SM: its shared memory and registers
// fill an SM), the batch is cut into as many slices as waves, each at most
// a wave: the loop of slice i then leaves SMs free on which the streaming
// pass of slice i+1 runs from the side stream, so only the first slice's
// pass is exposed.  The slices compute exactly what one launch would (every
// (b, h) and every row of the pass is independent).
cudaError_t launch_chunkwise_tc(const Params &p, bool out_bf16, const void *Q, const void *K,
                                const void *V, const float *s_in, float *s_out, void *O,
                                const void *G, void *Y, float eps, void *prep_ws, int *status,
                                cudaStream_t st) {
    if (!prep_ws)
        return launch_tc_rows(p, out_bf16, Q, K, V, s_in, s_out, O, G, Y, eps, 0, status, st);
    SideStream *ss = side_stream();
    // as many slices as waves, when every slice then fits in one wave (so
    // slicing never adds a wave); otherwise one launch
    constexpr int kMaxSlices = 16;
    const long long ctas_per_b = (long long)p.H * (p.dv / kTV);
    int slices = 1;
    if (ss) {
        const long long waves = (ctas_per_b * p.B + ss->sms - 1) / ss->sms;
        const long long per_slice = (p.B + waves - 1) / waves;  // batch elements, at most
        if (waves > 1 && waves <= std::min(p.B, kMaxSlices) && per_slice * ctas_per_b <= ss->sms)
            slices = (int)waves;
    }
    if (slices <= 1) {
        cudaError_t e = launch_chunkwise_prep(p, kC, Q, K, prep_ws, &Q, &K, st);
        if (e != cudaSuccess) return e;
        return launch_tc_rows(p, out_bf16, Q, K, V, s_in, s_out, O, G, Y, eps, 1, status, st);
    }
    // slice i: batch elements [b0(i), b0(i+1)); byte offsets per batch element
    auto b0 = [&](int i) { return (int)((long long)p.B * i / slices); };
    const size_t ob = out_bf16 ? 2 : 4;
    const size_t qk_b = (size_t)p.H * p.L * p.dk * 2, v_b = (size_t)p.H * p.L * p.dv * 2;
    const size_t o_b = (size_t)p.H * p.L * p.dv * ob, st_b = (size_t)p.H * p.dk * p.dv;
    const size_t ws_b = chunkwise_prep_bytes(p) / p.B;
    auto at = [](const void *base, size_t off) {
        return base ? static_cast<const void *>(static_cast<const uint8_t *>(base) + off) : nullptr;
    };
    auto at_w = [](void *base, size_t off) {
        return base ? static_cast<void *>(static_cast<uint8_t *>(base) + off) : nullptr;
    };
    auto sub = [&](int i) {
        Params q = p;
        q.B = b0(i + 1) - b0(i);
        return q;
    };
    const void *qh[kMaxSlices], *kt[kMaxSlices];  // prepared operands per slice
    auto prep = [&](int i, cudaStream_t on) {
        const size_t b = b0(i);
        return launch_chunkwise_prep(sub(i), kC, at(Q, b * qk_b), at(K, b * qk_b),
                                     at_w(prep_ws, b * ws_b), &qh[i], &kt[i], on);
    };
    // pass 0 on the caller's stream; the side stream starts after it (and so
    // after whatever the caller queued before), when the loop of slice 0
    // starts: the passes of the later slices run beside the loops
    std::lock_guard<std::mutex> lock(ss->mu);
    cudaError_t e = prep(0, st);
    if (e == cudaSuccess) e = cudaEventRecord(ss->start, st);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(ss->s, ss->start, 0);
    for (int i = 0; i < slices && e == cudaSuccess; ++i) {
        const size_t b = b0(i);
        e = launch_tc_rows(sub(i), out_bf16, qh[i], kt[i], at(V, b * v_b),
                           s_in ? s_in + b * st_b : nullptr, s_out ? s_out + b * st_b : nullptr,
                           at_w(O, b * o_b), at(G, b * v_b), at_w(Y, b * o_b), eps, 1, status, st);
        if (e == cudaSuccess && i + 1 < slices) {
            e = prep(i + 1, ss->s);
            if (e == cudaSuccess) e = cudaEventRecord(ss->ready, ss->s);
            if (e == cudaSuccess) e = cudaStreamWaitEvent(st, ss->ready, 0);
        }
    }
    return e;
}

cudaError_t launch_chunkwise_tc_rows(const Params &p, bool out_bf16, const void *Qh, const void *Kt,
                                     const void *V, const float *s_in, float *s_out, void *O,
                                     const void *G, void *Y, float eps, int *status,
                                     cudaStream_t st) {
    static_assert(kChunkBlock == kC, "the streaming pass and the loop share the row blocks");
    return launch_tc_rows(p, out_bf16, Qh, Kt, V, s_in, s_out, O, G, Y, eps, 1, status, st);
}

cudaError_t launch_chunkwise_tc_prepared(const Params &p, bool out_bf16, const void *Qh,
                                         RowLayout q_layout, const void *Kt, const void *V,
                                         RowLayout v_layout, bool v_head_major, const void *G,
                                         RowLayout g_layout, void *Y, void *O, float eps,
                                         int *status, cudaStream_t st) {
    return launch_chunkwise_ws(p, out_bf16, Qh, q_layout, Kt, bhld_layout(p, p.dk), V, v_layout, v_head_major, nullptr,
                               nullptr, O, G, g_layout, Y, eps, false, false, status, st);
}

}  // namespace ret
