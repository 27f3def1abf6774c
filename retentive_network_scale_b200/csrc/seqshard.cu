// seqshard.cu -- a long sequence cut into consecutive segments, joined
// through their states: across devices (ret_segment_state, ret_state_scan)
// and on one device (ret_chunkwise_segmented, for few long sequences).
//
// "Retentive Network" paper summary, section 2.1, chunkwise form (3):
// parallel inside a block of rows, a decayed state carried between blocks.
// The same recurrence holds between segments of any length: a segment of n
// rows that starts from state R leaves
//     R' = gamma^n R + U,   U = sum_{t<n} gamma^{n-1-t} k^_t^T v_t,
// where U depends on the segment alone.  So every device computes the U of
// its own segment at once (a streaming pass that turns and decay-weights the
// keys, then one product K~^T V on the tensor cores), the U are exchanged
// (an all-gather), and a
// scan gives each segment its entering state; the segment's outputs then
// come from ret_chunkwise started from that state.  On one device the same
// steps run for all segments at once: a [B][H][L][d] tensor read as
// [B][H*S][L/S][d] is S segment heads per head with uniform strides, so the
// chunk loop's streaming pass (whose weighted keys also serve the segment
// states), one launch for the segment states, one scan and one chunk-loop
// launch cover them, with S times the CTAs of the plain loop.
#include <mutex>

#include "launch.h"
#include "retention.h"

namespace ret {

// One cuBLAS handle per device for the batched GEMM fallback of the segment
// states (shapes off the tensor-core kernel), made on first use.
namespace {
constexpr int kBlasDevices = 64;
std::mutex g_blas_mu;
cublasHandle_t g_blas[kBlasDevices];
}  // namespace

std::mutex &blas_mutex() { return g_blas_mu; }

cublasHandle_t blas_handle(cudaStream_t st, void *workspace) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kBlasDevices) {
        cudaGetLastError();
        return nullptr;
    }
    if (!g_blas[dev] && cublasCreate(&g_blas[dev]) != CUBLAS_STATUS_SUCCESS) {
        g_blas[dev] = nullptr;
        return nullptr;
    }
    cublasHandle_t h = g_blas[dev];
    if (cublasSetStream(h, st) != CUBLAS_STATUS_SUCCESS ||
        cublasSetWorkspace(h, workspace, kBlasWorkspace) != CUBLAS_STATUS_SUCCESS)
        return nullptr;
    return h;
}

namespace {

constexpr size_t kAlign = 256;
size_t round_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// Decay exponents of one scan: R_rank = gamma^{n_in} R_0 + sum_{s<rank}
// gamma^{n[s]} U_s, with n[s] the tokens between segment s and `rank`.
struct ScanArgs {
    long long n[RET_MAX_SEGMENTS];
    long long n_in;
    int rank;
};

__device__ __forceinline__ float decay_pow_ll(float log2g, long long n) {
    return n == 0 ? 1.0f : exp2f((float)n * log2g);
}

// One thread: four consecutive state elements (d_v is a multiple of 4).
__global__ void __launch_bounds__(256)
state_scan_kernel(const Params p, const ScanArgs a, long long quads, size_t seg_elems,
                  const float *__restrict__ U_all, const float *__restrict__ state_in,
                  float *__restrict__ R) {
    const long long q = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (q >= quads) return;
    const size_t e = (size_t)q * 4;
    const int h = (int)((e / ((size_t)p.dk * p.dv)) % p.H);
    const float lg = p.log2g[h];
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (state_in) {
        const float f = decay_pow_ll(lg, a.n_in);
        const float4 x = *reinterpret_cast<const float4 *>(state_in + e);
        acc = make_float4(f * x.x, f * x.y, f * x.z, f * x.w);
    }
    for (int s = 0; s < a.rank; ++s) {
        const float f = decay_pow_ll(lg, a.n[s]);
        const float4 x = *reinterpret_cast<const float4 *>(U_all + s * seg_elems + e);
        acc.x = fmaf(f, x.x, acc.x);
        acc.y = fmaf(f, x.y, acc.y);
        acc.z = fmaf(f, x.z, acc.z);
        acc.w = fmaf(f, x.w, acc.w);
    }
    *reinterpret_cast<float4 *>(R + e) = acc;
}

bool sm100() {
    int dev = -1, major = 0, minor = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return major == 10 && minor == 0;
}

bool a16(const void *q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; }

// U_bh [d_k][d_v] = K~_bh^T V_bh for every (b, h) of p: on the tensor-core
// kernel of segstate.cu where it applies (d_k 64, 128 or 256, d_v 64 or a
// multiple of 128); otherwise as one cuBLAS batched GEMM, in column-major terms the
// (d_v x d_k) product V_cm (d_v x L) * K~_cm^T (L x d_k).
ret_status segment_gemm(const Params &p, const void *V, const void *kt, float *U,
                        void *blas_ws, cudaStream_t st) {
    if (segment_state_tc_supported(p)) {
        int *status = device_status_word();
        if (!status) return RET_ERR_CUDA;
        return launch_segment_state_tc(p, V, kt, 0, U, status, st) == cudaSuccess
                   ? RET_OK
                   : RET_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lock(blas_mutex());
    cublasHandle_t h = blas_handle(st, blas_ws);
    if (!h) return RET_ERR_CUDA;
    const float one = 1.f, zero = 0.f;
    const long long L = p.L, dk = p.dk, dv = p.dv;
    const cublasStatus_t r = cublasGemmStridedBatchedEx(
        h, CUBLAS_OP_N, CUBLAS_OP_T, (int)dv, (int)dk, (int)L, &one, V, CUDA_R_16BF, (int)dv,
        L * dv, kt, CUDA_R_16BF, (int)dk, L * dk, &zero, U, CUDA_R_32F, (int)dv, dk * dv,
        p.B * p.H, CUBLAS_COMPUTE_32F, CUBLAS_GEMM_DEFAULT);
    return r == CUBLAS_STATUS_SUCCESS ? RET_OK : RET_ERR_CUDA;
}

// The entering state of every segment of every sequence at once, segments
// of n rows each (R_0 = state_in or 0, R_{s+1} = gamma^n R_s + U_s): one
// thread per four elements of a (b, h) state walks its S segments in order.
// U and R are [B][H*S][d_k][d_v] (segment s of head h at h*S + s); state_in
// is [B][H][d_k][d_v].
__global__ void __launch_bounds__(256)
segment_scan_kernel(const Params p, int S, long long n, long long quads,
                    const float *__restrict__ U, const float *__restrict__ state_in,
                    float *__restrict__ R) {
    const long long q = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (q >= quads) return;
    const size_t per = (size_t)p.dk * p.dv;
    const size_t e = (size_t)q * 4;                  // element of the [B][H] states
    const size_t bh = e / per, off = e - bh * per;
    const int h = (int)(bh % p.H);
    const float g = decay_pow_ll(p.log2g[h], n);
    float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
    if (state_in) r = *reinterpret_cast<const float4 *>(state_in + e);
    const size_t first = (bh * S) * per + off;       // segment 0 of this (b, h)
    for (int s = 0; s < S; ++s) {
        *reinterpret_cast<float4 *>(R + first + (size_t)s * per) = r;
        const float4 u = *reinterpret_cast<const float4 *>(U + first + (size_t)s * per);
        r = make_float4(fmaf(g, r.x, u.x), fmaf(g, r.y, u.y), fmaf(g, r.z, u.z), fmaf(g, r.w, u.w));
    }
}

// [B][H][L] heads as [B][H*S][L/S] segment heads: decays repeated per
// segment, rows at their absolute positions.
Params segment_params(const Params &p, int S) {
    Params q = p;
    q.H = p.H * S;
    q.L = p.L / S;
    for (int h = p.H - 1; h >= 0; --h)
        for (int s = S - 1; s >= 0; --s) q.log2g[h * S + s] = p.log2g[h];
    q.seg_heads = S;
    q.seg_len = q.L;
    return q;
}

struct SegLayout {
    size_t prep, states, off_u, off_r, off_s, off_blas, bytes;
};

SegLayout seg_layout(const Params &p, int S) {
    const Params q = segment_params(p, S);
    SegLayout z{};
    z.prep = round_up(chunkwise_prep_bytes(q));
    z.states = round_up((size_t)q.B * q.H * q.dk * q.dv * sizeof(float));
    z.off_u = z.prep;
    z.off_r = z.off_u + z.states;
    z.off_s = z.off_r + z.states;
    z.off_blas = z.off_s + z.states;
    z.bytes = z.off_blas + kBlasWorkspace;
    return z;
}

}  // namespace

bool segmented_supported(const Params &p, int chunk, int S) {
    if (S < 1 || p.L % S != 0 || (long long)p.H * S > RET_MAX_HEADS ||
        (long long)p.B * p.H * S > 65535)  // one CTA row per segment head
        return false;
    return chunkwise_tc_supported(p, chunk, true) && segment_state_tc_supported(p);
}

size_t segmented_bytes(const Params &p, int S) { return seg_layout(p, S).bytes; }

int auto_segments(const Params &p, int chunk) {
    // the plain loop's CTAs; segments only when they leave most SMs idle,
    // as many as keep one wave (148 SMs) and at least four blocks of 128
    // rows per segment (below that the three extra launches cost more than
    // the shorter chain saves)
    const long long ctas = (long long)p.B * p.H * ((p.dv + 127) / 128);
    if (ctas >= 64) return 1;
    int S = 1;
    while (ctas * S * 2 <= 148 && p.L % (S * 2) == 0 && p.L / (S * 2) >= 4 * kChunkBlock &&
           segmented_supported(p, chunk, S * 2))
        S *= 2;
    return S;
}

cudaError_t launch_segmented(const Params &p, int S, bool out_bf16, const void *Q, const void *K,
                             const void *V, const float *state_in, float *state_out, void *O,
                             const void *G, void *Y, float eps, void *workspace, int *status,
                             cudaStream_t st) {
    const SegLayout z = seg_layout(p, S);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    float *U = reinterpret_cast<float *>(ws + z.off_u);
    float *R = reinterpret_cast<float *>(ws + z.off_r);
    float *Sout = reinterpret_cast<float *>(ws + z.off_s);
    const Params q = segment_params(p, S);
    // 1. the chunk loop's streaming pass: Q^ (with rotation) and K~, the keys
    //    turned and weighted by gamma^{m-1-j} within each block of m <= 128
    //    rows of each segment
    const void *qh = nullptr, *kt = nullptr;
    cudaError_t e = launch_chunkwise_prep(q, kChunkBlock, Q, K, ws, &qh, &kt, st);
    if (e != cudaSuccess) return e;
    // 2. every segment's own state from the same K~, each block's value rows
    //    scaled by the rest of the segment's weight
    if ((e = launch_segment_state_tc(q, V, kt, 2, U, status, st)) != cudaSuccess) return e;
    // 3. the state entering each segment
    const long long quads = (long long)p.B * p.H * p.dk * p.dv / 4;
    segment_scan_kernel<<<(unsigned)((quads + 255) / 256), 256, 0, st>>>(p, S, q.L, quads, U,
                                                                          state_in, R);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    note_launches(1);
    // 4. the chunk loop over all segments at once, each from its state (with
    //    the gate: G and Y of each segment's own rows)
    if ((e = launch_chunkwise_tc_rows(q, out_bf16, qh, kt, V, R, state_out ? Sout : nullptr, O, G,
                                      Y, eps, status, st)) != cudaSuccess)
        return e;
    // 5. the state after the last segment of each sequence
    if (state_out) {
        const size_t per = (size_t)p.dk * p.dv * sizeof(float);
        e = cudaMemcpy2DAsync(state_out, per, Sout + (size_t)(S - 1) * p.dk * p.dv, per * S, per,
                              (size_t)p.B * p.H, cudaMemcpyDeviceToDevice, st);
    }
    return e;
}

}  // namespace ret

extern "C" {

size_t ret_segment_state_workspace_size(const ret_desc *desc) {
    if (ret::validate_desc(desc) != RET_OK) return 0;
    const size_t rows = (size_t)desc->B * desc->H * desc->L;
    if (rows == 0) return 0;
    return ret::round_up(rows * desc->d_k * 2) + ret::kBlasWorkspace;
}

ret_status ret_segment_state(const ret_desc *desc, const void *K, const void *V, float *U,
                             void *workspace, size_t workspace_bytes, void *stream) {
    using namespace ret;
    ret_status s = validate_desc(desc);
    if (s != RET_OK) return s;
    if (desc->in_dtype != RET_BF16) return RET_ERR_DTYPE;
    if (desc->d_k % 8) return RET_ERR_SHAPE;  // 16-byte rows for the streaming pass
    const size_t bh = (size_t)desc->B * desc->H;
    if (bh == 0) return RET_OK;
    if (!U) return RET_ERR_NULL;
    if (!a16(U)) return RET_ERR_ALIGN;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (!sm100()) return RET_ERR_UNSUPPORTED;
    if (desc->L == 0) {  // an empty segment leaves the zero state
        return cudaMemsetAsync(U, 0, bh * desc->d_k * desc->d_v * sizeof(float), st) == cudaSuccess
                   ? RET_OK
                   : RET_ERR_CUDA;
    }
    if (!K || !V) return RET_ERR_NULL;
    if (!a16(K) || !a16(V)) return RET_ERR_ALIGN;
    if ((reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0) return RET_ERR_ALIGN;
    if (!workspace || workspace_bytes < ret_segment_state_workspace_size(desc))
        return RET_ERR_WORKSPACE;
    Params p;
    params_from_desc(desc, &p);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    void *kt = ws;
    // K~ = gamma^{L-1-t} k^_t: the whole segment as one block of rows
    if (launch_key_prep(p, desc->L, K, kt, st) != cudaSuccess) return RET_ERR_CUDA;
    return segment_gemm(p, V, kt, U, ws + round_up((size_t)bh * desc->L * desc->d_k * 2), st);
}

ret_status ret_state_scan(const ret_desc *desc, int n_seg, const int *seg_len, int rank,
                          const float *U_all, const float *state_in, float *R, void *stream) {
    using namespace ret;
    ret_status s = validate_desc(desc);
    if (s != RET_OK) return s;
    if (n_seg < 1 || n_seg > RET_MAX_SEGMENTS || rank < 0 || rank > n_seg) return RET_ERR_SHAPE;
    if (!seg_len) return RET_ERR_NULL;
    for (int i = 0; i < n_seg; ++i)
        if (seg_len[i] < 1) return RET_ERR_SHAPE;
    const size_t seg_elems = (size_t)desc->B * desc->H * desc->d_k * desc->d_v;
    if (seg_elems == 0) return RET_OK;
    if (!R || (rank > 0 && !U_all)) return RET_ERR_NULL;
    if (!a16(R) || (U_all && !a16(U_all)) || (state_in && !a16(state_in))) return RET_ERR_ALIGN;
    if (!sm100()) return RET_ERR_UNSUPPORTED;
    Params p;
    params_from_desc(desc, &p);
    ScanArgs a{};
    a.rank = rank;
    long long after = 0;  // tokens strictly between segment s and `rank`
    for (int i = rank - 1; i >= 0; --i) {
        a.n[i] = after;
        after += seg_len[i];
    }
    a.n_in = after;
    const long long quads = (long long)(seg_elems / 4);
    const long long blocks = (quads + 255) / 256;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    state_scan_kernel<<<(unsigned)blocks, 256, 0, st>>>(p, a, quads, seg_elems, U_all, state_in, R);
    if (cudaGetLastError() != cudaSuccess) return RET_ERR_CUDA;
    note_launches(1);
    return RET_OK;
}

namespace {

// The checks ret_chunkwise_segmented and its size share; fills p.
ret_status check_segmented(const ret_desc *desc, int chunk, int segments, ret::Params *p) {
    using namespace ret;
    ret_status s = validate_desc(desc);
    if (s != RET_OK) return s;
    if (desc->in_dtype != RET_BF16) return RET_ERR_DTYPE;
    if (chunk < 1 || segments < 1) return RET_ERR_ARG;
    if ((long long)desc->B * desc->L == 0) return RET_ERR_SHAPE;
    params_from_desc(desc, p);
    if (!segmented_supported(*p, chunk, segments)) return RET_ERR_SHAPE;
    return RET_OK;
}

}  // namespace

size_t ret_chunkwise_segmented_workspace_size(const ret_desc *desc, int chunk, int segments) {
    ret::Params p;
    if (check_segmented(desc, chunk, segments, &p) != RET_OK) return 0;
    return ret::seg_layout(p, segments).bytes;
}

ret_status ret_chunkwise_segmented(const ret_desc *desc, int chunk, int segments, const void *Q,
                                   const void *K, const void *V, const float *state_in,
                                   float *state_out, void *O, void *workspace,
                                   size_t workspace_bytes, void *stream) {
    using namespace ret;
    Params p;
    ret_status s = check_segmented(desc, chunk, segments, &p);
    if (s != RET_OK) return s;
    if (!Q || !K || !V || !O) return RET_ERR_NULL;
    if (!a16(Q) || !a16(K) || !a16(V) || !a16(O) || (state_in && !a16(state_in)) ||
        (state_out && !a16(state_out)))
        return RET_ERR_ALIGN;
    if ((reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0) return RET_ERR_ALIGN;
    const SegLayout z = seg_layout(p, segments);
    if (!workspace || workspace_bytes < z.bytes) return RET_ERR_WORKSPACE;
    if (!sm100()) return RET_ERR_UNSUPPORTED;
    int *status = device_status_word();
    if (!status) return RET_ERR_CUDA;
    return launch_segmented(p, segments, desc->out_dtype == RET_BF16, Q, K, V, state_in, state_out,
                            O, nullptr, nullptr, 0.f, workspace, status,
                            static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? RET_OK
               : RET_ERR_CUDA;
}

}  // extern "C"
