// seqshard.cu -- ret_segment_state and ret_state_scan: a long sequence cut
// into consecutive segments (one per device), joined through their states.
//
// "Retentive Network" paper summary, section 2.1, chunkwise form (3):
// parallel inside a block of rows, a decayed state carried between blocks.
// The same recurrence holds between segments of any length: a segment of n
// rows that starts from state R leaves
//     R' = gamma^n R + U,   U = sum_{t<n} gamma^{n-1-t} k^_t^T v_t,
// where U depends on the segment alone.  So every device computes the U of
// its own segment at once (a streaming pass that turns and decay-weights the
// keys, then one batched GEMM), the U are exchanged (an all-gather), and a
// scan gives each segment its entering state; the segment's outputs then
// come from ret_chunkwise started from that state.
#include <mutex>

#include "launch.h"
#include "retention.h"

namespace ret {
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

}  // namespace
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
    // U_bh [d_k][d_v] = K~_bh^T V_bh, i.e. in column-major terms the
    // (d_v x d_k) product V_cm (d_v x L) * K~_cm^T (L x d_k)
    std::lock_guard<std::mutex> lock(blas_mutex());
    cublasHandle_t h = blas_handle(st, ws + round_up((size_t)bh * desc->L * desc->d_k * 2));
    if (!h) return RET_ERR_CUDA;
    const float one = 1.f, zero = 0.f;
    const long long L = desc->L, dk = desc->d_k, dv = desc->d_v;
    const cublasStatus_t r = cublasGemmStridedBatchedEx(
        h, CUBLAS_OP_N, CUBLAS_OP_T, (int)dv, (int)dk, (int)L, &one, V, CUDA_R_16BF, (int)dv,
        L * dv, kt, CUDA_R_16BF, (int)dk, L * dk, &zero, U, CUDA_R_32F, (int)dv, dk * dv, (int)bh,
        CUBLAS_COMPUTE_32F, CUBLAS_GEMM_DEFAULT);
    return r == CUBLAS_STATUS_SUCCESS ? RET_OK : RET_ERR_CUDA;
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

}  // extern "C"
