// msr_layer.cu -- ret_msr_layer: the multi-scale retention layer around the
// chunkwise kernel.
//
// "Retentive Network" paper summary, section 2.1 (Q = (X W_Q) (.) Theta,
// K = (X W_K) (.) conj(Theta), V = X W_V, one decay per head) and section
// 2.2 (Y = GroupNorm_h(Concat(heads)); MSR(X) = (swish(X W_G) (.) Y) W_O):
//   P   = X [W_Q | W_K | W_V | W_G]          one bf16 GEMM, fp32 accumulate,
//                                            whose epilogue writes the Q and
//                                            K columns as Q^ and K~ (turned,
//                                            keys decay-weighted) per head
//   Y   = swish(G) (.) GroupNorm_h(O)        the fused chunkwise kernel, with
//                                            V and G read from P through
//                                            strided tensor maps
//   out = Y W_O                              one bf16 GEMM, fp32 accumulate
// Three launches, all this library's own kernels (the GEMM is gemm_tc.cu);
// nothing between them round-trips through a separate layout pass.
#include "launch.h"
#include "retention.h"

namespace {

constexpr int kMaxDevices = 64;
constexpr size_t kAlign = 256;

size_t round_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

struct LayerSizes {
    long long rows;   // B*L
    long long n_proj; // H*(2 d_k + 2 d_v)
    size_t proj, prep, y, off_prep, off_y, bytes;
};

LayerSizes sizes_of(const ret_desc *d) {
    LayerSizes s{};
    s.rows = (long long)d->B * d->L;
    s.n_proj = (long long)d->H * (2LL * d->d_k + 2LL * d->d_v);
    s.proj = (size_t)s.rows * s.n_proj * 2;
    s.prep = 2ull * s.rows * d->H * d->d_k * 2;
    s.y = (size_t)s.rows * d->H * d->d_v * 2;
    s.off_prep = round_up(s.proj);
    s.off_y = s.off_prep + round_up(s.prep);
    s.bytes = s.off_y + round_up(s.y);
    return s;
}

}  // namespace


extern "C" {

size_t ret_msr_layer_workspace_size(const ret_desc *desc, int d_model, int chunk) {
    if (ret::validate_desc(desc) != RET_OK || d_model < 8 || d_model % 8 || chunk < 1) return 0;
    if ((long long)desc->B * desc->L == 0) return 0;
    return sizes_of(desc).bytes;
}

ret_status ret_msr_layer(const ret_desc *desc, int d_model, int chunk, const void *X,
                         const void *W_qkvg, const void *W_o, float gn_eps, void *out,
                         void *workspace, size_t workspace_bytes, void *stream) {
    ret_status s = ret::validate_desc(desc);
    if (s != RET_OK) return s;
    if (desc->in_dtype != RET_BF16 || desc->out_dtype != RET_BF16) return RET_ERR_DTYPE;
    if (d_model < 8 || d_model % 8) return RET_ERR_SHAPE;
    if (chunk < 1 || !(gn_eps >= 0.0f && gn_eps < 3.0e38f)) return RET_ERR_ARG;
    ret::Params p;
    ret::params_from_desc(desc, &p);
    // the layer runs on the tensor-core chunkwise path only, at the head
    // shapes its tests cover (d_k 128 or 256, d_v a multiple of 128)
    if ((long long)desc->B * desc->L > 0 &&
        (!ret::chunkwise_tc_supported(p, chunk, true) || (p.dk != 128 && p.dk != 256) ||
         p.dv % 128 != 0))
        return RET_ERR_SHAPE;
    if ((long long)desc->B * desc->L == 0) return RET_OK;
    if (!X || !W_qkvg || !W_o || !out) return RET_ERR_NULL;
    auto a16 = [](const void *q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; };
    if (!a16(X) || !a16(W_qkvg) || !a16(W_o) || !a16(out)) return RET_ERR_ALIGN;
    if ((reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0) return RET_ERR_ALIGN;
    const LayerSizes z = sizes_of(desc);
    if (!workspace || workspace_bytes < z.bytes) return RET_ERR_WORKSPACE;
    int dev = -1, major = 0, minor = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
        cudaGetLastError();
        return RET_ERR_UNSUPPORTED;
    }
    if (major != 10 || minor != 0) return RET_ERR_UNSUPPORTED;
    int *status = ret::device_status_word();
    if (!status) return RET_ERR_CUDA;

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);

    const int H = desc->H, dk = desc->d_k, dv = desc->d_v;
    const auto *P = reinterpret_cast<const __nv_bfloat16 *>(ws);
    // 1. the four projections in one product, whose epilogue turns the Q
    //    and K columns (and weights the keys) into [B][H][L][d_k] arrays
    uint8_t *qh = ws + z.off_prep;
    uint8_t *kt = qh + z.prep / 2;
    if (ret::launch_gemm_proj(p, d_model, X, W_qkvg, ws, qh, kt, status, st) != cudaSuccess)
        return RET_ERR_CUDA;
    // 2. the chunk loop with the fused GroupNorm + gate; V and G are read as
    //    rows of H d_v columns of the projection
    const ret::RowLayout vg{z.n_proj, 0, (long long)desc->L * z.n_proj};
    cudaError_t e = ret::launch_chunkwise_tc_prepared(p, true, qh, ret::bhld_layout(p, dk), kt,
                                                      P + 2 * (size_t)H * dk, vg, false,
                                                      P + 2 * (size_t)H * dk + (size_t)H * dv, vg,
                                                      ws + z.off_y, nullptr, gn_eps, status, st);
    if (e != cudaSuccess) return RET_ERR_CUDA;
    // 3. the output projection
    const long long hdv = (long long)H * dv;
    if (ret::launch_gemm_tc(z.rows, d_model, hdv, ws + z.off_y, hdv, W_o, d_model, out, d_model,
                            status, st) != cudaSuccess)
        return RET_ERR_CUDA;
    return RET_OK;
}

}  // extern "C"
