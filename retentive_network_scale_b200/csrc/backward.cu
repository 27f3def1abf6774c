// backward.cu -- ret_backward: the gradients of O = Retention(Q, K, V)
// ("Retentive Network" paper summary, section 2.1, forms (1)-(3); the
// parallel and chunkwise forms are the training forms) with respect to Q,
// K and V, given dO, from a zero state.
//
// With q^_t = Theta_t q_t, k^_m = Theta_m k_m and
//   o_t = sum_{m<=t} gamma^{t-m} (q^_t . k^_m) v_m,
// the gradients are
//   dq^_t = sum_{m<=t} gamma^{t-m} (do_t . v_m) k^_m     causal
//   dk^_m = sum_{t>=m} gamma^{t-m} (v_m . do_t) q^_t     anti-causal
//   dv_m  = sum_{t>=m} gamma^{t-m} (k^_m . q^_t) do_t    anti-causal
//   dq_t = Theta_t^T dq^_t,  dk_m = Theta_m^T dk^_m.
// Each is a retention of rearranged operands: (query, key, value) =
// (dO, V, K^) causally, and (V, dO, Q^), (K^, Q^, dO) over the time-reversed
// sequences.  Retention is linear in its scores, so a contraction over d_v
// (the dO . V scores) splits into column blocks of 128 or 256 whose outputs
// add: every product then fits the tensor-core chunkwise kernel.  The
// operands are first copied (bf16) turned and/or time-reversed; the fp32
// partial outputs are summed, turned back and un-reversed at the end.
#include <algorithm>

#include "common.cuh"
#include "launch.h"
#include "retention.h"

namespace ret {
namespace {

constexpr int kThreads = 256;

// y (bf16, [B][H][L][d]) = x turned by the angle of row t's own position
// (ROT) and written at row t or, when `flip`, at row L-1-t.  One thread:
// 8 consecutive elements (4 pairs) of one row.
template <typename TI, bool ROT>
__global__ void __launch_bounds__(kThreads)
flip_turn_kernel(const Params p, int d, long long items, const TI *__restrict__ x,
                 __nv_bfloat16 *__restrict__ y, int flip) {
    __shared__ double s_theta[kMaxDk / 2];
    if constexpr (ROT) {
        stage_theta(p, s_theta, d / 2);
        __syncthreads();
    }
    const long long item = (long long)blockIdx.x * kThreads + threadIdx.x;
    if (item >= items) return;
    const int n8 = d / 8;
    const long long r = item / n8;
    const int c8 = (int)(item - r * n8);
    const int t = (int)(r % p.L);
    const long long rdst = flip ? r - t + (p.L - 1 - t) : r;
    float v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = ld(x, (size_t)r * d + c8 * 8 + e);
    if constexpr (ROT) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            float c, s;
            rot_cs(p.pos_offset + t, s_theta[c8 * 4 + e], &c, &s);
            rot_pair(v[2 * e], v[2 * e + 1], c, s);
        }
    }
    uint4 w;
    uint32_t *u = reinterpret_cast<uint32_t *>(&w);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        __nv_bfloat162 b2 = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
        u[e] = *reinterpret_cast<uint32_t *>(&b2);
    }
    *reinterpret_cast<uint4 *>(y + (size_t)rdst * d + c8 * 8) = w;
}

// out row t = the sum of the fp32 partials at row t (or L-1-t when `flip`),
// turned back by the angle of position pos_offset + t (ROT).
template <typename TO, bool ROT>
__global__ void __launch_bounds__(kThreads)
unturn_sum_kernel(const Params p, int d, long long items, const float *__restrict__ part0,
                  const float *__restrict__ part1, int flip, TO *__restrict__ out) {
    __shared__ double s_theta[kMaxDk / 2];
    if constexpr (ROT) {
        stage_theta(p, s_theta, d / 2);
        __syncthreads();
    }
    const long long item = (long long)blockIdx.x * kThreads + threadIdx.x;
    if (item >= items) return;
    const int n8 = d / 8;
    const long long r = item / n8;
    const int c8 = (int)(item - r * n8);
    const int t = (int)(r % p.L);
    const long long rsrc = flip ? r - t + (p.L - 1 - t) : r;
    float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int k = 0; k < 2; ++k) {
        const float *part = k == 0 ? part0 : part1;
        if (!part) continue;
        const float4 a = *reinterpret_cast<const float4 *>(part + (size_t)rsrc * d + c8 * 8);
        const float4 b = *reinterpret_cast<const float4 *>(part + (size_t)rsrc * d + c8 * 8 + 4);
        v[0] += a.x; v[1] += a.y; v[2] += a.z; v[3] += a.w;
        v[4] += b.x; v[5] += b.y; v[6] += b.z; v[7] += b.w;
    }
    if constexpr (ROT) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            float c, s;
            rot_cs(p.pos_offset + t, s_theta[c8 * 4 + e], &c, &s);
            rot_pair(v[2 * e], v[2 * e + 1], c, -s);  // Theta_t^T: the opposite turn
        }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) st(out, (size_t)r * d + c8 * 8 + e, v[e]);
}

constexpr size_t kAlign = 256;
size_t round_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// column blocks of d_v for the dO . V contractions: 256 wide, then one of 128
int split_dv(int dv, int *w) {  // at most two blocks for d_v <= 512
    int n = 0;
    for (int c = 0; c + 256 <= dv; c += 256) w[n++] = 256;
    if (dv % 256) w[n++] = 128;
    return n;
}

struct BwdLayout {
    size_t kh, qf, kf, vf, of, prep, part_dk, part_dv;  // offsets
    size_t bytes;
    int nsplit;
};

BwdLayout bwd_layout(const ret_desc *d) {
    BwdLayout z{};
    int w[8];
    z.nsplit = split_dv(d->d_v, w);
    const size_t rows = (size_t)d->B * d->H * d->L;
    const size_t bk = rows * d->d_k * 2, bv = rows * d->d_v * 2;
    size_t o = 0;
    z.kh = o; o += round_up(bk);
    z.qf = o; o += round_up(bk);
    z.kf = o; o += round_up(bk);
    z.vf = o; o += round_up(bv);
    z.of = o; o += round_up(bv);
    z.prep = o; o += round_up(2 * rows * 256 * 2);            // prepared Q^, K~ of one call
    z.part_dk = o; o += round_up(rows * d->d_k * 4) * 2 * z.nsplit;  // dQ^, dK^ partials
    z.part_dv = o; o += round_up(rows * d->d_v * 4);
    z.bytes = o;
    return z;
}

template <typename TI>
cudaError_t flip_turn(const Params &p, int d, const void *x, void *y, bool rot, bool flip,
                      cudaStream_t st) {
    const long long items = (long long)p.B * p.H * p.L * (d / 8);
    const long long blocks = (items + kThreads - 1) / kThreads;
    if (rot)
        flip_turn_kernel<TI, true><<<(unsigned)blocks, kThreads, 0, st>>>(
            p, d, items, static_cast<const TI *>(x), static_cast<__nv_bfloat16 *>(y), flip);
    else
        flip_turn_kernel<TI, false><<<(unsigned)blocks, kThreads, 0, st>>>(
            p, d, items, static_cast<const TI *>(x), static_cast<__nv_bfloat16 *>(y), flip);
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) note_launches(1);
    return e;
}

// (d_v <= 512, so a contraction over d_v has at most two column blocks)
template <typename TO>
cudaError_t unturn_sum(const Params &p, int d, const float *part0, const float *part1, bool flip,
                       bool rot, void *out, cudaStream_t st) {
    const long long items = (long long)p.B * p.H * p.L * (d / 8);
    const long long blocks = (items + kThreads - 1) / kThreads;
    if (rot)
        unturn_sum_kernel<TO, true><<<(unsigned)blocks, kThreads, 0, st>>>(p, d, items, part0, part1, flip,
                                                                           static_cast<TO *>(out));
    else
        unturn_sum_kernel<TO, false><<<(unsigned)blocks, kThreads, 0, st>>>(p, d, items, part0, part1, flip,
                                                                            static_cast<TO *>(out));
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) note_launches(1);
    return e;
}

// One retention product on the tensor cores: query/key rows read through
// `qk` (column offset already in the pointers), value rows [B][H][L][dv']
// contiguous, fp32 output [B][H][L][dv'].
cudaError_t product(const Params &base, int dqk, int dval, const void *q, const void *k,
                    RowLayout qk, const void *v, void *prep_ws, float *out, int *status,
                    cudaStream_t st) {
    Params p = base;
    p.dk = dqk;
    p.dv = dval;
    p.rotate = 0;  // the operands come turned already
    // only K~ is written: the query rows are read in place through `qk`
    const void *qh = nullptr, *kt = nullptr;
    cudaError_t e = launch_chunkwise_prep_strided(p, 128, q, k, qk, false, prep_ws, &qh, &kt, st);
    if (e != cudaSuccess) return e;
    return launch_chunkwise_tc_prepared(p, false, qh, qk, kt, v, bhld_layout(p, dval), true,
                                        nullptr, RowLayout{0, 0, 0}, nullptr, out, 0.f, status, st);
}

bool dims_ok(const ret_desc *d) {
    return (d->d_k == 128 || d->d_k == 256) && d->d_v % 128 == 0 && d->d_v <= kMaxDv;
}

}  // namespace
}  // namespace ret

extern "C" {

size_t ret_backward_workspace_size(const ret_desc *desc, int chunk) {
    if (ret::validate_desc(desc) != RET_OK || chunk < 1 || !ret::dims_ok(desc)) return 0;
    if ((long long)desc->B * desc->L == 0) return 0;
    return ret::bwd_layout(desc).bytes;
}

ret_status ret_backward(const ret_desc *desc, int chunk, const void *Q, const void *K,
                        const void *V, const void *dO, void *dQ, void *dK, void *dV,
                        void *workspace, size_t workspace_bytes, void *stream) {
    using namespace ret;
    ret_status s = validate_desc(desc);
    if (s != RET_OK) return s;
    if (desc->in_dtype != RET_BF16) return RET_ERR_DTYPE;
    if (chunk < 1) return RET_ERR_ARG;
    if (!dims_ok(desc)) return RET_ERR_SHAPE;
    Params p;
    params_from_desc(desc, &p);
    // every product runs on the tensor-core path: its decay condition
    if ((long long)desc->B * desc->L > 0 && !chunkwise_tc_supported(p, chunk, true))
        return RET_ERR_SHAPE;
    if ((long long)desc->B * desc->L == 0) return RET_OK;
    if (!Q || !K || !V || !dO || !dQ || !dK || !dV) return RET_ERR_NULL;
    auto a16 = [](const void *q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; };
    if (!a16(Q) || !a16(K) || !a16(V) || !a16(dO) || !a16(dQ) || !a16(dK) || !a16(dV))
        return RET_ERR_ALIGN;
    if ((reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0) return RET_ERR_ALIGN;
    const BwdLayout z = bwd_layout(desc);
    if (!workspace || workspace_bytes < z.bytes) return RET_ERR_WORKSPACE;
    int dev = -1, major = 0, minor = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
        cudaGetLastError();
        return RET_ERR_UNSUPPORTED;
    }
    if (major != 10 || minor != 0) return RET_ERR_UNSUPPORTED;
    int *status = device_status_word();
    if (!status) return RET_ERR_CUDA;

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    const int dk = desc->d_k, dv = desc->d_v;
    const bool rot = desc->rotate != 0;
    const size_t rows = (size_t)desc->B * desc->H * desc->L;
    void *Kh = ws + z.kh, *Qf = ws + z.qf, *Kf = ws + z.kf, *Vf = ws + z.vf, *Of = ws + z.of;
    void *prep = ws + z.prep;
    float *partA = reinterpret_cast<float *>(ws + z.part_dk);
    const size_t part_stride = round_up(rows * dk * 4) / 4;      // floats between partials
    float *partB = partA + part_stride * z.nsplit;
    float *partC = reinterpret_cast<float *>(ws + z.part_dv);

    cudaError_t e = cudaSuccess;
    auto run = [&](cudaError_t r) { if (e == cudaSuccess) e = r; };
    // 1. turned and/or time-reversed bf16 copies
    run(flip_turn<__nv_bfloat16>(p, dk, K, Kh, rot, false, st));
    run(flip_turn<__nv_bfloat16>(p, dk, Q, Qf, rot, true, st));
    run(flip_turn<__nv_bfloat16>(p, dk, K, Kf, rot, true, st));
    run(flip_turn<__nv_bfloat16>(p, dv, V, Vf, false, true, st));
    run(flip_turn<__nv_bfloat16>(p, dv, dO, Of, false, true, st));
    // 2. dQ^ (causal: dO, V, K^) and reversed dK^ (V, dO, Q^), per column block of d_v
    int w[8];
    const int n = split_dv(dv, w);
    const RowLayout full_v = bhld_layout(p, dv);
    const auto *dO8 = static_cast<const uint8_t *>(dO), *V8 = static_cast<const uint8_t *>(V);
    for (int i = 0, c0 = 0; i < n && e == cudaSuccess; c0 += w[i], ++i) {
        const size_t off = (size_t)c0 * 2;
        run(product(p, w[i], dk, dO8 + off, V8 + off, full_v, Kh, prep, partA + i * part_stride,
                    status, st));
        run(product(p, w[i], dk, static_cast<uint8_t *>(Vf) + off, static_cast<uint8_t *>(Of) + off,
                    full_v, Qf, prep, partB + i * part_stride, status, st));
    }
    // 3. reversed dV (K^, Q^, dO)
    run(product(p, dk, dv, Kf, Qf, bhld_layout(p, dk), Of, prep, partC, status, st));
    // 4. sums, the opposite turn, and back to forward time
    const float *a1 = n > 1 ? partA + part_stride : nullptr;
    const float *b1 = n > 1 ? partB + part_stride : nullptr;
    if (desc->out_dtype == RET_BF16) {
        run(unturn_sum<__nv_bfloat16>(p, dk, partA, a1, false, rot, dQ, st));
        run(unturn_sum<__nv_bfloat16>(p, dk, partB, b1, true, rot, dK, st));
        run(unturn_sum<__nv_bfloat16>(p, dv, partC, nullptr, true, false, dV, st));
    } else {
        run(unturn_sum<float>(p, dk, partA, a1, false, rot, dQ, st));
        run(unturn_sum<float>(p, dk, partB, b1, true, rot, dK, st));
        run(unturn_sum<float>(p, dv, partC, nullptr, true, false, dV, st));
    }
    return e == cudaSuccess ? RET_OK : RET_ERR_CUDA;
}

}  // extern "C"
