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
// (dO, V, K^) causally, and (V, dO, Q^), (K^, Q^, dO) anti-causally, which
// the tensor-core chunk loop runs in its reverse mode (blocks from last to
// first, mirrored mask and weights) on the operands as they are.
// Retention is linear in its scores, so a contraction over d_v (the dO . V
// scores) splits into column blocks of 128 or 256 whose outputs add: every
// product then fits the tensor-core chunkwise kernel.  With rotation, Q and
// K are first copied turned (bf16); the fp32 partial outputs are summed and
// turned back at the end.
#include <algorithm>

#include "common.cuh"
#include "launch.h"
#include "retention.h"

namespace ret {
namespace {

constexpr int kThreads = 256;
constexpr int kRows = 4;  // consecutive rows per thread in the copy passes

__device__ __forceinline__ uint4 ld_stream(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ float4 ld_stream_f4(const float *p) {
    const uint4 u = ld_stream(p);
    return make_float4(__uint_as_float(u.x), __uint_as_float(u.y), __uint_as_float(u.z),
                       __uint_as_float(u.w));
}

// One copy-pass work item: the 8-column chunk c8 of rows t0 .. t0+nr-1 of
// slice bh.  Items run chunk-fastest, so a warp reads whole rows.
struct CopyItem {
    int c8, t0, nr;
    long long bh;
};

__device__ __forceinline__ bool copy_item(const Params &p, int d, long long items, CopyItem *it) {
    const long long item = (long long)blockIdx.x * kThreads + threadIdx.x;
    if (item >= items) return false;
    const int n8 = d / 8;
    const int tiles = (p.L + kRows - 1) / kRows;
    it->c8 = (int)(item % n8);
    const long long rest = item / n8;
    it->t0 = (int)(rest % tiles) * kRows;
    it->bh = rest / tiles;
    it->nr = min(kRows, p.L - it->t0);
    return true;
}

// Angles of the four pairs of chunk c8 at position pos, and the per-row
// step theta_j: the first exact (fp64 reduction), the rest by rotation.
__device__ __forceinline__ void chunk_angles(const double *s_theta, int c8, long long pos, float *c,
                                             float *s, float *cs, float *ss) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const double th = s_theta[c8 * 4 + e];
        rot_cs_fast(pos, th, &c[e], &s[e]);
        __sincosf((float)th, &ss[e], &cs[e]);  // theta_j <= 1
    }
}

__device__ __forceinline__ void step_angles(float *c, float *s, const float *cs, const float *ss) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float cn = c[e] * cs[e] - s[e] * ss[e];
        s[e] = c[e] * ss[e] + s[e] * cs[e];
        c[e] = cn;
    }
}

// y (bf16, [B][H][L][d]) = x turned by the angle of row t's own position
// (ROT) and written at row t or, when `flip`, at row L-1-t.
template <bool ROT>
__global__ void __launch_bounds__(kThreads, 4)
flip_turn_kernel(const Params p, int d, long long items, const __nv_bfloat16 *__restrict__ x,
                 __nv_bfloat16 *__restrict__ y, int flip) {
    __shared__ double s_theta[kMaxDk / 2];
    if constexpr (ROT) {
        stage_theta(p, s_theta, d / 2);
        __syncthreads();
    }
    CopyItem it;
    if (!copy_item(p, d, items, &it)) return;
    const size_t base = (size_t)it.bh * p.L * d + (size_t)it.c8 * 8;
    uint4 w[kRows];
#pragma unroll
    for (int r = 0; r < kRows; ++r)
        if (r < it.nr) w[r] = ld_stream(x + base + (size_t)(it.t0 + r) * d);
    float c[4], s[4], cs[4], ss[4];
    if constexpr (ROT) chunk_angles(s_theta, it.c8, p.pos_offset + it.t0, c, s, cs, ss);
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
        if (r < it.nr) {
            if constexpr (ROT) {
                uint32_t *u = reinterpret_cast<uint32_t *>(&w[r]);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    float2 v = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&u[e]));
                    rot_pair(v.x, v.y, c[e], s[e]);
                    __nv_bfloat162 b2 = __floats2bfloat162_rn(v.x, v.y);
                    u[e] = *reinterpret_cast<uint32_t *>(&b2);
                }
                step_angles(c, s, cs, ss);
            }
            const int t = it.t0 + r;
            *reinterpret_cast<uint4 *>(y + base + (size_t)(flip ? p.L - 1 - t : t) * d) = w[r];
        }
    }
}

template <typename TO>
__device__ __forceinline__ void st8(TO *dst, const float *v);
template <>
__device__ __forceinline__ void st8<float>(float *dst, const float *v) {
    reinterpret_cast<float4 *>(dst)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4 *>(dst)[1] = make_float4(v[4], v[5], v[6], v[7]);
}
template <>
__device__ __forceinline__ void st8<__nv_bfloat16>(__nv_bfloat16 *dst, const float *v) {
    uint4 w;
    uint32_t *u = reinterpret_cast<uint32_t *>(&w);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        __nv_bfloat162 b2 = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
        u[e] = *reinterpret_cast<uint32_t *>(&b2);
    }
    *reinterpret_cast<uint4 *>(dst) = w;
}

// out row t = the sum of the fp32 partials at row t (or L-1-t when `flip`),
// turned back by the angle of position pos_offset + t (ROT).
template <typename TO, bool ROT>
__global__ void __launch_bounds__(kThreads, 4)
unturn_sum_kernel(const Params p, int d, long long items, const float *__restrict__ part0,
                  const float *__restrict__ part1, int flip, TO *__restrict__ out) {
    __shared__ double s_theta[kMaxDk / 2];
    if constexpr (ROT) {
        stage_theta(p, s_theta, d / 2);
        __syncthreads();
    }
    CopyItem it;
    if (!copy_item(p, d, items, &it)) return;
    const size_t base = (size_t)it.bh * p.L * d + (size_t)it.c8 * 8;
    float4 a[kRows][2];
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
        if (r < it.nr) {
            const int t = it.t0 + r;
            const size_t src = base + (size_t)(flip ? p.L - 1 - t : t) * d;
            a[r][0] = ld_stream_f4(part0 + src);
            a[r][1] = ld_stream_f4(part0 + src + 4);
            if (part1) {
                const float4 b0 = ld_stream_f4(part1 + src), b1 = ld_stream_f4(part1 + src + 4);
                a[r][0].x += b0.x; a[r][0].y += b0.y; a[r][0].z += b0.z; a[r][0].w += b0.w;
                a[r][1].x += b1.x; a[r][1].y += b1.y; a[r][1].z += b1.z; a[r][1].w += b1.w;
            }
        }
    }
    float c[4], s[4], cs[4], ss[4];
    if constexpr (ROT) chunk_angles(s_theta, it.c8, p.pos_offset + it.t0, c, s, cs, ss);
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
        if (r < it.nr) {
            float v[8] = {a[r][0].x, a[r][0].y, a[r][0].z, a[r][0].w,
                          a[r][1].x, a[r][1].y, a[r][1].z, a[r][1].w};
            if constexpr (ROT) {
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    rot_pair(v[2 * e], v[2 * e + 1], c[e], -s[e]);  // Theta_t^T: the opposite turn
                step_angles(c, s, cs, ss);
            }
            st8<TO>(out + base + (size_t)(it.t0 + r) * d, v);
        }
    }
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
    size_t kh, qh, prep, part_dk, part_dv;  // offsets (prep: two buffers)
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
    (void)bv;
    z.kh = o; o += d->rotate ? round_up(bk) : 0;  // turned K and Q
    z.qh = o; o += d->rotate ? round_up(bk) : 0;
    z.prep = o; o += round_up(2 * rows * 256 * 2) * 2;  // weighted keys of two products
    z.part_dk = o; o += round_up(rows * d->d_k * 4) * 2 * z.nsplit;  // dQ^, dK^ partials
    z.part_dv = o; o += round_up(rows * d->d_v * 4);
    z.bytes = o;
    return z;
}

long long copy_items(const Params &p, int d) {
    return (long long)p.B * p.H * ((p.L + kRows - 1) / kRows) * (d / 8);
}

cudaError_t flip_turn(const Params &p, int d, const void *x, void *y, bool rot, bool flip,
                      cudaStream_t st) {
    const long long items = copy_items(p, d);
    const long long blocks = (items + kThreads - 1) / kThreads;
    const auto *xs = static_cast<const __nv_bfloat16 *>(x);
    auto *yd = static_cast<__nv_bfloat16 *>(y);
    if (rot)
        flip_turn_kernel<true><<<(unsigned)blocks, kThreads, 0, st>>>(p, d, items, xs, yd, flip);
    else
        flip_turn_kernel<false><<<(unsigned)blocks, kThreads, 0, st>>>(p, d, items, xs, yd, flip);
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) note_launches(1);
    return e;
}

// (d_v <= 512, so a contraction over d_v has at most two column blocks)
template <typename TO>
cudaError_t unturn_sum(const Params &p, int d, const float *part0, const float *part1, bool flip,
                       bool rot, void *out, cudaStream_t st) {
    const long long items = copy_items(p, d);
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
// contiguous, fp32 output [B][H][L][dv'].  With acc_in the output is
// acc_in + the product, turned back by the rows' angles when `unturn`.
// It is two launches: the streaming pass that writes the weighted key rows
// K~ into prep_ws (product_keys), then the chunk loop (product_loop), so
// that the pass of the next product can run beside this one's loop.
Params product_params(const Params &base, int dqk, int dval, bool anti) {
    Params p = base;
    p.dk = dqk;
    p.dv = dval;
    p.rotate = 0;  // the operands come turned already
    p.reverse = anti ? 1 : 0;
    return p;
}

cudaError_t product_keys(const Params &p, const void *q, const void *k, RowLayout qk,
                         void *prep_ws, const void **kt, cudaStream_t st) {
    // only K~ is written: the query rows are read in place through `qk`
    const void *qh = nullptr;
    return launch_chunkwise_prep_strided(p, 128, q, k, qk, false, prep_ws, &qh, kt, st);
}

cudaError_t product_loop(const Params &p, const void *q, RowLayout qk, const void *kt,
                         const void *v, float *out, int *status, cudaStream_t st,
                         const float *acc_in = nullptr, bool unturn = false) {
    return launch_chunkwise_ws(p, false, q, qk, kt, bhld_layout(p, p.dk), v, bhld_layout(p, p.dv), true,
                               nullptr, nullptr, out, nullptr, RowLayout{0, 0, 0}, nullptr, 0.f, false,
                               false, status, st, acc_in, unturn ? 1 : 0);
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
    const void *Kh = rot ? static_cast<const void *>(ws + z.kh) : K;
    const void *Qh = rot ? static_cast<const void *>(ws + z.qh) : Q;
    void *prep = ws + z.prep;
    float *partA = reinterpret_cast<float *>(ws + z.part_dk);
    const size_t part_stride = round_up(rows * dk * 4) / 4;      // floats between partials
    float *partB = partA + part_stride * z.nsplit;
    // dV needs neither a second partial nor a turn: in fp32 the product
    // writes it in place
    const bool dv_direct = desc->out_dtype == RET_F32;
    float *partC = dv_direct ? static_cast<float *>(dV) : reinterpret_cast<float *>(ws + z.part_dv);

    cudaError_t e = cudaSuccess;
    auto run = [&](cudaError_t r) { if (e == cudaSuccess) e = r; };
    // The products, in order: dQ^ (causal: dO, V, K^) and dK^ (anti-causal:
    // V, dO, Q^) per column block of d_v, then dV (anti-causal: K^, Q^, dO).
    // In fp32 with two column blocks, the second block's products add the
    // first block's partials and turn the sums back in their epilogue,
    // writing dQ and dK themselves (no sum pass).
    struct Prod {
        Params p;
        const void *q, *k, *v;
        RowLayout qk;
        float *out;
        const float *acc_in;
        bool unturn, needs_qh;
    };
    Prod prods[2 * 8 + 1];
    int np = 0;
    int w[8];
    const int n = split_dv(dv, w);
    const RowLayout full_v = bhld_layout(p, dv);
    const auto *dO8 = static_cast<const uint8_t *>(dO), *V8 = static_cast<const uint8_t *>(V);
    const bool fold = desc->out_dtype == RET_F32 && n == 2;
    for (int i = 0, c0 = 0; i < n; c0 += w[i], ++i) {
        const size_t off = (size_t)c0 * 2;
        const bool last = fold && i == 1;
        prods[np++] = Prod{product_params(p, w[i], dk, false), dO8 + off, V8 + off, Kh, full_v,
                           last ? static_cast<float *>(dQ) : partA + i * part_stride,
                           last ? partA : nullptr, rot, false};
        prods[np++] = Prod{product_params(p, w[i], dk, true), V8 + off, dO8 + off, Qh, full_v,
                           last ? static_cast<float *>(dK) : partB + i * part_stride,
                           last ? partB : nullptr, rot, false};
    }
    prods[np++] = Prod{product_params(p, dk, dv, true), Kh, Qh, dO, bhld_layout(p, dk), partC,
                       nullptr, false, true};
    const size_t prep_b = round_up(2 * rows * 256 * 2);
    void *prep_buf[2] = {prep, static_cast<uint8_t *>(prep) + prep_b};
    const void *kt[2 * 8 + 1] = {};

    SideStreamRef side{};
    if (side_stream_ref(&side)) {
        // The weighting passes run on the side stream, each ahead of its
        // product, in two buffers used in turn: the pass of product j+1
        // fills the SMs that product j's loop (one wave or less) leaves
        // free, so only the first pass is exposed.  Events: ready = a pass
        // is done; aux[0..1] = the loop that read buffer 0 / 1 is done;
        // aux[2] = the turned copies are written.
        std::lock_guard<std::mutex> lock(*side.mu);
        run(cudaEventRecord(side.start, st));
        run(cudaStreamWaitEvent(side.s, side.start, 0));
        // 1. turned bf16 copies of K and Q, beside the first passes (which
        //    read V and dO only)
        if (rot) {
            run(flip_turn(p, dk, K, ws + z.kh, true, false, st));
            run(flip_turn(p, dk, Q, ws + z.qh, true, false, st));
        }
        run(cudaEventRecord(side.aux[2], st));
        // 2. the products
        for (int j = 0; j < np && e == cudaSuccess; ++j) {
            const Prod &r = prods[j];
            if (j >= 2) run(cudaStreamWaitEvent(side.s, side.aux[j % 2], 0));
            if (r.needs_qh) run(cudaStreamWaitEvent(side.s, side.aux[2], 0));
            run(product_keys(r.p, r.q, r.k, r.qk, prep_buf[j % 2], &kt[j], side.s));
            run(cudaEventRecord(side.ready, side.s));
            run(cudaStreamWaitEvent(st, side.ready, 0));
            run(product_loop(r.p, r.q, r.qk, kt[j], r.v, r.out, status, st, r.acc_in, r.unturn));
            run(cudaEventRecord(side.aux[j % 2], st));
        }
    } else {
        // no side stream: everything in order on the caller's stream
        if (rot) {
            run(flip_turn(p, dk, K, ws + z.kh, true, false, st));
            run(flip_turn(p, dk, Q, ws + z.qh, true, false, st));
        }
        for (int j = 0; j < np && e == cudaSuccess; ++j) {
            const Prod &r = prods[j];
            run(product_keys(r.p, r.q, r.k, r.qk, prep_buf[0], &kt[j], st));
            run(product_loop(r.p, r.q, r.qk, kt[j], r.v, r.out, status, st, r.acc_in, r.unturn));
        }
    }
    // 4. sums and the opposite turn
    const float *a1 = n > 1 ? partA + part_stride : nullptr;
    const float *b1 = n > 1 ? partB + part_stride : nullptr;
    if (desc->out_dtype == RET_BF16) {
        run(unturn_sum<__nv_bfloat16>(p, dk, partA, a1, false, rot, dQ, st));
        run(unturn_sum<__nv_bfloat16>(p, dk, partB, b1, false, rot, dK, st));
        run(unturn_sum<__nv_bfloat16>(p, dv, partC, nullptr, false, false, dV, st));
    } else if (!fold) {
        run(unturn_sum<float>(p, dk, partA, a1, false, rot, dQ, st));
        run(unturn_sum<float>(p, dk, partB, b1, false, rot, dK, st));
    }
    // (fp32 dV was written by its product)
    return e == cudaSuccess ? RET_OK : RET_ERR_CUDA;
}

}  // extern "C"
