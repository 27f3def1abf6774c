// prep.cu -- the two operands of the tensor-core chunkwise kernel that depend
// on the row position, prepared in one streaming pass over Q and K.
//
// "Retentive Network" paper summary, section 2.1: retention turns Q and K by
// the xPos angles (q^_t = Theta_t q_t, k^_t = Theta_t k_t), and the
// chunkwise form (3) weights key row j of a chunk of n rows by
// gamma^{n-1-j} in the state update.  The tensor-core kernel multiplies
//   Q^_t = Theta_t Q_t                        (Q itself without rotation)
//   K~_t = zeta_t Theta_t K_t,  zeta_t = gamma_h^{n-1-j}
// (t = chunk start + j; zeta_t = gamma_h^j for the anti-causal products of
// the backward pass, whose chunk loop runs from the last block to the first).  Computing them here, once per row, takes the
// turn off the kernel's critical path; inside the kernel the CUDA cores
// would turn each tile while the tensor cores wait, and every CTA of a head
// would turn the same rows.  The kernel then loads the prepared rows from
// the workspace by TMA.
//
// Layout: workspace = [Q^ : B*H*L*d_k bf16][K~ : B*H*L*d_k bf16] with
// rotation, [K~] without.  One thread takes one 16-byte column chunk (four
// pairs) of kRows consecutive rows of one (b, h): every load is issued
// before the arithmetic, Q and K share the angles, and the angles advance
// from the first one (reduced in fp64) by the per-row step theta_j.  Four
// rows per thread and four CTAs per SM keep the most bytes in flight (a
// measured choice: it reaches about 88% of the copy bandwidth).
#include <algorithm>

#include "common.cuh"
#include "launch.h"

namespace ret {
namespace {

constexpr int kRows = 4;
constexpr int kThreads = 256;

__device__ __forceinline__ uint4 ld_stream(const __nv_bfloat16 *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t pack2(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&v);
}

__device__ __forceinline__ float2 unpack2(uint32_t u) {
    return __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&u));
}

// ROT: turn Q and K (else K is only scaled); WQ: write Q^ (turned, or
// copied as it is when the source layout differs from the kernel's).
template <bool ROT, bool WQ>
__global__ void __launch_bounds__(kThreads, 4)
chunk_prep_kernel(const Params p, int chunk, long long items, const __nv_bfloat16 *__restrict__ Q,
                  const __nv_bfloat16 *__restrict__ K, RowLayout src, __nv_bfloat16 *__restrict__ qh,
                  __nv_bfloat16 *__restrict__ kt) {
    __shared__ double s_theta[kMaxDk / 2];
    if constexpr (ROT) {
        stage_theta(p, s_theta, p.dk / 2);
        __syncthreads();
    }
    const long long item = (long long)blockIdx.x * kThreads + threadIdx.x;
    if (item >= items) return;
    const int nch = p.dk / 8;
    const int tiles = (p.L + kRows - 1) / kRows;
    const int c16 = (int)(item % nch);
    const long long rest = item / nch;
    const int t0 = (int)(rest % tiles) * kRows;
    const int bh = (int)(rest / tiles);
    const int nr = min(kRows, p.L - t0);
    const size_t base = ((size_t)bh * p.L + t0) * p.dk + (size_t)c16 * 8;  // destination
    const size_t sbase = (size_t)(bh / p.H) * src.batch + (size_t)(bh % p.H) * src.head +
                         (size_t)t0 * src.row + (size_t)c16 * 8;

    uint4 xk[kRows], xq[kRows];
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
        if (r < nr) {
            xk[r] = ld_stream(K + sbase + (size_t)r * src.row);
            if constexpr (WQ) xq[r] = ld_stream(Q + sbase + (size_t)r * src.row);
        }
    }
    float c[4], s[4], cs[4], ss[4];
    if constexpr (ROT) {
        const long long pos0 =
            p.pos_offset + (long long)((bh % p.H) % p.seg_heads) * p.seg_len + t0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const double th = s_theta[c16 * 4 + e];
            rot_cs_fast(pos0, th, &c[e], &s[e]);
            __sincosf((float)th, &ss[e], &cs[e]);  // theta_j <= 1
        }
    }
    const float lg = p.log2g[bh % p.H];
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
        if (r < nr) {
            const int t = t0 + r, j = t % chunk;
            const int n = min(chunk, p.L - (t - j));
            const float z = decay_pow(lg, p.reverse ? j : n - 1 - j);
            uint32_t *uk = reinterpret_cast<uint32_t *>(&xk[r]);
            uint32_t *uq = reinterpret_cast<uint32_t *>(&xq[r]);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 k2 = unpack2(uk[e]);
                if constexpr (ROT) {
                    const float zc = z * c[e], zs = z * s[e];
                    if constexpr (WQ) {
                        const float2 q2 = unpack2(uq[e]);
                        uq[e] = pack2(q2.x * c[e] - q2.y * s[e], q2.x * s[e] + q2.y * c[e]);
                    }
                    uk[e] = pack2(k2.x * zc - k2.y * zs, k2.x * zs + k2.y * zc);
                    const float cn = c[e] * cs[e] - s[e] * ss[e];
                    s[e] = c[e] * ss[e] + s[e] * cs[e];
                    c[e] = cn;
                } else {
                    uk[e] = pack2(k2.x * z, k2.y * z);
                }
            }
            *reinterpret_cast<uint4 *>(kt + base + (size_t)r * p.dk) = xk[r];
            if constexpr (WQ) *reinterpret_cast<uint4 *>(qh + base + (size_t)r * p.dk) = xq[r];
        }
    }
}

}  // namespace

size_t chunkwise_prep_bytes(const Params &p) {
    const size_t one = (size_t)p.B * p.H * p.L * p.dk * sizeof(__nv_bfloat16);
    return p.rotate ? 2 * one : one;
}

cudaError_t launch_chunkwise_prep(const Params &p, int chunk, const void *Q, const void *K,
                                  void *workspace, const void **q_used, const void **k_used,
                                  cudaStream_t st) {
    return launch_chunkwise_prep_strided(p, chunk, Q, K, bhld_layout(p, p.dk), false, workspace,
                                         q_used, k_used, st);
}

cudaError_t launch_chunkwise_prep_strided(const Params &p, int chunk, const void *Q, const void *K,
                                          RowLayout src, bool always_q, void *workspace,
                                          const void **q_used, const void **k_used,
                                          cudaStream_t st) {
    const size_t rows = (size_t)p.B * p.H * p.L;
    const bool wq = p.rotate || always_q;
    __nv_bfloat16 *ws = static_cast<__nv_bfloat16 *>(workspace);
    __nv_bfloat16 *qh = wq ? ws : nullptr;
    __nv_bfloat16 *kt = wq ? ws + rows * p.dk : ws;
    const long long items =
        (long long)p.B * p.H * ((p.L + kRows - 1) / kRows) * (p.dk / 8);
    const long long blocks = (items + kThreads - 1) / kThreads;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
    const auto *q = static_cast<const __nv_bfloat16 *>(Q);
    const auto *k = static_cast<const __nv_bfloat16 *>(K);
    if (p.rotate)
        chunk_prep_kernel<true, true><<<(unsigned)blocks, kThreads, 0, st>>>(p, chunk, items, q, k, src, qh, kt);
    else if (wq)
        chunk_prep_kernel<false, true><<<(unsigned)blocks, kThreads, 0, st>>>(p, chunk, items, q, k, src, qh, kt);
    else
        chunk_prep_kernel<false, false><<<(unsigned)blocks, kThreads, 0, st>>>(p, chunk, items, q, k, src, qh, kt);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    note_launches(1);
    *q_used = wq ? qh : Q;
    *k_used = kt;
    return cudaSuccess;
}

cudaError_t launch_key_prep(const Params &p, int chunk, const void *K, void *kt,
                            cudaStream_t st) {
    const long long items =
        (long long)p.B * p.H * ((p.L + kRows - 1) / kRows) * (p.dk / 8);
    const long long blocks = (items + kThreads - 1) / kThreads;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
    const auto *k = static_cast<const __nv_bfloat16 *>(K);
    auto *out = static_cast<__nv_bfloat16 *>(kt);
    const RowLayout src = bhld_layout(p, p.dk);
    if (p.rotate)
        chunk_prep_kernel<true, false><<<(unsigned)blocks, kThreads, 0, st>>>(p, chunk, items, k, k, src, nullptr, out);
    else
        chunk_prep_kernel<false, false><<<(unsigned)blocks, kThreads, 0, st>>>(p, chunk, items, k, k, src, nullptr, out);
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) note_launches(1);
    return e;
}

}  // namespace ret
