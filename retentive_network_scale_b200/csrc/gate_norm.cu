// gate_norm.cu -- Y = swish(G) (.) GroupNorm_h(O), one group per head taken
// per token over its d_v channels ("Retentive Network" paper summary,
// section 2.2, the MSR equation; population variance, no affine terms).
//
// Bound by HBM (read O and G, write Y).  One warp per (b, t, h) row: each
// lane holds up to 16 of the row's d_v <= 512 values in registers as
// loaded (4-wide vector loads, O and G requested together), so the mean and
// variance (one pass of shifted sums) need no second read of memory.  The
// arithmetic runs on pairs of fp32 values and the sigmoid on the fast
// exponential and reciprocal, since a plain version is bound by instruction
// issue rather than by memory.
//
// The backward (gate_norm_backward_kernel) takes dY to dO and dG by the
// chain rule through the same three steps, with the same row ownership:
// n = (o - mu) r, r = 1/sqrt(var + eps); dG = dY n swish'(G) with
// swish'(g) = sigmoid(g) (1 + g (1 - sigmoid(g))); dn = dY swish(G);
// dO = r (dn - mean(dn) - n mean(dn n)).  O, G and dY are each read once,
// all three requested before the first reduction and held as loaded (dn
// in fp32) between the reductions; dO and dG are written once.  The kernel
// is bound by instruction issue, so the row statistics take one shifted
// pass, the sigmoid the fast exponential and reciprocal, and the rest runs
// on pairs of fp32 values (the paired add, mul and fma).
#include "common.cuh"
#include "launch.h"

namespace ret {
namespace {

constexpr int kThreadsB = 128;  // blocks of four warps, five per SM
constexpr int kPerLane = kMaxDv / 128;  // 4-vectors per lane

__device__ __forceinline__ void store4(float *p, const float *x) {
    *reinterpret_cast<float4 *>(p) = make_float4(x[0], x[1], x[2], x[3]);
}
__device__ __forceinline__ void store4(__nv_bfloat16 *p, const float *x) {
    __nv_bfloat162 a = __floats2bfloat162_rn(x[0], x[1]);
    __nv_bfloat162 b = __floats2bfloat162_rn(x[2], x[3]);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t *>(&a);
    u.y = *reinterpret_cast<uint32_t *>(&b);
    *reinterpret_cast<uint2 *>(p) = u;
}

// Two fp32 values in one 64-bit register pair (lo, hi), for the paired
// fp32 instructions (add, mul, fma on .f32x2).
__device__ __forceinline__ uint64_t p2(float lo, float hi) {
    uint64_t d;
    asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(lo), "f"(hi));
    return d;
}
__device__ __forceinline__ float p2_lo(uint64_t a) { return __uint_as_float(static_cast<uint32_t>(a)); }
__device__ __forceinline__ float p2_hi(uint64_t a) { return __uint_as_float(static_cast<uint32_t>(a >> 32)); }
__device__ __forceinline__ uint64_t p2_add(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t p2_mul(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t p2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

// Four consecutive elements as loaded (16 bytes of fp32 or 8 of bf16), so
// that a row's three inputs can all be in flight before any arithmetic.
template <typename T> struct Raw4;
template <> struct Raw4<float> {
    float4 v;
    // elements (2k, 2k+1) as a pair
    __device__ __forceinline__ uint64_t pair(int k) const { return k ? p2(v.z, v.w) : p2(v.x, v.y); }
    __device__ __forceinline__ void load(const float *p) { v = *reinterpret_cast<const float4 *>(p); }
    __device__ __forceinline__ void get(float *x) const { x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w; }
};
template <> struct Raw4<__nv_bfloat16> {
    uint2 v;
    __device__ __forceinline__ void load(const __nv_bfloat16 *p) { v = *reinterpret_cast<const uint2 *>(p); }
    // elements (2k, 2k+1) as a pair: a bf16 is the high half of its fp32
    __device__ __forceinline__ uint64_t pair(int k) const {
        const uint32_t u = k ? v.y : v.x;
        return p2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
    }
    __device__ __forceinline__ void get(float *x) const {
        float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&v.x));
        float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&v.y));
        x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
    }
};

// Offsets of row r = (b, t, h): into O / dO, and into G / dY / dG.
__device__ __forceinline__ void row_offsets(long long r, int L, int H, int dv, size_t &orow,
                                            size_t &gy) {
    const int h = (int)(r % H);
    const long long bt = r / H;
    const int t = (int)(bt % L);
    const long long b = bt / L;
    orow = (((size_t)b * H + h) * L + t) * dv;
    gy = (size_t)bt * H * dv + (size_t)h * dv;
}

template <typename TO_, typename TG>
__device__ __forceinline__ void load_row(const TO_ *O, const TG *G, const TG *dY, size_t orow,
                                         size_t gy, int dv, int lane, Raw4<TO_> *ro,
                                         Raw4<TG> *rg, Raw4<TG> *rdy) {
#pragma unroll
    for (int it = 0; it < kPerLane; ++it) {
        int e = 128 * it + 4 * lane;
        if (e < dv) {
            ro[it].load(O + orow + e);
            rg[it].load(G + gy + e);
            rdy[it].load(dY + gy + e);
        }
    }
}

// The row statistics shared by both directions: mean and variance of the
// row's O (held as loaded) from one pass of sums shifted by the row's first
// value, so that a large mean does not cancel the variance.  Returns the
// pairs (shift'), rs and nb with n = (o + shift') rs + nb the normalised
// row.
template <typename TO_>
__device__ __forceinline__ void row_stats(const Raw4<TO_> *ro, int dv, int lane, float eps,
                                          uint64_t &nshift2, uint64_t &rs2, uint64_t &nb2) {
    float x0[4];
    ro[0].get(x0);
    const float shift = __shfl_sync(0xffffffffu, x0[0], 0);
    nshift2 = p2(-shift, -shift);
    uint64_t s1 = 0, s2 = 0;  // (+0, +0) pairs
#pragma unroll
    for (int it = 0; it < kPerLane; ++it) {
        int e = 128 * it + 4 * lane;
        if (e < dv) {
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const uint64_t c = p2_add(ro[it].pair(k), nshift2);
                s1 = p2_add(s1, c);
                s2 = p2_fma(c, c, s2);
            }
        }
    }
    float t1 = p2_lo(s1) + p2_hi(s1), t2 = p2_lo(s2) + p2_hi(s2);
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) {
        t1 += __shfl_xor_sync(0xffffffffu, t1, m);
        t2 += __shfl_xor_sync(0xffffffffu, t2, m);
    }
    const float m1 = t1 / (float)dv;
    const float rs = rsqrtf(fmaxf(t2 / (float)dv - m1 * m1, 0.f) + eps);
    rs2 = p2(rs, rs);
    nb2 = p2(-m1 * rs, -m1 * rs);
}

// sigmoid of both values of a pair, by the fast exponential and reciprocal
// (a few units in the last place; it saturates to 0 or 1)
__device__ __forceinline__ uint64_t sigmoid2(uint64_t g) {
    return p2(__fdividef(1.0f, 1.0f + __expf(-p2_lo(g))), __fdividef(1.0f, 1.0f + __expf(-p2_hi(g))));
}

template <typename TO_, typename TG, typename TY>
__global__ void __launch_bounds__(kThreadsB, 5)
gate_norm_kernel(int B, int L, int H, int dv, const TO_ *O, const TG *G,
                 float eps, TY *Y) {
    const int lane = threadIdx.x & 31;
    const long long rows = (long long)B * L * H;
    const long long warps = (long long)gridDim.x * (kThreadsB / 32);
    for (long long r = (long long)blockIdx.x * (kThreadsB / 32) + threadIdx.x / 32; r < rows; r += warps) {
        size_t orow, gy;
        row_offsets(r, L, H, dv, orow, gy);
        // the row's O and G are requested together; O stays as loaded
        Raw4<TO_> ro[kPerLane];
        Raw4<TG> rg[kPerLane];
#pragma unroll
        for (int it = 0; it < kPerLane; ++it) {
            int e = 128 * it + 4 * lane;
            if (e < dv) {
                ro[it].load(O + orow + e);
                rg[it].load(G + gy + e);
            }
        }
        uint64_t nshift2, rs2, nb2;
        row_stats(ro, dv, lane, eps, nshift2, rs2, nb2);
#pragma unroll
        for (int it = 0; it < kPerLane; ++it) {
            int e = 128 * it + 4 * lane;
            if (e < dv) {
                float y[4];
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const uint64_t g = rg[it].pair(k);
                    const uint64_t n = p2_fma(p2_add(ro[it].pair(k), nshift2), rs2, nb2);
                    const uint64_t v = p2_mul(p2_mul(g, sigmoid2(g)), n);
                    y[2 * k] = p2_lo(v);
                    y[2 * k + 1] = p2_hi(v);
                }
                store4(Y + gy + e, y);
            }
        }
    }
}

template <typename TO_, typename TG, typename TY>
cudaError_t launch_t(int B, int L, int H, int dv, const void *O, const void *G,
                     float eps, void *Y, cudaStream_t st) {
    long long rows = (long long)B * L * H;
    long long blocks = (rows + (kThreadsB / 32) - 1) / (kThreadsB / 32);
    if (blocks > 148LL * 128) blocks = 148LL * 128;
    gate_norm_kernel<TO_, TG, TY><<<(unsigned)blocks, kThreadsB, 0, st>>>(
        B, L, H, dv, (const TO_ *)O, (const TG *)G, eps, (TY *)Y);
    cudaError_t err = cudaGetLastError();
    if (err == cudaSuccess) note_launches(1);
    return err;
}

template <typename TO_, typename TG>
cudaError_t launch_y(bool y_bf16, int B, int L, int H, int dv, const void *O,
                     const void *G, float eps, void *Y, cudaStream_t st) {
    return y_bf16 ? launch_t<TO_, TG, __nv_bfloat16>(B, L, H, dv, O, G, eps, Y, st)
                  : launch_t<TO_, TG, float>(B, L, H, dv, O, G, eps, Y, st);
}

template <typename TO_>
cudaError_t launch_g(bool g_bf16, bool y_bf16, int B, int L, int H, int dv,
                     const void *O, const void *G, float eps, void *Y, cudaStream_t st) {
    return g_bf16 ? launch_y<TO_, __nv_bfloat16>(y_bf16, B, L, H, dv, O, G, eps, Y, st)
                  : launch_y<TO_, float>(y_bf16, B, L, H, dv, O, G, eps, Y, st);
}

template <typename TO_, typename TG>
__global__ void __launch_bounds__(kThreadsB, 5)
gate_norm_backward_kernel(int B, int L, int H, int dv, const TO_ *O, const TG *G, const TG *dY,
                          float eps, TO_ *dO, TG *dG) {
    const int lane = threadIdx.x & 31;
    const long long rows = (long long)B * L * H;
    const long long warps = (long long)gridDim.x * (kThreadsB / 32);
    for (long long r = (long long)blockIdx.x * (kThreadsB / 32) + threadIdx.x / 32; r < rows; r += warps) {
        size_t orow, gy;
        row_offsets(r, L, H, dv, orow, gy);
        // the row's O, G and dY are requested together, before the
        // reductions that only O feeds
        Raw4<TO_> ro[kPerLane];
        Raw4<TG> rg[kPerLane], rdy[kPerLane];
        load_row(O, G, dY, orow, gy, dv, lane, ro, rg, rdy);
        // O stays as loaded and is converted again where it is used, which
        // is cheaper than holding the row in fp32 registers
        uint64_t nshift2, rs2, nb2;
        row_stats(ro, dv, lane, eps, nshift2, rs2, nb2);
        const float rs = p2_lo(rs2);
        const uint64_t one2 = p2(1.f, 1.f), mone2 = p2(-1.f, -1.f);
        // dn = dY swish(G) kept; dG written here
        uint64_t dn[kPerLane][2];
        uint64_t a_dn = 0, a_dnn = 0;
#pragma unroll
        for (int it = 0; it < kPerLane; ++it) {
            int e = 128 * it + 4 * lane;
            if (e < dv) {
                float dg[4];
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const uint64_t g = rg[it].pair(k), dy = rdy[it].pair(k);
                    const uint64_t sig = sigmoid2(g);
                    const uint64_t n = p2_fma(p2_add(ro[it].pair(k), nshift2), rs2, nb2);
                    dn[it][k] = p2_mul(dy, p2_mul(g, sig));
                    // swish'(g) = sig (1 + g (1 - sig))
                    const uint64_t ds = p2_mul(sig, p2_fma(g, p2_fma(sig, mone2, one2), one2));
                    const uint64_t d = p2_mul(p2_mul(dy, n), ds);
                    dg[2 * k] = p2_lo(d);
                    dg[2 * k + 1] = p2_hi(d);
                    a_dn = p2_add(a_dn, dn[it][k]);
                    a_dnn = p2_fma(dn[it][k], n, a_dnn);
                }
                store4(dG + gy + e, dg);
            }
        }
        float s_dn = p2_lo(a_dn) + p2_hi(a_dn), s_dnn = p2_lo(a_dnn) + p2_hi(a_dnn);
#pragma unroll
        for (int m = 16; m > 0; m >>= 1) {
            s_dn += __shfl_xor_sync(0xffffffffu, s_dn, m);
            s_dnn += __shfl_xor_sync(0xffffffffu, s_dnn, m);
        }
        // dO = rs (dn - mean(dn) - n mean(dn n)) = rs dn + (C n + Bc)
        const float m_dn = s_dn / (float)dv, m_dnn = s_dnn / (float)dv;
        const uint64_t C2 = p2(-rs * m_dnn, -rs * m_dnn), B2 = p2(-rs * m_dn, -rs * m_dn);
#pragma unroll
        for (int it = 0; it < kPerLane; ++it) {
            int e = 128 * it + 4 * lane;
            if (e < dv) {
                float d[4];
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const uint64_t n = p2_fma(p2_add(ro[it].pair(k), nshift2), rs2, nb2);
                    const uint64_t r = p2_fma(dn[it][k], rs2, p2_fma(n, C2, B2));
                    d[2 * k] = p2_lo(r);
                    d[2 * k + 1] = p2_hi(r);
                }
                store4(dO + orow + e, d);
            }
        }
    }
}

template <typename TO_, typename TG>
cudaError_t launch_backward_t(int B, int L, int H, int dv, const void *O, const void *G,
                              const void *dY, float eps, void *dO, void *dG, cudaStream_t st) {
    long long rows = (long long)B * L * H;
    long long blocks = (rows + (kThreadsB / 32) - 1) / (kThreadsB / 32);
    if (blocks > 148LL * 128) blocks = 148LL * 128;
    gate_norm_backward_kernel<TO_, TG><<<(unsigned)blocks, kThreadsB, 0, st>>>(
        B, L, H, dv, (const TO_ *)O, (const TG *)G, (const TG *)dY, eps, (TO_ *)dO, (TG *)dG);
    cudaError_t err = cudaGetLastError();
    if (err == cudaSuccess) note_launches(1);
    return err;
}

}  // namespace

cudaError_t launch_gate_norm_backward(int B, int L, int H, int dv, bool o_bf16, const void *O,
                                      bool g_bf16, const void *G, const void *dY, float eps,
                                      void *dO, void *dG, cudaStream_t st) {
    if ((long long)B * L * H == 0) return cudaSuccess;
    if (o_bf16)
        return g_bf16 ? launch_backward_t<__nv_bfloat16, __nv_bfloat16>(B, L, H, dv, O, G, dY, eps, dO, dG, st)
                      : launch_backward_t<__nv_bfloat16, float>(B, L, H, dv, O, G, dY, eps, dO, dG, st);
    return g_bf16 ? launch_backward_t<float, __nv_bfloat16>(B, L, H, dv, O, G, dY, eps, dO, dG, st)
                  : launch_backward_t<float, float>(B, L, H, dv, O, G, dY, eps, dO, dG, st);
}

cudaError_t launch_gate_norm(int B, int L, int H, int dv, bool o_bf16,
                             const void *O, bool g_bf16, const void *G,
                             float eps, bool y_bf16, void *Y, cudaStream_t st) {
    if ((long long)B * L * H == 0) return cudaSuccess;
    return o_bf16 ? launch_g<__nv_bfloat16>(g_bf16, y_bf16, B, L, H, dv, O, G, eps, Y, st)
                  : launch_g<float>(g_bf16, y_bf16, B, L, H, dv, O, G, eps, Y, st);
}

}  // namespace ret
