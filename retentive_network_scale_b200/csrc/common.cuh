// common.cuh -- parameters and device helpers shared by the retention kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "retention.h"

namespace ret {

constexpr int kMaxDk = 256;
constexpr int kMaxDv = 512;

// Everything a kernel needs about the problem, passed by value.  Decays are
// given as log2(gamma_h) so that gamma^n = exp2(n log2 gamma) for any n
// without repeated multiplication; gamma = 0 is log2 = -inf and is handled
// where n = 0 (gamma^0 = 1).
struct Params {
    int B, H, L, dk, dv;
    int rotate;
    long long pos_offset;
    float log2g[RET_MAX_HEADS];
    double theta[kMaxDk / 2];  // theta_j = base^(-2j/dk), fp64 from the host
    // Rows of head h sit at positions pos_offset + (h mod seg_heads) * seg_len
    // + t: a sequence read as seg_heads segments of seg_len rows, each segment
    // a head of its own ([B][H][L][d] is [B][H*S][L/S][d]).  1 and 0 for
    // plain heads; only the streaming pass reads them.
    int seg_heads;
    long long seg_len;
    // Anti-causal retention, o_t = sum over m >= t of gamma^{m-t} (q^_t . k^_m)
    // v_m (the time-reversed products of the backward pass): the streaming
    // pass weights key row j of a block by gamma^j and the tensor-core chunk
    // loop walks the blocks from last to first with the mirrored mask.  0
    // for the forward forms; no other kernel reads it.
    int reverse;
};

// ------------------------------------------------------------------ dtypes
__device__ __forceinline__ float ld(const float *p, size_t i) { return p[i]; }
__device__ __forceinline__ float ld(const __nv_bfloat16 *p, size_t i) {
    return __bfloat162float(p[i]);
}
__device__ __forceinline__ void st(float *p, size_t i, float v) { p[i] = v; }
__device__ __forceinline__ void st(__nv_bfloat16 *p, size_t i, float v) {
    p[i] = __float2bfloat16_rn(v);
}

// gamma^n for an integer n >= 0 (exactly 1 for n = 0, also when gamma = 0).
__device__ __forceinline__ float decay_pow(float log2g, int n) {
    return n == 0 ? 1.0f : exp2f((float)n * log2g);
}

// theta_0 .. theta_{n-1} into shared memory, by all threads of the block
// (the caller synchronises).  Kernel parameters are read through the
// constant cache, which serves one address per request: a per-thread index
// into Params::theta would be serialised across the warp, a shared-memory
// table is not.
__device__ __forceinline__ void stage_theta(const Params &p, double *s_theta, int n) {
    for (int i = threadIdx.x; i < n; i += blockDim.x) s_theta[i] = p.theta[i];
}

// cos and sin of pos * theta.  The product and its reduction to
// [-pi, pi] are done in fp64 so that positions of 10^5 and more keep full
// fp32 accuracy; the reduced angle then goes to sincosf.
__device__ __forceinline__ void rot_cs(long long pos, double theta, float *c,
                                       float *s) {
    const double two_pi = 6.283185307179586476925286766559;
    double a = (double)pos * theta;
    a -= two_pi * rint(a / two_pi);
    sincosf((float)a, s, c);
}

// cos and sin of pos * theta: the product and its reduction to [-pi, pi]
// in fp64, then the fast single-precision sine/cosine (absolute error near
// 2^-21 on that range).
__device__ __forceinline__ void rot_cs_fast(long long pos, double theta, float *c, float *s) {
    const double a = (double)pos * theta;
    const double k = rint(a * 0.15915494309189533577);
    __sincosf((float)fma(-k, 6.283185307179586477, a), s, c);
}

// xPos turn of one pair (x0, x1) by angle with cos c, sin s:
// (x0 + i x1) e^{i a} = (x0 c - x1 s) + i (x0 s + x1 c).
__device__ __forceinline__ void rot_pair(float &x0, float &x1, float c, float s) {
    float r0 = x0 * c - x1 * s;
    float r1 = x0 * s + x1 * c;
    x0 = r0;
    x1 = r1;
}

}  // namespace ret
