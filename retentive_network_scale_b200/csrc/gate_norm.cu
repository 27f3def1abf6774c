// gate_norm.cu -- Y = swish(G) (.) GroupNorm_h(O), one group per head taken
// per token over its d_v channels ("Retentive Network" paper summary,
// section 2.2, the MSR equation; population variance, no affine terms).
//
// Bound by HBM (read O and G, write Y).  One warp per (b, t, h) row: each
// lane holds up to 16 of the row's d_v <= 512 values in registers (4-wide
// vector loads), so the mean and the centred variance are two register
// passes and warp reductions with no second read of memory.
#include "common.cuh"
#include "launch.h"

namespace ret {
namespace {

constexpr int kThreads = 256;
constexpr int kPerLane = kMaxDv / 128;  // 4-vectors per lane

__device__ __forceinline__ void load4(const float *p, float *x) {
    float4 v = *reinterpret_cast<const float4 *>(p);
    x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
}
__device__ __forceinline__ void load4(const __nv_bfloat16 *p, float *x) {
    uint2 u = *reinterpret_cast<const uint2 *>(p);
    float2 a = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&u.x));
    float2 b = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&u.y));
    x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
}
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

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) v += __shfl_xor_sync(0xffffffffu, v, m);
    return v;
}

template <typename TO_, typename TG, typename TY>
__global__ void __launch_bounds__(kThreads)
gate_norm_kernel(int B, int L, int H, int dv, const TO_ *O, const TG *G,
                 float eps, TY *Y) {
    const int lane = threadIdx.x & 31;
    const long long rows = (long long)B * L * H;
    const long long warps = (long long)gridDim.x * (kThreads / 32);
    for (long long r = (long long)blockIdx.x * (kThreads / 32) + threadIdx.x / 32; r < rows; r += warps) {
        const int h = (int)(r % H);
        const long long bt = r / H;
        const int t = (int)(bt % L);
        const long long b = bt / L;
        const TO_ *o = O + (((size_t)b * H + h) * L + t) * dv;
        const size_t gy = (size_t)bt * H * dv + (size_t)h * dv;

        float x[kPerLane][4];
        float sum = 0.f;
#pragma unroll
        for (int it = 0; it < kPerLane; ++it) {
            int e = 128 * it + 4 * lane;
            if (e < dv) {
                load4(o + e, x[it]);
                sum += (x[it][0] + x[it][1]) + (x[it][2] + x[it][3]);
            }
        }
        const float mu = warp_sum(sum) / (float)dv;
        float sq = 0.f;
#pragma unroll
        for (int it = 0; it < kPerLane; ++it) {
            int e = 128 * it + 4 * lane;
            if (e < dv) {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    x[it][q] -= mu;
                    sq = fmaf(x[it][q], x[it][q], sq);
                }
            }
        }
        const float inv = rsqrtf(warp_sum(sq) / (float)dv + eps);
#pragma unroll
        for (int it = 0; it < kPerLane; ++it) {
            int e = 128 * it + 4 * lane;
            if (e < dv) {
                float g[4], y[4];
                load4(G + gy + e, g);
#pragma unroll
                for (int q = 0; q < 4; ++q) y[q] = g[q] / (1.0f + expf(-g[q])) * (x[it][q] * inv);
                store4(Y + gy + e, y);
            }
        }
    }
}

template <typename TO_, typename TG, typename TY>
cudaError_t launch_t(int B, int L, int H, int dv, const void *O, const void *G,
                     float eps, void *Y, cudaStream_t st) {
    long long rows = (long long)B * L * H;
    long long blocks = (rows + (kThreads / 32) - 1) / (kThreads / 32);
    if (blocks > 148LL * 64) blocks = 148LL * 64;
    gate_norm_kernel<TO_, TG, TY><<<(unsigned)blocks, kThreads, 0, st>>>(
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

}  // namespace

cudaError_t launch_gate_norm(int B, int L, int H, int dv, bool o_bf16,
                             const void *O, bool g_bf16, const void *G,
                             float eps, bool y_bf16, void *Y, cudaStream_t st) {
    if ((long long)B * L * H == 0) return cudaSuccess;
    return o_bf16 ? launch_g<__nv_bfloat16>(g_bf16, y_bf16, B, L, H, dv, O, G, eps, Y, st)
                  : launch_g<float>(g_bf16, y_bf16, B, L, H, dv, O, G, eps, Y, st);
}

}  // namespace ret
