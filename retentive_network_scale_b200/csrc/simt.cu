// simt.cu -- CUDA-core (FFMA, fp32 accumulate) kernels for the parallel and
// chunkwise retention forms.  They serve fp32 inputs, where tensor cores
// would round operands (TF32), and any shape the tensor-core kernel does not
// take.  Tiles of 32 rows/keys in shared memory; correctness over speed.
#include "common.cuh"
#include "launch.h"

namespace ret {
namespace {

constexpr int kThreads = 256;
constexpr int kTile = 32;      // rows per query tile, keys per key tile
constexpr int kParBV = 64;     // value columns per CTA, parallel kernel
constexpr int kChkBV = 32;     // value columns per CTA, chunkwise kernel

// Rows [r0, r0+kTile) of a [L][dk] slice into smem as fp32 (stride dk+1),
// turned by the xPos factor at absolute positions pos_offset + r.  Rows at
// or beyond `rend` are zero.
template <typename T>
__device__ void load_rot_rows(float *dst, const T *src, int r0, int rend,
                              const Params &p) {
    const int stride = p.dk + 1;
    if (p.rotate) {
        const int half = p.dk / 2;
        for (int idx = threadIdx.x; idx < kTile * half; idx += blockDim.x) {
            int r = idx / half, j = idx - r * half;
            float x0 = 0.f, x1 = 0.f;
            if (r0 + r < rend) {
                size_t base = (size_t)(r0 + r) * p.dk + 2 * j;
                x0 = ld(src, base);
                x1 = ld(src, base + 1);
                float c, s;
                rot_cs(p.pos_offset + r0 + r, p.theta[j], &c, &s);
                rot_pair(x0, x1, c, s);
            }
            dst[r * stride + 2 * j] = x0;
            dst[r * stride + 2 * j + 1] = x1;
        }
    } else {
        for (int idx = threadIdx.x; idx < kTile * p.dk; idx += blockDim.x) {
            int r = idx / p.dk, d = idx - r * p.dk;
            dst[r * stride + d] = (r0 + r < rend) ? ld(src, (size_t)(r0 + r) * p.dk + d) : 0.f;
        }
    }
}

// Rows [r0, r0+kTile), columns [c0, c0+bv) of a [L][dv] slice (stride bv+1).
template <typename T>
__device__ void load_v_rows(float *dst, const T *src, int r0, int rend, int c0,
                            int bv, int dv) {
    for (int idx = threadIdx.x; idx < kTile * bv; idx += blockDim.x) {
        int r = idx / bv, c = idx - r * bv;
        dst[r * (bv + 1) + c] = (r0 + r < rend && c0 + c < dv)
                                    ? ld(src, (size_t)(r0 + r) * dv + c0 + c)
                                    : 0.f;
    }
}

// ---------------------------------------------------------------- parallel
// O = (Q^ K^^T (.) D) V for one (b,h), a 32-row query tile and a 64-column
// slice of V.  grid = (ceil(L/32), B*H, ceil(dv/64)).
template <typename TI, typename TO>
__global__ void __launch_bounds__(kThreads)
parallel_simt_kernel(Params p, const TI *Q, const TI *K, const TI *V, TO *O) {
    extern __shared__ float smem[];
    const int ldk = p.dk + 1;
    float *Qs = smem;
    float *Ks = Qs + kTile * ldk;
    float *Vs = Ks + kTile * ldk;
    float *Ps = Vs + kTile * (kParBV + 1);

    const int bh = blockIdx.y, h = bh % p.H;
    const int q0 = blockIdx.x * kTile, c0 = blockIdx.z * kParBV;
    const size_t qk_off = (size_t)bh * p.L * p.dk, v_off = (size_t)bh * p.L * p.dv;
    const float lg = p.log2g[h];
    const int row = threadIdx.x / 8, sub = threadIdx.x % 8;

    load_rot_rows(Qs, Q + qk_off, q0, p.L, p);
    float acc[kParBV / 8];
#pragma unroll
    for (int u = 0; u < kParBV / 8; ++u) acc[u] = 0.f;

    for (int k0 = 0; k0 <= q0; k0 += kTile) {
        __syncthreads();
        load_rot_rows(Ks, K + qk_off, k0, p.L, p);
        load_v_rows(Vs, V + v_off, k0, p.L, c0, kParBV, p.dv);
        __syncthreads();
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            int key = sub + 8 * u;
            float s = 0.f;
            for (int d = 0; d < p.dk; ++d) s += Qs[row * ldk + d] * Ks[key * ldk + d];
            int n = q0 + row, m = k0 + key;
            Ps[row * (kTile + 1) + key] = (m <= n) ? s * decay_pow(lg, n - m) : 0.f;
        }
        __syncthreads();
        for (int key = 0; key < kTile; ++key) {
            float w = Ps[row * (kTile + 1) + key];
#pragma unroll
            for (int u = 0; u < kParBV / 8; ++u) acc[u] += w * Vs[key * (kParBV + 1) + sub + 8 * u];
        }
    }
    if (q0 + row < p.L) {
#pragma unroll
        for (int u = 0; u < kParBV / 8; ++u) {
            int c = c0 + sub + 8 * u;
            if (c < p.dv) st(O, v_off + (size_t)(q0 + row) * p.dv + c, acc[u]);
        }
    }
}

// --------------------------------------------------------------- chunkwise
// One CTA per (b,h) and 32-column slice of V; chunks in order, the state
// slice R [dk][32] in shared memory.  For each chunk of n rows: every row
// tile gets gamma^{j+1} q^ R plus its causal in-chunk part, then
// R <- gamma^n R + sum_j' gamma^{n-1-j'} k^_j'^T v_j'.
// grid = (B*H, ceil(dv/32)).
template <typename TI, typename TO>
__global__ void __launch_bounds__(kThreads)
chunkwise_simt_kernel(Params p, int chunk, const TI *Q, const TI *K, const TI *V,
                      const float *state_in, float *state_out, TO *O) {
    extern __shared__ float smem[];
    const int ldk = p.dk + 1, ldv = kChkBV + 1;
    float *Qs = smem;
    float *Ks = Qs + kTile * ldk;
    float *Vs = Ks + kTile * ldk;
    float *Ps = Vs + kTile * ldv;
    float *Rs = Ps + kTile * (kTile + 1);  // [dk][kChkBV]

    const int bh = blockIdx.x, h = bh % p.H, c0 = blockIdx.y * kChkBV;
    const size_t qk_off = (size_t)bh * p.L * p.dk, v_off = (size_t)bh * p.L * p.dv;
    const size_t s_off = (size_t)bh * p.dk * p.dv;
    const float lg = p.log2g[h];
    const int row = threadIdx.x / 8, sub = threadIdx.x % 8;

    for (int idx = threadIdx.x; idx < p.dk * kChkBV; idx += blockDim.x) {
        int d = idx / kChkBV, c = idx - d * kChkBV;
        Rs[idx] = (state_in && c0 + c < p.dv) ? state_in[s_off + (size_t)d * p.dv + c0 + c] : 0.f;
    }

    for (int cs = 0; cs < p.L; cs += chunk) {
        const int n = min(chunk, p.L - cs), ce = cs + n;
        for (int r0 = cs; r0 < ce; r0 += kTile) {
            __syncthreads();
            load_rot_rows(Qs, Q + qk_off, r0, ce, p);
            __syncthreads();
            // carried state: gamma^{j+1} q^_j R
            float acc[kChkBV / 8];
            const int j = r0 + row - cs;
            const float xi = decay_pow(lg, j + 1);
#pragma unroll
            for (int u = 0; u < kChkBV / 8; ++u) {
                float s = 0.f;
                for (int d = 0; d < p.dk; ++d) s += Qs[row * ldk + d] * Rs[d * kChkBV + sub + 8 * u];
                acc[u] = xi * s;
            }
            // inside the chunk: causal, decayed by gamma^{j-j'}
            for (int k0 = cs; k0 <= r0; k0 += kTile) {
                __syncthreads();
                load_rot_rows(Ks, K + qk_off, k0, ce, p);
                load_v_rows(Vs, V + v_off, k0, ce, c0, kChkBV, p.dv);
                __syncthreads();
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    int key = sub + 8 * u;
                    float s = 0.f;
                    for (int d = 0; d < p.dk; ++d) s += Qs[row * ldk + d] * Ks[key * ldk + d];
                    int nn = r0 + row, m = k0 + key;
                    Ps[row * (kTile + 1) + key] = (m <= nn && m < ce) ? s * decay_pow(lg, nn - m) : 0.f;
                }
                __syncthreads();
                for (int key = 0; key < kTile; ++key) {
                    float w = Ps[row * (kTile + 1) + key];
#pragma unroll
                    for (int u = 0; u < kChkBV / 8; ++u) acc[u] += w * Vs[key * ldv + sub + 8 * u];
                }
            }
            if (O && r0 + row < ce) {
#pragma unroll
                for (int u = 0; u < kChkBV / 8; ++u) {
                    int c = c0 + sub + 8 * u;
                    if (c < p.dv) st(O, v_off + (size_t)(r0 + row) * p.dv + c, acc[u]);
                }
            }
        }
        // state update; each thread owns the entries (d, c) with
        // c = tid % 32 and d = tid / 32 + 8 t.
        __syncthreads();
        const float gn = decay_pow(lg, n);
        const int c = threadIdx.x % kChkBV;
        for (int d = threadIdx.x / kChkBV; d < p.dk; d += kThreads / kChkBV) Rs[d * kChkBV + c] *= gn;
        for (int k0 = cs; k0 < ce; k0 += kTile) {
            __syncthreads();
            load_rot_rows(Ks, K + qk_off, k0, ce, p);
            load_v_rows(Vs, V + v_off, k0, ce, c0, kChkBV, p.dv);
            __syncthreads();
            for (int d = threadIdx.x / kChkBV; d < p.dk; d += kThreads / kChkBV) {
                float s = Rs[d * kChkBV + c];
                for (int key = 0; key < kTile && k0 + key < ce; ++key)
                    s += decay_pow(lg, ce - 1 - (k0 + key)) * Ks[key * ldk + d] * Vs[key * ldv + c];
                Rs[d * kChkBV + c] = s;
            }
        }
    }
    __syncthreads();
    if (state_out) {
        for (int idx = threadIdx.x; idx < p.dk * kChkBV; idx += blockDim.x) {
            int d = idx / kChkBV, c = idx - d * kChkBV;
            if (c0 + c < p.dv) state_out[s_off + (size_t)d * p.dv + c0 + c] = Rs[idx];
        }
    }
}

template <typename TI, typename TO>
cudaError_t launch_parallel_t(const Params &p, const void *Q, const void *K,
                              const void *V, void *O, cudaStream_t st) {
    size_t smem = sizeof(float) * (2 * kTile * (p.dk + 1) + kTile * (kParBV + 1) +
                                   kTile * (kTile + 1));
    auto kern = parallel_simt_kernel<TI, TO>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((p.L + kTile - 1) / kTile, p.B * p.H, (p.dv + kParBV - 1) / kParBV);
    kern<<<grid, kThreads, smem, st>>>(p, (const TI *)Q, (const TI *)K, (const TI *)V, (TO *)O);
    cudaError_t err = cudaGetLastError();
    if (err == cudaSuccess) note_launches(1);
    return err;
}

template <typename TI, typename TO>
cudaError_t launch_chunkwise_t(const Params &p, int chunk, const void *Q, const void *K,
                               const void *V, const float *s_in, float *s_out,
                               void *O, cudaStream_t st) {
    size_t smem = sizeof(float) * (2 * kTile * (p.dk + 1) + kTile * (kChkBV + 1) +
                                   kTile * (kTile + 1) + p.dk * kChkBV);
    auto kern = chunkwise_simt_kernel<TI, TO>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(p.B * p.H, (p.dv + kChkBV - 1) / kChkBV);
    kern<<<grid, kThreads, smem, st>>>(p, chunk, (const TI *)Q, (const TI *)K, (const TI *)V,
                                       s_in, s_out, (TO *)O);
    cudaError_t err = cudaGetLastError();
    if (err == cudaSuccess) note_launches(1);
    return err;
}

}  // namespace

cudaError_t launch_parallel_simt(const Params &p, bool in_bf16, bool out_bf16,
                                 const void *Q, const void *K, const void *V,
                                 void *O, cudaStream_t st) {
    if (in_bf16)
        return out_bf16 ? launch_parallel_t<__nv_bfloat16, __nv_bfloat16>(p, Q, K, V, O, st)
                        : launch_parallel_t<__nv_bfloat16, float>(p, Q, K, V, O, st);
    return out_bf16 ? launch_parallel_t<float, __nv_bfloat16>(p, Q, K, V, O, st)
                    : launch_parallel_t<float, float>(p, Q, K, V, O, st);
}

cudaError_t launch_chunkwise_simt(const Params &p, int chunk, bool in_bf16, bool out_bf16,
                                  const void *Q, const void *K, const void *V,
                                  const float *s_in, float *s_out, void *O,
                                  cudaStream_t st) {
    if (in_bf16)
        return out_bf16
                   ? launch_chunkwise_t<__nv_bfloat16, __nv_bfloat16>(p, chunk, Q, K, V, s_in, s_out, O, st)
                   : launch_chunkwise_t<__nv_bfloat16, float>(p, chunk, Q, K, V, s_in, s_out, O, st);
    return out_bf16 ? launch_chunkwise_t<float, __nv_bfloat16>(p, chunk, Q, K, V, s_in, s_out, O, st)
                    : launch_chunkwise_t<float, float>(p, chunk, Q, K, V, s_in, s_out, O, st);
}

}  // namespace ret
