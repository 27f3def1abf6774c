// decode.cu -- one recurrent retention step over the fp32 state:
//   S <- gamma S + k^^T v   (in place),   o = q^ S   (update, then read).
// "Retentive Network" paper summary, section 2.1, recurrent form (2).
//
// Bound by HBM: each step reads and writes the whole d_k x d_v fp32 state
// once (8 d_k d_v bytes per head) and does 4 flops per element.  One CTA
// owns COLS contiguous columns of one (b,h) state, all d_k rows: threads
// move 16-byte float4 pieces, TPR = COLS/4 threads cover a row segment, so a
// warp touches 32/TPR rows with fully used 128-byte lines.  Each thread keeps
// eight rows of loads in flight.  The column sums of q^ S are reduced
// through shared memory.  State traffic uses streaming (evict-first) hints:
// the state is larger than L2 and is not read again within the step.
#include "common.cuh"
#include "launch.h"
#include "tc_util.cuh"

namespace ret {
namespace {

constexpr int kThreads = 256;
constexpr int kRowsInFlight = 8;

__device__ __forceinline__ float4 load4(const float *p) { return *reinterpret_cast<const float4 *>(p); }
__device__ __forceinline__ float4 load4(const __nv_bfloat16 *p) {
    uint2 u = *reinterpret_cast<const uint2 *>(p);
    __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162 *>(&u.x);
    __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162 *>(&u.y);
    float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
    return make_float4(fa.x, fa.y, fb.x, fb.y);
}

template <typename TI, typename TO, int COLS>
__global__ void __launch_bounds__(kThreads)
recurrent_step_kernel(Params p, int ncol_tiles, const TI *q, const TI *k,
                      const TI *v, float *state, TO *o) {
    constexpr int TPR = COLS / 4;
    constexpr int RG = kThreads / TPR;
    __shared__ float qs[kMaxDk], ks[kMaxDk];
    __shared__ float red[kThreads * 4];

    const int bh = blockIdx.x / ncol_tiles, ct = blockIdx.x - bh * ncol_tiles;
    const int h = bh % p.H;
    const size_t qk_off = (size_t)bh * p.dk;

    // q^, k^ for this head into shared memory
    if (p.rotate) {
        for (int j = threadIdx.x; j < p.dk / 2; j += kThreads) {
            float c, s;
            rot_cs(p.pos_offset, p.theta[j], &c, &s);
            float q0 = ld(q, qk_off + 2 * j), q1 = ld(q, qk_off + 2 * j + 1);
            float k0 = ld(k, qk_off + 2 * j), k1 = ld(k, qk_off + 2 * j + 1);
            rot_pair(q0, q1, c, s);
            rot_pair(k0, k1, c, s);
            qs[2 * j] = q0; qs[2 * j + 1] = q1;
            ks[2 * j] = k0; ks[2 * j + 1] = k1;
        }
    } else {
        for (int i = threadIdx.x; i < p.dk; i += kThreads) {
            qs[i] = ld(q, qk_off + i);
            ks[i] = ld(k, qk_off + i);
        }
    }
    __syncthreads();

    const int tpr = threadIdx.x % TPR, rg = threadIdx.x / TPR;
    const int c = ct * COLS + 4 * tpr;
    const float4 vv = load4(v + (size_t)bh * p.dv + c);
    const float g = exp2f(p.log2g[h]);  // gamma (0 when log2 gamma = -inf)
    float *S = state + (size_t)bh * p.dk * p.dv + c;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);

    for (int i0 = rg; i0 < p.dk; i0 += RG * kRowsInFlight) {
        float4 s[kRowsInFlight];
#pragma unroll
        for (int u = 0; u < kRowsInFlight; ++u) {
            int i = i0 + u * RG;
            if (i < p.dk) s[u] = __ldcs(reinterpret_cast<const float4 *>(S + (size_t)i * p.dv));
        }
#pragma unroll
        for (int u = 0; u < kRowsInFlight; ++u) {
            int i = i0 + u * RG;
            if (i < p.dk) {
                const float ki = ks[i], qi = qs[i];
                s[u].x = fmaf(g, s[u].x, ki * vv.x);
                s[u].y = fmaf(g, s[u].y, ki * vv.y);
                s[u].z = fmaf(g, s[u].z, ki * vv.z);
                s[u].w = fmaf(g, s[u].w, ki * vv.w);
                __stcs(reinterpret_cast<float4 *>(S + (size_t)i * p.dv), s[u]);
                acc.x = fmaf(qi, s[u].x, acc.x);
                acc.y = fmaf(qi, s[u].y, acc.y);
                acc.z = fmaf(qi, s[u].z, acc.z);
                acc.w = fmaf(qi, s[u].w, acc.w);
            }
        }
    }

    // o[c'] = sum over row groups; red is [RG][COLS]
    red[rg * COLS + 4 * tpr + 0] = acc.x;
    red[rg * COLS + 4 * tpr + 1] = acc.y;
    red[rg * COLS + 4 * tpr + 2] = acc.z;
    red[rg * COLS + 4 * tpr + 3] = acc.w;
    __syncthreads();
    // level 1: thread t sums 4 row groups of column t % COLS
    constexpr int PARTS = kThreads / COLS;   // == RG / 4
    {
        const int cc = threadIdx.x % COLS, part = threadIdx.x / COLS;
        float sum = 0.f;
#pragma unroll
        for (int r = 0; r < 4; ++r) sum += red[(part * 4 + r) * COLS + cc];
        __syncthreads();
        red[part * COLS + cc] = sum;
    }
    __syncthreads();
    if (threadIdx.x < COLS) {
        float sum = 0.f;
        for (int part = 0; part < PARTS; ++part) sum += red[part * COLS + threadIdx.x];
        st(o, (size_t)bh * p.dv + ct * COLS + threadIdx.x, sum);
    }
}

// T > 1 consecutive tokens per sequence (positions pos_offset .. +T-1) in
// one pass over the state: every element runs its T updates in registers,
//   s <- gamma s + k^_t[i] v_t[c];   o_t[c] += q^_t[i] s   (t = 0 .. T-1),
// so the state is read and written once for all T tokens.  q, k, v, o are
// [B][H][T][d]; the rotated q^_t, k^_t of the head and the v_t of the CTA's
// columns sit in shared memory.  The column sums of all T tokens are reduced
// at the end: across the row groups of a warp by shuffles, then across the
// warps through shared memory in one pass.
constexpr int kMultiRowsInFlight = 4;
constexpr bool kMultiPacked = true;  // packed fp32 pairs on the rescaled path

template <typename TI, typename TO, int COLS, int TMAX, bool PACKED>
__global__ void __launch_bounds__(kThreads)
recurrent_multi_kernel(Params p, int T, int ncol_tiles, const TI *q, const TI *k, const TI *v,
                       float *state, TO *o) {
    constexpr int TPR = COLS / 4;
    constexpr int RG = kThreads / TPR;
    constexpr int kWarps = kThreads / 32;
    // q^_t and k^_t; after the state pass the same words hold the warps'
    // column sums
    __shared__ __align__(16) float qk[2 * TMAX * kMaxDk];
    __shared__ __align__(16) float vs[TMAX][COLS];
    __shared__ double s_theta[kMaxDk / 2];
    static_assert(kWarps * COLS <= 2 * kMaxDk, "column sums must fit in the q^/k^ words");
    auto qs = reinterpret_cast<float (*)[kMaxDk]>(qk);
    auto ks = reinterpret_cast<float (*)[kMaxDk]>(qk + TMAX * kMaxDk);
    auto red = reinterpret_cast<float (*)[TMAX][COLS]>(qk);

    const int bh = blockIdx.x / ncol_tiles, ct = blockIdx.x - bh * ncol_tiles;
    const int h = bh % p.H;
    const int dk = p.dk, dv = p.dv;
    // With gamma^T >= 2^-60 the T updates run on a rescaled state: with
    // s_t = gamma s_{t-1} + k_t v_t from s_{-1} = S,
    //   s_t = gamma^{t+1} a_t,  a_t = S + sum_{tau<=t} gamma^{-(tau+1)} k_tau v_tau,
    //   o_t = q_t . s_t = (gamma^{t+1} q_t) . a_t,
    // so with k~_t = gamma^{-(t+1)} k_t and q~_t = gamma^{t+1} q_t each token
    // costs a += k~ v and o += q~ a, and the state leaves as gamma^T a.  The
    // final scaling brings every term back to its own magnitude, so the
    // relative rounding is that of the direct form.  Other decays (gamma = 0
    // among them) take the direct form.
    const float lg = p.log2g[h];
    const bool scaled = (float)T * lg >= -60.f;
    auto fq = [&](int t) { return scaled ? exp2f((float)(t + 1) * lg) : 1.f; };
    auto fk = [&](int t) { return scaled ? exp2f(-(float)(t + 1) * lg) : 1.f; };

    // q^_t, k^_t (turned at position pos_offset + t) and this CTA's v_t columns
    if (p.rotate) {
        stage_theta(p, s_theta, dk / 2);
        __syncthreads();
        for (int idx = threadIdx.x; idx < T * (dk / 2); idx += kThreads) {
            const int t = idx / (dk / 2), j = idx - t * (dk / 2);
            const size_t base = ((size_t)bh * T + t) * dk;
            float c, sn;
            rot_cs_fast(p.pos_offset + t, s_theta[j], &c, &sn);
            float q0 = ld(q, base + 2 * j), q1 = ld(q, base + 2 * j + 1);
            float k0 = ld(k, base + 2 * j), k1 = ld(k, base + 2 * j + 1);
            rot_pair(q0, q1, c, sn);
            rot_pair(k0, k1, c, sn);
            const float a = fq(t), b = fk(t);
            qs[t][2 * j] = a * q0; qs[t][2 * j + 1] = a * q1;
            ks[t][2 * j] = b * k0; ks[t][2 * j + 1] = b * k1;
        }
    } else {
        for (int idx = threadIdx.x; idx < T * dk; idx += kThreads) {
            const int t = idx / dk, i = idx - t * dk;
            qs[t][i] = fq(t) * ld(q, ((size_t)bh * T + t) * dk + i);
            ks[t][i] = fk(t) * ld(k, ((size_t)bh * T + t) * dk + i);
        }
    }
    for (int idx = threadIdx.x; idx < T * COLS; idx += kThreads) {
        const int t = idx / COLS, cc = idx - t * COLS;
        vs[t][cc] = ld(v, ((size_t)bh * T + t) * dv + ct * COLS + cc);
    }
    __syncthreads();

    const int tpr = threadIdx.x % TPR, rg = threadIdx.x / TPR;
    const int c = ct * COLS + 4 * tpr;
    const float g = exp2f(lg);
    const float gT = scaled ? exp2f((float)T * lg) : 1.f;
    float *S = state + (size_t)bh * dk * dv + c;
    float4 acc[TMAX];
#pragma unroll
    for (int t = 0; t < TMAX; ++t) acc[t] = make_float4(0.f, 0.f, 0.f, 0.f);

    // packed fp32 pairs (x, y) and (z, w) of a float4
    union P4 {
        float4 f;
        uint64_t u[2];
    };
    for (int i0 = rg; i0 < dk; i0 += RG * kMultiRowsInFlight) {
        P4 s[kMultiRowsInFlight];
#pragma unroll
        for (int u = 0; u < kMultiRowsInFlight; ++u) {
            const int i = i0 + u * RG;
            if (i < dk) s[u].f = __ldcs(reinterpret_cast<const float4 *>(S + (size_t)i * dv));
        }
        if (scaled) {
#pragma unroll
            for (int t = 0; t < TMAX; ++t) {
                if (t < T) {
                    P4 vt, at;
                    vt.f = *reinterpret_cast<const float4 *>(&vs[t][4 * tpr]);
                    at.f = acc[t];
#pragma unroll
                    for (int u = 0; u < kMultiRowsInFlight; ++u) {
                        const int i = i0 + u * RG;
                        if (i < dk) {
                            const float ki = ks[t][i], qi = qs[t][i];
                            if constexpr (PACKED) {
                                const uint64_t K2 = tc::f2_make(ki, ki), Q2 = tc::f2_make(qi, qi);
                                s[u].u[0] = tc::f2_fma(K2, vt.u[0], s[u].u[0]);
                                s[u].u[1] = tc::f2_fma(K2, vt.u[1], s[u].u[1]);
                                at.u[0] = tc::f2_fma(Q2, s[u].u[0], at.u[0]);
                                at.u[1] = tc::f2_fma(Q2, s[u].u[1], at.u[1]);
                            } else {
                                s[u].f.x = fmaf(ki, vt.f.x, s[u].f.x);
                                s[u].f.y = fmaf(ki, vt.f.y, s[u].f.y);
                                s[u].f.z = fmaf(ki, vt.f.z, s[u].f.z);
                                s[u].f.w = fmaf(ki, vt.f.w, s[u].f.w);
                                at.f.x = fmaf(qi, s[u].f.x, at.f.x);
                                at.f.y = fmaf(qi, s[u].f.y, at.f.y);
                                at.f.z = fmaf(qi, s[u].f.z, at.f.z);
                                at.f.w = fmaf(qi, s[u].f.w, at.f.w);
                            }
                        }
                    }
                    acc[t] = at.f;
                }
            }
#pragma unroll
            for (int u = 0; u < kMultiRowsInFlight; ++u) {
                s[u].f.x *= gT;
                s[u].f.y *= gT;
                s[u].f.z *= gT;
                s[u].f.w *= gT;
            }
        } else {
#pragma unroll
            for (int t = 0; t < TMAX; ++t) {
                if (t < T) {
                    const float4 vt = *reinterpret_cast<const float4 *>(&vs[t][4 * tpr]);
#pragma unroll
                    for (int u = 0; u < kMultiRowsInFlight; ++u) {
                        const int i = i0 + u * RG;
                        if (i < dk) {
                            const float ki = ks[t][i], qi = qs[t][i];
                            s[u].f.x = fmaf(g, s[u].f.x, ki * vt.x);
                            s[u].f.y = fmaf(g, s[u].f.y, ki * vt.y);
                            s[u].f.z = fmaf(g, s[u].f.z, ki * vt.z);
                            s[u].f.w = fmaf(g, s[u].f.w, ki * vt.w);
                            acc[t].x = fmaf(qi, s[u].f.x, acc[t].x);
                            acc[t].y = fmaf(qi, s[u].f.y, acc[t].y);
                            acc[t].z = fmaf(qi, s[u].f.z, acc[t].z);
                            acc[t].w = fmaf(qi, s[u].f.w, acc[t].w);
                        }
                    }
                }
            }
        }
#pragma unroll
        for (int u = 0; u < kMultiRowsInFlight; ++u) {
            const int i = i0 + u * RG;
            if (i < dk) __stcs(reinterpret_cast<float4 *>(S + (size_t)i * dv), s[u].f);
        }
    }

    // o_t[c'] = the sum over row groups: the lanes of a warp that share this
    // thread's columns (lane bits TPR and up) by shuffles, then the warps
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int t = 0; t < TMAX; ++t) {
        if (t < T) {
#pragma unroll
            for (int off = TPR; off < 32; off <<= 1) {
                acc[t].x += __shfl_xor_sync(0xffffffffu, acc[t].x, off);
                acc[t].y += __shfl_xor_sync(0xffffffffu, acc[t].y, off);
                acc[t].z += __shfl_xor_sync(0xffffffffu, acc[t].z, off);
                acc[t].w += __shfl_xor_sync(0xffffffffu, acc[t].w, off);
            }
        }
    }
    __syncthreads();  // every thread is done with q^ and k^
#pragma unroll
    for (int t = 0; t < TMAX; ++t)
        if (t < T && lane < TPR) *reinterpret_cast<float4 *>(&red[warp][t][4 * tpr]) = acc[t];
    __syncthreads();
    for (int idx = threadIdx.x; idx < T * COLS; idx += kThreads) {
        const int t = idx / COLS, cc = idx - t * COLS;
        float tot = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) tot += red[w][t][cc];
        st(o, ((size_t)bh * T + t) * dv + ct * COLS + cc, tot);
    }
}

template <typename TI, typename TO, int TMAX>
cudaError_t launch_multi(const Params &p, int T, const void *q, const void *k, const void *v,
                         float *state, void *o, cudaStream_t st) {
    const int cols = (p.dv % 32 == 0) ? 32 : 4;
    const int tiles = p.dv / cols;
    const long long blocks = (long long)p.B * p.H * tiles;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    const TI *qq = (const TI *)q, *kk = (const TI *)k, *vv = (const TI *)v;
    TO *oo = (TO *)o;
    if (cols == 32)
        recurrent_multi_kernel<TI, TO, 32, TMAX, kMultiPacked><<<(unsigned)blocks, kThreads, 0, st>>>(p, T, tiles, qq, kk, vv, state, oo);
    else
        recurrent_multi_kernel<TI, TO, 4, TMAX, kMultiPacked><<<(unsigned)blocks, kThreads, 0, st>>>(p, T, tiles, qq, kk, vv, state, oo);
    cudaError_t err = cudaGetLastError();
    if (err == cudaSuccess) note_launches(1);
    return err;
}

template <typename TI, typename TO>
cudaError_t launch_multi_t(const Params &p, int T, const void *q, const void *k, const void *v,
                           float *state, void *o, cudaStream_t st) {
    if (T <= 4) return launch_multi<TI, TO, 4>(p, T, q, k, v, state, o, st);
    if (T <= 8) return launch_multi<TI, TO, 8>(p, T, q, k, v, state, o, st);
    return launch_multi<TI, TO, 16>(p, T, q, k, v, state, o, st);
}

template <typename TI, typename TO>
cudaError_t launch_t(const Params &p, const void *q, const void *k, const void *v,
                     float *state, void *o, cudaStream_t st) {
    int cols = (p.dv % 32 == 0) ? 32 : (p.dv % 16 == 0) ? 16 : (p.dv % 8 == 0) ? 8 : 4;
    int tiles = p.dv / cols;
    long long blocks = (long long)p.B * p.H * tiles;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    const TI *qq = (const TI *)q, *kk = (const TI *)k, *vv = (const TI *)v;
    TO *oo = (TO *)o;
    switch (cols) {
        case 32: recurrent_step_kernel<TI, TO, 32><<<(unsigned)blocks, kThreads, 0, st>>>(p, tiles, qq, kk, vv, state, oo); break;
        case 16: recurrent_step_kernel<TI, TO, 16><<<(unsigned)blocks, kThreads, 0, st>>>(p, tiles, qq, kk, vv, state, oo); break;
        case 8: recurrent_step_kernel<TI, TO, 8><<<(unsigned)blocks, kThreads, 0, st>>>(p, tiles, qq, kk, vv, state, oo); break;
        default: recurrent_step_kernel<TI, TO, 4><<<(unsigned)blocks, kThreads, 0, st>>>(p, tiles, qq, kk, vv, state, oo); break;
    }
    cudaError_t err = cudaGetLastError();
    if (err == cudaSuccess) note_launches(1);
    return err;
}

}  // namespace

cudaError_t launch_recurrent_step(const Params &p, bool in_bf16, bool out_bf16,
                                  const void *q, const void *k, const void *v,
                                  float *state, void *o, cudaStream_t st) {
    if (p.L > 1) {  // several tokens per sequence in one pass over the state
        if (in_bf16)
            return out_bf16 ? launch_multi_t<__nv_bfloat16, __nv_bfloat16>(p, p.L, q, k, v, state, o, st)
                            : launch_multi_t<__nv_bfloat16, float>(p, p.L, q, k, v, state, o, st);
        return out_bf16 ? launch_multi_t<float, __nv_bfloat16>(p, p.L, q, k, v, state, o, st)
                        : launch_multi_t<float, float>(p, p.L, q, k, v, state, o, st);
    }
    if (in_bf16)
        return out_bf16 ? launch_t<__nv_bfloat16, __nv_bfloat16>(p, q, k, v, state, o, st)
                        : launch_t<__nv_bfloat16, float>(p, q, k, v, state, o, st);
    return out_bf16 ? launch_t<float, __nv_bfloat16>(p, q, k, v, state, o, st)
                    : launch_t<float, float>(p, q, k, v, state, o, st);
}

}  // namespace ret
