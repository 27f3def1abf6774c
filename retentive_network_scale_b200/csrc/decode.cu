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
#include <algorithm>
#include <type_traits>

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
// [B][H][T][d].  A thread owns CPT adjacent columns of one head's state and
// streams through all d_k rows of them, so o_t of its columns is complete
// in its registers at the end: no reduction across threads.  A warp reads
// 32 CPT adjacent floats of a row per load (whole 128-byte lines); every
// thread keeps AHEAD rows of loads in flight in a ring of registers
// that is updated in place, the first of them issued before the operands
// are set up.  The operands of row i, the rotated (and rescaled, below)
// k~_t[i] and q~_t[i] for every t, sit in shared memory as packed fp32
// pairs (k, k, q, q), one 16-byte broadcast load per row and token; every
// update is a packed fused multiply-add on two columns, two rows at a time
// for independent chains, and v_t of the thread's columns stays in
// registers.
constexpr int kMultiThreads = 128;  // threads (columns / CPT) per CTA, at most

// Per token count: columns per thread (v_t and o_t live in registers), rows
// of loads in flight per thread (even) and the CTAs per SM the registers are
// budgeted for; measured on B200 at B=64, H=16, d_k=256, d_v=512.
template <int TMAX>
struct MultiCfg {
    static constexpr int CPT = TMAX > 8 ? 2 : 4;
    static constexpr int NPR = CPT / 2;  // fp32 pairs per row piece
    static constexpr int AHEAD = TMAX > 4 ? 10 : 8;
    static constexpr int MIN_CTAS = TMAX > 4 ? 3 : 4;
    static __host__ __device__ size_t rec_bytes(int dk) { return (size_t)dk * TMAX * 16; }
    static __host__ __device__ size_t smem_bytes(int dk) { return rec_bytes(dk) + (size_t)(kMaxDk / 2) * 8; }
};

template <int NPR>
struct Piece {
    uint64_t u[NPR];
};
__device__ __forceinline__ void ld_piece(Piece<2> &r, const float *p) {
    const ulonglong2 x = __ldcs(reinterpret_cast<const ulonglong2 *>(p));
    r.u[0] = x.x;
    r.u[1] = x.y;
}
__device__ __forceinline__ void ld_piece(Piece<1> &r, const float *p) {
    r.u[0] = __ldcs(reinterpret_cast<const unsigned long long *>(p));
}
__device__ __forceinline__ void st_piece(float *p, const Piece<2> &r) {
    __stcs(reinterpret_cast<ulonglong2 *>(p), make_ulonglong2(r.u[0], r.u[1]));
}
__device__ __forceinline__ void st_piece(float *p, const Piece<1> &r) {
    __stcs(reinterpret_cast<unsigned long long *>(p), (unsigned long long)r.u[0]);
}

template <typename TI, typename TO, int TMAX>
__global__ void __launch_bounds__(kMultiThreads, MultiCfg<TMAX>::MIN_CTAS)
recurrent_multi_kernel(Params p, int T, int ncol_tiles, const TI *q, const TI *k, const TI *v,
                       float *state, TO *o) {
    using Cfg = MultiCfg<TMAX>;
    constexpr int CPT = Cfg::CPT, NPR = Cfg::NPR;
    constexpr int R = Cfg::AHEAD;
    static_assert(R % 2 == 0, "rows go in pairs");
    extern __shared__ __align__(16) uint8_t dsm[];
    const int dk = p.dk, dv = p.dv;
    float4 *rec = reinterpret_cast<float4 *>(dsm);  // [dk][TMAX]: (k~, k~, q~, q~)
    double *s_theta = reinterpret_cast<double *>(dsm + Cfg::rec_bytes(dk));

    const int bh = blockIdx.x / ncol_tiles, ct = blockIdx.x - bh * ncol_tiles;
    const int h = bh % p.H;
    const int c = (ct * blockDim.x + threadIdx.x) * CPT;
    const bool active = c < dv;
    float *S = state + (size_t)bh * dk * dv + c;

    // rows 0 .. R-1 of the thread's columns, in flight during the set-up
    Piece<NPR> ring[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
        if (active && r < dk) ld_piece(ring[r], S + (size_t)r * dv);
        else
#pragma unroll
            for (int j = 0; j < NPR; ++j) ring[r].u[j] = 0ull;
    }
    Piece<NPR> vt[TMAX];  // zero past T
#pragma unroll
    for (int t = 0; t < TMAX; ++t)
#pragma unroll
        for (int j = 0; j < NPR; ++j) {
            const size_t base = ((size_t)bh * T + t) * dv + c + 2 * j;
            vt[t].u[j] = active && t < T ? tc::f2_make(ld(v, base), ld(v, base + 1)) : 0ull;
        }
    // With gamma^T >= 2^-60 the T updates run on a rescaled state: with
    // s_t = gamma s_{t-1} + k_t v_t from s_{-1} = S,
    //   s_t = gamma^{t+1} a_t,  a_t = S + sum_{tau<=t} gamma^{-(tau+1)} k_tau v_tau,
    //   o_t = q_t . s_t = (gamma^{t+1} q_t) . a_t,
    // so with k~_t = gamma^{-(t+1)} k_t and q~_t = gamma^{t+1} q_t each token
    // costs a += k~ v and o += q~ a, and the state leaves as gamma^T a.  The
    // final scaling brings every term back to its own magnitude, so the
    // relative rounding is that of the direct form.  Other decays (gamma = 0
    // among them) take the direct form with k~ = k^, q~ = q^.
    const float lg = p.log2g[h];
    const bool scaled = (float)T * lg >= -60.f;
    auto fq = [&](int t) { return scaled ? exp2f((float)(t + 1) * lg) : 1.f; };
    auto fk = [&](int t) { return scaled ? exp2f(-(float)(t + 1) * lg) : 1.f; };

    // operands (q~_t, k~_t turned at position pos_offset + t)
    if (p.rotate) {
        stage_theta(p, s_theta, dk / 2);
        __syncthreads();
        for (int idx = threadIdx.x; idx < T * (dk / 2); idx += blockDim.x) {
            const int t = idx / (dk / 2), j = idx - t * (dk / 2);
            const size_t base = ((size_t)bh * T + t) * dk;
            float cs, sn;
            rot_cs_fast(p.pos_offset + t, s_theta[j], &cs, &sn);
            float q0 = ld(q, base + 2 * j), q1 = ld(q, base + 2 * j + 1);
            float k0 = ld(k, base + 2 * j), k1 = ld(k, base + 2 * j + 1);
            rot_pair(q0, q1, cs, sn);
            rot_pair(k0, k1, cs, sn);
            const float a = fq(t), b = fk(t);
            rec[(2 * j) * TMAX + t] = make_float4(b * k0, b * k0, a * q0, a * q0);
            rec[(2 * j + 1) * TMAX + t] = make_float4(b * k1, b * k1, a * q1, a * q1);
        }
    } else {
        for (int idx = threadIdx.x; idx < T * dk; idx += blockDim.x) {
            const int t = idx / dk, i = idx - t * dk;
            const float kk = fk(t) * ld(k, ((size_t)bh * T + t) * dk + i);
            const float qq = fq(t) * ld(q, ((size_t)bh * T + t) * dk + i);
            rec[i * TMAX + t] = make_float4(kk, kk, qq, qq);
        }
    }
    // tokens T .. TMAX-1 carry zero operands: on the rescaled path they add
    // nothing (a += 0 v), so its loops need no test on t
    for (int idx = threadIdx.x; idx < (TMAX - T) * dk; idx += blockDim.x) {
        const int t = T + idx / dk, i = idx % dk;
        rec[i * TMAX + t] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    __syncthreads();
    if (!active) return;

    const float g = exp2f(lg);
    const uint64_t G2 = tc::f2_make(g, g);
    const float gT = exp2f((float)T * lg);
    const uint64_t GT2 = tc::f2_make(gT, gT);
    Piece<NPR> acc[TMAX];
#pragma unroll
    for (int t = 0; t < TMAX; ++t)
#pragma unroll
        for (int j = 0; j < NPR; ++j) acc[t].u[j] = 0ull;

    // rows i and (with TWO) i+1, updated in place in their ring slots and
    // stored
    auto rows = [&](auto sc, auto two, int i, Piece<NPR> &s0, Piece<NPR> &s1) {
        constexpr bool SC = decltype(sc)::value, TWO = decltype(two)::value;
        const float4 *rc = rec + i * TMAX;
#pragma unroll
        for (int t = 0; t < TMAX; ++t) {
            if (SC || t < T) {
                const ulonglong2 a = *reinterpret_cast<const ulonglong2 *>(rc + t);
                ulonglong2 b;
                if (TWO) b = *reinterpret_cast<const ulonglong2 *>(rc + TMAX + t);
#pragma unroll
                for (int j = 0; j < NPR; ++j) {
                    if (SC) {
                        s0.u[j] = tc::f2_fma(a.x, vt[t].u[j], s0.u[j]);
                        if (TWO) s1.u[j] = tc::f2_fma(b.x, vt[t].u[j], s1.u[j]);
                    } else {
                        s0.u[j] = tc::f2_fma(G2, s0.u[j], tc::f2_mul(a.x, vt[t].u[j]));
                        if (TWO) s1.u[j] = tc::f2_fma(G2, s1.u[j], tc::f2_mul(b.x, vt[t].u[j]));
                    }
                    acc[t].u[j] = tc::f2_fma(a.y, s0.u[j], acc[t].u[j]);
                    if (TWO) acc[t].u[j] = tc::f2_fma(b.y, s1.u[j], acc[t].u[j]);
                }
            }
        }
        if (SC) {
#pragma unroll
            for (int j = 0; j < NPR; ++j) {
                s0.u[j] = tc::f2_mul(GT2, s0.u[j]);
                if (TWO) s1.u[j] = tc::f2_mul(GT2, s1.u[j]);
            }
        }
        st_piece(S + (size_t)i * dv, s0);
        if (TWO) st_piece(S + (size_t)(i + 1) * dv, s1);
    };
    auto pass = [&](auto sc) {
        const std::true_type two;
        const std::false_type one;
        // whole groups of R rows: no tests on the row index; after a pair is
        // stored its slots take the rows R further on
        const int full = dk - dk % R;
#pragma unroll 1
        for (int i0 = 0; i0 < full; i0 += R) {
            const bool more = i0 + R < dk;
#pragma unroll
            for (int r = 0; r < R; r += 2) {
                rows(sc, two, i0 + r, ring[r], ring[r + 1]);
                if (more) {
                    if (i0 + R + r < dk) ld_piece(ring[r], S + (size_t)(i0 + R + r) * dv);
                    if (i0 + R + r + 1 < dk) ld_piece(ring[r + 1], S + (size_t)(i0 + R + r + 1) * dv);
                }
            }
        }
        // the last dk % R rows, already in slots 0 ..
#pragma unroll
        for (int r = 0; r < R; r += 2) {
            if (full + r + 1 < dk)
                rows(sc, two, full + r, ring[r], ring[r + 1]);
            else if (full + r < dk)
                rows(sc, one, full + r, ring[r], ring[r + 1]);
        }
    };
    if (scaled)
        pass(std::true_type{});
    else
        pass(std::false_type{});

#pragma unroll
    for (int t = 0; t < TMAX; ++t)
        if (t < T)
#pragma unroll
            for (int j = 0; j < NPR; ++j) {
                const size_t base = ((size_t)bh * T + t) * dv + c + 2 * j;
                st(o, base, tc::f2_lo(acc[t].u[j]));
                st(o, base + 1, tc::f2_hi(acc[t].u[j]));
            }
}

template <typename TI, typename TO, int TMAX>
cudaError_t launch_multi(const Params &p, int T, const void *q, const void *k, const void *v,
                         float *state, void *o, cudaStream_t st) {
    constexpr int CPT = MultiCfg<TMAX>::CPT;
    const int nthr = p.dv / CPT;  // d_v is a multiple of 4
    const int threads = std::min(kMultiThreads, (nthr + 31) / 32 * 32);
    const int tiles = (nthr + threads - 1) / threads;
    const long long blocks = (long long)p.B * p.H * tiles;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    auto kern = recurrent_multi_kernel<TI, TO, TMAX>;
    const size_t smem = MultiCfg<TMAX>::smem_bytes(p.dk);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)blocks, threads, smem, st>>>(p, T, tiles, (const TI *)q, (const TI *)k,
                                                  (const TI *)v, state, (TO *)o);
    e = cudaGetLastError();
    if (e == cudaSuccess) note_launches(1);
    return e;
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
