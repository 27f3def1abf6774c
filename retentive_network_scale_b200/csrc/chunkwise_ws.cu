// chunkwise_ws.cu -- chunkwise retention on the sm_100a tensor cores as a
// warp-specialised pipeline, with the per-head GroupNorm + swish gate fused.
//
// "Retentive Network" paper summary, section 2.1, chunkwise recurrent form
// (3): parallel inside a chunk, a decayed state carried between chunks.  For
// the chunk of n rows after state R, with xPos-rotated rows q^_j, k^_j:
//   o_j = sum_{j'<=j} gamma^{j-j'} (q^_j.k^_j') v_j' + gamma^{j+1} q^_j R
//   R  <- gamma^n R + sum_j' gamma^{n-1-j'} k^_j'^T v_j'
// The tensor cores see plain products only:
//   Rbar = bf16(gamma^n R),  O'' = Q^ Rbar + mask(Q^ K'^T) V',
//   o_j = gamma^{j+1-n} O''_j,  R <- gamma^n R + K'^T V'
// where the row weight zeta_j = gamma^{n-1-j} sits either on the key rows
// (K' = diag(zeta) K^, V' = V: rows prepared by the streaming pass, or
// turned and weighted here in shared memory as their tiles land) or on the
// value rows (K' = K^, V' = diag(zeta) V, applied here in shared memory;
// this needs no pass over Q and K at all when there is no rotation).  Both
// give gamma^{j+1-n} gamma^{n-1-j'} = gamma^{j-j'} term by term.  All
// factors stay in range while gamma^128 >= 2^-60.
//
// One CTA owns one (b, h) and 128 value columns (d_v = 64: one CTA with 64,
// the rest of its V tile zero); the CTAs of a head form a cluster.  d_k is
// 64, 128 or 256.  No role waits for a whole chunk to finish: every
// hand-over is an mbarrier, so the epilogue of chunk c runs while the
// tensor cores work on chunk c+1.  Roles (16 warps):
//   warp 0      issues the MMAs (one thread), chunk by chunk:
//               S = Q^ K'^T -> O'' = Q^ Rbar -> R^T += V'^T K' -> O'' += P V'
//   warp 1      issues the TMA loads of Q^, K', V as each buffer is released
//               by the products that read it (each load is issued thousands
//               of cycles before its product; no L2 prefetch, whose issue
//               was measured to hold the issuing thread for as long)
//   warp 2      scales the V tile by zeta (value-row mode only)
//   warp 3      announces this CTA's GroupNorm partials to the cluster (its
//               arrivals on the peers' barriers need not wait for the
//               epilogue's global loads and stores in flight)
//   warps 4-7   P = bf16(mask(S)) into tensor memory; then the state pass
//               (R^T <- gamma^{n'} R^T in TMEM and its bf16 copy Rbar^T in
//               shared memory for the next chunk, or state_out after the last);
//               with the rotation in the loop, then the xPos turn (and key
//               weights) of the next chunk's Q and K tiles
//   warps 8-15  the epilogue: O'' leaves tensor memory for registers at once
//               (the next chunk's O'' may then start), row statistics merged
//               across the cluster through distributed shared memory and
//               cluster-scope mbarriers, G read and Y written straight
//               between registers and global memory
// Global accesses of the epilogue are coalesced by 4 x 4 transposes of
// 16-byte pieces among groups of 4 lanes (shuffles): a thread holds one row
// (its TMEM lane), a load or store instruction covers 64 contiguous bytes
// of each of 8 rows.  G and Y therefore take no shared memory, which is what
// lets every buffer be released and reloaded independently.
//
// Tensor memory (512 columns): S [128 x 128] (P overwrites half of each
// 32-column group), O'' [128 x 128], R^T [128 x d_k].  Shared memory: Q^
// (d_k/64 blocks of 16 KB), K' and Rbar^T interleaved per 64-column block
// (32 KB each), V' (2 x 16 KB), barriers and the GroupNorm partials.
//
// Every wait is bounded (about 2 s of SM clock): on expiry the kernel
// latches RET_ERR_TIMEOUT in the device status word, every role leaves its
// loop, copies and MMAs still in flight get a bounded drain, the cluster
// meets once more so no peer is left reading this CTA's shared memory, and
// tensor memory is freed.
#include <cuda.h>

#include <cstring>
#include <type_traits>

#include "common.cuh"
#include "launch.h"
#include "tc_util.cuh"

namespace ret {
namespace {

using namespace tc;

constexpr int kC = 128;   // rows per block (MMA M)
constexpr int kTV = 128;  // value columns per CTA
constexpr int kThreads = 512;
constexpr int kMaxCluster = kMaxDv / kTV;
constexpr long long kTimeoutCycles = 4000000000LL;  // about 2 s

// QF/KF/VF: tile landed (TMA); VR: V' scaled (value-row mode); SSD: S done;
// SOD: Q^ Rbar done (Q^ and Rbar^T free); UD: state update done (K' free);
// PVD: P V' done (V' free, O'' final); PR: P written; RBL: the first half
// of Rbar^T (d-columns below d_k/2) written; RB: state pass done (all of
// Rbar^T and the decayed R^T ready); OF: O'' copied out by the epilogue;
// SL: this CTA's GroupNorm partials written; GX0/GX1: the partials of every
// CTA of the head published (by chunk parity).
// QR/KR: Q^ / K~ turned in shared memory (rotation in the loop only).
enum { QF = 0, KF, VF, VR, SSD, SOD, UD, PVD, PR, RBL, RB, OF, SL, GX0, GX1, QR, KR, kNumBars };

template <int DK>
struct Layout {
    static constexpr uint32_t kQ = 0;
    static constexpr uint32_t kQBytes = kC * DK * 2;
    static constexpr uint32_t kKR = kQ + kQBytes;  // [K' block | Rbar^T block] x DK/64
    static constexpr uint32_t kKRBytes = 2 * kC * DK * 2;
    static constexpr uint32_t kV = kKR + kKRBytes;
    static constexpr uint32_t kVBytes = kC * kTV * 2;
    static constexpr uint32_t kSmall = kV + kVBytes;
    static constexpr uint32_t kBar = kSmall;
    static constexpr uint32_t kTmemSlot = kSmall + 8 * kNumBars;
    static constexpr uint32_t kAbort = kTmemSlot + 4;
    // per row (mean, centred sum of squares) of this CTA's 128 columns, by
    // chunk parity; the peers read it remotely
    static constexpr uint32_t kSlot = kSmall + 256;
    static constexpr uint32_t kBytes = kSlot + 2 * 128 * 8;
    static_assert(8 * kNumBars + 8 <= 256, "small area");
    static __device__ __forceinline__ uint32_t k_blk(int kb) { return kKR + kb * 32768; }
    static __device__ __forceinline__ uint32_t rbar_blk(int kb) { return kKR + kb * 32768 + 16384; }
};

constexpr uint32_t kIdescSX = idesc_bf16(128, 128, 0, 0);  // S, O'': A Q^, B K' / Rbar^T rows
constexpr uint32_t kIdescPV = idesc_bf16(128, kTV, 0, 1);  // O'' += P V': A P (TMEM), B V' MN-major

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&v);
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t f2_of(const uint32_t *r) {
    return (static_cast<uint64_t>(r[1]) << 32) | r[0];
}
// a bf16 pair as a packed fp32 pair (lo, hi)
__device__ __forceinline__ uint64_t bf16x2_to_f2(uint32_t u) {
    return (static_cast<uint64_t>(u & 0xffff0000u) << 32) | (u << 16);
}
// swish(g) = g sigmoid(g) = h + h tanh(h), h = g / 2, on a bf16 pair (the
// hardware tanh approximation; one rounding to bf16 by the fused add)
__device__ __forceinline__ uint32_t swish_bf16x2(uint32_t g) {
    uint32_t h, t, s;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(h) : "r"(g), "r"(0x3f003f00u));
    asm("tanh.approx.bf16x2 %0, %1;" : "=r"(t) : "r"(h));
    asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(s) : "r"(h), "r"(t), "r"(h));
    return s;
}

__device__ __forceinline__ uint4 shfl_xor4(uint4 v, int s) {
    v.x = __shfl_xor_sync(0xffffffffu, v.x, s);
    v.y = __shfl_xor_sync(0xffffffffu, v.y, s);
    v.z = __shfl_xor_sync(0xffffffffu, v.z, s);
    v.w = __shfl_xor_sync(0xffffffffu, v.w, s);
    return v;
}
// 4 x 4 transpose of 16-byte elements among the 4 lanes of a group: lane m
// holding a[i] = X[m][i] ends with a[i] = X[i][m] (two butterfly stages,
// each lane keeping the half whose index bit matches its own).
__device__ __forceinline__ void xpose4(uint4 (&a)[4], int m) {
#pragma unroll
    for (int s = 2; s >= 1; s >>= 1) {
        const bool up = (m & s) != 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if ((i & s) == 0) {
                const uint4 r = shfl_xor4(up ? a[i] : a[i + s], s);
                if (up)
                    a[i] = r;
                else
                    a[i + s] = r;
            }
        }
    }
}

__device__ __forceinline__ uint4 ld_nc(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}
__device__ __forceinline__ void prefetch_l2(const void *p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}
__device__ __forceinline__ void st_na(void *p, uint4 v) {
    asm volatile("st.global.L1::no_allocate.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x),
                 "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

// Row c of Rbar^T (K-major, 128-byte swizzle): N (16 or 32) values of
// d-columns [d0, d0+N).
template <int DK, int N = 32>
__device__ __forceinline__ void st_rbarT_row(uint8_t *smem, int c, int d0, const float *v) {
    uint8_t *blk = smem + Layout<DK>::rbar_blk(d0 >> 6) + c * 128;
    const int ch0 = (d0 & 63) >> 3;
#pragma unroll
    for (int q = 0; q < N / 8; ++q) {
        uint4 w;
        w.x = pack_bf16(v[8 * q + 0], v[8 * q + 1]);
        w.y = pack_bf16(v[8 * q + 2], v[8 * q + 3]);
        w.z = pack_bf16(v[8 * q + 4], v[8 * q + 5]);
        w.w = pack_bf16(v[8 * q + 6], v[8 * q + 7]);
        *reinterpret_cast<uint4 *>(blk + (((ch0 + q) ^ (c & 7)) << 4)) = w;
    }
}

// The xPos turn of one landed 128-row tile in shared memory (128-byte
// swizzle, d_k/64 blocks of 64 columns `blk_stride` bytes apart): row r
// (position pos0 + r) has each pair (x_2j, x_2j+1) turned by
// (pos0 + r) theta_j and, for keys, scaled by zeta_r = gamma^{n-1-r}, the
// weight of the state update.  `nthr` threads, this one `ti`: a thread
// takes one 16-byte column chunk (4 pairs) and the rows r0, r0+RS, ...,
// two rows at a time in the lanes of packed fp32 pairs.  The angles start
// from an fp64 reduction and advance by 2 RS theta_j per step.  Rows at or
// past n are zeros from the load and stay as they are.
template <int DK>
__device__ __forceinline__ void turn_tile(uint8_t *smem, uint32_t blk0, uint32_t blk_stride,
                                          const Params &p, long long pos0, int n, bool keys,
                                          float lg, int ti, int nthr) {
    constexpr int NCH = DK / 8;  // 16-byte chunks per row
    const int RS = nthr / NCH;
    const int c16 = ti % NCH, r0 = ti / NCH;
    uint8_t *base = smem + blk0 + (c16 >> 3) * blk_stride;
    const int cw = c16 & 7;
    uint64_t C[4], NS[4], c2[4], s2[4], ns2[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const double th = p.theta[c16 * 4 + e];
        float ca, sa, cb, sb, cs, ss;
        rot_cs_fast(pos0 + r0, th, &ca, &sa);
        rot_cs_fast(pos0 + r0 + RS, th, &cb, &sb);
        rot_cs_fast(2 * RS, th, &cs, &ss);
        C[e] = f2_make(ca, cb);
        NS[e] = f2_make(-sa, -sb);
        c2[e] = f2_make(cs, cs);
        s2[e] = f2_make(ss, ss);
        ns2[e] = f2_make(-ss, -ss);
    }
    auto turn_pair = [&](uint4 &wa, uint4 &wb, int ra, int rb) {
        const float za = keys ? (ra < n ? decay_pow(lg, n - 1 - ra) : 0.f) : 1.f;
        const float zb = keys ? (rb < n ? decay_pow(lg, n - 1 - rb) : 0.f) : 1.f;
        const uint64_t Z = f2_make(za, zb);
        uint32_t *ua = reinterpret_cast<uint32_t *>(&wa);
        uint32_t *ub = reinterpret_cast<uint32_t *>(&wb);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            // x0 = low bf16, x1 = high bf16 of each row's pair
            const uint64_t X0 = (static_cast<uint64_t>(ub[e] << 16) << 32) | (ua[e] << 16);
            const uint64_t X1 = (static_cast<uint64_t>(ub[e] & 0xffff0000u) << 32) | (ua[e] & 0xffff0000u);
            const uint64_t NX0 = X0 ^ 0x8000000080000000ull;
            const uint64_t ZC = keys ? f2_mul(C[e], Z) : C[e];
            const uint64_t ZNS = keys ? f2_mul(NS[e], Z) : NS[e];
            const uint64_t Y0 = f2_fma(X1, ZNS, f2_mul(X0, ZC));   // x0 c - x1 s
            const uint64_t Y1 = f2_fma(X1, ZC, f2_mul(NX0, ZNS));  // x0 s + x1 c
            ua[e] = pack_bf16(f2_lo(Y0), f2_lo(Y1));
            ub[e] = pack_bf16(f2_hi(Y0), f2_hi(Y1));
            const uint64_t Cn = f2_fma(C[e], c2[e], f2_mul(NS[e], s2[e]));
            NS[e] = f2_fma(NS[e], c2[e], f2_mul(C[e], ns2[e]));
            C[e] = Cn;
        }
    };
    auto at = [&](int r) { return reinterpret_cast<uint4 *>(base + r * 128 + ((cw ^ (r & 7)) << 4)); };
    // rows r0 + RS k, four per step (the two rows of a packed pair RS apart)
#pragma unroll 1
    for (int ra = r0; ra < n; ra += 4 * RS) {
        const int rb = ra + RS, rc = ra + 2 * RS, rd = ra + 3 * RS;
        uint4 wa = *at(ra), wb = *at(rb), wc = *at(rc), wd = *at(rd);
        turn_pair(wa, wb, ra, rb);
        turn_pair(wc, wd, rc, rd);
        *at(ra) = wa;
        *at(rb) = wb;
        *at(rc) = wc;
        *at(rd) = wd;
    }
}

// R^T columns [D0, D1) of this thread's TMEM lane (value column `row`)
// after a chunk's state update: scaled by g2 (the next chunk's gamma^n,
// packed) back into TMEM and, as bf16, into Rbar^T for the next O''
// product; after the last chunk into state_out instead (`so` points at the
// lane's value column of d-row 0, or is null).  Units of W (16 or 32)
// columns; with PIPE the load of the next unit is in flight while the
// current one is processed (W more registers).
template <int DK, int D0, int D1, int W, bool PIPE>
__device__ __forceinline__ void state_cols(uint8_t *smem, uint32_t t_lane, int row, uint64_t g2,
                                           bool last, float *so, int dv) {
    static_assert((W == 16 || W == 32) && D0 % W == 0 && D1 % W == 0 && D1 > D0, "whole units");
    constexpr int NU = (D1 - D0) / W;
    constexpr int NB = PIPE ? 2 : 1;
    auto ld = [&](int col, uint32_t(&x)[W]) {
        if constexpr (W == 32) tmem_ld32(t_lane + col, x);
        else tmem_ld16(t_lane + col, x);
    };
    if (last) {
        // the final state, unit by unit
#pragma unroll 1
        for (int dd = D0; dd < D1; dd += W) {
            uint32_t x[W];
            ld(dd, x);
            tmem_wait_ld(x);
            if (so) {
#pragma unroll
                for (int i = 0; i < W; i += 2) {
                    const uint64_t y = f2_mul((static_cast<uint64_t>(x[i + 1]) << 32) | x[i], g2);
                    so[(size_t)(dd + i) * dv] = f2_lo(y);
                    so[(size_t)(dd + i + 1) * dv] = f2_hi(y);
                }
            }
        }
        return;
    }
    uint32_t r[NB][W];
    ld(D0, r[0]);
    tmem_wait_ld(r[0]);
#pragma unroll
    for (int u = 0; u < NU; ++u) {
        uint32_t(&cur)[W] = r[u % NB];
        if (PIPE && u + 1 < NU) ld(D0 + W * (u + 1), r[(u + 1) % NB]);
        const int dd = D0 + W * u;
        float v[W];
#pragma unroll
        for (int i = 0; i < W; i += 2) {
            const uint64_t x = f2_mul((static_cast<uint64_t>(cur[i + 1]) << 32) | cur[i], g2);
            v[i] = f2_lo(x);
            v[i + 1] = f2_hi(x);
        }
        st_rbarT_row<DK, W>(smem, row, dd, v);
#pragma unroll
        for (int i = 0; i < W; ++i) cur[i] = __float_as_uint(v[i]);
        if constexpr (W == 32) tmem_st32(t_lane + dd, cur);
        else tmem_st16(t_lane + dd, cur);
        if (u + 1 < NU) {
            if (!PIPE) ld(D0 + W * (u + 1), r[(u + 1) % NB]);
            tmem_wait_ld(r[(u + 1) % NB]);
        }
    }
}

// The starting state of R^T columns [D0, D1): gamma^{n_0} S_in^T into TMEM
// and its bf16 copy into Rbar^T (`si` points at the lane's value column of
// d-row 0, or is null for a lane past d_v: zeros); without a state
// (has_in false) zeros into Rbar^T only.
template <int DK, int D0, int D1>
__device__ __forceinline__ void state_init_cols(uint8_t *smem, uint32_t t_lane, int row, bool has_in,
                                                const float *si, float g0, int dv) {
#pragma unroll 1
    for (int d0 = D0; d0 < D1; d0 += 32) {
        float v[32];
        uint32_t r[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = si ? si[(size_t)(d0 + i) * dv] * g0 : 0.f;
        st_rbarT_row<DK>(smem, row, d0, v);
        if (has_in) {
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(v[i]);
            tmem_st32(t_lane + d0, r);
        }
    }
}

// 32 values of one row (this thread's, columns [col0, col0 + 32)) leave as
// TO, in pieces of 16 bytes that a 4 x 4 transpose among groups of 4 lanes
// gathers, so that one store instruction covers 64 contiguous bytes of 8
// rows: bf16 in one round, fp32 in two of 16 columns.  `pair(k)` gives
// columns col0 + 2k, col0 + 2k + 1 as a packed fp32 pair; `dst(i)` is the
// address of column 0 of row 4j+i of this lane's group (j = lane >> 2) and
// `ok(i)` whether that row exists.
template <typename TO, typename Pair, typename Dst, typename Ok>
__device__ __forceinline__ void store_row32(Pair pair, int m, int col0, Dst dst, Ok ok) {
    if constexpr (sizeof(TO) == 2) {
        uint4 a[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const uint64_t v0 = pair(4 * k), v1 = pair(4 * k + 1), v2 = pair(4 * k + 2), v3 = pair(4 * k + 3);
            a[k] = make_uint4(pack_bf16(f2_lo(v0), f2_hi(v0)), pack_bf16(f2_lo(v1), f2_hi(v1)),
                              pack_bf16(f2_lo(v2), f2_hi(v2)), pack_bf16(f2_lo(v3), f2_hi(v3)));
        }
        xpose4(a, m);
#pragma unroll
        for (int i = 0; i < 4; ++i)
            if (ok(i)) st_na(reinterpret_cast<__nv_bfloat16 *>(dst(i)) + col0 + 8 * m, a[i]);
    } else {
#pragma unroll
        for (int qq = 0; qq < 2; ++qq) {
            uint4 a[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint64_t v0 = pair(8 * qq + 2 * k), v1 = pair(8 * qq + 2 * k + 1);
                a[k] = make_uint4(static_cast<uint32_t>(v0), static_cast<uint32_t>(v0 >> 32),
                                  static_cast<uint32_t>(v1), static_cast<uint32_t>(v1 >> 32));
            }
            xpose4(a, m);
#pragma unroll
            for (int i = 0; i < 4; ++i)
                if (ok(i)) st_na(reinterpret_cast<float *>(dst(i)) + col0 + 16 * qq + 4 * m, a[i]);
        }
    }
}

template <int DK, typename TO, bool FUSE, bool REV, bool ROT>
__global__ void __launch_bounds__(kThreads, 1)
chunkwise_ws_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const Params p,
                    const float *__restrict__ state_in, float *__restrict__ state_out,
                    TO *__restrict__ O, const __nv_bfloat16 *__restrict__ G, long long g_row,
                    long long g_batch, TO *__restrict__ Y, float gn_eps, int zeta_v,
                    int v_head_major, int *status, const float *__restrict__ acc_in,
                    int acc_unturn) {
    using Ly = Layout<DK>;
    constexpr int KB = DK / 64;
    constexpr uint32_t kIdescU = idesc_bf16(128, DK, 1, 1);  // R^T += V'^T K' (both MN-major)
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t sbase = smem_u32(smem);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.y, h = bh % p.H, b = bh / p.H;
    const int v0 = blockIdx.x * kTV;
    const int dvr = min(kTV, p.dv - v0);  // value columns of this CTA: 128, or 64 when d_v = 64
    const float lg = p.log2g[h];
    const int L = p.L, dv = p.dv;
    const int nchunks = (L + kC - 1) / kC;
    const int nr = (int)gridDim.x;  // CTAs of this head (the cluster when FUSE)
    // the block of rows handled at step c: in order, or last to first for
    // the anti-causal form (the mask and the weights mirror within a block)
    constexpr bool rev = REV;
    auto blk = [&](int c) { return rev ? nchunks - 1 - c : c; };

    if (sbase & 1023u) {  // swizzle atoms need 1024-byte alignment (same for every CTA)
        if (tid == 0) atomicExch(status, (int)RET_ERR_CUDA);
        return;
    }
    auto bar = [&](int i) { return sbase + Ly::kBar + 8u * i; };
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Ly::kAbort);
    auto wait = [&](int i, uint32_t parity) {
        return mbar_wait_bounded(bar(i), parity, abort_flag, status, kTimeoutCycles);
    };

    if (tid == 0) {
        for (int i = 0; i < kNumBars; ++i) {
            uint32_t count = 1;
            // one arrival per warp of the role (lane 0, after the warp has met)
            if (i == VR) count = 1;
            if (i == PR || i == RBL || i == RB || i == QR || i == KR) count = 4;
            if (i == OF) count = 8;
            if (i == GX0 || i == GX1) count = nr;
            mbar_init(bar(i), count);
        }
        *abort_flag = 0;
        fence_mbar_init();
        fence_proxy_async_smem();
    }
    if (warp == 0) {
        tmem_alloc(sbase + Ly::kTmemSlot, 512);
        tmem_relinquish();
    }
    if (dvr < kTV) {
        // d_v = 64: the V tile's second block is never loaded and stays zero
        for (int i = tid; i < 16384 / 16; i += kThreads)
            reinterpret_cast<uint4 *>(smem + Ly::kV + 16384)[i] = make_uint4(0u, 0u, 0u, 0u);
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    if constexpr (FUSE) cluster_sync();  // every peer's barriers exist before any remote arrive
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + Ly::kTmemSlot);
    const uint32_t tS = tmem, tO = tmem + 128, tR = tmem + 256;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const int vx0 = v_head_major ? v0 : h * dv + v0, vz = v_head_major ? bh : b;

    // One arrival for the whole warp: every lane's earlier accesses (ordered
    // for the tensor cores / the async proxy by the fences each lane ran)
    // come before lane 0's arrival through the warp barrier.
    auto warp_arrive = [&](int i) {
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(i));
    };
    // Every role decides warp-uniformly whether to go on (a lane whose wait
    // ran out while another's completed must not leave its warp half way
    // through a .sync.aligned instruction or a barrier).
    auto wait_all = [&](int i, uint32_t parity) { return __all_sync(0xffffffffu, wait(i, parity)); };

    if (warp == 0) {
        // ============================================ MMA issue (one thread)
        const uint64_t dQ = sdesc_sw128(sbase + Ly::kQ, 16, 1024);
        const uint64_t dKR = sdesc_sw128(sbase + Ly::kKR, 16, 1024);
        const uint64_t dVa = sdesc_sw128(sbase + Ly::kV, 16384, 1024);
        const uint64_t dKb = sdesc_sw128(sbase + Ly::kKR, 32768, 1024);
        const bool has_in = state_in != nullptr;
        // part 0: S (B = K' rows), part 1: O'' (B = Rbar^T rows, 16 KB further)
        auto sx = [&](int part, int ks, bool acc) {
            const uint64_t off = (uint64_t)(((ks >> 2) * 16384 + (ks & 3) * 32) >> 4);
            const uint64_t offkr = (uint64_t)(((ks >> 2) * 32768 + part * 16384 + (ks & 3) * 32) >> 4);
            mma_ss(part ? tO : tS, dQ + off, dKR + offkr, kIdescSX, acc ? 1u : 0u);
        };
#pragma unroll 1
        for (int c = 0; c < nchunks; ++c) {
            const uint32_t par = c & 1, prv = par ^ 1;
            // S: the tiles of chunk c, and P of chunk c-1 consumed
            if (!(wait_all(ROT ? QR : QF, par) && wait_all(ROT ? KR : KF, par) &&
                  (c == 0 || wait_all(PVD, prv))))
                break;
            tc_fence_after();
            if (lane == 0) {
#pragma unroll
                for (int ks = 0; ks < DK / 16; ++ks) sx(0, ks, ks > 0);
                mma_commit(bar(SSD));
            }
            __syncwarp();
            // O'' = Q^ Rbar, over the d-columns of Rbar^T the state pass of
            // chunk c-1 has written (two halves), once O'' of c-1 is read out
            if (!(wait_all(RBL, par) && (c == 0 || wait_all(OF, prv)))) break;
            tc_fence_after();
            if (lane == 0) {
#pragma unroll
                for (int ks = 0; ks < DK / 32; ++ks) sx(1, ks, ks > 0);
            }
            __syncwarp();
            if (!wait_all(RB, par)) break;
            tc_fence_after();
            if (lane == 0) {
#pragma unroll
                for (int ks = DK / 32; ks < DK / 16; ++ks) sx(1, ks, true);
                mma_commit(bar(SOD));
            }
            __syncwarp();
            // R^T += V'^T K'
            if (!wait_all(zeta_v ? VR : VF, par)) break;
            tc_fence_after();
            if (lane == 0) {
                const bool acc0 = has_in || c > 0;
#pragma unroll
                for (int ks = 0; ks < kC / 16; ++ks) {
                    const uint64_t off = (uint64_t)((ks * 2048) >> 4);
                    mma_ss(tR, dVa + off, dKb + off, kIdescU, (ks > 0 || acc0) ? 1u : 0u);
                }
                mma_commit(bar(UD));
            }
            __syncwarp();
            // O'' += P V'
            if (!wait_all(PR, par)) break;
            tc_fence_after();
            if (lane == 0) {
#pragma unroll
                for (int ks = 0; ks < kC / 16; ++ks)
                    mma_ts(tO, tS + (ks >> 1) * 32 + (ks & 1) * 8, dVa + (uint64_t)((ks * 2048) >> 4),
                           kIdescPV, 1u);
                mma_commit(bar(PVD));
            }
            __syncwarp();
        }
    } else if (warp == 1) {
        // =================================================== TMA loads
        auto load_q = [&](int c) {
            mbar_expect_tx(bar(QF), Ly::kQBytes);
            for (int kb = 0; kb < KB; ++kb)
                tma_load_3d(sbase + Ly::kQ + kb * 16384, &tmQ, bar(QF), kb * 64, blk(c) * kC, bh);
        };
        auto load_k = [&](int c) {
            mbar_expect_tx(bar(KF), Ly::kQBytes);
            for (int kb = 0; kb < KB; ++kb)
                tma_load_3d(sbase + Ly::k_blk(kb), &tmK, bar(KF), kb * 64, blk(c) * kC, bh);
        };
        auto load_v = [&](int c) {
            mbar_expect_tx(bar(VF), dvr * kC * 2);
            for (int nb = 0; nb < dvr / 64; ++nb)
                tma_load_3d(sbase + Ly::kV + nb * 16384, &tmV, bar(VF), vx0 + nb * 64, blk(c) * kC, vz);
        };
        if (lane == 0) {
            load_q(0);
            load_k(0);
            load_v(0);
        }
#pragma unroll 1
        for (int c = 0; c + 1 < nchunks; ++c) {
            const uint32_t par = c & 1;
            if (!wait_all(SOD, par)) break;
            if (lane == 0) load_q(c + 1);
            if (!wait_all(UD, par)) break;
            if (lane == 0) load_k(c + 1);
            if (!wait_all(PVD, par)) break;
            if (lane == 0) load_v(c + 1);
            __syncwarp();
        }
    } else if (warp == 2) {
        // ======================= V' = diag(zeta) V (value-row mode only)
        if (zeta_v) {
#pragma unroll 1
            for (int c = 0; c < nchunks; ++c) {
                const int n = min(kC, L - blk(c) * kC);
                if (!wait_all(VF, c & 1)) break;
#pragma unroll 1
                for (int rr = 0; rr < 4; ++rr) {
                    const int r = lane + 32 * rr;  // rows of both 64-column blocks
                    const float z = r < n ? decay_pow(lg, rev ? r : n - 1 - r) : 0.f;
                    const uint64_t Z = f2_make(z, z);
#pragma unroll
                    for (int nb = 0; nb < 2; ++nb) {
                        uint8_t *rowp = smem + Ly::kV + nb * 16384 + r * 128;
#pragma unroll
                        for (int ch = 0; ch < 8; ++ch) {
                            // rows of a phase start at different 16-byte pieces: no bank conflicts
                            uint4 *ptr = reinterpret_cast<uint4 *>(rowp + (((ch + r) & 7) << 4));
                            uint4 w = *ptr;
                            uint32_t *u = reinterpret_cast<uint32_t *>(&w);
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const uint64_t x = f2_mul(bf16x2_to_f2(u[e]), Z);
                                u[e] = pack_bf16(f2_lo(x), f2_hi(x));
                            }
                            *ptr = w;
                        }
                    }
                }
                fence_proxy_async_smem();
                warp_arrive(VR);
            }
        }
    } else if (warp == 3) {
        // ============ GroupNorm partials of each chunk, announced to the cluster
        // The epilogue's slot writes are complete in this CTA's shared memory
        // once warp 3 observes SL (CTA-scope release and acquire), and a peer
        // reads that shared memory only after it has observed the arrival
        // that follows.
        if constexpr (FUSE) {
#pragma unroll 1
            for (int c = 0; c < nchunks; ++c) {
                const uint32_t par = c & 1;
                if (!wait_all(SL, par)) break;
                if (lane == 0)
                    for (int r = 0; r < nr; ++r) mbar_arrive_remote(map_to_rank(bar(par ? GX1 : GX0), r));
                __syncwarp();
            }
        }
    } else if (warp < 8) {
        // ================ P pass and state pass (warps 4-7, one TMEM lane each)
        const int row = tid & 127;  // chunk row for S, value column for R^T
        const int quad = warp & 3;
        const bool vcol = row < dvr;  // this lane's value column exists
        float *so = state_out && vcol ? state_out + (size_t)bh * DK * dv + v0 + row : nullptr;
        {
            // starting state: R^T = gamma^{n_0} S_in^T in TMEM and Rbar^T =
            // bf16 of the same; zeros without a state
            const float *si = state_in && vcol ? state_in + (size_t)bh * DK * dv + v0 + row : nullptr;
            state_init_cols<DK, 0, DK>(smem, tR + lane_base, row, state_in != nullptr, si,
                                       decay_pow(lg, min(kC, L - blk(0) * kC)), dv);
            tmem_wait_st();
            fence_proxy_async_smem();
            tc_fence_before();
            warp_arrive(RBL);
            warp_arrive(RB);
        }
        // With the rotation in the loop: Q^ and K~ of step c turned in shared
        // memory once their tiles land (the products wait on QR / KR)
        auto turn = [&](int c) {
            if constexpr (ROT) {
                const uint32_t par = c & 1;
                const int t0 = blk(c) * kC, n = min(kC, L - t0);
                const long long pos0 = p.pos_offset + t0;
                if (!wait_all(QF, par)) return false;
                turn_tile<DK>(smem, Ly::kQ, 16384, p, pos0, n, false, lg, tid - 128, 128);
                fence_proxy_async_smem();
                warp_arrive(QR);
                if (!wait_all(KF, par)) return false;
                turn_tile<DK>(smem, Ly::kKR, 32768, p, pos0, n, true, lg, tid - 128, 128);
                fence_proxy_async_smem();
                warp_arrive(KR);
            }
            return true;
        };
        bool turned = turn(0);
#pragma unroll 1
        for (int c = 0; c < nchunks && turned; ++c) {
            const uint32_t par = c & 1;
            const bool last = c + 1 == nchunks;
            const int n_next = last ? 0 : min(kC, L - (rev ? blk(c + 1) : c + 1) * kC);
            if (!wait_all(SSD, par)) break;
            tc_fence_after();
            // P = bf16(S) on keys j' <= j (j' >= j anti-causal), else 0: keys
            // [32 cb, 32 cb + 32) into columns [32 cb, 32 cb + 16); groups on
            // the far side of the diagonal block are zero for every row of
            // this warp
#pragma unroll 1
            for (int cb = 0; cb < 4; ++cb) {
                uint32_t pk[16];
                if (rev ? cb < quad : cb > quad) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) pk[i] = 0u;
                } else {
                    uint32_t a[32];
                    tmem_ld32(tS + lane_base + 32 * cb, a);
                    tmem_wait_ld(a);
                    if (rev ? cb > quad : cb < quad) {
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            pk[i] = pack_bf16(__uint_as_float(a[2 * i]), __uint_as_float(a[2 * i + 1]));
                    } else {
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const int k0 = 32 * cb + 2 * i;
                            const bool in0 = rev ? k0 >= row : k0 <= row;
                            const bool in1 = rev ? k0 + 1 >= row : k0 + 1 <= row;
                            pk[i] = pack_bf16(in0 ? __uint_as_float(a[2 * i]) : 0.f,
                                              in1 ? __uint_as_float(a[2 * i + 1]) : 0.f);
                        }
                    }
                }
                tmem_st16(tS + lane_base + 32 * cb, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            warp_arrive(PR);
            // state pass, once the state update has landed and the O''
            // product no longer reads Rbar^T
            if (!(wait_all(UD, par) && wait_all(SOD, par))) break;
            tc_fence_after();
            // (the first half of Rbar^T is published as soon as it is written)
            const float gnext = last ? 1.f : decay_pow(lg, n_next);
            const uint64_t g2 = f2_make(gnext, gnext);
            const uint32_t tl = tR + lane_base;
            if constexpr (DK >= 128) {
                state_cols<DK, 0, DK / 2, 32, true>(smem, tl, row, g2, last, so, dv);
                tmem_wait_st();
                fence_proxy_async_smem();
                tc_fence_before();
                warp_arrive(RBL);
                state_cols<DK, DK / 2, DK, 32, true>(smem, tl, row, g2, last, so, dv);
            } else {
                state_cols<DK, 0, DK, 32, true>(smem, tl, row, g2, last, so, dv);
            }
            tmem_wait_st();
            fence_proxy_async_smem();
            tc_fence_before();
            if constexpr (DK < 128) warp_arrive(RBL);
            warp_arrive(RB);
            if (!last && !(turned = turn(c + 1))) break;
        }
    } else {
        // ============================================ epilogue (warps 8-15)
        const int gtid = tid - 256;
        const int gwg = gtid >> 7;          // which 64 of the CTA's 128 columns
        const int quad = warp & 3;          // rows 32 quad .. 32 quad + 31
        const int row = 32 * quad + lane;   // this thread's row (TMEM lane)
        const int j4 = lane >> 2, m4 = lane & 3;  // groups of 4 lanes
        const int o0 = gwg * 64;
        const bool ocols = o0 < dvr;  // this thread's 64 columns exist (d_v = 64: group 0 only)
        // A segment head (p.seg_heads = S > 1: head h is segment h mod S of
        // head h / S, rows at (h mod S) * L of that head's sequence of S * L
        // rows) reads G and writes Y of its own rows of the real head.
        const int S = p.seg_heads, hr = h / S, sg = h - hr * S;
        const size_t ycol = (size_t)hr * dv + v0 + o0;  // column of Y / G of this thread's segment
        const size_t ypitch = (size_t)(p.H / S) * dv, yrow0 = (size_t)b * S * L + (size_t)sg * L;
        // rows of this lane group's 16-byte row pieces: 32 quad + 4 j4 + i
        auto grow = [&](int i) { return 32 * quad + 4 * j4 + i; };
        const __nv_bfloat16 *Gb = G + (size_t)b * g_batch + (size_t)sg * L * g_row + ycol;
        // With the gate, each chunk goes: G(c) loads issued; O''(c) copied
        // out of tensor memory (which is then released at once to the next
        // chunk's product); its row statistics published to the cluster;
        // then Y(c), once every CTA of the head has published.  The G loads
        // land while O'' is read out and the statistics are exchanged.  What
        // Y(c) needs of O'' is kept, per row segment of 64 columns, as
        // O'' - shift in bf16 (the shift is the segment's first value, so the
        // residuals are of the size of the row's spread and keep fp32's
        // range) with the shift.
        uint32_t rp[32];  // residuals of the chunk, bf16 pairs
        uint4 gp[8];      // its G, two halves of 32 columns (16-byte pieces as loaded, rows 4 j4 + i)
        float shift_p = 0.f, alpha_p = 1.f;
        int t0_p = 0, n_p = 0;
        // Y of chunk c_p (parity par_p), once every CTA of the head has
        // published its statistics.  A wait that runs out leaves the
        // chunk's Y unwritten; the group stops at the next barrier.
        auto finish = [&](int c_p) {
            const uint32_t par_p = c_p & 1;
            if (!mbar_wait_cluster_bounded(bar(par_p ? GX1 : GX0), (c_p >> 1) & 1, abort_flag,
                                           status, kTimeoutCycles))
                return;
            const uint32_t own = sbase + Ly::kSlot + (par_p * 128 + row) * 8;
            float2 e[kMaxCluster];
#pragma unroll
            for (int r = 0; r < kMaxCluster; ++r)
                if (r < nr) e[r] = ld_cluster_f32x2(map_to_rank(own, r));
            // each half to row `row`, 16-byte pieces 0..3 of its 32 columns
            xpose4(*reinterpret_cast<uint4(*)[4]>(gp), m4);
            xpose4(*reinterpret_cast<uint4(*)[4]>(gp + 4), m4);
            // swish(G) in place: sw[k] holds columns 2k, 2k+1
            uint32_t *sw = reinterpret_cast<uint32_t *>(gp);
#pragma unroll
            for (int k = 0; k < 32; ++k) sw[k] = swish_bf16x2(sw[k]);
            float mean = 0.f, m2 = 0.f;
#pragma unroll
            for (int r = 0; r < kMaxCluster; ++r)
                if (r < nr) mean += e[r].x;
            mean /= (float)nr;
#pragma unroll
            for (int r = 0; r < kMaxCluster; ++r)
                if (r < nr) m2 += e[r].y + (float)dvr * (e[r].x - mean) * (e[r].x - mean);
            const float var = m2 / (float)(nr * dvr);  // of O''; O = alpha O''
            const float scale = alpha_p * rsqrtf(alpha_p * alpha_p * var + gn_eps);
            const uint64_t SC = f2_make(scale, scale);
            const float off = (shift_p - mean) * scale;
            const uint64_t OFF = f2_make(off, off);
            // Y = swish(G) ((O'' - shift) scale + (shift - mean) scale)
#pragma unroll
            for (int hf = 0; hf < 2; ++hf)
                store_row32<TO>(
                    [&](int k) {
                        return f2_mul(f2_fma(bf16x2_to_f2(rp[16 * hf + k]), SC, OFF), bf16x2_to_f2(sw[16 * hf + k]));
                    },
                    m4, 32 * hf,
                    [&](int i) { return Y + (yrow0 + t0_p + grow(i)) * ypitch + ycol; },
                    [&](int i) { return ocols && grow(i) < n_p; });
        };
#pragma unroll 1
        for (int c = 0; c < nchunks; ++c) {
            const uint32_t par = c & 1;
            const int t0 = blk(c) * kC;
            const int n = min(kC, L - t0);
            auto row_ok = [&](int i) { return ocols && grow(i) < n; };
            if constexpr (FUSE) {
                // G of this chunk (coalesced: one instruction reads 64
                // contiguous bytes of each of 8 rows)
#pragma unroll
                for (int hf = 0; hf < 2; ++hf)
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int r = grow(i);
                        gp[4 * hf + i] = ocols && r < n ? ld_nc(Gb + (size_t)(t0 + r) * g_row + 32 * hf + 8 * m4)
                                                        : make_uint4(0u, 0u, 0u, 0u);
                    }
                // and the next chunk's G into L2 (a row segment of 64 columns
                // is one 128-byte line), so that its loads do not wait on HBM
                if (m4 == 0 && ocols && c + 1 < nchunks) {
                    const int t1 = rev ? blk(c + 1) * kC : t0 + kC, n1 = min(kC, L - t1);
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        if (grow(i) < n1) prefetch_l2(Gb + (size_t)(t1 + grow(i)) * g_row);
                }
            }
            {
                // with the gate the group meets at named barriers below, so it
                // decides together whether to go on
                bool ok = wait_all(PVD, par);
                if constexpr (FUSE) ok = named_sync_and(1, 256, ok);
                if (!ok) break;
            }
            tc_fence_after();
            // gamma^{row+1-n} (gamma^{-row} anti-causal)
            const float alpha = exp2f((float)(rev ? -row : row + 1 - n) * lg);
            const uint64_t A2 = f2_make(alpha, alpha);
            // O'' in two halves of 32 columns: O (when asked for), the
            // running statistics (shifted by the row's first value, even
            // and odd columns in packed fp32 lanes) and the residuals
            float shift = 0.f;
            uint64_t S1 = 0, S2 = 0;
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                uint32_t x[32];
                tmem_ld32(tO + lane_base + o0 + 32 * hf, x);
                tmem_wait_ld(x);
                if (hf == 1) {
                    tc_fence_before();
                    warp_arrive(OF);  // the next chunk's O'' may overwrite tensor memory
                }
                bool plain = O != nullptr;
                if constexpr (!FUSE) {
                    if (O && acc_in) {
                        // O = acc_in + this product, turned back by the angles of
                        // the row's position when acc_unturn (the second half of
                        // a backward gradient: the partial sum, then Theta_t^T)
                        plain = false;
                        const int col0 = v0 + o0 + 32 * hf;
                        float v[32];
                        const bool mine = ocols && row < n;
                        const float *ar = acc_in + ((size_t)bh * L + t0 + row) * dv + col0;
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            const float4 a4 = mine ? *reinterpret_cast<const float4 *>(ar + 4 * q)
                                                   : make_float4(0.f, 0.f, 0.f, 0.f);
                            const uint64_t s0 = f2_mul(f2_of(x + 4 * q), A2), s1 = f2_mul(f2_of(x + 4 * q + 2), A2);
                            v[4 * q] = a4.x + f2_lo(s0);
                            v[4 * q + 1] = a4.y + f2_hi(s0);
                            v[4 * q + 2] = a4.z + f2_lo(s1);
                            v[4 * q + 3] = a4.w + f2_hi(s1);
                        }
                        if (acc_unturn) {
                            const long long pos = p.pos_offset + t0 + row;
#pragma unroll
                            for (int e = 0; e < 16; ++e) {
                                float c, sn;
                                rot_cs_fast(pos, p.theta[col0 / 2 + e], &c, &sn);
                                const float a0 = v[2 * e], a1 = v[2 * e + 1];
                                v[2 * e] = a0 * c + a1 * sn;
                                v[2 * e + 1] = a1 * c - a0 * sn;
                            }
                        }
                        store_row32<TO>([&](int k) { return f2_make(v[2 * k], v[2 * k + 1]); }, m4, 32 * hf,
                                        [&](int i) { return O + ((size_t)bh * L + t0 + grow(i)) * dv + v0 + o0; },
                                        row_ok);
                    }
                }
                if (plain)
                    store_row32<TO>([&](int k) { return f2_mul(f2_of(x + 2 * k), A2); }, m4, 32 * hf,
                                    [&](int i) { return O + ((size_t)bh * L + t0 + grow(i)) * dv + v0 + o0; },
                                    row_ok);
                if constexpr (FUSE) {
                    if (hf == 0) shift = __uint_as_float(x[0]);
                    const uint64_t NSH = f2_make(-shift, -shift);
#pragma unroll
                    for (int i = 0; i < 32; i += 2) {
                        const uint64_t d = f2_add(f2_of(x + i), NSH);
                        S1 = f2_add(S1, d);
                        S2 = f2_fma(d, d, S2);
                        rp[16 * hf + i / 2] = pack_bf16(f2_lo(d), f2_hi(d));
                    }
                }
            }
            if constexpr (FUSE) {
                const float s1 = f2_lo(S1) + f2_hi(S1), s2 = f2_lo(S2) + f2_hi(S2);
                const float m_w = shift + s1 * (1.f / 64.f);
                const float m2_w = fmaxf(s2 - s1 * s1 * (1.f / 64.f), 0.f);
                // the two halves of the row merge (Chan's update, equal
                // counts) in this CTA's published slot
                float2 *slot = reinterpret_cast<float2 *>(smem + Ly::kSlot + (par * 128 + row) * 8);
                if (gwg == 1 && dvr == kTV) *slot = make_float2(m_w, m2_w);
                named_sync(1, 256);
                if (gwg == 0) {
                    if (dvr == kTV) {
                        const float2 o = *slot;
                        const float d = m_w - o.x;
                        *slot = make_float2(0.5f * (m_w + o.x), m2_w + o.y + 32.f * d * d);
                    } else {
                        *slot = make_float2(m_w, m2_w);  // the row's only 64 columns
                    }
                }
                named_sync(1, 256);
                // the slots are written (the barrier above ordered them before
                // this arrival); warp 3 announces them to the cluster
                if (gtid == 0) mbar_arrive(bar(SL));
                shift_p = shift;
                alpha_p = alpha;
                t0_p = t0;
                n_p = n;
            }
            if constexpr (FUSE) finish(c);
        }
    }

    __syncthreads();
    // After an abort, copies and MMAs still in flight get a bounded time to
    // land before the shared and tensor memory are released.
    if (tid == 0 && *abort_flag) {
        const long long start = clock64();
        while (clock64() - start < 20000000LL) __nanosleep(1000);
    }
    if constexpr (FUSE) cluster_sync();  // peers may still read this CTA's partials
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <int DK, typename TO, bool FUSE, bool REV = false, bool ROT = false>
cudaError_t launch_t(const Params &p, const CUtensorMap &mq, const CUtensorMap &mk,
                     const CUtensorMap &mv, const float *s_in, float *s_out, void *O,
                     const void *G, RowLayout g, void *Y, float eps, int zeta_v,
                     int v_head_major, int *status, cudaStream_t st,
                     const float *acc_in = nullptr, int acc_unturn = 0) {
    auto kern = chunkwise_ws_kernel<DK, TO, FUSE, REV, ROT>;
    const int smem = (int)Layout<DK>::kBytes;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((p.dv + kTV - 1) / kTV, p.B * p.H);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = FUSE ? (p.dv + kTV - 1) / kTV : 1;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, mq, mk, mv, p, s_in, s_out, (TO *)O,
                           (const __nv_bfloat16 *)G, g.row, g.batch, (TO *)Y, eps, zeta_v,
                           v_head_major, status, acc_in, acc_unturn);
    if (e == cudaSuccess) note_launches(1);
    return e;
}

template <int DK>
cudaError_t launch_dk(const Params &p, bool out_bf16, const CUtensorMap &mq, const CUtensorMap &mk,
                      const CUtensorMap &mv, const float *s_in, float *s_out, void *O,
                      const void *G, RowLayout g, void *Y, float eps, int zeta_v, int vhm, bool rot,
                      int *status, cudaStream_t st, const float *acc_in, int acc_unturn) {
    const bool fuse = Y != nullptr;
    if (acc_in && (out_bf16 || fuse || rot)) return cudaErrorInvalidValue;
    if (p.reverse) {
        // the anti-causal products of the backward pass: fp32 O, no gate
        if constexpr (DK >= 128) {
            if (!out_bf16 && !fuse && !rot)
                return launch_t<DK, float, false, true>(p, mq, mk, mv, s_in, s_out, O, G, g, Y, eps, zeta_v, vhm,
                                                        status, st, acc_in, acc_unturn);
        }
        return cudaErrorInvalidValue;
    }
    if (acc_in) return launch_t<DK, float, false>(p, mq, mk, mv, s_in, s_out, O, G, g, Y, eps, zeta_v, vhm,
                                                  status, st, acc_in, acc_unturn);
    if (rot) {
        // xPos turn of the landed tiles inside the loop (d_k 128 and 256)
        if constexpr (DK >= 128) {
            if (out_bf16)
                return fuse ? launch_t<DK, __nv_bfloat16, true, false, true>(p, mq, mk, mv, s_in, s_out, O, G, g, Y, eps, zeta_v, vhm, status, st)
                            : launch_t<DK, __nv_bfloat16, false, false, true>(p, mq, mk, mv, s_in, s_out, O, G, g, Y, eps, zeta_v, vhm, status, st);
            return fuse ? launch_t<DK, float, true, false, true>(p, mq, mk, mv, s_in, s_out, O, G, g, Y, eps, zeta_v, vhm, status, st)
                        : launch_t<DK, float, false, false, true>(p, mq, mk, mv, s_in, s_out, O, G, g, Y, eps, zeta_v, vhm, status, st);
        }
        return cudaErrorInvalidValue;
    }
    if (out_bf16)
        return fuse ? launch_t<DK, __nv_bfloat16, true>(p, mq, mk, mv, s_in, s_out, O, G, g, Y, eps, zeta_v, vhm, status, st)
                    : launch_t<DK, __nv_bfloat16, false>(p, mq, mk, mv, s_in, s_out, O, G, g, Y, eps, zeta_v, vhm, status, st);
    return fuse ? launch_t<DK, float, true>(p, mq, mk, mv, s_in, s_out, O, G, g, Y, eps, zeta_v, vhm, status, st)
                : launch_t<DK, float, false>(p, mq, mk, mv, s_in, s_out, O, G, g, Y, eps, zeta_v, vhm, status, st);
}

}  // namespace

cudaError_t launch_chunkwise_ws(const Params &p, bool out_bf16, const void *Q, RowLayout q_layout,
                                const void *K, RowLayout k_layout, const void *V, RowLayout v_layout,
                                bool v_head_major, const float *s_in, float *s_out, void *O,
                                const void *G, RowLayout g_layout, void *Y, float eps,
                                bool zeta_on_v, bool rotate_in_loop, int *status,
                                cudaStream_t st, const float *acc_in, int acc_unturn) {
    CUtensorMap mq, mk, mv;
    const int bh = p.B * p.H;
    if (!make_tma_map_bf16_strided(&mq, Q, p.dk, p.L, bh, q_layout.row, q_layout.head, kC) ||
        !make_tma_map_bf16_strided(&mk, K, p.dk, p.L, bh, k_layout.row, k_layout.head, kC))
        return cudaErrorInvalidValue;
    const bool ok = v_head_major
                        ? make_tma_map_bf16_strided(&mv, V, p.dv, p.L, bh, v_layout.row, v_layout.head, kC)
                        : make_tma_map_bf16_strided(&mv, V, p.H * p.dv, p.L, p.B, v_layout.row,
                                                    v_layout.batch, kC);
    if (!ok) return cudaErrorInvalidValue;
    const int zv = zeta_on_v ? 1 : 0, vhm = v_head_major ? 1 : 0;
    if (p.dk == 256)
        return launch_dk<256>(p, out_bf16, mq, mk, mv, s_in, s_out, O, G, g_layout, Y, eps, zv, vhm, rotate_in_loop, status, st, acc_in, acc_unturn);
    if (p.dk == 64)
        return launch_dk<64>(p, out_bf16, mq, mk, mv, s_in, s_out, O, G, g_layout, Y, eps, zv, vhm, rotate_in_loop, status, st, acc_in, acc_unturn);
    return launch_dk<128>(p, out_bf16, mq, mk, mv, s_in, s_out, O, G, g_layout, Y, eps, zv, vhm, rotate_in_loop, status, st, acc_in, acc_unturn);
}

}  // namespace ret
