// chunkwise_tc.cu -- chunkwise retention on the sm_100a tensor cores, with
// an optional fused per-head GroupNorm + swish gate epilogue.
//
// "Retentive Network" paper summary, section 2.1, chunkwise recurrent form
// (3): parallel inside a chunk, a decayed state carried between chunks.  For
// the chunk of n rows after state R, with xPos-rotated rows q^_j, k^_j:
//   o_j = sum_{j'<=j} gamma^{j-j'} (q^_j.k^_j') v_j' + gamma^{j+1} q^_j R
//   R  <- gamma^n R + sum_j' gamma^{n-1-j'} k^_j'^T v_j'
// The kernel evaluates it in a rescaled form that leaves the tensor cores
// nothing but plain products:
//   K~   = diag(zeta) K^,           zeta_j  = gamma^{n-1-j}   (fused into the turn of K)
//   Rbar = bf16(gamma^n R)          (the decayed state, kept that way in TMEM)
//   O''  = Q^ Rbar + mask(Q^ K~^T) V         (mask: keep j' <= j)
//   o_j  = alpha_j O''_j,           alpha_j = gamma^{j+1-n}
//   R    <- gamma^n R + K~^T V
// which is the same sum term by term (gamma^{j+1-n} gamma^{n-1-j'} =
// gamma^{j-j'}, gamma^{j+1-n} gamma^n = gamma^{j+1}).  All factors stay in
// range while gamma^128 >= 2^-60; other decays use the CUDA-core kernel.
//
// One CTA owns one (b, h) and a 128-column slice of V and walks the chunks
// in order.  Tensor memory (512 columns): S [128 x 128] (P, the bf16 mask
// of S, overwrites half of it and feeds the P V product as the A operand),
// O'' [128 x 128], and the fp32 state slice transposed, R^T [128 x d_k]
// (lanes are V columns).  Shared memory: TMA-loaded Q^, K~, V tiles
// (128-byte swizzle), with K~ and Rbar^T interleaved per 64-column block.
// Per chunk, thread 0 issues S = Q^ K~^T, then O'' = Q^ Rbar (the P pass
// runs on S meanwhile), then O'' += P V and R^T += V^T K~; every buffer is
// reloaded as soon as the last product that reads it completes, and the
// next chunk's tiles are prefetched into L2 a chunk ahead.  Q^ and K~ come
// prepared from the streaming pass (prep.cu) when the caller provides room
// for them; otherwise the two thread groups turn them in shared memory.
//
// Fused epilogue (Y = swish(G) (.) GroupNorm_h(O)): the CTAs of one head
// form a cluster along d_v; each reduces its 128 columns of a row to a mean
// and centred sum of squares, the partials are exchanged through
// distributed shared memory and merged (Chan's pairwise update), and every
// CTA normalises and gates its own columns.  The G tile lands in the Q^
// blocks 0,1 (free once the O'' product is done; the next chunk's blocks
// 0,1 are loaded after the gate pass), the gate factors are computed into
// registers between arriving at the exchange barrier and waiting on it, and
// Y leaves through the V tile and a TMA store.
//
// Every mbarrier wait is bounded: on expiry the kernel latches
// RET_ERR_TIMEOUT in the device status word and every thread skips the
// remaining work together (cluster barriers still run, so no CTA of a
// cluster is left waiting), in-flight copies and MMAs get a bounded drain,
// and TMEM is freed.
#include <cuda.h>

#include <algorithm>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "launch.h"
#include "tc_util.cuh"

namespace ret {
namespace {

using namespace tc;

constexpr int kC = 128;       // chunk rows (MMA M)
constexpr int kTV = 128;      // value columns per CTA (MMA N)
constexpr int kThreads = 512;
constexpr int kGroup = 256;   // two groups of two warpgroups
constexpr int kMaxCluster = kMaxDv / kTV;
constexpr long long kTimeoutCycles = 4000000000LL;  // about 2 s
constexpr float kMinLog2GammaTimesC = -60.f;        // gamma^C >= 2^-60

// Q^ arrives in two parts, blocks 0,1 (BQL) and the rest (BQH; d_k 256
// only), so that the S product can start on the part that lands first.
// BSS: S done (the P pass may start); BS: S and the Q^ Rbar part done.
enum { BQL = 0, BQH, BK, BV, BSS, BS, BU, BPV, BG, kNumBars };

template <int DK>
struct Layout {
    static constexpr uint32_t kQ = 0;                    // Q^: DK/64 blocks of 16 KB
    static constexpr uint32_t kQBytes = kC * DK * 2;
    // K^ and the bf16 state copy Rbar^T interleaved per 64-column block, so
    // that [K^ ; Rbar^T] is one 256-row K-major B operand of the S|X product:
    // block kb = [K^ rows 0..127 | Rbar^T rows (v columns) 0..127], 32 KB.
    static constexpr uint32_t kKR = kQ + kQBytes;
    static constexpr uint32_t kKRBytes = 2 * kC * DK * 2;
    static constexpr uint32_t kV = kKR + kKRBytes;       // V (then V'): 2 blocks of 16 KB
    static constexpr uint32_t kVBytes = kC * kTV * 2;
    static constexpr uint32_t kSmall = kV + kVBytes;
    static constexpr uint32_t kBar = kSmall;             // kNumBars mbarriers
    static constexpr uint32_t kTmemSlot = kSmall + 96;
    static constexpr uint32_t kAbort = kSmall + 100;
    // GroupNorm: this CTA's per-row (mean, centred sum of squares) of its
    // 128 columns, double-buffered by chunk parity; peers read it remotely.
    static constexpr uint32_t kGnOwn = kSmall + 128;     // [2][128] float2
    static constexpr uint32_t kBytes = kGnOwn + 2 * 128 * 8;
    static __device__ __forceinline__ uint32_t k_blk(int kb) { return kKR + kb * 32768; }
    static __device__ __forceinline__ uint32_t rbar_blk(int kb) { return kKR + kb * 32768 + 16384; }
};

// S = Q^ K~^T and O'' = Q^ Rbar : A Q^ (K-major), B 128 rows of K~ or of
// Rbar^T (K-major)
constexpr uint32_t kIdescSX = idesc_bf16(128, 128, 0, 0);
// O'' += P V' : A P from tensor memory, B V' (MN-major)
constexpr uint32_t kIdescPV = idesc_bf16(128, kTV, 0, 1);

__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                         int *status) {
    return mbar_wait_bounded(bar, parity, abort_flag, status, kTimeoutCycles);
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&v);
}

__device__ __forceinline__ float2 unpack_bf16(uint32_t u) {
    return __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&u));
}

// a bf16 pair as a packed fp32 pair (lo, hi): the bf16 bits are the top
// half of each fp32
__device__ __forceinline__ uint64_t bf16x2_to_f2(uint32_t u) {
    return (static_cast<uint64_t>(u & 0xffff0000u) << 32) | (u << 16);
}

__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

__device__ __forceinline__ uint64_t f2_of(const uint32_t *r) {
    return (static_cast<uint64_t>(r[1]) << 32) | r[0];
}

// Row c of Rbar^T (K-major, 128-byte swizzle, inside the interleaved K^ /
// Rbar^T blocks): the 32 values of d-columns [d0, d0+32).
template <int DK>
__device__ __forceinline__ void st_rbarT_row32(uint8_t *smem, int c, int d0, const float *v) {
    uint8_t *blk = smem + Layout<DK>::rbar_blk(d0 >> 6) + c * 128;
    const int ch0 = (d0 & 63) >> 3;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint4 w;
        w.x = pack_bf16(v[8 * q + 0], v[8 * q + 1]);
        w.y = pack_bf16(v[8 * q + 2], v[8 * q + 3]);
        w.z = pack_bf16(v[8 * q + 4], v[8 * q + 5]);
        w.w = pack_bf16(v[8 * q + 6], v[8 * q + 7]);
        *reinterpret_cast<uint4 *>(blk + (((ch0 + q) ^ (c & 7)) << 4)) = w;
    }
}

template <typename T>
__device__ __forceinline__ void st_row32(T *dst, const float *v);
template <>
__device__ __forceinline__ void st_row32<float>(float *dst, const float *v) {
#pragma unroll
    for (int i = 0; i < 32; i += 4)
        *reinterpret_cast<float4 *>(dst + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
}
template <>
__device__ __forceinline__ void st_row32<__nv_bfloat16>(__nv_bfloat16 *dst, const float *v) {
#pragma unroll
    for (int i = 0; i < 32; i += 8) {
        uint4 w;
        w.x = pack_bf16(v[i + 0], v[i + 1]);
        w.y = pack_bf16(v[i + 2], v[i + 3]);
        w.z = pack_bf16(v[i + 4], v[i + 5]);
        w.w = pack_bf16(v[i + 6], v[i + 7]);
        *reinterpret_cast<uint4 *>(dst + i) = w;
    }
}

// swish(g) = g sigmoid(g) = h + h tanh(h), h = g / 2, for a bf16 pair:
// halving is exact, the hardware's bf16x2 tanh approximation is the one
// special-function operation, and a fused multiply-add rounds the result
// once to bf16.  The gate factor then carries a relative error of a few
// bf16 units, next to the one rounding of Y itself to bf16.
__device__ __forceinline__ uint32_t swish_bf16x2(uint32_t g) {
    uint32_t h, t, s;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(h) : "r"(g), "r"(0x3f003f00u));  // (0.5, 0.5)
    asm("tanh.approx.bf16x2 %0, %1;" : "=r"(t) : "r"(h));
    asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(s) : "r"(h), "r"(t), "r"(h));
    return s;
}

template <int DK, typename TO, bool FUSE>
__global__ void __launch_bounds__(kThreads, 1)
chunkwise_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                    const __grid_constant__ CUtensorMap tmY, const __grid_constant__ CUtensorMap tmG,
                    const Params p,
                    const float *__restrict__ state_in, float *__restrict__ state_out,
                    TO *__restrict__ O, const __nv_bfloat16 *__restrict__ G, TO *__restrict__ Y,
                    float gn_eps, int pre, int v_head_major, int *status) {
    using Ly = Layout<DK>;
    constexpr int KB = DK / 64;         // 64-column blocks of Q^, K~, Rbar^T
    constexpr int KHI = KB - 2;         // Q^ blocks outside the staging area
    constexpr int NCH = DK / 8;         // 16-byte chunks per Q/K row
    constexpr int RGA = DK / 64;        // 32-column groups per thread in the state pass (group A)
    constexpr uint32_t kIdescU = idesc_bf16(128, DK, 1, 1);  // R^T += V^T K~ (both MN-major)
    constexpr bool kStage = sizeof(TO) == 2;  // bf16 Y tiles leave by TMA store (O: always)
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t sbase = smem_u32(smem);
    const int tid = threadIdx.x, warp = tid >> 5;
    const int wg = tid >> 7;        // warpgroup 0..3; each covers all 128 TMEM lanes
    const int row = tid & 127;      // TMEM lane: chunk row for S/O, V column for R^T
    const int grp = tid >> 8;       // 0: state pass and Q (warpgroups 0,1); 1: output and K (2,3)
    const int gtid = tid & 255;     // thread index within the group
    const int gwg = wg & 1;         // warpgroup within the group
    const int bh = blockIdx.y, h = bh % p.H, b = bh / p.H;
    const int v0 = blockIdx.x * kTV;
    const float lg = p.log2g[h];
    const int L = p.L, dv = p.dv;
    const int nchunks = (L + kC - 1) / kC;

    if (sbase & 1023u) {  // swizzle atoms need 1024-byte alignment (same for every CTA)
        if (tid == 0) atomicExch(status, (int)RET_ERR_CUDA);
        return;
    }
    auto bar = [&](int i) { return sbase + Ly::kBar + 8u * i; };
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Ly::kAbort);

    if (tid == 0) {
        for (int i = 0; i < kNumBars; ++i) mbar_init(bar(i), 1);
        *abort_flag = 0;
        fence_mbar_init();
        fence_proxy_async_smem();
    }
    if (warp == 0) {
        tmem_alloc(sbase + Ly::kTmemSlot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + Ly::kTmemSlot);
    const uint32_t tS = tmem, tO = tmem + 128, tR = tmem + 256;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;

    // Q^ blocks 0,1 (BQL) and the rest (BQH)
    auto load_q_lo = [&](int c) {
        mbar_expect_tx(bar(BQL), 2 * 16384);
        for (int kb = 0; kb < 2; ++kb)
            tma_load_3d(sbase + Ly::kQ + kb * 16384, &tmQ, bar(BQL), kb * 64, c * kC, bh);
    };
    auto load_q_hi = [&](int c) {
        if constexpr (KHI > 0) {
            mbar_expect_tx(bar(BQH), KHI * 16384);
            for (int kb = 2; kb < KB; ++kb)
                tma_load_3d(sbase + Ly::kQ + kb * 16384, &tmQ, bar(BQH), kb * 64, c * kC, bh);
        }
    };
    auto load_k = [&](int c) {
        mbar_expect_tx(bar(BK), Ly::kQBytes);
        for (int kb = 0; kb < KB; ++kb)
            tma_load_3d(sbase + Ly::k_blk(kb), &tmK, bar(BK), kb * 64, c * kC, bh);
    };
    // V as [B][H][L][d_v] (head-major) or as rows of H*d_v columns, like G
    const int vx0 = v_head_major ? v0 : h * dv + v0, vz = v_head_major ? bh : b;
    auto load_v = [&](int c) {
        mbar_expect_tx(bar(BV), Ly::kVBytes);
        for (int nb = 0; nb < 2; ++nb)
            tma_load_3d(sbase + Ly::kV + nb * 16384, &tmV, bar(BV), vx0 + nb * 64, c * kC, vz);
    };
    // the G tile of chunk c into the Q^ blocks 0,1 (free once the O''
    // product is done; the next chunk's blocks 0,1 follow the gate pass)
    auto load_g = [&](int c) {
        mbar_expect_tx(bar(BG), Ly::kVBytes);
        for (int nb = 0; nb < 2; ++nb)
            tma_load_3d(sbase + Ly::kQ + nb * 16384, &tmG, bar(BG), h * dv + v0 + nb * 64, c * kC, b);
    };
    // every tile chunk c will load, into L2 ahead of time (the Q^ and K~
    // blocks, which every CTA of the head loads, shared out among them)
    auto prefetch = [&](int c) {
        for (int kb = blockIdx.x; kb < KB; kb += gridDim.x) {
            tma_prefetch_3d(&tmQ, kb * 64, c * kC, bh);
            tma_prefetch_3d(&tmK, kb * 64, c * kC, bh);
        }
        for (int nb = 0; nb < 2; ++nb) {
            tma_prefetch_3d(&tmV, vx0 + nb * 64, c * kC, vz);
            if constexpr (FUSE) tma_prefetch_3d(&tmG, h * dv + v0 + nb * 64, c * kC, b);
        }
    };
    auto sync_alive = [&]() {
        __syncthreads();
        return *abort_flag == 0;
    };
    // group-local barrier (hardware barriers 1 and 2) and abort check
    auto gsync_alive = [&]() {
        named_sync(1 + grp, kGroup);
        return *abort_flag == 0;
    };
    const bool g_leader = gtid == 0;   // waits on mbarriers for its group

    // Turn (and for K~ scale by gamma^{n-1-r}) rows of the tile at blk0 with
    // `nthr` threads, this one being `ti`: thread -> 16-byte column chunk
    // (4 pairs) and the rows r0, r0+RS, r0+2RS, ... taken two at a time, the
    // two rows in the lanes of packed fp32 pairs.  Angles start exact (fp64
    // reduction) and advance by 2*RS*theta_j per step.
    auto rotate = [&](uint32_t blk0, uint32_t blk_stride, int c, int n, bool zeta, int ti, int nthr) {
        const int RS = nthr / NCH;
        const int c16 = ti % NCH, r0 = ti / NCH;
        const int blk = c16 >> 3, cw = c16 & 7;
        uint8_t *base = smem + blk0 + blk * blk_stride;
        uint64_t C[4], NS[4], c2[4], s2[4], ns2[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const double th = p.theta[c16 * 4 + e];
            float ca, sa, cb, sb, cs, ss;
            rot_cs_fast(p.pos_offset + (long long)c * kC + r0, th, &ca, &sa);
            rot_cs_fast(p.pos_offset + (long long)c * kC + r0 + RS, th, &cb, &sb);
            rot_cs_fast(2 * RS, th, &cs, &ss);
            C[e] = f2_make(ca, cb);
            NS[e] = f2_make(-sa, -sb);
            c2[e] = f2_make(cs, cs);
            s2[e] = f2_make(ss, ss);
            ns2[e] = f2_make(-ss, -ss);
        }
        // two row pairs per step: all four rows are loaded before any is written
        auto turn_pair = [&](uint4 &wa, uint4 &wb, int ra, int rb) {
            const float za = zeta ? (ra < n ? decay_pow(lg, n - 1 - ra) : 0.f) : 1.f;
            const float zb = zeta ? (rb < n ? decay_pow(lg, n - 1 - rb) : 0.f) : 1.f;
            const uint64_t Z = f2_make(za, zb);
            uint32_t *ua = reinterpret_cast<uint32_t *>(&wa);
            uint32_t *ub = reinterpret_cast<uint32_t *>(&wb);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                // x0 = low bf16, x1 = high bf16 of each row's pair
                const uint64_t X0 = (static_cast<uint64_t>(ub[e] << 16) << 32) | (ua[e] << 16);
                const uint64_t X1 = (static_cast<uint64_t>(ub[e] & 0xffff0000u) << 32) | (ua[e] & 0xffff0000u);
                const uint64_t NX0 = X0 ^ 0x8000000080000000ull;
                const uint64_t ZC = zeta ? f2_mul(C[e], Z) : C[e];
                const uint64_t ZNS = zeta ? f2_mul(NS[e], Z) : NS[e];
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
        // rows r0 + RS*k, k = 0..128/RS-1 (a multiple of 4); rows at or past n
        // are zeros from the load and are left as they are
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
    };
    // K~ = diag(zeta) K^ without rotation, `nthr` threads, this one `ti`
    auto scale_k = [&](int n, int ti, int nthr) {
        const int r = ti & 127;
        const float zeta = r < n ? decay_pow(lg, n - 1 - r) : 0.f;
#pragma unroll 1
        for (int kb = ti >> 7; kb < KB; kb += nthr >> 7) {
            uint8_t *krow = smem + Ly::k_blk(kb) + r * 128;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                uint4 *ptr = reinterpret_cast<uint4 *>(krow + (((q + r) & 7) << 4));
                uint4 w = *ptr;
                uint32_t *u = reinterpret_cast<uint32_t *>(&w);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 x = unpack_bf16(u[e]);
                    u[e] = pack_bf16(x.x * zeta, x.y * zeta);
                }
                *ptr = w;
            }
        }
    };
    auto prep_q = [&](int c, int n, int ti, int nthr) {
        if (p.rotate) rotate(Ly::kQ, 16384, c, n, false, ti, nthr);
    };
    auto prep_k = [&](int c, int n, int ti, int nthr) {
        if (p.rotate)
            rotate(Ly::kKR, 32768, c, n, true, ti, nthr);
        else
            scale_k(n, ti, nthr);
    };
    // MMA descriptors: fixed buffers, so only the start address moves
    const uint64_t dQ = sdesc_sw128(sbase + Ly::kQ, 16, 1024);          // A of [S|O''], K-major
    const uint64_t dKR = sdesc_sw128(sbase + Ly::kKR, 16, 1024);        // B of [S|O''], K-major
    const uint64_t dVa = sdesc_sw128(sbase + Ly::kV, 16384, 1024);      // A of R^T update, MN-major
    const uint64_t dKb = sdesc_sw128(sbase + Ly::kKR, 32768, 1024);     // B of R^T update, MN-major
    const uint64_t dVb = dVa;                                           // B of P V, MN-major

    if (tid == 0) {
        load_q_lo(0);
        load_q_hi(0);
        load_k(0);
        load_v(0);
        if constexpr (FUSE)
            for (int nb = 0; nb < 2; ++nb) tma_prefetch_3d(&tmG, h * dv + v0 + nb * 64, 0, b);
    }
    // Starting state: TMEM R^T = gamma^{n_0} S_in^T and Rbar^T = bf16 of the
    // same; zeros without a state (the S|X product then gives O'' = 0).
    const bool has_in = state_in != nullptr;
    {
        const float g0 = decay_pow(lg, min(kC, L));
        const int d_begin = wg * (DK / 4);
#pragma unroll 1
        for (int g = 0; g < DK / 128; ++g) {
            const int d0 = d_begin + 32 * g;
            float v[32];
            uint32_t r[32];
#pragma unroll
            for (int i = 0; i < 32; ++i)
                v[i] = has_in ? state_in[((size_t)bh * DK + d0 + i) * dv + v0 + row] * g0 : 0.f;
            st_rbarT_row32<DK>(smem, row, d0, v);
            if (has_in) {
#pragma unroll
                for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(v[i]);
                tmem_st32(tR + lane_base + d0, r);
            }
        }
        if (has_in) tmem_wait_st();
    }
    // chunk 0 (rows not prepared ahead): group A turns Q, group B prepares K~
    bool alive = true;
    if (!pre) {
        const int n0 = min(kC, L);
        if (g_leader) {
            if (grp == 0)
                (KHI == 0 || wait_bar(bar(BQH), 0, abort_flag, status)) &&
                    wait_bar(bar(BQL), 0, abort_flag, status);
            else
                wait_bar(bar(BK), 0, abort_flag, status);
        }
        alive = gsync_alive();
        if (alive) {
            if (grp == 0)
                prep_q(0, n0, gtid, kGroup);
            else
                prep_k(0, n0, gtid, kGroup);
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    alive = sync_alive();

#pragma unroll 1
    for (int c = 0; c < nchunks; ++c) {
        const uint32_t par = c & 1;  // every barrier completes once per chunk
        const int t0 = c * kC;
        const int n = min(kC, L - t0);
        const bool has_state = has_in || c > 0;
        const bool last = c + 1 == nchunks;
        const int n_next = last ? 0 : min(kC, L - t0 - kC);

        if (alive && tid == 32 && !last) prefetch(c + 1);  // off thread 0's path
        // V of this chunk, once the previous chunk's stores have read the V
        // tile (their last use of it; the products finished before the loop
        // barrier)
        if (alive && tid == kGroup && c > 0) {
            bulk_wait_read();
            load_v(c);
        }

        // ---- S = Q^ K~^T, then O'' = Q^ Rbar (thread 0; both over d_k in 16-
        // column steps: the Q^ blocks outside the staging area first, then
        // blocks 0,1, which may land later).  The P pass starts on S while
        // the tensor cores compute O''.
        if (alive && tid == 0) {
            bool ok = true;
            if (pre)  // prepared rows: nobody else has waited for the loads
                ok = (KHI == 0 || wait_bar(bar(BQH), par, abort_flag, status)) &&
                     wait_bar(bar(BK), par, abort_flag, status);
            tc_fence_after();
            // part 0: S (B = K~ rows), part 1: O'' (B = Rbar^T rows, 16 KB further)
            auto sx = [&](int part, int ks, bool acc) {
                const uint64_t off = (uint64_t)(((ks >> 2) * 16384 + (ks & 3) * 32) >> 4);
                const uint64_t offkr =
                    (uint64_t)(((ks >> 2) * 32768 + part * 16384 + (ks & 3) * 32) >> 4);
                mma_ss(part ? tO : tS, dQ + off, dKR + offkr, kIdescSX, acc ? 1u : 0u);
            };
            if (ok) {
#pragma unroll
                for (int ks = 8; ks < DK / 16; ++ks) sx(0, ks, ks > 8);
            }
            if (ok && pre) ok = wait_bar(bar(BQL), par, abort_flag, status);
            tc_fence_after();
            if (ok) {
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) sx(0, ks, KHI > 0 || ks > 0);
            }
            mma_commit(bar(BSS));
            if (ok) {
#pragma unroll
                for (int ks = 8; ks < DK / 16; ++ks) sx(1, ks, ks > 8);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) sx(1, ks, KHI > 0 || ks > 0);
            }
            mma_commit(bar(BS));
        }

        // ---- P = bf16(S) on j' <= j, else 0, into tensor memory, by warps
        // 1-15 as soon as S is done (warp 0 is still issuing the O'' product;
        // warp 4 also takes warp 0's lanes and keys); warp 0 meets them at
        // named barrier 4 before it issues P V.
        if (warp != 0) {
            if (alive && wait_bar(bar(BSS), par, abort_flag, status)) {
                tc_fence_after();
                // keys [c0, c0+32) of this warp's 32 lanes -> columns [c0, c0+16)
                auto mask_pack = [&](int c0) {
                    uint32_t a[32], pk[16];
                    tmem_ld32(tS + lane_base + c0, a);
                    tmem_wait_ld(a);
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int k0 = c0 + 2 * i;
                        pk[i] = pack_bf16(k0 <= row ? __uint_as_float(a[2 * i]) : 0.f,
                                          k0 + 1 <= row ? __uint_as_float(a[2 * i + 1]) : 0.f);
                    }
                    tmem_st16(tS + lane_base + c0, pk);
                };
                mask_pack(wg * 32);
                if (warp == 4) mask_pack(0);
                tmem_wait_st();
            }
            tc_fence_before();
            named_arrive(4, kThreads);
        } else {
            named_sync(4, kThreads);
        }
        alive = *abort_flag == 0;

        // Q^ and Rbar are no longer read once O'' is done: the next Q^ (with
        // the gate, G takes blocks 0,1 first), by thread 32 while thread 0
        // issues products
        if (alive && tid == 32 && wait_bar(bar(BS), par, abort_flag, status)) {
            if constexpr (FUSE) load_g(c);
            if (!last) {
                if constexpr (!FUSE) load_q_lo(c + 1);
                load_q_hi(c + 1);
            }
        }

        // ---- O'' += P V, then R^T += V^T K~ (the output pass starts first)
        if (alive && tid == 0 && wait_bar(bar(BV), par, abort_flag, status)) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < kC / 16; ++ks)
                mma_ts(tO, tS + (ks >> 1) * 32 + (ks & 1) * 8, dVb + (uint64_t)((ks * 2048) >> 4),
                       kIdescPV, 1u);
            mma_commit(bar(BPV));
#pragma unroll
            for (int ks = 0; ks < kC / 16; ++ks) {
                const uint64_t off = (uint64_t)((ks * 2048) >> 4);
                mma_ss(tR, dVa + off, dKb + off, kIdescU, (ks > 0 || has_state) ? 1u : 0u);
            }
            mma_commit(bar(BU));
        }

        if (grp == 0) {
            // ================= group A: state pass, then (rows not prepared) the next Q^
            if constexpr (FUSE) cluster_arrive();   // GroupNorm exchange barrier
            if (alive && tid == 0) {
                wait_bar(bar(BU), par, abort_flag, status);
                if (!last) load_k(c + 1);  // K~ is no longer read
            }
            alive = gsync_alive();
            tc_fence_after();
            if (alive) {
                const float gnext = last ? 1.f : decay_pow(lg, n_next);
                const int d_begin = gwg * (DK / 2);
                // R^T columns [d0, d0+32): decay, bf16 copy, back to TMEM; or state_out
                auto state32 = [&](uint32_t (&r)[32], int d0) {
                    float v[32];
                    const uint64_t G2 = f2_make(gnext, gnext);
#pragma unroll
                    for (int i = 0; i < 32; i += 2) {
                        const uint64_t x = f2_mul(f2_of(r + i), G2);
                        v[i] = f2_lo(x);
                        v[i + 1] = f2_hi(x);
                    }
                    if (last) {
                        if (state_out) {
#pragma unroll
                            for (int i = 0; i < 32; ++i)
                                state_out[((size_t)bh * DK + d0 + i) * dv + v0 + row] = v[i];
                        }
                    } else {
                        st_rbarT_row32<DK>(smem, row, d0, v);
#pragma unroll
                        for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(v[i]);
                        tmem_st32(tR + lane_base + d0, r);
                    }
                };
#pragma unroll 1
                for (int g = 0; g < RGA; g += 2) {
                    uint32_t ra[32], rb[32];
                    tmem_ld32(tR + lane_base + d_begin + 32 * g, ra);
                    tmem_ld32(tR + lane_base + d_begin + 32 * g + 32, rb);
                    tmem_wait_ld(ra);
                    tmem_wait_ld(rb);
                    state32(ra, d_begin + 32 * g);
                    state32(rb, d_begin + 32 * g + 32);
                }
                tmem_wait_st();
            }
            if (!pre) {
                if (alive && !last && g_leader)
                    (KHI == 0 || wait_bar(bar(BQH), par ^ 1, abort_flag, status)) &&
                        wait_bar(bar(BQL), par ^ 1, abort_flag, status);
                alive = gsync_alive();
                if (alive && !last) prep_q(c + 1, n_next, gtid, kGroup);
            }
            if constexpr (FUSE) cluster_wait();
        } else {
            // ================= group B: output (then, without prepared rows, the next K~)
            const int o0 = gwg * 64;   // this thread's 64 columns of the row, 32 at a time
            const size_t grow =
                ((size_t)b * L + t0 + row) * ((size_t)p.H * dv) + (size_t)h * dv + v0 + o0;
            // every thread observes the barriers it depends on itself: a
            // completed phase orders its own reads, no group barrier needed
            if (alive) alive = wait_bar(bar(BPV), par, abort_flag, status);
            tc_fence_after();
            const float alpha = exp2f((float)(row + 1 - n) * lg);  // gamma^{row+1-n}; lg finite
            // 32 columns of O'' (still in tensor memory until this iteration ends)
            auto ld_o = [&](int half, float *x) {
                uint32_t a[32];
                tmem_ld32(tO + lane_base + o0 + 32 * half, a);
                tmem_wait_ld(a);
#pragma unroll
                for (int i = 0; i < 32; ++i) x[i] = __uint_as_float(a[i]);
            };
            // bf16 tiles leave through the V tile (not read again this chunk
            // once the state update is done) and a TMA store; rows past the
            // sequence end are clipped.  The last store of a chunk is not
            // waited for here: the next chunk's V load waits for its read.
            auto stage32 = [&](int half, const float *vals) {
                uint8_t *dst = smem + Ly::kV + gwg * 16384 + row * 128;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint4 w;
                    w.x = pack_bf16(vals[8 * q + 0], vals[8 * q + 1]);
                    w.y = pack_bf16(vals[8 * q + 2], vals[8 * q + 3]);
                    w.z = pack_bf16(vals[8 * q + 4], vals[8 * q + 5]);
                    w.w = pack_bf16(vals[8 * q + 6], vals[8 * q + 7]);
                    *reinterpret_cast<uint4 *>(dst + (((4 * half + q) ^ (row & 7)) << 4)) = w;
                }
            };
            auto store_tile = [&](const CUtensorMap *map, int x0, int y0, int z0, bool restage) {
                fence_proxy_async_smem();
                named_sync(2, kGroup);
                if (g_leader) {
                    tma_store_3d(map, sbase + Ly::kV, x0, y0, z0);
                    tma_store_3d(map, sbase + Ly::kV + 16384, x0 + 64, y0, z0);
                    bulk_commit();
                    if (restage) bulk_wait_read();
                }
                if (restage) named_sync(2, kGroup);
            };
            // O = alpha O'' (staged tile or direct stores)
            auto emit_o = [&]() {
                if constexpr (sizeof(TO) == 2) {
#pragma unroll 1
                    for (int half = 0; half < 2; ++half) {
                        float x[32];
                        ld_o(half, x);
#pragma unroll
                        for (int i = 0; i < 32; ++i) x[i] *= alpha;
                        stage32(half, x);
                    }
                    store_tile(&tmO, v0, t0, bh, false);
                } else {
                    // fp32: two rounds of 32 columns per warpgroup (128-byte
                    // rows, one 16 KB box per warpgroup) through the V tile
#pragma unroll 1
                    for (int half = 0; half < 2; ++half) {
                        float x[32];
                        ld_o(half, x);
                        uint8_t *dst = smem + Ly::kV + gwg * 16384 + row * 128;
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            *reinterpret_cast<float4 *>(dst + ((q ^ (row & 7)) << 4)) =
                                make_float4(x[4 * q] * alpha, x[4 * q + 1] * alpha,
                                            x[4 * q + 2] * alpha, x[4 * q + 3] * alpha);
                        fence_proxy_async_smem();
                        named_sync(2, kGroup);
                        if (g_leader) {
                            tma_store_3d(&tmO, sbase + Ly::kV, v0 + 32 * half, t0, bh);
                            tma_store_3d(&tmO, sbase + Ly::kV + 16384, v0 + 64 + 32 * half, t0, bh);
                            bulk_commit();
                            if (half == 0) bulk_wait_read();
                        }
                        if (half == 0) named_sync(2, kGroup);
                    }
                }
            };
            // the products have read V (the state update is the last)
            auto v_free = [&]() {
                if (alive) alive = wait_bar(bar(BU), par, abort_flag, status);
            };
            if constexpr (!FUSE) {
                v_free();
                if (alive) emit_o();
            } else {
                const int nr = (int)gridDim.x;        // CTAs of this head = cluster size
                // Mean and centred sum of squares of this thread's 64 columns
                // in one pass, shifted by its first value (no cancellation
                // unless the mean sits many deviations from that sample);
                // even and odd columns in the two lanes of packed fp32 pairs.
                uint64_t S1 = 0, S2 = 0;
                float shift = 0.f;
                if (alive) {
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        uint32_t a[32];
                        tmem_ld32(tO + lane_base + o0 + 32 * half, a);
                        tmem_wait_ld(a);
                        if (half == 0) shift = __uint_as_float(a[0]);
                        const uint64_t NSH = f2_make(-shift, -shift);
#pragma unroll
                        for (int i = 0; i < 32; i += 2) {
                            const uint64_t d = f2_add(f2_of(a + i), NSH);
                            S1 = f2_add(S1, d);
                            S2 = f2_fma(d, d, S2);
                        }
                    }
                }
                const float s1 = f2_lo(S1) + f2_hi(S1), s2 = f2_lo(S2) + f2_hi(S2);
                const float m_w = shift + s1 * (1.f / 64.f);
                const float m2_w = fmaxf(s2 - s1 * s1 * (1.f / 64.f), 0.f);
                // The two warpgroups' halves merge (Chan's pairwise update,
                // equal counts) in this CTA's published slot; the peers read
                // it after the cluster barrier (double buffer by chunk parity:
                // a peer is never more than one chunk behind, the barrier sees
                // to that).
                const uint32_t own = sbase + Ly::kGnOwn + (par * 128 + row) * 8;
                float2 *slot = reinterpret_cast<float2 *>(smem + Ly::kGnOwn + (par * 128 + row) * 8);
                if (gwg == 1) *slot = make_float2(m_w, m2_w);
                named_sync(2, kGroup);
                if (gwg == 0) {
                    const float2 o = *slot;
                    const float d = m_w - o.x;
                    *slot = make_float2(0.5f * (m_w + o.x), m2_w + o.y + 32.f * d * d);
                }
                // swish(G) of this thread's 64 columns (bf16 pairs in
                // registers) from the G tile in the Q^ blocks 0,1 while the
                // peers reach the exchange barrier
                cluster_arrive();
                uint32_t sw[32];
                if (alive) alive = wait_bar(bar(BG), par, abort_flag, status);
                if (alive) {
                    const uint8_t *gt = smem + Ly::kQ + gwg * 16384 + row * 128;
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const uint4 w = *reinterpret_cast<const uint4 *>(gt + ((q ^ (row & 7)) << 4));
                        sw[4 * q + 0] = swish_bf16x2(w.x);
                        sw[4 * q + 1] = swish_bf16x2(w.y);
                        sw[4 * q + 2] = swish_bf16x2(w.z);
                        sw[4 * q + 3] = swish_bf16x2(w.w);
                    }
                }
                // the whole group has read G: the next Q^ blocks 0,1
                alive = gsync_alive();
                if (alive && g_leader && !last) load_q_lo(c + 1);
                cluster_wait();
                // the peers' partials (distributed shared memory), in flight
                // while the group waits for the products to release V
                float2 e[kMaxCluster];
                if (alive) {
#pragma unroll
                    for (int r = 0; r < kMaxCluster; ++r)
                        if (r < nr) e[r] = ld_cluster_f32x2(map_to_rank(own, r));
                }
                v_free();
                if (alive) {
                    uint32_t a[32];
                    tmem_ld32(tO + lane_base + o0, a);
                    float mean = 0.f, m2 = 0.f;
#pragma unroll
                    for (int r = 0; r < kMaxCluster; ++r)
                        if (r < nr) mean += e[r].x;
                    mean /= (float)nr;
#pragma unroll
                    for (int r = 0; r < kMaxCluster; ++r)
                        if (r < nr) m2 += e[r].y + (float)kTV * (e[r].x - mean) * (e[r].x - mean);
                    const float var = m2 / (float)(nr * kTV);  // of O'' ; O = alpha O''
                    const float scale = alpha * rsqrtf(alpha * alpha * var + gn_eps);
                    // (x - mean) scale as one fused multiply-add per pair
                    const uint64_t SC = f2_make(scale, scale);
                    const uint64_t NMS = f2_make(-mean * scale, -mean * scale);
                    // Y into the V tile
                    uint8_t *tile = smem + Ly::kV + gwg * 16384 + row * 128;
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        if (half == 1) tmem_ld32(tO + lane_base + o0 + 32, a);
                        tmem_wait_ld(a);
                        float x[32];
#pragma unroll
                        for (int k = 0; k < 16; ++k) {
                            const uint64_t y = f2_mul(f2_fma(f2_of(a + 2 * k), SC, NMS),
                                                      bf16x2_to_f2(sw[16 * half + k]));
                            x[2 * k] = f2_lo(y);
                            x[2 * k + 1] = f2_hi(y);
                        }
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            if constexpr (kStage) {
                                uint4 w;
                                w.x = pack_bf16(x[8 * q + 0], x[8 * q + 1]);
                                w.y = pack_bf16(x[8 * q + 2], x[8 * q + 3]);
                                w.z = pack_bf16(x[8 * q + 4], x[8 * q + 5]);
                                w.w = pack_bf16(x[8 * q + 6], x[8 * q + 7]);
                                *reinterpret_cast<uint4 *>(tile + (((4 * half + q) ^ (row & 7)) << 4)) = w;
                            }
                        }
                        if constexpr (!kStage)
                            if (row < n) st_row32<TO>(Y + grow + 32 * half, x);
                    }
                    if constexpr (kStage) store_tile(&tmY, h * dv + v0, t0, b, O != nullptr);
                    if (O) emit_o();
                }
            }
            if (!pre) {
                if (alive && g_leader && !last) wait_bar(bar(BK), par ^ 1, abort_flag, status);
                alive = gsync_alive();
                if (alive && !last) prep_k(c + 1, n_next, gtid, kGroup);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        alive = *abort_flag == 0;
    }

    if (tid == 0 || tid == kGroup) bulk_wait_all();  // output stores in flight
    if constexpr (FUSE) cluster_sync();  // peers may still write into this CTA's smem before it
    // After an abort, copies and MMAs still in flight get a bounded time to
    // land before the shared and tensor memory are released.
    if (tid == 0 && *abort_flag) {
        const long long start = clock64();
        while (clock64() - start < 20000000LL) __nanosleep(1000);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ------------------------------------------------------------------ host side
// G (and V when not head-major) are read as rows of H*d_v columns with the
// row / batch strides of `g` (the C ABI's [B][L][H*d_v] has H*d_v and
// L*H*d_v); the head stride does not apply to them.
struct Views {
    int v_head_major;
    RowLayout g;
};

template <int DK, typename TO, bool FUSE>
cudaError_t launch_t(const Params &p, const CUtensorMap &mq, const CUtensorMap &mk,
                     const CUtensorMap &mv, const float *s_in, float *s_out, void *O,
                     const void *G, void *Y, float eps, int pre, const Views &vw, int *status,
                     cudaStream_t st) {
    CUtensorMap mo, my, mg;
    std::memset(&mo, 0, sizeof(mo));
    std::memset(&my, 0, sizeof(my));
    std::memset(&mg, 0, sizeof(mg));
    if (sizeof(TO) == 2) {
        if (O && !make_tma_map_bf16(&mo, O, p.dv, p.L, p.B * p.H, kC)) return cudaErrorInvalidValue;
        if (Y && !make_tma_map_bf16(&my, Y, p.H * p.dv, p.L, p.B, kC)) return cudaErrorInvalidValue;
    } else if (O && !make_tma_map_f32(&mo, O, p.dv, p.L, p.B * p.H, kC)) {
        return cudaErrorInvalidValue;
    }
    if (G && !make_tma_map_bf16_strided(&mg, G, p.H * p.dv, p.L, p.B, vw.g.row, vw.g.batch, kC))
        return cudaErrorInvalidValue;
    auto kern = chunkwise_tc_kernel<DK, TO, FUSE>;
    const int smem = (int)Layout<DK>::kBytes;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.dv / kTV, p.B * p.H);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = FUSE ? p.dv / kTV : 1;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, mq, mk, mv, mo, my, mg, p, s_in, s_out, (TO *)O,
                           (const __nv_bfloat16 *)G, (TO *)Y, eps, pre, vw.v_head_major, status);
    if (e == cudaSuccess) note_launches(1);
    return e;
}

template <int DK>
cudaError_t launch_dk(const Params &p, bool out_bf16, const CUtensorMap &mq, const CUtensorMap &mk,
                      const CUtensorMap &mv, const float *s_in, float *s_out, void *O,
                      const void *G, void *Y, float eps, int pre, const Views &vw, int *status,
                      cudaStream_t st) {
    const bool fuse = Y != nullptr;
    if (out_bf16)
        return fuse ? launch_t<DK, __nv_bfloat16, true>(p, mq, mk, mv, s_in, s_out, O, G, Y, eps, pre, vw, status, st)
                    : launch_t<DK, __nv_bfloat16, false>(p, mq, mk, mv, s_in, s_out, O, G, Y, eps, pre, vw, status, st);
    return fuse ? launch_t<DK, float, true>(p, mq, mk, mv, s_in, s_out, O, G, Y, eps, pre, vw, status, st)
                : launch_t<DK, float, false>(p, mq, mk, mv, s_in, s_out, O, G, Y, eps, pre, vw, status, st);
}

}  // namespace

// The loop works in blocks of kC rows whatever the chunk: a chunk of
// kC * m rows is m consecutive blocks, and a chunk of 64 rows pairs up two
// chunks per block.  The chunkwise recurrence holds exactly at any row
// boundary (the state carried between blocks is the exact state after
// those rows), so either is the same computation; only the rounding
// differs.  d_k 64, d_v 64 and chunks of 64 rows are served by the
// pipelined kernel of chunkwise_ws.cu only: with rotation they need the
// streaming pass's workspace (chunkwise_tc_needs_prep).
bool chunkwise_tc_supported(const Params &p, int chunk, bool in_bf16) {
    const bool dk_ok = p.dk == 64 || p.dk == 128 || p.dk == 256;
    const bool dv_ok = p.dv == 64 || (p.dv % kTV == 0 && p.dv / kTV <= kMaxCluster);
    if (!in_bf16 || chunk % 64 != 0 || !dk_ok || !dv_ok || p.L < 1 || p.B * p.H < 1 ||
        (long long)p.B * p.H > 65535)
        return false;
    for (int h = 0; h < p.H; ++h)
        if (!(p.log2g[h] * kC >= kMinLog2GammaTimesC)) return false;  // also rejects gamma = 0
    return true;
}

bool chunkwise_tc_needs_prep(const Params &p, int chunk) {
    return p.rotate && (p.dk == 64 || p.dv == 64 || chunk % kC != 0);
}

namespace {

// The chunk loop on rows that are ready: prepared by the streaming pass
// (`pre`, the key rows carry their weight) or, without rotation and
// without a workspace for that pass, Q and K as they are (the loop then
// weights the value rows in shared memory, which measured slower than the
// pass).  Both run on the pipelined kernel of chunkwise_ws.cu; rotated rows
// that nobody prepared go to the kernel below, which turns them itself.
cudaError_t launch_tc_rows(const Params &p, bool out_bf16, const void *Q, const void *K,
                           const void *V, const float *s_in, float *s_out, void *O, const void *G,
                           void *Y, float eps, int pre, int *status, cudaStream_t st) {
    if (pre || !p.rotate) {
        const RowLayout hm = bhld_layout(p, p.dk), vl = bhld_layout(p, p.dv);
        // G [B][L][H d_v] of the real heads (segment heads: H = real heads x
        // seg_heads, L = rows of one segment; the batch stride is the same)
        const RowLayout gl{(long long)(p.H / p.seg_heads) * p.dv, 0, (long long)p.L * p.H * p.dv};
        return launch_chunkwise_ws(p, out_bf16, Q, hm, K, V, vl, true, s_in, s_out, O, G, gl, Y,
                                   eps, !pre, status, st);
    }
    CUtensorMap mq, mk, mv;
    const int bh = p.B * p.H;
    if (!make_tma_map_bf16(&mq, Q, p.dk, p.L, bh, kC) || !make_tma_map_bf16(&mk, K, p.dk, p.L, bh, kC) ||
        !make_tma_map_bf16(&mv, V, p.dv, p.L, bh, kC))
        return cudaErrorInvalidValue;
    const Views vw{1, RowLayout{(long long)p.H * p.dv, 0, (long long)p.L * p.H * p.dv}};
    if (p.dk == 256) return launch_dk<256>(p, out_bf16, mq, mk, mv, s_in, s_out, O, G, Y, eps, pre, vw, status, st);
    return launch_dk<128>(p, out_bf16, mq, mk, mv, s_in, s_out, O, G, Y, eps, pre, vw, status, st);
}

// A second stream per device on which the streaming pass of the next batch
// slice runs while the chunk loop of the current one holds the SMs, and the
// two events that join it to the caller's stream.  Made once; the lock
// keeps the enqueue sequences of concurrent callers apart.
struct SideStream {
    std::mutex mu;
    bool made = false, ok = false;
    cudaStream_t s = nullptr;
    cudaEvent_t start = nullptr, ready = nullptr;
    int sms = 0;
};
constexpr int kMaxDevices = 64;
SideStream g_side[kMaxDevices];

SideStream *side_stream() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return nullptr;
    }
    SideStream &ss = g_side[dev];
    std::lock_guard<std::mutex> lock(ss.mu);
    if (!ss.made) {
        ss.made = true;
        // the lowest priority: the loop's CTAs take the SMs first, the pass
        // fills those left over
        int least = 0, greatest = 0;
        ss.ok = cudaDeviceGetStreamPriorityRange(&least, &greatest) == cudaSuccess &&
                cudaStreamCreateWithPriority(&ss.s, cudaStreamNonBlocking, least) == cudaSuccess &&
                cudaEventCreateWithFlags(&ss.start, cudaEventDisableTiming) == cudaSuccess &&
                cudaEventCreateWithFlags(&ss.ready, cudaEventDisableTiming) == cudaSuccess &&
                cudaDeviceGetAttribute(&ss.sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess &&
                ss.sms > 0;
        if (!ss.ok) cudaGetLastError();
    }
    return ss.ok ? &ss : nullptr;
}

}  // namespace

// With room for them, the turned Q^ and scaled K~ are written once by a
// streaming pass and the kernel only loads them.  When the chunk loop needs
// more than one wave of CTAs (one per SM: its shared memory and registers
// fill an SM), the batch is cut into as many slices as waves, each at most
// a wave: the loop of slice i then leaves SMs free on which the streaming
// pass of slice i+1 runs from the side stream, so only the first slice's
// pass is exposed.  The slices compute exactly what one launch would (every
// (b, h) and every row of the pass is independent).
cudaError_t launch_chunkwise_tc(const Params &p, bool out_bf16, const void *Q, const void *K,
                                const void *V, const float *s_in, float *s_out, void *O,
                                const void *G, void *Y, float eps, void *prep_ws, int *status,
                                cudaStream_t st) {
    if (!prep_ws)
        return launch_tc_rows(p, out_bf16, Q, K, V, s_in, s_out, O, G, Y, eps, 0, status, st);
    SideStream *ss = side_stream();
    // as many slices as waves, when every slice then fits in one wave (so
    // slicing never adds a wave); otherwise one launch
    constexpr int kMaxSlices = 16;
    const long long ctas_per_b = (long long)p.H * (p.dv / kTV);
    int slices = 1;
    if (ss) {
        const long long waves = (ctas_per_b * p.B + ss->sms - 1) / ss->sms;
        const long long per_slice = (p.B + waves - 1) / waves;  // batch elements, at most
        if (waves > 1 && waves <= std::min(p.B, kMaxSlices) && per_slice * ctas_per_b <= ss->sms)
            slices = (int)waves;
    }
    if (slices <= 1) {
        cudaError_t e = launch_chunkwise_prep(p, kC, Q, K, prep_ws, &Q, &K, st);
        if (e != cudaSuccess) return e;
        return launch_tc_rows(p, out_bf16, Q, K, V, s_in, s_out, O, G, Y, eps, 1, status, st);
    }
    // slice i: batch elements [b0(i), b0(i+1)); byte offsets per batch element
    auto b0 = [&](int i) { return (int)((long long)p.B * i / slices); };
    const size_t ob = out_bf16 ? 2 : 4;
    const size_t qk_b = (size_t)p.H * p.L * p.dk * 2, v_b = (size_t)p.H * p.L * p.dv * 2;
    const size_t o_b = (size_t)p.H * p.L * p.dv * ob, st_b = (size_t)p.H * p.dk * p.dv;
    const size_t ws_b = chunkwise_prep_bytes(p) / p.B;
    auto at = [](const void *base, size_t off) {
        return base ? static_cast<const void *>(static_cast<const uint8_t *>(base) + off) : nullptr;
    };
    auto at_w = [](void *base, size_t off) {
        return base ? static_cast<void *>(static_cast<uint8_t *>(base) + off) : nullptr;
    };
    auto sub = [&](int i) {
        Params q = p;
        q.B = b0(i + 1) - b0(i);
        return q;
    };
    const void *qh[kMaxSlices], *kt[kMaxSlices];  // prepared operands per slice
    auto prep = [&](int i, cudaStream_t on) {
        const size_t b = b0(i);
        return launch_chunkwise_prep(sub(i), kC, at(Q, b * qk_b), at(K, b * qk_b),
                                     at_w(prep_ws, b * ws_b), &qh[i], &kt[i], on);
    };
    // pass 0 on the caller's stream; the side stream starts after it (and so
    // after whatever the caller queued before), when the loop of slice 0
    // starts: the passes of the later slices run beside the loops
    std::lock_guard<std::mutex> lock(ss->mu);
    cudaError_t e = prep(0, st);
    if (e == cudaSuccess) e = cudaEventRecord(ss->start, st);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(ss->s, ss->start, 0);
    for (int i = 0; i < slices && e == cudaSuccess; ++i) {
        const size_t b = b0(i);
        e = launch_tc_rows(sub(i), out_bf16, qh[i], kt[i], at(V, b * v_b),
                           s_in ? s_in + b * st_b : nullptr, s_out ? s_out + b * st_b : nullptr,
                           at_w(O, b * o_b), at(G, b * v_b), at_w(Y, b * o_b), eps, 1, status, st);
        if (e == cudaSuccess && i + 1 < slices) {
            e = prep(i + 1, ss->s);
            if (e == cudaSuccess) e = cudaEventRecord(ss->ready, ss->s);
            if (e == cudaSuccess) e = cudaStreamWaitEvent(st, ss->ready, 0);
        }
    }
    return e;
}

cudaError_t launch_chunkwise_tc_rows(const Params &p, bool out_bf16, const void *Qh, const void *Kt,
                                     const void *V, const float *s_in, float *s_out, void *O,
                                     const void *G, void *Y, float eps, int *status,
                                     cudaStream_t st) {
    static_assert(kChunkBlock == kC, "the streaming pass and the loop share the row blocks");
    return launch_tc_rows(p, out_bf16, Qh, Kt, V, s_in, s_out, O, G, Y, eps, 1, status, st);
}

cudaError_t launch_chunkwise_tc_prepared(const Params &p, bool out_bf16, const void *Qh,
                                         RowLayout q_layout, const void *Kt, const void *V,
                                         RowLayout v_layout, bool v_head_major, const void *G,
                                         RowLayout g_layout, void *Y, void *O, float eps,
                                         int *status, cudaStream_t st) {
    return launch_chunkwise_ws(p, out_bf16, Qh, q_layout, Kt, V, v_layout, v_head_major, nullptr,
                               nullptr, O, G, g_layout, Y, eps, false, status, st);
}

}  // namespace ret
