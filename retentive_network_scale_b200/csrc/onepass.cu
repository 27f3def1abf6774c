// onepass.cu -- the chunkwise form in one launch for problems too small to
// fill the GPU with chunk loops: every block of 128 rows of every head runs
// at once, and each block takes the state it starts from out of the
// per-block key-value sums its predecessors publish.
//
// "Retentive Network" paper summary, section 2.1, chunkwise recurrent form
// (3), unrolled over blocks: the state entering block j of a head is
//   R_j = sum_{i<j} gamma^{128 (j-1-i)} U_i,  U_i = sum_{r in block i} gamma^{n_i-1-r} k_r^T v_r
// (n_i = 128: only the last block can be short, and it has no successor).
// Block j with n rows then forms, as the chunk loop does,
//   O''_r = q_r Rbar + sum_{r'<=r} (q_r . k~_r') v_r',  o_r = gamma^{r+1-n} O''_r,
// with k~_r = gamma^{n-1-r} k_r and Rbar = bf16(gamma^n R_j); and with the
// gate, Y = swish(G) (.) GroupNorm_h(O) over the head's d_v columns (section
// 2.2), all of which this CTA holds.
//
// One CTA per (b, h, block), blockIdx.x = block + blocks * (b, h) (4 warps
// for d_v = 64, 8 for d_v = 128; see OCfg):
//   1. TMA loads of the block's Q, K, V tiles; K scaled to K~ in shared memory
//   2. U^T = V^T K~ on the tensor cores, read out and published to the
//      workspace with a flag (release at GPU scope)
//   3. S = Q K~^T, and P = bf16(mask(S)) back into tensor memory
//   4. the flags of the head's earlier blocks (a bounded wait), then
//      Rbar^T = bf16(sum_i gamma^{n + 128 (j-1-i)} U_i^T) into shared memory
//   5. O'' = Q Rbar + P V; the epilogue (decay scale, GroupNorm, gate) writes
//      Y or O
// A CTA waits only on CTAs of lower index of the same launch, which start
// before it; the CTAs an SM can hold (by their registers: four of 128
// threads, or two of 256) fit its 512 tensor-memory columns together (128 or
// 256 each), so no resident CTA waits for one that cannot start.  The flags
// are zeroed (a memset on the stream) before each launch.
//
// Shapes: d_k 64 or 128, d_v 64 or 128, bf16, no rotation, no carried state,
// at most kMaxBlocks blocks per head.  Every wait is bounded (about 2 s of SM
// clock) and latches RET_ERR_TIMEOUT in the device status word on expiry.
#include <cuda.h>

#include "common.cuh"
#include "launch.h"
#include "tc_util.cuh"

namespace ret {
namespace {

using namespace tc;

constexpr int kRowsBlk = 128;
constexpr int kMaxBlocks = 32;
constexpr long long kTimeoutCycles = 4000000000LL;  // about 2 s

// MU: U^T product done; MS: S done; MO: O'' done; LD: the tiles landed
enum { LD = 0, MU, MS, MO, kNumBars };

// Two shapes of CTA.  d_v = 64 ("compact"): 4 warps, one thread per row,
// 128 tensor-memory columns (S / P in the first 64 once P is packed, O'' in
// the last 64), so four CTAs share an SM.  d_v = 128: 8 warps, two threads
// per row (each half of the value columns), 256 columns (S / P, then O''),
// two CTAs per SM (their registers allow no more).  Either way every SM's
// CTAs fit its 512 columns together, so no allocation waits.
template <int DK, int DV>
struct OCfg {
    static constexpr bool kCompact = DV == 64;
    static constexpr int kThreads = kCompact ? 128 : 256;
    static constexpr int kHalves = kThreads / 128;               // threads per row
    static constexpr int kTmemCols = kCompact ? 128 : 256;
    static constexpr uint32_t kOCol = kCompact ? 64 : 128;       // O'' columns start here
    // shared memory: V (DV/64 blocks of 16 KB), Q and K (DK/64 blocks each);
    // Rbar^T replaces K~ once S and U are done.  With d_v = 64 the U^T
    // product (M = 128 value columns) also reads the 64 rows past V, which
    // are Q's: those result lanes are never read.
    static constexpr uint32_t kV = 0;
    static constexpr uint32_t kQ = kV + (DV / 64) * 16384;
    static constexpr uint32_t kTile = kRowsBlk * DK * 2;
    static constexpr uint32_t kK = kQ + kTile;
    static constexpr uint32_t kR = kK;
    static constexpr uint32_t kSmall = kK + kTile;
    static constexpr uint32_t kBar = kSmall;
    static constexpr uint32_t kTmemSlot = kSmall + 8 * kNumBars;
    static constexpr uint32_t kAbort = kTmemSlot + 4;
    static constexpr uint32_t kStat = kSmall + 64;               // 2 halves x 128 rows x (mean, M2)
    static constexpr uint32_t kBytes = kStat + (kCompact ? 0 : 2048);
    static_assert(kV + 2 * 16384 <= kSmall, "the U^T product's second A block stays in the tiles");
};

__device__ __forceinline__ uint32_t pk2(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&v);
}
// swish(g) = g sigmoid(g) = h + h tanh(h), h = g / 2, on a bf16 pair
__device__ __forceinline__ uint32_t swish2(uint32_t g) {
    uint32_t h, t, s;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(h) : "r"(g), "r"(0x3f003f00u));
    asm("tanh.approx.bf16x2 %0, %1;" : "=r"(t) : "r"(h));
    asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(s) : "r"(h), "r"(t), "r"(h));
    return s;
}
__device__ __forceinline__ uint32_t ld_acquire(const uint32_t *p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release(uint32_t *p, uint32_t v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Eight consecutive values to global memory (16-byte aligned) as TO.
__device__ __forceinline__ void st8(__nv_bfloat16 *dst, const float *v) {
    uint4 w;
    w.x = pk2(v[0], v[1]);
    w.y = pk2(v[2], v[3]);
    w.z = pk2(v[4], v[5]);
    w.w = pk2(v[6], v[7]);
    *reinterpret_cast<uint4 *>(dst) = w;
}
__device__ __forceinline__ void st8(float *dst, const float *v) {
    *reinterpret_cast<float4 *>(dst) = make_float4(v[0], v[1], v[2], v[3]);
    *reinterpret_cast<float4 *>(dst + 4) = make_float4(v[4], v[5], v[6], v[7]);
}

// Row c of a K-major 128-byte-swizzled tile of DK columns: N values (a
// multiple of 8, within one block of 64) of columns [d0, d0+N) as bf16.
template <int DK, int N>
__device__ __forceinline__ void st_row(uint8_t *tile, int c, int d0, const float *v) {
    static_assert(N % 8 == 0 && N <= 64, "whole 16-byte pieces of one block");
    uint8_t *blk = tile + (d0 >> 6) * 16384 + c * 128;
    const int ch0 = (d0 & 63) >> 3;
#pragma unroll
    for (int q = 0; q < N / 8; ++q) {
        uint4 w;
        w.x = pk2(v[8 * q + 0], v[8 * q + 1]);
        w.y = pk2(v[8 * q + 2], v[8 * q + 3]);
        w.z = pk2(v[8 * q + 4], v[8 * q + 5]);
        w.w = pk2(v[8 * q + 6], v[8 * q + 7]);
        *reinterpret_cast<uint4 *>(blk + (((ch0 + q) ^ (c & 7)) << 4)) = w;
    }
}

template <int DK, int DV, typename TO>
__global__ void __launch_bounds__(OCfg<DK, DV>::kThreads, DV == 64 ? 4 : 2)
onepass_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const Params p, int nb,
               float *__restrict__ Uws, uint32_t *__restrict__ flags,
               const __nv_bfloat16 *__restrict__ G, TO *__restrict__ Y, TO *__restrict__ O,
               float gn_eps, int *status) {
    using C = OCfg<DK, DV>;
    constexpr int NT = C::kThreads, HS = C::kHalves, KB = DK / 64;
    constexpr bool kCompact = C::kCompact;
    constexpr uint32_t kIdescU = idesc_bf16(128, DK, 1, 1);    // U^T = V^T K~ (both MN-major)
    constexpr uint32_t kIdescS = idesc_bf16(128, 128, 0, 0);   // S = Q K~^T
    constexpr uint32_t kIdescQR = idesc_bf16(128, DV, 0, 0);   // O'' = Q Rbar
    constexpr uint32_t kIdescPV = idesc_bf16(128, DV, 0, 1);   // O'' += P V
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t sbase = smem_u32(smem);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int j = (int)(blockIdx.x % nb), bh = (int)(blockIdx.x / nb);
    const int h = bh % p.H, b = bh / p.H;
    const int t0 = j * kRowsBlk, n = min(kRowsBlk, p.L - t0);
    const float lg = p.log2g[h];

    if (sbase & 1023u) {
        if (tid == 0) atomicExch(status, (int)RET_ERR_CUDA);
        return;
    }
    auto bar = [&](int i) { return sbase + C::kBar + 8u * i; };
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::kAbort);
    auto wait_bar = [&](int i) {
        return __all_sync(0xffffffffu, mbar_wait_bounded(bar(i), 0, abort_flag, status, kTimeoutCycles));
    };
    if (tid == 0) {
        for (int i = 0; i < kNumBars; ++i) mbar_init(bar(i), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(sbase + C::kTmemSlot, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + C::kTmemSlot);
    const uint32_t tS = tmem, tO = tmem + C::kOCol;  // tS holds U^T first, then S / P
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const int row = tid & 127, half = tid >> 7;      // half: 0 when one thread per row
    const int c0 = half * (DV / HS);                 // this thread's 64 value columns

    // ---- 1. the tiles
    if (tid == 0) {
        mbar_expect_tx(bar(LD), 2 * C::kTile + (uint32_t)(DV / 64) * 16384);
        for (int kb = 0; kb < KB; ++kb) {
            tma_load_3d(sbase + C::kQ + kb * 16384, &tmQ, bar(LD), kb * 64, t0, bh);
            tma_load_3d(sbase + C::kK + kb * 16384, &tmK, bar(LD), kb * 64, t0, bh);
        }
        for (int vb = 0; vb < DV / 64; ++vb)
            tma_load_3d(sbase + C::kV + vb * 16384, &tmV, bar(LD), vb * 64, t0, bh);
    }
    // the gate of this thread's row and 64 columns, in flight while the
    // products run
    uint4 g4[8];
    const size_t yrow = ((size_t)b * p.L + t0 + row) * ((size_t)p.H * DV) + (size_t)h * DV + c0;
    const bool row_ok = row < n;
    if (G) {
#pragma unroll
        for (int q = 0; q < 8; ++q)
            g4[q] = row_ok ? *reinterpret_cast<const uint4 *>(G + yrow + 8 * q) : make_uint4(0u, 0u, 0u, 0u);
    }
    // Every block-wide barrier below is reached by all threads; `ok` is made
    // the same for the whole CTA at each of them.
    bool ok = __syncthreads_and(wait_bar(LD));
    // K~ = diag(gamma^{n-1-r}) K in place (rows past n are zeros from the load)
    if (ok) {
        for (int i = tid; i < kRowsBlk * KB * 8; i += NT) {
            const int r = (i >> 3) % kRowsBlk, kb = i / (kRowsBlk * 8), ch = i & 7;
            const float z = r < n ? decay_pow(lg, n - 1 - r) : 0.f;
            uint4 *ptr = reinterpret_cast<uint4 *>(smem + C::kK + kb * 16384 + r * 128 + ch * 16);
            uint4 w = *ptr;
            uint32_t *u = reinterpret_cast<uint32_t *>(&w);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&u[e]));
                u[e] = pk2(f.x * z, f.y * z);
            }
            *ptr = w;
        }
    }
    fence_proxy_async_smem();
    __syncthreads();

    // ---- 2. U^T = V^T K~ (lanes: value columns, columns: d_k), published
    if (j + 1 < nb) {
        if (ok && tid == 0) {
            tc_fence_after();
            const uint64_t dVa = sdesc_sw128(sbase + C::kV, 16384, 1024);
            const uint64_t dKb = sdesc_sw128(sbase + C::kK, 16384, 1024);
#pragma unroll
            for (int ks = 0; ks < kRowsBlk / 16; ++ks) {
                const uint64_t off = (uint64_t)((ks * 2048) >> 4);
                mma_ss(tS, dVa + off, dKb + off, kIdescU, ks > 0 ? 1u : 0u);
            }
            mma_commit(bar(MU));
        }
        ok = __syncthreads_and(ok && wait_bar(MU));
        if (ok) {
            tc_fence_after();
            // this thread: value column `row`, d_k columns [half DK/HS, (half+1) DK/HS)
            float *U = Uws + ((size_t)bh * nb + j) * DK * DV;
#pragma unroll 1
            for (int k0 = half * (DK / HS); k0 < (half + 1) * (DK / HS); k0 += 32) {
                uint32_t x[32];
                tmem_ld32(tS + lane_base + k0, x);
                tmem_wait_ld(x);
                if (row < DV) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) U[(size_t)(k0 + i) * DV + row] = __uint_as_float(x[i]);
                }
            }
        }
        tc_fence_before();
        __syncthreads();
        // the release orders the whole CTA's stores (ordered before it by the
        // barrier) before the flag, for an acquire at GPU scope
        if (ok && tid == 0) st_release(flags + (size_t)bh * nb + j, 1u);
    }

    // ---- 3. S = Q K~^T, P = bf16(mask(S)) into tensor memory
    if (ok && tid == 0) {
        tc_fence_after();
        const uint64_t dQ = sdesc_sw128(sbase + C::kQ, 16, 1024);
        const uint64_t dK = sdesc_sw128(sbase + C::kK, 16, 1024);
#pragma unroll
        for (int ks = 0; ks < DK / 16; ++ks) {
            const uint64_t off = (uint64_t)(((ks >> 2) * 16384 + (ks & 3) * 32) >> 4);
            mma_ss(tS, dQ + off, dK + off, kIdescS, ks > 0 ? 1u : 0u);
        }
        mma_commit(bar(MS));
    }
    ok = __syncthreads_and(ok && wait_bar(MS));
    if (ok) {
        tc_fence_after();
        const int quad = warp & 3;
        // keys [32 cb, 32 cb + 32): compact, packed into columns
        // [16 cb, 16 cb + 16) in order (each row is one thread's, and group
        // cb's S is read before group cb+1's P lands on its columns);
        // otherwise into [32 cb, 32 cb + 16), each half of the CTA taking two
        // groups
#pragma unroll 1
        for (int cb = half * (4 / HS); cb < (half + 1) * (4 / HS); ++cb) {
            uint32_t pk[16];
            if (cb > quad) {
#pragma unroll
                for (int i = 0; i < 16; ++i) pk[i] = 0u;
            } else {
                uint32_t a[32];
                tmem_ld32(tS + lane_base + 32 * cb, a);
                tmem_wait_ld(a);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int k0 = 32 * cb + 2 * i;
                    pk[i] = pk2(k0 <= row ? __uint_as_float(a[2 * i]) : 0.f,
                                k0 + 1 <= row ? __uint_as_float(a[2 * i + 1]) : 0.f);
                }
            }
            tmem_st16(tS + lane_base + (kCompact ? 16 : 32) * cb, pk);
            if constexpr (kCompact) tmem_wait_st();
        }
        tmem_wait_st();
    }
    tc_fence_before();
    __syncthreads();

    // ---- 4. the entering state from the earlier blocks' sums; Rbar^T over K~
    if (j > 0) {
        if (ok && tid < 32) {
            // the lanes poll the flags of blocks lane, lane + 32, ... below j
            bool seen = true;
            const long long start = clock64();
            for (int i = lane; i < j && seen; i += 32) {
                while (ld_acquire(flags + (size_t)bh * nb + i) == 0u) {
                    if (*abort_flag || clock64() - start > kTimeoutCycles) {
                        seen = false;
                        break;
                    }
                }
            }
            if (!__all_sync(0xffffffffu, seen) && lane == 0) {
                *abort_flag = 1;
                atomicExch(status, (int)RET_ERR_TIMEOUT);
            }
        }
        __syncthreads();
        ok = ok && *abort_flag == 0;  // read after the barrier: the same for every thread
        if (ok) {
            // this thread: Rbar^T rows v0..v0+3 (value columns) and NE
            // consecutive d_k columns from k0, four columns per 16-byte load;
            // block i weighs gamma^{n + 128 (j-1-i)}, two blocks in flight
            constexpr int VQ = DV / 4, NE = DK * VQ / NT;
            const int v0 = 4 * (tid % VQ), k0 = (tid / VQ) * NE;
            const float *Ub = Uws + (size_t)bh * nb * DK * DV + (size_t)k0 * DV + v0;
            float4 acc[NE];
#pragma unroll
            for (int e = 0; e < NE; ++e) acc[e] = make_float4(0.f, 0.f, 0.f, 0.f);
            auto add = [&](float w, const float4 &x, float4 &a) {
                a.x = fmaf(w, x.x, a.x);
                a.y = fmaf(w, x.y, a.y);
                a.z = fmaf(w, x.z, a.z);
                a.w = fmaf(w, x.w, a.w);
            };
            int i = 0;
#pragma unroll 1
            for (; i + 2 <= j; i += 2) {
                float4 x0[NE], x1[NE];
#pragma unroll
                for (int e = 0; e < NE; ++e) {
                    x0[e] = __ldcg(reinterpret_cast<const float4 *>(Ub + (size_t)i * DK * DV + (size_t)e * DV));
                    x1[e] = __ldcg(reinterpret_cast<const float4 *>(Ub + (size_t)(i + 1) * DK * DV + (size_t)e * DV));
                }
                const float w0 = exp2f((float)(n + kRowsBlk * (j - 1 - i)) * lg);
                const float w1 = exp2f((float)(n + kRowsBlk * (j - 2 - i)) * lg);
#pragma unroll
                for (int e = 0; e < NE; ++e) {
                    add(w0, x0[e], acc[e]);
                    add(w1, x1[e], acc[e]);
                }
            }
            if (i < j) {
                const float w = exp2f((float)(n + kRowsBlk * (j - 1 - i)) * lg);
#pragma unroll
                for (int e = 0; e < NE; ++e)
                    add(w, __ldcg(reinterpret_cast<const float4 *>(Ub + (size_t)i * DK * DV + (size_t)e * DV)), acc[e]);
            }
            // the four rows' NE values into Rbar^T (over K~, whose products are done)
            float r0[NE], r1[NE], r2[NE], r3[NE];
#pragma unroll
            for (int e = 0; e < NE; ++e) {
                r0[e] = acc[e].x;
                r1[e] = acc[e].y;
                r2[e] = acc[e].z;
                r3[e] = acc[e].w;
            }
            st_row<DK, NE>(smem + C::kR, v0 + 0, k0, r0);
            st_row<DK, NE>(smem + C::kR, v0 + 1, k0, r1);
            st_row<DK, NE>(smem + C::kR, v0 + 2, k0, r2);
            st_row<DK, NE>(smem + C::kR, v0 + 3, k0, r3);
        }
        fence_proxy_async_smem();
        __syncthreads();
    }

    // ---- 5. O'' = Q Rbar + P V
    if (ok && tid == 0) {
        tc_fence_after();
        const uint64_t dQ = sdesc_sw128(sbase + C::kQ, 16, 1024);
        const uint64_t dR = sdesc_sw128(sbase + C::kR, 16, 1024);
        const uint64_t dV = sdesc_sw128(sbase + C::kV, 16384, 1024);
        if (j > 0) {
#pragma unroll
            for (int ks = 0; ks < DK / 16; ++ks) {
                const uint64_t off = (uint64_t)(((ks >> 2) * 16384 + (ks & 3) * 32) >> 4);
                mma_ss(tO, dQ + off, dR + off, kIdescQR, ks > 0 ? 1u : 0u);
            }
        }
#pragma unroll
        for (int ks = 0; ks < kRowsBlk / 16; ++ks) {
            const uint32_t pa = kCompact ? tS + ks * 8 : tS + (ks >> 1) * 32 + (ks & 1) * 8;
            mma_ts(tO, pa, dV + (uint64_t)((ks * 2048) >> 4), kIdescPV, (j > 0 || ks > 0) ? 1u : 0u);
        }
        mma_commit(bar(MO));
    }
    ok = __syncthreads_and(ok && wait_bar(MO));
    if (ok) {
        tc_fence_after();
        // this thread: row `row`, value columns [c0, c0 + 64)
        const float alpha = exp2f((float)(row + 1 - n) * lg);
        float o[64];
#pragma unroll
        for (int g = 0; g < 2; ++g) {
            uint32_t x[32];
            tmem_ld32(tO + lane_base + c0 + 32 * g, x);
            tmem_wait_ld(x);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[32 * g + i] = alpha * __uint_as_float(x[i]);
        }
        if (O && row_ok) {
            TO *orow = O + ((size_t)bh * p.L + t0 + row) * DV + c0;
#pragma unroll
            for (int q = 0; q < 8; ++q) st8(orow + 8 * q, o + 8 * q);
        }
        if (Y) {
            // GroupNorm over the row's d_v columns (merged with the other
            // half's through shared memory when two threads share a row:
            // Chan's update for two equal counts)
            float s1 = 0.f;
#pragma unroll
            for (int i = 0; i < 64; ++i) s1 += o[i];
            const float m_own = s1 * (1.f / 64.f);
            float q_own = 0.f;
#pragma unroll
            for (int i = 0; i < 64; ++i) {
                const float d = o[i] - m_own;
                q_own += d * d;
            }
            float mean = m_own, var = q_own * (1.f / 64.f);
            if constexpr (HS == 2) {
                float2 *slots = reinterpret_cast<float2 *>(smem + C::kStat);
                slots[half * 128 + row] = make_float2(m_own, q_own);
                named_sync(1, NT);
                const float2 oth = slots[(1 - half) * 128 + row];
                const float dm = m_own - oth.x;
                mean = 0.5f * (m_own + oth.x);
                var = (q_own + oth.y + 32.f * dm * dm) * (1.f / 128.f);
            }
            const float rs = rsqrtf(var + gn_eps);
            if (row_ok) {
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const uint32_t *gu = reinterpret_cast<const uint32_t *>(&g4[q]);
                    float yv[8];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const uint32_t sw = swish2(gu[e]);
                        const float2 sf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&sw));
                        yv[2 * e] = (o[8 * q + 2 * e] - mean) * rs * sf.x;
                        yv[2 * e + 1] = (o[8 * q + 2 * e + 1] - mean) * rs * sf.y;
                    }
                    st8(Y + yrow + 8 * q, yv);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (tid == 0 && *abort_flag) {
        const long long start = clock64();
        while (clock64() - start < 20000000LL) __nanosleep(1000);
    }
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

template <int DK, int DV, typename TO>
cudaError_t launch_op(const Params &p, const CUtensorMap &mq, const CUtensorMap &mk,
                      const CUtensorMap &mv, int nb, float *U, uint32_t *flags, const void *G,
                      void *Y, void *O, float eps, int *status, cudaStream_t st) {
    auto kern = onepass_kernel<DK, DV, TO>;
    const int smem = (int)OCfg<DK, DV>::kBytes;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)((size_t)p.B * p.H * nb);
    kern<<<grid, OCfg<DK, DV>::kThreads, smem, st>>>(mq, mk, mv, p, nb, U, flags,
                                       static_cast<const __nv_bfloat16 *>(G), static_cast<TO *>(Y),
                                       static_cast<TO *>(O), eps, status);
    e = cudaGetLastError();
    if (e == cudaSuccess) note_launches(1);
    return e;
}

}  // namespace

bool onepass_supported(const Params &p, bool in_bf16, bool has_state) {
    if (!in_bf16 || has_state || p.rotate || (p.dk != 64 && p.dk != 128) || (p.dv != 64 && p.dv != 128))
        return false;
    const long long nb = (p.L + kRowsBlk - 1) / kRowsBlk;
    if (p.L < 1 || nb > kMaxBlocks || (long long)p.B * p.H * nb > 2147483647LL) return false;
    for (int h = 0; h < p.H; ++h)
        if (!(p.log2g[h] * 128.f >= -60.f)) return false;  // the K~ weights stay in range
    return true;
}

size_t onepass_bytes(const Params &p) {
    const size_t nb = (p.L + kRowsBlk - 1) / kRowsBlk;
    const size_t u = (size_t)p.B * p.H * nb * p.dk * p.dv * sizeof(float);
    return (u + 255) / 256 * 256 + (size_t)p.B * p.H * nb * sizeof(uint32_t);
}

cudaError_t launch_onepass(const Params &p, bool out_bf16, const void *Q, const void *K,
                           const void *V, void *O, const void *G, void *Y, float eps,
                           void *workspace, int *status, cudaStream_t st) {
    const int nb = (p.L + kRowsBlk - 1) / kRowsBlk;
    const int bh = p.B * p.H;
    const size_t nbh = (size_t)bh * nb;
    const size_t u = nbh * p.dk * p.dv * sizeof(float);
    float *Uws = static_cast<float *>(workspace);
    uint32_t *flags = reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(workspace) + (u + 255) / 256 * 256);
    if ((G == nullptr) != (Y == nullptr)) return cudaErrorInvalidValue;
    CUtensorMap mq, mk, mv;
    if (!make_tma_map_bf16(&mq, Q, p.dk, p.L, bh, kRowsBlk) ||
        !make_tma_map_bf16(&mk, K, p.dk, p.L, bh, kRowsBlk) ||
        !make_tma_map_bf16(&mv, V, p.dv, p.L, bh, kRowsBlk))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaMemsetAsync(flags, 0, nbh * sizeof(uint32_t), st);
    if (e != cudaSuccess) return e;
#define RET_ONEPASS_GO(DK, DV)                                                                      \
    return out_bf16 ? launch_op<DK, DV, __nv_bfloat16>(p, mq, mk, mv, nb, Uws, flags, G, Y, O, eps, status, st) \
                    : launch_op<DK, DV, float>(p, mq, mk, mv, nb, Uws, flags, G, Y, O, eps, status, st)
    if (p.dk == 64 && p.dv == 64) RET_ONEPASS_GO(64, 64);
    if (p.dk == 64) RET_ONEPASS_GO(64, 128);
    if (p.dv == 64) RET_ONEPASS_GO(128, 64);
    RET_ONEPASS_GO(128, 128);
#undef RET_ONEPASS_GO
}

}  // namespace ret
