// parallel_tc.cu -- the parallel form of retention on the sm_100a tensor
// cores ("Retentive Network" paper summary, section 2.1, form (1)):
//     O = (Q^ K^^T (.) D) V,   D_nm = gamma^{n-m} for n >= m, else 0.
//
// Flash-style: one CTA owns a 128-row query tile, a slice of V columns
// (TV = 256, or 128 when d_v is not a multiple of 256, or 64 when d_v is
// 64) and one (b,h); d_k is 64, 128 or 256.  It
// walks the key tiles from the diagonal down:
//     S = Q^ K^_k^T            (tcgen05, fp32 in tensor memory)
//     P = S (.) D_tile         (CUDA cores: the decay as the rank-1 product
//                               gamma^{Delta+j} gamma^{-j'}, Delta = q0 - k0,
//                               and the causal mask on the diagonal tile;
//                               bf16 back into tensor memory)
//     O += P V_k               (tcgen05, A operand from tensor memory)
// Key tiles whose largest weight gamma^{Delta-127} is below 2^-150 add
// nothing representable in fp32; the walk stops there.  Roles (12 warps):
// one thread issues the MMAs -- S of tile t into one of two tensor-memory
// buffers, then P V of tile t-1 -- so that the P pass of one tile runs while
// the tensor cores multiply its neighbour; one thread issues the TMA loads of
// Q and of the next K tile once S has read the current one; another loads V
// in halves of 64 keys into a ring of three (so the next tile's first half
// lands while the current tile's products run, and its second half as soon
// as the current first half is consumed); warps 4-11 run the P pass and
// finally move the output tile out through shared memory and TMA stores.  Every hand-over is an mbarrier with
// a bounded wait.
//
// The rotation (xPos) is applied once per row by xpos_rotate_kernel into a
// workspace before this kernel runs: every key tile is read by many query
// tiles, so turning it inside would repeat the work per tile pair.
#include <cuda.h>

#include <cstring>

#include "common.cuh"
#include "launch.h"
#include "tc_util.cuh"

namespace ret {
namespace {

using namespace tc;

constexpr int kT = 128;         // query / key tile rows
constexpr int kThreads = 384;   // three warpgroups
constexpr long long kTimeoutCycles = 4000000000LL;
constexpr float kMinLog2GammaTimesT = -60.f;  // gamma^-127 stays below 2^60

// BQ/BK: tile landed; VF0-2: V half in ring slot s landed; VE0-2: the
// products that read ring slot s done (slot free); SD0/SD1: S of the tile in
// S buffer b done; PR0/PR1: P of buffer b written; PV0/PV1: P V of buffer
// b's tile done (the buffer free again).  The buffer barriers complete once
// every two key tiles and the ring's once every three halves, so no waiter
// can fall two phases behind.
enum { BQ = 0, BK, VF0, VF1, VF2, VE0, VE1, VE2, SD0, SD1, PR0, PR1, PV0, PV1, kNumBars };
constexpr int kRing = 3;  // V half tiles (64 keys) in flight

template <int DK, int TV>
struct PLayout {
    static constexpr uint32_t kQ = 0;                     // Q^: DK/64 blocks of 16 KB
    static constexpr uint32_t kQBytes = kT * DK * 2;
    static constexpr uint32_t kK = kQ + kQBytes;          // K^_k
    // V: a ring of kRing half tiles (64 keys x TV columns, TV/64 blocks of
    // 8 KB); at the end the first 2 slots stage the bf16 output tile
    static constexpr uint32_t kV = kK + kQBytes;
    static constexpr uint32_t kVBlock = (kT / 2) * 64 * 2;
    static constexpr uint32_t kVSlot = kVBlock * (TV / 64);
    static constexpr uint32_t kSmall = kV + kRing * kVSlot;
    static constexpr uint32_t kBar = kSmall;
    static constexpr uint32_t kTmemSlot = kSmall + 8 * kNumBars;
    static constexpr uint32_t kAbort = kTmemSlot + 4;
    static constexpr uint32_t kColScale = kSmall + 128;   // gamma^{-j'}, 128 floats
    static constexpr uint32_t kBytes = kColScale + 512;
    static_assert(8 * kNumBars + 8 <= 128, "small area");
    static_assert(kRing * kVSlot >= kT * TV * 2, "the output tile is staged in the V ring");
};

__device__ __forceinline__ bool pwait(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                      int *status) {
    return mbar_wait_bounded(bar, parity, abort_flag, status, kTimeoutCycles);
}

// Two consecutive 32-bit values of a tensor-memory load as a packed pair.
__device__ __forceinline__ uint64_t f2_pair(const uint32_t *r) {
    return (static_cast<uint64_t>(r[1]) << 32) | r[0];
}
// The pair with its low / high lane zeroed where asked.
__device__ __forceinline__ uint64_t f2_mask(uint64_t x, bool lo_zero, bool hi_zero) {
    if (lo_zero) x &= 0xffffffff00000000ull;
    if (hi_zero) x &= 0x00000000ffffffffull;
    return x;
}

__device__ __forceinline__ uint32_t pk_bf16(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&v);
}

template <int DK, int TV, typename TO>
__global__ void __launch_bounds__(kThreads, 1)
parallel_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                   const Params p, TO *__restrict__ O, int *status) {
    using Ly = PLayout<DK, TV>;
    constexpr int KB = DK / 64, VB = TV / 64;
    constexpr uint32_t kIdescS = idesc_bf16(128, 128, 0, 0);  // Q^ x K^ (both K-major)
    constexpr uint32_t kIdescPV = idesc_bf16(128, TV, 0, 1);  // P (tmem) x V (MN-major)
    constexpr bool kStage = sizeof(TO) == 2;
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t sbase = smem_u32(smem);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, row = tid & 127;
    const int nqt = (p.L + kT - 1) / kT;
    const int qt = nqt - 1 - (int)blockIdx.x;  // long rows of tiles first
    const int v0 = blockIdx.y * TV, bh = blockIdx.z, h = bh % p.H;
    const int q0 = qt * kT;
    const float lg = p.log2g[h];

    if (sbase & 1023u) {
        if (tid == 0) atomicExch(status, (int)RET_ERR_CUDA);
        return;
    }
    auto bar = [&](int i) { return sbase + Ly::kBar + 8u * i; };
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Ly::kAbort);
    float *colscale = reinterpret_cast<float *>(smem + Ly::kColScale);
    if (tid == 0) {
        for (int i = 0; i < kNumBars; ++i) mbar_init(bar(i), (i == PR0 || i == PR1) ? 8 : 1);
        *abort_flag = 0;
        fence_mbar_init();
        fence_proxy_async_smem();
    }
    if (warp == 0) {
        tmem_alloc(sbase + Ly::kTmemSlot, 512);
        tmem_relinquish();
    }
    if (tid < kT) colscale[tid] = exp2f(-(float)tid * lg);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + Ly::kTmemSlot);
    const uint32_t tO = tmem;
    auto tS = [&](int b) { return tmem + 256 + 128 * b; };
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;

    // last key tile with a representable weight: gamma^{Delta-127} >= 2^-150
    int kt_min = 0;
    if (lg < 0.f) {
        const int far = (int)floorf(-150.f / lg) + 127;  // largest Delta still kept
        kt_min = max(0, qt - far / kT);
    }
    const int nit = qt - kt_min + 1;  // key tiles qt, qt-1, ..., kt_min
    auto wait_all = [&](int i, uint32_t parity) {
        return __all_sync(0xffffffffu, pwait(bar(i), parity, abort_flag, status));
    };

    if (warp == 0) {
        // ====== MMA issue (one thread): S of tile it into buffer it & 1,
        // then P V of tile it-1 while the P pass works on tile it
        const uint64_t dQ = sdesc_sw128(sbase + Ly::kQ, 16, 1024);
        const uint64_t dK = sdesc_sw128(sbase + Ly::kK, 16, 1024);
        auto pv = [&](int j) {  // P V of tile j (buffer j & 1), one V half (64 keys) at a time
            const int b = j & 1;
            if (!wait_all(PR0 + b, (j >> 1) & 1)) return false;
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                const int hi = 2 * j + half, slot = hi % kRing;
                if (!wait_all(VF0 + slot, (hi / kRing) & 1)) return false;
                tc_fence_after();
                if (lane == 0) {
                    const uint64_t dV = sdesc_sw128(sbase + Ly::kV + slot * Ly::kVSlot, Ly::kVBlock, 1024);
#pragma unroll
                    for (int ks = 0; ks < kT / 32; ++ks)
                        mma_ts(tO, tS(b) + half * 64 + ks * 8, dV + (uint64_t)((ks * 2048) >> 4), kIdescPV,
                               (ks > 0 || half > 0 || j > 0) ? 1u : 0u);
                    mma_commit(bar(VE0 + slot));
                    if (half == 1) mma_commit(bar(PV0 + b));
                }
                __syncwarp();
            }
            return true;
        };
        bool ok = wait_all(BQ, 0);
#pragma unroll 1
        for (int it = 0; it < nit && ok; ++it) {
            const int b = it & 1;
            // the K tile, and buffer b free (P V of tile it-2 done)
            ok = wait_all(BK, it & 1) && (it < 2 || wait_all(PV0 + b, ((it - 2) >> 1) & 1));
            if (!ok) break;
            tc_fence_after();
            if (lane == 0) {
#pragma unroll
                for (int ks = 0; ks < DK / 16; ++ks) {
                    const uint64_t off = (uint64_t)(((ks >> 2) * 16384 + (ks & 3) * 32) >> 4);
                    mma_ss(tS(b), dQ + off, dK + off, kIdescS, ks > 0);
                }
                mma_commit(bar(SD0 + b));
            }
            __syncwarp();
            if (it > 0) ok = pv(it - 1);
        }
        if (ok) pv(nit - 1);
    } else if (warp == 1) {
        // ====== TMA loads of Q and K: the next K tile as soon as S has read
        // the current one
        auto load_k = [&](int kt) {
            mbar_expect_tx(bar(BK), Ly::kQBytes);
            for (int kb = 0; kb < KB; ++kb)
                tma_load_3d(sbase + Ly::kK + kb * 16384, &tmK, bar(BK), kb * 64, kt * kT, bh);
        };
        if (lane == 0) {
            mbar_expect_tx(bar(BQ), Ly::kQBytes);
            for (int kb = 0; kb < KB; ++kb)
                tma_load_3d(sbase + Ly::kQ + kb * 16384, &tmQ, bar(BQ), kb * 64, q0, bh);
            load_k(qt);
        }
#pragma unroll 1
        for (int it = 0; it + 1 < nit; ++it) {
            if (!wait_all(SD0 + (it & 1), (it >> 1) & 1)) break;
            if (lane == 0) load_k(qt - it - 1);
            __syncwarp();
        }
    } else if (warp == 2) {
        // ====== TMA loads of V, half a key tile at a time into the ring, as
        // soon as the products that read a slot's previous half are done
        // (the next tile's halves land while the current tile's products run)
#pragma unroll 1
        for (int hi = 0; hi < 2 * nit; ++hi) {
            const int slot = hi % kRing;
            if (hi >= kRing && !wait_all(VE0 + slot, (hi / kRing - 1) & 1)) break;
            if (lane == 0) {
                const int kt = qt - (hi >> 1), r0 = kt * kT + (hi & 1) * (kT / 2);
                const uint32_t dst = sbase + Ly::kV + slot * Ly::kVSlot;
                mbar_expect_tx(bar(VF0 + slot), Ly::kVSlot);
                for (int nb = 0; nb < VB; ++nb)
                    tma_load_3d(dst + nb * Ly::kVBlock, &tmV, bar(VF0 + slot), v0 + nb * 64, r0, bh);
            }
            __syncwarp();
        }
    } else if (warp >= 4) {
        // ====== P = S (.) D into tensor memory (warpgroup pw owns keys
        // [64 pw, 64 pw + 64)), then the output tile
        const int pw = (warp - 4) >> 2, gtid = tid - 128;
        const int k0 = pw * 64;
        bool ok = true;
#pragma unroll 1
        for (int it = 0; it < nit; ++it) {
            const int b = it & 1;
            const int delta = q0 - (qt - it) * kT;
            if (!wait_all(SD0 + b, (it >> 1) & 1)) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t a[32], c[32], pk[32];
            tmem_ld32(tS(b) + lane_base + k0, a);
            tmem_ld32(tS(b) + lane_base + k0 + 32, c);
            tmem_wait_ld(a);
            tmem_wait_ld(c);
            const float aj = exp2f((float)(delta + row) * lg);  // gamma^{Delta + j}
            const uint64_t A2 = f2_make(aj, aj);
            // the column weights gamma^{-j'} of this warpgroup's keys, four
            // at a time (one address for the whole warp: a broadcast)
            const float4 *cs4 = reinterpret_cast<const float4 *>(colscale + k0);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float4 wa = cs4[q], wb = cs4[8 + q];  // keys k0 + 4q.., k0 + 32 + 4q..
                const uint64_t w0 = f2_mul(A2, f2_make(wa.x, wa.y)), w1 = f2_mul(A2, f2_make(wa.z, wa.w));
                const uint64_t w2 = f2_mul(A2, f2_make(wb.x, wb.y)), w3 = f2_mul(A2, f2_make(wb.z, wb.w));
                uint64_t x0 = f2_mul(f2_pair(a + 4 * q), w0), x1 = f2_mul(f2_pair(a + 4 * q + 2), w1);
                uint64_t x2 = f2_mul(f2_pair(c + 4 * q), w2), x3 = f2_mul(f2_pair(c + 4 * q + 2), w3);
                if (delta == 0) {
                    // the diagonal tile: keys after the row's own position are masked
                    const int j = k0 + 4 * q;
                    x0 = f2_mask(x0, j > row, j + 1 > row);
                    x1 = f2_mask(x1, j + 2 > row, j + 3 > row);
                    x2 = f2_mask(x2, j + 32 > row, j + 33 > row);
                    x3 = f2_mask(x3, j + 34 > row, j + 35 > row);
                }
                pk[2 * q] = pk_bf16(f2_lo(x0), f2_hi(x0));
                pk[2 * q + 1] = pk_bf16(f2_lo(x1), f2_hi(x1));
                pk[16 + 2 * q] = pk_bf16(f2_lo(x2), f2_hi(x2));
                pk[16 + 2 * q + 1] = pk_bf16(f2_lo(x3), f2_hi(x3));
            }
            // keys [64w, 64w+64) -> columns [64w, 64w+32) of the buffer
            tmem_st32(tS(b) + lane_base + k0, pk);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(PR0 + b));
        }
        // the output tile once the last P V has landed (the group decides
        // together: it meets at a barrier before the store)
        const int last = nit - 1;
        ok = ok && wait_all(PV0 + (last & 1), (last >> 1) & 1);
        ok = named_sync_and(1, 256, ok);
        if (ok) {
            tc_fence_after();
            const int c0 = pw * (TV / 2);  // each warpgroup: TV/2 columns of the row
#pragma unroll 1
            for (int g = 0; g < TV / 64; ++g) {
                uint32_t a[32];
                tmem_ld32(tO + lane_base + c0 + 32 * g, a);
                tmem_wait_ld(a);
                const int col = c0 + 32 * g;
                if constexpr (kStage) {
                    // bf16 through the V tile (free: the last P V has read it)
                    uint8_t *dst = smem + Ly::kV + (col >> 6) * 16384 + row * 128;
                    const int ch0 = (col & 63) >> 3;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint4 w;
                        w.x = pk_bf16(__uint_as_float(a[8 * q + 0]), __uint_as_float(a[8 * q + 1]));
                        w.y = pk_bf16(__uint_as_float(a[8 * q + 2]), __uint_as_float(a[8 * q + 3]));
                        w.z = pk_bf16(__uint_as_float(a[8 * q + 4]), __uint_as_float(a[8 * q + 5]));
                        w.w = pk_bf16(__uint_as_float(a[8 * q + 6]), __uint_as_float(a[8 * q + 7]));
                        *reinterpret_cast<uint4 *>(dst + (((ch0 + q) ^ (row & 7)) << 4)) = w;
                    }
                } else if (q0 + row < p.L) {
                    float *dst = reinterpret_cast<float *>(O) + ((size_t)bh * p.L + q0 + row) * p.dv + v0 + col;
#pragma unroll
                    for (int i = 0; i < 32; i += 4)
                        *reinterpret_cast<float4 *>(dst + i) =
                            make_float4(__uint_as_float(a[i]), __uint_as_float(a[i + 1]),
                                        __uint_as_float(a[i + 2]), __uint_as_float(a[i + 3]));
                }
            }
            if constexpr (kStage) {
                fence_proxy_async_smem();
                named_sync(1, 256);
                if (gtid == 0) {
                    for (int nb = 0; nb < VB; ++nb)
                        tma_store_3d(&tmO, sbase + Ly::kV + nb * 16384, v0 + nb * 64, q0, bh);
                    bulk_commit();
                    bulk_wait_all();
                }
            }
        }
    }
    __syncthreads();
    // after an abort, copies and MMAs in flight get a bounded time to land
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

// xPos turn of [rows][dk] rows (row r at position pos_offset + r % L) into
// bf16.  Thread -> (16-byte output chunk = 4 pairs, block of 16 consecutive
// rows); the angles start exact and advance by theta_j per row.
template <typename TI>
__global__ void __launch_bounds__(256)
xpos_rotate_kernel(Params p, long long rows, const TI *__restrict__ x, __nv_bfloat16 *__restrict__ y) {
    constexpr int kRowsPerThread = 16;
    __shared__ double s_theta[kMaxDk / 2];
    stage_theta(p, s_theta, p.dk / 2);
    __syncthreads();
    const int nch = p.dk / 8;
    const long long items = (rows + kRowsPerThread - 1) / kRowsPerThread * nch;
    for (long long item = (long long)blockIdx.x * blockDim.x + threadIdx.x; item < items;
         item += (long long)gridDim.x * blockDim.x) {
        const int c16 = (int)(item % nch);
        const long long r0 = item / nch * kRowsPerThread;
        float c[4], s[4], sc[4], ss[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const double th = s_theta[c16 * 4 + e];
            rot_cs(p.pos_offset + r0 % p.L, th, &c[e], &s[e]);
            rot_cs(1, th, &sc[e], &ss[e]);
        }
        for (int k = 0; k < kRowsPerThread && r0 + k < rows; ++k) {
            const long long r = r0 + k;
            if (k > 0 && r % p.L == 0) {  // a new (b,h) slice starts: restart the angles
#pragma unroll
                for (int e = 0; e < 4; ++e) rot_cs(p.pos_offset, s_theta[c16 * 4 + e], &c[e], &s[e]);
            }
            const size_t base = (size_t)r * p.dk + c16 * 8;
            uint4 out;
            uint32_t *u = reinterpret_cast<uint32_t *>(&out);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                float x0 = ld(x, base + 2 * e), x1 = ld(x, base + 2 * e + 1);
                u[e] = pk_bf16(x0 * c[e] - x1 * s[e], x0 * s[e] + x1 * c[e]);
                const float cn = c[e] * sc[e] - s[e] * ss[e];
                s[e] = c[e] * ss[e] + s[e] * sc[e];
                c[e] = cn;
            }
            *reinterpret_cast<uint4 *>(y + base) = out;
        }
    }
}

template <int DK, int TV, typename TO>
cudaError_t launch_ptc(const Params &p, const CUtensorMap &mq, const CUtensorMap &mk,
                       const CUtensorMap &mv, const CUtensorMap &mo, void *O, int *status,
                       cudaStream_t st) {
    auto kern = parallel_tc_kernel<DK, TV, TO>;
    const int smem = (int)PLayout<DK, TV>::kBytes;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    dim3 grid((p.L + kT - 1) / kT, p.dv / TV, p.B * p.H);
    kern<<<grid, kThreads, smem, st>>>(mq, mk, mv, mo, p, (TO *)O, status);
    e = cudaGetLastError();
    if (e == cudaSuccess) note_launches(1);
    return e;
}

template <int DK, typename TO>
cudaError_t launch_ptc_tv(const Params &p, const CUtensorMap &mq, const CUtensorMap &mk,
                          const CUtensorMap &mv, const CUtensorMap &mo, void *O, int *status,
                          cudaStream_t st) {
    if (p.dv % 256 == 0) return launch_ptc<DK, 256, TO>(p, mq, mk, mv, mo, O, status, st);
    if (p.dv % 128 == 0) return launch_ptc<DK, 128, TO>(p, mq, mk, mv, mo, O, status, st);
    return launch_ptc<DK, 64, TO>(p, mq, mk, mv, mo, O, status, st);
}

}  // namespace

bool parallel_tc_supported(const Params &p, bool in_bf16) {
    if (!in_bf16 || (p.dk != 64 && p.dk != 128 && p.dk != 256) || (p.dv % 128 != 0 && p.dv != 64) ||
        p.L < 1 ||
        (long long)p.B * p.H > 65535 || (p.L + kT - 1) / kT > 2147483647)
        return false;
    for (int h = 0; h < p.H; ++h)
        if (!(p.log2g[h] * 127.f >= kMinLog2GammaTimesT)) return false;  // also rejects gamma = 0
    return true;
}

size_t parallel_tc_workspace(const Params &p) {
    return p.rotate ? (size_t)2 * p.B * p.H * p.L * p.dk * sizeof(__nv_bfloat16) : 0;
}

cudaError_t launch_parallel_tc(const Params &p, bool out_bf16, const void *Q, const void *K,
                               const void *V, void *O, void *workspace, int *status,
                               cudaStream_t st) {
    const long long rows = (long long)p.B * p.H * p.L;
    if (p.rotate) {
        // the turned Q^ and K^ in the workspace, then the products read them
        __nv_bfloat16 *qr = static_cast<__nv_bfloat16 *>(workspace);
        __nv_bfloat16 *kr = qr + (size_t)rows * p.dk;
        const long long items = (rows + 15) / 16 * (p.dk / 8);
        const int blocks = (int)std::min<long long>((items + 255) / 256, 148LL * 32);
        xpos_rotate_kernel<__nv_bfloat16><<<blocks, 256, 0, st>>>(p, rows, (const __nv_bfloat16 *)Q, qr);
        xpos_rotate_kernel<__nv_bfloat16><<<blocks, 256, 0, st>>>(p, rows, (const __nv_bfloat16 *)K, kr);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        note_launches(2);
        Q = qr;
        K = kr;
    }
    CUtensorMap mq, mk, mv, mo;
    std::memset(&mo, 0, sizeof(mo));
    const int bh = p.B * p.H;
    if (!make_tma_map_bf16(&mq, Q, p.dk, p.L, bh, kT) || !make_tma_map_bf16(&mk, K, p.dk, p.L, bh, kT) ||
        !make_tma_map_bf16(&mv, V, p.dv, p.L, bh, kT / 2))
        return cudaErrorInvalidValue;
    if (out_bf16 && !make_tma_map_bf16(&mo, O, p.dv, p.L, bh, kT)) return cudaErrorInvalidValue;
    if (p.dk == 256)
        return out_bf16 ? launch_ptc_tv<256, __nv_bfloat16>(p, mq, mk, mv, mo, O, status, st)
                        : launch_ptc_tv<256, float>(p, mq, mk, mv, mo, O, status, st);
    if (p.dk == 64)
        return out_bf16 ? launch_ptc_tv<64, __nv_bfloat16>(p, mq, mk, mv, mo, O, status, st)
                        : launch_ptc_tv<64, float>(p, mq, mk, mv, mo, O, status, st);
    return out_bf16 ? launch_ptc_tv<128, __nv_bfloat16>(p, mq, mk, mv, mo, O, status, st)
                    : launch_ptc_tv<128, float>(p, mq, mk, mv, mo, O, status, st);
}

}  // namespace ret
