// segstate.cu -- the state a segment of rows leaves from a zero start, on
// the sm_100a tensor cores.
//
// "Retentive Network" paper summary, section 2.1, chunkwise form (3): a
// block of n rows that starts from state R leaves gamma^n R + U with
//     U = sum_{t<n} gamma^{n-1-t} k^_t^T v_t,
// the block's own contribution.  With the weight gamma^{n-1-t} on the rows
// of one factor, U is one plain product, U = K~^T V, a reduction over the
// segment's rows.  The weight comes
//   - on the keys, K~_t = gamma^{n-1-t} k^_t (the streaming pass of prep.cu
//     with the segment as one block), or
//   - on the value rows (value mode 1), which warps 1-7 scale in shared
//     memory as each block of 128 rows lands, or
//   - split (value mode 2): keys weighted per block of 128 rows by the
//     streaming pass of the chunk loop, K~_t = gamma^{m-1-j} k^_t for row j
//     of a block of m rows, and the value rows of block b scaled by
//     gamma^{n - 128 b - m}, which makes up the rest of gamma^{n-1-t}.  One CTA
// owns one (b, h) and 128 value columns (d_v = 64: the 64, the rest of its
// V tile held at zero; d_k 64, 128 or 256) and accumulates U^T = V^T K~ in
// tensor memory over blocks of rows, which TMA brings through a ring of
// stages; its one MMA thread also reissues each stage's loads once the
// product that read it has completed.  A stage holds 128 rows at d_k 256
// and 64 rows at d_k 64 or 128, so that there two CTAs share an SM (96 KB
// or less of shared memory each) and a launch of up to 296 CTAs runs as
// one wave.  The eight warps then move U^T out
// of tensor memory into U [d_k][d_v] (fp32), one value column per lane.
//
// Every wait is bounded (about 2 s): on expiry RET_ERR_TIMEOUT is latched in
// the device status word, the CTA skips the rest, in-flight copies get a
// bounded drain and tensor memory is freed.
#include <cuda.h>

#include "common.cuh"
#include "launch.h"
#include "tc_util.cuh"

namespace ret {
namespace {

using namespace tc;

constexpr int kTV = 128;    // value columns per CTA (MMA M)
constexpr int kThreads = 256;                // warp 0 issues, warps 1-7 scale value rows
constexpr int kScalers = kThreads - 32;
constexpr long long kTimeoutCycles = 4000000000LL;

template <int DK>
struct SLayout {
    static constexpr int kRows = DK == 256 ? 128 : 64;    // rows per stage (the MMA's K extent)
    static constexpr uint32_t kBlk = kRows * 128;         // one 64-column block of a stage
    static constexpr int kStages = DK == 256 ? 2 : DK == 128 ? 3 : 4;
    static constexpr uint32_t kVBytes = kRows * kTV * 2;  // 2 blocks of 64 columns
    static constexpr uint32_t kKBytes = kRows * DK * 2;   // DK/64 blocks of 64 columns
    static constexpr uint32_t kStage = kVBytes + kKBytes;
    static constexpr uint32_t kBar = kStages * kStage;    // full[s], empty[s], ready[s], done
    static constexpr uint32_t kTmemSlot = kBar + 8 * (3 * kStages + 1);
    static constexpr uint32_t kAbort = kTmemSlot + 4;
    static constexpr uint32_t kBytes = kAbort + 4;
};

template <int DK>
__global__ void __launch_bounds__(kThreads, 1)
segment_state_kernel(const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmK,
                     const Params p, int zeta_v, float *__restrict__ U, int *status) {
    using Ly = SLayout<DK>;
    constexpr int NS = Ly::kStages;
    constexpr int kRows = Ly::kRows;
    constexpr uint32_t kBlk = Ly::kBlk;
    constexpr int KB = DK / 64;
    constexpr uint32_t kIdesc = idesc_bf16(128, DK, 1, 1);  // U^T += V^T K~ (both MN-major)
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t sbase = smem_u32(smem);
    const int tid = threadIdx.x, warp = tid >> 5;
    const int bh = blockIdx.y, v0 = blockIdx.x * kTV;
    const int L = p.L, dv = p.dv;
    const int dvr = min(kTV, dv - v0);  // value columns of this CTA: 128, or 64 when d_v = 64
    const float lg = p.log2g[bh % p.H];
    const int nblk = (L + kRows - 1) / kRows;
    if (sbase & 1023u) {
        if (tid == 0) atomicExch(status, (int)RET_ERR_CUDA);
        return;
    }
    auto full = [&](int s) { return sbase + Ly::kBar + 8u * s; };
    auto empty = [&](int s) { return sbase + Ly::kBar + 8u * (NS + s); };
    auto ready = [&](int s) { return sbase + Ly::kBar + 8u * (2 * NS + s); };
    const uint32_t done = sbase + Ly::kBar + 8u * (3 * NS);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Ly::kAbort);
    if (tid == 0) {
        for (int i = 0; i < 3 * NS + 1; ++i)
            mbar_init(sbase + Ly::kBar + 8u * i, (i >= 2 * NS && i < 3 * NS) ? kScalers / 32 : 1);
        *abort_flag = 0;
        fence_mbar_init();
        fence_proxy_async_smem();
    }
    if (warp == 0) {
        tmem_alloc(sbase + Ly::kTmemSlot, DK);
        tmem_relinquish();
    }
    if (dvr < kTV) {
        // d_v = 64: the second 64-column block of every stage's V tile is
        // never loaded and stays zero
        for (int s = 0; s < NS; ++s)
            for (int i = tid; i < (int)kBlk / 16; i += kThreads)
                reinterpret_cast<uint4 *>(smem + s * Ly::kStage + kBlk)[i] = make_uint4(0u, 0u, 0u, 0u);
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + Ly::kTmemSlot);

    if (tid == 0) {
        auto load = [&](int s, int blk) {
            const uint32_t st = sbase + s * Ly::kStage;
            mbar_expect_tx(full(s), dvr * kRows * 2 + Ly::kKBytes);
            for (int nb = 0; nb < dvr / 64; ++nb)
                tma_load_3d(st + nb * kBlk, &tmV, full(s), v0 + nb * 64, blk * kRows, bh);
            for (int kb = 0; kb < KB; ++kb)
                tma_load_3d(st + Ly::kVBytes + kb * kBlk, &tmK, full(s), kb * 64, blk * kRows, bh);
        };
        for (int s = 0; s < NS && s < nblk; ++s) load(s, s);
        bool ok = true;
#pragma unroll 1
        for (int blk = 0; blk < nblk && ok; ++blk) {
            const int s = blk % NS;
            const uint32_t par = (blk / NS) & 1;
            ok = mbar_wait_bounded(zeta_v ? ready(s) : full(s), par, abort_flag, status, kTimeoutCycles);
            if (!ok) break;
            tc_fence_after();
            const uint32_t st = sbase + s * Ly::kStage;
            const uint64_t dA = sdesc_sw128(st, kBlk, 1024);                   // V, MN-major
            const uint64_t dB = sdesc_sw128(st + Ly::kVBytes, kBlk, 1024);     // K~, MN-major
#pragma unroll
            for (int ks = 0; ks < kRows / 16; ++ks) {
                const uint64_t off = (uint64_t)((ks * 2048) >> 4);
                mma_ss(tmem, dA + off, dB + off, kIdesc, (blk > 0 || ks > 0) ? 1u : 0u);
            }
            mma_commit(empty(s));
            // the stage's next block, once this product has read it
            if (blk + NS < nblk) {
                ok = mbar_wait_bounded(empty(s), par, abort_flag, status, kTimeoutCycles);
                if (ok) load(s, blk + NS);
            }
        }
        mma_commit(done);
    } else if (zeta_v && warp > 0) {
        // V' = diag(zeta) V as each stage lands, zeta_t = gamma^{L-1-t}
        // (mode 1) or gamma^{L - 128 c - m} for row t of the c-th block of
        // 128 rows, which has m rows (mode 2, the blocks the keys were
        // weighted in): warps 1-7, one row per thread and pass (rows past L
        // are zeros)
        const int t = tid - 32;
        const int lane = tid & 31;
#pragma unroll 1
        for (int blk = 0; blk < nblk; ++blk) {
            const int s = blk % NS;
            const uint32_t par = (blk / NS) & 1;
            if (!__all_sync(0xffffffffu, mbar_wait_bounded(full(s), par, abort_flag, status,
                                                           kTimeoutCycles)))
                break;
            uint8_t *vt = smem + s * Ly::kStage;
#pragma unroll 1
            for (int r = t; r < kRows; r += kScalers) {
                const int row = blk * kRows + r;
                const int c0 = row - row % kChunkBlock;
                const int m = min(kChunkBlock, L - c0);
                const float z = row >= L ? 0.f
                                         : decay_pow(lg, zeta_v == 1 ? L - 1 - row : L - c0 - m);
                const uint64_t Z = f2_make(z, z);
#pragma unroll
                for (int nb = 0; nb < 2; ++nb)
                    if (nb * 64 < dvr)
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch) {
                        // rows of a phase start at different 16-byte pieces: no bank conflicts
                        uint4 *ptr = reinterpret_cast<uint4 *>(vt + nb * kBlk + r * 128 + (((ch + r) & 7) << 4));
                        uint4 w = *ptr;
                        uint32_t *u = reinterpret_cast<uint32_t *>(&w);
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const uint64_t hi = (static_cast<uint64_t>(u[e] & 0xffff0000u) << 32) | (u[e] << 16);
                            const uint64_t x = f2_mul(hi, Z);
                            __nv_bfloat162 pr = __floats2bfloat162_rn(f2_lo(x), f2_hi(x));
                            u[e] = *reinterpret_cast<uint32_t *>(&pr);
                        }
                        *ptr = w;
                    }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(ready(s));
        }
    }
    __syncthreads();
    // U[d][v0 + lane] of every d-column of U^T (lanes are value columns;
    // warps 0-3 take the first half of the d-columns, warps 4-7 the rest)
    const int row = tid & 127;
    const int dbeg = warp < 4 ? 0 : DK / 2;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    bool ok = *abort_flag == 0 && mbar_wait_bounded(done, 0, abort_flag, status, kTimeoutCycles);
    ok = __all_sync(0xffffffffu, ok);
    if (ok && *abort_flag == 0) {
        tc_fence_after();
#pragma unroll 1
        for (int d0 = dbeg; d0 < dbeg + DK / 2; d0 += 32) {
            uint32_t r[32];
            tmem_ld32(tmem + lane_base + d0, r);
            tmem_wait_ld(r);
#pragma unroll
            for (int i = 0; i < 32; ++i)
                if (row < dvr) U[((size_t)bh * DK + d0 + i) * dv + v0 + row] = __uint_as_float(r[i]);
        }
    }
    if (tid == 0 && *abort_flag) {
        const long long start = clock64();
        while (clock64() - start < 20000000LL) __nanosleep(1000);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, DK);
    }
}

template <int DK>
cudaError_t launch_dk(const Params &p, const CUtensorMap &mv, const CUtensorMap &mk, int zeta_v,
                      float *U, int *status, cudaStream_t st) {
    auto kern = segment_state_kernel<DK>;
    const int smem = (int)SLayout<DK>::kBytes;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    kern<<<dim3((p.dv + kTV - 1) / kTV, p.B * p.H), kThreads, smem, st>>>(mv, mk, p, zeta_v, U, status);
    e = cudaGetLastError();
    if (e == cudaSuccess) note_launches(1);
    return e;
}

}  // namespace

bool segment_state_tc_supported(const Params &p) {
    return (p.dk == 64 || p.dk == 128 || p.dk == 256) && (p.dv == 64 || p.dv % kTV == 0) &&
           p.dv <= kMaxDv && p.L >= 1 &&
           (long long)p.B * p.H >= 1 && (long long)p.B * p.H <= 65535;
}

cudaError_t launch_segment_state_tc(const Params &p, const void *V, const void *Kt, int zeta_v,
                                    float *U, int *status, cudaStream_t st) {
    CUtensorMap mv, mk;
    const int bh = p.B * p.H;
    const int rows = p.dk == 256 ? SLayout<256>::kRows : SLayout<128>::kRows;
    if (!make_tma_map_bf16(&mv, V, p.dv, p.L, bh, rows) || !make_tma_map_bf16(&mk, Kt, p.dk, p.L, bh, rows))
        return cudaErrorInvalidValue;
    if (p.dk == 256) return launch_dk<256>(p, mv, mk, zeta_v, U, status, st);
    if (p.dk == 64) return launch_dk<64>(p, mv, mk, zeta_v, U, status, st);
    return launch_dk<128>(p, mv, mk, zeta_v, U, status, st);
}

}  // namespace ret
