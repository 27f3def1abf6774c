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
//   V'   = diag(zeta) V,            zeta_j  = gamma^{n-1-j}
//   Rbar = bf16(gamma^n R)          (the decayed state, kept that way in TMEM)
//   O''  = Q^ Rbar + mask(Q^ K^^T) V'        (mask: keep j' <= j)
//   o_j  = alpha_j O''_j,           alpha_j = gamma^{j+1-n}
//   R    <- gamma^n R + K^^T V'
// which is the same sum term by term (gamma^{j+1-n} gamma^{n-1-j'} =
// gamma^{j-j'}, gamma^{j+1-n} gamma^n = gamma^{j+1}).  All factors stay in
// range while gamma^128 >= 2^-60; other decays use the CUDA-core kernel.
//
// One CTA owns one (b, h) and a 128-column slice of V and walks the chunks
// in order.  Tensor memory (512 columns): S [128 x 128] (P, the bf16 mask
// of S, overwrites half of it and feeds the P V' product as the A operand),
// O'' [128 x 128], and the fp32 state slice R [d_k x 128] as d_k/128 halves
// of 128 lanes.  Shared memory: TMA-loaded Q, K, V tiles (128-byte swizzle)
// and Rbar in the MN-major layout read as a B operand.  Loads of Q, K and V
// complete on separate barriers and are issued as soon as the MMAs that
// read the previous tile finish, so the next chunk's Q streams in while
// this chunk's state update runs.
//
// Fused epilogue (Y = swish(G) (.) GroupNorm_h(O)): the CTAs of one head
// form a cluster along d_v; each reduces its 128 columns of a row to a mean
// and centred sum of squares, the partials are exchanged through
// distributed shared memory and merged (Chan's pairwise update), and every
// CTA normalises and gates its own columns.
//
// Every mbarrier wait is bounded: on expiry the kernel latches
// RET_ERR_TIMEOUT in the device status word and every thread skips the
// remaining work together (cluster barriers still run, so no CTA of a
// cluster is left waiting), in-flight copies and MMAs get a bounded drain,
// and TMEM is freed.
#include <cuda.h>

#include "common.cuh"
#include "launch.h"
#include "tc_util.cuh"

namespace ret {
namespace {

using namespace tc;

constexpr int kC = 128;       // chunk rows (MMA M)
constexpr int kTV = 128;      // value columns per CTA (MMA N)
constexpr int kThreads = 256;
constexpr int kMaxCluster = kMaxDv / kTV;
constexpr long long kTimeoutCycles = 4000000000LL;  // about 2 s
constexpr float kMinLog2GammaTimesC = -60.f;        // gamma^C >= 2^-60

enum { BQ = 0, BK, BV, BS, BX, BU, BPV, kNumBars };

template <int DK>
struct Layout {
    static constexpr uint32_t kQ = 0;                    // Q^: DK/64 blocks of 16 KB
    static constexpr uint32_t kQBytes = kC * DK * 2;
    static constexpr uint32_t kK = kQ + kQBytes;         // K^
    static constexpr uint32_t kV = kK + kQBytes;         // V (then V'): 2 blocks of 16 KB
    static constexpr uint32_t kVBytes = kC * kTV * 2;
    static constexpr uint32_t kR = kV + kVBytes;         // Rbar: 2 column blocks of DK*128 B
    static constexpr uint32_t kRBytes = DK * kTV * 2;
    static constexpr uint32_t kSmall = kR + kRBytes;
    static constexpr uint32_t kBar = kSmall;             // kNumBars mbarriers
    static constexpr uint32_t kTmemSlot = kSmall + 64;
    static constexpr uint32_t kAbort = kSmall + 68;
    static constexpr uint32_t kRotStep = kSmall + 128;   // DK/2 float2
    static constexpr uint32_t kBytes = kRotStep + DK * 4;
    // GroupNorm scratch inside the V tile, which is dead between the P V'
    // product and the next V load.
    static constexpr uint32_t kGnPart = kV;              // [128] float2: second warpgroup's partials
    static constexpr uint32_t kGnStat = kV + 1024;       // [128] float2: per-row mean and scale
    static constexpr uint32_t kGnXchg = kV + 2048;       // [cluster rank][128] float2
};

constexpr uint32_t kIdescS = idesc_bf16(128, 128, 0, 0);   // Q^ (K-major) x K^ (K-major)
constexpr uint32_t kIdescX = idesc_bf16(128, kTV, 0, 1);   // Q^ x Rbar (MN-major)
constexpr uint32_t kIdescPV = idesc_bf16(128, kTV, 0, 1);  // P (tmem) x V' (MN-major)
constexpr uint32_t kIdescU = idesc_bf16(128, kTV, 1, 1);   // K^^T (MN-major) x V' (MN-major)

__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                         int *status) {
    const long long start = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (*abort_flag) return false;
        if (clock64() - start > kTimeoutCycles) {
            *abort_flag = 1;
            atomicExch(status, (int)RET_ERR_TIMEOUT);
            return false;
        }
    }
    return true;
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&v);
}

__device__ __forceinline__ float2 unpack_bf16(uint32_t u) {
    return __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&u));
}

// Row d of Rbar (MN-major B operand: blocks of 64 columns, each DK rows of
// 128 bytes, 128-byte swizzle): 32 values from column col0.
template <int DK>
__device__ __forceinline__ void st_rbar_row32(uint8_t *rbar, int d, int col0, const float *v) {
    const int blk = col0 >> 6;
    const int ch0 = (col0 & 63) >> 3;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint4 w;
        w.x = pack_bf16(v[8 * q + 0], v[8 * q + 1]);
        w.y = pack_bf16(v[8 * q + 2], v[8 * q + 3]);
        w.z = pack_bf16(v[8 * q + 4], v[8 * q + 5]);
        w.w = pack_bf16(v[8 * q + 6], v[8 * q + 7]);
        const int phys = (ch0 + q) ^ (d & 7);
        *reinterpret_cast<uint4 *>(rbar + blk * (DK * 128) + d * 128 + phys * 16) = w;
    }
}

// xPos turn of one [128 x DK] K-major swizzled tile in place.  Thread ->
// (16-byte column chunk = 4 pairs, starting row r0); it walks rows r0,
// r0+RS, ... and advances its four angles by RS*theta_j per step.
template <int DK>
__device__ void rotate_tile(uint8_t *tile, const float2 *rotstep, const Params &p, int t0, int n,
                            int tid) {
    constexpr int NCH = DK / 8;
    constexpr int RS = kThreads / NCH;
    const int c16 = tid % NCH;
    const int r0 = tid / NCH;
    const int blk = c16 >> 3, cw = c16 & 7;
    float c[4], s[4], sc[4], ss[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const int j = c16 * 4 + e;
        rot_cs(p.pos_offset + t0 + r0, p.theta[j], &c[e], &s[e]);
        sc[e] = rotstep[j].x;
        ss[e] = rotstep[j].y;
    }
#pragma unroll 2
    for (int r = r0; r < n; r += RS) {
        uint4 *ptr = reinterpret_cast<uint4 *>(tile + blk * 16384 + r * 128 + ((cw ^ (r & 7)) << 4));
        uint4 w = *ptr;
        uint32_t *u = reinterpret_cast<uint32_t *>(&w);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 x = unpack_bf16(u[e]);
            u[e] = pack_bf16(x.x * c[e] - x.y * s[e], x.x * s[e] + x.y * c[e]);
            const float cn = c[e] * sc[e] - s[e] * ss[e];
            s[e] = c[e] * ss[e] + s[e] * sc[e];
            c[e] = cn;
        }
        *ptr = w;
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

template <int DK, typename TO, bool FUSE>
__global__ void __launch_bounds__(kThreads, 1)
chunkwise_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const Params p,
                    const float *__restrict__ state_in, float *__restrict__ state_out,
                    TO *__restrict__ O, const __nv_bfloat16 *__restrict__ G, TO *__restrict__ Y,
                    float gn_eps, int *status) {
    using Ly = Layout<DK>;
    constexpr int NH = DK / 128;   // state halves of 128 rows
    constexpr int KB = DK / 64;    // 64-column blocks of Q^, K^
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t sbase = smem_u32(smem);
    const int tid = threadIdx.x, warp = tid >> 5;
    const int wg = tid >> 7;        // warpgroup
    const int row = tid & 127;      // TMEM lane of this thread
    const int bh = blockIdx.y, h = bh % p.H;
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
    float2 *rotstep = reinterpret_cast<float2 *>(smem + Ly::kRotStep);

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
    constexpr int kRS = kThreads / (DK / 8);
    if (p.rotate)
        for (int j = tid; j < DK / 2; j += kThreads) {
            float c, s;
            rot_cs(kRS, p.theta[j], &c, &s);
            rotstep[j] = make_float2(c, s);
        }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + Ly::kTmemSlot);
    const uint32_t tS = tmem, tO = tmem + 128, tR = tmem + 256;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    // Ownership of the state columns in the R passes: with two halves each
    // warpgroup takes one half; with one half they split its 128 columns.
    const int r_half = (NH == 2) ? wg : 0;
    const int r_col0 = (NH == 2) ? 0 : wg * 64;
    const int r_groups = (NH == 2) ? 4 : 2;
    const int r_d = r_half * 128 + row;
    // O / P: each warpgroup owns 64 columns of a row.
    const int o_col0 = wg * 64;

    auto load_q = [&](int c) {
        mbar_expect_tx(bar(BQ), Ly::kQBytes);
        for (int kb = 0; kb < KB; ++kb)
            tma_load_3d(sbase + Ly::kQ + kb * 16384, &tmQ, bar(BQ), kb * 64, c * kC, bh);
    };
    auto load_k = [&](int c) {
        mbar_expect_tx(bar(BK), Ly::kQBytes);
        for (int kb = 0; kb < KB; ++kb)
            tma_load_3d(sbase + Ly::kK + kb * 16384, &tmK, bar(BK), kb * 64, c * kC, bh);
    };
    auto load_v = [&](int c) {
        mbar_expect_tx(bar(BV), Ly::kVBytes);
        for (int nb = 0; nb < 2; ++nb)
            tma_load_3d(sbase + Ly::kV + nb * 16384, &tmV, bar(BV), v0 + nb * 64, c * kC, bh);
    };
    auto vdesc = [&](int ks) { return sdesc_sw128(sbase + Ly::kV + ks * 2048, 16384, 1024); };
    auto sync_alive = [&]() {
        __syncthreads();
        return *abort_flag == 0;
    };

    if (tid == 0) {
        load_q(0);
        load_k(0);
        load_v(0);
    }

    // starting state: TMEM R = gamma^{n_0} S_in and Rbar = bf16 of the same
    const bool has_in = state_in != nullptr;
    if (has_in) {
        const float g0 = decay_pow(lg, min(kC, L));
        const float *src = state_in + ((size_t)bh * DK + r_d) * dv + v0;
        for (int g = 0; g < r_groups; ++g) {
            const int col = r_col0 + 32 * g;
            float v[32];
            uint32_t r[32];
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
                const float4 x = *reinterpret_cast<const float4 *>(src + col + i);
                v[i] = x.x * g0; v[i + 1] = x.y * g0; v[i + 2] = x.z * g0; v[i + 3] = x.w * g0;
            }
            st_rbar_row32<DK>(smem + Ly::kR, r_d, col, v);
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(v[i]);
            tmem_st32(tR + r_half * 128 + lane_base + col, r);
        }
        tmem_wait_st();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    bool alive = sync_alive();

#pragma unroll 1
    for (int c = 0; c < nchunks; ++c) {
        const uint32_t par = c & 1;  // every barrier completes once per chunk
        const int t0 = c * kC;
        const int n = min(kC, L - t0);
        const bool has_state = has_in || c > 0;
        const bool last = c + 1 == nchunks;

        // ---- rotate Q and K of this chunk in place
        if (alive) {
            wait_bar(bar(BQ), par, abort_flag, status);
            wait_bar(bar(BK), par, abort_flag, status);
        }
        alive = sync_alive();
        if (alive && p.rotate) {
            rotate_tile<DK>(smem + Ly::kQ, rotstep, p, t0, n, tid);
            rotate_tile<DK>(smem + Ly::kK, rotstep, p, t0, n, tid);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        // ---- S = Q^ K^^T ; O'' = Q^ Rbar
        if (alive && tid == 0) {
            tc_fence_after();
#pragma unroll 1
            for (int ks = 0; ks < DK / 16; ++ks) {
                const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
                mma_ss(tS, sdesc_sw128(sbase + Ly::kQ + off, 16, 1024),
                       sdesc_sw128(sbase + Ly::kK + off, 16, 1024), kIdescS, ks > 0);
            }
            mma_commit(bar(BS));
            if (has_state) {
#pragma unroll 1
                for (int ks = 0; ks < DK / 16; ++ks) {
                    const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
                    mma_ss(tO, sdesc_sw128(sbase + Ly::kQ + off, 16, 1024),
                           sdesc_sw128(sbase + Ly::kR + ks * 2048, DK * 128, 1024), kIdescX, ks > 0);
                }
            }
            mma_commit(bar(BX));
        }

        // ---- V' = diag(zeta) V in place, while the MMAs run
        if (alive) wait_bar(bar(BV), par, abort_flag, status);
        alive = sync_alive();
        if (alive) {
            const float zeta = row < n ? decay_pow(lg, n - 1 - row) : 0.f;
            uint8_t *vrow = smem + Ly::kV + wg * 16384 + row * 128;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                uint4 *ptr = reinterpret_cast<uint4 *>(vrow + (((q + row) & 7) << 4));
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
        fence_proxy_async_smem();

        // ---- P = bf16(S) on j' <= j, else 0, into tensor memory
        if (alive) wait_bar(bar(BS), par, abort_flag, status);
        alive = sync_alive();
        tc_fence_after();
        if (alive) {
            uint32_t a[32], bb[32], pk[32];
            tmem_ld32(tS + lane_base + o_col0, a);
            tmem_ld32(tS + lane_base + o_col0 + 32, bb);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int k0 = o_col0 + 2 * i, k1 = o_col0 + 32 + 2 * i;
                pk[i] = pack_bf16(k0 <= row ? __uint_as_float(a[2 * i]) : 0.f,
                                  k0 + 1 <= row ? __uint_as_float(a[2 * i + 1]) : 0.f);
                pk[16 + i] = pack_bf16(k1 <= row ? __uint_as_float(bb[2 * i]) : 0.f,
                                       k1 + 1 <= row ? __uint_as_float(bb[2 * i + 1]) : 0.f);
            }
            // keys [0,64) -> columns [0,32), keys [64,128) -> columns [64,96)
            tmem_st32(tS + lane_base + o_col0, pk);
            tmem_wait_st();
        }
        tc_fence_before();
        __syncthreads();

        // ---- R += K^^T V' ; O'' += P V'
        if (alive && tid == 0) {
            tc_fence_after();
#pragma unroll 1
            for (int hh = 0; hh < NH; ++hh)
#pragma unroll 1
                for (int ks = 0; ks < kC / 16; ++ks)
                    mma_ss(tR + hh * 128, sdesc_sw128(sbase + Ly::kK + hh * 32768 + ks * 2048, 16384, 1024),
                           vdesc(ks), kIdescU, (ks > 0 || has_state) ? 1u : 0u);
            mma_commit(bar(BU));
#pragma unroll 1
            for (int ks = 0; ks < kC / 16; ++ks)
                mma_ts(tO, tS + (ks >> 2) * 64 + (ks & 3) * 8, vdesc(ks), kIdescPV,
                       (ks > 0 || has_state) ? 1u : 0u);
            mma_commit(bar(BPV));
            // Q^ is dead once S and O'' = Q^ Rbar are done: fetch the next Q
            if (!last && wait_bar(bar(BX), par, abort_flag, status)) load_q(c + 1);
        }

        // ---- state: R -> gamma^{n'} R in TMEM and Rbar; or state_out
        if (alive) wait_bar(bar(BU), par, abort_flag, status);
        alive = sync_alive();
        tc_fence_after();
        if (alive && tid == 0 && !last) load_k(c + 1);
        if (alive) {
            const float gnext = last ? 1.f : decay_pow(lg, min(kC, L - t0 - kC));
#pragma unroll 1
            for (int g = 0; g < r_groups; ++g) {
                const int col = r_col0 + 32 * g;
                uint32_t r[32];
                float v[32];
                tmem_ld32(tR + r_half * 128 + lane_base + col, r);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]) * gnext;
                if (last) {
                    if (state_out) st_row32<float>(state_out + ((size_t)bh * DK + r_d) * dv + v0 + col, v);
                } else {
                    st_rbar_row32<DK>(smem + Ly::kR, r_d, col, v);
#pragma unroll
                    for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(v[i]);
                    tmem_st32(tR + r_half * 128 + lane_base + col, r);
                }
            }
            tmem_wait_st();
        }

        // ---- epilogue: o_j = alpha_j O''_j (and the fused GroupNorm + gate)
        if (alive) wait_bar(bar(BPV), par, abort_flag, status);
        alive = sync_alive();
        tc_fence_after();
        const float alpha = exp2f((float)(row + 1 - n) * lg);  // gamma^{row+1-n}, lg finite here
        float x[64];
        if (alive) {
            uint32_t a[32], bb[32];
            tmem_ld32(tO + lane_base + o_col0, a);
            tmem_ld32(tO + lane_base + o_col0 + 32, bb);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                x[i] = __uint_as_float(a[i]);
                x[32 + i] = __uint_as_float(bb[i]);
            }
        }
        const size_t orow = ((size_t)bh * L + t0 + row) * dv + v0 + o_col0;
        if constexpr (!FUSE) {
            if (alive && row < n) {
                float y[64];
#pragma unroll
                for (int i = 0; i < 64; ++i) y[i] = x[i] * alpha;
                st_row32<TO>(O + orow, y);
                st_row32<TO>(O + orow + 32, y + 32);
            }
        } else {
            const int nr = (int)gridDim.x;        // CTAs of this head = cluster size
            const uint32_t rank = cluster_rank();
            const int b = bh / p.H;
            const size_t grow = ((size_t)b * L + t0 + row) * ((size_t)p.H * dv) + (size_t)h * dv + v0 + o_col0;
            uint4 gv[8];
            if (alive && row < n) {
#pragma unroll
                for (int q = 0; q < 8; ++q) gv[q] = *reinterpret_cast<const uint4 *>(G + grow + 8 * q);
            }
            float2 *part = reinterpret_cast<float2 *>(smem + Ly::kGnPart);
            float2 *stat = reinterpret_cast<float2 *>(smem + Ly::kGnStat);
            const float2 *xchg = reinterpret_cast<const float2 *>(smem + Ly::kGnXchg);
            // CTA-local mean and centred sum of squares of the row's 128 columns
            float s = 0.f;
#pragma unroll
            for (int i = 0; i < 64; ++i) s += x[i];
            if (wg == 1) part[row].x = s;
            __syncthreads();
            if (wg == 0) stat[row].x = (s + part[row].x) * (1.f / kTV);
            __syncthreads();
            const float mc = stat[row].x;
            float q2 = 0.f;
#pragma unroll
            for (int i = 0; i < 64; ++i) q2 = fmaf(x[i] - mc, x[i] - mc, q2);
            if (wg == 1) part[row].y = q2;
            // every CTA of the head is past its P V' product: V tiles are free
            cluster_sync();
            if (alive && wg == 0) {
                const float m2c = q2 + part[row].y;
                const uint32_t slot = sbase + Ly::kGnXchg + (rank * 128 + row) * 8;
                for (int r = 0; r < nr; ++r) st_cluster_f32x2(map_to_rank(slot, r), mc, m2c);
            }
            cluster_sync();
            if (alive && wg == 0) {
                float mean = 0.f;
                for (int r = 0; r < nr; ++r) mean += xchg[r * 128 + row].x;
                mean /= (float)nr;
                float m2 = 0.f;
                for (int r = 0; r < nr; ++r) {
                    const float2 e = xchg[r * 128 + row];
                    m2 += e.y + (float)kTV * (e.x - mean) * (e.x - mean);
                }
                const float var = m2 / (float)(nr * kTV);   // of O'' ; O = alpha O''
                stat[row] = make_float2(mean, alpha * rsqrtf(alpha * alpha * var + gn_eps));
            }
            __syncthreads();
            if (alive && row < n) {
                const float2 ms = stat[row];
                float y[64];
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const uint32_t *u = reinterpret_cast<const uint32_t *>(&gv[q]);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 g2 = unpack_bf16(u[e]);
                        const int i = 8 * q + 2 * e;
                        y[i] = g2.x / (1.f + expf(-g2.x)) * ((x[i] - ms.x) * ms.y);
                        y[i + 1] = g2.y / (1.f + expf(-g2.y)) * ((x[i + 1] - ms.x) * ms.y);
                    }
                }
                st_row32<TO>(Y + grow, y);
                st_row32<TO>(Y + grow + 32, y + 32);
                if (O) {
#pragma unroll
                    for (int i = 0; i < 64; ++i) y[i] = x[i] * alpha;
                    st_row32<TO>(O + orow, y);
                    st_row32<TO>(O + orow + 32, y + 32);
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        // the V tile (and the GroupNorm scratch in it) is free: next V
        if (alive && tid == 0 && !last) load_v(c + 1);
    }

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
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return static_cast<EncodeTiledFn>(nullptr);
        return reinterpret_cast<EncodeTiledFn>(f);
    }();
    return fn;
}

// [bh][rows][inner] bf16, boxes of 64 x 128 x 1 with 128-byte swizzle; rows
// past the end of a (b,h) slice read as zeros.
bool make_map(CUtensorMap *m, const void *base, int inner, int rows, int bh) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)rows, (cuuint64_t)bh};
    cuuint64_t strides[2] = {(cuuint64_t)inner * 2, (cuuint64_t)rows * inner * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)kC, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int DK, typename TO, bool FUSE>
cudaError_t launch_t(const Params &p, const CUtensorMap &mq, const CUtensorMap &mk,
                     const CUtensorMap &mv, const float *s_in, float *s_out, void *O,
                     const void *G, void *Y, float eps, int *status, cudaStream_t st) {
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
    e = cudaLaunchKernelEx(&cfg, kern, mq, mk, mv, p, s_in, s_out, (TO *)O,
                           (const __nv_bfloat16 *)G, (TO *)Y, eps, status);
    if (e == cudaSuccess) note_launches(1);
    return e;
}

template <int DK>
cudaError_t launch_dk(const Params &p, bool out_bf16, const CUtensorMap &mq, const CUtensorMap &mk,
                      const CUtensorMap &mv, const float *s_in, float *s_out, void *O,
                      const void *G, void *Y, float eps, int *status, cudaStream_t st) {
    const bool fuse = Y != nullptr;
    if (out_bf16)
        return fuse ? launch_t<DK, __nv_bfloat16, true>(p, mq, mk, mv, s_in, s_out, O, G, Y, eps, status, st)
                    : launch_t<DK, __nv_bfloat16, false>(p, mq, mk, mv, s_in, s_out, O, G, Y, eps, status, st);
    return fuse ? launch_t<DK, float, true>(p, mq, mk, mv, s_in, s_out, O, G, Y, eps, status, st)
                : launch_t<DK, float, false>(p, mq, mk, mv, s_in, s_out, O, G, Y, eps, status, st);
}

}  // namespace

bool chunkwise_tc_supported(const Params &p, int chunk, bool in_bf16) {
    if (!in_bf16 || chunk != kC || (p.dk != 128 && p.dk != 256) || p.dv % kTV != 0 ||
        p.dv / kTV > kMaxCluster || p.L < 1 || p.B * p.H < 1 || (long long)p.B * p.H > 65535)
        return false;
    for (int h = 0; h < p.H; ++h)
        if (!(p.log2g[h] * kC >= kMinLog2GammaTimesC)) return false;  // also rejects gamma = 0
    return true;
}

cudaError_t launch_chunkwise_tc(const Params &p, bool out_bf16, const void *Q, const void *K,
                                const void *V, const float *s_in, float *s_out, void *O,
                                const void *G, void *Y, float eps, int *status, cudaStream_t st) {
    CUtensorMap mq, mk, mv;
    const int bh = p.B * p.H;
    if (!make_map(&mq, Q, p.dk, p.L, bh) || !make_map(&mk, K, p.dk, p.L, bh) ||
        !make_map(&mv, V, p.dv, p.L, bh))
        return cudaErrorInvalidValue;
    if (p.dk == 256) return launch_dk<256>(p, out_bf16, mq, mk, mv, s_in, s_out, O, G, Y, eps, status, st);
    return launch_dk<128>(p, out_bf16, mq, mk, mv, s_in, s_out, O, G, Y, eps, status, st);
}

}  // namespace ret
