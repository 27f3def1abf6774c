// chunkwise_tc.cu -- chunkwise retention on the sm_100a tensor cores.
//
// "Retentive Network" paper summary, section 2.1, chunkwise recurrent form
// (3): parallel inside a chunk, a decayed state carried between chunks.  For
// the chunk of n rows starting after state R (rows j, keys j' < n):
//   S = Q^ K^^T                         (tcgen05, 128 x 128 x d_k)
//   P = S (.) D,  D[j][j'] = gamma^{j-j'} for j' <= j, else 0
//   O = diag(xi) (Q^ Rbar) + P V        xi_j = gamma^{j+1}
//   R <- gamma^n R + (diag(zeta) K^)^T V     zeta_j = gamma^{n-1-j}
// with Q^, K^ the xPos-rotated rows and Rbar the bf16 copy of R.
//
// One CTA owns one (b, h) and a 128-column slice of V, and walks the chunks
// in order.  Tensor memory (512 columns) holds S [128 x 128], O [128 x 128]
// and the fp32 state slice R [d_k x 128] as d_k/128 halves of 128 lanes.
// Shared memory holds the TMA-loaded Q, K, V tiles (128-byte swizzle; P
// reuses Q's space once Q^ is consumed) and Rbar in the MN-major layout the
// tensor core reads as its B operand.  CUDA-core passes between the MMA
// batches rotate Q and K in place, apply the decay to S, scale the carried
// term by xi and K^ by zeta, and move R between TMEM, its bf16 copy and
// (after the last chunk) the caller's state_out.
//
// Every mbarrier wait is bounded: on expiry the kernel latches
// RET_ERR_TIMEOUT in the device status word, all threads leave the loop
// together, in-flight copies and MMAs get a bounded drain, TMEM is freed.
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
constexpr long long kTimeoutCycles = 4000000000LL;  // about 2 s

template <int DK>
struct Layout {
    static constexpr uint32_t kQ = 0;                    // Q^ (later P): DK/64 blocks of 16 KB
    static constexpr uint32_t kQBytes = kC * DK * 2;
    static constexpr uint32_t kK = kQ + kQBytes;         // K^ (then zeta K^)
    static constexpr uint32_t kV = kK + kQBytes;         // V slice: 2 blocks of 16 KB
    static constexpr uint32_t kVBytes = kC * kTV * 2;
    static constexpr uint32_t kR = kV + kVBytes;         // Rbar: 2 column blocks of DK*128 B
    static constexpr uint32_t kRBytes = DK * kTV * 2;
    static constexpr uint32_t kP = kQ;
    static constexpr uint32_t kSmall = kR + kRBytes;
    static constexpr uint32_t kBarLoad = kSmall;
    static constexpr uint32_t kBarMma = kSmall + 8;
    static constexpr uint32_t kTmemSlot = kSmall + 16;
    static constexpr uint32_t kAbort = kSmall + 20;
    static constexpr uint32_t kColScale = kSmall + 32;   // 128 floats
    static constexpr uint32_t kRotStep = kColScale + 512;  // DK/2 float2
    static constexpr uint32_t kBytes = kRotStep + DK * 4;
};

constexpr uint32_t kIdescS = idesc_bf16(128, 128, 0, 0);   // Q^ (K-major) x K^ (K-major)
constexpr uint32_t kIdescX = idesc_bf16(128, kTV, 0, 1);   // Q^ x Rbar (MN-major)
constexpr uint32_t kIdescPV = idesc_bf16(128, kTV, 0, 1);  // P x V (MN-major)
constexpr uint32_t kIdescU = idesc_bf16(128, kTV, 1, 1);   // (zeta K^)^T (MN-major) x V

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

// Row `row` of a K-major, 128-byte-swizzled tile (64 bf16 per 128-byte row
// segment, blocks of 128 rows): 32 values starting at column `col0`
// (a multiple of 32).
__device__ __forceinline__ void st_kmajor_row32(uint8_t *tile, int row, int col0, const float *v) {
    const int blk = col0 >> 6;
    const int ch0 = (col0 & 63) >> 3;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint4 w;
        w.x = pack_bf16(v[8 * q + 0], v[8 * q + 1]);
        w.y = pack_bf16(v[8 * q + 2], v[8 * q + 3]);
        w.z = pack_bf16(v[8 * q + 4], v[8 * q + 5]);
        w.w = pack_bf16(v[8 * q + 6], v[8 * q + 7]);
        const int phys = (ch0 + q) ^ (row & 7);
        *reinterpret_cast<uint4 *>(tile + blk * 16384 + row * 128 + phys * 16) = w;
    }
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

// xPos turn of the Q and K tiles in place.  Thread -> (tile, 16-byte column
// chunk = 4 pairs, starting row r0); it walks rows r0, r0+RS, ... and steps
// its four angles by RS*theta_j with a complex multiply each row.
template <int DK>
__device__ void rotate_qk(uint8_t *q, uint8_t *k, const float2 *rotstep, const Params &p,
                          int t0, int n, int tid) {
    constexpr int NCH = DK / 8;
    constexpr int RS = kThreads / (2 * NCH);
    const int c16 = tid % NCH;
    const int rest = tid / NCH;
    uint8_t *base = rest < RS ? q : k;
    const int r0 = rest % RS;
    const int blk = c16 >> 3, cw = c16 & 7;
    float c[4], s[4], sc[4], ss[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const int j = c16 * 4 + e;
        rot_cs(p.pos_offset + t0 + r0, p.theta[j], &c[e], &s[e]);
        sc[e] = rotstep[j].x;
        ss[e] = rotstep[j].y;
    }
    for (int r = r0; r < n; r += RS) {
        uint4 *ptr = reinterpret_cast<uint4 *>(base + blk * 16384 + r * 128 + ((cw ^ (r & 7)) << 4));
        uint4 w = *ptr;
        uint32_t *u = reinterpret_cast<uint32_t *>(&w);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            float2 x = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&u[e]));
            float y0 = x.x * c[e] - x.y * s[e];
            float y1 = x.x * s[e] + x.y * c[e];
            u[e] = pack_bf16(y0, y1);
            float cn = c[e] * sc[e] - s[e] * ss[e];
            s[e] = c[e] * ss[e] + s[e] * sc[e];
            c[e] = cn;
        }
        *ptr = w;
    }
}

template <typename TO>
__device__ __forceinline__ void st_out32(TO *dst, const float *v);
template <>
__device__ __forceinline__ void st_out32<float>(float *dst, const float *v) {
#pragma unroll
    for (int i = 0; i < 32; i += 4)
        *reinterpret_cast<float4 *>(dst + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
}
template <>
__device__ __forceinline__ void st_out32<__nv_bfloat16>(__nv_bfloat16 *dst, const float *v) {
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

template <int DK, typename TO>
__global__ void __launch_bounds__(kThreads, 1)
chunkwise_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const Params p,
                    const float *__restrict__ state_in, float *__restrict__ state_out,
                    TO *__restrict__ O, int *status) {
    using Ly = Layout<DK>;
    constexpr int NH = DK / 128;
    constexpr int KB = DK / 64;
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t sbase = smem_u32(smem);
    const int tid = threadIdx.x, warp = tid >> 5;
    const int bh = blockIdx.y, h = bh % p.H;
    const int v0 = blockIdx.x * kTV;
    const float lg = p.log2g[h];
    const int L = p.L, dv = p.dv;
    const int nchunks = (L + kC - 1) / kC;

    if (sbase & 1023u) {  // swizzle atoms need 1024-byte alignment
        if (tid == 0) atomicExch(status, (int)RET_ERR_CUDA);
        return;
    }
    const uint32_t bar_load = sbase + Ly::kBarLoad, bar_mma = sbase + Ly::kBarMma;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Ly::kAbort);
    float *colscale = reinterpret_cast<float *>(smem + Ly::kColScale);
    float2 *rotstep = reinterpret_cast<float2 *>(smem + Ly::kRotStep);

    if (tid == 0) {
        mbar_init(bar_load, 1);
        mbar_init(bar_mma, 1);
        *abort_flag = 0;
        fence_mbar_init();
        fence_proxy_async_smem();
    }
    if (warp == 0) {
        tmem_alloc(sbase + Ly::kTmemSlot, 512);
        tmem_relinquish();
    }
    // gamma^{j-j'} = gamma^{j-64} * gamma^{64-j'} while gamma^-64 stays far
    // from overflow; otherwise one exp2 per element.
    const bool fast = (64.f * lg >= -120.f);
    for (int j = tid; j < kC; j += kThreads) colscale[j] = fast ? exp2f((float)(64 - j) * lg) : 0.f;
    constexpr int kRS = kThreads / (2 * DK / 8);
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
    const int row = tid & 127;  // TMEM lane of this thread (both warpgroups)

    auto issue_loads = [&](int c) {
        const int t0 = c * kC;
        mbar_expect_tx(bar_load, 2 * Ly::kQBytes + Ly::kVBytes);
        for (int kb = 0; kb < KB; ++kb)
            tma_load_3d(sbase + Ly::kQ + kb * 16384, &tmQ, bar_load, kb * 64, t0, bh);
        for (int kb = 0; kb < KB; ++kb)
            tma_load_3d(sbase + Ly::kK + kb * 16384, &tmK, bar_load, kb * 64, t0, bh);
        for (int nb = 0; nb < 2; ++nb)
            tma_load_3d(sbase + Ly::kV + nb * 16384, &tmV, bar_load, v0 + nb * 64, t0, bh);
    };
    bool load_pending = false, mma_pending = false;
    uint32_t load_parity = 0;
    if (tid == 0) {
        issue_loads(0);
        load_pending = true;
    }

    // starting state: TMEM R = gamma^{n_0} S_in, Rbar = bf16(S_in)
    const bool has_in = state_in != nullptr;
    if (has_in && tid < 128) {
        const float g0 = decay_pow(lg, min(kC, L));
        for (int hh = 0; hh < NH; ++hh) {
            const int d = hh * 128 + tid;
            const float *src = state_in + ((size_t)bh * DK + d) * dv + v0;
            for (int cb = 0; cb < 4; ++cb) {
                float v[32];
                uint32_t r[32];
#pragma unroll
                for (int i = 0; i < 32; i += 4) {
                    float4 x = *reinterpret_cast<const float4 *>(src + cb * 32 + i);
                    v[i] = x.x; v[i + 1] = x.y; v[i + 2] = x.z; v[i + 3] = x.w;
                }
                st_rbar_row32<DK>(smem + Ly::kR, d, cb * 32, v);
#pragma unroll
                for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(v[i] * g0);
                tmem_st32(tR + hh * 128 + lane_base + cb * 32, r);
            }
        }
        tmem_wait_st();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();

    uint32_t mma_parity = 0;
    for (int c = 0; c < nchunks; ++c) {
        const int t0 = c * kC;
        const int n = min(kC, L - t0);
        const bool has_state = has_in || c > 0;

        wait_bar(bar_load, c & 1, abort_flag, status);
        __syncthreads();
        if (*abort_flag) break;
        load_pending = false;

        if (p.rotate) rotate_qk<DK>(smem + Ly::kQ, smem + Ly::kK, rotstep, p, t0, n, tid);
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        // MMA batch 1: S = Q^ K^^T ; O = Q^ Rbar
        if (tid == 0) {
            tc_fence_after();
#pragma unroll 1
            for (int ks = 0; ks < DK / 16; ++ks) {
                const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
                mma_ss(tS, sdesc_sw128(sbase + Ly::kQ + off, 16, 1024),
                       sdesc_sw128(sbase + Ly::kK + off, 16, 1024), kIdescS, ks > 0);
            }
            if (has_state) {
#pragma unroll 1
                for (int ks = 0; ks < DK / 16; ++ks) {
                    const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
                    mma_ss(tO, sdesc_sw128(sbase + Ly::kQ + off, 16, 1024),
                           sdesc_sw128(sbase + Ly::kR + ks * 2048, DK * 128, 1024), kIdescX, ks > 0);
                }
            }
            mma_commit(bar_mma);
            mma_pending = true;
        }
        wait_bar(bar_mma, mma_parity, abort_flag, status);
        mma_parity ^= 1;
        __syncthreads();
        if (*abort_flag) break;
        mma_pending = false;
        tc_fence_after();

        if (tid < 128) {
            // P = S (.) D into the P tile; carried term scaled by xi
            const float a_j = fast ? exp2f((float)(row - 64) * lg) : 0.f;
#pragma unroll 1
            for (int cb = 0; cb < 4; ++cb) {
                uint32_t r[32];
                float v[32];
                tmem_ld32(tS + lane_base + cb * 32, r);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int jj = cb * 32 + i;
                    float w = 0.f;
                    if (jj <= row) w = fast ? a_j * colscale[jj] : decay_pow(lg, row - jj);
                    v[i] = __uint_as_float(r[i]) * w;
                }
                st_kmajor_row32(smem + Ly::kP, row, cb * 32, v);
            }
            if (has_state) {
                const float xi = decay_pow(lg, row + 1);
#pragma unroll 1
                for (int cb = 0; cb < 4; ++cb) {
                    uint32_t r[32];
                    tmem_ld32(tO + lane_base + cb * 32, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * xi);
                    tmem_st32(tO + lane_base + cb * 32, r);
                }
                tmem_wait_st();
            }
        } else {
            // zeta K^ in place (all chunks of row j get the same factor)
            const float zeta = row < n ? decay_pow(lg, n - 1 - row) : 0.f;
#pragma unroll 1
            for (int kb = 0; kb < KB; ++kb) {
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const int cc = (q + row) & 7;
                    uint4 *ptr = reinterpret_cast<uint4 *>(smem + Ly::kK + kb * 16384 + row * 128 + cc * 16);
                    uint4 w = *ptr;
                    uint32_t *u = reinterpret_cast<uint32_t *>(&w);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        float2 x = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&u[e]));
                        u[e] = pack_bf16(x.x * zeta, x.y * zeta);
                    }
                    *ptr = w;
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        // MMA batch 2: O += P V ; R += (zeta K^)^T V
        if (tid == 0) {
            tc_fence_after();
#pragma unroll 1
            for (int ks = 0; ks < kC / 16; ++ks) {
                const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
                mma_ss(tO, sdesc_sw128(sbase + Ly::kP + off, 16, 1024),
                       sdesc_sw128(sbase + Ly::kV + ks * 2048, 16384, 1024), kIdescPV,
                       (ks > 0 || has_state) ? 1u : 0u);
            }
#pragma unroll 1
            for (int hh = 0; hh < NH; ++hh)
#pragma unroll 1
                for (int ks = 0; ks < kC / 16; ++ks)
                    mma_ss(tR + hh * 128,
                           sdesc_sw128(sbase + Ly::kK + hh * 32768 + ks * 2048, 16384, 1024),
                           sdesc_sw128(sbase + Ly::kV + ks * 2048, 16384, 1024), kIdescU,
                           (ks > 0 || has_state) ? 1u : 0u);
            mma_commit(bar_mma);
            mma_pending = true;
        }
        wait_bar(bar_mma, mma_parity, abort_flag, status);
        mma_parity ^= 1;
        __syncthreads();
        if (*abort_flag) break;
        mma_pending = false;
        tc_fence_after();

        // Q, K, V and P are free: fetch the next chunk while R and O drain
        const bool last = (c + 1 == nchunks);
        if (tid == 0 && !last) {
            issue_loads(c + 1);
            load_pending = true;
            load_parity = (c + 1) & 1;
        }

        if (tid < 128) {
            const float gnext = last ? 0.f : decay_pow(lg, min(kC, L - t0 - kC));
#pragma unroll 1
            for (int hh = 0; hh < NH; ++hh) {
                const int d = hh * 128 + row;
#pragma unroll 1
                for (int cb = 0; cb < 4; ++cb) {
                    uint32_t r[32];
                    float v[32];
                    tmem_ld32(tR + hh * 128 + lane_base + cb * 32, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
                    if (last) {
                        if (state_out)
                            st_out32<float>(state_out + ((size_t)bh * DK + d) * dv + v0 + cb * 32, v);
                    } else {
                        st_rbar_row32<DK>(smem + Ly::kR, d, cb * 32, v);
#pragma unroll
                        for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(v[i] * gnext);
                        tmem_st32(tR + hh * 128 + lane_base + cb * 32, r);
                    }
                }
            }
            tmem_wait_st();
        } else {
#pragma unroll 1
            for (int cb = 0; cb < 4; ++cb) {
                uint32_t r[32];
                float v[32];
                tmem_ld32(tO + lane_base + cb * 32, r);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
                if (row < n) st_out32<TO>(O + ((size_t)bh * L + t0 + row) * dv + v0 + cb * 32, v);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
    }

    // After an abort, give copies and MMAs still in flight a bounded time to
    // land before the shared and tensor memory go away.
    if (tid == 0 && *abort_flag) {
        const long long start = clock64();
        while ((load_pending || mma_pending) && clock64() - start < kTimeoutCycles) {
            if (load_pending && mbar_try_wait(bar_load, load_parity)) load_pending = false;
            if (mma_pending && mbar_try_wait(bar_mma, mma_parity)) mma_pending = false;
        }
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

template <int DK, typename TO>
cudaError_t launch_t(const Params &p, const CUtensorMap &mq, const CUtensorMap &mk,
                     const CUtensorMap &mv, const float *s_in, float *s_out, void *O,
                     int *status, cudaStream_t st) {
    auto kern = chunkwise_tc_kernel<DK, TO>;
    const int smem = (int)Layout<DK>::kBytes;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    dim3 grid(p.dv / kTV, p.B * p.H);
    kern<<<grid, kThreads, smem, st>>>(mq, mk, mv, p, s_in, s_out, (TO *)O, status);
    e = cudaGetLastError();
    if (e == cudaSuccess) note_launches(1);
    return e;
}

}  // namespace

bool chunkwise_tc_supported(const Params &p, int chunk, bool in_bf16) {
    return in_bf16 && chunk == kC && (p.dk == 128 || p.dk == 256) && p.dv % kTV == 0 && p.L >= 1 &&
           (long long)p.B * p.H <= 65535 && p.B * p.H >= 1;
}

cudaError_t launch_chunkwise_tc(const Params &p, bool out_bf16, const void *Q, const void *K,
                                const void *V, const float *s_in, float *s_out, void *O,
                                int *status, cudaStream_t st) {
    CUtensorMap mq, mk, mv;
    const int bh = p.B * p.H;
    if (!make_map(&mq, Q, p.dk, p.L, bh) || !make_map(&mk, K, p.dk, p.L, bh) ||
        !make_map(&mv, V, p.dv, p.L, bh))
        return cudaErrorInvalidValue;
    if (p.dk == 256)
        return out_bf16 ? launch_t<256, __nv_bfloat16>(p, mq, mk, mv, s_in, s_out, O, status, st)
                        : launch_t<256, float>(p, mq, mk, mv, s_in, s_out, O, status, st);
    return out_bf16 ? launch_t<128, __nv_bfloat16>(p, mq, mk, mv, s_in, s_out, O, status, st)
                    : launch_t<128, float>(p, mq, mk, mv, s_in, s_out, O, status, st);
}

}  // namespace ret
