// gemm_tc.cu -- C = A B on the sm_100a tensor cores: the two dense
// projections of the multi-scale retention layer.
//
// "Retentive Network" paper summary, section 2.2: the layer forms
// Q, K, V (and the gate input X W_G) as products of X with the weight
// matrices, and multiplies the gated, normalised heads by W_O.  Both are
// plain products of a row-major bf16 matrix with a row-major bf16 weight
// matrix, accumulated in fp32 and stored as bf16:
//   C[M x N] = A[M x K] B[K x N]
//
// Persistent CTAs, in pairs (clusters of two, one CTA per SM): a pair walks
// output tiles of 256 x 256 (tile u, then u + pairs, ...; the N tiles of one
// row block are consecutive, so the pairs running at once share their A
// rows in L2 and the weights stay in L2).  Each CTA of a pair loads its own
// 128 rows of A and its own 128 columns of B, so an SM streams 32 KB per
// 64-deep stage for 256 x 256 x 64 products (a lone CTA with a 128 x 256
// tile would need 48 KB for half of that); the even CTA issues M = 256
// products that read the A rows and B columns of both CTAs and write each
// CTA's 128 result rows into its own tensor memory.  (M <= 128: one CTA per
// tile of 128 x 256, the same roles without the pairing.)  Roles (8 warps):
//   warp 0   issues the TMA loads of a stage (A: 128 rows x 64 k, K-major;
//            B: 64 k rows x 128 columns, two 64-column blocks, N-major)
//            once the products that read the stage before have completed;
//            the loads of both CTAs count on the even CTA's barrier
//   warp 1   (even CTA) issues the MMAs (one thread): per stage four
//            256 x 256 x 16 products into the tile's accumulator, then a
//            commit that frees the stage in both CTAs; after the last stage
//            of a tile a commit that hands the accumulators to both
//            epilogues
//   warps 4-7 the epilogue: each thread owns one row (its TMEM lane),
//            reads the accumulator 32 columns at a time, rounds to bf16
//            and stores 64-byte row pieces; then releases the accumulator
//            (an arrival on the even CTA's barrier)
// Tensor memory holds two accumulators (2 x 256 columns), so the epilogue
// of tile i runs while the tensor cores work on tile i+1.  Shared memory
// holds seven stages of 32 KB (four of 48 KB unpaired).
//
// Operands past M, N or K read as zeros from the TMA (so K needs no
// multiple of 64); stores past M or N are skipped (N a multiple of 8).
// Every wait is bounded (about 2 s of SM clock): on expiry the kernel
// latches RET_ERR_TIMEOUT in the device status word and every role leaves
// its loop; copies and MMAs in flight get a bounded drain before the
// shared and tensor memory are released.
#include <cuda.h>

#include <algorithm>

#include "common.cuh"
#include "launch.h"
#include "tc_util.cuh"

namespace ret {
namespace {

using namespace tc;

constexpr int kBM = 128, kBN = 256, kBK = 64;
constexpr int kThreads = 256;
constexpr uint32_t kABytes = kBM * kBK * 2;  // 16 KB: this CTA's 128 rows x 64 k
constexpr uint32_t kBBlock = kBK * 64 * 2;   // one 64-column block of B: 8 KB
constexpr long long kTimeoutCycles = 4000000000LL;  // about 2 s
constexpr int kProjBlock = 128;  // rows per block of the chunk loop the projection feeds

// PAIR: two CTAs of a cluster share each 256 x 256 tile: each loads its own
// 128 rows of A and its own 128 of the 256 columns of B, and the even CTA
// issues M = 256 products whose A rows and B columns come from both CTAs'
// shared memory and whose result rows land in each CTA's own tensor
// memory.  Alone: one CTA, a 128 x 256 tile, all of B's 256 columns.
template <bool PAIR>
struct Cfg {
    static constexpr int kStages = PAIR ? 7 : 4;
    static constexpr int kBCols = PAIR ? kBN / 2 : kBN;            // B columns loaded by a CTA
    static constexpr uint32_t kBBytes = kBBlock * (kBCols / 64);   // 16 or 32 KB
    static constexpr uint32_t kStageBytes = kABytes + kBBytes;     // 32 or 48 KB
    static constexpr uint32_t kData = kStages * kStageBytes;       // 224 or 192 KB
    // FULL[s]: stage s landed (the even CTA's barrier counts both CTAs'
    // bytes); EMPTY[s]: its products completed; ACCF[b]: accumulator b
    // final; ACCE[b]: accumulator b read out by the epilogue warps (of both
    // CTAs, counted at the even CTA)
    static constexpr int FULL = 0, EMPTY = kStages, ACCF = 2 * kStages, ACCE = 2 * kStages + 2,
                         kNumBars = 2 * kStages + 4;
    static constexpr uint32_t kBar = kData;
    static constexpr uint32_t kTmemSlot = kBar + 8 * kNumBars;
    static constexpr uint32_t kAbort = kTmemSlot + 4;
    static constexpr uint32_t kSmemBytes = kAbort + 4 + 1024;  // + alignment slack
    static constexpr uint32_t kIdesc = idesc_bf16(PAIR ? 2 * kBM : kBM, kBN, 0, 1);  // A K-major, B N-major
};

__device__ __forceinline__ uint32_t pack2(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&v);
}

// ---- the CTA-pair forms of the tcgen05 instructions (a kernel uses one
// cta_group throughout)
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void mma_ss_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrives on the barrier at `bar` (a shared-memory offset) in both CTAs of
// the pair once the products issued before have completed.
__device__ __forceinline__ void mma_commit_pair(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%0], %1;" ::"r"(bar), "h"((uint16_t)3)
        : "memory");
}
// TMA load into this CTA's shared memory whose completion is counted on a
// barrier of the pair (`bar_cluster`: a shared::cluster address, here the
// even CTA's).
__device__ __forceinline__ void tma_load_3d_pair(uint32_t dst, const CUtensorMap *map,
                                                 uint32_t bar_cluster, int c0, int c1, int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}
// One arrival on a barrier of the cluster (shared::cluster address),
// releasing this thread's earlier accesses at cluster scope.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(addr) : "memory");
}

// PROJ: C is the layer's projection P = X [W_Q | W_K | W_V | W_G] and the
// epilogue also does what the streaming pass would: the columns of the Q
// block leave turned by the xPos angles of their row's position, the
// columns of the K block turned and weighted by gamma_h^{n-1-j} (j the row's
// place in its block of 128 rows, n that block's rows), each into its own
// [B][H][L][d_k] array (qh, kt); only the V and G columns go to C.
template <bool PAIR, bool PROJ>
__global__ void __launch_bounds__(kThreads, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               int M, int N, int K, __nv_bfloat16 *__restrict__ C, long long ldc, int *status,
               const __grid_constant__ Params pp, __nv_bfloat16 *__restrict__ qh,
               __nv_bfloat16 *__restrict__ kt) {
    using G = Cfg<PAIR>;
    constexpr int kStages = G::kStages;
    extern __shared__ uint8_t smem_raw[];
    // swizzle atoms need 1024-byte alignment (the same offset in both CTAs
    // of a pair: the dynamic shared memory starts at the same address)
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(smem);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int rank = PAIR ? (int)cluster_rank() : 0;  // 0: the CTA that issues the products
    const int unit = PAIR ? (int)blockIdx.x / 2 : (int)blockIdx.x, units = PAIR ? (int)gridDim.x / 2 : (int)gridDim.x;
    constexpr int kTM = PAIR ? 2 * kBM : kBM;  // tile rows
    const int tiles_n = (N + kBN - 1) / kBN;
    const int ntiles = ((M + kTM - 1) / kTM) * tiles_n;
    const int kblocks = (K + kBK - 1) / kBK;

    auto bar = [&](int i) { return sbase + G::kBar + 8u * i; };
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + G::kAbort);
    auto wait = [&](int i, uint32_t parity) {
        return mbar_wait_bounded(bar(i), parity, abort_flag, status, kTimeoutCycles);
    };
    if (tid == 0) {
        for (int i = 0; i < G::kNumBars; ++i)
            mbar_init(bar(i), (i == G::ACCE || i == G::ACCE + 1) ? (PAIR ? 8 : 4) : 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 2) {
        if constexpr (PAIR) {
            tmem_alloc_pair(sbase + G::kTmemSlot, 512);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(sbase + G::kTmemSlot, 512);
            tmem_relinquish();
        }
    }
    tc_fence_before();
    __syncthreads();
    if constexpr (PAIR) cluster_sync();  // the peer's barriers exist before any remote arrival
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + G::kTmemSlot);
    // the barriers that count for a pair sit in the even CTA
    auto lead_bar = [&](int i) { return PAIR ? map_to_rank(bar(i), 0) : bar(i); };

    if (warp == 0 && lane == 0) {
        // ================================================= TMA producer
        long long it = 0;
        bool ok = true;
        for (int t = unit; t < ntiles && ok; t += units) {
            const int m0 = (t / tiles_n) * kTM + rank * kBM, n0 = (t % tiles_n) * kBN + rank * G::kBCols;
            for (int kb = 0; kb < kblocks; ++kb, ++it) {
                const int s = (int)(it % kStages);
                const uint32_t use = (uint32_t)(it / kStages);
                if (use > 0 && !wait(G::EMPTY + s, (use - 1) & 1)) {
                    ok = false;
                    break;
                }
                const uint32_t sa = sbase + s * G::kStageBytes, sb = sa + kABytes;
                if constexpr (PAIR) {
                    const uint32_t full = lead_bar(G::FULL + s);
                    if (rank == 0) mbar_expect_tx(bar(G::FULL + s), 2 * G::kStageBytes);
                    tma_load_3d_pair(sa, &tmA, full, kb * kBK, m0, 0);
#pragma unroll
                    for (int j = 0; j < G::kBCols / 64; ++j)
                        tma_load_3d_pair(sb + j * kBBlock, &tmB, full, n0 + 64 * j, kb * kBK, 0);
                } else {
                    mbar_expect_tx(bar(G::FULL + s), G::kStageBytes);
                    tma_load_3d(sa, &tmA, bar(G::FULL + s), kb * kBK, m0, 0);
#pragma unroll
                    for (int j = 0; j < G::kBCols / 64; ++j)
                        tma_load_3d(sb + j * kBBlock, &tmB, bar(G::FULL + s), n0 + 64 * j, kb * kBK, 0);
                }
            }
        }
        // every completion of this CTA's stages (for a pair: the arrivals
        // the other CTA's products send here) has landed before the CTA ends
        for (int s = 0; s < kStages && ok; ++s) {
            const long long uses = it / kStages + (s < it % kStages ? 1 : 0);
            if (uses > 0 && !wait(G::EMPTY + s, (uint32_t)(uses - 1) & 1)) ok = false;
        }
    } else if (warp == 1 && lane == 0 && rank == 0) {
        // ================================================= MMA issue
        long long it = 0;
        int tl = 0;  // tiles of this CTA so far
        bool ok = true;
        for (int t = unit; t < ntiles && ok; t += units, ++tl) {
            const int b = tl & 1;
            const uint32_t use = (uint32_t)(tl >> 1);
            // the epilogue has read this accumulator's previous tile
            if (use > 0 && !wait(G::ACCE + b, (use - 1) & 1)) break;
            tc_fence_after();
            const uint32_t d = tmem + b * kBN;
            for (int kb = 0; kb < kblocks; ++kb, ++it) {
                const int s = (int)(it % kStages);
                if (!wait(G::FULL + s, (uint32_t)(it / kStages) & 1)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t sa = sbase + s * G::kStageBytes, sb = sa + kABytes;
                const uint64_t da = sdesc_sw128(sa, 16, 1024);
                const uint64_t db = sdesc_sw128(sb, kBBlock, 1024);
#pragma unroll
                for (int ks = 0; ks < kBK / 16; ++ks) {
                    const uint64_t a = da + (uint64_t)((ks * 32) >> 4), bb = db + (uint64_t)((ks * 2048) >> 4);
                    const uint32_t acc = (kb > 0 || ks > 0) ? 1u : 0u;
                    if constexpr (PAIR) mma_ss_pair(d, a, bb, G::kIdesc, acc);
                    else mma_ss(d, a, bb, G::kIdesc, acc);
                }
                if constexpr (PAIR) mma_commit_pair(bar(G::EMPTY + s));
                else mma_commit(bar(G::EMPTY + s));
            }
            if (ok) {
                if constexpr (PAIR) mma_commit_pair(bar(G::ACCF + b));
                else mma_commit(bar(G::ACCF + b));
            }
        }
    } else if (warp >= 4) {
        // ================================================= epilogue
        const int quad = warp & 3;
        const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
        int tl = 0;
        for (int t = unit; t < ntiles; t += units, ++tl) {
            const int m0 = (t / tiles_n) * kTM + rank * kBM, n0 = (t % tiles_n) * kBN;
            const int b = tl & 1;
            if (!__all_sync(0xffffffffu, wait(G::ACCF + b, (uint32_t)(tl >> 1) & 1))) break;
            tc_fence_after();
            const int row = m0 + quad * 32 + lane;
            __nv_bfloat16 *crow = C + (size_t)row * ldc + n0;
            // (PROJ) this row's sequence, position and place in its block
            int pb = 0, pl = 0, pn = 0;
            if constexpr (PROJ) {
                pb = row / pp.L;
                pl = row - pb * pp.L;
                const int j0 = pl - pl % kProjBlock;
                pn = min(kProjBlock, pp.L - j0);
            }
#pragma unroll 1
            for (int c = 0; c < kBN / 32; ++c) {
                uint32_t x[32];
                tmem_ld32(tmem + lane_base + b * kBN + 32 * c, x);
                tmem_wait_ld(x);
                const int col0 = n0 + 32 * c;
                __nv_bfloat16 *dst = crow + 32 * c;
                if constexpr (PROJ) {
                    const int hdk = pp.H * pp.dk;
                    if (col0 < 2 * hdk) {
                        // a Q or K column chunk (32 columns of one head)
                        const bool key = col0 >= hdk;
                        const int cq = key ? col0 - hdk : col0;
                        const int h = cq / pp.dk, d0 = cq - h * pp.dk;
                        const float z = key ? decay_pow(pp.log2g[h], pn - 1 - (pl % kProjBlock)) : 1.f;
                        if (pp.rotate) {
                            const long long pos = pp.pos_offset + pl;
#pragma unroll
                            for (int e = 0; e < 16; ++e) {
                                float cs, sn;
                                rot_cs_fast(pos, pp.theta[d0 / 2 + e], &cs, &sn);
                                const float x0 = __uint_as_float(x[2 * e]), x1 = __uint_as_float(x[2 * e + 1]);
                                x[2 * e] = __float_as_uint(z * (x0 * cs - x1 * sn));
                                x[2 * e + 1] = __float_as_uint(z * (x0 * sn + x1 * cs));
                            }
                        } else if (key) {
#pragma unroll
                            for (int e = 0; e < 32; ++e) x[e] = __float_as_uint(z * __uint_as_float(x[e]));
                        }
                        dst = (key ? kt : qh) + (((size_t)pb * pp.H + h) * pp.L + pl) * pp.dk + d0;
                    } else {
                        dst = crow + 32 * c;
                    }
                }
                if (row < M) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int col = col0 + 8 * q;
                        if (col < N) {
                            uint4 w;
                            w.x = pack2(__uint_as_float(x[8 * q + 0]), __uint_as_float(x[8 * q + 1]));
                            w.y = pack2(__uint_as_float(x[8 * q + 2]), __uint_as_float(x[8 * q + 3]));
                            w.z = pack2(__uint_as_float(x[8 * q + 4]), __uint_as_float(x[8 * q + 5]));
                            w.w = pack2(__uint_as_float(x[8 * q + 6]), __uint_as_float(x[8 * q + 7]));
                            *reinterpret_cast<uint4 *>(dst + 8 * q) = w;
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if constexpr (PAIR) mbar_arrive_cluster(lead_bar(G::ACCE + b));
                else mbar_arrive(bar(G::ACCE + b));
            }
        }
    }

    __syncthreads();
    if (tid == 0 && *abort_flag) {
        const long long start = clock64();
        while (clock64() - start < 20000000LL) __nanosleep(1000);
    }
    tc_fence_before();
    __syncthreads();
    // a pair meets once more: neither CTA frees its tensor memory or leaves
    // while the other may still reach its shared memory
    if constexpr (PAIR) cluster_sync();
    if (warp == 2) {
        tc_fence_after();
        if constexpr (PAIR) tmem_dealloc_pair(tmem, 512);
        else tmem_dealloc(tmem, 512);
    }
}

int sm_count() {
    int dev = -1, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    return n;
}

}  // namespace

bool gemm_tc_supported(long long M, long long N, long long K, long long lda, long long ldb,
                       long long ldc) {
    return M >= 1 && N >= 8 && K >= 1 && M <= INT32_MAX && N <= INT32_MAX && K <= INT32_MAX &&
           N % 8 == 0 && lda % 8 == 0 && ldb % 8 == 0 && ldc % 8 == 0 && lda >= K && ldb >= N &&
           ldc >= N;
}

namespace {

template <bool PROJ>
cudaError_t launch_gemm(long long M, long long N, long long K, const void *A, long long lda,
                        const void *B, long long ldb, void *C, long long ldc, const Params &pp,
                        void *qh, void *kt, int *status, cudaStream_t st) {
    if (!gemm_tc_supported(M, N, K, lda, ldb, ldc)) return cudaErrorInvalidValue;
    // CTA pairs (256-row tiles) once there are enough rows to fill them
    const bool pair = M > kBM;
    const int tm = pair ? 2 * kBM : kBM;
    CUtensorMap ma, mb;
    if (!make_tma_map_bf16_strided(&ma, A, (int)K, (int)M, 1, lda, lda * M, kBM) ||
        !make_tma_map_bf16_strided(&mb, B, (int)N, (int)K, 1, ldb, ldb * K, kBK))
        return cudaErrorInvalidValue;
    const int sms = sm_count();
    if (sms < 2) return cudaErrorInvalidValue;
    const long long ntiles = ((M + tm - 1) / tm) * ((N + kBN - 1) / kBN);
    __nv_bfloat16 *c = static_cast<__nv_bfloat16 *>(C);
    __nv_bfloat16 *q = static_cast<__nv_bfloat16 *>(qh), *k = static_cast<__nv_bfloat16 *>(kt);
    cudaError_t e;
    if (pair) {
        const uint32_t smem = Cfg<true>::kSmemBytes;
        e = cudaFuncSetAttribute(gemm_tc_kernel<true, PROJ>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem);
        if (e != cudaSuccess) return e;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(2 * std::min<long long>(ntiles, sms / 2)), 1, 1);
        cfg.blockDim = dim3(kThreads, 1, 1);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, gemm_tc_kernel<true, PROJ>, ma, mb, (int)M, (int)N, (int)K, c, ldc,
                               status, pp, q, k);
    } else {
        const uint32_t smem = Cfg<false>::kSmemBytes;
        e = cudaFuncSetAttribute(gemm_tc_kernel<false, PROJ>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem);
        if (e != cudaSuccess) return e;
        const int grid = (int)std::min<long long>(ntiles, sms);
        gemm_tc_kernel<false, PROJ><<<grid, kThreads, smem, st>>>(ma, mb, (int)M, (int)N, (int)K, c, ldc,
                                                                 status, pp, q, k);
        e = cudaGetLastError();
    }
    if (e == cudaSuccess) note_launches(1);
    return e;
}

}  // namespace

cudaError_t launch_gemm_tc(long long M, long long N, long long K, const void *A, long long lda,
                           const void *B, long long ldb, void *C, long long ldc, int *status,
                           cudaStream_t st) {
    Params none{};
    return launch_gemm<false>(M, N, K, A, lda, B, ldb, C, ldc, none, nullptr, nullptr, status, st);
}

cudaError_t launch_gemm_proj(const Params &p, int d_model, const void *X, const void *W, void *P,
                             void *qh, void *kt, int *status, cudaStream_t st) {
    // every 32-column chunk of a tile lies in one head of one block
    if (p.dk % 32 != 0 || p.dv % 32 != 0 || !qh || !kt) return cudaErrorInvalidValue;
    const long long n_proj = (long long)p.H * (2LL * p.dk + 2LL * p.dv);
    return launch_gemm<true>((long long)p.B * p.L, n_proj, d_model, X, d_model, W, n_proj, P, n_proj,
                             p, qh, kt, status, st);
}

}  // namespace ret

extern "C" {

ret_status ret_gemm_bf16(long long M, long long N, long long K, const void *A, long long lda,
                         const void *B, long long ldb, void *C, long long ldc, void *stream) {
    if (M < 0 || N < 0 || K < 0) return RET_ERR_ARG;
    if (M == 0 || N == 0) return RET_OK;
    if (!ret::gemm_tc_supported(M, N, K, lda, ldb, ldc)) return RET_ERR_SHAPE;
    if (!A || !B || !C) return RET_ERR_NULL;
    auto a16 = [](const void *q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; };
    if (!a16(A) || !a16(B) || !a16(C)) return RET_ERR_ALIGN;
    int dev = -1, major = 0, minor = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
        cudaGetLastError();
        return RET_ERR_UNSUPPORTED;
    }
    if (major != 10 || minor != 0) return RET_ERR_UNSUPPORTED;
    int *status = ret::device_status_word();
    if (!status) return RET_ERR_CUDA;
    return ret::launch_gemm_tc(M, N, K, A, lda, B, ldb, C, ldc, status,
                               static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? RET_OK
               : RET_ERR_CUDA;
}

}  // extern "C"
