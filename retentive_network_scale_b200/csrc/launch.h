// launch.h -- internal launchers behind the C ABI (not exported).
#pragma once

#include <cublas_v2.h>
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "common.cuh"

namespace ret {

// Adds n to the process-wide launch counter (ret_kernel_launches).
void note_launches(int n);

cudaError_t launch_parallel_simt(const Params &p, bool in_bf16, bool out_bf16,
                                 const void *Q, const void *K, const void *V,
                                 void *O, cudaStream_t st);

cudaError_t launch_chunkwise_simt(const Params &p, int chunk, bool in_bf16,
                                  bool out_bf16, const void *Q, const void *K,
                                  const void *V, const float *s_in,
                                  float *s_out, void *O, cudaStream_t st);

// Tensor-core chunkwise kernel: bf16 inputs, chunk a multiple of 64
// (evaluated in blocks of 128 rows), d_k 64, 128 or 256, d_v 64 or a
// multiple of 128 (at most 512), every gamma_h^128 >= 2^-60.  With Y
// (and G) given it also writes Y = swish(G) (.) GroupNorm_h(O); O may then
// be NULL.
// With prep_ws (chunkwise_prep_bytes) the rows are first prepared by the
// streaming pass below; with NULL the kernel turns them itself (slower).
bool chunkwise_tc_supported(const Params &p, int chunk, bool in_bf16);
// Shapes of the tensor-core path whose rotated rows must come from the
// streaming pass (the workspace ret_chunkwise_prep_size gives).
bool chunkwise_tc_needs_prep(const Params &p, int chunk);
cudaError_t launch_chunkwise_tc(const Params &p, bool out_bf16, const void *Q, const void *K,
                                const void *V, const float *s_in, float *s_out, void *O,
                                const void *G, void *Y, float eps, void *prep_ws, int *status,
                                cudaStream_t st);

// The chunk loop alone on rows prepared by the streaming pass (blocks of
// kChunkBlock rows), one launch over the whole batch.
constexpr int kChunkBlock = 128;
cudaError_t launch_chunkwise_tc_rows(const Params &p, bool out_bf16, const void *Qh, const void *Kt,
                                     const void *V, const float *s_in, float *s_out, void *O,
                                     const void *G, void *Y, float eps, int *status,
                                     cudaStream_t st);

// Streaming pass: Q^ (rotation only) and K~ = gamma^{n-1-j} K^ per row of a
// chunk of `chunk` rows, bf16, into the workspace ([Q^][K~], or [K~] without
// rotation); *q_used / *k_used receive the operands to multiply.
size_t chunkwise_prep_bytes(const Params &p);
cudaError_t launch_chunkwise_prep(const Params &p, int chunk, const void *Q, const void *K,
                                  void *workspace, const void **q_used, const void **k_used,
                                  cudaStream_t st);

// Tensor map over [outer][rows][inner] bf16 with boxes of 64 x box_rows x 1
// and 128-byte swizzle; rows past the end read as zeros and are not written.
bool make_tma_map_bf16(CUtensorMap *m, const void *base, int inner, int rows, int outer, int box_rows);
// fp32 tensor map over [outer][rows][inner] with boxes of 32 x box_rows x 1
// (128-byte rows, 128-byte swizzle).
bool make_tma_map_f32(CUtensorMap *m, const void *base, int inner, int rows, int outer,
                      int box_rows);
// The same over a strided view: row_stride / outer_stride in elements
// (multiples of 8, i.e. 16 bytes).
bool make_tma_map_bf16_strided(CUtensorMap *m, const void *base, int inner, int rows, int outer,
                               long long row_stride, long long outer_stride, int box_rows);

// Element strides of a bf16 operand read as rows of (b, h, t): row t of head
// h of batch b starts at b*batch + h*head + t*row.
struct RowLayout {
    long long row, head, batch;
};
// [B][H][L][d], the layout of the C ABI's Q, K, V
inline RowLayout bhld_layout(const Params &p, int d) {
    return RowLayout{d, (long long)p.L * d, (long long)p.H * p.L * d};
}

// Tensor-core chunkwise kernel on rows already prepared: Q^ read through
// `q_layout` (head-major; its batch stride must be H times its head
// stride), K~ as [B][H][L][d_k], V and G through the given layouts (V as
// head-major rows when v_head_major, else as rows of H*d_v columns like G);
// writes Y ([B][L][H*d_v], with G) and/or O ([B][H][L][d_v]) in the output
// dtype.
cudaError_t launch_chunkwise_tc_prepared(const Params &p, bool out_bf16, const void *Qh,
                                         RowLayout q_layout, const void *Kt, const void *V,
                                         RowLayout v_layout, bool v_head_major, const void *G,
                                         RowLayout g_layout, void *Y, void *O, float eps,
                                         int *status, cudaStream_t st);
// Warp-specialised tensor-core chunk loop (chunkwise_ws.cu): the same
// shapes as the kernel above.  Q^ and K' are read through `q_layout` and
// `k_layout` (head-major), V through `v_layout` (head-major rows when
// v_head_major, else rows of H*d_v columns), G through `g_layout` (rows of
// H*d_v columns).  zeta_on_v: K' is K^ itself and the kernel weights the
// value rows by gamma^{n-1-j}; otherwise K' already carries that weight
// (the streaming pass).  rotate_in_loop: Q and K are the raw rows and the
// kernel turns the landed tiles (and weights the keys) in shared memory
// itself (d_k 128 or 256, plain heads).  Writes Y ([B][L][H*d_v], with G)
// and/or O ([B][H][L][d_v]) in the output dtype.  acc_in (fp32 O only, no
// gate, prepared rows): O = acc_in + the product, turned back by the angles
// of each row's position (Theta_t^T) when acc_unturn.
cudaError_t launch_chunkwise_ws(const Params &p, bool out_bf16, const void *Q, RowLayout q_layout,
                                const void *K, RowLayout k_layout, const void *V, RowLayout v_layout,
                                bool v_head_major, const float *s_in, float *s_out, void *O,
                                const void *G, RowLayout g_layout, void *Y, float eps,
                                bool zeta_on_v, bool rotate_in_loop, int *status,
                                cudaStream_t st, const float *acc_in = nullptr,
                                int acc_unturn = 0);

// The streaming pass reading Q and K through a layout; with always_q it
// writes Q^ even without rotation (then a plain copy into [B][H][L][d_k]),
// so the workspace holds 2*B*H*L*d_k values.
// The per-device side stream (lowest priority: kernels on it fill the SMs
// that a one-wave launch on the caller's stream leaves free) and events to
// join it to the caller's stream.  Made once per device; whoever enqueues
// on it holds *mu for the whole enqueue sequence.  False when it could not
// be made (the caller then queues everything on its own stream).
constexpr int kSideAuxEvents = 3;
struct SideStreamRef {
    std::mutex *mu;
    cudaStream_t s;
    cudaEvent_t start, ready, aux[kSideAuxEvents];
    int sms;
};
bool side_stream_ref(SideStreamRef *r);

cudaError_t launch_chunkwise_prep_strided(const Params &p, int chunk, const void *Q, const void *K,
                                          RowLayout src, bool always_q, void *workspace,
                                          const void **q_used, const void **k_used,
                                          cudaStream_t st);

// K~ alone (turned when p.rotate, and weighted by gamma^{n-1-j} per row of
// a chunk of `chunk` rows), bf16 [B][H][L][d_k], from K [B][H][L][d_k].
cudaError_t launch_key_prep(const Params &p, int chunk, const void *K, void *kt,
                            cudaStream_t st);

// C[M x N] = A[M x K] B[K x N] on the tensor cores (gemm_tc.cu): bf16
// row-major operands with leading dimensions lda, ldb, ldc (elements,
// multiples of 8), fp32 accumulation, bf16 C.  N a multiple of 8.
bool gemm_tc_supported(long long M, long long N, long long K, long long lda, long long ldb,
                       long long ldc);
cudaError_t launch_gemm_tc(long long M, long long N, long long K, const void *A, long long lda,
                           const void *B, long long ldb, void *C, long long ldc, int *status,
                           cudaStream_t st);

// The layer's projection P = X [W_Q | W_K | W_V | W_G] (X [B*L][d_model],
// P [B*L][H (2 d_k + 2 d_v)]) with the streaming pass folded into the
// epilogue: the Q and K columns leave as Q^ and K~ (turned when p.rotate,
// K~ weighted by gamma^{n-1-j} per block of 128 rows), bf16
// [B][H][L][d_k] into qh and kt; only the V and G columns are written to P.
cudaError_t launch_gemm_proj(const Params &p, int d_model, const void *X, const void *W, void *P,
                             void *qh, void *kt, int *status, cudaStream_t st);

// The current device's cuBLAS handle, bound to `st` and to kBlasWorkspace
// bytes of `workspace`; the caller holds blas_mutex() for as long as it
// uses the handle (a handle is not safe to share between host threads).
// NULL when the handle cannot be made or bound.
constexpr size_t kBlasWorkspace = 32ull << 20;
std::mutex &blas_mutex();
cublasHandle_t blas_handle(cudaStream_t st, void *workspace);

// U = sum_t gamma^{L-1-t} k^_t^T v_t per (b, h) ([d_k][d_v] fp32) on the
// tensor cores (segstate.cu): K~ [B][H][L][d_k], V [B][H][L][d_v], d_k 64,
// 128 or 256, d_v 64 or a multiple of 128.  zeta_v 0: the weight is on K~ already
// (the streaming pass with the segment as one block); 1: K~ = K^ and the
// kernel weights the value rows; 2: K~ carries the weights of 128-row
// blocks (the chunk loop's streaming pass) and the kernel scales each
// block's value rows by the rest.
bool segment_state_tc_supported(const Params &p);
cudaError_t launch_segment_state_tc(const Params &p, const void *V, const void *Kt, int zeta_v,
                                    float *U, int *status, cudaStream_t st);

// The chunkwise form with every sequence cut into S equal segments that run
// at once (seqshard.cu): streaming pass, segment states, scan of the
// entering states, one chunk-loop launch over the B*H*S segment heads (with
// the gate when G and Y are given), the final state copied out.  The
// workspace holds segmented_bytes(p, S), the streaming pass's rows first.
// auto_segments gives the S that ret_chunkwise uses when the plain loop
// would leave most SMs idle (1: none).
bool segmented_supported(const Params &p, int chunk, int S);
size_t segmented_bytes(const Params &p, int S);
int auto_segments(const Params &p, int chunk);
cudaError_t launch_segmented(const Params &p, int S, bool out_bf16, const void *Q, const void *K,
                             const void *V, const float *state_in, float *state_out, void *O,
                             const void *G, void *Y, float eps, void *workspace, int *status,
                             cudaStream_t st);

// The chunkwise form in one launch for few heads (onepass.cu): one CTA per
// block of 128 rows of every head, each taking its entering state from the
// key-value sums the head's earlier blocks publish to the workspace
// (onepass_bytes).  d_k and d_v 64 or 128, bf16, no rotation, no carried
// state, at most 32 blocks per head; writes Y (with G) and/or O.
bool onepass_supported(const Params &p, bool in_bf16, bool has_state);
size_t onepass_bytes(const Params &p);
cudaError_t launch_onepass(const Params &p, bool out_bf16, const void *Q, const void *K,
                           const void *V, void *O, const void *G, void *Y, float eps,
                           void *workspace, int *status, cudaStream_t st);

// Tensor-core parallel form: bf16 inputs, d_k 64, 128 or 256, d_v 64 or a
// multiple of 128, every gamma_h^127 >= 2^-60.  With rotation it first writes the turned
// Q^ and K^ (bf16) into the workspace (parallel_tc_workspace bytes).
bool parallel_tc_supported(const Params &p, bool in_bf16);
size_t parallel_tc_workspace(const Params &p);
cudaError_t launch_parallel_tc(const Params &p, bool out_bf16, const void *Q, const void *K,
                               const void *V, void *O, void *workspace, int *status,
                               cudaStream_t st);

// The description checks every entry point runs first (no CUDA calls).
ret_status validate_desc(const ret_desc *d);
// The kernels' parameters for a checked description.
void params_from_desc(const ret_desc *d, Params *p);

// Address of the device status word bounded waits latch errors into.
int *device_status_word();

cudaError_t launch_recurrent_step(const Params &p, bool in_bf16, bool out_bf16,
                                  const void *q, const void *k, const void *v,
                                  float *state, void *o, cudaStream_t st);

cudaError_t launch_gate_norm(int B, int L, int H, int dv, bool o_bf16,
                             const void *O, bool g_bf16, const void *G,
                             float eps, bool y_bf16, void *Y, cudaStream_t st);

// dO (O's type) and dG (G's type) of Y = swish(G) GroupNorm_h(O) given dY
// (G's type).
cudaError_t launch_gate_norm_backward(int B, int L, int H, int dv, bool o_bf16, const void *O,
                                      bool g_bf16, const void *G, const void *dY, float eps,
                                      void *dO, void *dG, cudaStream_t st);

}  // namespace ret
