/*
 * retention.h -- C ABI of the B200 multi-scale retention forward library
 * (libretention.so, hand-written CUDA for sm_100a).
 *
 * What is computed.  Per batch b and head h with scalar decay gamma_h, every
 * form returns
 *     o_n = sum_{m <= n} gamma_h^{n-m} (q^_n . k^_m) v_m ,
 * the scalar-gamma retention of "Retentive Network: A Successor to
 * Transformer for Large Language Models" (paper summary, blog.csdn.net
 * 132817411, section 2.1), where q^_n, k^_m are the rows turned by the xPos
 * factor e^{i n theta}: a row of even width d_k is read as d_k/2 complex
 * numbers (x[2j], x[2j+1]) and pair j is turned by the angle
 * pos * theta_j, theta_j = theta_base^(-2j/d_k), for Q and K alike, so the
 * score is the real part of (Q_n e^{in theta})(K_m e^{im theta})^dagger.
 * There is no 1/sqrt(d_k) score scale (the pages give none).
 *
 * Conventions shared by every entry point.
 *  - Pointers named as device pointers must be device memory of the current
 *    device (or managed memory); every one must be 16-byte aligned.  Pointers
 *    named as host pointers are read during the call only.
 *  - The caller owns every buffer and the stream.  The library allocates no
 *    device memory (cuBLAS allocates its own when the library first makes a
 *    handle on a device, for the shapes of ret_segment_state off its
 *    tensor-core kernel), keeps no
 *    per-call state, and never synchronises unless a function says so.
 *    `stream` is a cudaStream_t passed as void*; NULL is the legacy default
 *    stream.
 *  - Process-level objects, made once per device under a lock: the device
 *    status word of the bounded waits (a __device__ variable), the cuBLAS
 *    handle, and the side stream with five events on which ret_chunkwise
 *    runs the streaming pass of its next batch slice and ret_backward the
 *    key-weighting pass of its next product.  Calls from several host
 *    threads are safe; on one device they take those locks in turn while
 *    they enqueue work.
 *  - Arguments are checked before any launch.  A call that returns an error
 *    launched nothing and wrote nothing.  A call that returns RET_OK has only
 *    queued work: kernel faults surface on the stream, and a bounded device
 *    wait that gave up is reported by ret_last_device_status().
 *  - Layouts are dense and row-major:
 *        Q, K    [B][H][L][d_k]     V, O   [B][H][L][d_v]
 *        G, Y    [B][L][H*d_v]      state  [B][H][d_k][d_v]  (always fp32)
 *    Row t of a (b,h) slice sits at absolute position pos_offset + t.  A
 *    state is S after absorbing every token before the first row of the
 *    call, so prefill and decode must use continuous positions.
 *  - Limits: 1 <= H <= RET_MAX_HEADS, 1 <= d_k <= 256, 1 <= d_v <= 512,
 *    d_v a multiple of 4, d_k even when rotating; B, L >= 0 (zero sizes are
 *    accepted and do nothing); 0 <= gamma_h <= 1.
 *  - Only sm_100 devices are supported: elsewhere every compute entry point
 *    returns RET_ERR_UNSUPPORTED.  There is no fallback of any kind.
 */
#ifndef RETENTION_H
#define RETENTION_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

#define RET_MAX_HEADS 128
#define RET_MAX_DECODE_STEPS 16  /* tokens per ret_recurrent_step call */

typedef enum {
    RET_OK = 0,
    RET_ERR_NULL = 1,        /* a required pointer is NULL                    */
    RET_ERR_SHAPE = 2,       /* a size is negative or beyond the limits above */
    RET_ERR_DTYPE = 3,       /* dtype code not RET_F32 / RET_BF16             */
    RET_ERR_ALIGN = 4,       /* a device pointer is not 16-byte aligned       */
    RET_ERR_ARG = 5,         /* gamma outside [0,1] or not finite, chunk < 1,
                                odd d_k with rotation, eps < 0, bad base      */
    RET_ERR_WORKSPACE = 6,   /* workspace NULL or smaller than required       */
    RET_ERR_UNSUPPORTED = 7, /* not an sm_100 device                          */
    RET_ERR_CUDA = 8,        /* a CUDA runtime call or launch failed          */
    RET_ERR_TIMEOUT = 9      /* a bounded device wait gave up (see
                                ret_last_device_status)                        */
} ret_status;

typedef enum { RET_F32 = 0, RET_BF16 = 1 } ret_dtype;

/* Problem description.  The struct is read during the call only. */
typedef struct {
    int B, H, L, d_k, d_v;   /* L: 1..RET_MAX_DECODE_STEPS for
                                ret_recurrent_step                          */
    int in_dtype;            /* ret_dtype of Q, K, V (and G)                */
    int out_dtype;           /* ret_dtype of O (and Y)                      */
    const double *gamma;     /* HOST array [H]: decay of each head          */
    int rotate;              /* 0: no xPos rotation; 1: rotate Q and K      */
    double theta_base;       /* theta_j = theta_base^(-2j/d_k), e.g. 10000  */
    long long pos_offset;    /* absolute position of row 0 (>= 0)           */
} ret_desc;

/*
 * ret_parallel -- the parallel representation (section 2.1, form (1)):
 *     Retention(X) = (Q K^T (.) D) V,  D_nm = gamma^{n-m} (n >= m), else 0,
 * with Q, K rotated as above.  Q, K, V: device, in_dtype.  O: device,
 * out_dtype, fully overwritten.  No state in or out.
 *   workspace  device scratch of workspace_bytes; required only when
 *              ret_parallel_workspace_size() returns a non-zero size (it
 *              then receives the rotated Q and K in bf16).
 * Errors: RET_ERR_NULL, _SHAPE, _DTYPE, _ALIGN, _ARG, _WORKSPACE,
 * _UNSUPPORTED, _CUDA.
 */
ret_status ret_parallel(const ret_desc *desc, const void *Q, const void *K,
                        const void *V, void *O, void *workspace,
                        size_t workspace_bytes, void *stream);

/* Bytes of workspace ret_parallel needs for this description (0 when none).
 * Never fails (0 for descriptions ret_parallel would reject). */
size_t ret_parallel_workspace_size(const ret_desc *desc);

/*
 * ret_chunkwise -- the chunkwise recurrent representation (section 2.1,
 * form (3): parallel inside a chunk of `chunk` rows, a decayed state carried
 * between chunks).  For the chunk of n rows after state R:
 *     o_j = sum_{j'<=j} gamma^{j-j'} (q^_j.k^_{j'}) v_{j'} + gamma^{j+1} q^_j R
 *     R  <- gamma^n R + sum_{j'} gamma^{n-1-j'} k^_{j'}^T v_{j'}
 * (the recurrent form unrolled over the chunk; the last chunk may be short).
 * The result equals ret_parallel's up to rounding for every chunk size.
 * The tensor-core path works in blocks of 128 rows: a chunk of 128*m rows
 * is m consecutive blocks, a chunk of 64 rows two chunks per block (the
 * recurrence holds exactly at every row boundary, so this is the same
 * computation with different rounding).
 *   state_in  device fp32 [B][H][d_k][d_v] or NULL (zeros).
 *   state_out device fp32, or NULL; may alias state_in.
 *   O         device out_dtype [B][H][L][d_v], or NULL when only Y is wanted.
 *   G, Y      both NULL, or both device: G in_dtype, Y out_dtype
 *             [B][L][H*d_v]; then Y = swish(G) (.) GroupNorm_h(O) (as in
 *             ret_gate_norm) is written as well, with epsilon gn_eps.
 *   workspace device scratch of workspace_bytes; required only when
 *             ret_workspace_size() returns a non-zero size for this call.
 *             On the tensor-core path (bf16 inputs, chunk a multiple of
 *             64, d_k 64, 128 or 256, d_v 64 or a multiple of 128 up to
 *             512, gamma_h^128 >= 2^-60 for every head): with at least
 *             ret_chunkwise_prep_size() bytes the rotated Q and the
 *             decay-weighted K are prepared there in one streaming pass
 *             before the chunk loop (faster); with less, the loop turns
 *             the rows itself (d_k and d_v from 128 and chunks of 128*m
 *             only: for the other shapes of the path ret_workspace_size
 *             asks for the prep size when rotating) or, without rotation,
 *             weights the value rows itself.  With at least
 *             ret_chunkwise_fast_size() bytes a call on few heads cuts
 *             every sequence into segments that run at once (see there).
 *             Results agree either way up to rounding.
 * At least one of O and Y must be requested.
 * Errors: those of ret_parallel, plus RET_ERR_WORKSPACE.
 */
ret_status ret_chunkwise(const ret_desc *desc, int chunk, const void *Q,
                         const void *K, const void *V, const float *state_in,
                         float *state_out, void *O, const void *G, float gn_eps,
                         void *Y, void *workspace, size_t workspace_bytes,
                         void *stream);

/*
 * ret_chunkwise_gate_static -- no counterpart in the paper.  The same call as
 * ret_chunkwise with G and Y given and O = NULL, for callers that must not
 * allocate device memory while they run: for instance a service whose
 * device memory is reserved up front by a host framework, or one held to a
 * fixed memory budget once serving starts.  Such callers cannot provide the
 * workspace ret_chunkwise takes for shapes the tensor-core kernel does not
 * cover (an fp32 O of B*H*L*d_v floats, normalised into Y afterwards).
 * Here that scratch is a fixed array of RET_STATIC_SCRATCH_FLOATS floats
 * (16 MiB) inside the library; every device that loads the library holds
 * it until the process exits.  Nothing is allocated by this call.
 *   - Problems whose scratch would exceed the array return
 *     RET_ERR_WORKSPACE before anything runs.
 *   - The first call on each device that needs the array looks up its
 *     device address (cudaGetSymbolAddress) with that device current; make
 *     that first call before any stream capture.  A failed lookup returns
 *     RET_ERR_CUDA, leaves no CUDA error pending and is tried again by the
 *     next call.
 *   - All calls on a device share the array, which keeps the last call's
 *     contents; calls that overlap on the GPU (other streams or threads)
 *     race on it.
 * Arguments, layouts and other errors are those of ret_chunkwise; the
 * description, chunk and NULL checks come before the size check.
 */
#define RET_STATIC_SCRATCH_FLOATS (4u << 20)
ret_status ret_chunkwise_gate_static(const ret_desc *desc, int chunk, const void *Q,
                                     const void *K, const void *V, const float *state_in,
                                     float *state_out, const void *G, float gn_eps,
                                     void *Y, void *stream);

/* Bytes of workspace ret_chunkwise needs for this description and chunk
 * (0 when none).  Depends only on the arguments; never fails (returns 0
 * for descriptions that ret_chunkwise would reject). */
size_t ret_workspace_size(const ret_desc *desc, int chunk, int want_O,
                          int want_Y);

/* Bytes of OPTIONAL workspace with which ret_chunkwise takes its fastest
 * path for this description and chunk: on the tensor-core path the room of
 * ret_chunkwise_prep_size, or, when B*H*ceil(d_v/128) is below 64 (most
 * SMs would idle) and L splits into 2 to 16 equal segments of at least 512
 * rows, the room of ret_chunkwise_segmented_workspace_size for the number
 * of segments that keeps one CTA per SM: ret_chunkwise then cuts every
 * sequence into segments that run at once, with the gate when G and Y are
 * given (same result up to rounding).  0 when the tensor-core path does not
 * apply; never fails.  No counterpart in the paper. */
size_t ret_chunkwise_fast_size(const ret_desc *desc, int chunk);

/* Bytes of OPTIONAL workspace that let ret_chunkwise prepare its operands
 * ahead of the chunk loop (see ret_chunkwise): 2*B*H*L*d_k bf16 values
 * with rotation (the rotated Q, and K rotated and scaled by
 * gamma^{n-1-j} at offset j of its chunk of n rows), B*H*L*d_k without.
 * No counterpart in the paper: it is a layout choice of this library.
 * 0 when the tensor-core path does not apply (ret_workspace_size then
 * gives everything the call needs); never fails. */
size_t ret_chunkwise_prep_size(const ret_desc *desc, int chunk);

/* ret_chunkwise_prepare -- only the streaming pass that ret_chunkwise runs
 * first when its workspace holds ret_chunkwise_prep_size() bytes: the
 * rotated Q (bf16 [B][H][L][d_k], with rotation only) followed by
 * K~[b,h,t] = gamma_h^{n-1-j} Theta_t K[b,h,t] (bf16, same shape) for row t
 * at offset j of its block of n rows (section 2.1, chunkwise form (3): the
 * weight of key j' in the state update).  The tensor-core loop works in
 * blocks of 128 rows whatever `chunk` is (a multiple of 64; the recurrence
 * holds at every row boundary), so the weights follow those blocks.  No counterpart in the paper as a
 * call of its own; exported so that the pass can be timed or scheduled
 * apart.  Q, K device bf16; workspace device, caller-owned, overwritten.
 * Errors: RET_ERR_SHAPE when the tensor-core path does not apply (nothing
 * to prepare), _NULL, _ALIGN, _WORKSPACE (smaller than the prep size),
 * _UNSUPPORTED, _CUDA, and the description errors of ret_parallel. */
ret_status ret_chunkwise_prepare(const ret_desc *desc, int chunk,
                                 const void *Q, const void *K, void *workspace,
                                 size_t workspace_bytes, void *stream);

/* ret_chunkwise_prepared -- the chunk loop of ret_chunkwise alone, on rows
 * that ret_chunkwise_prepare wrote: the tensor-core loop, one launch over
 * the whole batch.  No counterpart in the paper as a call of its own;
 * exported for callers that schedule the streaming pass themselves, and so
 * that the loop can be timed apart.
 *   Qh  device bf16 [B][H][L][d_k]: the rotated Q from the workspace, or Q
 *       itself when desc->rotate is 0
 *   Kt  device bf16 [B][H][L][d_k]: the weighted K~ from the workspace
 *   V, state_in, state_out, O, G, gn_eps, Y  as ret_chunkwise
 * desc and chunk must be those the rows were prepared with.  Errors:
 * RET_ERR_SHAPE when the tensor-core path does not apply or the problem is
 * empty, and those of ret_chunkwise. */
ret_status ret_chunkwise_prepared(const ret_desc *desc, int chunk,
                                  const void *Qh, const void *Kt, const void *V,
                                  const float *state_in, float *state_out, void *O,
                                  const void *G, float gn_eps, void *Y, void *stream);

/*
 * ret_chunkwise_host -- no counterpart in the paper: ret_chunkwise from HOST
 * buffers to HOST buffers, the end-to-end form for callers whose Q, K, V, G
 * live in host memory.  Same description, layouts, dtypes and outputs as
 * ret_chunkwise (O and/or Y; G with Y), starting from a zero state and with
 * no state out.  The batch is cut into `slices` slices (1..B; more are
 * clamped to B) of ceil(B/slices) batch elements, and the slices flow through
 * two device slots on three streams, so that the host-to-device copies of
 * one slice, the compute of the previous one and the copy back of the one
 * before run at the same time.
 *   Q, K, V, G  host, read; O, Y host, written.  Page-locked memory
 *               (cudaHostAlloc / cudaHostRegister) lets the copies overlap;
 *               pageable memory works but the runtime stages those copies.
 *   dev_workspace  device, 256-byte aligned, at least
 *               ret_chunkwise_host_workspace_size() bytes; caller-owned.
 *   stream      the work starts after what is already queued on `stream`,
 *               and `stream` continues only once every copy back is done.
 *               Host buffers must stay valid until then.
 * Errors: those of ret_chunkwise, plus RET_ERR_ARG for slices < 1.  After a
 * failure the call waits for the copies it queued before it returns.
 */
ret_status ret_chunkwise_host(const ret_desc *desc, int chunk, const void *Q,
                              const void *K, const void *V, void *O,
                              const void *G, float gn_eps, void *Y, int slices,
                              void *dev_workspace, size_t dev_workspace_bytes,
                              void *stream);

/* Device workspace bytes ret_chunkwise_host needs (two slots of one slice
 * each, one slot when there is a single slice); 0 for descriptions it would
 * reject and for empty problems.  Never fails. */
size_t ret_chunkwise_host_workspace_size(const ret_desc *desc, int chunk,
                                         int want_O, int want_Y, int slices);

/*
 * ret_msr_layer -- the multi-scale retention layer (paper summary, section
 * 2.1: Q = (X W_Q) (.) Theta, K = (X W_K) (.) conj(Theta), V = X W_V, one
 * decay per head; section 2.2: Y = GroupNorm_h(Concat(heads)),
 * MSR(X) = (swish(X W_G) (.) Y) W_O):
 *     P   = X [W_Q | W_K | W_V | W_G]
 *     out = (swish(G) (.) GroupNorm_h(Retention(Q, K, V))) W_O
 * with the heads, rotation, decays and GroupNorm of ret_chunkwise, from a
 * zero state.
 *   X       device bf16 [B][L][d_model]
 *   W_qkvg  device bf16 [d_model][H*(2 d_k + 2 d_v)]: head h's columns of
 *           Q at h d_k, of K at H d_k + h d_k, of V at 2 H d_k + h d_v, of G
 *           at 2 H d_k + H d_v + h d_v
 *   W_o     device bf16 [H d_v][d_model]
 *   out     device bf16 [B][L][d_model]
 *   workspace  device, 256-byte aligned, at least
 *           ret_msr_layer_workspace_size() bytes (it holds P, the prepared
 *           Q and K, and Y).
 * desc->in_dtype and out_dtype are RET_BF16; d_model is a multiple of 8.
 * The layer runs on the tensor-core chunkwise path only (chunk a multiple of
 * 64, d_k 128 or 256, d_v a multiple of 128 up to 512, gamma_h^128 >=
 * 2^-60).  The two projections run on ret_gemm_bf16's tensor-core product
 * (fp32 accumulation); P and Y are held in bf16.
 * Errors: those of ret_chunkwise; RET_ERR_SHAPE off the tensor-core path.
 */
ret_status ret_msr_layer(const ret_desc *desc, int d_model, int chunk,
                         const void *X, const void *W_qkvg, const void *W_o,
                         float gn_eps, void *out, void *workspace,
                         size_t workspace_bytes, void *stream);

/* Device workspace bytes ret_msr_layer needs; 0 for descriptions it would
 * reject by their arguments and for empty problems.  Never fails. */
size_t ret_msr_layer_workspace_size(const ret_desc *desc, int d_model,
                                    int chunk);

/*
 * ret_gemm_bf16 -- C = A B, the dense product the layer's projections are
 * (paper summary, section 2.2: X W_Q, X W_K, X W_V, X W_G and the product
 * with W_O), on the tensor cores: bf16 operands, fp32 accumulation, bf16
 * result rounded to nearest even.
 *   A  device bf16, M rows of K values, row r at A + r*lda
 *   B  device bf16, K rows of N values, row k at B + k*ldb
 *   C  device bf16, M rows of N values, row r at C + r*ldc (written)
 * lda, ldb, ldc are in elements, multiples of 8, with lda >= K, ldb >= N,
 * ldc >= N; N is a multiple of 8; M, N, K fit in 32 bits.  C must not
 * overlap A or B.  M == 0 or N == 0 is an empty problem (RET_OK, nothing
 * launched).
 * Errors: RET_ERR_ARG (a negative size), RET_ERR_NULL, RET_ERR_SHAPE (K ==
 * 0, N not a multiple of 8, leading dimensions as above), RET_ERR_ALIGN
 * (a pointer not 16-byte aligned), RET_ERR_UNSUPPORTED (not an sm_100
 * device), RET_ERR_CUDA (launch failure).  A bounded wait that runs out
 * latches RET_ERR_TIMEOUT for ret_last_device_status.
 */
ret_status ret_gemm_bf16(long long M, long long N, long long K, const void *A,
                         long long lda, const void *B, long long ldb, void *C,
                         long long ldc, void *stream);

/*
 * ret_backward -- the gradients of the retention output O (as computed by
 * ret_parallel / ret_chunkwise, no gate, zero state) with respect to Q, K
 * and V, given dO (section 2.1: the parallel and chunkwise forms are the
 * training forms).  With q^_t = Theta_t q_t, k^_m = Theta_m k_m:
 *     dq^_t = sum_{m<=t} gamma^{t-m} (do_t . v_m) k^_m,
 *     dk^_m = sum_{t>=m} gamma^{t-m} (v_m . do_t) q^_t,
 *     dv_m  = sum_{t>=m} gamma^{t-m} (k^_m . q^_t) do_t,
 *     dq_t = Theta_t^T dq^_t, dk_m = Theta_m^T dk^_m.
 * Each is evaluated as a chunkwise retention of rearranged operands on the
 * tensor cores (the two anti-causal ones by the chunk loop's reverse mode,
 * on the operands in place; with rotation Q and K are first copied turned).
 * The key-weighting pass of each product runs on the library's side stream
 * (joined to `stream` by events), beside the previous product's loop.
 *   Q, K    device bf16 [B][H][L][d_k];  V, dO device bf16 [B][H][L][d_v]
 *   dQ, dK  device out_dtype [B][H][L][d_k];  dV device out_dtype
 *           [B][H][L][d_v]; all fully overwritten
 *   workspace  device, 256-byte aligned, at least
 *           ret_backward_workspace_size() bytes
 * Tensor-core shapes only: d_k 128 or 256, d_v a multiple of 128 up to 512,
 * chunk a multiple of 64, gamma_h^128 >= 2^-60 (else RET_ERR_SHAPE).
 * Errors: those of ret_chunkwise.
 */
ret_status ret_backward(const ret_desc *desc, int chunk, const void *Q,
                        const void *K, const void *V, const void *dO, void *dQ,
                        void *dK, void *dV, void *workspace,
                        size_t workspace_bytes, void *stream);

/* Device workspace bytes ret_backward needs (it depends on desc->rotate:
 * the turned copies of Q and K); 0 for descriptions it would reject by their
 * arguments and for empty problems.  Never fails. */
size_t ret_backward_workspace_size(const ret_desc *desc, int chunk);

/*
 * ret_segment_state -- the state a segment of a sequence leaves behind when
 * it starts from a zero state (section 2.1, form (3): the chunkwise state
 * recurrence holds at any row boundary, so between segments as between
 * chunks):
 *     U = sum_{t < L} gamma^{L-1-t} k^_t^T v_t,
 * k^_t turned at position pos_offset + t.  A segment of L rows that starts
 * from state R leaves gamma^L R + U.  To split a long sequence over several
 * devices, each computes the U of its own segment, the U are exchanged (an
 * all-gather), ret_state_scan gives each segment its entering state, and
 * ret_chunkwise with that state_in and the segment's pos_offset produces
 * the segment's outputs.
 *   K  device bf16 [B][H][L][d_k] (d_k a multiple of 8)
 *   V  device bf16 [B][H][L][d_v]
 *   U  device fp32 [B][H][d_k][d_v], fully overwritten (zeros when L = 0)
 *   workspace  device, 256-byte aligned, at least
 *              ret_segment_state_workspace_size() bytes
 * A streaming pass writes the turned, decay-weighted keys into the
 * workspace; one batched bf16 GEMM with fp32 accumulation (cuBLAS) forms U.
 * Errors: RET_ERR_NULL, _SHAPE, _DTYPE (bf16 inputs only), _ALIGN, _ARG,
 * _WORKSPACE, _UNSUPPORTED, _CUDA.
 */
ret_status ret_segment_state(const ret_desc *desc, const void *K, const void *V,
                             float *U, void *workspace, size_t workspace_bytes,
                             void *stream);

/* Device workspace bytes ret_segment_state needs; 0 for descriptions it
 * would reject by their arguments and for empty problems.  Never fails. */
size_t ret_segment_state_workspace_size(const ret_desc *desc);

#define RET_MAX_SEGMENTS 64  /* segments of one ret_state_scan */

/*
 * ret_state_scan -- the state entering segment `rank` of a sequence cut
 * into n_seg consecutive segments of seg_len[0..n_seg-1] rows, from the
 * segments' own states U_s (ret_segment_state) and the state before the
 * first segment:
 *     R_0 = state_in (zero when NULL),  R_{s+1} = gamma^{seg_len[s]} R_s + U_s,
 * returned for s = rank, 0 <= rank <= n_seg (rank = n_seg: the state after
 * the whole sequence).  desc supplies B, H, d_k, d_v and gamma (it must
 * pass the usual checks; its L and dtypes play no part).
 *   seg_len   HOST array [n_seg], every entry >= 1
 *   U_all     device fp32 [n_seg][B][H][d_k][d_v]; only segments below
 *             `rank` are read (may be NULL when rank = 0)
 *   state_in  device fp32 [B][H][d_k][d_v], or NULL
 *   R         device fp32 [B][H][d_k][d_v], fully overwritten
 * Errors: RET_ERR_NULL, _SHAPE (n_seg outside 1..RET_MAX_SEGMENTS, rank
 * outside 0..n_seg, a seg_len below 1), _ALIGN, _ARG, _UNSUPPORTED, _CUDA.
 */
ret_status ret_state_scan(const ret_desc *desc, int n_seg, const int *seg_len,
                          int rank, const float *U_all, const float *state_in,
                          float *R, void *stream);

/*
 * ret_chunkwise_segmented -- ret_chunkwise for few long sequences, on one
 * device: every sequence is cut into `segments` equal segments of L /
 * segments rows, which run at once (the chunkwise recurrence of section
 * 2.1, form (3), holds between segments as between chunks).  Each segment's
 * own state comes from the streaming pass's keys and a tensor-core
 * reduction over its rows, a scan gives every segment its entering state, and
 * one launch of the tensor-core chunk loop computes all segments, each from
 * its state: S times the CTAs of the plain loop, for B*H*d_v/128 well below
 * the number of SMs.  Same result as ret_chunkwise up to rounding.
 *   Q, K  device bf16 [B][H][L][d_k];  V device bf16 [B][H][L][d_v]
 *   state_in   device fp32 [B][H][d_k][d_v] or NULL (zero state)
 *   state_out  device fp32 [B][H][d_k][d_v] or NULL: after the last row
 *   O          device out_dtype [B][H][L][d_v], fully overwritten
 *   workspace  device, 256-byte aligned, at least
 *              ret_chunkwise_segmented_workspace_size() bytes
 * Tensor-core shapes only; L a multiple of `segments`, H * segments <=
 * RET_MAX_HEADS, B * H * segments <= 65535 (else RET_ERR_SHAPE).  No gate
 * (use ret_gate_norm on O).  Errors: those of ret_chunkwise.
 */
ret_status ret_chunkwise_segmented(const ret_desc *desc, int chunk, int segments,
                                   const void *Q, const void *K, const void *V,
                                   const float *state_in, float *state_out,
                                   void *O, void *workspace, size_t workspace_bytes,
                                   void *stream);

/* Device workspace bytes ret_chunkwise_segmented needs; 0 for calls it
 * would reject by their arguments.  Never fails. */
size_t ret_chunkwise_segmented_workspace_size(const ret_desc *desc, int chunk,
                                              int segments);

/*
 * ret_selftest_wait_timeout -- diagnostic, no counterpart in the paper.
 * Queues one small kernel on `stream` that waits on an mbarrier nothing
 * completes, through the same bounded wait every tensor-core kernel uses,
 * giving up after `cycles` SM clock cycles (1000 to 4e9, i.e. up to about
 * 2 s).  The expected outcome is the failure path of a stalled copy or
 * product: RET_ERR_TIMEOUT latched in the device status word (read and
 * cleared by ret_last_device_status), the kernel ending normally and the
 * device staying usable.  Returns RET_OK once the kernel is queued;
 * RET_ERR_ARG for `cycles` out of range, _UNSUPPORTED, _CUDA.
 */
ret_status ret_selftest_wait_timeout(long long cycles, void *stream);

/*
 * ret_recurrent_step -- the recurrent representation (section 2.1, form
 * (2)) for desc->L = T consecutive tokens of every sequence (1 <= T <=
 * RET_MAX_DECODE_STEPS): for n = pos_offset .. pos_offset+T-1,
 *     S_n = gamma S_{n-1} + k^_n^T v_n,  then  o_n = q^_n S_n
 * (update first, then read).  desc->pos_offset is the absolute position of
 * the first token.  The state is read and written once for all T tokens,
 * so T > 1 (several accepted tokens, or a chunk of a draft) costs about the
 * HBM traffic of one token.
 *   q, k   device in_dtype [B][H][T][d_k];  v device in_dtype [B][H][T][d_v]
 *   state  device fp32 [B][H][d_k][d_v], updated in place
 *   o      device out_dtype [B][H][T][d_v]
 * (with T = 1 these are [B][H][d]).  Errors: those of ret_parallel, and
 * RET_ERR_SHAPE for T outside 1..RET_MAX_DECODE_STEPS.
 */
ret_status ret_recurrent_step(const ret_desc *desc, const void *q,
                              const void *k, const void *v, float *state,
                              void *o, void *stream);

/*
 * ret_gate_norm -- section 2.2: Y = swish(G) (.) GroupNorm_h(O), one group
 * per head taken per token over its d_v channels, population variance, no
 * affine parameters, swish(x) = x sigmoid(x):
 *     Y[b,t,h*d_v+c] = swish(G[b,t,h*d_v+c]) (O[b,h,t,c] - mu) / sqrt(var + eps)
 *   O  device o_dtype [B][H][L][d_v];  G device g_dtype [B][L][H*d_v]
 *   Y  device y_dtype [B][L][H*d_v], fully overwritten
 * Errors: RET_ERR_NULL, _SHAPE, _DTYPE, _ALIGN, _ARG (eps < 0), _UNSUPPORTED,
 * _CUDA.
 */
ret_status ret_gate_norm(int B, int L, int H, int d_v, int o_dtype,
                         const void *O, int g_dtype, const void *G, float eps,
                         int y_dtype, void *Y, void *stream);

/*
 * ret_gate_norm_backward -- gradients of section 2.2's output
 * Y = swish(G) (.) GroupNorm_h(O) (the computation of ret_gate_norm) with
 * respect to O and G, given dY, by the chain rule through its three steps
 * (per (b, t, h) row of d_v channels, n = (O - mu) / sqrt(var + eps)):
 *     dG = dY (.) n (.) swish'(G),  swish'(g) = sigmoid(g) (1 + g (1 - sigmoid(g)))
 *     dn = dY (.) swish(G)
 *     dO = (dn - mean(dn) - n mean(dn (.) n)) / sqrt(var + eps)
 * The paper summary gives the forward only; this is its derivative, the
 * step a training pass takes before the retention backward (ret_backward
 * takes the dO written here).
 *   O   device o_dtype [B][H][L][d_v], the retention output of the forward
 *   G   device g_dtype [B][L][H*d_v];  dY  device g_dtype [B][L][H*d_v]
 *   dO  device o_dtype [B][H][L][d_v];  dG  device g_dtype [B][L][H*d_v]
 * Both outputs are fully overwritten and must not alias an input.  fp32
 * arithmetic.  Errors: RET_ERR_NULL, _SHAPE (as ret_gate_norm), _DTYPE,
 * _ALIGN, _ARG (eps < 0 or not finite), _UNSUPPORTED, _CUDA.
 */
ret_status ret_gate_norm_backward(int B, int L, int H, int d_v, int o_dtype,
                                  const void *O, int g_dtype, const void *G,
                                  const void *dY, float eps, void *dO, void *dG,
                                  void *stream);

/* Synchronises `stream`, then returns and clears the device status word
 * that bounded waits in the kernels latch (RET_ERR_TIMEOUT), or
 * RET_ERR_CUDA when the stream reports an error. */
ret_status ret_last_device_status(void *stream);

/* Number of kernels this library has launched in this process so far, over
 * all devices and threads (benchmarks count their launches with it). */
unsigned long long ret_kernel_launches(void);

/* Static, NUL-terminated description of a status code. */
const char *ret_status_string(ret_status status);

/*
 * ret_msr_gammas -- section 2.2: the decay of head h of the multi-scale
 * retention layer, gamma_h = 1 - 2^(-5-h) for h = 0 .. H-1 (short windows
 * for the first heads, long ones for the last).  A host function: it writes
 * the H doubles of `gamma` (HOST memory, caller-owned), ready to be the
 * `gamma` array of a ret_desc.  Errors: RET_ERR_NULL, RET_ERR_SHAPE for H
 * outside 1..RET_MAX_HEADS.
 */
ret_status ret_msr_gammas(int H, double *gamma);

#ifdef __cplusplus
}
#endif

#endif /* RETENTION_H */
