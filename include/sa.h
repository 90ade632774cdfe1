/*
 * sa.h -- C ABI of the Sketch Attention (SA) compression library (libsa.so).
 *
 * What it computes.  One SA layer of SequenceO1, as section 2.1 ("Sketch
 * Attention") of the reading notes "SequenceO1：用可缓存的低秩草图实现端到端十万级用户历史建模"
 * defines it.  For each user b with history X_b (n_b x d, one row per
 * behaviour), shared prototypes P (k x d) and projections W_Q, W_K (d x d):
 *
 *     S   = (P W_Q)(X_b W_K)^T * scale                 k x n_b affinities
 *     A   = softmax of S over the PROTOTYPE axis j      every column sums to 1
 *     X~_b = A X_b                                      k x d sketch, no value projection
 *     m_b  = A 1                                        k per-prototype masses
 *
 * (sum_j m_bj = n_b; X~_bj / m_bj is the mass-normalised sketch.)  The
 * library evaluates S through Q' = P W_Q W_K^T * scale, the rearrangement
 * section 1 of the same notes describes for single-query cross-attention,
 * so the key projection X W_K is never formed; and it fuses affinity,
 * stable softmax and aggregation in one pass over X without writing the
 * k x n matrices to memory, as section 2.4 describes for FlashSA, over
 * ragged batches.
 *
 * Conventions.
 *  - Device pointers are CUDA device memory of the current device (the one
 *    current when the query was prepared).  Host pointers are host memory.
 *  - All arrays are dense and row-major.  bf16 data is IEEE bfloat16 bit
 *    patterns (uint16); fp32 data is IEEE binary32.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Device-side work is enqueued on it and runs asynchronously unless an
 *    entry point says otherwise.
 *  - The caller owns every buffer it passes; the library owns only what is
 *    inside an sa_query (freed by sa_sketch_free).
 *  - Host-side argument errors are reported immediately and nothing is
 *    enqueued.  Offsets live on the device, so their validity is checked on
 *    the device: a bad offsets array never causes an out-of-bounds access,
 *    but it makes the outputs unspecified and raises a device flag that
 *    sa_read_device_status reports.
 */
#ifndef SA_H_
#define SA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum sa_status {
  SA_OK = 0,
  SA_ERR_INVALID_ARG = 1,  /* null pointer, bad size, misaligned buffer, wrong device */
  SA_ERR_UNSUPPORTED = 2,  /* shape/dtype/GPU without a kernel in this build */
  SA_ERR_WORKSPACE = 3,    /* workspace smaller than sa_workspace_bytes() */
  SA_ERR_CUDA = 4,         /* a CUDA runtime call or kernel launch failed */
  SA_ERR_DEVICE_FLAG = 5   /* a kernel flagged bad offsets or a timed-out wait */
} sa_status;

typedef enum sa_dtype {
  SA_BF16 = 0, /* bf16 inputs, tensor-core pass, fp32 accumulation */
  SA_FP32 = 1  /* fp32 inputs, CUDA-core pass, fp64 accumulation */
} sa_dtype;

/* Device flag bits reported through sa_read_device_status. */
#define SA_DEVFLAG_OFFSET0_NONZERO 1u  /* offsets[0] != 0 */
#define SA_DEVFLAG_OFFSETS_DECREASE 2u /* offsets[b] > offsets[b+1] for some b */
#define SA_DEVFLAG_OFFSET_LAST 4u      /* offsets[batch] != total_rows */
#define SA_DEVFLAG_TIMEOUT 8u          /* a kernel's bounded wait gave up */
#define SA_DEVFLAG_SMEM_ALIGN 16u      /* a kernel found its shared memory misaligned (no work done) */
#define SA_DEVFLAG_ACTION_TYPE 32u     /* an action type id >= the producer's n_types */

/* Opaque handle: the precomputed query Q' for one weight set. */
typedef struct sa_query_s* sa_query;

/*
 * sa_prepare_query -- precompute Q' = P W_Q W_K^T * scale (times log2 e) for
 * one set of SA parameters (section 2.1: P^(0) in R^{k x d}, W_Q, W_K in
 * R^{d x d}; section 1: the query/key rearrangement).
 *
 *   P     device, k x d, dtype          shared prototypes P^(0)
 *   W_Q   device, d x d, dtype          query projection
 *   W_K   device, d x d, dtype          key projection
 *   k     1 <= k <= 1024                number of prototypes
 *   d     64, 128 or 256                embedding width
 *   scale finite                        affinity scale (1/sqrt(d) in the paper's setting)
 *   dtype SA_BF16 or SA_FP32            element type of P, W_Q, W_K and of X later
 *   stream                              the precompute kernel runs on it
 *   out   host; receives the handle
 *
 * Allocates device memory (cudaMalloc) for Q' and for W_Q W_K^T * scale
 * (d x d fp32, used by sa_sketch_forward_user_queries).  P, W_Q and W_K are read by
 * a kernel enqueued on `stream`; they must stay alive until it completes.
 * Returns SA_ERR_UNSUPPORTED for shapes without a kernel, or for a GPU
 * other than sm_100.  bf16: d = 64 and 128 take any k <= 1024 (k > 128 runs
 * on clusters of ceil(k / 128) CTAs, each holding 128 prototypes; section
 * 2.2 of the notes puts the final layers at about a thousand prototypes),
 * d = 256 takes k <= 256 (k > 64 on pairs of CTAs).  fp32: k <= 256.
 */
sa_status sa_prepare_query(const void* P, const void* W_Q, const void* W_K, int k, int d,
                           float scale, sa_dtype dtype, void* stream, sa_query* out);

/* Releases a query and its device memory (synchronises with the device).
 * NULL is a no-op. */
void sa_sketch_free(sa_query q);

/* Bytes of device workspace sa_sketch_forward needs for a batch of `batch`
 * users and `total_rows` rows.  Independent of the batch size beyond a fixed
 * bound (it scales with the number of SMs, not with the number of users).
 * Per-user queries need more: sa_workspace_bytes_user_queries. */
size_t sa_workspace_bytes(sa_query q, int64_t batch, int64_t total_rows);

/*
 * sa_sketch_forward -- one SA layer over a ragged batch (section 2.1; ragged
 * batches and fused tiling: section 2.4).
 *
 *   q           prepared query
 *   X           device, total_rows x d, q's dtype; user b owns rows
 *               [offsets[b], offsets[b+1]).  16-byte aligned.
 *   offsets     device, int64, batch + 1 entries: offsets[0] == 0,
 *               non-decreasing, offsets[batch] == total_rows.  No padding:
 *               rows outside a user's range never contribute to it
 *               (section 3.1: padding must not receive mass).
 *   batch       number of users B >= 0
 *   total_rows  N >= 0, < 2^31 - 256
 *   X_tilde     device out, B x k x d fp32 (16-byte aligned): the sketches
 *   mass        device out, B x k fp32: m_bj = sum_i A_ji
 *   workspace   device, >= sa_workspace_bytes(q, B, N) bytes, 256-byte
 *               aligned; no initial contents needed; one call at a time
 *   stream      work is enqueued here; outputs are ready when it is done
 *
 * A user with no rows gets X~ = 0 and m = 0.  Results are bitwise
 * reproducible for the same inputs on the same GPU model.
 */
sa_status sa_sketch_forward(sa_query q, const void* X, const int64_t* offsets, int64_t batch,
                            int64_t total_rows, float* X_tilde, float* mass, void* workspace,
                            size_t workspace_bytes, void* stream);

/*
 * sa_sketch_forward_user_queries -- the SA step of a refinement layer: user
 * b's rows are queried by its own k x d matrix Q_b in place of P (section
 * 2.2 "Stacked Refinement" of the same notes: layer l starts from the shared
 * prototypes and queries the original X with the previous layer's sketch).
 * For each user b:
 *
 *     S_b = (Q_b W_Q)(X_b W_K)^T * scale,  A_b = softmax over prototypes,
 *     X~_b = A_b X_b,  m_b = A_b 1
 *
 * with W_Q, W_K and scale those of `q` (its P is not used).  The library
 * forms Q'_b = Q_b (W_Q W_K^T * scale) in fp32 for every user (a kernel on
 * `stream`, into the workspace) and runs the same fused pass, which loads
 * each user's Q'_b where that user's rows begin.
 *
 *   q           prepared query (supplies d, k, dtype, W_Q, W_K, scale)
 *   queries     device, B x k x d fp32 (4-byte aligned): Q_b for every user
 *               (for example the previous layer's X~, or a function of it);
 *               not modified
 *   X, offsets, batch, total_rows, X_tilde, mass, stream
 *               as for sa_sketch_forward
 *   workspace   device, >= sa_workspace_bytes_user_queries(q, B, N) bytes,
 *               256-byte aligned; one call at a time
 *
 * Every query shape that sa_sketch_forward runs takes per-user queries.
 * Returns SA_ERR_INVALID_ARG if queries is NULL with B > 0 or if B * k_pad
 * reaches 2^31 (k_pad as sa_query_info reports), otherwise as
 * sa_sketch_forward.  An empty user gets X~ = 0 and m = 0 whatever its Q_b.
 */
size_t sa_workspace_bytes_user_queries(sa_query q, int64_t batch, int64_t total_rows);
/* The first two of the three kernels (Q'_b for every user, then the fused
 * pass); sa_sketch_finalize with the same arguments (minus `queries`)
 * completes the layer, as for sa_sketch_partials. */
sa_status sa_sketch_partials_user_queries(sa_query q, const float* queries, const void* X,
                                          const int64_t* offsets, int64_t batch,
                                          int64_t total_rows, float* X_tilde, float* mass,
                                          void* workspace, size_t workspace_bytes, void* stream);
sa_status sa_sketch_forward_user_queries(sa_query q, const float* queries, const void* X,
                                         const int64_t* offsets, int64_t batch,
                                         int64_t total_rows, float* X_tilde, float* mass,
                                         void* workspace, size_t workspace_bytes, void* stream);

/*
 * The two kernels sa_sketch_forward enqueues, for callers that schedule (or
 * time) them separately.  sa_sketch_partials runs the fused pass over X,
 * writing users that lie inside one CTA's row range to the outputs and the
 * others to partial slots in the workspace; sa_sketch_finalize then sums the
 * partial slots in a fixed order, zero-fills empty users and validates the
 * offsets.  Calling both, in this order, on one stream with the same
 * arguments equals sa_sketch_forward.
 */
sa_status sa_sketch_partials(sa_query q, const void* X, const int64_t* offsets, int64_t batch,
                             int64_t total_rows, float* X_tilde, float* mass, void* workspace,
                             size_t workspace_bytes, void* stream);
sa_status sa_sketch_finalize(sa_query q, const void* X, const int64_t* offsets, int64_t batch,
                             int64_t total_rows, float* X_tilde, float* mass, void* workspace,
                             size_t workspace_bytes, void* stream);

/*
 * sa_sketch_forward_host -- the same layer on HOST buffers (end-to-end use).
 *
 *   X_host        host, total_rows x d, q's dtype (pinned memory copies fastest)
 *   offsets_host  host, batch + 1 int64 (validated on the host before any copy)
 *   X_tilde_host  host out, B x k x d fp32
 *   mass_host     host out, B x k fp32
 *   device_buffer device, >= sa_host_path_device_bytes(q, B, N), 256-byte aligned
 *
 * Copies X and the offsets to device_buffer, runs sa_sketch_forward there,
 * copies the results back and synchronises `stream` before returning.
 */
size_t sa_host_path_device_bytes(sa_query q, int64_t batch, int64_t total_rows);
sa_status sa_sketch_forward_host(sa_query q, const void* X_host, const int64_t* offsets_host,
                                 int64_t batch, int64_t total_rows, float* X_tilde_host,
                                 float* mass_host, void* device_buffer,
                                 size_t device_buffer_bytes, void* stream);

/*
 * sa_read_device_status -- synchronises `stream`, reads the device flags of
 * the last call that used `workspace` and clears them.  Returns SA_OK if no
 * flag was set, SA_ERR_DEVICE_FLAG otherwise (with the SA_DEVFLAG_* bits in
 * *flags_out if it is not NULL), SA_ERR_CUDA if the copy failed.
 */
sa_status sa_read_device_status(void* workspace, size_t workspace_bytes, void* stream,
                                uint32_t* flags_out);

/*
 * sa_sketch_forward_noalloc -- sa_sketch_forward for callers that cannot
 * allocate device memory.  (The SequenceO1 paper has no counterpart to this
 * entry point; it exists for callers of this library.)
 *
 * Some callers cannot call cudaMalloc or any other allocator where they run
 * the SA layer: code inside an allocator's own hooks, code under a memory
 * pool that must not grow, or hosts that hand the library only fixed,
 * pre-registered buffers.  This call takes the same inputs and outputs as
 * sa_sketch_forward, but in place of a caller-provided workspace it uses a
 * fixed 32 MiB scratch array inside the library's device image.  Every GPU
 * that loads the library's module holds that array until the process exits.
 * Under CUDA's default lazy module loading the module, and with it the
 * array, is loaded on a device by the first call there; a call with
 * batch = 0 does only that set-up, so a caller can make it while allocating
 * is still allowed.  Later calls allocate nothing.
 *
 *   q, X, offsets, batch, total_rows, X_tilde, mass, stream
 *                     as for sa_sketch_forward
 *   device_flags_out  device, 2 uint32 words (4-byte aligned), or NULL:
 *                     receives, in stream order, this call's device flags
 *                     (word 0: the SA_DEVFLAG_OFFSET* bits, word 1:
 *                     SA_DEVFLAG_TIMEOUT and SA_DEVFLAG_SMEM_ALIGN), which sa_read_device_status
 *                     reports for the workspace path
 *
 * Returns SA_ERR_WORKSPACE when the call needs more scratch than the array
 * holds (sa_workspace_bytes(q, batch, total_rows) > 32 MiB; this covers
 * every query with k * d <= 128 * 128 on a 148-SM GPU), SA_ERR_CUDA if the
 * array's address cannot be looked up, and otherwise what sa_sketch_forward
 * returns.
 *
 * The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current) and caches it with the
 * ID of the device's context; make that first call before any stream
 * capture on the device.  After a device reset the next call runs in a new
 * context and looks the address up again (the module is reloaded then).
 * All calls share the one array, so calls whose work overlaps on the GPU
 * (other streams, other host threads) race on it and give wrong results:
 * serialise them.
 */
sa_status sa_sketch_forward_noalloc(sa_query q, const void* X, const int64_t* offsets,
                                    int64_t batch, int64_t total_rows, float* X_tilde,
                                    float* mass, uint32_t* device_flags_out, void* stream);

/*
 * sa_mass_normalise -- the mass-normalised sketch X~_bj / m_bj (0 where
 * m_bj == 0), the weighted mean of user b's rows under prototype j (section
 * 2.1: the sketch is a weighted aggregation; its masses make it a mean),
 * e.g. as the query of the next refinement layer (section 2.2).
 *
 *   X_tilde  device, batch x k x d fp32 (16-byte aligned), as written by
 *            sa_sketch_forward
 *   mass     device, batch x k fp32
 *   batch    B >= 0;  k >= 1;  d >= 4, a multiple of 4
 *   out      device, batch x k x d fp32 (16-byte aligned); may be X_tilde
 *   stream   the kernel is enqueued here
 *
 * Returns SA_ERR_INVALID_ARG for bad sizes, null pointers or misalignment.
 */
sa_status sa_mass_normalise(const float* X_tilde, const float* mass, int64_t batch, int k, int d,
                            float* out, void* stream);

/*
 * sa_sketch_backward -- gradients of one SA layer (section 2.2 of the notes:
 * the compression module is trained end to end by the ranking loss; the
 * page prints no backward, so these follow from section 2.1's forward by
 * the chain rule).  For upstream gradients G_b = dL/dX~_b and g_b = dL/dm_b:
 *
 *     dA  = G X^T + g 1^T,   dS = A * (dA - 1 c^T),  c_i = sum_j A_ji dA_ji
 *     dX  = A^T G + dS^T Q'              (Q' = P W_Q W_K^T * scale)
 *     R   = dS X,   dP = scale R W_K W_Q^T,
 *     dW_Q = scale P^T R W_K,   dW_K = scale R^T P W_Q
 *
 * One tcgen05 pass over X recomputes the softmax per 128-row tile (no saved
 * activations), writes dX and accumulates R per user; small GEMMs turn R
 * into the parameter gradients.
 *
 *   q           prepared bf16 query with d in {64, 128} and k <= 128
 *               (others: SA_ERR_UNSUPPORTED)
 *   queries     device B x k x d fp32 (per-user queries, as for
 *               sa_sketch_forward_user_queries) or NULL (the shared P)
 *   P_f32       device k x d fp32: the prototypes q was prepared with (read
 *               only when queries is NULL)
 *   W_Q_f32, W_K_f32   device d x d fp32: the projections q was prepared with
 *   X, offsets, batch, total_rows   as for sa_sketch_forward
 *   G           device B x k x d fp32: dL/dX~
 *   g           device B x k fp32: dL/dm, or NULL (zero)
 *   dX          device out, total_rows x d bf16 (16-byte aligned)
 *   dP          device out, k x d fp32 summed over users (shared P), or
 *               B x k x d fp32 per user (with queries: dL/dQ_b)
 *   dW_Q, dW_K  device out, d x d fp32, summed over users
 *   workspace   device, >= sa_workspace_bytes_backward(q, B, N) bytes,
 *               256-byte aligned; one call at a time
 *
 * Device flags (bad offsets, timeouts) are read with sa_read_device_status
 * on the workspace.  Rows of empty users contribute nothing.
 */
size_t sa_workspace_bytes_backward(sa_query q, int64_t batch, int64_t total_rows);
sa_status sa_sketch_backward(sa_query q, const float* queries, const float* P_f32,
                             const float* W_Q_f32, const float* W_K_f32, const void* X,
                             const int64_t* offsets, int64_t batch, int64_t total_rows,
                             const float* G, const float* g, void* dX, float* dP, float* dW_Q,
                             float* dW_K, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Stacked refinement layers (section 2.2 "Stacked Refinement" of the same
 * notes).  Layer l queries the ORIGINAL history X with the previous layer's
 * sketches (layer 1 with the shared prototypes: X~^(0) = P^(0)) and then
 * updates every (user, prototype) row of width d:
 *
 *     z   = LN1(prev_bj + X~_bj / m_bj)          (X~/m is 0 where m_bj = 0)
 *     out = LN2(z + (SiLU(z W1) * (z W3)) W2)
 *
 * where X~, m are that layer's SA outputs, LN normalises over the d features
 * (biased variance, eps 1e-5) with gain gamma and shift beta, and the FFN is
 * SwiGLU-gated with hidden width h and no biases.  The page lost the layer's
 * formulas; this is the reading its text supports (the aggregation added to
 * the previous state and normalised, then a residual feed-forward network):
 * the aggregation enters mass-normalised, a weighted mean of the user's
 * rows, whose scale does not grow with the history length.  Every layer has
 * its own sa_query (W_Q, W_K, scale) and sa_refine (LN and FFN parameters).
 */
typedef struct sa_refine_s* sa_refine;

/*
 * sa_prepare_refine -- the LN and FFN parameters of one refinement layer.
 *
 *   W1, W3   device, d x h fp32, row-major (z W1, z W3)
 *   W2       device, h x d fp32, row-major
 *   gamma1, beta1, gamma2, beta2   device, d fp32 each (LN1, LN2)
 *   d        64 or 128 (256: SA_ERR_UNSUPPORTED)
 *   h        hidden width, a multiple of 128, 128 <= h <= 4096
 *   stream   the copies (bf16, transposed) are made by kernels on it
 *   out      host; receives the handle
 *
 * Allocates device memory for the parameters; the inputs may be freed once
 * `stream` has passed this call.  Errors: SA_ERR_INVALID_ARG (null,
 * misaligned, bad d or h), SA_ERR_UNSUPPORTED (d = 256, or not sm_100),
 * SA_ERR_CUDA.
 */
sa_status sa_prepare_refine(const float* W1, const float* W3, const float* W2,
                            const float* gamma1, const float* beta1, const float* gamma2,
                            const float* beta2, int d, int h, void* stream, sa_refine* out);

/* Releases a refinement handle and its device memory.  NULL is a no-op. */
void sa_refine_free(sa_refine r);

/*
 * sa_refine_update -- the update after a layer's SA step, for batch * k rows
 * (one tcgen05 kernel: LN1, the FFN on the tensor cores in bf16 with fp32
 * accumulation, LN2; the norms in fp32).
 *
 *   prev         device fp32, 16-byte aligned: batch x k x d, or k x d
 *                shared by every user when prev_shared != 0 (layer 1: P)
 *   X_tilde      device, batch x k x d fp32 (16-byte aligned): the layer's
 *                SA sketches
 *   mass         device, batch x k fp32: the layer's masses
 *   batch, k     batch >= 0, k >= 1
 *   out          device, batch x k x d fp32 (16-byte aligned); must not
 *                overlap the inputs
 *   device_flags device uint32 (or NULL): SA_DEVFLAG_TIMEOUT is OR-ed in if
 *                a bounded wait in the kernel gave up
 *   stream       the kernel is enqueued here
 */
sa_status sa_refine_update(sa_refine r, const float* prev, int prev_shared, const float* X_tilde,
                           const float* mass, int64_t batch, int k, float* out,
                           uint32_t* device_flags, void* stream);

/*
 * sa_refine_layer_forward -- one refinement layer over a ragged batch: the
 * SA step (section 2.1 with the layer's query; per-user queries for l >= 2)
 * followed by sa_refine_update.
 *
 *   q          the layer's SA query (its W_Q, W_K, scale; its P for layer 1)
 *   r          the layer's LN and FFN parameters (same d as q; q bf16)
 *   prev       device fp32: NULL for layer 1 (the query and the residual are
 *              the shared prototypes, given as P_f32), else the previous
 *              layer's sketches, batch x k x d
 *   P_f32      device, k x d fp32: the prototypes q was prepared with, as
 *              fp32 (read only when prev is NULL)
 *   X, offsets, batch, total_rows   as for sa_sketch_forward
 *   out        device, batch x k x d fp32: X~^(l); must not overlap prev
 *   workspace  device, >= sa_workspace_bytes_refine_layer(q, batch,
 *              total_rows), 256-byte aligned; one call at a time
 *
 * Device flags (bad offsets, timeouts) are read with sa_read_device_status
 * on the workspace, as for sa_sketch_forward.
 */
size_t sa_workspace_bytes_refine_layer(sa_query q, int64_t batch, int64_t total_rows);
sa_status sa_refine_layer_forward(sa_query q, sa_refine r, const float* prev, const float* P_f32,
                                  const void* X, const int64_t* offsets, int64_t batch,
                                  int64_t total_rows, float* out, void* workspace,
                                  size_t workspace_bytes, void* stream);

/*
 * sa_refine_stack_forward -- `layers` refinement layers in sequence (the
 * final configuration of section 2.2 has two): layer 1 from P_f32, each
 * later layer queried by the previous layer's output; every layer reads the
 * original X.  qs[l], rs[l] are layer l's handles (all with the same k, d).
 *
 *   out        device, batch x k x d fp32: X~^(layers)
 *   workspace  device, >= sa_workspace_bytes_refine_stack(qs[0], batch,
 *              total_rows) (which also holds the layers' intermediate
 *              sketches), 256-byte aligned
 */
size_t sa_workspace_bytes_refine_stack(sa_query q, int64_t batch, int64_t total_rows);
sa_status sa_refine_stack_forward(int layers, const sa_query* qs, const sa_refine* rs,
                                  const float* P_f32, const void* X, const int64_t* offsets,
                                  int64_t batch, int64_t total_rows, float* out, void* workspace,
                                  size_t workspace_bytes, void* stream);

/*
 * Sketch cache (section 2.4 "Local KVCache" of the same notes; section 2.3,
 * Figure 2: hit -> the stored sketch, miss -> one compression).  Only the
 * user-side sketch (X~_b and m_b, k x d and k fp32) is stored, keyed by the
 * user, the model version, the history timestamp and the sketch
 * configuration, for a time-to-live, in a device pool of `capacity` slots.
 * Times are seconds on any clock the caller chooses (passed as `now`).
 *
 * Decisions (the page names the key, the TTL and capacity eviction and no
 * more; this is the reading built):
 *  - an entry is fresh while now - t_insert < ttl; a lookup that finds an
 *    expired entry counts a miss and drops it;
 *  - a hit refreshes the entry's last-use time;
 *  - an insert of a new key takes the free slot with the smallest index,
 *    else evicts the expired entry inserted earliest, else the least
 *    recently used entry (ties: the smaller slot);
 *  - inserting a key that is present replaces its sketch in place and
 *    restarts its TTL; within one call, of two equal keys the later wins.
 * The index is host memory guarded by a mutex; the sketches move only on
 * the device.  Calls on one cache that move data (lookup, insert, forward)
 * must be ordered with one another by the caller: the library reuses one
 * device slot list, so use one stream per cache.  Every call must be made
 * with the cache's device current (SA_ERR_INVALID_ARG otherwise), and `now`
 * must be finite (SA_ERR_INVALID_ARG otherwise).  SA_ERR_CUDA from a call
 * also covers a failed host allocation in the index; the cache's index may
 * then be partly updated, so free the cache.
 */
typedef struct sa_cache_key {
  int64_t user;
  int64_t model_version;
  int64_t history_ts;
  int64_t config;
} sa_cache_key;

typedef struct sa_cache_s* sa_cache;

/* A cache of `capacity` sketches of k x d (k >= 1, d >= 4 and a multiple of
 * 4, capacity >= 1) with a time-to-live of ttl_seconds (> 0).  Allocates
 * capacity * k * (d + 1) * 4 bytes on the current device (SA_ERR_INVALID_ARG
 * if that count does not fit in size_t).  Errors: SA_ERR_INVALID_ARG,
 * SA_ERR_CUDA. */
sa_status sa_cache_create(int k, int d, int64_t capacity, double ttl_seconds, sa_cache* out);

/* Waits for the cache's device, then releases the cache and its device
 * memory (any device may be current; it is current again on return).  NULL
 * is a no-op. */
void sa_cache_free(sa_cache c);

/*
 * sa_cache_lookup -- for each of `batch` keys (host array): hit[b] (host
 * out) = 1 if a fresh entry exists, else 0; for each hit a kernel on
 * `stream` copies the entry into X_tilde[b] (device, batch x k x d fp32,
 * 16-byte aligned) and mass[b] (device, batch x k fp32).  Rows of misses
 * are left as they were.  The decisions are taken on the host before the
 * call returns; the copies complete with the stream.
 */
sa_status sa_cache_lookup(sa_cache c, const sa_cache_key* keys, int64_t batch, double now,
                          uint8_t* hit, float* X_tilde, float* mass, void* stream);

/*
 * sa_cache_insert -- stores X_tilde[b], mass[b] (device, layout as for
 * lookup) under keys[b] (host) at time `now`, evicting as described above.
 * The copies are kernels on `stream`; the sources must stay unchanged until
 * they complete.
 */
sa_status sa_cache_insert(sa_cache c, const sa_cache_key* keys, int64_t batch, double now,
                          const float* X_tilde, const float* mass, void* stream);

/* Host-side counters: entries held, hits, misses (expired ones included),
 * evictions.  Any pointer may be NULL. */
sa_status sa_cache_stats(sa_cache c, int64_t* entries, int64_t* hits, int64_t* misses,
                         int64_t* evictions);

/*
 * sa_cache_forward -- one SA layer served through the cache: look the keys
 * up and copy the hits to the outputs; each run of consecutive missed users
 * (whose rows and outputs are contiguous) is compressed in place by one
 * sa_sketch_forward over its range of X, and its sketches are inserted.
 *
 *   c, q           a cache and a prepared query of the same k and d
 *   keys           host, batch keys
 *   offsets_host   host, batch + 1 int64 (validated on the host): the same
 *                  ragged layout as sa_sketch_forward's device offsets
 *   X              device, total_rows x d, q's dtype, 16-byte aligned
 *   X_tilde, mass  device outputs as for sa_sketch_forward
 *   hit            host out, batch bytes: 1 where the cache served the user
 *   workspace      device, >= sa_cache_forward_workspace_bytes(q, batch,
 *                  total_rows), 256-byte aligned; the SA pass's device
 *                  flags are read with sa_read_device_status on it, as for
 *                  sa_sketch_forward
 *
 * Returns once the host work is done and everything is enqueued on `stream`.
 */
size_t sa_cache_forward_workspace_bytes(sa_query q, int64_t batch, int64_t total_rows);
sa_status sa_cache_forward(sa_cache c, sa_query q, const sa_cache_key* keys, double now,
                           const void* X, const int64_t* offsets_host, int64_t batch,
                           int64_t total_rows, float* X_tilde, float* mass, uint8_t* hit,
                           void* workspace, size_t workspace_bytes, void* stream);

/*
 * Width adapter (section 2.3): Y = X~ W_A with W_A in R^{d x D} and no bias,
 * mapping every sketch row to the ranking model's width (D = 1024 in the
 * final configuration).  The adapted sketch is shared by a request's targets
 * but not cached (section 2.4).  One tcgen05 kernel: X~ rounded to bf16,
 * W_A held as bf16, fp32 accumulation, Y written as bf16.
 */
typedef struct sa_adapter_s* sa_adapter;

/* W_A: device, d x D fp32 (4-byte aligned); d 64 or 128; D a positive
 * multiple of 256.  A kernel on `stream` makes the bf16 copy; W_A may be
 * freed once the stream has passed this call.  Errors: SA_ERR_INVALID_ARG,
 * SA_ERR_UNSUPPORTED (not sm_100), SA_ERR_CUDA. */
sa_status sa_prepare_adapter(const float* W_A, int d, int D, void* stream, sa_adapter* out);

/* Releases an adapter.  NULL is a no-op. */
void sa_adapter_free(sa_adapter a);

/*
 * sa_adapter_forward -- Y (device out, rows x D bf16, 16-byte aligned) =
 * X_tilde (device, rows x d fp32, 16-byte aligned) W_A, for rows = batch * k
 * sketch rows.  device_flags (device uint32, or NULL): SA_DEVFLAG_TIMEOUT or
 * SA_DEVFLAG_SMEM_ALIGN is OR-ed in if the kernel gave up.
 */
sa_status sa_adapter_forward(sa_adapter a, const float* X_tilde, int64_t rows, void* out,
                             uint32_t* device_flags, void* stream);

/*
 * Action-side fusion (section 2.2 "Stacked Refinement 与动作侧融合" of the
 * same notes): the producer of the history matrix X.  For behaviour i with
 * item embedding e_i (d wide) and action type id t_i:
 *
 *     x_i = e_i + (SiLU(z_i W1) * (z_i W3)) W2,   z_i = [e_i ; table[t_i]],
 *
 * W1, W3 (d + d_a) x h with the e-rows first, W2 h x d, no biases, the
 * action table n_types x d_a.  The page gives the abstract form (a SwiGLU
 * network over the concatenation, residual on e_i) and no more; this is
 * the reading built.  The library folds table W1[d:] and table W3[d:] into
 * per-type rows at prepare time, so the producer's products have K = d.
 */
typedef struct sa_action_s* sa_action;

/*
 * sa_prepare_action -- the producer's parameters.
 *
 *   W1, W3        device, (d + d_a) x h fp32, row-major, 4-byte aligned
 *   W2            device, h x d fp32
 *   action_table  device, n_types x d_a fp32
 *   d             64 or 128
 *   d_a           1 <= d_a <= 4096
 *   h             a multiple of 64, 64 <= h <= 4096
 *   n_types       1 <= n_types <= 16
 *   stream        the bf16 copies and the per-type rows are made by a kernel
 *                 on it; the inputs may be freed once the stream has passed
 *                 this call
 *
 * Errors: SA_ERR_INVALID_ARG, SA_ERR_UNSUPPORTED (not sm_100), SA_ERR_CUDA.
 */
sa_status sa_prepare_action(const float* W1, const float* W3, const float* W2,
                            const float* action_table, int d, int d_a, int h, int n_types,
                            void* stream, sa_action* out);

/* Waits for the producer's device, then releases the producer (any device
 * may be current; it is current again on return).  NULL is a no-op. */
void sa_action_free(sa_action act);

/*
 * sa_action_fuse -- X = the fused rows for `rows` behaviours (one tcgen05
 * kernel; bf16 products with fp32 accumulation, the gate in fp32, X rounded
 * to bf16).
 *
 *   E             device, rows x d bf16, 16-byte aligned: item embeddings
 *   types         device, rows uint8: action type ids; an id >= n_types
 *                 contributes no action term and raises SA_DEVFLAG_ACTION_TYPE
 *   rows          0 <= rows < 2^31 - 256
 *   X             device out, rows x d bf16, 16-byte aligned; must not
 *                 overlap E
 *   device_flags  device uint32 (or NULL): SA_DEVFLAG_* bits OR-ed in
 */
sa_status sa_action_fuse(sa_action act, const void* E, const uint8_t* types, int64_t rows, void* X,
                         uint32_t* device_flags, void* stream);

/*
 * sa_action_sketch_forward -- the producer followed by one SA layer over its
 * output: X is written to the workspace and compressed by sa_sketch_forward
 * (q bf16, the same d as act).  offsets, batch, total_rows, X_tilde, mass
 * as for sa_sketch_forward; workspace >=
 * sa_workspace_bytes_action_sketch(q, batch, total_rows), 256-byte aligned.
 * Device flags of both kernels are read with sa_read_device_status on the
 * workspace.
 */
size_t sa_workspace_bytes_action_sketch(sa_query q, int64_t batch, int64_t total_rows);
sa_status sa_action_sketch_forward(sa_action act, sa_query q, const void* E, const uint8_t* types,
                                   const int64_t* offsets, int64_t batch, int64_t total_rows,
                                   float* X_tilde, float* mass, void* workspace,
                                   size_t workspace_bytes, void* stream);

/* Static description of a status code. */
const char* sa_status_string(sa_status s);

/* Shape of a prepared query: k, d, dtype, and the padded prototype count
 * the tensor-core pass uses (0 for fp32). */
sa_status sa_query_info(sa_query q, int* k, int* d, int* dtype, int* k_pad);

#ifdef __cplusplus
}
#endif

#endif /* SA_H_ */
