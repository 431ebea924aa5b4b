/*
 * tsp.h - C ABI of the TSP (Tensor + Sequence Parallelism) per-rank layer
 * forward, and the backward of its MLP half, for NVIDIA B200 (sm_100a).
 *
 * The method (zubnet.ai news item "Zyphra TSP folds TP+SP onto one GPU
 * axis", paragraphs 1-2): tensor parallelism (weights split) and sequence
 * parallelism (tokens split) are folded onto ONE mesh axis of size D.  Each
 * rank holds 1/D of the weights and 1/D of the tokens.  For attention the
 * weight shards are broadcast one after another and every rank applies each
 * shard to its own tokens; K/V are all-gathered under a zigzag sequence
 * partition.  For the MLP a ring passes the weight shards point to point, so
 * the MLP output is a sum of shard contributions computed locally and no
 * all-reduce is needed.
 *
 * This library computes what ONE rank computes for one dense decoder layer.
 * On one GPU the broadcast, ring and all-gather become loops over shard
 * pointers that already sit in device memory; ranks can be run one after
 * another.  Layer form: pre-LayerNorm (gamma=1, beta=0, biased variance,
 * eps inside the square root), multi-head causal attention with as many K/V
 * heads as Q heads and no positional encoding, GELU (tanh form), no biases:
 *
 *     Y1 = X + Attn(LN1(X)) Wo,       Y = Y1 + GELU(LN2(Y1) W1) W2.
 *
 * Conventions shared by every call
 *   - All matrices are row-major.  "K-major [n, k]" means n rows of k
 *     contiguous elements (the layout of a Linear layer's weight).
 *   - Tokens: the T-token sequence is cut into 2D chunks of c = T/(2D)
 *     tokens; rank r holds chunk r then chunk 2D-1-r.  "Rank-local order"
 *     is that order: local row i < c is global position r*c + i, local row
 *     i >= c is global position (2D-1-r)*c + (i-c).  L = 2c local tokens.
 *   - Shard k of the attention weights is head group k (heads
 *     k*H/D .. (k+1)*H/D-1, i.e. hidden columns k*h/D .. (k+1)*h/D-1); shard
 *     k of the FFN is FFN columns k*F/D .. (k+1)*F/D-1.
 *   - K/V full-sequence tensors are [T, h] fp16 in natural (global) order,
 *     head j in columns j*d .. (j+1)*d-1.
 *   - Number formats: the model's tensors (X, the weights, Y) are bf16; the
 *     operands of every matmul inside the layer (LayerNorm outputs, Q, K, V,
 *     softmax probabilities, attention output, GELU output, weight shards)
 *     are held in fp16 - the same 16 bits and tensor-core rate, three more
 *     significand bits - with fp32 accumulation; the residual stream
 *     X + attention is fp32.  Conversions round to nearest even and
 *     saturate at +-65504.
 *   - Every device buffer is allocated and freed by the caller.  Functions
 *     that take a stream only enqueue work on it (asynchronous) unless
 *     stated otherwise; the library allocates no device memory and keeps no
 *     state between calls.  One exception: tsp_kv_project_noalloc's scratch
 *     is a 64 MiB file-scope device array of this library (held on every
 *     device that loads it until exit), whose device address the library
 *     caches per device and CUDA context; that array keeps the last call's
 *     contents, and calls that overlap on the GPU race on it.
 *   - Every entry point and launch step is an NVTX range (named after the
 *     call) for Nsight timelines.
 *   - Host-detectable errors are returned synchronously and nothing is
 *     enqueued.  There is no fallback path: an unsupported shape is an
 *     error.  Device-side events are recorded in a status section (a status
 *     word, then a flags word) at the start of the workspace, of the MLP
 *     backward's workspace and of the packed shard buffer, and reported by
 *     tsp_get_device_status: a bounded wait inside a kernel that ran out
 *     (TSP_ERR_TIMEOUT), or a conversion to fp16 that saturated
 *     (TSP_ERR_SATURATED: a weight beyond +-65504 when packing, or a Q, K,
 *     V, GELU output or recomputed pre-activation beyond it in a GEMM
 *     epilogue).  LayerNorm outputs (|y| < sqrt(h)) and attention outputs (a
 *     convex combination of fp16 V rows) cannot leave the range.
 */
#ifndef TSP_H_
#define TSP_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#define TSP_MAX_D 16
#define TSP_N_STEP_EVENTS 8
#define TSP_N_WS_OFFSETS 9

typedef enum {
  TSP_OK = 0,
  TSP_ERR_INVALID_ARG = 1, /* null pointer, rank out of range, T % 2D != 0, H % D, F % D, ... */
  TSP_ERR_UNSUPPORTED = 2, /* a shape the kernels do not implement (see tsp_check_dims) */
  TSP_ERR_CUDA = 3,        /* a CUDA runtime call failed; see tsp_last_cuda_error */
  TSP_ERR_TIMEOUT = 4,     /* a bounded wait inside a kernel ran out */
  TSP_ERR_WORKSPACE = 5,   /* workspace or buffer smaller than required */
  TSP_ERR_SATURATED = 6,   /* a value outside fp16's range (|x| > 65504) was
                              clamped to +-65504 on conversion: the results are
                              finite but may be wrong (device status only) */
  TSP_ERR_BOUNDS = 7       /* an index check of the debug build (compiled with
                              -DTSP_DEBUG) failed and the access was skipped
                              (device status only; the normal build has none) */
} tsp_status;

/* Layer and sequence sizes. */
typedef struct {
  int64_t T;           /* sequence length (global tokens); T % (2D) == 0 */
  int32_t h;           /* hidden size; h == n_heads * head_dim */
  int32_t n_heads;     /* H: attention heads (Q and K/V) */
  int32_t head_dim;    /* d: 64 or 128 */
  int32_t ffn;         /* F: FFN width */
  float ln_eps;        /* LayerNorm epsilon (1e-5 for the 7B layer) */
  float softmax_scale; /* applied to q.k; 1/sqrt(d) for the 7B layer */
} tsp_dims;

/* Per-shard device pointers (fp16), each shard one contiguous K-major
 * buffer:  wq/wk/wv[k] [h/D, h],  wo[k] [h, h/D],  w1[k] [F/D, h],
 * w2[k] [h, F/D].  Only entries 0..D-1 are read.  Pointers must be 16-byte
 * aligned.  tsp_pack_shards builds them from the bf16 model weights. */
typedef struct {
  int32_t D;
  const void* wq[TSP_MAX_D];
  const void* wk[TSP_MAX_D];
  const void* wv[TSP_MAX_D];
  const void* wo[TSP_MAX_D];
  const void* w1[TSP_MAX_D];
  const void* w2[TSP_MAX_D];
} tsp_weights;

/* Output dtypes of tsp_layer_forward. */
#define TSP_OUT_BF16 0
#define TSP_OUT_F32 1

/* Short English text for a status code (static storage). */
const char* tsp_status_string(int status);

/* Text of the last CUDA error seen by this thread (static per-thread storage). */
const char* tsp_last_cuda_error(void);

/* Checks sizes against what the kernels implement; returns TSP_OK,
 * TSP_ERR_INVALID_ARG or TSP_ERR_UNSUPPORTED.  Supported: head_dim 64 or
 * 128, h % 64 == 0, h <= 8192 (the LayerNorm kernels hold a row as at most
 * 8 groups of 4 values per thread of a 256-thread block), h/D % 64 == 0,
 * F/D % 64 == 0, H % D == 0, F % D == 0, 1 <= D <= TSP_MAX_D,
 * T % (2D) == 0, T < 2^31.  Pure host function. */
int tsp_check_dims(const tsp_dims* dims, int D);

/* Zigzag index map [zubnet.ai TSP item, paragraph 2: "zigzag partition"]:
 * d_idx[i] = global position of rank `rank`'s local token i, for
 * i in [0, T/D).  d_idx: device int32 [T/D].  Bit-exact integer result. */
int tsp_zigzag_index(int64_t T, int D, int rank, int32_t* d_idx, cudaStream_t stream);

/* Bytes of one packed shard buffer for all six weights at this D: a
 * 1 KiB status section (read by tsp_get_device_status on the buffer's base
 * address), then the shards. */
size_t tsp_shard_buffer_bytes(const tsp_dims* dims, int D);

/* Splits full weights into per-rank shards [zubnet.ai TSP item, paragraph 1:
 * "each GPU holds 1/D of the weights"].  w_full[6] = {Wq, Wk, Wv, Wo, W1, W2}
 * are device bf16 in the math orientation y = x W ([in, out]: Wq/Wk/Wv/Wo
 * [h, h], W1 [h, F], W2 [F, h]).  Writes the K-major fp16 shards into d_buf
 * (tsp_shard_buffer_bytes bytes, caller-owned, 16-byte aligned) and fills
 * *out with pointers into d_buf.  A weight beyond +-65504 is clamped and
 * recorded in d_buf's status section (tsp_get_device_status(d_buf, ...)
 * then returns TSP_ERR_SATURATED). */
int tsp_pack_shards(const tsp_dims* dims, int D, const void* const w_full[6],
                    void* d_buf, size_t buf_bytes, tsp_weights* out, cudaStream_t stream);

/* Workspace bytes that tsp_kv_project / tsp_layer_forward / tsp_rank_step
 * need for one rank at this D (activations of L = T/D tokens plus a status
 * word).  The workspace is caller-owned device memory, 256-byte aligned. */
size_t tsp_workspace_bytes(const tsp_dims* dims, int D);

/* Byte offsets inside the workspace of the per-rank intermediates, for
 * inspection after a call and as inputs of the backward (all rank-local
 * order, row-major):
 *   off[0] status section,  off[1] LN output xn fp16 [L, h] (LN2's output
 *   after tsp_layer_forward),  off[2] Q fp16 [L, h],  off[3] attention
 *   output A fp16 [L, h],  off[4] Y1 = X + attention projection, fp32
 *   [L, h],  off[5] H = GELU(LN2(Y1) W1) fp16 [L, F],  off[6] scheduler
 *   counters,  off[7] total bytes,  off[8] the attention's log-sum-exp stash
 *   fp32 [H][2][c_pad]: per head j, local chunk g (0: chunk r, 1: chunk
 *   2D-1-r) and row i of the chunk, log2 of sum_k 2^(scale * log2(e) *
 *   q_i . k_k) over the row's causal keys (c_pad = c rounded up to a
 *   multiple of 128; rows i >= c are not written).  Returns TSP_OK,
 *   TSP_ERR_INVALID_ARG or TSP_ERR_UNSUPPORTED. */
int tsp_workspace_offsets(const tsp_dims* dims, int D, size_t off[TSP_N_WS_OFFSETS]);

/* Clears a status section - the workspace's, the MLP backward workspace's
 * or the shard buffer's: its status and flags words (enqueued on `stream`). */
int tsp_reset_device_status(void* ws, cudaStream_t stream);

/* Synchronises `stream`, then reads a status section (see
 * tsp_reset_device_status): TSP_ERR_TIMEOUT if a bounded wait ran out, else
 * TSP_ERR_BOUNDS if an index check of the debug build failed, else
 * TSP_ERR_SATURATED if an fp16 conversion saturated, else TSP_OK.  All are
 * sticky until tsp_reset_device_status. */
int tsp_get_device_status(const void* ws, cudaStream_t stream);

/* K/V projection of one rank's tokens [zubnet.ai TSP item, paragraph 2:
 * every rank applies each weight shard to its own tokens; K/V are then
 * all-gathered with the zigzag partition]:
 *     K[pos(i)] = LN1(x_local[i]) Wk,   V[pos(i)] = LN1(x_local[i]) Wv
 * for all D shards (head groups), written at the tokens' GLOBAL rows of
 * k_full / v_full ([T, h] fp16) - the place the all-gather puts them.
 * x_local: bf16 [T/D, h] rank-local order.  With D=1, rank 0 this projects
 * a whole natural-order sequence.  ws: tsp_workspace_bytes(dims, D). */
int tsp_kv_project(const tsp_dims* dims, const tsp_weights* w, int rank,
                   const void* x_local, void* k_full, void* v_full,
                   void* ws, size_t ws_bytes, cudaStream_t stream);

/* tsp_kv_project for callers that cannot allocate device memory.  The paper
 * has no counterpart: this is a deployment variant of tsp_kv_project, not a
 * step of the method.  Some callers are handed only their input and output
 * buffers and own no device allocator (a plugin inside a host framework that
 * manages all device memory), and some must not call cudaMalloc on their hot
 * path because it can synchronise the device or fail at run time.  This
 * entry point computes exactly what tsp_kv_project computes (same kernels,
 * bit-identical K and V) and takes no workspace: its scratch - the LN1
 * output of the rank's tokens and a status word - is a file-scope device
 * array of 64 MiB inside this library, held by every GPU that loads the
 * library until the process exits.  Limit: T/D * h * 2 + 1024 bytes must fit
 * in 64 MiB (e.g. 8191 tokens at h = 4096); larger sizes return
 * TSP_ERR_WORKSPACE with a message in tsp_last_cuda_error.  The first call on
 * a device looks up the array's device address (cudaGetSymbolAddress) with
 * that device current; make that first call before any stream capture.  All
 * calls share the one array, which keeps the last call's contents (the call
 * clears its status and flags words itself): calls that overlap on the GPU
 * - from different streams or threads - race on it, so order them.  The
 * array's device address is cached per device and per CUDA context: after a
 * cudaDeviceReset, or a primary context released and created again, the
 * next call looks it up anew in the new context.  A device-side timeout or
 * an fp16 saturation inside this call is recorded in the array's status
 * section; tsp_kv_project_noalloc_status reads it.  No cudaMalloc, cudaFree
 * or allocating library routine is used.  Arguments as in tsp_kv_project. */
int tsp_kv_project_noalloc(const tsp_dims* dims, const tsp_weights* w, int rank,
                           const void* x_local, void* k_full, void* v_full, cudaStream_t stream);

/* Synchronises `stream`, then reads the status section of
 * tsp_kv_project_noalloc's static scratch (the last call's, on the current
 * device): TSP_OK, TSP_ERR_TIMEOUT or TSP_ERR_SATURATED, as
 * tsp_get_device_status.  The paper has no counterpart. */
int tsp_kv_project_noalloc_status(cudaStream_t stream);

/* The rank's layer forward given the all-gathered K/V [zubnet.ai TSP item,
 * paragraphs 1-2, 4]:
 *   Xn = LN1(x_local);  for each shard k: Q_k = Xn Wq_k^T,
 *   A_k = causal softmax(scale Q_k K_k^T) V_k  (query at global position p
 *   sees keys 0..p),  Y1 = x_local + sum_k A_k Wo_k^T;
 *   Y = Y1 + sum_k GELU(LN2(Y1) W1_k^T) W2_k^T  (the shard sum is local:
 *   no all-reduce).
 * x_local bf16 [T/D, h] rank-local order; k_full, v_full fp16 [T, h]
 * natural order (read only); y_local [T/D, h] rank-local order, bf16
 * (y_dtype TSP_OUT_BF16) or fp32 (TSP_OUT_F32); the bf16 result is the
 * fp32 result rounded to nearest even.  step_events: NULL, or
 * TSP_N_STEP_EVENTS caller-created events recorded on `stream` after the
 * launches of LN1, Q, attention, O, LN2, W1, W2 (event 0 before LN1). */
int tsp_layer_forward(const tsp_dims* dims, const tsp_weights* w, int rank,
                      const void* x_local, const void* k_full, const void* v_full,
                      void* y_local, int y_dtype, void* ws, size_t ws_bytes,
                      cudaStream_t stream, cudaEvent_t* step_events);

/* One whole TSP rank step: tsp_kv_project of the rank's own tokens followed
 * by tsp_layer_forward, with LN1 computed once and the Q, K and V
 * projections done in one launch.  k_full / v_full are read-write: the
 * rank's own rows are written, the other ranks' rows must already be there.
 * step_events as in tsp_layer_forward (the Q launch also projects K/V). */
int tsp_rank_step(const tsp_dims* dims, const tsp_weights* w, int rank,
                  const void* x_local, void* k_full, void* v_full,
                  void* y_local, int y_dtype, void* ws, size_t ws_bytes,
                  cudaStream_t stream, cudaEvent_t* step_events);

/* tsp_rank_step with the token buffers in HOST memory: copies h_x_local
 * ([T/D, h] bf16) to `d_x_staging` (device, T/D*h*2 bytes, caller-owned),
 * runs the step, copies the result back to h_y_local, all enqueued on
 * `stream`.  Pinned host memory makes the copies asynchronous.
 * compute_after (may be null): the step's kernels wait for this event, after
 * the host-to-device copy has been enqueued; compute_done (may be null) is
 * recorded when they end, before the device-to-host copy.  A caller that
 * alternates steps between two streams chains each step's compute_after to
 * the previous step's compute_done: the copies of one step then overlap the
 * kernels of the other while the kernels of consecutive steps never share
 * the GPU.  Both events are the caller's; neither is waited on by the host. */
int tsp_rank_step_host(const tsp_dims* dims, const tsp_weights* w, int rank,
                       const void* h_x_local, void* d_x_staging,
                       void* k_full, void* v_full, void* d_y_staging,
                       void* h_y_local, int y_dtype, void* ws, size_t ws_bytes,
                       cudaStream_t stream, cudaEvent_t compute_after, cudaEvent_t compute_done);

/* Workspace bytes of tsp_attn_backward at this D (status section, work
 * queue counter, Delta); 0 on a bad argument. */
size_t tsp_attn_backward_workspace_bytes(const tsp_dims* dims, int D);

/* Backward of one rank's causal attention against the all-gathered K/V
 * [zubnet.ai TSP item, paragraph 1: the validated workload is training;
 * paragraph 2: every rank attends its own zigzag tokens against the K/V of
 * the whole sequence, so its dK and dV reach all T keys and are summed over
 * the ranks - the reduce-scatter back to the key owners].  The chain rule
 * through the forward (the pages give no backward), per head, for query row i
 * at global position p(i) and its keys k <= p(i):
 *   P = 2^(scale * log2(e) * q_i . k_k - lse2_i)  (lse2 from the forward),
 *   dP = dO V^T,  Delta_i = rowsum(dO_i * O_i),
 *   dS = scale * P * (dP - Delta),
 *   dQ = dS K,  dK += dS^T Q,  dV += P^T dO.
 * q: fp16 [T/D, h] (the forward's Q), o: fp16 [T/D, h] (the forward's
 * attention output A), d_o: fp16 [T/D, h] (the gradient of A), all
 * rank-local order; k_full, v_full: fp16 [T, h] natural order; lse: the
 * forward's stash (tsp_workspace_offsets off[8], same dims, D and rank).
 * dq: fp32 [T/D, h], overwritten.  dk_full, dv_full: fp32 [T, h] natural
 * order, ADDED to (zero them before the first rank; running every rank adds
 * up the whole sequence's gradients); calls that add to the same buffers
 * must not overlap on the GPU.  P, dS and dO enter the tensor cores as fp16;
 * scores, Delta and every accumulation are fp32.  ws:
 * tsp_attn_backward_workspace_bytes(dims, D) bytes, 256-byte aligned, its
 * status section read by tsp_get_device_status.  Pointers 16-byte aligned. */
int tsp_attn_backward(const tsp_dims* dims, int D, int rank, const void* q, const void* k_full,
                      const void* v_full, const void* o, const void* lse, const void* d_o, void* dq,
                      void* dk_full, void* dv_full, void* ws, size_t ws_bytes, cudaStream_t stream);

/* Workspace bytes of tsp_mlp_backward at this D (its own status word first,
 * then the recomputed and transposed activations); 0 on a bad argument. */
size_t tsp_mlp_backward_workspace_bytes(const tsp_dims* dims, int D);

/* Backward of the MLP half of the layer for one rank's tokens [zubnet.ai
 * TSP item, paragraph 1: the validated workload is training; paragraphs
 * 2 and 4: the MLP is a sum over FFN shards with no all-reduce].  For the
 * rank's residual rows Y1 and the loss gradient dY of Y = Y1 + GELU(LN2(Y1)
 * W1) W2 (the chain rule; the pages give no backward):
 *   Xn2 = LN2(Y1) and U = Xn2 W1 are recomputed (fp16, as in the forward;
 *   U by the fp16 shards in `w`),
 *   dU = (dY W2^T) * GELU'(U)        (bf16),
 *   dY1 = dY + LN2'(Y1)^T (dU W1^T)  (fp32),
 *   dW1 = Xn2^T dU,  dW2 = GELU(U)^T dY  (fp32, summed over the rank's
 *   tokens; Xn2 and GELU(U) enter these two products as bf16).
 * The products with dY, dU and their transposes run on bf16 tensor-core
 * operands: W1 and W2 are read from the caller's full bf16 weights in the
 * math orientation, w1_full [h, F] and w2_full [F, h] row-major.  Shard k's
 * gradient is columns k*F/D .. (k+1)*F/D-1 of dW1 and the same rows of dW2.
 * y1: fp32 [T/D, h] and dy: bf16 [T/D, h], both rank-local order (read
 * only); dy1: fp32 [T/D, h]; dw1: fp32 [h, F]; dw2: fp32 [F, h]; every
 * pointer 16-byte aligned.  With T = 0 only dw1 and dw2 are written (zeros)
 * and y1, dy, dy1 may be NULL.  bws: tsp_mlp_backward_workspace_bytes(dims, D)
 * bytes, also the status word that tsp_get_device_status reads.  h and F
 * must be multiples of 256 and T/D a multiple of 128 (TSP_ERR_UNSUPPORTED
 * otherwise, before anything is enqueued).  step_events: NULL, or TSP_N_STEP_EVENTS
 * caller-created events recorded on `stream` before the first launch and
 * after LN2 + U, dU, dXn2, the LN2 backward, the transposes, dW1 and dW2. */
int tsp_mlp_backward(const tsp_dims* dims, const tsp_weights* w,
                     const void* w1_full, const void* w2_full,
                     const void* y1, const void* dy, void* dy1, void* dw1, void* dw2,
                     void* bws, size_t bws_bytes, cudaStream_t stream,
                     cudaEvent_t* step_events);

/* Workspace bytes of tsp_layer_backward at this D (the MLP half's sections,
 * its status section first, then the attention half's); 0 on a bad
 * argument. */
size_t tsp_layer_backward_workspace_bytes(const tsp_dims* dims, int D);

/* One rank's share of the whole layer's backward [zubnet.ai TSP item,
 * paragraph 1: the validated workload is training; paragraph 2: the
 * attention shards are applied to the rank's own tokens against the
 * all-gathered K/V, and the MLP shards' contributions are summed locally].
 * The chain rule through the forward (the pages give none), for the rank's
 * rows and the loss gradient dY of its output:
 *   the MLP half as tsp_mlp_backward: dY1, dW1, dW2;
 *   dA = dY1 Wo^T (fp16),  dWo = A^T dY1;
 *   the attention as tsp_attn_backward: dQ, and dK, dV for every key;
 *   dWq = LN1(X)^T dQ,  dX = dY1 + LN1'(X)^T (dQ Wq^T).
 * What the key owners add after the dK/dV reduce-scatter (LN1'^T (dK Wk^T +
 * dV Wv^T), dWk, dWv) is tsp_kv_backward.  Inputs: w (fp16 shards, for the
 * recomputed U) and w_full = {Wq, Wk, Wv, Wo, W1, W2} bf16 in the math
 * orientation [in, out] (operands of the gradient products, bf16 as in
 * tsp_mlp_backward); x_local bf16 [T/D, h]; fwd_ws: the workspace of this
 * rank's tsp_layer_forward or tsp_rank_step (same dims, D and rank; read:
 * Q, A, Y1 and the log-sum-exp stash); k_full, v_full fp16 [T, h] as in that
 * forward; dy bf16 [T/D, h].  Outputs: dx fp32 [T/D, h] (overwritten);
 * dwq, dwo fp32 [h, h], dw1 fp32 [h, F], dw2 fp32 [F, h]: this rank's
 * contributions summed over its tokens (overwritten); dk_full, dv_full fp32
 * [T, h] natural order, ADDED to (see tsp_attn_backward).  Same shape limits
 * as tsp_mlp_backward.  bws: tsp_layer_backward_workspace_bytes bytes,
 * 256-byte aligned; its status section (read by tsp_get_device_status) is at
 * its start.  step_events: NULL, or TSP_N_STEP_EVENTS events recorded before
 * the first launch and after the MLP half, dA, dWo, the attention, the dQ
 * and LN1 preparations, dWq, and dX. */
int tsp_layer_backward(const tsp_dims* dims, const tsp_weights* w, const void* const w_full[6], int rank,
                       const void* x_local, const void* fwd_ws, size_t fwd_ws_bytes, const void* k_full,
                       const void* v_full, const void* dy, void* dx, void* dwq, void* dwo, void* dw1, void* dw2,
                       void* dk_full, void* dv_full, void* bws, size_t bws_bytes, cudaStream_t stream,
                       cudaEvent_t* step_events);

/* Workspace bytes of tsp_kv_backward at this D; 0 on a bad argument. */
size_t tsp_kv_backward_workspace_bytes(const tsp_dims* dims, int D);

/* The key owner's part of the layer's backward, once dK and dV of the whole
 * sequence have been summed over the ranks [zubnet.ai TSP item, paragraph 2:
 * K/V were all-gathered with the zigzag partition, so their gradients are
 * reduce-scattered back to the ranks that own those tokens]: for rank
 * `rank`'s own tokens at global positions pos(i),
 *   dX[i] += LN1'(X_i)^T (dK[pos(i)] Wk^T + dV[pos(i)] Wv^T),
 *   dWk = LN1(X)^T dK[pos],  dWv = LN1(X)^T dV[pos]  (this rank's tokens).
 * w_full as in tsp_layer_backward (Wk, Wv read); x_local bf16 [T/D, h];
 * dk_full, dv_full fp32 [T, h] (read; each rank reads only its own rows);
 * dx fp32 [T/D, h] added to (tsp_layer_backward's output); dwk, dwv fp32
 * [h, h] overwritten.  dK and dV enter their products as bf16.  kws:
 * tsp_kv_backward_workspace_bytes bytes, 256-byte aligned, status section
 * first. */
int tsp_kv_backward(const tsp_dims* dims, int D, const void* const w_full[6], int rank, const void* x_local,
                    const void* dk_full, const void* dv_full, void* dx, void* dwk, void* dwv, void* kws,
                    size_t kws_bytes, cudaStream_t stream);

/* ---- Tensor-parallel baseline layer ------------------------------------
 * The layer TSP is compared with [zubnet.ai TSP item, paragraphs 1-2: TSP
 * against tensor parallelism (TP, and TP with sequence parallelism), whose
 * MLP needs an all-reduce].  A TP rank k of D holds the same shards as TSP
 * rank k - head group k of Wq, Wk, Wv (columns) and Wo (rows), FFN block k
 * of W1 (columns) and W2 (rows) - but every one of the T tokens:
 *   Y1 = X + sum_k Attn_k(LN1(X) Wq_k, LN1(X) Wk_k, LN1(X) Wv_k) Wo_k^T,
 *   Y  = Y1 + sum_k GELU(LN2(Y1) W1_k^T) W2_k^T,
 * and each sum over k is an all-reduce across the D ranks.  On one GPU the
 * ranks run in turn and the all-reduce is tsp_tp_all_reduce, a sum over the
 * ranks' partial products in device memory.  Operand formats as in the TSP
 * layer (fp16 matmul operands, fp32 accumulation and residual stream). */

/* Workspace bytes of one TP rank (tsp_tp_attention_partial and
 * tsp_tp_mlp_partial share it; status section first); 0 on a bad argument. */
size_t tsp_tp_workspace_bytes(const tsp_dims* dims, int D);

/* TP rank k's partial of the attention half: LN1(X) over all T tokens, its
 * head group's Q, K, V, causal attention over the whole sequence, and
 * A_k Wo_k^T.  x: bf16 [T, h] natural order; part: fp32 [T, h] written; w:
 * the packed shards (w->D = D, the TP degree). */
int tsp_tp_attention_partial(const tsp_dims* dims, const tsp_weights* w, int k, const void* x, void* part,
                             void* ws, size_t ws_bytes, cudaStream_t stream);

/* TP rank k's partial of the MLP half: GELU(LN2(Y1) W1_k^T) W2_k^T over all T
 * tokens.  y1: fp32 [T, h]; part: fp32 [T, h] written. */
int tsp_tp_mlp_partial(const tsp_dims* dims, const tsp_weights* w, int k, const void* y1, void* part, void* ws,
                       size_t ws_bytes, cudaStream_t stream);

/* The all-reduce of the TP layer on one GPU: out = resid + sum of the
 * n_parts fp32 [T, h] partials (1 <= n_parts <= TSP_MAX_D).  resid: fp32
 * (resid_f32 = 1) or bf16 [T, h]; out: TSP_OUT_F32 or TSP_OUT_BF16 [T, h]. */
int tsp_tp_all_reduce(const tsp_dims* dims, int n_parts, const void* const parts[], const void* resid,
                      int resid_f32, void* out, int out_dtype, cudaStream_t stream);

/* ---- Per-shard steps --------------------------------------------------
 * One rank's layer forward taken shard by shard, for running the TSP
 * exchange across GPUs [zubnet.ai TSP item, paragraph 2: the attention
 * shards are broadcast one after another and every rank applies each to its
 * own tokens, K/V are all-gathered under the zigzag partition, and the MLP
 * shards pass around a ring], where each weight shard and each head group's
 * K/V arrive one at a time and the transfer of the next overlaps the
 * compute of the current one.  Composed in order they compute what
 * tsp_layer_forward computes (the shard sums accumulate in the fp32 output
 * instead of inside one product):
 *   xn1 = LN1(x);  y1 = x;
 *   for each head group k: tsp_shard_qkv, all-gather K_k/V_k,
 *       tsp_shard_attention, tsp_shard_accumulate(a_k, Wo_k, y1);
 *   xn2 = LN2(y1);  y = y1;
 *   for each FFN block k: tsp_shard_ffn_up, tsp_shard_accumulate(h_k, W2_k, y).
 * Shard pointers are the packed fp16 shards of tsp_pack_shards.  ws:
 * tsp_shard_workspace_bytes() bytes, 256-byte aligned, status section first
 * (tsp_get_device_status). */
size_t tsp_shard_workspace_bytes(void);

/* y = LN(x) fp16 [rows, h] for x bf16 (x_f32 = 0) or fp32 (x_f32 = 1),
 * biased variance, eps inside the square root, gamma = 1, beta = 0. */
int tsp_layernorm(int64_t rows, int h, float eps, const void* x, int x_f32, void* y, cudaStream_t stream);

/* Head group k of the rank's projections: q_k = xn1 Wq_k^T fp16 [T/D, h/D]
 * (rank-local rows); K_k, V_k = xn1 Wk_k^T, xn1 Wv_k^T written at the rank's
 * GLOBAL rows of k_k, v_k fp16 [T, h/D] (what the all-gather then fills in
 * for the other ranks).  xn1: fp16 [T/D, h]. */
int tsp_shard_qkv(const tsp_dims* dims, int D, int rank, const void* wq_k, const void* wk_k, const void* wv_k,
                  const void* xn1, void* q_k, void* k_k, void* v_k, void* ws, cudaStream_t stream);

/* Causal attention of head group k: a_k fp16 [T/D, h/D] from q_k [T/D, h/D]
 * and the group's all-gathered k_k, v_k [T, h/D] (natural order). */
int tsp_shard_attention(const tsp_dims* dims, int D, int rank, const void* q_k, const void* k_k, const void* v_k,
                        void* a_k, void* ws, cudaStream_t stream);

/* FFN block k: h_k = GELU(xn2 W1_k^T) fp16 [T/D, F/D], xn2 fp16 [T/D, h]. */
int tsp_shard_ffn_up(const tsp_dims* dims, int D, const void* w1_k, const void* xn2, void* h_k, void* ws,
                     cudaStream_t stream);

/* y += act w_k^T for one shard: act fp16 [T/D, k_dim] with k_dim = h/D (the
 * attention output a_k, w_k = Wo_k) or F/D (h_k, w_k = W2_k); y fp32
 * [T/D, h], read and written in place. */
int tsp_shard_accumulate(const tsp_dims* dims, int D, const void* act, int k_dim, const void* w_k, void* y,
                         void* ws, cudaStream_t stream);

/* Fault-detection self test: launches one block that waits on a barrier
 * nothing will ever complete, with a limit of `timeout_ns` nanoseconds
 * (at most 2e9).  The wait gives up, the kernel records TSP_ERR_TIMEOUT in
 * the workspace status word and returns normally, so the context stays
 * usable.  ws: at least 256 bytes; NULL targets the status section of
 * tsp_kv_project_noalloc's static scratch (read by
 * tsp_kv_project_noalloc_status). */
int tsp_selftest_wait_timeout(void* ws, uint64_t timeout_ns, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* TSP_H_ */
