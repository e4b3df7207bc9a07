/*
 * pi_sparse_ffn.h — C ABI of the activation-sparse FFN decode path (sm_100a / B200).
 *
 * The operation: PowerInfer's neuron-aware sparse FFN at decode time, as the pages
 * describe it.
 *   - A small per-layer predictor says which FFN neurons will fire. Only those neurons
 *     are computed; the others are skipped (unite.ai "PowerInfer: Mesin Inferensi LLM
 *     Cepat dengan GPU Konsumen", §"Fase Online: Mesin Inferensi LLM yang Sadar Neuron"
 *     and §"Prediktor Kepadatan Adaptif").
 *   - Neuron-aware operators read the individual rows (up/gate) and columns (down) of
 *     the active neurons. There is no conversion to a dense format (same page,
 *     §"Operator yang Sadar Neuron").
 *   - Neurons that fire often ("hot") are placed by firing frequency. A neuron table
 *     maps every placed neuron back to its original position (same page,
 *     §"Penempatan dan Pengelolaan Neuron"; KPD "PowerInfer: Fast Large Language Model
 *     Serving with a Consumer-grade GPU", §"Метод").
 *   - Activations: ReLU, ReGLU and squared ReLU (GeekNews "Tüketici sınıfı GPU takılı
 *     PC'lerde yüksek hızlı büyük dil modeli serving", §"Kısıtlar ve SSS": the method
 *     serves the ReLU family, whose exact zeros can be skipped).
 *     Weights: fp32, fp16 or Q4_0 (same page, §"Kuantizasyon ve uyumluluk").
 *
 * Per layer and token x (d = d_model, f = d_ff, r = rank):
 *   u      = P1^T x                                  P1: [d x r]
 *   logit_i = sum_k P2[k,i] u_k - t_i                P2: [r x f], t: [f]
 *   bit i   = (logit_i > 0), strict
 *   idx     = ascending ids of the neurons whose bit is set for any token of the batch
 *   ReLU :  a_i = max(0, w_up_i . x + b_i)
 *   ReGLU:  a_i = max(0, w_gate_i . x + b_i) * (w_up_i . x)
 *   ReLU^2: a_i = max(0, w_up_i . x + b_i)^2
 *   a[b,i] = 0 where token b's own bit is 0
 *   y_j     = sum over active i of W_down[j,i] * a_i          (fp32 accumulation)
 *   stack:  v = x + y;  x' = (v - mean(v)) / sqrt(var(v) + 1e-6), in fp32, stored in
 *           the activation dtype. The pages have no layer stack; this residual plus a
 *           mean-centred normalisation is this library's reading.
 *
 * Conventions
 *   - Every call returns a pi_status. PI_OK is 0.
 *   - Arguments are validated synchronously, before anything is enqueued. A call that
 *     fails validation enqueues nothing.
 *   - Work is enqueued on the given stream and runs asynchronously. pi_load_layer and
 *     pi_reorder_hot_prefix are the exceptions: they synchronise the stream before
 *     they return.
 *   - Buffers the caller passes (x, y, mask, idx, count, logits, trace) are device
 *     memory that the caller owns. They must not alias one another.
 *   - Layer and workspace objects are owned by the library. Free them with
 *     pi_free_layer and pi_workspace_free.
 *   - Errors detected on the device: a grid-barrier wait that ran out, or an active
 *     count beyond d_ff. They set an error word in the workspace; the kernel then
 *     returns without hanging. Read it with pi_stream_status.
 *   - Mask words are uint32 and least-significant-bit first: bit j of word w is
 *     neuron 32*w + j. Indices are in the layer's stored order. That order is the
 *     original order until pi_reorder_hot_prefix is called; pi_get_perm maps stored
 *     order back to original ids.
 *   - Supported dtype families (w, x, p): (F32, F32, F32), (F16, F16, F16) and
 *     (Q4_0, F16, F16). Any other combination returns PI_ERR_UNSUPPORTED.
 *   - Limits: d_ff % 32 == 0; d_model % 64 == 0 (Q4_0: % 256 == 0); 1 <= rank <= d_model;
 *     1 <= B <= PI_MAX_BATCH. PI_ERR_ARG otherwise.
 */
#ifndef PI_SPARSE_FFN_H
#define PI_SPARSE_FFN_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#define PI_MAX_BATCH 32

typedef enum {
  PI_OK = 0,
  PI_ERR_ARG = 1,          /* bad pointer, size, shape or combination */
  PI_ERR_UNSUPPORTED = 2,  /* valid request the library does not implement */
  PI_ERR_OOM = 3,          /* device allocation failed */
  PI_ERR_CUDA = 4,         /* a CUDA runtime call failed (launch, copy, sync) */
  PI_ERR_TIMEOUT = 5,      /* a device-side wait gave up (see pi_stream_status) */
  PI_ERR_DEVICE = 6        /* a device-side check failed (see pi_stream_status) */
} pi_status;

typedef enum { PI_F32 = 0, PI_F16 = 1, PI_Q4_0 = 2 } pi_dtype;
typedef enum { PI_RELU = 0, PI_REGLU = 1, PI_RELU2 = 2 } pi_act;

/* Shape and types of one FFN layer. */
typedef struct {
  int d_model;       /* d */
  int d_ff;          /* f, a multiple of 32 */
  int rank;          /* r, predictor rank */
  pi_act act;        /* PI_RELU, PI_RELU2 (squared ReLU): bias on up; PI_REGLU: bias on gate */
  pi_dtype w_dtype;  /* up/gate/down weights */
  pi_dtype x_dtype;  /* activations x (F32 or F16) */
  pi_dtype p_dtype;  /* predictor P1/P2 (F32 or F16) */
} pi_layer_desc;

/* Device pointers to one layer's weights, in the caller's layout. pi_load_layer copies
 * them; the caller may free them once it returns.
 *   F32/F16: w_up [f x d] and w_gate [f x d] are row-major (row i = neuron i);
 *            w_down is [d x f] row-major; the library stores it transposed.
 *   Q4_0:    w_up / w_gate / w_down are nibble planes uint8 [f][d/32][16]. Byte j of
 *            a block holds element j in its low four bits and element j+16 in its
 *            high four bits. s_up / s_gate / s_down are fp16 scale planes [f][d/32].
 *            The value is (q - 8) * scale. The down weights are given neuron-major
 *            ([f] rows of d), the axis the blocks run along.
 *   w_gate / s_gate are NULL for ReLU and squared ReLU. s_* are NULL unless w_dtype is Q4_0.
 *   bias [f] f32, thresh [f] f32; p1 [d x r] and p2 [r x f] row-major in p_dtype. */
typedef struct {
  const void* w_up;
  const void* w_gate;
  const void* w_down;
  const void* s_up;
  const void* s_gate;
  const void* s_down;
  const float* bias;
  const void* p1;
  const void* p2;
  const float* thresh;
} pi_layer_weights;

typedef struct pi_layer pi_layer;
typedef struct pi_workspace pi_workspace;

/* Optional per-layer capture for pi_decode_stack. Any member may be NULL. Layer l's
 * records start at l * (per-layer size).
 *   x      [L+1][B][d] in the activation dtype: x[l] is layer l's input; x[L] is the output
 *   logits [L][B][f] f32
 *   mask   [L][B][f/32] u32
 *   idx    [L][f] i32; only the first count[l] entries of layer l are written
 *   count  [L] i32
 *   idx and count are the compaction of the layer's mask, so they are filled only
 *   together and only with mask (PI_ERR_ARG otherwise).
 *   y      [L][B][d] f32, the FFN output before the residual and the normalisation */
typedef struct {
  void* x;
  float* logits;
  uint32_t* mask;
  int32_t* idx;
  int32_t* count;
  float* y;
} pi_trace;

/* ---------------------------------------------------------------- layers */

/* Copy one layer into library-owned device memory, in the library's own layout.
 *   - One contiguous record per neuron: [gate row | up row | 16-byte bias header], so
 *     one copy brings everything a neuron's gate/up dot products need.
 *   - The down weights neuron-major, one row of d_model per neuron, so a block can read
 *     its own column slice of each active neuron's row.
 *   - P1 is stored transposed and P2 neuron-major.
 * desc and w are host structs holding device pointers. Synchronises `stream` before it
 * returns. On success *out holds the layer. */
pi_status pi_load_layer(const pi_layer_desc* desc, const pi_layer_weights* w,
                        cudaStream_t stream, pi_layer** out);

/* Re-store the layer's neurons by descending firing frequency, ties by ascending
 * original id. The order is built on the device. Every per-neuron tensor moves with
 * its neuron: up/gate/down rows, bias, P2 columns and thresholds. The neuron table
 * (pi_get_perm) is updated to match.
 *   freq:      device f32[d_ff], the measured firing frequency of each neuron in the
 *              layer's current stored order.
 *   hot_count: -1, or the length of the hot prefix in [0, d_ff]. It is validated and
 *              kept; the kernels do not read it (the hot order itself is what they use:
 *              it places the always-firing neurons first, and its frequencies set how
 *              many own records every block keeps before the mask exchange).
 * Synchronises `stream` before it returns. Calling it again composes the orders. */
pi_status pi_reorder_hot_prefix(pi_layer* layer, const float* freq, int hot_count,
                                cudaStream_t stream);

/* perm_out: device int32[d_ff]; perm_out[stored position] = original neuron id. */
pi_status pi_get_perm(const pi_layer* layer, int32_t* perm_out, cudaStream_t stream);

/* Copy back the layer's descriptor (host struct). */
pi_status pi_layer_get_desc(const pi_layer* layer, pi_layer_desc* out);

void pi_free_layer(pi_layer* layer);

/* ---------------------------------------------------------------- workspace */

/* Scratch for the kernels: the cross-block exchange words (the predictor vector u,
 * every block's mask words, h of the active neurons, the stack's x + y and its
 * moments, and every block's partial y for the row-owned down pass: grid x d_model_max
 * words of 8 bytes), the launch words, the device error word, and the multi-launch
 * path's mask, index and partial-sum buffers. It is sized for the largest shapes it
 * will serve: calls with larger d_model, d_ff, rank, B or L return PI_ERR_ARG. A
 * workspace serves one stream at a time. Calls that overlap on the device and share a
 * workspace race. */
pi_status pi_workspace_create(int d_model_max, int d_ff_max, int rank_max, int B_max,
                              int L_max, pi_workspace** out);
void pi_workspace_free(pi_workspace* ws);

/* Synchronise `stream`, then read and clear the workspace's device error word.
 * Returns PI_OK, PI_ERR_TIMEOUT or PI_ERR_DEVICE. After an error the barrier words
 * are reset, so the workspace stays usable. */
pi_status pi_stream_status(pi_workspace* ws, cudaStream_t stream);

/* Running total, over every FFN call made with this workspace, of the active-list
 * lengths the kernels processed (host out; synchronous). It is used to count the bytes
 * a run actually read. */
pi_status pi_workspace_active_total(pi_workspace* ws, unsigned long long* out);

/* Per-layer union active count of the last pi_decode_stack call (host out [L];
 * synchronous). */
pi_status pi_workspace_layer_counts(pi_workspace* ws, int32_t* host_out, int L);

/* Diagnostic: launch grid barriers whose target one block more than the grid can never
 * reach. Every wait must give up after timeout_ns and report it. pi_stream_status then
 * returns PI_ERR_TIMEOUT and resets the workspace's barrier words. It checks that a
 * device-side wait ends without hanging the GPU. */
pi_status pi_diag_barrier_timeout(pi_workspace* ws, long long timeout_ns, cudaStream_t stream);

/* Diagnostic: with `on`, every later pi_decode_stack on this workspace records each
 * block's SM cycle counter at up to 64 points of every layer. Consumer warp 0: 0 layer
 * start, 1 u rows published, 2 u received, 3 logits done, 4 own list and mask words
 * published, 6 list barrier passed, 8 first record landed, 9 gate/up dots done, 25 h
 * words of the first chunks received, 26 every warp past the h barrier, 27 the down
 * copies of chunk 0 landed, 28 down products done, 10 down slice summed, 11 v and
 * moments published, 12 every v and moment received, 13 glue done. First helper thread:
 * 5 every block's mask words received, 29 the rest of the list handed over, 23 down
 * list built, 7 down copies issued. Slot 14 holds the block's own active count, 15 the
 * layer's active count, 17 the cycles thread 0 polls for h and 18 the cycles spent
 * waiting for P2 rows. With `on` = 2 the stamps come from the GPU's global nanosecond
 * timer instead, so blocks can be compared with one another. With `on` = 0 recording
 * stops and the buffer is freed. */
pi_status pi_diag_phase_clocks_enable(pi_workspace* ws, int on);

/* Copy the first n stamps ([grid][L_max][64], int64) to host memory (synchronous). */
pi_status pi_diag_phase_clocks_read(pi_workspace* ws, long long* host_out, size_t n);

/* Blocks per launch of the fused kernel on this workspace's device (its SM count). */
int pi_device_grid(pi_workspace* ws);

/* ---------------------------------------------------------------- hot path */

/* Predictor. x: device [B][d] in x_dtype. mask: device u32 [B][f/32].
 * logits: NULL, or device f32 [B][f]. Logits are computed in fp32: u is accumulated
 * in fp32 from the stored weights, then logit = P2^T u - t. */
pi_status pi_predict(const pi_layer* layer, const void* x, int B, uint32_t* mask,
                     float* logits, pi_workspace* ws, cudaStream_t stream);

/* Bytes of the static device scratch behind pi_predict_noalloc (256 KiB). */
#define PI_NOALLOC_SCRATCH_BYTES (256u * 1024u)

/* pi_predict without a workspace: the predictor launch of pi_predict, with the same
 * outputs and the same bits wherever both serve the shape. It allocates no memory: its
 * cross-block scratch is one static device array of PI_NOALLOC_SCRATCH_BYTES per device.
 * The pages have no counterpart; this entry point is this library's own. It is for
 * callers that cannot allocate device memory when they call it, such as a serving loop
 * that has already handed all free HBM to its weights and KV cache, or a plug-in that
 * sees only a stream and plain pointers and has nowhere to keep a workspace between
 * calls.
 *
 * Shapes served: only those the single persistent launch serves, that is 1 to 4 tokens
 *   (1 to 2 for Q4_0) with d_model up to 12288 (fp16, 1 token), 8192 (fp16 2 tokens,
 *   Q4_0), 4096 (fp16 4 tokens, fp32 1-2 tokens) or 2048 (fp32 4 tokens). Other shapes,
 *   which pi_predict runs on its multi-launch path, return PI_ERR_UNSUPPORTED before
 *   anything is enqueued, the first call's set-up included.
 * status: device i32, owned by the caller (required). After the launch it receives
 *   PI_OK, PI_ERR_TIMEOUT (a bounded device-side wait gave up) or PI_ERR_DEVICE (a
 *   device-side check failed). After an error the scratch is reset on the device for
 *   the next call. The word is written only when the call returns PI_OK; after any
 *   other return it keeps what it held.
 * Scratch needed: 256 + round256(B * rank * 8) bytes. A shape that needs more than
 *   PI_NOALLOC_SCRATCH_BYTES returns PI_ERR_UNSUPPORTED and enqueues nothing.
 * Set-up: the first call on each device takes the array's address, clears it and
 *   synchronises `stream` before it returns. Make that first call before any stream
 *   capture begins. The set-up is kept for the life of the process: after
 *   cudaDeviceReset (or anything else that destroys the device's primary context) this
 *   entry point must not be called again on that device.
 * Calls share the one array per device. Two calls that may run at the same time (on
 *   different streams, or from different threads without ordering) race on it and
 *   give undefined results. Order them on one stream or with events. */
pi_status pi_predict_noalloc(const pi_layer* layer, const void* x, int B, uint32_t* mask,
                             float* logits, int32_t* status, cudaStream_t stream);

/* Compaction. idx (device i32 [d_ff]) receives the ascending ids of the neurons whose
 * bit is set for any of the B tokens (the OR of mask[0..B-1]). *count (device i32)
 * receives their number. Only the first *count entries of idx are written. */
pi_status pi_compact_active(const uint32_t* mask, int B, int d_ff, int32_t* idx,
                            int32_t* count, cudaStream_t stream);

/* Sparse FFN over an active list. x: device [B][d] (x_dtype). mask: device
 * [B][f/32] per-token bits. idx/count: the active list, for example from
 * pi_compact_active. Every id in idx must have its bit set in at least one token's
 * mask. y: device f32 [B][d] (overwritten).
 * Only the active rows are read. Sums run in fp32 and are deterministic: the same
 * inputs give the same bits. */
pi_status pi_sparse_ffn(const pi_layer* layer, const void* x, int B, const uint32_t* mask,
                        const int32_t* idx, const int32_t* count, float* y,
                        pi_workspace* ws, cudaStream_t stream);

/* A whole decode step through L layers: predictor, compaction, sparse FFN and stack
 * glue for each layer. At 1-4 tokens, when the layer fits the persistent kernel, one
 * launch runs the whole step. Otherwise (5-32 tokens, or layers too wide for it) each
 * layer runs a fixed sequence of kernels: tensor-core row tiles for the predictor and
 * gate/up, compaction, the down columns and the glue. The host does not synchronise
 * inside either way. x_inout: device [B][d] in the activation dtype. It holds x_0 on
 * entry and x_L on return. All layers must share one descriptor except for the
 * predictor rank, which may differ from layer to layer (the pages size each layer's
 * predictor by its own sparsity: unite.ai "PowerInfer: Mesin Inferensi LLM Cepat dengan
 * GPU Konsumen", §"Prediktor Kepadatan Adaptif"); the workspace's rank_max must cover the
 * largest. trace may be NULL. */
pi_status pi_decode_stack(pi_layer* const* layers, int L, void* x_inout, int B,
                          const pi_trace* trace, pi_workspace* ws, cudaStream_t stream);

/* pi_decode_stack driven from host memory. It copies x_host (B*d elements in the
 * activation dtype) to the device, runs the stack, and copies x_L back to x_out_host.
 * It then synchronises `stream` and returns pi_stream_status. Pinned host buffers make
 * the copies asynchronous. x_host and x_out_host may be the same buffer. */
pi_status pi_decode_stack_host(pi_layer* const* layers, int L, const void* x_host,
                               void* x_out_host, int B, pi_workspace* ws,
                               cudaStream_t stream);

/* ---------------------------------------------------------------- misc */

const char* pi_status_str(pi_status s);

/* Compile-time version of this ABI (major * 10000 + minor * 100 + patch). */
int pi_abi_version(void);

/* Number of kernels this library has launched in the calling process so far, on any
 * device and stream (layout, predictor, compaction, FFN and service kernels alike;
 * memsets and copies are not kernels of this library and are not counted).  The count is
 * taken on the host at each launch, so the difference between two reads brackets the
 * launches of the calls made in between.  Thread-safe; never fails. */
uint64_t pi_kernel_launches(void);

#ifdef __cplusplus
}
#endif

#endif /* PI_SPARSE_FFN_H */
