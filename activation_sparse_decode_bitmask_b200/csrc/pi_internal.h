// Internal definitions shared by the library's translation units (not part of the ABI).
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "../../include/pi_sparse_ffn.h"

namespace pi {

// ---------------------------------------------------------------- device-side errors
enum DevErr : int {
  DEV_OK = 0,
  DEV_ERR_GRID_TIMEOUT = 1,   // a grid-barrier wait ran out
  DEV_ERR_RING_TIMEOUT = 2,   // a shared-memory ring wait ran out
  DEV_ERR_LIST = 3,           // an active list longer than the block can hold
  DEV_ERR_INDEX = 4,          // an index or count outside [0, d_ff]
  DEV_ERR_BAD_FREQ = 5,       // a non-finite firing frequency
};

// Launch epochs tag the cross-block exchange words (tag = epoch * 1024 + layer * 8 +
// exchange, 32 bits).  An epoch that is a multiple of 2^22 would give layer 0's first
// exchange the tag 0, the tag of a cleared word, so such epochs are skipped.
constexpr uint32_t kEpochWrap = 1u << 22;
__host__ __device__ inline uint32_t next_launch_epoch(uint32_t e) {
  ++e;
  if (e % kEpochWrap == 0) ++e;
  return e;
}

// dtype families (w, x, p)
enum Family : int { FAM_F32 = 0, FAM_F16 = 1, FAM_Q4 = 2 };

// Kernel launch geometry of the fused kernel: 16 consumer warps + 1 producer warp.
constexpr int kConsumerWarps = 16;
constexpr int kConsumerThreads = kConsumerWarps * 32;
constexpr int kThreads = kConsumerThreads + 32;
constexpr int kMaxOwn = 512;          // owned neurons per block (d_ff <= 512 * grid)
constexpr int kMaxOwnWords = kMaxOwn / 32;
constexpr int kMaxPieces = 16;        // 16-byte down units one block owns
constexpr int kMaxList = 512;         // active neurons a block may process in one layer
constexpr int kMaxLayers = 100;       // layers of one pi_decode_stack call
constexpr int kMaxGrid = 256;         // blocks of the fused kernel (SMs)
constexpr int kDiagSlots = 64;        // diagnostic stamps per block and layer

// Library-owned, re-laid-out layer, as the fused kernel sees it.
struct LayerDev {
  const uint8_t* rec;     // [f][rec_stride] per-neuron record [gate row][up row][16-byte header: bias],
                          // followed by the down rows [f][dn_stride] (neuron-major)
  const uint8_t* p1t;     // [r][p1_row]       P1 transposed, p_dtype
  const uint8_t* p2o;     // [G][nown_max][p2_stride(r)] predictor row + (t, b) of neuron c + m*G
  int keep_floor;         // own records every block keeps before the mask exchange (0 = none)
  int r;                  // this layer's predictor rank (layers of one stack may differ)
};

// Bytes of one owner-major predictor row of rank r: r values of p_bytes, then (t, b),
// rounded to 16.
__host__ __device__ inline int p2_stride_of(int r, int p_bytes) { return (r * p_bytes + 8 + 15) / 16 * 16; }

}  // namespace pi

struct pi_layer {
  pi_layer_desc desc;
  int family;
  int row_bytes;    // one weight row (d elements) in the record
  int rec_stride;   // bytes per neuron record (gate? + up + bias header), multiple of 16
  int gate_off, up_off;   // byte offsets of the rows in a record (gate_off -1 for ReLU)
  int bias_off;     // byte offset of the record's 16-byte header holding the bias (f32)
  int dn_stride;    // bytes per down row (multiple of 16)
  size_t dn_off;    // byte offset of the down rows in the record allocation (f * rec_stride)
  int p1_row;       // bytes of one P1^T row (d * p_bytes)
  int p2_stride;    // bytes per neuron predictor row (r * p_bytes + 8, rounded to 16)
  int G;            // blocks the owner-major predictor layout was built for (the SM count)
  int nown_max;     // ceil(f / G): predictor rows per block, padded
  uint8_t* rec;     // records, then the down rows
  uint8_t* p1t;
  uint8_t* p2o;
  float* bias;      // [f] stored order
  float* thresh;    // [f] stored order
  int32_t* perm;    // [f] stored position -> original id
  float* freq_sorted;  // [f] firing frequency in stored order (after a reorder), else null
  float* freq_host;    // host copy of freq_sorted (descending), or null
  int keep_floor[4];   // per batch 1..4: own records every block keeps before balancing
  int hot_count;    // -1: derived per batch from freq_sorted
  int device;
};

struct pi_workspace {
  int d_max, f_max, r_max, B_max, L_max;
  int grid;          // blocks of the fused kernel (one per SM)
  int device;
  uint64_t* ux;      // [B_max][r_max]          tagged u
  uint64_t* mx;      // [grid][4][kMaxOwnWords] tagged own mask words
  uint64_t* hx;      // [f_max + grid][B_max]   tagged h: owner o's records from word o * nown_max on
  uint64_t* vx;      // [B][d] tagged x + y, then [B][grid][2] the column slices' sums and sums of squares
  uint64_t* yx;      // [grid][d_max] tagged partial y of each block (row-owned down pass, one token)
  uint32_t* bar;     // [0] probe barrier count, [1] exit count, [2] launch epoch (tags)
  int* err;          // device error word
  unsigned long long* active_total;  // running sum of active-list lengths (all calls)
  int32_t* layer_count;              // [L_max] per-layer union active count of the last stack
  void* x_dev;       // [B_max][d_max] staging for pi_decode_stack_host (fp32 size)
  // batched path (B_max > 4 only)
  __half* u_hi;      // [32][r_max] u as fp16 high part
  __half* u_lo;      // [32][r_max] u low part
  uint32_t* bmask;   // [32][f_max/32]
  int32_t* bidx;     // [f_max]
  int32_t* bcount;   // [1]
  float* bh;         // [f_max][32] h of the active neurons
  float* by;         // [32][d_max] FFN output
  float* bpart;      // split partial sums of the row kernels
  size_t bpart_floats;
  float* bypart;     // split partial sums of the down kernel
  long long* phase_clk;  // diagnostics: [grid][L_max][12] stamps, or null when off
  int phase_global;      // 1: stamps from the global ns timer
  void* x_host_pinned;
};

namespace pi {

// Counts one kernel launch of this library (read by pi_kernel_launches).
void note_launch();

// Parameters of one launch of the fused kernel.
struct FusedParams {
  int mode;            // bit 1: predictor, bit 2: FFN, bit 4: stack glue (layer loop)
  int L, B, d, f;
  int r;               // the largest predictor rank of the launch's layers (u buffer size)
  int grid;
  int row_bytes, rec_stride, gate_off, up_off, bias_off, p1_row, p2_stride;
  int dn_stride;       // bytes per down row
  int act_square;      // squared ReLU: h = max(0, up + b)^2 (the ReLU instantiation squares)
  long long dn_off;    // byte offset of the down rows behind a layer's records
  int ring_bytes, p1_rows_per_item, nown_max;
  int inflight_budget; // bytes of bulk copies one block keeps in flight at most (one item at least)
  int p2_item_bytes;   // target bytes of one copy of predictor rows (a layer's rows per copy follow)
  int nw;              // 32-bit words of one block's own bits per token: ceil(nown_max / 32)
  int dunits;          // 16-byte down units of a row: d/4 (fp32), d/8 (fp16), d/32 (Q4_0 blocks)
  int pmax;            // most down units one block owns: ceil(dunits / grid), <= kMaxPieces
  int dch;             // active entries per down chunk (each chunk's rows fit one half of dbuf)
  // dynamic shared-memory layout (byte offsets)
  int off_ring, off_xs, off_us, off_ob, off_dlist, off_dbuf, off_dsc, off_dred, off_hs;
  LayerDev layers[kMaxLayers];
  // inputs / outputs
  const void* x_in;          // [B][d] activation dtype
  void* x_out;               // [B][d] activation dtype (stack)
  uint32_t* mask_out;        // [B][f/32] (predict), zeroed by the host
  float* logits_out;         // [B][f] (predict) or null
  const uint32_t* mask_in;   // [B][f/32] (ffn)
  const int32_t* idx_in;     // [f] (ffn)
  const int32_t* count_in;   // (ffn)
  float* y_out;              // [B][d] (ffn)
  pi_trace trace;            // (stack)
  // workspace
  uint64_t* ux;
  uint64_t* mx;
  uint64_t* hx;
  uint64_t* vx;        // [B][d] v, then [B][grid][2] slice moments
  uint64_t* yx;        // [G][d] partial y of every block (row-owned down pass)
  uint32_t* bar;
  int* err;
  unsigned long long* active_total;
  int32_t* layer_count;
  long long barrier_timeout_ns;   // grid-barrier probe wait budget (global timer)
  long long wait_cycles;          // fused-kernel wait budget in SM cycles
  int barrier_extra;   // added to the barrier target (diagnostics: forces a timeout)
  long long* phase_clk;  // diagnostics: SM cycle stamps per block, layer and phase, or null
  int phase_global;      // stamps from the global ns timer instead of the SM cycle counter
  unsigned poll_ns;      // back-off between polling rounds of the cross-block exchanges
};

enum : int { MODE_PREDICT = 1, MODE_FFN = 2, MODE_GLUE = 4 };

cudaError_t launch_fused(int family, int act, int B, const FusedParams& p, size_t smem_bytes,
                         cudaStream_t stream);
// Fills the shared-memory layout, item sizes and down-chunk geometry of `p` (whose shape,
// record and grid fields are set) within `budget` bytes; false if the shape does not fit.
bool fused_plan_smem(FusedParams& p, int family, size_t budget, size_t& smem_bytes);
bool fused_supported(int family, int B, int d);
cudaError_t launch_barrier_probe(const FusedParams& p, int rounds, cudaStream_t stream);

// Batched path (up to 32 tokens, fp16 family): tensor-core tiles for every contraction.
struct BatchedLayer {
  int d, f, r, G, nown_max;
  const uint8_t* rec;
  int rec_stride, up_off, gate_off;
  const uint8_t* dn;     // down rows [f][dn_stride]
  int dn_stride;
  const uint8_t* p1t;
  int p1_row;
  const uint8_t* p2o;
  int p2_stride;
  const float* thresh;
  const float* bias;
  int act_square;        // squared ReLU
};
bool batched_supported(int family, int B, int d, int r);
cudaError_t batched_predict(const BatchedLayer& L, const void* x, int B, uint32_t* mask, float* logits,
                            __half* u_hi, __half* u_lo, float* part, size_t part_floats, cudaStream_t s);
cudaError_t batched_ffn(const BatchedLayer& L, const void* x, int B, const uint32_t* mask, const int32_t* idx,
                        const int32_t* count, float* h, float* y, float* part, size_t part_floats, float* ypart,
                        int* err, cudaStream_t s);
size_t batched_part_floats(int d_max, int f_max, int r_max);
size_t batched_ypart_floats(int d_max);
cudaError_t batched_glue(const void* x, const float* y, int B, int d, void* x_out, void* trace_x, cudaStream_t s);
cudaError_t batched_count(const int32_t* count, unsigned long long* total, int32_t* layer_count, cudaStream_t s);

cudaError_t launch_compact(const uint32_t* mask, int B, int f, int32_t* idx, int32_t* count,
                           cudaStream_t stream);

}  // namespace pi
