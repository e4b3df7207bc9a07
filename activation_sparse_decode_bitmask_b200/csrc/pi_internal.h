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

// dtype families (w, x, p)
enum Family : int { FAM_F32 = 0, FAM_F16 = 1, FAM_Q4 = 2 };

// Kernel launch geometry of the fused kernel: 16 consumer warps + 1 producer warp.
constexpr int kConsumerWarps = 16;
constexpr int kConsumerThreads = kConsumerWarps * 32;
constexpr int kThreads = kConsumerThreads + 32;
constexpr int kMaxOwn = 512;          // owned neurons per block (d_ff <= 512 * grid)
constexpr int kMaxList = 512;         // active neurons a block may process in one layer
constexpr int kMaxLayers = 100;       // layers of one pi_decode_stack call
constexpr int kMaxGrid = 256;         // blocks of the fused kernel (SMs)
constexpr int kDiagSlots = 64;        // diagnostic stamps per block and layer

// Library-owned, re-laid-out layer.
struct LayerDev {
  const uint8_t* rec;     // [f][rec_stride]   per-neuron record [gate][up][down]
  const uint8_t* p1t;     // [r][p1_row]       P1 transposed, p_dtype
  const uint8_t* p2o;     // [G][nown_max][p2_stride] predictor row + (t, b) of neuron c + m*G
  int hot;                // hot-prefix length at this call's batch, 0 = none
  int keep_floor;         // records every block keeps of its own before balancing (0 = none)
};

}  // namespace pi

struct pi_layer {
  pi_layer_desc desc;
  int family;
  int row_bytes;    // one weight row (d elements) in the record
  int rec_stride;   // bytes per neuron record (gate? + up + down), multiple of 16
  int gate_off, up_off, down_off;   // byte offsets of the rows in a record (gate_off -1 for ReLU)
  int bias_off;     // byte offset of the record's 16-byte header holding the bias (f32)
  int p1_row;       // bytes of one P1^T row (d * p_bytes)
  int p2_stride;    // bytes per neuron predictor row (r * p_bytes + 8, rounded to 16)
  int G;            // blocks the owner-major predictor layout was built for (the SM count)
  int nown_max;     // ceil(f / G): predictor rows per block, padded
  uint8_t* rec;
  uint8_t* p1t;
  uint8_t* p2o;
  float* bias;      // [f] stored order
  float* thresh;    // [f] stored order
  int32_t* perm;    // [f] stored position -> original id
  float* freq_sorted;  // [f] firing frequency in stored order (after a reorder), else null
  float* freq_host;    // host copy of freq_sorted (descending), or null
  int keep_floor[4];   // per batch 1..4: own records every block keeps before balancing
  int hot_count;    // -1: derived per batch from freq_sorted
  int hot_len_b[33];   // per batch 1..32: hot-prefix length (set with freq_host)
  int device;
};

struct pi_workspace {
  int d_max, f_max, r_max, B_max, L_max;
  int grid;          // blocks of the fused kernel (one per SM)
  int device;
  uint64_t* ux;      // [B_max][r_max]          tagged u
  uint64_t* px;      // [grid][B_max][d_max]    tagged y partials
  uint64_t* vx;      // [B_max][d_max]          tagged x + y
  uint64_t* sx;      // [B_max][grid][2]        tagged slice sums and sums of squares
  uint64_t* cx;      // [grid]                  tagged own active counts (balance)
  uint64_t* lx;      // [grid][kMaxOwn]         tagged own active list entries (balance)
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
  int L, B, d, f, r;
  int grid;
  int row_bytes, rec_stride, gate_off, up_off, down_off, bias_off, p1_row, p2_stride;
  int ring_bytes, p1_rows_per_item, p2_rows_per_item, nown_max;
  int rec_window;      // ring_bytes / rec_stride - 2: at least 1, so three records fit in the ring
  int nslices;
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
  uint64_t* px;
  uint64_t* vx;
  uint64_t* sx;
  uint64_t* cx;        // tagged own active counts [grid]; null: no balancing (each block keeps its own)
  uint64_t* lx;        // tagged own active list entries [grid][kMaxOwn]
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
size_t fused_fixed_smem(int B, int d, int r, int grid, int nown_max, int family);
bool fused_supported(int family, int B, int d);
cudaError_t launch_barrier_probe(const FusedParams& p, int rounds, cudaStream_t stream);

// Batched path (up to 32 tokens, fp16 family): tensor-core tiles for every contraction.
struct BatchedLayer {
  int d, f, r, G, nown_max;
  const uint8_t* rec;
  int rec_stride, up_off, gate_off, down_off;
  const uint8_t* p1t;
  int p1_row;
  const uint8_t* p2o;
  int p2_stride;
  const float* thresh;
  const float* bias;
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
