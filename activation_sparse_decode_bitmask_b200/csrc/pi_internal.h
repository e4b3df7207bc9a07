// Internal definitions shared by the library's translation units (not part of the ABI).
#pragma once
#include <cstddef>
#include <cstdint>
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

// Kernel launch geometry of the fused kernel: 8 consumer warps + 1 producer warp.
constexpr int kConsumerWarps = 8;
constexpr int kConsumerThreads = kConsumerWarps * 32;
constexpr int kThreads = kConsumerThreads + 32;
constexpr int kMaxSlots = 48;
constexpr int kMaxOwn = 512;          // owned neurons per block (d_ff <= 512 * grid)
constexpr int kMaxList = 512;         // active neurons a block may process in one layer
constexpr int kMaxLayers = 128;       // layers of one pi_decode_stack call

// Library-owned, re-laid-out layer.
struct LayerDev {
  const uint8_t* rec;     // [f][rec_stride]   per-neuron record [gate][up][down]
  const uint8_t* p1t;     // [r][p1_row]       P1 transposed, p_dtype
  const uint8_t* p2n;     // [f][p2_stride]    per-neuron predictor row + (t, b) header
};

}  // namespace pi

struct pi_layer {
  pi_layer_desc desc;
  int family;
  int row_bytes;    // one weight row (d elements) in the record
  int rec_stride;   // bytes per neuron record (gate? + up + down), multiple of 16
  int gate_off, up_off, down_off;   // byte offsets of the rows in a record (gate_off -1 for ReLU)
  int p1_row;       // bytes of one P1^T row (d * p_bytes)
  int p2_stride;    // bytes per neuron predictor row (r * p_bytes + 8, rounded to 16)
  uint8_t* rec;
  uint8_t* p1t;
  uint8_t* p2n;
  float* bias;      // [f] stored order
  float* thresh;    // [f] stored order
  int32_t* perm;    // [f] stored position -> original id
  float* freq_sorted;  // [f] firing frequency in stored order (after a reorder), else null
  int hot_count;    // -1: derived per batch from freq_sorted
  int device;
};

struct pi_workspace {
  int d_max, f_max, r_max, B_max, L_max;
  int grid;          // blocks of the fused kernel (one per SM)
  int device;
  float* u;          // [B_max][r_max]
  uint32_t* maskbuf; // [2][B_max][f_max/32]
  float* partials;   // [grid][B_max][d_max]
  float* v;          // [B_max][d_max]
  float* xb;         // [2][B_max][d_max]
  float* ssq;        // [B_max][grid]
  uint32_t* bar;     // [0] arrive counter, [1] exit counter (reset by the last block out)
  int* err;          // device error word
  unsigned long long* active_total;  // running sum of active-list lengths (all calls)
  int32_t* layer_count;              // [L_max] per-layer union active count of the last stack
  void* x_dev;       // [B_max][d_max] staging for pi_decode_stack_host (fp32 size)
  void* x_host_pinned;
};

namespace pi {

// Parameters of one launch of the fused kernel.
struct FusedParams {
  int mode;            // bit 1: predictor, bit 2: FFN, bit 4: stack glue (layer loop)
  int L, B, d, f, r;
  int grid;
  int row_bytes, rec_stride, gate_off, up_off, down_off, p1_row, p2_stride;
  int slot_bytes, nslots, rows_per_p2slot;
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
  float* u;
  uint32_t* maskbuf;
  float* partials;
  float* v;            // [B][d] x + y of the current layer
  float* xb;           // [2][B][d] fp32 layer inputs, by layer parity
  float* ssq;
  uint32_t* bar;
  int* err;
  unsigned long long* active_total;
  int32_t* layer_count;
  long long barrier_timeout_ns;
  int barrier_extra;   // added to the barrier target (diagnostics: forces a timeout)
};

enum : int { MODE_PREDICT = 1, MODE_FFN = 2, MODE_GLUE = 4 };

cudaError_t launch_fused(int family, int act, int B, const FusedParams& p, size_t smem_bytes,
                         cudaStream_t stream);
size_t fused_smem_bytes(const FusedParams& p);
size_t fused_fixed_smem(int B, int r);
bool fused_supported(int family, int B, int d);
cudaError_t launch_barrier_probe(const FusedParams& p, int rounds, cudaStream_t stream);

cudaError_t launch_compact(const uint32_t* mask, int B, int f, int32_t* idx, int32_t* count,
                           cudaStream_t stream);

}  // namespace pi
