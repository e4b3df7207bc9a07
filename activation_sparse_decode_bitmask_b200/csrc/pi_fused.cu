// The fused persistent kernel of the activation-sparse FFN decode path.
//
// One block per SM: 8 consumer warps and 1 producer warp.  The producer streams every
// byte the block needs from HBM into a byte ring in shared memory, as a few large bulk
// copies per item: the block's P1^T rows, its own neurons' predictor rows (stored
// contiguously per block), and one [gate | up | down] record per active neuron it
// processes.  It runs ahead of the consumers as far as the ring allows, so the next
// layer's predictor is in flight while the consumers wait on cross-block exchanges.
//
// Per layer, for block c of G (stack mode):
//   P-a  u_k = P1^T[k] . x for the block's rank rows k (one warp per row) -> u exchange
//   P-b  logit_i = P2^T[i] . u - t_i for the block's own neurons i = c, c+G, c+2G, ...
//        (8 rows per warp pass); bit = logit > 0
//   list the block's own active neurons, ascending: nothing is exchanged, so the
//        producer starts on the records as soon as the block's own bits are known
//   F    for each of its records: one warp forms the gate/up dot products with x
//          ReLU : h = max(0, w_up_i . x + b_i)    ReGLU: max(0, w_gate_i . x + b_i) * (w_up_i . x)
//          h[b] = 0 where token b's bit is 0
//        then all threads add h * w_down_i into y (registers, fp32, one thread per 16 B)
//        -> partial exchange
//   R    block s < nslices owns a column slice: v = x + sum_c partial_c in ascending c,
//        and the slice's sum and sum of squares -> v / moments exchange
//   glue x' = (v - mean(v)) / sqrt(var(v) + 1e-6) from the slices' sums and sums of
//        squares, rounded to the activation dtype
// Mask words (predict output, trace) are OR-ed in by the owner blocks of their bits.
// Cross-block exchanges use 64-bit words {tag, value}: a reader polls the words
// themselves until every tag matches, so data and completion arrive together and no grid
// barrier is needed.  Tags are unique per launch (a device epoch advanced by the last
// block out), per layer and per exchange.  Every sum runs in a fixed order, so results
// are bitwise reproducible.
#include <cuda_fp16.h>
#include <cstdint>

#include "pi_internal.h"
#include "pi_ptx.cuh"
#include "pi_rowmath.cuh"

namespace pi {

namespace {

constexpr float kRmsEps = 1e-6f;
constexpr int kRedBar = 1;          // named barrier id among consumers
constexpr int kMaxColGroups = 4;    // 32-column groups per reduce slice
constexpr int kItems = 32;          // ring items in flight (mbarrier pairs)
constexpr int kBalK = 12;           // list entries every block publishes at least (balance)
constexpr uint32_t kSleepNs = 20000;  // suspend hint of blocking mbarrier waits (wakes on completion)
constexpr int kHr = 48;             // F h slots: >= kItems + the dot lookahead (16)

struct Smem {
  uint64_t full[kItems];
  uint64_t empty[kItems];
  uint64_t list_ready;          // the first part of the block's list is in place
  uint64_t list2_ready;         // the whole list is in place
  uint64_t f_done;              // the consumers have taken every F record of the layer
  int abort_flag;
  int nlist_a;                  // records of the first part of the list
  int nlist;
  int count;                   // active neurons of the layer (union over tokens)
  int pad;
  uint32_t item_pos[kItems];   // producer bookkeeping of items in flight
  uint32_t item_size[kItems];
  float gmean[4];   // glue: mean and standard deviation of v per token
  float gsd[4];
  float red[2][kConsumerWarps][16];   // block reductions: warp partials (double-buffered)
  uint64_t hready[kHr];         // F: the dot partials of record s (mod kHr) are in hpart[s]
  float hpart[kHr][16];         // [warp of the record's group][token][gate/up]
  int32_t list[kMaxList];
  uint8_t list_bits[kMaxList];
  uint8_t own_bits[kMaxOwn];
  int32_t cnt[kMaxGrid];        // every block's own active count (balance)
  uint32_t bsnap[kMaxGrid * 12];   // every block's first list entries (balance), kBalK per block
  int32_t xpre[kMaxGrid + 1];   // exclusive prefix of the blocks' excess over the target
  int32_t bal[4];               // target, this block's deficit start, total excess
  int32_t wsum[3][kConsumerWarps];   // per-warp partials of the balance's block scans
};

// Diagnostics: SM cycle stamps at phase boundaries, [block][layer][kPhases].
constexpr int kPhases = kDiagSlots;
__device__ __forceinline__ long long stamp_now(const FusedParams& p) {
  return p.phase_global ? (long long)globaltimer_ns() : clock64();
}
__device__ __forceinline__ void stamp(const FusedParams& p, int l, int ph) {
  if (p.phase_clk && threadIdx.x == 0)
    p.phase_clk[((size_t)blockIdx.x * p.L + l) * kPhases + ph] = stamp_now(p);
}
__device__ __forceinline__ void stamp_val(const FusedParams& p, int l, int ph, long long v) {
  if (p.phase_clk && threadIdx.x == 0) p.phase_clk[((size_t)blockIdx.x * p.L + l) * kPhases + ph] = v;
}
__device__ __forceinline__ long long diag_clock(const FusedParams& p) { return p.phase_clk ? clock64() : 0; }
__device__ __forceinline__ void pstamp(const FusedParams& p, int l, int ph) {
  if (p.phase_clk) p.phase_clk[((size_t)blockIdx.x * p.L + l) * kPhases + ph] = stamp_now(p);
}

// Bounded waits count SM cycles (clock64 is cheap to read; the global timer is not):
// `limit` is the wait budget converted to cycles at an upper bound of the SM clock.
__device__ __forceinline__ uint64_t wait_start() { return (uint64_t)clock64(); }
__device__ __forceinline__ bool timed_out(uint64_t t0, long long limit) {
  return (long long)((uint64_t)clock64() - t0) > limit;
}
__device__ __forceinline__ void set_abort(Smem& sm, int* err, int code) {
  atomicExch(err, code);
  *(volatile int*)&sm.abort_flag = 1;
}
__device__ __forceinline__ bool aborted(Smem& sm) { return *(volatile int*)&sm.abort_flag != 0; }

// ------------------------------------------------------------------ tagged words
__device__ __forceinline__ uint64_t tagged(uint32_t bits, uint32_t tag) { return ((uint64_t)tag << 32) | bits; }
__device__ __forceinline__ void st_tag(uint64_t* p, float v, uint32_t tag) {
  asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" ::"l"(p), "l"(tagged(__float_as_uint(v), tag)) : "memory");
}
__device__ __forceinline__ void st_tag2(uint64_t* p, float v0, float v1, uint32_t tag) {
  asm volatile("st.relaxed.gpu.global.v2.b64 [%0], {%1, %2};" ::"l"(p), "l"(tagged(__float_as_uint(v0), tag)),
               "l"(tagged(__float_as_uint(v1), tag))
               : "memory");
}
__device__ __forceinline__ uint64_t ld_tag(const uint64_t* p) {
  uint64_t w;
  asm volatile("ld.relaxed.gpu.global.b64 %0, [%1];" : "=l"(w) : "l"(p) : "memory");
  return w;
}
__device__ __forceinline__ void ld_tag2(const uint64_t* p, uint64_t& a, uint64_t& b) {
  asm volatile("ld.relaxed.gpu.global.v2.b64 {%0, %1}, [%2];" : "=l"(a), "=l"(b) : "l"(p) : "memory");
}
__device__ __forceinline__ bool tag_ok(uint64_t w, uint32_t tag) { return (uint32_t)(w >> 32) == tag; }
__device__ __forceinline__ float tag_val(uint64_t w) { return __uint_as_float((uint32_t)w); }

// Butterfly reduce-scatter of 8 per-lane partial sums (per token) across the warp: on
// return, out[b] in every lane is the full sum of row (lane >> 2) & 7.  The order of
// the additions is fixed, so the sums are reproducible.
template <int NB>
__device__ __forceinline__ void reduce_scatter8(const float (&a)[8][NB], int lane, float (&out)[NB]) {
  const bool h16 = lane & 16, h8 = lane & 8, h4 = lane & 4;
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    float s4[4], s2[2];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float send = h16 ? a[i][b] : a[i + 4][b];
      const float keep = h16 ? a[i + 4][b] : a[i][b];
      s4[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const float send = h8 ? s4[i] : s4[i + 2];
      const float keep = h8 ? s4[i + 2] : s4[i];
      s2[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
    float s1 = (h4 ? s2[1] : s2[0]) + __shfl_xor_sync(0xffffffffu, h4 ? s2[0] : s2[1], 4);
    s1 += __shfl_xor_sync(0xffffffffu, s1, 2);
    s1 += __shfl_xor_sync(0xffffffffu, s1, 1);
    out[b] = s1;
  }
}

// Poll the tagged words base[first + k*stride] (k < MAXK, index < n) until every one
// carries `tag`: each round issues all outstanding loads together, so a round costs one
// L2 round trip whatever the number of words (bounded).
template <int MAXK>
__device__ __forceinline__ void poll_words(const uint64_t* base, int first, int stride, int n, uint32_t tag,
                                           uint64_t (&w)[MAXK], Smem& sm, const FusedParams& p) {
  uint32_t need = 0;
#pragma unroll
  for (int k = 0; k < MAXK; ++k) {
    w[k] = 0;
    if (first + k * stride < n) need |= 1u << k;
  }
  uint64_t t0 = 0;
  bool started = false;
  while (need) {
    // every load of the round is issued before any tag is looked at, so the round costs
    // one L2 round trip whatever the number of words
#pragma unroll
    for (int k = 0; k < MAXK; ++k)
      if (need >> k & 1u) w[k] = ld_tag(base + first + k * stride);
#pragma unroll
    for (int k = 0; k < MAXK; ++k)
      if ((need >> k & 1u) && tag_ok(w[k], tag)) need &= ~(1u << k);
    if (!need || aborted(sm)) break;
    if (!started) {
      t0 = wait_start();
      started = true;
    } else if (timed_out(t0, p.wait_cycles)) {
      set_abort(sm, p.err, DEV_ERR_GRID_TIMEOUT);
      break;
    }
    if (p.poll_ns) __nanosleep(p.poll_ns);   // back off: many blocks poll the same lines
  }
}

// ------------------------------------------------------------------ ring (shared by both sides)
__device__ __forceinline__ uint32_t ring_place(uint32_t& head, uint32_t size, uint32_t cap) {
  uint32_t pos = head;
  if (pos + size > cap) pos = 0;
  head = pos + size;
  return pos;
}

struct ConsumerRing {
  uint8_t* base;
  uint32_t cap, head, item;
};

// Position of the next item (in order) without waiting for it.
__device__ __forceinline__ const uint8_t* ring_next(ConsumerRing& r, uint32_t size) {
  return r.base + ring_place(r.head, size, r.cap);
}
// Wait until ring item `item` has landed (bounded).
// Wait until phase `par` of `bar` has completed (bounded).
__device__ __forceinline__ void bar_wait(uint64_t* bar, uint32_t par, Smem& sm, const FusedParams& p) {
  if (!aborted(sm) && !mbar_try_wait(bar, par)) {
    const uint64_t t0 = wait_start();
    while (!mbar_try_wait_sleep(bar, par, kSleepNs)) {
      if (aborted(sm)) break;
      if (timed_out(t0, p.wait_cycles)) { set_abort(sm, p.err, DEV_ERR_RING_TIMEOUT); break; }
    }
  }
}
__device__ __forceinline__ void ring_wait_item(uint32_t item, Smem& sm, const FusedParams& p) {
  bar_wait(&sm.full[item % kItems], (item / kItems) & 1u, sm, p);
}
// Warp-collective wait for ring item `item`: lane 0 waits on the barrier (acquire) and
// __syncwarp passes the visibility of the landed bytes on to the other lanes, so the
// mbarrier sees one waiter per warp instead of 32.
__device__ __forceinline__ void ring_wait_item_warp(uint32_t item, Smem& sm, const FusedParams& p) {
  if ((threadIdx.x & 31) == 0) ring_wait_item(item, sm, p);
  __syncwarp();
}
__device__ __forceinline__ void ring_release_item(uint32_t item, Smem& sm) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(&sm.empty[item % kItems]);
}

// ------------------------------------------------------------------ activations
template <int FAM>
__device__ __forceinline__ float round_act(float v) {
  if constexpr (FAM == FAM_F32) return v;
  else return __half2float(__float2half_rn(v));
}
template <int FAM>
__device__ __forceinline__ void store_act(void* base, size_t idx, float v) {
  if constexpr (FAM == FAM_F32) reinterpret_cast<float*>(base)[idx] = v;
  else reinterpret_cast<__half*>(base)[idx] = __float2half_rn(v);
}
template <int FAM>
__device__ __forceinline__ float load_act(const void* base, size_t idx) {
  if constexpr (FAM == FAM_F32) return reinterpret_cast<const float*>(base)[idx];
  else return __half2float(reinterpret_cast<const __half*>(base)[idx]);
}

__device__ __forceinline__ int slice_begin(int s, int ns, int ngroups) {
  return (int)((long long)s * ngroups / ns) * 32;
}
__device__ __forceinline__ uint32_t tag_of(uint32_t epoch, int l, int e) {
  return epoch * 1024u + (uint32_t)l * 8u + (uint32_t)e;
}

__host__ __device__ constexpr int pow2_ceil(int v) { return v <= 1 ? 1 : 2 * pow2_ceil((v + 1) / 2); }
__host__ __device__ constexpr int log2_exact(int v) { return v <= 1 ? 0 : 1 + log2_exact(v / 2); }

// Warps that share the gate/up dots of one F record: 4 (8 for Q4_0, whose units cost
// more arithmetic), fewer where the partials of the group would not fit a 16-float slot.
__host__ __device__ constexpr int f_group_warps(int fam, int act, int nb) {
  return (fam == FAM_Q4 ? 8 : 4) * nb * (act == PI_REGLU ? 2 : 1) <= 16 ? (fam == FAM_Q4 ? 8 : 4)
                                                                        : 16 / (nb * (act == PI_REGLU ? 2 : 1));
}

// This lane's partial gate/up dot products of one F record (at shared address rec) with
// every token's x (xs: [NB][d] at shared address xs) over the units q0, q0 + qs, ... in
// ascending order.
template <int FAM, int ACT, int NB>
__device__ __forceinline__ void record_dot(uint32_t rec, uint32_t xs, const FusedParams& p, int nunits, int q0,
                                           int qs, float (&au)[NB], float (&ag)[NB]) {
  constexpr int XW = Fam<FAM>::XW;
#pragma unroll
  for (int b = 0; b < NB; ++b) au[b] = ag[b] = 0.f;
  const uint32_t up = rec + (uint32_t)p.up_off, gate = rec + (uint32_t)p.gate_off;
  if constexpr (FAM == FAM_Q4) {
    // x units widen to 16 fp32 values: one token at a time keeps them in registers
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      float su[1] = {0.f}, sg[1] = {0.f};
#pragma unroll 2
      for (int q = q0; q < nunits; q += qs) {
        uint32_t xu[1][XW];
        lds_x_unit<FAM, 1>(xs + (uint32_t)(b * p.d * 2), p.d, q, xu);
        unit_dot<FAM, 1>(up, p.d, q, xu, su);
        if constexpr (ACT == PI_REGLU) unit_dot<FAM, 1>(gate, p.d, q, xu, sg);
      }
      au[b] = su[0];
      ag[b] = sg[0];
    }
  } else {
#pragma unroll 4
    for (int q = q0; q < nunits; q += qs) {
      uint32_t xu[NB][XW];
      lds_x_unit<FAM, NB>(xs, p.d, q, xu);
      unit_dot<FAM, NB>(up, p.d, q, xu, au);
      if constexpr (ACT == PI_REGLU) unit_dot<FAM, NB>(gate, p.d, q, xu, ag);
    }
  }
}

// Balance the active records across blocks.  Every block publishes its own active count
// and its list entries (id | token bits << 24).  After reading all counts, every block
// derives the same assignment from them alone: target T = max(ceil(N / G), floor); a
// block keeps its first min(n_c, T) own records; the records past T of the blocks above
// the target, in (block, position) order, fill the blocks below it in block order.  So
// every block ends with T or fewer records and the assignment is a function of the data
// and the layer's floor only.  A block's first min(n_c, floor) records are its own in
// any case, so they are fetched while this runs.  Returns the block's new list length;
// the taken records follow its own in sm.list.
__device__ __forceinline__ int balance_list(int n_own, int floor, uint32_t tag_c, Smem& sm, const FusedParams& p, int c,
                                            int G, int t, int warp, int lane, int l) {
  // publish the count and at least kBalK entries (padded), so that one polling round can
  // read every count and every block's first kBalK entries
  if (t < max(n_own, kBalK))
    st_tag(p.lx + (size_t)c * kMaxOwn + t,
           __uint_as_float(t < n_own ? ((uint32_t)sm.list[t] | ((uint32_t)sm.list_bits[t] << 24)) : 0u), tag_c);
  if (t == 0) st_tag(p.cx + c, __int_as_float(n_own), tag_c);
  stamp(p, l, 22);
  {
    // chunks of 4 words per thread: one round for up to 2048 words (157 blocks)
    constexpr int MQ = 4;
    const int nq = G * (1 + kBalK);
    for (int base = 0; base < nq; base += MQ * kConsumerThreads) {
      uint64_t w[MQ];
      uint32_t need = 0;
#pragma unroll
      for (int i = 0; i < MQ; ++i) {
        w[i] = 0;
        if (base + t + i * kConsumerThreads < nq) need |= 1u << i;
      }
      bool started = false;
      uint64_t tp = 0;
      while (need) {
#pragma unroll
        for (int i = 0; i < MQ; ++i)
          if (need >> i & 1u) {
            const int q = base + t + i * kConsumerThreads;
            const uint64_t* src = (q < G) ? p.cx + q : p.lx + (size_t)((q - G) / kBalK) * kMaxOwn + (q - G) % kBalK;
            w[i] = ld_tag(src);
          }
#pragma unroll
        for (int i = 0; i < MQ; ++i)
          if ((need >> i & 1u) && tag_ok(w[i], tag_c)) need &= ~(1u << i);
        if (!need || aborted(sm)) break;
        if (!started) { tp = wait_start(); started = true; }
        else if (timed_out(tp, p.wait_cycles)) { set_abort(sm, p.err, DEV_ERR_GRID_TIMEOUT); break; }
        if (p.poll_ns) __nanosleep(p.poll_ns);
      }
#pragma unroll
      for (int i = 0; i < MQ; ++i) {
        const int q = base + t + i * kConsumerThreads;
        if (q < G) sm.cnt[q] = __float_as_int(tag_val(w[i]));
        else if (q < nq) sm.bsnap[q - G] = (uint32_t)w[i];
      }
    }
  }
  stamp(p, l, 23);
  named_bar_sync(kRedBar, kConsumerThreads);
  stamp(p, l, 24);
  // block-wide: N = sum of the counts, T, the exclusive prefix of the excess over T, and
  // this block's deficit start (the deficits of the blocks before it), in fixed orders
  const int cv = (t < G) ? sm.cnt[t] : 0;
  {
    int v = cv;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) sm.wsum[0][warp] = v;
  }
  named_bar_sync(kRedBar, kConsumerThreads);
  int n = 0;
#pragma unroll
  for (int w = 0; w < kConsumerWarps; ++w) n += sm.wsum[0][w];
  const int Tb = max((n + G - 1) / G, floor);
  const int ex = (t < G) ? max(0, cv - Tb) : 0;
  const int de = (t < c) ? max(0, Tb - cv) : 0;
  int incl = ex, dsum = de;
#pragma unroll
  for (int k = 1; k < 32; k <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, k);
    if (lane >= k) incl += v;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, o);
  if (lane == 31) sm.wsum[1][warp] = incl;
  if (lane == 0) sm.wsum[2][warp] = dsum;
  named_bar_sync(kRedBar, kConsumerThreads);
  {
    int off = 0, total = 0, dstart_all = 0;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) {
      if (w < warp) off += sm.wsum[1][w];
      total += sm.wsum[1][w];
      dstart_all += sm.wsum[2][w];
    }
    if (t < G) sm.xpre[t] = off + incl - ex;
    if (t == 0) {
      sm.xpre[G] = total;
      sm.bal[0] = Tb;
      sm.bal[1] = dstart_all;
      sm.bal[2] = total;
    }
  }
  named_bar_sync(kRedBar, kConsumerThreads);
  const int T = sm.bal[0], dstart = sm.bal[1], xtotal = sm.bal[2];
  const int keep = min(n_own, T);
  const int deficit = max(0, T - n_own);
  const int ntake = max(0, min(dstart + deficit, xtotal) - dstart);
  stamp(p, l, 25);
  if (t < ntake) {
    const int x = dstart + t;
    int lo = 0, hi = G;   // owner o: xpre[o] <= x < xpre[o + 1]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (sm.xpre[mid] <= x) lo = mid;
      else hi = mid;
    }
    const int k = T + (x - sm.xpre[lo]);
    uint32_t v;
    if (k < kBalK) {
      v = sm.bsnap[lo * kBalK + k];
    } else {   // past the snapshot (a block far above the target): read it now
      uint64_t w[1];
      poll_words<1>(p.lx + (size_t)lo * kMaxOwn + k, 0, 1, 1, tag_c, w, sm, p);
      v = (uint32_t)w[0];
    }
    sm.list[keep + t] = (int32_t)(v & 0xFFFFFFu);
    sm.list_bits[keep + t] = (uint8_t)(v >> 24);
  }
  named_bar_sync(kRedBar, kConsumerThreads);
  return keep + ntake;
}

// ------------------------------------------------------------------ the kernel
template <int FAM, int ACT, int NB, int NU>
__global__ void __launch_bounds__(kThreads, 1) fused_kernel(const FusedParams p) {
  constexpr int UE = Fam<FAM>::UE;
  constexpr int XW = Fam<FAM>::XW;
  constexpr int PB = Fam<FAM>::PB;
  using XT = typename Fam<FAM>::X;
  extern __shared__ __align__(128) uint8_t dsmem[];
  Smem& sm = *reinterpret_cast<Smem*>(dsmem);
  uint8_t* ring_base = dsmem + ((sizeof(Smem) + 127) / 128) * 128;
  XT* xs = reinterpret_cast<XT*>(ring_base + p.ring_bytes);            // [NB][d] current input
  float* u_s = reinterpret_cast<float*>(xs + (size_t)NB * p.d);        // [NB][r]
  float* red2 = u_s + (size_t)NB * p.r;                                // [8][NB][4][32]

  const int c = blockIdx.x, G = gridDim.x;
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const bool do_pred = p.mode & MODE_PREDICT, do_ffn = p.mode & MODE_FFN, do_glue = p.mode & MODE_GLUE;
  const int d = p.d, f = p.f, r = p.r, B = p.B;
  const int k0 = (int)((long long)c * r / G), k1 = (int)((long long)(c + 1) * r / G);
  const int nown = (c < f) ? (f - c + G - 1) / G : 0;
  const int nunits = d / UE;
  const int words = f / 32;
  const uint32_t epoch = *reinterpret_cast<volatile const uint32_t*>(p.bar + 2);

  if (t == 0) {
    for (int s = 0; s < kItems; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], kConsumerWarps);
    }
    mbar_init(&sm.list_ready, 1);
    mbar_init(&sm.list2_ready, 1);
    mbar_init(&sm.f_done, 1);
    for (int s = 0; s < kHr; ++s) mbar_init(&sm.hready[s], f_group_warps(FAM, ACT, NB));
    sm.abort_flag = 0;
    sm.nlist = 0;
    mbar_fence_init();
  }
  __syncthreads();

  // ================================================================ producer warp
  if (warp == kConsumerWarps) {
    if (lane == 0) {
      uint32_t head = 0, issued = 0, oldest = 0;
      // Reserve ring space for the next item: wait (in order) for the release of every
      // older item that overlaps it, and of the item that last used its barrier pair.
      auto reserve = [&](uint32_t size, uint32_t& pos) -> bool {
        pos = ring_place(head, size, p.ring_bytes);
        while (oldest < issued) {
          bool must = issued - oldest >= (uint32_t)kItems;
          if (!must) {
            for (uint32_t j = oldest; j < issued; ++j) {
              const uint32_t a = sm.item_pos[j % kItems], e = a + sm.item_size[j % kItems];
              if (pos < e && a < pos + size) { must = true; break; }
            }
          }
          if (!must) break;
          uint64_t* eb = &sm.empty[oldest % kItems];
          const uint32_t par = (oldest / kItems) & 1u;
          if (!mbar_try_wait(eb, par)) {
            const uint64_t t0 = wait_start();
            while (!mbar_try_wait_sleep(eb, par, kSleepNs)) {
              if (aborted(sm)) return false;
              if (timed_out(t0, p.wait_cycles)) { set_abort(sm, p.err, DEV_ERR_RING_TIMEOUT); return false; }
            }
          }
          ++oldest;
        }
        return !aborted(sm);
      };
      auto begin_item = [&](uint32_t size, uint8_t*& dst, uint64_t*& fb) -> bool {
        uint32_t pos;
        if (!reserve(size, pos)) return false;
        sm.item_pos[issued % kItems] = pos;
        sm.item_size[issued % kItems] = size;
        dst = ring_base + pos;
        fb = &sm.full[issued % kItems];
        mbar_arrive_expect_tx(fb, size);
        ++issued;
        return true;
      };
      bool ok = true;
      for (int l = 0; l < p.L && ok; ++l) {
        const LayerDev Ld = p.layers[l];
        uint8_t* dst;
        uint64_t* fb;
        if (do_pred && do_ffn && l > 0) {
          // the predictor rows of this layer are not needed before the glue of the last
          // one ends: start their copies once this block has taken its last F record, so
          // that they do not compete with the F records other blocks still wait for
          const uint64_t t0 = wait_start();
          while (!mbar_try_wait_sleep(&sm.f_done, (uint32_t)((l - 1) & 1), kSleepNs)) {
            if (aborted(sm)) { ok = false; break; }
            if (timed_out(t0, p.wait_cycles)) { set_abort(sm, p.err, DEV_ERR_RING_TIMEOUT); ok = false; break; }
          }
          if (!ok) break;
        }
        if (do_pred) {
          for (int k = k0; k < k1 && ok; k += p.p1_rows_per_item) {
            const int n = min(p.p1_rows_per_item, k1 - k);
            const uint32_t bytes = (uint32_t)n * p.p1_row;
            if (!(ok = begin_item(bytes, dst, fb))) break;
            bulk_g2s(dst, Ld.p1t + (size_t)k * p.p1_row, bytes, fb);
          }
          const uint8_t* own = Ld.p2o + (size_t)c * p.nown_max * p.p2_stride;
          for (int m = 0; m < nown && ok; m += p.p2_rows_per_item) {
            const int n = min(p.p2_rows_per_item, nown - m);
            const uint32_t bytes = (uint32_t)n * p.p2_stride;
            if (!(ok = begin_item(bytes, dst, fb))) break;
            bulk_g2s(dst, own + (size_t)m * p.p2_stride, bytes, fb);
          }
        }
        if (do_ffn && ok) {
          pstamp(p, l, 9);
          const uint64_t t0 = wait_start();
          while (!mbar_try_wait_sleep(&sm.list_ready, (uint32_t)(l & 1), kSleepNs)) {
            if (aborted(sm)) { ok = false; break; }
            if (timed_out(t0, p.wait_cycles)) { set_abort(sm, p.err, DEV_ERR_RING_TIMEOUT); ok = false; break; }
          }
          pstamp(p, l, 10);
          // Ask HBM for every record at once (L2 prefetch needs no shared memory); the
          // ring copies then find them in L2 as space frees up.  The first part of the
          // list is known before the balancing exchange ends, the rest after it.
          const int na = ok ? sm.nlist_a : 0;
          for (int e = 0; e < na && ok; ++e)
            prefetch_l2_bulk(Ld.rec + (size_t)sm.list[e] * p.rec_stride, (uint32_t)p.rec_stride);
          int e = 0;
          for (; e < na && ok; ++e) {
            if (!(ok = begin_item((uint32_t)p.rec_stride, dst, fb))) break;
            bulk_g2s(dst, Ld.rec + (size_t)sm.list[e] * p.rec_stride, (uint32_t)p.rec_stride, fb);
          }
          if (ok) {
            const uint64_t t0 = wait_start();
            while (!mbar_try_wait_sleep(&sm.list2_ready, (uint32_t)(l & 1), kSleepNs)) {
              if (aborted(sm)) { ok = false; break; }
              if (timed_out(t0, p.wait_cycles)) { set_abort(sm, p.err, DEV_ERR_RING_TIMEOUT); ok = false; break; }
            }
          }
          const int n = ok ? sm.nlist : 0;
          for (int q = na; q < n && ok; ++q)
            prefetch_l2_bulk(Ld.rec + (size_t)sm.list[q] * p.rec_stride, (uint32_t)p.rec_stride);
          for (; e < n && ok; ++e) {
            if (!(ok = begin_item((uint32_t)p.rec_stride, dst, fb))) break;
            bulk_g2s(dst, Ld.rec + (size_t)sm.list[e] * p.rec_stride, (uint32_t)p.rec_stride, fb);
          }
          pstamp(p, l, 11);
        }
      }
      // drain: never leave the block while a bulk copy may still write shared memory
      const uint32_t first = issued > (uint32_t)kItems ? issued - kItems : 0u;
      for (uint32_t s = first; s < issued; ++s) {
        uint64_t* fb = &sm.full[s % kItems];
        const uint32_t par = (s / kItems) & 1u;
        const uint64_t t0 = wait_start();
        while (!mbar_try_wait_sleep(fb, par, kSleepNs)) {
          if (timed_out(t0, p.wait_cycles)) { atomicExch(p.err, DEV_ERR_RING_TIMEOUT); break; }
        }
      }
    }
    return;
  }

  // ================================================================ consumers
  ConsumerRing ring{ring_base, (uint32_t)p.ring_bytes, 0u, 0u};

  // the input x of the first layer into shared memory
  for (int idx = t; idx < B * d; idx += kConsumerThreads) xs[idx] = reinterpret_cast<const XT*>(p.x_in)[idx];
  for (int idx = B * d + t; idx < NB * d; idx += kConsumerThreads) xs[idx] = XT(0.f);

  const int ngroups = d / 32;
  const int nslices = p.nslices;
  const bool slice_owner = c < nslices;
  const int col0 = slice_owner ? slice_begin(c, nslices, ngroups) : 0;
  const int col1 = slice_owner ? slice_begin(c + 1, nslices, ngroups) : 0;
  const int ng = (col1 - col0) / 32;
  // slice owners keep their slice of the current layer input (fp32) for the residual:
  // warp b holds token b, lane = column within a 32-column group
  float xsl[kMaxColGroups];
#pragma unroll
  for (int gq = 0; gq < kMaxColGroups; ++gq) xsl[gq] = 0.f;
  if (do_glue && slice_owner && warp < B) {
#pragma unroll
    for (int gq = 0; gq < kMaxColGroups; ++gq)
      if (gq < ng) {
        const size_t idx = (size_t)warp * d + col0 + 32 * gq + lane;
        xsl[gq] = load_act<FAM>(p.x_in, idx);
        if (p.trace.x) store_act<FAM>(p.trace.x, idx, xsl[gq]);
      }
  }
  named_bar_sync(kRedBar, kConsumerThreads);

  int redbuf = 0;   // which half of sm.red the next block reduction uses
  uint32_t fseq = 0;  // F records of earlier layers (h slot of record e: (fseq + e) % kHr)
  for (int l = 0; l < p.L; ++l) {
    const uint32_t tag_u = tag_of(epoch, l, 0), tag_p = tag_of(epoch, l, 1), tag_v = tag_of(epoch, l, 2),
                   tag_c = tag_of(epoch, l, 3);
    int nlist = 0;
    bool signaled_a = false;   // the first part of the list was handed over already
    stamp(p, l, 0);
    // this layer's x units, fp32, in registers for P-a and F
    uint32_t xr[NU][NB][XW];
#pragma unroll
    for (int j = 0; j < NU; ++j) {
      const int q = t + kConsumerThreads * j;
      if (q < nunits) {
        load_x_unit<FAM, NB>(xs, d, q, xr[j]);
      } else {
#pragma unroll
        for (int b = 0; b < NB; ++b)
#pragma unroll
          for (int e = 0; e < XW; ++e) xr[j][b][e] = 0u;
      }
    }

    if (do_pred) {
      // ---------------------------------------------------------- P-a: u rows of this block
      // Every thread dots its x units with each row; a warp reduce-scatter and a 16-warp
      // sum in shared memory finish 16 / NB rows per pass.
      constexpr int RP = 16 / NB;
      for (int k = k0; k < k1; k += p.p1_rows_per_item) {
        const int n = min(p.p1_rows_per_item, k1 - k);
        const uint8_t* item = ring_next(ring, (uint32_t)n * p.p1_row);
        ring_wait_item_warp(ring.item, sm, p);
        if (k == k0) stamp(p, l, 13);
        for (int i0 = 0; i0 < n; i0 += RP) {
          float v[16];
#pragma unroll
          for (int s2 = 0; s2 < 16; ++s2) v[s2] = 0.f;
#pragma unroll
          for (int i = 0; i < RP; ++i) {
            if (i0 + i < n) {
              const uint32_t row = smem_u32(item) + (uint32_t)((i0 + i) * p.p1_row);
              float acc[NB];
#pragma unroll
              for (int b = 0; b < NB; ++b) acc[b] = 0.f;
#pragma unroll
              for (int j = 0; j < NU; ++j)
                if (t + kConsumerThreads * j < nunits) unit_dot_p<FAM, NB>(row, t + kConsumerThreads * j, xr[j], acc);
#pragma unroll
              for (int b = 0; b < NB; ++b) v[i * NB + b] = acc[b];
            }
          }
          const float sw = reduce_scatter<16>(v, lane);
          float* red = &sm.red[redbuf][0][0];
          redbuf ^= 1;
          if ((lane & 1) == 0) red[warp * 16 + (lane >> 1)] = sw;
          named_bar_sync(kRedBar, kConsumerThreads);
          if (t < RP * NB) {
            const int i = t / NB, b = t % NB;
            if (i0 + i < n && b < B) {
              float u = 0.f;
#pragma unroll
              for (int w = 0; w < kConsumerWarps; ++w) u += red[w * 16 + t];
              st_tag(p.ux + (size_t)b * r + k + i0 + i, u, tag_u);
            }
          }
        }
        ring_release_item(ring.item++, sm);
      }
      stamp(p, l, 1);
      // ---------------------------------------------------------- u exchange
      {
        constexpr int KU = 6 * NB;   // r <= 1536
        uint64_t w[KU];
        poll_words<KU>(p.ux, t, kConsumerThreads, B * r, tag_u, w, sm, p);
#pragma unroll
        for (int k = 0; k < KU; ++k)
          if (t + k * kConsumerThreads < B * r) u_s[t + k * kConsumerThreads] = tag_val(w[k]);
      }
      named_bar_sync(kRedBar, kConsumerThreads);
      stamp(p, l, 2);

      // ---------------------------------------------------------- P-b: own logits
      // A warp takes 8 rows at a time: lane q accumulates the 16-byte chunks q, q+32, ...
      // of all 8 rows, then a butterfly reduce-scatter leaves the whole dot of row
      // (lane >> 2) & 7 in lanes 4j..4j+3 (9 shuffles for 8 rows).
      uint32_t* mask_dst = do_glue ? (p.trace.mask ? p.trace.mask + (size_t)l * B * words : nullptr) : p.mask_out;
      const int rchunks = r * PB / 16;
      long long pb_wait = 0;   // diagnostics: cycles spent waiting for P2 items
      for (int m0 = 0; m0 < nown; m0 += p.p2_rows_per_item) {
        const int n = min(p.p2_rows_per_item, nown - m0);
        const uint8_t* item = ring_next(ring, (uint32_t)n * p.p2_stride);
        const long long wt0 = diag_clock(p);
        ring_wait_item_warp(ring.item, sm, p);
        pb_wait += diag_clock(p) - wt0;
        if (m0 == 0) stamp(p, l, 12);
        for (int mb = warp * 8; mb < n; mb += kConsumerWarps * 8) {
          uint32_t rows[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) rows[i] = smem_u32(item) + (uint32_t)(min(mb + i, n - 1) * p.p2_stride);   // past n: repeats, unused
          float acc[8][NB];
#pragma unroll
          for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int b = 0; b < NB; ++b) acc[i][b] = 0.f;
          for (int q = lane; q < rchunks; q += 32) {
            if constexpr (PB == 4) {
              float4 uu[NB];
#pragma unroll
              for (int b = 0; b < NB; ++b) uu[b] = *reinterpret_cast<const float4*>(u_s + b * r + 4 * q);
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const float4 w = u4f(lds128(rows[i] + 16u * q));
#pragma unroll
                for (int b = 0; b < NB; ++b)
                  acc[i][b] = fmaf(w.w, uu[b].w, fmaf(w.z, uu[b].z, fmaf(w.y, uu[b].y, fmaf(w.x, uu[b].x, acc[i][b]))));
              }
            } else {
              float4 u0[NB], u1[NB];
#pragma unroll
              for (int b = 0; b < NB; ++b) {
                u0[b] = *reinterpret_cast<const float4*>(u_s + b * r + 8 * q);
                u1[b] = *reinterpret_cast<const float4*>(u_s + b * r + 8 * q + 4);
              }
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const uint4 w = lds128(rows[i] + 16u * q);
                const float2 a = h2f2(w.x), bb = h2f2(w.y), cc = h2f2(w.z), e = h2f2(w.w);
#pragma unroll
                for (int b = 0; b < NB; ++b) {
                  float s = acc[i][b];
                  s = fmaf(a.x, u0[b].x, s); s = fmaf(a.y, u0[b].y, s); s = fmaf(bb.x, u0[b].z, s);
                  s = fmaf(bb.y, u0[b].w, s); s = fmaf(cc.x, u1[b].x, s); s = fmaf(cc.y, u1[b].y, s);
                  s = fmaf(e.x, u1[b].z, s); s = fmaf(e.y, u1[b].w, s);
                  acc[i][b] = s;
                }
              }
            }
          }
          float dot[NB];
          reduce_scatter8<NB>(acc, lane, dot);
          const int m = mb + ((lane >> 2) & 7);
          if ((lane & 3) == 0 && m < n) {
            uint32_t trow = rows[0];
#pragma unroll
            for (int i = 1; i < 8; ++i) if (i == ((lane >> 2) & 7)) trow = rows[i];
            const float ti = lds_f32(trow + (uint32_t)(r * PB));
            const int i = c + (m0 + m) * G;
            uint32_t bits = 0;
#pragma unroll
            for (int b = 0; b < NB; ++b) {
              if (b < B) {
                const float lg = dot[b] - ti;
                if (lg > 0.f) {
                  bits |= 1u << b;
                  if (mask_dst) atomicOr(mask_dst + (size_t)b * words + (i >> 5), 1u << (i & 31));
                }
                if (p.logits_out) p.logits_out[(size_t)b * f + i] = lg;
                if (p.trace.logits) p.trace.logits[((size_t)l * B + b) * f + i] = lg;
              }
            }
            sm.own_bits[m0 + m] = (uint8_t)bits;
          }
        }
        ring_release_item(ring.item++, sm);
      }
      named_bar_sync(kRedBar, kConsumerThreads);
      stamp(p, l, 7);
      stamp_val(p, l, 18, pb_wait);

      // ---------------------------------------------------------- own active list
      // Block c processes the active neurons it owns, i = c + m*G in ascending m: the
      // list needs nothing from other blocks.
      if (warp == 0) {
        int base = 0;
        for (int mm = 0; mm < nown; mm += 32) {
          const int m = mm + lane;
          const uint32_t tb = (m < nown) ? sm.own_bits[m] : 0u;
          const uint32_t bal = __ballot_sync(0xffffffffu, tb != 0u);
          if (tb) {
            const int e = base + __popc(bal & ((1u << lane) - 1u));
            sm.list[e] = c + m * G;
            sm.list_bits[e] = (uint8_t)tb;
          }
          base += __popc(bal);
        }
        if (lane == 0) sm.count = base;
      }
      named_bar_sync(kRedBar, kConsumerThreads);
      nlist = sm.count;
      if (t == 0 && do_ffn && nlist > 0) {
        atomicAdd(p.active_total, (unsigned long long)nlist);
        if (p.layer_count) atomicAdd(p.layer_count + l, nlist);
      }
      stamp(p, l, 15);
      if (do_ffn && p.cx) {
        // the first part (own records every block keeps) goes to the producer now
        const int floor = p.layers[l].keep_floor;
        if (t == 0) {
          sm.nlist_a = min(nlist, floor);
          mbar_arrive(&sm.list_ready);
        }
        signaled_a = true;
        nlist = balance_list(nlist, floor, tag_c, sm, p, c, G, t, warp, lane, l);
      }
      stamp_val(p, l, 14, nlist);
    } else if (do_ffn) {
      // ---------------------------------------------------------- list from the caller
      int cnt = __ldg(p.count_in);
      if (cnt < 0 || cnt > f) {
        if (t == 0) atomicExch(p.err, DEV_ERR_INDEX);
        cnt = 0;
      }
      const int a0 = (int)((long long)c * cnt / G), a1 = (int)((long long)(c + 1) * cnt / G);
      nlist = a1 - a0;
      if (nlist > kMaxList) {
        if (t == 0) atomicExch(p.err, DEV_ERR_LIST);
        nlist = 0;
      }
      for (int e = t; e < nlist; e += kConsumerThreads) {
        int i = __ldg(p.idx_in + a0 + e);
        if (i < 0 || i >= f) { atomicExch(p.err, DEV_ERR_INDEX); i = 0; }
        uint32_t bits = 0;
        for (int b = 0; b < B; ++b) bits |= ((__ldg(p.mask_in + (size_t)b * words + (i >> 5)) >> (i & 31)) & 1u) << b;
        sm.list[e] = i;
        sm.list_bits[e] = (uint8_t)bits;
      }
      if (t == 0) atomicAdd(p.active_total, (unsigned long long)nlist);
    }

    if (!do_ffn) break;   // predictor only
    named_bar_sync(kRedBar, kConsumerThreads);
    if (t == 0) {
      if (!signaled_a) {
        sm.nlist_a = nlist;
        mbar_arrive(&sm.list_ready);
      }
      sm.nlist = nlist;
      mbar_arrive(&sm.list2_ready);
    }
    stamp(p, l, 3);

    // ------------------------------------------------------------ F: records
    // The 16 consumer warps form groups of KG; group g takes the gate/up dots of records
    // g, g + 16/KG, ... with no block barrier: each warp of the group waits for the record
    // to land, dots its slice of the units with x from shared memory, reduces across its
    // lanes, posts its partial sums in the record's h slot and arrives on the slot's
    // barrier.  Every thread then adds h * (its units of each down row) into its y units
    // in list order: it waits on each record's slot, sums the KG partials in a fixed order,
    // forms h and releases the record.  A warp dots a record only while it is fewer than R
    // records ahead of its own down-row cursor, so the records a warp waits for always
    // fit in the ring beside the ones not yet released.  Sums run in a fixed order
    // whatever the timing.
    float y[NU][NB][UE];
#pragma unroll
    for (int j = 0; j < NU; ++j)
#pragma unroll
      for (int b = 0; b < NB; ++b)
#pragma unroll
        for (int e = 0; e < UE; ++e) y[j][b][e] = 0.f;
    {
      constexpr int NV = (ACT == PI_REGLU) ? 2 : 1;
      constexpr int NVAL = NB * NV;                 // partial sums per warp and record
      constexpr int V = pow2_ceil(NVAL);
      constexpr int LG = log2_exact(V);
      constexpr int KG = f_group_warps(FAM, ACT, NB);
      constexpr int NG = kConsumerWarps / KG;       // records dotted at once
      static_assert(KG * NVAL <= 16 && kConsumerWarps % KG == 0, "h slot layout");
      // records E .. E + R - 1 fit in the ring together (at most one record's worth of
      // space is lost where the placement wraps)
      const int R = max(1, min((int)(ring.cap / (uint32_t)p.rec_stride) - 1, kConsumerWarps));
      const uint32_t base = smem_u32(ring.base), xsa = smem_u32(xs);
      const uint32_t item0 = ring.item;
      const int kq = warp % KG;
      long long f_wait = 0, d_wait = 0;   // diagnostics: cycles thread 0 waits for h / for records
      int ed = warp / KG;                  // next record this warp's group dots
      uint32_t hd = ring.head;             // ring head before record id (dot cursor)
      int id = 0;
      for (int ea = 0; ea < nlist; ++ea) {
        while (ed < nlist && ed < ea + R) {
          uint32_t pos = 0;
          for (; id <= ed; ++id) pos = ring_place(hd, (uint32_t)p.rec_stride, ring.cap);
          const long long wt0 = diag_clock(p);
          ring_wait_item_warp(item0 + ed, sm, p);
          d_wait += diag_clock(p) - wt0;
          if (ed == 0) stamp(p, l, 5);
          float au[NB], ag[NB];
          record_dot<FAM, ACT, NB>(base + pos, xsa, p, nunits, 32 * kq + lane, 32 * KG, au, ag);
          float v[V];
#pragma unroll
          for (int i = 0; i < V; ++i) v[i] = 0.f;
#pragma unroll
          for (int b = 0; b < NB; ++b) {
            v[b * NV] = au[b];
            if constexpr (ACT == PI_REGLU) v[b * NV + 1] = ag[b];
          }
          const float sw = reduce_scatter<V>(v, lane);   // lane k: value k >> (5 - LG)
          const uint32_t s = (fseq + (uint32_t)ed) % kHr;
          if ((lane & ((32 >> LG) - 1)) == 0 && (lane >> (5 - LG)) < NVAL) sm.hpart[s][kq * NVAL + (lane >> (5 - LG))] = sw;
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.hready[s]);
          ed += NG;
        }
        const uint32_t pa = ring_place(ring.head, (uint32_t)p.rec_stride, ring.cap);
        const uint32_t sq = fseq + (uint32_t)ea;
        const long long wt0 = diag_clock(p);
        if (lane == 0) bar_wait(&sm.hready[sq % kHr], (sq / kHr) & 1u, sm, p);
        __syncwarp();
        f_wait += diag_clock(p) - wt0;
        const float* hp = sm.hpart[sq % kHr];
        float sv[NVAL];
#pragma unroll
        for (int i = 0; i < NVAL; ++i) {
          float a = hp[i];
#pragma unroll
          for (int k = 1; k < KG; ++k) a += hp[k * NVAL + i];
          sv[i] = a;
        }
        const float bi = lds_f32(base + pa + (uint32_t)p.bias_off);
        const uint32_t bits = sm.list_bits[ea];
        float h[NB];
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          float a;
          if constexpr (ACT == PI_REGLU) a = fmaxf(sv[b * NV + 1] + bi, 0.f) * sv[b * NV];
          else a = fmaxf(sv[b * NV] + bi, 0.f);
          h[b] = (b < B && ((bits >> b) & 1u)) ? a : 0.f;
        }
        const uint32_t drow = base + pa + (uint32_t)p.down_off;
#pragma unroll
        for (int j = 0; j < NU; ++j)
          if (t + kConsumerThreads * j < nunits) unit_axpy<FAM, NB>(drow, d, t + kConsumerThreads * j, h, y[j]);
        ring_release_item(item0 + ea, sm);
      }
      ring.item = item0 + (uint32_t)nlist;
      fseq += (uint32_t)nlist;
      if (t == 0) mbar_arrive(&sm.f_done);
      stamp(p, l, 20);
      stamp_val(p, l, 19, f_wait);
      stamp_val(p, l, 21, d_wait);
    }
    // publish the partial y of this block as tagged words
    {
      uint64_t* part = p.px + (size_t)c * B * d;
#pragma unroll
      for (int b = 0; b < NB; ++b)
#pragma unroll
        for (int j = 0; j < NU; ++j) {
          const int q = t + kConsumerThreads * j;
          if (b < B && q < nunits) {
            uint64_t* dst = part + (size_t)b * d + (size_t)q * UE;
#pragma unroll
            for (int e = 0; e < UE; e += 2) st_tag2(dst + e, y[j][b][e], y[j][b][e + 1], tag_p);
          }
        }
    }
    stamp(p, l, 4);

    // ------------------------------------------------------------ R: slice reduce
    if (slice_owner) {
      // warp w sums partial rows cc = w, w+8, ...; KU rows' words are read together so
      // the L2 round trips overlap; sums run in ascending cc (fixed order)
      constexpr int KU = 10 / NB;   // 16 warps x 10 rows: all 148 partials in one round at one token
      float acc[NB][kMaxColGroups];
#pragma unroll
      for (int b = 0; b < NB; ++b)
#pragma unroll
        for (int gq = 0; gq < kMaxColGroups; ++gq) acc[b][gq] = 0.f;
      const uint64_t t0 = wait_start();
      for (int gq = 0; gq < ng; ++gq) {
        for (int cc0 = warp; cc0 < G; cc0 += kConsumerWarps * KU) {
          float tmp[KU][NB];
          uint32_t need = 0;
#pragma unroll
          for (int k = 0; k < KU; ++k)
#pragma unroll
            for (int b = 0; b < NB; ++b) {
              tmp[k][b] = 0.f;
              if (cc0 + kConsumerWarps * k < G && b < B) need |= 1u << (k * NB + b);
            }
          while (need) {
            uint64_t wk[KU][NB];
#pragma unroll
            for (int k = 0; k < KU; ++k)
#pragma unroll
              for (int b = 0; b < NB; ++b) {
                wk[k][b] = 0;
                if (need >> (k * NB + b) & 1u)
                  wk[k][b] = ld_tag(p.px + ((size_t)(cc0 + kConsumerWarps * k) * B + b) * d + col0 + 32 * gq + lane);
              }
#pragma unroll
            for (int k = 0; k < KU; ++k)
#pragma unroll
              for (int b = 0; b < NB; ++b)
                if ((need >> (k * NB + b) & 1u) && tag_ok(wk[k][b], tag_p)) {
                  tmp[k][b] = tag_val(wk[k][b]);
                  need &= ~(1u << (k * NB + b));
                }
            if (need && aborted(sm)) break;
            if (need && timed_out(t0, p.wait_cycles)) { set_abort(sm, p.err, DEV_ERR_GRID_TIMEOUT); break; }
            if (need && p.poll_ns) __nanosleep(p.poll_ns);
          }
#pragma unroll
          for (int k = 0; k < KU; ++k)
#pragma unroll
            for (int b = 0; b < NB; ++b) acc[b][gq] += tmp[k][b];
        }
      }
#pragma unroll
      for (int b = 0; b < NB; ++b)
#pragma unroll
        for (int gq = 0; gq < kMaxColGroups; ++gq)
          red2[((warp * NB + b) * kMaxColGroups + gq) * 32 + lane] = acc[b][gq];
      named_bar_sync(kRedBar, kConsumerThreads);
      // warp b finishes token b's columns, summing the warps' parts in a fixed order
      if (warp < NB && warp < B) {
        const int b = warp;
        float sq = 0.f, sv = 0.f;
#pragma unroll
        for (int gq = 0; gq < kMaxColGroups; ++gq) {
          if (gq < ng) {
            float yv = 0.f;
#pragma unroll
            for (int w = 0; w < kConsumerWarps; ++w) yv += red2[((w * NB + b) * kMaxColGroups + gq) * 32 + lane];
            const int j = col0 + 32 * gq + lane;
            if (do_glue) {
              const float vv = xsl[gq] + yv;
              xsl[gq] = vv;   // holds v until the glue turns it into the next input
              sq += vv * vv;
              sv += vv;
              st_tag(p.vx + (size_t)b * d + j, vv, tag_v);
              if (p.trace.y) p.trace.y[((size_t)l * B + b) * d + j] = yv;
            } else {
              p.y_out[(size_t)b * d + j] = yv;
            }
          }
        }
        if (do_glue) {
          sq = warp_sum(sq);
          sv = warp_sum(sv);
          if (lane == 0) {
            st_tag(p.sx + ((size_t)b * G + c) * 2, sv, tag_v);
            st_tag(p.sx + ((size_t)b * G + c) * 2 + 1, sq, tag_v);
          }
        }
      }
    }
    if (!do_glue) break;
    stamp(p, l, 6);

    // ------------------------------------------------------------ glue: x' = (v - mean) / sd
    // One polling round reads both what the slice owners published: every thread polls its
    // v pairs of the first chunk and a few of the slices' (sum, sum of squares) words.
    {
      const int npairs = B * d / 2;
      const int nmom = 2 * nslices * B;
      constexpr int MQ = (2 * kMaxGrid * 4 + kConsumerThreads - 1) / kConsumerThreads;
      uint64_t w0[8], w1[8], wm[MQ];
      uint32_t need = 0, needm = 0;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        w0[k] = w1[k] = 0;
        if (t + k * kConsumerThreads < npairs) need |= 1u << k;
      }
#pragma unroll
      for (int i = 0; i < MQ; ++i) {
        wm[i] = 0;
        if (t + i * kConsumerThreads < nmom) needm |= 1u << i;
      }
      {
        bool started = false;
        uint64_t tp = 0;
        while (need | needm) {
#pragma unroll
          for (int k = 0; k < 8; ++k)
            if (need >> k & 1u) ld_tag2(p.vx + 2 * (size_t)(t + k * kConsumerThreads), w0[k], w1[k]);
#pragma unroll
          for (int i = 0; i < MQ; ++i)
            if (needm >> i & 1u) {
              const int q = t + i * kConsumerThreads;
              const int bq = q / (2 * nslices), cq = (q >> 1) % nslices;
              wm[i] = ld_tag(p.sx + ((size_t)bq * G + cq) * 2 + (q & 1));
            }
#pragma unroll
          for (int k = 0; k < 8; ++k)
            if ((need >> k & 1u) && tag_ok(w0[k], tag_v) && tag_ok(w1[k], tag_v)) need &= ~(1u << k);
#pragma unroll
          for (int i = 0; i < MQ; ++i)
            if ((needm >> i & 1u) && tag_ok(wm[i], tag_v)) needm &= ~(1u << i);
          if (!(need | needm) || aborted(sm)) break;
          if (!started) { tp = wait_start(); started = true; }
          else if (timed_out(tp, p.wait_cycles)) { set_abort(sm, p.err, DEV_ERR_GRID_TIMEOUT); break; }
          if (p.poll_ns) __nanosleep(p.poll_ns);
        }
      }
      named_bar_sync(kRedBar, kConsumerThreads);   // the slice reduce is done with red2; nobody reads xs
      stamp(p, l, 16);
      float* mom = red2;                            // [B][nslices][2]
#pragma unroll
      for (int i = 0; i < MQ; ++i)
        if (t + i * kConsumerThreads < nmom) mom[t + i * kConsumerThreads] = tag_val(wm[i]);
      named_bar_sync(kRedBar, kConsumerThreads);
      if (warp < NB) {
        float s = 0.f, s2 = 0.f;
        if (warp < B)
          for (int cq = lane; cq < nslices; cq += 32) {
            s += mom[(warp * nslices + cq) * 2];
            s2 += mom[(warp * nslices + cq) * 2 + 1];
          }
        const float sum = warp_sum(s);
        s2 = warp_sum(s2);
        if (lane == 0) {
          const float mean = sum / (float)d;
          const float var = fmaxf(s2 / (float)d - mean * mean, 0.f);
          sm.gmean[warp] = mean;
          sm.gsd[warp] = sqrtf(var + kRmsEps);
        }
      }
      named_bar_sync(kRedBar, kConsumerThreads);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int pr = t + k * kConsumerThreads;
        if (pr < npairs) {
          const int idx = 2 * pr, b = idx / d;
          const float mean = sm.gmean[b], sd = sm.gsd[b];
          xs[idx] = XT(round_act<FAM>((tag_val(w0[k]) - mean) / sd));
          xs[idx + 1] = XT(round_act<FAM>((tag_val(w1[k]) - mean) / sd));
        }
      }
      // pairs past the first chunk (wide layers or several tokens): published already
      for (int base = 8 * kConsumerThreads; base < npairs; base += 8 * kConsumerThreads) {
#pragma unroll
        for (int k = 0; k < 8; ++k) w0[k] = w1[k] = 0;
        need = 0;
#pragma unroll
        for (int k = 0; k < 8; ++k)
          if (base + t + k * kConsumerThreads < npairs) need |= 1u << k;
        bool started = false;
        uint64_t tp = 0;
        while (need) {
#pragma unroll
          for (int k = 0; k < 8; ++k)
            if (need >> k & 1u) ld_tag2(p.vx + 2 * (size_t)(base + t + k * kConsumerThreads), w0[k], w1[k]);
#pragma unroll
          for (int k = 0; k < 8; ++k)
            if ((need >> k & 1u) && tag_ok(w0[k], tag_v) && tag_ok(w1[k], tag_v)) need &= ~(1u << k);
          if (!need || aborted(sm)) break;
          if (!started) { tp = wait_start(); started = true; }
          else if (timed_out(tp, p.wait_cycles)) { set_abort(sm, p.err, DEV_ERR_GRID_TIMEOUT); break; }
          if (p.poll_ns) __nanosleep(p.poll_ns);
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int pr = base + t + k * kConsumerThreads;
          if (pr < npairs) {
            const int idx = 2 * pr, b = idx / d;
            const float mean = sm.gmean[b], sd = sm.gsd[b];
            xs[idx] = XT(round_act<FAM>((tag_val(w0[k]) - mean) / sd));
            xs[idx + 1] = XT(round_act<FAM>((tag_val(w1[k]) - mean) / sd));
          }
        }
      }
      stamp(p, l, 17);
      // slice owners: the new input of their slice, the trace, and the output
      if (slice_owner && warp < NB && warp < B) {
        const int b = warp;
        const float mean = sm.gmean[b], sd = sm.gsd[b];
#pragma unroll
        for (int gq = 0; gq < kMaxColGroups; ++gq)
          if (gq < ng) {
            const size_t j = (size_t)b * d + col0 + 32 * gq + lane;
            xsl[gq] = round_act<FAM>((xsl[gq] - mean) / sd);
            if (p.trace.x) store_act<FAM>(p.trace.x, (size_t)(l + 1) * B * d + j, xsl[gq]);
            if (l == p.L - 1) store_act<FAM>(p.x_out, j, xsl[gq]);
          }
      }
      named_bar_sync(kRedBar, kConsumerThreads);
    }
    stamp(p, l, 8);
  }

  // last block out: advance the epoch (new tags for the next launch) and reset the count
  named_bar_sync(kRedBar, kConsumerThreads);
  if (t == 0) {
    __threadfence();
    const uint32_t prev = atomicAdd(p.bar + 1, 1u);
    if (prev == (uint32_t)G - 1) {
      atomicExch(p.bar + 2, epoch + 1u);
      atomicExch(p.bar + 1, 0u);
    }
  }
}

// ------------------------------------------------------------------ grid barrier probe
// A kernel that only runs grid barriers; with barrier_extra > 0 the target can never be
// reached, so every wait must give up after barrier_timeout_ns and report it.
__global__ void __launch_bounds__(kThreads, 1) barrier_probe_kernel(const FusedParams p, int rounds) {
  __shared__ int abort_flag;
  if (threadIdx.x == 0) abort_flag = 0;
  __syncthreads();
  if (threadIdx.x >= kConsumerThreads) return;
  uint32_t epoch = 0;
  for (int i = 0; i < rounds; ++i) {
    named_bar_sync(kRedBar, kConsumerThreads);
    ++epoch;
    if (threadIdx.x == 0 && !abort_flag) {
      const uint32_t target = epoch * (uint32_t)gridDim.x + (uint32_t)p.barrier_extra;
      red_release_gpu_add(p.bar, 1u);
      const uint64_t t0 = wait_start();
      while (ld_acquire_gpu(p.bar) < target) {
        if (timed_out(t0, p.wait_cycles)) {
          atomicExch(p.err, DEV_ERR_GRID_TIMEOUT);
          abort_flag = 1;
          break;
        }
      }
    }
    named_bar_sync(kRedBar, kConsumerThreads);
  }
  named_bar_sync(kRedBar, kConsumerThreads);
  if (threadIdx.x == 0) {
    __threadfence();
    const uint32_t prev = atomicAdd(p.bar + 1, 1u);
    if (prev == (uint32_t)gridDim.x - 1) {
      atomicExch(p.bar, 0u);
      atomicExch(p.bar + 1, 0u);
    }
  }
}

constexpr int ue_of(int fam) { return fam == FAM_F32 ? 4 : fam == FAM_F16 ? 8 : 16; }

// Largest d_model each (family, tokens) pair serves, and the unit count per consumer
// thread that covers it; a launch takes the smallest count that covers its d, so x and y
// in registers stay small.
constexpr int d_max_of(int fam, int nb) {
  return fam == FAM_F32 ? (nb == 4 ? 2048 : 4096)
                        : fam == FAM_F16 ? (nb == 1 ? 12288 : nb == 2 ? 8192 : 4096) : (nb <= 2 ? 8192 : 0);
}
constexpr int nu_max(int fam, int nb) {
  return (d_max_of(fam, nb) / ue_of(fam) + kConsumerThreads - 1) / kConsumerThreads;
}

int nb_of(int B) { return B <= 1 ? 1 : B <= 2 ? 2 : B <= 4 ? 4 : 0; }

template <int FAM, int ACT, int NB, int NU>
cudaError_t launch_t(const FusedParams& p, size_t smem, cudaStream_t stream) {
  auto kern = fused_kernel<FAM, ACT, NB, NU>;
  static int configured = 0;   // the attribute is per function; raise it when a launch needs more
  if ((int)smem > configured) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    configured = (int)smem;
  }
  void* args[] = {const_cast<FusedParams*>(&p)};
  return cudaLaunchCooperativeKernel((const void*)kern, dim3(p.grid), dim3(kThreads), args, smem, stream);
}

template <int FAM, int ACT, int NB>
cudaError_t launch_nu(const FusedParams& p, size_t smem, cudaStream_t stream) {
  constexpr int M = nu_max(FAM, NB);
  const int nunits = p.d / ue_of(FAM);
  const int nu = (nunits + kConsumerThreads - 1) / kConsumerThreads;
  if constexpr (M >= 1) if (nu <= 1) return launch_t<FAM, ACT, NB, 1>(p, smem, stream);
  if constexpr (M >= 2) if (nu == 2) return launch_t<FAM, ACT, NB, 2>(p, smem, stream);
  if constexpr (M >= 3) if (nu == 3) return launch_t<FAM, ACT, NB, 3>(p, smem, stream);
  if constexpr (M >= 4) if (nu == 4) return launch_t<FAM, ACT, NB, 4>(p, smem, stream);
  if constexpr (M >= 5) if (nu == 5) return launch_t<FAM, ACT, NB, 5>(p, smem, stream);
  if constexpr (M >= 6) if (nu == 6) return launch_t<FAM, ACT, NB, 6>(p, smem, stream);
  static_assert(M <= 6, "unit counts above 6 are not instantiated");
  return cudaErrorNotSupported;
}

template <int FAM, int ACT>
cudaError_t launch_nb(int B, const FusedParams& p, size_t smem, cudaStream_t stream) {
  switch (nb_of(B)) {
    case 1: return launch_nu<FAM, ACT, 1>(p, smem, stream);
    case 2: return launch_nu<FAM, ACT, 2>(p, smem, stream);
    case 4:
      if constexpr (FAM != FAM_Q4) return launch_nu<FAM, ACT, 4>(p, smem, stream);
      else return cudaErrorNotSupported;
  }
  return cudaErrorNotSupported;
}

}  // namespace

bool fused_supported(int family, int B, int d) {
  const int nb = nb_of(B);
  if (nb == 0) return false;
  return d <= d_max_of(family, nb);
}

size_t fused_fixed_smem(int B, int d, int r, int grid, int nown_max, int family) {
  const int nb = nb_of(B) ? nb_of(B) : 4;
  const size_t xbytes = family == FAM_F32 ? 4 : 2;
  return ((sizeof(Smem) + 127) / 128) * 128 + (size_t)nb * d * xbytes + (size_t)nb * r * sizeof(float) +
         (size_t)kConsumerWarps * nb * kMaxColGroups * 32 * sizeof(float) + 128;
}


cudaError_t launch_fused(int family, int act, int B, const FusedParams& p, size_t smem, cudaStream_t stream) {
  if (family == FAM_F32)
    return act == PI_REGLU ? launch_nb<FAM_F32, PI_REGLU>(B, p, smem, stream)
                           : launch_nb<FAM_F32, PI_RELU>(B, p, smem, stream);
  if (family == FAM_F16)
    return act == PI_REGLU ? launch_nb<FAM_F16, PI_REGLU>(B, p, smem, stream)
                           : launch_nb<FAM_F16, PI_RELU>(B, p, smem, stream);
  if (family == FAM_Q4)
    return act == PI_REGLU ? launch_nb<FAM_Q4, PI_REGLU>(B, p, smem, stream)
                           : launch_nb<FAM_Q4, PI_RELU>(B, p, smem, stream);
  return cudaErrorNotSupported;
}

cudaError_t launch_barrier_probe(const FusedParams& p, int rounds, cudaStream_t stream) {
  void* args[] = {const_cast<FusedParams*>(&p), &rounds};
  return cudaLaunchCooperativeKernel((const void*)barrier_probe_kernel, dim3(p.grid), dim3(kThreads), args, 0,
                                     stream);
}

}  // namespace pi
