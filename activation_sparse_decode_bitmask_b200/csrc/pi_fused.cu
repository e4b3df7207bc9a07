// The fused persistent kernel of the activation-sparse FFN decode path.
//
// One block per SM: 16 consumer warps and 1 producer warp.  The producer streams the
// block's predictor rows and the [gate | up | bias] record of every active neuron the
// block dots from HBM into a byte ring in shared memory, as bulk copies completing on
// mbarriers.  It runs ahead of the consumers as far as the ring allows, so the next
// layer's predictor is in flight while the consumers finish the current one.
//
// Per layer, for block c of G (stack mode):
//   P-a   u_k = P1^T[k] . x for the block's rank rows k -> u exchange
//   P-b   logit_i = P2^T[i] . u - t_i for the block's own neurons i = c, c+G, c+2G, ...;
//         bit = logit > 0.  The block lists its own active neurons and hands the first
//         of them (a floor set from the firing frequencies) to the producer at once.
//   mask  every block publishes its own bit words; one polling round gives every block
//         every bit.  From the union counts each block derives the same balanced
//         assignment: it keeps up to T of its own active neurons and takes the excess of
//         the blocks above T, so every block dots at most T = max(ceil(N/G), floor).
//   F     gate/up dot products of the assigned records (a group of warps per record):
//           ReLU : h = max(0, w_up_i . x + b_i)    ReGLU: max(0, w_gate_i . x + b_i) * (w_up_i . x)
//           squared ReLU: h = max(0, w_up_i . x + b_i)^2
//           h[b] = 0 where token b's bit is 0
//         -> h exchange (one tagged word per neuron and token)
//   down  block c owns a slice of the d output columns.  While F runs, its threads copy
//         their slice of every active neuron's down row into shared memory (cp.async);
//         then y[slice] = sum over the active neurons of h_i * W_down[i][slice], in a fixed
//         order, and v = x + y with the slice's sum and sum of squares -> v exchange
//   glue  x' = (v - mean(v)) / sqrt(var(v) + 1e-6) from every slice's v and moments,
//         rounded to the activation dtype
// The down projection is column-owned: a block reads only its slice of each active down
// row, so nothing like a d-long partial sum per block is ever exchanged; the exchanges
// carry r values (u), f/32 bit words (mask), one value per active neuron (h) and d
// values (v) per token.
// Mask words (predict output, trace) are OR-ed in by the owner blocks of their bits.
// Cross-block exchanges use 64-bit words {tag, value}: a reader polls the words
// themselves until every tag matches, so data and completion arrive together and no grid
// barrier is needed.  Tags are unique per launch (a device epoch advanced by the last
// block out), per layer and per exchange.  Every sum runs in a fixed order, so results
// are bitwise reproducible.
#include <cuda_fp16.h>
#include <algorithm>
#include <cstdint>

#include "pi_internal.h"
#include "pi_ptx.cuh"
#include "pi_rowmath.cuh"

namespace pi {

namespace {

constexpr float kNormEps = 1e-6f;
constexpr int kRedBar = 1;          // named barrier id among consumers
constexpr int kItems = 32;          // ring items in flight (mbarrier pairs)
constexpr uint32_t kSleepNs = 20000;  // suspend hint of blocking mbarrier waits (wakes on completion)
constexpr int kHr = 48;             // F h slots: more than kItems, so a slot is free before its reuse
constexpr int kMaxDch = 1024;       // entries per down chunk

enum Exchange : int { EX_U = 0, EX_M = 1, EX_H = 2, EX_V = 3 };

struct Smem {
  uint64_t full[kItems];
  uint64_t empty[kItems];
  uint64_t list_ready;          // the kept part of the block's list is in place
  uint64_t list2_ready;         // the whole list is in place
  int abort_flag;
  int nlist_a;                  // records of the kept part of the list
  int nlist;
  int count;                    // own active neurons of the layer (union over tokens)
  uint32_t item_pos[kItems];    // producer bookkeeping of items in flight
  uint32_t item_size[kItems];
  float gmean[4];               // glue: mean and standard deviation of v per token
  float gsd[4];
  float red[2][kConsumerWarps][16];   // block reductions: warp partials (double-buffered)
  int hcnt[kHr];                // F: warps of the record's group that posted partials
  float hpart[kHr][16];         // [warp of the record's group][token][gate/up]
  int32_t list[kMaxList];       // the neurons this block dots, kept ones first
  int32_t list_ent[kMaxList];   // their positions in the layer's entry order (h word index)
  uint8_t list_bits[kMaxList];
  uint8_t own_bits[kMaxOwn];
  int32_t cnt[kMaxGrid];        // union active count of every block's own neurons
  int32_t pre[kMaxGrid + 1];    // exclusive prefix of cnt: entries in owner-major order
  int32_t xpre[kMaxGrid + 1];   // exclusive prefix of the blocks' excess over the target
  int32_t bal[4];               // target, this block's deficit start, total excess
  int32_t wsum[3][kConsumerWarps];   // per-warp partials of block scans
};

// Diagnostics: SM cycle (or global ns) stamps at phase boundaries, [block][layer][slot].
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
__device__ __forceinline__ void st_tag_u(uint64_t* p, uint32_t v, uint32_t tag) {
  asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" ::"l"(p), "l"(tagged(v, tag)) : "memory");
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

__device__ __forceinline__ uint32_t lds_u32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}

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
// Release an item: the 16 consumer warps owe 16 arrivals per item; a warp that stands
// for `cnt` of them arrives with that count.
__device__ __forceinline__ void ring_release_item(uint32_t item, Smem& sm, uint32_t cnt = 1) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) {
    if (cnt == 1) mbar_arrive(&sm.empty[item % kItems]);
    else mbar_arrive_cnt(&sm.empty[item % kItems], cnt);
  }
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
template <int FAM, typename XT>
__device__ __forceinline__ float xs_val(const XT* xs, int idx) {
  if constexpr (FAM == FAM_F32) return xs[idx];
  else return __half2float(xs[idx]);
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

// Elements of one 16-byte down unit: 4 fp32, 8 fp16, or the 32 weights of a Q4_0 block.
__host__ __device__ constexpr int down_unit_elems(int fam) { return fam == FAM_F32 ? 4 : fam == FAM_F16 ? 8 : 32; }

// Position of the k-th (from 0) set bit of u; u has more than k set bits.
__device__ __forceinline__ int select_bit(uint32_t u, int k) {
  int pos = 0, n = __popc(u & 0xFFFFu);
  if (k >= n) { k -= n; u >>= 16; pos += 16; }
  n = __popc(u & 0xFFu);
  if (k >= n) { k -= n; u >>= 8; pos += 8; }
  n = __popc(u & 0xFu);
  if (k >= n) { k -= n; u >>= 4; pos += 4; }
  n = __popc(u & 0x3u);
  if (k >= n) { k -= n; u >>= 2; pos += 2; }
  if (k >= (int)(u & 1u)) pos += 1;
  return pos;
}

// Exclusive prefix sums over the consumer threads of K values per thread (thread order),
// with the totals.  Integer sums: the result is exact.
template <int K>
__device__ __forceinline__ void block_excl_scan(const int (&v)[K], int (&excl)[K], int (&tot)[K], Smem& sm, int warp,
                                                int lane) {
  int incl[K];
#pragma unroll
  for (int k = 0; k < K; ++k) {
    incl[k] = v[k];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int x = __shfl_up_sync(0xffffffffu, incl[k], o);
      if (lane >= o) incl[k] += x;
    }
    if (lane == 31) sm.wsum[k][warp] = incl[k];
  }
  named_bar_sync(kRedBar, kConsumerThreads);
#pragma unroll
  for (int k = 0; k < K; ++k) {
    int off = 0, total = 0;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) {
      const int s = sm.wsum[k][w];
      if (w < warp) off += s;
      total += s;
    }
    excl[k] = off + incl[k] - v[k];
    tot[k] = total;
  }
  named_bar_sync(kRedBar, kConsumerThreads);   // sm.wsum is free again
}

// Union over the tokens of block o's own bit word w (ob: [G][NB][nw]).
template <int NB>
__device__ __forceinline__ uint32_t union_word(const uint32_t* ob, int o, int w, int nw) {
  uint32_t u = 0;
#pragma unroll
  for (int b = 0; b < NB; ++b) u |= ob[((size_t)o * NB + b) * nw + w];
  return u;
}

// Own index m of the k-th active neuron of block o, from the union of its bit words.
template <int NB>
__device__ __forceinline__ int owner_select(const uint32_t* ob, int o, int k, int nw) {
  for (int w = 0; w < nw; ++w) {
    const uint32_t u = union_word<NB>(ob, o, w, nw);
    const int n = __popc(u);
    if (k < n) return 32 * w + select_bit(u, k);
    k -= n;
  }
  return -1;   // unreachable with consistent counts
}

template <int NB>
__device__ __forceinline__ uint32_t owner_token_bits(const uint32_t* ob, int o, int m, int nw) {
  uint32_t bits = 0;
#pragma unroll
  for (int b = 0; b < NB; ++b) bits |= ((ob[((size_t)o * NB + b) * nw + (m >> 5)] >> (m & 31)) & 1u) << b;
  return bits;
}

// ------------------------------------------------------------------ gate/up dots
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
#pragma unroll 4
  for (int q = q0; q < nunits; q += qs) {
    uint32_t xu[NB][XW];
    lds_x_unit<FAM, NB>(xs, p.d, q, xu);
    unit_dot<FAM, NB>(up, p.d, q, xu, au);
    if constexpr (ACT == PI_REGLU) unit_dot<FAM, NB>(gate, p.d, q, xu, ag);
  }
}

// ------------------------------------------------------------------ down units
// acc[b][e] += h[b] * (element e of a 16-byte down unit at shared address a); Q4_0 units
// are whole 32-weight blocks whose fp16 scale is `sc`.
template <int FAM, int NB>
__device__ __forceinline__ void down_unit_fma(uint32_t a, float sc, const float (&h)[NB],
                                              float (&acc)[NB][down_unit_elems(FAM)]) {
  if constexpr (FAM == FAM_F32) {
    const float4 w = u4f(lds128(a));
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      acc[b][0] = fmaf(h[b], w.x, acc[b][0]); acc[b][1] = fmaf(h[b], w.y, acc[b][1]);
      acc[b][2] = fmaf(h[b], w.z, acc[b][2]); acc[b][3] = fmaf(h[b], w.w, acc[b][3]);
    }
  } else if constexpr (FAM == FAM_F16) {
    float w[8];
    widen8(lds128(a), w);
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[b][e] = fmaf(h[b], w[e], acc[b][e]);
  } else {
    // byte j of the block: element j in its low nibble, element j + 16 in its high one
    const uint4 nb = lds128(a);
    const uint32_t wv[4] = {nb.x, nb.y, nb.z, nb.w};
    float hs[NB];
#pragma unroll
    for (int b = 0; b < NB; ++b) hs[b] = h[b] * sc;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const uint32_t lo = wv[m] & 0x0F0F0F0Fu, hi = (wv[m] >> 4) & 0x0F0F0F0Fu;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float cl = q4_val(lo, k), ch = q4_val(hi, k);
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          acc[b][4 * m + k] = fmaf(hs[b], cl, acc[b][4 * m + k]);
          acc[b][16 + 4 * m + k] = fmaf(hs[b], ch, acc[b][16 + 4 * m + k]);
        }
      }
    }
  }
}

// ------------------------------------------------------------------ the kernel
template <int FAM, int ACT, int NB, int NU>
__global__ void __launch_bounds__(kThreads, 1) fused_kernel(const FusedParams p) {
  constexpr int UE = Fam<FAM>::UE;
  constexpr int XW = Fam<FAM>::XW;
  constexpr int PB = Fam<FAM>::PB;
  constexpr int PE = down_unit_elems(FAM);
  using XT = typename Fam<FAM>::X;
  extern __shared__ __align__(128) uint8_t dsmem[];
  Smem& sm = *reinterpret_cast<Smem*>(dsmem);
  uint8_t* ring_base = dsmem + p.off_ring;
  XT* xs = reinterpret_cast<XT*>(dsmem + p.off_xs);                  // [NB][d] current input
  float* u_s = reinterpret_cast<float*>(dsmem + p.off_us);           // [NB][r]
  uint32_t* ob = reinterpret_cast<uint32_t*>(dsmem + p.off_ob);      // [G][NB][nw] every block's own bits
  int32_t* dlist = reinterpret_cast<int32_t*>(dsmem + p.off_dlist);  // [2][dch] neuron of each chunk entry
  float* dred = reinterpret_cast<float*>(dsmem + p.off_dred);        // down reduction / v slice / moments
  const uint32_t dbuf_u = smem_u32(dsmem + p.off_dbuf);              // [2][dch][pmax] 16-byte down units
  const uint32_t dsc_u = smem_u32(dsmem + p.off_dsc);                // Q4_0: [2][dch][pmax] scale words

  const int c = blockIdx.x, G = gridDim.x;
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const bool do_pred = p.mode & MODE_PREDICT, do_ffn = p.mode & MODE_FFN, do_glue = p.mode & MODE_GLUE;
  const int d = p.d, f = p.f, B = p.B;
  const int nown = (c < f) ? (f - c + G - 1) / G : 0;
  const int nunits = d / UE;
  const int words = f / 32;
  const int nw = p.nw;
  const int dch = p.dch, pmax = p.pmax;
  // the block's down slice: 16-byte units [cu0, cu1) of every down row.  In the down
  // phase lpe consecutive lanes take one entry (lane % lpe is the unit, so the lanes of an
  // entry read one contiguous piece of its row) and a warp takes epw entries per pass:
  // this lane handles unit dw of the entries de0, de0 + dstep, ... of every chunk
  const int cu0 = (int)((long long)c * p.dunits / G), cu1 = (int)((long long)(c + 1) * p.dunits / G);
  const int npc = cu1 - cu0;
  const int lpe = npc <= 1 ? 1 : npc <= 2 ? 2 : npc <= 4 ? 4 : npc <= 8 ? 8 : 16;
  const int epw = 32 / lpe;
  const int dw = (lane % lpe) < npc ? lane % lpe : -1;
  const int de0 = warp * epw + lane / lpe;
  const int dstep = kConsumerWarps * epw;
  const int col0 = cu0 * PE, ncol = npc * PE;
  const uint32_t epoch = *reinterpret_cast<volatile const uint32_t*>(p.bar + 2);

  if (t == 0) {
    for (int s = 0; s < kItems; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], kConsumerWarps);
    }
    mbar_init(&sm.list_ready, 1);
    mbar_init(&sm.list2_ready, 1);
    for (int s = 0; s < kHr; ++s) sm.hcnt[s] = 0;
    sm.abort_flag = 0;
    sm.nlist = 0;
    mbar_fence_init();
  }
  __syncthreads();

  // ================================================================ producer warp
  if (warp == kConsumerWarps) {
    if (lane == 0) {
      uint32_t head = 0, issued = 0, oldest = 0;
      uint32_t landed = 0, inflight = 0;   // items known to have landed; bytes issued beyond them
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
      // Keep at most inflight_budget bytes of this block's copies in flight (one item at
      // least): more would not raise the block's share of HBM bandwidth, only the queueing
      // delay every latency-critical exchange word waits behind.
      auto throttle = [&](uint32_t size) -> bool {
        while (landed < issued && inflight + size > (uint32_t)p.inflight_budget) {
          uint64_t* fb = &sm.full[landed % kItems];
          const uint32_t par = (landed / kItems) & 1u;
          if (!mbar_try_wait(fb, par)) {
            const uint64_t t0 = wait_start();
            while (!mbar_try_wait_sleep(fb, par, kSleepNs)) {
              if (aborted(sm)) return false;
              if (timed_out(t0, p.wait_cycles)) { set_abort(sm, p.err, DEV_ERR_RING_TIMEOUT); return false; }
            }
          }
          inflight -= sm.item_size[landed % kItems];
          ++landed;
        }
        return !aborted(sm);
      };
      auto begin_item = [&](uint32_t size, uint8_t*& dst, uint64_t*& fb) -> bool {
        uint32_t pos;
        if (!throttle(size)) return false;
        if (!reserve(size, pos)) return false;
        // released items have landed: account for them before their slot is reused
        while (landed < oldest) {
          inflight -= sm.item_size[landed % kItems];
          ++landed;
        }
        inflight += size;
        sm.item_pos[issued % kItems] = pos;
        sm.item_size[issued % kItems] = size;
        dst = ring_base + pos;
        fb = &sm.full[issued % kItems];
        mbar_arrive_expect_tx(fb, size);
        ++issued;
        return true;
      };
      auto wait_list = [&](uint64_t* bar, uint32_t par) -> bool {
        const uint64_t t0 = wait_start();
        while (!mbar_try_wait_sleep(bar, par, kSleepNs)) {
          if (aborted(sm)) return false;
          if (timed_out(t0, p.wait_cycles)) { set_abort(sm, p.err, DEV_ERR_RING_TIMEOUT); return false; }
        }
        return true;
      };
      bool ok = true;
      for (int l = 0; l < p.L && ok; ++l) {
        const LayerDev Ld = p.layers[l];
        const int r = Ld.r;
        const int k0 = (int)((long long)c * r / G), k1 = (int)((long long)(c + 1) * r / G);
        const int p2_stride = p2_stride_of(r, PB);
        const int p2_rows = max(1, min(p.nown_max, p.p2_item_bytes / p2_stride));
        uint8_t* dst;
        uint64_t* fb;
        if (do_pred) {
          for (int k = k0; k < k1 && ok; k += p.p1_rows_per_item) {
            const int n = min(p.p1_rows_per_item, k1 - k);
            const uint32_t bytes = (uint32_t)n * p.p1_row;
            if (!(ok = begin_item(bytes, dst, fb))) break;
            bulk_g2s(dst, Ld.p1t + (size_t)k * p.p1_row, bytes, fb);
          }
          const uint8_t* own = Ld.p2o + (size_t)c * p.nown_max * p2_stride;
          for (int m = 0; m < nown && ok; m += p2_rows) {
            const int n = min(p2_rows, nown - m);
            const uint32_t bytes = (uint32_t)n * p2_stride;
            if (!(ok = begin_item(bytes, dst, fb))) break;
            bulk_g2s(dst, own + (size_t)m * p2_stride, bytes, fb);
          }
        }
        if (do_ffn && ok) {
          pstamp(p, l, 20);
          ok = wait_list(&sm.list_ready, (uint32_t)(l & 1));
          pstamp(p, l, 21);
          // The kept part of the list is known before the mask exchange ends, the rest
          // after it.
          const int na = ok ? sm.nlist_a : 0;
          int e = 0;
          for (; e < na && ok; ++e) {
            if (!(ok = begin_item((uint32_t)p.rec_stride, dst, fb))) break;
            bulk_g2s(dst, Ld.rec + (size_t)sm.list[e] * p.rec_stride, (uint32_t)p.rec_stride, fb);
          }
          if (ok) ok = wait_list(&sm.list2_ready, (uint32_t)(l & 1));
          const int n = ok ? sm.nlist : 0;
          for (; e < n && ok; ++e) {
            if (!(ok = begin_item((uint32_t)p.rec_stride, dst, fb))) break;
            bulk_g2s(dst, Ld.rec + (size_t)sm.list[e] * p.rec_stride, (uint32_t)p.rec_stride, fb);
          }
          pstamp(p, l, 22);
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
  // the trace's layer-0 input: every block writes its own columns
  if (do_glue && p.trace.x)
    for (int q = t; q < B * ncol; q += kConsumerThreads) {
      const size_t idx = (size_t)(q / ncol) * d + col0 + q % ncol;
      store_act<FAM>(p.trace.x, idx, load_act<FAM>(p.x_in, idx));
    }
  named_bar_sync(kRedBar, kConsumerThreads);

  int redbuf = 0;     // which half of sm.red the next block reduction uses
  uint32_t fseq = 0;  // F records of earlier layers (h slot of record e: (fseq + e) % kHr)
  for (int l = 0; l < p.L; ++l) {
    const LayerDev Ld = p.layers[l];
    const int r = Ld.r;
    const int k0 = (int)((long long)c * r / G), k1 = (int)((long long)(c + 1) * r / G);
    const int p2_stride = p2_stride_of(r, PB);
    const int p2_rows = max(1, min(p.nown_max, p.p2_item_bytes / p2_stride));
    const uint32_t tag_u = tag_of(epoch, l, EX_U), tag_m = tag_of(epoch, l, EX_M), tag_h = tag_of(epoch, l, EX_H),
                   tag_v = tag_of(epoch, l, EX_V);
    int nlist = 0;      // records this block dots
    int ntotal = 0;     // active entries of the layer (the down list)
    bool signaled_a = false;
    stamp(p, l, 0);
    // this layer's x units, fp32, in registers for P-a
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
      for (int m0 = 0; m0 < nown; m0 += p2_rows) {
        const int n = min(p2_rows, nown - m0);
        const uint8_t* item = ring_next(ring, (uint32_t)n * p2_stride);
        const long long wt0 = diag_clock(p);
        ring_wait_item_warp(ring.item, sm, p);
        pb_wait += diag_clock(p) - wt0;
        for (int mb = warp * 8; mb < n; mb += kConsumerWarps * 8) {
          uint32_t rows[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) rows[i] = smem_u32(item) + (uint32_t)(min(mb + i, n - 1) * p2_stride);   // past n: repeats, unused
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
      stamp(p, l, 3);
      stamp_val(p, l, 18, pb_wait);
      if (!do_ffn) break;   // predictor only

      // ---------------------------------------------------------- own active list + bits
      // Block c's own neurons are i = c + m*G in ascending m.  Warp w < nw also publishes
      // word w of the block's own bits for every token (the mask exchange).
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
      for (int w = warp; w < nw; w += kConsumerWarps) {
        const int m = 32 * w + lane;
        const uint32_t tb = (m < nown) ? sm.own_bits[m] : 0u;
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          const uint32_t word = __ballot_sync(0xffffffffu, (tb >> b) & 1u);
          if (lane == 0 && b < B) st_tag_u(p.mx + ((size_t)c * 4 + b) * kMaxOwnWords + w, word, tag_m);
        }
      }
      named_bar_sync(kRedBar, kConsumerThreads);
      const int n_own = sm.count;
      const int floor = Ld.keep_floor;
      // the kept part (own records every block keeps whatever the counts) goes to the
      // producer now, so its copies run during the mask exchange
      if (t == 0) {
        sm.nlist_a = min(n_own, floor);
        mbar_arrive(&sm.list_ready);
      }
      signaled_a = true;
      stamp(p, l, 4);

      // ---------------------------------------------------------- mask exchange
      {
        const int per = B * nw;
        const int nq = G * per;
        constexpr int MQ = 16;
        if (NB > B)
          for (int q = t; q < G * NB * nw; q += kConsumerThreads)
            if ((q / nw) % NB >= B) ob[q] = 0u;
        for (int base = 0; base < nq; base += MQ * kConsumerThreads) {
          uint64_t w[MQ];
          uint32_t need = 0;
#pragma unroll
          for (int i = 0; i < MQ; ++i) {
            w[i] = 0;
            if (base + t + i * kConsumerThreads < nq) need |= 1u << i;
          }
          bool started = false;
          uint64_t tp0 = 0;
          while (need) {
#pragma unroll
            for (int i = 0; i < MQ; ++i)
              if (need >> i & 1u) {
                const int q = base + t + i * kConsumerThreads;
                const int o = q / per, rem = q % per;
                w[i] = ld_tag(p.mx + ((size_t)o * 4 + rem / nw) * kMaxOwnWords + rem % nw);
              }
#pragma unroll
            for (int i = 0; i < MQ; ++i)
              if ((need >> i & 1u) && tag_ok(w[i], tag_m)) need &= ~(1u << i);
            if (!need || aborted(sm)) break;
            if (!started) { tp0 = wait_start(); started = true; }
            else if (timed_out(tp0, p.wait_cycles)) { set_abort(sm, p.err, DEV_ERR_GRID_TIMEOUT); break; }
            if (p.poll_ns) __nanosleep(p.poll_ns);
          }
#pragma unroll
          for (int i = 0; i < MQ; ++i) {
            const int q = base + t + i * kConsumerThreads;
            if (q < nq) {
              // only bits of neurons the owner has can be set (a word of an aborted
              // exchange may hold anything)
              const int o = q / per, rem = q % per, ww = rem % nw;
              const int nown_o = (o < f) ? (f - o + G - 1) / G : 0;
              const int nv = min(32, max(0, nown_o - 32 * ww));
              const uint32_t valid = nv >= 32 ? 0xFFFFFFFFu : ((1u << nv) - 1u);
              ob[((size_t)o * NB + rem / nw) * nw + ww] = (uint32_t)w[i] & valid;
            }
          }
        }
      }
      named_bar_sync(kRedBar, kConsumerThreads);
      stamp(p, l, 5);
      if (t < G) {
        int n = 0;
        for (int w = 0; w < nw; ++w) n += __popc(union_word<NB>(ob, t, w, nw));
        sm.cnt[t] = n;
      }
      named_bar_sync(kRedBar, kConsumerThreads);

      // ---------------------------------------------------------- balanced assignment
      // N = the sum of the counts; target T = max(ceil(N / G), floor).  Block c keeps its
      // first min(n_c, T) own entries; the entries past T of the blocks above the target,
      // in (block, position) order, fill the blocks below it in block order.  Every block
      // derives the same assignment from the counts alone.
      {
        const int cv = (t < G) ? sm.cnt[t] : 0;
        int v1[1] = {cv}, e1[1], s1[1];
        block_excl_scan<1>(v1, e1, s1, sm, warp, lane);
        const int N = s1[0];
        const int T = max((N + G - 1) / G, floor);
        int v2[2] = {(t < G) ? max(0, cv - T) : 0, (t < G) ? max(0, T - cv) : 0}, e2[2], s2[2];
        block_excl_scan<2>(v2, e2, s2, sm, warp, lane);
        if (t < G) {
          sm.pre[t] = e1[0];
          sm.xpre[t] = e2[0];
        }
        if (t == c) sm.bal[1] = e2[1];
        if (t == 0) {
          sm.pre[G] = N;
          sm.xpre[G] = s2[0];
          sm.bal[0] = T;
          sm.bal[2] = s2[0];
        }
        named_bar_sync(kRedBar, kConsumerThreads);
        const int dstart = sm.bal[1], xtotal = sm.bal[2];
        const int keep = min(n_own, T);
        const int deficit = max(0, T - n_own);
        const int ntake = max(0, min(dstart + deficit, xtotal) - dstart);
        for (int q = t; q < keep; q += kConsumerThreads) sm.list_ent[q] = sm.pre[c] + q;
        for (int q = t; q < ntake; q += kConsumerThreads) {
          const int x = dstart + q;
          int lo = 0, hi = G;   // owner o: xpre[o] <= x < xpre[o + 1]
          while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (sm.xpre[mid] <= x) lo = mid;
            else hi = mid;
          }
          const int k = T + (x - sm.xpre[lo]);
          const int m = owner_select<NB>(ob, lo, k, nw);
          const int i = lo + max(m, 0) * G;
          sm.list[keep + q] = i < f ? i : 0;
          sm.list_ent[keep + q] = sm.pre[lo] + k;
          sm.list_bits[keep + q] = (uint8_t)owner_token_bits<NB>(ob, lo, max(m, 0), nw);
        }
        nlist = keep + ntake;
        ntotal = N;
      }
      if (t == 0) {
        atomicAdd(p.active_total, (unsigned long long)nlist);
        if (p.layer_count) atomicAdd(p.layer_count + l, nlist);
      }
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
        sm.list_ent[e] = a0 + e;
        sm.list_bits[e] = (uint8_t)bits;
      }
      if (t == 0) atomicAdd(p.active_total, (unsigned long long)nlist);
      ntotal = cnt;
    }

    named_bar_sync(kRedBar, kConsumerThreads);
    if (t == 0) {
      if (!signaled_a) {
        sm.nlist_a = nlist;
        mbar_arrive(&sm.list_ready);
      }
      sm.nlist = nlist;
      mbar_arrive(&sm.list2_ready);
    }
    stamp(p, l, 6);
    stamp_val(p, l, 14, nlist);
    stamp_val(p, l, 15, ntotal);

    // ------------------------------------------------------------ down list and copies
    // Chunk k holds the active entries [k*dch, (k+1)*dch) of the layer in owner-major
    // order (the caller's order for a given list); dlist half k%2 holds their neuron ids
    // and dbuf half k%2 their units [cu0, cu1).  Each thread copies, and later reads,
    // only its own slots, so its cp.async groups alone order the copies and the reads.
    const int nchunks = (ntotal + dch - 1) / dch;
    const uint8_t* dn = Ld.rec + p.dn_off;
    auto build_dlist = [&](int k) {
      const int lo = k * dch, hi = min(ntotal, lo + dch);
      int32_t* dl = dlist + (k & 1) * dch;
      if (do_pred) {
        for (int o = t; o < G; o += kConsumerThreads) {
          const int e0 = sm.pre[o], e1 = e0 + sm.cnt[o];
          if (e1 <= lo || e0 >= hi) continue;
          int e = e0;
          for (int w = 0; w < nw && e < hi; ++w) {
            uint32_t u = union_word<NB>(ob, o, w, nw);
            const int n = __popc(u);
            if (e + n <= lo) { e += n; continue; }
            while (u && e < hi) {
              const int bit = __ffs(u) - 1;
              u &= u - 1;
              if (e >= lo) dl[e - lo] = o + (32 * w + bit) * G;
              ++e;
            }
          }
        }
      } else {
        for (int e = lo + t; e < hi; e += kConsumerThreads) {
          int i = __ldg(p.idx_in + e);
          if (i < 0 || i >= f) i = 0;   // reported above
          dl[e - lo] = i;
        }
      }
    };
    auto issue_down = [&](int k) {
      if (dw < 0) return;
      const int lo = k * dch, hi = min(ntotal, lo + dch);
      const int32_t* dl = dlist + (k & 1) * dch;
      const int half = (k & 1) * dch;
      for (int e = lo + de0; e < hi; e += dstep) {
        const int i = dl[e - lo];
        const uint8_t* row = dn + (size_t)i * p.dn_stride;
        const uint32_t slot = (uint32_t)((half + e - lo) * pmax + dw);
        cpa16(dbuf_u + slot * 16u, row + (size_t)(cu0 + dw) * 16);
        if constexpr (FAM == FAM_Q4) cpa4(dsc_u + slot * 4u, row + (size_t)(d >> 1) + (size_t)((cu0 + dw) >> 1) * 4);
      }
    };
    build_dlist(0);
    if (nchunks > 1) build_dlist(1);
    named_bar_sync(kRedBar, kConsumerThreads);
    issue_down(0);
    cpa_commit();
    if (nchunks > 1) issue_down(1);
    cpa_commit();
    stamp(p, l, 7);

    // ------------------------------------------------------------ F: records -> h
    // The 16 consumer warps form groups of KG; group g dots records g, g + 16/KG, ...
    // with no block barrier: each warp of the group waits for the record to land, dots
    // its slice of the units with x from shared memory, reduces across its lanes and
    // posts its partial sums in the record's h slot.  The last warp of the group to post
    // sums the group's partials in a fixed order, forms h and publishes it.
    {
      constexpr int NV = (ACT == PI_REGLU) ? 2 : 1;
      constexpr int NVAL = NB * NV;                 // partial sums per warp and record
      constexpr int V = pow2_ceil(NVAL);
      constexpr int LG = log2_exact(V);
      constexpr int KG = f_group_warps(FAM, ACT, NB);
      constexpr int NG = kConsumerWarps / KG;       // records dotted at once
      static_assert(KG * NVAL <= 16 && kConsumerWarps % KG == 0, "h slot layout");
      const uint32_t base = smem_u32(ring.base), xsa = smem_u32(xs);
      const uint32_t item0 = ring.item;
      const int kq = warp % KG;
      long long f_wait = 0;   // diagnostics: cycles warp 0 waits for records
      uint32_t hd = ring.head;   // ring head before record id (dot cursor)
      int id = 0;
      for (int e = warp / KG; e < nlist; e += NG) {
        uint32_t pos = 0;
        for (; id <= e; ++id) pos = ring_place(hd, (uint32_t)p.rec_stride, ring.cap);
        const long long wt0 = diag_clock(p);
        ring_wait_item_warp(item0 + e, sm, p);
        f_wait += diag_clock(p) - wt0;
        if (e == 0) stamp(p, l, 8);
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
        const uint32_t s = (fseq + (uint32_t)e) % kHr;
        if ((lane & ((32 >> LG) - 1)) == 0 && (lane >> (5 - LG)) < NVAL) sm.hpart[s][kq * NVAL + (lane >> (5 - LG))] = sw;
        const float bi = lds_f32(base + pos + (uint32_t)p.bias_off);
        __syncwarp();
        if (lane == 0) {
          __threadfence_block();
          if (atomicAdd(&sm.hcnt[s], 1) == KG - 1) {
            __threadfence_block();
            const volatile float* hp = sm.hpart[s];
            const int ent = sm.list_ent[e];
            const uint32_t bits = sm.list_bits[e];
#pragma unroll
            for (int b = 0; b < NB; ++b) {
              if (b < B) {
                float su = hp[b * NV], sg = 0.f;
#pragma unroll
                for (int k = 1; k < KG; ++k) su += hp[k * NVAL + b * NV];
                if constexpr (ACT == PI_REGLU) {
                  sg = hp[b * NV + 1];
#pragma unroll
                  for (int k = 1; k < KG; ++k) sg += hp[k * NVAL + b * NV + 1];
                }
                float a;
                if constexpr (ACT == PI_REGLU) {
                  a = fmaxf(sg + bi, 0.f) * su;
                } else {
                  a = fmaxf(su + bi, 0.f);
                  if (p.act_square) a *= a;
                }
                st_tag(p.hx + (size_t)ent * B + b, ((bits >> b) & 1u) ? a : 0.f, tag_h);
              }
            }
            sm.hcnt[s] = 0;
          }
        }
        ring_release_item(item0 + e, sm, (uint32_t)(kConsumerWarps / KG));
      }
      for (int q = 0; q < nlist; ++q) ring_place(ring.head, (uint32_t)p.rec_stride, ring.cap);
      ring.item = item0 + (uint32_t)nlist;
      fseq += (uint32_t)nlist;
      stamp_val(p, l, 19, f_wait);
    }
    stamp(p, l, 9);

    // ------------------------------------------------------------ down: y of the slice
    float acc[NB][PE];
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
      for (int e = 0; e < PE; ++e) acc[b][e] = 0.f;
    long long h_wait = 0;   // diagnostics: cycles thread 0 polls for h
    for (int k = 0; k < nchunks; ++k) {
      cpa_wait_but_newest();   // this thread's copies of chunk k have landed
      if (dw >= 0) {
        const int lo = k * dch, hi = min(ntotal, lo + dch);
        const int32_t* dl = dlist + (k & 1) * dch;
        const int half = (k & 1) * dch;
        constexpr int HB = NB == 1 ? 8 : NB == 2 ? 4 : 2;   // entries whose h words one polling round reads
        for (int eb = lo + de0; eb < hi; eb += HB * dstep) {
          uint64_t hw[HB][NB];
          uint32_t need = 0;
#pragma unroll
          for (int q = 0; q < HB; ++q)
#pragma unroll
            for (int b = 0; b < NB; ++b) {
              hw[q][b] = 0;
              if (eb + q * dstep < hi && b < B) need |= 1u << (q * NB + b);
            }
          const long long wt0 = diag_clock(p);
          bool started = false;
          uint64_t tp0 = 0;
          while (need) {
#pragma unroll
            for (int q = 0; q < HB; ++q)
#pragma unroll
              for (int b = 0; b < NB; ++b)
                if (need >> (q * NB + b) & 1u) hw[q][b] = ld_tag(p.hx + (size_t)(eb + q * dstep) * B + b);
#pragma unroll
            for (int q = 0; q < HB; ++q)
#pragma unroll
              for (int b = 0; b < NB; ++b)
                if ((need >> (q * NB + b) & 1u) && tag_ok(hw[q][b], tag_h)) need &= ~(1u << (q * NB + b));
            if (!need || aborted(sm)) break;
            if (!started) { tp0 = wait_start(); started = true; }
            else if (timed_out(tp0, p.wait_cycles)) { set_abort(sm, p.err, DEV_ERR_GRID_TIMEOUT); break; }
            if (p.poll_ns) __nanosleep(p.poll_ns);
          }
          h_wait += diag_clock(p) - wt0;
#pragma unroll
          for (int q = 0; q < HB; ++q) {
            const int e = eb + q * dstep;
            if (e < hi) {
              float h[NB];
#pragma unroll
              for (int b = 0; b < NB; ++b) h[b] = b < B ? tag_val(hw[q][b]) : 0.f;
              const uint32_t slot = (uint32_t)((half + e - lo) * pmax + dw);
              float sc = 0.f;
              if constexpr (FAM == FAM_Q4) {
                const uint32_t sw = lds_u32(dsc_u + slot * 4u);
                sc = __half2float(__ushort_as_half((unsigned short)(((cu0 + dw) & 1) ? (sw >> 16) : (sw & 0xFFFFu))));
              }
              down_unit_fma<FAM, NB>(dbuf_u + slot * 16u, sc, h, acc);
            }
          }
        }
      }
      if (k + 2 < nchunks) {
        named_bar_sync(kRedBar, kConsumerThreads);   // every thread is done with dlist half k%2
        build_dlist(k + 2);
        named_bar_sync(kRedBar, kConsumerThreads);
        issue_down(k + 2);
      }
      cpa_commit();
    }
    cpa_wait_all();
    stamp_val(p, l, 17, h_wait);
    stamp(p, l, 10);

    // ------------------------------------------------------------ slice reduction
    // The lanes of a warp that hold the same unit are summed by a butterfly over the lane
    // bits above the unit bits; then the warps are summed in ascending order.
    {
      constexpr int V = NB * PE;
#pragma unroll
      for (int b = 0; b < NB; ++b)
#pragma unroll
        for (int e = 0; e < PE; ++e) {
          float v = acc[b][e];
          for (int o = lpe; o < 32; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
          acc[b][e] = v;
        }
      if (lane < lpe && dw >= 0) {
#pragma unroll
        for (int b = 0; b < NB; ++b)
#pragma unroll
          for (int e = 0; e < PE; ++e) dred[(warp * pmax + dw) * V + b * PE + e] = acc[b][e];
      }
      named_bar_sync(kRedBar, kConsumerThreads);
      float* vsl = dred + kConsumerWarps * pmax * V;   // [NB][ncol] v of the slice
      if (t < B * ncol) {
        const int b = t / ncol, q = t % ncol, w = q / PE, e = q % PE;
        float y = 0.f;
        for (int k = 0; k < kConsumerWarps; ++k) y += dred[(k * pmax + w) * V + b * PE + e];
        const int col = col0 + q;
        if (do_glue) {
          const float v = xs_val<FAM>(xs, b * d + col) + y;
          vsl[b * ncol + q] = v;
          st_tag(p.vx + (size_t)b * d + col, v, tag_v);
          if (p.trace.y) p.trace.y[((size_t)l * B + b) * d + col] = y;
        } else {
          p.y_out[(size_t)b * d + col] = y;
        }
      }
      if (!do_glue) break;
      named_bar_sync(kRedBar, kConsumerThreads);
      if (warp < NB) {
        float s = 0.f, s2 = 0.f;
        if (warp < B)
          for (int q = lane; q < ncol; q += 32) {
            const float v = vsl[warp * ncol + q];
            s += v;
            s2 += v * v;
          }
        s = warp_sum(s);
        s2 = warp_sum(s2);
        if (lane == 0 && warp < B) {
          st_tag(p.sx + ((size_t)warp * G + c) * 2, s, tag_v);
          st_tag(p.sx + ((size_t)warp * G + c) * 2 + 1, s2, tag_v);
        }
      }
    }
    stamp(p, l, 11);

    // ------------------------------------------------------------ glue: x' = (v - mean) / sd
    // One polling round reads every v and every slice's (sum, sum of squares).
    {
      const int npairs = B * d / 2;
      const int nmom = 2 * G * B;
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
        uint64_t tp0 = 0;
        while (need | needm) {
#pragma unroll
          for (int k = 0; k < 8; ++k)
            if (need >> k & 1u) ld_tag2(p.vx + 2 * (size_t)(t + k * kConsumerThreads), w0[k], w1[k]);
#pragma unroll
          for (int i = 0; i < MQ; ++i)
            if (needm >> i & 1u) wm[i] = ld_tag(p.sx + t + i * kConsumerThreads);
#pragma unroll
          for (int k = 0; k < 8; ++k)
            if ((need >> k & 1u) && tag_ok(w0[k], tag_v) && tag_ok(w1[k], tag_v)) need &= ~(1u << k);
#pragma unroll
          for (int i = 0; i < MQ; ++i)
            if ((needm >> i & 1u) && tag_ok(wm[i], tag_v)) needm &= ~(1u << i);
          if (!(need | needm) || aborted(sm)) break;
          if (!started) { tp0 = wait_start(); started = true; }
          else if (timed_out(tp0, p.wait_cycles)) { set_abort(sm, p.err, DEV_ERR_GRID_TIMEOUT); break; }
          if (p.poll_ns) __nanosleep(p.poll_ns);
        }
      }
      named_bar_sync(kRedBar, kConsumerThreads);   // nobody reads vsl or xs any more
      stamp(p, l, 12);
      float* mom = dred;                            // [B][G][2]
#pragma unroll
      for (int i = 0; i < MQ; ++i)
        if (t + i * kConsumerThreads < nmom) mom[t + i * kConsumerThreads] = tag_val(wm[i]);
      named_bar_sync(kRedBar, kConsumerThreads);
      if (warp < NB) {
        float s = 0.f, s2 = 0.f;
        if (warp < B)
          for (int cq = lane; cq < G; cq += 32) {
            s += mom[(warp * G + cq) * 2];
            s2 += mom[(warp * G + cq) * 2 + 1];
          }
        const float sum = warp_sum(s);
        s2 = warp_sum(s2);
        if (lane == 0) {
          const float mean = sum / (float)d;
          const float var = fmaxf(s2 / (float)d - mean * mean, 0.f);
          sm.gmean[warp] = mean;
          sm.gsd[warp] = sqrtf(var + kNormEps);
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
        uint64_t tp0 = 0;
        while (need) {
#pragma unroll
          for (int k = 0; k < 8; ++k)
            if (need >> k & 1u) ld_tag2(p.vx + 2 * (size_t)(base + t + k * kConsumerThreads), w0[k], w1[k]);
#pragma unroll
          for (int k = 0; k < 8; ++k)
            if ((need >> k & 1u) && tag_ok(w0[k], tag_v) && tag_ok(w1[k], tag_v)) need &= ~(1u << k);
          if (!need || aborted(sm)) break;
          if (!started) { tp0 = wait_start(); started = true; }
          else if (timed_out(tp0, p.wait_cycles)) { set_abort(sm, p.err, DEV_ERR_GRID_TIMEOUT); break; }
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
      named_bar_sync(kRedBar, kConsumerThreads);
      // every block writes its own columns of the trace and of the output
      if (p.trace.x || l == p.L - 1)
        for (int q = t; q < B * ncol; q += kConsumerThreads) {
          const int b = q / ncol;
          const size_t j = (size_t)b * d + col0 + q % ncol;
          const float xv = xs_val<FAM>(xs, (int)j);
          if (p.trace.x) store_act<FAM>(p.trace.x, (size_t)(l + 1) * B * d + j, xv);
          if (l == p.L - 1) store_act<FAM>(p.x_out, j, xv);
        }
    }
    stamp(p, l, 13);
  }

  // last block out: advance the epoch (new tags for the next launch) and reset the count
  named_bar_sync(kRedBar, kConsumerThreads);
  if (t == 0) {
    __threadfence();
    const uint32_t prev = atomicAdd(p.bar + 1, 1u);
    if (prev == (uint32_t)G - 1) {
      atomicExch(p.bar + 2, next_launch_epoch(epoch));
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
// thread that covers it; a launch takes the smallest count that covers its d, so x in
// registers stays small.
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

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

}  // namespace

bool fused_supported(int family, int B, int d) {
  const int nb = nb_of(B);
  if (nb == 0) return false;
  return d <= d_max_of(family, nb);
}

bool fused_plan_smem(FusedParams& p, int family, size_t budget, size_t& smem_bytes) {
  const int nb = nb_of(p.B);
  if (nb == 0) return false;
  const int G = p.grid;
  const size_t xbytes = family == FAM_F32 ? 4 : 2;
  const int pe = down_unit_elems(family);
  p.nw = (p.nown_max + 31) / 32;
  p.dunits = p.d / pe;
  p.pmax = (p.dunits + G - 1) / G;
  if (p.nw > kMaxOwnWords || p.pmax > kMaxPieces || p.pmax < 1) return false;
  // ring items: whole neuron records; P1^T rows grouped into ~32 KB copies; the block's own
  // P2 rows in copies of up to 48 KB
  const int cap = std::max(p.rec_stride, 32 * 1024);
  p.p1_rows_per_item = std::max(1, cap / p.p1_row);
  p.p2_item_bytes = std::max(cap, 48 * 1024);
  // the largest copy of predictor rows any layer makes: its rows per copy times its stride,
  // at most max(p2_item_bytes, one row of the largest rank)
  const long long max_p2_item = std::max((long long)p.p2_item_bytes, (long long)p.p2_stride);
  const long long max_item = std::max({(long long)p.rec_stride, (long long)p.p1_rows_per_item * p.p1_row,
                                       max_p2_item});
  const size_t dred_floats = std::max((size_t)(kConsumerWarps + 1) * p.pmax * nb * pe, (size_t)nb * G * 2);
  size_t off = round_up(sizeof(Smem), 128);
  const size_t fixed_tail = round_up((size_t)nb * p.d * xbytes, 16) + round_up((size_t)nb * p.r * 4, 16) +
                            round_up((size_t)G * nb * p.nw * 4, 16) + round_up(dred_floats * 4, 16);
  // per chunk entry: its dlist slot and its units (plus a scale word per Q4_0 unit), twice
  const size_t entry_bytes = 2 * (4 + (size_t)p.pmax * 16 + (family == FAM_Q4 ? (size_t)p.pmax * 4 : 0));
  const size_t ring_min = std::max((size_t)112 * 1024, (size_t)(2 * max_item));
  if (budget < off + fixed_tail + ring_min + 64 * entry_bytes + 256) return false;
  size_t dch = (budget - off - fixed_tail - ring_min - 256) / entry_bytes;
  dch = std::min(dch, (size_t)kMaxDch);
  p.dch = (int)dch;
  const size_t down_bytes = round_up(dch * entry_bytes, 128);
  p.ring_bytes = (int)((budget - off - fixed_tail - down_bytes - 256) / 128 * 128);
  if (p.ring_bytes < 2 * max_item || max_item >= (1 << 20)) return false;
  p.off_ring = (int)off;
  off += (size_t)p.ring_bytes;
  p.off_xs = (int)off;
  off += round_up((size_t)nb * p.d * xbytes, 16);
  p.off_us = (int)off;
  off += round_up((size_t)nb * p.r * 4, 16);
  p.off_ob = (int)off;
  off += round_up((size_t)G * nb * p.nw * 4, 16);
  p.off_dred = (int)off;
  off += round_up(dred_floats * 4, 16);
  p.off_dlist = (int)off;
  off += round_up((size_t)2 * dch * 4, 16);
  p.off_dbuf = (int)off;
  off += (size_t)2 * dch * p.pmax * 16;
  p.off_dsc = (int)off;
  off += family == FAM_Q4 ? (size_t)2 * dch * p.pmax * 4 : 0;
  smem_bytes = round_up(off, 128);
  return smem_bytes <= budget;
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
