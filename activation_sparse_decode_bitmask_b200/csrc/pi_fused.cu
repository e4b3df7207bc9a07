// The fused persistent kernel of the activation-sparse FFN decode path.
//
// One block per SM: 16 consumer warps and 1 producer warp.  The producer streams the
// block's predictor rows and the [gate | up | bias] record of every neuron the block dots
// from HBM into a byte ring in shared memory, as bulk copies completing on mbarriers.
// A layer's predictor rows wait until the previous layer's records are dotted, so the
// records have HBM to themselves and the predictor copies fill the exchanges after them.
//
// Per layer, for block c of G (stack mode):
//   P-a   u_k = P1^T[k] . x for the block's rank rows k -> u exchange
//   P-b   logit_i = P2^T[i] . u - t_i for the block's own neurons i = c, c+G, c+2G, ...;
//         bit = logit > 0.  The block lists its own active neurons, publishes its bit
//         words and hands the first na of the list (a floor set from the firing
//         frequencies) to the producer at once.
//   F     warps 0..7 dot records as they land (a group of warps per record):
//           ReLU : h = max(0, w_up_i . x + b_i)    ReGLU: max(0, w_gate_i . x + b_i) * (w_up_i . x)
//           squared ReLU: h = max(0, w_up_i . x + b_i)^2
//           h[b] = 0 where token b's bit is 0
//         -> h exchange: owner o's k-th active neuron publishes h at word o * nown_max + k
//   help  meanwhile warps 8..15 poll every block's bit words, count them, and derive the
//         same balanced assignment in every block: target T = ceil(N / G); a block dots
//         at most max(T, na) of its own records and takes the excess of the blocks above
//         T in block order.  They list the rest of the block's records for the producer
//         and the F warps, build the layer's down list (all N active neurons in owner-major
//         order with their h words) and copy the block's slice of every listed down row
//         into shared memory (cp.async, completing on an mbarrier).  Down-list chunks past
//         the second are built and copied by every consumer thread during the down pass.
//   down  block c owns a slice of the d output columns: once the h words are in,
//         y[slice] = sum over the active neurons of h_i * W_down[i][slice], in a fixed
//         order, and v = x + y with the slice's sum and sum of squares -> v exchange
//         With one token and more active neurons than three down-list chunks hold, the down
//         pass is row-owned instead: each block reads the full down rows of the records it
//         dotted (bulk copies after the records), adds h times its units of each row into
//         registers, publishes its partial y (d words), and sums its column slice over all
//         blocks' partials (small scattered slice copies would limit it otherwise).
//   glue  x' = (v - mean(v)) / sqrt(var(v) + 1e-6) from every slice's v and moments,
//         rounded to the activation dtype
// The down projection is column-owned: a block reads only its slice of each active down
// row, so nothing like a d-long partial sum per block is ever exchanged; the exchanges
// carry r values (u), f/32 bit words (mask), one value per active neuron (h) and d
// values (v) per token.  An own record that its owner dots although a taker dots it too
// publishes the same value twice (both blocks hold the same x and sum in the same order).
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
constexpr int kHr = 48;             // F h slots: more than kItems, so a slot is free before its reuse
constexpr uint32_t kSleepNs = 20000;  // suspend hint of blocking mbarrier waits (wakes on completion)
constexpr int kMaxDch = 1024;       // entries per down chunk
constexpr int kFWarps = 8;          // consumer warps that dot records; the others help
constexpr int kHelperThreads = (kConsumerWarps - kFWarps) * 32;
static_assert(2 * kHelperThreads >= kMaxGrid, "the helpers take two owners a thread");
constexpr int kAssignBar = 2;       // F warps + helpers: the taken records are listed
constexpr int kHelpBar = 3;         // helpers only

enum Exchange : int { EX_U = 0, EX_M = 1, EX_H = 2, EX_V = 3, EX_Y = 4 };

// Row-owned down pass (one token, layers whose active list exceeds three down chunks): each
// thread keeps the partial y of the down units t, t + 512, ... (at most kRoUnits of them).
__host__ __device__ constexpr int ro_units(int fam) { return fam == FAM_Q4 ? 1 : 3; }

struct Smem {
  uint64_t full[kItems];
  uint64_t empty[kItems];
  int abort_flag;
  int count;                    // own active neurons of the layer (union over tokens)
  uint64_t item_at[kItems];     // producer bookkeeping: unwrapped ring offset of items in flight
  uint32_t item_size[kItems];
  float gmean[4];               // glue: mean and 1 / standard deviation of v per token
  float gsd[4];
  float red[2][kConsumerWarps][16];   // block reductions: warp partials (double-buffered)
  int hcnt[kHr];                // F: warps of the record's group that posted partials
  float hpart[kHr][16];         // F: [warp of the record's group][token][gate/up]
  int32_t list[kMaxList];       // the neurons this block dots: its own active ones, then taken ones
  int32_t list_hid[kMaxList];   // h word of each taken entry
  uint8_t list_bits[kMaxList];
  uint8_t own_bits[kMaxOwn];
  int32_t pre[kMaxGrid + 1];    // exclusive prefix of cnt: entries in owner-major order
  int32_t xpre[kMaxGrid + 1];   // exclusive prefix of the owners' excess over the target
  int32_t wsum[2][kConsumerWarps];   // helper scans: the warps' totals
  int32_t wall[kConsumerWarps]; // block scan of the consumer threads' word runs
  uint64_t list_ready;          // the first na records of the list are in place
  uint64_t list2_ready;         // all nrec records of the list are in place
  int na;                       // records handed to the producer before the mask exchange
  int own_cnt;                  // own records this block dots (list entries [0, own_cnt))
  int nrec;                     // records this block dots: own_cnt own ones, then taken ones
  int keep_t;                   // own records whose down rows this block takes (row-owned pass)
  int ro;                       // this layer's down pass is row-owned
  uint64_t dfull[2];            // down chunk copies of each half landed
  uint64_t fdone;               // the layer's neuron records are dotted (the producer's gate)
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
// the same stamp from the first helper thread
__device__ __forceinline__ void hstamp(const FusedParams& p, int l, int ph) {
  if (p.phase_clk && threadIdx.x == kFWarps * 32)
    p.phase_clk[((size_t)blockIdx.x * p.L + l) * kPhases + ph] = stamp_now(p);
}
__device__ __forceinline__ void stamp_val(const FusedParams& p, int l, int ph, long long v) {
  if (p.phase_clk && threadIdx.x == 0) p.phase_clk[((size_t)blockIdx.x * p.L + l) * kPhases + ph] = v;
}
__device__ __forceinline__ long long diag_clock(const FusedParams& p) { return p.phase_clk ? clock64() : 0; }

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
__device__ __forceinline__ bool tag_ok(uint64_t w, uint32_t tag) { return (uint32_t)(w >> 32) == tag; }

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

// Poll the n tagged words src + at(q), q in [0, n), with the npw consumer warps from
// thread tbase on only (the other warps go on to the caller's named barrier and issue
// nothing meanwhile): MQ
// words per lane and round, all loads of a round issued before any tag is checked.  The
// 32-bit payload of word q goes to dst[q].
template <int MQ, typename At>
__device__ __forceinline__ void poll_words(const uint64_t* src, At at, int n, int npw, uint32_t tag, uint32_t* dst,
                                           Smem& sm, const FusedParams& p, int tbase = 0) {
  const int t = (int)threadIdx.x - tbase;
  if (t < 0) return;
  if (t >= npw * 32) return;
  const int nthr = npw * 32;
  for (int b0 = 0; b0 < n; b0 += MQ * nthr) {
    uint64_t w[MQ];
    uint32_t need = 0;
#pragma unroll
    for (int i = 0; i < MQ; ++i) {
      w[i] = 0;
      if (b0 + t + i * nthr < n) need |= 1u << i;
    }
    bool started = false;
    uint64_t t0 = 0;
    while (need) {
#pragma unroll
      for (int i = 0; i < MQ; ++i)
        if (need >> i & 1u) w[i] = ld_tag(src + at(b0 + t + i * nthr));
#pragma unroll
      for (int i = 0; i < MQ; ++i)
        if ((need >> i & 1u) && tag_ok(w[i], tag)) need &= ~(1u << i);
      if (!need || aborted(sm)) break;
      if (!started) { t0 = wait_start(); started = true; }
      else if (timed_out(t0, p.wait_cycles)) { set_abort(sm, p.err, DEV_ERR_GRID_TIMEOUT); break; }
      if (p.poll_ns) __nanosleep(p.poll_ns);
    }
#pragma unroll
    for (int i = 0; i < MQ; ++i)
      if (b0 + t + i * nthr < n) dst[b0 + t + i * nthr] = (uint32_t)w[i];
  }
}

// The same over the consecutive words src[0..n).
template <int MQ>
__device__ __forceinline__ void poll_linear(const uint64_t* src, int n, int npw, uint32_t tag, uint32_t* dst, Smem& sm,
                                         const FusedParams& p) {
  poll_words<MQ>(src, [](int q) { return (size_t)q; }, n, npw, tag, dst, sm, p);
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

// Warps that share the gate/up dots of one F record: 4, or 2 where the partials of a
// group of 4 would not fit a 16-float slot; either divides the kFWarps F warps.
__host__ __device__ constexpr int f_group_warps(int act, int nb) {
  return 4 * nb * (act == PI_REGLU ? 2 : 1) <= 16 ? 4 : 2;
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

// Union over the B tokens of block o's own bit word w (ob: [G][B][nw]).
__device__ __forceinline__ uint32_t union_word(const uint32_t* ob, int o, int w, int nw, int B) {
  uint32_t u = 0;
  for (int b = 0; b < B; ++b) u |= ob[((size_t)o * B + b) * nw + w];
  return u;
}

// Own index m of the k-th active neuron of block o, from the union of its bit words.
__device__ __forceinline__ int owner_select(const uint32_t* ob, int o, int k, int nw, int B) {
  for (int w = 0; w < nw; ++w) {
    const uint32_t u = union_word(ob, o, w, nw, B);
    const int n = __popc(u);
    if (k < n) return 32 * w + select_bit(u, k);
    k -= n;
  }
  return -1;   // unreachable with consistent counts
}

__device__ __forceinline__ uint32_t owner_token_bits(const uint32_t* ob, int o, int m, int nw, int B) {
  uint32_t bits = 0;
  for (int b = 0; b < B; ++b) bits |= ((ob[((size_t)o * B + b) * nw + (m >> 5)] >> (m & 31)) & 1u) << b;
  return bits;
}

// ------------------------------------------------------------------ gate/up dots
// This lane's partial gate/up dot products of one neuron record (at shared address rec)
// with every token's x (xs: [NB][d] at shared address xs) over the units q0, q0 + qs, ...
// in ascending order.
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
__global__ void __launch_bounds__(kThreads, 1) fused_kernel(const __grid_constant__ FusedParams p) {
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
  uint32_t* ob = reinterpret_cast<uint32_t*>(dsmem + p.off_ob);      // [G][B][nw] every block's own bits
  int32_t* dlist = reinterpret_cast<int32_t*>(dsmem + p.off_dlist);  // [2][dch] neuron of each chunk entry
  int32_t* dhid = dlist + 2 * p.dch;                                  // [2][dch] its h word (per token)
  float* dred = reinterpret_cast<float*>(dsmem + p.off_dred);        // down reduction / v slice / moments
  float* hrec = dred;   // h of each dotted record, one token (read by a row-owned down pass,
                        // which leaves dred unused; F writes it before any slice reduction)
  const uint32_t dbuf_u = smem_u32(dsmem + p.off_dbuf);              // [2][dch][pmax] 16-byte down units
  const uint32_t dsc_u = smem_u32(dsmem + p.off_dsc);                // Q4_0: [2][dch][pmax] scale words
  float* hs = reinterpret_cast<float*>(dsmem + p.off_hs);            // [2 * dch][B] h of the resident entries

  const int c = blockIdx.x, G = gridDim.x;
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const bool do_pred = p.mode & MODE_PREDICT, do_ffn = p.mode & MODE_FFN, do_glue = p.mode & MODE_GLUE;
  const int d = p.d, f = p.f, B = p.B;
  const int nown = (c < f) ? (f - c + G - 1) / G : 0;
  // blocks o < own_rem own nown_max neurons, the others nown_max - 1
  const int nown_max = p.nown_max;
  const int own_rem = f - (nown_max - 1) * G;
  const int nunits = d / UE;
  const int words = f / 32;
  const int nw = p.nw;
  // helpers: this thread's run of the G * nw mask words
  const int wpt = (G * nw + kHelperThreads - 1) / kHelperThreads;
  const int wj0 = min(G * nw, max(0, (int)threadIdx.x - kFWarps * 32) * wpt);
  const int wj1 = min(G * nw, wj0 + wpt);
  const int dch = p.dch, pmax = p.pmax;
  // the block's down slice: 16-byte units [cu0, cu1) of every down row.  In the down
  // phase lpe consecutive lanes take one entry (lane % lpe is the unit, so the lanes of an
  // entry read one contiguous piece of its row) and a warp takes epw entries per pass:
  // this lane handles unit dw of the entries de0, de0 + dstep, ... of every chunk
  const int cu0 = (int)((unsigned)c * (unsigned)p.dunits / (unsigned)G);
  const int cu1 = (int)((unsigned)(c + 1) * (unsigned)p.dunits / (unsigned)G);
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
    for (int s = 0; s < kHr; ++s) sm.hcnt[s] = 0;
    mbar_init(&sm.fdone, 1);
    mbar_init(&sm.list_ready, 1);
    mbar_init(&sm.list2_ready, 1);
    mbar_init(&sm.dfull[0], kConsumerThreads);
    mbar_init(&sm.dfull[1], kConsumerThreads);
    sm.abort_flag = 0;
    mbar_fence_init();
  }
  __syncthreads();

  // ================================================================ producer warp
  if (warp == kConsumerWarps) {
    if (lane == 0) {
      uint32_t head = 0, issued = 0, oldest = 0;
      uint32_t landed = 0, inflight = 0;   // items known to have landed; bytes issued beyond them
      // Reserve ring space for the next item.  Items sit in the ring in issue order, none
      // across its end; with offsets counted without wrapping (one more lap at each wrap),
      // an older item can share bytes with the new one only if the new one ends more than
      // one ring length past the older one's start.  Such items are the oldest ones still
      // held, so the producer waits for releases in order until the oldest held item is
      // clear (and no more than kItems - 1 are held).
      uint32_t lap = 0;
      uint64_t at_new = 0;
      auto reserve = [&](uint32_t size, uint32_t& pos) -> bool {
        pos = head;
        if (pos + size > (uint32_t)p.ring_bytes) {
          pos = 0;
          ++lap;
        }
        head = pos + size;
        at_new = (uint64_t)lap * (uint32_t)p.ring_bytes + pos;
        while (oldest < issued) {
          if (issued - oldest < (uint32_t)kItems &&
              at_new + size <= sm.item_at[oldest % kItems] + (uint32_t)p.ring_bytes)
            break;
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
        sm.item_at[issued % kItems] = at_new;
        sm.item_size[issued % kItems] = size;
        dst = ring_base + pos;
        fb = &sm.full[issued % kItems];
        mbar_arrive_expect_tx(fb, size);
        ++issued;
        return true;
      };
      auto wait_list = [&](uint64_t* bar, uint32_t par) -> bool {
        if (mbar_try_wait(bar, par)) return true;
        const uint64_t t0 = wait_start();
        while (!mbar_try_wait_sleep(bar, par, kSleepNs)) {
          if (aborted(sm)) return false;
          if (timed_out(t0, p.wait_cycles)) { set_abort(sm, p.err, DEV_ERR_RING_TIMEOUT); return false; }
        }
        return true;
      };
      // One issue site for every item: per layer the P1^T rows in copies of
      // p1_rows_per_item, the own P2 rows in copies of p2_rows, then one record per list
      // entry: the first na as soon as the block's own list is known, the rest once the
      // helpers have listed them.
      bool ok = true;
      for (int l = 0; l < p.L && ok; ++l) {
        // Layer l's predictor rows wait until layer l - 1's records are dotted: until then
        // the records' reads have HBM to themselves, and the exchanges after them leave
        // HBM idle for these copies.
        if (l > 0 && do_ffn) {
          const uint32_t par = (uint32_t)((l - 1) & 1);
          if (!mbar_try_wait(&sm.fdone, par)) {
            const uint64_t t0 = wait_start();
            while (!mbar_try_wait_sleep(&sm.fdone, par, kSleepNs)) {
              if (aborted(sm)) { ok = false; break; }
              if (timed_out(t0, p.wait_cycles)) { set_abort(sm, p.err, DEV_ERR_RING_TIMEOUT); ok = false; break; }
            }
            if (!ok) break;
          }
        }
        const LayerDev Ld = p.layers[l];
        const int r = Ld.r;
        const int k0 = (int)((unsigned)c * (unsigned)r / (unsigned)G);
        const int k1 = (int)((unsigned)(c + 1) * (unsigned)r / (unsigned)G);
        const int p2_stride = p2_stride_of(r, PB);
        const int p2_rows = max(1, min(p.nown_max, p.p2_item_bytes / p2_stride));
        const uint8_t* own = Ld.p2o + (size_t)c * p.nown_max * p2_stride;
        const int n1 = do_pred ? (k1 - k0 + p.p1_rows_per_item - 1) / p.p1_rows_per_item : 0;
        const int n2 = do_pred ? (nown + p2_rows - 1) / p2_rows : 0;
        int na = 0, n = 0;   // records: handed over first, in all (known once listed)
        int nd = 0, keep_t = 0, own_c = 0;   // row-owned layers: down rows after the records
        for (int it = 0; ok; ++it) {
          const uint8_t* src;
          uint32_t bytes;
          if (it < n1) {
            const int k = k0 + it * p.p1_rows_per_item;
            src = Ld.p1t + (size_t)k * p.p1_row;
            bytes = (uint32_t)min(p.p1_rows_per_item, k1 - k) * p.p1_row;
          } else if (it < n1 + n2) {
            const int m = (it - n1) * p2_rows;
            src = own + (size_t)m * p2_stride;
            bytes = (uint32_t)min(p2_rows, nown - m) * p2_stride;
          } else {
            if (!do_ffn) break;
            const int e = it - n1 - n2;
            if (e == 0) {
              if (!(ok = wait_list(&sm.list_ready, (uint32_t)(l & 1)))) break;
              na = n = sm.na;
            }
            if (e == na && n == na) {
              if (!(ok = wait_list(&sm.list2_ready, (uint32_t)(l & 1)))) break;
              n = sm.nrec;
              if (sm.ro) {
                keep_t = sm.keep_t;
                own_c = sm.own_cnt;
                nd = keep_t + (n - own_c);
              }
            }
            if (e < n) {
              src = Ld.rec + (size_t)sm.list[e] * p.rec_stride;
              bytes = (uint32_t)p.rec_stride;
            } else {
              const int j = e - n;   // down row j: own entries below T, then the taken ones
              if (j >= nd) break;
              const int ent = j < keep_t ? j : own_c + (j - keep_t);
              src = Ld.rec + p.dn_off + (size_t)sm.list[ent] * p.dn_stride;
              bytes = (uint32_t)p.dn_stride;
            }
          }
          uint8_t* dst;
          uint64_t* fb;
          if (!(ok = begin_item(bytes, dst, fb))) break;
          bulk_g2s(dst, src, bytes, fb);
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
  uint32_t dphase[2] = {0u, 0u};   // completed phases of dfull[0], dfull[1]
  for (int l = 0; l < p.L; ++l) {
    const LayerDev Ld = p.layers[l];
    const int r = Ld.r;
    const int k0 = (int)((unsigned)c * (unsigned)r / (unsigned)G);
    const int k1 = (int)((unsigned)(c + 1) * (unsigned)r / (unsigned)G);
    const int p2_stride = p2_stride_of(r, PB);
    const int p2_rows = max(1, min(p.nown_max, p.p2_item_bytes / p2_stride));
    const uint32_t tag_u = tag_of(epoch, l, EX_U), tag_m = tag_of(epoch, l, EX_M), tag_h = tag_of(epoch, l, EX_H),
                   tag_v = tag_of(epoch, l, EX_V), tag_y = tag_of(epoch, l, EX_Y);
    int nlist = 0;      // records this block dots
    int ntotal = 0;     // active entries of the layer (the down list)
    int hid0 = 0;       // h word of the block's first record: records publish h in list order
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
      poll_linear<8>(p.ux, B * r, kConsumerWarps, tag_u, reinterpret_cast<uint32_t*>(u_s), sm, p);
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
          if (lane == 0 && b < B) st_tag_u(p.mx + ((size_t)c * B + b) * nw + w, word, tag_m);
        }
      }
      if (t == 0) {
        // own records handed to the producer now, whatever the exchange says
        sm.na = min(sm.count, max(Ld.keep_floor, 1));
        mbar_arrive(&sm.list_ready);
      }
      named_bar_sync(kRedBar, kConsumerThreads);
      nlist = sm.count;
      hid0 = c * nown_max;
      stamp(p, l, 4);
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
      const int a0 = (int)((unsigned)c * (unsigned)cnt / (unsigned)G);
      const int a1 = (int)((unsigned)(c + 1) * (unsigned)cnt / (unsigned)G);
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
      if (t == 0) {
        atomicAdd(p.active_total, (unsigned long long)nlist);
        sm.na = sm.own_cnt = sm.nrec = nlist;
        sm.ro = 0;
        mbar_arrive(&sm.list_ready);
      }
      ntotal = cnt;
      hid0 = a0;
    }

    named_bar_sync(kRedBar, kConsumerThreads);
    stamp(p, l, 6);
    stamp_val(p, l, 14, nlist);

    // ------------------------------------------------------------ down list and copies
    // Chunk k holds the active entries [k*dch, (k+1)*dch) of the layer in owner-major
    // order (the caller's order for a given list); dlist half k%2 holds their neuron ids,
    // dhid half k%2 the index of their h words (owner o's records publish h from word
    // o * nown_max on; a caller's list, at its entry index) and dbuf half k%2 their units
    // [cu0, cu1).  The helper warps build the halves and copy the units (cp.async); the
    // copies of half j complete a phase of dfull[j].
    const uint8_t* dn = Ld.rec + p.dn_off;
    const int ht = t - kFWarps * 32;   // helper thread index (>= 0 in the helper warps)
    int woff = 0;                      // helpers: the layer's entries before this thread's mask words
    // chunks k .. k + nk - 1 (nk = 2 only from an even k: the two halves in order)
    // Word runs: the helpers' (one run a helper thread, its first entry at woff) and, for
    // chunks past the second, every consumer thread's (wa0, wa1, aoff).
    auto build_dlist = [&](int k, int nk, int rj0, int rj1, int roff, int tid, int nthr) {
      const int lo = k * dch, hi = min(ntotal, lo + nk * dch);
      int32_t* dl = dlist + (k & 1) * dch;
      int32_t* dh = dhid + (k & 1) * dch;
      if (do_pred) {
        // this thread's run of mask words, its first entry at roff: set bits in order
        int e = roff;
        int o = rj0 / nw, w = rj0 - o * nw;
        const uint32_t dla = smem_u32(dl), dha = smem_u32(dh);
        for (int j = rj0; j < rj1 && e < hi; ++j) {
          uint32_t u = union_word(ob, o, w, nw, B);
          const int n = __popc(u);
          if (e + n > lo) {
            const int pre_o = sm.pre[o];
            while (u && e < hi) {
              const int bit = __ffs(u) - 1;
              u &= u - 1;
              if (e >= lo) {
                sts_u32(dla + 4u * (uint32_t)(e - lo), (uint32_t)(o + (32 * w + bit) * G));
                // owner o's h words start at o * nown_max
                sts_u32(dha + 4u * (uint32_t)(e - lo), (uint32_t)(o * nown_max + (e - pre_o)));
              }
              ++e;
            }
          } else {
            e += n;
          }
          if (++w == nw) {
            w = 0;
            ++o;
          }
        }
      } else {
        for (int e = lo + tid; e < hi; e += nthr) {
          int i = __ldg(p.idx_in + e);
          if (i < 0 || i >= f) i = 0;   // reported above
          dl[e - lo] = i;
          dh[e - lo] = e;
        }
      }
    };
    // helper lane mapping of the copies: the F mapping of the down pass over 4 warps
    const int hde0 = (warp - kFWarps) * epw + lane / lpe;
    const int hdstep = (kConsumerWarps - kFWarps) * epw;
    auto issue_down = [&](int k, int ef, int es) {
      if (dw >= 0) {
        const int lo = k * dch, hi = min(ntotal, lo + dch);
        const int32_t* dl = dlist + (k & 1) * dch;
        const int half = (k & 1) * dch;
        for (int e = lo + ef; e < hi; e += es) {
          const int i = dl[e - lo];
          const uint8_t* row = dn + (size_t)i * p.dn_stride;
          const uint32_t slot = (uint32_t)((half + e - lo) * pmax + dw);
          cpa16(dbuf_u + slot * 16u, row + (size_t)(cu0 + dw) * 16);
          if constexpr (FAM == FAM_Q4)
            cpa4(dsc_u + slot * 4u, row + (size_t)(d >> 1) + (size_t)((cu0 + dw) >> 1) * 4);
        }
      }
      cpa_arrive_noinc(&sm.dfull[k & 1]);
    };

    // ------------------------------------------------------------ F: records -> h
    // Warps below kFWarps form groups of KG; group g dots records g, g + NG, ... in ring
    // order: each warp of the group waits for the record to land, dots its slice of the
    // units with x from shared memory, reduces across its lanes and posts its partial
    // sums in the record's h slot.  The last warp of the group to post sums the group's
    // partials in a fixed order, forms h and publishes it.  Records past na wait for the
    // helpers' list (kAssignBar).  The helper warps take the mask exchange, the balanced
    // assignment, the down list and the down copies meanwhile.
    if (warp < kFWarps) {
      constexpr int NV = (ACT == PI_REGLU) ? 2 : 1;
      constexpr int NVAL = NB * NV;                 // partial sums per warp and record
      constexpr int V = pow2_ceil(NVAL);
      constexpr int LG = log2_exact(V);
      constexpr int KG = f_group_warps(ACT, NB);
      constexpr int NG = kFWarps / KG;              // records dotted at once
      static_assert(KG * NVAL <= 16 && kFWarps % KG == 0 && kHr % NG == 0, "h slot layout");
      const uint32_t base = smem_u32(ring.base), xsa = smem_u32(xs);
      const uint32_t item0 = ring.item;
      const int kq = warp % KG;
      uint32_t hd = ring.head;   // ring head before record id (dot cursor)
      int id = 0;
      const int na = sm.na;
      int nrec = na, own_cnt = na;
      for (int e = warp / KG;; e += NG) {
        if (e >= na && nrec == na && own_cnt == na) {
          named_bar_sync(kAssignBar, kConsumerThreads);   // the rest of the list is in place
          nrec = sm.nrec;
          own_cnt = sm.own_cnt;
          if (nrec == na) own_cnt = -1;   // (no second wait)
        }
        if (e >= nrec) break;
        uint32_t pos = 0;
        for (; id <= e; ++id) pos = ring_place(hd, (uint32_t)p.rec_stride, ring.cap);
        ring_wait_item_warp(item0 + e, sm, p);
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
        if ((lane & ((32 >> LG) - 1)) == 0 && (lane >> (5 - LG)) < NVAL)
          sm.hpart[s][kq * NVAL + (lane >> (5 - LG))] = sw;
        const float bi = lds_f32(base + pos + (uint32_t)p.bias_off);
        __syncwarp();
        if (lane == 0) {
          __threadfence_block();
          if (atomicAdd(&sm.hcnt[s], 1) == KG - 1) {
            __threadfence_block();
            const volatile float* hp = sm.hpart[s];
            const int ent = e < max(own_cnt, na) ? hid0 + e : sm.list_hid[e];
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
                if (b == 0) hrec[e] = (bits & 1u) ? a : 0.f;
              }
            }
            sm.hcnt[s] = 0;
          }
        }
        ring_release_item(item0 + e, sm, (uint32_t)(kConsumerWarps / KG));
      }
      stamp(p, l, 9);
      if (t == 0) mbar_arrive(&sm.fdone);
    } else {
      if (do_pred) {
        // ---------------------------------------------------------- mask exchange
        poll_words<8>(p.mx, [](int q) { return (size_t)q; }, G * B * nw, kConsumerWarps - kFWarps, tag_m, ob, sm, p,
                      kFWarps * 32);
        named_bar_sync(kHelpBar, kHelperThreads);
        hstamp(p, l, 5);
        // The mask words in owner-major order (word j: owner j / nw, word j % nw) are
        // split into runs of consecutive words, one run a helper thread.  Only bits of
        // neurons the owner has can be set (a word of an aborted exchange may hold
        // anything): the rest are cleared in place.
        int wcnt = 0;
        for (int j = wj0; j < wj1; ++j) {
          const int o = j / nw, w = j - o * nw;
          const int nown_o = o < own_rem ? nown_max : nown_max - 1;
          const int nv = min(32, max(0, nown_o - 32 * w));
          const uint32_t valid = nv >= 32 ? 0xFFFFFFFFu : ((1u << nv) - 1u);
          uint32_t u = 0;
          for (int b = 0; b < B; ++b) {
            uint32_t* wp = ob + ((size_t)o * B + b) * nw + w;
            const uint32_t x = *wp & valid;
            *wp = x;
            u |= x;
          }
          wcnt += __popc(u);
        }
        // the prefix of the counts, then of the excess over T and of the shortfall
        const int hw = warp - kFWarps;
        auto helper_scan = [&](int v, int slot, int& total) -> int {   // exclusive prefix over helpers
          int incl = v;
#pragma unroll
          for (int k = 1; k < 32; k <<= 1) {
            const int x = __shfl_up_sync(0xffffffffu, incl, k);
            if (lane >= k) incl += x;
          }
          if (lane == 31) sm.wsum[slot][hw] = incl;
          named_bar_sync(kHelpBar, kHelperThreads);
          int off = 0;
          total = 0;
#pragma unroll
          for (int w = 0; w < kConsumerWarps - kFWarps; ++w) {
            const int x = sm.wsum[slot][w];
            off += w < hw ? x : 0;
            total += x;
          }
          return off + incl - v;   // exclusive
        };
        int N = 0;
        woff = helper_scan(wcnt, 0, N);   // entries before this thread's first word
        {
          int e = woff;
          for (int j = wj0; j < wj1; ++j) {
            const int o = j / nw, w = j - o * nw;
            if (w == 0) sm.pre[o] = e;
            e += __popc(union_word(ob, o, w, nw, B));
          }
          if (ht == 0) sm.pre[G] = N;
        }
        named_bar_sync(kHelpBar, kHelperThreads);
        int n2[2];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int o = 2 * ht + i;
          n2[i] = o < G ? sm.pre[o + 1] - sm.pre[o] : 0;
        }
        const int T = max(1, (N + G - 1) / G);
        // the excess over T and the shortfall below it, scanned together
        const int x0 = max(0, n2[0] - T), x1 = max(0, n2[1] - T);
        const int s0 = (2 * ht < G) ? max(0, T - n2[0]) : 0, s1 = (2 * ht + 1 < G) ? max(0, T - n2[1]) : 0;
        int px, ps, xtotal;
        {
          int ix = x0 + x1, is = s0 + s1;
#pragma unroll
          for (int k = 1; k < 32; k <<= 1) {
            const int a = __shfl_up_sync(0xffffffffu, ix, k), b = __shfl_up_sync(0xffffffffu, is, k);
            if (lane >= k) {
              ix += a;
              is += b;
            }
          }
          if (lane == 31) {
            sm.wsum[1][hw] = ix;
            sm.wsum[1][kConsumerWarps / 2 + hw] = is;
          }
          named_bar_sync(kHelpBar, kHelperThreads);
          int ox = 0, os = 0;
          xtotal = 0;
#pragma unroll
          for (int w = 0; w < kConsumerWarps - kFWarps; ++w) {
            const int a = sm.wsum[1][w], b = sm.wsum[1][kConsumerWarps / 2 + w];
            ox += w < hw ? a : 0;
            os += w < hw ? b : 0;
            xtotal += a;
          }
          px = ox + ix - (x0 + x1);
          ps = os + is - (s0 + s1);
        }
        if (2 * ht < G) sm.xpre[2 * ht] = px;
        if (2 * ht + 1 < G) sm.xpre[2 * ht + 1] = px + x0;
        if (ht == 0) sm.xpre[G] = xtotal;
        if (2 * ht == c) sm.wsum[0][kConsumerWarps - 1] = ps;
        if (2 * ht + 1 == c) sm.wsum[0][kConsumerWarps - 1] = ps + s0;
        named_bar_sync(kHelpBar, kHelperThreads);
        const int n_own = nlist;
        const int dstart = sm.wsum[0][kConsumerWarps - 1];
        // this block dots its first own_cnt own records (those already handed to the
        // producer included) and then the taken ones, listed from entry own_cnt on
        const int own_cnt = max(min(n_own, T), sm.na);
        const int deficit = max(0, T - n_own);
        const int ntake = max(0, min(dstart + deficit, xtotal) - dstart);
        if (ht == 0) {
          sm.own_cnt = own_cnt;
          sm.nrec = own_cnt + ntake;
          // more active neurons than three down chunks hold: the row-owned down pass (one
          // token), each block over the down rows of the records it dots, own ones past T
          // left to their takers
          sm.ro = (B == 1 && N > 3 * dch && p.dunits <= kConsumerThreads * ro_units(FAM) &&
                   G * PE * 4 <= 32 * dch) ? 1 : 0;
          sm.keep_t = min(n_own, T);
        }
        for (int q = ht; q < ntake; q += kHelperThreads) {
          const int x = dstart + q;
          int lo = 0, hi = G;   // owner o: xpre[o] <= x < xpre[o + 1]
          while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (sm.xpre[mid] <= x) lo = mid;
            else hi = mid;
          }
          const int k = T + (x - sm.xpre[lo]);
          const int m = owner_select(ob, lo, k, nw, B);
          const int i = lo + max(m, 0) * G;
          sm.list[own_cnt + q] = i < f ? i : 0;
          sm.list_bits[own_cnt + q] = (uint8_t)(m >= 0 ? owner_token_bits(ob, lo, m, nw, B) : 0u);
          sm.list_hid[own_cnt + q] = lo * nown_max + k;
        }
        ntotal = N;
      }
      named_bar_sync(kHelpBar, kHelperThreads);
      if (ht == 0) mbar_arrive(&sm.list2_ready);          // the producer copies the rest
      named_bar_arrive(kAssignBar, kConsumerThreads);   // the F warps dot it
      hstamp(p, l, 29);
      const int nchunks = sm.ro ? 0 : (ntotal + dch - 1) / dch;
      build_dlist(0, 2, wj0, wj1, woff, ht, kHelperThreads);
      named_bar_sync(kHelpBar, kHelperThreads);
      hstamp(p, l, 23);
      if (nchunks > 0) issue_down(0, hde0, hdstep);
      if (nchunks > 1) issue_down(1, hde0, hdstep);
      hstamp(p, l, 7);
    }
    if (do_pred) ntotal = sm.pre[G];   // every warp: the layer's active count
    const bool ro = sm.ro != 0;
    const int nchunks = ro ? 0 : (ntotal + dch - 1) / dch;
    stamp_val(p, l, 15, ntotal);

    // ------------------------------------------------------------ down: y of the slice
    float acc[NB][PE];
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
      for (int e = 0; e < PE; ++e) acc[b][e] = 0.f;
    long long h_wait = 0;   // diagnostics: cycles thread 0 polls for h
    // The h words of resident entries (at their dhid words) are polled by every consumer
    // thread at once (one polling round) into shared memory: chunks 0 and 1 together, later
    // chunks one at a time.  Entry e of chunk k sits in slot e - (k - k % 2) * dch.
    auto poll_h = [&](int e_lo, int e_hi, int slot0) {
      const long long wt0 = diag_clock(p);
      const int32_t* hid = dhid + slot0;
      poll_words<8>(p.hx, [&](int q) { return (size_t)hid[q / B] * B + (size_t)(q % B); }, (e_hi - e_lo) * B,
                    kConsumerWarps, tag_h, reinterpret_cast<uint32_t*>(hs) + (size_t)slot0 * B, sm, p);
      h_wait += diag_clock(p) - wt0;
    };
    // every warp is past F and the down list halves 0 and 1 are built
    named_bar_sync(kRedBar, kConsumerThreads);
    if (warp < kFWarps) {   // the F warps' arrivals on the copies of chunks 0 and 1 (none)
      if (nchunks > 0) cpa_arrive_noinc(&sm.dfull[0]);
      if (nchunks > 1) cpa_arrive_noinc(&sm.dfull[1]);
    }
    // chunks past the second are built and copied by every consumer thread: each takes a
    // run of the mask words, its first entry from a block scan of the runs' counts
    int wa0 = 0, wa1 = 0, aoff = 0;
    if (do_pred && nchunks > 2) {
      const int wpa = (G * nw + kConsumerThreads - 1) / kConsumerThreads;
      wa0 = min(G * nw, t * wpa);
      wa1 = min(G * nw, wa0 + wpa);
      int cnt = 0;
      for (int j = wa0; j < wa1; ++j) {
        const int o = j / nw;
        cnt += __popc(union_word(ob, o, j - o * nw, nw, B));
      }
      int incl = cnt;
#pragma unroll
      for (int k = 1; k < 32; k <<= 1) {
        const int x = __shfl_up_sync(0xffffffffu, incl, k);
        if (lane >= k) incl += x;
      }
      if (lane == 31) sm.wall[warp] = incl;
      named_bar_sync(kRedBar, kConsumerThreads);
      int off = 0;
      for (int w = 0; w < warp; ++w) off += sm.wall[w];
      aoff = off + incl - cnt;
    }
    {
      // the ring past this layer's records (every consumer keeps the same ring state)
      const int nr = sm.nrec;
      for (int q = 0; q < nr; ++q) ring_place(ring.head, (uint32_t)p.rec_stride, ring.cap);
      ring.item += (uint32_t)nr;
      fseq += (uint32_t)nr;
    }
    if (ro) {
      // ------------------------------------------------------------ row-owned down pass
      // The down rows of the records this block dotted follow them in the ring; thread t
      // adds h times its units t, t + 512, ... of each row, in list order, and publishes
      // its partial y (tagged words, d a block).
      constexpr int RU = ro_units(FAM);
      const int keep_t = sm.keep_t, own_c = sm.own_cnt;
      const int nd = keep_t + (sm.nrec - own_c);
      const uint32_t base = smem_u32(ring.base);
      float ra[RU][1][PE];
#pragma unroll
      for (int u = 0; u < RU; ++u)
#pragma unroll
        for (int e = 0; e < PE; ++e) ra[u][0][e] = 0.f;
      for (int j = 0; j < nd; ++j) {
        const uint32_t pos = ring_place(ring.head, (uint32_t)p.dn_stride, ring.cap);
        ring_wait_item_warp(ring.item, sm, p);
        const float h1[1] = {hrec[j < keep_t ? j : own_c + (j - keep_t)]};
#pragma unroll
        for (int u = 0; u < RU; ++u) {
          const int unit = t + u * kConsumerThreads;
          if (unit < p.dunits) {
            float sc = 0.f;
            if constexpr (FAM == FAM_Q4) sc = lds_h2f(base + pos + (uint32_t)(d >> 1) + 2u * (uint32_t)unit);
            down_unit_fma<FAM, 1>(base + pos + 16u * (uint32_t)unit, sc, h1, ra[u]);
          }
        }
        ring_release_item(ring.item++, sm);
      }
#pragma unroll
      for (int u = 0; u < RU; ++u) {
        const int unit = t + u * kConsumerThreads;
        if (unit < p.dunits)
#pragma unroll
          for (int e = 0; e < PE; ++e) st_tag(p.yx + (size_t)c * d + (size_t)unit * PE + e, ra[u][0][e], tag_y);
      }
    }
    for (int k = 0; k < nchunks; ++k) {
      const int lo = k * dch, hi = min(ntotal, lo + dch);
      if (k == 0) poll_h(0, min(ntotal, 2 * dch), 0);
      else if (k >= 2) poll_h(lo, hi, (k & 1) * dch);
      if (k == 0) stamp(p, l, 25);
      if (k != 1) named_bar_sync(kRedBar, kConsumerThreads);
      if (k == 0) stamp(p, l, 26);
      bar_wait(&sm.dfull[k & 1], dphase[k & 1] & 1u, sm, p);   // the copies of chunk k have landed
      ++dphase[k & 1];
      if (k == 0) stamp(p, l, 27);
      if (dw >= 0) {
        const int half = (k & 1) * dch;
        for (int e = lo + de0; e < hi; e += dstep) {
          float h[NB];
#pragma unroll
          for (int b = 0; b < NB; ++b) h[b] = b < B ? hs[(size_t)(half + e - lo) * B + b] : 0.f;
          const uint32_t slot = (uint32_t)((half + e - lo) * pmax + dw);
          float sc = 0.f;
          if constexpr (FAM == FAM_Q4) {
            const uint32_t sw = lds_u32(dsc_u + slot * 4u);
            sc = __half2float(__ushort_as_half((unsigned short)(((cu0 + dw) & 1) ? (sw >> 16) : (sw & 0xFFFFu))));
          }
          down_unit_fma<FAM, NB>(dbuf_u + slot * 16u, sc, h, acc);
        }
      }
      if (k + 2 < nchunks) {
        named_bar_sync(kRedBar, kConsumerThreads);   // every thread is done with dlist, hs and dbuf half k%2
        build_dlist(k + 2, 1, wa0, wa1, aoff, t, kConsumerThreads);
        named_bar_sync(kRedBar, kConsumerThreads);   // chunk k + 2's dlist and dhid are in place
        issue_down(k + 2, de0, dstep);
      }
    }
    stamp(p, l, 28);
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
      if (lane < lpe && dw >= 0 && !ro) {
#pragma unroll
        for (int b = 0; b < NB; ++b)
#pragma unroll
          for (int e = 0; e < PE; ++e) dred[(warp * pmax + dw) * V + b * PE + e] = acc[b][e];
      }
      // row-owned layers: every block's partial y of this block's columns
      float* ybuf = reinterpret_cast<float*>(dsmem + p.off_dbuf);   // [G][ncol]
      if (ro)
        poll_words<8>(p.yx, [&](int q) { const int g = q / ncol; return (size_t)g * d + col0 + (q - g * ncol); },
                      G * ncol, kConsumerWarps, tag_y, reinterpret_cast<uint32_t*>(ybuf), sm, p);
      named_bar_sync(kRedBar, kConsumerThreads);
      // warp b forms token b's slice: y, v = x + y and its (sum, sum of squares), which
      // follow v in the exchange array
      if (warp < B) {
        const int b = warp;
        float s = 0.f, s2 = 0.f;
        for (int q = lane; q < ncol; q += 32) {
          const int w = q / PE, e = q % PE;
          float y = 0.f;
          if (ro)
            for (int g = 0; g < G; ++g) y += ybuf[g * ncol + q];
          else
            for (int k = 0; k < kConsumerWarps; ++k) y += dred[(k * pmax + w) * V + b * PE + e];
          const int col = col0 + q;
          if (do_glue) {
            const float v = xs_val<FAM>(xs, b * d + col) + y;
            st_tag(p.vx + (size_t)b * d + col, v, tag_v);
            if (p.trace.y) p.trace.y[((size_t)l * B + b) * d + col] = y;
            s += v;
            s2 += v * v;
          } else {
            p.y_out[(size_t)b * d + col] = y;
          }
        }
        if (do_glue) {
          s = warp_sum(s);
          s2 = warp_sum(s2);
          if (lane == 0) {
            st_tag(p.vx + (size_t)B * d + ((size_t)b * G + c) * 2, s, tag_v);
            st_tag(p.vx + (size_t)B * d + ((size_t)b * G + c) * 2 + 1, s2, tag_v);
          }
        }
      }
      if (!do_glue) break;
      if (ro) named_bar_sync(kRedBar, kConsumerThreads);   // ybuf is read before the glue reuses it
    }
    stamp(p, l, 11);

    // ------------------------------------------------------------ glue: x' = (v - mean) / sd
    // The consumer threads poll every slice's (sum, sum of squares), which follow v in the
    // same array, and then all of v into the down buffers (free now); the moments give
    // each token's mean and 1 / sd, and every thread forms its elements of x'.
    {
      float* gbuf = reinterpret_cast<float*>(dsmem + p.off_dlist);   // [B][d] v, then [B][G][2]
      // the moments, published after v, first: the repeated polls then touch only the
      // few lines they sit in, and v is usually complete at the first look
      poll_linear<8>(p.vx + (size_t)B * d, 2 * B * G, kConsumerWarps, tag_v,
                     reinterpret_cast<uint32_t*>(gbuf) + (size_t)B * d, sm, p);
      poll_linear<16>(p.vx, B * d, kConsumerWarps, tag_v, reinterpret_cast<uint32_t*>(gbuf), sm, p);
      named_bar_sync(kRedBar, kConsumerThreads);
      stamp(p, l, 12);
      if (warp < B) {
        const float* mom = gbuf + (size_t)B * d + (size_t)warp * G * 2;
        float s = 0.f, s2 = 0.f;
        for (int cq = lane; cq < G; cq += 32) {
          s += mom[2 * cq];
          s2 += mom[2 * cq + 1];
        }
        const float sum = warp_sum(s);
        s2 = warp_sum(s2);
        if (lane == 0) {
          const float mean = sum / (float)d;
          const float var = fmaxf(s2 / (float)d - mean * mean, 0.f);
          sm.gmean[warp] = mean;
          sm.gsd[warp] = 1.0f / sqrtf(var + kNormEps);   // one division per token; elements multiply
        }
      }
      named_bar_sync(kRedBar, kConsumerThreads);
      for (int b = 0; b < B; ++b) {
        const float mean = sm.gmean[b], inv = sm.gsd[b];
        for (int j = t; j < d; j += kConsumerThreads)
          xs[b * d + j] = XT(round_act<FAM>((gbuf[b * d + j] - mean) * inv));
      }
      named_bar_sync(kRedBar, kConsumerThreads);
      // every block writes its own columns of the trace and of the output
      if (p.trace.x || l == p.L - 1)
        for (int b = 0; b < B; ++b)
          for (int q = t; q < ncol; q += kConsumerThreads) {
            const int j = b * d + col0 + q;
            const float xv = xs_val<FAM>(xs, j);
            if (p.trace.x) store_act<FAM>(p.trace.x, (size_t)(l + 1) * B * d + j, xv);
            if (l == p.L - 1) store_act<FAM>(p.x_out, (size_t)j, xv);
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
  const size_t dred_floats = std::max((size_t)kConsumerWarps * p.pmax * nb * pe, (size_t)kMaxList);
  size_t off = round_up(sizeof(Smem), 128);
  const size_t fixed_tail = round_up((size_t)nb * p.d * xbytes, 16) + round_up((size_t)nb * p.r * 4, 16) +
                            round_up((size_t)G * nb * p.nw * 4, 16) + round_up(dred_floats * 4, 16);
  // per chunk entry: its dlist and dhid slots and its units (plus a scale word per Q4_0
  // unit), twice
  const size_t entry_bytes = 2 * (8 + (size_t)nb * 4 + (size_t)p.pmax * 16 + (family == FAM_Q4 ? (size_t)p.pmax * 4 : 0));
  const size_t ring_min = std::max((size_t)112 * 1024, (size_t)(2 * max_item));
  if (budget < off + fixed_tail + ring_min + 64 * entry_bytes + 256) return false;
  size_t dch = (budget - off - fixed_tail - ring_min - 256) / entry_bytes;
  dch = std::min(dch, (size_t)kMaxDch);
  p.dch = (int)dch;
  // the glue reuses the down region (dlist .. hs) for all of v and the slice moments
  const size_t glue_bytes = ((size_t)nb * p.d + 2 * (size_t)nb * G) * 4;
  if (dch * entry_bytes < glue_bytes) dch = std::min((size_t)kMaxDch, (glue_bytes + entry_bytes - 1) / entry_bytes);
  if (dch * entry_bytes < glue_bytes) return false;
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
  off += round_up((size_t)4 * dch * 4, 16);
  p.off_dbuf = (int)off;
  off += (size_t)2 * dch * p.pmax * 16;
  p.off_dsc = (int)off;
  off += family == FAM_Q4 ? (size_t)2 * dch * p.pmax * 4 : 0;
  p.off_hs = (int)off;
  off += (size_t)2 * dch * nb * 4;
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
