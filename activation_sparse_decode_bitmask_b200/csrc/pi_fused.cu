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
//        (one warp per row, four rows at a time); bit = logit > 0 -> bitmap exchange
//   list every block reads every block's bitmap, so all know the active set; the
//        active neurons are split evenly: block c takes a contiguous share of them in
//        (owner block, owner position) order
//   F    for each of its records: one warp forms the gate/up dot products with x
//          ReLU : h = max(0, w_up_i . x + b_i)    ReGLU: max(0, w_gate_i . x + b_i) * (w_up_i . x)
//          h[b] = 0 where token b's bit is 0
//        then all threads add h * w_down_i into y (registers, fp32, one thread per 16 B)
//        -> partial exchange
//   R    block s < nslices owns a column slice: v = x + sum_c partial_c in ascending c,
//        and the slice's sum and sum of squares -> v / moments exchange
//   glue x' = (v - mean(v)) / sqrt(var(v) + 1e-6) from the slices' sums and sums of
//        squares, rounded to the activation dtype
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
constexpr int kMaxBatch = 16;       // records per F batch (one warp each)

struct Smem {
  uint64_t full[kItems];
  uint64_t empty[kItems];
  uint64_t list_ready;
  uint64_t layer_start;
  int abort_flag;
  int nlist;
  int count;                   // active neurons of the layer (union over tokens)
  int pad;
  uint32_t item_pos[kItems];   // producer bookkeeping of items in flight
  uint32_t item_size[kItems];
  float gmean[4];   // glue: mean and standard deviation of v per token
  float gsd[4];
  float hbuf[kMaxList][4];      // h of the layer's records, by list position
  int hflag[kMaxList];          // = layer + 1 once hbuf[e] is written
  int32_t list[kMaxList];
  uint8_t list_bits[kMaxList];
  uint8_t own_bits[kMaxOwn];
  int32_t cstart[kMaxGrid + 1];   // prefix of active counts over owner blocks
  int scan[kConsumerWarps + 1];
};

// Diagnostics: SM cycle stamps at phase boundaries, [block][layer][kPhases].
constexpr int kPhases = 20;
__device__ __forceinline__ long long stamp_now(const FusedParams& p) {
  return p.phase_global ? (long long)globaltimer_ns() : clock64();
}
__device__ __forceinline__ void stamp(const FusedParams& p, int l, int ph) {
  if (p.phase_clk && threadIdx.x == 0)
    p.phase_clk[((size_t)blockIdx.x * p.L + l) * kPhases + ph] = stamp_now(p);
}
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
      if (need >> k & 1u) {
        w[k] = ld_tag(base + first + k * stride);
        if (tag_ok(w[k], tag)) need &= ~(1u << k);
      }
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
__device__ __forceinline__ void ring_wait_item(uint32_t item, Smem& sm, const FusedParams& p) {
  uint64_t* bar = &sm.full[item % kItems];
  const uint32_t par = (item / kItems) & 1u;
  if (!aborted(sm) && !mbar_try_wait(bar, par)) {
    const uint64_t t0 = wait_start();
    while (!mbar_try_wait(bar, par)) {
      if (aborted(sm)) break;
      if (timed_out(t0, p.wait_cycles)) { set_abort(sm, p.err, DEV_ERR_RING_TIMEOUT); break; }
    }
  }
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

// ------------------------------------------------------------------ the kernel
template <int FAM, int ACT, int NB, int NU>
__global__ void __launch_bounds__(kThreads, 1) fused_kernel(const FusedParams p) {
  constexpr int UE = Fam<FAM>::UE;
  constexpr int PB = Fam<FAM>::PB;
  using XT = typename Fam<FAM>::X;
  extern __shared__ __align__(128) uint8_t dsmem[];
  Smem& sm = *reinterpret_cast<Smem*>(dsmem);
  uint8_t* ring_base = dsmem + ((sizeof(Smem) + 127) / 128) * 128;
  XT* xs = reinterpret_cast<XT*>(ring_base + p.ring_bytes);            // [NB][d] current input
  float* u_s = reinterpret_cast<float*>(xs + (size_t)NB * p.d);        // [NB][r]
  float* red2 = u_s + (size_t)NB * p.r;                                // [8][NB][4][32]
  uint32_t* bm = reinterpret_cast<uint32_t*>(red2 + kConsumerWarps * NB * kMaxColGroups * 32);   // [B][G][W]

  const int c = blockIdx.x, G = gridDim.x;
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const bool do_pred = p.mode & MODE_PREDICT, do_ffn = p.mode & MODE_FFN, do_glue = p.mode & MODE_GLUE;
  const int d = p.d, f = p.f, r = p.r, B = p.B;
  const int k0 = (int)((long long)c * r / G), k1 = (int)((long long)(c + 1) * r / G);
  const int nown = (c < f) ? (f - c + G - 1) / G : 0;
  const int W = (p.nown_max + 31) / 32;   // bitmap words per block and token
  const int nunits = d / UE;
  const int words = f / 32;
  const uint32_t epoch = *reinterpret_cast<volatile const uint32_t*>(p.bar + 2);
  const bool trace_idx = do_glue && (p.trace.idx || p.trace.count);

  if (t == 0) {
    for (int s = 0; s < kItems; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], kConsumerWarps);
    }
    mbar_init(&sm.list_ready, 1);
    mbar_init(&sm.layer_start, 1);
    for (int e = 0; e < kMaxList; ++e) sm.hflag[e] = 0;
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
            while (!mbar_try_wait(eb, par)) {
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
        if (do_pred && p.gate_producer && l > 0) {
          // experiment: keep the producer quiet until the consumers start this layer
          const uint64_t t0 = wait_start();
          while (!mbar_try_wait(&sm.layer_start, (uint32_t)(l & 1))) {
            if (aborted(sm)) { ok = false; break; }
            if (timed_out(t0, p.wait_cycles)) { set_abort(sm, p.err, DEV_ERR_RING_TIMEOUT); ok = false; break; }
          }
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
          while (!mbar_try_wait(&sm.list_ready, (uint32_t)(l & 1))) {
            if (aborted(sm)) { ok = false; break; }
            if (timed_out(t0, p.wait_cycles)) { set_abort(sm, p.err, DEV_ERR_RING_TIMEOUT); ok = false; break; }
          }
          pstamp(p, l, 10);
          const int n = ok ? sm.nlist : 0;
          // Ask HBM for every record of the block at once (L2 prefetch needs no shared
          // memory); the ring copies below then find them in L2 as space frees up.
          for (int e = 0; e < n && ok; ++e)
            prefetch_l2_bulk(Ld.rec + (size_t)sm.list[e] * p.rec_stride, (uint32_t)p.rec_stride);
          // Warm L2 with the next layer's predictor rows of this block while this layer's
          // records stream: that bulk traffic then lands in the F phase instead of slowing
          // the cross-block exchanges that follow it, and the ring copies of those rows
          // later come from L2.  The prefetches are issued after the first records.
          const bool warm = do_pred && l + 1 < p.L;
          const int first_recs = min(n, 2);
          for (int e = 0; e < first_recs && ok; ++e) {
            if (!(ok = begin_item((uint32_t)p.rec_stride, dst, fb))) break;
            bulk_g2s(dst, Ld.rec + (size_t)sm.list[e] * p.rec_stride, (uint32_t)p.rec_stride, fb);
          }
          if (warm && ok) {
            const LayerDev Ln = p.layers[l + 1];
            if (k1 > k0) prefetch_l2_bulk(Ln.p1t + (size_t)k0 * p.p1_row, (uint32_t)(k1 - k0) * p.p1_row);
            if (nown > 0)
              prefetch_l2_bulk(Ln.p2o + (size_t)c * p.nown_max * p.p2_stride, (uint32_t)nown * p.p2_stride);
          }
          for (int e = first_recs; e < n && ok; ++e) {
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
        while (!mbar_try_wait(fb, par)) {
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

  for (int l = 0; l < p.L; ++l) {
    const uint32_t tag_u = tag_of(epoch, l, 0), tag_p = tag_of(epoch, l, 1), tag_v = tag_of(epoch, l, 2),
                   tag_b = tag_of(epoch, l, 3);
    int nlist = 0;
    stamp(p, l, 0);
    if (t == 0) mbar_arrive(&sm.layer_start);

    if (do_pred) {
      // ---------------------------------------------------------- P-a: u rows, a warp per row
      for (int k = k0; k < k1; k += p.p1_rows_per_item) {
        const int n = min(p.p1_rows_per_item, k1 - k);
        const uint8_t* item = ring_next(ring, (uint32_t)n * p.p1_row);
        ring_wait_item(ring.item, sm, p);
        if (k == k0) stamp(p, l, 13);
        for (int kk = warp; kk < n; kk += kConsumerWarps) {
          float acc[NB];
          warp_dot_p<FAM, NB>(item + (size_t)kk * p.p1_row, xs, d, acc);
          if (lane < B) {
            float v = acc[0];
#pragma unroll
            for (int b = 1; b < NB; ++b) if (lane == b) v = acc[b];
            st_tag(p.ux + (size_t)lane * r + k + kk, v, tag_u);
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

      // ---------------------------------------------------------- P-b: own logits, 4 rows per warp
      const int rchunks = r * PB / 16;
      for (int m0 = 0; m0 < nown; m0 += p.p2_rows_per_item) {
        const int n = min(p.p2_rows_per_item, nown - m0);
        const uint8_t* item = ring_next(ring, (uint32_t)n * p.p2_stride);
        ring_wait_item(ring.item, sm, p);
        if (m0 == 0) stamp(p, l, 12);
        for (int mb = warp * 4; mb < n; mb += kConsumerWarps * 4) {
          float acc[4][NB];
#pragma unroll
          for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int b = 0; b < NB; ++b) acc[i][b] = 0.f;
          for (int q = lane; q < rchunks; q += 32) {
            if constexpr (PB == 4) {
              float4 uu[NB];
#pragma unroll
              for (int b = 0; b < NB; ++b) uu[b] = *reinterpret_cast<const float4*>(u_s + b * r + 4 * q);
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                if (mb + i < n) {
                  const float4 w = *reinterpret_cast<const float4*>(item + (size_t)(mb + i) * p.p2_stride + 16 * q);
#pragma unroll
                  for (int b = 0; b < NB; ++b)
                    acc[i][b] = fmaf(w.x, uu[b].x, fmaf(w.y, uu[b].y, fmaf(w.z, uu[b].z, fmaf(w.w, uu[b].w, acc[i][b]))));
                }
              }
            } else {
              float4 u0[NB], u1[NB];
#pragma unroll
              for (int b = 0; b < NB; ++b) {
                u0[b] = *reinterpret_cast<const float4*>(u_s + b * r + 8 * q);
                u1[b] = *reinterpret_cast<const float4*>(u_s + b * r + 8 * q + 4);
              }
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                if (mb + i < n) {
                  const uint4 w = *reinterpret_cast<const uint4*>(item + (size_t)(mb + i) * p.p2_stride + 16 * q);
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
          }
#pragma unroll
          for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int b = 0; b < NB; ++b) acc[i][b] = warp_sum(acc[i][b]);
          if (lane < 4 && mb + lane < n) {
            const int m = mb + lane;
            const uint8_t* prow = item + (size_t)m * p.p2_stride;
            const float ti = *reinterpret_cast<const float*>(prow + (size_t)r * PB);
            const int i = c + (m0 + m) * G;
            uint32_t bits = 0;
#pragma unroll
            for (int b = 0; b < NB; ++b) {
              float lgv = acc[0][b];
#pragma unroll
              for (int ii = 1; ii < 4; ++ii) if (lane == ii) lgv = acc[ii][b];
              if (b < B) {
                const float lg = lgv - ti;
                if (lg > 0.f) bits |= 1u << b;
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

      // ---------------------------------------------------------- bitmap exchange
      // publish this block's per-token bitmap words (bit m of word m/32 = own neuron m)
      for (int qb = warp; qb < W * B; qb += kConsumerWarps) {
        const int q = qb % W, b = qb / W;
        const int m = 32 * q + lane;
        const uint32_t bit = (m < nown) ? ((sm.own_bits[m] >> b) & 1u) : 0u;
        const uint32_t word = __ballot_sync(0xffffffffu, bit != 0);
        if (lane == 0) st_tag_u(p.bx + ((size_t)b * G + c) * W + q, word, tag_b);
      }
      for (int base = 0; base < B * G * W; base += 8 * kConsumerThreads) {
        uint64_t w[8];
        poll_words<8>(p.bx + base, t, kConsumerThreads, B * G * W - base, tag_b, w, sm, p);
#pragma unroll
        for (int k = 0; k < 8; ++k)
          if (base + t + k * kConsumerThreads < B * G * W) bm[base + t + k * kConsumerThreads] = (uint32_t)w[k];
      }
      named_bar_sync(kRedBar, kConsumerThreads);
      stamp(p, l, 14);
      // active count per owner block (union over tokens), prefix over blocks
      if (t < G) {
        int n = 0;
        for (int q = 0; q < W; ++q) {
          uint32_t un = 0;
          for (int b = 0; b < B; ++b) un |= bm[((size_t)b * G + t) * W + q];
          n += __popc(un);
        }
        sm.cstart[t + 1] = n;
      }
      named_bar_sync(kRedBar, kConsumerThreads);
      if (warp == 0) {   // inclusive scan over the G (<= kMaxGrid) block counts
        int carry = 0;
        for (int c0 = 0; c0 < G; c0 += 32) {
          int v = (c0 + lane < G) ? sm.cstart[c0 + lane + 1] : 0;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, v, o);
            if (lane >= o) v += u;
          }
          if (c0 + lane < G) sm.cstart[c0 + lane + 1] = v + carry;
          carry += __shfl_sync(0xffffffffu, v, 31);
        }
        if (lane == 0) { sm.cstart[0] = 0; sm.count = carry; }
      }
      named_bar_sync(kRedBar, kConsumerThreads);
      stamp(p, l, 15);
      const int count = sm.count;
      // this block's even share of the active neurons, in (owner block, owner position) order
      const int a0 = (int)((long long)c * count / G), a1 = (int)((long long)(c + 1) * count / G);
      nlist = min(a1 - a0, kMaxList);
      if (t < G && sm.cstart[t] < a1 && sm.cstart[t + 1] > a0) {
        int pos = sm.cstart[t];
        for (int q = 0; q < W && pos < a1; ++q) {
          uint32_t un = 0;
          for (int b = 0; b < B; ++b) un |= bm[((size_t)b * G + t) * W + q];
          while (un && pos < a1) {
            const int bit = __ffs(un) - 1;
            un &= un - 1;
            if (pos >= a0 && pos - a0 < kMaxList) {
              const int m = 32 * q + bit;
              const int e = pos - a0;
              uint32_t tb = 0;
              for (int b = 0; b < B; ++b) tb |= ((bm[((size_t)b * G + t) * W + q] >> bit) & 1u) << b;
              sm.list[e] = t + m * G;
              sm.list_bits[e] = (uint8_t)tb;
            }
            ++pos;
          }
        }
      }
      if (t == 0 && c == 0 && do_ffn) {
        atomicAdd(p.active_total, (unsigned long long)count);
        if (p.layer_count) p.layer_count[l] = count;
      }
      if (t == 0 && a1 - a0 > kMaxList) atomicExch(p.err, DEV_ERR_LIST);
      // mask words (predict output or trace): block c assembles words w = c, c+G, ...
      uint32_t* mask_dst = do_glue ? (p.trace.mask ? p.trace.mask + (size_t)l * B * words : nullptr) : p.mask_out;
      if (mask_dst) {
        for (int wb = c + G * warp; wb < words * B; wb += G * kConsumerWarps) {
          const int b = wb / words, w = wb % words;
          const int i = 32 * w + lane;
          const int oc = i % G, om = i / G;
          const uint32_t bit = (bm[((size_t)b * G + oc) * W + (om >> 5)] >> (om & 31)) & 1u;
          const uint32_t word = __ballot_sync(0xffffffffu, bit != 0);
          if (lane == 0) mask_dst[(size_t)b * words + w] = word;
        }
      }
      // trace: ascending index list and count of the layer (the union over tokens)
      if (trace_idx && c == 0) {
        int base = 0;
        for (int w0 = 0; w0 < words; w0 += kConsumerThreads) {
          const int w = w0 + t;
          uint32_t un = 0;
          if (w < words)
            for (int j = 0; j < 32; ++j) {
              const int i = 32 * w + j, oc = i % G, om = i / G;
              uint32_t bit = 0;
              for (int b = 0; b < B; ++b) bit |= (bm[((size_t)b * G + oc) * W + (om >> 5)] >> (om & 31)) & 1u;
              un |= bit << j;
            }
          const int cnt = __popc(un);
          int incl = cnt;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
          }
          if (lane == 31) sm.scan[warp] = incl;
          named_bar_sync(kRedBar, kConsumerThreads);
          int wb = 0, tot = 0;
          for (int q = 0; q < kConsumerWarps; ++q) { if (q < warp) wb += sm.scan[q]; tot += sm.scan[q]; }
          int pos = base + wb + incl - cnt;
          if (p.trace.idx)
            while (un) {
              const int bit = __ffs(un) - 1;
              un &= un - 1;
              p.trace.idx[(size_t)l * f + pos++] = w * 32 + bit;
            }
          base += tot;
          named_bar_sync(kRedBar, kConsumerThreads);
        }
        if (t == 0 && p.trace.count) p.trace.count[l] = base;
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
        sm.list_bits[e] = (uint8_t)bits;
      }
      if (t == 0) atomicAdd(p.active_total, (unsigned long long)nlist);
    }

    if (!do_ffn) break;   // predictor only
    named_bar_sync(kRedBar, kConsumerThreads);
    if (t == 0) {
      sm.nlist = nlist;
      mbar_arrive(&sm.list_ready);
    }
    stamp(p, l, 3);

    // ------------------------------------------------------------ F: gather + scatter in batches
    float y[NB][NU][UE];
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
      for (int j = 0; j < NU; ++j)
#pragma unroll
        for (int e = 0; e < UE; ++e) y[b][j][e] = 0.f;
    // Records stream through the ring in windows of p.batch; warp k of a window forms the
    // dot products of its record and flags h, and every warp adds each record's down row
    // as soon as that record's h is flagged (no block-wide barrier in between).
    const int hval = l + 1;
    for (int e0 = 0; e0 < nlist; e0 += p.batch) {
      const int nb = min(p.batch, nlist - e0);
      uint32_t rpos[kMaxBatch];
      const uint32_t item0 = ring.item;
#pragma unroll
      for (int k = 0; k < kMaxBatch; ++k)
        rpos[k] = (k < nb) ? (uint32_t)(ring_next(ring, (uint32_t)p.rec_stride) - ring.base) : 0u;
      if (warp < nb) {
        uint32_t pos = rpos[0];
#pragma unroll
        for (int k = 1; k < kMaxBatch; ++k) if (warp == k) pos = rpos[k];
        const uint8_t* rec = ring.base + pos;
        ring_wait_item(item0 + warp, sm, p);
        if (e0 == 0 && warp == 0) stamp(p, l, 5);
        float ua[NB], ga[NB];
        if constexpr (ACT == PI_REGLU) {
          warp_dot_w2<FAM, NB>(rec + p.up_off, rec + p.gate_off, xs, d, ua, ga);
        } else {
          warp_dot_w<FAM, NB>(rec + p.up_off, xs, d, ua);
#pragma unroll
          for (int b = 0; b < NB; ++b) ga[b] = 0.f;
        }
        if (lane == 0) {
          const int e = e0 + warp;
          const uint32_t bits = sm.list_bits[e];
          const float bi = *reinterpret_cast<const float*>(rec + p.bias_off);
#pragma unroll
          for (int b = 0; b < NB; ++b) {
            float a;
            if constexpr (ACT == PI_REGLU) a = fmaxf(ga[b] + bi, 0.f) * ua[b];
            else a = fmaxf(ua[b] + bi, 0.f);
            sm.hbuf[e][b] = ((bits >> b) & 1u) ? a : 0.f;
          }
          __threadfence_block();
          *(volatile int*)&sm.hflag[e] = hval;
        }
        __syncwarp();
      }
      for (int k = 0; k < nb; ++k) {
        uint32_t pos = rpos[0];
#pragma unroll
        for (int kk = 1; kk < kMaxBatch; ++kk) if (k == kk) pos = rpos[kk];
        const int e = e0 + k;
        if (*(volatile int*)&sm.hflag[e] != hval) {
          const uint64_t t0 = wait_start();
          while (*(volatile int*)&sm.hflag[e] != hval) {
            if (aborted(sm)) break;
            if (timed_out(t0, p.wait_cycles)) { set_abort(sm, p.err, DEV_ERR_RING_TIMEOUT); break; }
          }
        }
        __threadfence_block();
        ring_wait_item(item0 + k, sm, p);   // completed already: makes the data visible here
        float h[NB];
#pragma unroll
        for (int b = 0; b < NB; ++b) h[b] = sm.hbuf[e][b];
        axpy_units<FAM, NB, NU>(ring.base + pos + p.down_off, nunits, d, h, y);
        ring_release_item(item0 + k, sm);
      }
      ring.item = item0 + nb;
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
            for (int e = 0; e < UE; e += 2) st_tag2(dst + e, y[b][j][e], y[b][j][e + 1], tag_p);
          }
        }
    }
    stamp(p, l, 4);

    // ------------------------------------------------------------ R: slice reduce
    if (slice_owner) {
      // warp w sums partial rows cc = w, w+8, ...; KU rows' words are read together so
      // the L2 round trips overlap; sums run in ascending cc (fixed order)
      constexpr int KU = 20 / NB;
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
#pragma unroll
            for (int k = 0; k < KU; ++k)
#pragma unroll
              for (int b = 0; b < NB; ++b)
                if (need >> (k * NB + b) & 1u) {
                  const int cc = cc0 + kConsumerWarps * k;
                  const uint64_t w = ld_tag(p.px + ((size_t)cc * B + b) * d + col0 + 32 * gq + lane);
                  if (tag_ok(w, tag_p)) { tmp[k][b] = tag_val(w); need &= ~(1u << (k * NB + b)); }
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

    // ------------------------------------------------------------ glue: x' = v / rms
    {
      if (warp < NB) {
        float s = 0.f;
        float s2 = 0.f;
        if (warp < B) {
          // words (sum, sum of squares) of every slice, interleaved: even lanes read sums,
          // odd lanes sums of squares (32 is even, so a lane keeps its parity)
          uint64_t w[2 * kMaxGrid / 32];
          poll_words<2 * kMaxGrid / 32>(p.sx + (size_t)warp * G * 2, lane, 32, 2 * nslices, tag_v, w, sm, p);
#pragma unroll
          for (int k = 0; k < 2 * kMaxGrid / 32; ++k)
            if (lane + 32 * k < 2 * nslices) s += tag_val(w[k]);
        }
        const float sum = warp_sum((lane & 1) ? 0.f : s);
        s2 = warp_sum((lane & 1) ? s : 0.f);
        if (lane == 0) {
          const float mean = sum / (float)d;
          const float var = fmaxf(s2 / (float)d - mean * mean, 0.f);
          sm.gmean[warp] = mean;
          sm.gsd[warp] = sqrtf(var + kRmsEps);
        }
      }
      named_bar_sync(kRedBar, kConsumerThreads);
      stamp(p, l, 16);   // rms known; every warp is done reading xs
      {
        const int npairs = B * d / 2;
        for (int base = 0; base < npairs; base += 8 * kConsumerThreads) {
          uint64_t w0[8], w1[8];
          uint32_t need = 0;
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            w0[k] = w1[k] = 0;
            if (base + t + k * kConsumerThreads < npairs) need |= 1u << k;
          }
          bool started = false;
          uint64_t tp = 0;
          while (need) {
#pragma unroll
            for (int k = 0; k < 8; ++k)
              if (need >> k & 1u) {
                ld_tag2(p.vx + 2 * (size_t)(base + t + k * kConsumerThreads), w0[k], w1[k]);
                if (tag_ok(w0[k], tag_v) && tag_ok(w1[k], tag_v)) need &= ~(1u << k);
              }
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

// Largest per-thread unit count of each (family, tokens) instantiation.
template <int FAM, int NB> struct NUof;
template <> struct NUof<FAM_F32, 1> { static constexpr int v = 2; };
template <> struct NUof<FAM_F32, 2> { static constexpr int v = 2; };
template <> struct NUof<FAM_F32, 4> { static constexpr int v = 2; };
template <> struct NUof<FAM_F16, 1> { static constexpr int v = 3; };
template <> struct NUof<FAM_F16, 2> { static constexpr int v = 2; };
template <> struct NUof<FAM_F16, 4> { static constexpr int v = 1; };
template <> struct NUof<FAM_Q4, 1> { static constexpr int v = 1; };
template <> struct NUof<FAM_Q4, 2> { static constexpr int v = 1; };

constexpr int ue_of(int fam) { return fam == FAM_F32 ? 4 : fam == FAM_F16 ? 8 : 32; }

int nu_max(int fam, int nb) {
  switch (fam) {
    case FAM_F32: return 2;
    case FAM_F16: return nb == 1 ? 3 : nb == 2 ? 2 : 1;
    case FAM_Q4: return nb <= 2 ? 1 : 0;
  }
  return 0;
}

int nb_of(int B) { return B <= 1 ? 1 : B <= 2 ? 2 : B <= 4 ? 4 : 0; }

template <int FAM, int ACT, int NB>
cudaError_t launch_t(const FusedParams& p, size_t smem, cudaStream_t stream) {
  auto kern = fused_kernel<FAM, ACT, NB, NUof<FAM, NB>::v>;
  static int configured = 0;   // the attribute is per function; raise it when a launch needs more
  if ((int)smem > configured) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    configured = (int)smem;
  }
  void* args[] = {const_cast<FusedParams*>(&p)};
  return cudaLaunchCooperativeKernel((const void*)kern, dim3(p.grid), dim3(kThreads), args, smem, stream);
}

template <int FAM, int ACT>
cudaError_t launch_nb(int B, const FusedParams& p, size_t smem, cudaStream_t stream) {
  switch (nb_of(B)) {
    case 1: return launch_t<FAM, ACT, 1>(p, smem, stream);
    case 2: return launch_t<FAM, ACT, 2>(p, smem, stream);
    case 4:
      if constexpr (FAM != FAM_Q4) return launch_t<FAM, ACT, 4>(p, smem, stream);
      else return cudaErrorNotSupported;
  }
  return cudaErrorNotSupported;
}

}  // namespace

bool fused_supported(int family, int B, int d) {
  const int nb = nb_of(B);
  if (nb == 0) return false;
  const int nu = nu_max(family, nb);
  if (nu == 0) return false;
  return d <= nu * ue_of(family) * kConsumerThreads;
}

size_t fused_fixed_smem(int B, int d, int r, int grid, int nown_max, int family) {
  const int nb = nb_of(B) ? nb_of(B) : 4;
  const size_t xbytes = family == FAM_F32 ? 4 : 2;
  const size_t W = (size_t)(nown_max + 31) / 32;
  return ((sizeof(Smem) + 127) / 128) * 128 + (size_t)nb * d * xbytes + (size_t)nb * r * sizeof(float) +
         (size_t)kConsumerWarps * nb * kMaxColGroups * 32 * sizeof(float) + (size_t)nb * grid * W * 4 + 128;
}

int fused_max_batch() { return kMaxBatch; }

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
