// The fused persistent kernel of the activation-sparse FFN decode path.
//
// One block per SM, 8 consumer warps + 1 producer warp.  The producer streams every
// byte the block needs (predictor rows, then the active neurons' weight rows) from HBM
// into a ring of shared-memory slots with bulk copies completing on mbarriers.  It runs
// ahead of the consumers as far as the ring allows, so the next layer's predictor rows
// are already in flight while the consumers sit in grid barriers.
//
// Per layer (stack mode), for block c of G:
//   P-a  u_k = P1^T[k] . x for the block's rank rows k            -> u (global)
//        grid barrier
//   P-b  logit_i = P2^T[i] . u - t_i for the block's own neurons i = c, c+G, c+2G, ...
//        bit = logit > 0; the mask word bits are published with atomicOr
//   F    for each own neuron whose bit is set for some token (ascending i):
//          ReLU : h = max(0, w_up_i . x + b_i)          ReGLU: max(0, w_gate_i . x + b_i) * (w_up_i . x)
//          h[b] = 0 where token b's bit is 0;  y_partial += h * w_down_i (registers, fp32)
//        y_partial -> partials[c]; grid barrier
//   R    block s < nslices owns a column slice: v = x + sum_c partials[c] (fixed order),
//        sum of squares of the slice; grid barrier
//   glue x' = v / sqrt(sum_s ssq_s / d + 1e-6), rounded to the activation dtype
// Owning neurons at neuron granularity (i mod G) lets a block start gathering its active
// rows as soon as its own logits are known, with no global compaction in between, and
// spreads the frequently firing neurons evenly over the blocks.  Every reduction runs in
// a fixed order, so results are bitwise reproducible.
#include <cuda_fp16.h>
#include <cstdint>

#include "pi_internal.h"
#include "pi_ptx.cuh"

namespace pi {

namespace {

constexpr float kRmsEps = 1e-6f;
constexpr int kRedBar = 1;          // named barrier id among consumers
constexpr int kMaxColGroups = 4;    // 32-column groups per reduce slice

template <int FAM> struct Fam;
template <> struct Fam<FAM_F32> { static constexpr int UE = 4;  static constexpr int PB = 4; };
template <> struct Fam<FAM_F16> { static constexpr int UE = 8;  static constexpr int PB = 2; };
template <> struct Fam<FAM_Q4>  { static constexpr int UE = 32; static constexpr int PB = 2; };

struct Smem {
  uint64_t full[kMaxSlots];
  uint64_t empty[kMaxSlots];
  uint64_t list_ready;
  int abort_flag;
  int nlist;
  int nown;
  int pad0;
  float red[2][kConsumerWarps][8];
  float rms[4];
  int32_t list[kMaxList];
  float list_bias[kMaxList];
  uint8_t list_bits[kMaxList];
  uint8_t own_bits[kMaxOwn];
  float own_bias[kMaxOwn];
  int scan[kConsumerThreads / 32 + 1];
};

__device__ __forceinline__ bool timed_out(uint64_t t0, long long limit) {
  return (long long)(globaltimer_ns() - t0) > limit;
}

// ------------------------------------------------------------------ ring (consumer side)
struct Ring {
  uint8_t* base;
  int slot_bytes;
  int nslots;
  uint32_t seq;
  __device__ uint8_t* slot(uint32_t s) const { return base + (size_t)(s % nslots) * slot_bytes; }
};

__device__ __forceinline__ uint8_t* ring_wait(Ring& r, Smem& sm, uint32_t s, long long limit, int* err) {
  uint64_t* bar = &sm.full[s % r.nslots];
  uint32_t par = (s / r.nslots) & 1u;
  if (!sm.abort_flag) {
    if (!mbar_try_wait(bar, par)) {
      uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(bar, par)) {
        if (*(volatile int*)&sm.abort_flag) break;
        if (timed_out(t0, limit)) {
          atomicExch(err, DEV_ERR_RING_TIMEOUT);
          *(volatile int*)&sm.abort_flag = 1;
          break;
        }
      }
    }
  }
  return r.slot(s);
}
__device__ __forceinline__ void ring_release(Ring& r, Smem& sm, uint32_t s) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(&sm.empty[s % r.nslots]);
}

// ------------------------------------------------------------------ grid barrier
__device__ bool grid_barrier(const FusedParams& p, Smem& sm, uint32_t& epoch) {
  named_bar_sync(kRedBar, kConsumerThreads);
  ++epoch;
  if (threadIdx.x == 0 && !sm.abort_flag) {
    const uint32_t target = epoch * (uint32_t)gridDim.x + (uint32_t)p.barrier_extra;
    red_release_gpu_add(p.bar, 1u);
    if (ld_acquire_gpu(p.bar) < target) {
      uint64_t t0 = globaltimer_ns();
      while (ld_acquire_gpu(p.bar) < target) {
        if (timed_out(t0, p.barrier_timeout_ns)) {
          atomicExch(p.err, DEV_ERR_GRID_TIMEOUT);
          *(volatile int*)&sm.abort_flag = 1;
          break;
        }
      }
    }
  }
  named_bar_sync(kRedBar, kConsumerThreads);
  return !sm.abort_flag;
}

// ------------------------------------------------------------------ reductions
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Sum NV values over the 256 consumer threads; every consumer gets the totals.
template <int NV>
__device__ __forceinline__ void block_sum(float (&v)[NV], Smem& sm, int& buf) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
  for (int i = 0; i < NV; ++i) v[i] = warp_sum(v[i]);
  if (lane == 0) {
#pragma unroll
    for (int i = 0; i < NV; ++i) sm.red[buf][warp][i] = v[i];
  }
  named_bar_sync(kRedBar, kConsumerThreads);
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) s += sm.red[buf][w][i];
    v[i] = s;
  }
  buf ^= 1;
}

// ------------------------------------------------------------------ per-thread row math
// A weight row (d elements) is split in units of UE elements (16 bytes of fp32/fp16
// weights, or one 32-weight Q4_0 block).  Consumer thread t owns units t + 256*j.
template <int FAM, int NB, int NU>
struct RowMath {
  static constexpr int UE = Fam<FAM>::UE;

  // dot of a weight row with x for every token
  __device__ static void dot(const uint8_t* row, int nunits, int d, const float (&x)[NB][NU][UE],
                             float (&acc)[NB]) {
    const int t = threadIdx.x;
#pragma unroll
    for (int j = 0; j < NU; ++j) {
      const int q = t + kConsumerThreads * j;
      if (q < nunits) {
        if constexpr (FAM == FAM_F32) {
          const float4 w = *reinterpret_cast<const float4*>(row + 16 * q);
#pragma unroll
          for (int b = 0; b < NB; ++b)
            acc[b] += w.x * x[b][j][0] + w.y * x[b][j][1] + w.z * x[b][j][2] + w.w * x[b][j][3];
        } else if constexpr (FAM == FAM_F16) {
          const uint4 w = *reinterpret_cast<const uint4*>(row + 16 * q);
          const float2 a = h2f2(w.x), bb = h2f2(w.y), c = h2f2(w.z), e = h2f2(w.w);
#pragma unroll
          for (int b = 0; b < NB; ++b)
            acc[b] += a.x * x[b][j][0] + a.y * x[b][j][1] + bb.x * x[b][j][2] + bb.y * x[b][j][3] +
                      c.x * x[b][j][4] + c.y * x[b][j][5] + e.x * x[b][j][6] + e.y * x[b][j][7];
        } else {
          const uint4 nb = *reinterpret_cast<const uint4*>(row + 16 * q);
          const float s = __half2float(*reinterpret_cast<const __half*>(row + (d >> 1) + 2 * q));
          const uint32_t wv[4] = {nb.x, nb.y, nb.z, nb.w};
          float part[NB];
#pragma unroll
          for (int b = 0; b < NB; ++b) part[b] = 0.f;
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            const uint32_t lo = wv[m] & 0x0F0F0F0Fu, hi = (wv[m] >> 4) & 0x0F0F0F0Fu;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              // 2^23 + code as a float, minus 2^23 + 8: exactly (code - 8)
              const float cl = __uint_as_float(__byte_perm(lo, 0x4B000000u, 0x7540 + k)) - 8388616.f;
              const float ch = __uint_as_float(__byte_perm(hi, 0x4B000000u, 0x7540 + k)) - 8388616.f;
#pragma unroll
              for (int b = 0; b < NB; ++b)
                part[b] += cl * x[b][j][4 * m + k] + ch * x[b][j][4 * m + k + 16];
            }
          }
#pragma unroll
          for (int b = 0; b < NB; ++b) acc[b] += s * part[b];
        }
      }
    }
  }

  // y += h * row for every token
  __device__ static void axpy(const uint8_t* row, int nunits, int d, const float (&h)[NB],
                              float (&y)[NB][NU][UE]) {
    const int t = threadIdx.x;
#pragma unroll
    for (int j = 0; j < NU; ++j) {
      const int q = t + kConsumerThreads * j;
      if (q < nunits) {
        if constexpr (FAM == FAM_F32) {
          const float4 w = *reinterpret_cast<const float4*>(row + 16 * q);
#pragma unroll
          for (int b = 0; b < NB; ++b) {
            y[b][j][0] += h[b] * w.x; y[b][j][1] += h[b] * w.y;
            y[b][j][2] += h[b] * w.z; y[b][j][3] += h[b] * w.w;
          }
        } else if constexpr (FAM == FAM_F16) {
          const uint4 w = *reinterpret_cast<const uint4*>(row + 16 * q);
          const float2 a = h2f2(w.x), bb = h2f2(w.y), c = h2f2(w.z), e = h2f2(w.w);
#pragma unroll
          for (int b = 0; b < NB; ++b) {
            y[b][j][0] += h[b] * a.x;  y[b][j][1] += h[b] * a.y;
            y[b][j][2] += h[b] * bb.x; y[b][j][3] += h[b] * bb.y;
            y[b][j][4] += h[b] * c.x;  y[b][j][5] += h[b] * c.y;
            y[b][j][6] += h[b] * e.x;  y[b][j][7] += h[b] * e.y;
          }
        } else {
          const uint4 nb = *reinterpret_cast<const uint4*>(row + 16 * q);
          const float s = __half2float(*reinterpret_cast<const __half*>(row + (d >> 1) + 2 * q));
          const uint32_t wv[4] = {nb.x, nb.y, nb.z, nb.w};
          float hs[NB];
#pragma unroll
          for (int b = 0; b < NB; ++b) hs[b] = h[b] * s;
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            const uint32_t lo = wv[m] & 0x0F0F0F0Fu, hi = (wv[m] >> 4) & 0x0F0F0F0Fu;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const float cl = __uint_as_float(__byte_perm(lo, 0x4B000000u, 0x7540 + k)) - 8388616.f;
              const float ch = __uint_as_float(__byte_perm(hi, 0x4B000000u, 0x7540 + k)) - 8388616.f;
#pragma unroll
              for (int b = 0; b < NB; ++b) {
                y[b][j][4 * m + k] += hs[b] * cl;
                y[b][j][4 * m + k + 16] += hs[b] * ch;
              }
            }
          }
        }
      }
    }
  }

  // dot of a P1^T row (p dtype) with x, using the x unit layout of the family
  __device__ static void dot_p1(const uint8_t* row, int nunits, const float (&x)[NB][NU][UE],
                                float (&acc)[NB]) {
    const int t = threadIdx.x;
    if constexpr (FAM == FAM_F32 || FAM == FAM_F16) {
      // same element type and unit layout as the weight rows
      dot(row, nunits, 0, x, acc);
    } else {
#pragma unroll
      for (int j = 0; j < NU; ++j) {
        const int q = t + kConsumerThreads * j;
        if (q < nunits) {
#pragma unroll
          for (int i0 = 0; i0 < 4; ++i0) {
            const int i = (i0 + t) & 3;   // rotate the 16-byte chunk order across threads
            const uint4 w = *reinterpret_cast<const uint4*>(row + 64 * q + 16 * i);
            const float2 a = h2f2(w.x), bb = h2f2(w.y), c = h2f2(w.z), e = h2f2(w.w);
#pragma unroll
            for (int b = 0; b < NB; ++b) {
              const float* xv = &x[b][j][8 * i];
              acc[b] += a.x * xv[0] + a.y * xv[1] + bb.x * xv[2] + bb.y * xv[3] + c.x * xv[4] +
                        c.y * xv[5] + e.x * xv[6] + e.y * xv[7];
            }
          }
        }
      }
    }
  }
};

// load x (activation dtype, [B][d]) into the thread's units, rounding already applied
template <int FAM, int NB, int NU>
__device__ __forceinline__ void load_x(const void* src, int B, int d, float (&x)[NB][NU][Fam<FAM>::UE]) {
  constexpr int UE = Fam<FAM>::UE;
  const int nunits = d / UE;
  const int t = threadIdx.x;
#pragma unroll
  for (int b = 0; b < NB; ++b)
#pragma unroll
    for (int j = 0; j < NU; ++j) {
      const int q = t + kConsumerThreads * j;
#pragma unroll
      for (int e = 0; e < UE; ++e) x[b][j][e] = 0.f;
      if (b < B && q < nunits) {
        if constexpr (FAM == FAM_F32) {
          const float4 v = reinterpret_cast<const float4*>(src)[(size_t)b * (d / 4) + q];
          x[b][j][0] = v.x; x[b][j][1] = v.y; x[b][j][2] = v.z; x[b][j][3] = v.w;
        } else {
          const __half* hp = reinterpret_cast<const __half*>(src) + (size_t)b * d + (size_t)q * UE;
#pragma unroll
          for (int e = 0; e < UE; e += 8) {
            const uint4 w = *reinterpret_cast<const uint4*>(hp + e);
            const float2 a = h2f2(w.x), bb = h2f2(w.y), c = h2f2(w.z), f = h2f2(w.w);
            x[b][j][e + 0] = a.x;  x[b][j][e + 1] = a.y;  x[b][j][e + 2] = bb.x; x[b][j][e + 3] = bb.y;
            x[b][j][e + 4] = c.x;  x[b][j][e + 5] = c.y;  x[b][j][e + 6] = f.x;  x[b][j][e + 7] = f.y;
          }
        }
      }
    }
}

__device__ __forceinline__ int slice_begin(int s, int ns, int ngroups) { return (int)((long long)s * ngroups / ns) * 32; }

// ------------------------------------------------------------------ the kernel
template <int FAM, int ACT, int NB, int NU>
__global__ void __launch_bounds__(kThreads, 1) fused_kernel(const FusedParams p) {
  constexpr int UE = Fam<FAM>::UE;
  constexpr int PB = Fam<FAM>::PB;
  extern __shared__ __align__(128) uint8_t dsmem[];
  Smem& sm = *reinterpret_cast<Smem*>(dsmem);
  uint8_t* ring_base = dsmem + ((sizeof(Smem) + 127) / 128) * 128;
  float* u_s = reinterpret_cast<float*>(ring_base + (size_t)p.nslots * p.slot_bytes);   // [NB][r]
  float* red2 = u_s + NB * p.r;                                                      // reduce scratch

  const int c = blockIdx.x, G = gridDim.x;
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const bool do_pred = p.mode & MODE_PREDICT, do_ffn = p.mode & MODE_FFN, do_glue = p.mode & MODE_GLUE;
  const int d = p.d, f = p.f, r = p.r, B = p.B;
  const int k0 = (int)((long long)c * r / G), k1 = (int)((long long)(c + 1) * r / G);
  const int nown = (c < f) ? (f - c + G - 1) / G : 0;
  const int nunits = d / UE;
  const int words = f / 32;

  if (t == 0) {
    for (int s = 0; s < p.nslots; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], kConsumerWarps);
    }
    mbar_init(&sm.list_ready, 1);
    sm.abort_flag = 0;
    sm.nlist = 0;
    mbar_fence_init();
  }
  __syncthreads();

  // ================================================================ producer warp
  if (warp == kConsumerWarps) {
    if (lane == 0) {
      uint32_t seq = 0;
      auto acquire = [&](uint32_t s) -> bool {
        if (s >= (uint32_t)p.nslots) {
          uint64_t* eb = &sm.empty[s % p.nslots];
          const uint32_t par = ((s / p.nslots) & 1u) ^ 1u;
          if (!mbar_try_wait(eb, par)) {
            uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(eb, par)) {
              if (*(volatile int*)&sm.abort_flag) return false;
              if (timed_out(t0, p.barrier_timeout_ns)) {
                atomicExch(p.err, DEV_ERR_RING_TIMEOUT);
                *(volatile int*)&sm.abort_flag = 1;
                return false;
              }
            }
          }
        }
        return !*(volatile int*)&sm.abort_flag;
      };
      auto issue = [&](const uint8_t* src, uint32_t bytes) -> bool {
        if (!acquire(seq)) return false;
        uint8_t* dst = ring_base + (size_t)(seq % p.nslots) * p.slot_bytes;
        uint64_t* fb = &sm.full[seq % p.nslots];
        mbar_arrive_expect_tx(fb, bytes);
        bulk_g2s(dst, src, bytes, fb);
        ++seq;
        return true;
      };
      bool ok = true;
      for (int l = 0; l < p.L && ok; ++l) {
        const LayerDev Ld = p.layers[l];
        if (do_pred) {
          for (int k = k0; k < k1 && ok; ++k) ok = issue(Ld.p1t + (size_t)k * p.p1_row, p.p1_row);
          for (int m0 = 0; m0 < nown && ok; m0 += p.rows_per_p2slot) {
            const int n = min(p.rows_per_p2slot, nown - m0);
            if (!acquire(seq)) { ok = false; break; }
            uint8_t* dst = ring_base + (size_t)(seq % p.nslots) * p.slot_bytes;
            uint64_t* fb = &sm.full[seq % p.nslots];
            mbar_arrive_expect_tx(fb, (uint32_t)(n * p.p2_stride));
            for (int m = 0; m < n; ++m) {
              const int i = c + (m0 + m) * G;
              bulk_g2s(dst + (size_t)m * p.p2_stride, Ld.p2n + (size_t)i * p.p2_stride, p.p2_stride, fb);
            }
            ++seq;
          }
        }
        if (do_ffn && ok) {
          // wait for the consumers' active list of this layer
          uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(&sm.list_ready, (uint32_t)(l & 1))) {
            if (*(volatile int*)&sm.abort_flag) { ok = false; break; }
            if (timed_out(t0, p.barrier_timeout_ns)) {
              atomicExch(p.err, DEV_ERR_RING_TIMEOUT);
              *(volatile int*)&sm.abort_flag = 1;
              ok = false;
              break;
            }
          }
          const int n = ok ? sm.nlist : 0;
          for (int e = 0; e < n && ok; ++e) {
            const uint8_t* rec = Ld.rec + (size_t)sm.list[e] * p.rec_stride;
            if (ACT == PI_REGLU) ok = issue(rec + p.gate_off, p.row_bytes);
            if (ok) ok = issue(rec + p.up_off, p.row_bytes);
            if (ok) ok = issue(rec + p.down_off, p.row_bytes);
          }
        }
      }
      // drain: never leave the block while a bulk copy may still write shared memory
      const uint32_t first = seq > (uint32_t)p.nslots ? seq - p.nslots : 0u;
      for (uint32_t s = first; s < seq; ++s) {
        uint64_t* fb = &sm.full[s % p.nslots];
        const uint32_t par = (s / p.nslots) & 1u;
        uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(fb, par)) {
          if (timed_out(t0, p.barrier_timeout_ns)) { atomicExch(p.err, DEV_ERR_RING_TIMEOUT); break; }
        }
      }
    }
    return;
  }

  // ================================================================ consumers
  Ring ring{ring_base, p.slot_bytes, p.nslots, 0};
  uint32_t epoch = 0;
  int rbuf = 0;
  float x[NB][NU][UE];
  load_x<FAM, NB, NU>(p.x_in, B, d, x);

  const int ngroups = d / 32;
  const int nslices = p.nslices;
  const bool slice_owner = c < nslices;
  const int col0 = slice_owner ? slice_begin(c, nslices, ngroups) : 0;
  const int col1 = slice_owner ? slice_begin(c + 1, nslices, ngroups) : 0;

  // layer-0 input into the trace and, for the residual, into the fp32 input buffer xb[0]
  if (do_glue && slice_owner) {
    for (int idx = t; idx < B * (col1 - col0); idx += kConsumerThreads) {
      const int b = idx / (col1 - col0), j = col0 + idx % (col1 - col0);
      float xv;
      if constexpr (FAM == FAM_F32) xv = reinterpret_cast<const float*>(p.x_in)[(size_t)b * d + j];
      else xv = __half2float(reinterpret_cast<const __half*>(p.x_in)[(size_t)b * d + j]);
      p.xb[(size_t)b * d + j] = xv;
      if (p.trace.x) {
        if constexpr (FAM == FAM_F32) reinterpret_cast<float*>(p.trace.x)[(size_t)b * d + j] = xv;
        else reinterpret_cast<__half*>(p.trace.x)[(size_t)b * d + j] = __float2half_rn(xv);
      }
    }
  }
  // the first layer's mask buffer starts at zero
  if (do_glue) {
    const int w0 = (int)((long long)c * words * B / G), w1 = (int)((long long)(c + 1) * words * B / G);
    for (int w = w0 + t; w < w1; w += kConsumerThreads) p.maskbuf[w] = 0u;
  }

  for (int l = 0; l < p.L; ++l) {
    const LayerDev Ld = p.layers[l];
    uint32_t* mask_l = do_glue ? p.maskbuf + (size_t)(l & 1) * B * words : p.mask_out;
    int nlist = 0;

    if (do_pred) {
      // ---------------------------------------------------------- P-a: u rows
      for (int k = k0; k < k1; ++k) {
        const uint8_t* row = ring_wait(ring, sm, ring.seq, p.barrier_timeout_ns, p.err);
        float acc[NB];
#pragma unroll
        for (int b = 0; b < NB; ++b) acc[b] = 0.f;
        RowMath<FAM, NB, NU>::dot_p1(row, nunits, x, acc);
        ring_release(ring, sm, ring.seq++);
        block_sum<NB>(acc, sm, rbuf);
        if (t == 0) {
#pragma unroll
          for (int b = 0; b < NB; ++b)
            if (b < B) p.u[(size_t)b * r + k] = acc[b];
        }
      }
      grid_barrier(p, sm, epoch);
      for (int idx = t; idx < B * r; idx += kConsumerThreads) u_s[idx] = __ldcg(p.u + idx);
      if (do_glue) {   // zero the next layer's mask buffer (read by nobody until then)
        uint32_t* nxt = p.maskbuf + (size_t)((l + 1) & 1) * B * words;
        const int w0 = (int)((long long)c * words * B / G), w1 = (int)((long long)(c + 1) * words * B / G);
        for (int w = w0 + t; w < w1; w += kConsumerThreads) nxt[w] = 0u;
      }
      named_bar_sync(kRedBar, kConsumerThreads);

      // ---------------------------------------------------------- P-b: own logits
      const int rchunks = r * PB / 16;
      for (int m0 = 0; m0 < nown; m0 += p.rows_per_p2slot) {
        const int n = min(p.rows_per_p2slot, nown - m0);
        const uint8_t* slot = ring_wait(ring, sm, ring.seq, p.barrier_timeout_ns, p.err);
        for (int m = warp; m < n; m += kConsumerWarps) {
          const uint8_t* prow = slot + (size_t)m * p.p2_stride;
          float acc[NB];
#pragma unroll
          for (int b = 0; b < NB; ++b) acc[b] = 0.f;
          for (int q = lane; q < rchunks; q += 32) {
            if constexpr (PB == 4) {
              const float4 w = *reinterpret_cast<const float4*>(prow + 16 * q);
#pragma unroll
              for (int b = 0; b < NB; ++b) {
                const float4 uu = *reinterpret_cast<const float4*>(u_s + b * r + 4 * q);
                acc[b] += w.x * uu.x + w.y * uu.y + w.z * uu.z + w.w * uu.w;
              }
            } else {
              const uint4 w = *reinterpret_cast<const uint4*>(prow + 16 * q);
              const float2 a = h2f2(w.x), bb = h2f2(w.y), cc = h2f2(w.z), e = h2f2(w.w);
#pragma unroll
              for (int b = 0; b < NB; ++b) {
                const float4 u0 = *reinterpret_cast<const float4*>(u_s + b * r + 8 * q);
                const float4 u1 = *reinterpret_cast<const float4*>(u_s + b * r + 8 * q + 4);
                acc[b] += a.x * u0.x + a.y * u0.y + bb.x * u0.z + bb.y * u0.w + cc.x * u1.x +
                          cc.y * u1.y + e.x * u1.z + e.y * u1.w;
              }
            }
          }
#pragma unroll
          for (int b = 0; b < NB; ++b) acc[b] = warp_sum(acc[b]);
          if (lane == 0) {
            const float ti = *reinterpret_cast<const float*>(prow + (size_t)r * PB);
            const float bi = *reinterpret_cast<const float*>(prow + (size_t)r * PB + 4);
            const int i = c + (m0 + m) * G;
            uint32_t bits = 0;
#pragma unroll
            for (int b = 0; b < NB; ++b) {
              if (b < B) {
                const float lg = acc[b] - ti;
                if (lg > 0.f) bits |= 1u << b;
                if (p.logits_out) p.logits_out[(size_t)b * f + i] = lg;
                if (p.trace.logits) p.trace.logits[((size_t)l * B + b) * f + i] = lg;
              }
            }
            sm.own_bits[m0 + m] = (uint8_t)bits;
            sm.own_bias[m0 + m] = bi;
          }
        }
        ring_release(ring, sm, ring.seq++);
      }
      named_bar_sync(kRedBar, kConsumerThreads);

      // ---------------------------------------------------------- own active list
      {
        // 2 own neurons per thread (nown <= 512), ascending order kept by a block scan
        const int m_a = 2 * t, m_b = 2 * t + 1;
        const uint32_t ba = (m_a < nown) ? sm.own_bits[m_a] : 0u;
        const uint32_t bb = (m_b < nown) ? sm.own_bits[m_b] : 0u;
        const int cnt = (ba != 0) + (bb != 0);
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int v = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += v;
        }
        if (lane == 31) sm.scan[warp] = incl;
        named_bar_sync(kRedBar, kConsumerThreads);
        int wbase = 0;
        for (int w = 0; w < warp; ++w) wbase += sm.scan[w];
        int total = 0;
        for (int w = 0; w < kConsumerWarps; ++w) total += sm.scan[w];
        int pos = wbase + incl - cnt;
        if (ba) {
          const int i = c + m_a * G;
          sm.list[pos] = i; sm.list_bits[pos] = (uint8_t)ba; sm.list_bias[pos] = sm.own_bias[m_a]; ++pos;
          for (int b = 0; b < B; ++b)
            if (ba >> b & 1u) atomicOr(mask_l + (size_t)b * words + (i >> 5), 1u << (i & 31));
        }
        if (bb) {
          const int i = c + m_b * G;
          sm.list[pos] = i; sm.list_bits[pos] = (uint8_t)bb; sm.list_bias[pos] = sm.own_bias[m_b];
          for (int b = 0; b < B; ++b)
            if (bb >> b & 1u) atomicOr(mask_l + (size_t)b * words + (i >> 5), 1u << (i & 31));
        }
        nlist = total;
        if (t == 0) {
          sm.nlist = total;
          if (do_ffn) {
            atomicAdd(p.active_total, (unsigned long long)total);
            if (p.layer_count) atomicAdd(p.layer_count + l, total);
          }
        }
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
        sm.list_bias[e] = *reinterpret_cast<const float*>(Ld.p2n + (size_t)i * p.p2_stride + (size_t)r * PB + 4);
      }
      if (t == 0) {
        sm.nlist = nlist;
        atomicAdd(p.active_total, (unsigned long long)nlist);
      }
    }

    if (do_ffn) {
      named_bar_sync(kRedBar, kConsumerThreads);
      if (t == 0) mbar_arrive(&sm.list_ready);
      // ---------------------------------------------------------- F: gather + scatter
      float y[NB][NU][UE];
#pragma unroll
      for (int b = 0; b < NB; ++b)
#pragma unroll
        for (int j = 0; j < NU; ++j)
#pragma unroll
          for (int e = 0; e < UE; ++e) y[b][j][e] = 0.f;
      for (int e = 0; e < nlist; ++e) {
        const uint32_t bits = sm.list_bits[e];
        const float bi = sm.list_bias[e];
        float acc[2 * NB];
#pragma unroll
        for (int i = 0; i < 2 * NB; ++i) acc[i] = 0.f;
        if constexpr (ACT == PI_REGLU) {
          const uint8_t* g = ring_wait(ring, sm, ring.seq, p.barrier_timeout_ns, p.err);
          float ga[NB];
#pragma unroll
          for (int b = 0; b < NB; ++b) ga[b] = 0.f;
          RowMath<FAM, NB, NU>::dot(g, nunits, d, x, ga);
          ring_release(ring, sm, ring.seq++);
#pragma unroll
          for (int b = 0; b < NB; ++b) acc[NB + b] = ga[b];
        }
        {
          const uint8_t* u = ring_wait(ring, sm, ring.seq, p.barrier_timeout_ns, p.err);
          float ua[NB];
#pragma unroll
          for (int b = 0; b < NB; ++b) ua[b] = 0.f;
          RowMath<FAM, NB, NU>::dot(u, nunits, d, x, ua);
          ring_release(ring, sm, ring.seq++);
#pragma unroll
          for (int b = 0; b < NB; ++b) acc[b] = ua[b];
        }
        block_sum<2 * NB>(acc, sm, rbuf);
        float h[NB];
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          float a;
          if constexpr (ACT == PI_REGLU) a = fmaxf(acc[NB + b] + bi, 0.f) * acc[b];
          else a = fmaxf(acc[b] + bi, 0.f);
          h[b] = ((bits >> b) & 1u) ? a : 0.f;
        }
        const uint8_t* dn = ring_wait(ring, sm, ring.seq, p.barrier_timeout_ns, p.err);
        RowMath<FAM, NB, NU>::axpy(dn, nunits, d, h, y);
        ring_release(ring, sm, ring.seq++);
      }
      // partial y of this block
      float* part = p.partials + (size_t)c * B * d;
#pragma unroll
      for (int b = 0; b < NB; ++b)
#pragma unroll
        for (int j = 0; j < NU; ++j) {
          const int q = t + kConsumerThreads * j;
          if (b < B && q < nunits) {
            float* dst = part + (size_t)b * d + (size_t)q * UE;
#pragma unroll
            for (int e = 0; e < UE; e += 4)
              *reinterpret_cast<float4*>(dst + e) = make_float4(y[b][j][e], y[b][j][e + 1], y[b][j][e + 2], y[b][j][e + 3]);
          }
        }
      grid_barrier(p, sm, epoch);

      // ---------------------------------------------------------- R: slice reduce
      if (slice_owner) {
        const int ng = (col1 - col0) / 32;   // 32-column groups in this slice
        float acc[NB][kMaxColGroups];
#pragma unroll
        for (int b = 0; b < NB; ++b)
#pragma unroll
          for (int gq = 0; gq < kMaxColGroups; ++gq) acc[b][gq] = 0.f;
        for (int cc = warp; cc < G; cc += kConsumerWarps) {
          const float* src = p.partials + (size_t)cc * B * d;
#pragma unroll
          for (int b = 0; b < NB; ++b)
#pragma unroll
            for (int gq = 0; gq < kMaxColGroups; ++gq)
              if (b < B && gq < ng) acc[b][gq] += __ldcg(src + (size_t)b * d + col0 + 32 * gq + lane);
        }
#pragma unroll
        for (int b = 0; b < NB; ++b)
#pragma unroll
          for (int gq = 0; gq < kMaxColGroups; ++gq)
            red2[((warp * NB + b) * kMaxColGroups + gq) * 32 + lane] = acc[b][gq];
        named_bar_sync(kRedBar, kConsumerThreads);
        // warp w finishes token (w % NB)'s column groups; fixed summation order over warps
        if (warp < NB && warp < B) {
          const int b = warp;
          float sq = 0.f;
          for (int gq = 0; gq < ng; ++gq) {
            float yv = 0.f;
#pragma unroll
            for (int w = 0; w < kConsumerWarps; ++w) yv += red2[((w * NB + b) * kMaxColGroups + gq) * 32 + lane];
            const int j = col0 + 32 * gq + lane;
            if (do_glue) {
              const float vv = __ldcg(p.xb + (size_t)(l & 1) * B * d + (size_t)b * d + j) + yv;
              p.v[(size_t)b * d + j] = vv;
              sq += vv * vv;
              if (p.trace.y) p.trace.y[((size_t)l * B + b) * d + j] = yv;
            } else {
              p.y_out[(size_t)b * d + j] = yv;
            }
          }
          if (do_glue) {
            sq = warp_sum(sq);
            if (lane == 0) p.ssq[(size_t)b * G + c] = sq;
          }
        }
      }
      // trace: mask words, compact index list and count of this layer (complete now)
      if (do_glue && (p.trace.idx || p.trace.count || p.trace.mask) && c == G - 1) {
        if (p.trace.mask)
          for (int w = t; w < B * words; w += kConsumerThreads)
            p.trace.mask[(size_t)l * B * words + w] = __ldcg(mask_l + w);
        // block-wide ordered compaction of the union of the B masks
        int base = 0;
        for (int w0 = 0; w0 < words; w0 += kConsumerThreads) {
          const int w = w0 + t;
          uint32_t un = 0;
          if (w < words)
            for (int b = 0; b < B; ++b) un |= __ldcg(mask_l + (size_t)b * words + w);
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
      if (!do_glue) break;
      grid_barrier(p, sm, epoch);

      // ---------------------------------------------------------- glue: x' = v / rms
      if (t < NB) {
        float s = 0.f;
        if (t < B)
          for (int q = 0; q < nslices; ++q) s += __ldcg(p.ssq + (size_t)t * G + q);
        sm.rms[t] = sqrtf(s / (float)d + kRmsEps);
      }
      named_bar_sync(kRedBar, kConsumerThreads);
#pragma unroll
      for (int b = 0; b < NB; ++b)
#pragma unroll
        for (int j = 0; j < NU; ++j) {
          const int q = t + kConsumerThreads * j;
          if (b < B && q < nunits) {
            const float inv = sm.rms[b];
            const float* src = p.v + (size_t)b * d + (size_t)q * UE;
#pragma unroll
            for (int e = 0; e < UE; e += 4) {
              const float4 vv = __ldcg(reinterpret_cast<const float4*>(src + e));
              const float o[4] = {vv.x / inv, vv.y / inv, vv.z / inv, vv.w / inv};
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                if constexpr (FAM == FAM_F32) x[b][j][e + k] = o[k];
                else x[b][j][e + k] = __half2float(__float2half_rn(o[k]));
              }
            }
          }
        }
      // slice owners keep the new input in fp32 for the next layer's residual (xb is
      // double-buffered by layer parity: the other copy was last read before this
      // layer's first grid barrier), and write the trace / output
      if (slice_owner) {
        float* xn = p.xb + (size_t)((l + 1) & 1) * B * d;
        for (int idx = t; idx < B * (col1 - col0); idx += kConsumerThreads) {
          const int b = idx / (col1 - col0), j = col0 + idx % (col1 - col0);
          float xv = __ldcg(p.v + (size_t)b * d + j) / sm.rms[b];
          if constexpr (FAM != FAM_F32) xv = __half2float(__float2half_rn(xv));
          xn[(size_t)b * d + j] = xv;
          if (p.trace.x) {
            if constexpr (FAM == FAM_F32) reinterpret_cast<float*>(p.trace.x)[((size_t)(l + 1) * B + b) * d + j] = xv;
            else reinterpret_cast<__half*>(p.trace.x)[((size_t)(l + 1) * B + b) * d + j] = __float2half_rn(xv);
          }
          if (l == p.L - 1) {
            if constexpr (FAM == FAM_F32) reinterpret_cast<float*>(p.x_out)[(size_t)b * d + j] = xv;
            else reinterpret_cast<__half*>(p.x_out)[(size_t)b * d + j] = __float2half_rn(xv);
          }
        }
      }
    } else {
      break;   // predictor only
    }
  }

  // last block out resets the barrier words for the next launch
  named_bar_sync(kRedBar, kConsumerThreads);
  if (t == 0) {
    __threadfence();
    const uint32_t prev = atomicAdd(p.bar + 1, 1u);
    if (prev == (uint32_t)G - 1) {
      atomicExch(p.bar, 0u);
      atomicExch(p.bar + 1, 0u);
    }
  }
}

// A kernel that only runs grid barriers; with barrier_extra > 0 the target can never be
// reached, so every wait must give up after barrier_timeout_ns and report it.
__global__ void __launch_bounds__(kThreads, 1) barrier_probe_kernel(const FusedParams p, int rounds) {
  __shared__ Smem sm;
  if (threadIdx.x == 0) sm.abort_flag = 0;
  __syncthreads();
  if (threadIdx.x >= kConsumerThreads) return;
  uint32_t epoch = 0;
  for (int i = 0; i < rounds; ++i) grid_barrier(p, sm, epoch);
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
template <> struct NUof<FAM_F32, 1> { static constexpr int v = 4; };
template <> struct NUof<FAM_F32, 2> { static constexpr int v = 4; };
template <> struct NUof<FAM_F32, 4> { static constexpr int v = 4; };
template <> struct NUof<FAM_F16, 1> { static constexpr int v = 6; };
template <> struct NUof<FAM_F16, 2> { static constexpr int v = 4; };
template <> struct NUof<FAM_F16, 4> { static constexpr int v = 2; };
template <> struct NUof<FAM_Q4, 1> { static constexpr int v = 2; };
template <> struct NUof<FAM_Q4, 2> { static constexpr int v = 1; };

constexpr int ue_of(int fam) { return fam == FAM_F32 ? 4 : fam == FAM_F16 ? 8 : 32; }

int nu_max(int fam, int nb) {
  switch (fam) {
    case FAM_F32: return 4;
    case FAM_F16: return nb == 1 ? 6 : nb == 2 ? 4 : 2;
    case FAM_Q4: return nb == 1 ? 2 : nb == 2 ? 1 : 0;
  }
  return 0;
}

int nb_of(int B) { return B <= 1 ? 1 : B <= 2 ? 2 : B <= 4 ? 4 : 0; }

template <int FAM, int ACT, int NB>
cudaError_t launch_t(const FusedParams& p, size_t smem, cudaStream_t stream) {
  auto kern = fused_kernel<FAM, ACT, NB, NUof<FAM, NB>::v>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
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

size_t fused_fixed_smem(int B, int r) {
  const int nb = nb_of(B) ? nb_of(B) : 4;
  return ((sizeof(Smem) + 127) / 128) * 128 + (size_t)nb * r * sizeof(float) +
         (size_t)kConsumerWarps * nb * kMaxColGroups * 32 * sizeof(float);
}

size_t fused_smem_bytes(const FusedParams& p) {
  return fused_fixed_smem(p.B, p.r) + (size_t)p.nslots * p.slot_bytes;
}

cudaError_t launch_fused(int family, int act, int B, const FusedParams& p, size_t smem,
                         cudaStream_t stream) {
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
  return cudaLaunchCooperativeKernel((const void*)barrier_probe_kernel, dim3(p.grid), dim3(kThreads),
                                     args, 0, stream);
}

}  // namespace pi
