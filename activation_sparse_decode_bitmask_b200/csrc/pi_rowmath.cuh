// Row arithmetic of the fused kernel.
//   warp dots: one warp forms the dot product of a row held in shared memory with the
//              tokens' x (also in shared memory); lanes stride over 16-byte chunks, the
//              sum is reduced with shuffles and returned in every lane
//   axpy:      the down projection y += h * row, one thread per 16-byte unit of y
// Rows are fp32, fp16 or Q4_0 (32-weight blocks: 16 bytes of nibbles, element j in the
// low four bits of byte j and element j + 16 in the high four bits, then the fp16 scales
// of all blocks of the row); x is fp32 for the fp32 family and fp16 otherwise.  Products
// and sums are formed in fp32.
#pragma once
#include <cuda_fp16.h>
#include <cstdint>

#include "pi_internal.h"
#include "pi_ptx.cuh"

namespace pi {

template <int FAM> struct Fam;
template <> struct Fam<FAM_F32> { static constexpr int UE = 4;  static constexpr int PB = 4; using X = float; };
template <> struct Fam<FAM_F16> { static constexpr int UE = 8;  static constexpr int PB = 2; using X = __half; };
template <> struct Fam<FAM_Q4>  { static constexpr int UE = 32; static constexpr int PB = 2; using X = __half; };

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// 2^23 + code as a float, minus 2^23 + 8: exactly (code - 8) for a 4-bit code in byte k
__device__ __forceinline__ float q4_val(uint32_t nibbles_in_bytes, int k) {
  return __uint_as_float(__byte_perm(nibbles_in_bytes, 0x4B000000u, 0x7540 + k)) - 8388616.f;
}

// Sum over 8 fp16 weights (one 16-byte chunk) times 8 x values.
__device__ __forceinline__ float dot8_h(const uint4 w, const uint4 xv) {
  const float2 w0 = h2f2(w.x), w1 = h2f2(w.y), w2 = h2f2(w.z), w3 = h2f2(w.w);
  const float2 x0 = h2f2(xv.x), x1 = h2f2(xv.y), x2 = h2f2(xv.z), x3 = h2f2(xv.w);
  float s = w0.x * x0.x;
  s = fmaf(w0.y, x0.y, s); s = fmaf(w1.x, x1.x, s); s = fmaf(w1.y, x1.y, s);
  s = fmaf(w2.x, x2.x, s); s = fmaf(w2.y, x2.y, s); s = fmaf(w3.x, x3.x, s); s = fmaf(w3.y, x3.y, s);
  return s;
}

// Warp dot of a row in the p dtype (fp32 for the fp32 family, else fp16) with x.
// xs: [NB][d] in the family's x type.  acc[b] holds the full sum in every lane.
template <int FAM, int NB>
__device__ __forceinline__ void warp_dot_p(const uint8_t* row, const void* xs, int d, float (&acc)[NB]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int b = 0; b < NB; ++b) acc[b] = 0.f;
  if constexpr (FAM == FAM_F32) {
    const float4* w4 = reinterpret_cast<const float4*>(row);
    const float* x = reinterpret_cast<const float*>(xs);
#pragma unroll 4
    for (int q = lane; q < d / 4; q += 32) {
      const float4 w = w4[q];
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        const float4 xv = reinterpret_cast<const float4*>(x + (size_t)b * d)[q];
        acc[b] = fmaf(w.x, xv.x, fmaf(w.y, xv.y, fmaf(w.z, xv.z, fmaf(w.w, xv.w, acc[b]))));
      }
    }
  } else {
    const uint4* w4 = reinterpret_cast<const uint4*>(row);
    const __half* x = reinterpret_cast<const __half*>(xs);
#pragma unroll 4
    for (int q = lane; q < d / 8; q += 32) {
      const uint4 w = w4[q];
#pragma unroll
      for (int b = 0; b < NB; ++b) acc[b] += dot8_h(w, reinterpret_cast<const uint4*>(x + (size_t)b * d)[q]);
    }
  }
#pragma unroll
  for (int b = 0; b < NB; ++b) acc[b] = warp_sum(acc[b]);
}

// Warp dot of a weight row (family format) with x.
template <int FAM, int NB>
__device__ __forceinline__ void warp_dot_w(const uint8_t* row, const void* xs, int d, float (&acc)[NB]) {
  if constexpr (FAM != FAM_Q4) {
    warp_dot_p<FAM, NB>(row, xs, d, acc);
  } else {
    const int lane = threadIdx.x & 31;
    const uint4* nib = reinterpret_cast<const uint4*>(row);
    const __half* scl = reinterpret_cast<const __half*>(row + (d >> 1));
    const __half* x = reinterpret_cast<const __half*>(xs);
#pragma unroll
    for (int b = 0; b < NB; ++b) acc[b] = 0.f;
#pragma unroll 2
    for (int q = lane; q < d / 32; q += 32) {
      const uint4 nb = nib[q];
      const float s = __half2float(scl[q]);
      const uint32_t wv[4] = {nb.x, nb.y, nb.z, nb.w};
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        const uint4* xq = reinterpret_cast<const uint4*>(x + (size_t)b * d + 32 * q);
        const uint4 xa = xq[0], xb = xq[1], xc = xq[2], xd = xq[3];   // elements 0-7, 8-15, 16-23, 24-31
        const uint32_t xl[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
        const uint32_t xh[8] = {xc.x, xc.y, xc.z, xc.w, xd.x, xd.y, xd.z, xd.w};
        float part = 0.f;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const uint32_t lo = wv[m] & 0x0F0F0F0Fu, hi = (wv[m] >> 4) & 0x0F0F0F0Fu;
          const float2 l0 = h2f2(xl[2 * m]), l1 = h2f2(xl[2 * m + 1]);   // x[4m .. 4m+3]
          const float2 h0 = h2f2(xh[2 * m]), h1 = h2f2(xh[2 * m + 1]);   // x[16+4m .. 16+4m+3]
          part = fmaf(q4_val(lo, 0), l0.x, part); part = fmaf(q4_val(lo, 1), l0.y, part);
          part = fmaf(q4_val(lo, 2), l1.x, part); part = fmaf(q4_val(lo, 3), l1.y, part);
          part = fmaf(q4_val(hi, 0), h0.x, part); part = fmaf(q4_val(hi, 1), h0.y, part);
          part = fmaf(q4_val(hi, 2), h1.x, part); part = fmaf(q4_val(hi, 3), h1.y, part);
        }
        acc[b] = fmaf(s, part, acc[b]);
      }
    }
#pragma unroll
    for (int b = 0; b < NB; ++b) acc[b] = warp_sum(acc[b]);
  }
}

// Warp dots of two weight rows (up and gate of one neuron) with x, reading x once.
template <int FAM, int NB>
__device__ __forceinline__ void warp_dot_w2(const uint8_t* row_a, const uint8_t* row_b, const void* xs, int d,
                                            float (&acc_a)[NB], float (&acc_b)[NB]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int b = 0; b < NB; ++b) acc_a[b] = acc_b[b] = 0.f;
  if constexpr (FAM == FAM_F32) {
    const float4* wa = reinterpret_cast<const float4*>(row_a);
    const float4* wb = reinterpret_cast<const float4*>(row_b);
    const float* x = reinterpret_cast<const float*>(xs);
#pragma unroll 4
    for (int q = lane; q < d / 4; q += 32) {
      const float4 a = wa[q], c = wb[q];
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        const float4 xv = reinterpret_cast<const float4*>(x + (size_t)b * d)[q];
        acc_a[b] = fmaf(a.x, xv.x, fmaf(a.y, xv.y, fmaf(a.z, xv.z, fmaf(a.w, xv.w, acc_a[b]))));
        acc_b[b] = fmaf(c.x, xv.x, fmaf(c.y, xv.y, fmaf(c.z, xv.z, fmaf(c.w, xv.w, acc_b[b]))));
      }
    }
  } else if constexpr (FAM == FAM_F16) {
    const uint4* wa = reinterpret_cast<const uint4*>(row_a);
    const uint4* wb = reinterpret_cast<const uint4*>(row_b);
    const __half* x = reinterpret_cast<const __half*>(xs);
#pragma unroll 4
    for (int q = lane; q < d / 8; q += 32) {
      const uint4 a = wa[q], c = wb[q];
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        const uint4 xv = reinterpret_cast<const uint4*>(x + (size_t)b * d)[q];
        acc_a[b] += dot8_h(a, xv);
        acc_b[b] += dot8_h(c, xv);
      }
    }
  } else {
    warp_dot_w<FAM, NB>(row_a, xs, d, acc_a);
    warp_dot_w<FAM, NB>(row_b, xs, d, acc_b);
    return;
  }
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    acc_a[b] = warp_sum(acc_a[b]);
    acc_b[b] = warp_sum(acc_b[b]);
  }
}

// y[b] += h[b] * row for the thread's units (consumer thread t owns units t + kConsumerThreads*j).
template <int FAM, int NB, int NU>
__device__ __forceinline__ void axpy_units(const uint8_t* row, int nunits, int d, const float (&h)[NB],
                                           float (&y)[NB][NU][Fam<FAM>::UE]) {
  const int t = threadIdx.x;
#pragma unroll
  for (int j = 0; j < NU; ++j) {
    const int q = t + kConsumerThreads * j;
    if (q < nunits) {
      if constexpr (FAM == FAM_F32) {
        const float4 w = reinterpret_cast<const float4*>(row)[q];
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          y[b][j][0] = fmaf(h[b], w.x, y[b][j][0]); y[b][j][1] = fmaf(h[b], w.y, y[b][j][1]);
          y[b][j][2] = fmaf(h[b], w.z, y[b][j][2]); y[b][j][3] = fmaf(h[b], w.w, y[b][j][3]);
        }
      } else if constexpr (FAM == FAM_F16) {
        const uint4 w = reinterpret_cast<const uint4*>(row)[q];
        const float2 a = h2f2(w.x), bb = h2f2(w.y), c = h2f2(w.z), e = h2f2(w.w);
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          y[b][j][0] = fmaf(h[b], a.x, y[b][j][0]);  y[b][j][1] = fmaf(h[b], a.y, y[b][j][1]);
          y[b][j][2] = fmaf(h[b], bb.x, y[b][j][2]); y[b][j][3] = fmaf(h[b], bb.y, y[b][j][3]);
          y[b][j][4] = fmaf(h[b], c.x, y[b][j][4]);  y[b][j][5] = fmaf(h[b], c.y, y[b][j][5]);
          y[b][j][6] = fmaf(h[b], e.x, y[b][j][6]);  y[b][j][7] = fmaf(h[b], e.y, y[b][j][7]);
        }
      } else {
        const uint4 nb = reinterpret_cast<const uint4*>(row)[q];
        const float s = __half2float(reinterpret_cast<const __half*>(row + (d >> 1))[q]);
        const uint32_t wv[4] = {nb.x, nb.y, nb.z, nb.w};
        float hs[NB];
#pragma unroll
        for (int b = 0; b < NB; ++b) hs[b] = h[b] * s;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const uint32_t lo = wv[m] & 0x0F0F0F0Fu, hi = (wv[m] >> 4) & 0x0F0F0F0Fu;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float cl = q4_val(lo, k), ch = q4_val(hi, k);
#pragma unroll
            for (int b = 0; b < NB; ++b) {
              y[b][j][4 * m + k] = fmaf(hs[b], cl, y[b][j][4 * m + k]);
              y[b][j][4 * m + k + 16] = fmaf(hs[b], ch, y[b][j][4 * m + k + 16]);
            }
          }
        }
      }
    }
  }
}

}  // namespace pi
