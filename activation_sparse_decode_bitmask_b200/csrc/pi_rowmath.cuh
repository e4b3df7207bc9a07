// Row arithmetic of the fused kernel.
//
// Consumer thread t owns the units q = t + kConsumerThreads * j (j < NU) of every d-long
// row: 4 elements for fp32, 8 for fp16 and 16 (half a Q4_0 block) for Q4_0.  It keeps
// its units of every token's x and y in registers as fp32 for a whole layer, so a row's
// dot product is a per-thread partial sum over the thread's units (the caller reduces
// the partials across the block) and the down projection y += h * row needs no
// cross-thread step at all.
//
// Q4_0 rows: 32-weight blocks; the row holds the 16 nibble bytes of every block (byte j
// has element j in its low four bits and element j + 16 in its high four bits), then the
// fp16 scales of all its blocks.  Value = (code - 8) * scale.  A unit is the low or the
// high nibbles of one block.  Products and sums are formed in fp32.
#pragma once
#include <cuda_fp16.h>
#include <cstdint>

#include "pi_internal.h"
#include "pi_ptx.cuh"

namespace pi {

template <int FAM> struct Fam;
template <> struct Fam<FAM_F32> { static constexpr int UE = 4;  static constexpr int PB = 4; using X = float; };
template <> struct Fam<FAM_F16> { static constexpr int UE = 8;  static constexpr int PB = 2; using X = __half; };
template <> struct Fam<FAM_Q4>  { static constexpr int UE = 16; static constexpr int PB = 2; using X = __half; };

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// 2^23 + code as a float, minus 2^23 + 8: exactly (code - 8) for a 4-bit code in byte k
__device__ __forceinline__ float q4_val(uint32_t nibbles_in_bytes, int k) {
  return __uint_as_float(__byte_perm(nibbles_in_bytes, 0x4B000000u, 0x7540 + k)) - 8388616.f;
}

// 8 fp16 values of a 16-byte chunk, widened
__device__ __forceinline__ void widen8(const uint4 v, float* o) {
  const float2 a = h2f2(v.x), b = h2f2(v.y), c = h2f2(v.z), e = h2f2(v.w);
  o[0] = a.x; o[1] = a.y; o[2] = b.x; o[3] = b.y; o[4] = c.x; o[5] = c.y; o[6] = e.x; o[7] = e.y;
}

// Unit q of every token's x (xs: [NB][d] in the family's x type), widened to fp32.
template <int FAM, int NB>
__device__ __forceinline__ void load_x_unit(const void* xs, int d, int q, float (&xu)[NB][Fam<FAM>::UE]) {
  constexpr int UE = Fam<FAM>::UE;
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    if constexpr (FAM == FAM_F32) {
      const float4 v = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(xs) + (size_t)b * d)[q];
      xu[b][0] = v.x; xu[b][1] = v.y; xu[b][2] = v.z; xu[b][3] = v.w;
    } else {
      const uint4* src = reinterpret_cast<const uint4*>(reinterpret_cast<const __half*>(xs) + (size_t)b * d + UE * q);
#pragma unroll
      for (int c = 0; c < UE / 8; ++c) widen8(src[c], &xu[b][8 * c]);
    }
  }
}

// acc[b] += (unit q of a weight row) . xu[b]
template <int FAM, int NB>
__device__ __forceinline__ void unit_dot(const uint8_t* row, int d, int q, const float (&xu)[NB][Fam<FAM>::UE],
                                         float (&acc)[NB]) {
  if constexpr (FAM == FAM_F32) {
    const float4 w = reinterpret_cast<const float4*>(row)[q];
#pragma unroll
    for (int b = 0; b < NB; ++b)
      acc[b] = fmaf(w.w, xu[b][3], fmaf(w.z, xu[b][2], fmaf(w.y, xu[b][1], fmaf(w.x, xu[b][0], acc[b]))));
  } else if constexpr (FAM == FAM_F16) {
    float w[8];
    widen8(reinterpret_cast<const uint4*>(row)[q], w);
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      float s = acc[b], s2 = w[4] * xu[b][4];
      s = fmaf(w[0], xu[b][0], s); s2 = fmaf(w[5], xu[b][5], s2);
      s = fmaf(w[1], xu[b][1], s); s2 = fmaf(w[6], xu[b][6], s2);
      s = fmaf(w[2], xu[b][2], s); s2 = fmaf(w[7], xu[b][7], s2);
      s = fmaf(w[3], xu[b][3], s);
      acc[b] = s + s2;
    }
  } else {
    const int blk = q >> 1;
    const uint4 nb = reinterpret_cast<const uint4*>(row)[blk];
    const float sc = __half2float(reinterpret_cast<const __half*>(row + (d >> 1))[blk]);
    const int sh = (q & 1) * 4;
    const uint32_t wv[4] = {(nb.x >> sh) & 0x0F0F0F0Fu, (nb.y >> sh) & 0x0F0F0F0Fu, (nb.z >> sh) & 0x0F0F0F0Fu,
                            (nb.w >> sh) & 0x0F0F0F0Fu};
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      float s = 0.f, s2 = 0.f;
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        s = fmaf(q4_val(wv[m], 0), xu[b][4 * m], s);
        s2 = fmaf(q4_val(wv[m], 1), xu[b][4 * m + 1], s2);
        s = fmaf(q4_val(wv[m], 2), xu[b][4 * m + 2], s);
        s2 = fmaf(q4_val(wv[m], 3), xu[b][4 * m + 3], s2);
      }
      acc[b] = fmaf(sc, s + s2, acc[b]);
    }
  }
}

// acc[b] += (unit q of a predictor row in the p dtype: fp32 for the fp32 family, else
// fp16) . xu[b]
template <int FAM, int NB>
__device__ __forceinline__ void unit_dot_p(const uint8_t* row, int q, const float (&xu)[NB][Fam<FAM>::UE],
                                           float (&acc)[NB]) {
  constexpr int UE = Fam<FAM>::UE;
  if constexpr (FAM == FAM_F32) {
    unit_dot<FAM_F32, NB>(row, 0, q, xu, acc);
  } else {
    const uint4* src = reinterpret_cast<const uint4*>(row + (size_t)q * UE * 2);
#pragma unroll
    for (int c = 0; c < UE / 8; ++c) {
      float w[8];
      widen8(src[c], w);
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        float s = acc[b], s2 = w[4] * xu[b][8 * c + 4];
        s = fmaf(w[0], xu[b][8 * c + 0], s); s2 = fmaf(w[5], xu[b][8 * c + 5], s2);
        s = fmaf(w[1], xu[b][8 * c + 1], s); s2 = fmaf(w[6], xu[b][8 * c + 6], s2);
        s = fmaf(w[2], xu[b][8 * c + 2], s); s2 = fmaf(w[7], xu[b][8 * c + 7], s2);
        s = fmaf(w[3], xu[b][8 * c + 3], s);
        acc[b] = s + s2;
      }
    }
  }
}

// yu[b] += h[b] * (unit q of a weight row)
template <int FAM, int NB>
__device__ __forceinline__ void unit_axpy(const uint8_t* row, int d, int q, const float (&h)[NB],
                                          float (&yu)[NB][Fam<FAM>::UE]) {
  if constexpr (FAM == FAM_F32) {
    const float4 w = reinterpret_cast<const float4*>(row)[q];
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      yu[b][0] = fmaf(h[b], w.x, yu[b][0]); yu[b][1] = fmaf(h[b], w.y, yu[b][1]);
      yu[b][2] = fmaf(h[b], w.z, yu[b][2]); yu[b][3] = fmaf(h[b], w.w, yu[b][3]);
    }
  } else if constexpr (FAM == FAM_F16) {
    float w[8];
    widen8(reinterpret_cast<const uint4*>(row)[q], w);
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
      for (int e = 0; e < 8; ++e) yu[b][e] = fmaf(h[b], w[e], yu[b][e]);
  } else {
    const int blk = q >> 1;
    const uint4 nb = reinterpret_cast<const uint4*>(row)[blk];
    const float sc = __half2float(reinterpret_cast<const __half*>(row + (d >> 1))[blk]);
    const int sh = (q & 1) * 4;
    const uint32_t wv[4] = {(nb.x >> sh) & 0x0F0F0F0Fu, (nb.y >> sh) & 0x0F0F0F0Fu, (nb.z >> sh) & 0x0F0F0F0Fu,
                            (nb.w >> sh) & 0x0F0F0F0Fu};
    float hs[NB];
#pragma unroll
    for (int b = 0; b < NB; ++b) hs[b] = h[b] * sc;
#pragma unroll
    for (int m = 0; m < 4; ++m)
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float cv = q4_val(wv[m], k);
#pragma unroll
        for (int b = 0; b < NB; ++b) yu[b][4 * m + k] = fmaf(hs[b], cv, yu[b][4 * m + k]);
      }
  }
}

// Butterfly reduce-scatter of 16 per-lane values across the warp: on return every lane
// holds the warp's sum of value (lane >> 1).  The pairing of the additions is the same
// for every value, so a value's sum does not depend on its slot.
__device__ __forceinline__ float reduce_scatter16(float (&v)[16], int lane) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const bool up = lane & 16;
    const float send = up ? v[i] : v[i + 8];
    const float keep = up ? v[i + 8] : v[i];
    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const bool up = lane & 8;
    const float send = up ? v[i] : v[i + 4];
    const float keep = up ? v[i + 4] : v[i];
    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const bool up = lane & 4;
    const float send = up ? v[i] : v[i + 2];
    const float keep = up ? v[i + 2] : v[i];
    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
  }
  {
    const bool up = lane & 2;
    const float send = up ? v[0] : v[1];
    const float keep = up ? v[1] : v[0];
    v[0] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
  }
  return v[0] + __shfl_xor_sync(0xffffffffu, v[0], 1);
}

}  // namespace pi
