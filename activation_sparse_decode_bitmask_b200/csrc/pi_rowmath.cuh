// Row arithmetic of the fused kernel.
//
// Consumer thread t owns the units q = t + kConsumerThreads * j (j < NU) of a d-long
// row: 4 elements for fp32, 8 for fp16 and 16 (half a Q4_0 block) for Q4_0.  It keeps its
// units of every token's x in registers for the predictor's first stage, and a row's dot
// product is a per-thread partial sum over the thread's units (the caller reduces the
// partials across the warp and the block).
//
// x units are kept as they are stored: fp32 values for the fp32 family, fp16 pairs for the
// fp16 and Q4_0 families.  fp16 weights meet fp16 x through fma.rn.f32.f16: the product of
// two fp16 values is exact in fp32, so only the fp32 sums round.
//
// Q4_0 rows: 32-weight blocks; the row holds the 16 nibble bytes of every block (byte j
// has element j in its low four bits and element j + 16 in its high four bits), then the
// fp16 scales of all its blocks.  Value = (code - 8) * scale.  A unit is the low or the
// high nibbles of one block.  Two codes become one fp16 pair exactly: a code q under the
// exponent pattern of 1024 is the fp16 value 1024 + q, and one packed subtraction of 1032
// leaves q - 8 (integers below 2048 are exact in fp16).  The pair then meets x like an
// fp16 weight pair, and the block's scale multiplies the unit's sum once.
#pragma once
#include <cuda_fp16.h>
#include <cstdint>

#include "pi_internal.h"
#include "pi_ptx.cuh"

namespace pi {

template <int FAM> struct Fam;
// UE: elements per unit; PB: bytes per predictor element; XW: 32-bit registers that hold
// one token's unit of x (fp32 values, or fp16 pairs for the fp16 and Q4_0 families, whose
// dots use fp16 x fp16 products accumulated in fp32)
template <> struct Fam<FAM_F32> { static constexpr int UE = 4;  static constexpr int PB = 4; static constexpr int XW = 4;  using X = float; };
template <> struct Fam<FAM_F16> { static constexpr int UE = 8;  static constexpr int PB = 2; static constexpr int XW = 4;  using X = __half; };
template <> struct Fam<FAM_Q4>  { static constexpr int UE = 16; static constexpr int PB = 2; static constexpr int XW = 8;  using X = __half; };

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

// Loads from shared memory by 32-bit shared-window address (the ring holds every row)
__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}
__device__ __forceinline__ void sts_u32(uint32_t a, uint32_t v) {
  asm volatile("st.shared.u32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}
__device__ __forceinline__ float lds_f32(uint32_t a) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ float lds_h2f(uint32_t a) {
  unsigned short v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
  return __half2float(__ushort_as_half(v));
}
// Read-only streaming loads from global memory (weights that no kernel writes meanwhile)
__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 v;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
      : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
      : "l"(p));
  return v;
}
__device__ __forceinline__ float ldg_h2f(const void* p) {
  unsigned short v;
  asm("ld.global.nc.u16 %0, [%1];" : "=h"(v) : "l"(p));
  return __half2float(__ushort_as_half(v));
}
__device__ __forceinline__ float4 u4f(uint4 v) {
  return make_float4(__uint_as_float(v.x), __uint_as_float(v.y), __uint_as_float(v.z), __uint_as_float(v.w));
}

// acc + lo(w) * lo(x) and acc2 + hi(w) * hi(x): fp16 x fp16 products (exact in fp32)
// added in fp32 with one rounding each
__device__ __forceinline__ void fma2_h(uint32_t w2, uint32_t x2, float& acc, float& acc2) {
  asm("{\n .reg .f16 wl, wh, xl, xh;\n mov.b32 {wl, wh}, %2;\n mov.b32 {xl, xh}, %3;\n"
      " fma.rn.f32.f16 %0, wl, xl, %0;\n fma.rn.f32.f16 %1, wh, xh, %1;\n}"
      : "+f"(acc), "+f"(acc2)
      : "r"(w2), "r"(x2));
}

// Unit q of every token's x (xs: [NB][d] in the family's x type) in registers.
template <int FAM, int NB>
__device__ __forceinline__ void load_x_unit(const void* xs, int d, int q, uint32_t (&xu)[NB][Fam<FAM>::XW]) {
  constexpr int UE = Fam<FAM>::UE;
  constexpr int XB = FAM == FAM_F32 ? 4 : 2;
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(xs) + (size_t)XB * (b * d + UE * q));
#pragma unroll
    for (int c = 0; c < Fam<FAM>::XW / 4; ++c) {
      const uint4 v = src[c];
      xu[b][4 * c] = v.x; xu[b][4 * c + 1] = v.y; xu[b][4 * c + 2] = v.z; xu[b][4 * c + 3] = v.w;
    }
  }
}

// The same from shared memory (xs: shared address of [NB][d] in the family's x type)
template <int FAM, int NB>
__device__ __forceinline__ void lds_x_unit(uint32_t xs, int d, int q, uint32_t (&xu)[NB][Fam<FAM>::XW]) {
  constexpr int UE = Fam<FAM>::UE;
  constexpr uint32_t XB = FAM == FAM_F32 ? 4u : 2u;   // bytes per x element
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    const uint32_t a = xs + XB * (uint32_t)(b * d + UE * q);
#pragma unroll
    for (int c = 0; c < Fam<FAM>::XW / 4; ++c) {
      const uint4 v = lds128(a + 16u * c);
      xu[b][4 * c] = v.x; xu[b][4 * c + 1] = v.y; xu[b][4 * c + 2] = v.z; xu[b][4 * c + 3] = v.w;
    }
  }
}

// Two Q4_0 codes (bytes k and k + 1 of `codes`, each 0..15) as the fp16 pair
// (code_k - 8, code_{k+1} - 8), exactly: 0x64cc is the fp16 value 1024 + cc.
template <int K>
__device__ __forceinline__ uint32_t q4_pair(uint32_t codes) {
  const uint32_t biased = __byte_perm(codes, 0x00006464u, K == 0 ? 0x5140u : 0x5342u);
  const __half2 v = __hsub2(*reinterpret_cast<const __half2*>(&biased), __floats2half2_rn(1032.f, 1032.f));
  return *reinterpret_cast<const uint32_t*>(&v);
}

// Byte offset, within a weight row, of the 16 bytes unit q reads: the unit itself, or
// for Q4_0 the code block it is one half of.
template <int FAM>
__device__ __forceinline__ uint32_t unit_byte(int q) {
  return FAM == FAM_Q4 ? 16u * (uint32_t)(q >> 1) : 16u * (uint32_t)q;
}

// acc[b] += (unit q of a weight row) . xu[b], from the unit's 16 bytes w (and for Q4_0
// the block's fp16 scale sc)
template <int FAM, int NB>
__device__ __forceinline__ void unit_dot_w(const uint4 w, float sc, int q, const uint32_t (&xu)[NB][Fam<FAM>::XW],
                                           float (&acc)[NB]) {
  if constexpr (FAM == FAM_F32) {
    const float4 v = u4f(w);
#pragma unroll
    for (int b = 0; b < NB; ++b)
      acc[b] = fmaf(v.w, __uint_as_float(xu[b][3]),
                    fmaf(v.z, __uint_as_float(xu[b][2]),
                         fmaf(v.y, __uint_as_float(xu[b][1]), fmaf(v.x, __uint_as_float(xu[b][0]), acc[b]))));
  } else if constexpr (FAM == FAM_F16) {
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      float s = acc[b], s2 = 0.f;
      fma2_h(w.x, xu[b][0], s, s2);
      fma2_h(w.y, xu[b][1], s, s2);
      fma2_h(w.z, xu[b][2], s, s2);
      fma2_h(w.w, xu[b][3], s, s2);
      acc[b] = s + s2;
    }
  } else {
    const int sh = (q & 1) * 4;
    const uint32_t wv[4] = {(w.x >> sh) & 0x0F0F0F0Fu, (w.y >> sh) & 0x0F0F0F0Fu, (w.z >> sh) & 0x0F0F0F0Fu,
                            (w.w >> sh) & 0x0F0F0F0Fu};
    uint32_t wp[8];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      wp[2 * m] = q4_pair<0>(wv[m]);       // elements 4m, 4m + 1 of the unit
      wp[2 * m + 1] = q4_pair<1>(wv[m]);   // elements 4m + 2, 4m + 3
    }
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      float s = 0.f, s2 = 0.f;
#pragma unroll
      for (int k = 0; k < 8; ++k) fma2_h(wp[k], xu[b][k], s, s2);
      acc[b] = fmaf(sc, s + s2, acc[b]);
    }
  }
}

// The same with the row in shared memory (row: shared address; d: the row's length)
template <int FAM, int NB>
__device__ __forceinline__ void unit_dot(uint32_t row, int d, int q, const uint32_t (&xu)[NB][Fam<FAM>::XW],
                                         float (&acc)[NB]) {
  const uint4 w = lds128(row + unit_byte<FAM>(q));
  const float sc = FAM == FAM_Q4 ? lds_h2f(row + (uint32_t)(d >> 1) + 2u * (uint32_t)(q >> 1)) : 0.f;
  unit_dot_w<FAM, NB>(w, sc, q, xu, acc);
}

// acc[b] += (unit q of a predictor row in the p dtype: fp32 for the fp32 family, else
// fp16) . xu[b]
template <int FAM, int NB>
__device__ __forceinline__ void unit_dot_p(uint32_t row, int q, const uint32_t (&xu)[NB][Fam<FAM>::XW],
                                           float (&acc)[NB]) {
  constexpr int UE = Fam<FAM>::UE;
  if constexpr (FAM == FAM_F32 || FAM == FAM_F16) {
    unit_dot<FAM, NB>(row, 0, q, xu, acc);
  } else {
    // fp16 predictor row: 16 elements per unit, two 16-byte chunks
    const uint32_t src = row + (uint32_t)q * UE * 2;
    const uint4 w0 = lds128(src), w1 = lds128(src + 16u);
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      float s = acc[b], s2 = 0.f;
      fma2_h(w0.x, xu[b][0], s, s2); fma2_h(w0.y, xu[b][1], s, s2);
      fma2_h(w0.z, xu[b][2], s, s2); fma2_h(w0.w, xu[b][3], s, s2);
      fma2_h(w1.x, xu[b][4], s, s2); fma2_h(w1.y, xu[b][5], s, s2);
      fma2_h(w1.z, xu[b][6], s, s2); fma2_h(w1.w, xu[b][7], s, s2);
      acc[b] = s + s2;
    }
  }
}

// Butterfly reduce-scatter of V (a power of two, <= 16) per-lane values across the
// warp: on return every lane holds the warp's sum of value lane >> (5 - log2 V).  The
// lanes are paired at offsets 16, 8, 4, 2, 1 in that order for every V and every value,
// so a value's sum does not depend on V or on its slot.
template <int V>
__device__ __forceinline__ float reduce_scatter(float (&v)[V], int lane) {
  static_assert(V >= 1 && V <= 16 && (V & (V - 1)) == 0, "V must be a power of two <= 16");
#pragma unroll
  for (int o = 16, n = V / 2; n >= 1; o >>= 1, n >>= 1) {
    const bool up = lane & o;
#pragma unroll
    for (int i = 0; i < n; ++i) {
      const float send = up ? v[i] : v[i + n];
      const float keep = up ? v[i + n] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
  float s = v[0];
#pragma unroll
  for (int o = 16 / V; o >= 1; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  return s;
}

}  // namespace pi
