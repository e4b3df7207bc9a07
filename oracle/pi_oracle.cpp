// Oracle: a plain, slow, obviously correct CPU statement of the activation-sparse FFN at
// decode time, in C++ loops with double accumulation.
//
// TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's CPU
// baseline leg load this library (through oracle/cpp.py).  It shares no code, header or
// table with the CUDA library, and neither links the other.
//
// Sources (three web pages about PowerInfer; cited by page title and section):
//   [GN]  GeekNews "Tüketici sınıfı GPU takılı PC'lerde yüksek hızlı büyük dil modeli
//         serving", sections "Kuantizasyon ve uyumluluk", "Kısıtlar ve SSS".
//   [KPD] КПД "PowerInfer: Fast Large Language Model Serving with a Consumer-grade GPU",
//         section "Метод".
//   [UAI] unite.ai "PowerInfer: Mesin Inferensi LLM Cepat dengan GPU Konsumen", sections
//         "Fase Online: Mesin Inferensi LLM yang Sadar Neuron", "Prediktor Kepadatan
//         Adaptif", "Operator yang Sadar Neuron".
//
// Stored values are read in their stored formats and widened exactly to double: fp32,
// fp16 (IEEE binary16, decoded here bit by bit) and Q4_0 (32 four-bit codes q sharing
// one fp16 scale s, value (q - 8) * s; byte j of a block holds element j in its low
// nibble and element j + 16 in its high nibble).
//
// Layouts (the generator's): up/gate [f][d] row-major, down [d][f] row-major for fp32 and
// fp16; Q4_0 up/gate/down as nibble planes [f][d/32][16] and scale planes [f][d/32], the
// down weights neuron-major.  P1 [d][r], P2 [r][f] in the predictor dtype; bias and
// threshold [f] fp32.
//
// Every sum runs over its index in ascending order.  The loops over independent outputs
// may be shared among OpenMP threads; no sum is split, so the results do not depend on
// the thread count.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

enum { DT_F32 = 0, DT_F16 = 1, DT_Q4_0 = 2 };
enum { ACT_RELU = 0, ACT_REGLU = 1, ACT_RELU2 = 2 };

// IEEE binary16 -> double, exactly: sign, 5-bit exponent (bias 15), 10-bit fraction;
// exponent 0 holds subnormals (fraction * 2^-24), exponent 31 infinities and NaNs.
double half_to_double(uint16_t h) {
  const int sign = (h >> 15) & 1, e = (h >> 10) & 0x1F, m = h & 0x3FF;
  double v;
  if (e == 0) v = std::ldexp((double)m, -24);
  else if (e == 31) v = m ? NAN : INFINITY;
  else v = std::ldexp((double)(1024 + m), e - 25);
  return sign ? -v : v;
}

// float -> binary16 with round-to-nearest, ties to even (what a cast of an fp32 value to
// fp16 does): the value is scaled to an integer count of the target's units and rounded.
uint16_t float_to_half(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  const uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
  const double a = std::fabs((double)f);
  if (std::isnan(f)) return (uint16_t)(sign | 0x7E00u);
  if (a >= 65520.0) return (uint16_t)(sign | 0x7C00u);   // rounds to infinity
  int e;
  std::frexp(a, &e);                 // a = m * 2^e, m in [0.5, 1)
  int ue = e - 11;                   // unit of the last of 11 significant bits
  if (ue < -24) ue = -24;            // subnormal range: the unit is 2^-24
  const double q = a / std::ldexp(1.0, ue);    // exact (power-of-two scaling)
  double n = std::floor(q);
  const double rem = q - n;
  if (rem > 0.5 || (rem == 0.5 && std::fmod(n, 2.0) == 1.0)) n += 1.0;
  // n * 2^ue is the rounded value; encode it
  const double r = n * std::ldexp(1.0, ue);
  if (r == 0.0) return sign;
  int re;
  std::frexp(r, &re);
  if (re - 1 < -14) {                // subnormal: fraction = r / 2^-24
    return (uint16_t)(sign | (uint16_t)(r / std::ldexp(1.0, -24)));
  }
  const int exp_field = re - 1 + 15;
  const double frac = r / std::ldexp(1.0, re - 1) - 1.0;   // in [0, 1)
  return (uint16_t)(sign | (uint16_t)(exp_field << 10) | (uint16_t)(frac * 1024.0));
}

}  // namespace

extern "C" {

// One layer in its stored formats.  Pointers are host memory owned by the caller.
typedef struct {
  int d, f, r, act, w_dtype, p_dtype;
  const void* w_up;        // fp: [f][d]; Q4_0: nibbles [f][d/32][16]
  const void* w_gate;      // same, ReGLU only (else null)
  const void* w_down;      // fp: [d][f]; Q4_0: nibbles [f][d/32][16] (neuron-major)
  const uint16_t* s_up;    // Q4_0 scales [f][d/32] (fp16 bits), else null
  const uint16_t* s_gate;
  const uint16_t* s_down;
  const float* bias;       // [f]
  const void* p1;          // [d][r] in p_dtype
  const void* p2;          // [r][f] in p_dtype
  const float* thresh;     // [f]
} pio_layer;

double pio_half_to_double(uint16_t h) { return half_to_double(h); }
uint16_t pio_float_to_half(float f) { return float_to_half(f); }

void pio_set_threads(int n) {
#ifdef _OPENMP
  omp_set_num_threads(n > 0 ? n : 1);
#else
  (void)n;
#endif
}
int pio_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

}  // extern "C"

namespace {

double pvalue(int dt, const void* base, size_t i) {
  return dt == DT_F32 ? (double)static_cast<const float*>(base)[i] : half_to_double(static_cast<const uint16_t*>(base)[i]);
}

// Element j of the Q4_0 row `row` of a plane ([rows][d/32][16] nibbles, [rows][d/32] scales).
double q4_value(const void* nib, const uint16_t* sc, int d, size_t row, int j) {
  const int blk = j / 32, k = j % 32;
  const uint8_t byte = static_cast<const uint8_t*>(nib)[(row * (d / 32) + blk) * 16 + (k % 16)];
  const int q = k < 16 ? (byte & 0x0F) : (byte >> 4);
  return (double)(q - 8) * half_to_double(sc[row * (d / 32) + blk]);
}

// Weight of neuron i at input/output element j: up/gate row i element j, and W_down[j][i].
double w_up(const pio_layer* L, int i, int j) {
  if (L->w_dtype == DT_Q4_0) return q4_value(L->w_up, L->s_up, L->d, i, j);
  return pvalue(L->w_dtype, L->w_up, (size_t)i * L->d + j);
}
double w_gate(const pio_layer* L, int i, int j) {
  if (L->w_dtype == DT_Q4_0) return q4_value(L->w_gate, L->s_gate, L->d, i, j);
  return pvalue(L->w_dtype, L->w_gate, (size_t)i * L->d + j);
}
double w_down(const pio_layer* L, int j, int i) {
  if (L->w_dtype == DT_Q4_0) return q4_value(L->w_down, L->s_down, L->d, i, j);
  return pvalue(L->w_dtype, L->w_down, (size_t)j * L->f + i);
}

// a_{b,i}: ReLU max(0, up + b); ReGLU max(0, gate + b) * up; squared ReLU max(0, up + b)^2.
// [GN] §"Kısıtlar ve SSS": ReLU-family activations give exact zeros that can be skipped.
double activation(const pio_layer* L, const double* x, int i) {
  double up = 0.0;
  for (int j = 0; j < L->d; ++j) up += w_up(L, i, j) * x[j];
  if (L->act == ACT_REGLU) {
    double gate = 0.0;
    for (int j = 0; j < L->d; ++j) gate += w_gate(L, i, j) * x[j];
    const double g = gate + (double)L->bias[i];
    return (g > 0.0 ? g : 0.0) * up;
  }
  const double a = up + (double)L->bias[i];
  const double rl = a > 0.0 ? a : 0.0;
  return L->act == ACT_RELU2 ? rl * rl : rl;
}

}  // namespace

extern "C" {

// Predictor, [UAI] §"Prediktor Kepadatan Adaptif": a small per-layer predictor says
// which neurons will be active.  Read here as a linear low-rank map with a per-neuron
// threshold: u_k = sum_j P1[j][k] x_j; logit_i = sum_k P2[k][i] u_k - t_i.
// x [B][d] double; logits [B][f].
int pio_predict(const pio_layer* L, int B, const double* x, double* logits) {
  const int d = L->d, f = L->f, r = L->r;
  std::vector<double> u((size_t)B * r);
  for (int b = 0; b < B; ++b) {
#pragma omp parallel for schedule(static)
    for (int k = 0; k < r; ++k) {
      double s = 0.0;
      for (int j = 0; j < d; ++j) s += pvalue(L->p_dtype, L->p1, (size_t)j * r + k) * x[(size_t)b * d + j];
      u[(size_t)b * r + k] = s;
    }
#pragma omp parallel for schedule(static)
    for (int i = 0; i < f; ++i) {
      double s = 0.0;
      for (int k = 0; k < r; ++k) s += pvalue(L->p_dtype, L->p2, (size_t)k * f + i) * u[(size_t)b * r + k];
      logits[(size_t)b * f + i] = s - (double)L->thresh[i];
    }
  }
  return 0;
}

// Mask words: neuron i fires iff logit_i > 0 (strict); bit j of word w is neuron 32w + j.
void pio_pack_mask(const double* logits, int B, int f, uint32_t* words) {
  for (int b = 0; b < B; ++b)
    for (int w = 0; w < f / 32; ++w) {
      uint32_t v = 0;
      for (int j = 0; j < 32; ++j)
        if (logits[(size_t)b * f + 32 * w + j] > 0.0) v |= 1u << j;
      words[(size_t)b * (f / 32) + w] = v;
    }
}

// Compaction, [UAI] §"Operator yang Sadar Neuron": the active neurons (the union over the
// batch) are listed in ascending order and touched one by one.  Returns the count.
int pio_compact(const uint32_t* words, int B, int f, int32_t* idx) {
  int n = 0;
  for (int i = 0; i < f; ++i) {
    uint32_t any = 0;
    for (int b = 0; b < B; ++b) any |= (words[(size_t)b * (f / 32) + i / 32] >> (i % 32)) & 1u;
    if (any) idx[n++] = i;
  }
  return n;
}

// Sparse FFN, [UAI] §"Fase Online: Mesin Inferensi LLM yang Sadar Neuron" and §"Operator
// yang Sadar Neuron": only the listed neurons are computed, row by row for up/gate and
// column by column for down; token b's a_{b,i} is 0 where its own mask bit is 0.
// y_{b,j} = sum over the list in order of W_down[j][i] * a_{b,i}.
// masks [B][f] bytes (0/1); idx [count]; y [B][d].
int pio_sparse_ffn(const pio_layer* L, int B, const double* x, const uint8_t* masks, const int32_t* idx, int count,
                   double* y) {
  const int d = L->d, f = L->f;
  std::vector<double> a((size_t)B * count);
  for (int b = 0; b < B; ++b) {
#pragma omp parallel for schedule(dynamic, 16)
    for (int k = 0; k < count; ++k) {
      const int i = idx[k];
      a[(size_t)b * count + k] = masks[(size_t)b * f + i] ? activation(L, x + (size_t)b * d, i) : 0.0;
    }
#pragma omp parallel for schedule(static)
    for (int j = 0; j < d; ++j) {
      double s = 0.0;
      for (int k = 0; k < count; ++k) s += w_down(L, j, idx[k]) * a[(size_t)b * count + k];
      y[(size_t)b * d + j] = s;
    }
  }
  return 0;
}

// The dense FFN: every neuron, no predictor (the reference for the sparse = dense
// invariant and the dense CPU baseline).
int pio_dense_ffn(const pio_layer* L, int B, const double* x, double* y) {
  const int f = L->f;
  std::vector<int32_t> all(f);
  for (int i = 0; i < f; ++i) all[i] = i;
  std::vector<uint8_t> ones((size_t)B * f, 1);
  return pio_sparse_ffn(L, B, x, ones.data(), all.data(), f, y);
}

// The true mask: neuron i passes a nonzero value through its ReLU, i.e. its firing
// pre-activation (up + b for ReLU and squared ReLU, gate + b for ReGLU) is > 0.
// out [B][f] bytes.
int pio_true_mask(const pio_layer* L, int B, const double* x, uint8_t* out) {
  const int d = L->d, f = L->f;
  for (int b = 0; b < B; ++b) {
#pragma omp parallel for schedule(static)
    for (int i = 0; i < f; ++i) {
      double s = 0.0;
      for (int j = 0; j < d; ++j)
        s += (L->act == ACT_REGLU ? w_gate(L, i, j) : w_up(L, i, j)) * x[(size_t)b * d + j];
      out[(size_t)b * f + i] = (s + (double)L->bias[i]) > 0.0;
    }
  }
  return 0;
}

// Stack glue (the pages have no layer stack; this library's reading): v = x + y;
// x' = (v - mean v) / sqrt(var v + 1e-6) per token; x_dtype 0 rounds x' to fp32, 1 to
// fp32 then fp16, -1 leaves it in double.
void pio_glue(int B, int d, const double* x, const double* y, int x_dtype, double* x_next) {
  std::vector<double> v(d);
  for (int b = 0; b < B; ++b) {
    double s = 0.0;
    for (int j = 0; j < d; ++j) {
      v[j] = x[(size_t)b * d + j] + y[(size_t)b * d + j];
      s += v[j];
    }
    const double mean = s / d;
    double q = 0.0;
    for (int j = 0; j < d; ++j) q += (v[j] - mean) * (v[j] - mean);
    const double sd = std::sqrt(q / d + 1e-6);
    for (int j = 0; j < d; ++j) {
      const double o = (v[j] - mean) / sd;
      double out = o;
      if (x_dtype == 0) out = (double)(float)o;
      else if (x_dtype == 1) out = half_to_double(float_to_half((float)o));
      x_next[(size_t)b * d + j] = out;
    }
  }
}

// One layer of the stack: predict, mask words, compaction, sparse FFN, glue.
int pio_layer_step(const pio_layer* L, int B, const double* x, int x_dtype, double* logits, uint32_t* words,
                   int32_t* idx, int* count, double* y, double* x_next) {
  const int f = L->f;
  pio_predict(L, B, x, logits);
  pio_pack_mask(logits, B, f, words);
  const int n = pio_compact(words, B, f, idx);
  *count = n;
  std::vector<uint8_t> masks((size_t)B * f);
  for (size_t q = 0; q < masks.size(); ++q) masks[q] = logits[q] > 0.0;
  pio_sparse_ffn(L, B, x, masks.data(), idx, n, y);
  pio_glue(B, L->d, x, y, x_dtype, x_next);
  return 0;
}

}  // extern "C"
