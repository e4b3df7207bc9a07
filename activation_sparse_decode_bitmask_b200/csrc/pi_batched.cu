// The batched path: 5 to 32 tokens per call, fp16 family.
//
// At these batch sizes every step of a layer is a dense contraction over the rows it
// touches, so each runs on the tensor cores: tiles of 16 rows x 8 tokens, K in steps of
// 16 (mma.sync m16n8k16, fp16 operands, fp32 accumulation), operands staged through
// shared memory with cp.async and read with ldmatrix.
//   u       = P1^T x           rows: P1^T rows (contiguous)         tokens: x (fp16)
//   logit   = P2^T u - t       rows: P2 columns (owner-major rows)  tokens: u as fp16 hi + lo
//   h       = act(W x + b)     rows: gate/up rows of the active neurons (gathered by idx)
//   y       = sum_i h_i Wd_i   columns of the down rows of the active neurons; h as fp16 hi + lo
// fp16 x fp16 products are exact in fp32; u and h are fp32 values carried as the sum of
// two fp16 numbers (hi = fp16(v), lo = fp16(v - hi)), about 22 significant bits, so no
// step rounds an intermediate to fp16.  The active neurons are processed in the order of
// idx; the neurons at the front of the stored order are the hot prefix, so the first
// row tiles of every layer are its dense hot block and the rest are gathered cold rows.
// Every sum runs in a fixed order: results are bitwise reproducible.
#include <cuda_fp16.h>
#include <algorithm>
#include <cstdint>

#include "pi_internal.h"
#include "pi_ptx.cuh"

namespace pi {

namespace {

constexpr int kBW = 4;                    // warps per block
constexpr int kRows = 16 * kBW;           // rows (or columns) per block
constexpr int kKC = 128;                  // K elements staged per chunk (256 bytes of each row)
constexpr int kPad = kKC * 2 + 16;        // bytes per staged row: the 16-byte pad keeps ldmatrix conflict-free
constexpr int kMaxKSplit = 32;            // K splits of a row kernel at most
constexpr int kMaxDownSplit = 16;         // neuron splits of the down kernel at most
constexpr int kDM = 2;                    // 16-column tiles per warp in the down kernel
constexpr int kDCols = 16 * kDM * kBW;    // columns per down block
constexpr int kDN = 64;                   // neurons staged per down chunk
constexpr int kDPad = kDCols * 2 + 16;    // bytes per staged down row slice
constexpr int kHPad = kDN * 2 + 16;       // bytes per staged token row of h

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t a, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(a));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t a, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(a));
}
__device__ __forceinline__ void ldsm_x2(uint32_t a, uint32_t (&r)[2]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];" : "=r"(r[0]), "=r"(r[1]) : "r"(a));
}
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
__device__ __forceinline__ void split_h(float v, __half& hi, __half& lo) {
  hi = __float2half_rn(v);
  lo = __float2half_rn(v - __half2float(hi));
}

// ------------------------------------------------------------------ rows x tokens
// part[split][row][token] = sum over the split's K range of Rows[row][k] * Tok[token][k]
// for a block of 64 rows and all tokens.  Rows are fp16 rows found through the mode's
// addressing; Tok is [B][K] fp16 (plus a [B][K] low part when SPLIT).  Chunks of 64 K
// stream through a 3-stage cp.async pipeline.  An epilogue kernel then sums the splits in
// order and finishes the mode's step.
enum RowMode { ROWS_P1 = 0, ROWS_P2 = 1, ROWS_FFN = 2 };
constexpr int kStages = 3;

struct RowTokArgs {
  int mode, nrows_static, K, B, ksplit;
  const int32_t* count;        // ROWS_FFN: number of active rows (device)
  const uint8_t* base;         // row storage
  int stride;                  // bytes between consecutive rows (P1) or per record / P2 row
  int G, nown_max;             // ROWS_P2: owner-major placement of neuron rows
  const int32_t* idx;          // ROWS_FFN: stored ids of the active neurons
  int up_off, gate_off;        // ROWS_FFN: byte offsets of the rows in a record (gate < 0: ReLU)
  int f;
  const __half* tok;           // [B][K]
  const __half* tok_lo;        // [B][K] or null
  float* part;                 // [ksplit][NMAT][nrows_static][32]
  int* err;                    // device error word (index or count out of range)
};

template <int NT, int NMAT, bool SPLIT>
__global__ void __launch_bounds__(32 * kBW) rowtok_kernel(const RowTokArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int NS = SPLIT ? 2 : 1;
  constexpr int BP = NT * 8;                                   // padded tokens
  constexpr int ROWS_B = NMAT * kRows * kPad, TOK_B = NS * BP * kPad, STAGE_B = ROWS_B + TOK_B;
  int nrows = a.nrows_static;
  if (a.mode == ROWS_FFN) {
    const int cnt = *a.count;
    if (cnt < 0 || cnt > a.nrows_static) {
      if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) atomicExch(a.err, DEV_ERR_INDEX);
      return;
    }
    nrows = cnt;
  }
  const int row0 = blockIdx.x * kRows;
  if (row0 >= nrows) return;
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int nch = a.K / kKC;
  const int c_begin = (int)((long long)blockIdx.y * nch / a.ksplit);
  const int c_end = (int)((long long)(blockIdx.y + 1) * nch / a.ksplit);

  // byte address of row j (clamped into range: rows past the end repeat the last one and
  // their results are never used), matrix m
  auto row_ptr = [&](int j, int m) -> const uint8_t* {
    j = min(j, nrows - 1);
    if (a.mode == ROWS_P1) return a.base + (size_t)j * a.stride;
    if (a.mode == ROWS_P2) return a.base + ((size_t)(j % a.G) * a.nown_max + j / a.G) * a.stride;
    int i = __ldg(a.idx + j);
    if (i < 0 || i >= a.f) {   // a bad id reads neuron 0 and is reported
      atomicExch(a.err, DEV_ERR_INDEX);
      i = 0;
    }
    return a.base + (size_t)i * a.stride + (m == 0 ? a.up_off : a.gate_off);
  };
  // the block's row addresses, once: the same rows stream through every K chunk
  __shared__ const uint8_t* rowp[NMAT][kRows];
  for (int e = t; e < NMAT * kRows; e += 32 * kBW) rowp[e / kRows][e % kRows] = row_ptr(row0 + e % kRows, e / kRows);
  __syncthreads();
  const uint32_t base_u = smem_u32(smem);
  auto stage_chunk = [&](int ch, int buf) {
    const int k0 = ch * kKC;
    const uint32_t rows_u = base_u + (uint32_t)(buf * STAGE_B), tok_u = rows_u + ROWS_B;
    constexpr int PC = kKC * 2 / 16;   // 16-byte pieces per staged row
    for (int e = t; e < NMAT * kRows * PC; e += 32 * kBW) {
      const int m = e / (kRows * PC), rr = (e / PC) % kRows, pc = e % PC;
      cp_async16(rows_u + (uint32_t)((m * kRows + rr) * kPad + pc * 16), rowp[m][rr] + (size_t)k0 * 2 + pc * 16);
    }
    for (int e = t; e < NS * BP * PC; e += 32 * kBW) {
      const int s = e / (BP * PC), b = (e / PC) % BP, pc = e % PC;
      const __half* src = (s == 0 ? a.tok : a.tok_lo) + (size_t)min(b, a.B - 1) * a.K + k0 + pc * 8;
      cp_async16(tok_u + (uint32_t)((s * BP + b) * kPad + pc * 16), src);
    }
  };

  float c[NMAT][NT][4];
#pragma unroll
  for (int m = 0; m < NMAT; ++m)
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) c[m][n][e] = 0.f;

#pragma unroll
  for (int s = 0; s < kStages - 1; ++s) {
    if (c_begin + s < c_end) stage_chunk(c_begin + s, s);
    cp_async_commit();
  }
  for (int ch = c_begin; ch < c_end; ++ch) {
    cp_async_wait_1();
    __syncthreads();   // chunk ch landed for every thread; chunk ch - 1's buffer is free
    if (ch + kStages - 1 < c_end) stage_chunk(ch + kStages - 1, (ch + kStages - 1 - c_begin) % kStages);
    cp_async_commit();
    const int buf = (ch - c_begin) % kStages;
    const uint32_t rows_u = base_u + (uint32_t)(buf * STAGE_B), tok_u = rows_u + ROWS_B;
#pragma unroll
    for (int ks = 0; ks < kKC / 16; ++ks) {
      uint32_t af[NMAT][4];
#pragma unroll
      for (int m = 0; m < NMAT; ++m) {
        const int r = warp * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
        const int kk = ks * 16 + 8 * (lane >> 4);
        ldsm_x4(rows_u + (uint32_t)((m * kRows + r) * kPad + kk * 2), af[m]);
      }
#pragma unroll
      for (int n = 0; n < NT; ++n) {
#pragma unroll
        for (int s = 0; s < NS; ++s) {
          uint32_t bf[2];
          const int b = n * 8 + (lane & 7);
          const int kk = ks * 16 + 8 * ((lane >> 3) & 1);
          ldsm_x2(tok_u + (uint32_t)((s * BP + b) * kPad + kk * 2), bf);
#pragma unroll
          for (int m = 0; m < NMAT; ++m) mma16816(c[m][n], af[m], bf);
        }
      }
    }
  }
  cp_async_wait_all();

  // raw partials: thread holds rows g and g + 8 of the warp's tile, tokens 2t and 2t + 1
  // of every 8-token tile
  const int g = lane >> 2, tq = lane & 3;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int j = row0 + warp * 16 + g + 8 * half;
    if (j >= nrows) continue;
#pragma unroll
    for (int m = 0; m < NMAT; ++m)
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        float2 v = make_float2(c[m][n][2 * half], c[m][n][2 * half + 1]);
        *reinterpret_cast<float2*>(a.part + (((size_t)blockIdx.y * NMAT + m) * a.nrows_static + j) * 32 + n * 8 + 2 * tq) = v;
      }
  }
}

// Sum the splits of part (fixed order) and finish the mode's step, one thread per
// (row, token).
struct RowEpiArgs {
  int mode, nrows_static, B, ksplit, nmat;
  int squared;                 // ROWS_FFN: squared ReLU
  const int32_t* count;
  const int32_t* idx;
  int f;
  const float* part;
  __half* u_hi;                // ROWS_P1: [B][r]
  __half* u_lo;
  const float* thresh;         // ROWS_P2
  float* logits;               // [B][f] or null
  uint32_t* mask;              // [B][f/32], zeroed by the caller
  const float* bias;           // ROWS_FFN
  const uint32_t* mask_in;     // [B][f/32]
  float* h;                    // [count][32]
};

__global__ void __launch_bounds__(256) rowtok_epilogue(const RowEpiArgs a) {
  int nrows = a.nrows_static;
  if (a.mode == ROWS_FFN) {
    const int cnt = *a.count;
    if (cnt < 0 || cnt > a.nrows_static) return;   // reported by the row kernel
    nrows = cnt;
  }
  const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int j = (int)(e / 32), b = (int)(e % 32);
  if (j >= nrows) return;
  float v[2] = {0.f, 0.f};
  for (int s = 0; s < a.ksplit; ++s)
    for (int m = 0; m < a.nmat; ++m) v[m] += a.part[(((size_t)s * a.nmat + m) * a.nrows_static + j) * 32 + b];
  if (a.mode == ROWS_P1) {
    if (b < a.B) {
      __half hi, lo;
      split_h(v[0], hi, lo);
      a.u_hi[(size_t)b * a.nrows_static + j] = hi;
      a.u_lo[(size_t)b * a.nrows_static + j] = lo;
    }
  } else if (a.mode == ROWS_P2) {
    if (b < a.B) {
      const float lg = v[0] - __ldg(a.thresh + j);
      if (a.logits) a.logits[(size_t)b * a.f + j] = lg;
      if (lg > 0.f) atomicOr(a.mask + (size_t)b * (a.f / 32) + (j >> 5), 1u << (j & 31));
    }
  } else {
    float hv = 0.f;
    if (b < a.B) {
      int i = __ldg(a.idx + j);
      if (i < 0 || i >= a.f) i = 0;   // reported by the row kernel
      const uint32_t bit = (__ldg(a.mask_in + (size_t)b * (a.f / 32) + (i >> 5)) >> (i & 31)) & 1u;
      const float bi = __ldg(a.bias + i);
      float act = (a.nmat == 2) ? fmaxf(v[1] + bi, 0.f) * v[0] : fmaxf(v[0] + bi, 0.f);   // matrix 1: gate
      if (a.squared) act *= act;   // squared ReLU
      hv = bit ? act : 0.f;
    }
    a.h[(size_t)j * 32 + b] = hv;
  }
}

// ------------------------------------------------------------------ down projection
// ypart[split][b][c] = sum over the split's neurons j of h[j][b] * Wd[idx[j]][c], for a
// block of 64 columns and all tokens: the columns' slices of the active down rows are
// staged [neuron][column] and read transposed; then the splits are summed in order.
struct DownArgs {
  const int32_t* count;
  int fmax, d, B, nsplit;
  const uint8_t* rec;
  int rec_stride, down_off;
  const int32_t* idx;
  const float* h;      // [count][32]
  float* ypart;        // [nsplit][B][d]
};

template <int NT>
__global__ void __launch_bounds__(32 * kBW) down_kernel(const DownArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int BP = NT * 8;
  // a stage: the chunk's down-row slices, h as fp16 hi / lo [2][BP], and h as copied (fp32 [kDN][BP])
  constexpr int W_B = kDN * kDPad, HS_B = 2 * BP * kHPad, STAGE_B = W_B + HS_B + kDN * BP * 4;
  constexpr int PC = kDCols * 2 / 16;          // 16-byte pieces of a row slice
  constexpr int PW = kDN * PC / (32 * kBW);    // row-slice pieces per thread and chunk
  constexpr int PH = BP / 4;                   // 16-byte pieces of a neuron's h
  static_assert(kDN * PC % (32 * kBW) == 0 && kDN * PH % (32 * kBW) == 0, "down staging");
  int count = *a.count;
  if (count < 0 || count > a.fmax) count = 0;   // reported by the gate/up kernel; y becomes 0
  const int nch = (count + kDN - 1) / kDN;
  const int c_begin = (int)((long long)blockIdx.y * nch / a.nsplit);
  const int c_end = (int)((long long)(blockIdx.y + 1) * nch / a.nsplit);
  const int c0 = blockIdx.x * kDCols;
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const uint32_t base_u = smem_u32(smem);
  // The neuron index of each of this thread's row-slice pieces of a chunk is loaded one
  // chunk before the copies that need it, so no copy waits on a global load.
  auto load_idx = [&](int ch, int (&iv)[PW]) {
#pragma unroll
    for (int u = 0; u < PW; ++u) {
      const int jj = (t + u * 32 * kBW) / PC;
      iv[u] = ch < c_end ? __ldg(a.idx + min(ch * kDN + jj, count - 1)) : 0;
    }
  };
  auto stage = [&](int ch, int buf, const int (&iv)[PW]) {
    const int j0 = ch * kDN;
    const uint32_t w_u = base_u + (uint32_t)(buf * STAGE_B), hr_u = w_u + W_B + HS_B;
#pragma unroll
    for (int u = 0; u < PW; ++u) {
      const int e = t + u * 32 * kBW, jj = e / PC, pc = e % PC;
      int i = iv[u];
      if (i < 0 || i >= a.fmax) i = 0;   // reported by the gate/up kernel
      cp_async16(w_u + (uint32_t)(jj * kDPad + pc * 16),
                 a.rec + (size_t)i * a.rec_stride + a.down_off + (size_t)c0 * 2 + pc * 16);
    }
    // h rows past count are clamped to the last one and zeroed when converted
#pragma unroll
    for (int u = 0; u < kDN * PH / (32 * kBW); ++u) {
      const int e = t + u * 32 * kBW, jj = e / PH, pc = e % PH;
      cp_async16(hr_u + (uint32_t)((jj * BP + pc * 4) * 4), a.h + (size_t)min(j0 + jj, count - 1) * 32 + pc * 4);
    }
  };
  float c[kDM][NT][4];
#pragma unroll
  for (int mt = 0; mt < kDM; ++mt)
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) c[mt][n][e] = 0.f;
  int iv[PW];
#pragma unroll
  for (int s = 0; s < kStages - 1; ++s) {
    if (c_begin + s < c_end) {
      load_idx(c_begin + s, iv);
      stage(c_begin + s, s, iv);
    }
    cp_async_commit();
  }
  load_idx(c_begin + kStages - 1, iv);
  for (int ch = c_begin; ch < c_end; ++ch) {
    const int buf = (ch - c_begin) % kStages;
    const uint32_t w_u = base_u + (uint32_t)(buf * STAGE_B), h_u = w_u + W_B;
    cp_async_wait_1();
    __syncthreads();   // weights and h of chunk ch are in place; chunk ch - 1's buffer is free
    if (ch + kStages - 1 < c_end) stage(ch + kStages - 1, (ch + kStages - 1 - c_begin) % kStages, iv);
    cp_async_commit();
    load_idx(ch + kStages, iv);   // consumed by the next iteration's copies
    // h of the chunk, split into fp16 hi / lo (neurons past count contribute zero)
    {
      const int j0 = ch * kDN;
      const float* hr = reinterpret_cast<const float*>(smem + buf * STAGE_B + W_B + HS_B);
      for (int e = t; e < BP * kDN; e += 32 * kBW) {
        const int b = e / kDN, jj = e % kDN;
        const float v = (j0 + jj < count && b < a.B) ? hr[jj * BP + b] : 0.f;
        __half hi, lo;
        split_h(v, hi, lo);
        reinterpret_cast<__half*>(smem + buf * STAGE_B + W_B + (size_t)b * kHPad)[jj] = hi;
        reinterpret_cast<__half*>(smem + buf * STAGE_B + W_B + (size_t)(BP + b) * kHPad)[jj] = lo;
      }
    }
    __syncthreads();   // h of chunk ch is split
#pragma unroll
    for (int ks = 0; ks < kDN / 16; ++ks) {
      uint32_t bf[NT][2][2];
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int s = 0; s < 2; ++s) {
          const int b = n * 8 + (lane & 7);
          const int jj = ks * 16 + 8 * ((lane >> 3) & 1);
          ldsm_x2(h_u + (uint32_t)((s * BP + b) * kHPad + jj * 2), bf[n][s]);
        }
#pragma unroll
      for (int mt = 0; mt < kDM; ++mt) {
        uint32_t af[4];
        const int jj = ks * 16 + (lane & 7) + 8 * (lane >> 4);                 // neuron (K) of this lane's row address
        const int cc = (warp * kDM + mt) * 16 + 8 * ((lane >> 3) & 1);       // column (M) offset
        ldsm_x4_t(w_u + (uint32_t)(jj * kDPad + cc * 2), af);
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          mma16816(c[mt][n], af, bf[n][0]);
          mma16816(c[mt][n], af, bf[n][1]);
        }
      }
    }
    __syncthreads();   // every thread is done with this buffer before its h is rewritten
  }
  cp_async_wait_all();
  const int g = lane >> 2, tq = lane & 3;
#pragma unroll
  for (int mt = 0; mt < kDM; ++mt)
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int col = c0 + (warp * kDM + mt) * 16 + g + 8 * (e >> 1);
        const int b = n * 8 + 2 * tq + (e & 1);
        if (b < a.B && col < a.d) a.ypart[((size_t)blockIdx.y * a.B + b) * a.d + col] = c[mt][n][e];
      }
}

__global__ void __launch_bounds__(256) down_reduce(const float* ypart, int nsplit, int n, float* y) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= n) return;
  float v = 0.f;
  for (int s = 0; s < nsplit; ++s) v += ypart[(size_t)s * n + e];
  y[e] = v;
}

// ------------------------------------------------------------------ stack glue
// x' = round_fp16((v - mean v) / sqrt(var v + 1e-6)), v = x + y, one block per token;
// the sums run in a fixed order.
__global__ void __launch_bounds__(256) glue_kernel(const __half* x, const float* y, int d, __half* x_out,
                                                   __half* trace_x) {
  __shared__ float red[2][8];
  const int b = blockIdx.x, t = threadIdx.x, lane = t & 31, warp = t >> 5;
  float s = 0.f, s2 = 0.f;
  for (int j = t; j < d; j += 256) {
    const float v = __half2float(x[(size_t)b * d + j]) + y[(size_t)b * d + j];
    s += v;
    s2 += v * v;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    s += __shfl_xor_sync(0xffffffffu, s, o);
    s2 += __shfl_xor_sync(0xffffffffu, s2, o);
  }
  if (lane == 0) { red[0][warp] = s; red[1][warp] = s2; }
  __syncthreads();
  float sum = 0.f, sumsq = 0.f;
#pragma unroll
  for (int w = 0; w < 8; ++w) { sum += red[0][w]; sumsq += red[1][w]; }
  const float mean = sum / (float)d;
  const float sd = sqrtf(fmaxf(sumsq / (float)d - mean * mean, 0.f) + 1e-6f);
  __syncthreads();
  for (int j = t; j < d; j += 256) {
    const float v = __half2float(x[(size_t)b * d + j]) + y[(size_t)b * d + j];
    const __half o = __float2half_rn((v - mean) / sd);
    x_out[(size_t)b * d + j] = o;
    if (trace_x) trace_x[(size_t)b * d + j] = o;
  }
}

// K splits: enough blocks to cover the SMs a few times over, at least two chunks each.
int ksplit_for(int row_blocks, int nch) {
  const int target = 4 * 148;
  int s = (target + row_blocks - 1) / max(row_blocks, 1);
  s = min(s, max(1, nch / 2));
  return max(1, min(s, kMaxKSplit));
}

// Raise a kernel's dynamic shared memory limit once (per kernel, per size increase), so
// the hot launch sequence makes no extra driver calls.
template <typename K>
cudaError_t smem_attr_once(K kern, size_t smem, int& configured) {
  if ((int)smem <= configured) return cudaSuccess;
  const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e == cudaSuccess) configured = (int)smem;
  return e;
}

template <int NT>
cudaError_t launch_rowtok_nt(const RowTokArgs& a, int nmat, int blocks, cudaStream_t s) {
  const bool split = a.tok_lo != nullptr;
  const int ns = split ? 2 : 1;
  const size_t smem = (size_t)kStages * ((size_t)nmat * kRows * kPad + (size_t)ns * NT * 8 * kPad);
  const dim3 grid(blocks, a.ksplit);
  static int conf2 = 0, conf_split = 0, conf1 = 0;
  cudaError_t e;
  if (nmat == 2) {
    if (split) return cudaErrorNotSupported;
    auto k = rowtok_kernel<NT, 2, false>;
    if ((e = smem_attr_once(k, smem, conf2)) != cudaSuccess) return e;
    note_launch();
    k<<<grid, 32 * kBW, smem, s>>>(a);
  } else if (split) {
    auto k = rowtok_kernel<NT, 1, true>;
    if ((e = smem_attr_once(k, smem, conf_split)) != cudaSuccess) return e;
    note_launch();
    k<<<grid, 32 * kBW, smem, s>>>(a);
  } else {
    auto k = rowtok_kernel<NT, 1, false>;
    if ((e = smem_attr_once(k, smem, conf1)) != cudaSuccess) return e;
    note_launch();
    k<<<grid, 32 * kBW, smem, s>>>(a);
  }
  return cudaGetLastError();
}

// The row kernel for rows_max rows (an upper bound when the count is on the device), then
// its epilogue.
cudaError_t launch_rows(RowTokArgs a, RowEpiArgs ep, int nmat, int rows_max, size_t part_floats, cudaStream_t s) {
  const int blocks = (rows_max + kRows - 1) / kRows;
  if (blocks <= 0) return cudaSuccess;
  a.ksplit = ksplit_for(blocks, a.K / kKC);
  const size_t per_split = (size_t)nmat * a.nrows_static * 32;
  a.ksplit = (int)std::max<size_t>(1, std::min<size_t>(a.ksplit, part_floats / per_split));
  if (per_split > part_floats) return cudaErrorInvalidValue;
  cudaError_t e = cudaErrorNotSupported;
  switch ((a.B + 7) / 8) {
    case 1: e = launch_rowtok_nt<1>(a, nmat, blocks, s); break;
    case 2: e = launch_rowtok_nt<2>(a, nmat, blocks, s); break;
    case 3: e = launch_rowtok_nt<3>(a, nmat, blocks, s); break;
    case 4: e = launch_rowtok_nt<4>(a, nmat, blocks, s); break;
  }
  if (e != cudaSuccess) return e;
  ep.ksplit = a.ksplit;
  ep.nmat = nmat;
  ep.part = a.part;
  const long long n = (long long)rows_max * 32;
  note_launch();
  rowtok_epilogue<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(ep);
  return cudaGetLastError();
}

template <int NT>
cudaError_t launch_down_nt(const DownArgs& a, cudaStream_t s) {
  const size_t smem = (size_t)kStages * ((size_t)kDN * kDPad + 2 * (size_t)NT * 8 * kHPad + (size_t)kDN * NT * 8 * 4);
  auto k = down_kernel<NT>;
  static int conf = 0;
  const cudaError_t e = smem_attr_once(k, smem, conf);
  if (e != cudaSuccess) return e;
  note_launch();
  k<<<dim3((a.d + kDCols - 1) / kDCols, a.nsplit), 32 * kBW, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

bool batched_supported(int family, int B, int d, int r) {
  return family == FAM_F16 && B >= 1 && B <= 32 && d % kKC == 0 && r % kKC == 0 && d % kDCols == 0;
}

cudaError_t batched_predict(const BatchedLayer& L, const void* x, int B, uint32_t* mask, float* logits,
                            __half* u_hi, __half* u_lo, float* part, size_t part_floats, cudaStream_t s) {
  RowTokArgs a{};
  a.mode = ROWS_P1;
  a.nrows_static = L.r;
  a.K = L.d;
  a.B = B;
  a.base = L.p1t;
  a.stride = L.p1_row;
  a.tok = reinterpret_cast<const __half*>(x);
  a.part = part;
  RowEpiArgs ea{};
  ea.mode = ROWS_P1;
  ea.nrows_static = L.r;
  ea.B = B;
  ea.u_hi = u_hi;
  ea.u_lo = u_lo;
  cudaError_t e = launch_rows(a, ea, 1, L.r, part_floats, s);
  if (e != cudaSuccess) return e;
  RowTokArgs b{};
  b.mode = ROWS_P2;
  b.nrows_static = L.f;
  b.K = L.r;
  b.B = B;
  b.base = L.p2o;
  b.stride = L.p2_stride;
  b.G = L.G;
  b.nown_max = L.nown_max;
  b.tok = u_hi;
  b.tok_lo = u_lo;
  b.part = part;
  RowEpiArgs eb{};
  eb.mode = ROWS_P2;
  eb.nrows_static = L.f;
  eb.B = B;
  eb.f = L.f;
  eb.thresh = L.thresh;
  eb.logits = logits;
  eb.mask = mask;
  return launch_rows(b, eb, 1, L.f, part_floats, s);
}

cudaError_t batched_ffn(const BatchedLayer& L, const void* x, int B, const uint32_t* mask, const int32_t* idx,
                        const int32_t* count, float* h, float* y, float* part, size_t part_floats, float* ypart,
                        int* err, cudaStream_t s) {
  const int nmat = L.gate_off >= 0 ? 2 : 1;
  RowTokArgs a{};
  a.mode = ROWS_FFN;
  a.nrows_static = L.f;
  a.count = count;
  a.K = L.d;
  a.B = B;
  a.base = L.rec;
  a.stride = L.rec_stride;
  a.idx = idx;
  a.up_off = L.up_off;
  a.gate_off = L.gate_off;
  a.f = L.f;
  a.tok = reinterpret_cast<const __half*>(x);
  a.part = part;
  a.err = err;
  RowEpiArgs ea{};
  ea.mode = ROWS_FFN;
  ea.nrows_static = L.f;
  ea.B = B;
  ea.count = count;
  ea.idx = idx;
  ea.f = L.f;
  ea.bias = L.bias;
  ea.squared = L.act_square;
  ea.mask_in = mask;
  ea.h = h;
  cudaError_t e = launch_rows(a, ea, nmat, L.f, part_floats, s);
  if (e != cudaSuccess) return e;
  DownArgs dn{};
  dn.count = count;
  dn.fmax = L.f;
  dn.d = L.d;
  dn.B = B;
  dn.rec = L.dn;
  dn.rec_stride = L.dn_stride;
  dn.down_off = 0;
  dn.idx = idx;
  dn.h = h;
  dn.ypart = ypart;
  const int col_blocks = (L.d + kDCols - 1) / kDCols;
  dn.nsplit = std::min(kMaxDownSplit, std::max(1, (4 * 148 + col_blocks - 1) / col_blocks));
  switch ((B + 7) / 8) {
    case 1: e = launch_down_nt<1>(dn, s); break;
    case 2: e = launch_down_nt<2>(dn, s); break;
    case 3: e = launch_down_nt<3>(dn, s); break;
    case 4: e = launch_down_nt<4>(dn, s); break;
    default: e = cudaErrorNotSupported;
  }
  if (e != cudaSuccess) return e;
  const int n = B * L.d;
  note_launch();
  down_reduce<<<(n + 255) / 256, 256, 0, s>>>(ypart, dn.nsplit, n, y);
  return cudaGetLastError();
}

size_t batched_part_floats(int d_max, int f_max, int r_max) {
  // row kernels: up to kMaxKSplit splits of the rank rows, and (bounded by this size)
  // splits of the d_ff rows for two matrices; 32 token slots per row
  return std::max((size_t)kMaxKSplit * r_max, (size_t)8 * 2 * f_max) * 32;
}
size_t batched_ypart_floats(int d_max) { return (size_t)kMaxDownSplit * 32 * d_max; }

namespace {
__global__ void count_add_kernel(const int32_t* count, unsigned long long* total, int32_t* layer_count) {
  const int c = *count;
  atomicAdd(total, (unsigned long long)c);
  if (layer_count) *layer_count = c;
}
}  // namespace

cudaError_t batched_count(const int32_t* count, unsigned long long* total, int32_t* layer_count, cudaStream_t s) {
  note_launch();
  count_add_kernel<<<1, 1, 0, s>>>(count, total, layer_count);
  return cudaGetLastError();
}

cudaError_t batched_glue(const void* x, const float* y, int B, int d, void* x_out, void* trace_x, cudaStream_t s) {
  note_launch();
  glue_kernel<<<B, 256, 0, s>>>(reinterpret_cast<const __half*>(x), y, d, reinterpret_cast<__half*>(x_out),
                                reinterpret_cast<__half*>(trace_x));
  return cudaGetLastError();
}

}  // namespace pi
