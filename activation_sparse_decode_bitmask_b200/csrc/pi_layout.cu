// Set-up kernels: re-lay a caller's layer into the library's layout, build the
// hot-neuron order on the device, permute a layer into it, and compact a mask into an
// ascending active-index list.
#include <cuda_fp16.h>
#include <cstdint>

#include "pi_internal.h"
#include "pi_layout.h"

namespace pi {

namespace {

// Row of neuron n in the owner-major predictor layout: block n % G, position n / G.
__device__ __forceinline__ long long owner_row(int n, int G, int nmax) {
  return G > 0 ? (long long)(n % G) * nmax + n / G : (long long)n;
}

// dst row c gets src column c: dst[row(c) * dst_stride + dst_off + r * sizeof(T)] = src[r * src_ld + c]
// (row(c) = c, or the owner-major row when G > 0)
template <typename T>
__global__ void transpose_kernel(const T* __restrict__ src, int rows, int cols, long long src_ld,
                                 uint8_t* __restrict__ dst, long long dst_stride, long long dst_off,
                                 int G, int nmax) {
  __shared__ T tile[32][33];
  const int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
  for (int k = threadIdx.y; k < 32; k += blockDim.y) {
    const int r = r0 + k, c = c0 + threadIdx.x;
    if (r < rows && c < cols) tile[k][threadIdx.x] = src[(long long)r * src_ld + c];
  }
  __syncthreads();
  for (int k = threadIdx.y; k < 32; k += blockDim.y) {
    const int c = c0 + k, r = r0 + threadIdx.x;
    if (r < rows && c < cols)
      *reinterpret_cast<T*>(dst + owner_row(c, G, nmax) * dst_stride + dst_off + (long long)r * sizeof(T)) =
          tile[threadIdx.x][k];
  }
}

// dst + i*dst_stride + dst_off  <-  src + i*src_stride + src_off, `bytes` per row (multiple of 4)
__global__ void copy_rows_kernel(const uint8_t* __restrict__ src, long long src_stride, long long src_off,
                                 uint8_t* __restrict__ dst, long long dst_stride, long long dst_off,
                                 int rows, int bytes, const int32_t* __restrict__ order) {
  const int i = blockIdx.x;
  if (i >= rows) return;
  const int si = order ? order[i] : i;
  const uint8_t* s = src + (long long)si * src_stride + src_off;
  uint8_t* d = dst + (long long)i * dst_stride + dst_off;
  if ((bytes & 15) == 0 && (((uintptr_t)s | (uintptr_t)d) & 15) == 0) {
    for (int k = threadIdx.x; k < bytes / 16; k += blockDim.x)
      reinterpret_cast<uint4*>(d)[k] = reinterpret_cast<const uint4*>(s)[k];
  } else {
    for (int k = threadIdx.x; k < bytes / 4; k += blockDim.x)
      reinterpret_cast<uint32_t*>(d)[k] = reinterpret_cast<const uint32_t*>(s)[k];
  }
}

// per-neuron predictor header: (t_i, b_i) after the r predictor values
__global__ void p2_header_kernel(const float* __restrict__ thresh, const float* __restrict__ bias, int f,
                                 uint8_t* __restrict__ p2o, int p2_stride, int hdr_off, int G, int nmax) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= f) return;
  float* h = reinterpret_cast<float*>(p2o + owner_row(i, G, nmax) * p2_stride + hdr_off);
  h[0] = thresh[i];
  h[1] = bias[i];
}

// one float per row: dst + i*stride + off <- v[i]
__global__ void row_scalar_kernel(const float* __restrict__ v, int f, uint8_t* __restrict__ dst, long long stride,
                                  long long off) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < f) *reinterpret_cast<float*>(dst + (long long)i * stride + off) = v[i];
}

// owner-major rows permuted by neuron: dst row(n) <- src row(order[n])
__global__ void gather_owner_rows_kernel(const uint8_t* __restrict__ src, uint8_t* __restrict__ dst,
                                         const int32_t* __restrict__ order, int f, int G, int nmax, int stride) {
  const int n = blockIdx.x;
  if (n >= f) return;
  const uint4* s = reinterpret_cast<const uint4*>(src + owner_row(order[n], G, nmax) * stride);
  uint4* d = reinterpret_cast<uint4*>(dst + owner_row(n, G, nmax) * stride);
  for (int k = threadIdx.x; k < stride / 16; k += blockDim.x) d[k] = s[k];
}

__global__ void gather_f32_kernel(const float* __restrict__ src, const int32_t* __restrict__ order, int n,
                                  float* __restrict__ dst) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) dst[i] = src[order[i]];
}
__global__ void gather_i32_kernel(const int32_t* __restrict__ src, const int32_t* __restrict__ order, int n,
                                  int32_t* __restrict__ dst) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) dst[i] = src[order[i]];
}
__global__ void iota_kernel(int32_t* p, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) p[i] = i;
}

// rank_i = #{j : f_j > f_i} + #{j < i : f_j == f_i}: the position of neuron i in the
// order by descending frequency with ties by ascending index.  O(n^2) comparisons,
// trivially parallel and exact; order[rank_i] = i.
__global__ void hot_rank_kernel(const float* __restrict__ freq, int n, int32_t* __restrict__ order,
                                int* __restrict__ bad) {
  __shared__ float tile[1024];
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  const float fi = i < n ? freq[i] : 0.f;
  if (i < n && !isfinite(fi)) atomicExch(bad, 1);
  int rank = 0;
  for (int j0 = 0; j0 < n; j0 += 1024) {
    __syncthreads();
    for (int k = threadIdx.x; k < 1024; k += blockDim.x) tile[k] = (j0 + k < n) ? freq[j0 + k] : 0.f;
    __syncthreads();
    const int jn = min(1024, n - j0);
    if (i < n)
      for (int k = 0; k < jn; ++k) {
        const float fj = tile[k];
        rank += (fj > fi) || (fj == fi && j0 + k < i);
      }
  }
  if (i < n) order[rank] = i;
}

// Ordered compaction of the OR of B masks into ascending indices, one block.
__global__ void __launch_bounds__(1024) compact_kernel(const uint32_t* __restrict__ mask, int B, int f,
                                                       int32_t* __restrict__ idx, int32_t* __restrict__ count) {
  __shared__ int wsum[32];
  __shared__ int s_base;
  const int words = f / 32;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  if (t == 0) s_base = 0;
  __syncthreads();
  for (int w0 = 0; w0 < words; w0 += blockDim.x) {
    const int w = w0 + t;
    uint32_t un = 0;
    if (w < words)
      for (int b = 0; b < B; ++b) un |= mask[(long long)b * words + w];
    const int cnt = __popc(un);
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const int nw = blockDim.x / 32;
      int v = lane < nw ? wsum[lane] : 0;
      int inc = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += u;
      }
      if (lane < nw) wsum[lane] = inc - v;   // exclusive prefix of warp totals
    }
    __syncthreads();
    int pos = s_base + wsum[warp] + incl - cnt;
    while (un) {
      const int bit = __ffs(un) - 1;
      un &= un - 1;
      idx[pos++] = w * 32 + bit;
    }
    __syncthreads();
    if (t == blockDim.x - 1) s_base += wsum[warp] + incl;
    __syncthreads();
  }
  if (t == 0) *count = s_base;
}

}  // namespace

static dim3 tgrid(int rows, int cols) { return dim3((cols + 31) / 32, (rows + 31) / 32); }

cudaError_t relayout_transpose(const void* src, int esize, int rows, int cols, long long src_ld,
                               uint8_t* dst, long long dst_stride, long long dst_off, cudaStream_t s,
                               int G, int nmax) {
  const dim3 blk(32, 8);
  if (esize != 4 && esize != 2) return cudaErrorInvalidValue;
  note_launch();
  if (esize == 4)
    transpose_kernel<uint32_t><<<tgrid(rows, cols), blk, 0, s>>>(static_cast<const uint32_t*>(src), rows, cols,
                                                                  src_ld, dst, dst_stride, dst_off, G, nmax);
  else
    transpose_kernel<uint16_t><<<tgrid(rows, cols), blk, 0, s>>>(static_cast<const uint16_t*>(src), rows, cols,
                                                                  src_ld, dst, dst_stride, dst_off, G, nmax);
  return cudaGetLastError();
}

cudaError_t relayout_copy_rows(const void* src, long long src_stride, long long src_off, uint8_t* dst,
                               long long dst_stride, long long dst_off, int rows, int bytes,
                               const int32_t* order, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  note_launch();
  copy_rows_kernel<<<rows, 128, 0, s>>>(static_cast<const uint8_t*>(src), src_stride, src_off, dst, dst_stride,
                                        dst_off, rows, bytes, order);
  return cudaGetLastError();
}

cudaError_t relayout_p2_header(const float* thresh, const float* bias, int f, uint8_t* p2o, int p2_stride,
                               int hdr_off, int G, int nmax, cudaStream_t s) {
  note_launch();
  p2_header_kernel<<<(f + 255) / 256, 256, 0, s>>>(thresh, bias, f, p2o, p2_stride, hdr_off, G, nmax);
  return cudaGetLastError();
}

cudaError_t relayout_row_scalar(const float* v, int f, uint8_t* dst, long long stride, long long off, cudaStream_t s) {
  note_launch();
  row_scalar_kernel<<<(f + 255) / 256, 256, 0, s>>>(v, f, dst, stride, off);
  return cudaGetLastError();
}

cudaError_t gather_owner_rows(const uint8_t* src, uint8_t* dst, const int32_t* order, int f, int G, int nmax,
                              int stride, cudaStream_t s) {
  note_launch();
  gather_owner_rows_kernel<<<f, 128, 0, s>>>(src, dst, order, f, G, nmax, stride);
  return cudaGetLastError();
}

cudaError_t hot_order(const float* freq, int n, int32_t* order, int* bad, cudaStream_t s) {
  note_launch();
  hot_rank_kernel<<<(n + 255) / 256, 256, 0, s>>>(freq, n, order, bad);
  return cudaGetLastError();
}

cudaError_t gather_f32(const float* src, const int32_t* order, int n, float* dst, cudaStream_t s) {
  note_launch();
  gather_f32_kernel<<<(n + 255) / 256, 256, 0, s>>>(src, order, n, dst);
  return cudaGetLastError();
}
cudaError_t gather_i32(const int32_t* src, const int32_t* order, int n, int32_t* dst, cudaStream_t s) {
  note_launch();
  gather_i32_kernel<<<(n + 255) / 256, 256, 0, s>>>(src, order, n, dst);
  return cudaGetLastError();
}
cudaError_t iota_i32(int32_t* p, int n, cudaStream_t s) {
  note_launch();
  iota_kernel<<<(n + 255) / 256, 256, 0, s>>>(p, n);
  return cudaGetLastError();
}

cudaError_t launch_compact(const uint32_t* mask, int B, int f, int32_t* idx, int32_t* count, cudaStream_t s) {
  note_launch();
  compact_kernel<<<1, 1024, 0, s>>>(mask, B, f, idx, count);
  return cudaGetLastError();
}

}  // namespace pi
