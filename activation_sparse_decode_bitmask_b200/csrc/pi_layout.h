// Set-up kernels (layout, hot order, compaction); see pi_layout.cu.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace pi {
// G > 0: destination rows are laid out owner-major (row of n = (n % G) * nmax + n / G)
cudaError_t relayout_transpose(const void* src, int esize, int rows, int cols, long long src_ld,
                               uint8_t* dst, long long dst_stride, long long dst_off, cudaStream_t s,
                               int G = 0, int nmax = 0);
cudaError_t relayout_copy_rows(const void* src, long long src_stride, long long src_off, uint8_t* dst,
                               long long dst_stride, long long dst_off, int rows, int bytes,
                               const int32_t* order, cudaStream_t s);
cudaError_t relayout_p2_header(const float* thresh, const float* bias, int f, uint8_t* p2o, int p2_stride,
                               int hdr_off, int G, int nmax, cudaStream_t s);
cudaError_t relayout_row_scalar(const float* v, int f, uint8_t* dst, long long stride, long long off, cudaStream_t s);
cudaError_t gather_owner_rows(const uint8_t* src, uint8_t* dst, const int32_t* order, int f, int G, int nmax,
                              int stride, cudaStream_t s);
cudaError_t hot_order(const float* freq, int n, int32_t* order, int* bad, cudaStream_t s);
cudaError_t gather_f32(const float* src, const int32_t* order, int n, float* dst, cudaStream_t s);
cudaError_t gather_i32(const int32_t* src, const int32_t* order, int n, int32_t* dst, cudaStream_t s);
cudaError_t iota_i32(int32_t* p, int n, cudaStream_t s);
}  // namespace pi
