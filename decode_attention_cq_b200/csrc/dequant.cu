// cq_dequant: codes -> alpha + step * code, for checks only (CalibQuant
// article, Method 2: the cache is represented by integers, a per-channel scale
// and a per-channel bias). Evaluated in double, rounded once to the dtype.
#include "common.cuh"
#include "kernels.h"

namespace cq {

namespace {

template <int BITS>
__device__ __forceinline__ int read_code(const uint8_t* row, cq_layout layout, int i, int j) {
  size_t byte;
  int bit;
  if (layout == CQ_LAYOUT_CANONICAL) {
    byte = (size_t)i * (kD * BITS / 8) + (j * BITS) / 8;
    bit = (j * BITS) % 8;
  } else if (layout == CQ_LAYOUT_OCTET_K) {  // P = 8 / BITS tokens per byte
    byte = (size_t)(i / (8 / BITS)) * kD + j;
    bit = (i % (8 / BITS)) * BITS;
  } else {  // tiles of 32 P tokens
    constexpr int kTile = 32 * (8 / BITS);
    byte = (size_t)(i / kTile) * 4096 + j * 32 + (i % kTile) / (8 / BITS);
    bit = (i % (8 / BITS)) * BITS;
  }
  return (row[byte] >> bit) & ((1 << BITS) - 1);
}

template <typename T, int BITS>
__global__ void __launch_bounds__(256) k_dequant(const uint8_t* __restrict__ codes,
                                                 const T* __restrict__ alpha,
                                                 const T* __restrict__ scale, cq_layout layout,
                                                 int n, size_t row_bytes, T* __restrict__ out) {
  const int row = blockIdx.y;
  const size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= (size_t)n * kD) return;
  const int i = (int)(e / kD), j = (int)(e % kD);
  const int c = read_code<BITS>(codes + (size_t)row * row_bytes, layout, i, j);
  const double a = (double)DT<T>::f(alpha[(size_t)row * kD + j]);
  const double s = (double)DT<T>::f(scale[(size_t)row * kD + j]);
  out[(size_t)row * n * kD + e] = DT<T>::from_double(__dadd_rn(a, __dmul_rn(s, (double)c)));
}

template <typename T>
cudaError_t run(const uint8_t* codes, const T* alpha, const T* scale, cq_layout layout, int rows,
                int n, int bits, T* out, cudaStream_t stream) {
  size_t row_bytes;
  if (layout == CQ_LAYOUT_CANONICAL) row_bytes = (size_t)n * kD * bits / 8;
  else if (layout == CQ_LAYOUT_OCTET_K) row_bytes = (size_t)((n + 8 / bits - 1) / (8 / bits)) * kD;
  else row_bytes = (size_t)((n + 256 / bits - 1) / (256 / bits)) * 4096;
  const dim3 grid((unsigned)(((size_t)n * kD + 255) / 256), rows);
  switch (bits) {
    case 1: k_dequant<T, 1><<<grid, 256, 0, stream>>>(codes, alpha, scale, layout, n, row_bytes, out); break;
    case 2: k_dequant<T, 2><<<grid, 256, 0, stream>>>(codes, alpha, scale, layout, n, row_bytes, out); break;
    case 4: k_dequant<T, 4><<<grid, 256, 0, stream>>>(codes, alpha, scale, layout, n, row_bytes, out); break;
    default: k_dequant<T, 8><<<grid, 256, 0, stream>>>(codes, alpha, scale, layout, n, row_bytes, out); break;
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_dequant(const uint8_t* codes, const void* alpha, const void* scale, cq_dtype dt,
                           cq_layout layout, int rows, int n, int bits, void* out,
                           cudaStream_t stream) {
  if (dt == CQ_F16)
    return run<half>(codes, static_cast<const half*>(alpha), static_cast<const half*>(scale), layout,
                     rows, n, bits, static_cast<half*>(out), stream);
  return run<float>(codes, static_cast<const float*>(alpha), static_cast<const float*>(scale),
                    layout, rows, n, bits, static_cast<float*>(out), stream);
}

}  // namespace cq
