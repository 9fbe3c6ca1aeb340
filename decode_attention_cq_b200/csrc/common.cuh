// Internal helpers shared by the libcalibq kernels (not part of the C ABI).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "calibq.h"
#include "kernels.h"

namespace cq {

// Function attributes (dynamic shared memory, cluster sizes) belong to a device
// context, so the launchers record per device that they have set them.
constexpr int kMaxDevices = 64;
inline int current_device() {
  int dev = 0;
  return cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < kMaxDevices ? dev : -1;
}
// SM count of the current device, read once per device (0 if unknown).
inline int device_sms() {
  static int count[kMaxDevices] = {};  // benign race: every caller stores the same value
  const int dev = current_device();
  int c = 0;
  if (dev < 0) return 0;
  if (count[dev] == 0 && cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess)
    count[dev] = c;
  return count[dev];
}

// ---------------------------------------------------------------- dtypes ----
template <typename T>
struct DT;
template <>
struct DT<half> {
  static __device__ __forceinline__ float f(half v) { return __half2float(v); }
  static __device__ __forceinline__ half from_double(double v) { return __double2half(v); }
  static __device__ __forceinline__ half from_float(float v) { return __float2half_rn(v); }
};
template <>
struct DT<float> {
  static __device__ __forceinline__ float f(float v) { return v; }
  static __device__ __forceinline__ float from_double(double v) { return __double2float_rn(v); }
  static __device__ __forceinline__ float from_float(float v) { return v; }
};

// Eight consecutive elements of a row as floats (16 bytes of half, 32 of float).
__device__ __forceinline__ void load8(const half* p, float (&v)[8]) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  const half2* h = reinterpret_cast<const half2*>(&u);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 f = __half22float2(h[e]);
    v[2 * e] = f.x;
    v[2 * e + 1] = f.y;
  }
}
__device__ __forceinline__ void load8(const float* p, float (&v)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// ------------------------------------------------------------ rounding ----
// Code of x in channel [alpha, beta] with L = 2^bits - 1 (CalibQuant article,
// Method 1): nearest integer to (x - alpha) * L / (beta - alpha), ties to even,
// decided on the IEEE double evaluation ((x - alpha) * L) / (beta - alpha).
//
// A float candidate r_f = (x - alpha) * inv (inv = L / (beta - alpha) in
// float) is within 4 * 2^-24 relative of the real quotient (three roundings
// plus the binary16/32 -> float conversion being exact), i.e. within
// 255 * 2.4e-7 < 2^-12 absolute. Whenever r_f is farther than 2^-12 from a
// half-integer it therefore rounds like the exact value; otherwise the double
// evaluation decides.
__device__ __forceinline__ int quant_code(float xf, float af, float inv, double ad, double bd,
                                          int L) {
  const float r = (xf - af) * inv;
  const float fr = r - floorf(r);
  int c;
  if (fabsf(fr - 0.5f) > 0x1p-12f) {
    c = __float2int_rn(r);
  } else {
    const double rd =
        __ddiv_rn(__dmul_rn(__dsub_rn((double)xf, ad), (double)L), __dsub_rn(bd, ad));
    c = __double2int_rn(rd);
  }
  c = min(max(c, 0), L);
  return inv > 0.f ? c : 0;
}

// 1-bit codes: with L = 1 the rounding rule above reduces to code = [x - alpha >
// (beta - alpha) / 2] = [2x > alpha + beta] (a tie gives 0, as round-half-to-
// even of 1/2 does; a constant channel gives 0). With alpha + beta held as the
// exact pair s_hi + s_lo (two_sum), the float test fl(2x - s_hi) > s_lo is exact:
// when 2x and s_hi are within a factor of two the subtraction is exact
// (Sterbenz); otherwise |2x - s_hi| >= |s_hi| / 2 > |s_lo| and rounding cannot
// move it across s_lo.
__device__ __forceinline__ void two_sum(float a, float b, float& hi, float& lo) {
  hi = __fadd_rn(a, b);
  const float t = __fsub_rn(hi, a);
  lo = __fadd_rn(__fsub_rn(a, __fsub_rn(hi, t)), __fsub_rn(b, t));
}
__device__ __forceinline__ uint32_t code1(float x, float s_hi, float s_lo) {
  return __fmaf_rn(2.f, x, -s_hi) > s_lo ? 1u : 0u;
}

}  // namespace cq
