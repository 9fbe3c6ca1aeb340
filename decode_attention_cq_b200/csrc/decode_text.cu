// Mixed caches: the full-precision text tokens next to a quantized visual
// cache (the CalibQuant article quantizes the visual KV cache; text tokens keep
// their precision). The visual part is attended by an octet decode kernel in
// partial mode (normalized fp32 result + ln sum exp of its calibrated logits);
// this kernel attends the G = 4 query heads of one (batch, kv-head) row over
// the text keys / values with an online softmax on the raw logits sigma q.k,
// and merges both parts by their log-sum-exps into the final output:
//   o = (e^{lse_v} o_v + sum_j e^{x_j} v_j) / (e^{lse_v} + sum_j e^{x_j}).
#include <float.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "text_attend.cuh"

namespace cq {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kG = 4;

__device__ __forceinline__ void load4(const half* p, float (&v)[4]) {
  txt::Raw4<half>::to_float(txt::Raw4<half>::load(p), v);
}
__device__ __forceinline__ void load4(const float* p, float (&v)[4]) {
  txt::Raw4<float>::to_float(txt::Raw4<float>::load(p), v);
}

// grid: one CTA per (batch, kv-head) row; each warp attends its share of the
// row's text tokens (txt::warp_text_attend), then the warps' parts and the
// visual part are merged by their log-sum-exps.
template <typename T>
__global__ void __launch_bounds__(kThreads) k_text_merge(const T* __restrict__ q, const T* __restrict__ kt,
                                                         const T* __restrict__ vt, int n_text,
                                                         const float* __restrict__ part_o,
                                                         const float* __restrict__ part_lse, T* __restrict__ out,
                                                         int Hq, int Hkv, float sigma) {
  __shared__ float s_m[kWarps][kG], s_l[kWarps][kG];
  __shared__ float s_acc[kWarps][kG][kD];
  const int row = blockIdx.x, b = row / Hkv, hkv = row % Hkv;
  // warp index broadcast from lane 0: known warp-uniform, so shuffles under branches and
  // loops on it need no reconvergence
  const int t = threadIdx.x, warp = __shfl_sync(0xffffffffu, t >> 5, 0), lane = t & 31;
  const size_t bh0 = (size_t)b * Hq + (size_t)kG * hkv;  // first query head of the row

  float qv[kG][4];
#pragma unroll
  for (int h = 0; h < kG; ++h) load4(q + (bh0 + h) * kD + 4 * lane, qv[h]);
  float m[kG], l[kG], acc[kG][4];
  txt::warp_text_attend<T, kWarps>(qv, kt + (size_t)row * n_text * kD + 4 * lane,
                                   vt + (size_t)row * n_text * kD + 4 * lane, n_text, sigma, warp, lane, m, l, acc);
#pragma unroll
  for (int h = 0; h < kG; ++h) {
    if (lane == 0) {
      s_m[warp][h] = m[h];
      s_l[warp][h] = l[h];
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) s_acc[warp][h][4 * lane + c] = acc[h][c];
  }
  __syncthreads();
  // thread (h, ch), two per thread: merge the warps' text parts and the visual part
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int idx = 2 * t + e, h = idx >> 7, ch = idx & 127;
    const size_t bh = bh0 + h;
    const float lse_v = part_lse[bh];
    float M = lse_v;
    for (int w = 0; w < kWarps; ++w)
      if (s_l[w][h] > 0.f) M = fmaxf(M, s_m[w][h]);
    const float wv = expf(lse_v - M);
    float num = wv * part_o[bh * kD + ch], den = wv;
    for (int w = 0; w < kWarps; ++w) {
      if (s_l[w][h] > 0.f) {
        const float f = expf(s_m[w][h] - M);
        num = fmaf(f, s_acc[w][h][ch], num);
        den = fmaf(f, s_l[w][h], den);
      }
    }
    out[bh * kD + ch] = DT<T>::from_float(num / den);
  }
}

}  // namespace

size_t text_merge_workspace_bytes(int B, int Hq) {
  return (size_t)B * Hq * kD * sizeof(float) + (size_t)B * Hq * sizeof(float);
}

cudaError_t launch_text_merge(const DecodeArgs& a, cq_dtype dt, const void* k_text, const void* v_text, int n_text,
                              cudaStream_t stream) {
  const int rows = a.B * a.Hkv;
  if (dt == CQ_F16)
    k_text_merge<half><<<rows, kThreads, 0, stream>>>(
        static_cast<const half*>(a.q), static_cast<const half*>(k_text), static_cast<const half*>(v_text), n_text,
        a.part_o, a.part_lse, static_cast<half*>(a.out), a.Hq, a.Hkv, a.sigma);
  else
    k_text_merge<float><<<rows, kThreads, 0, stream>>>(
        static_cast<const float*>(a.q), static_cast<const float*>(k_text), static_cast<const float*>(v_text), n_text,
        a.part_o, a.part_lse, static_cast<float*>(a.out), a.Hq, a.Hkv, a.sigma);
  return cudaGetLastError();
}

}  // namespace cq
