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

namespace cq {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kG = 4;

// Four consecutive elements of a row: raw (as loaded) and as floats.
template <typename T>
struct Raw4;
template <>
struct Raw4<half> {
  using type = uint2;
  __device__ static type load(const half* p) { return __ldg(reinterpret_cast<const uint2*>(p)); }
  __device__ static type zero() { return make_uint2(0u, 0u); }
  __device__ static void to_float(const type& u, float (&v)[4]) {
    const float2 a = __half22float2(*reinterpret_cast<const half2*>(&u.x));
    const float2 b = __half22float2(*reinterpret_cast<const half2*>(&u.y));
    v[0] = a.x;
    v[1] = a.y;
    v[2] = b.x;
    v[3] = b.y;
  }
};
template <>
struct Raw4<float> {
  using type = float4;
  __device__ static type load(const float* p) { return __ldg(reinterpret_cast<const float4*>(p)); }
  __device__ static type zero() { return make_float4(0.f, 0.f, 0.f, 0.f); }
  __device__ static void to_float(const type& u, float (&v)[4]) {
    v[0] = u.x;
    v[1] = u.y;
    v[2] = u.z;
    v[3] = u.w;
  }
};
__device__ __forceinline__ void load4(const half* p, float (&v)[4]) { Raw4<half>::to_float(Raw4<half>::load(p), v); }
__device__ __forceinline__ void load4(const float* p, float (&v)[4]) { Raw4<float>::to_float(Raw4<float>::load(p), v); }

// grid: one CTA per (batch, kv-head) row. Warp w takes batches of 8 text
// tokens (batch w, w + 8, ...); lane l holds channels 4 l .. 4 l + 3 of the
// keys and values. The 32 partial dot products of a batch (8 tokens x 4 heads)
// are summed over the lanes with one transposed butterfly (31 shuffles), after
// which lane l owns the logit of token l / 4, head l % 4.
template <typename T>
__global__ void __launch_bounds__(kThreads) k_text_merge(const T* __restrict__ q, const T* __restrict__ kt,
                                                         const T* __restrict__ vt, int n_text,
                                                         const float* __restrict__ part_o,
                                                         const float* __restrict__ part_lse, T* __restrict__ out,
                                                         int Hq, int Hkv, float sigma) {
  constexpr int kBatch = 8;
  __shared__ float s_m[kWarps][kG], s_l[kWarps][kG];
  __shared__ float s_acc[kWarps][kG][kD];
  const int row = blockIdx.x, b = row / Hkv, hkv = row % Hkv;
  // warp index broadcast from lane 0: known warp-uniform, so shuffles under branches and
  // loops on it need no reconvergence
  const int t = threadIdx.x, warp = __shfl_sync(0xffffffffu, t >> 5, 0), lane = t & 31;
  const int my_h = lane & 3;  // head of the logit this lane owns after the butterfly
  const size_t bh0 = (size_t)b * Hq + (size_t)kG * hkv;  // first query head of the row

  float qv[kG][4];
#pragma unroll
  for (int h = 0; h < kG; ++h) load4(q + (bh0 + h) * kD + 4 * lane, qv[h]);
  float m[kG], l[kG], acc[kG][4];
#pragma unroll
  for (int h = 0; h < kG; ++h) {
    m[h] = -FLT_MAX;
    l[h] = 0.f;
    acc[h][0] = acc[h][1] = acc[h][2] = acc[h][3] = 0.f;
  }
  const T* kr = kt + (size_t)row * n_text * kD + 4 * lane;
  const T* vr = vt + (size_t)row * n_text * kD + 4 * lane;
  using R = Raw4<T>;
  // the next pass's keys and values are loaded while this pass computes
  typename R::type kraw[kBatch], vraw[kBatch];
#pragma unroll
  for (int u = 0; u < kBatch; ++u) {
    const int j = kBatch * warp + u;
    kraw[u] = j < n_text ? R::load(kr + (size_t)j * kD) : R::zero();
    vraw[u] = j < n_text ? R::load(vr + (size_t)j * kD) : R::zero();
  }
  // every warp runs every pass (a pass past the end masks all its tokens): the
  // butterfly's shuffles must not sit in a loop whose trip count the compiler
  // sees as per-thread, where each costs several times its latency
  for (int jb = 0; jb < n_text; jb += kBatch * kWarps) {
    const int j0 = jb + kBatch * warp;
    typename R::type kcur[kBatch], vcur[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      kcur[u] = kraw[u];
      vcur[u] = vraw[u];
      const int j = j0 + kBatch * kWarps + u;
      kraw[u] = j < n_text ? R::load(kr + (size_t)j * kD) : R::zero();
      vraw[u] = j < n_text ? R::load(vr + (size_t)j * kD) : R::zero();
    }
    float dv[kBatch * kG];  // partial dots, index 4 token + head
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      float kv[4];
      R::to_float(kcur[u], kv);
#pragma unroll
      for (int h = 0; h < kG; ++h)
        dv[kG * u + h] = qv[h][0] * kv[0] + qv[h][1] * kv[1] + qv[h][2] * kv[2] + qv[h][3] * kv[3];
    }
    // transposed butterfly: after the step with offset s, lane l keeps the
    // indices whose bit s matches its own; at the end dv[0] = full dot of index l
#pragma unroll
    for (int s = 16; s >= 1; s >>= 1) {
      const bool upper = lane & s;
#pragma unroll
      for (int i = 0; i < s; ++i) {
        const float send = upper ? dv[i] : dv[i + s];
        const float keep = upper ? dv[i + s] : dv[i];
        dv[i] = keep + __shfl_xor_sync(0xffffffffu, send, s);
      }
    }
    const bool valid = j0 + (lane >> 2) < n_text;
    const float x = valid ? sigma * dv[0] : -FLT_MAX;
    // batch maximum and weights per head: lanes with equal lane % 4
    float bm = x;
    bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 4));
    bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 8));
    bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 16));
    float mine_m = m[0];
#pragma unroll
    for (int h = 1; h < kG; ++h)
      if (my_h == h) mine_m = m[h];
    const float mn = fmaxf(mine_m, bm);
    const float p = valid ? expf(x - mn) : 0.f;
    const float sc = expf(mine_m - mn);
    float ps = p;
    ps += __shfl_xor_sync(0xffffffffu, ps, 4);
    ps += __shfl_xor_sync(0xffffffffu, ps, 8);
    ps += __shfl_xor_sync(0xffffffffu, ps, 16);
    // every lane updates its 4 channels of all 4 heads
    float vv[kBatch][4];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) R::to_float(vcur[u], vv[u]);
#pragma unroll
    for (int h = 0; h < kG; ++h) {
      const float sch = __shfl_sync(0xffffffffu, sc, h);
      const float mh = __shfl_sync(0xffffffffu, mn, h);
      const float lh = __shfl_sync(0xffffffffu, ps, h);
      l[h] = fmaf(l[h], sch, lh);
      m[h] = mh;
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[h][c] *= sch;
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const float pu = __shfl_sync(0xffffffffu, p, 4 * u + h);
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[h][c] = fmaf(pu, vv[u][c], acc[h][c]);
      }
    }
  }
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
