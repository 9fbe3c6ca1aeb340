// One warp's share of a decode step's attention over full-precision text tokens
// (mixed caches: the quantized visual tokens are attended by the octet
// kernels, the text tokens keep their precision). Used by the text-merge
// kernel and by the one-CTA-per-row decode kernel. Internal header.
#pragma once

#include <cuda_fp16.h>
#include <float.h>
#include <stdint.h>

namespace cq {
namespace txt {

constexpr int kG = 4;      // query heads per kv-head
constexpr int kBatch = 8;  // text tokens per warp pass
constexpr int kDim = 128;  // head dimension

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

// Warp `warp` of kWarps takes the text tokens in batches of 8 (batch warp,
// warp + kWarps, ...); lane l holds channels 4 l .. 4 l + 3 of the keys and
// values (kr, vr point at channel 4 l of the row's first token; qv holds the
// same channels of the G = 4 queries). The 32 partial dot products of a batch
// (8 tokens x 4 heads) are summed over the lanes with one transposed butterfly
// (31 shuffles), after which lane l owns the logit sigma q.k of token l / 4,
// head l % 4. The warp keeps, per head, a running maximum m, sum of weights l
// and weighted value sum acc (its lane's 4 channels); the next batch's keys and
// values are loaded while the current one computes. The loop's trip count
// depends on n_text only: a shuffle inside a loop whose trip count the
// compiler sees as per-thread costs several times its latency.
template <typename T, int kWarps>
__device__ __forceinline__ void warp_text_attend(const float (&qv)[kG][4], const T* __restrict__ kr,
                                                 const T* __restrict__ vr, int n_text, float sigma, int warp,
                                                 int lane, float (&m)[kG], float (&l)[kG], float (&acc)[kG][4]) {
  using R = Raw4<T>;
  const int my_h = lane & 3;  // head of the logit this lane owns after the butterfly
#pragma unroll
  for (int h = 0; h < kG; ++h) {
    m[h] = -FLT_MAX;
    l[h] = 0.f;
    acc[h][0] = acc[h][1] = acc[h][2] = acc[h][3] = 0.f;
  }
  typename R::type kraw[kBatch], vraw[kBatch];
#pragma unroll
  for (int u = 0; u < kBatch; ++u) {
    const int j = kBatch * warp + u;
    kraw[u] = j < n_text ? R::load(kr + (size_t)j * kDim) : R::zero();
    vraw[u] = j < n_text ? R::load(vr + (size_t)j * kDim) : R::zero();
  }
  for (int jb = 0; jb < n_text; jb += kBatch * kWarps) {
    const int j0 = jb + kBatch * warp;
    typename R::type kcur[kBatch], vcur[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      kcur[u] = kraw[u];
      vcur[u] = vraw[u];
      const int j = j0 + kBatch * kWarps + u;
      kraw[u] = j < n_text ? R::load(kr + (size_t)j * kDim) : R::zero();
      vraw[u] = j < n_text ? R::load(vr + (size_t)j * kDim) : R::zero();
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
}

}  // namespace txt
}  // namespace cq
