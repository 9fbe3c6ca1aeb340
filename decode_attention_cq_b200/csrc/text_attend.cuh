// A warp's share of a decode step's attention over full-precision text tokens
// (mixed caches: the quantized visual tokens are attended by the octet
// kernels, the text tokens keep their precision). Used by the text-merge
// kernel and by the one-CTA-per-row decode kernel. Internal header.
#pragma once

#include <cuda_fp16.h>
#include <float.h>
#include <stdint.h>

#include "mma_util.cuh"

namespace cq {
namespace txt {

constexpr int kG = 4;      // query heads per kv-head
constexpr int kBatch = 8;  // text tokens per warp pass
constexpr int kDim = 128;  // head dimension
constexpr int kChunkTokens = 64;     // f16 text tokens per shared-memory chunk (keys or values)
constexpr int kChunkBytes = 16384;   // two 128-byte-swizzled boxes of 64 channels (8 KB each)
constexpr float kLog2e = 1.4426950408889634f;

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

// f16 text tokens on the tensor cores. The keys and the values of every 64
// tokens arrive as chunks g0 + 2 p and g0 + 2 p + 1 (p = 0 .. ntp - 1), each two
// boxes of 64 channels x 64 tokens with the 128-byte swizzle (16-byte chunk c
// of token row r at c ^ (r & 7)). `chunks` gives a chunk's shared-memory
// address once it has landed (wait) and takes the warp's release of it.
// Warp group warp >> 2 (of two) takes every other chunk pair, warp & 3 a
// 16-token slice of it:
//   S = Q K^T       A = the four query heads (rows 4..15 zero), B = key rows
//                   (ldmatrix), f32 accumulators;
//   online softmax  on the raw logits sigma S, per head;
//   O^T += V^T P^T  A = value rows, transposed by ldmatrix; B = P in f16,
//                   which is S's accumulator fragment as it stands (the lane
//                   holding S[head g][tokens 2 tq, 2 tq + 1] is the lane whose
//                   B fragment needs exactly those); the weight sums use the
//                   same rounded values.
// On return: m = running maximum of head g (lanes with g < 4; every lane of a
// group agrees), l = this lane's part of the head's weight sum, o[x] = rows
// 16 x + g and 16 x + g + 8 (channels) of O^T, columns (heads) 2 tq, 2 tq + 1.
template <class Chunks>
__device__ __forceinline__ void text_mma(Chunks& chunks, int g0, const half* q, int ntp, int n_text, float sigma,
                                         int warp, int lane, float& m, float& l, float (&o)[8][4]) {
  using namespace mu;
  const int g = lane >> 2, tq = lane & 3, grp = warp >> 2, sl = warp & 3;
  uint32_t qa[8][4];
#pragma unroll
  for (int s = 0; s < 8; ++s) {
    const uint32_t* qw = reinterpret_cast<const uint32_t*>(q + (g & 3) * kDim + 16 * s + 2 * tq);
    qa[s][0] = g < kG ? qw[0] : 0u;  // q[g][16 s + 2 tq ..]
    qa[s][1] = 0u;
    qa[s][2] = g < kG ? qw[4] : 0u;  // q[g][16 s + 8 + 2 tq ..]
    qa[s][3] = 0u;
  }
  m = -FLT_MAX;
  l = 0.f;
#pragma unroll
  for (int x = 0; x < 8; ++x) o[x][0] = o[x][1] = o[x][2] = o[x][3] = 0.f;
  const int mat = lane >> 3, r = lane & 7;
  const uint32_t rowoff = (uint32_t)(16 * sl + 8 * (mat >> 1) + r) * 128u;  // this lane's ldmatrix row
  for (int tp0 = 0; tp0 < ntp; tp0 += 2) {
    const int tp = tp0 + grp, gk = g0 + 2 * tp, gv = gk + 1;
    const bool act = tp < ntp;
    float sacc[2][4];
#pragma unroll
    for (int n = 0; n < 2; ++n) sacc[n][0] = sacc[n][1] = sacc[n][2] = sacc[n][3] = 0.f;
    if (act) {
      const uint32_t kt = chunks.wait(gk) + rowoff;
#pragma unroll
      for (int s = 0; s < 8; ++s) {  // channels 16 s .. 16 s + 15
        const uint32_t c = (uint32_t)(2 * (s & 3) + (mat & 1));
        uint32_t b[4];
        ldsm_x4(kt + (uint32_t)((s >> 2) * (kChunkBytes / 2)) + ((c ^ (uint32_t)r) << 4), b);
        mma_f16(sacc[0], qa[s], b[0], b[1]);
        mma_f16(sacc[1], qa[s], b[2], b[3]);
      }
      chunks.release(gk);
    }
    // logits of head g at tokens 64 tp + 16 sl + 8 n + 2 tq + e
    const int t0 = kChunkTokens * tp + 16 * sl + 2 * tq;
    float x[2][2], tmax = -FLT_MAX;
    bool ok[2][2];
#pragma unroll
    for (int n = 0; n < 2; ++n)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        ok[n][e] = act && g < kG && t0 + 8 * n + e < n_text;
        x[n][e] = ok[n][e] ? sigma * sacc[n][e] : -FLT_MAX;
        tmax = fmaxf(tmax, x[n][e]);
      }
    tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 1));
    tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 2));
    const float mnew = fmaxf(m, tmax);
    const float sc = ex2_approx((m - mnew) * kLog2e);  // 1 while nothing was seen, 0 on the first tokens
    uint32_t pb[2];
    float psum = 0.f;
#pragma unroll
    for (int n = 0; n < 2; ++n) {
      const float p0 = ok[n][0] ? ex2_approx((x[n][0] - mnew) * kLog2e) : 0.f;
      const float p1 = ok[n][1] ? ex2_approx((x[n][1] - mnew) * kLog2e) : 0.f;
      const __half2 h2 = __floats2half2_rn(p0, p1);
      pb[n] = *reinterpret_cast<const uint32_t*>(&h2);
      const float2 back = __half22float2(h2);  // the weights the MMA uses
      psum += back.x + back.y;
    }
    l = fmaf(l, sc, psum);
    m = mnew;
    // O^T columns are heads 2 tq, 2 tq + 1: their factors sit in lanes 8 tq, 8 tq + 4
    const float sc0 = __shfl_sync(0xffffffffu, sc, 8 * tq), sc1 = __shfl_sync(0xffffffffu, sc, 8 * tq + 4);
#pragma unroll
    for (int xx = 0; xx < 8; ++xx) {
      o[xx][0] *= sc0;
      o[xx][1] *= sc1;
      o[xx][2] *= sc0;
      o[xx][3] *= sc1;
    }
    if (act) {
      const uint32_t vt = chunks.wait(gv) + rowoff;
#pragma unroll
      for (int xx = 0; xx < 8; ++xx) {  // channels 16 xx .. 16 xx + 15
        const uint32_t c = (uint32_t)(2 * (xx & 3) + (mat & 1));
        uint32_t av[4];
        ldsm_x4_trans(vt + (uint32_t)((xx >> 2) * (kChunkBytes / 2)) + ((c ^ (uint32_t)r) << 4), av);
        mma_f16(o[xx], av, pb[0], pb[1]);
      }
      chunks.release(gv);
    }
  }
}

}  // namespace txt
}  // namespace cq
