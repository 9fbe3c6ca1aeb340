// cq_quantize_kv kernels: per-channel statistics and bit packing
// (CalibQuant article, Method 1: uniform b-bit quantization with the range
// [alpha, beta] refined per channel over the n tokens of each (batch, head)).
//
// Two launches, both HBM-bound reads of the input cache:
//   k_stats  grid (rows, S): per-split per-channel min/max -> workspace
//   k_pack   grid (rows, tiles): folds the S partials into alpha/beta, writes
//            alpha and the step (once per row) and the packed codes of its tile.
#include <float.h>

#include <type_traits>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace cq {

namespace {

constexpr int kThreads = 256;
constexpr int kTpr = kD / 8;            // threads per token row (8 channels each)
constexpr int kRpi = kThreads / kTpr;   // token rows per iteration

// Where the pack functions read token rows from (the row in global memory).
template <typename T>
struct GlobalRows {
  const T* __restrict__ row0;  // token 0 of the (batch, head) row
  __device__ __forceinline__ void load8(int i, int ch, float (&v)[8]) const {
    cq::load8(row0 + (size_t)i * kD + ch, v);
  }
  // the same eight binary16 values as four packed pairs
  __device__ __forceinline__ void load8h(int i, int ch, uint32_t (&w)[4]) const {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(row0 + (size_t)i * kD + ch));
    w[0] = u.x;
    w[1] = u.y;
    w[2] = u.z;
    w[3] = u.w;
  }
};

// Per-channel min / max of tokens [i0, i1) of one row; thread j < kD gets
// channel j's pair. 16 threads cover a token row (8 channels each).
// smn, smx: kRpi x kD floats each of shared scratch.
template <typename T>
__device__ __forceinline__ void tile_minmax(const T* __restrict__ xrow, int i0, int i1, float& a, float& b,
                                            float (*smn)[kD], float (*smx)[kD]) {
  const int cg = threadIdx.x % kTpr, r = threadIdx.x / kTpr;
  float mn[8], mx[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    mn[e] = FLT_MAX;
    mx[e] = -FLT_MAX;
  }
  const T* base = xrow + cg * 8;
  if constexpr (std::is_same<T, half>::value) {
    // binary16 extremes are binary16 values: packed pairs, no conversions
    __half2 mn2[4], mx2[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      mn2[p] = __half2half2(__ushort_as_half(0x7c00u));  // +inf
      mx2[p] = __half2half2(__ushort_as_half(0xfc00u));  // -inf
    }
#pragma unroll 8
    for (int i = i0 + r; i < i1; i += kRpi) {
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(base + (size_t)i * kD));
      const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        mn2[p] = __hmin2(mn2[p], h[p]);
        mx2[p] = __hmax2(mx2[p], h[p]);
      }
    }
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      mn[2 * p] = __low2float(mn2[p]);
      mn[2 * p + 1] = __high2float(mn2[p]);
      mx[2 * p] = __low2float(mx2[p]);
      mx[2 * p + 1] = __high2float(mx2[p]);
    }
  } else {
#pragma unroll 8
    for (int i = i0 + r; i < i1; i += kRpi) {
      float v[8];
      load8(base + (size_t)i * kD, v);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        mn[e] = fminf(mn[e], v[e]);
        mx[e] = fmaxf(mx[e], v[e]);
      }
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    smn[r][cg * 8 + e] = mn[e];
    smx[r][cg * 8 + e] = mx[e];
  }
  __syncthreads();
  a = FLT_MAX;
  b = -FLT_MAX;
  if (threadIdx.x < kD) {
    for (int q = 0; q < kRpi; ++q) {
      a = fminf(a, smn[q][threadIdx.x]);
      b = fmaxf(b, smx[q][threadIdx.x]);
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(kThreads) k_stats(const T* __restrict__ x, int n, int S,
                                                    float* __restrict__ part) {
  const int row = blockIdx.x, s = blockIdx.y;
  const int per = (n + S - 1) / S;
  const int i0 = s * per, i1 = min(n, i0 + per);
  __shared__ float smn[kRpi][kD], smx[kRpi][kD];
  float a, b;
  tile_minmax<T>(x + (size_t)row * n * kD, i0, i1, a, b, smn, smx);
  if (threadIdx.x < kD) {
    float* out = part + ((size_t)row * S + s) * 2 * kD;
    out[threadIdx.x] = a;
    out[kD + threadIdx.x] = b;
  }
}

// A row's folded statistics, shared by the CTA that packs one of its tiles.
struct RowStats {
  float alpha[kD], beta[kD];
  float inv[kD];     // L / (beta - alpha), 0 for a constant channel
  uint16_t thr[kD];  // binary16 rows: bits of the smallest binary16 above (alpha + beta) / 2
};

// 1-bit code of a binary16 value x: [x > (alpha + beta) / 2] (the rounding rule
// with L = 1, see code1). alpha and beta are binary16 values, so their mean mu is
// exact in double, and x > mu holds exactly when x >= the smallest binary16 above
// mu: one packed comparison per two values decides the codes.
__device__ __forceinline__ uint16_t half_above_mid(float a, float b) {
  const double mu = ((double)a + (double)b) * 0.5;
  const uint16_t h = __half_as_ushort(__double2half(mu));  // nearest, ties to even
  if ((double)__half2float(__ushort_as_half(h)) > mu) return h;  // nearest is above: nothing between
  if ((h & 0x7fffu) == 0) return 0x0001u;                        // +-0: the smallest subnormal
  return (h & 0x8000u) ? (uint16_t)(h - 1u) : (uint16_t)(h + 1u);  // one step up
}

// Per pair of channels (2p, 2p + 1): 0xffff in each half whose value is >= its threshold.
__device__ __forceinline__ uint32_t ge_mask(uint32_t x2, uint32_t thr2) {
  return __hge2_mask(*reinterpret_cast<const __half2*>(&x2), *reinterpret_cast<const __half2*>(&thr2));
}

// Folds the S partials of `row` ([S][min, max][kD], global or shared memory)
// into shared alpha/beta/inv; with `write` also stores the row's alpha and step.
template <typename T>
__device__ __forceinline__ void fold_stats(const float* p, int S, int L, bool write, int row,
                                           RowStats& st,
                                           T* __restrict__ alpha_out, T* __restrict__ scale_out) {
  if (threadIdx.x < kD) {
    const int j = threadIdx.x;
    float a = FLT_MAX, b = -FLT_MAX;
    for (int s = 0; s < S; ++s) {
      a = fminf(a, p[s * 2 * kD + j]);
      b = fmaxf(b, p[s * 2 * kD + kD + j]);
    }
    st.alpha[j] = a;
    st.beta[j] = b;
    st.inv[j] = (b > a) ? (float)L / (b - a) : 0.f;
    if constexpr (std::is_same<T, half>::value) st.thr[j] = half_above_mid(a, b);
    if (write) {
      alpha_out[(size_t)row * kD + j] = DT<T>::from_float(a);  // exact: an input value
      const double step = __ddiv_rn(__dsub_rn((double)b, (double)a), (double)L);
      scale_out[(size_t)row * kD + j] = DT<T>::from_double(step);
    }
  }
  __syncthreads();
}

// Canonical layout: each thread turns 8 channels of one token into 8*BITS bits.
template <typename T, int BITS, typename Src>
__device__ __forceinline__ void k_pack_canonical_tile(const Src& src, int n, int row, int tile, int tile_tokens,
    const RowStats& st, uint8_t* __restrict__ codes) {
  constexpr int L = (1 << BITS) - 1;
  const int cg = threadIdx.x % kTpr, r = threadIdx.x / kTpr;
  if constexpr (BITS == 1 && std::is_same<T, half>::value) {
    // channel 2p's code from the low half of pair p lands on bit 2p, channel
    // 2p + 1's from the high half on bit 17 + 2p (folded down to 2p + 1)
    uint32_t th[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) th[p] = st.thr[cg * 8 + 2 * p] | ((uint32_t)st.thr[cg * 8 + 2 * p + 1] << 16);
    const int i0 = tile * tile_tokens, i1 = min(n, i0 + tile_tokens);
    uint8_t* cr = codes + (size_t)row * n * (kD / 8) + cg;
    for (int i = i0 + r; i < i1; i += kRpi) {
      uint32_t w[4], acc = 0;
      src.load8h(i, cg * 8, w);
#pragma unroll
      for (int p = 0; p < 4; ++p) acc |= ge_mask(w[p], th[p]) & ((1u << (2 * p)) | (1u << (17 + 2 * p)));
      cr[(size_t)i * (kD / 8)] = (uint8_t)(acc | (acc >> 16));
    }
  } else {
    float af[8], inv[8], hi[8], lo[8];
    double ad[8], bd[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      af[e] = st.alpha[cg * 8 + e];
      inv[e] = st.inv[cg * 8 + e];
      ad[e] = (double)af[e];
      bd[e] = (double)st.beta[cg * 8 + e];
      two_sum(af[e], st.beta[cg * 8 + e], hi[e], lo[e]);  // used for 1-bit codes
    }
    const int i0 = tile * tile_tokens, i1 = min(n, i0 + tile_tokens);
    uint8_t* cr = codes + (size_t)row * n * (kD * BITS / 8) + cg * BITS;
    for (int i = i0 + r; i < i1; i += kRpi) {
      float v[8];
      src.load8(i, cg * 8, v);
      uint64_t packed = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        if constexpr (BITS == 1)
          packed |= (uint64_t)code1(v[e], hi[e], lo[e]) << e;
        else
          packed |= (uint64_t)quant_code(v[e], af[e], inv[e], ad[e], bd[e], L) << (e * BITS);
      }
      uint8_t* dst = cr + (size_t)i * (kD * BITS / 8);
      if (BITS == 1) *dst = (uint8_t)packed;
      if (BITS == 2) *reinterpret_cast<uint16_t*>(dst) = (uint16_t)packed;
      if (BITS == 4) *reinterpret_cast<uint32_t*>(dst) = (uint32_t)packed;
      if (BITS == 8) *reinterpret_cast<uint64_t*>(dst) = packed;
    }
  }
}

template <typename T, int BITS>
__global__ void __launch_bounds__(kThreads) k_pack_canonical(
    const T* __restrict__ x, int n, int S, int tile_tokens, const float* __restrict__ part,
    uint8_t* __restrict__ codes, T* __restrict__ alpha_out, T* __restrict__ scale_out) {
  __shared__ RowStats st;
  const int row = blockIdx.x;
  fold_stats<T>(part + (size_t)row * S * 2 * kD, S, (1 << BITS) - 1, blockIdx.y == 0, row, st, alpha_out,
                scale_out);
  k_pack_canonical_tile<T, BITS>(GlobalRows<T>{x + (size_t)row * n * kD}, n, row, blockIdx.y, tile_tokens, st, codes);
}

// OCTET_K layout (bits = 1): a thread owns one token octet (8 tokens) x 8
// channels, i.e. 8 consecutive bytes of the layout.
template <typename T, typename Src>
__device__ __forceinline__ void k_pack_octet_k_tile(const Src& src, int n, int row, int tile, int tile_tokens,
    const RowStats& st, uint8_t* __restrict__ codes) {
  const int cb = threadIdx.x % kTpr, r = threadIdx.x / kTpr;
  if constexpr (std::is_same<T, half>::value) {
    // token k's codes of channel pair p go to bits k (channel 2p) and 16 + k
    // (channel 2p + 1) of acc[p]; two byte permutes give the 8 channel bytes
    uint32_t th[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) th[p] = st.thr[cb * 8 + 2 * p] | ((uint32_t)st.thr[cb * 8 + 2 * p + 1] << 16);
    const int octets = (n + 7) / 8;
    const int m0 = tile * (tile_tokens / 8), m1 = min(octets, m0 + tile_tokens / 8);
    uint8_t* cr = codes + (size_t)row * octets * kD + cb * 8;
    for (int m = m0 + r; m < m1; m += kRpi) {
      uint32_t acc[4] = {0u, 0u, 0u, 0u};
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        if (8 * m + k < n) {
          uint32_t w[4];
          src.load8h(8 * m + k, cb * 8, w);
#pragma unroll
          for (int p = 0; p < 4; ++p) acc[p] |= ge_mask(w[p], th[p]) & (0x00010001u << k);
        }
      }
      *reinterpret_cast<uint2*>(cr + (size_t)m * kD) =
          make_uint2(__byte_perm(acc[0], acc[1], 0x6420), __byte_perm(acc[2], acc[3], 0x6420));
    }
  } else {
    float hi[8], lo[8];  // alpha + beta of the thread's channels as an exact pair
#pragma unroll
    for (int e = 0; e < 8; ++e) two_sum(st.alpha[cb * 8 + e], st.beta[cb * 8 + e], hi[e], lo[e]);
    const int octets = (n + 7) / 8;
    const int m0 = tile * (tile_tokens / 8), m1 = min(octets, m0 + tile_tokens / 8);
    uint8_t* cr = codes + (size_t)row * octets * kD + cb * 8;
    for (int m = m0 + r; m < m1; m += kRpi) {
      uint64_t bytes = 0;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int i = 8 * m + k;
        if (i < n) {
          float v[8];
          src.load8(i, cb * 8, v);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            bytes |= (uint64_t)code1(v[e], hi[e], lo[e]) << (8 * e + k);
        }
      }
      *reinterpret_cast<uint64_t*>(cr + (size_t)m * kD) = bytes;
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(kThreads) k_pack_octet_k(
    const T* __restrict__ x, int n, int S, int tile_tokens, const float* __restrict__ part,
    uint8_t* __restrict__ codes, T* __restrict__ alpha_out, T* __restrict__ scale_out) {
  __shared__ RowStats st;
  const int row = blockIdx.x;
  fold_stats<T>(part + (size_t)row * S * 2 * kD, S, 1, blockIdx.y == 0, row, st, alpha_out,
                scale_out);
  k_pack_octet_k_tile<T>(GlobalRows<T>{x + (size_t)row * n * kD}, n, row, blockIdx.y, tile_tokens, st, codes);
}

// OCTET_V layout (bits = 1): channel j's 32-byte row of a 256-token layout
// tile is the 256-bit vector of its codes in token order (byte o = tokens
// 8 o .. 8 o + 7). The CTA takes its tile 256 tokens at a time and assembles
// each 4 KB layout tile in shared memory (rows padded to 9 words), then writes
// it out with coalesced 4-byte stores.
//  - binary16: a thread takes one octet x 8 channels at a time, like the
//    octet-K pack (each load instruction of a warp covers two token rows), and
//    drops its 8 channel bytes into the staged tile;
//  - binary32: warp w owns tokens 32 w .. 32 w + 31, i.e. word w of every
//    channel's row. Lane l reads channels 8 (l % 16) .. + 7 of tokens
//    16 (l / 16) .. + 15, sets one bit per token in a 16-bit word per channel,
//    and the two half-warps join their halves with one exchange.
template <typename T, typename Src>
__device__ __forceinline__ void k_pack_octet_v_tile(const Src& src, int n, int row, int tile, int tile_tokens,
    const RowStats& st, uint8_t* __restrict__ codes) {
  __shared__ uint32_t stage[kD * 9];  // [channel][word 0..7, padding]
  const int n_pad = (n + 255) / 256 * 256;
  const int v0 = tile * (tile_tokens / 256), v1 = min(n_pad / 256, v0 + tile_tokens / 256);
  uint8_t* cr = codes + (size_t)row * (n_pad / 256) * 4096;
  if constexpr (std::is_same<T, half>::value) {
    uint8_t* sb = reinterpret_cast<uint8_t*>(stage);
    const int cg = threadIdx.x % kTpr, r = threadIdx.x / kTpr;
    uint32_t th[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) th[p] = st.thr[8 * cg + 2 * p] | ((uint32_t)st.thr[8 * cg + 2 * p + 1] << 16);
    for (int vt = v0; vt < v1; ++vt) {
#pragma unroll
      for (int oo = 0; oo < 2; ++oo) {
        const int o = r + kRpi * oo, tok0 = vt * 256 + 8 * o;  // octet o of the layout tile
        uint32_t acc[4] = {0u, 0u, 0u, 0u};  // bit k / 16 + k: token tok0 + k of channel 8 cg + 2p / + 1
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          if (tok0 + k < n) {
            uint32_t w[4];
            src.load8h(tok0 + k, 8 * cg, w);
#pragma unroll
            for (int p = 0; p < 4; ++p) acc[p] |= ge_mask(w[p], th[p]) & (0x00010001u << k);
          }
        }
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          sb[(8 * cg + 2 * p) * 36 + o] = (uint8_t)acc[p];
          sb[(8 * cg + 2 * p + 1) * 36 + o] = (uint8_t)(acc[p] >> 16);
        }
      }
      __syncthreads();
      uint32_t* dst = reinterpret_cast<uint32_t*>(cr + (size_t)vt * 4096);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int w = (int)threadIdx.x + kThreads * k;  // word w: channel w / 8, word w % 8 of its row
        dst[w] = stage[(w >> 3) * 9 + (w & 7)];
      }
      __syncthreads();
    }
  } else {
    __shared__ float s_hi[kD], s_lo[kD];  // alpha + beta per channel as an exact pair
    if (threadIdx.x < kD) two_sum(st.alpha[threadIdx.x], st.beta[threadIdx.x], s_hi[threadIdx.x], s_lo[threadIdx.x]);
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, cg = lane & 15, hh = lane >> 4;
    float hi[8], lo[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      hi[e] = s_hi[8 * cg + e];
      lo[e] = s_lo[8 * cg + e];
    }
    for (int vt = v0; vt < v1; ++vt) {
      const int tok0 = vt * 256 + 32 * warp + 16 * hh;
      uint32_t acc[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};  // bit i: token tok0 + i
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        if (tok0 + i < n) {
          float v[8];
          src.load8(tok0 + i, 8 * cg, v);
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[e] |= code1(v[e], hi[e], lo[e]) << i;
        }
      }
      uint32_t word[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const uint32_t other = __shfl_xor_sync(0xffffffffu, acc[e], 16);
        word[e] = hh ? (other | (acc[e] << 16)) : (acc[e] | (other << 16));
      }
      // lane (cg, hh) stores channels 8 cg + 4 hh .. 8 cg + 4 hh + 3
#pragma unroll
      for (int j2 = 0; j2 < 4; ++j2) stage[(8 * cg + 4 * hh + j2) * 9 + warp] = hh ? word[4 + j2] : word[j2];
      __syncthreads();
      uint32_t* dst = reinterpret_cast<uint32_t*>(cr + (size_t)vt * 4096);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int w = (int)threadIdx.x + kThreads * k;  // word w: channel w / 8, word w % 8 of its row
        dst[w] = stage[(w >> 3) * 9 + (w & 7)];
      }
      __syncthreads();
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(kThreads) k_pack_octet_v(
    const T* __restrict__ x, int n, int S, int tile_tokens, const float* __restrict__ part,
    uint8_t* __restrict__ codes, T* __restrict__ alpha_out, T* __restrict__ scale_out) {
  __shared__ RowStats st;
  const int row = blockIdx.x;
  fold_stats<T>(part + (size_t)row * S * 2 * kD, S, 1, blockIdx.y == 0, row, st, alpha_out,
                scale_out);
  k_pack_octet_v_tile<T>(GlobalRows<T>{x + (size_t)row * n * kD}, n, row, blockIdx.y, tile_tokens, st, codes);
}

// OCTET_K layout with BITS in {2, 4, 8}: P = 8 / BITS tokens share a byte; a
// thread owns one byte group (P tokens) x 8 channels, i.e. 8 consecutive bytes.
template <typename T, int BITS, typename Src>
__device__ __forceinline__ void k_pack_octet_k_b_tile(const Src& src, int n, int row, int tile, int tile_tokens,
    const RowStats& st, uint8_t* __restrict__ codes) {
  constexpr int L = (1 << BITS) - 1, P = 8 / BITS;
  const int cb = threadIdx.x % kTpr, r = threadIdx.x / kTpr;
  float af[8], inv[8];
  double ad[8], bd[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    af[e] = st.alpha[cb * 8 + e];
    inv[e] = st.inv[cb * 8 + e];
    ad[e] = (double)af[e];
    bd[e] = (double)st.beta[cb * 8 + e];
  }
  const int groups = (n + P - 1) / P;
  const int m0 = tile * (tile_tokens / P), m1 = min(groups, m0 + tile_tokens / P);
  uint8_t* cr = codes + (size_t)row * groups * kD + cb * 8;
  for (int m = m0 + r; m < m1; m += kRpi) {
    uint64_t bytes = 0;
#pragma unroll
    for (int k = 0; k < P; ++k) {
      const int i = P * m + k;
      if (i < n) {
        float v[8];
        src.load8(i, cb * 8, v);
#pragma unroll
        for (int e = 0; e < 8; ++e)
          bytes |= (uint64_t)quant_code(v[e], af[e], inv[e], ad[e], bd[e], L) << (8 * e + BITS * k);
      }
    }
    *reinterpret_cast<uint64_t*>(cr + (size_t)m * kD) = bytes;
  }
}

template <typename T, int BITS>
__global__ void __launch_bounds__(kThreads) k_pack_octet_k_b(
    const T* __restrict__ x, int n, int S, int tile_tokens, const float* __restrict__ part,
    uint8_t* __restrict__ codes, T* __restrict__ alpha_out, T* __restrict__ scale_out) {
  __shared__ RowStats st;
  const int row = blockIdx.x;
  fold_stats<T>(part + (size_t)row * S * 2 * kD, S, (1 << BITS) - 1, blockIdx.y == 0, row, st, alpha_out,
                scale_out);
  k_pack_octet_k_b_tile<T, BITS>(GlobalRows<T>{x + (size_t)row * n * kD}, n, row, blockIdx.y, tile_tokens, st, codes);
}

// OCTET_V layout with BITS in {2, 4, 8}: tiles of 32 P tokens; byte column q of
// a tile holds tokens P q .. P q + P - 1. A warp owns one tile: lane q builds
// byte column q of every channel (consecutive lanes write consecutive bytes).
template <typename T, int BITS, typename Src>
__device__ __forceinline__ void k_pack_octet_v_b_tile(const Src& src, int n, int row, int tile, int tile_tokens,
    const RowStats& st, uint8_t* __restrict__ codes) {
  constexpr int L = (1 << BITS) - 1, P = 8 / BITS, kTile = 32 * P;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int tiles = (n + kTile - 1) / kTile;
  const int v0 = tile * (tile_tokens / kTile), v1 = min(tiles, v0 + tile_tokens / kTile);
  uint8_t* cr = codes + (size_t)row * tiles * 4096;
  for (int vt = v0 + warp; vt < v1; vt += kThreads / 32) {
#pragma unroll 1
    for (int cg = 0; cg < kD / 8; ++cg) {
      uint32_t bytes[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
      for (int k = 0; k < P; ++k) {
        const int i = vt * kTile + P * lane + k;
        if (i < n) {
          float v[8];
          src.load8(i, cg * 8, v);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int j = cg * 8 + e;
            bytes[e] |= (uint32_t)quant_code(v[e], st.alpha[j], st.inv[j], (double)st.alpha[j], (double)st.beta[j], L)
                        << (BITS * k);
          }
        }
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) cr[(size_t)vt * 4096 + (cg * 8 + e) * 32 + lane] = (uint8_t)bytes[e];
    }
  }
}

template <typename T, int BITS>
__global__ void __launch_bounds__(kThreads) k_pack_octet_v_b(
    const T* __restrict__ x, int n, int S, int tile_tokens, const float* __restrict__ part,
    uint8_t* __restrict__ codes, T* __restrict__ alpha_out, T* __restrict__ scale_out) {
  __shared__ RowStats st;
  const int row = blockIdx.x;
  fold_stats<T>(part + (size_t)row * S * 2 * kD, S, (1 << BITS) - 1, blockIdx.y == 0, row, st, alpha_out,
                scale_out);
  k_pack_octet_v_b_tile<T, BITS>(GlobalRows<T>{x + (size_t)row * n * kD}, n, row, blockIdx.y, tile_tokens, st, codes);
}

// Single-read fill: one thread-block cluster per row, one CTA per tile of
// tile_tokens tokens. Each CTA first asks L2 for its whole tile (bulk
// prefetches, no registers held), takes the min / max of the tile, pushes them to
// every CTA of the cluster (distributed shared memory), folds the row's
// statistics from what it received (the same fold as the two-launch path, so
// alpha, step and codes are identical) and packs its own tile. The pack re-reads
// the tile the CTA has just read: the launcher caps the CTAs resident per SM so
// that the tiles in flight stay well inside L2, and HBM sees the input once.
constexpr int kFillMaxCl = 16;

template <typename T, int BITS, int LAYOUT, typename Src>
__device__ __forceinline__ void pack_tile(const Src& src, int n, int row, int tile, int tile_tokens,
                                          const RowStats& st,
                                          uint8_t* __restrict__ codes) {
  if constexpr (LAYOUT == CQ_LAYOUT_CANONICAL) {
    k_pack_canonical_tile<T, BITS>(src, n, row, tile, tile_tokens, st, codes);
  } else if constexpr (LAYOUT == CQ_LAYOUT_OCTET_K) {
    if constexpr (BITS == 1)
      k_pack_octet_k_tile<T>(src, n, row, tile, tile_tokens, st, codes);
    else
      k_pack_octet_k_b_tile<T, BITS>(src, n, row, tile, tile_tokens, st, codes);
  } else {
    if constexpr (BITS == 1)
      k_pack_octet_v_tile<T>(src, n, row, tile, tile_tokens, st, codes);
    else
      k_pack_octet_v_b_tile<T, BITS>(src, n, row, tile, tile_tokens, st, codes);
  }
}

template <typename T, int BITS, int LAYOUT>
__global__ void __launch_bounds__(kThreads, 4) k_fill(const T* __restrict__ x, int n, int cl, int tile_tokens,
                                                      uint8_t* __restrict__ codes, T* __restrict__ alpha_out,
                                                      T* __restrict__ scale_out) {
  // dynamic: the per-row-group min / max of pass 1 (also what pads the CTA's
  // shared memory to the residency cap)
  extern __shared__ __align__(128) uint8_t fill_dyn[];
  __shared__ float recv[kFillMaxCl][2][kD];  // every CTA's (min, max) per channel
  __shared__ RowStats st;
  float(*smn)[kD] = reinterpret_cast<float(*)[kD]>(fill_dyn + ((128u - (tc::smem_u32(fill_dyn) & 127u)) & 127u));
  float(*smx)[kD] = smn + kRpi;
  const uint32_t rank = tc::cluster_rank();
  const int row = blockIdx.x / cl;
  tc::cluster_arrive_relaxed();  // matched by the wait before the first peer store
  const int i0 = (int)rank * tile_tokens, i1 = min(n, i0 + tile_tokens);
  const T* xrow = x + (size_t)row * n * kD;
  {
    // the whole tile is requested into L2 at once (16 KB per request), so HBM
    // sees every resident CTA's tile in flight; both passes below read from L2
    constexpr int kReq = 16 * 1024;
    const char* tile0 = reinterpret_cast<const char*>(xrow + (size_t)i0 * kD);
    const int bytes = (i1 - i0) * kD * (int)sizeof(T);
    if ((int)threadIdx.x * kReq < bytes)
      tc::prefetch_l2_bulk(tile0 + (size_t)threadIdx.x * kReq, (uint32_t)min(kReq, bytes - (int)threadIdx.x * kReq));
  }
  float a, b;
  tile_minmax<T>(xrow, i0, i1, a, b, smn, smx);
  tc::cluster_wait();  // every CTA of the cluster is running
  if (threadIdx.x < kD) {
    for (int r = 0; r < cl; ++r) {
      tc::st_peer_f32(&recv[rank][0][threadIdx.x], (uint32_t)r, a);
      tc::st_peer_f32(&recv[rank][1][threadIdx.x], (uint32_t)r, b);
    }
  }
  tc::cluster_sync();  // every partial has landed; no peer access after this point
  constexpr int L = (1 << BITS) - 1;
  fold_stats<T>(&recv[0][0][0], cl, L, rank == 0, row, st, alpha_out, scale_out);
  pack_tile<T, BITS, LAYOUT>(GlobalRows<T>{xrow}, n, row, (int)rank, tile_tokens, st, codes);
}

// Tile of the single-read fill for a row of n tokens (0: not supported, use
// the two-launch path): 512 tokens up to n = 8192, 1024 up to n = 16384.
int fill_tile_tokens(int n) {
  if (n <= 512 * kFillMaxCl) return 512;
  if (n <= 1024 * kFillMaxCl) return 1024;
  return 0;
}

template <typename T, int BITS, int LAYOUT>
cudaError_t launch_fill(const T* x, int rows, int n, uint8_t* codes, T* alpha, T* scale, cudaStream_t stream) {
  const int tile = fill_tile_tokens(n);
  const int cl = (n + tile - 1) / tile;
  // Dynamic shared memory: the pass-1 scratch, padded to cap residency at 4 CTAs
  // per SM: 4 x 148 tiles of 512 tokens x 256 B = 76 MB in flight, inside the
  // 126 MB L2, so each tile's second read hits L2 (at 1024-token tiles the cap
  // is the same). Static + dynamic = 46 KB: more than 228 KB / 5, and within
  // the 48 KB a launch may use without opting in.
  constexpr int kTotal = 46 * 1024;
  constexpr int kScratch = 2 * kRpi * kD * (int)sizeof(float) + 128;  // + alignment
  static int pads[kMaxDevices];  // per device, + 1 once set (benign race: every caller computes the same values)
  const int dev = current_device();
  if (dev < 0) return cudaErrorInvalidDevice;
  if (pads[dev] == 0) {
    cudaError_t e = cudaFuncSetAttribute(k_fill<T, BITS, LAYOUT>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    cudaFuncAttributes fa;
    if (e == cudaSuccess) e = cudaFuncGetAttributes(&fa, k_fill<T, BITS, LAYOUT>);
    if (e != cudaSuccess) return e;
    const int pad = (int)fa.sharedSizeBytes + kScratch < kTotal ? kTotal - (int)fa.sharedSizeBytes : kScratch;
    pads[dev] = 1 + pad;
  }
  const int pad = pads[dev] - 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(rows * cl), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = (size_t)pad;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)cl;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k_fill<T, BITS, LAYOUT>, x, n, cl, tile, codes, alpha, scale);
}

template <typename T, int LAYOUT>
cudaError_t launch_fill_bits(const T* x, int rows, int n, int bits, uint8_t* codes, T* alpha, T* scale,
                             cudaStream_t stream) {
  switch (bits) {
    case 1: return launch_fill<T, 1, LAYOUT>(x, rows, n, codes, alpha, scale, stream);
    case 2: return launch_fill<T, 2, LAYOUT>(x, rows, n, codes, alpha, scale, stream);
    case 4: return launch_fill<T, 4, LAYOUT>(x, rows, n, codes, alpha, scale, stream);
    default: return launch_fill<T, 8, LAYOUT>(x, rows, n, codes, alpha, scale, stream);
  }
}

}  // namespace

int quantize_splits(int rows, int n) {
  // Enough (row, split) blocks to fill the GPU a few times over, and at least
  // 512 tokens per split.
  int s = (1024 + rows - 1) / rows;
  const int cap = (n + 511) / 512;
  if (s > cap) s = cap;
  return s < 1 ? 1 : s;
}

bool quantize_uses_workspace(int rows, int n) {
  return !(fill_tile_tokens(n) > 0 &&
           (long long)rows * ((n + fill_tile_tokens(n) - 1) / fill_tile_tokens(n)) <= 0x7fffffffLL);
}

template <typename T>
static cudaError_t launch_quantize_t(const T* x, int rows, int n, int bits, cq_layout layout,
                                     uint8_t* codes, T* alpha, T* scale, float* part,
                                     cudaStream_t stream) {
  if (!quantize_uses_workspace(rows, n)) {
    cudaError_t e;
    if (layout == CQ_LAYOUT_CANONICAL)
      e = launch_fill_bits<T, CQ_LAYOUT_CANONICAL>(x, rows, n, bits, codes, alpha, scale, stream);
    else if (layout == CQ_LAYOUT_OCTET_K)
      e = launch_fill_bits<T, CQ_LAYOUT_OCTET_K>(x, rows, n, bits, codes, alpha, scale, stream);
    else
      e = launch_fill_bits<T, CQ_LAYOUT_OCTET_V>(x, rows, n, bits, codes, alpha, scale, stream);
    return e == cudaSuccess ? cudaGetLastError() : e;
  }
  const int S = quantize_splits(rows, n);
  k_stats<T><<<dim3(rows, S), kThreads, 0, stream>>>(x, n, S, part);
  const int tile = 1024;
  if (layout == CQ_LAYOUT_CANONICAL) {
    const dim3 grid(rows, (n + tile - 1) / tile);
    switch (bits) {
      case 1: k_pack_canonical<T, 1><<<grid, kThreads, 0, stream>>>(x, n, S, tile, part, codes, alpha, scale); break;
      case 2: k_pack_canonical<T, 2><<<grid, kThreads, 0, stream>>>(x, n, S, tile, part, codes, alpha, scale); break;
      case 4: k_pack_canonical<T, 4><<<grid, kThreads, 0, stream>>>(x, n, S, tile, part, codes, alpha, scale); break;
      default: k_pack_canonical<T, 8><<<grid, kThreads, 0, stream>>>(x, n, S, tile, part, codes, alpha, scale); break;
    }
  } else if (layout == CQ_LAYOUT_OCTET_K) {
    const int P = 8 / bits, n_pad = (n + P - 1) / P * P;
    const dim3 grid(rows, (n_pad + tile - 1) / tile);
    switch (bits) {
      case 1: k_pack_octet_k<T><<<grid, kThreads, 0, stream>>>(x, n, S, tile, part, codes, alpha, scale); break;
      case 2: k_pack_octet_k_b<T, 2><<<grid, kThreads, 0, stream>>>(x, n, S, tile, part, codes, alpha, scale); break;
      case 4: k_pack_octet_k_b<T, 4><<<grid, kThreads, 0, stream>>>(x, n, S, tile, part, codes, alpha, scale); break;
      default: k_pack_octet_k_b<T, 8><<<grid, kThreads, 0, stream>>>(x, n, S, tile, part, codes, alpha, scale); break;
    }
  } else {
    const int vtile = 32 * (8 / bits), n_pad = (n + vtile - 1) / vtile * vtile;
    const dim3 grid(rows, (n_pad + tile - 1) / tile);
    switch (bits) {
      case 1: k_pack_octet_v<T><<<grid, kThreads, 0, stream>>>(x, n, S, tile, part, codes, alpha, scale); break;
      case 2: k_pack_octet_v_b<T, 2><<<grid, kThreads, 0, stream>>>(x, n, S, tile, part, codes, alpha, scale); break;
      case 4: k_pack_octet_v_b<T, 4><<<grid, kThreads, 0, stream>>>(x, n, S, tile, part, codes, alpha, scale); break;
      default: k_pack_octet_v_b<T, 8><<<grid, kThreads, 0, stream>>>(x, n, S, tile, part, codes, alpha, scale); break;
    }
  }
  return cudaGetLastError();
}

cudaError_t launch_quantize(const void* x, cq_dtype dt, int rows, int n, int bits, cq_layout layout,
                            uint8_t* codes, void* alpha, void* scale, void* workspace,
                            cudaStream_t stream) {
  float* part = static_cast<float*>(workspace);
  if (dt == CQ_F16)
    return launch_quantize_t<half>(static_cast<const half*>(x), rows, n, bits, layout, codes,
                                   static_cast<half*>(alpha), static_cast<half*>(scale), part, stream);
  return launch_quantize_t<float>(static_cast<const float*>(x), rows, n, bits, layout, codes,
                                  static_cast<float*>(alpha), static_cast<float*>(scale), part, stream);
}

size_t quantize_workspace_bytes(int rows, int n) {
  return (size_t)rows * quantize_splits(rows, n) * 2 * kD * sizeof(float);
}

}  // namespace cq

// ---------------------------------------------------------------------------
// Fixed scratch for cq_quantize_kv_noalloc: the per-split channel min/max
// partials live in a file-scope device array instead of a caller workspace.
// Every GPU that loads the library holds it until the process exits. Host
// code must not hand the symbol itself to a kernel (it is a host-side stand-in
// for the device array), so its device address is looked up once per device
// (with that device current) and kept; cudaDeviceReset makes that address
// stale, so no call may follow a reset of a device this process used.
#include <mutex>

namespace cq {

namespace {
constexpr size_t kStaticScratchBytes = 4u << 20;  // 4 MiB = 4096 (row, split) partials
static __device__ __align__(256) unsigned char g_quantize_scratch[kStaticScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};
}  // namespace

size_t quantize_static_scratch_bytes() { return kStaticScratchBytes; }

cudaError_t quantize_static_scratch(void** ptr) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_quantize_scratch);  // with `dev` current
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *ptr = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace cq
