// Generic decode attention over canonical-layout codes (any bits, any GQA
// group size up to 32), CUDA cores, three launches:
//
//   k_scores     x_i = sigma*(q.alpha_K) + (sigma*q (.) s_K) . c^K_i per token
//                (post-scaled logits, CalibQuant article Method 2) + per-chunk
//                min/max of every (batch, query-head) row
//   k_softmax_v  row range -> calibration slope (Method 3) -> softmax weights
//                -> per-chunk sum_i p_i c^V_i and sum_i p_i
//   k_merge      o = alpha_V + s_V (.) acc / l
//
// Calibration needs the range of the whole row before any weight is known,
// hence the split. The logits go through the workspace (L2-resident for
// moderate sizes). The tensor-core path for the 1-bit octet layouts lives in
// decode_octet.cu.
#include <float.h>

#include "common.cuh"
#include "kernels.h"

namespace cq {

namespace {

constexpr int kThreads = 256;
constexpr int kChunk = 256;   // tokens per block
constexpr int kMaxG = 32;     // query heads per kv-head supported here

struct Ws {
  float* scores;  // [B*Hq][n]
  float* mm;      // [B*Hq][C][2]
  float* acc;     // [B*Hq][C][kD]
  float* l;       // [B*Hq][C]
};

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

__host__ __device__ inline Ws carve(void* base, int B, int Hq, int n) {
  const int C = (n + kChunk - 1) / kChunk;
  const size_t rows = (size_t)B * Hq;
  char* p = static_cast<char*>(base);
  Ws w;
  w.scores = reinterpret_cast<float*>(p);
  p += align256(rows * n * sizeof(float));
  w.mm = reinterpret_cast<float*>(p);
  p += align256(rows * C * 2 * sizeof(float));
  w.acc = reinterpret_cast<float*>(p);
  p += align256(rows * C * kD * sizeof(float));
  w.l = reinterpret_cast<float*>(p);
  return w;
}

template <int BITS>
__device__ __forceinline__ float code_of(const uint32_t* words, int j) {
  constexpr uint32_t L = (1u << BITS) - 1;
  return (float)((words[(j * BITS) >> 5] >> ((j * BITS) & 31)) & L);
}

template <typename T, int BITS>
__global__ void __launch_bounds__(kThreads) k_scores(DecodeArgs a, Ws ws) {
  constexpr int NW = kD * BITS / 32;  // 32-bit words per token
  const int G = a.Hq / a.Hkv;
  const int bg = blockIdx.x, b = bg / a.Hkv, g = bg % a.Hkv;
  const int C = gridDim.y;
  __shared__ float sW[kMaxG][kD];
  __shared__ float sc0[kMaxG];
  __shared__ float smn[kThreads / 32][kMaxG], smx[kThreads / 32][kMaxG];
  const T* q = static_cast<const T*>(a.q) + ((size_t)b * a.Hq + (size_t)g * G) * kD;
  const T* al = static_cast<const T*>(a.k_alpha) + (size_t)bg * kD;
  const T* sc = static_cast<const T*>(a.k_scale) + (size_t)bg * kD;
  for (int e = threadIdx.x; e < G * kD; e += kThreads) {
    const int h = e / kD, j = e % kD;
    sW[h][j] = a.sigma * DT<T>::f(q[(size_t)h * kD + j]) * DT<T>::f(sc[j]);
  }
  const int lane = threadIdx.x & 31, warp = __shfl_sync(0xffffffffu, (int)threadIdx.x >> 5, 0);  // warp-uniform
  // passes over the heads with a trip count from G only: shuffles under a loop
  // on the warp index cost several times their latency
  for (int h0 = 0; h0 < G; h0 += kThreads / 32) {
    const int h = h0 + warp;
    float s = 0.f;
    if (h < G)
      for (int j = lane; j < kD; j += 32) s += DT<T>::f(q[(size_t)h * kD + j]) * DT<T>::f(al[j]);
#pragma unroll
    for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0 && h < G) sc0[h] = a.sigma * s;
  }
  __syncthreads();

  const int i = blockIdx.y * kChunk + threadIdx.x;
  const bool live = i < a.n;
  uint32_t words[NW];
  if (live) {
    const uint4* src = reinterpret_cast<const uint4*>(a.k_codes + ((size_t)bg * a.n + i) * (NW * 4));
#pragma unroll
    for (int w = 0; w < NW / 4; ++w) {
      const uint4 u = __ldg(src + w);
      words[4 * w] = u.x; words[4 * w + 1] = u.y; words[4 * w + 2] = u.z; words[4 * w + 3] = u.w;
    }
  } else {
#pragma unroll
    for (int w = 0; w < NW; ++w) words[w] = 0;
  }
  float* srow = ws.scores + ((size_t)b * a.Hq + (size_t)g * G) * a.n;
  for (int h0 = 0; h0 < G; h0 += 4) {
    float x[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) x[u] = (h0 + u < G) ? sc0[h0 + u] : 0.f;
#pragma unroll 4
    for (int j = 0; j < kD; ++j) {
      const float c = code_of<BITS>(words, j);
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (h0 + u < G) x[u] = fmaf(sW[h0 + u][j], c, x[u]);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int h = h0 + u;
      if (h >= G) break;
      if (live) srow[(size_t)h * a.n + i] = x[u];
      float mn = live ? x[u] : FLT_MAX, mx = live ? x[u] : -FLT_MAX;
#pragma unroll
      for (int o = 16; o; o >>= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      }
      if (lane == 0) {
        smn[warp][h] = mn;
        smx[warp][h] = mx;
      }
    }
  }
  __syncthreads();
  for (int h = threadIdx.x; h < G; h += kThreads) {
    float mn = FLT_MAX, mx = -FLT_MAX;
    for (int w = 0; w < kThreads / 32; ++w) {
      mn = fminf(mn, smn[w][h]);
      mx = fmaxf(mx, smx[w][h]);
    }
    float* o = ws.mm + (((size_t)b * a.Hq + (size_t)g * G + h) * C + blockIdx.y) * 2;
    o[0] = mn;
    o[1] = mx;
  }
}

template <typename T, int BITS>
__global__ void __launch_bounds__(kThreads) k_softmax_v(DecodeArgs a, Ws ws) {
  constexpr int NW = kD * BITS / 32;
  const int G = a.Hq / a.Hkv;
  const int bg = blockIdx.x, b = bg / a.Hkv, g = bg % a.Hkv;
  const int C = gridDim.y;
  __shared__ float sA[kMaxG], sRef[kMaxG];
  __shared__ float sP[kMaxG][kChunk];
  __shared__ float sAcc[2][kD];
  const size_t row0 = (size_t)b * a.Hq + (size_t)g * G;
  // row range -> slope of the calibration map and the largest calibrated logit
  for (int h = threadIdx.x; h < G; h += kThreads) {
    float m = FLT_MAX, M = -FLT_MAX;
    const float* mm = ws.mm + (row0 + h) * C * 2;
    for (int c = 0; c < C; ++c) {
      m = fminf(m, mm[2 * c]);
      M = fmaxf(M, mm[2 * c + 1]);
    }
    float slope = 1.f;
    if (a.calib && M > m) slope = (a.tau_hi * M - a.tau_lo * m) / (M - m);
    sA[h] = slope;
    sRef[h] = fmaxf(slope * m, slope * M);
  }
  __syncthreads();
  const int i0 = blockIdx.y * kChunk;
  for (int e = threadIdx.x; e < G * kChunk; e += kThreads) {
    const int h = e / kChunk, u = e % kChunk, i = i0 + u;
    float p = 0.f;
    if (i < a.n) p = __expf(sA[h] * ws.scores[(row0 + h) * a.n + i] - sRef[h]);
    sP[h][u] = p;
  }
  __syncthreads();
  // sum of weights of this chunk
  const int lane = threadIdx.x & 31, warp = __shfl_sync(0xffffffffu, (int)threadIdx.x >> 5, 0);  // warp-uniform
  for (int h0 = 0; h0 < G; h0 += kThreads / 32) {  // trip count from G only (see above)
    const int h = h0 + warp;
    float s = 0.f;
    if (h < G)
      for (int u = lane; u < kChunk; u += 32) s += sP[h][u];
#pragma unroll
    for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0 && h < G) ws.l[(row0 + h) * C + blockIdx.y] = s;
  }
  // sum_i p_i c_ij: thread = (channel j, half of the chunk)
  const int j = threadIdx.x & (kD - 1), half = threadIdx.x >> 7;
  const int u0 = half * (kChunk / 2), u1 = min(u0 + kChunk / 2, a.n - i0);
  const uint32_t* vrow = reinterpret_cast<const uint32_t*>(a.v_codes) + (size_t)bg * a.n * NW;
  const int wj = (j * BITS) >> 5, sj = (j * BITS) & 31;
  constexpr uint32_t L = (1u << BITS) - 1;
  for (int h0 = 0; h0 < G; h0 += 4) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int u = u0; u < u1; ++u) {
      const float c = (float)((__ldg(vrow + (size_t)(i0 + u) * NW + wj) >> sj) & L);
#pragma unroll
      for (int v = 0; v < 4; ++v)
        if (h0 + v < G) acc[v] = fmaf(sP[h0 + v][u], c, acc[v]);
    }
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int h = h0 + v;
      if (h >= G) break;
      sAcc[half][j] = acc[v];
      __syncthreads();
      if (half == 0) ws.acc[((row0 + h) * C + blockIdx.y) * kD + j] = sAcc[0][j] + sAcc[1][j];
      __syncthreads();
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(kD) k_merge(DecodeArgs a, Ws ws, int C) {
  const size_t row = blockIdx.x;  // b*Hq + h
  const int b = (int)(row / a.Hq), h = (int)(row % a.Hq);
  const int G = a.Hq / a.Hkv, g = h / G;
  const int j = threadIdx.x;
  float l = 0.f, acc = 0.f;
  for (int c = 0; c < C; ++c) {
    l += ws.l[row * C + c];
    acc += ws.acc[(row * C + c) * kD + j];
  }
  const size_t kv = ((size_t)b * a.Hkv + g) * kD + j;
  const float alpha = DT<T>::f(static_cast<const T*>(a.v_alpha)[kv]);
  const float step = DT<T>::f(static_cast<const T*>(a.v_scale)[kv]);
  static_cast<T*>(a.out)[row * kD + j] = DT<T>::from_float(alpha + step * (acc / l));
}

template <typename T, int BITS>
cudaError_t run(const DecodeArgs& a, void* workspace, cudaStream_t stream) {
  const int C = (a.n + kChunk - 1) / kChunk;
  Ws ws = carve(workspace, a.B, a.Hq, a.n);
  const dim3 grid(a.B * a.Hkv, C);
  k_scores<T, BITS><<<grid, kThreads, 0, stream>>>(a, ws);
  k_softmax_v<T, BITS><<<grid, kThreads, 0, stream>>>(a, ws);
  k_merge<T><<<a.B * a.Hq, kD, 0, stream>>>(a, ws, C);
  return cudaGetLastError();
}

template <typename T>
cudaError_t run_t(const DecodeArgs& a, void* workspace, cudaStream_t stream) {
  switch (a.bits) {
    case 1: return run<T, 1>(a, workspace, stream);
    case 2: return run<T, 2>(a, workspace, stream);
    case 4: return run<T, 4>(a, workspace, stream);
    default: return run<T, 8>(a, workspace, stream);
  }
}

}  // namespace

size_t decode_generic_workspace_bytes(int B, int Hq, int n) {
  const int C = (n + kChunk - 1) / kChunk;
  const size_t rows = (size_t)B * Hq;
  return align256(rows * n * sizeof(float)) + align256(rows * C * 2 * sizeof(float)) +
         align256(rows * C * kD * sizeof(float)) + align256(rows * C * sizeof(float));
}

cudaError_t launch_decode_generic(const DecodeArgs& a, cq_dtype dt, void* workspace,
                                  cudaStream_t stream) {
  if (dt == CQ_F16) return run_t<half>(a, workspace, stream);
  return run_t<float>(a, workspace, stream);
}

}  // namespace cq
