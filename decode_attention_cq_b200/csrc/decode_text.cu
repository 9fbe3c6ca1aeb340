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
#include "mma_util.cuh"
#include "tc.cuh"
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
// row's text tokens (txt::warp_text_attend: f32 tokens, or none), then the
// warps' parts and the visual part are merged by their log-sum-exps.
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

// ---- f16 text tokens on the tensor cores (txt::text_mma) ----------------
// The row's keys and values stream through a ring of four 16 KB slots: chunk
// gi holds the keys (gi even) or the values (gi odd) of tokens 64 (gi / 2) ..,
// as two tensor copies of 64 channels with the 128-byte swizzle (tokens past
// the row's end arrive as zeros). Each slot completes on its own mbarrier; the
// four warps reading a chunk release it through a shared counter, and the one
// that completes the count issues the chunk that reuses the slot.
constexpr int kSlots = 4;
// Parity waits: a warp may wait on a slot's next use only once its previous
// use has landed. The two warp groups take alternate chunk pairs (keys, values)
// from chunk 0, so with a multiple of 4 slots each group reuses only its own
// two slots.
static_assert(kSlots % 4 == 0, "warp groups must own their ring slots");

struct TextRing {
  uint64_t full[kSlots];
  uint32_t released[kSlots];  // warp releases of each slot so far (8 shares per use)
  uint32_t uses[kSlots];      // copies issued into each slot so far
  int err;                    // a bounded wait ran out
};

struct MergeChunks {
  TextRing& R;
  uint8_t* ring;
  uint32_t ring_u;
  const CUtensorMap* kmap;
  const CUtensorMap* vmap;
  int row, nall;
  __device__ __forceinline__ void issue(int gi) {
    const int s = gi % kSlots;
    atomicAdd(&R.uses[s], 1u);
    tc::mbar_arrive_expect_tx(&R.full[s], txt::kChunkBytes);
    uint8_t* dst = ring + (size_t)s * txt::kChunkBytes;
    const CUtensorMap* m = (gi & 1) ? vmap : kmap;
    tc::tma_load_3d(dst, m, 0, (gi >> 1) * txt::kChunkTokens, row, &R.full[s]);
    tc::tma_load_3d(dst + txt::kChunkBytes / 2, m, 128, (gi >> 1) * txt::kChunkTokens, row, &R.full[s]);
  }
  __device__ __forceinline__ uint32_t wait(int gi) {
    mu::warp_wait_copies(&R.full[gi % kSlots], (uint32_t)(gi / kSlots) & 1u, &R.err);
    return ring_u + (uint32_t)((gi % kSlots) * txt::kChunkBytes);
  }
  __device__ __forceinline__ void release(int gi) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) {
      const int s = gi % kSlots;
      __threadfence_block();  // this warp's reads of the slot come before the release
      const uint32_t done = atomicAdd(&R.released[s], 2u) + 2u;
      if (done == 8u * (uint32_t)(gi / kSlots + 1) && gi + kSlots < nall) {
        __threadfence_block();
        tc::fence_proxy_async();
        issue(gi + kSlots);
      }
    }
  }
};

// grid: one CTA per (batch, kv-head) row, 256 threads, dynamic shared memory =
// the ring (+ alignment): every warp attends its share of the row's text
// tokens on the tensor cores, then the warps' parts and the visual part are
// merged by their log-sum-exps.
__global__ void __launch_bounds__(kThreads) k_text_merge_mma(const half* __restrict__ q, int n_text,
                                                             const float* __restrict__ part_o,
                                                             const float* __restrict__ part_lse,
                                                             half* __restrict__ out, int Hq, int Hkv, float sigma,
                                                             const __grid_constant__ CUtensorMap kmap,
                                                             const __grid_constant__ CUtensorMap vmap) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* ring = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
  __shared__ TextRing R;
  __shared__ __align__(16) half s_q[kG * kD];
  __shared__ float s_m[kWarps][kG], s_l[kWarps][kG];
  const int row = blockIdx.x, b = row / Hkv, hkv = row % Hkv;
  const int t = threadIdx.x, warp = __shfl_sync(0xffffffffu, t >> 5, 0), lane = t & 31;
  const int g = lane >> 2, tq = lane & 3;
  const size_t bh0 = (size_t)b * Hq + (size_t)kG * hkv;  // first query head of the row
  const int ntp = (n_text + txt::kChunkTokens - 1) / txt::kChunkTokens;
  MergeChunks chunks{R, ring, tc::smem_u32(ring), &kmap, &vmap, row, 2 * ntp};
  if (t == 0) {
    R.err = 0;
    for (int s = 0; s < kSlots; ++s) {
      tc::mbar_init(&R.full[s], 1);
      R.released[s] = 0;
      R.uses[s] = 0;
    }
    tc::fence_mbar_init();
    for (int gi = 0; gi < kSlots && gi < 2 * ntp; ++gi) chunks.issue(gi);
  }
  if (t < kG * kD / 8)  // the four query rows, 16 bytes per thread
    reinterpret_cast<uint4*>(s_q)[t] = reinterpret_cast<const uint4*>(q + bh0 * kD)[t];
  __syncthreads();

  float m, l, o[8][4];
  txt::text_mma(chunks, 0, s_q, ntp, n_text, sigma, warp, lane, m, l, o);
  l += __shfl_xor_sync(0xffffffffu, l, 1);
  l += __shfl_xor_sync(0xffffffffu, l, 2);
  __syncthreads();  // every chunk is read: the ring becomes the parts' scratch
  float* s_acc = reinterpret_cast<float*>(ring);  // [warp][head][channel]
  if (g < kG && tq == 0) {
    s_m[warp][g] = m;
    s_l[warp][g] = l;
  }
  if (tq < 2) {
    float* h0 = s_acc + (warp * kG + 2 * tq) * kD;  // head 2 tq; head 2 tq + 1 follows
#pragma unroll
    for (int xx = 0; xx < 8; ++xx) {
      h0[16 * xx + g] = o[xx][0];
      h0[kD + 16 * xx + g] = o[xx][1];
      h0[16 * xx + g + 8] = o[xx][2];
      h0[kD + 16 * xx + g + 8] = o[xx][3];
    }
  }
  __syncthreads();
  const bool bad = R.err != 0;
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
        num = fmaf(f, s_acc[(w * kG + h) * kD + ch], num);
        den = fmaf(f, s_l[w][h], den);
      }
    }
    out[bh * kD + ch] = __float2half_rn(bad ? __int_as_float(0x7fc00000) : num / den);
  }
  // on the error path, copies still in flight land before the CTA exits
  if (t == 0 && bad) {
    for (int s = 0; s < kSlots; ++s)
      if (R.uses[s] > 0) tc::mbar_wait(&R.full[s], (R.uses[s] - 1) & 1u, mu::kSpin);
  }
}

}  // namespace

size_t text_merge_workspace_bytes(int B, int Hq) {
  return (size_t)B * Hq * kD * sizeof(float) + (size_t)B * Hq * sizeof(float);
}

cudaError_t launch_text_merge(const DecodeArgs& a, cq_dtype dt, const void* k_text, const void* v_text, int n_text,
                              cudaStream_t stream) {
  const int rows = a.B * a.Hkv;
  if (dt == CQ_F16 && n_text > 0) {
    constexpr size_t kSmem = (size_t)kSlots * txt::kChunkBytes + 1024;  // ring + alignment
    static bool attr_sets[kMaxDevices];  // per device (benign race: every caller sets the same value)
    const int attr_dev = current_device();
    if (attr_dev < 0) return cudaErrorInvalidDevice;
    bool& attr_set = attr_sets[attr_dev];
    if (!attr_set) {
      const cudaError_t e =
          cudaFuncSetAttribute(k_text_merge_mma, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem);
      if (e != cudaSuccess) return e;
      attr_set = true;
    }
    CUtensorMap kmap, vmap;
    if (!mu::encode_3d_box(&kmap, k_text, kD * sizeof(half), (uint64_t)n_text, (uint64_t)rows, 128,
                           txt::kChunkTokens, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !mu::encode_3d_box(&vmap, v_text, kD * sizeof(half), (uint64_t)n_text, (uint64_t)rows, 128,
                           txt::kChunkTokens, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
    k_text_merge_mma<<<rows, kThreads, kSmem, stream>>>(static_cast<const half*>(a.q), n_text, a.part_o,
                                                        a.part_lse, static_cast<half*>(a.out), a.Hq, a.Hkv,
                                                        a.sigma, kmap, vmap);
  } else if (dt == CQ_F16)
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
