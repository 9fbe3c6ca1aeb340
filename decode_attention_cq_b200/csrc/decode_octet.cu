// Fused 1-bit decode attention on the 5th-generation tensor cores (tcgen05,
// sm_100a) over the octet code layouts. One thread-block cluster per
// (batch, kv-head) row; each CTA of the cluster owns a contiguous slice of
// tokens and keeps that slice's logits in shared memory.
//
// Method (CalibQuant article): logits x_i = sigma q.alpha_K + (sigma q (.) s_K)
// . c^K_i on the integer codes (Method 2, post-scaling), calibration map g on
// the row's score range (Method 3), softmax, and o = alpha_V + s_V (.)
// sum_i p_i c^V_i / sum_i p_i (Method 2 applied to V).
//
// How the contractions reach the tensor core:
//  * K side (per 1024-token tile, M = 128 token octets): tensor-memory lane m
//    holds octet m's 128 bytes; masking bit k of every byte gives the int8
//    operand "code of token 8m+k times 2^k" for all 128 channels. B is the
//    per-row weight vector w_h = sigma q_h (.) s_K in 22-bit fixed point,
//    split into three int8 limbs per head (N = 16: 4 heads x 4 limb slots).
//    D (int32, TMEM) = 2^k * sum_j c_j * limb_j; the epilogue recombines limbs.
//  * V side (per 256-token tile, M = 128 channels): lane j holds channel j's
//    32 bytes; bit k gives "code of token 8q+k times 2^k" for the 32 octets q.
//    B holds p_i * 2^(31-k) as four uint8 limbs per head (N = 16), so every
//    bit position accumulates into the same int32 D = sum_i c_ij p_i 2^31.
//  * The softmax needs the row's full score range before any weight exists,
//    so the cluster exchanges (min, max) through distributed shared memory,
//    then sums the partial V accumulators the same way.
// No workspace, one launch per decode step.
#include <float.h>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace cq {

namespace {

constexpr int kThreads = 128;
constexpr int kG = 4;             // query heads per kv-head
constexpr int kKTile = 1024;      // tokens per K-side tile (128 octets)
constexpr int kVTile = 256;       // tokens per V-side tile (32 octets)
constexpr int kPrefSlice = 2048;  // preferred tokens per CTA (logits kept in shared memory)
constexpr int kMaxSlice = 8192;   // largest slice: n <= 65536 with 8-CTA clusters
constexpr int kCtasPerSm = 4;     // 4 x 128 TMEM columns, <= 128 registers per thread
constexpr uint32_t kTmemCols = 128;
constexpr uint32_t kColA = 0;     // K: 2 buffers x 4 chunks x 8 cols; V: 8 bits x 8 cols
constexpr uint32_t kColDK = 64;   // K accumulators: 2 buffers x 16 cols
constexpr uint32_t kColDV = 96;   // V accumulator: 16 cols
constexpr uint32_t kSpin = 1u << 22;
constexpr size_t kMinSmem = 48 * 1024;  // keeps at most four CTAs (4 x 128 TMEM columns) per SM
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kWMax = (1 << 21) - 1;  // 22-bit signed fixed point for the K-side weights
constexpr int kVPrefetch = 3;     // V tiles in flight per thread

struct Smem {
  uint8_t bk[4][512];        // K-side B: 32 channels x 16 (head, limb) bytes per chunk, MN-major
  uint8_t bv[2][8][512];     // V-side B: 32 octets x 16 (head, limb) bytes per bit, double-buffered
  float part_acc[kG][kD];    // this CTA's sum_i p_i c_ij (limbs recombined)
  float part_l[kG];          // this CTA's sum_i p_i
  float mM[kG][2];           // this CTA's logit range per head
  float red[4][kG][2];       // per-warp reduction scratch
  float c0[kG];              // sigma q.alpha_K
  float kscale[kG];          // fixed-point step of w_h
  float alog2[kG];           // calibration slope * log2(e)
  float ref[kG];             // largest calibrated logit * log2(e)
  uint64_t mbar_k[2];
  uint64_t mbar_v[2];
  uint32_t tmem_base;
  int err;
};

__host__ __device__ constexpr size_t align1k(size_t x) { return (x + 1023) & ~(size_t)1023; }

__device__ __forceinline__ uint4 ldg_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// 2^x with the hardware approximation (relative error about 2^-22).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float warp_min(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// 32 bytes of one V-side lane (channel t of a 256-token tile).
struct VWords {
  uint4 lo, hi;
};

template <typename T>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    k_decode_octet(DecodeArgs a, int cl, int slice_tokens) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  Smem& S = *reinterpret_cast<Smem*>(smem_raw);
  float* scores = reinterpret_cast<float*>(smem_raw + align1k(sizeof(Smem)));  // [kG][slice_tokens]

  // warp index broadcast from lane 0: known warp-uniform, so shuffles under branches and
  // loops on it need no reconvergence
  const int t = threadIdx.x, warp = __shfl_sync(0xffffffffu, t >> 5, 0), lane = t & 31;
  const uint32_t rank = tc::cluster_rank();
  const int row = blockIdx.x / cl;  // b * Hkv + g
  const int b = row / a.Hkv, g = row % a.Hkv;
  const int n = a.n;
  const int octets = (n + 7) >> 3;
  const int nk = (n + kKTile - 1) / kKTile;
  const int kt0 = (int)((rank * nk) / cl), kt1 = (int)(((rank + 1) * nk) / cl);
  const int t0 = kt0 * kKTile, t1 = min(n, kt1 * kKTile);
  const int vt0 = t0 / kVTile, vt1 = (t1 + kVTile - 1) / kVTile;
  const uint8_t* kc = a.k_codes + (size_t)row * octets * kD;
  const uint8_t* vc = a.v_codes + (size_t)row * ((n + kVTile - 1) / kVTile) * 4096;

  // The first K tile's codes are requested before anything else so that their
  // latency overlaps the setup below.
  uint32_t w32[32];
  auto load_k_tile = [&](int kt) {
    const int oct = kt * (kKTile / 8) + t;
    if (oct < octets) {
      const uint4* src = reinterpret_cast<const uint4*>(kc + (size_t)oct * kD);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint4 u = ldg_stream(src + i);
        w32[4 * i] = u.x;
        w32[4 * i + 1] = u.y;
        w32[4 * i + 2] = u.z;
        w32[4 * i + 3] = u.w;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) w32[i] = 0;
    }
  };
  if (kt0 < kt1) load_k_tile(kt0);

  // ---------------------------------------------------------------- setup
  if (warp == 0) {
    tc::tmem_alloc(&S.tmem_base, kTmemCols);
    tc::tmem_relinquish();
  }
  if (t == 0) {
    tc::mbar_init(&S.mbar_k[0], 1);
    tc::mbar_init(&S.mbar_k[1], 1);
    tc::mbar_init(&S.mbar_v[0], 1);
    tc::mbar_init(&S.mbar_v[1], 1);
    tc::fence_mbar_init();
    S.err = 0;
  }
  // post-scaled weights w_h[j] = sigma q_h[j] s_K[j] and bias c0_h = sigma q_h . alpha_K
  const T* qp = static_cast<const T*>(a.q) + ((size_t)b * a.Hq + (size_t)kG * g) * kD;
  const float sk = DT<T>::f(static_cast<const T*>(a.k_scale)[(size_t)row * kD + t]);
  const float ak = DT<T>::f(static_cast<const T*>(a.k_alpha)[(size_t)row * kD + t]);
  float w[kG];
#pragma unroll
  for (int h = 0; h < kG; ++h) {
    const float qv = DT<T>::f(qp[h * kD + t]);
    w[h] = a.sigma * qv * sk;
    const float amax = warp_max(fabsf(w[h]));
    const float qa = warp_sum(qv * ak);
    if (lane == 0) {
      S.red[warp][h][0] = amax;
      S.red[warp][h][1] = qa;
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = S.tmem_base;
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
  if (t < kG) {
    float amax = 0.f, qa = 0.f;
    for (int q = 0; q < 4; ++q) {
      amax = fmaxf(amax, S.red[q][t][0]);
      qa += S.red[q][t][1];
    }
    S.c0[t] = a.sigma * qa;
    S.kscale[t] = amax > 0.f ? amax / (float)kWMax : 0.f;
  }
  __syncthreads();
  {
    uint32_t limbs[kG];
#pragma unroll
    for (int h = 0; h < kG; ++h) {
      const float inv = S.kscale[h] > 0.f ? 1.f / S.kscale[h] : 0.f;
      int wi = __float2int_rn(w[h] * inv);
      wi = max(-kWMax, min(kWMax, wi));
      limbs[h] = (uint32_t)(wi & 127) | ((uint32_t)((wi >> 7) & 127) << 8) |
                 ((uint32_t)((wi >> 14) & 255) << 16);
    }
    *reinterpret_cast<uint4*>(&S.bk[t >> 5][(t & 31) * 16]) = make_uint4(limbs[0], limbs[1], limbs[2], limbs[3]);
  }
  tc::fence_proxy_async();
  __syncthreads();

  // --------------------------------------------------------------- K side
  // One step per (tile, bit position k): store the masked codes of bit k into
  // A[s&1], issue its four chunk MMAs into D[s&1], then finish the previous
  // step (wait for its MMAs, read D, write logits) while these run.
  // Logits are kept as scores[h][k][octet] (octet relative to the slice).
  constexpr uint32_t kIdescK = tc::idesc_i8(true, 16);
  const int slice_oct = slice_tokens / 8;
  float kscale[kG], c0[kG];
#pragma unroll
  for (int h = 0; h < kG; ++h) {
    kscale[h] = S.kscale[h];
    c0[h] = S.c0[h];
  }
  float mn[kG], mx[kG];
#pragma unroll
  for (int h = 0; h < kG; ++h) {
    mn[h] = FLT_MAX;
    mx[h] = -FLT_MAX;
  }
  uint32_t ph_k0 = 0u, ph_k1 = 0u;
  auto wait_k = [&](int which) {
    uint32_t& ph = which ? ph_k1 : ph_k0;
    if (S.err == 0 && !tc::mbar_wait(&S.mbar_k[which], ph, kSpin)) S.err = 1;
    ph ^= 1u;
  };
  // logits of step `sp` (tile kt0 + sp/8, bit sp%8) from D[sp&1]
  auto finish_k = [&](int sp) {
    const int buf = sp & 1, k = sp & 7, kt = kt0 + (sp >> 3);
    wait_k(buf);
    tc::fence_after_sync();
    uint32_t dv[16];
    tc::ld_x16(tbase + lane_off + kColDK + buf * 16, dv);
    tc::wait_ld();
    const bool valid = kt * kKTile + 8 * t + k < n;
    const float pow2 = __int_as_float((127 - k) << 23);  // 2^-k
    const int o = (kt - kt0) * (kKTile / 8) + t;
#pragma unroll
    for (int h = 0; h < kG; ++h) {
      const float v = fmaf(16384.f, (float)(int)dv[4 * h + 2],
                           fmaf(128.f, (float)(int)dv[4 * h + 1], (float)(int)dv[4 * h]));
      const float x = fmaf(v, kscale[h] * pow2, c0[h]);
      if (valid) {
        mn[h] = fminf(mn[h], x);
        mx[h] = fmaxf(mx[h], x);
      }
      scores[((size_t)h * 8 + k) * slice_oct + o] = x;
    }
    tc::fence_before_sync();
  };
  const int steps = (kt1 - kt0) * 8;
  for (int sp = 0; sp < steps; ++sp) {
    const int buf = sp & 1, k = sp & 7;
    const uint32_t m = 0x01010101u << k;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = w32[8 * c + i] & m;
      tc::st_x8(tbase + lane_off + kColA + buf * 32 + c * 8, v);
    }
    // all bit positions of this tile are in flight: fetch the next tile
    if (k == 7 && kt0 + (sp >> 3) + 1 < kt1) load_k_tile(kt0 + (sp >> 3) + 1);
    tc::wait_st();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (t == 0 && S.err == 0) {
#pragma unroll
      for (int c = 0; c < 4; ++c)
        tc::mma_i8_ts(tbase + kColDK + buf * 16, tbase + kColA + buf * 32 + c * 8,
                      tc::smem_desc(S.bk[c], 128, 512), kIdescK, c > 0 ? 1u : 0u);
      tc::mma_commit(&S.mbar_k[buf]);
    }
    if (sp > 0) finish_k(sp - 1);
  }
  if (steps > 0) finish_k(steps - 1);

  // -------------------------------------------- score range of the whole row
#pragma unroll
  for (int h = 0; h < kG; ++h) {
    const float m = warp_min(mn[h]), M = warp_max(mx[h]);
    if (lane == 0) {
      S.red[warp][h][0] = m;
      S.red[warp][h][1] = M;
    }
  }
  // V codes of the first tiles are requested before the cluster exchange.
  VWords ring[kVPrefetch];
  auto load_v_tile = [&](int vt, VWords& dst) {
    if (vt < vt1) {
      const uint4* src = reinterpret_cast<const uint4*>(vc + (size_t)vt * 4096 + t * 32);
      dst.lo = ldg_stream(src);
      dst.hi = ldg_stream(src + 1);
    }
  };
#pragma unroll
  for (int p = 0; p < kVPrefetch; ++p) load_v_tile(vt0 + p, ring[p]);
  __syncthreads();
  if (t < kG) {
    float m = FLT_MAX, M = -FLT_MAX;
    for (int q = 0; q < 4; ++q) {
      m = fminf(m, S.red[q][t][0]);
      M = fmaxf(M, S.red[q][t][1]);
    }
    S.mM[t][0] = m;
    S.mM[t][1] = M;
  }
  tc::cluster_sync();
  if (t < kG) {
    float m = FLT_MAX, M = -FLT_MAX;
    for (int r = 0; r < cl; ++r) {
      m = fminf(m, tc::ld_peer_f32(&S.mM[t][0], r));
      M = fmaxf(M, tc::ld_peer_f32(&S.mM[t][1], r));
    }
    float slope = 1.f;
    if (a.calib && M > m) slope = (a.tau_hi * M - a.tau_lo * m) / (M - m);
    S.alog2[t] = slope * kLog2e;
    S.ref[t] = fmaxf(slope * m, slope * M) * kLog2e;
  }
  __syncthreads();

  // --------------------------------------------------------------- V side
  // Per tile: softmax weights -> B (double-buffered in shared memory) while
  // the previous tile's MMAs run; then wait for them, refill the single A
  // buffer in TMEM and issue this tile's eight MMAs.
  constexpr uint32_t kIdescV = tc::idesc_i8(false, 16);
  const int hp = t & 3, grp = t >> 2;
  const float alog2 = S.alog2[hp], ref = S.ref[hp];
  float lsum = 0.f;
  uint32_t ph_v0 = 0u, ph_v1 = 0u;  // parity of the next completion of mbar_v[0] / mbar_v[1]
  auto wait_v = [&](int which) {
    uint32_t& ph = which ? ph_v1 : ph_v0;
    if (S.err == 0 && !tc::mbar_wait(&S.mbar_v[which], ph, kSpin)) S.err = 1;
    ph ^= 1u;
  };
  for (int vt = vt0; vt < vt1; ++vt) {
    const int it = vt - vt0, buf = it & 1;
    // B: softmax weights of tokens 256 vt + 8 grp + k for head hp, scaled by 2^(31-k)
    // bv[buf] was last read by the MMAs of tile it-2, waited for in iteration it-1
    const int i0 = vt * kVTile + 8 * grp;
    const int o = (i0 - t0) >> 3;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      uint32_t pi = 0;
      if (i0 + k < n) {
        const float x = scores[((size_t)hp * 8 + k) * slice_oct + o];
        const float p = ex2_approx(fmaf(x, alog2, (float)(31 - k) - ref));  // p_i * 2^(31-k)
        pi = __float2uint_rn(p);
        lsum = fmaf(p, __int_as_float((127 - 31 + k) << 23), lsum);  // sum_i p_i
      }
      *reinterpret_cast<uint32_t*>(&S.bv[buf][k][grp * 16 + 4 * hp]) = pi;
    }
    tc::fence_proxy_async();
    if (it >= 1) {  // the single TMEM A buffer was read by the MMAs of tile it-1
      wait_v(buf ^ 1);
      tc::fence_after_sync();
    }
    // A: channel t's 32 octet bytes of this tile, one bit position per MMA
    const VWords cur = ring[0];
#pragma unroll
    for (int p = 0; p + 1 < kVPrefetch; ++p) ring[p] = ring[p + 1];
    load_v_tile(vt + kVPrefetch, ring[kVPrefetch - 1]);
    const uint32_t wv[8] = {cur.lo.x, cur.lo.y, cur.lo.z, cur.lo.w, cur.hi.x, cur.hi.y, cur.hi.z, cur.hi.w};
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const uint32_t m = 0x01010101u << k;
      uint32_t v8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) v8[i] = wv[i] & m;
      tc::st_x8(tbase + lane_off + kColA + k * 8, v8);
    }
    tc::wait_st();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (t == 0 && S.err == 0) {
#pragma unroll
      for (int k = 0; k < 8; ++k)
        tc::mma_i8_ts(tbase + kColDV, tbase + kColA + k * 8, tc::smem_desc(S.bv[buf][k], 128, 512),
                      kIdescV, (it == 0 && k == 0) ? 0u : 1u);
      tc::mma_commit(&S.mbar_v[buf]);
    }
  }
  if (vt1 > vt0) wait_v((vt1 - vt0 - 1) & 1);  // the last tile's commit is the only one not waited for
  tc::fence_after_sync();
  uint32_t dv[16];
  tc::ld_x16(tbase + lane_off + kColDV, dv);
  tc::wait_ld();
  const bool failed = S.err != 0;
#pragma unroll
  for (int h = 0; h < kG; ++h) {
    const float acc = (float)(int)dv[4 * h] * 0x1p-31f + (float)(int)dv[4 * h + 1] * 0x1p-23f +
                      (float)(int)dv[4 * h + 2] * 0x1p-15f + (float)(int)dv[4 * h + 3] * 0x1p-7f;
    S.part_acc[h][t] = acc;
  }
  // sum of weights per head: lanes with equal (lane & 3) share a head
  float ls = lsum;
  ls += __shfl_xor_sync(0xffffffffu, ls, 4);
  ls += __shfl_xor_sync(0xffffffffu, ls, 8);
  ls += __shfl_xor_sync(0xffffffffu, ls, 16);
  if (lane < kG) S.red[warp][lane][0] = ls;
  __syncthreads();
  if (t < kG) {
    float l = 0.f;
    for (int q = 0; q < 4; ++q) l += S.red[q][t][0];
    S.part_l[t] = failed ? __int_as_float(0x7fc00000) : l;
    if (failed && t == 0 && a.status != nullptr) atomicOr(a.status, CQ_DEVICE_WAIT_TIMEOUT);
  }
  tc::cluster_sync();

  // --------------------------------------- rank 0 merges the cluster and stores
  if (rank == 0) {
    const size_t kv = (size_t)row * kD + t;
    const float alpha = DT<T>::f(static_cast<const T*>(a.v_alpha)[kv]);
    const float step = DT<T>::f(static_cast<const T*>(a.v_scale)[kv]);
    T* out = static_cast<T*>(a.out) + ((size_t)b * a.Hq + (size_t)kG * g) * kD;
#pragma unroll
    for (int h = 0; h < kG; ++h) {
      float acc = 0.f, l = 0.f;
      for (int r = 0; r < cl; ++r) {
        acc += tc::ld_peer_f32(&S.part_acc[h][t], r);
        l += tc::ld_peer_f32(&S.part_l[h], r);
      }
      out[h * kD + t] = DT<T>::from_float(fmaf(step, acc / l, alpha));
    }
  }
  tc::cluster_sync();  // peers keep their shared memory until rank 0 has read it

  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tbase, kTmemCols);
}

// Cluster size: enough CTAs that each keeps at most kPrefSlice tokens (more
// only when n needs more than 8 CTAs of that size), then the
// power of two (<= 8, <= number of K tiles) whose wave count best fills the
// GPU at kCtasPerSm CTAs per SM.
int pick_cluster(int rows, int nk, int sms) {
  int cl = 1;
  while (cl < 8 && cl * kPrefSlice < nk * kKTile) cl *= 2;
  if (cl * kMaxSlice < nk * kKTile) return -1;
  int best = cl;
  double best_eff = -1.0;
  for (int c = cl; c <= 8 && c <= nk; c *= 2) {
    const double waves = (double)rows * c / ((double)sms * kCtasPerSm);
    const double eff = waves / ceil(waves);
    if (eff > best_eff + 0.02) {
      best_eff = eff;
      best = c;
    }
  }
  return best;
}

template <typename T>
cudaError_t run(const DecodeArgs& a, cudaStream_t stream) {
  static int sm_counts[kMaxDevices];  // per device; only sizes the cluster choice
  const int dev = current_device();
  if (dev < 0) return cudaErrorInvalidDevice;
  if (sm_counts[dev] == 0) {
    int c = 0;
    sm_counts[dev] = cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess ? c : 148;
  }
  const int sms = sm_counts[dev];
  const int rows = a.B * a.Hkv;
  const int nk = (a.n + kKTile - 1) / kKTile;
  const int cl = pick_cluster(rows, nk, sms);
  if (cl < 0) return cudaErrorNotSupported;
  const int slice_tokens = ((nk + cl - 1) / cl) * kKTile;
  size_t smem = align1k(sizeof(Smem)) + (size_t)kG * slice_tokens * sizeof(float);
  if (smem < kMinSmem) smem = kMinSmem;
  static bool attr_sets[kMaxDevices];  // per device (benign race: every caller sets the same value)
  const int attr_dev = current_device();
  if (attr_dev < 0) return cudaErrorInvalidDevice;
  bool& attr_set = attr_sets[attr_dev];
  if (!attr_set) {
    const size_t max_smem = align1k(sizeof(Smem)) + (size_t)kG * kMaxSlice * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(k_decode_octet<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)(max_smem > kMinSmem ? max_smem : kMinSmem));
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(rows * cl), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)cl;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k_decode_octet<T>, a, cl, slice_tokens);
}

}  // namespace

cudaError_t launch_decode_octet(const DecodeArgs& a, cq_dtype dt, cudaStream_t stream) {
  if (dt == CQ_F16) return run<half>(a, stream);
  return run<float>(a, stream);
}

}  // namespace cq
