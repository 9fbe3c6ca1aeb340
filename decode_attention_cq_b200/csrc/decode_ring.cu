// Fused decode attention for 2-, 4- and 8-bit codes in the octet layouts, on
// register-fed tensor-core MMAs (mma.sync m16n8k32, u8 x s8/u8 -> s32).
//
// Method (CalibQuant article): logits x_i = sigma q.alpha_K + (sigma q (.) s_K)
// . c^K_i on the integer codes (Method 2, post-scaling), calibration map g on
// the row's score range (Method 3), softmax, o = alpha_V + s_V (.)
// sum_i p_i c^V_i / sum_i p_i (Method 2 applied to V).
//
// With b-bit codes a byte holds P = 8 / b tokens; masking sub-position k of
// every byte ((2^b - 1) << k b) gives the 8-bit operand "code of token P m + k
// times 2^(k b)", so the 1-bit construction carries over with P sub-positions
// instead of 8 bit positions: K side A = masked code bytes of 16 byte rows x
// 32 channels, B = the weights w_h = sigma q_h (.) s_K in three int8 limbs;
// V side A = softmax weights p 2^(31 - k b) in four uint8 limbs, B = masked
// code bytes of 8 channels.
//
// One thread-block cluster per (batch, kv-head) row, one CTA per 2048-token
// slice, whatever b is. Only the slice's logits (later its weight fragments,
// 16 bytes per token) stay resident; the codes (32 b KB per slice for K and
// again for V) stream through a ring of four 16 KB tensor copies: K
// chunks first, then V chunks, so the first V chunks load while the cluster
// exchanges the logit range. A slot is refilled once all eight warps have
// released it (full / empty mbarriers, every wait bounded).
#include <float.h>

#include "common.cuh"
#include "kernels.h"
#include "mma_util.cuh"
#include "tc.cuh"

namespace cq {

namespace {

using namespace mu;

constexpr int kThreads = 256;  // 8 warps
constexpr int kWarps = kThreads / 32;
constexpr int kSlice = 2048;         // tokens per CTA
constexpr int kMaxCl = 16;           // 16-CTA clusters need the non-portable size
constexpr int kWMax = (1 << 21) - 1;
constexpr int kLimbRow = 132;        // bytes per limb row (spreads the B-fragment loads over banks)
constexpr int kRecv = kG * 140;      // >= kG * cl * ceil(kD / cl) for every cl <= 16 (560 at cl = 14)
constexpr int kPartStride = kD + 8;  // floats per (warp pair, head) row of the partial sums
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kChunkBytes = 16384;   // one ring slot: 8 K units or 4 V tiles
constexpr int kChunkRows = 128;      // 128-byte rows (K byte rows or V lines) per slot

template <typename T>
struct RingFixed {
  // raw rows (dtype T): q of the 4 heads, alpha_K, s_K, alpha_V, s_V
  alignas(16) uint8_t stage[8 * kD * sizeof(T)];
  uint64_t bar_rows, full[4], empty[4];
  int err;                          // a bounded wait ran out
  uint8_t limb[kG * 3][kLimbRow];   // K-side weight limbs: row 3 h + l, byte = channel
  float red[kWarps][kG][2];         // per-warp reduction scratch
  float mM[kMaxCl][kG][2];          // every peer's logit range per head (pushed to all)
  float part_l[kMaxCl][kG];         // every peer's sum of weights (pushed to all)
  float lsum[kWarps][kG];           // per-warp sum of weights
  float c0[kG], kscale[kG], alog2[kG], ref[kG];
  float cst[kG];                    // g(x) - slope x: the calibration's constant term
  float recv[kRecv];                // [src][h][channel - first owned channel]
};

// Ring slots (SLOTS): 4 with 2 CTAs per SM (more bytes in flight per CTA)
// while the launch fits in two waves of 2 CTAs per SM, 2 with 3 CTAs per SM
// (more CTAs resident) beyond that. Measured on B200 at n = 8192: batch 16
// takes 4 (2-bit 40.9 -> 37.9 us, 8-bit 78.6 -> 67.8 us); batch 64 takes 2
// (2-bit 117.2 -> 103.1 us, 4-bit 146.5 -> 129.2 us, 8-bit 211.1 -> 194.6 us);
// batch 32, 2-bit: 67.4 -> 62.9 us with 2.
inline int ring_slots_for(long long ctas, int sms) { return sms > 0 && ctas <= 4LL * sms ? 4 : 2; }

// logits / weight fragments (16 B per token) | ring (slots x 16 KB) | fixed part
template <typename T, int SLOTS>
constexpr size_t ring_smem_bytes() {
  return (size_t)kSlice * 16 + (size_t)SLOTS * kChunkBytes + sizeof(RingFixed<T>);
}

// kmap: K codes as [rows][byte rows][128 B]; vmap: V codes as [rows][tiles *
// 32][128 B] (a 128-byte line holds 4 channels' 32 bytes of a tile). Both use
// the 128-byte swizzle (chunk c of line l lands at chunk c ^ (l & 7)).
template <typename T, int BITS, int SLOTS>
__global__ void __launch_bounds__(kThreads, SLOTS == 2 ? 3 : 2)
    k_decode_ring(const __grid_constant__ DecodeArgs a, int cl, const __grid_constant__ CUtensorMap kmap,
                  const __grid_constant__ CUtensorMap vmap) {
  constexpr int P = 8 / BITS;         // tokens per code byte
  constexpr int kUnitTok = 16 * P;    // tokens per K unit (16 byte rows, 2 KB)
  constexpr int kTileTok = 32 * P;    // tokens per V tile (32 byte columns, 4 KB)
  constexpr int kUnitWords = 64 * P;  // logit words per unit (16 byte rows x P x 4 heads)
  constexpr uint32_t kSubMask = 0x01010101u * ((1u << BITS) - 1u);  // sub-position 0 of every byte
  constexpr int kSlots = SLOTS;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // the 128-byte swizzle of the copies repeats every 1024 bytes: align to it
  uint8_t* sL = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* ring = sL + (size_t)kSlice * 16;
  RingFixed<T>& F = *reinterpret_cast<RingFixed<T>*>(ring + kSlots * kChunkBytes);
  float* sLf = reinterpret_cast<float*>(sL);   // logits, unit u at words [kUnitWords u, ...)
  float* sPart = reinterpret_cast<float*>(ring);  // per warp-pair partial sums (after the V side)
  const uint32_t sL_u = tc::smem_u32(sL), ring_u = tc::smem_u32(ring);

  // warp index broadcast from lane 0: known warp-uniform, so shuffles under branches and
  // loops on it need no reconvergence
  const int t = threadIdx.x, warp = __shfl_sync(0xffffffffu, t >> 5, 0), lane = t & 31, g = lane >> 2, tq = lane & 3;
  const uint32_t rank = tc::cluster_rank();
  const int row = blockIdx.x / cl;
  const int b = row / a.Hkv, hkv = row % a.Hkv;
  const int n = a.n;
  const int nvt = (n + kTileTok - 1) / kTileTok;
  const int vt0 = (int)((rank * nvt) / cl), vt1 = (int)(((rank + 1) * nvt) / cl);
  const int t0 = vt0 * kTileTok, t1 = min(n, vt1 * kTileTok);
  const int nvtl = vt1 - vt0;                            // V tiles of this CTA
  const int nunits = (t1 - t0 + kUnitTok - 1) / kUnitTok;  // K units of this CTA
  const int nk = (nunits + kWarps - 1) / kWarps;         // K chunks (one unit per warp)
  const int nv = (nvtl + 3) / 4;                         // V chunks (one tile per warp pair)
  const int nchunks = nk + nv;
  volatile int* err = &F.err;

  // chunk gi of the ring sequence (K chunks, then V chunks) into slot gi % kSlots;
  // rows past the row's end arrive as zeros
  auto issue = [&](int gi) {
    const int slot = gi % kSlots;
    tc::mbar_arrive_expect_tx(&F.full[slot], kChunkBytes);
    if (gi < nk)
      tc::tma_load_3d(ring + slot * kChunkBytes, &kmap, 0, t0 / P + gi * kChunkRows, row, &F.full[slot]);
    else
      tc::tma_load_3d(ring + slot * kChunkBytes, &vmap, 0, vt0 * 32 + (gi - nk) * kChunkRows, row, &F.full[slot]);
  };
  // after every warp released the slot of chunk gi: refill it with chunk gi + kSlots
  auto refill = [&](int gi) {
    if (t == 0 && gi + kSlots < nchunks) {
      if (tc::mbar_wait(&F.empty[gi % kSlots], (uint32_t)(gi / kSlots) & 1u, kSpin)) {
        tc::fence_proxy_async();
        issue(gi + kSlots);
      } else {
        *err = 1;
      }
    }
  };

  // ---- 1. query and statistics rows (bulk copies), first two code chunks
  if (t == 0) {
    F.err = 0;
    tc::mbar_init(&F.bar_rows, 1);
    for (int i = 0; i < kSlots; ++i) {
      tc::mbar_init(&F.full[i], 1);
      tc::mbar_init(&F.empty[i], kWarps);
    }
    tc::fence_mbar_init();
    constexpr uint32_t kRow = kD * sizeof(T);
    const uint8_t* qrow = static_cast<const uint8_t*>(a.q) + ((size_t)b * a.Hq + (size_t)kG * hkv) * kRow;
    const size_t stat = (size_t)row * kRow;
    tc::mbar_arrive_expect_tx(&F.bar_rows, 8 * kRow);
    tc::bulk_load(F.stage, qrow, kG * kRow, &F.bar_rows);
    tc::bulk_load(F.stage + 4 * kRow, static_cast<const uint8_t*>(a.k_alpha) + stat, kRow, &F.bar_rows);
    tc::bulk_load(F.stage + 5 * kRow, static_cast<const uint8_t*>(a.k_scale) + stat, kRow, &F.bar_rows);
    tc::bulk_load(F.stage + 6 * kRow, static_cast<const uint8_t*>(a.v_alpha) + stat, kRow, &F.bar_rows);
    tc::bulk_load(F.stage + 7 * kRow, static_cast<const uint8_t*>(a.v_scale) + stat, kRow, &F.bar_rows);
    for (int gi = 0; gi < kSlots && gi < nchunks; ++gi) issue(gi);
  }
  tc::cluster_arrive_relaxed();  // matched by the wait before the first peer store
  __syncthreads();               // barrier initialisation is visible

  // ---- 2. post-scaled K weights w_h = sigma q_h (.) s_K in 22-bit fixed point
  const T* sRows = reinterpret_cast<const T*>(F.stage);  // q[4][kD], alpha_K, s_K, alpha_V, s_V
  wait_copies(&F.bar_rows, 0, err);
  float w[kG];
  // Every warp runs this (warps 4..7 repeat channels 0..127 and store nothing):
  // a shuffle the compiler cannot prove convergent, e.g. under a branch on the
  // thread index, costs several times its latency.
  {
    const int ch = t & (kD - 1);
    const float ak = DT<T>::f(sRows[4 * kD + ch]);
    const float sk = DT<T>::f(sRows[5 * kD + ch]);
    float amax[kG], qa[kG];
#pragma unroll
    for (int h = 0; h < kG; ++h) {
      const float qv = DT<T>::f(sRows[h * kD + ch]);
      w[h] = a.sigma * qv * sk;
      amax[h] = fabsf(w[h]);
      qa[h] = qv * ak;
    }
    // the four heads' reductions interleaved, with no branch between them
#pragma unroll
    for (int o = 16; o; o >>= 1)
#pragma unroll
      for (int h = 0; h < kG; ++h) {
        amax[h] = fmaxf(amax[h], __shfl_xor_sync(0xffffffffu, amax[h], o));
        qa[h] += __shfl_xor_sync(0xffffffffu, qa[h], o);
      }
    if (lane == 0 && warp < kD / 32) {
#pragma unroll
      for (int h = 0; h < kG; ++h) {
        F.red[warp][h][0] = amax[h];
        F.red[warp][h][1] = qa[h];
      }
    }
  }
  __syncthreads();
  if (warp < kD / 32) {  // t < kD
#pragma unroll
    for (int h = 0; h < kG; ++h) {
      const float amax = fmaxf(fmaxf(F.red[0][h][0], F.red[1][h][0]), fmaxf(F.red[2][h][0], F.red[3][h][0]));
      const float ks = amax * (1.f / (float)kWMax);              // any scale works: w is rounded with this one
      const float inv = ks > 0.f ? __fdividef(1.f, ks) : 0.f;  // approximate: the clamp below bounds w
      const int wi = max(-kWMax, min(kWMax, __float2int_rn(w[h] * inv)));
      F.limb[3 * h + 0][t] = (uint8_t)(wi & 127);
      F.limb[3 * h + 1][t] = (uint8_t)((wi >> 7) & 127);
      F.limb[3 * h + 2][t] = (uint8_t)((wi >> 14) & 255);
      if (t == h) {
        F.kscale[h] = ks;
        F.c0[h] = a.sigma * (F.red[0][h][1] + F.red[1][h][1] + F.red[2][h][1] + F.red[3][h][1]);
      }
    }
  }
  __syncthreads();
  // B fragments of the K side: bk[c][tile][half] holds channels 32c + 16 half + 4 tq + (0..3);
  // tile 0 column g = (head g/2, limb g%2), tile 1 column g = (head g/2, limb 2) for even g, 0 for odd g.
  uint32_t bk[4][2][2];
#pragma unroll
  for (int c = 0; c < 4; ++c)
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int j = 32 * c + 16 * half + 4 * tq;
      bk[c][0][half] = *reinterpret_cast<const uint32_t*>(&F.limb[3 * (g >> 1) + (g & 1)][j]);
      bk[c][1][half] = (g & 1) ? 0u : *reinterpret_cast<const uint32_t*>(&F.limb[3 * (g >> 1) + 2][j]);
    }
  const float c0 = F.c0[tq], kscale = F.kscale[tq];

  // ---- 3. K side: chunk gk holds units 8 gk .. 8 gk + 7, warp w takes unit 8 gk + w
  // (16 byte rows x 128 channels); the unit's logits go to its slot of the logit area
  constexpr int KK = P >= 2 ? 2 : 1;  // sub-positions per pass (independent accumulators)
  float mn = FLT_MAX, mx = -FLT_MAX;  // logit range of head tq over this lane's tokens
  for (int gk = 0; gk < nk; ++gk) {
    const int slot = gk % kSlots;
    wait_copies(&F.full[slot], (uint32_t)(gk / kSlots) & 1u, err);
    const int u = kWarps * gk + warp;
    if (u < nunits) {
      uint32_t af[4][4];  // A fragments of chunks c = 0..3 (rows = byte rows {g, g+8} of the unit)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int m = lane >> 3, r8 = 8 * (m & 1) + (lane & 7), c16 = 2 * c + (m >> 1);
        ldsm_x4(ring_u + slot * kChunkBytes + warp * 2048 + r8 * 128 + ((c16 ^ (lane & 7)) << 4), af[c]);
      }
      float* lg = sLf + u * kUnitWords;
      const int tok = t0 + kUnitTok * u + P * g;  // token of byte row g, sub-position 0
      const bool full = t0 + kUnitTok * (u + 1) <= t1;
#pragma unroll
      for (int k = 0; k < P; k += KK) {
        int d[KK][2][4];  // [sub-position k + kk][tile][reg]
#pragma unroll
        for (int kk = 0; kk < KK; ++kk)
#pragma unroll
          for (int tl = 0; tl < 2; ++tl) d[kk][tl][0] = d[kk][tl][1] = d[kk][tl][2] = d[kk][tl][3] = 0;
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int kk = 0; kk < KK; ++kk) {
            const uint32_t msk = kSubMask << ((k + kk) * BITS);
            const uint32_t am[4] = {af[c][0] & msk, af[c][1] & msk, af[c][2] & msk, af[c][3] & msk};
            mma_u8s8(d[kk][0], am, bk[c][0][0], bk[c][0][1]);
            mma_u8s8(d[kk][1], am, bk[c][1][0], bk[c][1][1]);
          }
        // d[kk][0] = (row g | g+8, cols 2tq, 2tq+1) = head tq limbs 0, 1; d[kk][1] col 2tq = head tq limb 2
#pragma unroll
        for (int kk = 0; kk < KK; ++kk) {
          const float sc = kscale * __int_as_float((127 - (k + kk) * BITS) << 23);  // step * 2^-(k b)
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            const int d01 = d[kk][0][2 * r] + (d[kk][0][2 * r + 1] << 7);  // |d01| < 2^30
            const float v = fmaf(16384.f, (float)d[kk][1][2 * r], (float)d01);
            const float x = fmaf(v, sc, c0);
            if (full || tok + 8 * P * r + k + kk < t1) {
              mn = fminf(mn, x);
              mx = fmaxf(mx, x);
            }
            lg[logit_pos(u, k + kk, tq, g + 8 * r)] = x;
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) tc::mbar_arrive(&F.empty[slot]);
    refill(gk);
  }

  // ---- 4. logit range of the whole row (cluster), calibration slope
  // lanes with equal tq hold the same head
  mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, 4));
  mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, 8));
  mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, 16));
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
  if (lane < kG) {
    F.red[warp][lane][0] = mn;
    F.red[warp][lane][1] = mx;
  }
  __syncthreads();
  tc::cluster_wait();  // every CTA of the cluster is running
  if (t < kG * kMaxCl) {  // thread (h, r): push this CTA's range of head h to peer r
    const int h = t & 3, r = t >> 2;
    float m = FLT_MAX, M = -FLT_MAX;
#pragma unroll
    for (int q = 0; q < kWarps; ++q) {
      m = fminf(m, F.red[q][h][0]);
      M = fmaxf(M, F.red[q][h][1]);
    }
    if (r < cl) {
      tc::st_peer_f32(&F.mM[rank][h][0], r, m);
      tc::st_peer_f32(&F.mM[rank][h][1], r, M);
    }
  }
  tc::cluster_sync();
  if (t < kG) {
    float m = FLT_MAX, M = -FLT_MAX;
    for (int r = 0; r < cl; ++r) {
      m = fminf(m, F.mM[r][t][0]);
      M = fmaxf(M, F.mM[r][t][1]);
    }
    float slope = 1.f, cst = 0.f;
    if (a.calib && M > m) {
      slope = (a.tau_hi * M - a.tau_lo * m) / (M - m);
      cst = a.tau_lo * m - slope * m;  // g(x) = slope x + cst
    }
    F.alog2[t] = slope * kLog2e;
    F.ref[t] = fmaxf(slope * m, slope * M) * kLog2e;
    F.cst[t] = cst;
  }
  __syncthreads();

  // ---- 5. softmax weights P = p_i 2^(31 - k b) as four uint8 limbs in the
  // A-fragment order of the V side, over the logits (a tile's 2 units of logits
  // hold exactly its P x 512 bytes of fragments). Thread (tsub, k, h, grp) takes
  // sub-position k, head h, byte columns 4 grp .. 4 grp + 3 of tiles tsub,
  // tsub + b, ... (at most 8 per thread); all of them are read before any
  // fragment is written.
  float lsum = 0.f;
  {
    const int tsub = t / (32 * P), k = (t / 32) % P, h = (lane >> 3) & 3, grp = lane & 7;
    const float alog2 = F.alog2[h], bias = (float)(31 - k * BITS) - F.ref[h];
    const float unscale = __int_as_float((127 - 31 + k * BITS) << 23);  // 2^(k b - 31)
    // byte columns 4 grp .. of tile lt: unit 2 lt + grp / 4, byte rows 4 (grp % 4) ..
    const float* src = sLf + (grp >> 2) * kUnitWords + logit_pos(grp >> 2, k, h, 4 * (grp & 3));
    // lane 4 h + grp % 4 holds A rows h (limb 0) and h + 8 (limb 2); lane + 16 rows h + 4, h + 12
    uint8_t* dst = sL + (size_t)(k * 32 + 4 * h + (grp & 3)) * 16 + (grp >> 2) * 8;
    float4 xv[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int lt = tsub + i * BITS;
      if (lt < nvtl) xv[i] = *reinterpret_cast<const float4*>(src + (size_t)lt * 2 * kUnitWords);
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int lt = tsub + i * BITS;
      if (lt >= nvtl) break;
      const float xs[4] = {xv[i].x, xv[i].y, xv[i].z, xv[i].w};
      const int i0 = t0 + lt * kTileTok + 4 * P * grp + k;  // token of byte column 4 grp
      uint32_t Pw[4];
      if (t0 + (lt + 1) * kTileTok <= t1) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float p = ex2_approx(fmaf(xs[j], alog2, bias));
          Pw[j] = __float2uint_rn(p);
          lsum += p;
        }
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const bool ok = i0 + P * j < t1;
          const float p = ex2_approx(fmaf(xs[j], alog2, bias));
          Pw[j] = ok ? __float2uint_rn(p) : 0u;
          lsum += ok ? p : 0.f;
        }
      }
      // word l = byte l of Pw[0..3]
      const uint32_t lo01 = __byte_perm(Pw[0], Pw[1], 0x5140), hi01 = __byte_perm(Pw[0], Pw[1], 0x7362);
      const uint32_t lo23 = __byte_perm(Pw[2], Pw[3], 0x5140), hi23 = __byte_perm(Pw[2], Pw[3], 0x7362);
      const uint32_t w0 = __byte_perm(lo01, lo23, 0x5410), w1 = __byte_perm(lo01, lo23, 0x7632);
      const uint32_t w2 = __byte_perm(hi01, hi23, 0x5410), w3 = __byte_perm(hi01, hi23, 0x7632);
      *reinterpret_cast<uint2*>(dst + (size_t)lt * 512 * P) = make_uint2(w0, w2);
      *reinterpret_cast<uint2*>(dst + (size_t)lt * 512 * P + 256) = make_uint2(w1, w3);
    }
    lsum *= unscale;
    // lanes with equal h: xor over grp
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 1);
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 2);
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 4);
    if (grp == 0) F.lsum[warp][h] = lsum;
  }
  __syncthreads();  // the weight fragments are complete

  // ---- 6. V side: chunk gv holds tiles 4 gv .. 4 gv + 3; warp pair p takes tile
  // 4 gv + p, warp parity picks channels 64 hc .. 64 hc + 63. D rows (limb, head).
  const int hc = warp & 1, pair = warp >> 1;
  int acc[8][4];
#pragma unroll
  for (int j = 0; j < 8; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0;
  for (int gv = 0; gv < nv; ++gv) {
    const int gi = nk + gv, slot = gi % kSlots;
    wait_copies(&F.full[slot], (uint32_t)(gi / kSlots) & 1u, err);
    const int lt = 4 * gv + pair;
    if (lt < nvtl) {
      const uint32_t tile_u = ring_u + slot * kChunkBytes + pair * 4096;
      const uint32_t frag_u = sL_u + lt * 512 * P + lane * 16;
      uint32_t bv[8][2];
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        const int mat = lane >> 3, half = mat & 1;
        const int ch = 64 * hc + 16 * p + 8 * (mat >> 1) + (lane & 7);
        uint32_t r[4];
        ldsm_x4(tile_u + (ch >> 2) * 128 + (((((ch & 3) << 1) | half) ^ ((ch >> 2) & 7)) << 4), r);
        bv[2 * p][0] = r[0];
        bv[2 * p][1] = r[1];
        bv[2 * p + 1][0] = r[2];
        bv[2 * p + 1][1] = r[3];
      }
#pragma unroll
      for (int k = 0; k < P; ++k) {
        uint32_t af[4];
        lds128(frag_u + k * 512, af);
        const uint32_t msk = kSubMask << (k * BITS);
#pragma unroll
        for (int j = 0; j < 8; ++j) mma_u8u8(acc[j], af, bv[j][0] & msk, bv[j][1] & msk);
      }
    }
    __syncwarp();
    if (lane == 0) tc::mbar_arrive(&F.empty[slot]);
    refill(gi);
  }

  // ---- 7. combine limbs (lane and lane ^ 16), sum the warp pairs, scatter to the owners
  // Lane with g < 4 holds limbs 0 and 2 of head g, lane + 16 limbs 1 and 3.
  __syncthreads();  // every warp is done with the ring: the partial sums reuse it
  {
    const float s_lo = (g < 4) ? 0x1p-31f : 0x1p-23f, s_hi = (g < 4) ? 0x1p-15f : 0x1p-7f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      float v[2];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        v[c] = fmaf((float)acc[j][c + 2], s_hi, (float)acc[j][c] * s_lo);
        v[c] += __shfl_xor_sync(0xffffffffu, v[c], 16);
      }
      if (lane < 16)
        *reinterpret_cast<float2*>(sPart + (pair * kG + g) * kPartStride + 64 * hc + 8 * j + 2 * tq) =
            make_float2(v[0], v[1]);
    }
  }
  __syncthreads();
  // CTA r of the cluster owns channels [r kD / cl, (r + 1) kD / cl); recv rows are ceil(kD / cl) wide
  const int wrecv = (kD + cl - 1) / cl;
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int idx = 2 * t + e, h = idx >> 7, ch = idx & 127;
    float s = 0.f;
#pragma unroll
    for (int q = 0; q < kWarps / 2; ++q) s += sPart[(q * kG + h) * kPartStride + ch];
    int owner = 0;
    while ((owner + 1) * kD / cl <= ch) ++owner;
    const int first = owner * kD / cl;
    tc::st_peer_f32(&F.recv[((int)rank * kG + h) * wrecv + ch - first], (uint32_t)owner, s);
  }
  if (t < kG * kMaxCl) {  // thread (h, r): this CTA's sum of weights of head h to peer r
    const int h = t & 3, r = t >> 2;
    if (r < cl) {
      float l = 0.f;
#pragma unroll
      for (int q = 0; q < kWarps; ++q) l += F.lsum[q][h];
      tc::st_peer_f32(&F.part_l[rank][h], (uint32_t)r, l);
    }
  }
  tc::cluster_sync();

  // ---- 8. every CTA finishes its channels: o = alpha_V + s_V (.) sum c p / sum p
  {
    const int first = (int)rank * kD / cl, width = ((int)rank + 1) * kD / cl - first;
    for (int e = t; e < kG * width; e += kThreads) {
      const int h = e / width, ch = first + e % width;
      float s = 0.f, l = 0.f;
      for (int r = 0; r < cl; ++r) {
        s += F.recv[(r * kG + h) * wrecv + ch - first];
        l += F.part_l[r][h];
      }
      const float alpha = DT<T>::f(sRows[6 * kD + ch]);
      const float step = *err ? __int_as_float(0x7fc00000) : DT<T>::f(sRows[7 * kD + ch]);
      const size_t bh = (size_t)b * a.Hq + (size_t)kG * hkv + h;
      if (a.part_o == nullptr) {
        static_cast<T*>(a.out)[bh * kD + ch] = DT<T>::from_float(fmaf(step, s / l, alpha));
      } else {
        a.part_o[bh * kD + ch] = fmaf(step, s / l, alpha);
        // sum_i exp(y_i) = 2^ref sum_i p_i e^cst with p_i = 2^(x_i alog2 - ref)
        if (ch == 0) a.part_lse[bh] = fmaf(F.ref[h], 0.6931471805599453f, logf(l)) + F.cst[h];
      }
    }
  }
  if (*err && t == 0) {  // let copies still in flight land before the CTA's memory is reused
    report_timeout(a.status);
    tc::mbar_wait(&F.bar_rows, 0, kSpin);
    for (int gi = nchunks - kSlots; gi < nchunks; ++gi)
      if (gi >= 0) tc::mbar_wait(&F.full[gi % kSlots], (uint32_t)(gi / kSlots) & 1u, kSpin);
  }
}

template <typename T, int BITS, int SLOTS>
cudaError_t run_bits(const DecodeArgs& a, int rows, int nvt, int cl, cudaStream_t stream) {
  constexpr int P = 8 / BITS;
  const size_t smem = ring_smem_bytes<T, SLOTS>() + 1024;  // slack to align to the 1024-byte swizzle atom
  static bool attr_sets[kMaxDevices];  // per device (benign race: every caller sets the same value)
  const int attr_dev = current_device();
  if (attr_dev < 0) return cudaErrorInvalidDevice;
  bool& attr_set = attr_sets[attr_dev];
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(k_decode_ring<T, BITS, SLOTS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(k_decode_ring<T, BITS, SLOTS>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  CUtensorMap kmap, vmap;
  const uint64_t byte_rows = (uint64_t)(a.n + P - 1) / P;
  if (!encode_3d(&kmap, a.k_codes, 128, byte_rows, (uint64_t)rows, kChunkRows, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_3d(&vmap, a.v_codes, 128, (uint64_t)nvt * 32, (uint64_t)rows, kChunkRows, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
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
  return cudaLaunchKernelEx(&cfg, k_decode_ring<T, BITS, SLOTS>, a, cl, kmap, vmap);
}

template <typename T, int BITS>
cudaError_t run_bits(const DecodeArgs& a, cudaStream_t stream) {
  constexpr int kTileTok = 32 * (8 / BITS);
  const int rows = a.B * a.Hkv;
  const int nvt = (a.n + kTileTok - 1) / kTileTok;
  const int per = kSlice / kTileTok;  // V tiles per CTA
  const int cl = (nvt + per - 1) / per;
  if (cl > kMaxCl || (long long)rows * cl > 0x7fffffffLL) return cudaErrorNotSupported;
  if (ring_slots_for((long long)rows * cl, device_sms()) == 4) return run_bits<T, BITS, 4>(a, rows, nvt, cl, stream);
  return run_bits<T, BITS, 2>(a, rows, nvt, cl, stream);
}

template <typename T>
cudaError_t run(const DecodeArgs& a, cudaStream_t stream) {
  switch (a.bits) {
    case 2: return run_bits<T, 2>(a, stream);
    case 4: return run_bits<T, 4>(a, stream);
    case 8: return run_bits<T, 8>(a, stream);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace

bool decode_ring_supports(int n, int bits) {
  if (bits != 2 && bits != 4 && bits != 8) return false;
  return n >= 1 && n <= kMaxCl * kSlice;
}

cudaError_t launch_decode_ring(const DecodeArgs& a, cq_dtype dt, cudaStream_t stream) {
  if (!decode_ring_supports(a.n, a.bits)) return cudaErrorNotSupported;
  if (dt == CQ_F16) return run<half>(a, stream);
  return run<float>(a, stream);
}

}  // namespace cq
