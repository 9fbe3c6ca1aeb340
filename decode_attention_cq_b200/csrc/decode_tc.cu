// Fused 1-bit decode attention on the 5th-generation tensor cores: one
// persistent CTA per SM owns all 512 tensor-memory columns and works through
// whole (batch, kv-head) rows.
//
// Method (CalibQuant article): logits x_i = sigma q.alpha_K + (sigma q (.) s_K)
// . c^K_i on the integer codes (Method 2, post-scaling), calibration map g on
// the row's score range (Method 3), softmax, o = alpha_V + s_V (.)
// sum_i p_i c^V_i / sum_i p_i (Method 2 applied to V).
//
// Both contractions run as tcgen05.mma.kind::i8 (M = 128, N = 16, K = 32, A in
// tensor memory, B in shared memory, int32 accumulators in tensor memory):
//  * K side, one unit per (block of 128 octets = 1024 tokens, bit k): lane m of
//    A holds octet m's 128 code bytes masked to bit k ("code of token 8m + k
//    times 2^k" per channel); B holds the weights w_h = sigma q_h (.) s_K in
//    22-bit fixed point as three int8 limbs per head (columns 4 h + l). The
//    accumulators start from the bit pattern of 1.5 * 2^23 so that each reads
//    back as a float with one subtraction.
//  * V side, one unit per (256-token tile, half of the bit positions): lane j
//    of A holds channel j's 32 octet bytes masked to bit k; B holds p_i
//    2^(31 - k) as four uint8 limbs per head, so every bit accumulates into
//    the same int32 sum of c_ij p_i 2^31.
// The calibration slope needs the range of every logit of the row before any
// weight exists, so the row's fp32 logits (16 B per token) stay in shared
// memory between the two sides and the range is a barrier inside the CTA.
//
// 16 warps in 4 groups of 4: warp 4 g + q reaches tensor-memory lanes 32 q ..
// 32 q + 31, so a group covers the 128 lanes of its own 128 columns. Group g
// takes K blocks g, g + 4, .. and V tiles g, g + 4, .. of every row. Each warp
// writes its lanes of a unit's A operand and arrives on the slot's mbarrier;
// the unit's MMAs are issued by one warp of the group in turn (unit k by warp
// k % 4), which waits for the other three: a warp issues one MMA about every
// 50 cycles, so the issuing is spread over the warps and the four groups
// issue in parallel. Per row:
//  1. K side: one TMA copy per K block (16 KB, 128-byte swizzle); each warp
//     loads its octet row into registers, the last one to do so starts the
//     group's next copy; per bit k the masked codes go to A slot k % 2, the
//     MMAs into D slot k % 4, and the logits of the unit two back are read:
//     x = c0 + step 2^-k (D0 + 2^7 D1 + 2^14 D2), stored with the row range;
//  2. range: warp shuffles and one CTA barrier; then the next row's weight
//     limbs (head g by group g) while this row's V side runs;
//  3. V side: per half-tile each warp writes the softmax weights of one bit
//     (B) and the masked V codes of its 32 channels (A); the half-tiles'
//     MMAs rotate over the four warps, each into its own accumulator (so every
//     accumulator receives MMAs from one thread, in order), and the four are
//     added exactly at the end;
//  4. output: o = alpha_V + s_V (.) sum D_V / sum p, head g by group g.
// Every mbarrier wait is bounded; a wait that runs out makes the outputs NaN.
// No workspace; 1 <= n <= 8192 tokens per row; one launch per decode step.
#include <float.h>

#include "common.cuh"
#include "kernels.h"
#include "mma_util.cuh"
#include "tc.cuh"

namespace cq {

namespace {

using namespace mu;

constexpr int kWarpsTc = 16;
constexpr int kGroups = 4;
constexpr int kThreadsTc = kWarpsTc * 32;  // 512
constexpr int kBlkOct = 128;               // octets per K block (M)
constexpr int kBlkBytes = kBlkOct * kD;    // 16 KB
constexpr int kVTileTc = 256;              // tokens per V tile
constexpr int kMaxNTc = 8192;
constexpr int kMaxOct = kMaxNTc / 8;
constexpr int kWMaxTc = (1 << 21) - 1;      // 22-bit signed fixed point for the K weights
constexpr uint32_t kBiasBits = 0x4B400000u;  // 1.5 * 2^23: an int32 d added to it reads as 1.5 * 2^23 + d
constexpr float kBiasF = 12582912.0f;
constexpr float kLog2eTc = 1.4426950408889634f;
constexpr uint32_t kSpinTc = 1u << 22;  // bound on the probes of every mbarrier wait

// Tensor-memory columns of group g start at 128 g: A slots at +0 / +32 (32
// columns = 128 code bytes per lane on the K side, four bits x 8 columns on
// the V side); K side D slot s at +64 + 16 s (s = 0..3); V side accumulator of
// warp q at +64 + 16 q.
constexpr uint32_t kColD = 64;

struct TcSmem {
  float4 logit[8][kMaxOct];          // [bit][octet]: the 4 heads' logits of token 8 octet + bit
  uint8_t kblk[kGroups][kBlkBytes];  // K codes: one block per group (128-byte swizzle)
  uint8_t bv[kGroups][2][4][512];    // V-side B: [group][slot][bit in half][32 octets x 16 B]
  uint8_t bk[4][512];                // K-side B: [32-channel chunk][32 channels x 16 B]
  float part[kGroups][kG][kD];       // per group: sum_i c_ij p_i of its tiles
  uint64_t kload[kGroups];
  uint64_t kdone[kGroups][4], vdone[kGroups][2];
  uint64_t kfull[kGroups][2], vfull[kGroups][2];  // the four warps' A (and V-side B) parts of a slot are in place
  uint32_t fcnt[kGroups];                          // arrivals per K block (the last one refills)
  float red[kWarpsTc][kG][2];  // per warp: logit range per head
  float lsum[kWarpsTc][kG];    // per warp: sum of softmax weights per head
  float sred[kGroups][4][2];   // setup: per group, per warp (max |w|, q.alpha)
  alignas(16) float c0[kG];
  alignas(16) float kscale[kG];
  int err;
  uint32_t tmem_base;
};

constexpr size_t kSmemTc = sizeof(TcSmem) + 1024;  // + alignment of the swizzled K blocks
static_assert(kSmemTc <= 227 * 1024, "one CTA per SM must fit in shared memory");
static_assert(kSmemTc > 228 * 1024 / 2, "two CTAs per SM would contend for tensor memory");

// 2^-k for k = 0..31 (exact)
__device__ __forceinline__ float pow2_neg(int k) { return __int_as_float((127 - k) << 23); }

__device__ __forceinline__ float bits_to_count(uint32_t d) { return __uint_as_float(d) - kBiasF; }

__device__ __forceinline__ void st_x16_same(uint32_t taddr, uint32_t v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1};" ::"r"(taddr),
      "r"(v)
      : "memory");
}
__device__ __forceinline__ float4 lds_f4(const float4* p) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(tc::smem_u32(p))
               : "memory");
  return v;
}
__device__ __forceinline__ uint4 ldg_v4(const uint8_t* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// D[tmem] (+)= A[tmem] x B[smem], kind::i8, issued by one thread (the form
// without an output-lane mask).
__device__ __forceinline__ void mma_i8(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d),
      "r"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

// Count one arrival (release, and acquire of the earlier ones); returns the
// count before it.
__device__ __forceinline__ uint32_t count_in(uint32_t* cnt) {
  uint32_t old;
  asm volatile("atom.acq_rel.cta.shared::cta.add.u32 %0, [%1], 1;" : "=r"(old) : "r"(tc::smem_u32(cnt)) : "memory");
  return old;
}

// One probe of the phase with the given parity; a thread whose phase is not
// complete may be suspended for up to `ns` nanoseconds first.
__device__ __forceinline__ bool try_wait_ns(uint64_t* mbar, uint32_t parity, uint32_t ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(tc::smem_u32(mbar)), "r"(parity), "r"(ns)
      : "memory");
  return ok != 0;
}

// The whole warp waits for the phase of `bar` with the given parity, each lane
// sleeping in try_wait rather than spinning; a wait that runs out (kSpinTc
// probes) flags the CTA.
__device__ __forceinline__ void wait_bar(uint64_t* bar, uint32_t parity, volatile int* err) {
  uint32_t i = 0;
  while (!try_wait_ns(bar, parity, 1000000u))
    if (++i == kSpinTc) {
      *err = 1;
      break;
    }
  __syncwarp();
}

__device__ __forceinline__ float warp_min_tc(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Blocks and tiles of group g in a row: g, g + 4, ... < total.
__device__ __forceinline__ int group_count(int total, int g) {
  return total > g ? (total - g + kGroups - 1) / kGroups : 0;
}

template <typename T>
__global__ void __launch_bounds__(kThreadsTc, 1)
    k_decode_tc(const __grid_constant__ DecodeArgs a, int rows, const __grid_constant__ CUtensorMap kmap) {
  extern __shared__ uint8_t smem_raw[];
  TcSmem& S = *reinterpret_cast<TcSmem*>(smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u));

  const int t = threadIdx.x, warp = __shfl_sync(0xffffffffu, t >> 5, 0), lane = t & 31;
  const int g = warp >> 2, q = warp & 3;
  const int ch = 32 * q + lane;  // channel (setup, V side, output) / octet within a K block
  const int n = a.n, octets = (n + 7) >> 3;
  const int nkb = (octets + kBlkOct - 1) / kBlkOct;  // K blocks of a row
  const int nvt = (n + kVTileTc - 1) / kVTileTc;     // V tiles of a row
  const int nb = group_count(nkb, g), nv = group_count(nvt, g);
  const size_t vrow_bytes = (size_t)nvt * 4096;
  volatile int* err = &S.err;

  if (t == 0) {
    S.err = 0;
    for (int gg = 0; gg < kGroups; ++gg) {
      tc::mbar_init(&S.kload[gg], 1);
      for (int i = 0; i < 4; ++i) tc::mbar_init(&S.kdone[gg][i], 1);
      for (int i = 0; i < 2; ++i) {
        tc::mbar_init(&S.vdone[gg][i], 1);
        tc::mbar_init(&S.kfull[gg][i], 4);
        tc::mbar_init(&S.vfull[gg][i], 4);
      }
      S.fcnt[gg] = 0;
    }
    tc::fence_mbar_init();
  }
  if (warp == 0) {
    tc::tmem_alloc(&S.tmem_base, 512);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = S.tmem_base;
  const uint32_t lane_off = (uint32_t)(32 * q) << 16;
  const uint32_t gcol = tmem + lane_off + 128u * g;  // this warp's lanes of the group's columns
  const uint32_t mcol = tmem + 128u * g;             // the group's columns (MMA operands)
  constexpr uint32_t kIdescK = tc::idesc_i8(true, 16), kIdescV = tc::idesc_i8(false, 16);
  // descriptors of B blocks 512 bytes apart differ by 512 / 16 in the start-address field
  const uint64_t dk0 = tc::smem_desc(S.bk[0], 128, 512), dv0 = tc::smem_desc(S.bv[g][0][0], 128, 512);

  // K block b of group g in row `row` -> shared memory (one thread)
  auto load_block = [&](int row, int b) {
    tc::mbar_arrive_expect_tx(&S.kload[g], kBlkBytes);
    tc::tma_load_3d(S.kblk[g], &kmap, 0, (g + kGroups * b) * kBlkOct, row, &S.kload[g]);
  };
  // q, alpha_K, s_K of head g / channel ch
  auto load_setup = [&](int row, float& qv, float& ak, float& sk) {
    const int b = row / a.Hkv, hkv = row % a.Hkv;
    qv = DT<T>::f(static_cast<const T*>(a.q)[((size_t)b * a.Hq + (size_t)kG * hkv + g) * kD + ch]);
    ak = DT<T>::f(static_cast<const T*>(a.k_alpha)[(size_t)row * kD + ch]);
    sk = DT<T>::f(static_cast<const T*>(a.k_scale)[(size_t)row * kD + ch]);
  };
  // head g's weights w = sigma q (.) s_K as three int8 limbs (B of the K side)
  // and its constant term; group g's 128 threads, one channel each
  auto setup = [&](float qv, float ak, float sk) {
    const float w = a.sigma * qv * sk;
    const float am = warp_max(fabsf(w));
    const float qa = warp_sum(qv * ak);
    if (lane == 0) {
      S.sred[g][q][0] = am;
      S.sred[g][q][1] = qa;
    }
    tc::bar_sync(1 + g, 128);
    const float amax = fmaxf(fmaxf(S.sred[g][0][0], S.sred[g][1][0]), fmaxf(S.sred[g][2][0], S.sred[g][3][0]));
    const float ks = amax * (1.f / (float)kWMaxTc);
    const float inv = ks > 0.f ? __fdividef(1.f, ks) : 0.f;  // approximate: the clamp bounds w
    const int wi = max(-kWMaxTc, min(kWMaxTc, __float2int_rn(w * inv)));
    *reinterpret_cast<uint32_t*>(&S.bk[ch >> 5][(ch & 31) * 16 + 4 * g]) =
        (uint32_t)(wi & 127) | ((uint32_t)((wi >> 7) & 127) << 8) | ((uint32_t)((wi >> 14) & 255) << 16);
    if (q == 0 && lane == 0) {
      S.kscale[g] = ks;
      S.c0[g] = a.sigma * (S.sred[g][0][1] + S.sred[g][1][1] + S.sred[g][2][1] + S.sred[g][3][1]);
    }
    tc::fence_proxy_async();
  };

  {
    float qv, ak, sk;
    if ((int)blockIdx.x < rows) {
      if (q == 0 && lane == 0 && nb > 0) load_block(blockIdx.x, 0);
      load_setup(blockIdx.x, qv, ak, sk);
      setup(qv, ak, sk);
    }
  }
  __syncthreads();  // the first row's weight limbs are in place

  uint32_t kbc = 0, vs = 0;
  for (int row = blockIdx.x; row < rows; row += gridDim.x) {
    const bool more = row + (int)gridDim.x < rows;
    // ---- 1. K side. Unit 8 c + k (bit k of the group's c-th block) masks into
    // A slot k % 2, accumulates into D slot k % 4, and its logits are read back
    // two units later; with 8 units per block every slot and parity is a
    // constant of k.
    float mn[kG], mx[kG];
#pragma unroll
    for (int h = 0; h < kG; ++h) {
      mn[h] = FLT_MAX;
      mx[h] = -FLT_MAX;
    }
    float c0v[kG], ksv[kG];
#pragma unroll
    for (int h = 0; h < kG; ++h) {
      c0v[h] = S.c0[h];
      ksv[h] = S.kscale[h];
    }
    // logits of bit k of block kb from D slot k % 4
    auto epilogue = [&](int kb, int k) {
      uint32_t d[16];
      tc::ld_x16(gcol + kColD + 16u * (uint32_t)(k & 3), d);
      tc::wait_ld();
      const float pw = pow2_neg(k);
      float x[kG];
#pragma unroll
      for (int h = 0; h < kG; ++h) {
        const float d0 = bits_to_count(d[4 * h]), d1 = bits_to_count(d[4 * h + 1]), d2 = bits_to_count(d[4 * h + 2]);
        x[h] = fmaf(fmaf(16384.f, d2, fmaf(128.f, d1, d0)), ksv[h] * pw, c0v[h]);
      }
      const int oct = kBlkOct * kb + ch;
      if (8 * oct + k < n) {
#pragma unroll
        for (int h = 0; h < kG; ++h) {
          mn[h] = fminf(mn[h], x[h]);
          mx[h] = fmaxf(mx[h], x[h]);
        }
      }
      S.logit[k][oct] = make_float4(x[0], x[1], x[2], x[3]);
    };
#pragma unroll 1
    for (int bi = 0; bi < nb; ++bi) {
      const int kb = g + kGroups * bi;
      uint32_t raw[32];
      wait_bar(&S.kload[g], kbc & 1u, err);
      {
        const uint32_t base = tc::smem_u32(S.kblk[g]) + (uint32_t)ch * 128u;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t r4[4];
          lds128(base + ((uint32_t)(c ^ (ch & 7)) << 4), r4);
          raw[4 * c] = r4[0];
          raw[4 * c + 1] = r4[1];
          raw[4 * c + 2] = r4[2];
          raw[4 * c + 3] = r4[3];
        }
      }
      __syncwarp();
      if (lane == 0 && (count_in(&S.fcnt[g]) & 3u) == 3u) {  // the last warp out starts the next copy
        if (bi + 1 < nb) load_block(row, bi + 1);
        else if (more) load_block(row + gridDim.x, 0);
      }
      const bool first = kbc == 0;  // no unit before this block anywhere
      ++kbc;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        // A slot k % 2 was read by the unit two back: bit k - 2 of this block (D
        // slot (k - 2) % 4 in its use 0 for bits 0..3, parity 0, use 1 for bits
        // 4, 5, parity 1) or bit k + 6 of the previous block (use 1, parity 1)
        if (k >= 2 || !first) wait_bar(&S.kdone[g][(k + 2) & 3], k >= 2 && k < 6 ? 0u : 1u, err);
        tc::fence_after_sync();
        {
          const uint32_t m = 0x01010101u << k;
          uint32_t v[32];
#pragma unroll
          for (int x = 0; x < 32; ++x) v[x] = raw[x] & m;
          tc::st_x32(gcol + 32u * (uint32_t)(k & 1), v);
        }
        st_x16_same(gcol + kColD + 16u * (uint32_t)(k & 3), kBiasBits);  // read back two units later
        tc::wait_st();
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&S.kfull[g][k & 1]);
        if (q == (k & 3)) {  // warp k % 4 issues bit k: slot k % 2, its (k / 2)-th use in the block
          wait_bar(&S.kfull[g][k & 1], (uint32_t)(k >> 1) & 1u, err);
          tc::fence_after_sync();
          if (lane == 0) {
            if (*err == 0) {
#pragma unroll
              for (int c = 0; c < 4; ++c)
                mma_i8(mcol + kColD + 16u * (uint32_t)(k & 3), mcol + 32u * (uint32_t)(k & 1) + 8u * c,
                       dk0 + 32u * c, kIdescK, 1u);
            }
            tc::mma_commit(&S.kdone[g][k & 3]);
          }
          __syncwarp();
        }
        if (k >= 2) epilogue(kb, k - 2);
        else if (bi > 0) epilogue(kb - kGroups, k + 6);
      }
    }
    if (nb > 0) {  // the row's last two units: bits 6 and 7 of the last block
      const int kb = g + kGroups * (nb - 1);
      wait_bar(&S.kdone[g][2], 1u, err);
      tc::fence_after_sync();
      epilogue(kb, 6);
      wait_bar(&S.kdone[g][3], 1u, err);
      tc::fence_after_sync();
      epilogue(kb, 7);
    }
    tc::fence_before_sync();

    // ---- 2. ahead of the barrier: this row's first V codes and statistics and
    // the next row's setup values; then the row range
    const uint8_t* vrow = a.v_codes + (size_t)row * vrow_bytes + (size_t)ch * 32;
    uint4 nlo = make_uint4(0, 0, 0, 0), nhi = nlo;
    if (nv > 0) {
      nlo = ldg_v4(vrow + (size_t)g * 4096);
      nhi = ldg_v4(vrow + (size_t)g * 4096 + 16);
    }
    const float av = DT<T>::f(static_cast<const T*>(a.v_alpha)[(size_t)row * kD + ch]);
    const float sv = DT<T>::f(static_cast<const T*>(a.v_scale)[(size_t)row * kD + ch]);
    float qv = 0.f, ak = 0.f, sk = 0.f;
    if (more) load_setup(row + gridDim.x, qv, ak, sk);
    float alog2[kG], ref[kG];
#pragma unroll
    for (int h = 0; h < kG; ++h) {
      const float m = warp_min_tc(mn[h]), M = warp_max(mx[h]);
      if (lane == 0) {
        S.red[warp][h][0] = m;
        S.red[warp][h][1] = M;
      }
    }
    __syncthreads();  // every logit and range of the row; every K MMA of the row is complete
#pragma unroll
    for (int h = 0; h < kG; ++h) {
      float m = S.red[lane & 15][h][0], M = S.red[lane & 15][h][1];
#pragma unroll
      for (int o = 8; o; o >>= 1) {
        m = fminf(m, __shfl_xor_sync(0xffffffffu, m, o));
        M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
      }
      float slope = 1.f;
      if (a.calib && M > m) slope = (a.tau_hi * M - a.tau_lo * m) / (M - m);
      alog2[h] = slope * kLog2eTc;
      ref[h] = fmaxf(slope * m, slope * M) * kLog2eTc;
    }
    if (more) setup(qv, ak, sk);  // the next row's weight limbs (this row's K MMAs are done)

    // ---- 3. V side: half-tile j (bits 4 (j & 1) .. + 3 of tile j / 2) in slot vs % 2;
    // the warp that completes a half-tile runs its MMAs into its own accumulator
    st_x16_same(gcol + kColD, 0u);  // the four accumulators of this warp's lanes start at zero
    st_x16_same(gcol + kColD + 16u, 0u);
    st_x16_same(gcol + kColD + 32u, 0u);
    st_x16_same(gcol + kColD + 48u, 0u);
    float lsum[kG] = {0.f, 0.f, 0.f, 0.f};
    {
#pragma unroll 1
      for (int j = 0; j < nv; ++j, ++vs) {  // vs: tiles of this group so far
        const int vt = g + kGroups * j;
        const uint32_t wv[8] = {nlo.x, nlo.y, nlo.z, nlo.w, nhi.x, nhi.y, nhi.z, nhi.w};
        if (j + 1 < nv) {
          nlo = ldg_v4(vrow + (size_t)(vt + kGroups) * 4096);
          nhi = ldg_v4(vrow + (size_t)(vt + kGroups) * 4096 + 16);
        }
        const bool full = kVTileTc * (vt + 1) <= n;
#pragma unroll
        for (int h = 0; h < 2; ++h) {  // bits 4 h .. 4 h + 3 in slot h
          const int k = 4 * h + q;      // the bit whose B rows this warp writes
          const float4 lg = lds_f4(&S.logit[k][32 * vt + lane]);
          const bool valid = full || kVTileTc * vt + 8 * lane + k < n;
          const float xs[kG] = {lg.x, lg.y, lg.z, lg.w};
          const float back = pow2_neg(31 - k);
          uint32_t pi[kG];
#pragma unroll
          for (int hh = 0; hh < kG; ++hh) {
            const float p2 = ex2_approx(fmaf(xs[hh], alog2[hh], (float)(31 - k) - ref[hh]));  // p 2^(31-k)
            pi[hh] = valid ? __float2uint_rn(p2) : 0u;
            lsum[hh] = valid ? fmaf(p2, back, lsum[hh]) : lsum[hh];
          }
          // the slot's previous tile has been read by its MMAs
          if (vs > 0) wait_bar(&S.vdone[g][h], (vs - 1) & 1u, err);
          sts128(tc::smem_u32(&S.bv[g][h][q][lane * 16]), pi);
          tc::fence_proxy_async();
          tc::fence_after_sync();
          {
            uint32_t v[32];
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {
              const uint32_t m = 0x01010101u << (4 * h + k4);
#pragma unroll
              for (int x = 0; x < 8; ++x) v[8 * k4 + x] = wv[x] & m;
            }
            tc::st_x32(gcol + 32u * (uint32_t)h, v);
          }
          tc::wait_st();
          tc::fence_before_sync();
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(&S.vfull[g][h]);
          if (q == (int)((2u * vs + (uint32_t)h) & 3u)) {  // half-tiles rotate over the warps' accumulators
            wait_bar(&S.vfull[g][h], vs & 1u, err);
            tc::fence_after_sync();
            if (lane == 0) {
              if (*err == 0) {
#pragma unroll
                for (int k4 = 0; k4 < 4; ++k4)
                  mma_i8(mcol + kColD + 16u * q, mcol + 32u * (uint32_t)h + 8u * k4,
                         dv0 + 32u * (4u * (uint32_t)h + (uint32_t)k4), kIdescV, 1u);
              }
              tc::mma_commit(&S.vdone[g][h]);
            }
            __syncwarp();
          }
        }
      }
    }
    // the row's last two half-tiles; then this group's sums for this warp's channels
    if (nv > 0) {  // the row's last tile, both halves
      wait_bar(&S.vdone[g][0], (vs - 1) & 1u, err);
      wait_bar(&S.vdone[g][1], (vs - 1) & 1u, err);
    }
    tc::wait_st();
    tc::fence_after_sync();
    {
      // which warp issued a half-tile varies from call to call: the four
      // accumulators are added exactly (int32) before the one conversion
      int sum[16];
#pragma unroll
      for (int x = 0; x < 16; ++x) sum[x] = 0;
#pragma unroll
      for (int qq = 0; qq < 4; ++qq) {
        uint32_t d[16];
        tc::ld_x16(gcol + kColD + 16u * qq, d);
        tc::wait_ld();
#pragma unroll
        for (int x = 0; x < 16; ++x) sum[x] += (int)d[x];
      }
#pragma unroll
      for (int h = 0; h < kG; ++h)
        S.part[g][h][ch] = (float)sum[4 * h] * 0x1p-31f + (float)sum[4 * h + 1] * 0x1p-23f +
                           (float)sum[4 * h + 2] * 0x1p-15f + (float)sum[4 * h + 3] * 0x1p-7f;
    }
#pragma unroll
    for (int h = 0; h < kG; ++h) {
      const float l = warp_sum(lsum[h]);
      if (lane == 0) S.lsum[warp][h] = l;
    }
    tc::fence_before_sync();
    __syncthreads();  // the row's sums; the next row's limbs; every read of this row's logits is done

    // ---- 4. output: head g, channel ch
    {
      float lt = 0.f;
#pragma unroll
      for (int w = 0; w < kWarpsTc; ++w) lt += S.lsum[w][g];
      const float acc = S.part[0][g][ch] + S.part[1][g][ch] + S.part[2][g][ch] + S.part[3][g][ch];
      const int b = row / a.Hkv, hkv = row % a.Hkv;
      const float o = *err ? __int_as_float(0x7fc00000) : fmaf(sv, acc / lt, av);
      static_cast<T*>(a.out)[((size_t)b * a.Hq + (size_t)kG * hkv + g) * kD + ch] = DT<T>::from_float(o);
    }
  }

  if (t == 0 && *err) report_timeout(a.status);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 0) tc::tmem_dealloc(tmem, 512);
}

template <typename T>
cudaError_t run(const DecodeArgs& a, cudaStream_t stream) {
  const int rows = a.B * a.Hkv;
  static int sms[kMaxDevices];  // per device: SM count, 0 until the attributes are set
  const int dev = current_device();
  if (dev < 0) return cudaErrorInvalidDevice;
  if (sms[dev] == 0) {
    int c = 0;
    cudaError_t e = cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(k_decode_tc<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemTc);
    if (e != cudaSuccess) return e;
    sms[dev] = c;
  }
  CUtensorMap kmap;
  if (!encode_3d(&kmap, a.k_codes, kD, (uint64_t)(a.n + 7) / 8, (uint64_t)rows, kBlkOct,
                 CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  const int grid = rows < sms[dev] ? rows : sms[dev];
  k_decode_tc<T><<<grid, kThreadsTc, kSmemTc, stream>>>(a, rows, kmap);
  return cudaGetLastError();
}

}  // namespace

bool decode_tc_supports(int n) { return n >= 1 && n <= kMaxNTc; }

cudaError_t launch_decode_tc(const DecodeArgs& a, cq_dtype dt, cudaStream_t stream) {
  if (!decode_tc_supports(a.n) || a.part_o != nullptr || a.n_text > 0) return cudaErrorNotSupported;
  if (dt == CQ_F16) return run<half>(a, stream);
  return run<float>(a, stream);
}

}  // namespace cq
