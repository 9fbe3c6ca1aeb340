// Fused 1-bit decode attention on register-fed tensor-core MMAs
// (mma.sync m16n8k32, u8 x s8/u8 -> s32) over the octet code layouts; the
// default path for bits = 1, Hq = 4 Hkv, n <= 32768.
//
// Method (CalibQuant article): logits x_i = sigma q.alpha_K + (sigma q (.) s_K)
// . c^K_i on the integer codes (Method 2, post-scaling), calibration map g on
// the row's score range (Method 3), softmax, o = alpha_V + s_V (.)
// sum_i p_i c^V_i / sum_i p_i (Method 2 applied to V).
//
// One thread-block cluster per (batch, kv-head) row, one CTA per slice of at
// most S tokens (S = 2048, or 4096 for n > 16384). Each CTA
//  1. streams its slice of K and V codes into shared memory with a few tensor
//     copies issued by one thread (128-byte swizzle, so that ldmatrix reads are
//     conflict-free), completing on mbarriers;
//  2. K side: per unit of 16 token octets (128 tokens) a warp loads the A
//     fragments of all 128 channels with ldmatrix; masking bit k of every byte
//     gives "code of token 8 r + k times 2^k" for octet row r. B holds the
//     weights w_h = sigma q_h (.) s_K as a 22-bit fixed-point number split into
//     three int8 limbs (two N = 8 tiles: heads x limbs). The unit's logits
//     (2 KB) overwrite its codes (2 KB), which the warp holds in registers;
//  3. exchanges the logit range with the other CTAs of the row (distributed
//     shared memory) and derives the calibration slope;
//  4. turns logits into softmax weights p_i 2^(31-k) as four uint8 limbs,
//     written in A-fragment order over the logits;
//  5. V side: A = weight limbs (16 rows = 4 limbs x 4 heads, K = 32 octets of
//     one bit position), B = masked codes of 8 channels (ldmatrix); a warp
//     pair splits the 128 channels, the four pairs split the tiles;
//  6. sums the warps, scatters the (head, channel) partial sums over the
//     cluster so that every CTA owns a range of channels, and writes o.
// Everything stays on chip; one launch per decode step, no workspace.
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
constexpr int kUnit = 128;     // tokens per K-side unit (16 octets, 2 KB of codes)
constexpr int kVTile = 256;    // tokens per V-side tile (32 octets, 4 KB of codes)
constexpr int kMaxCl = 8;
constexpr int kWMax = (1 << 21) - 1;
constexpr int kLimbRow = 132;  // bytes per limb row (padding spreads the B-fragment loads over banks)
constexpr int kRecv = kG * 136;  // >= kG * cl * ceil(kD / cl) for every cl <= 8
constexpr int kPartStride = kD + 8;  // floats per (warp pair, head) row of the partial sums
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kKBoxRows = 128;      // octet rows per K tensor-copy box (8 units, 16 KB)
constexpr int kMaxKBoxes = 4;       // 4096-token slices
constexpr int kVBoxLines = 256;     // 128-byte V lines per tensor-copy box (8 tiles, 32 KB)

struct Fixed {
  // raw rows (dtype T) staged first: q of the 4 heads, alpha_K, s_K, alpha_V, s_V
  alignas(16) uint8_t stage[8 * kD * 4];
  uint64_t bar_rows, bar_v, bar_k[kMaxKBoxes];  // copy completion, one phase per launch
  int err;                                      // a bounded wait ran out
  uint8_t limb[kG * 3][kLimbRow];  // K-side weight limbs: row 3 h + l, byte = channel
  float red[kWarps][kG][2];        // per-warp reduction scratch
  float mM[kMaxCl][kG][2];         // every peer's logit range per head (pushed to all)
  float part_l[kMaxCl][kG];        // every peer's sum of weights (pushed to all)
  float lsum[kWarps][kG];          // per-warp sum of weights
  float c0[kG], kscale[kG], alog2[kG], ref[kG];
  float cst[kG];                    // g(x) - slope x: the calibration's constant term
  float recv[kRecv];               // [src][h][channel - first owned channel], stride ceil(kD / cl)
};

// Shared memory for a slice of S tokens: K codes / logits / weight fragments
// (S/8 x 128 B) | V codes / partial sums (S/256 x 4 KB) | fixed part.
__host__ __device__ constexpr size_t smem_bytes(int slice) {
  return (size_t)slice / 8 * 128 + (size_t)slice / kVTile * 4096 + sizeof(Fixed);
}

// kmap: K codes as [rows][octets][128 B]; vmap: V codes as [rows][tiles * 32][128 B]
// (a 128-byte line holds 4 channels' 32 bytes of a tile). Both use the 128-byte
// swizzle: 16-byte chunk c of line l lands at chunk c ^ (l & 7), which keeps
// every ldmatrix phase on 32 distinct banks.
template <typename T, int S>
__global__ void __launch_bounds__(kThreads, S == 2048 ? 3 : 1)
    k_decode_mma(const __grid_constant__ DecodeArgs a, int cl, const __grid_constant__ CUtensorMap kmap,
                 const __grid_constant__ CUtensorMap vmap) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // the 128-byte swizzle of the K copies repeats every 1024 bytes: align to it
  uint8_t* sK = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);                      // [S/8][128] codes, 16-byte chunks swizzled by octet
  uint8_t* sV = sK + (size_t)S / 8 * 128;      // [S/256 tiles][32 lines][128 B] codes, swizzled
  Fixed& F = *reinterpret_cast<Fixed*>(sV + (size_t)S / kVTile * 4096);
  float* sL = reinterpret_cast<float*>(sK);    // logits, unit u at floats [512 u, 512 u + 512)
  uint8_t* sFrag = sK;                         // weight-limb A fragments, tile lt at bytes [4096 lt, ...)
  float* sPart = reinterpret_cast<float*>(sV);  // per warp-pair partial sums (after the V side)

  // warp index broadcast from lane 0: known warp-uniform, so shuffles under branches and
  // loops on it need no reconvergence
  const int t = threadIdx.x, warp = __shfl_sync(0xffffffffu, t >> 5, 0), lane = t & 31, g = lane >> 2, tq = lane & 3;
  const uint32_t rank = tc::cluster_rank();
  const int row = blockIdx.x / cl;
  const int b = row / a.Hkv, hkv = row % a.Hkv;
  const int n = a.n;
  const int nvt = (n + kVTile - 1) / kVTile;
  const int vt0 = (int)((rank * nvt) / cl), vt1 = (int)(((rank + 1) * nvt) / cl);
  const int t0 = vt0 * kVTile, t1 = min(n, vt1 * kVTile);
  const int nvtl = vt1 - vt0;                        // V tiles of this CTA
  const int nunits = (t1 - t0 + kUnit - 1) / kUnit;  // K units of this CTA
  const uint32_t sK_u = tc::smem_u32(sK), sV_u = tc::smem_u32(sV);

  // ---- 1. one thread streams the query and statistics rows, then this slice's
  // codes into shared memory with bulk / tensor copies (no per-thread copy
  // instructions stand in the way of the other warps' shared-memory traffic)
  const int nkbox = (nunits * 16 + kKBoxRows - 1) / kKBoxRows;  // K boxes of 8 units
  volatile int* err = &F.err;
  if (t == 0) {
    F.err = 0;
    tc::mbar_init(&F.bar_rows, 1);
    tc::mbar_init(&F.bar_v, 1);
    for (int i = 0; i < kMaxKBoxes; ++i) tc::mbar_init(&F.bar_k[i], 1);
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
    for (int i = 0; i < nkbox; ++i) {  // octet rows past the row's end arrive as zeros
      tc::mbar_arrive_expect_tx(&F.bar_k[i], kKBoxRows * 128);
      tc::tma_load_3d(sK + (size_t)i * kKBoxRows * 128, &kmap, 0, t0 / 8 + i * kKBoxRows, row, &F.bar_k[i]);
    }
    const int nvbox = (nvtl * 32 + kVBoxLines - 1) / kVBoxLines;  // lines past the row's end arrive as zeros
    tc::mbar_arrive_expect_tx(&F.bar_v, (uint32_t)nvbox * kVBoxLines * 128);
    for (int i = 0; i < nvbox; ++i)
      tc::tma_load_3d(sV + (size_t)i * kVBoxLines * 128, &vmap, 0, vt0 * 32 + i * kVBoxLines, row, &F.bar_v);
  }
  tc::cluster_arrive_relaxed();  // matched by the wait before the first peer store
  __syncthreads();               // barrier initialisation is visible

  // ---- 2. post-scaled K weights w_h = sigma q_h (.) s_K in 22-bit fixed point
  const T* sRows = reinterpret_cast<const T*>(F.stage);  // q[4][kD], alpha_K, s_K, alpha_V, s_V
  wait_copies(&F.bar_rows, 0, err, a.wait_probes);
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

  // ---- 3. K side: warp w takes units w, w + 8, ... (unit w + 8 i is in copy box i);
  // per unit 16 octets x 128 channels
  float mn = FLT_MAX, mx = -FLT_MAX;  // logit range of head tq over this lane's tokens
  for (int u = warp; u < nunits; u += kWarps) {
    wait_copies(&F.bar_k[u / kWarps], 0, err, a.wait_probes);
    uint32_t af[4][4];  // A fragments of chunks c = 0..3 (rows = octets 16u + {g, g+8})
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int m = lane >> 3, r8 = 8 * (m & 1) + (lane & 7), c16 = 2 * c + (m >> 1);
      ldsm_x4(sK_u + u * 2048 + r8 * 128 + ((c16 ^ (lane & 7)) << 4), af[c]);
    }
    float* lg = sL + u * 512;  // this unit's logits overwrite its codes (held in af)
    const int tok = t0 + kUnit * u + 8 * g;  // token of octet row g, bit 0
#pragma unroll
    for (int k = 0; k < 8; k += 2) {
      int d[2][2][4];  // [bit k + kk][tile][reg]
#pragma unroll
      for (int kk = 0; kk < 2; ++kk)
#pragma unroll
        for (int tl = 0; tl < 2; ++tl) d[kk][tl][0] = d[kk][tl][1] = d[kk][tl][2] = d[kk][tl][3] = 0;
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
          const uint32_t msk = 0x01010101u << (k + kk);
          const uint32_t am[4] = {af[c][0] & msk, af[c][1] & msk, af[c][2] & msk, af[c][3] & msk};
          mma_u8s8(d[kk][0], am, bk[c][0][0], bk[c][0][1]);
          mma_u8s8(d[kk][1], am, bk[c][1][0], bk[c][1][1]);
        }
      // d[kk][0] = (row g | g+8, cols 2tq, 2tq+1) = head tq limbs 0, 1; d[kk][1] col 2tq = head tq limb 2
#pragma unroll
      for (int kk = 0; kk < 2; ++kk) {
        const float sc = kscale * __int_as_float((127 - k - kk) << 23);  // step * 2^-k
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int d01 = d[kk][0][2 * r] + (d[kk][0][2 * r + 1] << 7);  // |d01| < 2^29
          const float v = fmaf(16384.f, (float)d[kk][1][2 * r], (float)d01);
          const float x = fmaf(v, sc, c0);
          if (tok + 64 * r + k + kk < t1) {
            mn = fminf(mn, x);
            mx = fmaxf(mx, x);
          }
          lg[logit_pos(u, k + kk, tq, g + 8 * r)] = x;
        }
      }
    }
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

  // ---- 5. softmax weights P = p_i 2^(31-k) as four uint8 limbs in the A-fragment
  // order of the V side, over the logits. Thread (k = warp, h, grp) takes the
  // tokens 8 (4 grp + j) + k, j = 0..3, of every V tile; A row m = 4 limb + h,
  // A column = octet within the tile. A tile's logits are all read (group of
  // up to 8 tiles, then a barrier) before its fragments are written.
  float lsum = 0.f;
  {
    const int k = warp, h = (lane >> 3) & 3, grp = lane & 7;
    const float alog2 = F.alog2[h], bias = (float)(31 - k) - F.ref[h];
    const float unscale = __int_as_float((127 - 31 + k) << 23);  // 2^(k-31)
    // octets 4 grp .. 4 grp + 3 of tile lt: unit 2 lt + grp / 4, octets 4 (grp % 4) ..
    const float* src = sL + (grp >> 2) * 512 + logit_pos(grp >> 2, k, h, 4 * (grp & 3));
    // lane 4 h + grp % 4 holds A rows h (limb 0) and h + 8 (limb 2); lane + 16 rows h + 4, h + 12
    uint8_t* dst = sFrag + (size_t)(k * 32 + 4 * h + (grp & 3)) * 16 + (grp >> 2) * 8;
#pragma unroll 1
    for (int lt0 = 0; lt0 < nvtl; lt0 += 8) {
      float4 xv[8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (lt0 + i < nvtl) xv[i] = *reinterpret_cast<const float4*>(src + (lt0 + i) * 1024);
      __syncthreads();
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int lt = lt0 + i;
        if (lt >= nvtl) break;
        const float xs[4] = {xv[i].x, xv[i].y, xv[i].z, xv[i].w};
        const int i0 = t0 + lt * kVTile + 32 * grp + k;  // token of j = 0
        uint32_t P[4];
        if (t0 + (lt + 1) * kVTile <= t1) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float p = ex2_approx(fmaf(xs[j], alog2, bias));
            P[j] = __float2uint_rn(p);
            lsum += p;
          }
        } else {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const bool ok = i0 + 8 * j < t1;
            const float p = ex2_approx(fmaf(xs[j], alog2, bias));
            P[j] = ok ? __float2uint_rn(p) : 0u;
            lsum += ok ? p : 0.f;
          }
        }
        // word l = byte l of P[0..3]
        const uint32_t lo01 = __byte_perm(P[0], P[1], 0x5140), hi01 = __byte_perm(P[0], P[1], 0x7362);
        const uint32_t lo23 = __byte_perm(P[2], P[3], 0x5140), hi23 = __byte_perm(P[2], P[3], 0x7362);
        const uint32_t w0 = __byte_perm(lo01, lo23, 0x5410), w1 = __byte_perm(lo01, lo23, 0x7632);
        const uint32_t w2 = __byte_perm(hi01, hi23, 0x5410), w3 = __byte_perm(hi01, hi23, 0x7632);
        *reinterpret_cast<uint2*>(dst + (size_t)lt * 4096) = make_uint2(w0, w2);
        *reinterpret_cast<uint2*>(dst + (size_t)lt * 4096 + 256) = make_uint2(w1, w3);
      }
    }
    lsum *= unscale;
    // lanes with equal h: xor over grp
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 1);
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 2);
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 4);
    if (grp == 0) F.lsum[warp][h] = lsum;
  }
  wait_copies(&F.bar_v, 0, err, a.wait_probes);
  __syncthreads();  // the weight fragments are complete

  // ---- 6. V side: warp pair p = warp / 2 takes tiles p, p + 4, ...; warp parity
  // picks channels 64 hc .. 64 hc + 63. D rows (limb, head), columns channels.
  const int hc = warp & 1, pair = warp >> 1;
  int acc[8][4];
#pragma unroll
  for (int j = 0; j < 8; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0;
  for (int lt = pair; lt < nvtl; lt += kWarps / 2) {
    const uint32_t tile_u = sV_u + lt * 4096, frag_u = sK_u + lt * 4096 + lane * 16;
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
    for (int k = 0; k < 8; ++k) {
      uint32_t af[4];
      lds128(frag_u + k * 512, af);
      const uint32_t msk = 0x01010101u << k;
#pragma unroll
      for (int j = 0; j < 8; ++j) mma_u8u8(acc[j], af, bv[j][0] & msk, bv[j][1] & msk);
    }
  }

  // ---- 7. combine limbs (lane and lane ^ 16), sum the warp pairs, scatter to the owners
  // Lane with g < 4 holds limbs 0 and 2 of head g, lane + 16 limbs 1 and 3.
  __syncthreads();  // every warp is done with the V codes: the partial sums reuse them
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
    tc::mbar_wait(&F.bar_v, 0, kSpin);
    for (int i = 0; i < nkbox; ++i) tc::mbar_wait(&F.bar_k[i], 0, kSpin);
  }
}

template <typename T, int S>
cudaError_t run_slice(const DecodeArgs& a, int rows, int cl, cudaStream_t stream) {
  const size_t smem = smem_bytes(S) + 1024;  // slack to align the codes to the 1024-byte swizzle atom
  static bool attr_sets[kMaxDevices];  // per device (benign race: every caller sets the same value)
  const int attr_dev = current_device();
  if (attr_dev < 0) return cudaErrorInvalidDevice;
  bool& attr_set = attr_sets[attr_dev];
  if (!attr_set) {
    const cudaError_t e =
        cudaFuncSetAttribute(k_decode_mma<T, S>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int octets = (a.n + 7) / 8, nvt = (a.n + kVTile - 1) / kVTile;
  CUtensorMap kmap, vmap;
  if (!encode_3d(&kmap, a.k_codes, kD, (uint64_t)octets, (uint64_t)rows, kKBoxRows, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_3d(&vmap, a.v_codes, 128, (uint64_t)nvt * 32, (uint64_t)rows, kVBoxLines, CU_TENSOR_MAP_SWIZZLE_128B))
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
  return cudaLaunchKernelEx(&cfg, k_decode_mma<T, S>, a, cl, kmap, vmap);
}

template <typename T>
cudaError_t run(const DecodeArgs& a, cudaStream_t stream) {
  const int rows = a.B * a.Hkv;
  const int nvt = (a.n + kVTile - 1) / kVTile;
  const bool small = nvt <= kMaxCl * (2048 / kVTile);  // n <= 16384: 3 CTAs per SM
  const int per = (small ? 2048 : 4096) / kVTile;
  const int cl = (nvt + per - 1) / per;
  if (cl > kMaxCl || (long long)rows * cl > 0x7fffffffLL) return cudaErrorNotSupported;
  return small ? run_slice<T, 2048>(a, rows, cl, stream) : run_slice<T, 4096>(a, rows, cl, stream);
}

}  // namespace

bool decode_mma_supports(int n) { return n >= 1 && n <= kMaxCl * 4096; }

cudaError_t launch_decode_mma(const DecodeArgs& a, cq_dtype dt, cudaStream_t stream) {
  if (!decode_mma_supports(a.n)) return cudaErrorNotSupported;
  if (dt == CQ_F16) return run<half>(a, stream);
  return run<float>(a, stream);
}

}  // namespace cq
