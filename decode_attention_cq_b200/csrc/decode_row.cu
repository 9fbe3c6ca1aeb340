// Fused 1-bit decode attention, one CTA per (batch, kv-head) row, logits held
// in tensor memory; register-fed tensor-core MMAs (mma.sync m16n8k32, 8-bit
// operands, s32 accumulators) over the octet code layouts.
//
// Method (CalibQuant article): logits x_i = sigma q.alpha_K + (sigma q (.) s_K)
// . c^K_i on the integer codes (Method 2, post-scaling), calibration map g on
// the row's score range (Method 3), softmax, o = alpha_V + s_V (.)
// sum_i p_i c^V_i / sum_i p_i (Method 2 applied to V).
//
// Why one CTA per row: the calibration slope needs the range of ALL logits of
// the row before any softmax weight exists. Splitting a row over a cluster
// makes every slice wait twice on its peers (range, then partial sums); here
// the range is a barrier inside the CTA. The row's logits (n x 4 heads x 4 B,
// 128 KB at n = 8192) do not fit next to a code ring in shared memory for two
// CTAs per SM, so they live in tensor memory (256 columns per CTA, two CTAs
// per SM), written and read back by the thread that owns them.
//
// Tiles of 256 tokens (32 octets), 8 warps, two CTAs per SM:
//  1. one thread copies the q / alpha / s rows and the first chunks of codes
//     while warp 0 allocates tensor memory;
//     the K codes and after them the V codes stream through a ring of 16 KB
//     slots (4 tiles each; tensor copies with the 128-byte swizzle, completing
//     on a full mbarrier per slot, every wait bounded). A shared counter per
//     slot collects the warps' releases, and the warp whose release empties
//     the slot issues the copy that reuses it: no thread waits for a slot;
//  2. the weights w_h = sigma q_h (.) s_K become 22-bit fixed point in three
//     int8 limbs, held as the A operand: rows 4 l + h (limb l, head h);
//  3. K side: warp w takes tiles w, w + 8, ...; B = the codes of 8 octets x 32
//     channels, masked to bit k (one octet byte holds 8 tokens of a channel;
//     masking bit k leaves "code of token 8 o + k times 2^k"). The octet each
//     B column stands for is chosen so that the thread holding D rows g, g + 8
//     and columns 2 tq, 2 tq + 1 of the four N = 8 tiles ends up with head
//     g % 4 of octets 4 tq + i and 16 + 4 tq + i (i = 0..3): exactly the
//     tokens whose softmax weights it needs for the V side's A fragment. Bits
//     are taken in pairs (k, k + 1); after one exchange between lanes l and
//     l ^ 16 (the lanes holding limbs 0, 2 and limb 1 of one head), lane l < 16
//     owns bit k and lane l + 16 bit k + 1. Each lane stores its 8 logits per
//     bit pair in its own tensor-memory lane;
//  4. the row range per head (warp shuffles + one CTA barrier) gives the
//     calibration slope;
//  5. each lane turns its 32 logit columns of a tile, in place, into its A-fragment
//     words of the tile's 8 bit positions for the V side: P = p 2^(31-k) for its
//     own bit of every pair, a swap with lane ^ 16, byte permutes into limb rows
//     (rows 4 limb + head, columns octets); each warp of a pair forms half of
//     the bit positions of the pair's next tile while it issues the current
//     tile's V MMAs, and a 64-thread barrier per tile hands the halves over;
//  6. V side: warp pair (q, q + 4) (the two warps sharing a tensor-memory lane
//     quarter) takes tiles q, q + 4, ... and splits the 128 channels; A = the
//     tile's fragments loaded from tensor memory, B = V codes of 8 channels
//     masked to bit k. Sum_l 2^(8l-31) D_l = sum c p;
//  7. the four warp pairs' sums meet in shared memory; o = alpha_V + s_V (.)
//     sum c p / sum p; with text tokens (a mixed cache) the warps first attend
//     them (f16: through the ring and the tensor cores) and the output merges
//     both parts by their log-sum-exps.
// No workspace; n <= 8192 tokens per row. One launch per decode step, plus,
// past two full waves of rows, a second one that splits the rows beyond a
// whole number of SM counts over 2-CTA clusters (decode_row_split_rows).
#include <float.h>

#include <type_traits>

#include "common.cuh"
#include "kernels.h"
#include "mma_util.cuh"
#include "tc.cuh"
#include "text_attend.cuh"

namespace cq {

namespace {

using namespace mu;

constexpr int kThreads = 256;  // 8 warps
constexpr int kTile = 256;              // tokens per tile (32 octets, 4 KB of codes per side)
constexpr int kChunkTiles = 4;          // tiles per ring slot
constexpr int kChunkBytes = kChunkTiles * 4096;
constexpr int kSlots = 4;
// The ring's waits are parity waits, so a warp may wait on a slot's next use
// only once the slot's previous use has landed. Each warp group reuses only
// the slots of chunks it consumes itself: K chunks alternate between warps
// 0-3 and 4-7 (slots of one parity each), every warp reads every V chunk (and
// a CTA barrier separates the two sides), and the two groups take alternate
// text chunk pairs (two slots each). That needs kSlots to be a multiple of 4.
static_assert(kSlots % 4 == 0, "warp groups must own their ring slots");
constexpr int kMaxTiles = 32;  // n <= 8192: 8 tiles per tensor-memory lane quarter, 256 columns
constexpr int kWMax = (1 << 21) - 1;
constexpr int kLimbRow = 132;  // bytes per limb row (padding spreads the fragment loads over banks)
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kTextTile = txt::kChunkTokens;  // text tokens per ring chunk (f16: 64 x 256 B keys or values)
static_assert(txt::kChunkBytes == 4 * 4096, "a text chunk fills one ring slot");
constexpr int kMinSmem = 80 * 1024;  // > 228 KB / 3: at most two CTAs (2 x 256 columns) per SM

struct RowFixed {
  alignas(16) uint8_t stage[8 * kD * 4];  // q of the 4 heads, alpha_K, s_K, alpha_V, s_V (dtype T)
  uint64_t full[kSlots], bar_rows;
  uint32_t released[kSlots];  // warp releases of each slot so far (8 per use)
  uint32_t uses[kSlots];      // copies issued into each slot so far
  int err;                    // a bounded wait ran out
  uint32_t tmem_base;  // written by tcgen05.alloc
  uint8_t limb[kG * 3][kLimbRow];  // weight limbs: row 3 h + l, byte = channel
  float red[8][kG][2];             // per-warp reduction scratch
  float lsum[8][kG];               // per warp: sum of its softmax weights
  float c0[kG], kscale[kG], alog2[kG], ref[kG], cst[kG];
  alignas(16) float part[4][kG][kD];  // per warp pair: sum_i c_ij p_i
  // a row split over a 2-CTA cluster: what the peer pushed
  float xm[2][kG][2];   // [rank][head]: (min, max) of the rank's logits
  float xpart[kG][kD];  // rank 1's sum_i c_ij p_i (at rank 0)
  float xl[kG];         // rank 1's sum_i p_i (at rank 0)
  float xerr;           // rank 1's error flag (at rank 0)
};

__host__ __device__ constexpr size_t row_smem_bytes() {
  return (size_t)kSlots * kChunkBytes + sizeof(RowFixed) + 1024;  // + alignment to the swizzle atom
}


// Byte l of each of p0..p3 -> one word (column order), and byte l + 2 -> another.
__device__ __forceinline__ void gather_limbs(uint32_t p0, uint32_t p1, uint32_t p2, uint32_t p3, uint32_t sel,
                                             uint32_t& lo, uint32_t& hi) {
  const uint32_t t01 = __byte_perm(p0, p1, sel), t23 = __byte_perm(p2, p3, sel);
  lo = __byte_perm(t01, t23, 0x5410);
  hi = __byte_perm(t01, t23, 0x7632);
}

// Octet (0..31 within a tile) of a lane's value i (0..7): 4 tq + i, then 16 + 4 tq + i - 4.
__device__ __forceinline__ int lane_octet(int tq, int i) { return (i < 4) ? 4 * tq + i : 12 + 4 * tq + i; }

// What the ring streams for one row: the K codes, the V codes (nchunk chunks
// each), then, for a mixed cache in f16, the keys and the values of the text
// tokens (one chunk each per 64 tokens).
struct Ring {
  const CUtensorMap* kmap;
  const CUtensorMap* vmap;
  const CUtensorMap* ktmap;
  const CUtensorMap* vtmap;
  int row, tile0, nchunk, nall;  // tile0: first tile of the row this CTA takes
};

// Chunk gi (0 .. nall - 1) lands in slot gi % kSlots: the K codes of tiles
// tile0 + 4 gi .. + 3, then (gi >= nchunk) the V codes of tiles tile0 + 4 (gi - nchunk) ..,
// then (gi >= 2 nchunk) alternately the keys and the values of 64 text tokens
// as two boxes of 64 channels (8 KB each). Tiles and tokens past the row's end
// arrive as zeros (tensor-copy bounds fill).
__device__ __forceinline__ void issue_chunk(RowFixed& F, uint8_t* ring, const Ring& R, int gi) {
  const int s = gi % kSlots;
  atomicAdd(&F.uses[s], 1u);
  tc::mbar_arrive_expect_tx(&F.full[s], kChunkBytes);
  uint8_t* dst = ring + (size_t)s * kChunkBytes;
  if (gi < R.nchunk) {
    tc::tma_load_3d(dst, R.kmap, 0, (R.tile0 + gi * kChunkTiles) * 32, R.row, &F.full[s]);
  } else if (gi < 2 * R.nchunk) {
    tc::tma_load_3d(dst, R.vmap, 0, (R.tile0 + (gi - R.nchunk) * kChunkTiles) * 32, R.row, &F.full[s]);
  } else {
    const int tt = gi - 2 * R.nchunk;
    const CUtensorMap* m = (tt & 1) ? R.vtmap : R.ktmap;
    tc::tma_load_3d(dst, m, 0, (tt >> 1) * kTextTile, R.row, &F.full[s]);
    tc::tma_load_3d(dst + kChunkBytes / 2, m, 128, (tt >> 1) * kTextTile, R.row, &F.full[s]);
  }
}

// A warp is done reading chunk gi (its share of the slot's 8 releases is
// `share`); the warp that completes the slot's releases issues the chunk that
// reuses it, so no thread ever waits for a slot to drain.
__device__ __forceinline__ void release_chunk(RowFixed& F, uint8_t* ring, const Ring& R, int gi, uint32_t share) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) {
    const int s = gi % kSlots;
    __threadfence_block();  // this warp's reads of the slot come before the release
    const uint32_t done = atomicAdd(&F.released[s], share) + share;
    if (done == 8u * (uint32_t)(gi / kSlots + 1) && gi + kSlots < R.nall) {
      __threadfence_block();
      tc::fence_proxy_async();
      issue_chunk(F, ring, R, gi + kSlots);
    }
  }
}

// The ring's text chunks as txt::text_mma consumes them: chunk gi's slot
// once its copy has landed, and the warp's release of it (four warps per
// text chunk).
struct RowTextChunks {
  RowFixed& F;
  uint8_t* ring;
  uint32_t ring_u;
  const Ring& R;
  volatile int* err;
  __device__ __forceinline__ uint32_t wait(int gi) {
    warp_wait_copies(&F.full[gi % kSlots], (uint32_t)(gi / kSlots) & 1u, err);
    return ring_u + (uint32_t)((gi % kSlots) * kChunkBytes);
  }
  __device__ __forceinline__ void release(int gi) { release_chunk(F, ring, R, gi, 2); }
};

// kmap: K codes as [rows][octets][128 B]; vmap: V codes as [rows][tiles * 32][128 B]
// (a 128-byte line holds 4 channels' 32 bytes of a tile). Both with the
// 128-byte swizzle: 16-byte chunk c of line l lands at chunk c ^ (l & 7).
// kSplit: each row is split over a cluster of two CTAs (rank r takes tiles
// r * ceil(nt / 2) ..); the ranks exchange the logit range and rank 1 hands its
// partial sums to rank 0, which writes the row. Plain decodes only (no text
// tokens, no partial mode). Rows row0 .. of this launch.
template <typename T, bool kSplit>
__global__ void __launch_bounds__(kThreads, 2)
    k_decode_row(const __grid_constant__ DecodeArgs a, uint32_t tmem_cols, int row0,
                 const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                 const __grid_constant__ CUtensorMap ktmap, const __grid_constant__ CUtensorMap vtmap) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* ring = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
  RowFixed& F = *reinterpret_cast<RowFixed*>(ring + (size_t)kSlots * kChunkBytes);
  const uint32_t ring_u = tc::smem_u32(ring);

  // the warp index broadcast from lane 0 is known to be warp-uniform, so branches
  // and loops on it keep the warp converged: shuffles inside them stay cheap
  const int t = threadIdx.x, warp = __shfl_sync(0xffffffffu, t >> 5, 0), lane = t & 31, g = lane >> 2, tq = lane & 3;
  const int rank = kSplit ? (int)tc::cluster_rank() : 0;
  const int row = row0 + (kSplit ? (int)blockIdx.x / 2 : (int)blockIdx.x), b = row / a.Hkv, hkv = row % a.Hkv;
  const int n = a.n;
  const int nt = (n + kTile - 1) / kTile;                     // tiles of the row
  const int nt_first = kSplit ? (nt + 1) / 2 : nt;             // tiles of rank 0
  const int tile0 = rank == 0 ? 0 : nt_first;                  // this CTA's first tile
  const int ntl = rank == 0 ? nt_first : nt - nt_first;        // this CTA's tiles
  const int nchunk = (ntl + kChunkTiles - 1) / kChunkTiles;    // ring chunks per side
  // f16 text tokens of a mixed cache stream through the ring after the V codes
  // and meet the tensor cores; f32 ones are read directly by the warps
  constexpr bool kTextMma = std::is_same<T, half>::value;
  const int ntp = kTextMma ? (a.n_text + kTextTile - 1) / kTextTile : 0;  // text key / value chunk pairs
  const Ring R{&kmap, &vmap, &ktmap, &vtmap, row, tile0, nchunk, 2 * nchunk + 2 * ntp};
  volatile int* err = &F.err;
  if constexpr (kSplit) tc::cluster_arrive_relaxed();  // matched by the wait before the first peer store
  // a launch of split rows that follows this one on the stream may start now
  if constexpr (!kSplit) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // ---- 1. barriers, tensor memory, the query and statistics rows, the first
  // chunks: warp 1 sets up and issues the copies while warp 0 allocates
  if (t == 32) {
    F.err = 0;
    for (int s = 0; s < kSlots; ++s) {
      tc::mbar_init(&F.full[s], 1);
      F.released[s] = 0;
      F.uses[s] = 0;
    }
    tc::mbar_init(&F.bar_rows, 1);
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
    for (int gi = 0; gi < kSlots && gi < R.nall; ++gi) issue_chunk(F, ring, R, gi);
  }
  if (warp == 0) {
    tc::tmem_alloc(&F.tmem_base, tmem_cols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = F.tmem_base;

  {
    // ---- 2. post-scaled K weights w_h = sigma q_h (.) s_K in 22-bit fixed point
    const T* sRows = reinterpret_cast<const T*>(F.stage);  // q[4][kD], alpha_K, s_K, alpha_V, s_V
    warp_wait_copies(&F.bar_rows, 0, err);
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
        const float ks = amax * (1.f / (float)kWMax);  // any scale works: w is rounded with this one
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

    // A fragments of the K side, per 32-channel chunk c: row g = (limb g / 4,
    // head g % 4), row g + 8 = (limb 2, head g) for g < 4, zero for g >= 4.
    const bool lo = lane < 16;  // lo lanes hold limbs 0 and 2 of head g, hi lanes limb 1 of head g - 4
    const int h = g & 3;        // the head of every value this lane holds
    uint32_t wa[4][4];
    {
      const uint8_t* r0 = F.limb[3 * h + (g >> 2)];
      const uint8_t* r1 = F.limb[3 * h + 2];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int j = 32 * c + 4 * tq;
        wa[c][0] = *reinterpret_cast<const uint32_t*>(r0 + j);
        wa[c][1] = lo ? *reinterpret_cast<const uint32_t*>(r1 + j) : 0u;
        wa[c][2] = *reinterpret_cast<const uint32_t*>(r0 + j + 16);
        wa[c][3] = lo ? *reinterpret_cast<const uint32_t*>(r1 + j + 16) : 0u;
      }
    }
    const float c0 = F.c0[h], kscale = F.kscale[h];
    const uint32_t tlane = tmem + ((uint32_t)(32 * (warp & 3)) << 16);  // this warp's lane quarter

    // ---- 3. K side: chunk c's tile 4 c + (warp & 3) belongs to warp (4 c + (warp & 3)) % 8
    float mn = FLT_MAX, mx = -FLT_MAX;  // logit range of head h over this lane's tokens
    // Every warp runs every pass (a shuffle inside a loop whose trip count the
    // compiler sees as per-thread costs several times its latency); a pass
    // without a tile computes on zero codes and stores nothing.
    for (int pass = 0; pass < nchunk; pass += 2) {
      const int c = pass + (warp >> 2), s = c % kSlots, j = kChunkTiles * c + (warp & 3);
      const bool act = c < nchunk, have = act && j < ntl;
      if (act) warp_wait_copies(&F.full[s], (uint32_t)(c / kSlots) & 1u, err);
      uint32_t bk[4][4][2];  // [32-channel chunk][N tile][reg]
      if (have) {
        // lane provides row (lane & 7) of matrix lane >> 3; matrix (N tile 2x + m / 2, half m % 2)
        const uint32_t tile_u = ring_u + (uint32_t)(s * kChunkBytes + (warp & 3) * 4096);
        const int m = lane >> 3, r = lane & 7;
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          const int jn = 2 * x + (m >> 1);
          const int oct = 2 * jn + 12 * (jn >> 1) + 4 * (r >> 1) + (r & 1);  // octet of B column r
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            uint32_t rr[4];
            ldsm_x4(tile_u + oct * 128 + (((2 * cc + (m & 1)) ^ (oct & 7)) << 4), rr);
            bk[cc][2 * x][0] = rr[0];
            bk[cc][2 * x][1] = rr[1];
            bk[cc][2 * x + 1][0] = rr[2];
            bk[cc][2 * x + 1][1] = rr[3];
          }
        }
      } else {
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
#pragma unroll
          for (int jn = 0; jn < 4; ++jn) bk[cc][jn][0] = bk[cc][jn][1] = 0u;
      }
      if (act) release_chunk(F, ring, R, c, 2);  // K side: four warps per chunk
      const int jg = tile0 + j;                              // the row's tile index
      const bool ragged = !have || kTile * (jg + 1) > n;    // some token of the tile is not this CTA's
      const uint32_t col0 = tlane + (uint32_t)(32 * (j >> 2));
#pragma unroll
      for (int kp = 0; kp < 4; ++kp) {
        int d[2][4][4];  // [bit 2 kp + kk][N tile][reg]
#pragma unroll
        for (int kk = 0; kk < 2; ++kk)
#pragma unroll
          for (int jn = 0; jn < 4; ++jn) d[kk][jn][0] = d[kk][jn][1] = d[kk][jn][2] = d[kk][jn][3] = 0;
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
          const uint32_t msk = 0x01010101u << (2 * kp + kk);
#pragma unroll
          for (int cc = 0; cc < 4; ++cc)
#pragma unroll
            for (int jn = 0; jn < 4; ++jn) mma_s8u8(d[kk][jn], wa[cc], bk[cc][jn][0] & msk, bk[cc][jn][1] & msk);
        }
        // lo lanes finish bit 2 kp, hi lanes bit 2 kp + 1: x = D0 + 2^7 D1 + 2^14 D2
        const int kown = 2 * kp + (lo ? 0 : 1);
        const float sc = kscale * __int_as_float((127 - kown) << 23);  // step * 2^-k
        uint32_t out[8];
#pragma unroll
        for (int jn = 0; jn < 4; ++jn)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int i = 2 * jn + e;
            const int send =
                lo ? __float_as_int(fmaf(16384.f, (float)d[1][jn][2 + e], (float)d[1][jn][e])) : d[0][jn][e];
            const int recv = __shfl_xor_sync(0xffffffffu, send, 16);
            float x;
            if (lo) {
              const int d01 = d[0][jn][e] + (recv << 7);  // |d01| < 2^29
              x = fmaf(16384.f, (float)d[0][jn][2 + e], (float)d01);
            } else {
              x = fmaf(128.f, (float)d[1][jn][e], __int_as_float(recv));
            }
            const float xl = fmaf(x, sc, c0);
            if (!ragged || (have && kTile * jg + 8 * lane_octet(tq, i) + kown < n)) {
              mn = fminf(mn, xl);
              mx = fmaxf(mx, xl);
            }
            out[i] = __float_as_uint(xl);
          }
        if (have) tc::st_x8(col0 + 8 * kp, out);
      }
    }
    tc::wait_st();

    // ---- 4. logit range of the row, calibration slope
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, 1));
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, 2));
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, 16));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
    if (lo && tq == 0) {
      F.red[warp][g][0] = mn;
      F.red[warp][g][1] = mx;
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if constexpr (kSplit) {
      // this CTA's range into F.xm[rank] of both CTAs; the cluster barrier publishes it
      tc::cluster_wait();  // (arrived at the start) the peer is running: its shared memory exists
      if (t < kG) {
        float m = FLT_MAX, M = -FLT_MAX;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          m = fminf(m, F.red[q][t][0]);
          M = fmaxf(M, F.red[q][t][1]);
        }
        F.xm[rank][t][0] = m;
        F.xm[rank][t][1] = M;
        tc::st_peer_f32(&F.xm[rank][t][0], (uint32_t)(rank ^ 1), m);
        tc::st_peer_f32(&F.xm[rank][t][1], (uint32_t)(rank ^ 1), M);
      }
      tc::cluster_sync();
    }
    if (t < kG) {
      float m = FLT_MAX, M = -FLT_MAX;
      if constexpr (kSplit) {
        m = fminf(F.xm[0][t][0], F.xm[1][t][0]);
        M = fmaxf(F.xm[0][t][1], F.xm[1][t][1]);
      } else {
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          m = fminf(m, F.red[q][t][0]);
          M = fmaxf(M, F.red[q][t][1]);
        }
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

    // ---- 5./6. softmax weights and the V side, interleaved. A lane's 32 logit
    // columns of a tile become, in place, its A-fragment words of the tile's 8
    // bit positions (column 4 k + r = register r of bit k): P = p 2^(31-k) for its
    // own bit of every pair, a swap with lane ^ 16 (the lane holding the same
    // head's other limbs), byte permutes into limb rows. Warp pair (q, q + 4)
    // (the two warps sharing a tensor-memory lane quarter) takes tiles q, q + 4,
    // ...; warp q + 4 hc forms bit positions 4 hc .. 4 hc + 3 of the pair's next
    // tile while it issues the MMAs of the current one, and a 64-thread barrier
    // per tile hands the two halves over. On the V side hc picks channels
    // 64 hc .. 64 hc + 63: A = the tile's fragments from tensor memory, B = V codes
    // of 8 channels masked to bit k.
    const int q = warp & 3, hc = warp >> 2;
    float lsum = 0.f;
    const float alog2 = F.alog2[h], ref = F.ref[h];
    const uint32_t sel = lo ? 0x6240u : 0x7351u;  // bytes (limb, limb + 2) of two words: limbs 0, 2 or 1, 3
    // this warp's half of tile 4 c + q's fragments, one bit pair (kp = 2 hc + kp2) at a time
    auto form_half = [&](int c) {
      const int j = kChunkTiles * c + q;
      const bool live = j < ntl;                             // a tile of this CTA
      const int jg = tile0 + j;                              // the row's tile index
      const bool ragged = !live || kTile * (jg + 1) > n;     // some token of the tile is masked
#pragma unroll
      for (int kp2 = 0; kp2 < 2; ++kp2) {
        const int kp = 2 * hc + kp2;
        const uint32_t col = tlane + (uint32_t)(32 * c + 8 * kp);
        uint32_t xs[8], outw[8];
        tc::ld_x8(col, xs);
        tc::wait_ld();
        const int kown = 2 * kp + (lo ? 0 : 1);
        const float bias = (float)(31 - kown) - ref;
        const float unscale = __int_as_float((127 - 31 + kown) << 23);  // 2^(k - 31)
        uint32_t pown[8], poth[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float p = ex2_approx(fmaf(__uint_as_float(xs[i]), alog2, bias));
          const bool ok = !ragged || (live && kTile * jg + 8 * lane_octet(tq, i) + kown < n);
          pown[i] = ok ? __float2uint_rn(p) : 0u;
          lsum = ok ? fmaf(p, unscale, lsum) : lsum;
          poth[i] = __shfl_xor_sync(0xffffffffu, pown[i], 16);
        }
        // bit 2 kp: the lo lanes' weights; bit 2 kp + 1: the hi lanes'
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
          uint32_t P[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) P[i] = ((kk == 0) == lo) ? pown[i] : poth[i];
          gather_limbs(P[0], P[1], P[2], P[3], sel, outw[4 * kk], outw[4 * kk + 1]);
          gather_limbs(P[4], P[5], P[6], P[7], sel, outw[4 * kk + 2], outw[4 * kk + 3]);
        }
        tc::st_x8(col, outw);  // columns 8 kp .. 8 kp + 7 = bits 2 kp, 2 kp + 1
      }
      tc::wait_st();
      tc::fence_before_sync();
      switch (q) {  // barrier 1 + q: warps q and q + 4
        case 0: tc::bar_sync_id<1>(64); break;
        case 1: tc::bar_sync_id<2>(64); break;
        case 2: tc::bar_sync_id<3>(64); break;
        default: tc::bar_sync_id<4>(64); break;
      }
      tc::fence_after_sync();
    };
    form_half(0);

    int acc[8][4];
#pragma unroll
    for (int jn = 0; jn < 8; ++jn) acc[jn][0] = acc[jn][1] = acc[jn][2] = acc[jn][3] = 0;
    for (int c = 0; c < nchunk; ++c) {
      const int gi = nchunk + c, s = gi % kSlots, j = kChunkTiles * c + q;
      warp_wait_copies(&F.full[s], (uint32_t)(gi / kSlots) & 1u, err);
      uint32_t bv[8][2];
      if (j < ntl) {
        const uint32_t tile_u = ring_u + (uint32_t)(s * kChunkBytes + q * 4096);
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
      } else {
#pragma unroll
        for (int jn = 0; jn < 8; ++jn) bv[jn][0] = bv[jn][1] = 0u;
      }
      release_chunk(F, ring, R, gi, 1);  // V side: all eight warps per chunk
      uint32_t fr[32];  // A fragments of the tile's 8 bit positions (zero past the row's end)
      tc::ld_x16(tlane + (uint32_t)(32 * c), *reinterpret_cast<uint32_t(*)[16]>(&fr[0]));
      tc::ld_x16(tlane + (uint32_t)(32 * c + 16), *reinterpret_cast<uint32_t(*)[16]>(&fr[16]));
      tc::wait_ld();
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint32_t af[4] = {fr[4 * k], fr[4 * k + 1], fr[4 * k + 2], fr[4 * k + 3]};
        const uint32_t msk = 0x01010101u << k;
#pragma unroll
        for (int jn = 0; jn < 8; ++jn) mma_u8u8(acc[jn], af, bv[jn][0] & msk, bv[jn][1] & msk);
      }
      if (c + 1 < nchunk) form_half(c + 1);
    }
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 1);
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 2);
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 16);
    if (lo && tq == 0) F.lsum[warp][g] = lsum;

    // ---- 7. limbs combined (lane and lane ^ 16), the pairs summed, o written
    float* part = &F.part[0][0][0];  // [pair][head][channel]
    {
      const float s_lo = lo ? 0x1p-31f : 0x1p-23f, s_hi = lo ? 0x1p-15f : 0x1p-7f;
#pragma unroll
      for (int jn = 0; jn < 8; ++jn) {
        float v[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          v[e] = fmaf((float)acc[jn][e + 2], s_hi, (float)acc[jn][e] * s_lo);
          v[e] += __shfl_xor_sync(0xffffffffu, v[e], 16);
        }
        if (lo)
          *reinterpret_cast<float2*>(part + (q * kG + g) * kD + 64 * hc + 8 * jn + 2 * tq) = make_float2(v[0], v[1]);
      }
    }

    // ---- 8. text tokens of a mixed cache (none in a plain decode): each warp
    // attends its share of the row's full-precision tokens with an online softmax
    // on the raw logits sigma q.k; merged below by log-sum-exp. Once every warp
    // is past the ring's last chunk, the ring holds the warps' parts.
    float* t_acc = reinterpret_cast<float*>(ring);  // [warp][head][channel]
    float* t_ml = t_acc + 8 * kG * kD;              // [warp][head][running maximum, sum of weights]
    if (a.n_text > 0) {
      if constexpr (kTextMma) {
        float tm, tl, o[8][4];
        RowTextChunks chunks{F, ring, ring_u, R, err};
        txt::text_mma(chunks, 2 * nchunk, sRows, ntp, a.n_text, a.sigma, warp, lane, tm, tl, o);
        tl += __shfl_xor_sync(0xffffffffu, tl, 1);
        tl += __shfl_xor_sync(0xffffffffu, tl, 2);
        __syncthreads();  // the ring's text chunks are all read
        if (g < kG && tq == 0) {
          t_ml[(warp * kG + g) * 2] = tm;
          t_ml[(warp * kG + g) * 2 + 1] = tl;
        }
        if (tq < 2) {
          float* h0 = t_acc + (warp * kG + 2 * tq) * kD;  // head 2 tq; head 2 tq + 1 follows
#pragma unroll
          for (int xx = 0; xx < 8; ++xx) {
            h0[16 * xx + g] = o[xx][0];
            h0[kD + 16 * xx + g] = o[xx][1];
            h0[16 * xx + g + 8] = o[xx][2];
            h0[kD + 16 * xx + g + 8] = o[xx][3];
          }
        }
      } else {
        float qv[kG][4];
#pragma unroll
        for (int hh = 0; hh < kG; ++hh)
#pragma unroll
          for (int c = 0; c < 4; ++c) qv[hh][c] = DT<T>::f(sRows[hh * kD + 4 * lane + c]);
        float tm[kG], tl[kG], tacc[kG][4];
        const size_t toff = (size_t)row * a.n_text * kD + 4 * lane;
        txt::warp_text_attend<T, 8>(qv, static_cast<const T*>(a.k_text) + toff,
                                    static_cast<const T*>(a.v_text) + toff, a.n_text, a.sigma, warp, lane, tm, tl,
                                    tacc);
#pragma unroll
        for (int hh = 0; hh < kG; ++hh) {
          if (lane == 0) {
            t_ml[(warp * kG + hh) * 2] = tm[hh];
            t_ml[(warp * kG + hh) * 2 + 1] = tl[hh];
          }
#pragma unroll
          for (int c = 0; c < 4; ++c) t_acc[(warp * kG + hh) * kD + 4 * lane + c] = tacc[hh][c];
        }
      }
    }
    __syncthreads();
    if constexpr (kSplit) {
      // rank 1 hands its sums (and its error flag) to rank 0 and is done
      if (rank == 1) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int idx = 2 * t + e, hh = idx >> 7, ch = idx & 127;
          float sum = 0.f;
#pragma unroll
          for (int p = 0; p < 4; ++p) sum += part[(p * kG + hh) * kD + ch];
          tc::st_peer_f32(&F.xpart[hh][ch], 0u, sum);
        }
        if (t < kG) {
          float l = 0.f;
#pragma unroll
          for (int w8 = 0; w8 < 8; ++w8) l += F.lsum[w8][t];
          tc::st_peer_f32(&F.xl[t], 0u, l);
        }
        if (t == 0) tc::st_peer_f32(&F.xerr, 0u, *err ? 1.f : 0.f);
      }
      tc::cluster_sync();
    }
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      if (kSplit && rank != 0) continue;
      const int idx = 2 * t + e, hh = idx >> 7, ch = idx & 127;
      float sum = 0.f, l = 0.f;
#pragma unroll
      for (int p = 0; p < 4; ++p) sum += part[(p * kG + hh) * kD + ch];
#pragma unroll
      for (int w8 = 0; w8 < 8; ++w8) l += F.lsum[w8][hh];
      if constexpr (kSplit) {
        sum += F.xpart[hh][ch];
        l += F.xl[hh];
      }
      const bool bad = *err || (kSplit && F.xerr != 0.f);
      const float alpha = DT<T>::f(sRows[6 * kD + ch]);
      const float step = bad ? __int_as_float(0x7fc00000) : DT<T>::f(sRows[7 * kD + ch]);
      const size_t bh = (size_t)b * a.Hq + (size_t)kG * hkv + hh;
      if (a.n_text > 0) {
        // quantized part: weights exp(y_i - Y), Y = ref ln 2 + cst; sum l, and
        // sum p (alpha + s c) = alpha l + s sum c p; text parts by their maxima
        const float Y = fmaf(F.ref[hh], 0.6931471805599453f, F.cst[hh]);
        float M = Y;
        for (int w8 = 0; w8 < 8; ++w8)
          if (t_ml[(w8 * kG + hh) * 2 + 1] > 0.f) M = fmaxf(M, t_ml[(w8 * kG + hh) * 2]);
        const float fv = expf(Y - M);
        float num = fv * fmaf(step, sum, alpha * l), den = fv * l;
        for (int w8 = 0; w8 < 8; ++w8) {
          const float tlw = t_ml[(w8 * kG + hh) * 2 + 1];
          if (tlw > 0.f) {
            const float f = expf(t_ml[(w8 * kG + hh) * 2] - M);
            num = fmaf(f, t_acc[(w8 * kG + hh) * kD + ch], num);
            den = fmaf(f, tlw, den);
          }
        }
        static_cast<T*>(a.out)[bh * kD + ch] = DT<T>::from_float(num / den);
      } else if (a.part_o == nullptr) {
        static_cast<T*>(a.out)[bh * kD + ch] = DT<T>::from_float(fmaf(step, sum / l, alpha));
      } else {
        a.part_o[bh * kD + ch] = fmaf(step, sum / l, alpha);
        // sum_i exp(y_i) = 2^ref sum_i p_i e^cst with p_i = 2^(x_i alog2 - ref)
        if (ch == 0) a.part_lse[bh] = fmaf(F.ref[hh], 0.6931471805599453f, logf(l)) + F.cst[hh];
      }
    }
  }

  // ---- teardown: tensor memory back; on the error path, copies still in flight land first
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, tmem_cols);
  }
  if (t == 0 && *err) {
    report_timeout(a.status);
    for (int s = 0; s < kSlots; ++s)
      if (F.uses[s] > 0) tc::mbar_wait(&F.full[s], (F.uses[s] - 1) & 1u, kSpin);
  }
  // The split launch starts while the whole rows still run. Its last CTA (the
  // last to be scheduled) waits for them before it exits, so the split grid
  // does not complete before the whole-row grid, and work after the decode on
  // the stream sees every row; the other CTAs free their SM slots at once.
  if constexpr (kSplit)
    if (blockIdx.x == gridDim.x - 1) asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Tensor-memory columns for a CTA's tiles: 32 per tile of a lane quarter, a
// power of two >= 32.
uint32_t tmem_cols_for(int tiles) {
  uint32_t cols = 32;
  while (cols < 32u * (uint32_t)((tiles + 3) / 4)) cols <<= 1;
  return cols;
}

template <typename T, bool kSplit>
cudaError_t set_row_attributes(size_t smem) {
  static bool attr_sets[kMaxDevices];  // per device (benign race: every caller sets the same value)
  const int attr_dev = current_device();
  if (attr_dev < 0) return cudaErrorInvalidDevice;
  bool& attr_set = attr_sets[attr_dev];
  if (attr_set) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(k_decode_row<T, kSplit>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e == cudaSuccess)  // two CTAs per SM need the largest shared-memory carve-out
    e = cudaFuncSetAttribute(k_decode_row<T, kSplit>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             (int)cudaSharedmemCarveoutMaxShared);
  if (e == cudaSuccess) attr_set = true;
  return e;
}

template <typename T>
cudaError_t run_row(const DecodeArgs& a, cudaStream_t stream) {
  const int rows = a.B * a.Hkv;
  const int nt = (a.n + kTile - 1) / kTile;
  const size_t smem = row_smem_bytes() > (size_t)kMinSmem ? row_smem_bytes() : (size_t)kMinSmem;
  cudaError_t e = set_row_attributes<T, false>(smem);
  if (e != cudaSuccess) return e;
  CUtensorMap kmap, vmap;
  if (!encode_3d(&kmap, a.k_codes, kD, (uint64_t)(a.n + 7) / 8, (uint64_t)rows, kChunkTiles * 32,
                 CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_3d(&vmap, a.v_codes, 128, (uint64_t)nt * 32, (uint64_t)rows, kChunkTiles * 32,
                 CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  CUtensorMap ktmap = kmap, vtmap = vmap;  // stand-ins, never read, without f16 text tokens
  if (std::is_same<T, half>::value && a.n_text > 0 &&
      (!encode_3d_box(&ktmap, a.k_text, kD * sizeof(half), (uint64_t)a.n_text, (uint64_t)rows, 128, kTextTile,
                      CU_TENSOR_MAP_SWIZZLE_128B) ||
       !encode_3d_box(&vtmap, a.v_text, kD * sizeof(half), (uint64_t)a.n_text, (uint64_t)rows, 128, kTextTile,
                      CU_TENSOR_MAP_SWIZZLE_128B)))
    return cudaErrorInvalidValue;

  const int split = decode_row_split_rows(rows, a.n, a.n_text == 0 && a.part_o == nullptr);
  const int whole = rows - split;
  if (whole > 0) {
    k_decode_row<T, false><<<whole, kThreads, smem, stream>>>(a, tmem_cols_for(nt), 0, kmap, vmap, ktmap, vtmap);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (split > 0) {
    // the halves go into the same stream as a programmatic dependent launch:
    // every whole-row CTA lets it start as soon as it runs, and it reads and
    // writes nothing of theirs, so its CTAs take SM slots as whole rows finish
    if ((e = set_row_attributes<T, true>(smem)) != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(2 * split), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    if ((e = cudaLaunchKernelEx(&cfg, k_decode_row<T, true>, a, tmem_cols_for((nt + 1) / 2), whole, kmap, vmap,
                                ktmap, vtmap)) != cudaSuccess)
      return e;
  }
  return cudaSuccess;
}

}  // namespace

bool decode_row_supports(int n) { return n >= 1 && n <= kMaxTiles * kTile; }

// Two rows per SM run at once. Past two full waves, the rows beyond a whole
// number of SM counts would leave some SMs one row more than the others; in
// a plain decode those rows run as halves on 2-CTA clusters, in a second
// launch (programmatic dependent: it overlaps the whole rows on the same
// stream), so that the halves spread over the SMs. Only while
// they are at most half the SM count: beyond that most SMs would take a half
// on top of their whole rows and the halves' own cost (set-up, the two
// exchanges) outweighs the balance (measured on B200: 512 rows of 8192 tokens
// 86.9 -> 83.1 us, 384 rows 69.8 -> 72.7 us).
int decode_row_split_rows(int rows, int n, bool plain) {
  const int sms = device_sms(), nt = (n + kTile - 1) / kTile;
  if (!plain || nt < 2 || sms <= 0 || rows <= 2 * sms) return 0;
  const int rest = rows % sms;
  return rest <= sms / 2 ? rest : 0;
}

cudaError_t launch_decode_row(const DecodeArgs& a, cq_dtype dt, cudaStream_t stream) {
  if (!decode_row_supports(a.n)) return cudaErrorNotSupported;
  if (dt == CQ_F16) return run_row<half>(a, stream);
  return run_row<float>(a, stream);
}

}  // namespace cq
