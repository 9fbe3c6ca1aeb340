// Building blocks shared by the register-fed decode kernels: ldmatrix /
// shared-memory loads, the 8-bit mma.sync forms, warp reductions, the logit
// placement in shared memory, bounded copy waits, and tensor-map encoding.
#pragma once

#include <cuda.h>  // CUtensorMap (encoded through the runtime's driver entry point; no libcuda link)
#include <cuda_runtime.h>
#include <stdint.h>

#include "calibq.h"
#include "tc.cuh"

namespace cq {
namespace mu {

constexpr int kG = 4;                 // query heads per kv-head
constexpr uint32_t kSpin = 1u << 24;  // bound on every mbarrier wait (about a second)

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr)
               : "memory");
}
// The same four 8x8 matrices, each transposed on the way into registers.
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr)
               : "memory");
}
__device__ __forceinline__ void lds128(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr)
               : "memory");
}

__device__ __forceinline__ void sts128(uint32_t addr, const uint32_t (&r)[4]) {
  asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3])
               : "memory");
}

// D += A (16x32 u8, row) x B (32x8 s8, col). Register-only: the compiler may
// interleave independent MMAs.
__device__ __forceinline__ void mma_u8s8(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// D += A (16x32 s8, row) x B (32x8 u8, col)
__device__ __forceinline__ void mma_s8u8(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// D += A (16x32 u8, row) x B (32x8 u8, col)
__device__ __forceinline__ void mma_u8u8(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// D += A (16x16 f16, row) x B (16x8 f16, col), f32 accumulators
__device__ __forceinline__ void mma_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
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

// Position (in floats, within its unit's 2 KB) of the logit of octet o (0..15)
// of a unit, bit position k, head h. Rows of 16 floats; odd units swap row
// pairs and heads 2, 3 swap octet halves, so that both the K-side stores and
// the softmax-side float4 loads are free of bank conflicts.
__device__ __forceinline__ int logit_pos(int unit, int k, int h, int o) {
  return (((k * kG + h) ^ (unit & 1)) << 4) + (o ^ ((h >> 1) << 3));
}

// Every thread waits for the copy phase; a wait that runs out flags the CTA
// (its outputs become NaN) instead of hanging. probes = 0: the default bound
// (try_wait, about a second); otherwise that many non-suspending probes.
__device__ __forceinline__ void wait_copies(uint64_t* bar, uint32_t parity, volatile int* err,
                                            uint32_t probes = 0) {
  bool ok = false;
  if (probes == 0) {
    ok = tc::mbar_wait(bar, parity, kSpin);
  } else {
    for (uint32_t i = 0; i < probes && !ok; ++i) ok = tc::mbar_test_wait(bar, parity);
  }
  if (!ok) *err = 1;
}

// Report a CTA's timed-out wait in the caller's status word (one thread).
__device__ __forceinline__ void report_timeout(int* status) {
  if (status != nullptr) atomicOr(status, CQ_DEVICE_WAIT_TIMEOUT);
}

// The same for a whole warp: every lane probes without suspending and the warp
// leaves together once every lane has seen the phase complete, so no lane
// trails the others into the next warp-collective instruction.
__device__ __forceinline__ void warp_wait_copies(uint64_t* bar, uint32_t parity, volatile int* err) {
  for (uint32_t i = 0; i < kSpin; ++i)
    if (__all_sync(0xffffffffu, tc::mbar_test_wait(bar, parity))) return;
  *err = 1;
}

// ---------------------------------------------------------------- host side
using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiled encode_fn() {
  static EncodeTiled fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<EncodeTiled>(p);
  }();
  return fn;
}

// 3-D uint8 map {inner bytes, mid, outer} with box {box_inner, box_mid, 1}.
inline bool encode_3d_box_uncached(CUtensorMap* m, const void* base, uint64_t inner, uint64_t mid, uint64_t outer,
                                   uint32_t box_inner, uint32_t box_mid, CUtensorMapSwizzle swz) {
  const EncodeTiled fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[3] = {inner, mid, outer};
  const cuuint64_t strides[2] = {inner, inner * mid};
  const cuuint32_t box[3] = {box_inner, box_mid, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The same through a small per-thread cache of recent encodings: a decode loop
// passes the same buffers every step, and an encoding depends on its arguments
// only, so a hit returns exactly the map the encoder would write.
inline bool encode_3d_box(CUtensorMap* m, const void* base, uint64_t inner, uint64_t mid, uint64_t outer,
                          uint32_t box_inner, uint32_t box_mid, CUtensorMapSwizzle swz) {
  struct Entry {
    CUtensorMap map;
    const void* base;
    uint64_t inner, mid, outer;
    uint32_t box_inner, box_mid;
    int swz;
    bool used;
  };
  constexpr int kEntries = 8;
  thread_local Entry cache[kEntries] = {};
  thread_local int next = 0;
  for (Entry& e : cache)
    if (e.used && e.base == base && e.inner == inner && e.mid == mid && e.outer == outer &&
        e.box_inner == box_inner && e.box_mid == box_mid && e.swz == (int)swz) {
      *m = e.map;
      return true;
    }
  if (!encode_3d_box_uncached(m, base, inner, mid, outer, box_inner, box_mid, swz)) return false;
  Entry& e = cache[next];
  next = (next + 1) % kEntries;
  e.map = *m;
  e.base = base;
  e.inner = inner;
  e.mid = mid;
  e.outer = outer;
  e.box_inner = box_inner;
  e.box_mid = box_mid;
  e.swz = (int)swz;
  e.used = true;
  return true;
}

// 3-D uint8 map {inner bytes, mid, outer} with box {inner, box_mid, 1}.
inline bool encode_3d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t mid, uint64_t outer, uint32_t box_mid,
                      CUtensorMapSwizzle swz) {
  return encode_3d_box(m, base, inner, mid, outer, (uint32_t)inner, box_mid, swz);
}

}  // namespace mu
}  // namespace cq
