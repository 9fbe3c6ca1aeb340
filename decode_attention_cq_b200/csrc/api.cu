// The libcalibq C ABI: host-side validation and dispatch (see include/calibq.h).
#include <atomic>
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include <limits>

#include <cuda.h>  // CUdeviceptr, CUresult (the driver entry point, no libcuda link)

#include "calibq.h"
#include "common.cuh"
#include "kernels.h"

namespace {

using cq::kD;

constexpr int kVersion = 10000;  // 1.0.0

bool valid_bits(int bits) { return bits == 1 || bits == 2 || bits == 4 || bits == 8; }
bool valid_dtype(cq_dtype dt) { return dt == CQ_F16 || dt == CQ_F32; }
bool valid_layout(cq_layout l) {
  return l == CQ_LAYOUT_CANONICAL || l == CQ_LAYOUT_OCTET_K || l == CQ_LAYOUT_OCTET_V;
}
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// cuMemGetAddressRange through the runtime's driver entry point (the library
// does not link libcuda): the extent of the allocation that holds a pointer.
using GetAddressRange = CUresult (*)(CUdeviceptr*, size_t*, CUdeviceptr);
GetAddressRange address_range_fn() {
  static const GetAddressRange fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuMemGetAddressRange", &p, 12000, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<GetAddressRange>(p);
  }();
  return fn;
}

// Allocations that passed check_ptr on this host thread: [base, end) of device
// memory of device `dev`, or of managed memory (dev = -1). A call passes up to
// ten pointers, most of them into the same few allocations, and a decode loop
// passes the same buffers every step; a pointer inside a remembered allocation
// is accepted without a driver query (each costs a few tenths of a
// microsecond). Replaced round robin.
struct SeenAlloc {
  uintptr_t base = 0, end = 0;
  int dev = -2;
};
constexpr int kSeenAllocs = 16;
thread_local SeenAlloc g_seen[kSeenAllocs];
thread_local int g_seen_next = 0;

// Device memory of the current device (or managed memory) and 16-byte aligned.
cq_status check_ptr(const void* p) {
  if (p == nullptr || !aligned16(p)) return CQ_ERR_INVALID_ARG;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return CQ_ERR_CUDA;
  const uintptr_t u = reinterpret_cast<uintptr_t>(p);
  for (const SeenAlloc& a : g_seen)
    if (u >= a.base && u < a.end && (a.dev == dev || a.dev == -1)) return CQ_OK;
  cudaPointerAttributes attr;
  cudaError_t e = cudaPointerGetAttributes(&attr, p);
  if (e != cudaSuccess) {
    cudaGetLastError();  // clear the sticky-free error of an unknown pointer
    return CQ_ERR_INVALID_ARG;
  }
  if (attr.type != cudaMemoryTypeDevice && attr.type != cudaMemoryTypeManaged)
    return CQ_ERR_INVALID_ARG;
  if (attr.type == cudaMemoryTypeDevice && attr.device != dev) return CQ_ERR_INVALID_ARG;
  CUdeviceptr base = 0;
  size_t bytes = 0;
  const GetAddressRange range = address_range_fn();
  if (range != nullptr && range(&base, &bytes, (CUdeviceptr)u) == CUDA_SUCCESS && bytes > 0) {
    g_seen[g_seen_next] = SeenAlloc{(uintptr_t)base, (uintptr_t)base + bytes,
                                    attr.type == cudaMemoryTypeManaged ? -1 : dev};
    g_seen_next = (g_seen_next + 1) % kSeenAllocs;
  }
  return CQ_OK;
}

// 1-bit octet-layout decode kernels: "row" (one CTA per row, logits in tensor
// memory, n <= 8192), "cluster" (a cluster of CTAs per row, n <= 32768),
// "tcgen05" (5th-generation tensor cores, n <= 65536) and "pipe" (one
// persistent CTA per SM whose warps feed tcgen05 MMAs, plain decodes with
// n <= 8192; measured slower than "row" on B200, so only on request).
// cq_set_decode_kernel, else the environment variable CALIBQ_DECODE_KERNEL,
// may name one to use wherever it supports the call; otherwise the choice
// between the row and the cluster kernel is the one with the smaller
// estimated step time, and the tcgen05 kernel takes what neither supports.
enum class Kernel1 { kAuto, kRow, kCluster, kTcgen05, kPipe };

Kernel1 env_kernel() {
  static const Kernel1 forced = [] {
    const char* v = getenv("CALIBQ_DECODE_KERNEL");
    if (v == nullptr) return Kernel1::kAuto;
    if (strcmp(v, "row") == 0) return Kernel1::kRow;
    if (strcmp(v, "cluster") == 0) return Kernel1::kCluster;
    if (strcmp(v, "tcgen05") == 0) return Kernel1::kTcgen05;
    if (strcmp(v, "pipe") == 0) return Kernel1::kPipe;
    return Kernel1::kAuto;
  }();
  return forced;
}

std::atomic<int> g_set_kernel{-1};  // cq_set_decode_kernel's choice; -1: none made

Kernel1 forced_kernel() {
  const int v = g_set_kernel.load(std::memory_order_relaxed);
  return v < 0 ? env_kernel() : static_cast<Kernel1>(v);
}

// SM count of the current device (read once per device).
int sm_count() {
  static std::atomic<int> counts[cq::kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= cq::kMaxDevices) return 0;
  int c = counts[dev].load(std::memory_order_relaxed);
  if (c == 0) {
    if (cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    counts[dev].store(c, std::memory_order_relaxed);
  }
  return c;
}

// Step-time estimates (microseconds on B200) of the two kernels for `rows`
// (batch, kv-head) rows of n tokens, fitted to measurements at n = 3328 and
// 8192 over 128 to 512 rows (every point within about 3 us). The row kernel
// runs two CTAs per SM: t1 is a row alone on its SM, t2 a wave of two per SM,
// and a partial last wave costs 0.6 t1 when it leaves at most one row per SM,
// else 0.8 t2; a plain decode whose leftover rows run as split halves
// (decode_row_split_rows) gains about 0.1 t2. The cluster kernel's time grows
// about linearly in the rows.
double est_row_us(int n, long long rows, int sms, bool split) {
  const double t1 = 12.8 + 0.00243 * n, t2 = 16.7 + 0.0037 * n;
  if (rows <= sms) return t1;
  const long long slots = 2LL * sms, full = rows / slots, rest = rows % slots;
  if (full == 0) return t2;
  return (double)full * t2 + (rest == 0 ? 0.0 : rest <= sms ? 0.6 * t1 : 0.8 * t2) - (split ? 0.1 * t2 : 0.0);
}
double est_cluster_us(int n, long long rows) { return 11.7 + (double)rows * (0.0065 + 1.77e-5 * n); }

// partial: the visual part of a two-launch mixed call (no tcgen05 kernel);
// plain: a decode with no text tokens and no partial result (rows may split).
Kernel1 choose_1bit(int n, int rows, bool partial, bool plain) {
  const Kernel1 f = forced_kernel();
  const bool pipe = plain && cq::decode_tc_supports(n);
  if (f == Kernel1::kPipe && pipe) return Kernel1::kPipe;
  if (f == Kernel1::kRow && cq::decode_row_supports(n)) return Kernel1::kRow;
  if (f == Kernel1::kCluster && cq::decode_mma_supports(n)) return Kernel1::kCluster;
  if (f == Kernel1::kTcgen05 && !partial) return Kernel1::kTcgen05;
  const int sms = sm_count();
  const bool split = plain && cq::decode_row_split_rows(rows, n, true) > 0;
  if (cq::decode_row_supports(n) && sms > 0 && est_row_us(n, rows, sms, split) < est_cluster_us(n, rows))
    return Kernel1::kRow;
  if (cq::decode_mma_supports(n)) return Kernel1::kCluster;
  return partial ? Kernel1::kAuto : Kernel1::kTcgen05;  // kAuto: none
}

cudaError_t launch_decode_1bit(const cq::DecodeArgs& a, cq_dtype dt, cudaStream_t s) {
  switch (choose_1bit(a.n, a.B * a.Hkv, a.part_o != nullptr, a.part_o == nullptr && a.n_text == 0)) {
    case Kernel1::kRow: return cq::launch_decode_row(a, dt, s);
    case Kernel1::kCluster: return cq::launch_decode_mma(a, dt, s);
    case Kernel1::kTcgen05: return cq::launch_decode_octet(a, dt, s);
    case Kernel1::kPipe: return cq::launch_decode_tc(a, dt, s);
    default: return cudaErrorNotSupported;
  }
}

#define CQ_TRY(expr)                 \
  do {                               \
    const cq_status _s = (expr);     \
    if (_s != CQ_OK) return _s;      \
  } while (0)

// Sizes shared by every entry point.
cq_status check_shape(int B, int H, int n, int d, int bits) {
  if (B < 1 || H < 1 || n < 1) return CQ_ERR_INVALID_ARG;
  if (!valid_bits(bits)) return CQ_ERR_INVALID_ARG;
  if (d != kD) return CQ_ERR_UNSUPPORTED;
  // every element index must fit comfortably in 63 bits and rows in a grid dimension
  if ((double)B * H * n * d > 9.0e15) return CQ_ERR_INVALID_ARG;
  if ((long long)B * H > (long long)std::numeric_limits<int>::max()) return CQ_ERR_INVALID_ARG;
  return CQ_OK;
}

cq_status row_bytes(cq_layout layout, int n, int bits, size_t* out) {
  if (!valid_layout(layout) || !valid_bits(bits)) return CQ_ERR_INVALID_ARG;
  switch (layout) {
    case CQ_LAYOUT_CANONICAL: *out = (size_t)n * kD * bits / 8; return CQ_OK;
    case CQ_LAYOUT_OCTET_K:  // 8 / bits tokens per byte
      *out = (size_t)((n + 8 / bits - 1) / (8 / bits)) * kD;
      return CQ_OK;
    default:  // tiles of 256 / bits tokens
      *out = (size_t)((n + 256 / bits - 1) / (256 / bits)) * 4096;
      return CQ_OK;
  }
}

cq_status cuda_status(cudaError_t e) { return e == cudaSuccess ? CQ_OK : CQ_ERR_CUDA; }

cq::DecodeArgs make_args(const void* q, const uint8_t* k_codes, const void* k_alpha, const void* k_scale,
                         const uint8_t* v_codes, const void* v_alpha, const void* v_scale, int B, int Hq, int Hkv,
                         int n, int d, int bits, float softmax_scale, cq_calib calib, void* out) {
  cq::DecodeArgs a;
  a.q = q;
  a.k_codes = k_codes;
  a.k_alpha = k_alpha;
  a.k_scale = k_scale;
  a.v_codes = v_codes;
  a.v_alpha = v_alpha;
  a.v_scale = v_scale;
  a.out = out;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.n = n;
  a.bits = bits;
  a.sigma = softmax_scale == 0.f ? 1.0f / sqrtf((float)d) : softmax_scale;
  a.calib = calib.enabled ? 1 : 0;
  a.tau_lo = calib.tau_lo;
  a.tau_hi = calib.tau_hi;
  return a;
}

}  // namespace

extern "C" {

int cq_version(void) { return kVersion; }

const char* cq_status_string(cq_status status) {
  switch (status) {
    case CQ_OK: return "CQ_OK";
    case CQ_ERR_INVALID_ARG: return "CQ_ERR_INVALID_ARG: null, misaligned or host pointer, or a bad size/enum";
    case CQ_ERR_UNSUPPORTED: return "CQ_ERR_UNSUPPORTED: valid request outside the supported set";
    case CQ_ERR_WORKSPACE: return "CQ_ERR_WORKSPACE: workspace missing or too small";
    case CQ_ERR_CUDA: return "CQ_ERR_CUDA: a CUDA call or kernel launch failed";
  }
  return "unknown cq_status";
}

cq_status cq_codes_bytes(cq_layout layout, int B, int H, int n, int d, int bits, size_t* bytes) {
  if (bytes == nullptr) return CQ_ERR_INVALID_ARG;
  CQ_TRY(check_shape(B, H, n, d, bits));
  size_t rb = 0;
  CQ_TRY(row_bytes(layout, n, bits, &rb));
  *bytes = (size_t)B * H * rb;
  return CQ_OK;
}

cq_status cq_quantize_kv_workspace_size(int B, int H, int n, int d, size_t* bytes) {
  if (bytes == nullptr) return CQ_ERR_INVALID_ARG;
  CQ_TRY(check_shape(B, H, n, d, 1));
  *bytes = cq::quantize_workspace_bytes(B * H, n);
  return CQ_OK;
}

cq_status cq_quantize_kv(const void* x, cq_dtype dt, int B, int H, int n, int d, int bits,
                         cq_layout layout, uint8_t* codes, void* alpha, void* scale,
                         void* workspace, size_t ws_bytes, cq_stream_t stream) {
  if (!valid_dtype(dt)) return CQ_ERR_INVALID_ARG;
  CQ_TRY(check_shape(B, H, n, d, bits));
  size_t rb = 0;
  CQ_TRY(row_bytes(layout, n, bits, &rb));
  CQ_TRY(check_ptr(x));
  CQ_TRY(check_ptr(codes));
  CQ_TRY(check_ptr(alpha));
  CQ_TRY(check_ptr(scale));
  const size_t need = cq::quantize_workspace_bytes(B * H, n);
  if (workspace == nullptr || ws_bytes < need) return CQ_ERR_WORKSPACE;
  CQ_TRY(check_ptr(workspace));
  return cuda_status(cq::launch_quantize(x, dt, B * H, n, bits, layout, codes, alpha, scale,
                                         workspace, reinterpret_cast<cudaStream_t>(stream)));
}

cq_status cq_quantize_kv_noalloc(const void* x, cq_dtype dt, int B, int H, int n, int d, int bits,
                                 cq_layout layout, uint8_t* codes, void* alpha, void* scale,
                                 cq_stream_t stream) {
  if (!valid_dtype(dt)) return CQ_ERR_INVALID_ARG;
  CQ_TRY(check_shape(B, H, n, d, bits));
  size_t rb = 0;
  CQ_TRY(row_bytes(layout, n, bits, &rb));
  // only the two-launch path (n > 16384) keeps statistics in the scratch
  if (cq::quantize_uses_workspace(B * H, n) &&
      cq::quantize_workspace_bytes(B * H, n) > cq::quantize_static_scratch_bytes())
    return CQ_ERR_UNSUPPORTED;
  CQ_TRY(check_ptr(x));
  CQ_TRY(check_ptr(codes));
  CQ_TRY(check_ptr(alpha));
  CQ_TRY(check_ptr(scale));
  void* scratch = nullptr;
  if (cq::quantize_static_scratch(&scratch) != cudaSuccess) return CQ_ERR_CUDA;
  return cuda_status(cq::launch_quantize(x, dt, B * H, n, bits, layout, codes, alpha, scale,
                                         scratch, reinterpret_cast<cudaStream_t>(stream)));
}

cq_status cq_decode_attn_workspace_size(cq_layout k_layout, cq_layout v_layout, int B, int Hq,
                                        int Hkv, int n, int d, int bits, size_t* bytes) {
  if (bytes == nullptr) return CQ_ERR_INVALID_ARG;
  CQ_TRY(check_shape(B, Hq, n, d, bits));
  if (Hkv < 1 || Hq % Hkv) return CQ_ERR_INVALID_ARG;
  if (!valid_layout(k_layout) || !valid_layout(v_layout)) return CQ_ERR_INVALID_ARG;
  if (k_layout == CQ_LAYOUT_CANONICAL && v_layout == CQ_LAYOUT_CANONICAL) {
    *bytes = cq::decode_generic_workspace_bytes(B, Hq, n);
    return CQ_OK;
  }
  if (k_layout == CQ_LAYOUT_OCTET_K && v_layout == CQ_LAYOUT_OCTET_V) {
    *bytes = 0;
    return CQ_OK;
  }
  return CQ_ERR_UNSUPPORTED;
}

const char* cq_decode_kernel_name(cq_layout k_layout, cq_layout v_layout, int B, int Hq, int Hkv, int n, int d,
                                  int bits) {
  if (check_shape(B, Hq, n, d, bits) != CQ_OK || Hkv < 1 || Hq % Hkv) return nullptr;
  const int G = Hq / Hkv;
  if (k_layout == CQ_LAYOUT_CANONICAL && v_layout == CQ_LAYOUT_CANONICAL)
    return G <= 32 ? "k_scores + k_softmax_v + k_merge" : nullptr;
  if (k_layout != CQ_LAYOUT_OCTET_K || v_layout != CQ_LAYOUT_OCTET_V || G != 4) return nullptr;
  if (bits != 1) return cq::decode_ring_supports(n, bits) ? "k_decode_ring" : nullptr;
  if (n > 65536) return nullptr;
  switch (choose_1bit(n, B * Hkv, false, true)) {
    case Kernel1::kRow: return "k_decode_row";
    case Kernel1::kCluster: return "k_decode_mma";
    case Kernel1::kPipe: return "k_decode_tc";
    default: return "k_decode_octet";
  }
}

int cq_decode_launch_count(cq_layout k_layout, cq_layout v_layout, int B, int Hq, int Hkv, int n, int d, int bits,
                           int n_text) {
  if (n_text < 0) return 0;
  const char* name = cq_decode_kernel_name(k_layout, v_layout, B, Hq, Hkv, n, d, bits);
  if (name == nullptr) return 0;
  if (k_layout == CQ_LAYOUT_CANONICAL) return n_text > 0 ? 0 : 3;  // mixed calls take the octet layouts only
  if (bits != 1) return n_text > 0 ? 2 : 1;                          // ring kernel (partial), text merge
  if (n_text > 0) {  // the row kernel attends the text tokens itself; the others hand over to the text merge
    if (n > 32768) return 0;
    return choose_1bit(n, B * Hkv, false, false) == Kernel1::kRow ? 1 : 2;
  }
  if (choose_1bit(n, B * Hkv, false, true) == Kernel1::kRow)
    return 1 + (cq::decode_row_split_rows(B * Hkv, n, true) > 0 ? 1 : 0);
  return 1;
}

cq_status cq_set_decode_kernel(cq_decode_kernel which) {
  switch (which) {
    case CQ_KERNEL_AUTO: g_set_kernel.store((int)Kernel1::kAuto); return CQ_OK;
    case CQ_KERNEL_ROW: g_set_kernel.store((int)Kernel1::kRow); return CQ_OK;
    case CQ_KERNEL_CLUSTER: g_set_kernel.store((int)Kernel1::kCluster); return CQ_OK;
    case CQ_KERNEL_TCGEN05: g_set_kernel.store((int)Kernel1::kTcgen05); return CQ_OK;
    case CQ_KERNEL_PIPE: g_set_kernel.store((int)Kernel1::kPipe); return CQ_OK;
    case CQ_KERNEL_ENV: g_set_kernel.store(-1); return CQ_OK;
    default: return CQ_ERR_INVALID_ARG;
  }
}

cq_status cq_decode_attn(const void* q, cq_dtype dt, const uint8_t* k_codes, const void* k_alpha,
                         const void* k_scale, cq_layout k_layout, const uint8_t* v_codes,
                         const void* v_alpha, const void* v_scale, cq_layout v_layout, int B,
                         int Hq, int Hkv, int n, int d, int bits, float softmax_scale,
                         cq_calib calib, void* out, void* workspace, size_t ws_bytes,
                         cq_stream_t stream) {
  return cq_decode_attn_ex(q, dt, k_codes, k_alpha, k_scale, k_layout, v_codes, v_alpha, v_scale, v_layout, B, Hq,
                           Hkv, n, d, bits, softmax_scale, calib, out, workspace, ws_bytes, nullptr, 0u, stream);
}

cq_status cq_decode_attn_ex(const void* q, cq_dtype dt, const uint8_t* k_codes, const void* k_alpha,
                            const void* k_scale, cq_layout k_layout, const uint8_t* v_codes,
                            const void* v_alpha, const void* v_scale, cq_layout v_layout, int B,
                            int Hq, int Hkv, int n, int d, int bits, float softmax_scale,
                            cq_calib calib, void* out, void* workspace, size_t ws_bytes,
                            int* status, unsigned wait_probes, cq_stream_t stream) {
  if (!valid_dtype(dt)) return CQ_ERR_INVALID_ARG;
  CQ_TRY(check_shape(B, Hq, n, d, bits));
  if (Hkv < 1 || Hq % Hkv) return CQ_ERR_INVALID_ARG;
  if (!valid_layout(k_layout) || !valid_layout(v_layout)) return CQ_ERR_INVALID_ARG;
  if (!isfinite(softmax_scale) || softmax_scale < 0.f) return CQ_ERR_INVALID_ARG;
  if (calib.enabled && (!isfinite(calib.tau_lo) || !isfinite(calib.tau_hi))) return CQ_ERR_INVALID_ARG;
  size_t rb = 0;
  CQ_TRY(row_bytes(k_layout, n, bits, &rb));
  CQ_TRY(row_bytes(v_layout, n, bits, &rb));
  const bool generic = k_layout == CQ_LAYOUT_CANONICAL && v_layout == CQ_LAYOUT_CANONICAL;
  const bool octet = k_layout == CQ_LAYOUT_OCTET_K && v_layout == CQ_LAYOUT_OCTET_V;
  if (!generic && !octet) return CQ_ERR_UNSUPPORTED;
  const int G = Hq / Hkv;
  if (generic && G > 32) return CQ_ERR_UNSUPPORTED;
  if (octet && (G != 4 || (bits == 1 ? n > 65536 : !cq::decode_ring_supports(n, bits))))
    return CQ_ERR_UNSUPPORTED;
  const void* ptrs[] = {q, k_codes, k_alpha, k_scale, v_codes, v_alpha, v_scale, out};
  for (const void* p : ptrs) CQ_TRY(check_ptr(p));
  if (status != nullptr) CQ_TRY(check_ptr(status));
  cq::DecodeArgs a = make_args(q, k_codes, k_alpha, k_scale, v_codes, v_alpha, v_scale, B, Hq, Hkv, n, d, bits,
                               softmax_scale, calib, out);
  a.status = status;
  a.wait_probes = wait_probes;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (generic) {
    const size_t need = cq::decode_generic_workspace_bytes(B, Hq, n);
    if (workspace == nullptr || ws_bytes < need) return CQ_ERR_WORKSPACE;
    CQ_TRY(check_ptr(workspace));
    return cuda_status(cq::launch_decode_generic(a, dt, workspace, s));
  }
  const cudaError_t e = bits != 1 ? cq::launch_decode_ring(a, dt, s) : launch_decode_1bit(a, dt, s);
  if (e == cudaErrorNotSupported) return CQ_ERR_UNSUPPORTED;
  return cuda_status(e);
}

cq_status cq_decode_attn_mixed_workspace_size(int B, int Hq, int d, size_t* bytes) {
  if (bytes == nullptr || B < 1 || Hq < 1) return CQ_ERR_INVALID_ARG;
  if (d != kD) return CQ_ERR_UNSUPPORTED;
  *bytes = cq::text_merge_workspace_bytes(B, Hq);
  return CQ_OK;
}

cq_status cq_decode_attn_mixed(const void* q, cq_dtype dt, const uint8_t* k_codes, const void* k_alpha,
                               const void* k_scale, const uint8_t* v_codes, const void* v_alpha,
                               const void* v_scale, int n_vis, int bits, const void* k_text, const void* v_text,
                               int n_text, int B, int Hq, int Hkv, int d, float softmax_scale, cq_calib calib,
                               void* out, void* workspace, size_t ws_bytes, cq_stream_t stream) {
  if (!valid_dtype(dt)) return CQ_ERR_INVALID_ARG;
  CQ_TRY(check_shape(B, Hq, n_vis, d, bits));
  if (Hkv < 1 || Hq % Hkv || n_text < 0) return CQ_ERR_INVALID_ARG;
  if (!isfinite(softmax_scale) || softmax_scale < 0.f) return CQ_ERR_INVALID_ARG;
  if (calib.enabled && (!isfinite(calib.tau_lo) || !isfinite(calib.tau_hi))) return CQ_ERR_INVALID_ARG;
  if ((double)B * Hkv * n_text * d > 9.0e15) return CQ_ERR_INVALID_ARG;
  if (Hq / Hkv != 4) return CQ_ERR_UNSUPPORTED;
  if (bits == 1 ? !cq::decode_mma_supports(n_vis) : !cq::decode_ring_supports(n_vis, bits))
    return CQ_ERR_UNSUPPORTED;
  const void* ptrs[] = {q, k_codes, k_alpha, k_scale, v_codes, v_alpha, v_scale, out};
  for (const void* p : ptrs) CQ_TRY(check_ptr(p));
  if (n_text > 0) {
    CQ_TRY(check_ptr(k_text));
    CQ_TRY(check_ptr(v_text));
  }
  const size_t need = cq::text_merge_workspace_bytes(B, Hq);
  if (workspace == nullptr || ws_bytes < need) return CQ_ERR_WORKSPACE;
  CQ_TRY(check_ptr(workspace));
  cq::DecodeArgs a = make_args(q, k_codes, k_alpha, k_scale, v_codes, v_alpha, v_scale, B, Hq, Hkv, n_vis, d,
                               bits, softmax_scale, calib, out);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (bits == 1 && choose_1bit(n_vis, B * Hkv, false, false) == Kernel1::kRow) {
    // one launch: the row kernel attends the text tokens after the quantized ones
    a.k_text = k_text;
    a.v_text = v_text;
    a.n_text = n_text;
    return cuda_status(cq::launch_decode_row(a, dt, s));
  }
  a.part_o = static_cast<float*>(workspace);
  a.part_lse = a.part_o + (size_t)B * Hq * kD;
  cudaError_t e = bits != 1 ? cq::launch_decode_ring(a, dt, s) : launch_decode_1bit(a, dt, s);
  if (e == cudaErrorNotSupported) return CQ_ERR_UNSUPPORTED;
  if (e != cudaSuccess) return CQ_ERR_CUDA;
  return cuda_status(cq::launch_text_merge(a, dt, k_text, v_text, n_text, s));
}

cq_status cq_dequant(const uint8_t* codes, const void* alpha, const void* scale, cq_dtype dt,
                     cq_layout layout, int B, int H, int n, int d, int bits, void* out,
                     cq_stream_t stream) {
  if (!valid_dtype(dt)) return CQ_ERR_INVALID_ARG;
  CQ_TRY(check_shape(B, H, n, d, bits));
  size_t rb = 0;
  CQ_TRY(row_bytes(layout, n, bits, &rb));
  if ((long long)B * H > 65535) return CQ_ERR_UNSUPPORTED;
  const void* ptrs[] = {codes, alpha, scale, out};
  for (const void* p : ptrs) CQ_TRY(check_ptr(p));
  return cuda_status(cq::launch_dequant(codes, alpha, scale, dt, layout, B * H, n, bits, out,
                                        reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"
