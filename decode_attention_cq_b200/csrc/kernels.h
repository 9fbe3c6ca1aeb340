// Launchers behind the libcalibq C ABI (internal; arguments already validated).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "calibq.h"

namespace cq {

constexpr int kD = 128;  // head dimension supported by every kernel

// ---- quantize.cu
int quantize_splits(int rows, int n);
size_t quantize_workspace_bytes(int rows, int n);
// Whether cq_quantize_kv takes the two-launch path that keeps per-split
// statistics in the workspace (the single-read fill uses none).
bool quantize_uses_workspace(int rows, int n);
cudaError_t launch_quantize(const void* x, cq_dtype dt, int rows, int n, int bits, cq_layout layout,
                            uint8_t* codes, void* alpha, void* scale, void* workspace,
                            cudaStream_t stream);
// Device address (current device) and size of the library's fixed quantize scratch.
size_t quantize_static_scratch_bytes();
cudaError_t quantize_static_scratch(void** ptr);

// ---- dequant.cu
cudaError_t launch_dequant(const uint8_t* codes, const void* alpha, const void* scale, cq_dtype dt,
                           cq_layout layout, int rows, int n, int bits, void* out,
                           cudaStream_t stream);

// ---- decode_generic.cu (canonical layouts, any bits, any group size)
struct DecodeArgs {
  const void* q;
  const uint8_t* k_codes;
  const void* k_alpha;
  const void* k_scale;
  const uint8_t* v_codes;
  const void* v_alpha;
  const void* v_scale;
  void* out;
  int B, Hq, Hkv, n, bits;
  float sigma;
  int calib;
  float tau_lo, tau_hi;
  // Partial mode (octet kernels only): when part_o is set, the kernel writes the
  // normalized result in fp32 to part_o [B][Hq][d] and ln sum_i exp(y_i) of the
  // calibrated logits y = g(x) to part_lse [B][Hq] instead of writing out.
  float* part_o = nullptr;
  float* part_lse = nullptr;
  // Mixed caches in one launch (k_decode_row only): full-precision text tokens
  // [B][Hkv][n_text][d] in the input dtype, attended after the quantized ones in
  // the same softmax (their logits sigma q.k as they are, their values as stored).
  const void* k_text = nullptr;
  const void* v_text = nullptr;
  int n_text = 0;
  // Device status word (may be null): a CTA whose bounded wait ran out ORs
  // CQ_DEVICE_WAIT_TIMEOUT into it (its rows are NaN).
  int* status = nullptr;
  // Probes of each wait for a copy in k_decode_mma (whose copies are issued once
  // per launch) before it gives up; 0 = the default bound (about a second).
  uint32_t wait_probes = 0;
};
size_t decode_generic_workspace_bytes(int B, int Hq, int n);
cudaError_t launch_decode_generic(const DecodeArgs& a, cq_dtype dt, void* workspace,
                                  cudaStream_t stream);

// ---- decode_octet.cu (octet layouts, bits = 1, Hq = 4 Hkv, tensor cores)
cudaError_t launch_decode_octet(const DecodeArgs& a, cq_dtype dt, cudaStream_t stream);

// ---- decode_text.cu (mixed caches: full-precision text tokens + merge with the
// partial result of a quantized visual part; G = 4)
size_t text_merge_workspace_bytes(int B, int Hq);
cudaError_t launch_text_merge(const DecodeArgs& a, cq_dtype dt, const void* k_text, const void* v_text, int n_text,
                              cudaStream_t stream);

// ---- decode_ring.cu (octet layouts, bits in {2, 4, 8}, Hq = 4 Hkv, n <= 32768, mma.sync)
bool decode_ring_supports(int n, int bits);
cudaError_t launch_decode_ring(const DecodeArgs& a, cq_dtype dt, cudaStream_t stream);

// ---- decode_mma.cu (octet layouts, bits = 1, Hq = 4 Hkv, n <= 32768, mma.sync)
bool decode_mma_supports(int n);
cudaError_t launch_decode_mma(const DecodeArgs& a, cq_dtype dt, cudaStream_t stream);
// One CTA per (batch, kv-head) row with the logits in tensor memory (1 bit,
// octet layouts, Hq = 4 Hkv, n <= 8192).
bool decode_row_supports(int n);
// Rows of a plain decode (no text tokens, no partial result) that the row
// kernel runs as halves on 2-CTA clusters in a second launch (0: none).
int decode_row_split_rows(int rows, int n, bool plain);
cudaError_t launch_decode_row(const DecodeArgs& a, cq_dtype dt, cudaStream_t stream);

// ---- decode_tc.cu (1 bit, octet layouts, Hq = 4 Hkv, n <= 8192, plain decodes:
// one persistent CTA per SM, tcgen05 MMAs fed by worker warps, dedicated issuers)
bool decode_tc_supports(int n);
cudaError_t launch_decode_tc(const DecodeArgs& a, cq_dtype dt, cudaStream_t stream);

}  // namespace cq
