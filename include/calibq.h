/*
 * libcalibq -- CalibQuant's visual-KV-cache quantization and decode attention
 * on NVIDIA B200 (sm_100a).
 *
 * Source of the method: the CalibQuant article (QbitAI's write-up of
 * "CalibQuant: 1-Bit KV Cache Quantization for Multimodal LLMs", arXiv
 * 2502.14882), sections "Method 1" (channel-wise b-bit quantization),
 * "Method 2" (post-scaling) and "Method 3" (post-quantization calibration).
 *
 * Conventions shared by every entry point:
 *
 *  - All tensor pointers are DEVICE pointers owned by the caller (device or
 *    managed memory of the current device; host pointers are rejected with
 *    CQ_ERR_INVALID_ARG). The library never allocates device memory and
 *    creates no streams or events in these calls. Host-side state: the kernel
 *    choice set by cq_set_decode_kernel (process-wide), and per host thread a
 *    small cache of encoded tensor maps and of the device allocations that
 *    earlier calls validated (a pointer inside one of those is accepted
 *    without asking the driver again, so a pointer into memory freed since is
 *    not caught: pass no dangling pointers). Calls are thread-safe.
 *  - Work is enqueued asynchronously on `stream` (NULL = the legacy default
 *    stream). A returned CQ_OK means the launch was enqueued; kernel faults
 *    surface on the stream like any CUDA error.
 *  - Arguments are validated on the host before anything is launched; on any
 *    error nothing is launched and no output is written.
 *  - Supported: head dim d = 128, bits in {1, 2, 4, 8}, n >= 1, Hq a multiple
 *    of Hkv. Tensors are dense and contiguous (row-major, last index fastest).
 *  - dtype CQ_F16 = IEEE binary16, CQ_F32 = IEEE binary32.
 */
#ifndef CALIBQ_H
#define CALIBQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; declared here so the header needs no CUDA headers. */
typedef struct CUstream_st* cq_stream_t;

typedef enum cq_status {
  CQ_OK = 0,
  CQ_ERR_INVALID_ARG = 1, /* null / misaligned / host pointer, bad size, bad enum */
  CQ_ERR_UNSUPPORTED = 2, /* valid request outside the supported set (e.g. d != 128) */
  CQ_ERR_WORKSPACE = 3,   /* workspace missing or smaller than the *_workspace_size query */
  CQ_ERR_CUDA = 4         /* a CUDA runtime call or launch failed */
} cq_status;

typedef enum cq_dtype { CQ_F16 = 0, CQ_F32 = 1 } cq_dtype;

/*
 * Bit layouts of a packed code row (one (batch, head) pair). A row holds the
 * codes of tokens 0..n-1 (padded where stated); rows follow each other with no
 * gap, so the codes buffer is [B][H][row_bytes].
 *
 * CQ_LAYOUT_CANONICAL (any bits; row_bytes = n * d * bits / 8):
 *   token-major. Token i occupies d*bits/8 bytes starting at i*d*bits/8;
 *   channel j's code is stored at bits [j*bits, j*bits+bits) of the token's
 *   little-endian bit string, i.e. at bit (j*bits) % 32 of little-endian
 *   uint32 word (j*bits)/32 of the token.
 *
 * CQ_LAYOUT_OCTET_K (bits in {1, 2, 4, 8}, d = 128; P = 8 / bits tokens share
 *   a byte; row_bytes = ceil(n/P) * 128): one byte per (P consecutive tokens,
 *   channel). Token i, channel j:
 *       byte = (i / P) * 128 + j,         code at bits [(i % P) * bits, +bits).
 *   For bits = 1: byte = (i >> 3) * 128 + j, bit = i & 7. (Row m of the
 *   [n/P][128] byte matrix is one row of the K-side tensor-core operand;
 *   masking sub-position k of every byte gives "code of token P m + k times
 *   2^(k bits)" as an 8-bit operand.)
 *
 * CQ_LAYOUT_OCTET_V (bits in {1, 2, 4, 8}, d = 128; row_bytes =
 *   ceil(n / (32 P)) * 4096): the same bytes, transposed per tile of 32 P
 *   tokens (256 for bits = 1). Token i, channel j:
 *       byte = (i / (32 P)) * 4096 + j * 32 + (i % (32 P)) / P,
 *       code at bits [(i % P) * bits, +bits).
 *   For bits = 1: byte = (i >> 8) * 4096 + j * 32 + ((i & 255) >> 3), bit =
 *   i & 7. (Channel j's 32 bytes of a tile are one column of the V-side
 *   operand.)
 *
 * Padding tokens (n..padded-1) of the octet layouts hold code 0 and are
 * ignored by cq_decode_attn.
 */
typedef enum cq_layout {
  CQ_LAYOUT_CANONICAL = 0,
  CQ_LAYOUT_OCTET_K = 1,
  CQ_LAYOUT_OCTET_V = 2
} cq_layout;

/*
 * Calibration g of the pre-softmax scores (Method 3). When enabled, every
 * (batch, query-head) score row x with range [m, M] is mapped linearly onto
 * [tau_lo*m, tau_hi*M]:
 *     g(x) = tau_lo*m + (x - m) * (tau_hi*M - tau_lo*m) / (M - m),
 * and a row with M == m is left unchanged. (The article fixes g as the linear
 * map of the row's score range onto a target interval given by parameters;
 * the interval [tau_lo*m, tau_hi*M] is this library's reading.) tau = (1, 1)
 * is the identity. Requires finite tau_lo, tau_hi.
 */
typedef struct cq_calib {
  int enabled;
  float tau_lo;
  float tau_hi;
} cq_calib;

/* Library version as 10000*major + 100*minor + patch. */
int cq_version(void);

/* Static, never-NULL description of a status code. */
const char* cq_status_string(cq_status status);

/*
 * Bytes of a packed codes buffer [B][H][row_bytes] for the given layout.
 * Pure host function; CQ_ERR_INVALID_ARG for bad sizes, CQ_ERR_UNSUPPORTED
 * for a layout/bits/d combination outside the supported set.
 */
cq_status cq_codes_bytes(cq_layout layout, int B, int H, int n, int d, int bits, size_t* bytes);

/*
 * Workspace (device bytes, 256-byte aligned pointer) needed by cq_quantize_kv.
 */
cq_status cq_quantize_kv_workspace_size(int B, int H, int n, int d, size_t* bytes);

/*
 * Channel-wise b-bit quantization of one cache tensor (Method 1). Call once
 * for K and once for V.
 *
 *   x       [B][H][n][d] in dtype `dt` (16-byte aligned).
 *   codes   packed codes, cq_codes_bytes(layout, ...) bytes (16-byte aligned).
 *   alpha   [B][H][d] in `dt`: per-channel minimum over the n tokens (exact).
 *   scale   [B][H][d] in `dt`: per-channel step (beta - alpha) / (2^bits - 1),
 *           computed in double and rounded once to `dt` (0 for a constant channel).
 *   workspace / ws_bytes: at least cq_quantize_kv_workspace_size(...) bytes.
 *
 * Code of element x of channel j: the nearest integer to the real number
 * (x - alpha_j) * L / (beta_j - alpha_j), L = 2^bits - 1, ties to even, taken
 * on the IEEE double evaluation ((x - alpha) * L) / (beta - alpha); 0 when
 * beta_j == alpha_j. (For binary16 inputs this is the exact real rounding.)
 * The octet layouts take bits in {1, 2, 4, 8} with d = 128.
 *
 * Execution: for n <= 16384 one launch reads x once (a thread-block cluster
 * per (b, h) row exchanges the channel statistics on chip, and each CTA packs
 * the tile it has just read); longer rows take two launches (statistics into
 * the workspace, then pack). Both give identical alpha, scale and codes.
 */
cq_status cq_quantize_kv(const void* x, cq_dtype dt, int B, int H, int n, int d, int bits,
                         cq_layout layout, uint8_t* codes, void* alpha, void* scale,
                         void* workspace, size_t ws_bytes, cq_stream_t stream);

/*
 * cq_quantize_kv without a caller workspace. (Not part of the method: the
 * article has no counterpart; this is a deployment convenience.)
 *
 * Some embedders cannot give the library scratch device memory: a serving
 * runtime that has already reserved all of HBM for its own KV-cache pool (a
 * cudaMalloc there fails or fragments the pool), or a caller on a
 * latency-critical path where cudaMalloc/cudaFree would implicitly
 * synchronize the device. This entry point takes the same arguments as
 * cq_quantize_kv minus the workspace, allocates nothing (no cudaMalloc, no
 * cudaFree, no allocating library routine) and keeps its scratch -- the
 * per-split channel minima and maxima of the two-launch path that rows with
 * n > 16384 take -- in a fixed 4 MiB array compiled into the library, which
 * every GPU that loads the library holds until the process exits. Rows with
 * n <= 16384 take the single-read fill, which needs no scratch at all.
 *
 *  - Limit: a request on the two-launch path whose scratch
 *    (cq_quantize_kv_workspace_size) exceeds 4 MiB returns
 *    CQ_ERR_UNSUPPORTED and launches nothing; this is decided from the sizes
 *    alone, before the pointers are looked at.
 *  - The first call on each device looks up that device's address of the
 *    array (with the device current) and keeps it; make that first call
 *    before any stream capture. cudaDeviceReset invalidates the kept address:
 *    do not call this entry point on a device after resetting it.
 *  - Every call, on any stream, shares the one array: calls whose kernels
 *    overlap on the GPU race with each other. Serialize them (one stream, or
 *    events). The array keeps the previous call's contents; nothing in it has
 *    to start at zero because every call overwrites what it reads.
 *  - Unlike the rest of the library this entry point has global state (the
 *    array and the per-device address cache, guarded by a mutex).
 */
cq_status cq_quantize_kv_noalloc(const void* x, cq_dtype dt, int B, int H, int n, int d, int bits,
                                 cq_layout layout, uint8_t* codes, void* alpha, void* scale,
                                 cq_stream_t stream);

/*
 * Workspace needed by cq_decode_attn for this layout pair (0 for the octet
 * layouts, which keep every intermediate on chip).
 */
cq_status cq_decode_attn_workspace_size(cq_layout k_layout, cq_layout v_layout, int B, int Hq,
                                        int Hkv, int n, int d, int bits, size_t* bytes);

/*
 * One decode step of grouped-query attention over the packed caches, with
 * post-scaling (Method 2) and optional calibration (Method 3):
 *
 *   x_i = sigma * ( q . alpha_K + (q (.) s_K) . c^K_i )          (logits)
 *   y   = g(x) if calib.enabled else x                           (per row)
 *   p_i = exp(y_i - max y) / sum_j exp(y_j - max y)
 *   o   = alpha_V + s_V (.) sum_i p_i c^V_i
 *
 * Query head h reads kv-head h / (Hq/Hkv). sigma = softmax_scale, or
 * 1/sqrt(d) when softmax_scale == 0.
 *
 *   q        [B][Hq][d] in `dt`;   out [B][Hq][d] in `dt`.
 *   k_codes/v_codes: packed as written by cq_quantize_kv with k_layout/v_layout;
 *   k_alpha, k_scale, v_alpha, v_scale: [B][Hkv][d] in `dt`.
 *
 * Supported layout pairs: (CANONICAL, CANONICAL) for any bits and any Hq/Hkv;
 * (OCTET_K, OCTET_V) for d = 128, Hq = 4*Hkv and n <= 65536 at bits = 1
 * (n <= 32768 at bits 2, 4, 8) -- the tensor-core path, one launch per call
 * (two for some batches of the 1-bit row kernel: cq_decode_launch_count).
 * The octet kernels hold the four query heads of a kv-head in the rows of
 * one tensor-core tile, so any other ratio Hq/Hkv with the octet layouts
 * returns CQ_ERR_UNSUPPORTED; such models store their cache in the CANONICAL
 * layout, whose CUDA-core kernels take any ratio but run several times
 * slower (about 7x at 1 bit, n = 8192, batch 16 on B200).
 * cq_decode_kernel_name says which kernel a call launches; the 1-bit kernels
 * agree with each other within the output tolerance, not bit for bit.
 */
cq_status cq_decode_attn(const void* q, cq_dtype dt, const uint8_t* k_codes, const void* k_alpha,
                         const void* k_scale, cq_layout k_layout, const uint8_t* v_codes,
                         const void* v_alpha, const void* v_scale, cq_layout v_layout, int B,
                         int Hq, int Hkv, int n, int d, int bits, float softmax_scale,
                         cq_calib calib, void* out, void* workspace, size_t ws_bytes,
                         cq_stream_t stream);

/* Bit of the device status word of cq_decode_attn_ex: a bounded wait of a
 * decode kernel ran out; the rows of the CTAs concerned were written as NaN. */
#define CQ_DEVICE_WAIT_TIMEOUT 1

/*
 * cq_decode_attn with a device-side error report. Every wait of the decode
 * kernels for data (copies from global memory, tensor-core results) is
 * bounded; a wait that runs out does not hang the GPU: the CTA writes NaN to
 * its output rows, lets the copies it issued land, and returns. The host-side
 * status (the return value) cannot know about it, since the call returns
 * before the kernels run; this entry point reports it on the device instead:
 *
 *   status       NULL, or device memory holding one int (16-byte aligned, like
 *                every pointer of this library): when any CTA's wait ran out,
 *                CQ_DEVICE_WAIT_TIMEOUT is ORed into it. Nothing else is
 *                written there; the caller zeroes it before the call and reads
 *                it after synchronizing `stream`.
 *   wait_probes  0 for the kernels' own bounds (about a second of waiting).
 *                Otherwise each wait for a copy in "k_decode_mma" (the kernel
 *                whose copies are all issued at the start of the launch) gives
 *                up after that many non-blocking probes: a diagnostic that
 *                exercises the timeout path (1 makes it give up while the
 *                copies are still in flight). The other kernels keep their own
 *                bounds, since their copy rings must not be re-armed before a
 *                copy has landed.
 *
 * Everything else is as for cq_decode_attn, which is this call with
 * status = NULL and wait_probes = 0.
 */
cq_status cq_decode_attn_ex(const void* q, cq_dtype dt, const uint8_t* k_codes, const void* k_alpha,
                            const void* k_scale, cq_layout k_layout, const uint8_t* v_codes,
                            const void* v_alpha, const void* v_scale, cq_layout v_layout, int B,
                            int Hq, int Hkv, int n, int d, int bits, float softmax_scale,
                            cq_calib calib, void* out, void* workspace, size_t ws_bytes,
                            int* status, unsigned wait_probes, cq_stream_t stream);

/*
 * Name of the kernel that cq_decode_attn launches for these layouts and sizes
 * on the current device, or NULL when the call would not launch one (invalid
 * or unsupported arguments). Host-only; reads the device's SM count once.
 *   1 bit, octet layouts: "k_decode_row" (one CTA per (sequence, kv-head) row,
 *     two per SM, n <= 8192), "k_decode_mma" (a cluster of CTAs per row,
 *     n <= 32768) or "k_decode_octet" (tcgen05, n <= 65536). Between the
 *     first two the library takes the one with the smaller estimated step
 *     time for B * Hkv rows of n tokens (an estimate fitted to measurements on
 *     B200: the row kernel for long rows and full waves of two rows per SM,
 *     the cluster kernel for short rows and for batches that leave the row
 *     kernel a thin last wave); the tcgen05 kernel takes longer rows.
 *     cq_set_decode_kernel, else the environment variable
 *     CALIBQ_DECODE_KERNEL = pipe | row | cluster | tcgen05 (read once per process),
 *     forces one of them wherever it supports n. "k_decode_tc" (pipe: one
 *     persistent CTA per SM working through whole rows, n <= 8192, plain
 *     decodes, its warps feeding 5th-generation tensor-core MMAs) is chosen
 *     only when forced.
 *   2, 4, 8 bits, octet layouts: "k_decode_ring".
 *   Canonical layouts: "k_scores + k_softmax_v + k_merge" (three launches).
 * The returned string is static; the caller does not free it.
 */
const char* cq_decode_kernel_name(cq_layout k_layout, cq_layout v_layout, int B, int Hq, int Hkv, int n, int d,
                                  int bits);

/*
 * Number of kernel launches that cq_decode_attn (n_text = 0) or
 * cq_decode_attn_mixed (n_text > 0 text tokens) makes for these arguments on
 * the current device, or 0 when the call would launch none. Host-only.
 *   canonical layouts: 3; octet layouts: 1 per call, except that a mixed
 *   call hands the text tokens to a second kernel unless the row kernel takes
 *   them, and that a plain 1-bit call on the row kernel with more than two
 *   waves of rows (two rows per SM) runs the rows beyond a whole number of SM
 *   counts, when they are at most half the SM count, as half rows on 2-CTA
 *   clusters in a second launch on the same stream (a programmatic dependent
 *   launch: it overlaps the whole rows, and reads or writes nothing of theirs).
 *   No call creates streams or events; every call can be captured into a
 *   CUDA graph, the first one of a process included.
 */
int cq_decode_launch_count(cq_layout k_layout, cq_layout v_layout, int B, int Hq, int Hkv, int n, int d, int bits,
                           int n_text);

/* 1-bit octet-layout decode kernels, for cq_set_decode_kernel. */
typedef enum cq_decode_kernel {
  CQ_KERNEL_ENV = -1,     /* CALIBQ_DECODE_KERNEL decides, else the estimate (the initial state) */
  CQ_KERNEL_AUTO = 0,     /* the estimate decides, whatever the environment says */
  CQ_KERNEL_ROW = 1,      /* "k_decode_row" wherever n <= 8192 */
  CQ_KERNEL_CLUSTER = 2,  /* "k_decode_mma" wherever n <= 32768 */
  CQ_KERNEL_TCGEN05 = 3,  /* "k_decode_octet" (plain decodes; mixed calls choose as with AUTO) */
  CQ_KERNEL_PIPE = 4      /* "k_decode_tc" (plain decodes with n <= 8192; others choose as with AUTO) */
} cq_decode_kernel;

/*
 * Force (or stop forcing) the 1-bit octet-layout decode kernel for every later
 * cq_decode_attn, cq_decode_attn_mixed and cq_decode_kernel_name call of the
 * process. A forced kernel that does not support a call's n falls back to the
 * estimate. The kernels' outputs agree within the output tolerance, not bit
 * for bit. Host-only; takes effect for calls made after it returns (a call
 * racing with it on another thread may use either choice).
 * Returns CQ_ERR_INVALID_ARG for a value outside cq_decode_kernel.
 */
cq_status cq_set_decode_kernel(cq_decode_kernel which);

/*
 * Workspace of cq_decode_attn_mixed: the visual part's partial result
 * (B * Hq * d floats) and its log-sum-exps (B * Hq floats).
 */
cq_status cq_decode_attn_mixed_workspace_size(int B, int Hq, int d, size_t* bytes);

/*
 * One decode step over a mixed cache: n_vis quantized visual tokens (the
 * article quantizes the visual KV cache) followed by n_text full-precision
 * text tokens, in one softmax:
 *
 *   x_i = sigma * ( q . alpha_K + (q (.) s_K) . c^K_i )   visual logits (Method 2)
 *   y_i = g(x_i), g fitted to the range of the visual logits only (Method 3)
 *   z_j = sigma * q . k_j                                 text logits, not calibrated
 *   o   = ( sum_i e^{y_i} (alpha_V + s_V (.) c^V_i) + sum_j e^{z_j} v_j )
 *         / ( sum_i e^{y_i} + sum_j e^{z_j} )
 *
 * (Which tokens the calibration sees, and that g's constant term is kept so
 * that visual and text logits share one scale, is this library's reading; the
 * article applies g to the scores of the quantized cache.)
 *
 *   visual codes: k_codes in CQ_LAYOUT_OCTET_K, v_codes in CQ_LAYOUT_OCTET_V,
 *     bits in {1, 2, 4, 8}, statistics [B][Hkv][d] in `dt`;
 *   k_text, v_text: [B][Hkv][n_text][d] in `dt` (may be NULL when n_text = 0);
 *   q, out: [B][Hq][d] in `dt`; Hq = 4 * Hkv; d = 128;
 *   n_vis <= 32768; workspace: cq_decode_attn_mixed_workspace_size bytes.
 * With 1-bit codes, when cq_decode_kernel_name names "k_decode_row", one
 * launch on `stream`: that kernel attends the text tokens after the visual
 * ones (f16 keys and values on the tensor cores, probabilities rounded to f16
 * for the value product; f32 on the CUDA cores). Otherwise two launches
 * (visual partial result into the workspace, then text + merge). The
 * workspace is required in both cases.
 */
cq_status cq_decode_attn_mixed(const void* q, cq_dtype dt, const uint8_t* k_codes, const void* k_alpha,
                               const void* k_scale, const uint8_t* v_codes, const void* v_alpha,
                               const void* v_scale, int n_vis, int bits, const void* k_text,
                               const void* v_text, int n_text, int B, int Hq, int Hkv, int d,
                               float softmax_scale, cq_calib calib, void* out, void* workspace,
                               size_t ws_bytes, cq_stream_t stream);

/*
 * Dequantize packed codes back to floating point (for checks only):
 *   out[b][h][i][j] = alpha[b][h][j] + scale[b][h][j] * code(i, j),
 * evaluated in double and rounded once to `dt`.
 *   out [B][H][n][d] in `dt`.
 */
cq_status cq_dequant(const uint8_t* codes, const void* alpha, const void* scale, cq_dtype dt,
                     cq_layout layout, int B, int H, int n, int d, int bits, void* out,
                     cq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* CALIBQ_H */
