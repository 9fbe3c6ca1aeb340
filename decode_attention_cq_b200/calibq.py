"""Thin ctypes binding of libcalibq (argument marshalling only).

Every function here has the name of the C entry point it calls and does no
arithmetic of the method: it allocates output tensors with torch (device
memory), passes raw pointers, the current torch stream and sizes, and raises
``CalibqError`` on any non-OK status. All compute runs in the CUDA kernels of
``lib/libcalibq.so``; when that library is missing the import of any function
fails loudly -- there is no CPU fallback.
"""

from __future__ import annotations

import ctypes
import functools
import os
from dataclasses import dataclass

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "lib", "libcalibq.so")

CQ_OK, CQ_ERR_INVALID_ARG, CQ_ERR_UNSUPPORTED, CQ_ERR_WORKSPACE, CQ_ERR_CUDA = range(5)
CQ_F16, CQ_F32 = 0, 1
LAYOUT_CANONICAL, LAYOUT_OCTET_K, LAYOUT_OCTET_V = 0, 1, 2
KERNEL_ENV, KERNEL_AUTO, KERNEL_ROW, KERNEL_CLUSTER, KERNEL_TCGEN05, KERNEL_PIPE = -1, 0, 1, 2, 3, 4

ENTRY_POINTS = (
    "cq_version",
    "cq_status_string",
    "cq_codes_bytes",
    "cq_quantize_kv_workspace_size",
    "cq_quantize_kv",
    "cq_quantize_kv_noalloc",
    "cq_decode_attn_workspace_size",
    "cq_decode_kernel_name",
    "cq_set_decode_kernel",
    "cq_decode_launch_count",
    "cq_decode_attn",
    "cq_decode_attn_ex",
    "cq_decode_attn_mixed_workspace_size",
    "cq_decode_attn_mixed",
    "cq_dequant",
)


class CalibqError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)}")


class cq_calib(ctypes.Structure):
    _fields_ = [("enabled", ctypes.c_int), ("tau_lo", ctypes.c_float), ("tau_hi", ctypes.c_float)]


_P, _I, _SZ, _F = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
_SIGS = {
    "cq_version": ([], _I),
    "cq_status_string": ([_I], ctypes.c_char_p),
    "cq_codes_bytes": ([_I, _I, _I, _I, _I, _I, ctypes.POINTER(_SZ)], _I),
    "cq_quantize_kv_workspace_size": ([_I, _I, _I, _I, ctypes.POINTER(_SZ)], _I),
    "cq_quantize_kv": ([_P, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _SZ, _P], _I),
    "cq_quantize_kv_noalloc": ([_P, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P], _I),
    "cq_decode_attn_workspace_size": ([_I, _I, _I, _I, _I, _I, _I, _I, ctypes.POINTER(_SZ)], _I),
    "cq_decode_kernel_name": ([_I, _I, _I, _I, _I, _I, _I, _I], ctypes.c_char_p),
    "cq_set_decode_kernel": ([_I], _I),
    "cq_decode_launch_count": ([_I, _I, _I, _I, _I, _I, _I, _I, _I], _I),
    "cq_decode_attn": ([_P, _I, _P, _P, _P, _I, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F,
                        cq_calib, _P, _P, _SZ, _P], _I),
    "cq_decode_attn_ex": ([_P, _I, _P, _P, _P, _I, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F,
                           cq_calib, _P, _P, _SZ, _P, ctypes.c_uint, _P], _I),
    "cq_decode_attn_mixed_workspace_size": ([_I, _I, _I, ctypes.POINTER(_SZ)], _I),
    "cq_decode_attn_mixed": ([_P, _I, _P, _P, _P, _P, _P, _P, _I, _I, _P, _P, _I, _I, _I, _I, _I, _F,
                              cq_calib, _P, _P, _SZ, _P], _I),
    "cq_dequant": ([_P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _P, _P], _I),
}

_lib = None


def load() -> ctypes.CDLL:
    """Load libcalibq.so once (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libcalibq is not built ({LIB_PATH} missing); "
                              "run `python -m decode_attention_cq_b200.build_lib`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGS.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = res
        _lib = lib
    return _lib


def status_string(status: int) -> str:
    return load().cq_status_string(status).decode()


def _check(status: int, what: str):
    if status != CQ_OK:
        raise CalibqError(status, what)


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.float16:
        return CQ_F16
    if t.dtype == torch.float32:
        return CQ_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(stream, t: torch.Tensor | None = None) -> int:
    """The stream handle to launch on: `stream`, else the current stream of
    t's device (of the current device without t)."""
    if stream is not None:
        return stream.cuda_stream
    if _raw_stream is not None and t is not None and t.is_cuda:
        return _raw_stream(t.get_device())
    return torch.cuda.current_stream().cuda_stream


@functools.lru_cache(maxsize=64)
def _calib(enabled: bool, tau_lo: float, tau_hi: float) -> "cq_calib":
    # passed by value: one instance per distinct setting can be shared
    return cq_calib(int(enabled), tau_lo, tau_hi)


@dataclass
class QuantizedCache:
    """Packed codes plus stored per-channel alpha and step of one cache tensor."""

    codes: torch.Tensor  # uint8 [B, H, row_bytes]
    alpha: torch.Tensor  # [B, H, d] in the input dtype
    scale: torch.Tensor  # [B, H, d] in the input dtype
    layout: int
    bits: int
    n: int

    @property
    def shape(self):
        B, H, d = self.alpha.shape
        return B, H, self.n, d


def cq_version() -> int:
    return load().cq_version()


def cq_codes_bytes(layout: int, B: int, H: int, n: int, d: int, bits: int) -> int:
    out = ctypes.c_size_t(0)
    _check(load().cq_codes_bytes(layout, B, H, n, d, bits, ctypes.byref(out)), "cq_codes_bytes")
    return out.value


def cq_quantize_kv_workspace_size(B: int, H: int, n: int, d: int) -> int:
    out = ctypes.c_size_t(0)
    _check(load().cq_quantize_kv_workspace_size(B, H, n, d, ctypes.byref(out)),
           "cq_quantize_kv_workspace_size")
    return out.value


def cq_quantize_kv(x: torch.Tensor, bits: int, layout: int = LAYOUT_CANONICAL, *,
                   out: QuantizedCache | None = None, workspace: torch.Tensor | None = None,
                   stream=None) -> QuantizedCache:
    """Quantize one [B, H, n, d] cache tensor; returns (codes, alpha, scale)."""
    B, H, n, d = x.shape
    if out is None:
        nbytes = cq_codes_bytes(layout, B, H, n, d, bits)
        out = QuantizedCache(
            codes=torch.empty(B, H, nbytes // (B * H), dtype=torch.uint8, device=x.device),
            alpha=torch.empty(B, H, d, dtype=x.dtype, device=x.device),
            scale=torch.empty(B, H, d, dtype=x.dtype, device=x.device),
            layout=layout, bits=bits, n=n)
    if workspace is None:
        ws = cq_quantize_kv_workspace_size(B, H, n, d)
        workspace = torch.empty(max(ws, 1), dtype=torch.uint8, device=x.device)
    _check(load().cq_quantize_kv(_ptr(x), _dt(x), B, H, n, d, bits, layout, _ptr(out.codes),
                                 _ptr(out.alpha), _ptr(out.scale), _ptr(workspace),
                                 workspace.numel(), _stream(stream, x)), "cq_quantize_kv")
    return out


def cq_quantize_kv_noalloc(x: torch.Tensor, bits: int, layout: int = LAYOUT_CANONICAL, *,
                           out: QuantizedCache | None = None, stream=None) -> QuantizedCache:
    """cq_quantize_kv with the library's fixed scratch instead of a workspace
    (for callers that cannot allocate device memory; see include/calibq.h)."""
    B, H, n, d = x.shape
    if out is None:
        nbytes = cq_codes_bytes(layout, B, H, n, d, bits)
        out = QuantizedCache(
            codes=torch.empty(B, H, nbytes // (B * H), dtype=torch.uint8, device=x.device),
            alpha=torch.empty(B, H, d, dtype=x.dtype, device=x.device),
            scale=torch.empty(B, H, d, dtype=x.dtype, device=x.device),
            layout=layout, bits=bits, n=n)
    _check(load().cq_quantize_kv_noalloc(_ptr(x), _dt(x), B, H, n, d, bits, layout, _ptr(out.codes),
                                         _ptr(out.alpha), _ptr(out.scale), _stream(stream, x)),
           "cq_quantize_kv_noalloc")
    return out


def cq_decode_attn_workspace_size(k_layout: int, v_layout: int, B: int, Hq: int, Hkv: int, n: int,
                                  d: int, bits: int) -> int:
    out = ctypes.c_size_t(0)
    _check(load().cq_decode_attn_workspace_size(k_layout, v_layout, B, Hq, Hkv, n, d, bits,
                                                ctypes.byref(out)), "cq_decode_attn_workspace_size")
    return out.value


def cq_decode_kernel_name(k_layout: int, v_layout: int, B: int, Hq: int, Hkv: int, n: int, d: int,
                          bits: int) -> str | None:
    """Name of the kernel cq_decode_attn launches for these arguments, or None."""
    name = load().cq_decode_kernel_name(k_layout, v_layout, B, Hq, Hkv, n, d, bits)
    return None if name is None else name.decode()


def cq_decode_launch_count(k_layout: int, v_layout: int, B: int, Hq: int, Hkv: int, n: int, d: int,
                           bits: int, n_text: int = 0) -> int:
    """Kernel launches of one cq_decode_attn (n_text = 0) or cq_decode_attn_mixed
    call for these arguments (0: none)."""
    return load().cq_decode_launch_count(k_layout, v_layout, B, Hq, Hkv, n, d, bits, n_text)


def cq_set_decode_kernel(which: int) -> None:
    """Force a 1-bit octet decode kernel for the rest of the process
    (KERNEL_PIPE / KERNEL_ROW / KERNEL_CLUSTER / KERNEL_TCGEN05), let the estimate decide
    (KERNEL_AUTO), or go back to the environment (KERNEL_ENV)."""
    _check(load().cq_set_decode_kernel(int(which)), "cq_set_decode_kernel")


def cq_decode_attn(q: torch.Tensor, k: QuantizedCache, v: QuantizedCache, *,
                   calib=(False, 1.0, 1.0), softmax_scale: float = 0.0,
                   out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                   stream=None) -> torch.Tensor:
    """One decode step over packed K/V; returns out [B, Hq, d] in q's dtype."""
    B, Hq, d = q.shape
    _, Hkv, n, _ = k.shape
    if out is None:
        out = torch.empty_like(q)
    if workspace is None and k.layout == LAYOUT_CANONICAL:  # the octet path takes none
        ws = cq_decode_attn_workspace_size(k.layout, v.layout, B, Hq, Hkv, n, d, k.bits)
        workspace = torch.empty(ws, dtype=torch.uint8, device=q.device) if ws else None
    cal = _calib(bool(calib[0]), float(calib[1]), float(calib[2]))
    _check(load().cq_decode_attn(_ptr(q), _dt(q), _ptr(k.codes), _ptr(k.alpha), _ptr(k.scale),
                                 k.layout, _ptr(v.codes), _ptr(v.alpha), _ptr(v.scale), v.layout,
                                 B, Hq, Hkv, n, d, k.bits, float(softmax_scale), cal, _ptr(out),
                                 _ptr(workspace), 0 if workspace is None else workspace.numel(),
                                 _stream(stream, q)), "cq_decode_attn")
    return out


DEVICE_WAIT_TIMEOUT = 1  # bit of the device status word (CQ_DEVICE_WAIT_TIMEOUT)


def cq_decode_attn_ex(q: torch.Tensor, k: QuantizedCache, v: QuantizedCache, status: torch.Tensor, *,
                      wait_probes: int = 0, calib=(False, 1.0, 1.0), softmax_scale: float = 0.0,
                      out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                      stream=None) -> torch.Tensor:
    """cq_decode_attn that ORs DEVICE_WAIT_TIMEOUT into `status` (an int32
    device tensor the caller zeroes) when a kernel's bounded wait ran out;
    wait_probes > 0 bounds the cluster kernel's copy waits to that many probes."""
    B, Hq, d = q.shape
    _, Hkv, n, _ = k.shape
    if out is None:
        out = torch.empty_like(q)
    if workspace is None and k.layout == LAYOUT_CANONICAL:  # the octet path takes none
        ws = cq_decode_attn_workspace_size(k.layout, v.layout, B, Hq, Hkv, n, d, k.bits)
        workspace = torch.empty(ws, dtype=torch.uint8, device=q.device) if ws else None
    if status.dtype != torch.int32 or not status.is_cuda:
        raise ValueError("status must be an int32 CUDA tensor")
    cal = _calib(bool(calib[0]), float(calib[1]), float(calib[2]))
    _check(load().cq_decode_attn_ex(_ptr(q), _dt(q), _ptr(k.codes), _ptr(k.alpha), _ptr(k.scale),
                                    k.layout, _ptr(v.codes), _ptr(v.alpha), _ptr(v.scale), v.layout,
                                    B, Hq, Hkv, n, d, k.bits, float(softmax_scale), cal, _ptr(out),
                                    _ptr(workspace), 0 if workspace is None else workspace.numel(),
                                    _ptr(status), int(wait_probes), _stream(stream, q)), "cq_decode_attn_ex")
    return out


def cq_decode_attn_mixed_workspace_size(B: int, Hq: int, d: int) -> int:
    out = ctypes.c_size_t()
    _check(load().cq_decode_attn_mixed_workspace_size(B, Hq, d, ctypes.byref(out)),
           "cq_decode_attn_mixed_workspace_size")
    return out.value


def cq_decode_attn_mixed(q: torch.Tensor, k: QuantizedCache, v: QuantizedCache,
                         k_text: torch.Tensor | None, v_text: torch.Tensor | None, *,
                         calib=(False, 1.0, 1.0), softmax_scale: float = 0.0,
                         out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                         stream=None) -> torch.Tensor:
    """Decode over quantized visual K/V (octet layouts) followed by full-precision
    text K/V [B, Hkv, n_text, d] in q's dtype (None or n_text = 0 for none)."""
    B, Hq, d = q.shape
    _, Hkv, n, _ = k.shape
    n_text = 0 if k_text is None else k_text.shape[2]
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = torch.empty(cq_decode_attn_mixed_workspace_size(B, Hq, d), dtype=torch.uint8,
                                device=q.device)
    cal = _calib(bool(calib[0]), float(calib[1]), float(calib[2]))
    _check(load().cq_decode_attn_mixed(_ptr(q), _dt(q), _ptr(k.codes), _ptr(k.alpha), _ptr(k.scale),
                                       _ptr(v.codes), _ptr(v.alpha), _ptr(v.scale), n, k.bits,
                                       _ptr(k_text), _ptr(v_text), n_text, B, Hq, Hkv, d,
                                       float(softmax_scale), cal, _ptr(out), _ptr(workspace),
                                       workspace.numel(), _stream(stream, q)), "cq_decode_attn_mixed")
    return out


def cq_dequant(cache: QuantizedCache, *, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """codes -> alpha + step * code as [B, H, n, d] (checks only)."""
    B, H, n, d = cache.shape
    if out is None:
        out = torch.empty(B, H, n, d, dtype=cache.alpha.dtype, device=cache.alpha.device)
    _check(load().cq_dequant(_ptr(cache.codes), _ptr(cache.alpha), _ptr(cache.scale),
                             _dt(cache.alpha), cache.layout, B, H, n, d, cache.bits, _ptr(out),
                             _stream(stream, cache.codes)), "cq_dequant")
    return out
