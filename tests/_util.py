"""Shared helpers for the GPU parity tests (comparison rules, oracle calls)."""

import numpy as np
import torch

import oracle

# Spec tolerance on attention outputs: per (batch, query-head) row,
# max_j |o_gpu - o_ref| / max_j |o_ref| <= 2e-3.
OUT_RTOL = 2e-3

DT = {torch.float16: "f16", torch.float32: "f32"}


def row_rel_err(out_gpu, out_ref):
    """max over rows of max_j |diff| / max_j |ref| (rows = all leading dims)."""
    g = np.asarray(out_gpu, dtype=np.float64)
    r = np.asarray(out_ref, dtype=np.float64)
    num = np.abs(g - r).max(axis=-1)
    den = np.abs(r).max(axis=-1)
    return float((num / np.maximum(den, 1e-30)).max())


def ref_output_rounded(out_ref, torch_dtype):
    """The fp64 oracle output rounded once to the output dtype (the GPU's storage)."""
    npd = np.float16 if torch_dtype == torch.float16 else np.float32
    return out_ref.astype(npd).astype(np.float64)


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def oracle_quantize(x_cpu_tensor, bits):
    return oracle.quantize_cache(f64(x_cpu_tensor), bits, DT[x_cpu_tensor.dtype])
