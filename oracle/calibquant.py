"""CalibQuant quantize -> dequantize -> attend, in float64 on the CPU.

TEST INFRASTRUCTURE ONLY (see the package docstring). Array conventions:

* a cache tensor X is ``[B, H, n, d]`` (batch, kv-head, token, channel);
* a query tensor q is ``[B, Hq, d]`` with ``Hq = G * Hkv``;
* per-channel statistics are ``[B, H, d]``;
* codes are int64 arrays ``[B, H, n, d]`` with values in ``{0 .. 2^b - 1}``
  (bit packing lives in ``layouts.py``).

All arithmetic is IEEE float64 unless a step says otherwise.
"""

from __future__ import annotations

import numpy as np

__all__ = [
    "levels",
    "channel_stats",
    "quantize_codes",
    "stored_stats",
    "dequantize",
    "scores_dequantized",
    "scores_post_scaled",
    "calibrate",
    "softmax",
    "attend_dequantized",
    "attend_post_scaled",
    "quantize_cache",
    "decode_attention",
    "decode_attention_mixed",
]

_STORE = {"f16": np.float16, "f32": np.float32}


def _f64(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


def levels(bits: int) -> int:
    """Largest code L = 2^b - 1 of b-bit uniform quantization (Method 1)."""
    if bits not in (1, 2, 4, 8):
        raise ValueError(f"bits must be 1, 2, 4 or 8, got {bits}")
    return (1 << bits) - 1


def channel_stats(x):
    """Per-channel range of one cache matrix (Method 1).

    For each (batch, kv-head) the cache is a matrix K in R^{n x d}; the article
    refines the range [alpha, beta] per channel instead of using one global
    range: alpha_j = min_i K_ij and beta_j = max_i K_ij over the n tokens.

    x: ``[..., n, d]`` -> (alpha, beta), each ``[..., d]`` float64. Both are
    input values, so they are exact.
    """
    x = _f64(x)
    if x.shape[-2] < 1:
        raise ValueError("need at least one token")
    return x.min(axis=-2), x.max(axis=-2)


def quantize_codes(x, alpha, beta, bits: int):
    """b-bit integer codes of x in [alpha, beta] (Method 1).

    The article maps x to the integer round((x - alpha) / (beta - alpha) *
    (2^b - 1)) with a round-to-nearest operator. Readings taken where the page
    is silent:

    * ties go to the even integer (IEEE default);
    * a constant channel (beta == alpha, e.g. n == 1) gets code 0;
    * the rounding decision is taken on r = ((x - alpha) * L) / (beta - alpha)
      with each operation in IEEE float64 round-to-nearest-even. For fp16
      inputs every step before the divide is exact and the divide cannot land
      on a tie unless the real quotient is one, so this equals rounding the
      exact real quotient (pinned against exact rationals in the tests).

    x: ``[..., n, d]``; alpha, beta: ``[..., d]`` -> int64 codes ``[..., n, d]``.
    """
    L = levels(bits)
    x = _f64(x)
    a = _f64(alpha)[..., None, :]
    b = _f64(beta)[..., None, :]
    rng = b - a
    num = (x - a) * L
    with np.errstate(divide="ignore", invalid="ignore"):
        r = num / rng
    c = np.rint(np.where(rng > 0, r, 0.0))  # np.rint rounds half to even
    return np.clip(c, 0, L).astype(np.int64)


def stored_stats(alpha, beta, bits: int, dtype: str):
    """Per-channel offset and step as stored beside the codes (Method 2).

    The quantized cache is represented by integers plus a per-channel scale
    factor and bias term. Readings: the bias is alpha itself (stored exactly:
    it is an input value), the scale is the step s = (beta - alpha) / L rounded
    once to the storage dtype, and the storage dtype is the input's dtype.

    Returns (alpha_stored, s_stored) as numpy arrays of the storage dtype.
    """
    L = levels(bits)
    st = _STORE[dtype]
    a = _f64(alpha)
    s = (_f64(beta) - a) / L
    return a.astype(st), s.astype(st)


def dequantize(codes, alpha_s, s_s):
    """x_hat = alpha + s * c with the stored per-channel alpha and s (Method 2).

    codes: ``[..., n, d]``; alpha_s, s_s: ``[..., d]`` -> float64 ``[..., n, d]``.
    """
    return _f64(alpha_s)[..., None, :] + _f64(s_s)[..., None, :] * _f64(codes)


def _group_kv(kv, hq: int):
    """Repeat kv-heads so query head h reads kv-head h // G (reading: GQA)."""
    hkv = kv.shape[1]
    if hq % hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    return np.repeat(kv, hq // hkv, axis=1)


def _sigma(d: int, softmax_scale: float) -> float:
    return 1.0 / np.sqrt(d) if softmax_scale == 0 else float(softmax_scale)


def scores_dequantized(q, k_hat, softmax_scale: float = 0.0):
    """Attention logits of one decode step on the dequantized K cache.

    x_i = sigma * <q, k_hat_i> for every token i (the generation-time attention
    of Method 2, written before the reordering). sigma = 1/sqrt(d) by default
    (reading: the standard scale). Query head h reads kv-head h // G.

    q: ``[B, Hq, d]``; k_hat: ``[B, Hkv, n, d]`` -> ``[B, Hq, n]``.
    """
    q = _f64(q)
    k = _group_kv(_f64(k_hat), q.shape[1])
    return _sigma(q.shape[-1], softmax_scale) * np.einsum("bhd,bhnd->bhn", q, k)


def scores_post_scaled(q, codes, alpha_s, s_s, softmax_scale: float = 0.0):
    """The same logits in the post-scaled order of Method 2.

    <q, alpha + s (.) c> = <q, alpha> + <q (.) s, c>: the per-channel
    dequantization is folded into the query once per step, and the product is
    taken against the integer codes directly.
    """
    q = _f64(q)
    hq = q.shape[1]
    c = _group_kv(_f64(codes), hq)
    a = _group_kv(_f64(alpha_s)[:, :, None, :], hq)[:, :, 0, :]
    s = _group_kv(_f64(s_s)[:, :, None, :], hq)[:, :, 0, :]
    sig = _sigma(q.shape[-1], softmax_scale)
    bias = np.einsum("bhd,bhd->bh", q, a)
    w = q * s
    return sig * (bias[..., None] + np.einsum("bhd,bhnd->bhn", w, c))


def calibrate(x, tau_lo: float, tau_hi: float):
    """Post-quantization calibration g of the pre-softmax scores (Method 3).

    With every entry of a score row in [m, M] (m = min, M = max over the
    row's n tokens), g is the linear map sending [m, M] onto the target
    interval; the row is replaced by g(x). Reading (the interval was lost from
    the page): the target is [tau_lo * m, tau_hi * M], i.e.

        g(x) = tau_lo * m + (x - m) * (tau_hi * M - tau_lo * m) / (M - m).

    (tau_lo, tau_hi) = (1, 1) is the identity. A row with M == m is left as is.

    x: ``[..., n]`` -> same shape.
    """
    x = _f64(x)
    m = x.min(axis=-1, keepdims=True)
    M = x.max(axis=-1, keepdims=True)
    span = M - m
    with np.errstate(divide="ignore", invalid="ignore"):
        y = tau_lo * m + (x - m) * (tau_hi * M - tau_lo * m) / span
    return np.where(span > 0, y, x)


def softmax(y):
    """Row softmax p_i = exp(y_i - max y) / sum_j exp(y_j - max y)."""
    y = _f64(y)
    e = np.exp(y - y.max(axis=-1, keepdims=True))
    return e / e.sum(axis=-1, keepdims=True)


def attend_dequantized(p, v_hat):
    """o = sum_i p_i v_hat_i on the dequantized V cache.

    p: ``[B, Hq, n]``; v_hat: ``[B, Hkv, n, d]`` -> ``[B, Hq, d]``.
    """
    v = _group_kv(_f64(v_hat), p.shape[1])
    return np.einsum("bhn,bhnd->bhd", _f64(p), v)


def attend_post_scaled(p, codes, alpha_s, s_s):
    """The same weighted sum in the post-scaled order of Method 2.

    sum_i p_i (alpha + s (.) c_i) = alpha * sum_i p_i + s (.) sum_i p_i c_i.
    """
    p = _f64(p)
    hq = p.shape[1]
    c = _group_kv(_f64(codes), hq)
    a = _group_kv(_f64(alpha_s)[:, :, None, :], hq)[:, :, 0, :]
    s = _group_kv(_f64(s_s)[:, :, None, :], hq)[:, :, 0, :]
    return a * p.sum(axis=-1)[..., None] + s * np.einsum("bhn,bhnd->bhd", p, c)


def quantize_cache(x, bits: int, dtype: str):
    """Method 1 on one cache tensor: statistics, codes, stored alpha and step.

    x: ``[B, H, n, d]`` -> dict(codes, alpha, scale, beta) where codes are
    int64 ``[B, H, n, d]`` and alpha/scale are in the storage dtype.
    """
    alpha, beta = channel_stats(x)
    codes = quantize_codes(x, alpha, beta, bits)
    a_s, s_s = stored_stats(alpha, beta, bits, dtype)
    return {"codes": codes, "alpha": a_s, "scale": s_s, "beta": beta}


def decode_attention(q, k, v, bits: int, dtype: str, calib=(False, 1.0, 1.0),
                     softmax_scale: float = 0.0, check_forms: bool = True):
    """One decode step of CalibQuant attention, end to end, in float64.

    q: ``[B, Hq, d]``; k, v: ``[B, Hkv, n, d]`` (the full-precision caches);
    calib: (enabled, tau_lo, tau_hi). Steps: quantize K and V channel-wise
    (Method 1), logits on the dequantized K (Method 2), calibration g per
    (batch, query head) row (Method 3) when enabled, softmax, weighted sum of
    the dequantized V.

    With ``check_forms`` the post-scaled orderings of Method 2 are evaluated
    as well and must agree with the dequantize-then-attend forms to 1e-12
    relative to the magnitude of the terms.

    Returns dict(out [B, Hq, d] float64, scores, y, p, kq, vq).
    """
    enabled, tau_lo, tau_hi = calib
    kq = quantize_cache(k, bits, dtype)
    vq = quantize_cache(v, bits, dtype)
    k_hat = dequantize(kq["codes"], kq["alpha"], kq["scale"])
    v_hat = dequantize(vq["codes"], vq["alpha"], vq["scale"])
    x = scores_dequantized(q, k_hat, softmax_scale)
    y = calibrate(x, tau_lo, tau_hi) if enabled else x
    p = softmax(y)
    out = attend_dequantized(p, v_hat)
    if check_forms:
        x2 = scores_post_scaled(q, kq["codes"], kq["alpha"], kq["scale"], softmax_scale)
        mag = _sigma(q.shape[-1], softmax_scale) * np.einsum(
            "bhd,bhnd->bhn", np.abs(_f64(q)), _group_kv(np.abs(k_hat), q.shape[1]))
        assert np.all(np.abs(x - x2) <= 1e-12 * (mag + 1e-300)), "post-scaled logits disagree"
        o2 = attend_post_scaled(p, vq["codes"], vq["alpha"], vq["scale"])
        vmag = attend_dequantized(p, np.abs(v_hat))
        assert np.all(np.abs(out - o2) <= 1e-12 * (vmag + 1e-300)), "post-scaled output disagrees"
    return {"out": out, "scores": x, "y": y, "p": p, "kq": kq, "vq": vq}


def decode_attention_mixed(q, k_vis, v_vis, k_text, v_text, bits: int, dtype: str,
                           calib=(False, 1.0, 1.0), softmax_scale: float = 0.0):
    """One decode step over a mixed cache: quantized visual tokens, then
    full-precision text tokens, in one softmax, in float64.

    The article quantizes the visual KV cache (Methods 1 and 2) and calibrates
    the scores of that quantized cache (Method 3). Reading for a cache that also
    holds text tokens: g is fitted to the range of the visual logits only and
    applied to them with its constant term (so visual and text logits share one
    scale); text logits sigma <q, k_j> are used as they are and their values
    as stored.

    q: ``[B, Hq, d]``; k_vis, v_vis: ``[B, Hkv, n_vis, d]`` (full precision,
    quantized here); k_text, v_text: ``[B, Hkv, n_text, d]``.
    Returns dict(out [B, Hq, d], p [B, Hq, n_vis + n_text]).
    """
    enabled, tau_lo, tau_hi = calib
    kq = quantize_cache(k_vis, bits, dtype)
    vq = quantize_cache(v_vis, bits, dtype)
    k_hat = dequantize(kq["codes"], kq["alpha"], kq["scale"])
    v_hat = dequantize(vq["codes"], vq["alpha"], vq["scale"])
    x = scores_dequantized(q, k_hat, softmax_scale)
    y = calibrate(x, tau_lo, tau_hi) if enabled else x
    z = scores_dequantized(q, k_text, softmax_scale)  # plain sigma <q, k_j>
    p = softmax(np.concatenate([y, z], axis=-1))
    n_vis = y.shape[-1]
    out = attend_dequantized(p[..., :n_vis], v_hat) + attend_dequantized(p[..., n_vis:], _f64(v_text))
    return {"out": out, "p": p}
