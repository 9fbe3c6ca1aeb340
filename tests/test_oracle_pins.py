"""Pins of the fp64 oracle against facts fixed outside the oracle itself.

Each test checks the oracle against something other than its own formulas:
exact rational arithmetic, hand-worked ties, a library attention routine,
closed forms, or invariants the CalibQuant article's method implies. They run
without a GPU.
"""

from fractions import Fraction
import os

import numpy as np
import pytest
import torch

import oracle
from decode_attention_cq_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _exact_code(x, a, b, bits):
    """Round-half-even of the exact real (x - a) * L / (b - a) with Fractions."""
    L = (1 << bits) - 1
    if b == a:
        return 0
    r = (Fraction(float(x)) - Fraction(float(a))) * L / (Fraction(float(b)) - Fraction(float(a)))
    return round(r)  # Fraction.__round__ rounds half to even


def _round_fraction(fr, np_dtype):
    """Single correctly-rounded (half-to-even) conversion of a Fraction to np_dtype."""
    c = np_dtype(float(fr))
    cands = {c, np.nextafter(c, np_dtype(np.inf)), np.nextafter(c, np_dtype(-np.inf))}
    best = None
    for v in cands:
        if not np.isfinite(v):
            continue
        err = abs(Fraction(float(v)) - fr)
        if best is None or err < best[0]:
            best = (err, v)
        elif err == best[0]:  # tie between two neighbours: pick the even significand
            bits_v = v.view(np.uint16 if np_dtype == np.float16 else np.uint32)
            if int(bits_v) % 2 == 0:
                best = (err, v)
    return best[1]


def _small_cache(dtype, seed, n=40, d=8, B=2, H=2):
    g = torch.Generator().manual_seed(seed)
    x = synth.make_cache(B, H, n, d, dtype, 1, g, "cpu")
    return x.to(torch.float64).numpy()


@pytest.mark.parametrize("bits", [1, 2, 4, 8])
@pytest.mark.parametrize("dtype", ["f16", "f32"])
def test_codes_match_exact_rationals(bits, dtype):
    x = _small_cache(dtype, seed=bits * 7 + (dtype == "f16"))
    alpha, beta = oracle.channel_stats(x)
    codes = oracle.quantize_codes(x, alpha, beta, bits)
    B, H, n, d = x.shape
    for bb in range(B):
        for h in range(H):
            for j in range(d):
                a, b = alpha[bb, h, j], beta[bb, h, j]
                for i in range(n):
                    assert codes[bb, h, i, j] == _exact_code(x[bb, h, i, j], a, b, bits)


@pytest.mark.parametrize("bits", [1, 2, 4, 8])
def test_codes_in_range_and_extremes_map_to_0_and_L(bits):
    x = _small_cache("f16", seed=100 + bits, n=300, d=16)
    alpha, beta = oracle.channel_stats(x)
    c = oracle.quantize_codes(x, alpha, beta, bits)
    L = (1 << bits) - 1
    assert c.min() >= 0 and c.max() <= L
    # the per-channel min maps to 0 and the max to L (2-bit codes are 0..3 etc.)
    amin = x.argmin(axis=2)
    amax = x.argmax(axis=2)
    for bb in range(x.shape[0]):
        for h in range(x.shape[1]):
            for j in range(x.shape[3]):
                assert c[bb, h, amin[bb, h, j], j] == 0
                assert c[bb, h, amax[bb, h, j], j] == L
    if bits == 2:
        assert set(np.unique(c)) == {0, 1, 2, 3}


def test_ties_from_golden_file():
    rows = []
    with open(os.path.join(GOLDEN, "ties.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                rows.append(line.split())
    assert len(rows) >= 15
    for bits, a, b, x, want in rows:
        bits, want = int(bits), int(want)
        col = np.array([float(a), float(b), float(x)])[None, None, :, None]
        al, be = oracle.channel_stats(col)
        c = oracle.quantize_codes(col, al, be, bits)
        assert c[0, 0, 2, 0] == want, (bits, a, b, x)


def test_constant_channel_and_single_token():
    x = np.zeros((1, 1, 5, 4))
    x[..., 1] = 3.25  # constant channel
    x[0, 0, :, 0] = np.arange(5)
    al, be = oracle.channel_stats(x)
    c = oracle.quantize_codes(x, al, be, 1)
    assert np.all(c[..., 1:] == 0)
    a_s, s_s = oracle.stored_stats(al, be, 1, "f32")
    assert s_s[0, 0, 1] == 0 and a_s[0, 0, 1] == np.float32(3.25)
    one = x[:, :, :1, :]
    al1, be1 = oracle.channel_stats(one)
    assert np.all(oracle.quantize_codes(one, al1, be1, 4) == 0)


@pytest.mark.parametrize("bits", [1, 2, 4, 8])
@pytest.mark.parametrize("dtype,npd", [("f16", np.float16), ("f32", np.float32)])
def test_stored_scale_is_single_rounding_of_exact_step(bits, dtype, npd):
    x = _small_cache(dtype, seed=300 + bits, n=64, d=16)
    al, be = oracle.channel_stats(x)
    a_s, s_s = oracle.stored_stats(al, be, bits, dtype)
    L = (1 << bits) - 1
    assert a_s.dtype == npd and s_s.dtype == npd
    assert np.array_equal(a_s.astype(np.float64), al)  # alpha is an input value
    for idx in np.ndindex(al.shape):
        exact = (Fraction(float(be[idx])) - Fraction(float(al[idx]))) / L
        assert s_s[idx] == _round_fraction(exact, npd), idx


@pytest.mark.parametrize("bits", [1, 2, 4, 8])
def test_dequantization_error_bound(bits):
    x = _small_cache("f16", seed=400 + bits, n=200, d=16)
    q = oracle.quantize_cache(x, bits, "f16")
    xh = oracle.dequantize(q["codes"], q["alpha"], q["scale"])
    L = (1 << bits) - 1
    s_exact = (q["beta"] - q["alpha"].astype(np.float64)) / L
    bound = s_exact / 2 + L * np.abs(q["scale"].astype(np.float64) - s_exact)
    assert np.all(np.abs(x - xh) <= bound[..., None, :] * (1 + 1e-12) + 1e-300)


def test_dequantize_closed_form():
    codes = np.array([[[[0, 1], [3, 2]]]])
    a = np.array([[[-1.0, 0.5]]])
    s = np.array([[[0.25, 2.0]]])
    xh = oracle.dequantize(codes, a, s)
    assert np.array_equal(xh, np.array([[[[-1.0, 2.5], [-0.25, 4.5]]]]))


def _case(B=2, Hq=8, Hkv=2, n=96, d=32, dtype="f16", seed=5):
    q, k, v = synth.make_case(B, Hq, Hkv, n, d, dtype, outliers=2, seed=seed)
    f = lambda t: t.to(torch.float64).numpy()
    return f(q), f(k), f(v)


@pytest.mark.parametrize("bits", [1, 2, 4])
def test_post_scaled_forms_equal_dequantized_forms(bits):
    q, k, v = _case()
    kq = oracle.quantize_cache(k, bits, "f16")
    vq = oracle.quantize_cache(v, bits, "f16")
    kh = oracle.dequantize(kq["codes"], kq["alpha"], kq["scale"])
    vh = oracle.dequantize(vq["codes"], vq["alpha"], vq["scale"])
    x1 = oracle.scores_dequantized(q, kh)
    x2 = oracle.scores_post_scaled(q, kq["codes"], kq["alpha"], kq["scale"])
    assert np.allclose(x1, x2, rtol=1e-12, atol=1e-12)
    p = oracle.softmax(x1)
    o1 = oracle.attend_dequantized(p, vh)
    o2 = oracle.attend_post_scaled(p, vq["codes"], vq["alpha"], vq["scale"])
    assert np.allclose(o1, o2, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("tau", [(1.0, 1.0), (0.8, 0.9), (1.0, 0.5), (0.5, 1.0)])
def test_calibration_sends_range_to_target_interval(tau):
    rng = np.random.default_rng(7)
    x = rng.normal(size=(3, 4, 50)) * 5 + 1
    y = oracle.calibrate(x, *tau)
    m, M = x.min(-1), x.max(-1)
    im, iM = x.argmin(-1), x.argmax(-1)
    ym = np.take_along_axis(y, im[..., None], -1)[..., 0]
    yM = np.take_along_axis(y, iM[..., None], -1)[..., 0]
    assert np.allclose(ym, tau[0] * m, rtol=0, atol=1e-12)
    assert np.allclose(yM, tau[1] * M, rtol=0, atol=1e-12)
    # linear: equal steps in x give equal steps in y
    xs = np.concatenate([m[..., None], (m + M)[..., None] / 2, M[..., None], x], -1)
    ys = oracle.calibrate(xs, *tau)
    assert np.allclose(ys[..., 1] - ys[..., 0], ys[..., 2] - ys[..., 1], atol=1e-10)
    if tau == (1.0, 1.0):
        assert np.allclose(y, x, atol=1e-12)


def test_calibration_of_constant_row_is_identity():
    x = np.full((1, 1, 7), 2.5)
    assert np.array_equal(oracle.calibrate(x, 0.8, 0.9), x)


def test_softmax_rows_sum_to_one_and_match_scipy():
    from scipy.special import softmax as sp_softmax
    rng = np.random.default_rng(3)
    y = rng.normal(size=(4, 5, 33)) * 30
    p = oracle.softmax(y)
    assert np.allclose(p.sum(-1), 1.0, atol=1e-14)
    assert np.allclose(p, sp_softmax(y, axis=-1), rtol=1e-12, atol=1e-300)


@pytest.mark.parametrize("bits", [1, 2])
@pytest.mark.parametrize("calib", [(False, 1, 1), (True, 0.8, 0.9), (True, 1.0, 0.5)])
def test_output_in_convex_hull_of_dequantized_values(bits, calib):
    q, k, v = _case(seed=11)
    r = oracle.decode_attention(q, k, v, bits, "f16", calib)
    a = np.repeat(r["vq"]["alpha"].astype(np.float64), 4, axis=1)
    s = np.repeat(r["vq"]["scale"].astype(np.float64), 4, axis=1)
    L = (1 << bits) - 1
    assert np.all(r["out"] >= a - 1e-12) and np.all(r["out"] <= a + L * s + 1e-12)
    assert np.allclose(r["p"].sum(-1), 1.0, atol=1e-13)


def test_single_token_returns_v():
    q, k, v = _case(n=1)
    r = oracle.decode_attention(q, k, v, 1, "f16", (True, 0.8, 0.9))
    assert np.array_equal(r["out"], np.repeat(v[:, :, 0, :], 4, axis=1))


def test_zero_query_gives_mean_of_dequantized_v():
    q, k, v = _case()
    r = oracle.decode_attention(np.zeros_like(q), k, v, 1, "f16", (True, 0.8, 0.9))
    vh = oracle.dequantize(r["vq"]["codes"], r["vq"]["alpha"], r["vq"]["scale"])
    assert np.allclose(r["out"], np.repeat(vh.mean(axis=2), 4, axis=1), rtol=1e-13, atol=1e-13)


def test_token_permutation_invariance():
    q, k, v = _case(seed=21)
    perm = np.random.default_rng(0).permutation(k.shape[2])
    r1 = oracle.decode_attention(q, k, v, 2, "f16", (True, 0.8, 0.9))
    r2 = oracle.decode_attention(q, k[:, :, perm], v[:, :, perm], 2, "f16", (True, 0.8, 0.9))
    assert np.allclose(r1["out"], r2["out"], rtol=1e-12, atol=1e-12)


def test_gqa_equals_mha_on_repeated_kv():
    q, k, v = _case(seed=31)
    G = q.shape[1] // k.shape[1]
    r1 = oracle.decode_attention(q, k, v, 1, "f16", (True, 0.8, 0.9))
    r2 = oracle.decode_attention(q, np.repeat(k, G, axis=1), np.repeat(v, G, axis=1), 1, "f16", (True, 0.8, 0.9))
    assert np.allclose(r1["out"], r2["out"], rtol=1e-13, atol=1e-13)
    # and the grouping is h -> h // G: swapping two kv-heads changes which query heads move
    k2, v2 = k[:, ::-1].copy(), v[:, ::-1].copy()
    r3 = oracle.decode_attention(q, k2, v2, 1, "f16", (True, 0.8, 0.9))
    assert not np.allclose(r1["out"][:, :G], r3["out"][:, :G])


@pytest.mark.parametrize("bits", [1, 4])
def test_uncalibrated_equals_library_sdpa_on_dequantized_cache(bits):
    q, k, v = _case(seed=41)
    r = oracle.decode_attention(q, k, v, bits, "f16", (False, 1, 1))
    kh = oracle.dequantize(r["kq"]["codes"], r["kq"]["alpha"], r["kq"]["scale"])
    vh = oracle.dequantize(r["vq"]["codes"], r["vq"]["alpha"], r["vq"]["scale"])
    G = q.shape[1] // k.shape[1]
    qt = torch.from_numpy(q)[:, :, None, :]
    kt = torch.from_numpy(np.repeat(kh, G, axis=1))
    vt = torch.from_numpy(np.repeat(vh, G, axis=1))
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt)[:, :, 0, :].numpy()
    assert np.allclose(r["out"], ref, rtol=1e-10, atol=1e-10)
    # tau = (1, 1) with calibration on is the same as off
    r11 = oracle.decode_attention(q, k, v, bits, "f16", (True, 1.0, 1.0))
    assert np.allclose(r11["out"], r["out"], rtol=1e-12, atol=1e-12)


def test_calibration_matches_library_sdpa_with_rescaled_logits():
    """g is affine with slope a, so softmax(g(x)) = softmax(a x) = SDPA with scale a*sigma."""
    q, k, v = _case(seed=51, B=1, Hq=4, Hkv=1)
    tau = (0.8, 0.9)
    r = oracle.decode_attention(q, k, v, 1, "f16", (True, *tau))
    x = r["scores"]
    m, M = x.min(-1), x.max(-1)
    a = (tau[1] * M - tau[0] * m) / (M - m)  # slope of the map [m, M] -> [tau_lo m, tau_hi M]
    kh = oracle.dequantize(r["kq"]["codes"], r["kq"]["alpha"], r["kq"]["scale"])
    vh = oracle.dequantize(r["vq"]["codes"], r["vq"]["alpha"], r["vq"]["scale"])
    for h in range(4):
        qt = torch.from_numpy(q[:, h:h + 1])[:, :, None, :]
        ref = torch.nn.functional.scaled_dot_product_attention(
            qt, torch.from_numpy(kh), torch.from_numpy(vh), scale=float(a[0, h]) / np.sqrt(q.shape[-1]))
        assert np.allclose(r["out"][:, h], ref[:, 0, 0].numpy(), rtol=1e-10, atol=1e-10)


def test_eight_bits_approach_exact_attention():
    q, k, v = _case(seed=61)
    r = oracle.decode_attention(q, k, v, 8, "f16", (False, 1, 1))
    G = q.shape[1] // k.shape[1]
    qt = torch.from_numpy(q)[:, :, None, :]
    exact = torch.nn.functional.scaled_dot_product_attention(
        qt, torch.from_numpy(np.repeat(k, G, 1)), torch.from_numpy(np.repeat(v, G, 1)))[:, :, 0].numpy()
    # bound: logits move by at most eps = sigma * sum |q_j| * (s_j/2 + 255 |s_j - s~_j|),
    # softmax weights by a factor within e^{+-2 eps}, values by s_V/2 + ...
    sk = np.repeat(r["kq"]["scale"].astype(np.float64), G, 1)
    eps = (np.abs(q) * sk).sum(-1) / np.sqrt(q.shape[-1])  # >= the bound above (s/2 + rounding < s)
    sv = np.repeat(r["vq"]["scale"].astype(np.float64), G, 1)
    vrange = np.repeat(np.abs(v).max(axis=2), G, 1)
    bound = (np.exp(2 * eps)[..., None] - 1) * vrange + sv
    assert np.all(np.abs(r["out"] - exact) <= bound)
    assert np.max(np.abs(r["out"] - exact)) < 0.05 * np.max(np.abs(exact))


def _text(seed, B, Hkv, n_text, d):
    g = torch.Generator().manual_seed(seed)
    return (synth.make_cache(B, Hkv, n_text, d, "f16", 0, g, "cpu").to(torch.float64).numpy(),
            synth.make_cache(B, Hkv, n_text, d, "f16", 0, g, "cpu").to(torch.float64).numpy())


def test_mixed_cache_without_text_is_plain_decode():
    q, k, v = _case(seed=71)
    kt = np.zeros((k.shape[0], k.shape[1], 0, k.shape[3]))
    for calib in ((False, 1, 1), (True, 0.8, 0.9)):
        r = oracle.decode_attention(q, k, v, 1, "f16", calib)
        rm = oracle.decode_attention_mixed(q, k, v, kt, kt, 1, "f16", calib)
        assert np.allclose(rm["out"], r["out"], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("bits", [1, 4])
def test_mixed_cache_matches_library_sdpa(bits):
    """Uncalibrated: textbook attention over [dequantized visual; text] tokens.
    Calibrated: the visual logits become a x + c (a = slope, c = the constant of
    the map [m, M] -> [tau_lo m, tau_hi M]), i.e. keys scaled by a and an additive
    mask c on the visual positions."""
    q, k, v = _case(seed=73, B=1, Hq=4, Hkv=1)
    kt, vt = _text(74, 1, 1, 17, q.shape[-1])
    r0 = oracle.decode_attention(q, k, v, bits, "f16", (False, 1, 1))
    kh = oracle.dequantize(r0["kq"]["codes"], r0["kq"]["alpha"], r0["kq"]["scale"])
    vh = oracle.dequantize(r0["vq"]["codes"], r0["vq"]["alpha"], r0["vq"]["scale"])
    d, n_vis = q.shape[-1], k.shape[2]
    sig = 1 / np.sqrt(d)
    rm = oracle.decode_attention_mixed(q, k, v, kt, vt, bits, "f16", (False, 1, 1))
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[:, :, None, :], torch.from_numpy(np.repeat(np.concatenate([kh, kt], 2), 4, 1)),
        torch.from_numpy(np.repeat(np.concatenate([vh, vt], 2), 4, 1)))[:, :, 0].numpy()
    assert np.allclose(rm["out"], ref, rtol=1e-10, atol=1e-10)
    tau = (0.8, 0.9)
    rc = oracle.decode_attention_mixed(q, k, v, kt, vt, bits, "f16", (True, *tau))
    x = sig * np.einsum("bhd,bnd->bhn", q, kh[:, 0])  # visual logits, every head
    m, M = x.min(-1), x.max(-1)
    a = (tau[1] * M - tau[0] * m) / (M - m)
    c = tau[0] * m - a * m
    for h in range(4):
        keys = np.concatenate([a[0, h] * kh[0, 0], kt[0, 0]], 0)[None, None]
        vals = np.concatenate([vh[0, 0], vt[0, 0]], 0)[None, None]
        mask = np.concatenate([np.full(n_vis, c[0, h]), np.zeros(kt.shape[2])])[None, None, None, :]
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q[:, h:h + 1])[:, :, None, :], torch.from_numpy(keys), torch.from_numpy(vals),
            attn_mask=torch.from_numpy(mask))
        assert np.allclose(rc["out"][0, h], ref[0, 0, 0].numpy(), rtol=1e-10, atol=1e-10)


def test_mixed_cache_duplicate_tokens_leave_attention_unchanged():
    """Text tokens equal to the dequantized visual tokens (calibration off):
    every token appears twice, which does not change the softmax average."""
    q, k, v = _case(seed=75)
    r = oracle.decode_attention(q, k, v, 2, "f16", (False, 1, 1))
    kh = oracle.dequantize(r["kq"]["codes"], r["kq"]["alpha"], r["kq"]["scale"])
    vh = oracle.dequantize(r["vq"]["codes"], r["vq"]["alpha"], r["vq"]["scale"])
    rm = oracle.decode_attention_mixed(q, k, v, kh, vh, 2, "f16", (False, 1, 1))
    assert np.allclose(rm["out"], r["out"], rtol=1e-12, atol=1e-12)
