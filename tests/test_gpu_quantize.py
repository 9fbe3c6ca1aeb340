"""GPU parity of cq_quantize_kv and cq_dequant against the fp64 oracle.

Codes, packed bytes (padding included), stored alpha and step must match the
oracle bit for bit; dequantized values must equal the oracle's float64
dequantization rounded once to the storage dtype.
"""

import numpy as np
import pytest
import torch

import oracle
from decode_attention_cq_b200 import calibq as cq
from decode_attention_cq_b200 import synth

from _util import f64, oracle_quantize

pytestmark = pytest.mark.gpu

LAYOUTS = {
    "canonical": cq.LAYOUT_CANONICAL,
    "octet_k": cq.LAYOUT_OCTET_K,
    "octet_v": cq.LAYOUT_OCTET_V,
}


def _cache(B, H, n, dtype, seed, outliers=2):
    g = torch.Generator().manual_seed(seed)
    return synth.make_cache(B, H, n, 128, dtype, outliers, g, "cpu")


def _check_quantized(x_cpu, qc, bits, layout):
    ref = oracle_quantize(x_cpu, bits)
    B, H, n, d = x_cpu.shape
    alpha = qc.alpha.cpu().numpy()
    scale = qc.scale.cpu().numpy()
    assert np.array_equal(alpha.view(np.uint8), ref["alpha"].view(np.uint8)), "alpha differs"
    assert np.array_equal(scale.view(np.uint8), ref["scale"].view(np.uint8)), "scale differs"
    packed = qc.codes.cpu().numpy()
    want = oracle.pack_codes(ref["codes"], layout, bits)
    assert packed.shape == want.shape
    if not np.array_equal(packed, want):
        got = oracle.unpack_codes(packed, layout, n, d, bits)
        bad = np.argwhere(got != ref["codes"])
        raise AssertionError(f"{len(bad)} codes differ, first at {bad[:5].tolist()}")
    return ref


@pytest.mark.parametrize("dtype", ["f16", "f32"])
@pytest.mark.parametrize("bits", [1, 2, 4, 8])
@pytest.mark.parametrize("n", [1, 7, 300, 1500])
def test_canonical_codes_bit_exact(cuda_device, dtype, bits, n):
    x = _cache(2, 3, n, dtype, seed=bits * 100 + n)
    qc = cq.cq_quantize_kv(x.to(cuda_device), bits, cq.LAYOUT_CANONICAL)
    torch.cuda.synchronize()
    _check_quantized(x, qc, bits, cq.LAYOUT_CANONICAL)


@pytest.mark.parametrize("dtype", ["f16", "f32"])
@pytest.mark.parametrize("layout", ["octet_k", "octet_v"])
@pytest.mark.parametrize("n", [1, 8, 9, 255, 256, 257, 1024, 2049, 3328])
def test_octet_codes_bit_exact(cuda_device, dtype, layout, n):
    x = _cache(2, 2, n, dtype, seed=n + 7)
    qc = cq.cq_quantize_kv(x.to(cuda_device), 1, LAYOUTS[layout])
    torch.cuda.synchronize()
    _check_quantized(x, qc, 1, LAYOUTS[layout])


@pytest.mark.parametrize("dtype", ["f16", "f32"])
@pytest.mark.parametrize("layout", ["octet_k", "octet_v"])
@pytest.mark.parametrize("bits", [2, 4, 8])
@pytest.mark.parametrize("n", [1, 3, 31, 33, 64, 65, 129, 1000, 2049])
def test_octet_multibit_codes_bit_exact(cuda_device, dtype, layout, bits, n):
    """b-bit octet layouts (8/b tokens per byte): ragged tails inside a byte
    group and inside a V tile of 256/b tokens."""
    x = _cache(2, 2, n, dtype, seed=1000 * bits + n)
    qc = cq.cq_quantize_kv(x.to(cuda_device), bits, LAYOUTS[layout])
    torch.cuda.synchronize()
    _check_quantized(x, qc, bits, LAYOUTS[layout])


def test_exact_ties_and_constant_channels(cuda_device):
    """Inputs that sit exactly on rounding ties and channels with beta == alpha."""
    n = 64
    x = torch.zeros(1, 2, n, 128, dtype=torch.float16)
    # channel c: values 0 .. 63 * step so (x - alpha) * L / range hits exact halves often
    for c in range(128):
        x[0, 0, :, c] = torch.arange(n, dtype=torch.float32) * (0.25 + (c % 5)) - (c % 7)
    x[0, 1] = 3.5  # every channel constant
    for bits in (1, 2, 4, 8):
        for layout in (cq.LAYOUT_CANONICAL, cq.LAYOUT_OCTET_K, cq.LAYOUT_OCTET_V):
            qc = cq.cq_quantize_kv(x.to(cuda_device), bits, layout)
            torch.cuda.synchronize()
            ref = _check_quantized(x, qc, bits, layout)
            assert np.all(ref["codes"][0, 1] == 0)


@pytest.mark.parametrize("layout", ["canonical", "octet_k", "octet_v"])
def test_dequant_matches_oracle(cuda_device, layout):
    bits_list = [1, 2, 4, 8]
    for dtype in ("f16", "f32"):
        for bits in bits_list:
            x = _cache(1, 2, 333, dtype, seed=bits + 3)
            qc = cq.cq_quantize_kv(x.to(cuda_device), bits, LAYOUTS[layout])
            got = cq.cq_dequant(qc).cpu()
            ref = oracle_quantize(x, bits)
            xh = oracle.dequantize(ref["codes"], ref["alpha"], ref["scale"])
            want = xh.astype(np.float16 if dtype == "f16" else np.float32)
            assert np.array_equal(got.numpy().view(np.uint8), want.view(np.uint8))


def test_full_size_sampled_rows(cuda_device):
    """The n=8192, batch-64 workload quantized whole on the GPU; sampled
    (batch, kv-head) rows checked bit-exactly against the oracle."""
    w = synth.WORKLOADS["internvl8b_n8192_b64"]
    q, k, v = synth.make_workload(w, device=cuda_device)
    for x, layout in ((k, cq.LAYOUT_OCTET_K), (v, cq.LAYOUT_OCTET_V)):
        qc = cq.cq_quantize_kv(x, 1, layout)
        torch.cuda.synchronize()
        for (b, h) in ((0, 0), (17, 3), (63, 7)):
            xr = x[b:b + 1, h:h + 1].cpu()
            sub = cq.QuantizedCache(qc.codes[b:b + 1, h:h + 1].contiguous(),
                                    qc.alpha[b:b + 1, h:h + 1].contiguous(),
                                    qc.scale[b:b + 1, h:h + 1].contiguous(), layout, 1, w.n)
            _check_quantized(xr, sub, 1, layout)
    del q, k, v
    torch.cuda.empty_cache()


@pytest.mark.parametrize("dtype", ["f16", "f32"])
def test_one_bit_midpoints_across_exponent_ranges(cuda_device, dtype):
    """1-bit codes decide x > (alpha + beta) / 2 exactly even when alpha + beta
    is not representable in float: channels span tiny to large magnitudes and
    most tokens sit on or next to the exact midpoint."""
    npd = np.float16 if dtype == "f16" else np.float32
    rng = np.random.default_rng(11)
    n, d = 96, 128
    x = np.zeros((1, 1, n, d), dtype=npd)
    for c in range(d):
        lo_mag = float(npd(2.0 ** rng.integers(-14, 0)))
        hi_mag = float(npd(rng.uniform(1.0, 6.0e4 if dtype == "f16" else 1.0e6)))
        a, b = npd(-lo_mag if c % 2 else lo_mag), npd(hi_mag)
        if a > b:
            a, b = b, a
        mid = (float(a) + float(b)) / 2.0  # exact in double
        m = npd(mid)
        around = [m]
        for _ in range(6):
            around.append(np.nextafter(around[-1], npd(np.inf), dtype=npd))
        below = [m]
        for _ in range(6):
            below.append(np.nextafter(below[-1], npd(-np.inf), dtype=npd))
        vals = [a, b] + around + below[1:]
        col = np.array(vals + list(rng.uniform(float(a), float(b), n - len(vals))), dtype=npd)
        x[0, 0, :, c] = col
    xt = torch.from_numpy(x)
    for layout in (cq.LAYOUT_CANONICAL, cq.LAYOUT_OCTET_K, cq.LAYOUT_OCTET_V):
        qc = cq.cq_quantize_kv(xt.to(cuda_device), 1, layout)
        torch.cuda.synchronize()
        _check_quantized(xt, qc, 1, layout)


@pytest.mark.parametrize("layout", ["canonical", "octet_k", "octet_v"])
@pytest.mark.parametrize("bits", [1, 2, 4, 8])
@pytest.mark.parametrize("n", [8192, 8193, 16384, 16385])
def test_codes_bit_exact_across_fill_limits(cuda_device, layout, bits, n):
    """Rows on both sides of the single-read fill's limits: 512-token tiles up
    to n = 8192, 1024-token tiles up to 16384, the two-pass statistics + pack
    path above. Codes, alpha and step bit for bit against the oracle."""
    x = _cache(1, 2, n, "f16", seed=n * 3 + bits)
    qc = cq.cq_quantize_kv(x.to(cuda_device), bits, LAYOUTS[layout])
    torch.cuda.synchronize()
    _check_quantized(x, qc, bits, LAYOUTS[layout])


@pytest.mark.parametrize("n", [8193, 16385])
def test_one_bit_f32_codes_across_fill_limits(cuda_device, n):
    x = _cache(1, 2, n, "f32", seed=n + 5)
    for layout in (cq.LAYOUT_OCTET_K, cq.LAYOUT_OCTET_V):
        qc = cq.cq_quantize_kv(x.to(cuda_device), 1, layout)
        torch.cuda.synchronize()
        _check_quantized(x, qc, 1, layout)


# The +-65504 channel: steps past the largest finite value overflow to inf (and
# are dropped), and its step 131008 is stored as +inf by the oracle and the
# library alike.
@np.errstate(over="ignore")
def test_one_bit_f16_thresholds_at_zero_subnormals_and_extremes(cuda_device):
    """Binary16 1-bit codes are decided against the smallest binary16 above the
    channel midpoint mu = (alpha + beta) / 2. Every way of finding it is met:
    - mu = 0, where the threshold is the smallest subnormal;
    - mu between -2^-24 and 0, and between 0 and 2^-24;
    - mu an exact negative subnormal, where one step up reaches -0;
    - mu halfway between subnormals;
    - mu halfway between the two largest finite values;
    - a constant channel at 65504, where the threshold is +inf;
    - mu = 0 with both signed zeros among the tokens.
    Codes, alpha and step are compared bit-exactly with the oracle in every
    layout, with a ragged token count."""
    f = np.float16
    sub = lambda k: f(k * 2.0 ** -24)  # noqa: E731  (k times the smallest subnormal)
    cases = [  # (alpha, beta, tokens inside [alpha, beta] that must appear)
        (f(-1), f(1), [f(0), f(-0.0), sub(1), -sub(1), sub(3), -sub(2)]),
        (-sub(1), sub(2), [f(0), f(-0.0), sub(1)]),
        (-sub(2), sub(1), [f(0), f(-0.0), -sub(1)]),
        (-sub(3), sub(1), [-sub(1), -sub(2), f(-0.0), f(0)]),
        (sub(3), sub(8), [sub(4), sub(5), sub(6), sub(7)]),
        (f(65472), f(65504), []),
        (f(-65504), f(65504), [f(0), f(-0.0), sub(1), -sub(1), f(65472), f(-65472)]),
        (f(65504), f(65504), []),
        (f(-2.0 ** -14), f(2.0 ** -14), [sub(1), -sub(1), f(0), f(-0.0), sub(1023), -sub(1023)]),
    ]
    rng = np.random.default_rng(5)
    n, d = 77, 128
    x = np.zeros((1, 2, n, d), dtype=f)
    for c in range(d):
        a, b, extra = cases[c % len(cases)]
        mid = (float(a) + float(b)) / 2.0  # exact in double
        near = [f(mid)]
        for step in (np.inf, -np.inf):
            v = f(mid)
            for _ in range(3):
                v = np.nextafter(v, f(step), dtype=f)
                near.append(v)
        near = [v for v in near if a <= v <= b and np.isfinite(v)]
        vals = [a, b] + extra + near
        rest = rng.uniform(float(a), float(b), n - len(vals)).astype(f)
        col = np.array(vals + list(rest), dtype=f)
        x[0, 0, :, c] = col
        x[0, 1, :, c] = col[rng.permutation(n)]
    xt = torch.from_numpy(x)
    for layout in (cq.LAYOUT_CANONICAL, cq.LAYOUT_OCTET_K, cq.LAYOUT_OCTET_V):
        qc = cq.cq_quantize_kv(xt.to(cuda_device), 1, layout)
        torch.cuda.synchronize()
        _check_quantized(xt, qc, 1, layout)
