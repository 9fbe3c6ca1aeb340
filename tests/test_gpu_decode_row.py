"""GPU parity of the one-CTA-per-row 1-bit decode kernel against the fp64
oracle: calibration
variants in both dtypes, the degenerate cases of the method (all logits
equal, constant channels, a single token) and determinism. The kernel is
forced (cq_set_decode_kernel) and each test checks that it is the one
launched; 38 sequences x 4 kv-heads = 152 rows."""

import pytest
import torch

import oracle
from decode_attention_cq_b200 import calibq as cq
from decode_attention_cq_b200 import synth

from _util import OUT_RTOL, f64, ref_output_rounded, row_rel_err

pytestmark = pytest.mark.gpu

B, HKV = 38, 4
CALIBS = [(False, 1.0, 1.0), (True, 0.8, 0.9), (True, 1.0, 0.5), (True, 0.5, 1.0)]


def _check_row_kernel(n):
    assert cq.cq_decode_kernel_name(cq.LAYOUT_OCTET_K, cq.LAYOUT_OCTET_V, B, 4 * HKV, HKV, n, 128, 1) == "k_decode_row"


def _quant(k, v, device):
    return (cq.cq_quantize_kv(k.to(device), 1, cq.LAYOUT_OCTET_K),
            cq.cq_quantize_kv(v.to(device), 1, cq.LAYOUT_OCTET_V))


def _err(out, q, k, v, calib):
    dt = "f16" if q.dtype == torch.float16 else "f32"
    ref = oracle.decode_attention(f64(q), f64(k), f64(v), 1, dt, calib)["out"]
    return row_rel_err(out.float().cpu().numpy(), ref_output_rounded(ref, q.dtype))


@pytest.mark.parametrize("calib", CALIBS)
@pytest.mark.parametrize("dtype", ["f16", "f32"])
def test_row_kernel_calibrations_and_dtypes(row_kernel, calib, dtype):
    n = 1000  # four 256-token tiles, the last one ragged
    _check_row_kernel(n)
    q, k, v = synth.make_case(B, 4 * HKV, HKV, n, 128, dtype, outliers=4, seed=101)
    kq, vq = _quant(k, v, row_kernel)
    out = cq.cq_decode_attn(q.to(row_kernel), kq, vq, calib=calib)
    torch.cuda.synchronize()
    assert _err(out, q, k, v, calib) <= OUT_RTOL


def test_row_kernel_equal_logits(row_kernel):
    """Zero query: every logit is the same, the range is empty (M = m), the
    calibration leaves it as is and the weights are uniform."""
    n = 600
    _check_row_kernel(n)
    q, k, v = synth.make_case(B, 4 * HKV, HKV, n, 128, "f16", seed=5)
    q.zero_()
    kq, vq = _quant(k, v, row_kernel)
    for calib in CALIBS[:2]:
        out = cq.cq_decode_attn(q.to(row_kernel), kq, vq, calib=calib)
        torch.cuda.synchronize()
        assert _err(out, q, k, v, calib) <= OUT_RTOL


def test_row_kernel_constant_channels(row_kernel):
    """beta == alpha in every channel: codes are 0, the step is 0, and the
    output is the constant value exactly."""
    n = 300
    _check_row_kernel(n)
    k = torch.full((B, HKV, n, 128), 1.5, dtype=torch.float16)
    v = torch.full((B, HKV, n, 128), -0.75, dtype=torch.float16)
    q = torch.randn(B, 4 * HKV, 128, generator=torch.Generator().manual_seed(3)).half()
    kq, vq = _quant(k, v, row_kernel)
    out = cq.cq_decode_attn(q.to(row_kernel), kq, vq, calib=CALIBS[1]).cpu()
    assert torch.all(out == -0.75)


def test_row_kernel_single_token(row_kernel):
    """One token: its weight is 1 and the output is its value, which a 1-bit
    code with alpha = beta = x reproduces exactly."""
    _check_row_kernel(1)
    q, k, v = synth.make_case(B, 4 * HKV, HKV, 1, 128, "f16", seed=6)
    kq, vq = _quant(k, v, row_kernel)
    out = cq.cq_decode_attn(q.to(row_kernel), kq, vq, calib=CALIBS[1]).cpu()
    assert torch.equal(out, v[:, :, 0, :].repeat_interleave(4, dim=1))


def test_row_kernel_deterministic(row_kernel):
    n = 3000
    _check_row_kernel(n)
    q, k, v = synth.make_case(B, 4 * HKV, HKV, n, 128, "f16", seed=9)
    kq, vq = _quant(k, v, row_kernel)
    qd = q.to(row_kernel)
    o1 = cq.cq_decode_attn(qd, kq, vq, calib=CALIBS[1]).clone()
    for _ in range(3):
        o2 = cq.cq_decode_attn(qd, kq, vq, calib=CALIBS[1])
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)


@pytest.mark.parametrize("n", [8192, 3000, 257])
def test_row_kernel_split_rows(row_kernel, n):
    """More than two waves of rows (two per SM): the rows beyond a whole number
    of SM counts run as halves on 2-CTA clusters, in a second launch. Every
    such row, and whole rows around them, against the oracle."""
    Bb, Hkv = 40, 8  # 320 rows
    rows = Bb * Hkv
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    split = rows % sms if rows > 2 * sms and (n + 255) // 256 >= 2 and rows % sms <= sms // 2 else 0
    K, V = cq.LAYOUT_OCTET_K, cq.LAYOUT_OCTET_V
    assert cq.cq_decode_launch_count(K, V, Bb, 4 * Hkv, Hkv, n, 128, 1) == (2 if split else 1)
    q, k, v = synth.make_case(Bb, 4 * Hkv, Hkv, n, 128, "f16", outliers=4, seed=n + 13)
    kq, vq = _quant(k, v, row_kernel)
    calib = CALIBS[1]
    out = cq.cq_decode_attn(q.to(row_kernel), kq, vq, calib=calib).cpu()
    first_split_batch = (rows - split) // Hkv
    batches = sorted({0, Bb // 2, max(0, first_split_batch - 1)} | set(range(first_split_batch, Bb)))
    for b in batches:
        sl = slice(b, b + 1)
        ref = oracle.decode_attention(f64(q[sl]), f64(k[sl]), f64(v[sl]), 1, "f16", calib)["out"]
        err = row_rel_err(out[sl].float().numpy(), ref_output_rounded(ref, torch.float16))
        assert err <= OUT_RTOL, (n, b, err)


def test_split_rows_are_ordered_before_later_stream_work(row_kernel):
    """The split rows start while the whole rows still run (a programmatic
    dependent launch), yet work queued after the call on the same stream must
    see every row: a device copy and a host copy taken right after the call,
    with no synchronization in between, equal the output read after it."""
    Bb, Hkv, n = 40, 8, 8192  # 320 rows: 24 of them run split on B200
    K, V = cq.LAYOUT_OCTET_K, cq.LAYOUT_OCTET_V
    assert cq.cq_decode_launch_count(K, V, Bb, 4 * Hkv, Hkv, n, 128, 1) == 2
    q, k, v = synth.make_case(Bb, 4 * Hkv, Hkv, n, 128, "f16", outliers=4, seed=77, device=row_kernel)
    kq, vq = _quant(k, v, row_kernel)
    out = torch.empty_like(q)
    host = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    for _ in range(5):
        out.fill_(float("nan"))
        cq.cq_decode_attn(q, kq, vq, calib=CALIBS[1], out=out)
        snap = out.clone()
        host.copy_(out, non_blocking=True)
        torch.cuda.synchronize()
        assert not torch.isnan(out).any()
        assert torch.equal(snap, out)
        assert torch.equal(host, out.cpu())
