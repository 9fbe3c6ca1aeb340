"""GPU parity of the persistent tcgen05 1-bit decode kernel (one CTA per SM
working through whole rows; forced with cq_set_decode_kernel) against the
fp64 oracle: ragged token counts that span several K blocks (1024 tokens)
and V tiles (256 tokens), both dtypes, every calibration variant, more rows
than SMs (several rows per CTA, where the pipeline state carries over from
row to row), the degenerate cases of the method and bitwise determinism."""

import pytest
import torch

import oracle
from decode_attention_cq_b200 import calibq as cq
from decode_attention_cq_b200 import synth

from _util import OUT_RTOL, f64, ref_output_rounded, row_rel_err

pytestmark = pytest.mark.gpu

CALIBS = [(False, 1.0, 1.0), (True, 0.8, 0.9), (True, 1.0, 0.5), (True, 0.5, 1.0)]
K, V = cq.LAYOUT_OCTET_K, cq.LAYOUT_OCTET_V


def _name(B, Hkv, n):
    return cq.cq_decode_kernel_name(K, V, B, 4 * Hkv, Hkv, n, 128, 1)


def _quant(k, v, device):
    return cq.cq_quantize_kv(k.to(device), 1, K), cq.cq_quantize_kv(v.to(device), 1, V)


def _err(out, q, k, v, calib):
    dt = "f16" if q.dtype == torch.float16 else "f32"
    ref = oracle.decode_attention(f64(q), f64(k), f64(v), 1, dt, calib)["out"]
    return row_rel_err(out.float().cpu().numpy(), ref_output_rounded(ref, q.dtype))


@pytest.mark.parametrize("n", [1, 7, 255, 257, 1000, 1025, 2049, 3000, 8192])
def test_pipe_ragged_lengths(pipe_kernel, n):
    B, Hkv = 3, 4
    assert _name(B, Hkv, n) == "k_decode_tc"
    q, k, v = synth.make_case(B, 4 * Hkv, Hkv, n, 128, "f16", outliers=4, seed=n + 101)
    kq, vq = _quant(k, v, pipe_kernel)
    out = cq.cq_decode_attn(q.to(pipe_kernel), kq, vq, calib=CALIBS[1])
    torch.cuda.synchronize()
    assert _err(out, q, k, v, CALIBS[1]) <= OUT_RTOL


@pytest.mark.parametrize("calib", CALIBS)
@pytest.mark.parametrize("dtype", ["f16", "f32"])
def test_pipe_calibrations_and_dtypes(pipe_kernel, calib, dtype):
    B, Hkv, n = 5, 4, 1500
    q, k, v = synth.make_case(B, 4 * Hkv, Hkv, n, 128, dtype, outliers=4, seed=202)
    kq, vq = _quant(k, v, pipe_kernel)
    out = cq.cq_decode_attn(q.to(pipe_kernel), kq, vq, calib=calib)
    torch.cuda.synchronize()
    assert _err(out, q, k, v, calib) <= OUT_RTOL


@pytest.mark.parametrize("n", [300, 4100])
def test_pipe_many_rows_per_cta(pipe_kernel, n):
    """More rows than SMs: every CTA runs several rows back to back (the K-block
    copies of the next row start during the current one, the pipeline's slot
    counters carry over). A spread of sequences, including the last ones."""
    B, Hkv = 40, 8  # 320 rows
    assert _name(B, Hkv, n) == "k_decode_tc"
    q, k, v = synth.make_case(B, 4 * Hkv, Hkv, n, 128, "f16", outliers=4, seed=n + 7)
    kq, vq = _quant(k, v, pipe_kernel)
    out = cq.cq_decode_attn(q.to(pipe_kernel), kq, vq, calib=CALIBS[1]).cpu()
    for b in (0, 1, 17, 18, 19, 36, 37, 38, 39):
        sl = slice(b, b + 1)
        ref = oracle.decode_attention(f64(q[sl]), f64(k[sl]), f64(v[sl]), 1, "f16", CALIBS[1])["out"]
        err = row_rel_err(out[sl].float().numpy(), ref_output_rounded(ref, torch.float16))
        assert err <= OUT_RTOL, (n, b, err)


def test_pipe_equal_logits_and_single_token(pipe_kernel):
    """Zero query (all logits equal: uniform weights) and n = 1 (the output is
    the token's value, exactly)."""
    B, Hkv = 4, 4
    q, k, v = synth.make_case(B, 4 * Hkv, Hkv, 700, 128, "f16", seed=5)
    q.zero_()
    kq, vq = _quant(k, v, pipe_kernel)
    for calib in CALIBS[:2]:
        out = cq.cq_decode_attn(q.to(pipe_kernel), kq, vq, calib=calib)
        torch.cuda.synchronize()
        assert _err(out, q, k, v, calib) <= OUT_RTOL
    q, k, v = synth.make_case(B, 4 * Hkv, Hkv, 1, 128, "f16", seed=6)
    kq, vq = _quant(k, v, pipe_kernel)
    out = cq.cq_decode_attn(q.to(pipe_kernel), kq, vq, calib=CALIBS[1]).cpu()
    assert torch.equal(out, v[:, :, 0, :].repeat_interleave(4, dim=1))


def test_pipe_deterministic(pipe_kernel):
    B, Hkv, n = 40, 8, 3000  # several rows per CTA
    q, k, v = synth.make_case(B, 4 * Hkv, Hkv, n, 128, "f16", seed=9)
    kq, vq = _quant(k, v, pipe_kernel)
    qd = q.to(pipe_kernel)
    o1 = cq.cq_decode_attn(qd, kq, vq, calib=CALIBS[1]).clone()
    for _ in range(3):
        o2 = cq.cq_decode_attn(qd, kq, vq, calib=CALIBS[1])
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)


def test_pipe_not_taken_for_mixed_or_long_rows(cuda_device):
    cq.cq_set_decode_kernel(cq.KERNEL_PIPE)
    try:
        assert _name(2, 2, 8193) != "k_decode_tc"  # n > 8192
        assert cq.cq_decode_launch_count(K, V, 2, 8, 2, 1000, 128, 1, 16) >= 1  # mixed calls: another kernel
    finally:
        cq.cq_set_decode_kernel(cq.KERNEL_ENV)
