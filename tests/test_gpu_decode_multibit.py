"""GPU parity of the b-bit octet decode path (b in {2, 4, 8}: codes streamed
through a shared-memory ring, logits resident) against the fp64 oracle, within
the 2e-3 per-row relative tolerance: ragged lengths inside a byte group and a
V tile, every calibration variant and dtype, rows long enough for 5- to
16-CTA clusters, agreement with the canonical path, and the bit-sweep
workload (batch 16, n = 8192) sampled."""

import numpy as np
import pytest
import torch

import oracle
from decode_attention_cq_b200 import calibq as cq
from decode_attention_cq_b200 import synth

from _util import OUT_RTOL, f64, ref_output_rounded, row_rel_err

pytestmark = pytest.mark.gpu

CALIBS = [(False, 1.0, 1.0), (True, 0.8, 0.9), (True, 1.0, 0.5), (True, 0.5, 1.0)]


def _quant(k, v, bits, device):
    return (cq.cq_quantize_kv(k.to(device), bits, cq.LAYOUT_OCTET_K),
            cq.cq_quantize_kv(v.to(device), bits, cq.LAYOUT_OCTET_V))


def _ref(q, k, v, bits, calib):
    dt = "f16" if q.dtype == torch.float16 else "f32"
    return oracle.decode_attention(f64(q), f64(k), f64(v), bits, dt, calib)["out"]


def _err(out, ref, dtype):
    return row_rel_err(out.float().cpu().numpy(), ref_output_rounded(ref, dtype))


@pytest.mark.parametrize("bits", [2, 4, 8])
@pytest.mark.parametrize("n", [1, 3, 33, 64, 65, 129, 1000, 2048, 2049, 3328])
def test_ragged_lengths(cuda_device, bits, n):
    q, k, v = synth.make_case(2, 8, 2, n, 128, "f16", outliers=4, seed=100 * bits + n)
    kq, vq = _quant(k, v, bits, cuda_device)
    for calib in CALIBS[:2]:
        out = cq.cq_decode_attn(q.to(cuda_device), kq, vq, calib=calib)
        torch.cuda.synchronize()
        assert _err(out, _ref(q, k, v, bits, calib), torch.float16) <= OUT_RTOL, (bits, n, calib)


@pytest.mark.parametrize("bits", [2, 4, 8])
@pytest.mark.parametrize("dtype", ["f16", "f32"])
def test_calibration_variants_and_dtypes(cuda_device, bits, dtype):
    q, k, v = synth.make_case(3, 12, 3, 1500, 128, dtype, outliers=4, seed=77 + bits)
    kq, vq = _quant(k, v, bits, cuda_device)
    for calib in CALIBS:
        out = cq.cq_decode_attn(q.to(cuda_device), kq, vq, calib=calib)
        torch.cuda.synchronize()
        assert _err(out, _ref(q, k, v, bits, calib), q.dtype) <= OUT_RTOL, (bits, dtype, calib)


@pytest.mark.parametrize("bits,n", [(2, 8192), (4, 10000), (8, 16384), (2, 20000), (4, 32768)])
def test_long_rows_use_larger_clusters(cuda_device, bits, n):
    q, k, v = synth.make_case(1, 4, 1, n, 128, "f16", outliers=4, seed=n + bits)
    kq, vq = _quant(k, v, bits, cuda_device)
    out = cq.cq_decode_attn(q.to(cuda_device), kq, vq, calib=CALIBS[1])
    torch.cuda.synchronize()
    assert _err(out, _ref(q, k, v, bits, CALIBS[1]), torch.float16) <= OUT_RTOL


@pytest.mark.parametrize("bits", [2, 4, 8])
def test_matches_canonical_path_and_is_deterministic(cuda_device, bits):
    q, k, v = synth.make_case(4, 16, 4, 2100, 128, "f16", outliers=4, seed=8 + bits)
    qd = q.to(cuda_device)
    kq, vq = _quant(k, v, bits, cuda_device)
    kc = cq.cq_quantize_kv(k.to(cuda_device), bits, cq.LAYOUT_CANONICAL)
    vc = cq.cq_quantize_kv(v.to(cuda_device), bits, cq.LAYOUT_CANONICAL)
    o1 = cq.cq_decode_attn(qd, kq, vq, calib=CALIBS[1]).clone()
    o2 = cq.cq_decode_attn(qd, kc, vc, calib=CALIBS[1])
    o3 = cq.cq_decode_attn(qd, kq, vq, calib=CALIBS[1])
    torch.cuda.synchronize()
    assert row_rel_err(o1.float().cpu().numpy(), o2.float().cpu().numpy()) <= OUT_RTOL
    assert torch.equal(o1, o3)


def test_degenerate_inputs(cuda_device):
    for bits in (2, 4, 8):
        q, k, v = synth.make_case(1, 4, 1, 300, 128, "f16", seed=5 + bits)
        q.zero_()  # all logits equal: mean of the dequantized V
        kq, vq = _quant(k, v, bits, cuda_device)
        out = cq.cq_decode_attn(q.to(cuda_device), kq, vq, calib=CALIBS[1])
        torch.cuda.synchronize()
        assert _err(out, _ref(q, k, v, bits, CALIBS[1]), torch.float16) <= OUT_RTOL
        q3, k3, v3 = synth.make_case(2, 8, 2, 1, 128, "f16", seed=6 + bits)  # one token: o = v
        kq3, vq3 = _quant(k3, v3, bits, cuda_device)
        out3 = cq.cq_decode_attn(q3.to(cuda_device), kq3, vq3, calib=CALIBS[1]).cpu()
        assert torch.equal(out3, v3[:, :, 0, :].repeat_interleave(4, dim=1))


@pytest.mark.parametrize("bits", [2, 4, 8])
def test_bitsweep_n8192_batch16_sampled(cuda_device, bits):
    """The bit-sweep workload (batch 16, 32/8 heads, n = 8192): sequences 0 and
    15 recomputed by the oracle, every row checked for the convex hull
    alpha_V <= o <= alpha_V + (2^b - 1) s_V."""
    w = synth.WORKLOADS["bitsweep_n8192_b16"]
    q, k, v = synth.make_workload(w, device=cuda_device)
    kq, vq = _quant(k, v, bits, cuda_device)
    out = cq.cq_decode_attn(q, kq, vq, calib=CALIBS[1])
    torch.cuda.synchronize()
    for b in (0, 15):
        ref = _ref(q[b:b + 1].cpu(), k[b:b + 1].cpu(), v[b:b + 1].cpu(), bits, CALIBS[1])
        assert _err(out[b:b + 1], ref, torch.float16) <= OUT_RTOL, b
    a = vq.alpha.float().repeat_interleave(4, dim=1)
    s = vq.scale.float().repeat_interleave(4, dim=1) * ((1 << bits) - 1)
    o = out.float()
    tol = 1e-3 * (a.abs() + s.abs())
    assert torch.all(o >= a - tol) and torch.all(o <= a + s + tol)
    del q, k, v
    torch.cuda.empty_cache()


@pytest.mark.parametrize("bits", [2, 4, 8])
def test_large_launch_two_slot_ring(cuda_device, bits):
    """A launch past two waves of 2 CTAs per SM (batch 40, n = 8192: 1280
    CTAs of 2048 tokens) takes the 2-slot ring with 3 CTAs per SM; the first,
    a middle and the last sequence against the oracle, and every row inside
    the convex hull alpha_V <= o <= alpha_V + (2^b - 1) s_V."""
    B, Hkv, n = 40, 8, 8192
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert B * Hkv * 4 > 4 * sms  # the launch this test is for
    q, k, v = synth.make_case(B, 4 * Hkv, Hkv, n, 128, "f16", outliers=4, seed=900 + bits, device=cuda_device)
    kq, vq = _quant(k, v, bits, cuda_device)
    out = cq.cq_decode_attn(q, kq, vq, calib=CALIBS[1])
    torch.cuda.synchronize()
    for b in (0, B // 2, B - 1):
        ref = _ref(q[b:b + 1].cpu(), k[b:b + 1].cpu(), v[b:b + 1].cpu(), bits, CALIBS[1])
        assert _err(out[b:b + 1], ref, torch.float16) <= OUT_RTOL, b
    a = vq.alpha.float().repeat_interleave(4, dim=1)
    s = vq.scale.float().repeat_interleave(4, dim=1) * ((1 << bits) - 1)
    o = out.float()
    tol = 1e-3 * (a.abs() + s.abs())
    assert torch.all(o >= a - tol) and torch.all(o <= a + s + tol)
    del q, k, v
    torch.cuda.empty_cache()
