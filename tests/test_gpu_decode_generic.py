"""GPU parity of cq_decode_attn on canonical layouts (every bit width, any GQA
group) against the fp64 oracle, within the 2e-3 per-row relative tolerance."""

import numpy as np
import pytest
import torch

import oracle
from decode_attention_cq_b200 import calibq as cq
from decode_attention_cq_b200 import synth

from _util import OUT_RTOL, f64, ref_output_rounded, row_rel_err

pytestmark = pytest.mark.gpu

CALIBS = [(False, 1.0, 1.0), (True, 0.8, 0.9), (True, 1.0, 0.5), (True, 0.5, 1.0)]


def _run(q, k, v, bits, calib, device, softmax_scale=0.0):
    kq = cq.cq_quantize_kv(k.to(device), bits, cq.LAYOUT_CANONICAL)
    vq = cq.cq_quantize_kv(v.to(device), bits, cq.LAYOUT_CANONICAL)
    out = cq.cq_decode_attn(q.to(device), kq, vq, calib=calib, softmax_scale=softmax_scale)
    torch.cuda.synchronize()
    return out.cpu()


def _ref(q, k, v, bits, calib, softmax_scale=0.0):
    dt = "f16" if q.dtype == torch.float16 else "f32"
    return oracle.decode_attention(f64(q), f64(k), f64(v), bits, dt, calib, softmax_scale)["out"]


@pytest.mark.parametrize("bits", [1, 2])
@pytest.mark.parametrize("calib", CALIBS)
def test_tiny_single_head_fp32(cuda_device, bits, calib):
    """B=1, one query head, one kv-head, n=256, fp32 (the tiny workload)."""
    w = synth.WORKLOADS["tiny_n256"]
    q, k, v = synth.make_workload(w)
    out = _run(q, k, v, bits, calib, cuda_device)
    ref = _ref(q, k, v, bits, calib)
    assert row_rel_err(out.numpy(), ref) <= OUT_RTOL


@pytest.mark.parametrize("bits", [1, 2, 4, 8])
@pytest.mark.parametrize("n", [1, 5, 256, 777])
@pytest.mark.parametrize("G", [1, 4, 6])
def test_gqa_ragged(cuda_device, bits, n, G):
    q, k, v = synth.make_case(2, 2 * G, 2, n, 128, "f16", outliers=2, seed=bits * 31 + n + G)
    for calib in (CALIBS[0], CALIBS[1]):
        out = _run(q, k, v, bits, calib, cuda_device)
        ref = _ref(q, k, v, bits, calib)
        assert row_rel_err(out.numpy(), ref_output_rounded(ref, torch.float16)) <= OUT_RTOL, calib


def test_single_token_is_v(cuda_device):
    q, k, v = synth.make_case(2, 8, 2, 1, 128, "f16", seed=3)
    out = _run(q, k, v, 1, CALIBS[1], cuda_device)
    assert torch.equal(out, v[:, :, 0, :].repeat_interleave(4, dim=1))


def test_zero_query_is_mean(cuda_device):
    q, k, v = synth.make_case(1, 4, 1, 300, 128, "f16", seed=4)
    q.zero_()
    out = _run(q, k, v, 2, CALIBS[1], cuda_device)
    ref = _ref(q, k, v, 2, CALIBS[1])
    assert row_rel_err(out.numpy(), ref) <= OUT_RTOL


def test_explicit_softmax_scale(cuda_device):
    q, k, v = synth.make_case(1, 8, 2, 200, 128, "f32", seed=5)
    out = _run(q, k, v, 4, CALIBS[1], cuda_device, softmax_scale=0.05)
    ref = _ref(q, k, v, 4, CALIBS[1], softmax_scale=0.05)
    assert row_rel_err(out.numpy(), ref) <= OUT_RTOL


@pytest.mark.parametrize("bits", [1, 2, 4, 8])
def test_bit_sweep_sampled_rows(cuda_device, bits):
    """n=8192, batch 16, 32/8 heads (the bit-width sweep); rows of two sequences
    are recomputed by the oracle."""
    w = synth.WORKLOADS["bitsweep_n8192_b16"]
    q, k, v = synth.make_workload(w, device=cuda_device)
    out = _run(q, k, v, bits, CALIBS[1], cuda_device)
    for b in (0, 11):
        ref = _ref(q[b:b + 1].cpu(), k[b:b + 1].cpu(), v[b:b + 1].cpu(), bits, CALIBS[1])
        assert row_rel_err(out[b:b + 1].numpy(), ref_output_rounded(ref, torch.float16)) <= OUT_RTOL
    del q, k, v
    torch.cuda.empty_cache()
