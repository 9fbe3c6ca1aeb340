"""GPU parity of the mixed-cache decode (quantized visual tokens in the octet
layouts + full-precision text tokens in one softmax) against the fp64 oracle,
within the 2e-3 per-row relative tolerance, for every bit width, text lengths
from 0 up, with and without calibration, both dtypes; and equality with the
plain decode when there are no text tokens."""

import pytest
import torch

import oracle
from decode_attention_cq_b200 import calibq as cq
from decode_attention_cq_b200 import synth

from _util import OUT_RTOL, f64, ref_output_rounded, row_rel_err

pytestmark = pytest.mark.gpu


def _case(B, Hkv, n_vis, n_text, dtype, bits, seed):
    q, k, v = synth.make_case(B, 4 * Hkv, Hkv, n_vis, 128, dtype, outliers=4, seed=seed)
    g = torch.Generator().manual_seed(seed + 1)
    kt = synth.make_cache(B, Hkv, n_text, 128, dtype, 0, g, "cpu")
    vt = synth.make_cache(B, Hkv, n_text, 128, dtype, 0, g, "cpu")
    return q, k, v, kt, vt


@pytest.mark.parametrize("bits", [1, 2, 4, 8])
@pytest.mark.parametrize("n_vis,n_text", [(257, 0), (257, 1), (1000, 37), (3328, 300), (9000, 64)])
def test_mixed_matches_oracle(cuda_device, bits, n_vis, n_text):
    q, k, v, kt, vt = _case(2, 2, n_vis, n_text, "f16", bits, seed=bits * 1000 + n_vis + n_text)
    kq = cq.cq_quantize_kv(k.to(cuda_device), bits, cq.LAYOUT_OCTET_K)
    vq = cq.cq_quantize_kv(v.to(cuda_device), bits, cq.LAYOUT_OCTET_V)
    for calib in ((False, 1.0, 1.0), (True, 0.8, 0.9)):
        out = cq.cq_decode_attn_mixed(q.to(cuda_device), kq, vq, kt.to(cuda_device), vt.to(cuda_device),
                                      calib=calib)
        torch.cuda.synchronize()
        ref = oracle.decode_attention_mixed(f64(q), f64(k), f64(v), f64(kt), f64(vt), bits, "f16", calib)["out"]
        err = row_rel_err(out.float().cpu().numpy(), ref_output_rounded(ref, torch.float16))
        assert err <= OUT_RTOL, (bits, n_vis, n_text, calib, err)


def test_mixed_f32_and_explicit_scale(cuda_device):
    q, k, v, kt, vt = _case(1, 3, 1500, 90, "f32", 1, seed=5)
    kq = cq.cq_quantize_kv(k.to(cuda_device), 1, cq.LAYOUT_OCTET_K)
    vq = cq.cq_quantize_kv(v.to(cuda_device), 1, cq.LAYOUT_OCTET_V)
    out = cq.cq_decode_attn_mixed(q.to(cuda_device), kq, vq, kt.to(cuda_device), vt.to(cuda_device),
                                  calib=(True, 1.0, 0.5), softmax_scale=0.05)
    torch.cuda.synchronize()
    ref = oracle.decode_attention_mixed(f64(q), f64(k), f64(v), f64(kt), f64(vt), 1, "f32", (True, 1.0, 0.5),
                                        softmax_scale=0.05)["out"]
    assert row_rel_err(out.cpu().numpy(), ref_output_rounded(ref, torch.float32)) <= OUT_RTOL


@pytest.mark.parametrize("bits", [1, 4])
def test_mixed_without_text_equals_plain_decode(cuda_device, bits):
    q, k, v, _, _ = _case(2, 2, 2049, 0, "f16", bits, seed=9)
    qd = q.to(cuda_device)
    kq = cq.cq_quantize_kv(k.to(cuda_device), bits, cq.LAYOUT_OCTET_K)
    vq = cq.cq_quantize_kv(v.to(cuda_device), bits, cq.LAYOUT_OCTET_V)
    plain = cq.cq_decode_attn(qd, kq, vq, calib=(True, 0.8, 0.9))
    mixed = cq.cq_decode_attn_mixed(qd, kq, vq, None, None, calib=(True, 0.8, 0.9))
    torch.cuda.synchronize()
    assert torch.equal(plain, mixed)


ROW_CASES = [("f16", 700, 50), ("f16", 1, 1), ("f16", 257, 63), ("f16", 3328, 64), ("f16", 1000, 65),
             ("f16", 8192, 300), ("f16", 64, 129), ("f16", 2048, 1024), ("f32", 700, 50), ("f32", 8192, 300)]


def _check_row_kernel(B, Hkv, n_vis):
    assert cq.cq_decode_kernel_name(cq.LAYOUT_OCTET_K, cq.LAYOUT_OCTET_V, B, 4 * Hkv, Hkv, n_vis, 128, 1) == "k_decode_row"


@pytest.mark.parametrize("dtype,n_vis,n_text", ROW_CASES)
def test_mixed_through_the_row_kernel(row_kernel, dtype, n_vis, n_text):
    """The one-CTA-per-row kernel (forced), which attends the text tokens in
    the same launch (f16: through the ring and the
    tensor cores, 64 tokens per chunk, whole and partial chunks, odd and even
    chunk-pair counts; f32: on the CUDA cores); and equality with the plain
    decode without text."""
    B, Hkv = 38, 4  # 152 rows: at least one per SM
    cuda_device = row_kernel
    _check_row_kernel(B, Hkv, n_vis)
    q, k, v, kt, vt = _case(B, Hkv, n_vis, n_text, dtype, 1, seed=77 + n_vis + n_text)
    qd = q.to(cuda_device)
    kq = cq.cq_quantize_kv(k.to(cuda_device), 1, cq.LAYOUT_OCTET_K)
    vq = cq.cq_quantize_kv(v.to(cuda_device), 1, cq.LAYOUT_OCTET_V)
    calib = (True, 0.8, 0.9)
    out = cq.cq_decode_attn_mixed(qd, kq, vq, kt.to(cuda_device), vt.to(cuda_device), calib=calib)
    plain = cq.cq_decode_attn(qd, kq, vq, calib=calib)
    mixed0 = cq.cq_decode_attn_mixed(qd, kq, vq, None, None, calib=calib)
    torch.cuda.synchronize()
    ref = oracle.decode_attention_mixed(f64(q), f64(k), f64(v), f64(kt), f64(vt), 1, dtype, calib)["out"]
    rd = torch.float16 if dtype == "f16" else torch.float32
    assert row_rel_err(out.float().cpu().numpy(), ref_output_rounded(ref, rd)) <= OUT_RTOL
    assert torch.equal(plain, mixed0)


@pytest.mark.parametrize("text_scale", [0.05, 4.0])
def test_row_kernel_text_logits_far_from_visual(row_kernel, text_scale):
    """Text keys scaled so that the text logits sit well inside (0.05) or far
    above (4.0) the visual ones: the log-sum-exp merge has to keep whichever
    side carries the weight."""
    B, Hkv = 38, 4
    cuda_device = row_kernel
    _check_row_kernel(B, Hkv, 1500)
    q, k, v, kt, vt = _case(B, Hkv, 1500, 200, "f16", 1, seed=31)
    kt = (kt.double() * text_scale).to(torch.float16)
    qd = q.to(cuda_device)
    kq = cq.cq_quantize_kv(k.to(cuda_device), 1, cq.LAYOUT_OCTET_K)
    vq = cq.cq_quantize_kv(v.to(cuda_device), 1, cq.LAYOUT_OCTET_V)
    calib = (True, 0.8, 0.9)
    out = cq.cq_decode_attn_mixed(qd, kq, vq, kt.to(cuda_device), vt.to(cuda_device), calib=calib)
    torch.cuda.synchronize()
    ref = oracle.decode_attention_mixed(f64(q), f64(k), f64(v), f64(kt), f64(vt), 1, "f16", calib)["out"]
    assert row_rel_err(out.float().cpu().numpy(), ref_output_rounded(ref, torch.float16)) <= OUT_RTOL
