"""Host-side validation with real device buffers: every bad call returns its
status and launches nothing (outputs stay untouched)."""

import pytest
import torch

from decode_attention_cq_b200 import calibq as cq

pytestmark = pytest.mark.gpu


def _qc(device, n=64, layout=cq.LAYOUT_CANONICAL, bits=1, dtype=torch.float16, H=2):
    x = torch.randn(1, H, n, 128, device=device).to(dtype)
    return x, cq.cq_quantize_kv(x, bits, layout)


def test_quantize_rejections(cuda_device):
    x, qc = _qc(cuda_device)
    lib = cq.load()
    ws = torch.empty(cq.cq_quantize_kv_workspace_size(1, 2, 64, 128), dtype=torch.uint8, device=cuda_device)
    sentinel = qc.codes.clone()
    s = torch.cuda.current_stream().cuda_stream
    args = lambda **kw: dict(dict(x=x.data_ptr(), codes=qc.codes.data_ptr(), alpha=qc.alpha.data_ptr(),
                                  scale=qc.scale.data_ptr(), ws=ws.data_ptr(), nws=ws.numel()), **kw)

    def call(a, layout=0, bits=1):
        return lib.cq_quantize_kv(a["x"], 0, 1, 2, 64, 128, bits, layout, a["codes"], a["alpha"],
                                  a["scale"], a["ws"], a["nws"], s)

    assert call(args()) == cq.CQ_OK
    torch.cuda.synchronize()
    sentinel = qc.codes.clone()
    host = torch.empty(64 * 128 * 2, dtype=torch.uint8)
    assert call(args(x=host.data_ptr())) == cq.CQ_ERR_INVALID_ARG           # host pointer
    assert call(args(x=x.data_ptr() + 2)) == cq.CQ_ERR_INVALID_ARG          # misaligned
    assert call(args(nws=ws.numel() - 1)) == cq.CQ_ERR_WORKSPACE            # small workspace
    assert call(args(ws=None)) == cq.CQ_ERR_WORKSPACE
    assert call(args(), layout=1, bits=3) == cq.CQ_ERR_INVALID_ARG          # bits not in {1, 2, 4, 8}
    assert call(args(), layout=7, bits=1) == cq.CQ_ERR_INVALID_ARG          # unknown layout
    torch.cuda.synchronize()
    assert torch.equal(qc.codes, sentinel)


def test_decode_rejections(cuda_device):
    _, kq = _qc(cuda_device, layout=cq.LAYOUT_OCTET_K)
    _, vq = _qc(cuda_device, layout=cq.LAYOUT_OCTET_V)
    _, kc = _qc(cuda_device)
    q = torch.randn(1, 8, 128, device=cuda_device).half()
    out = torch.full_like(q, 7.0)
    # mixed layouts
    with pytest.raises(cq.CalibqError) as e:
        cq.cq_decode_attn(q, kc, vq, out=out, workspace=torch.empty(1 << 20, dtype=torch.uint8, device=cuda_device))
    assert e.value.status == cq.CQ_ERR_UNSUPPORTED
    # octet path needs 4 query heads per kv-head
    q6 = torch.randn(1, 6, 128, device=cuda_device).half()
    with pytest.raises(cq.CalibqError) as e:
        cq.cq_decode_attn(q6, kq, vq)
    assert e.value.status in (cq.CQ_ERR_UNSUPPORTED, cq.CQ_ERR_INVALID_ARG)
    # generic path: workspace too small
    _, vc = _qc(cuda_device)
    with pytest.raises(cq.CalibqError) as e:
        cq.cq_decode_attn(q, kc, vc, out=out, workspace=torch.empty(16, dtype=torch.uint8, device=cuda_device))
    assert e.value.status == cq.CQ_ERR_WORKSPACE
    # non-finite calibration parameters
    with pytest.raises(cq.CalibqError) as e:
        cq.cq_decode_attn(q, kc, vc, out=out, calib=(True, float("inf"), 0.9))
    assert e.value.status == cq.CQ_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert torch.all(out == 7.0)


def test_octet_path_length_limit(cuda_device):
    """n above 65536 is refused by the tensor-core path (its logits live on chip)."""
    n = 65537
    x = torch.zeros(1, 1, n, 128, device=cuda_device).half()
    kq = cq.cq_quantize_kv(x, 1, cq.LAYOUT_OCTET_K)
    vq = cq.cq_quantize_kv(x, 1, cq.LAYOUT_OCTET_V)
    q = torch.zeros(1, 4, 128, device=cuda_device).half()
    with pytest.raises(cq.CalibqError) as e:
        cq.cq_decode_attn(q, kq, vq)
    assert e.value.status == cq.CQ_ERR_UNSUPPORTED


def test_validated_allocations_are_remembered_per_allocation(cuda_device):
    """A pointer inside an allocation that an earlier call validated is
    accepted without a new driver query; pointers the driver would reject are
    still rejected after device buffers have been remembered."""
    x, qc = _qc(cuda_device, n=64, H=4)
    lib = cq.load()
    s = torch.cuda.current_stream().cuda_stream
    ws = torch.empty(cq.cq_quantize_kv_workspace_size(1, 2, 64, 128), dtype=torch.uint8, device=cuda_device)

    def call(xp, codes=qc.codes.data_ptr()):
        return lib.cq_quantize_kv(xp, 0, 1, 2, 64, 128, 1, 0, codes, qc.alpha.data_ptr(), qc.scale.data_ptr(),
                                  ws.data_ptr(), ws.numel(), s)

    assert call(x.data_ptr()) == cq.CQ_OK
    # heads 2..3 of the same tensor: same allocation, 16-byte aligned
    assert call(x.data_ptr() + 2 * 64 * 128 * 2) == cq.CQ_OK
    host = torch.empty(64 * 128 * 2, dtype=torch.uint8)
    assert call(host.data_ptr()) == cq.CQ_ERR_INVALID_ARG
    assert call(x.data_ptr(), codes=host.data_ptr()) == cq.CQ_ERR_INVALID_ARG
    assert call(x.data_ptr() + 16 + 2) == cq.CQ_ERR_INVALID_ARG  # misaligned, inside a remembered allocation
    torch.cuda.synchronize()
    # the same buffers through the binding, many times: outputs stay exact
    want = cq.cq_quantize_kv(x, 1, cq.LAYOUT_CANONICAL)
    for _ in range(3):
        got = cq.cq_quantize_kv(x, 1, cq.LAYOUT_CANONICAL)
        assert torch.equal(got.codes, want.codes)
