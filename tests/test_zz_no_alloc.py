"""cq_quantize_kv_noalloc: the quantizer for callers that cannot allocate
device memory (for instance a serving runtime whose KV-cache pool already owns
all of HBM). It keeps its scratch in a fixed array inside the library, so it is
checked here, through the C ABI, against cq_quantize_kv with a caller
workspace: two calls in a row on different inputs must both reproduce that
entry point's codes, alpha and step exactly, and a request larger than the
fixed scratch must be refused without writing anything.

Named so that pytest collects it last."""

import pytest
import torch

from decode_attention_cq_b200 import calibq as cq
from decode_attention_cq_b200 import synth

pytestmark = pytest.mark.gpu


def _noalloc(x, bits, layout):
    B, H, n, d = x.shape
    nbytes = cq.cq_codes_bytes(layout, B, H, n, d, bits)
    codes = torch.empty(B, H, nbytes // (B * H), dtype=torch.uint8, device=x.device)
    alpha = torch.empty(B, H, d, dtype=x.dtype, device=x.device)
    scale = torch.empty(B, H, d, dtype=x.dtype, device=x.device)
    st = cq.load().cq_quantize_kv_noalloc(
        x.data_ptr(), cq.CQ_F16 if x.dtype == torch.float16 else cq.CQ_F32, B, H, n, d, bits, layout,
        codes.data_ptr(), alpha.data_ptr(), scale.data_ptr(), torch.cuda.current_stream().cuda_stream)
    return st, codes, alpha, scale


@pytest.mark.parametrize("layout,bits,dtype", [(cq.LAYOUT_CANONICAL, 1, "f16"), (cq.LAYOUT_CANONICAL, 4, "f32"),
                                               (cq.LAYOUT_OCTET_K, 1, "f16"), (cq.LAYOUT_OCTET_V, 1, "f16")])
def test_two_calls_match_the_workspace_entry_point(cuda_device, layout, bits, dtype):
    gen = torch.Generator().manual_seed(1234 + bits)
    inputs = [synth.make_cache(4, 8, n, 128, dtype, 4, gen, "cpu").to(cuda_device) for n in (3000, 1777)]
    results = [_noalloc(x, bits, layout) for x in inputs]  # back to back on one stream
    torch.cuda.synchronize()
    for x, (st, codes, alpha, scale) in zip(inputs, results):
        assert st == cq.CQ_OK, cq.status_string(st)
        ref = cq.cq_quantize_kv(x, bits, layout)
        torch.cuda.synchronize()
        assert torch.equal(codes, ref.codes)
        assert torch.equal(alpha.view(torch.uint8), ref.alpha.view(torch.uint8))
        assert torch.equal(scale.view(torch.uint8), ref.scale.view(torch.uint8))


def test_request_beyond_the_fixed_scratch_is_refused(cuda_device):
    # 4097 (batch, head) rows need 4097 KiB of partials: one more than the 4 MiB scratch
    x = torch.randn(1, 4097, 1, 128, device=cuda_device).half()
    st, codes, alpha, scale = _noalloc(x, 1, cq.LAYOUT_CANONICAL)
    assert st == cq.CQ_ERR_UNSUPPORTED
    assert cq.cq_quantize_kv_workspace_size(1, 4097, 1, 128) > 4 << 20
    x2 = torch.randn(1, 4096, 1, 128, device=cuda_device).half()
    st2, codes2, _, _ = _noalloc(x2, 1, cq.LAYOUT_CANONICAL)
    torch.cuda.synchronize()
    assert st2 == cq.CQ_OK
    assert torch.equal(codes2, cq.cq_quantize_kv(x2, 1, cq.LAYOUT_CANONICAL).codes)
