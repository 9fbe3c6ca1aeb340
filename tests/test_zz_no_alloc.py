"""cq_quantize_kv_noalloc: the quantizer for callers that cannot allocate
device memory (for instance a serving runtime whose KV-cache pool already owns
all of HBM, or a latency-critical path where cudaMalloc would synchronize the
device). It keeps the scratch of its two-launch path (rows longer than 16384
tokens: per-split channel minima and maxima) in a fixed array inside the
library. Checked here through the C ABI: two calls in a row on different
inputs long enough to use that array must each reproduce the fp64 oracle's
codes, alpha and step bit for bit, and the same bytes as cq_quantize_kv with a
caller workspace; short rows (no scratch) must be accepted whatever their
number; a request whose scratch exceeds the array is refused before anything
is launched.

Named so that pytest collects it last."""

import numpy as np
import pytest
import torch

import oracle
from decode_attention_cq_b200 import calibq as cq
from decode_attention_cq_b200 import synth

from _util import oracle_quantize

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


def _check_oracle(x_cpu, codes, alpha, scale, bits, layout):
    ref = oracle_quantize(x_cpu, bits)
    assert np.array_equal(alpha.cpu().numpy().view(np.uint8), ref["alpha"].view(np.uint8)), "alpha differs"
    assert np.array_equal(scale.cpu().numpy().view(np.uint8), ref["scale"].view(np.uint8)), "scale differs"
    assert np.array_equal(codes.cpu().numpy(), oracle.pack_codes(ref["codes"], layout, bits)), "codes differ"


@pytest.mark.parametrize("layout,bits,dtype", [(cq.LAYOUT_CANONICAL, 1, "f16"), (cq.LAYOUT_CANONICAL, 4, "f32"),
                                               (cq.LAYOUT_OCTET_K, 1, "f32"), (cq.LAYOUT_OCTET_V, 1, "f16"),
                                               (cq.LAYOUT_OCTET_K, 2, "f16")])
def test_two_calls_through_the_fixed_scratch(cuda_device, layout, bits, dtype):
    # n > 16384: the two-launch path, whose statistics go through the fixed array;
    # the second call has different sizes and data, so a stale or misplaced
    # partial from the first one would change its result
    gen = torch.Generator().manual_seed(1234 + bits)
    shapes = [(1, 4, 20000), (1, 6, 17000)]
    inputs = [synth.make_cache(B, H, n, 128, dtype, 4, gen, "cpu") for B, H, n in shapes]
    for B, H, n in shapes:
        assert cq.cq_quantize_kv_workspace_size(B, H, n, 128) > 0
    results = [_noalloc(x.to(cuda_device), bits, layout) for x in inputs]  # back to back on one stream
    torch.cuda.synchronize()
    for x, (st, codes, alpha, scale) in zip(inputs, results):
        assert st == cq.CQ_OK, cq.status_string(st)
        _check_oracle(x, codes, alpha, scale, bits, layout)
        ref = cq.cq_quantize_kv(x.to(cuda_device), bits, layout)
        torch.cuda.synchronize()
        assert torch.equal(codes, ref.codes)
        assert torch.equal(alpha.view(torch.uint8), ref.alpha.view(torch.uint8))
        assert torch.equal(scale.view(torch.uint8), ref.scale.view(torch.uint8))


def test_short_rows_need_no_scratch(cuda_device):
    # 4097 (batch, head) rows of one token: their workspace would exceed the
    # array, but the single-read fill uses none, so the call is accepted
    assert cq.cq_quantize_kv_workspace_size(1, 4097, 1, 128) > 4 << 20
    x = torch.randn(1, 4097, 1, 128, generator=torch.Generator().manual_seed(5)).half()
    st, codes, alpha, scale = _noalloc(x.to(cuda_device), 1, cq.LAYOUT_CANONICAL)
    torch.cuda.synchronize()
    assert st == cq.CQ_OK
    _check_oracle(x, codes, alpha, scale, 1, cq.LAYOUT_CANONICAL)


def test_request_beyond_the_fixed_scratch_is_refused(cuda_device):
    # 4097 rows of 16385 tokens need 4097 KiB of partials, one more than the
    # 4 MiB array: refused from the sizes alone, before any pointer is used
    assert cq.cq_quantize_kv_workspace_size(1, 4097, 16385, 128) > 4 << 20
    st = cq.load().cq_quantize_kv_noalloc(None, cq.CQ_F16, 1, 4097, 16385, 128, 1, cq.LAYOUT_CANONICAL,
                                          None, None, None, None)
    assert st == cq.CQ_ERR_UNSUPPORTED
    # the largest accepted request on that path: 4096 rows
    assert cq.cq_quantize_kv_workspace_size(1, 4096, 16385, 128) <= 4 << 20
    st = cq.load().cq_quantize_kv_noalloc(None, cq.CQ_F16, 1, 4096, 16385, 128, 1, cq.LAYOUT_CANONICAL,
                                          None, None, None, None)
    assert st == cq.CQ_ERR_INVALID_ARG  # past the limit check: now the null pointers are refused
