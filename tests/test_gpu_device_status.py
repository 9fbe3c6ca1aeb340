"""The decode kernels' device-side error report (cq_decode_attn_ex). Every
wait of a decode kernel for data is bounded; one that runs out makes the CTA
write NaN rows and return instead of hanging, and is reported in a device
status word the caller reads after synchronizing. The timeout path is made to
run on a normal input by bounding the cluster kernel's copy waits to one
non-blocking probe (its copies are all issued at the start of the launch, so
they are still in flight when it gives up; they land before the CTA exits).
No copy is broken and nothing faults; the context stays usable."""

import pytest
import torch

import oracle
from decode_attention_cq_b200 import calibq as cq
from decode_attention_cq_b200 import synth

from _util import OUT_RTOL, f64, ref_output_rounded, row_rel_err

pytestmark = pytest.mark.gpu

CALIB = (True, 0.8, 0.9)
K, V = cq.LAYOUT_OCTET_K, cq.LAYOUT_OCTET_V


def _case(device, B=8, Hkv=8, n=8192, seed=77):
    q, k, v = synth.make_case(B, 4 * Hkv, Hkv, n, 128, "f16", outliers=4, seed=seed)
    return q, k, v, cq.cq_quantize_kv(k.to(device), 1, K), cq.cq_quantize_kv(v.to(device), 1, V)


def _check(out, q, k, v, batches):
    for b in batches:
        sl = slice(b, b + 1)
        ref = oracle.decode_attention(f64(q[sl]), f64(k[sl]), f64(v[sl]), 1, "f16", CALIB, check_forms=False)["out"]
        assert row_rel_err(out[sl].float().cpu().numpy(), ref_output_rounded(ref, torch.float16)) <= OUT_RTOL, b


def test_timed_out_wait_is_reported_and_the_context_stays_usable(cuda_device):
    q, k, v, kq, vq = _case(cuda_device)
    status = torch.zeros(4, dtype=torch.int32, device=cuda_device)
    cq.cq_set_decode_kernel(cq.KERNEL_CLUSTER)
    try:
        assert cq.cq_decode_kernel_name(K, V, 8, 32, 8, 8192, 128, 1) == "k_decode_mma"
        qd = q.to(cuda_device)
        out = cq.cq_decode_attn_ex(qd, kq, vq, status, wait_probes=1, calib=CALIB)
        torch.cuda.synchronize()
        assert int(status[0]) == cq.DEVICE_WAIT_TIMEOUT
        assert int(status[1:].abs().sum()) == 0  # only the one word is written
        assert torch.isnan(out.float()).any()  # the rows of the CTAs that gave up
        # same stream, same context: the default bounds give the right answer and no report
        status.zero_()
        out = cq.cq_decode_attn_ex(qd, kq, vq, status, calib=CALIB)
        torch.cuda.synchronize()
        assert int(status[0]) == 0
        _check(out, q, k, v, (0, 7))
    finally:
        cq.cq_set_decode_kernel(cq.KERNEL_ENV)


@pytest.mark.parametrize("kernel", ["auto", "row", "pipe"])
def test_normal_calls_report_nothing(cuda_device, kernel):
    q, k, v, kq, vq = _case(cuda_device, B=4, n=3000, seed=78)
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    choice = {"auto": cq.KERNEL_AUTO, "row": cq.KERNEL_ROW, "pipe": cq.KERNEL_PIPE}[kernel]
    cq.cq_set_decode_kernel(choice)
    try:
        out = cq.cq_decode_attn_ex(q.to(cuda_device), kq, vq, status, calib=CALIB)
        torch.cuda.synchronize()
        assert int(status[0]) == 0
        _check(out, q, k, v, (0, 3))
    finally:
        cq.cq_set_decode_kernel(cq.KERNEL_ENV)
