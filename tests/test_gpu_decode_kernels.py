"""The 1-bit octet-layout decode kernels against the fp64 oracle: the
one-CTA-per-row kernel (n <= 8192, chosen when the batch gives every SM a
row), the cluster kernel (n <= 32768) and the tcgen05 kernel (longer rows),
each also forced with CALIBQ_DECODE_KERNEL in a child process so that the
selection, read once per process, applies. A forced kernel that does not take
n falls back to the default choice."""

import json
import os
import subprocess
import sys

import pytest

from _util import OUT_RTOL

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
CASES = [[1, 1, [True, 0.8, 0.9]], [7, 1, [True, 0.8, 0.9]], [255, 1, [True, 0.8, 0.9]],
         [256, 1, [False, 1.0, 1.0]], [300, 2, [False, 1.0, 1.0]], [1024, 1, [True, 0.8, 0.9]],
         [1025, 2, [True, 0.8, 0.9]], [2049, 1, [True, 1.0, 0.5]], [3328, 1, [True, 0.8, 0.9]],
         [4097, 1, [True, 0.8, 0.9]], [8191, 1, [True, 0.5, 1.0]], [8192, 1, [True, 0.8, 0.9]],
         [600, 80, [True, 0.8, 0.9]], [10000, 1, [True, 0.5, 1.0]], [12000, 1, [True, 0.8, 0.9]],
         [14000, 1, [True, 0.8, 0.9]], [20000, 1, [True, 0.8, 0.9]]]


def _run(kernel):
    env = dict(os.environ)
    env.pop("CALIBQ_DECODE_KERNEL", None)
    if kernel:
        env["CALIBQ_DECODE_KERNEL"] = kernel
    res = subprocess.run([sys.executable, os.path.join(HERE, "_kernel_select_worker.py"), json.dumps(CASES)],
                         env=env, capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    return json.loads(res.stdout.strip().splitlines()[-1])


def _expected(kernel, n):
    """The documented choice: a forced kernel where it takes n; otherwise, for
    n <= 8192, the row or the cluster kernel (an estimate of their step times
    decides), then the cluster kernel up to n = 32768, then the tcgen05 one."""
    if kernel == "row" and n <= 8192:
        return {"k_decode_row"}
    if kernel == "cluster" and n <= 32768:
        return {"k_decode_mma"}
    if kernel == "tcgen05":
        return {"k_decode_octet"}
    if n <= 8192:
        return {"k_decode_row", "k_decode_mma"}
    return {"k_decode_mma"} if n <= 32768 else {"k_decode_octet"}


@pytest.mark.parametrize("kernel", [None, "row", "cluster", "tcgen05"])
def test_octet_kernels_match_oracle(cuda_device, kernel):
    r = _run(kernel)
    for (n, batch, calib), e, name in zip(CASES, r["errs"], r["names"]):
        assert name in _expected(kernel, n), (kernel, n, batch, name)
        assert e <= OUT_RTOL, (kernel, n, calib, e)
