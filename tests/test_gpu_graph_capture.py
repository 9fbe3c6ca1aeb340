"""Every cq_decode_attn call can be captured into a CUDA graph, the first one
of a process included: the library creates no streams or events and
synchronizes nothing inside a call. Run in a fresh child process so that the
captured call really is the first."""

import json
import os
import subprocess
import sys

import pytest

from _util import OUT_RTOL

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


def test_first_call_is_captured_and_replayed(cuda_device):
    res = subprocess.run([sys.executable, os.path.join(HERE, "_graph_capture_worker.py")],
                         capture_output=True, text=True, timeout=900)
    assert res.returncode == 0, res.stderr[-3000:]
    line = json.loads(res.stdout.strip().splitlines()[-1])
    assert line["kernel"] == "k_decode_row" and line["launches"] == 2  # whole rows + split rows
    assert not line["captured_nonzero"]
    for b, e in line["errs"].items():
        assert e <= OUT_RTOL, (b, e)
