"""Runs in a child process whose environment picks the octet decode kernel
(CALIBQ_DECODE_KERNEL is read once per process); prints one JSON line with the
per-case row-relative errors against the fp64 oracle and the kernel each case
ran."""

import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

import torch  # noqa: E402

import oracle  # noqa: E402
from decode_attention_cq_b200 import calibq as cq  # noqa: E402
from decode_attention_cq_b200 import synth  # noqa: E402

from _util import f64, ref_output_rounded, row_rel_err  # noqa: E402


def main():
    cases = json.loads(sys.argv[1])
    errs, names = [], []
    for n, batch, calib in cases:
        names.append(cq.cq_decode_kernel_name(cq.LAYOUT_OCTET_K, cq.LAYOUT_OCTET_V, batch, 8, 2, n, 128, 1))
        q, k, v = synth.make_case(batch, 4 * 2, 2, n, 128, "f16", outliers=4, seed=n)
        kq = cq.cq_quantize_kv(k.to("cuda:0"), 1, cq.LAYOUT_OCTET_K)
        vq = cq.cq_quantize_kv(v.to("cuda:0"), 1, cq.LAYOUT_OCTET_V)
        out = cq.cq_decode_attn(q.to("cuda:0"), kq, vq, calib=tuple(calib))
        torch.cuda.synchronize()
        ref = oracle.decode_attention(f64(q), f64(k), f64(v), 1, "f16", tuple(calib))["out"]
        errs.append(row_rel_err(out.float().cpu().numpy(), ref_output_rounded(ref, torch.float16)))
    print(json.dumps({"errs": errs, "names": names}))


if __name__ == "__main__":
    main()
