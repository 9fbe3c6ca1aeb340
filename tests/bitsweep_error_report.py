"""Output error of the bit-width sweep against the fp64 oracle.

    python tests/bitsweep_error_report.py [--sequences 0 15]

For each b in {1, 2, 4, 8} at bitsweep_n8192_b16 (batch 16, 32 / 8 heads,
d = 128, n = 8192; the same seeded inputs as ``bench.py --bit-sweep``), one
JSON line with the largest and the mean per-row relative error
max_j |o - o_ref| / max_j |o_ref| of the library's output (octet layouts,
tensor-core path, calibration tau = (0.8, 0.9)) against the oracle's,
over every (batch, query-head) row of the sampled sequences. Needs a GPU;
the oracle runs on the host (about 4 s per sequence and b).
"""

import argparse
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(HERE))
sys.path.insert(0, HERE)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import oracle  # noqa: E402
from decode_attention_cq_b200 import calibq as cq  # noqa: E402
from decode_attention_cq_b200 import synth  # noqa: E402

from _util import f64, ref_output_rounded  # noqa: E402

CALIB = (True, 0.8, 0.9)


def row_errors(out, ref):
    num = np.abs(out - ref).max(axis=-1)
    den = np.maximum(np.abs(ref).max(axis=-1), 1e-30)
    return (num / den).ravel()


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--sequences", type=int, nargs="+", default=[0, 15])
    args = ap.parse_args(argv)
    dev = torch.device("cuda", 0)
    w = synth.WORKLOADS["bitsweep_n8192_b16"]
    q, k, v = synth.make_workload(w, device=dev)
    qc, kc, vc = q.cpu(), k.cpu(), v.cpu()
    for bits in (1, 2, 4, 8):
        kq = cq.cq_quantize_kv(k, bits, cq.LAYOUT_OCTET_K)
        vq = cq.cq_quantize_kv(v, bits, cq.LAYOUT_OCTET_V)
        out = cq.cq_decode_attn(q, kq, vq, calib=CALIB).float().cpu().numpy()
        errs = []
        for b in args.sequences:
            ref = oracle.decode_attention(f64(qc[b:b + 1]), f64(kc[b:b + 1]), f64(vc[b:b + 1]), bits, "f16", CALIB,
                                          check_forms=False)["out"]
            errs.append(row_errors(out[b:b + 1], ref_output_rounded(ref, torch.float16)))
        e = np.concatenate(errs)
        print(json.dumps({"workload": "bitsweep_n8192_b16", "bits": bits, "sequences": args.sequences,
                          "rows": int(e.size), "max_row_rel_err": float(e.max()), "mean_row_rel_err": float(e.mean()),
                          "tolerance": 2e-3,
                          "kernel": cq.cq_decode_kernel_name(cq.LAYOUT_OCTET_K, cq.LAYOUT_OCTET_V, w.batch, w.hq,
                                                             w.hkv, w.n, w.d, bits)}), flush=True)


if __name__ == "__main__":
    main()
