"""Child process for test_gpu_graph_capture: the first cq_decode_attn call of
the process is made inside CUDA-graph capture (the default, global capture
mode), at the bench workload (batch 64, n = 8192: whole rows plus split rows
in a programmatic dependent launch); the graph is replayed and sampled
sequences are compared with the fp64 oracle. Prints one JSON line."""

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

CALIB = (True, 0.8, 0.9)


def main():
    dev = torch.device("cuda", 0)
    w = synth.WORKLOADS["internvl8b_n8192_b64"]
    q, k, v = synth.make_workload(w, device=dev)
    K, V = cq.LAYOUT_OCTET_K, cq.LAYOUT_OCTET_V
    kq = cq.cq_quantize_kv(k, 1, K)
    vq = cq.cq_quantize_kv(v, 1, V)
    out = torch.zeros_like(q)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):  # the process's first decode call
        cq.cq_decode_attn(q, kq, vq, calib=CALIB, out=out)
    captured_nonzero = bool(out.abs().sum().item() != 0)  # capture does not run the kernels
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    qc, kc, vc = q.cpu(), k.cpu(), v.cpu()
    errs = {}
    for b in (0, 31, 55, 60, 63):
        ref = oracle.decode_attention(f64(qc[b:b + 1]), f64(kc[b:b + 1]), f64(vc[b:b + 1]), 1, "f16", CALIB,
                                      check_forms=False)["out"]
        errs[b] = row_rel_err(out[b:b + 1].float().cpu().numpy(), ref_output_rounded(ref, torch.float16))
    print(json.dumps({"errs": errs, "captured_nonzero": captured_nonzero,
                      "kernel": cq.cq_decode_kernel_name(K, V, w.batch, w.hq, w.hkv, w.n, w.d, 1),
                      "launches": cq.cq_decode_launch_count(K, V, w.batch, w.hq, w.hkv, w.n, w.d, 1)}))


if __name__ == "__main__":
    main()
