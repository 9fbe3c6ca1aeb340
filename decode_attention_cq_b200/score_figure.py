"""Exact / Quant / Quant-C attention-score distributions on a synthetic cache.

The CalibQuant article (Method 3, the figure after it) shows that 1-bit
quantization of the K cache widens the distribution of attention scores (its
dequantized values sit at the channel extremes), and that the calibration map
g pulls it back towards the full-precision ("Exact") one. This module rebuilds
that comparison on a seeded InternVL-2.5-shaped cache:

* Exact   -- logits sigma q.k on the full-precision keys;
* Quant   -- logits on the 1-bit keys (quantized and dequantized by libcalibq);
* Quant-C -- Quant logits after g (calibration interval [tau_lo m, tau_hi M]).

It reports, per series, the spread of the logits, the largest softmax weight,
the divergence KL(Exact || series) of the softmax rows, and a histogram of the
logits over common bins. Usage (needs a GPU and the built library):

    python -m decode_attention_cq_b200.score_figure [--n 3328] [--tau 0.8 0.9] [--out report.md]
"""

from __future__ import annotations

import argparse
import sys

import torch

from . import calibq as cq
from . import synth


def calibrate(x: torch.Tensor, tau_lo: float, tau_hi: float) -> torch.Tensor:
    """g on each row of x: [m, M] -> [tau_lo m, tau_hi M] (rows with M == m unchanged)."""
    m = x.min(dim=-1, keepdim=True).values
    M = x.max(dim=-1, keepdim=True).values
    span = M - m
    y = tau_lo * m + (x - m) * (tau_hi * M - tau_lo * m) / torch.where(span > 0, span, torch.ones_like(span))
    return torch.where(span > 0, y, x)


def score_series(n: int = 3328, tau=(0.8, 0.9), seed: int = 1, heads: int = 32, kv_heads: int = 8,
                 device: str = "cuda:0"):
    """Logits [Hq, n] of the three series for one sequence (float64 on the device)."""
    q, k, _ = synth.make_case(1, heads, kv_heads, n, 128, "f16", outliers=4, seed=seed, device=device)
    kq = cq.cq_quantize_kv(k, 1, cq.LAYOUT_CANONICAL)
    k_hat = cq.cq_dequant(kq)
    sigma = 128 ** -0.5
    g = heads // kv_heads

    def logits(keys):
        kk = keys.double().repeat_interleave(g, dim=1)[0]  # [Hq, n, d]
        return sigma * torch.einsum("hd,hnd->hn", q.double()[0], kk)

    exact = logits(k)
    quant = logits(k_hat)
    return {"Exact": exact, "Quant": quant, "Quant-C": calibrate(quant, *tau)}


def summarize(series: dict, bins: int = 24):
    """Per-series statistics and a common-bin histogram of the logits."""
    p_exact = torch.softmax(series["Exact"], dim=-1)
    lo = min(float(s.min()) for s in series.values())
    hi = max(float(s.max()) for s in series.values())
    edges = torch.linspace(lo, hi, bins + 1, dtype=torch.float64)
    rows = {}
    for name, x in series.items():
        p = torch.softmax(x, dim=-1)
        kl = (p_exact * (torch.log(p_exact + 1e-300) - torch.log(p + 1e-300))).sum(-1).mean()
        hist = torch.histc(x.flatten().cpu(), bins=bins, min=lo, max=hi)
        rows[name] = {"std": float(x.std()), "min": float(x.min()), "max": float(x.max()),
                      "max_p": float(p.max(dim=-1).values.mean()), "kl": float(kl), "hist": hist.tolist()}
    return {"edges": edges.tolist(), "series": rows}


def report(summary: dict, n: int, tau) -> str:
    lines = [f"# Attention-score distributions, 1-bit K cache, n = {n}, tau = {tau[0]}, {tau[1]}", "",
             "| series | logit std | min | max | mean max weight | KL(Exact || series) |",
             "|---|---|---|---|---|---|"]
    for name, r in summary["series"].items():
        lines.append(f"| {name} | {r['std']:.3f} | {r['min']:.2f} | {r['max']:.2f} | {r['max_p']:.4f} | {r['kl']:.4f} |")
    lines += ["", "Logit histogram (counts per bin):", "",
              "| bin | " + " | ".join(summary["series"]) + " |", "|---|" + "---|" * len(summary["series"])]
    e = summary["edges"]
    for i in range(len(e) - 1):
        counts = " | ".join(str(int(r["hist"][i])) for r in summary["series"].values())
        lines.append(f"| [{e[i]:.2f}, {e[i + 1]:.2f}) | {counts} |")
    return "\n".join(lines) + "\n"


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--n", type=int, default=3328)
    ap.add_argument("--tau", type=float, nargs=2, default=(0.8, 0.9))
    ap.add_argument("--seed", type=int, default=1)
    ap.add_argument("--out", default=None)
    args = ap.parse_args(argv)
    text = report(summarize(score_series(args.n, tuple(args.tau), args.seed)), args.n, tuple(args.tau))
    if args.out:
        with open(args.out, "w") as f:
            f.write(text)
    sys.stdout.write(text)
    return 0


if __name__ == "__main__":
    raise SystemExit(main())
