"""The Exact / Quant / Quant-C score-distribution tool: its calibration map
matches the oracle's g (CPU), and on the GPU the rebuilt figure shows what
the CalibQuant article's figure shows -- 1-bit keys widen the logit
distribution and calibration pulls the softmax rows back towards Exact."""

import numpy as np
import pytest
import torch

import oracle
from decode_attention_cq_b200 import score_figure


@pytest.mark.parametrize("tau", [(0.8, 0.9), (1.0, 0.5), (1.0, 1.0)])
def test_calibration_matches_oracle(tau):
    x = torch.randn(5, 77, dtype=torch.float64) * 3
    x[2] = 1.5  # a constant row stays as it is
    got = score_figure.calibrate(x, *tau).numpy()
    assert np.allclose(got, oracle.calibrate(x.numpy(), *tau), rtol=1e-12, atol=1e-12)


@pytest.mark.gpu
def test_figure_reproduces_the_calibration_effect(cuda_device):
    series = score_figure.score_series(n=1200, tau=(0.8, 0.9), seed=3, device=cuda_device)
    s = score_figure.summarize(series)["series"]
    assert s["Quant"]["std"] > s["Exact"]["std"]          # 1-bit keys widen the logits
    assert s["Quant-C"]["std"] < s["Quant"]["std"]        # g pulls them in
    assert s["Quant-C"]["kl"] < s["Quant"]["kl"]          # and the softmax closer to Exact
    assert s["Exact"]["kl"] == pytest.approx(0.0, abs=1e-12)
    for r in s.values():
        assert sum(r["hist"]) == pytest.approx(32 * 1200)


@pytest.mark.gpu
def test_figure_series_match_the_oracle(cuda_device):
    """The three series element by element against the oracle on the same
    seeded inputs: Exact = sigma q.k, Quant = the same on the oracle's 1-bit
    dequantized keys (rounded once to f16, as the library stores them),
    Quant-C = the oracle's calibration map g of Quant."""
    from decode_attention_cq_b200 import synth

    n, tau, seed = 1200, (0.8, 0.9), 3
    series = score_figure.score_series(n=n, tau=tau, seed=seed, device=cuda_device)
    q, k, _ = synth.make_case(1, 32, 8, n, 128, "f16", outliers=4, seed=seed, device=cuda_device)  # as the tool draws them
    qd, kd = q.cpu().double().numpy(), k.cpu().double().numpy()
    kq = oracle.quantize_cache(kd, 1, "f16")
    k_hat = oracle.dequantize(kq["codes"], kq["alpha"], kq["scale"]).astype(np.float16).astype(np.float64)
    want = {"Exact": oracle.scores_dequantized(qd, kd)[0],
            "Quant": oracle.scores_dequantized(qd, k_hat)[0]}
    want["Quant-C"] = oracle.calibrate(want["Quant"], *tau)
    for name, ref in want.items():
        got = series[name].cpu().numpy()
        assert got.shape == ref.shape
        assert np.allclose(got, ref, rtol=1e-9, atol=1e-9 * np.abs(ref).max()), name
