"""The W / rho ablation on the planted generator, through the GPU kernels
(HyQuant digest, results paragraph: a larger window or a higher
vertical-line ratio lowers the error; README Overview: the hybrid keeps the
important keys FP16).  Errors are relative L2 against the same kernels with
every key FP16 (W >= L), on a 2K prefix: the hybrid beats uniform low-bit
storage, and the error falls as W or rho grows."""
import pytest
import torch

pytestmark = pytest.mark.gpu


def test_error_falls_with_window_and_ratio():
    import bench
    rows = bench.ablation_sweep(torch.device("cuda", 0), Ls=2048, Ws=(0, 128, 512), rhos=(0, 500, 2000), steps=3)
    e = {(r["W"], round(r["rho"] * 10000)): r for r in rows}
    for key in ("prefill_rel_l2", "decode_rel_l2"):
        assert e[(128, 500)][key] < e[(0, 0)][key], key                     # hybrid < uniform low-bit
        for rho in (0, 500, 2000):
            assert e[(512, rho)][key] < e[(128, rho)][key] < e[(0, rho)][key], (key, rho)
        for W in (0, 128, 512):
            assert e[(W, 2000)][key] < e[(W, 500)][key] < e[(W, 0)][key], (key, W)
