"""Stored values: hand-worked kernel values, and the oracle's own PR1 output (regression)."""
import json
import os

import numpy as np

from laplacian_nystr_attention_avg_b200.inputs import WORKLOADS, make_inputs
from oracle import lfa_oracle as O

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_kernel_hand_values():
    with open(os.path.join(GOLDEN, "kernel_hand_values.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        k = O.laplacian_kernel(np.array([c["x"]]), np.array([c["y"]]), c["lam"])[0, 0]
        assert abs(k - c["k"]) <= 1e-15, c


def test_pr1_regression():
    wl = WORKLOADS["pr1"]
    x = make_inputs(wl)
    g = np.load(os.path.join(GOLDEN, "pr1_oracle.npz"))
    fw = O.forward(x.Q.numpy(), x.V.numpy(), x.dwc.numpy(), wl, whiten=True)
    fu = O.forward(x.Q.numpy(), x.V.numpy(), x.dwc.numpy(), wl, whiten=False)
    for name, got in (("O", fw.O), ("O_attn", fw.O_attn), ("O_unw", fu.O), ("O_attn_unw", fu.O_attn),
                      ("C", fw.units[0].C), ("X", fw.units[0].X)):
        ref = g[name]
        assert np.allclose(got, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max()), name
