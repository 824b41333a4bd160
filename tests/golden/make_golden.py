"""Writes the stored oracle outputs under tests/golden/ (calls only oracle/ and the input generator).

Run from the repository root:  python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from laplacian_nystr_attention_avg_b200.inputs import WORKLOADS, make_inputs  # noqa: E402
from oracle import lfa_oracle as O  # noqa: E402


def main():
    wl = WORKLOADS["pr1"]
    x = make_inputs(wl)
    fw = O.forward(x.Q.numpy(), x.V.numpy(), x.dwc.numpy(), wl, whiten=True)
    fu = O.forward(x.Q.numpy(), x.V.numpy(), x.dwc.numpy(), wl, whiten=False)
    u = fw.units[0]
    np.savez_compressed(os.path.join(HERE, "pr1_oracle.npz"), O=fw.O, O_attn=fw.O_attn,
                        O_unw=fu.O, O_attn_unw=fu.O_attn, C=u.C, X=u.X, L=u.L)
    meta = {"workload": "pr1", "seed": 0, "alpha": u.alpha.alpha, "alpha_pages": u.alpha.alpha_pages,
            "fallback": u.alpha.fallback, "norm2": u.alpha.norm2,
            "ns_residual_fro": [r[0] for r in u.ns_residuals]}
    with open(os.path.join(HERE, "pr1_oracle.json"), "w") as f:
        json.dump(meta, f, indent=1)


if __name__ == "__main__":
    main()
