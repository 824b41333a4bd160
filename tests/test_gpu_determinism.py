"""Back-to-back forwards on one handle are bit-identical.

The fused kernel's CTAs meet only through flags and shared memory, and a missing barrier shows up
as a result that depends on what an earlier launch left in an SM's shared memory or on warp timing:
some units come out wrong in some calls, while a single call (all the parity tests make) looks
right. So every call of a run of back-to-back forwards, alternately into one reused output buffer
(holding the previous result) and into a fresh one, must equal the first call bit for bit. The
per-stage path is held to the same rule.
"""
import pytest
import torch

from tests import parity_util as pu

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,calls", [("pvt1", 60), ("pvt2", 60), ("hr49", 20), ("hr196", 6), ("pr1", 20)])
def test_back_to_back_forwards_are_bit_identical(name, calls):
    wl = pu.workload(name)
    x = pu.inputs_for(wl)
    mod = pu.gpu_module(wl, True, False)
    Q, V = x.Q_store.cuda(), x.V_store.cuda()
    ref = mod.forward(Q, V).clone()
    O = mod.new_output()
    bad = []
    for k in range(calls):
        out = mod.forward(Q, V, O if k % 2 else None)
        if not torch.equal(out, ref):
            bad.append(k)
    st, _ = mod.info()
    assert st == 0
    assert not bad, f"{name} ({mod.path}): calls {bad[:10]} differ from the first"
