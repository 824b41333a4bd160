"""A bounded wait of the fused forward runs out, on purpose and safely, and the handle recovers.

lfa_debug_spin_test makes the next forward wait for a landmark flag value that nothing sets, with
every wait for a flag written by another thread block bounded by a short budget. Nothing faults or
hangs: the waits expire, the call sets the timeout bit and completes with invalid outputs, and
lfa_get_info reports LFA_ERR_TIMEOUT and re-arms the flags. The next forward must then be
bit-identical to one from before the test.
"""
import pytest
import torch

from laplacian_nystr_attention_avg_b200 import lfa
from tests import parity_util as pu

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["pvt1", "pvt2"])
def test_flag_waits_run_out_and_the_next_forward_is_clean(name):
    wl = pu.workload(name)
    x = pu.inputs_for(wl)
    mod = pu.gpu_module(wl, True, False)
    assert mod.path == "fused"
    Q, V = x.Q_store.cuda(), x.V_store.cuda()
    clean = mod.forward(Q, V).clone()
    st, _ = mod.info()
    assert st == lfa.LFA_OK
    mod.arm_spin_test(2000)          # about 1 us at the SM clock
    mod.forward(Q, V)
    st, _ = mod.info()
    assert st == lfa.LFA_ERR_TIMEOUT
    again = mod.forward(Q, V)
    st, _ = mod.info()
    assert st == lfa.LFA_OK
    assert torch.equal(again, clean)


def test_spin_test_needs_the_fused_path(monkeypatch):
    monkeypatch.setenv("LFA_FORWARD_PATH", "generic")
    mod = pu.gpu_module(pu.workload("pvt2"), True, False)
    with pytest.raises(lfa.LfaError) as e:
        mod.arm_spin_test(2000)
    assert e.value.status == lfa.LFA_ERR_UNSUPPORTED
