"""lfa_forward_noalloc: the handle-free forward over the library's static scratch area.

Through the C ABI: two calls in a row match the handle-based lfa_forward on the same
inputs within the forward parity tolerance, the second call leaves the device's free
memory unchanged, and a configuration that needs more scratch than the static area
holds is rejected before any device work. This file is named to be collected last, so
the checks also run after every other test has used the device.
"""
from __future__ import annotations

import ctypes

import pytest
import torch

from laplacian_nystr_attention_avg_b200 import lfa
from tests import parity_util as pu


def test_noalloc_rejects_config_beyond_scratch():
    # m = 196 landmarks for 8 units needs about 20 MiB of scratch (16 MiB available);
    # the pointers are never dereferenced because the size check comes first
    cfg = lfa.make_config(pu.workload("hr196"), True)
    fake = ctypes.c_void_p(1 << 20)
    st = lfa.load().lfa_forward_noalloc(ctypes.byref(cfg), fake, fake, fake, fake, None)
    assert st == lfa.LFA_ERR_SCRATCH_LIMIT
    assert "scratch" in lfa.status_string(st)
    bad = lfa.make_config(pu.workload("hr196", r=5), True)    # 112 % 5 != 0
    assert lfa.load().lfa_forward_noalloc(ctypes.byref(bad), fake, fake, fake, fake, None) == \
        lfa.LFA_ERR_INVALID_ARG


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["pr1", "pvt1", "pvt2", "hr49"])
def test_noalloc_matches_forward_two_calls(name):
    wl = pu.workload(name)
    x = pu.inputs_for(wl)
    mod = pu.gpu_module(wl, True, False)
    Q, V = x.Q_store.cuda(), x.V_store.cuda()
    ref = mod.forward(Q, V)
    O1 = torch.full_like(ref, float("nan"))
    O2 = torch.full_like(ref, float("nan"))
    lfa.forward_noalloc(mod.cfg, mod.weight, Q, V, O1)
    torch.cuda.synchronize()
    free_before, _ = torch.cuda.mem_get_info()
    lfa.forward_noalloc(mod.cfg, mod.weight, Q, V, O2)
    torch.cuda.synchronize()
    free_after, _ = torch.cuda.mem_get_info()
    assert free_after == free_before
    units = tuple(range(wl.units))
    bf16 = wl.dtype == "bf16"
    want = pu.unit_rows(ref, units)
    for O in (O1, O2):
        err = pu.o_error(pu.unit_rows(O, units), want, bf16)
        assert err <= pu.o_tolerance(bf16), f"{name}: no-alloc vs lfa_forward error {err:.3e}"
    assert torch.equal(O1, O2)
