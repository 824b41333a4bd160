"""The C-ABI library loads and exports what include/lfa.h declares; host-side validation.

No compute call is made here (no GPU needed): only entry points that return before
touching the device.
"""
import ctypes
import os

import pytest

from laplacian_nystr_attention_avg_b200 import build as lfa_build
from laplacian_nystr_attention_avg_b200 import lfa
from laplacian_nystr_attention_avg_b200.inputs import WORKLOADS


@pytest.fixture(scope="module")
def lib():
    lfa_build.build()
    return lfa.load()


def test_exports_every_declared_symbol(lib):
    names = lfa.header_symbols()
    assert "lfa_forward" in names and "lfa_backward" in names and "lfa_create" in names
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/lfa.h but not exported"


def test_status_strings(lib):
    for s in range(7):
        assert lfa.status_string(s) and lfa.status_string(s) != "unknown status"
    assert lfa.status_string(99) == "unknown status"


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_workspace_size_valid_configs(lib, name):
    cfg = lfa.make_config(WORKLOADS[name])
    n = lfa.workspace_size(cfg)
    assert n > 0 and n % 256 == 0


def _cfg(**kw):
    base = dict(B=1, heads=1, H=16, W=16, d=32, r=4, lambda_=4.0, eps=1e-6, T=20, dtype=lfa.LFA_F32, whiten=1)
    base.update(kw)
    return lfa.Config(**base)


@pytest.mark.parametrize("kw,expect", [
    (dict(H=15), lfa.LFA_ERR_INVALID_ARG),              # H % r != 0
    (dict(W=18), lfa.LFA_ERR_INVALID_ARG),              # W % r != 0
    (dict(lambda_=0.0), lfa.LFA_ERR_INVALID_ARG),
    (dict(lambda_=-1.0), lfa.LFA_ERR_INVALID_ARG),
    (dict(lambda_=float("nan")), lfa.LFA_ERR_INVALID_ARG),
    (dict(eps=-1e-6), lfa.LFA_ERR_INVALID_ARG),
    (dict(T=-1), lfa.LFA_ERR_INVALID_ARG),
    (dict(T=65), lfa.LFA_ERR_INVALID_ARG),
    (dict(B=0), lfa.LFA_ERR_INVALID_ARG),
    (dict(r=0), lfa.LFA_ERR_INVALID_ARG),
    (dict(whiten=4), lfa.LFA_ERR_INVALID_ARG),          # 0 raw, 1 per unit, 2 batch-pooled, 3 reading B
    (dict(whiten=3, H=64, W=68, r=4), lfa.LFA_ERR_UNSUPPORTED),   # reading B: m = 272 > 256 too
    (dict(whiten=-1), lfa.LFA_ERR_INVALID_ARG),
    (dict(d=48), lfa.LFA_ERR_UNSUPPORTED),
    (dict(d=128), lfa.LFA_ERR_UNSUPPORTED),
    (dict(dtype=7), lfa.LFA_ERR_UNSUPPORTED),
    (dict(H=64, W=68, r=4), lfa.LFA_ERR_UNSUPPORTED),   # m = 272 > 256
])
def test_create_rejects_bad_configs(lib, kw, expect):
    cfg = _cfg(**kw)
    assert lfa.workspace_size(cfg) == 0
    h = ctypes.c_void_p()
    st = lib.lfa_create(ctypes.byref(cfg), 256, 256, 1 << 20, ctypes.byref(h))
    assert st == expect
    assert not h.value


def test_reading_b_accepts_the_largest_m(lib):
    # whiten = 3 streams the landmark covariance in 64 x 64 blocks: m = 256 (and a ragged m) plan
    for kw in (dict(H=64, W=64, r=4), dict(H=52, W=76, r=4)):
        assert lfa.workspace_size(_cfg(whiten=3, **kw)) > 0


def test_solver_calls_validate_before_any_device_work(lib):
    assert lfa.solver_workspace_size(0, 49) == 0
    assert lfa.solver_workspace_size(1, 0) == 0
    assert lfa.solver_workspace_size(1, 257) == 0
    n = lfa.solver_workspace_size(3, 49)
    assert n >= 2 * 3 * 49 * 49 * 4
    bad = lfa.LFA_ERR_INVALID_ARG
    p = 256   # an aligned non-null address; every call below must fail its checks before using it
    cg = lib.lfa_cg_solve
    assert cg(None, p, p, 1, 49, 8, 5, None) == bad
    assert cg(p, None, p, 1, 49, 8, 5, None) == bad
    assert cg(p, p, None, 1, 49, 8, 5, None) == bad
    assert cg(p + 4, p, p, 1, 49, 8, 5, None) == bad          # misaligned
    assert cg(p, p, p, 0, 49, 8, 5, None) == bad              # U
    assert cg(p, p, p, 1, 257, 8, 5, None) == bad             # m > 256
    assert cg(p, p, p, 1, 49, 0, 5, None) == bad              # nrhs
    assert cg(p, p, p, 1, 49, 8, -1, None) == bad             # iters
    ns = lib.lfa_ns_solve
    assert ns(None, p, 1, 49, 20, p, n, None, None) == bad
    assert ns(p, p, 1, 49, 65, p, n, None, None) == bad       # T > 64
    assert ns(p, p, 1, 49, -1, p, n, None, None) == bad
    assert ns(p, p, 3, 49, 20, p, n - 1, None, None) == bad   # workspace too small
    assert ns(p, p, 3, 49, 20, p + 16, n, None, None) == bad  # workspace not 256-byte aligned
    assert ns(p, p, 1, 0, 20, p, n, None, None) == bad


def test_create_rejects_null_and_misaligned(lib):
    cfg = _cfg()
    h = ctypes.c_void_p()
    n = lfa.workspace_size(cfg)
    assert lib.lfa_create(ctypes.byref(cfg), None, 256, n, ctypes.byref(h)) == lfa.LFA_ERR_INVALID_ARG
    assert lib.lfa_create(ctypes.byref(cfg), 256, None, n, ctypes.byref(h)) == lfa.LFA_ERR_INVALID_ARG
    assert lib.lfa_create(ctypes.byref(cfg), 256, 256 + 16, n, ctypes.byref(h)) == lfa.LFA_ERR_INVALID_ARG
    assert lib.lfa_create(ctypes.byref(cfg), 256 + 4, 256, n, ctypes.byref(h)) == lfa.LFA_ERR_INVALID_ARG
    assert lib.lfa_create(ctypes.byref(cfg), 256, 256, n - 1, ctypes.byref(h)) == lfa.LFA_ERR_INVALID_ARG
    assert lib.lfa_create(ctypes.byref(cfg), 256, 256, n, None) == lfa.LFA_ERR_INVALID_ARG


def test_null_handle_calls(lib):
    assert lib.lfa_forward(None, 16, 16, 16, None) == lfa.LFA_ERR_INVALID_ARG
    assert lib.lfa_backward(None, 16, 16, 16, 16, 16, None) == lfa.LFA_ERR_INVALID_ARG
    assert lib.lfa_destroy(None) == lfa.LFA_ERR_INVALID_ARG
    assert lib.lfa_forward_path(None) == b"invalid"


def test_workspace_holds_no_n_by_m_matrix(lib):
    # C (N x m) is never stored: at N = 65536, m = 256, d = 32 the whole workspace stays below
    # the 64 MiB that one fp32 C of a single unit would take. It grows with N only through the
    # row-partition partials (at most 296 partitions) and the backward's fp32 dQ staging (N x d).
    n = lfa.workspace_size(_cfg(H=256, W=256, r=16, d=32, T=24))
    assert 0 < n < 65536 * 256 * 4


def test_library_needs_no_python_or_torch(lib):
    # the dynamic section of the built library lists its shared-library dependencies
    import subprocess
    out = subprocess.run(["readelf", "-d", lfa.LIB_PATH], capture_output=True, text=True, check=True).stdout
    needed = [line.split("[")[1].split("]")[0] for line in out.splitlines() if "(NEEDED)" in line]
    assert needed, out
    for n in needed:
        assert "python" not in n and "torch" not in n and "c10" not in n, n
