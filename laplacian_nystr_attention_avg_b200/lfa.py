"""Thin ctypes binding of liblfa.so (include/lfa.h). Argument marshalling only.

PyTorch supplies device memory and streams; every step of the attention path runs
in the library's CUDA kernels. If the library is missing this module raises: there
is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import List, Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "liblfa.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "lfa.h")

LFA_OK, LFA_ERR_INVALID_ARG, LFA_ERR_UNSUPPORTED, LFA_ERR_CUDA, LFA_ERR_STATE, \
    LFA_ERR_TIMEOUT, LFA_ERR_NONFINITE, LFA_ERR_SCRATCH_LIMIT = range(8)
LFA_NOALLOC_SCRATCH_BYTES = 16 << 20
LFA_F32, LFA_BF16 = 0, 1
LFA_WHITEN_BATCH = 2   # cfg.whiten: column statistics pooled per head over the batch
LFA_WHITEN_FULL = 3    # cfg.whiten: Reading B, whitening of the columns of the whole Nystrom matrix


class Config(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("heads", ctypes.c_int), ("H", ctypes.c_int), ("W", ctypes.c_int),
                ("d", ctypes.c_int), ("r", ctypes.c_int), ("lambda_", ctypes.c_float),
                ("eps", ctypes.c_float), ("T", ctypes.c_int), ("dtype", ctypes.c_int),
                ("whiten", ctypes.c_int)]


class UnitInfo(ctypes.Structure):
    _fields_ = [("alpha_fallback", ctypes.c_int), ("alpha", ctypes.c_float),
                ("lambda_max", ctypes.c_float), ("ns_residual_fro", ctypes.c_float),
                ("kappa", ctypes.c_float)]


class LfaError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


_lib: Optional[ctypes.CDLL] = None


def _declare(lib: ctypes.CDLL) -> None:
    vp, sz, ci = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
    cfgp = ctypes.POINTER(Config)
    sig = {
        "lfa_workspace_size": (sz, [cfgp]),
        "lfa_create": (ci, [cfgp, vp, vp, sz, ctypes.POINTER(vp)]),
        "lfa_forward": (ci, [vp, vp, vp, vp, vp]),
        "lfa_forward_host": (ci, [vp, vp, vp, vp, vp, vp, vp, vp]),
        "lfa_forward_host_async": (ci, [vp, vp, vp, vp, vp, vp, vp, vp]),
        "lfa_forward_noalloc": (ci, [cfgp, vp, vp, vp, vp, vp]),
        "lfa_backward": (ci, [vp, vp, vp, vp, vp, vp, vp]),
        "lfa_get_info": (ci, [vp, ctypes.POINTER(UnitInfo), ci, vp]),
        "lfa_destroy": (ci, [vp]),
        "lfa_status_string": (ctypes.c_char_p, [ci]),
        "lfa_debug_cross_kernel": (ci, [vp, vp, ci, vp, vp]),
        "lfa_debug_capture_cross": (ci, [vp, ci, vp, vp]),
        "lfa_debug_spin_test": (ci, [vp, ctypes.c_longlong]),
        "lfa_debug_context": (ci, [vp, ci, vp, vp, vp, vp, vp]),
        "lfa_forward_path": (ctypes.c_char_p, [vp]),
        "lfa_set_profile_events": (ci, [vp, vp, vp]),
        "lfa_dominant_kernel": (ctypes.c_char_p, [vp]),
        "lfa_launches_per_forward": (ci, [vp]),
        "lfa_debug_trace": (ci, [vp, vp]),
        "lfa_fused_grid": (ci, [vp]),
        "lfa_debug_selftest": (ci, [ci, vp, vp, vp, ci, vp, ci, vp, vp]),
        "lfa_sp_workspace_size": (sz, [cfgp, ci, ci]),
        "lfa_sp_create": (ci, [cfgp, ci, ci, vp, vp, sz, ctypes.POINTER(vp)]),
        "lfa_sp_partial_size": (ci, [vp]),
        "lfa_sp_pool": (ci, [vp, vp, vp, vp]),
        "lfa_sp_pass1": (ci, [vp, vp, vp, vp, vp, vp]),
        "lfa_sp_pass2": (ci, [vp, vp, vp, vp, vp, vp, vp]),
        "lfa_solver_workspace_size": (sz, [ci, ci]),
        "lfa_ns_solve": (ci, [vp, vp, ci, ci, ci, vp, sz, ctypes.POINTER(UnitInfo), vp]),
        "lfa_cg_solve": (ci, [vp, vp, vp, ci, ci, ci, ci, vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args


def load() -> ctypes.CDLL:
    """Open liblfa.so from the package directory (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"liblfa.so not found at {LIB_PATH}; build it with "
                               "`python -m laplacian_nystr_attention_avg_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        _declare(lib)
        _lib = lib
    return _lib


def header_symbols() -> List[str]:
    """Names of the entry points declared in include/lfa.h."""
    with open(HEADER_PATH) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(lfa_[a-z_]+)\s*\(", text)))


def selftest(mode: int, A: Optional[torch.Tensor], B: Optional[torch.Tensor], param: int = 0,
             tma_src: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Run one tensor-core / TMA building-block self-test; returns D [128, 64] fp32 (device)."""
    dev = (A if A is not None else tma_src).device
    D = torch.zeros((128, 64), dtype=torch.float32, device=dev)
    status = torch.zeros((1,), dtype=torch.int32, device=dev)
    rows = 0 if tma_src is None else tma_src.shape[0]
    _check(load().lfa_debug_selftest(int(mode), _ptr(A), _ptr(B), _ptr(D), int(param), _ptr(tma_src), int(rows),
                                     _ptr(status), _stream(None)), "lfa_debug_selftest")
    torch.cuda.synchronize()
    if int(status.item()) != 0:
        raise LfaError(LFA_ERR_TIMEOUT, "lfa_debug_selftest")
    return D


def status_string(status: int) -> str:
    return load().lfa_status_string(int(status)).decode()


def _check(status: int, what: str) -> None:
    if status != LFA_OK:
        raise LfaError(status, what)


def make_config(wl, whiten=True) -> Config:
    """lfa_config from a Workload (laplacian_nystr_attention_avg_b200.inputs).

    whiten: True (per-unit column statistics), False (raw C), "batch" (statistics
    pooled per head over the batch; cfg.whiten = LFA_WHITEN_BATCH) or "full" (Reading B:
    the columns of the whole Nystrom matrix; cfg.whiten = LFA_WHITEN_FULL).
    """
    wv = {"batch": LFA_WHITEN_BATCH, "full": LFA_WHITEN_FULL}.get(whiten, None) if isinstance(whiten, str) \
        else (1 if whiten else 0)
    if wv is None:
        raise ValueError(f"whiten: {whiten!r}")
    return Config(wl.B, wl.heads, wl.H, wl.W, wl.d, wl.r, float(wl.lam), float(wl.eps), int(wl.T),
                  LFA_BF16 if wl.dtype == "bf16" else LFA_F32, wv)


def workspace_size(cfg: Config) -> int:
    return int(load().lfa_workspace_size(ctypes.byref(cfg)))


def solver_workspace_size(U: int, m: int) -> int:
    return int(load().lfa_solver_workspace_size(int(U), int(m)))


def ns_solve(W: torch.Tensor, T: int, stream=None):
    """lfa_ns_solve: the forward pass's T-step Newton-Schulz approximation of W^-1 for each of the
    U symmetric positive-definite matrices W [U, m, m] (device float32). Returns (X, [UnitInfo])."""
    if W.dim() != 3 or W.shape[1] != W.shape[2]:
        raise ValueError(f"W: expected [U, m, m], got {tuple(W.shape)}")
    U, m = int(W.shape[0]), int(W.shape[1])
    _require(W, "W", (U, m, m), torch.float32, W.device)
    X = torch.empty_like(W)
    nbytes = solver_workspace_size(U, m)
    if nbytes == 0:
        raise LfaError(LFA_ERR_INVALID_ARG, "lfa_solver_workspace_size")
    ws = torch.empty((nbytes + 256,), dtype=torch.uint8, device=W.device)
    off = (-ws.data_ptr()) % 256
    info = (UnitInfo * U)()
    _check(load().lfa_ns_solve(_ptr(W), _ptr(X), U, m, int(T), ctypes.c_void_p(ws.data_ptr() + off), nbytes,
                               info, _stream(stream)), "lfa_ns_solve")
    return X, list(info)


def cg_solve(W: torch.Tensor, B: torch.Tensor, iters: int, stream=None) -> torch.Tensor:
    """lfa_cg_solve: conjugate gradients for W Y = B, W [U, m, m] symmetric positive definite,
    B [U, m, nrhs] (device float32), exactly `iters` iterations from Y = 0. Returns Y."""
    if W.dim() != 3 or W.shape[1] != W.shape[2] or B.dim() != 3:
        raise ValueError(f"W [U, m, m] and B [U, m, nrhs] expected, got {tuple(W.shape)}, {tuple(B.shape)}")
    U, m, nrhs = int(W.shape[0]), int(W.shape[1]), int(B.shape[2])
    _require(W, "W", (U, m, m), torch.float32, W.device)
    _require(B, "B", (U, m, nrhs), torch.float32, W.device)
    Y = torch.empty_like(B)
    _check(load().lfa_cg_solve(_ptr(W), _ptr(B), _ptr(Y), U, m, nrhs, int(iters), _stream(stream)), "lfa_cg_solve")
    return Y


def forward_noalloc(cfg: Config, dwc_weight: torch.Tensor, Q: torch.Tensor, V: torch.Tensor,
                    O: torch.Tensor, stream=None) -> torch.Tensor:
    """lfa_forward_noalloc: handle-free forward over the library's static scratch area.

    dwc_weight: device float32 [heads, d, 3, 3]; Q, V, O: device [B, heads, N, d] in the
    config's dtype. Raises LfaError (LFA_ERR_SCRATCH_LIMIT) when the config does not fit.
    """
    shape, dt = _cfg_shape(cfg), _cfg_dtype(cfg)
    _require(Q, "Q", shape, dt)
    _require(V, "V", shape, dt, Q.device)
    _require(O, "O", shape, dt, Q.device)
    _require(dwc_weight, "dwc_weight", (cfg.heads, cfg.d, 3, 3), torch.float32, Q.device)
    _check(load().lfa_forward_noalloc(ctypes.byref(cfg), _ptr(dwc_weight), _ptr(Q), _ptr(V), _ptr(O),
                                      _stream(stream)), "lfa_forward_noalloc")
    return O


def _require(t: torch.Tensor, name: str, shape, dtype, device=None, host: bool = False) -> None:
    """Reject a tensor the library would read or write out of bounds: wrong dtype, shape, layout or
    device. (The library sees only a pointer, so these checks live in the binding.)"""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if host:
        if t.device.type != "cpu":
            raise ValueError(f"{name}: expected a host tensor")
    elif t.device.type != "cuda" or (device is not None and t.device != device):
        raise ValueError(f"{name}: on {t.device}, expected {device if device is not None else 'a CUDA device'}")


def _cfg_shape(cfg: Config):
    return (cfg.B, cfg.heads, cfg.H * cfg.W, cfg.d)


def _cfg_dtype(cfg: Config):
    return torch.bfloat16 if cfg.dtype == LFA_BF16 else torch.float32


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


class LaplacianNystromAttention:
    """One configured attention call: owns a torch-allocated workspace and an lfa handle.

    dwc_weight: float32 [heads, d, 3, 3] (moved to the device). Q, V, O tensors are
    [B, heads, N, d] contiguous in the config's dtype on the same device.
    """

    def __init__(self, cfg: Config, dwc_weight: torch.Tensor, device: str = "cuda"):
        self.lib = load()
        self.cfg = cfg
        self.device = torch.device(device)
        if self.device.type == "cuda" and self.device.index is None:
            self.device = torch.device("cuda", torch.cuda.current_device())
        self.dtype = torch.bfloat16 if cfg.dtype == LFA_BF16 else torch.float32
        self.units = cfg.B * cfg.heads
        self.N = cfg.H * cfg.W
        self.m = (cfg.H // cfg.r) * (cfg.W // cfg.r)
        self.shape = (cfg.B, cfg.heads, self.N, cfg.d)
        self.weight = dwc_weight.to(self.device, torch.float32).contiguous()
        _require(self.weight, "dwc_weight", (cfg.heads, cfg.d, 3, 3), torch.float32, self.device)
        nbytes = workspace_size(cfg)
        if nbytes == 0:
            raise LfaError(LFA_ERR_INVALID_ARG, "lfa_workspace_size")
        self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        h = ctypes.c_void_p()
        _check(self.lib.lfa_create(ctypes.byref(cfg), self.weight.data_ptr(), self.workspace.data_ptr(),
                                   nbytes, ctypes.byref(h)), "lfa_create")
        self.handle = h

    @property
    def path(self) -> str:
        return self.lib.lfa_forward_path(self.handle).decode()

    @property
    def launches_per_forward(self) -> int:
        return int(self.lib.lfa_launches_per_forward(self.handle))

    @property
    def dominant_kernel(self) -> str:
        return self.lib.lfa_dominant_kernel(self.handle).decode()

    def set_profile_events(self, begin=None, end=None) -> None:
        """Bracket the dominant kernel of later forwards with two torch.cuda.Event objects."""
        for ev in (begin, end):
            if ev is not None and not ev.cuda_event:
                ev.record()          # torch creates the CUDA event lazily, on first record
        b = None if begin is None else begin.cuda_event
        e = None if end is None else end.cuda_event
        _check(self.lib.lfa_set_profile_events(self.handle, b, e), "lfa_set_profile_events")

    @property
    def fused_grid(self) -> int:
        return int(self.lib.lfa_fused_grid(self.handle))

    def set_trace(self, buf: Optional[torch.Tensor]) -> None:
        """Record fused-kernel phase timestamps into buf (int64 [grid, 32], device) or stop (None)."""
        _check(self.lib.lfa_debug_trace(self.handle, _ptr(buf)), "lfa_debug_trace")

    def new_output(self) -> torch.Tensor:
        return torch.empty(self.shape, dtype=self.dtype, device=self.device)

    def forward(self, Q: torch.Tensor, V: torch.Tensor, O: Optional[torch.Tensor] = None,
                stream=None) -> torch.Tensor:
        if O is None:
            O = self.new_output()
        for name, t in (("Q", Q), ("V", V), ("O", O)):
            _require(t, name, self.shape, self.dtype, self.device)
        _check(self.lib.lfa_forward(self.handle, _ptr(Q), _ptr(V), _ptr(O), _stream(stream)), "lfa_forward")
        return O

    def forward_host(self, Q_host, V_host, O_host, Q_dev, V_dev, O_dev, stream=None) -> None:
        for name, t in (("Q_host", Q_host), ("V_host", V_host), ("O_host", O_host)):
            _require(t, name, self.shape, self.dtype, host=True)
        for name, t in (("Q_dev", Q_dev), ("V_dev", V_dev), ("O_dev", O_dev)):
            _require(t, name, self.shape, self.dtype, self.device)
        _check(self.lib.lfa_forward_host(self.handle, _ptr(Q_host), _ptr(V_host), _ptr(O_host), _ptr(Q_dev),
                                         _ptr(V_dev), _ptr(O_dev), _stream(stream)), "lfa_forward_host")

    def forward_host_async(self, Q_host, V_host, O_host, Q_dev, V_dev, O_dev, stream=None) -> None:
        """lfa_forward_host_async: enqueue copies in, the forward and the copy out; O_host is ready once
        `stream` has been synchronised."""
        for name, t in (("Q_host", Q_host), ("V_host", V_host), ("O_host", O_host)):
            _require(t, name, self.shape, self.dtype, host=True)
        for name, t in (("Q_dev", Q_dev), ("V_dev", V_dev), ("O_dev", O_dev)):
            _require(t, name, self.shape, self.dtype, self.device)
        _check(self.lib.lfa_forward_host_async(self.handle, _ptr(Q_host), _ptr(V_host), _ptr(O_host), _ptr(Q_dev),
                                               _ptr(V_dev), _ptr(O_dev), _stream(stream)), "lfa_forward_host_async")

    def backward(self, Q, V, dO, dQ=None, dV=None, stream=None):
        if dQ is None:
            dQ = self.new_output()
        if dV is None:
            dV = self.new_output()
        for name, t in (("Q", Q), ("V", V), ("dO", dO), ("dQ", dQ), ("dV", dV)):
            _require(t, name, self.shape, self.dtype, self.device)
        _check(self.lib.lfa_backward(self.handle, _ptr(Q), _ptr(V), _ptr(dO), _ptr(dQ), _ptr(dV),
                                     _stream(stream)), "lfa_backward")
        return dQ, dV

    def info(self, stream=None):
        """(status, [UnitInfo]) of the most recent forward; synchronises the stream."""
        arr = (UnitInfo * self.units)()
        st = self.lib.lfa_get_info(self.handle, arr, self.units, _stream(stream))
        if st not in (LFA_OK, LFA_ERR_TIMEOUT, LFA_ERR_NONFINITE):
            raise LfaError(st, "lfa_get_info")
        return st, list(arr)

    def cross_kernel(self, Q: torch.Tensor, unit: int, stream=None) -> torch.Tensor:
        C = torch.empty((self.N, self.m), dtype=torch.float32, device=self.device)
        _check(self.lib.lfa_debug_cross_kernel(self.handle, _ptr(Q), int(unit), _ptr(C), _stream(stream)),
               "lfa_debug_cross_kernel")
        return C

    def capture_cross(self, Q: torch.Tensor, V: torch.Tensor, unit: int, O: Optional[torch.Tensor] = None,
                      stream=None):
        """(C, shift) of `unit` as one forward computes it (lfa_debug_capture_cross + lfa_forward), each
        fp32 [N, m]: the C that pass 2 uses and the column shift subtracted before its bf16 rounding."""
        C = torch.empty((self.N, self.m), dtype=torch.float32, device=self.device)
        S = torch.empty((self.N, self.m), dtype=torch.float32, device=self.device)
        _check(self.lib.lfa_debug_capture_cross(self.handle, int(unit), _ptr(C), _ptr(S)),
               "lfa_debug_capture_cross")
        self.forward(Q, V, O, stream)
        return C, S

    def arm_spin_test(self, budget_cycles: int) -> None:
        """lfa_debug_spin_test: the next forward's cross-block waits run out after budget_cycles."""
        _check(self.lib.lfa_debug_spin_test(self.handle, int(budget_cycles)), "lfa_debug_spin_test")

    def context(self, unit: int, stream=None):
        d = self.cfg.d
        L = torch.empty((self.m, d), dtype=torch.float32, device=self.device)
        X = torch.empty((self.m, self.m), dtype=torch.float32, device=self.device)
        mu = torch.empty((self.m,), dtype=torch.float32, device=self.device)
        s = torch.empty((self.m,), dtype=torch.float32, device=self.device)
        _check(self.lib.lfa_debug_context(self.handle, int(unit), _ptr(L), _ptr(X), _ptr(mu), _ptr(s),
                                          _stream(stream)), "lfa_debug_context")
        return L, X, mu, s

    def close(self) -> None:
        if getattr(self, "handle", None):
            self.lib.lfa_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class SeqSplitBand:
    """A band of grid rows [y0, y0 + ny) of every unit (lfa_sp_create): the library's three band
    calls. Q, V, O of the band are [B, heads, ny * W, d] in the config's dtype on one device."""

    def __init__(self, cfg: Config, y0: int, ny: int, dwc_weight: torch.Tensor, device: str = "cuda"):
        self.lib = load()
        self.cfg = cfg
        self.y0, self.ny = int(y0), int(ny)
        self.device = torch.device(device)
        if self.device.type == "cuda" and self.device.index is None:
            self.device = torch.device("cuda", torch.cuda.current_device())
        self.dtype = torch.bfloat16 if cfg.dtype == LFA_BF16 else torch.float32
        self.m = (cfg.H // cfg.r) * (cfg.W // cfg.r)
        self.shape = (cfg.B, cfg.heads, self.ny * cfg.W, cfg.d)
        self.weight = dwc_weight.to(self.device, torch.float32).contiguous()
        _require(self.weight, "dwc_weight", (cfg.heads, cfg.d, 3, 3), torch.float32, self.device)
        nbytes = int(self.lib.lfa_sp_workspace_size(ctypes.byref(cfg), self.y0, self.ny))
        if nbytes == 0:
            raise LfaError(LFA_ERR_INVALID_ARG, "lfa_sp_workspace_size")
        self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        h = ctypes.c_void_p()
        _check(self.lib.lfa_sp_create(ctypes.byref(cfg), self.y0, self.ny, self.weight.data_ptr(),
                                      self.workspace.data_ptr(), nbytes, ctypes.byref(h)), "lfa_sp_create")
        self.handle = h
        self.S = int(self.lib.lfa_sp_partial_size(h))

    def pool(self, Q: torch.Tensor, stream=None) -> torch.Tensor:
        _require(Q, "Q", self.shape, self.dtype, self.device)
        L = torch.empty((self.cfg.B, self.cfg.heads, self.m, self.cfg.d), dtype=torch.float32, device=self.device)
        _check(self.lib.lfa_sp_pool(self.handle, _ptr(Q), _ptr(L), _stream(stream)), "lfa_sp_pool")
        return L

    def pass1(self, Q: torch.Tensor, V: torch.Tensor, L: torch.Tensor, stream=None) -> torch.Tensor:
        for name, t in (("Q", Q), ("V", V)):
            _require(t, name, self.shape, self.dtype, self.device)
        _require(L, "L", (self.cfg.B, self.cfg.heads, self.m, self.cfg.d), torch.float32, self.device)
        part = torch.empty((self.cfg.B, self.cfg.heads, self.S), dtype=torch.float64, device=self.device)
        _check(self.lib.lfa_sp_pass1(self.handle, _ptr(Q), _ptr(V), _ptr(L), _ptr(part), _stream(stream)),
               "lfa_sp_pass1")
        return part

    def pass2(self, Q, V, halo, part, O, stream=None):
        for name, t in (("Q", Q), ("V", V), ("O", O)):
            _require(t, name, self.shape, self.dtype, self.device)
        _require(halo, "halo", (self.cfg.B, self.cfg.heads, 2, self.cfg.W, self.cfg.d), self.dtype, self.device)
        _require(part, "partials", (self.cfg.B, self.cfg.heads, self.S), torch.float64, self.device)
        _check(self.lib.lfa_sp_pass2(self.handle, _ptr(Q), _ptr(V), _ptr(halo), _ptr(part), _ptr(O),
                                     _stream(stream)), "lfa_sp_pass2")
        return O

    def close(self) -> None:
        if getattr(self, "handle", None):
            self.lib.lfa_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
