"""B200 (sm_100a) Mamba-3 SSM layer scan -- Python binding of include/m3.h.

The functions below carry the C ABI's names and only marshal arguments: they
check tensor placement, dtype and contiguity, turn tensors into device
pointers and call ``libm3.so`` through ctypes on the current torch stream.
Every step of the scan runs in the library's CUDA kernels; there is no
PyTorch or CPU implementation behind these calls, and importing the package
fails if the library has not been built (``python -m
selective_state_space_m3_b200.build``).

With ``M3_DEBUG_BOUNDS=1`` in the environment at import, the package loads
``libm3_debug.so`` instead: the same kernels with every global and
shared-memory index checked (failed checks skip the access and are counted;
read them with :func:`m3_debug_bounds_report`).  It is built beside the
release library (``python -m selective_state_space_m3_b200.build --all``).
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Optional

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
DEBUG_BOUNDS = os.environ.get("M3_DEBUG_BOUNDS", "") == "1"
LIB_PATH = os.path.join(_PKG, "libm3_debug.so" if DEBUG_BOUNDS else "libm3.so")

M3_OK, M3_ERR_INVALID_ARG, M3_ERR_UNSUPPORTED, M3_ERR_WORKSPACE, M3_ERR_CUDA, M3_ERR_DEVICE_TIMEOUT = range(6)
M3_F32, M3_BF16 = 0, 1


class M3Error(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {m3_status_string(status)} (status {status})")


class _Dims(ctypes.Structure):
    _fields_ = [(k, ctypes.c_int) for k in
                ("batch", "seqlen", "nheads", "ngroups", "headdim", "dstate", "rank", "chunk",
                 "io_dtype")]


class _Carry(ctypes.Structure):
    _fields_ = [("h", ctypes.c_void_p), ("prev_B", ctypes.c_void_p), ("prev_x", ctypes.c_void_p)]


class _BoundsReport(ctypes.Structure):
    _fields_ = [("enabled", ctypes.c_int), ("failures", ctypes.c_uint), ("site", ctypes.c_int),
                ("index", ctypes.c_longlong), ("limit", ctypes.c_longlong)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: the CUDA library must be built "
                          "(python -m selective_state_space_m3_b200.build"
                          f"{' --debug' if DEBUG_BOUNDS else ''})")
    lib = ctypes.CDLL(LIB_PATH)
    V, S, I = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
    D, C = ctypes.POINTER(_Dims), ctypes.POINTER(_Carry)
    lib.m3_scan_workspace_size.argtypes = [D, ctypes.POINTER(S)]
    lib.m3_scan_fwd.argtypes = [D, V, V, V, V, V, V, V, C, V, C, V, S, V]
    lib.m3_step.argtypes = [D, C, V, V, V, V, V, V, V, V, V]
    lib.m3_rope_bc.argtypes = [D, V, V, V, V, V, V, V, V]
    lib.m3_device_status.argtypes = [V, V]
    IP = ctypes.POINTER(I)
    lib.m3_scan_plan.argtypes = [D, IP, IP, IP, IP]
    lib.m3_scan_plan.restype = I
    lib.m3_scan_fwd_static.argtypes = [D, V, V, V, V, V, V, V, C, V, C, V]
    lib.m3_scan_fwd_static.restype = I
    lib.m3_static_forget_device.argtypes = []
    lib.m3_static_forget_device.restype = I
    lib.m3_selftest_bounded_wait.argtypes = [V, S, V]
    lib.m3_selftest_bounded_wait.restype = I
    lib.m3_debug_bounds_report.argtypes = [ctypes.POINTER(_BoundsReport), I]
    lib.m3_debug_bounds_report.restype = I
    LL = ctypes.c_longlong
    lib.m3_selftest_bounds_check.argtypes = [V, LL, LL, LL, V]
    lib.m3_selftest_bounds_check.restype = I
    lib.m3_scan_bwd_workspace_size.argtypes = [D, ctypes.POINTER(S)]
    lib.m3_scan_bwd_workspace_size.restype = I
    lib.m3_scan_bwd.argtypes = [D, V, V, V, V, V, V, V, C, V, C, V, V, V, V, V, V, V, C, V, S, V]
    lib.m3_scan_bwd.restype = I
    lib.m3_scan_phase_workspace_size.argtypes = [D, I, ctypes.POINTER(S)]
    lib.m3_scan_phase_workspace_size.restype = I
    lib.m3_scan_fwd_phase.argtypes = [D, I, V, V, V, V, V, V, V, V, V, C, V, C, V, S, V]
    lib.m3_scan_fwd_phase.restype = I
    lib.m3_scan_fwd_damped.argtypes = [D, I, V, V, V, V, V, V, V, C, V, C, V]
    lib.m3_scan_fwd_damped.restype = I
    lib.m3_scan_fwd_reflect.argtypes = [D, V, V, V, V, V, V, V, V, C, V, C, V]
    lib.m3_scan_fwd_reflect.restype = I
    lib.m3_status_string.argtypes = [I]
    lib.m3_status_string.restype = ctypes.c_char_p
    for f in ("m3_scan_workspace_size", "m3_scan_fwd", "m3_step", "m3_rope_bc", "m3_device_status"):
        getattr(lib, f).restype = I
    return lib


_lib = _load()

# every symbol include/m3.h declares (checked by the CPU test suite)
ABI_SYMBOLS = ("m3_scan_workspace_size", "m3_scan_fwd", "m3_step", "m3_rope_bc",
               "m3_scan_plan", "m3_device_status", "m3_selftest_bounded_wait", "m3_debug_bounds_report",
               "m3_selftest_bounds_check", "m3_scan_fwd_static",
               "m3_static_forget_device", "m3_scan_bwd_workspace_size", "m3_scan_bwd", "m3_scan_phase_workspace_size",
               "m3_scan_fwd_phase", "m3_scan_fwd_damped", "m3_scan_fwd_reflect", "m3_status_string")


@dataclasses.dataclass
class Dims:
    batch: int
    seqlen: int
    nheads: int
    ngroups: int
    headdim: int
    dstate: int
    rank: int = 1
    chunk: int = 64
    io_dtype: int = M3_BF16

    def c(self) -> _Dims:
        return _Dims(self.batch, self.seqlen, self.nheads, self.ngroups, self.headdim,
                     self.dstate, self.rank, self.chunk, self.io_dtype)


@dataclasses.dataclass
class Carry:
    h: Optional[torch.Tensor] = None        # [b][h][n][p] float32
    prev_B: Optional[torch.Tensor] = None   # [b][h][r][n] io dtype
    prev_x: Optional[torch.Tensor] = None   # [b][h][r][p] io dtype

    def c(self) -> _Carry:
        return _Carry(_ptr(self.h), _ptr(self.prev_B), _ptr(self.prev_x))


def io_dtype_of(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return M3_BF16
    if t.dtype == torch.float32:
        return M3_F32
    raise TypeError(f"io tensors must be float32 or bfloat16, got {t.dtype}")


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("m3 takes device tensors")
    if not t.is_contiguous():
        raise ValueError("m3 takes contiguous tensors")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check(status: int, what: str):
    if status != M3_OK:
        raise M3Error(status, what)


def m3_status_string(status: int) -> str:
    return _lib.m3_status_string(int(status)).decode()


def m3_scan_workspace_size(dims: Dims) -> int:
    n = ctypes.c_size_t(0)
    d = dims.c()
    _check(_lib.m3_scan_workspace_size(ctypes.byref(d), ctypes.byref(n)), "m3_scan_workspace_size")
    return int(n.value)


def m3_scan_plan(dims: Dims) -> dict:
    """Host-only: launches per call, segments, chunk length used, path."""
    d = dims.c()
    out = [ctypes.c_int(0) for _ in range(4)]
    _check(_lib.m3_scan_plan(ctypes.byref(d), *[ctypes.byref(o) for o in out]), "m3_scan_plan")
    return dict(launches=out[0].value, segments=out[1].value, chunk_used=out[2].value,
                path=("simt", "tcgen05")[out[3].value])


def m3_scan_fwd(dims: Dims, x, B, C, dt, A, lam, theta, y, workspace,
                init: Optional[Carry] = None, final_state: Optional[Carry] = None, stream=None) -> None:
    """Chunked prefill (see include/m3.h).  All tensors on the device,
    contiguous, in the ABI's layouts; ``y`` and ``final_state`` are written."""
    d = dims.c()
    ci = init.c() if init is not None else None
    cf = final_state.c() if final_state is not None else None
    st = _lib.m3_scan_fwd(ctypes.byref(d), _ptr(x), _ptr(B), _ptr(C), _ptr(dt), _ptr(A), _ptr(lam),
                          _ptr(theta), ctypes.byref(ci) if ci is not None else None, _ptr(y),
                          ctypes.byref(cf) if cf is not None else None, _ptr(workspace),
                          workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "m3_scan_fwd")


def m3_scan_fwd_static(dims: Dims, x, B, C, dt, A, lam, theta, y,
                       init: Optional[Carry] = None, final_state: Optional[Carry] = None, stream=None) -> None:
    """m3_scan_fwd without a workspace, for callers that cannot allocate device
    memory: the scratch is a fixed array inside the library (see include/m3.h
    for the size limit and for why overlapping calls must be serialised)."""
    d = dims.c()
    ci = init.c() if init is not None else None
    cf = final_state.c() if final_state is not None else None
    st = _lib.m3_scan_fwd_static(ctypes.byref(d), _ptr(x), _ptr(B), _ptr(C), _ptr(dt), _ptr(A), _ptr(lam),
                                 _ptr(theta), ctypes.byref(ci) if ci is not None else None, _ptr(y),
                                 ctypes.byref(cf) if cf is not None else None, _stream(stream))
    _check(st, "m3_scan_fwd_static")


def m3_static_forget_device() -> None:
    """Drop the static scratch array's cached address for the current device
    (only needed after a device reset)."""
    _check(_lib.m3_static_forget_device(), "m3_static_forget_device")


def m3_step(dims: Dims, state: Carry, x, B, C, dt, A, lam, theta, y, stream=None) -> None:
    """One decode token; ``state`` is updated in place."""
    d = dims.c()
    cs = state.c()
    st = _lib.m3_step(ctypes.byref(d), ctypes.byref(cs), _ptr(x), _ptr(B), _ptr(C), _ptr(dt),
                      _ptr(A), _ptr(lam), _ptr(theta), _ptr(y), _stream(stream))
    _check(st, "m3_step")


def m3_rope_bc(dims: Dims, B, C, dt, theta, B_rot, C_rot, phase=None, stream=None) -> None:
    d = dims.c()
    st = _lib.m3_rope_bc(ctypes.byref(d), _ptr(B), _ptr(C), _ptr(dt), _ptr(theta), _ptr(B_rot),
                         _ptr(C_rot), _ptr(phase), _stream(stream))
    _check(st, "m3_rope_bc")


def m3_device_status(workspace, stream=None) -> int:
    """Synchronises the stream; returns (and clears) the workspace status."""
    return int(_lib.m3_device_status(_ptr(workspace), _stream(stream)))


def m3_selftest_bounded_wait(workspace, stream=None) -> None:
    """Launch the bounded-wait diagnostic; read the result with m3_device_status."""
    _check(_lib.m3_selftest_bounded_wait(_ptr(workspace), workspace.numel() * workspace.element_size(),
                                         _stream(stream)), "m3_selftest_bounded_wait")


def m3_debug_bounds_report(clear: bool = False) -> dict:
    """The index checks' record (synchronises the device in the debug build):
    enabled (1 in libm3_debug.so), failures, and site / index / limit of the
    first failure."""
    r = _BoundsReport()
    _check(_lib.m3_debug_bounds_report(ctypes.byref(r), int(bool(clear))), "m3_debug_bounds_report")
    return {"enabled": r.enabled, "failures": r.failures, "site": r.site, "index": r.index, "limit": r.limit}


def m3_selftest_bounds_check(buffer, index: int, limit: int, stream=None) -> None:
    """Debug build: one thread stores 1.0 to buffer[index] if index < limit
    (float32 device buffer; index and limit within its size)."""
    if buffer.dtype != torch.float32:
        raise TypeError("the self-test buffer is float32")
    _check(_lib.m3_selftest_bounds_check(_ptr(buffer), buffer.numel(), int(index), int(limit), _stream(stream)),
           "m3_selftest_bounds_check")


def m3_scan_bwd_workspace_size(dims: Dims) -> int:
    n = ctypes.c_size_t(0)
    d = dims.c()
    _check(_lib.m3_scan_bwd_workspace_size(ctypes.byref(d), ctypes.byref(n)), "m3_scan_bwd_workspace_size")
    return n.value


def m3_scan_bwd(dims: Dims, x, B, C, dt, A, lam, theta, dy, grads: dict, workspace,
                init: Optional[Carry] = None, d_final: Optional[Carry] = None,
                d_init: Optional[Carry] = None, stream=None) -> None:
    """Backward pass (see include/m3.h).  ``grads`` holds the float32 output
    tensors dx, dB, dC, ddt, dA, dlam, dtheta; ``d_final`` / ``d_init`` are
    Carry objects of float32 tensors (members may be None)."""
    d = dims.c()
    ci = init.c() if init is not None else None
    cf = d_final.c() if d_final is not None else None
    cd = d_init.c() if d_init is not None else None
    g = grads
    st = _lib.m3_scan_bwd(ctypes.byref(d), _ptr(x), _ptr(B), _ptr(C), _ptr(dt), _ptr(A), _ptr(lam), _ptr(theta),
                          ctypes.byref(ci) if ci is not None else None, _ptr(dy),
                          ctypes.byref(cf) if cf is not None else None,
                          _ptr(g["dx"]), _ptr(g["dB"]), _ptr(g["dC"]), _ptr(g["ddt"]), _ptr(g["dA"]),
                          _ptr(g["dlam"]), _ptr(g["dtheta"]), ctypes.byref(cd) if cd is not None else None,
                          _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "m3_scan_bwd")


M3_PHASE_NATIVE, M3_PHASE_ZERO, M3_PHASE_REVERSE, M3_PHASE_SHUFFLE, M3_PHASE_FIXED, \
    M3_PHASE_WRITE_ONLY, M3_PHASE_READ_ONLY = range(7)


def m3_scan_phase_workspace_size(dims: Dims, mode: int) -> int:
    n = ctypes.c_size_t(0)
    d = dims.c()
    _check(_lib.m3_scan_phase_workspace_size(ctypes.byref(d), int(mode), ctypes.byref(n)),
           "m3_scan_phase_workspace_size")
    return n.value


def m3_scan_fwd_phase(dims: Dims, mode: int, x, B, C, dt, A, lam, theta, y, workspace, perm=None, freq=None,
                      init: Optional[Carry] = None, final_state: Optional[Carry] = None, stream=None) -> None:
    """m3_scan_fwd under a phase intervention (see include/m3.h).  ``perm``
    (SHUFFLE) and ``freq`` (FIXED) are host sequences / arrays."""
    d = dims.c()
    ci = init.c() if init is not None else None
    cf = final_state.c() if final_state is not None else None
    perm_c = (ctypes.c_int * len(perm))(*[int(v) for v in perm]) if perm is not None else None
    freq_c = None
    if freq is not None:
        flat = [float(v) for v in np.asarray(freq, dtype=np.float32).ravel()]
        freq_c = (ctypes.c_float * len(flat))(*flat)
    st = _lib.m3_scan_fwd_phase(ctypes.byref(d), int(mode),
                                ctypes.cast(perm_c, ctypes.c_void_p) if perm_c is not None else None,
                                ctypes.cast(freq_c, ctypes.c_void_p) if freq_c is not None else None,
                                _ptr(x), _ptr(B), _ptr(C), _ptr(dt), _ptr(A), _ptr(lam), _ptr(theta),
                                ctypes.byref(ci) if ci is not None else None, _ptr(y),
                                ctypes.byref(cf) if cf is not None else None, _ptr(workspace),
                                workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "m3_scan_fwd_phase")


M3_DAMP_UNDER, M3_DAMP_CRITICAL, M3_DAMP_OVER = range(3)


def m3_scan_fwd_damped(dims: Dims, regime: int, x, B, C, dt, A, lam, theta, y,
                       init: Optional[Carry] = None, final_state: Optional[Carry] = None, stream=None) -> None:
    """The scan under a damping regime (M3_DAMP_UNDER / CRITICAL / OVER; see
    include/m3.h).  No workspace."""
    d = dims.c()
    ci = init.c() if init is not None else None
    cf = final_state.c() if final_state is not None else None
    st = _lib.m3_scan_fwd_damped(ctypes.byref(d), int(regime), _ptr(x), _ptr(B), _ptr(C), _ptr(dt), _ptr(A),
                                 _ptr(lam), _ptr(theta), ctypes.byref(ci) if ci is not None else None, _ptr(y),
                                 ctypes.byref(cf) if cf is not None else None, _stream(stream))
    _check(st, "m3_scan_fwd_damped")


def m3_scan_fwd_reflect(dims: Dims, u, x, B, C, dt, A, lam, theta, y,
                        init: Optional[Carry] = None, final_state: Optional[Carry] = None, stream=None) -> None:
    """The scan with the low-rank reflection term; ``u`` [b][t][g][n] in the
    io dtype (see include/m3.h).  No workspace."""
    d = dims.c()
    ci = init.c() if init is not None else None
    cf = final_state.c() if final_state is not None else None
    st = _lib.m3_scan_fwd_reflect(ctypes.byref(d), _ptr(u), _ptr(x), _ptr(B), _ptr(C), _ptr(dt), _ptr(A),
                                  _ptr(lam), _ptr(theta), ctypes.byref(ci) if ci is not None else None, _ptr(y),
                                  ctypes.byref(cf) if cf is not None else None, _stream(stream))
    _check(st, "m3_scan_fwd_reflect")


def raw_lib():
    """The ctypes handle (for calls that pass raw pointers)."""
    return _lib


__all__ = ["Dims", "Carry", "M3Error", "m3_scan_workspace_size", "m3_scan_fwd", "m3_step",
           "m3_rope_bc", "m3_scan_plan", "m3_device_status", "m3_selftest_bounded_wait", "m3_debug_bounds_report",
           "m3_selftest_bounds_check", "DEBUG_BOUNDS", "m3_scan_fwd_static",
           "m3_static_forget_device", "m3_scan_bwd_workspace_size", "m3_scan_bwd", "m3_status_string",
           "m3_scan_phase_workspace_size", "m3_scan_fwd_phase", "m3_scan_fwd_damped", "m3_scan_fwd_reflect",
           "M3_DAMP_UNDER", "M3_DAMP_CRITICAL", "M3_DAMP_OVER", "io_dtype_of", "ABI_SYMBOLS",
           "M3_F32", "M3_BF16", "raw_lib", "LIB_PATH"]
