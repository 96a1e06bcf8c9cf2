"""fp64 CPU oracle of the Mamba-3 SSM layer scan -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s cpu-baseline /
reference leg may import this package.  The product package
``selective_state_space_m3_b200`` never imports it, and the two share no code.

The arithmetic lives in ``m3_oracle.c`` (plain C, double precision, the literal
token-by-token recurrence); this module only compiles it with gcc and marshals
float64 numpy arrays through ctypes.

Passages followed (page titles and sections):
  * "Mamba-3" summary (b-lab.team), section 1 "Exponential-Trapezoidal
    Discretization": h_t = a_t h_{t-1} + b_t B_{t-1} x_{t-1} + g_t B_t x_t with
    a_t = exp(dt A), b_t = (1-lam) dt exp(dt A), g_t = lam dt.
  * same page, section 2 "Complex-Valued State Space Model": Proposition 2
    (block-diagonal R(dt theta[i]) rotations, y = C^T h) and Proposition 3
    (the rotation moved onto B and C as a cumulative phase, oracle_rope_bc).
  * same page, section 3 "MIMO": B, C in R^{N x R}, x in R^{P x R}.
  * "Understanding Mamba-3 Through Oscillatory Dynamics", sections 2.2, 4.1,
    4.2 and appendix C.2: the damping-regime variants (scan_damped).
  * the low-rank reflection extension's abstract (listed on the same paper's
    page) and appendix C.4 of that paper: scan_reflect.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "m3_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB = os.path.join(_BUILD, "libm3oracle.so")
_lock = threading.Lock()
_lib = None


class _Dims(ctypes.Structure):
    _fields_ = [(k, ctypes.c_int) for k in
                ("batch", "seqlen", "nheads", "ngroups", "headdim", "dstate", "rank")]


def build(force: bool = False) -> str:
    """Compile m3_oracle.c into oracle/_build/libm3oracle.so (gcc, -O2, OpenMP)."""
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-std=c99",
                        "-o", tmp, _SRC, "-lm"], check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _bind(lib):
    P = ctypes.POINTER(ctypes.c_double)
    D = ctypes.POINTER(_Dims)
    lib.oracle_scan.argtypes = [D] + [P] * 14
    lib.oracle_scan.restype = ctypes.c_int
    lib.oracle_step.argtypes = [D] + [P] * 11
    lib.oracle_step.restype = ctypes.c_int
    lib.oracle_scan_bwd.argtypes = [D] + [P] * 24
    lib.oracle_scan_bwd.restype = ctypes.c_int
    lib.oracle_rope_bc.argtypes = [D] + [P] * 7
    lib.oracle_rope_bc.restype = ctypes.c_int
    lib.oracle_scan_damped.argtypes = [D, ctypes.c_int] + [P] * 14
    lib.oracle_scan_damped.restype = ctypes.c_int
    lib.oracle_scan_reflect.argtypes = [D] + [P] * 15
    lib.oracle_scan_reflect.restype = ctypes.c_int
    lib.oracle_num_threads.argtypes = []
    lib.oracle_num_threads.restype = ctypes.c_int
    lib.oracle_set_num_threads.argtypes = [ctypes.c_int]
    lib.oracle_set_num_threads.restype = None
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = _bind(ctypes.CDLL(build()))
    return _lib


def compile_variant(source_text: str, tag: str):
    """Compile a modified copy of the oracle source (tests plant mistakes in
    it to show that the pins catch them) and return a ctypes handle usable as
    the ``lib=`` argument of scan/step/rope_bc.  The copy is built in a
    temporary directory that is removed once the library is loaded (the
    loaded image stays valid after its file is unlinked)."""
    import tempfile
    with tempfile.TemporaryDirectory(prefix=f"m3oracle_{tag}_") as tmp:
        src = os.path.join(tmp, "variant.c")
        so = os.path.join(tmp, "variant.so")
        with open(src, "w") as f:
            f.write(source_text)
        subprocess.run(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-std=c99",
                        "-o", so, src, "-lm"], check=True)
        return _bind(ctypes.CDLL(so))


def source_text() -> str:
    with open(_SRC) as f:
        return f.read()


def _p(a):
    if a is None:
        return None
    assert a.dtype == np.float64 and a.flags["C_CONTIGUOUS"], "oracle takes C-contiguous float64"
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _f64(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float64)


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def set_num_threads(n: int) -> None:
    """OpenMP threads of later oracle calls (timing only: every (b, h) is
    computed by one thread, so the results do not depend on it)."""
    _load().oracle_set_num_threads(int(n))


def scan(x, B, C, dt, A, lam, theta, init_h=None, init_pB=None, init_pX=None, lib=None):
    """Full-sequence oracle.

    x [b,t,h,r,p]; B, C [b,t,g,r,n]; dt, lam [b,t,h]; A [h]; theta [b,t,g,n/2];
    optional carry init_h [b,h,n,p], init_pB [b,h,r,n], init_pX [b,h,r,p].
    Returns (y [b,t,h,r,p], h [b,h,n,p], prev_B [b,h,r,n], prev_x [b,h,r,p]).
    """
    x, B, C, dt, A, lam, theta = map(_f64, (x, B, C, dt, A, lam, theta))
    init_h, init_pB, init_pX = map(_f64, (init_h, init_pB, init_pX))
    b, L, H, R, P = x.shape
    G, N = B.shape[2], B.shape[4]
    d = _Dims(b, L, H, G, P, N, R)
    y = np.zeros((b, L, H, R, P))
    hL = np.zeros((b, H, N, P))
    pB = np.zeros((b, H, R, N))
    pX = np.zeros((b, H, R, P))
    rc = (lib or _load()).oracle_scan(ctypes.byref(d), _p(x), _p(B), _p(C), _p(dt), _p(A), _p(lam),
                             _p(theta), _p(init_h), _p(init_pB), _p(init_pX),
                             _p(y), _p(hL), _p(pB), _p(pX))
    if rc != 0:
        raise ValueError("oracle_scan rejected its arguments")
    return y, hL, pB, pX


def scan_bwd(x, B, C, dt, A, lam, theta, dy, init_h=None, init_pB=None, init_pX=None,
             dh=None, dpB=None, dpX=None, lib=None):
    """Gradients of J = sum <dy, y> + <dh, h_L> + <dpB, prev_B_L> + <dpX, prev_x_L>
    with respect to every input of scan() (shapes as there).  Returns a dict
    with dx, dB, dC (B and C summed over the heads of a group), ddt, dA, dlam,
    dtheta, d_init_h, d_init_pB, d_init_pX."""
    x, B, C, dt, A, lam, theta, dy = map(_f64, (x, B, C, dt, A, lam, theta, dy))
    init_h, init_pB, init_pX, dh, dpB, dpX = map(_f64, (init_h, init_pB, init_pX, dh, dpB, dpX))
    b, L, H, R, P = x.shape
    G, N = B.shape[2], B.shape[4]
    d = _Dims(b, L, H, G, P, N, R)
    out = {"dx": np.zeros_like(x), "dB": np.zeros_like(B), "dC": np.zeros_like(C),
           "ddt": np.zeros_like(dt), "dA": np.zeros_like(A), "dlam": np.zeros_like(lam),
           "dtheta": np.zeros_like(theta), "d_init_h": np.zeros((b, H, N, P)),
           "d_init_pB": np.zeros((b, H, R, N)), "d_init_pX": np.zeros((b, H, R, P))}
    rc = (lib or _load()).oracle_scan_bwd(
        ctypes.byref(d), _p(x), _p(B), _p(C), _p(dt), _p(A), _p(lam), _p(theta),
        _p(init_h), _p(init_pB), _p(init_pX), _p(dy), _p(dh), _p(dpB), _p(dpX),
        _p(out["dx"]), _p(out["dB"]), _p(out["dC"]), _p(out["ddt"]), _p(out["dA"]), _p(out["dlam"]),
        _p(out["dtheta"]), _p(out["d_init_h"]), _p(out["d_init_pB"]), _p(out["d_init_pX"]))
    if rc != 0:
        raise ValueError("oracle_scan_bwd rejected its arguments")
    return out


DAMPING_REGIMES = ("under", "critical", "over")


def _scan_variant(fn, lead, x, B, C, dt, A, lam, theta, init_h, init_pB, init_pX):
    x, B, C, dt, A, lam, theta = map(_f64, (x, B, C, dt, A, lam, theta))
    init_h, init_pB, init_pX = map(_f64, (init_h, init_pB, init_pX))
    b, L, H, R, P = x.shape
    G, N = B.shape[2], B.shape[4]
    d = _Dims(b, L, H, G, P, N, R)
    y = np.zeros((b, L, H, R, P))
    hL = np.zeros((b, H, N, P))
    pB = np.zeros((b, H, R, N))
    pX = np.zeros((b, H, R, P))
    rc = fn(ctypes.byref(d), *lead, _p(x), _p(B), _p(C), _p(dt), _p(A), _p(lam), _p(theta),
            _p(init_h), _p(init_pB), _p(init_pX), _p(y), _p(hL), _p(pB), _p(pX))
    if rc != 0:
        raise ValueError(f"{fn.__name__} rejected its arguments")
    return y, hL, pB, pX


def scan_damped(regime, x, B, C, dt, A, lam, theta, init_h=None, init_pB=None, init_pX=None, lib=None):
    """Damping-regime variant ("Understanding Mamba-3 Through Oscillatory
    Dynamics", sections 2.2, 4.1, 4.2, appendix C.2): rotary pair i of token t
    evolves under dt (A I + theta[i] K_s), K_s = [[0, -1], [s, 0]], with
    s = +1 (under, Mamba-3), 0 (critical), -1 (over); inputs, layouts and
    returns as scan().  ``regime`` is a DAMPING_REGIMES name or 0/1/2."""
    rg = DAMPING_REGIMES.index(regime) if isinstance(regime, str) else int(regime)
    lb = lib or _load()
    return _scan_variant(lb.oracle_scan_damped, (ctypes.c_int(rg),), x, B, C, dt, A, lam, theta,
                         init_h, init_pB, init_pX)


def scan_reflect(u, x, B, C, dt, A, lam, theta, init_h=None, init_pB=None, init_pX=None, lib=None):
    """Low-rank reflection extension: Mamba-3's transition with the diagonal
    alpha_t I replaced by alpha_t (I - 2 u u^T / u^T u), u [b,t,g,n] an
    input-dependent direction (u = 0: no reflection); otherwise as scan()."""
    u = _f64(u)
    lb = lib or _load()
    return _scan_variant(lb.oracle_scan_reflect, (_p(u),), x, B, C, dt, A, lam, theta,
                         init_h, init_pB, init_pX)


PHASE_MODES = ("native", "zero", "reverse", "shuffle", "fixed", "write_only", "read_only")


def scan_phase(mode, x, B, C, dt, A, lam, theta, perm=None, freq=None, init_h=None, init_pB=None,
               init_pX=None, lib=None):
    """The scan under a phase intervention ("Understanding Mamba-3 Through
    Oscillatory Dynamics", section 5.3, appendix D.4; fixed rotations,
    section 4.3), written as its definition: the first five modes change
    theta and run scan(); write_only / read_only run the theta = 0 scan on
    per-head operands of which one side is rotated by the cumulative phase
    (rope_bc, Proposition 3) and the other is not.  Returns scan()'s tuple."""
    mode = PHASE_MODES.index(mode) if isinstance(mode, str) else int(mode)
    x, B, C, dt, A, lam, theta = map(_f64, (x, B, C, dt, A, lam, theta))
    kw = dict(init_h=init_h, init_pB=init_pB, init_pX=init_pX, lib=lib)
    if mode == 0:
        return scan(x, B, C, dt, A, lam, theta, **kw)
    if mode == 1:
        return scan(x, B, C, dt, A, lam, np.zeros_like(theta), **kw)
    if mode == 2:
        return scan(x, B, C, dt, A, lam, -theta, **kw)
    if mode == 3:
        return scan(x, B, C, dt, A, lam, theta[..., np.asarray(perm)], **kw)
    if mode == 4:
        fq = np.asarray(freq, dtype=np.float64)            # [G][N/2]
        return scan(x, B, C, dt, A, lam, np.broadcast_to(fq, theta.shape).copy(), **kw)
    H = x.shape[2]
    G = B.shape[2]
    Br, Cr, _ = rope_bc(B, C, dt, theta, nheads=H, lib=lib)
    Bh = np.repeat(B, H // G, axis=2)
    Ch = np.repeat(C, H // G, axis=2)
    th0 = np.zeros(theta.shape[:2] + (H, theta.shape[3]))
    if mode == 5:
        return scan(x, Br, Ch, dt, A, lam, th0, **kw)
    return scan(x, Bh, Cr, dt, A, lam, th0, **kw)


def step(h, prev_B, prev_x, x, B, C, dt, A, lam, theta, lib=None):
    """One decode token.  h [b,h,n,p], prev_B [b,h,r,n], prev_x [b,h,r,p];
    x [b,h,r,p]; B, C [b,g,r,n]; dt, lam [b,h]; A [h]; theta [b,g,n/2].
    Returns (y [b,h,r,p], h', prev_B', prev_x') as new arrays."""
    h, prev_B, prev_x = (np.array(a, dtype=np.float64, order="C", copy=True)
                         for a in (h, prev_B, prev_x))
    x, B, C, dt, A, lam, theta = map(_f64, (x, B, C, dt, A, lam, theta))
    b, H, R, P = x.shape
    G, N = B.shape[1], B.shape[3]
    d = _Dims(b, 1, H, G, P, N, R)
    y = np.zeros((b, H, R, P))
    rc = (lib or _load()).oracle_step(ctypes.byref(d), _p(h), _p(prev_B), _p(prev_x), _p(x), _p(B),
                             _p(C), _p(dt), _p(A), _p(lam), _p(theta), _p(y))
    if rc != 0:
        raise ValueError("oracle_step rejected its arguments")
    return y, h, prev_B, prev_x


def rope_bc(B, C, dt, theta, nheads, lib=None):
    """Cumulative phase and rotated B, C per head.
    Returns (B_rot [b,t,h,r,n], C_rot [b,t,h,r,n], phase [b,t,h,n/2])."""
    B, C, dt, theta = map(_f64, (B, C, dt, theta))
    b, L, G, R, N = B.shape
    d = _Dims(b, L, nheads, G, 1, N, R)
    Bo = np.zeros((b, L, nheads, R, N))
    Co = np.zeros((b, L, nheads, R, N))
    ph = np.zeros((b, L, nheads, N // 2))
    rc = (lib or _load()).oracle_rope_bc(ctypes.byref(d), _p(B), _p(C), _p(dt), _p(theta),
                                _p(Bo), _p(Co), _p(ph))
    if rc != 0:
        raise ValueError("oracle_rope_bc rejected its arguments")
    return Bo, Co, ph
