"""The product path has no CPU fallback (no GPU needed).

* Without libm3.so the package does not import: it raises ImportError (and
  likewise without libm3_debug.so when M3_DEBUG_BOUNDS=1 asks for it).
* Every entry point refuses host tensors before anything reaches the
  library, so no computation can silently run on the host.
* Neither the package's Python nor its CUDA sources reach the oracle, and
  importing the package loads no oracle module.
"""
import glob
import os
import shutil
import subprocess
import sys

import pytest
import torch

import selective_state_space_m3_b200 as m3

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "selective_state_space_m3_b200")


def test_missing_library_fails_the_import(tmp_path):
    dst = tmp_path / "selective_state_space_m3_b200"
    dst.mkdir()
    for f in glob.glob(os.path.join(PKG, "*.py")):
        shutil.copy(f, dst)
    assert not (dst / "libm3.so").exists()
    r = subprocess.run([sys.executable, "-c", "import selective_state_space_m3_b200"], cwd=tmp_path,
                       env={**os.environ, "PYTHONPATH": str(tmp_path)}, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode != 0
    assert "ImportError" in r.stderr and "libm3.so is missing" in r.stderr


def test_missing_debug_library_fails_the_import_under_the_debug_switch(tmp_path):
    """M3_DEBUG_BOUNDS=1 asks for the index-checked library: with only the
    release library present the import fails too (no quiet fallback to it)."""
    dst = tmp_path / "selective_state_space_m3_b200"
    dst.mkdir()
    for f in glob.glob(os.path.join(PKG, "*.py")):
        shutil.copy(f, dst)
    shutil.copy(os.path.join(PKG, "libm3.so"), dst)
    assert not (dst / "libm3_debug.so").exists()
    r = subprocess.run([sys.executable, "-c", "import selective_state_space_m3_b200"], cwd=tmp_path,
                       env={**os.environ, "PYTHONPATH": str(tmp_path), "M3_DEBUG_BOUNDS": "1"},
                       capture_output=True, text=True, timeout=300)
    assert r.returncode != 0
    assert "ImportError" in r.stderr and "libm3_debug.so is missing" in r.stderr


def _host_case():
    b, L, H, G, R, P, N = 1, 4, 2, 2, 1, 16, 16
    dims = m3.Dims(b, L, H, G, P, N, R, 16, m3.M3_F32)
    f = lambda *s: torch.zeros(*s, dtype=torch.float32)
    t = dict(x=f(b, L, H, R, P), B=f(b, L, G, R, N), C=f(b, L, G, R, N), dt=f(b, L, H), A=f(H),
             lam=f(b, L, H), theta=f(b, L, G, N // 2), y=f(b, L, H, R, P))
    return dims, t, f


def test_every_entry_point_refuses_host_tensors():
    dims, t, f = _host_case()
    ws = torch.zeros(1 << 16, dtype=torch.uint8)
    carry = m3.Carry(f(1, 2, 16, 16), f(1, 2, 1, 16), f(1, 2, 1, 16))
    grads = {k: f(1) for k in ("dx", "dB", "dC", "ddt", "dA", "dlam", "dtheta")}
    args = (t["x"], t["B"], t["C"], t["dt"], t["A"], t["lam"], t["theta"])
    calls = [
        lambda: m3.m3_scan_fwd(dims, *args, t["y"], ws),
        lambda: m3.m3_scan_fwd_static(dims, *args, t["y"]),
        lambda: m3.m3_step(dims, carry, *args, t["y"]),
        lambda: m3.m3_rope_bc(dims, t["B"], t["C"], t["dt"], t["theta"], f(1), f(1)),
        lambda: m3.m3_scan_bwd(dims, *args, t["y"], grads, ws),
        lambda: m3.m3_scan_fwd_phase(dims, m3.M3_PHASE_ZERO, *args, t["y"], ws),
    ]
    for call in calls:
        with pytest.raises(ValueError, match="device tensors"):
            call()


def test_product_sources_never_reach_the_oracle():
    srcs = glob.glob(os.path.join(PKG, "*.py")) + glob.glob(os.path.join(PKG, "csrc", "*"))
    srcs += glob.glob(os.path.join(ROOT, "include", "*.h"))
    assert srcs
    for s in srcs:
        text = open(s, errors="replace").read()
        for needle in ("import oracle", "from oracle", "m3_oracle", "oracle/", "liboracle"):
            assert needle not in text, f"{os.path.relpath(s, ROOT)} names {needle!r}"


def test_importing_the_package_loads_no_oracle_module():
    code = ("import sys, selective_state_space_m3_b200\n"
            "bad = [k for k in sys.modules if k == 'oracle' or k.startswith('oracle.')]\n"
            "so = [l for l in open('/proc/self/maps') if 'oracle' in l]\n"
            "assert not bad and not so, (bad, so)\n")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
