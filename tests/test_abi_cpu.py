"""CPU checks of the C ABI (no GPU, no kernel launches).

* libm3.so loads and exports every function include/m3.h declares.
* Host-side validation returns its status before anything is enqueued: the
  pointers passed here are never dereferenced (bad sizes, misalignment and
  small workspaces are all rejected first).
* The workspace-size query is host-only.
"""
import ctypes
import os
import re
import subprocess

import pytest

import selective_state_space_m3_b200 as m3

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "m3.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(m3_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_abi():
    assert set(declared_functions()) == set(m3.ABI_SYMBOLS)


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(m3.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", m3.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(m3_[a-z0-9_]+)$", out, flags=re.M))
    assert set(declared_functions()) <= exported


def test_status_strings():
    for s in range(6):
        assert m3.m3_status_string(s)
    assert m3.m3_status_string(99) == "unknown status"


LIB = m3.raw_lib()
GOOD = 0x10000          # 16-byte aligned fake device addresses (never touched)
BAD = 0x10008


def dims(**kw):
    base = dict(batch=2, seqlen=64, nheads=4, ngroups=2, headdim=16, dstate=16, rank=2, chunk=16,
                io_dtype=m3.M3_BF16)
    base.update(kw)
    return m3.Dims(**base)


def scan_status(d, ptr=GOOD, ws=GOOD, ws_bytes=1 << 30, y=GOOD, init=None, fin=None):
    cd = d.c()
    return LIB.m3_scan_fwd(ctypes.byref(cd), ptr, ptr, ptr, ptr, ptr, ptr, ptr,
                           ctypes.byref(init) if init is not None else None, y,
                           ctypes.byref(fin) if fin is not None else None, ws, ws_bytes, None)


def test_workspace_size_is_host_only_and_positive():
    n = m3.m3_scan_workspace_size(dims())
    assert n >= 256 and n % 256 == 0
    n2 = m3.m3_scan_workspace_size(dims(batch=1, nheads=1, ngroups=1, seqlen=4096))
    assert n2 > 256          # a long single sequence is split into segments


@pytest.mark.parametrize("bad", [
    dict(dstate=15), dict(nheads=3, ngroups=2), dict(batch=-1), dict(seqlen=-1), dict(rank=0),
    dict(headdim=0), dict(chunk=0), dict(io_dtype=7), dict(ngroups=0),
])
def test_scan_rejects_bad_dims(bad):
    assert scan_status(dims(**bad)) == m3.M3_ERR_INVALID_ARG


def test_scan_rejects_null_and_misaligned_pointers():
    assert scan_status(dims(), ptr=0) == m3.M3_ERR_INVALID_ARG
    assert scan_status(dims(), ptr=BAD) == m3.M3_ERR_INVALID_ARG
    assert scan_status(dims(), y=BAD) == m3.M3_ERR_INVALID_ARG
    bad_carry = m3._Carry(BAD, None, None)
    assert scan_status(dims(), init=bad_carry) == m3.M3_ERR_INVALID_ARG
    assert scan_status(dims(), fin=bad_carry) == m3.M3_ERR_INVALID_ARG


def test_scan_rejects_small_or_missing_workspace():
    need = m3.m3_scan_workspace_size(dims())
    assert scan_status(dims(), ws_bytes=need - 1) == m3.M3_ERR_WORKSPACE
    assert scan_status(dims(), ws=0) == m3.M3_ERR_WORKSPACE
    assert scan_status(dims(), ws=BAD) == m3.M3_ERR_WORKSPACE


def test_unsupported_sizes():
    n = ctypes.c_size_t(0)
    cd = dims(dstate=2048).c()
    assert LIB.m3_scan_workspace_size(ctypes.byref(cd), ctypes.byref(n)) == m3.M3_ERR_UNSUPPORTED


def test_step_rejects_bad_arguments():
    d = dims().c()
    good = m3._Carry(GOOD, GOOD, GOOD)
    args = [GOOD] * 8
    assert LIB.m3_step(ctypes.byref(d), None, *args, None) == m3.M3_ERR_INVALID_ARG
    assert LIB.m3_step(ctypes.byref(d), ctypes.byref(m3._Carry(GOOD, None, GOOD)), *args,
                       None) == m3.M3_ERR_INVALID_ARG
    assert LIB.m3_step(ctypes.byref(d), ctypes.byref(m3._Carry(BAD, GOOD, GOOD)), *args,
                       None) == m3.M3_ERR_INVALID_ARG
    d_odd = dims(dstate=9).c()
    assert LIB.m3_step(ctypes.byref(d_odd), ctypes.byref(good), *args, None) == m3.M3_ERR_INVALID_ARG
    d_bad_p = dims(headdim=12).c()      # P/4 = 3: not a power of two
    assert LIB.m3_step(ctypes.byref(d_bad_p), ctypes.byref(good), *args, None) == m3.M3_ERR_UNSUPPORTED


def test_rope_rejects_bad_arguments():
    d = dims().c()
    assert LIB.m3_rope_bc(ctypes.byref(d), GOOD, 0, GOOD, GOOD, GOOD, GOOD, None,
                          None) == m3.M3_ERR_INVALID_ARG
    assert LIB.m3_rope_bc(ctypes.byref(d), GOOD, GOOD, GOOD, GOOD, GOOD, GOOD, BAD,
                          None) == m3.M3_ERR_INVALID_ARG


def test_null_dims():
    n = ctypes.c_size_t(0)
    assert LIB.m3_scan_workspace_size(None, ctypes.byref(n)) == m3.M3_ERR_INVALID_ARG
    assert LIB.m3_device_status(None, None) == m3.M3_ERR_INVALID_ARG


def test_plan_picks_the_tensor_core_path_for_bf16_layers():
    import m3_synth
    from tests._util import dims_of
    p0 = m3.m3_scan_plan(dims_of(m3_synth.SISO_TINY))
    assert p0["path"] == "simt" and p0["chunk_used"] == 32
    for s in (m3_synth.SISO_LAYER, m3_synth.MIMO_R4_LAYER, m3_synth.LONG_SISO):
        p = m3.m3_scan_plan(dims_of(s))
        assert p["path"] == "tcgen05"
        assert p["chunk_used"] == 128 // s.rank
        assert p["launches"] == (1 if p["segments"] == 1 else 3)
    # the 1.5B MIMO layer has 256 sequences: one segment each, one launch
    assert m3.m3_scan_plan(dims_of(m3_synth.MIMO_R4_LAYER))["segments"] == 1


def _bwd_status(d, ptr=GOOD, ws=GOOD, ws_bytes=1 << 34, dy=GOOD):
    cd = d.c()
    return LIB.m3_scan_bwd(ctypes.byref(cd), ptr, ptr, ptr, ptr, ptr, ptr, ptr, None, dy, None,
                           ptr, ptr, ptr, ptr, ptr, ptr, ptr, None, ws, ws_bytes, None)


def test_bwd_rejects_before_launching():
    d = dims(headdim=16, dstate=16, rank=2)
    n = m3.m3_scan_bwd_workspace_size(d)
    assert n > 256
    assert _bwd_status(dims(headdim=48)) == m3.M3_ERR_UNSUPPORTED       # P not 16/32/64
    assert _bwd_status(dims(rank=5, headdim=16, dstate=16)) == m3.M3_ERR_UNSUPPORTED
    assert _bwd_status(dims(nheads=3, ngroups=2)) == m3.M3_ERR_INVALID_ARG
    assert _bwd_status(d, ptr=BAD) == m3.M3_ERR_INVALID_ARG
    assert _bwd_status(d, dy=0) == m3.M3_ERR_INVALID_ARG
    assert _bwd_status(d, ws_bytes=n - 1) == m3.M3_ERR_WORKSPACE
    assert _bwd_status(d, ws=0) == m3.M3_ERR_WORKSPACE


def _phase_status(d, mode, perm=None, freq=None, ws_bytes=1 << 34):
    cd = d.c()
    pc = (ctypes.c_int * len(perm))(*perm) if perm is not None else None
    fc = (ctypes.c_float * len(freq))(*freq) if freq is not None else None
    return LIB.m3_scan_fwd_phase(ctypes.byref(cd), mode, ctypes.cast(pc, ctypes.c_void_p) if pc else None,
                                 ctypes.cast(fc, ctypes.c_void_p) if fc else None,
                                 GOOD, GOOD, GOOD, GOOD, GOOD, GOOD, GOOD, None, GOOD, None, GOOD, ws_bytes, None)


def test_phase_rejects_before_launching():
    d = dims(dstate=16)                        # 8 rotary pairs
    assert _phase_status(d, 7) == m3.M3_ERR_INVALID_ARG
    assert _phase_status(d, m3.M3_PHASE_SHUFFLE) == m3.M3_ERR_INVALID_ARG                 # no perm
    assert _phase_status(d, m3.M3_PHASE_SHUFFLE, perm=[0, 1, 2, 3, 4, 5, 6, 6]) == m3.M3_ERR_INVALID_ARG
    assert _phase_status(d, m3.M3_PHASE_SHUFFLE, perm=[0, 1, 2, 3, 4, 5, 6, 8]) == m3.M3_ERR_INVALID_ARG
    assert _phase_status(d, m3.M3_PHASE_FIXED) == m3.M3_ERR_INVALID_ARG                   # no freq
    n = m3.m3_scan_phase_workspace_size(d, m3.M3_PHASE_READ_ONLY)
    assert n > m3.m3_scan_workspace_size(d)
    assert _phase_status(d, m3.M3_PHASE_READ_ONLY, ws_bytes=n - 1) == m3.M3_ERR_WORKSPACE


def test_empty_problems_return_ok_before_touching_anything():
    """batch = 0 (and L = 0 for the per-sequence calls) is a valid call with
    nothing to do: it returns M3_OK with null data pointers and enqueues no
    kernel; the plan reports zero launches."""
    e = dims(batch=0)
    assert scan_status(e, ptr=0, y=0) == m3.M3_OK
    assert m3.m3_scan_plan(e)["launches"] == 0
    assert m3.m3_scan_plan(dims(seqlen=0))["launches"] == 0
    d = e.c()
    assert LIB.m3_step(ctypes.byref(d), ctypes.byref(m3._Carry(None, None, None)), *([None] * 8),
                       None) == m3.M3_OK
    for empty in (e, dims(seqlen=0)):
        d = empty.c()
        assert LIB.m3_rope_bc(ctypes.byref(d), None, None, None, None, None, None, None,
                              None) == m3.M3_OK


def _variant_status(d, regime=0, u=GOOD, ptr=GOOD, reflect=False):
    cd = d.c()
    if reflect:
        return LIB.m3_scan_fwd_reflect(ctypes.byref(cd), u, ptr, ptr, ptr, ptr, ptr, ptr, ptr, None, ptr, None,
                                       None)
    return LIB.m3_scan_fwd_damped(ctypes.byref(cd), regime, ptr, ptr, ptr, ptr, ptr, ptr, ptr, None, ptr, None,
                                  None)


def test_variants_reject_before_launching():
    """Damped and reflection scans: a bad regime, unsupported shapes (rank 3,
    dstate not a multiple of 8 or above 256, headdim not a multiple of 16),
    null or misaligned pointers all return before any launch; an empty call
    is OK with null pointers."""
    d = dims(headdim=16, dstate=16, rank=2)
    assert _variant_status(d, regime=3) == m3.M3_ERR_INVALID_ARG
    assert _variant_status(d, regime=-1) == m3.M3_ERR_INVALID_ARG
    assert _variant_status(dims(rank=3)) == m3.M3_ERR_UNSUPPORTED
    assert _variant_status(dims(dstate=12)) == m3.M3_ERR_UNSUPPORTED
    assert _variant_status(dims(dstate=512)) == m3.M3_ERR_UNSUPPORTED
    assert _variant_status(dims(headdim=24)) == m3.M3_ERR_UNSUPPORTED
    assert _variant_status(d, ptr=BAD) == m3.M3_ERR_INVALID_ARG
    assert _variant_status(d, reflect=True, u=BAD) == m3.M3_ERR_INVALID_ARG
    assert _variant_status(d, reflect=True, u=None) == m3.M3_ERR_INVALID_ARG
    for e in (dims(batch=0), dims(seqlen=0)):
        assert _variant_status(e, ptr=None) == m3.M3_OK
        assert _variant_status(e, ptr=None, reflect=True, u=None) == m3.M3_OK


def test_static_forget_device_needs_a_current_device():
    """m3_static_forget_device only clears a cached address: with a device it
    returns M3_OK (twice in a row too), without one M3_ERR_CUDA; it never
    launches anything."""
    st = LIB.m3_static_forget_device()
    assert st in (m3.M3_OK, m3.M3_ERR_CUDA)
    assert LIB.m3_static_forget_device() == st


def test_release_build_has_no_index_checks():
    """libm3.so: the bounds report says 'disabled' without touching a device,
    and the checks' self-test validates its arguments, then refuses
    (M3_ERR_UNSUPPORTED) without launching."""
    if m3.DEBUG_BOUNDS:
        pytest.skip("the package was imported with the index-checked library")
    assert m3.m3_debug_bounds_report() == {"enabled": 0, "failures": 0, "site": 0, "index": 0, "limit": 0}
    assert LIB.m3_debug_bounds_report(None, 0) == m3.M3_ERR_INVALID_ARG
    st = LIB.m3_selftest_bounds_check
    assert st(GOOD, 64, 40, 32, None) == m3.M3_ERR_UNSUPPORTED
    assert st(None, 64, 40, 32, None) == m3.M3_ERR_INVALID_ARG      # no buffer
    assert st(GOOD, 64, 64, 32, None) == m3.M3_ERR_INVALID_ARG      # index past the buffer
    assert st(GOOD, 64, -1, 32, None) == m3.M3_ERR_INVALID_ARG
    assert st(GOOD, 64, 3, 65, None) == m3.M3_ERR_INVALID_ARG       # limit past the buffer
    assert st(GOOD, 0, 0, 0, None) == m3.M3_ERR_INVALID_ARG


def test_debug_library_is_built_and_exports_every_symbol():
    """libm3_debug.so (the index-checked build) sits beside libm3.so, exports
    the same ABI, and is what the package loads under M3_DEBUG_BOUNDS=1; its
    report needs a device (M3_ERR_CUDA without one)."""
    dbg = os.path.join(os.path.dirname(m3.LIB_PATH), "libm3_debug.so")
    assert os.path.exists(dbg)
    out = subprocess.run(["nm", "-D", "--defined-only", dbg], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(m3_[a-z0-9_]+)$", out, flags=re.M))
    assert set(declared_functions()) <= exported
    code = (
        "import torch, selective_state_space_m3_b200 as m3\n"
        "assert m3.DEBUG_BOUNDS and m3.LIB_PATH.endswith('libm3_debug.so'), m3.LIB_PATH\n"
        "lib = m3.raw_lib()\n"
        "assert lib.m3_selftest_bounds_check(0x10000, 64, 64, 32, None) == m3.M3_ERR_INVALID_ARG\n"
        "if not torch.cuda.is_available():\n"
        "    try:\n"
        "        m3.m3_debug_bounds_report()\n"
        "        raise SystemExit('report without a device')\n"
        "    except m3.M3Error as e:\n"
        "        assert e.status == m3.M3_ERR_CUDA, e\n"
        "print('debug ok')\n")
    env = dict(os.environ, M3_DEBUG_BOUNDS="1", PYTHONPATH=ROOT)
    r = subprocess.run([os.sys.executable, "-c", code], capture_output=True, text=True, env=env, cwd=ROOT, timeout=300)
    assert r.returncode == 0 and "debug ok" in r.stdout, r.stdout + r.stderr
