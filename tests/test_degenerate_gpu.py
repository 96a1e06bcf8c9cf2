"""Parity of the CUDA path with the fp64 oracle on the degenerate cases of the
recurrence ("Mamba-3" summary, b-lab.team, sections 1-2), through the C ABI
(needs a B200):

* lambda = 1: the trapezoid rule collapses to Mamba-2's exponential-Euler
  step (no pending beta term);
* lambda = 0: only the pending beta term feeds the state;
* theta = 0: no rotation, the real diagonal SSM;
* dt = 0 on a run of tokens: those tokens neither decay nor feed the state
  (alpha = 1, beta = gamma = 0), so the state passes through unchanged;
* large theta (|dt theta| up to ~60 rad per token): the cumulative phase wraps
  many times per tile.

Each case runs on the tensor-core prefill (bf16, R = 4 and R = 1, several
tiles, a ragged tail, sequences cut into segments) and on the float32 SIMT
prefill, and, for the bf16 R = 4 shape, through the decode step token by
token.  Bounds as in test_parity_gpu: relative L2 and per-element max-abs
within 2e-2 (bf16) or 1e-4 (float32) of the block's scale.
"""
import numpy as np
import pytest
import torch

import m3_synth
import oracle
from tests._util import dims_of, empty_carry, f64, gpu_scan, max_abs, rel_l2, tol_for

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import selective_state_space_m3_b200 as m3


def _check(name, got, want, tol):
    r = rel_l2(got, want)
    ma = max_abs(got, want)
    scale = float(np.max(np.abs(want))) if np.size(want) else 0.0
    print(f"{name}: rel_l2={r:.3e} max_abs={ma:.3e} (max|want|={scale:.3e})")
    assert np.all(np.isfinite(np.asarray(got, np.float64))), name
    assert r <= tol, f"{name}: rel_l2 {r:.3e} > {tol:.1e}"
    assert ma <= tol * scale, f"{name}: max_abs {ma:.3e} > {tol:.1e} x {scale:.3e}"


def _degenerate(inp, case):
    out = {k: v.clone() for k, v in inp.items()}
    if case == "lambda1":
        out["lam"].fill_(1.0)
    elif case == "lambda0":
        out["lam"].fill_(0.0)
    elif case == "theta0":
        out["theta"].zero_()
    elif case == "dt0_run":
        L = out["dt"].shape[1]
        out["dt"][:, L // 3: L // 3 + 40] = 0.0
    elif case == "large_theta":
        out["theta"].mul_(8.0)                      # |theta| up to 8 pi
        out["dt"].clamp_(max=2.5)
    else:
        raise ValueError(case)
    return out


CASES = ["lambda1", "lambda0", "theta0", "dt0_run", "large_theta"]
SHAPES = [
    (m3_synth.ScanShape(2, 3 * 32 + 7, 4, 4, 64, 128, 4, 64, "bf16", 0.0, 91), "tc_r4"),
    (m3_synth.ScanShape(1, 2 * 128 + 9, 3, 3, 64, 128, 1, 64, "bf16", 0.0, 92), "tc_r1"),
    (m3_synth.ScanShape(2, 150, 2, 1, 16, 16, 2, 32, "f32", 0.0, 93), "simt_f32"),
]


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("shape,name", SHAPES, ids=[n for _, n in SHAPES])
def test_degenerate_scan_matches_oracle(shape, name, case):
    inp = _degenerate(m3_synth.make_scan_inputs(shape), case)
    want_tc = shape.dtype == "bf16"
    assert (m3.m3_scan_plan(dims_of(shape))["path"] == "tcgen05") == want_tc
    y, fin = gpu_scan(shape, inp)
    yo, ho, bo, xo = oracle.scan(**{k: f64(v) for k, v in inp.items()})
    tol = tol_for(shape.dtype)
    _check(f"{name}/{case} y", f64(y), yo, tol)
    _check(f"{name}/{case} h", f64(fin.h), ho, tol)
    np.testing.assert_array_equal(f64(fin.prev_B), bo)
    np.testing.assert_array_equal(f64(fin.prev_x), xo)


@pytest.mark.parametrize("case", CASES)
def test_degenerate_segments_match_oracle(case, monkeypatch):
    """The same cases with every sequence cut into 3 segments (summary pass,
    combine, main pass)."""
    monkeypatch.setenv("M3_SCAN_NSEG", "3")
    shape = m3_synth.ScanShape(1, 5 * 32 + 3, 2, 2, 64, 128, 4, 64, "bf16", 0.0, 94)
    assert m3.m3_scan_plan(dims_of(shape))["segments"] == 3
    inp = _degenerate(m3_synth.make_scan_inputs(shape), case)
    y, fin = gpu_scan(shape, inp)
    yo, ho, _, _ = oracle.scan(**{k: f64(v) for k, v in inp.items()})
    _check(f"segments/{case} y", f64(y), yo, 2e-2)
    _check(f"segments/{case} h", f64(fin.h), ho, 2e-2)


@pytest.mark.parametrize("case", CASES)
def test_degenerate_decode_matches_oracle(case):
    """The decode step token by token on the same cases (bf16, R = 4), from a
    zero carry, every y compared."""
    shape = m3_synth.ScanShape(2, 24, 4, 4, 64, 128, 4, 64, "bf16", 0.0, 95)
    inp = _degenerate(m3_synth.make_scan_inputs(shape), case)
    b, L, H, R, P = inp["x"].shape
    G, N = inp["B"].shape[2], inp["B"].shape[4]
    carry = empty_carry(shape)
    state = m3.Carry(carry.h.zero_(), carry.prev_B.zero_(), carry.prev_x.zero_())
    d = m3.Dims(b, 1, H, G, P, N, R, 1, m3.M3_BF16)
    A = inp["A"].cuda()
    yo, ho, _, _ = oracle.scan(**{k: f64(v) for k, v in inp.items()})
    for t in range(L):
        tok = {k: inp[k][:, t].contiguous().cuda() for k in ("x", "B", "C", "dt", "lam", "theta")}
        y = torch.empty_like(tok["x"])
        m3.m3_step(d, state, tok["x"], tok["B"], tok["C"], tok["dt"], A, tok["lam"], tok["theta"], y)
        torch.cuda.synchronize()
        _check(f"decode/{case} t{t} y", f64(y), yo[:, t], 2e-2)
    _check(f"decode/{case} h", f64(state.h), ho, 2e-2)
