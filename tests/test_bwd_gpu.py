"""Parity of the backward pass (m3_scan_bwd) with the oracle's reverse mode
(needs a B200).

The oracle's gradient is itself pinned by finite differences of the forward
oracle (tests/test_oracle_pins.py).  Every gradient is compared element by
element, relative L2 per tensor.  The GPU computes in float32 from the same
stored inputs; the bound 1e-4 is the forward's float32 bound (the backward
is a float32 recurrence of the same length), except dA, a sum over every
token of the sequence(s) with mixed signs, checked at 1e-3.
"""
import numpy as np
import pytest
import torch

import m3_synth
import oracle
from tests._util import dims_of, f64, max_abs, rel_l2

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import selective_state_space_m3_b200 as m3


def _check(name, got, want, tol):
    r = rel_l2(got, want)
    print(f"{name}: rel_l2={r:.3e} max_abs={max_abs(got, want):.3e}")
    assert np.all(np.isfinite(np.asarray(got, np.float64))), name
    assert r <= tol, f"{name}: rel_l2 {r:.3e} > {tol:.1e}"


def _gpu_bwd(shape, inp, dy, init=None, d_final=None, want_init=False):
    dev = {k: v.cuda() for k, v in inp.items()}
    d = dims_of(shape)
    b, L, H, G, R, P, N = shape.batch, shape.seqlen, shape.nheads, shape.ngroups, shape.rank, shape.headdim, shape.dstate
    f = dict(device="cuda", dtype=torch.float32)
    g = {"dx": torch.empty(b, L, H, R, P, **f), "dB": torch.empty(b, L, G, R, N, **f),
         "dC": torch.empty(b, L, G, R, N, **f), "ddt": torch.empty(b, L, H, **f), "dA": torch.empty(H, **f),
         "dlam": torch.empty(b, L, H, **f), "dtheta": torch.empty(b, L, G, N // 2, **f)}
    ws = torch.zeros(m3.m3_scan_bwd_workspace_size(d), dtype=torch.uint8, device="cuda")
    di = None
    if want_init:
        di = m3.Carry(torch.empty(b, H, N, P, **f), torch.empty(b, H, R, N, **f), torch.empty(b, H, R, P, **f))
    m3.m3_scan_bwd(d, dev["x"], dev["B"], dev["C"], dev["dt"], dev["A"], dev["lam"], dev["theta"],
                   dy.cuda(), g, ws, init=init, d_final=d_final, d_init=di)
    torch.cuda.synchronize()
    return g, di


def _compare(tag, g, ref, tol=1e-4, skip=(), di=None):
    for k in ("dx", "dB", "dC", "ddt", "dlam", "dtheta", "dA"):
        if k in skip:
            continue
        _check(f"{tag} {k}", f64(g[k]), ref[k], 1e-3 if k == "dA" else tol)
    if di is not None:
        _check(f"{tag} d_init_h", f64(di.h), ref["d_init_h"], tol)
        _check(f"{tag} d_init_pB", f64(di.prev_B), ref["d_init_pB"], tol)
        _check(f"{tag} d_init_pX", f64(di.prev_x), ref["d_init_pX"], tol)


CASES = [
    # several 16-token checkpoint blocks and a ragged tail; shared group
    (m3_synth.ScanShape(2, 100, 2, 1, 16, 16, 2, 32, "f32", 0.0, 91), "f32_mimo_shared"),
    (m3_synth.ScanShape(1, 70, 3, 3, 64, 128, 4, 64, "bf16", 0.0, 92), "bf16_r4_layer_dims"),
    (m3_synth.ScanShape(2, 45, 4, 2, 32, 32, 1, 64, "bf16", -1.0, 93), "bf16_siso"),
    (m3_synth.ScanShape(1, 33, 2, 2, 16, 64, 3, 16, "f32", 0.0, 94), "f32_r3"),
]


@pytest.mark.parametrize("shape,name", CASES, ids=[n for _, n in CASES])
@pytest.mark.parametrize("carry", [False, True])
def test_scan_bwd_matches_oracle(shape, name, carry):
    inp = m3_synth.make_scan_inputs(shape)
    b, L, H, R, P, N = shape.batch, shape.seqlen, shape.nheads, shape.rank, shape.headdim, shape.dstate
    rng = np.random.default_rng(shape.seed + 7)
    io = torch.float32 if shape.dtype == "f32" else torch.bfloat16
    dy = torch.from_numpy(rng.standard_normal((b, L, H, R, P)).astype(np.float32)).to(io)
    init = d_final = None
    okw = {}
    if carry:
        c = m3_synth.make_carry(b, H, N, P, R, shape.dtype, shape.seed + 8, scale=0.5)
        init = m3.Carry(c["h"].cuda(), c["prev_B"].cuda(), c["prev_x"].cuda())
        fin = {k: torch.from_numpy(rng.standard_normal(s).astype(np.float32))
               for k, s in (("h", (b, H, N, P)), ("pB", (b, H, R, N)), ("pX", (b, H, R, P)))}
        d_final = m3.Carry(fin["h"].cuda(), fin["pB"].cuda(), fin["pX"].cuda())
        okw = dict(init_h=f64(c["h"]), init_pB=f64(c["prev_B"]), init_pX=f64(c["prev_x"]),
                   dh=f64(fin["h"]), dpB=f64(fin["pB"]), dpX=f64(fin["pX"]))
    g, di = _gpu_bwd(shape, inp, dy, init=init, d_final=d_final, want_init=carry)
    ref = oracle.scan_bwd(**{k: f64(v) for k, v in inp.items()}, dy=f64(dy), **okw)
    _compare(f"{name} carry={carry}", g, ref, di=di)


def test_scan_bwd_layer_shape_sampled():
    """The R=4 layer's full shape (8 x 4096 tokens, 32 heads, one group per
    head), sampled (b, h) against the oracle run on that slice alone.  dA
    sums over the batch, so it is compared through its own slice sum."""
    shape = m3_synth.MIMO_R4_LAYER
    inp = m3_synth.make_scan_inputs(shape)
    b, L, H, R, P = shape.batch, shape.seqlen, shape.nheads, shape.rank, shape.headdim
    rng = np.random.default_rng(2024)
    dy = torch.from_numpy(rng.standard_normal((b, L, H, R, P)).astype(np.float32)).to(torch.bfloat16)
    g, _ = _gpu_bwd(shape, inp, dy)
    for (bb, hh) in [(0, 0), (6, 21)]:
        sl = lambda v: f64(v[bb:bb + 1, :, hh:hh + 1])
        one = {k: sl(v) for k, v in inp.items() if k != "A"}
        one["A"] = f64(inp["A"][hh:hh + 1])
        ref = oracle.scan_bwd(**one, dy=sl(dy))
        got = {k: g[k][bb:bb + 1, :, hh:hh + 1] for k in ("dx", "dB", "dC", "ddt", "dlam", "dtheta")}
        _compare(f"layer b{bb} h{hh}", got, ref, skip=("dA",))


def test_scan_bwd_empty_sequence():
    """L = 0: the carry-in gradient is the carry-out gradient, dA is zero."""
    shape = m3_synth.ScanShape(2, 0, 2, 2, 16, 16, 1, 32, "f32", 0.0, 95)
    d = dims_of(shape)
    f = dict(device="cuda", dtype=torch.float32)
    z = torch.empty(0, **f)
    dh = torch.randn(2, 2, 16, 16, **f)
    g = {"dx": z, "dB": z, "dC": z, "ddt": z, "dA": torch.full((2,), 7.0, **f), "dlam": z, "dtheta": z}
    di = m3.Carry(torch.empty(2, 2, 16, 16, **f), torch.empty(2, 2, 1, 16, **f), torch.empty(2, 2, 1, 16, **f))
    ws = torch.zeros(max(256, m3.m3_scan_bwd_workspace_size(d)), dtype=torch.uint8, device="cuda")
    m3.m3_scan_bwd(d, z, z, z, z, torch.zeros(2, **f), z, z, z, g, ws,
                   d_final=m3.Carry(dh, None, None), d_init=di)
    torch.cuda.synchronize()
    assert torch.equal(di.h, dh)
    assert torch.count_nonzero(g["dA"]) == 0
    assert torch.count_nonzero(di.prev_B) == 0 and torch.count_nonzero(di.prev_x) == 0


def test_scan_bwd_layer_homogeneity_full_size():
    """At the R=4 layer's full size, identities that need no oracle: with no
    carry-in, J = sum <dy, y> is linear in x, in B and in C, so the backward's
    <dx, x>, <dB, B> and <dC, C> are the same number, J.  Against J computed
    from the forward's y the bound is the forward's own: |J_fwd - J| is at most
    the y error (relative L2 2e-2) times ||y|| ||dy|| (Cauchy-Schwarz); the sum
    cancels heavily, so J_fwd alone is a loose check."""
    shape = m3_synth.MIMO_R4_LAYER
    inp = m3_synth.make_scan_inputs(shape)
    b, L, H, R, P = shape.batch, shape.seqlen, shape.nheads, shape.rank, shape.headdim
    rng = np.random.default_rng(77)
    dy = torch.from_numpy(rng.standard_normal((b, L, H, R, P)).astype(np.float32)).to(torch.bfloat16)
    dev = {k: v.cuda() for k, v in inp.items()}
    d = dims_of(shape)
    y = torch.empty_like(dev["x"])
    ws = torch.zeros(m3.m3_scan_workspace_size(d), dtype=torch.uint8, device="cuda")
    m3.m3_scan_fwd(d, dev["x"], dev["B"], dev["C"], dev["dt"], dev["A"], dev["lam"], dev["theta"], y, ws)
    dyd = dy.cuda().double()
    J_fwd = float((y.double() * dyd).sum())
    bound = 2e-2 * float(y.double().norm()) * float(dyd.norm())
    g, _ = _gpu_bwd(shape, inp, dy)
    v = {k: float((g["d" + k].double() * dev[k].double()).sum()) for k in ("x", "B", "C")}
    print(f"homogeneity: <dx,x>={v['x']:.6e} <dB,B>={v['B']:.6e} <dC,C>={v['C']:.6e} J_fwd={J_fwd:.6e} "
          f"bound={bound:.3e}")
    assert abs(v["B"] - v["x"]) <= 1e-3 * abs(v["x"]), v
    assert abs(v["C"] - v["x"]) <= 1e-3 * abs(v["x"]), v
    assert abs(v["x"] - J_fwd) <= bound, (v, J_fwd, bound)
