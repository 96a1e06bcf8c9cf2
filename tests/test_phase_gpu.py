"""Parity of the phase interventions (m3_scan_fwd_phase) with the oracle's
definition of each (oracle.scan_phase, pinned on the CPU) -- needs a B200.

Each mode runs on the tensor-core path (bf16, N=128, P=64, R=4) and on the
float32 SIMT path, with B / C shared by two heads (so the one-sided modes
exercise the per-head copy), within the forward's tolerances."""
import numpy as np
import pytest
import torch

import m3_synth
import oracle
from tests._util import dims_of, f64, max_abs, rel_l2, tol_for

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import selective_state_space_m3_b200 as m3

MODES = ["native", "zero", "reverse", "shuffle", "fixed", "write_only", "read_only"]
SHAPES = [
    (m3_synth.ScanShape(2, 150, 4, 2, 64, 128, 4, 64, "bf16", 0.0, 101), "tc_r4"),
    (m3_synth.ScanShape(1, 90, 4, 2, 16, 16, 2, 32, "f32", 0.0, 102), "simt_f32"),
]


@pytest.mark.parametrize("shape,sname", SHAPES, ids=[n for _, n in SHAPES])
@pytest.mark.parametrize("mode", MODES)
def test_phase_mode_matches_oracle(shape, sname, mode):
    inp = m3_synth.make_scan_inputs(shape)
    dev = {k: v.cuda() for k, v in inp.items()}
    d = dims_of(shape)
    NH, G = shape.dstate // 2, shape.ngroups
    rng = np.random.default_rng(shape.seed)
    perm = list(rng.permutation(NH)) if mode == "shuffle" else None
    freq = rng.uniform(-np.pi, np.pi, (G, NH)).astype(np.float32) if mode == "fixed" else None
    mi = MODES.index(mode)
    y = torch.empty_like(dev["x"])
    f = dict(device="cuda")
    fin = m3.Carry(torch.empty(shape.batch, shape.nheads, shape.dstate, shape.headdim, **f),
                   torch.empty(shape.batch, shape.nheads, shape.rank, shape.dstate, dtype=dev["B"].dtype, **f),
                   torch.empty(shape.batch, shape.nheads, shape.rank, shape.headdim, dtype=dev["x"].dtype, **f))
    ws = torch.zeros(m3.m3_scan_phase_workspace_size(d, mi), dtype=torch.uint8, device="cuda")
    m3.m3_scan_fwd_phase(d, mi, dev["x"], dev["B"], dev["C"], dev["dt"], dev["A"], dev["lam"], dev["theta"], y, ws,
                         perm=perm, freq=freq, final_state=fin)
    assert m3.m3_device_status(ws) == m3.M3_OK
    yo, ho, _, _ = oracle.scan_phase(mode, **{k: f64(v) for k, v in inp.items()}, perm=perm,
                                     freq=None if freq is None else freq.astype(np.float64))
    tol = tol_for(shape.dtype)
    for name, got, want in (("y", f64(y), yo), ("h", f64(fin.h), ho)):
        r = rel_l2(got, want)
        print(f"{sname} {mode} {name}: rel_l2={r:.3e} max_abs={max_abs(got, want):.3e}")
        assert r <= tol, (sname, mode, name, r)
