"""m3_scan_fwd_static: the prefill for callers that cannot allocate device
memory (for example a plugin whose host engine owns all device memory, or a
loop that must not enter the allocator after start-up).  It runs the same
kernels as m3_scan_fwd with the scratch taken from a fixed array inside the
library instead of a caller-provided workspace.

Checked through the C ABI against m3_scan_fwd on the same inputs, on two
calls in a row with different shapes that both use the scratch (several
segments per sequence), so the second call also shows that what the first
call left in the shared array does not leak into its result.  This file is
named to be collected last; it also passes when run alone.
"""
import numpy as np
import pytest
import torch

import m3_synth
from tests._util import dims_of, empty_carry, f64, rel_l2

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import selective_state_space_m3_b200 as m3


def _both(shape, seed_carry):
    inp = m3_synth.make_scan_inputs(shape)
    dev = {k: v.cuda() for k, v in inp.items()}
    c = m3_synth.make_carry(shape.batch, shape.nheads, shape.dstate, shape.headdim, shape.rank,
                            shape.dtype, seed_carry, scale=0.3)
    init = m3.Carry(c["h"].cuda(), c["prev_B"].cuda(), c["prev_x"].cuda())
    d = dims_of(shape)
    plan = m3.m3_scan_plan(d)
    assert plan["segments"] > 1                 # the scratch is really used
    need = m3.m3_scan_workspace_size(d)
    assert 256 < need <= 32 << 20
    # existing entry point with a caller-provided workspace
    y_ref = torch.empty_like(dev["x"])
    fin_ref = empty_carry(shape)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    m3.m3_scan_fwd(d, dev["x"], dev["B"], dev["C"], dev["dt"], dev["A"], dev["lam"], dev["theta"],
                   y_ref, ws, init=init, final_state=fin_ref)
    # the variant without a workspace
    y = torch.full_like(dev["x"], float("nan"))
    fin = empty_carry(shape)
    m3.m3_scan_fwd_static(d, dev["x"], dev["B"], dev["C"], dev["dt"], dev["A"], dev["lam"], dev["theta"],
                          y, init=init, final_state=fin)
    torch.cuda.synchronize()
    tol = 1e-4 if shape.dtype == "f32" else 2e-2
    assert np.all(np.isfinite(f64(y)))
    assert rel_l2(f64(y), f64(y_ref)) <= tol
    assert rel_l2(f64(fin.h), f64(fin_ref.h)) <= tol
    assert torch.equal(fin.prev_B, fin_ref.prev_B) and torch.equal(fin.prev_x, fin_ref.prev_x)


def test_static_scratch_matches_workspace_path_twice():
    # tensor-core path, rank 4, 4 sequences cut into several segments each
    _both(m3_synth.ScanShape(1, 1500, 4, 4, 64, 128, 4, 64, "bf16", 0.0, 81), 81)
    # then a different shape on the SIMT float32 path, reusing the array
    _both(m3_synth.ScanShape(1, 700, 2, 1, 16, 16, 2, 32, "f32", 0.0, 82), 82)


def test_static_scratch_rejects_sizes_beyond_its_limit():
    # 64 sequences of a 256 x 128 float32 state in 4 segments need ~64 MiB
    shape = m3_synth.ScanShape(1, 4096, 64, 64, 128, 256, 1, 64, "bf16", 0.0, 83)
    d = dims_of(shape)
    assert m3.m3_scan_workspace_size(d) > 32 << 20
    z = torch.zeros(16, device="cuda")
    with pytest.raises(m3.M3Error) as e:
        m3.m3_scan_fwd_static(d, z, z, z, z, z, z, z, z)
    assert e.value.status == m3.M3_ERR_WORKSPACE


def test_forgetting_the_cached_address_looks_it_up_again():
    # what a caller does after a device reset; here the context is unchanged,
    # so the looked-up address must simply serve the next call as before
    m3.m3_static_forget_device()
    _both(m3_synth.ScanShape(1, 900, 2, 2, 64, 128, 4, 64, "bf16", 0.0, 84), 84)
