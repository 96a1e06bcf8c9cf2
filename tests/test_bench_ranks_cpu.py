"""The multi-rank plumbing of bench.py, run as two gloo ranks on the CPU.

With N GPUs the bench runs N independent replicas (one seeded problem per
rank, no collective on the data path); the only collectives are the timing
barrier and the max over ranks.  These tests run that plumbing with the gloo
backend: the ranks agree on the slowest time, each rank draws a different
problem of the same shape, and the reported value is the whole job's tokens
over the slowest rank's time.
"""
import json
import os
import socket
import sys
import types

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import m3_synth
    args = types.SimpleNamespace(layer=bench.LAYER, batch=1)
    cx = bench.Ctx(args, device="cpu")
    my_ms = 10.0 + 5.0 * rank                     # rank 1 is the slow one
    cx.barrier()
    slowest = cx.max_over_ranks(my_ms)
    shape = bench.rank_shape(bench.LAYER, cx.rank, batch=1)
    small = m3_synth.shrink(shape, seqlen=8, nheads=2, ngroups=2)
    x = m3_synth.make_scan_inputs(small)["x"].float()
    cx.close()
    with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
        json.dump({"slowest": slowest, "seed": shape.seed, "batch": shape.batch,
                   "x0": x.flatten()[:4].tolist(), "world": cx.world}, f)


def test_two_gloo_ranks_agree_on_the_slowest_time_and_draw_distinct_problems(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    r = [json.load(open(tmp_path / f"r{k}.json")) for k in range(world)]
    assert r[0]["slowest"] == r[1]["slowest"] == 15.0
    assert r[0]["world"] == r[1]["world"] == 2
    assert r[0]["seed"] != r[1]["seed"]
    assert r[0]["x0"] != r[1]["x0"]
    assert r[0]["batch"] == r[1]["batch"] == 1


def test_throughput_counts_every_rank_over_the_slowest_time():
    # 2 ranks x 8 sequences x 4096 tokens, 10 steps, slowest rank 20 ms in total
    v = bench.throughput(2, 8 * 4096, 10, 20.0)
    assert v == pytest.approx(2 * 8 * 4096 * 10 / 0.020)
    assert bench.throughput(1, 8 * 4096, 10, 20.0) == pytest.approx(v / 2)


def test_single_rank_context_needs_no_process_group():
    args = types.SimpleNamespace(layer=bench.LAYER, batch=0)
    env = {k: os.environ.pop(k) for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK") if k in os.environ}
    try:
        cx = bench.Ctx(args, device="cpu")
        assert cx.world == 1 and cx.max_over_ranks(3.5) == 3.5
        cx.barrier()
        cx.close()
    finally:
        os.environ.update(env)


def test_traffic_is_reported_only_for_the_captured_sources_and_plan():
    d = bench.source_digest("scan_tc_kernel")
    assert len(d) == 16 and d == bench.source_digest("scan_tc_kernel")
    assert d != bench.source_digest("step_pipe_kernel")
    caps = {"scan_tc_kernel": ("mimo_r4_layer", 1, 123, d)}
    t, src = bench.captured_traffic("scan_tc_kernel", "mimo_r4_layer", 1, captures=caps)
    assert t == 123 and d in src
    # another plan, another workload, other sources, no capture: no figure
    assert bench.captured_traffic("scan_tc_kernel", "mimo_r4_layer", 4, captures=caps)[0] is None
    assert bench.captured_traffic("scan_tc_kernel", "long_siso", 1, captures=caps)[0] is None
    stale = {"scan_tc_kernel": ("mimo_r4_layer", 1, 123, "0" * 16)}
    t, why = bench.captured_traffic("scan_tc_kernel", "mimo_r4_layer", 1, captures=stale)
    assert t is None and "changed" in why
    assert bench.captured_traffic("step_pipe_kernel", "decode", captures=caps)[0] is None
    # every committed capture names a known kernel and a digest of its sources
    for k, cap in bench.CAPTURES.items():
        assert k in bench.KERNEL_SOURCES
        assert cap is None or (len(cap) == 4 and len(cap[3]) == 16)


def test_bench_defaults_are_one_gpu_and_minutes_of_work(monkeypatch):
    monkeypatch.setattr(sys, "argv", ["bench.py"])
    a = bench.parse()
    assert a.gpus == 1 and a.warmup >= 3 and 1 <= a.steps <= 200
    assert a.impl == "ours" and a.layer == bench.LAYER and a.decode_steps == 1000
    assert not a.no_bwd and not a.no_phase    # every measured part runs by default


def test_reference_arm_prints_on_rank_0_only():
    """Under torchrun the oracle arm runs on rank 0 alone; another rank exits 0
    at once, prints nothing and joins no process group."""
    import subprocess
    env = {**os.environ, "RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1",
           "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(_free_port())}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "3"], env=env, cwd=ROOT, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_prefill_roofline_arithmetic():
    """The algorithmic bytes and FLOPs of the R=4 layer prefill, from tensor
    shapes alone (meta tensors): 3336 B per token-head (x 512, y 512, B and C
    2048, theta 256, dt and lambda 8) plus A and the final carry once, and
    (Q+1) R^2 (N+P) + 4 R N P = 330,752 FLOP per token-head at Q = 64."""
    import torch
    import m3_synth
    s = m3_synth.MIMO_R4_LAYER
    b, L, H, G, R, P, N = s.batch, s.seqlen, s.nheads, s.ngroups, s.rank, s.headdim, s.dstate

    def m(*shape, dtype=torch.float32):
        return torch.empty(*shape, dtype=dtype, device="meta")

    bf = torch.bfloat16
    t = {"x": m(b, L, H, R, P, dtype=bf), "B": m(b, L, G, R, N, dtype=bf), "C": m(b, L, G, R, N, dtype=bf),
         "dt": m(b, L, H), "A": m(H), "lam": m(b, L, H), "theta": m(b, L, G, N // 2)}
    fin = types.SimpleNamespace(h=m(b, H, N, P), prev_B=m(b, H, R, N, dtype=bf), prev_x=m(b, H, R, P, dtype=bf))
    token_heads = b * L * H
    carry = b * H * (N * P * 4 + R * N * 2 + R * P * 2)
    got = bench.algorithmic_bytes(t, m(b, L, H, R, P, dtype=bf), fin)
    assert got == 3336 * token_heads + 4 * H + carry == 3_506_831_488
    assert bench.algorithmic_flops(s, 64) == 330_752 * token_heads
    # the tcgen05 path's chunk at R = 4 (one 128-row tile = 32 tokens):
    # 33 * 16 * 192 + 4 * 4 * 128 * 64 = 232,448 FLOP per token-head
    assert bench.algorithmic_flops(s, 32) == 232_448 * token_heads
