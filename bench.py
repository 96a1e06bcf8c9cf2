#!/usr/bin/env python
"""Throughput of the Mamba-3 SSM layer scan on B200 GPUs.

Default workload: the chunked prefill (m3_scan_fwd) of the 1.5B-scale MIMO
layer -- batch 8, 32 heads, L = 4096, P = 64, N = 128, rank 4, chunk 64,
bfloat16 x/B/C, float32 dt/A/lambda/theta -- on synthetic seeded inputs
(m3_synth).  One step = one m3_scan_fwd over the whole batch, final carry
included.  The same run reports, each in its own object: "e2e" (pinned host
inputs in and y out inside the timed region), "rope" (m3_rope_bc), "bwd"
(m3_scan_bwd), "phase" (two phase interventions), "layers" (the SISO layer and
the long-context SISO layer), "decode" (m3_step, batch 256, 32 heads, rank 4,
carry from the prefill), "variants" (damping regimes and reflection on the
SISO layer) and "cpu_baseline" (the fp64 oracle on a bounded sample).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (torchrun, one rank per GPU) every rank runs its own independent
batch (weak scaling, no collective on the data path); the timed region is
bracketed by a barrier and device syncs, and the max over ranks is reported.
``--impl reference`` times the fp64 CPU oracle on a bounded sample of the
same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "tokens/sec per SSM layer (chunked fwd, decode step) and % of roofline on 1 B200"
LAYER = "mimo_r4_layer"       # the 1.5B-like MIMO layer
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--decode-steps", type=int, default=1000)
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-rope", action="store_true", help="skip the m3_rope_bc measurement")
    ap.add_argument("--no-layers", action="store_true",
                    help="skip the SISO and long-context SISO prefill objects")
    ap.add_argument("--no-bwd", action="store_true", help="skip the backward pass m3_scan_bwd")
    ap.add_argument("--no-phase", action="store_true", help="skip the two phase interventions")
    # accepted for older command lines: the two measurements now run by default
    ap.add_argument("--bwd", action="store_true", help=argparse.SUPPRESS)
    ap.add_argument("--phase", action="store_true", help=argparse.SUPPRESS)
    ap.add_argument("--no-variants", action="store_true",
                    help="skip the damping-regime and reflection variants")
    ap.add_argument("--batch", type=int, default=0,
                    help="override the layer's batch (profiling captures of a smaller case)")
    ap.add_argument("--workload", choices=["both", "prefill", "decode"], default="both",
                    help="decode alone starts from a seeded random carry (profiling captures)")
    ap.add_argument("--decode-batch", type=int, default=0,
                    help="override the decode batch (profiling captures of a smaller case)")
    ap.add_argument("--layer", choices=["siso_layer", "mimo_r4_layer", "long_siso"], default=LAYER,
                    help="prefill workload: the R=4 MIMO layer (default, the headline), the SISO "
                         "layer or the long-context SISO layer")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return dict(hbm=float(j["hbm_gbs"]), bf16=float(j["bf16_tflops"]),
                    bf16_sus=float(j.get("bf16_tflops_sustained", j["bf16_tflops"])), src="measured")
    return dict(hbm=FALLBACK_HBM_GBS, bf16=FALLBACK_BF16_TFLOPS, bf16_sus=1400.0, src="fallback")


# ------------------------------------------------------------ clocks (NVML) --
class ClockSampler:
    """Samples SM clock and clock-event reasons every 5 ms in a thread."""
    BITS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
            0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks",
            0x1: "gpu_idle"}

    def __init__(self, device_index: int):
        self.samples, self.reasons, self.ok = [], set(), False
        self._stop = threading.Event()
        self.active = False
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid.encode())
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.fn = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
            self.ok = True
        except Exception as e:  # noqa: BLE001
            self.err = repr(e)

    def _run(self):
        while not self._stop.is_set():
            try:
                if self.active:
                    mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                    bits = self.fn(self.h)
                    util = self.nv.nvmlDeviceGetUtilizationRates(self.h).gpu
                    self.samples.append((mhz, bits, util))
            except Exception:  # noqa: BLE001
                pass
            time.sleep(0.005)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self.ok:
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"error": getattr(self, "err", "nvml unavailable")}
        loaded = [s for s in self.samples if s[2] > 0] or self.samples
        reasons = set()
        for _, bits, _ in loaded:
            for b, name in self.BITS.items():
                if bits & b and name != "gpu_idle":
                    reasons.add(name)
        return {"sm_mhz": statistics.median([s[0] for s in loaded]) if loaded else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(reasons), "samples": len(loaded)}


# ----------------------------------------------------------------- sizes --
def algorithmic_bytes(t: dict, y, fin) -> int:
    """Compulsory bytes of one prefill: every input read once, y and the final
    carry written once."""
    n = sum(v.numel() * v.element_size() for v in t.values())
    n += y.numel() * y.element_size()
    for v in (fin.h, fin.prev_B, fin.prev_x):
        n += v.numel() * v.element_size()
    return n


def algorithmic_flops(s, chunk: int) -> float:
    """Causal chunked-scan FLOPs per token-head at chunk length `chunk` (the
    one the plan runs): intra-chunk Gram + masked product ((Q+1) R^2 (N+P)),
    plus the state terms (chunk output C~ S and chunk state B~^T X: 4 R N P)."""
    Q, R, N, P = chunk, s.rank, s.dstate, s.headdim
    per = (Q + 1) * R * R * (N + P) + 4 * R * N * P
    return float(per) * s.batch * s.seqlen * s.nheads


# ------------------------------------------------------------- reference --
def oracle_sample_timing(budget_s: float, min_calls: int = 2, max_calls: int = 20, fixed_calls: int = 0,
                         warmup: int = 1):
    """The fp64 oracle on a bounded sample of the headline workload: batch row
    0 of 8, the whole sequence, all heads (fewer heads when one call would not
    fit the budget).  `warmup` untimed calls, then timed calls: `fixed_calls`
    if given, else as many as fit in `budget_s` (between min_calls and
    max_calls).  Returns (layer tokens per second, seconds per call, calls,
    heads)."""
    import numpy as np
    import torch
    import m3_synth
    import oracle
    s = m3_synth.LAYERS[LAYER]
    sub = m3_synth.shrink(s, batch=1)
    f = {k: v.to(torch.float64).numpy() for k, v in m3_synth.make_scan_inputs(sub).items()}
    t0 = time.perf_counter()
    oracle.scan(**f)
    first = time.perf_counter() - t0
    heads = s.nheads
    calls = fixed_calls if fixed_calls > 0 else int(min(max_calls, max(min_calls, budget_s // max(first, 1e-6))))
    if (calls + warmup) * first > 1.5 * budget_s:
        # the oracle runs one (b, h) per thread, so a call costs whole rounds of
        # `cores` heads: keep as many rounds as fit in the budget (at least one)
        cores = max(1, oracle.num_threads())
        rounds_all = -(-s.nheads // cores)
        rounds = int(rounds_all * budget_s / ((calls + warmup) * first))
        heads = max(1, min(s.nheads, max(rounds, 1) * cores))
        assert s.ngroups == s.nheads          # one group per head: heads and groups slice together
        f = {k: (v[:heads] if k == "A" else np.ascontiguousarray(v[:, :, :heads])) for k, v in f.items()}
    for _ in range(max(warmup - 1, 0)):
        oracle.scan(**f)
    t0 = time.perf_counter()
    for _ in range(calls):
        oracle.scan(**f)
    dt = (time.perf_counter() - t0) / max(calls, 1)
    toks = sub.batch * sub.seqlen * heads / s.nheads      # layer tokens: all heads of a token
    return toks / dt, dt, calls, heads


def oracle_sample_text(heads: int, calls: int) -> str:
    return (f"batch row 0 of 8 ({heads} of 32 heads x 4096 tokens) per call, {calls} timed calls after "
            "a warm-up call, scaled to layer tokens")


def run_reference(args, rank):
    if rank != 0:
        return 0
    import m3_synth
    import oracle
    s = m3_synth.LAYERS[LAYER]
    val, dt, calls, heads = oracle_sample_timing(budget_s=120.0, fixed_calls=args.steps,
                                                 warmup=max(args.warmup, 1))
    cores = oracle.num_threads()
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": m3_synth.NAMES[LAYER], "global_batch": s.batch, "seq_len": s.seqlen,
                       "sample": f"batch row 0 of 8, {heads} of 32 heads, full L=4096 per step"},
            "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": cores, "host_cpus": os.cpu_count(),
                             "kind": "oracle", "sample": oracle_sample_text(heads, calls)},
            "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


def cpu_baseline_sample():
    """The oracle on a bounded sample of the same workload, timed on this
    host's cores the same way as the reference arm (warm-up call, then about
    15 s of timed calls)."""
    import oracle
    val, dt, calls, heads = oracle_sample_timing(budget_s=15.0)
    out = {"value": val, "unit": "tokens/s", "cores": oracle.num_threads(), "host_cpus": os.cpu_count(),
           "kind": "oracle", "sample": oracle_sample_text(heads, calls), "seconds_per_call": dt}
    out["single_thread"] = oracle_single_thread()
    out["decode"] = oracle_decode_sample()
    return out


def oracle_decode_sample(budget_s: float = 5.0):
    """The oracle's decode step on a fixed subset of the decode workload:
    sequences j = 0 mod 16 of the 256 (all 32 heads), seeded carry and
    tokens, as many steps as fit in about `budget_s` after one warm-up step;
    tokens/s counts one token per sequence and step."""
    import numpy as np
    import torch
    import m3_synth
    import oracle
    dec = m3_synth.DECODE
    sub = list(range(0, dec.batch, 16))
    c = m3_synth.make_carry(dec.batch, dec.nheads, dec.dstate, dec.headdim, dec.rank, dec.dtype, dec.seed,
                            scale=0.5)
    f64 = lambda t: t.to(torch.float64).numpy()
    h, pB, pX = f64(c["h"])[sub], f64(c["prev_B"])[sub], f64(c["prev_x"])[sub]
    A = -np.exp(np.linspace(-2, 1, dec.nheads))
    toks = [{k: f64(v)[sub] for k, v in m3_synth.make_decode_token(dec, k).items()} for k in range(4)]

    def one(k):
        t = toks[k % len(toks)]
        return oracle.step(h, pB, pX, t["x"], t["B"], t["C"], t["dt"], A, t["lam"], t["theta"])

    t0 = time.perf_counter()
    _, h, pB, pX = one(0)
    first = max(time.perf_counter() - t0, 1e-6)
    n = int(max(2, min(200, budget_s // first)))
    t0 = time.perf_counter()
    for k in range(n):
        _, h, pB, pX = one(k + 1)
    dt = (time.perf_counter() - t0) / n
    return {"value": len(sub) / dt, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"decode step on {len(sub)} of 256 sequences (j = 0 mod 16, all 32 heads), "
                      f"{n} timed steps after a warm-up step"}


def oracle_single_thread():
    """The oracle on one host thread, on the two small SISO workloads in full
    (the tiny one and the 4 x 2048-token, 8-head layer): a per-core figure
    beside the all-cores sample."""
    import torch
    import m3_synth
    import oracle
    res = {}
    cores = oracle.num_threads()
    oracle.set_num_threads(1)
    try:
        for name in ("siso_tiny", "siso_layer"):
            s = m3_synth.LAYERS[name]
            f = {k: v.to(torch.float64).numpy() for k, v in m3_synth.make_scan_inputs(s).items()}
            t0 = time.perf_counter()
            oracle.scan(**f)
            dt = time.perf_counter() - t0
            res[name] = {"tokens_per_s": s.batch * s.seqlen / dt, "seconds": dt}
    finally:
        oracle.set_num_threads(cores)
    return res


# ------------------------------------------------------------------ ours --
class Ctx:
    """Per-process state shared by the measured parts.  `device="cpu"` runs
    the same rank plumbing over gloo (the host-logic tests use it)."""

    def __init__(self, args, device: str = "cuda"):
        import torch
        import torch.distributed as dist
        self.args = args
        self.device = device
        self.rank = int(os.environ.get("RANK", "0"))
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        if device == "cuda":
            torch.cuda.set_device(self.local)
        if self.world > 1:
            import datetime
            if device == "cuda":
                dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                        device_id=torch.device("cuda", self.local))
            else:
                dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
        self.dist = dist
        self.pk = peaks()
        self.stream = torch.cuda.current_stream() if device == "cuda" else None

    def barrier(self):
        if self.world > 1:
            self.dist.barrier()

    def max_over_ranks(self, v: float) -> float:
        import torch
        if self.world == 1:
            return v
        t = torch.tensor([v], device=self.device, dtype=torch.float64)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.world > 1:
            self.dist.barrier()
            self.dist.destroy_process_group()


L2_BYTES = 126 * 1024 * 1024

# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum of one launch,
# from ncu) of the dominant kernel of each measured part, keyed to what was
# captured: the kernel, the workload and plan it ran, and a digest of the
# kernel's sources at capture time.  A figure is reported only while the
# built sources still have that digest and the timed launch has that
# workload and plan; otherwise "traffic" is null and the reason is given.
# The ncu commands are in profiles/.
KERNEL_SOURCES = {
    "scan_tc_kernel": ("k_scan_tc.cu", "tc_ptx.cuh", "m3_common.cuh", "m3_kernels.h", "m3_bounds.cuh"),
    "step_pipe_kernel": ("k_step.cu", "m3_common.cuh", "m3_kernels.h", "m3_bounds.cuh"),
    "rope_block_kernel": ("k_rope.cu", "m3_common.cuh", "m3_kernels.h", "m3_bounds.cuh"),
}
CAPTURES = {
    # kernel: (workload, plan segments or None, bytes per launch, source digest)
    "scan_tc_kernel": ("mimo_r4_layer_b8_h32_L4096_P64_N128_Q64_bf16", 1,
                       2_982_624_000 + 525_852_416, "09d664a50f617954"),
    "step_pipe_kernel": ("decode_mimo_r4_b256_h32_P64_N128_x1000", None,
                         304_190_208 + 224_724_480, "87cab08d84241421"),
    "rope_block_kernel": ("mimo_r4_layer_b8_h32_L4096_P64_N128_Q64_bf16", None,
                          2_423_474_432 + 2_379_173_888, "722d31272b55c86c"),
}


def source_digest(kernel: str) -> str:
    """sha256 (first 16 hex digits) of the kernel's source files, in order."""
    import hashlib
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "selective_state_space_m3_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def captured_traffic(kernel: str, workload: str, segments=None, captures=None):
    """(bytes per launch, source) of the capture that matches, else (None, why)."""
    cap = (CAPTURES if captures is None else captures).get(kernel)
    if cap is None:
        return None, "no ncu capture of this kernel on the current sources"
    c_work, c_seg, c_bytes, c_digest = cap
    if c_work != workload or (c_seg is not None and c_seg != segments):
        return None, f"capture is of {c_work} (segments {c_seg}), not of this launch"
    digest = source_digest(kernel)
    if digest != c_digest:
        return None, f"kernel sources changed since the capture (digest {digest}, captured {c_digest})"
    return c_bytes, f"ncu dram__bytes_read.sum + dram__bytes_write.sum of one launch, sources {digest}"


def throughput(world: int, tokens_per_rank: int, steps: int, total_ms: float) -> float:
    """Whole-job tokens/s: every rank processed `tokens_per_rank` per step and
    the slowest rank's time is the job's time."""
    return world * tokens_per_rank * steps / (total_ms / 1e3)


def rank_shape(layer: str, rank: int, batch: int = 0):
    """Each rank runs its own seeded problem of the same shape (weak scaling)."""
    import m3_synth
    s = m3_synth.LAYERS[layer]
    s = m3_synth.shrink(s, seed=s.seed + 1000 * rank)
    if batch > 0:
        s = m3_synth.shrink(s, batch=batch)
    return s


def run_prefill(cx, line):
    """The chunked prefill of one layer workload (default: the R=4 MIMO
    layer); fills the headline keys of `line` and returns what the e2e and
    decode parts reuse."""
    import torch
    import m3_synth
    import selective_state_space_m3_b200 as m3
    args, pk, stream = cx.args, cx.pk, cx.stream
    s = rank_shape(args.layer, cx.rank, args.batch)
    host = m3_synth.make_scan_inputs(s)
    dev = {k: v.cuda() for k, v in host.items()}
    io = m3.M3_BF16 if s.dtype == "bf16" else m3.M3_F32
    d = m3.Dims(s.batch, s.seqlen, s.nheads, s.ngroups, s.headdim, s.dstate, s.rank, s.chunk, io)
    plan = m3.m3_scan_plan(d)
    y = torch.empty_like(dev["x"])
    ws = torch.zeros(m3.m3_scan_workspace_size(d), dtype=torch.uint8, device="cuda")
    fin = m3.Carry(torch.empty(s.batch, s.nheads, s.dstate, s.headdim, device="cuda"),
                   torch.empty(s.batch, s.nheads, s.rank, s.dstate, device="cuda", dtype=dev["x"].dtype),
                   torch.empty(s.batch, s.nheads, s.rank, s.headdim, device="cuda", dtype=dev["x"].dtype))
    abytes = algorithmic_bytes(dev, y, fin)
    # inputs smaller than twice the L2 are evicted between timed launches
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device="cuda") if abytes < 2 * L2_BYTES else None

    def step():
        m3.m3_scan_fwd(d, dev["x"], dev["B"], dev["C"], dev["dt"], dev["A"], dev["lam"], dev["theta"],
                       y, ws, final_state=fin, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert m3.m3_device_status(ws) == m3.M3_OK

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    with ClockSampler(cx.local) as clk:
        clk.active = True
        cx.barrier()
        torch.cuda.synchronize()
        t_all0 = torch.cuda.Event(enable_timing=True)
        t_all1 = torch.cuda.Event(enable_timing=True)
        t_all0.record(stream)
        for e0, e1 in ev:
            if flush is not None:
                flush.zero_()
            e0.record(stream)
            step()
            e1.record(stream)
        t_all1.record(stream)
        torch.cuda.synchronize()
        cx.barrier()
        clk.active = False
    assert m3.m3_device_status(ws) == m3.M3_OK
    launch_ms = [e0.elapsed_time(e1) for e0, e1 in ev]
    per_launch_ms = statistics.mean(launch_ms)
    # with a flush between launches the step time is the launches alone
    own_ms = t_all0.elapsed_time(t_all1) if flush is None else sum(launch_ms)
    total_ms = cx.max_over_ranks(own_ms)
    ms_per_step = total_ms / args.steps
    tokens = s.batch * s.seqlen
    value = throughput(cx.world, tokens, args.steps, total_ms)
    unflushed = None
    if flush is not None:
        # the same launches back to back, inputs left in L2: reported beside
        # the flushed figure, never as the value
        cx.barrier()
        torch.cuda.synchronize()
        u0 = torch.cuda.Event(enable_timing=True)
        u1 = torch.cuda.Event(enable_timing=True)
        u0.record(stream)
        for _ in range(args.steps):
            step()
        u1.record(stream)
        torch.cuda.synchronize()
        cx.barrier()
        assert m3.m3_device_status(ws) == m3.M3_OK
        u_ms = cx.max_over_ranks(u0.elapsed_time(u1))
        unflushed = {"ms_per_step": u_ms / args.steps,
                     "tokens_per_s": throughput(cx.world, tokens, args.steps, u_ms),
                     "l2": "not flushed: inputs stay in L2 between launches"}

    aflops = algorithmic_flops(s, plan["chunk_used"])
    achieved_gbs = abytes / (per_launch_ms / 1e3) / 1e9
    tflops = aflops / (per_launch_ms / 1e3) / 1e12
    workload = m3_synth.NAMES[args.layer] if args.batch <= 0 else m3_synth.NAMES[args.layer] + f"_batch{s.batch}"
    traffic, traffic_src = captured_traffic("scan_tc_kernel", workload, plan["segments"])
    if plan["launches"] != 1:
        traffic, traffic_src = None, "plan has several launches; capture covers one kernel launch"
    line.update({
        "value": value, "ms_per_step": ms_per_step,
        "config": {"workload": workload,
                   "global_batch": s.batch * cx.world,
                   "seq_len": s.seqlen, "nheads": s.nheads, "headdim": s.headdim, "dstate": s.dstate,
                   "rank": s.rank, "chunk": s.chunk,
                   "parallelism": "replicas" if cx.world == 1 else f"dp{cx.world}",
                   "l2": ("inputs %.2f GB per step >> 126 MB L2; no flush" % (abytes / 1e9)) if flush is None
                   else "L2 flushed (252 MB write) before every timed launch",
                   "path": plan["path"], "segments": plan["segments"], "chunk_used": plan["chunk_used"]},
        "roofline": {"bound": "hbm", "achieved": achieved_gbs, "peak": pk["hbm"], "unit": "GB/s",
                     "frac": achieved_gbs / pk["hbm"], "traffic": traffic, "traffic_source": traffic_src,
                     "peak_source": pk["src"],
                     "kernel": "m3_scan_fwd (whole call: %d launch%s)" % (
                         plan["launches"], "" if plan["launches"] == 1 else "es"),
                     "algorithmic_bytes_per_launch": abytes,
                     "tensor_tflops": tflops, "tensor_frac_of_bf16_peak": tflops / pk["bf16"]},
        "clocks": clk.summary(),
        "gpu_launches": plan["launches"] * args.steps})
    if unflushed is not None:
        line["unflushed"] = unflushed
    def run(dv, yy, st):
        m3.m3_scan_fwd(d, dv["x"], dv["B"], dv["C"], dv["dt"], dv["A"], dv["lam"], dv["theta"],
                       yy, ws, final_state=fin, stream=st)

    return dict(s=s, host=host, dev=dev, y=y, fin=fin, step=step, run=run, tokens=tokens)


def run_layer(cx, name):
    """m3_scan_fwd on another prefill workload (the SISO layer, or the
    long-context SISO layer), timed like the headline: CUDA events around
    each call on the launching stream, L2 flushed before each call when the
    inputs are smaller than twice the L2.  Each call is timed twice: launched
    eagerly, and captured once in a CUDA graph and replayed (the plan's
    launches then follow each other on the device with no host in between);
    the graph figure is the object's ms_per_call."""
    import torch
    import m3_synth
    import selective_state_space_m3_b200 as m3
    args, pk, stream = cx.args, cx.pk, cx.stream
    s = rank_shape(name, cx.rank)
    dev = {k: v.cuda() for k, v in m3_synth.make_scan_inputs(s).items()}
    io = m3.M3_BF16 if s.dtype == "bf16" else m3.M3_F32
    d = m3.Dims(s.batch, s.seqlen, s.nheads, s.ngroups, s.headdim, s.dstate, s.rank, s.chunk, io)
    plan = m3.m3_scan_plan(d)
    y = torch.empty_like(dev["x"])
    ws = torch.zeros(m3.m3_scan_workspace_size(d), dtype=torch.uint8, device="cuda")
    fin = m3.Carry(torch.empty(s.batch, s.nheads, s.dstate, s.headdim, device="cuda"),
                   torch.empty(s.batch, s.nheads, s.rank, s.dstate, device="cuda", dtype=dev["x"].dtype),
                   torch.empty(s.batch, s.nheads, s.rank, s.headdim, device="cuda", dtype=dev["x"].dtype))
    abytes = algorithmic_bytes(dev, y, fin)
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device="cuda") if abytes < 2 * L2_BYTES else None

    def call(st):
        m3.m3_scan_fwd(d, dev["x"], dev["B"], dev["C"], dev["dt"], dev["A"], dev["lam"], dev["theta"],
                       y, ws, final_state=fin, stream=st)

    for _ in range(max(3, args.warmup)):
        call(stream)
    torch.cuda.synchronize()
    assert m3.m3_device_status(ws) == m3.M3_OK
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call(torch.cuda.current_stream())
    g.replay()
    torch.cuda.synchronize()
    n = max(5, min(args.steps, 20))

    def timed(fn):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        cx.barrier()
        torch.cuda.synchronize()
        for e0, e1 in ev:
            if flush is not None:
                flush.zero_()
            e0.record(stream)
            fn()
            e1.record(stream)
        torch.cuda.synchronize()
        cx.barrier()
        return cx.max_over_ranks(statistics.mean(e0.elapsed_time(e1) for e0, e1 in ev))

    with ClockSampler(cx.local) as clk:
        clk.active = True
        eager_ms = timed(lambda: call(stream))
        graph_ms = timed(g.replay)
        clk.active = False
    unflushed_ms = None
    if flush is not None:
        # the graph replays back to back, inputs left in L2 (reported beside
        # the flushed figure, never as it)
        cx.barrier()
        torch.cuda.synchronize()
        u0, u1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        u0.record(stream)
        for _ in range(n):
            g.replay()
        u1.record(stream)
        torch.cuda.synchronize()
        cx.barrier()
        unflushed_ms = cx.max_over_ranks(u0.elapsed_time(u1)) / n
    assert m3.m3_device_status(ws) == m3.M3_OK
    del g
    gbs = abytes / (graph_ms / 1e3) / 1e9
    tflops = algorithmic_flops(s, plan["chunk_used"]) / (graph_ms / 1e3) / 1e12
    out = {"workload": m3_synth.NAMES[name], "ms_per_call": graph_ms, "eager_ms_per_call": eager_ms,
           "tokens_per_s": cx.world * s.batch * s.seqlen / (graph_ms / 1e3),
           "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm"], "unit": "GB/s",
                        "frac": gbs / pk["hbm"], "peak_source": pk["src"], "algorithmic_bytes_per_launch": abytes,
                        "traffic": None, "traffic_source": "no ncu capture of this workload on the current sources",
                        "kernel": "m3_scan_fwd (whole call: %d launch%s, CUDA graph)" % (
                            plan["launches"], "" if plan["launches"] == 1 else "es"),
                        "tensor_tflops": tflops, "tensor_frac_of_bf16_peak": tflops / pk["bf16"]},
           "plan": {"path": plan["path"], "segments": plan["segments"], "launches": plan["launches"],
                    "chunk_used": plan["chunk_used"]},
           "l2": ("inputs %.2f GB >> 126 MB L2; no flush" % (abytes / 1e9)) if flush is None
           else "L2 flushed (252 MB write) before every timed call",
           "clocks": clk.summary(), "gpu_launches": (3 if flush is not None else 2) * n * plan["launches"],
           "calls_timed": n}
    if unflushed_ms is not None:
        out["unflushed_ms_per_call"] = unflushed_ms
    del flush, ws, dev
    return out


def run_e2e(cx, line, pf):
    """Pinned host buffers in, y out, the copies inside the timed region.
    Every step copies its inputs in on a copy stream, runs m3_scan_fwd on the
    compute stream and reads y back on a third stream; the device inputs and
    y are double buffered, so that one step's device-to-host read overlaps
    the next step's host-to-device copy (the link's two directions are
    independent).  The timed region runs from the first copy in to the last
    read back."""
    import torch
    pinned = {k: v.pin_memory() for k, v in pf["host"].items()}
    devs = [pf["dev"], {k: torch.empty_like(v) for k, v in pf["dev"].items()}]
    ys = [pf["y"], torch.empty_like(pf["y"])]
    y_host = [torch.empty(pf["y"].shape, dtype=pf["y"].dtype).pin_memory() for _ in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in pinned.values())
    d2h = y_host[0].numel() * y_host[0].element_size()
    ke = max(2, min(cx.args.steps, 4))
    s_in, s_out, s_c = torch.cuda.Stream(), torch.cuda.Stream(), cx.stream

    def steps(n):
        free = [None, None]                    # buffer j's last read-back done
        last = None
        for k in range(n):
            j = k % 2
            with torch.cuda.stream(s_in):
                if free[j] is not None:
                    s_in.wait_event(free[j])
                for name, v in pinned.items():
                    devs[j][name].copy_(v, non_blocking=True)
                e_in = torch.cuda.Event()
                e_in.record(s_in)
            s_c.wait_event(e_in)
            pf["run"](devs[j], ys[j], s_c)
            e_c = torch.cuda.Event()
            e_c.record(s_c)
            with torch.cuda.stream(s_out):
                s_out.wait_event(e_c)
                y_host[j].copy_(ys[j], non_blocking=True)
                last = torch.cuda.Event()
                last.record(s_out)
            free[j] = last
        return last

    steps(2)
    torch.cuda.synchronize()
    cx.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    done = steps(ke)
    s_out.wait_event(done)
    e1.record(s_out)
    torch.cuda.synchronize()
    cx.barrier()
    ms = cx.max_over_ranks(e0.elapsed_time(e1))
    line["e2e"] = {"value": cx.world * pf["tokens"] * ke / (ms / 1e3), "unit": "tokens/s",
                   "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": ke,
                   "overlap": "step k's read-back overlaps step k+1's copy in (double-buffered device inputs)"}
    del devs[1], ys[1]


def run_rope(cx, line, pf):
    """m3_rope_bc (cumulative phase and rotated B, C per head) on the layer's
    inputs: its own roofline, since it is the one standalone HBM-bound pass."""
    import torch
    import selective_state_space_m3_b200 as m3
    args, pk, stream = cx.args, cx.pk, cx.stream
    s, dev = pf["s"], pf["dev"]
    io = dev["B"].dtype
    Bo = torch.empty((s.batch, s.seqlen, s.nheads, s.rank, s.dstate), device="cuda", dtype=io)
    Co = torch.empty_like(Bo)
    ph = torch.empty((s.batch, s.seqlen, s.nheads, s.dstate // 2), device="cuda", dtype=torch.float32)
    d = m3.Dims(s.batch, s.seqlen, s.nheads, s.ngroups, s.headdim, s.dstate, s.rank, s.chunk,
                m3.M3_BF16 if s.dtype == "bf16" else m3.M3_F32)

    def call():
        m3.m3_rope_bc(d, dev["B"], dev["C"], dev["dt"], dev["theta"], Bo, Co, ph, stream=stream)

    for _ in range(max(3, args.warmup)):
        call()
    torch.cuda.synchronize()
    n = max(5, min(args.steps, 20))
    cx.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(n):
        call()
    e1.record(stream)
    torch.cuda.synchronize()
    cx.barrier()
    ms = cx.max_over_ranks(e0.elapsed_time(e1)) / n
    nbytes = sum(dev[k].numel() * dev[k].element_size() for k in ("B", "C", "dt", "theta"))
    nbytes += sum(v.numel() * v.element_size() for v in (Bo, Co, ph))
    gbs = nbytes / (ms / 1e3) / 1e9
    rope_traffic, rope_src = captured_traffic("rope_block_kernel", line["config"]["workload"])
    line["rope"] = {"workload": "rope_bc_" + line["config"]["workload"], "ms_per_call": ms,
                    "tokens_per_s": cx.world * s.batch * s.seqlen / (ms / 1e3),
                    "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm"], "unit": "GB/s",
                                 "frac": gbs / pk["hbm"], "algorithmic_bytes_per_launch": nbytes,
                                 "traffic": rope_traffic, "traffic_source": rope_src},
                    "gpu_launches": n, "l2": "inputs and outputs %.1f GB >> L2; no flush" % (nbytes / 1e9)}
    del Bo, Co, ph


def run_bwd(cx, line, pf):
    """m3_scan_bwd on the layer: the gradients of sum <dy, y> with respect to
    every input (float32 outputs), dy seeded."""
    import numpy as np
    import torch
    import selective_state_space_m3_b200 as m3
    args, pk, stream = cx.args, cx.pk, cx.stream
    s, dev = pf["s"], pf["dev"]
    b, L, H, G, R, P, N = s.batch, s.seqlen, s.nheads, s.ngroups, s.rank, s.headdim, s.dstate
    rng = np.random.default_rng(s.seed + 77)
    dy = torch.from_numpy(rng.standard_normal((b, L, H, R, P)).astype(np.float32)).to(dev["x"].dtype).cuda()
    f = dict(device="cuda", dtype=torch.float32)
    g = {"dx": torch.empty(b, L, H, R, P, **f), "dB": torch.empty(b, L, G, R, N, **f),
         "dC": torch.empty(b, L, G, R, N, **f), "ddt": torch.empty(b, L, H, **f), "dA": torch.empty(H, **f),
         "dlam": torch.empty(b, L, H, **f), "dtheta": torch.empty(b, L, G, N // 2, **f)}
    d = m3.Dims(b, L, H, G, P, N, R, s.chunk, m3.M3_BF16 if s.dtype == "bf16" else m3.M3_F32)
    ws = torch.zeros(m3.m3_scan_bwd_workspace_size(d), dtype=torch.uint8, device="cuda")

    def call():
        m3.m3_scan_bwd(d, dev["x"], dev["B"], dev["C"], dev["dt"], dev["A"], dev["lam"], dev["theta"],
                       dy, g, ws, stream=stream)

    call()
    torch.cuda.synchronize()
    n = 3
    cx.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(n):
        call()
    e1.record(stream)
    torch.cuda.synchronize()
    cx.barrier()
    ms = cx.max_over_ranks(e0.elapsed_time(e1)) / n
    nbytes = sum(dev[k].numel() * dev[k].element_size() for k in dev) + dy.numel() * dy.element_size()
    nbytes += sum(v.numel() * v.element_size() for v in g.values())
    gbs = nbytes / (ms / 1e3) / 1e9
    line["bwd"] = {"workload": "scan_bwd_" + line["config"]["workload"], "ms_per_call": ms,
                   "tokens_per_s": cx.world * b * L / (ms / 1e3),
                   "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm"], "unit": "GB/s",
                                "frac": gbs / pk["hbm"], "algorithmic_bytes_per_launch": nbytes,
                                "traffic": None},
                   "gpu_launches": 2 * n, "kernels": "checkpoint forward + reverse (SIMT, float32)"}
    del g, ws, dy


def run_phase(cx, line, pf):
    """m3_scan_fwd_phase on the layer for two interventions (reversed phase:
    a theta rewrite; rotation on readout only: m3_rope_bc plus a theta = 0
    scan), against the prefill's algorithmic bytes."""
    import torch
    import selective_state_space_m3_b200 as m3
    args, pk, stream = cx.args, cx.pk, cx.stream
    s, dev = pf["s"], pf["dev"]
    d = m3.Dims(s.batch, s.seqlen, s.nheads, s.ngroups, s.headdim, s.dstate, s.rank, s.chunk,
                m3.M3_BF16 if s.dtype == "bf16" else m3.M3_F32)
    y = torch.empty_like(dev["x"])
    out = {}
    for name, mode in (("reverse", m3.M3_PHASE_REVERSE), ("read_only", m3.M3_PHASE_READ_ONLY)):
        ws = torch.zeros(m3.m3_scan_phase_workspace_size(d, mode), dtype=torch.uint8, device="cuda")

        def call():
            m3.m3_scan_fwd_phase(d, mode, dev["x"], dev["B"], dev["C"], dev["dt"], dev["A"], dev["lam"],
                                 dev["theta"], y, ws, stream=stream)

        for _ in range(3):
            call()
        torch.cuda.synchronize()
        n = 10
        cx.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n):
            call()
        e1.record(stream)
        torch.cuda.synchronize()
        cx.barrier()
        assert m3.m3_device_status(ws) == m3.M3_OK
        ms = cx.max_over_ranks(e0.elapsed_time(e1)) / n
        gbs = line["roofline"]["algorithmic_bytes_per_launch"] / (ms / 1e3) / 1e9
        out[name] = {"ms_per_call": ms, "tokens_per_s": cx.world * s.batch * s.seqlen / (ms / 1e3),
                     "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm"], "unit": "GB/s",
                                  "frac": gbs / pk["hbm"], "traffic": None,
                                  "algorithmic_bytes_per_launch": line["roofline"]["algorithmic_bytes_per_launch"]}}
        del ws
    line["phase"] = out


def fp32_peak_tflops(sm_max_mhz) -> float:
    """FP32 FMA roofline of the CUDA cores: 148 SMs x 128 FP32 lanes x 2 FLOP
    per FMA x the maximum SM clock (1965 MHz on this machine's B200s)."""
    return 148 * 128 * 2 * float(sm_max_mhz or 1965) * 1e6 / 1e12


def variant_flops(s, reflect: bool) -> float:
    """Algorithmic FLOPs of the token-by-token recurrence per call: per state
    element and token, the pending beta term (2R + 1), the 2x2 pair block (3),
    the input term (2R + 1) and the readout (2R); the reflection adds its
    projection and update (4)."""
    per = 6 * s.rank + 5 + (4 if reflect else 0)
    return float(per) * s.dstate * s.headdim * s.batch * s.seqlen * s.nheads


def run_variants(cx, line):
    """The transition variants on the SISO layer workload (batch 4, 8 heads,
    L = 2048, bf16): the critically damped and overdamped regimes
    (m3_scan_fwd_damped) and the low-rank reflection (m3_scan_fwd_reflect),
    token by token in float32 on the CUDA cores (roofline: FP32 FMA rate).
    The 25 MB of inputs are evicted from L2 before every timed launch."""
    import torch
    import m3_synth
    import selective_state_space_m3_b200 as m3
    args, pk, stream = cx.args, cx.pk, cx.stream
    s = m3_synth.shrink(m3_synth.SISO_LAYER, seed=m3_synth.SISO_LAYER.seed + 1000 * cx.rank)
    host = m3_synth.make_scan_inputs(s)
    dev = {k: v.cuda() for k, v in host.items()}
    theta_over = m3_synth.overdamped_theta(host, s).cuda()
    u = m3_synth.make_reflect_direction(s).cuda()
    d = m3.Dims(s.batch, s.seqlen, s.nheads, s.ngroups, s.headdim, s.dstate, s.rank, s.chunk, m3.M3_BF16)
    y = torch.empty_like(dev["x"])
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device="cuda")
    nbytes = sum(v.numel() * v.element_size() for v in dev.values()) + y.numel() * y.element_size()
    out = {}
    calls = {
        "critical": lambda: m3.m3_scan_fwd_damped(d, m3.M3_DAMP_CRITICAL, dev["x"], dev["B"], dev["C"], dev["dt"],
                                                  dev["A"], dev["lam"], dev["theta"], y, stream=stream),
        "over": lambda: m3.m3_scan_fwd_damped(d, m3.M3_DAMP_OVER, dev["x"], dev["B"], dev["C"], dev["dt"],
                                              dev["A"], dev["lam"], theta_over, y, stream=stream),
        "reflect": lambda: m3.m3_scan_fwd_reflect(d, u, dev["x"], dev["B"], dev["C"], dev["dt"], dev["A"],
                                                  dev["lam"], dev["theta"], y, stream=stream),
    }
    with ClockSampler(cx.local) as clk:
        for name, call in calls.items():
            for _ in range(3):
                call()
            torch.cuda.synchronize()
            n = 10
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
            cx.barrier()
            clk.active = True
            for e0, e1 in ev:
                flush.zero_()
                e0.record(stream)
                call()
                e1.record(stream)
            torch.cuda.synchronize()
            clk.active = False
            cx.barrier()
            ms = cx.max_over_ranks(statistics.mean(e0.elapsed_time(e1) for e0, e1 in ev))
            fl = variant_flops(s, name == "reflect")
            peak = fp32_peak_tflops(clk.max_mhz if clk.ok else None)
            tf = fl / (ms / 1e3) / 1e12
            out[name] = {"ms_per_call": ms, "tokens_per_s": cx.world * s.batch * s.seqlen / (ms / 1e3),
                         "roofline": {"bound": "alu", "achieved": tf, "peak": peak, "unit": "TFLOP/s",
                                      "frac": tf / peak, "algorithmic_flops_per_launch": fl,
                                      "peak_source": "148 SMs x 128 FP32 lanes x 2 x max SM clock",
                                      "hbm_frac": nbytes / (ms / 1e3) / 1e9 / pk["hbm"], "traffic": None},
                         "gpu_launches": n}
    out["workload"] = m3_synth.NAMES["siso_layer"]
    out["l2"] = "L2 flushed (252 MB write) before every timed launch"
    out["clocks"] = clk.summary()
    line["variants"] = out
    del flush


def run_decode(cx, line, pf):
    """m3_step x decode_steps captured in one CUDA graph; the carry comes from
    the prefill's final state (tiled, sequence j <- batch row j mod 8), or
    from a seeded random carry when the decode runs alone."""
    import torch
    import m3_synth
    import selective_state_space_m3_b200 as m3
    args, pk, stream = cx.args, cx.pk, cx.stream
    dec = m3_synth.DecodeShape(seed=m3_synth.DECODE.seed + 1000 * cx.rank)
    if args.decode_batch > 0:
        dec = dataclasses_replace(dec, batch=args.decode_batch)
    if pf is not None and args.layer == LAYER:
        fin = pf["fin"]
        reps = -(-dec.batch // fin.h.shape[0])
        state = m3.Carry(fin.h.repeat(reps, 1, 1, 1)[:dec.batch].contiguous(),
                         fin.prev_B.repeat(reps, 1, 1, 1)[:dec.batch].contiguous(),
                         fin.prev_x.repeat(reps, 1, 1, 1)[:dec.batch].contiguous())
        Ad = pf["dev"]["A"]
    else:
        c = m3_synth.make_carry(dec.batch, dec.nheads, dec.dstate, dec.headdim, dec.rank, dec.dtype,
                                dec.seed, scale=0.5)
        state = m3.Carry(c["h"].cuda(), c["prev_B"].cuda(), c["prev_x"].cuda())
        Ad = (-torch.exp(torch.linspace(-2, 1, dec.nheads))).cuda()
    pool = 64      # distinct tokens (22 MB each at batch 256; 1.4 GB >> L2), cycled
    toks = []
    for k in range(pool):
        t = m3_synth.make_decode_token(dec, k)
        toks.append({n: v.cuda() for n, v in t.items()})
    dd = m3.Dims(dec.batch, 1, dec.nheads, dec.ngroups, dec.headdim, dec.dstate, dec.rank, 1, m3.M3_BF16)
    yd = torch.empty_like(toks[0]["x"])
    S = args.decode_steps

    def run_steps(n, st):
        for k in range(n):
            t = toks[k % pool]
            m3.m3_step(dd, state, t["x"], t["B"], t["C"], t["dt"], Ad, t["lam"], t["theta"], yd, stream=st)

    run_steps(3, stream)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run_steps(S, torch.cuda.current_stream())
    g.replay()
    torch.cuda.synchronize()
    reps_t = 2
    with ClockSampler(cx.local) as clk2:
        clk2.active = True
        cx.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps_t):
            g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        cx.barrier()
        clk2.active = False
    ms = cx.max_over_ranks(e0.elapsed_time(e1))
    per_step_us = ms * 1e3 / (reps_t * S)
    t0 = toks[0]
    step_bytes = (2 * state.h.numel() * 4 + 2 * (state.prev_B.numel() + state.prev_x.numel()) * 2 +
                  sum(v.numel() * v.element_size() for v in t0.values()) + yd.numel() * 2 + Ad.numel() * 4)
    gbs = step_bytes / (per_step_us * 1e-6) / 1e9
    dec_work = m3_synth.NAMES["decode"] if dec.batch == 256 else f"decode_b{dec.batch}"
    dec_traffic, dec_src = captured_traffic("step_pipe_kernel", dec_work)
    line["decode"] = {"workload": dec_work,
                      "tokens_per_s": cx.world * dec.batch / (per_step_us * 1e-6),
                      "us_per_step": per_step_us, "steps_timed": reps_t * S,
                      "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm"], "unit": "GB/s",
                                   "frac": gbs / pk["hbm"], "algorithmic_bytes_per_launch": step_bytes,
                                   "traffic": dec_traffic, "traffic_source": dec_src},
                      "gpu_launches": reps_t * S, "clocks": clk2.summary(),
                      "carry": "prefill final state" if pf is not None and args.layer == LAYER
                      else "seeded random",
                      "inputs": f"{pool} distinct tokens cycled"}
    del g


def dataclasses_replace(obj, **kw):
    import dataclasses
    return dataclasses.replace(obj, **kw)


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank)
    cx = Ctx(args)
    line = {"metric": METRIC, "value": None, "unit": "tokens/s", "n_gpus": cx.world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": None, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic"}
    pf = None
    if args.workload in ("both", "prefill"):
        pf = run_prefill(cx, line)
        if not args.no_e2e:
            run_e2e(cx, line, pf)
        if not args.no_rope:
            run_rope(cx, line, pf)
        if not args.no_bwd:
            run_bwd(cx, line, pf)
        if not args.no_phase:
            run_phase(cx, line, pf)
        if args.layer == LAYER and not args.no_layers:
            # the other two prefill workloads, each in its own object
            line["layers"] = {n: run_layer(cx, n) for n in ("siso_layer", "long_siso")}
    if args.workload in ("both", "decode") and not args.no_decode:
        run_decode(cx, line, pf)
    if args.workload == "both" and not args.no_variants:
        run_variants(cx, line)
    if cx.world == 1 and not args.no_cpu and args.workload != "decode" and args.layer == LAYER:
        line["cpu_baseline"] = cpu_baseline_sample()
    cx.close()
    if cx.rank == 0:
        print(json.dumps(line))
    return 0


if __name__ == "__main__":
    sys.exit(main())
