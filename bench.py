#!/usr/bin/env python
"""Throughput benchmark of the Mamba-3 SSM layer core (libm3) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one pass of the whole hot path over one batch of the 1.5B-scale layer (batch 2,
seqlen 32768, 32 heads x 128, d_state 128, MIMO rank 4, bf16 x/B/C, fp32 state): m3_scan_fwd
over the 2 x 32768 prompt tokens, then m3_decode_step for one more token per sequence from the
final state.  value = tokens/s over all ranks (weak scaling: every rank runs its own batch; no
data-path collective).  Inputs are seeded and synthetic; one input set (1.25 GB) is larger
than L2, and two sets alternate between steps.

Extra keys: "prefill" / "decode" give each kernel measured on its own ("prefill.p1_layer" the
page-1-shaped layer, "prefill.sweep_l15b" the 1.5B-scale layer at 2K and 8K tokens; decode on
the 1.5B-scale layer at batch 128, "decode.sweep" batches 1, 16 and 512); "roofline" is the
dominant kernel (the tensor-core prefill) against MEASURED_PEAKS.json; "cpu_baseline" times the
fp64 oracle (test infrastructure) on a bounded sample and compares its outputs with the GPU's;
"e2e" times the same step through the C ABI with pinned host buffers and the host<->device
copies inside the timed region.

--impl reference times the fp64 CPU oracle alone (the reference arm of this build).
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "Mamba-3 SSM tokens/s (prefill, decode) and % of tensor-core / HBM roofline"
WORKLOAD = "l15b_32k"
EXTRA_PREFILL = "p1_layer"
DECODE_WORKLOAD = "decode_b128"
L2_BYTES = 126 * 1024 * 1024

# dram bytes read and written by one m3_scan_fwd on the headline workload (state pass + full
# pass), from the committed ncu summary of that kernel; None whenever the kernel has changed
# since the counters were taken.
PREFILL_DRAM = {"read": 4 * 281106432, "write": 4 * 103955968,
                "note": "ncu dram__bytes_read/write.sum of both launches on l15b_8k (the same 2-segment plan), "
                        "scaled by tokens to l15b_32k; writes below algorithmic: the last ~100 MB of y is "
                        "still in L2 when the kernel ends"}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


# ------------------------------------------------------------------ algorithmic counts

def prefill_bytes(d):
    """Algorithmic HBM bytes of one m3_scan_fwd: every input read once, y written once,
    state (h, carry) read and written once."""
    r, w = prefill_bytes_rw(d)
    return r + w


def prefill_bytes_rw(d):
    """(read, written) algorithmic bytes of one m3_scan_fwd: x, B, C, theta, dt, A, lam and
    the state read once; y and the state written once."""
    b, L, H, P, N, R, G = (d[k] for k in ("b", "L", "H", "P", "N", "R", "G"))
    e = 2 if d["dtype"] == "bf16" else 4
    tok = b * L
    state = b * H * (N * P + R * N + P) * 4
    read = tok * (H * P * e + 2 * G * R * N * e + G * (N // 2) * 4 + 3 * H * 4) + state
    written = tok * H * P * e + state
    return read, written


def prefill_flops(d, chunk=32):
    """Algorithmic FLOPs of the chunked scan at the model's chunk length (dense chunk
    tiles): per token and head 2 Q R^2 (N + P) (intra-chunk C B^T and its product
    with X) + 4 R N P (state readout and state update)."""
    b, L, H, P, N, R = (d[k] for k in ("b", "L", "H", "P", "N", "R"))
    intra = 2 * chunk * R * R * (N + P)
    inter = 4 * R * N * P
    return b * L * H * (intra + inter), b * L * H * intra


def decode_bytes(d):
    """Algorithmic HBM bytes of one m3_decode_step: state read + written, token I/O."""
    b, H, P, N, R, G = (d[k] for k in ("b", "H", "P", "N", "R", "G"))
    e = 2 if d["dtype"] == "bf16" else 4
    state = 2 * b * H * (N * P + R * N + P) * 4
    io = b * (2 * H * P * e + 2 * G * R * N * e + G * (N // 2) * 4 + 3 * H * 4)
    return state + io


def decode_flops(d):
    b, H, P, N, R = (d[k] for k in ("b", "H", "P", "N", "R"))
    # per state element: rank-R u_t and u_{t-1} (4R), rotation + decay + add (~8), readout (2R)
    return b * H * N * P * (6 * R + 8)


# ------------------------------------------------------------------ peaks, clocks

def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            j = json.load(f)
        return dict(hbm=float(j["hbm_gbs"]), bf16=float(j["bf16_tflops"]),
                    bf16_sus=float(j.get("bf16_tflops_sustained", j["bf16_tflops"])), src="measured")
    except Exception:
        return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


_SAMPLER = r"""
import sys, time, pynvml
pynvml.nvmlInit()
h = pynvml.nvmlDeviceGetHandleByIndex(int(sys.argv[1]))
print("max", pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM), flush=True)
while True:
    try:
        print(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM),
              pynvml.nvmlDeviceGetCurrentClocksEventReasons(h), flush=True)
    except Exception:
        pass
    time.sleep(float(sys.argv[2]))
"""


class ClockSampler:
    """Samples SM clock and clock-event reasons with NVML (read-only queries) from a
    separate process while the timed region runs."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, index, period=0.002):
        self.index, self.period = index, period
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.proc = None

    def __enter__(self):
        import subprocess
        try:
            self.proc = subprocess.Popen([sys.executable, "-c", _SAMPLER, str(self.index), str(self.period)],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            first = self.proc.stdout.readline().split()   # wait until sampling runs
            if first and first[0] == "max":
                self.max_mhz = int(first[1])
        except Exception as e:  # sampling is best effort; the line says so
            log(f"clock sampling unavailable: {e}")
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(3 * self.period)
            self.proc.terminate()
            out, _ = self.proc.communicate(timeout=10)
            for line in out.splitlines():
                f = line.split()
                if len(f) == 2:
                    self.samples.append(int(f[0]))
                    mask = int(f[1])
                    for bit, name in self.REASONS.items():
                        if mask & bit:
                            self.reasons.add(name)
        return False

    def summary(self):
        med = statistics.median(self.samples) if self.samples else None
        return {"sm_mhz": med, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples), "source": "nvml, separate process"}


# ------------------------------------------------------------------ our arm

def dist_setup(n_gpus):
    import torch
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    import torch
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()


def max_over_ranks(x, world, device="cuda"):
    """Max of a per-rank scalar (a timed region) over all ranks of the process group."""
    import torch
    if world == 1:
        return float(x)
    import torch.distributed as dist
    t = torch.tensor([float(x)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(base_seed, rank):
    """Every rank draws its own batch (weak scaling: independent sequences per rank)."""
    return base_seed + 7919 * rank


def job_throughput(tokens_per_rank_step, steps, world, max_ms):
    """Whole-job tokens/s: all ranks' tokens over the slowest rank's timed region."""
    return world * tokens_per_rank_step * steps / (max_ms / 1e3)


def make_ring(inp, n_sets, device):
    """n_sets device copies of the layer inputs (distinct buffers, same values) plus
    per-set y buffers and states, so consecutive steps touch > L2 bytes."""
    import torch
    from selective_state_space_53_b200 import m3
    sets = []
    for _ in range(n_sets):
        dev = m3.to_device(inp, device)
        dims = m3.dims_of(inp)
        st, keep = m3.state_tensors(dims, device=device)
        y = torch.empty_like(dev["x"])
        sets.append(dict(dev=dev, state=st, keep=keep, y=y))
    return sets


def token_slice(dev, t):
    seq = ("x", "dt", "A", "lam", "B", "C", "theta")
    return {k: (v[:, t].contiguous() if (v is not None and k in seq) else v) for k, v in dev.items()}


def _prefill_record(name, cfg, ms, peaks):
    """Throughput and roofline fractions of one m3_scan_fwd of `cfg` that took `ms`."""
    by = prefill_bytes(cfg)
    fl, fl_intra = prefill_flops(cfg)
    sec = ms * 1e-3
    return {
        "workload": "%s m3_scan_fwd b%d L%d H%d P%d N%d R%d" % (name, cfg["b"], cfg["L"], cfg["H"], cfg["P"],
                                                              cfg["N"], cfg["R"]),
        "tokens_per_s": cfg["b"] * cfg["L"] / sec, "ms_per_launch": ms,
        "tflops": fl / sec / 1e12,
        "tensor_frac_of_measured_burst": fl / sec / 1e12 / peaks["bf16"],
        "tensor_frac_of_measured_sustained": fl / sec / 1e12 / peaks["bf16_sus"],
        "intra_chunk_tflops": fl_intra / sec / 1e12,
        "intra_chunk_frac_of_measured_burst": fl_intra / sec / 1e12 / peaks["bf16"],
        "intra_chunk_frac_of_measured_sustained": fl_intra / sec / 1e12 / peaks["bf16_sus"],
        "hbm_gbs": by / sec / 1e9, "hbm_frac_of_measured": by / sec / 1e9 / peaks["hbm"],
        "algorithmic_bytes": by, "algorithmic_flops": fl,
    }


def run_ours(args):
    import numpy as np
    import torch
    from selective_state_space_53_b200 import m3
    from selective_state_space_53_b200.inputs import CONFIGS, SEEDS, config_inputs

    rank, world, local = dist_setup(args.gpus)
    device = f"cuda:{local}"
    peaks = measured_peaks()
    cfg = dict(CONFIGS[WORKLOAD])
    log(f"drawing the {WORKLOAD} inputs")
    inp = config_inputs(WORKLOAD, seed=rank_seed(SEEDS[WORKLOAD], rank))
    dims = m3.dims_of(inp)
    dims1 = m3.dims_of(inp, L=1)
    per_set = prefill_bytes(cfg)
    n_sets = max(2, -(-3 * L2_BYTES // per_set))
    ring = make_ring(inp, n_sets, device)
    # the decode token of each set: a fresh draw's first token
    tok_inp = config_inputs(WORKLOAD, seed=rank_seed(SEEDS[WORKLOAD] + 100, rank), L=1)
    tok_dev = token_slice(m3.to_device(tok_inp, device), 0)
    for s in ring:
        s["state1"] = m3.State.wrap(dims1, *s["keep"])
        s["y1"] = torch.empty_like(tok_dev["x"])
    ws_bytes = m3.m3_scan_workspace_size(dims)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=device)  # steps run in stream order
    stream = torch.cuda.current_stream()

    def step(i, ev=None):
        s = ring[i % n_sets]
        if ev is not None:
            ev[0].record(stream)
        m3.scan(dims, s["dev"], s["state"], y=s["y"], workspace=ws)
        if ev is not None:
            ev[1].record(stream)
        m3.decode(dims1, tok_dev, s["state1"], y=s["y1"])

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    assert m3.m3_check() == 0

    # ---- timed region: K steps, events per prefill launch for the roofline
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier(world)
        t0.record(stream)
        for i in range(args.steps):
            step(args.warmup + i, evs[i])
        t1.record(stream)
        barrier(world)
    assert m3.m3_check() == 0
    ms_local = t0.elapsed_time(t1)
    ms = max_over_ranks(ms_local, world)
    prefill_ms = [a.elapsed_time(b) for a, b in evs]
    tokens_step = cfg["b"] * (cfg["L"] + 1)
    value = job_throughput(tokens_step, args.steps, world, ms)
    gpu_launches = (3 if ws_bytes > 0 else 2) * args.steps  # [state pass] + full pass + decode

    pf_ms = statistics.mean(prefill_ms)
    prefill = _prefill_record(WORKLOAD, cfg, pf_ms, peaks)
    prefill["ms_per_launch_min_max"] = [min(prefill_ms), max(prefill_ms)]
    alg_r, alg_w = prefill_bytes_rw(cfg)
    traffic = None
    if PREFILL_DRAM is not None:
        traffic = PREFILL_DRAM["read"] + PREFILL_DRAM["write"]
    roofline = {
        "kernel": "m3_scan_fwd (scan_ws_kernel: state pass + full pass)",
        "bound": "tensor",
        "achieved": prefill["tflops"],
        "peak": peaks["bf16"],
        "unit": "TFLOP/s",
        "frac": prefill["tensor_frac_of_measured_burst"],
        "traffic": traffic,
        "traffic_read": None if PREFILL_DRAM is None else PREFILL_DRAM["read"],
        "traffic_write": None if PREFILL_DRAM is None else PREFILL_DRAM["write"],
        "traffic_note": None if PREFILL_DRAM is None else PREFILL_DRAM["note"],
        "algorithmic_read": alg_r, "algorithmic_write": alg_w,
        "peak_source": "measured (MEASURED_PEAKS.json, bf16 burst)" if peaks["src"] == "measured" else "fallback",
        "frac_of_sustained": prefill["tensor_frac_of_measured_sustained"],
        "intra_chunk_frac": prefill["intra_chunk_frac_of_measured_burst"],
        "intra_chunk_frac_of_sustained": prefill["intra_chunk_frac_of_measured_sustained"],
        "other_bound_frac": prefill["hbm_frac_of_measured"],
    }
    # the oracle comparison: one more call on set 0 from a zero state (the timed steps continue
    # each set's state from the step before)
    s0 = ring[0]
    for t in s0["keep"]:
        t.zero_()
    m3.scan(dims, s0["dev"], s0["state"], y=s0["y"], workspace=ws)
    torch.cuda.synchronize()
    assert m3.m3_check() == 0
    y_sample = s0["y"]

    decode = run_decode(args, device, peaks) if not args.no_decode else None
    if decode is not None and not args.no_decode_sweep:
        # the rest of the decode batch sweep of the 1.5B-scale layer, one line each
        decode["sweep"] = {}
        for nm in ("decode_b1", "decode_b16", "decode_b512", "decode_p1_b128"):
            r = run_decode(args, device, peaks, nm)
            decode["sweep"][nm] = {k: r[k] for k in ("us_per_step", "tokens_per_s", "hbm_gbs", "hbm_frac_of_measured")}
            torch.cuda.empty_cache()
    if not args.no_prefill_sweep:
        prefill[EXTRA_PREFILL] = run_prefill_one(args, device, peaks, EXTRA_PREFILL)
        prefill["sweep_l15b"] = run_prefill_sweep(args, device, peaks)
    stack = run_stack(args, device, peaks) if not args.no_stack else None
    backward = run_backward(args, device) if not args.no_backward else None
    e2e = run_e2e(args, inp, tok_inp, device, world) if not args.no_e2e else None
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded; shapes of the 1.5B-scale layer)",
        "config": {"workload": f"{WORKLOAD}: m3_scan_fwd over b{cfg['b']} x L{cfg['L']} (H{cfg['H']} P{cfg['P']} "
                               f"N{cfg['N']} R{cfg['R']}, chunk 32) + 1 m3_decode_step",
                   "global_batch": cfg["b"] * world, "seq_len": cfg["L"], "parallelism": f"dp{world}",
                   "l2": f"{n_sets} input sets of {per_set / 2**20:.0f} MiB each (> L2), alternating"},
        "roofline": roofline, "prefill": prefill, "decode": decode, "stack": stack, "backward": backward, "e2e": e2e,
        "gpu_launches": gpu_launches, "clocks": clk.summary(),
    }
    if rank == 0 and not args.no_cpu:
        line["cpu_baseline"] = cpu_baseline(cfg, inp, y_sample, seconds=args.cpu_seconds)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_prefill_one(args, device, peaks, name, calls=5):
    """m3_scan_fwd alone on workload `name`: mean of `calls` calls after 2 warm-up calls, each on
    its own copy of the inputs when one copy fits in L2."""
    import torch
    from selective_state_space_53_b200 import m3
    from selective_state_space_53_b200.inputs import CONFIGS, config_inputs
    cfg = dict(CONFIGS[name])
    inp = config_inputs(name)
    dims = m3.dims_of(inp)
    per_set = prefill_bytes(cfg)
    n_sets = max(1, -(-2 * L2_BYTES // per_set))
    ring = make_ring(inp, n_sets, device)
    ws_bytes = m3.m3_scan_workspace_size(dims)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()
    for i in range(2):
        s = ring[i % n_sets]
        m3.scan(dims, s["dev"], s["state"], y=s["y"], workspace=ws)
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(calls)]
    for i, (a, b) in enumerate(evs):
        s = ring[i % n_sets]
        a.record(stream)
        m3.scan(dims, s["dev"], s["state"], y=s["y"], workspace=ws)
        b.record(stream)
    torch.cuda.synchronize()
    assert m3.m3_check() == 0
    ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
    out = _prefill_record(name, cfg, ms, peaks)
    out["input_sets"] = n_sets
    del ring, ws
    torch.cuda.empty_cache()
    return out


def run_prefill_sweep(args, device, peaks):
    """m3_scan_fwd on the 1.5B-scale layer (b2, H32 P128 N128 R4) at seqlen 2K and 8K (32K is the
    headline workload)."""
    return {name: run_prefill_one(args, device, peaks, name) for name in ("l15b_2k", "l15b_8k")}


def run_decode(args, device, peaks, name=DECODE_WORKLOAD):
    """m3_decode_step on the 1.5B-scale layer (batch 128 by default: state 256 MiB > L2)."""
    import torch
    from selective_state_space_53_b200 import m3
    from selective_state_space_53_b200.inputs import CONFIGS, SEEDS, make_inputs, make_state
    cfg = dict(CONFIGS[name])
    steps = args.decode_steps
    cfg_draw = dict(cfg, L=min(steps, 16))
    inp = make_inputs(seed=SEEDS[name], **cfg_draw)
    dims1 = m3.dims_of(inp, L=1)
    h, cB, cx = make_state(cfg["b"], cfg["H"], cfg["P"], cfg["N"], cfg["R"], seed=7, scale=0.1)
    # a ring of independent states when one state fits twice in L2 (batch 1 and 16), so that
    # every step reads and writes its state in HBM
    state_bytes = 2 * cfg["b"] * cfg["H"] * (cfg["N"] * cfg["P"] + cfg["R"] * cfg["N"] + cfg["P"]) * 4
    n_states = max(1, -(-2 * L2_BYTES // state_bytes))
    states = []
    for _ in range(n_states):
        st, keep = m3.state_tensors(dims1, device=device, h=h, carry_B=cB, carry_x=cx)
        states.append((st, keep))
    dev = m3.to_device(inp, device)
    toks = [token_slice(dev, t) for t in range(cfg_draw["L"])]
    y = torch.empty_like(toks[0]["x"])
    stream = torch.cuda.current_stream()
    for i in range(3):
        m3.decode(dims1, toks[i % len(toks)], states[i % n_states][0], y=y)
    torch.cuda.synchronize()
    # capture the steps in a CUDA graph: launch overhead out of the per-token time
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(steps):
            m3.decode(dims1, toks[i % len(toks)], states[i % n_states][0], y=y)
    g.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    g.replay()
    b.record(stream)
    torch.cuda.synchronize()
    assert m3.m3_check() == 0
    ms = a.elapsed_time(b) / steps
    by = decode_bytes(cfg)
    fl = decode_flops(cfg)
    del g
    return {"workload": "%s: m3_decode_step, b%d H%d P%d N%d R%d, CUDA graph of %d steps over %d state(s) "
                        "(%.0f MiB)" % (name, cfg["b"], cfg["H"], cfg["P"], cfg["N"], cfg["R"], steps, n_states,
                                        n_states * state_bytes / 2 / 2**20),
            "tokens_per_s": cfg["b"] / (ms * 1e-3), "us_per_step": ms * 1e3,
            "hbm_gbs": by / (ms * 1e-3) / 1e9, "hbm_frac_of_measured": by / (ms * 1e-3) / 1e9 / peaks["hbm"],
            "tflops": fl / (ms * 1e-3) / 1e12, "algorithmic_bytes": by}


def run_backward(args, device, names=("p1_layer", "l15b_2k"), calls=2):
    """m3_scan_bwd (every gradient) on the page-1 layer and the 1.5B-scale layer at 2K tokens: the
    mean of `calls` calls after one warm-up call, gradient and workspace buffers allocated once."""
    import torch
    from selective_state_space_53_b200 import m3
    from selective_state_space_53_b200.inputs import CONFIGS, config_inputs
    out = {}
    for name in names:
        cfg = dict(CONFIGS[name])
        inp = config_inputs(name)
        dims = m3.dims_of(inp)
        dev = m3.to_device(inp, device)
        st, keep = m3.state_tensors(dims, device=device)
        g = torch.Generator(device="cpu").manual_seed(31)
        dy = torch.randn(dev["x"].shape, generator=g).to(dev["x"].dtype).to(device)
        m3.scan_backward(dims, dev, st, dy)
        torch.cuda.synchronize()
        stream = torch.cuda.current_stream()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(calls):
            m3.scan_backward(dims, dev, st, dy)
        b.record(stream)
        torch.cuda.synchronize()
        assert m3.m3_check() == 0
        ms = a.elapsed_time(b) / calls
        out[name] = {"workload": "%s: m3_scan_bwd b%d L%d H%d P%d N%d R%d, every gradient" %
                                 (name, cfg["b"], cfg["L"], cfg["H"], cfg["P"], cfg["N"], cfg["R"]),
                     "ms_per_call": ms, "tokens_per_s": cfg["b"] * cfg["L"] / (ms * 1e-3),
                     "note": "token-sequential SIMT kernel with checkpointed recomputation (one to four "
                             "blocks per (batch, head), each owning a slice of the columns); includes allocation "
                             "of the gradient buffers and workspace"}
        del dev, st, keep, dy
        torch.cuda.empty_cache()
    return out


def run_stack(args, device, peaks):
    """The 12-layer stack of the page-1 language-model shape (b8 L4096): the whole forward
    (torch projections around the libm3 core) and its 12 core calls alone."""
    import torch
    from selective_state_space_53_b200 import m3
    from selective_state_space_53_b200.inputs import CONFIGS
    from selective_state_space_53_b200.stack import Mamba3Stack, StackShape
    cfg = dict(CONFIGS["p1_stack"])
    shape = StackShape(layers=cfg["layers"], H=cfg["H"], P=cfg["P"], N=cfg["N"], R=cfg["R"], G=cfg["G"])
    b, L = cfg["b"], cfg["L"]
    stack = Mamba3Stack(shape, seed=1002, device=device)
    gen = torch.Generator(device="cpu").manual_seed(2002)
    u = torch.randn(b, L, shape.d_model, generator=gen).to(torch.bfloat16).to(device)
    stream = torch.cuda.current_stream()
    # core operands of every layer, for timing the core calls alone
    dims = stack.dims(b, L)
    ws = torch.empty(max(m3.m3_scan_workspace_size(dims), 16), dtype=torch.uint8, device=device)
    ops = [stack.core_inputs(u, layer)[0] for layer in stack.layers]
    st, keep = m3.state_tensors(dims, device=device)
    y = torch.empty_like(ops[0]["x"])
    for _ in range(2):
        stack.forward(u)
        for dev in ops:
            m3.scan(dims, dev, st, y=y, workspace=ws)
    torch.cuda.synchronize()
    iters = 3
    a, c = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(iters):
        stack.forward(u)
    c.record(stream)
    torch.cuda.synchronize()
    fwd_ms = a.elapsed_time(c) / iters
    a.record(stream)
    for _ in range(iters):
        for dev in ops:
            m3.scan(dims, dev, st, y=y, workspace=ws)
    c.record(stream)
    torch.cuda.synchronize()
    assert m3.m3_check() == 0
    core_ms = a.elapsed_time(c) / iters
    layer_cfg = dict(cfg, dtype="bf16")
    by = shape.layers * prefill_bytes(layer_cfg)
    return {"workload": "p1_stack: 12 layers x (b8 L4096, H24 P64 N64 R2), forward prefill; torch projections "
                        "around the libm3 core, which applies the front-end to the raw projections",
            "tokens_per_s": b * L / (fwd_ms * 1e-3), "ms_per_forward": fwd_ms,
            "core_tokens_per_s": b * L / (core_ms * 1e-3), "core_ms_per_forward": core_ms,
            "core_hbm_frac_of_measured": by / (core_ms * 1e-3) / 1e9 / peaks["hbm"]}


def run_e2e(args, inp, tok_inp, device, world):
    """Same step through the C ABI from pinned host buffers: H2D of the step's inputs,
    prefill + decode, D2H of y (prefill and decode outputs).  Steps are pipelined over two
    buffer sets and three streams (copy in, compute, copy out), ordered by events: step i's
    inputs go in while step i-1 computes and step i-2's outputs come back.  Every step's copies
    lie inside the timed region."""
    import torch
    from selective_state_space_53_b200 import m3
    host = {}
    for k in ("x", "dt", "A", "lam", "B", "C", "theta", "bias_B", "bias_C", "W_x", "W_o", "D"):
        a = getattr(inp, k)
        if a is None:
            host[k] = None
            continue
        t = torch.from_numpy(a)
        if k in ("x", "B", "C"):
            t = t.to(torch.bfloat16)
        host[k] = t.pin_memory()
    htok = {}
    for k in ("x", "dt", "A", "lam", "B", "C", "theta"):
        t = torch.from_numpy(getattr(tok_inp, k)[:, 0].copy())
        if k in ("x", "B", "C"):
            t = t.to(torch.bfloat16)
        htok[k] = t.pin_memory()
    dims = m3.dims_of(inp)
    dims1 = m3.dims_of(inp, L=1)
    st, keep = m3.state_tensors(dims, device=device)
    st1 = m3.State.wrap(dims1, *keep)
    ws = torch.empty(max(m3.m3_scan_workspace_size(dims), 16), dtype=torch.uint8, device=device)
    bufs = []
    for _ in range(2):
        dev = {k: (None if v is None else torch.empty_like(v, device=device)) for k, v in host.items()}
        dtok = {k: torch.empty_like(v, device=device) for k, v in htok.items()}
        for k in ("bias_B", "bias_C", "W_x", "W_o", "D"):
            dtok[k] = dev[k]
        y = torch.empty_like(dev["x"])
        y1 = torch.empty_like(dtok["x"])
        bufs.append(dict(dev=dev, dtok=dtok, y=y, y1=y1,
                         y_host=torch.empty_like(y, device="cpu").pin_memory(),
                         y1_host=torch.empty_like(y1, device="cpu").pin_memory(),
                         h2d=torch.cuda.Event(), comp=torch.cuda.Event(), d2h=torch.cuda.Event(), used=False))
    h2d = sum(v.numel() * v.element_size() for v in host.values() if v is not None) + \
        sum(v.numel() * v.element_size() for v in htok.values())
    d2h = bufs[0]["y"].numel() * bufs[0]["y"].element_size() + bufs[0]["y1"].numel() * bufs[0]["y1"].element_size()
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(device=device), torch.cuda.Stream(device=device)

    def step(i):
        bf = bufs[i % 2]
        with torch.cuda.stream(s_in):
            if bf["used"]:
                s_in.wait_event(bf["comp"])  # step i-2 has consumed this buffer's inputs
            for k, v in host.items():
                if v is not None:
                    bf["dev"][k].copy_(v, non_blocking=True)
            for k, v in htok.items():
                bf["dtok"][k].copy_(v, non_blocking=True)
            bf["h2d"].record(s_in)
        comp.wait_event(bf["h2d"])
        if bf["used"]:
            comp.wait_event(bf["d2h"])  # step i-2's outputs have left this buffer
        m3.scan(dims, bf["dev"], st, y=bf["y"], workspace=ws)
        m3.decode(dims1, bf["dtok"], st1, y=bf["y1"])
        bf["comp"].record(comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(bf["comp"])
            bf["y_host"].copy_(bf["y"], non_blocking=True)
            bf["y1_host"].copy_(bf["y1"], non_blocking=True)
            bf["d2h"].record(s_out)
        bf["used"] = True

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    n = max(1, min(args.steps, 30))
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    a.record(comp)
    s_in.wait_stream(comp)
    s_out.wait_stream(comp)
    for i in range(n):
        step(args.warmup + i)
    comp.wait_stream(s_in)
    comp.wait_stream(s_out)
    b.record(comp)
    barrier(world)
    ms = max_over_ranks(a.elapsed_time(b), world) / n
    tokens = inp.dims["b"] * (inp.dims["L"] + 1)
    return {"value": world * tokens / (ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": ms, "steps": n,
            "pipelining": "2 buffer sets; copy-in, compute and copy-out streams ordered by events"}


# ------------------------------------------------------------------ fp64 oracle (CPU)

def _prefix(inp, Lp):
    """The first Lp tokens of every sequence of a draw (the recurrence is causal, so the
    oracle's outputs on them are the full run's first Lp outputs)."""
    import copy
    sub = copy.copy(inp)
    for k in ("x", "dt", "A", "lam", "B", "C", "theta"):
        setattr(sub, k, getattr(inp, k)[:, :Lp])
    sub.dims = dict(inp.dims, L=Lp)
    return sub


def _oracle_time(inp, pairs, threads=0):
    """(seconds, y) of the oracle on the (batch, head) pairs of a draw."""
    from oracle import oracle as orc
    t = time.perf_counter()
    y, _, _, _ = orc.scan_inputs(inp, sel=pairs, threads=threads)
    return time.perf_counter() - t, y


def _sample_len(inp, pairs, seconds, probe_len=64):
    """Prefix length whose oracle run over `pairs` takes about `seconds`."""
    t, _ = _oracle_time(_prefix(inp, probe_len), pairs)
    per_tok = t / probe_len
    Lp = int(seconds / max(per_tok, 1e-9))
    return max(probe_len, min(inp.dims["L"], (Lp // 64) * 64))


def cpu_baseline(cfg, inp, y_gpu, seconds=12.0):
    """The fp64 oracle as it stands, OpenMP over (batch, head) on all host cores, on a bounded
    sample: every (batch, head) sequence of the layer over a prefix of the tokens, sized to take
    about `seconds`.  tokens/s counts layer tokens (a layer token needs all H heads).  The same
    sample checks the GPU: its y on those tokens against the oracle's (max relative error and
    elementwise error, the bf16 tolerance 2e-2)."""
    import numpy as np
    from oracle import oracle as orc
    H, b = cfg["H"], cfg["b"]
    allp = [(bi, hi) for bi in range(b) for hi in range(H)]
    cores = orc.max_threads()
    Lp = _sample_len(inp, allp, seconds)
    sub = _prefix(inp, Lp)
    t, yr = _oracle_time(sub, allp)
    yg = y_gpu[:, :Lp].float().cpu().numpy().astype(np.float64)
    err = float(np.abs(yg - yr).max() / max(np.abs(yr).max(), 1e-300))
    floor = 1e-3 * np.abs(yr).max()
    elem = float((np.abs(yg - yr) / np.maximum(np.abs(yr), floor)).max())
    return {"value": len(allp) * Lp / H / t, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"all {len(allp)} (batch, head) sequences of {WORKLOAD} over their first {Lp} of "
                      f"{cfg['L']} tokens ({t:.1f} s); tokens/s counts layer tokens (all {H} heads)",
            "seconds": t,
            "parity": {"y_max_rel_err": err, "y_elementwise_rel_err": elem, "tolerance": 2e-2,
                       "tokens": Lp, "sequences": len(allp),
                       "metric": "max|gpu - oracle| / max|oracle| over the sample; elementwise: "
                                 "|gpu - oracle| / max(|oracle|, 1e-3 max|oracle|)"}}


def run_reference(args):
    """Reference arm: the fp64 oracle on the host cores, on the same workload and metric."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from oracle import oracle as orc
    from selective_state_space_53_b200.inputs import CONFIGS, SEEDS, make_inputs
    cfg = dict(CONFIGS[WORKLOAD])
    H, b = cfg["H"], cfg["b"]
    cores = orc.max_threads()
    allp = [(bi, hi) for bi in range(b) for hi in range(H)]
    # each step: every (batch, head) sequence over a prefix of the tokens, sized so that the
    # whole run takes about three minutes; the draw has the workload's shapes and seed
    Lmax = 4096
    draw = dict(cfg, L=Lmax)
    draw.pop("layers", None)
    inp = make_inputs(seed=SEEDS[WORKLOAD], **draw)
    per_step = 180.0 / max(1, args.steps + args.warmup)
    Lp = _sample_len(inp, allp, per_step)
    sub = _prefix(inp, Lp)
    for i in range(args.warmup):
        _oracle_time(sub, allp)
    t = 0.0
    for i in range(args.steps):
        t += _oracle_time(sub, allp)[0]
    layer_tokens_per_step = len(allp) * Lp / H
    value = layer_tokens_per_step * args.steps / t
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded; shapes of the 1.5B-scale layer)",
        "config": {"workload": f"{WORKLOAD}: m3_scan_fwd over b{cfg['b']} x L{cfg['L']} (H{cfg['H']} P{cfg['P']} "
                               f"N{cfg['N']} R{cfg['R']}, chunk 32) + 1 m3_decode_step",
                   "global_batch": b, "seq_len": cfg["L"], "parallelism": "host cores"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"each step: all {len(allp)} (batch, head) sequences over their first {Lp} "
                                   f"tokens; tokens/s counts layer tokens (all {H} heads)"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--decode-steps", type=int, default=1024)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu", action="store_true", help="skip the oracle timing")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-decode-sweep", action="store_true", help="decode at batch 128 only")
    ap.add_argument("--no-prefill-sweep", action="store_true", help="skip the 1.5B-scale layer prefill sweep")
    ap.add_argument("--no-stack", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-backward", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
