"""Run one entry point of libm3 on a named workload a few times, for profilers.

    python -m selective_state_space_53_b200.run_case --workload l15b_8k --op scan --calls 3
    python -m selective_state_space_53_b200.run_case --workload decode_b1 --op decode --calls 8

The inputs are the seeded draw of the workload (``inputs.config_inputs``), uploaded once;
each call runs through the C ABI on the current stream, and the library's error flag is
checked at the end.  ``--L`` (and ``--b --H --P --N --R``, ``--dtype``) override the workload's sizes and storage type
(a smaller capture of the same kernel, or another kernel's shape);
``--raw`` passes the draw as raw projections (M3_FLAG_RAW_INPUTS).  Prints one line with the
mean time of the calls (CUDA events; not a bench figure under a profiler).
"""

from __future__ import annotations

import argparse
import json


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="l15b_8k")
    ap.add_argument("--op", choices=["scan", "decode", "bwd"], default="scan")
    ap.add_argument("--calls", type=int, default=3)
    ap.add_argument("--L", type=int, default=0, help="sequence length override")
    for k in ("b", "H", "P", "N", "R"):
        ap.add_argument("--" + k, type=int, default=0, help=f"{k} override")
    ap.add_argument("--dtype", choices=["bf16", "f32"], default=None, help="storage dtype override")
    ap.add_argument("--raw", action="store_true")
    args = ap.parse_args()

    import torch
    from . import m3
    from .inputs import CONFIGS, SEEDS, make_inputs, make_raw_inputs

    cfg = dict(CONFIGS[args.workload])
    cfg.pop("layers", None)
    for k in ("L", "b", "H", "P", "N", "R"):
        if getattr(args, k):
            cfg[k] = getattr(args, k)
    if args.dtype:
        cfg["dtype"] = args.dtype
    seed = SEEDS.get(args.workload, 0)
    if args.raw:
        inp = make_raw_inputs(seed=seed, **cfg)
    else:
        inp = make_inputs(seed=seed, **cfg)
    flags = m3.M3_FLAG_RAW_INPUTS if args.raw else 0
    dev = m3.to_device(inp, "cuda")
    stream = torch.cuda.current_stream()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]

    if args.op == "scan":
        dims = m3.dims_of(inp, flags=flags)
        st, keep = m3.state_tensors(dims, device="cuda")
        ws = torch.empty(max(m3.m3_scan_workspace_size(dims), 16), dtype=torch.uint8, device="cuda")
        y = torch.empty_like(dev["x"])

        def call():
            m3.scan(dims, dev, st, y=y, workspace=ws)
        units = cfg["b"] * cfg["L"]
    elif args.op == "decode":
        dims = m3.dims_of(inp, L=1, flags=flags)
        st, keep = m3.state_tensors(dims, device="cuda")
        seq = ("x", "dt", "A", "lam", "theta", "B", "C")
        tok = {k: (v[:, 0].contiguous() if (v is not None and k in seq) else v) for k, v in dev.items()}
        y = torch.empty_like(tok["x"])

        def call():
            m3.decode(dims, tok, st, y=y)
        units = cfg["b"]
    else:
        dims = m3.dims_of(inp, flags=flags)
        st, keep = m3.state_tensors(dims, device="cuda")
        dy = torch.randn(dev["x"].shape, generator=torch.Generator().manual_seed(seed + 1)).to(dev["x"].dtype).cuda()

        def call():
            m3.scan_backward(dims, dev, st, dy)
        units = cfg["b"] * cfg["L"]

    call()
    torch.cuda.synchronize()
    ev[0].record(stream)
    for _ in range(args.calls):
        call()
    ev[1].record(stream)
    torch.cuda.synchronize()
    rc = m3.m3_check()
    if rc != 0:
        raise SystemExit(f"m3_check reported {rc}")
    ms = ev[0].elapsed_time(ev[1]) / args.calls
    print(json.dumps({"workload": args.workload, "op": args.op, "L": cfg["L"], "raw": args.raw,
                      "calls": args.calls, "ms_per_call": ms, "units_per_s": units / (ms * 1e-3)}))


if __name__ == "__main__":
    main()
