"""Run fused linear cross-entropy on one seeded case, for profiling and timing.

    python -m linear_cross_entropy_04_b200.run_case --BT 4096 --H 4096 --V 32768 \\
        [--chunk-rows 2048] [--calls 1] [--workload llama3_8b_seq] [--time]

Inputs follow the named workload's recipe (distribution, ignore fraction,
seed) at the given sizes. Every call runs the whole path once. Used as the
command under ncu (small cases) and for quick per-shape timings.
"""
import argparse
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="llama3_8b_seq")
    ap.add_argument("--BT", type=int)
    ap.add_argument("--H", type=int)
    ap.add_argument("--V", type=int)
    ap.add_argument("--chunk-rows", type=int, default=0)
    ap.add_argument("--grad-w-accum", default="output")
    ap.add_argument("--calls", type=int, default=1)
    ap.add_argument("--no-grad-x", action="store_true")
    ap.add_argument("--no-grad-w", action="store_true")
    ap.add_argument("--time", action="store_true", help="time the calls with CUDA events and phases")
    a = ap.parse_args()

    import torch

    import linear_cross_entropy_04_b200 as flce
    from linear_cross_entropy_04_b200 import _binding as B
    from linear_cross_entropy_04_b200.inputs import WORKLOADS, make_inputs

    w = WORKLOADS[a.workload]
    d = make_inputs(w, BT=a.BT, H=a.H, V=a.V)
    dt = torch.bfloat16 if d["dtype"] == "bf16" else torch.float32
    X = torch.from_numpy(d["X"]).to(dt).cuda()
    W = torch.from_numpy(d["W"]).to(dt).cuda()
    t = torch.from_numpy(d["target"]).cuda()
    out = (torch.empty((), device="cuda"), None if a.no_grad_x else torch.empty_like(X),
           None if a.no_grad_w else torch.empty_like(W))
    kw = dict(chunk_rows=a.chunk_rows, grad_w_accum=a.grad_w_accum, out=out, return_stats=True,
              want_grad_X=not a.no_grad_x, want_grad_W=not a.no_grad_w)
    if a.time:
        for _ in range(2):
            flce.fused_linear_cross_entropy(X, W, t, **kw)
        torch.cuda.synchronize()
        flce.phase_times(reset=True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(a.calls):
        st = flce.fused_linear_cross_entropy(X, W, t, flags=B.FLAG_TIME_PHASES if a.time else 0, **kw)[3]
    e1.record()
    torch.cuda.synchronize()
    err = flce.device_error()
    res = {"BT": d["BT"], "H": d["H"], "V": d["V"], "stats": st, "device_error": err,
           "ms_per_call": e0.elapsed_time(e1) / a.calls}
    if a.time:
        res["phases_ms_per_call"] = {k: v[0] / a.calls for k, v in flce.phase_times(reset=True).items()}
        res["tflops"] = 6.0 * d["BT"] * d["H"] * d["V"] / (res["ms_per_call"] / 1e3) / 1e12
    print(json.dumps(res))
    return 1 if err else 0


if __name__ == "__main__":
    sys.exit(main())
