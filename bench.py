"""Benchmark: fused linear cross-entropy forward + backward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one full pass of the path (count, logits GEMM + online softmax,
row combine, in-place dlogits, grad_X/grad_W GEMMs, loss) over one batch of
synthetic tokens of the named workload (default: Llama-3-8B lm_head, BT=4096,
H=4096, V=128256, bf16). Inputs stay resident in HBM; W alone (1.05 GB) is
larger than the 126 MB L2, so no L2 flush is needed between steps.

With N > 1 (torchrun), every rank runs its own batch (weak scaling) with a
replica of W, and the step adds the data-parallel exchange: an all-reduce of
the non-ignored row count before the loss, then of the loss, then grad_W
summed over ranks (below). --dp takes that path, collectives included, on one
rank too.

--impl reference times the float64 CPU oracle on bounded samples of the same
workload (rank 0 only); it is the slow baseline the pages' method is exact to.

Other paths (one GPU, their own JSON lines):
  --path ce                 logits-given cross-entropy vs torch cross_entropy + backward
  --path preference --kind  a fused-linear preference-loss step vs PyTorch on materialised logits
With N > 1 grad_W is reduce-scattered by rows after the step (NCCL; each rank keeps
V/N rows, the sharded-gradient setting of the pages' FSDP benchmark);
--grad-w-exchange all_reduce gives every rank all of it, and --grad-w-exchange fused
(or --dp-fused-grad-w) lets the grad_W GEMM's epilogue add each tile into the owner
rank's symmetric-memory shard over NVLink.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "FLCE fwd+bwd tokens/sec and TFLOP/s (% of B200 bf16 peak), peak workspace"
UNIT = "tokens/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="llama3_8b_seq")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=24,
                    help="host-buffer steps timed end to end (the pipeline's fill and drain are included)")
    ap.add_argument("--e2e-slots", type=int, default=2, help="device buffer sets of the host pipeline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU time of the oracle sample")
    ap.add_argument("--chunk-rows", type=int, default=0)
    ap.add_argument("--grad-w-accum", default="output", choices=["output", "fp32"])
    ap.add_argument("--schedule", default="stored", choices=["stored", "recompute"],
                    help="stored: row chunks keep their logits store (6*BT*H*V tensor FLOPs, the default); "
                         "recompute: vocabulary chunks, logits rebuilt after an lse pass (8*BT*H*V)")
    ap.add_argument("--workspace-limit-mib", type=int, default=0, help="chunk store budget (0: the library default)")
    ap.add_argument("--grad-w-exchange", default="reduce_scatter", choices=["reduce_scatter", "all_reduce", "fused"],
                    help="N > 1: how grad_W is summed over ranks. reduce_scatter (default): NCCL reduce-scatter "
                         "after the step, each rank keeps V/N rows (the sharded-gradient setting of the pages' "
                         "FSDP benchmark); all_reduce: every rank gets all of grad_W; fused: the grad_W GEMM's "
                         "epilogue adds each tile into the owner rank's shard over NVLink (symmetric memory)")
    ap.add_argument("--dp-fused-grad-w", action="store_true", help="the same as --grad-w-exchange fused")
    ap.add_argument("--dp", action="store_true",
                    help="take the data-parallel code path (collectives included) even on one rank")
    ap.add_argument("--path", default="flce", choices=["flce", "ce", "preference"],
                    help="flce: the fused lm_head + loss step (default); ce: cross-entropy of given logits; "
                         "preference: a fused-linear preference loss step (--kind)")
    ap.add_argument("--kind", default="dpo", choices=["dpo", "orpo", "cpo", "simpo", "kto"],
                    help="preference loss for --path preference")
    ap.add_argument("--seq-len", type=int, default=512, help="tokens per sequence for --path preference")
    ap.add_argument("--BT", type=int, default=0, help="profiling: cut the workload to this many tokens")
    ap.add_argument("--H", type=int, default=0, help="profiling: hidden size override")
    ap.add_argument("--V", type=int, default=0, help="profiling: vocabulary size override")
    return ap.parse_args()


EXCHANGE_NAMES = {"reduce_scatter": "NCCL reduce-scatter by rows (each rank keeps V/N rows of grad_W)",
                  "all_reduce": "NCCL all-reduce", "fused": "fused reduce-scatter in the grad_W GEMM"}


def grad_w_exchange(args, V: int, world: int):
    """How grad_W is summed over `world` ranks (None on one GPU, unless --dp).
    The row reduce-scatter needs V divisible by the world size; otherwise
    all-reduce."""
    if world <= 1 and not args.dp:
        return None
    ex = "fused" if args.dp_fused_grad_w else args.grad_w_exchange
    if ex == "reduce_scatter" and V % world:
        return "all_reduce"
    return ex


def workload(args):
    """The named workload, or the same recipe at the --BT/--H/--V sizes (small
    cases for profiling); an overridden workload is renamed after its sizes."""
    import dataclasses

    from linear_cross_entropy_04_b200.inputs import WORKLOADS

    w = WORKLOADS[args.workload]
    over = {k: getattr(args, k) for k in ("BT", "H", "V") if getattr(args, k)}
    if not over:
        return w
    w = dataclasses.replace(w, **over)
    return dataclasses.replace(w, name=f"{args.workload} recipe at {w.BT}x{w.H}x{w.V}")


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """nvidia-smi clock / throttle samples, kept only where they fall inside
    the timed region (mark_start / mark_end bracket it on the host clock)."""

    Q = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, index, period_ms=100):
        self.index = index
        self.period_ms = period_ms
        self.proc = None
        self.window = None
        fd, self.path = tempfile.mkstemp(prefix=f"flce_clocks_rank{index}_", suffix=".csv")
        os.close(fd)

    def __enter__(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", str(self.period_ms)],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def mark_start(self):
        self._t0 = time.time()

    def mark_end(self):
        self.window = (self._t0, time.time())

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    @staticmethod
    def _stamp(txt):
        import datetime

        for fmt in ("%Y/%m/%d %H:%M:%S.%f", "%Y/%m/%d %H:%M:%S"):
            try:
                return datetime.datetime.strptime(txt, fmt).timestamp()
            except ValueError:
                pass
        return None

    def summary(self):
        if not self.proc or not os.path.exists(self.path):
            if os.path.exists(self.path):
                os.unlink(self.path)
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        rows = []
        with open(self.path) as fh:
            lines = fh.readlines()
        os.unlink(self.path)
        for ln in lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 10:
                continue
            try:
                rows.append((self._stamp(f[0]), float(f[2]), float(f[3]), float(f[4]), f[6:10]))
            except ValueError:
                continue
        return self.summarize(rows, self.window, self.period_ms)

    @classmethod
    def summarize(cls, rows, window, period_ms=100):
        """rows: (unix time, sm MHz, max MHz, watts, [4 reason fields]). Samples
        inside the window are used; a window shorter than the sample period
        takes the samples within one period of it and says so."""
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        scope = "timed region"
        sel = rows
        if window is not None and all(r[0] is not None for r in rows):
            sel = [r for r in rows if window[0] <= r[0] <= window[1]]
            if not sel:
                pad = period_ms / 1e3
                sel = [r for r in rows if window[0] - pad <= r[0] <= window[1] + pad]
                scope = "within one sample period of the timed region"
            if not sel:
                return {"sm_mhz": None, "sm_max_mhz": rows[-1][2], "reasons": ["unsampled"],
                        "samples": 0, "scope": "no sample near the timed region"}
        else:
            scope = "whole run (no timestamps)"
        reasons = set()
        for r in sel:
            for n, v in zip(cls.NAMES, r[4]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(r[1] for r in sel), "sm_max_mhz": sel[-1][2],
                "reasons": sorted(reasons), "samples": len(sel), "power_w": statistics.median(r[3] for r in sel),
                "scope": scope}


# ---------------------------------------------------------------- recorded ncu traffic

# everything that decides what the captured launches do: the kernels, and the
# host code that picks their chunking, tile order and launch split
KERNEL_SOURCES = ["linear_cross_entropy_04_b200/csrc/" + f
                  for f in ("tc_gemm2.cuh", "tc_gemm.cuh", "ptx.cuh", "aux_kernels.cuh", "flce.cu")]


def code_only(text: str) -> str:
    """C/C++/CUDA source with its comments removed and whitespace collapsed (no
    string literal in these files holds a comment marker)."""
    import re

    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return " ".join(text.split())


def kernel_source_hash():
    """sha256 (first 16 hex digits) of the code of the files that decide what the
    GEMM launches do; comments and layout do not count."""
    import hashlib

    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        h.update(code_only(open(os.path.join(ROOT, f), encoding="utf-8").read()).encode())
        h.update(b"\0")
    return h.hexdigest()[:16]


def recorded_traffic(workload):
    """DRAM bytes per GEMM launch from the committed ncu summary of this
    workload, if it was taken on the current kernel source (else None)."""
    p = os.path.join(ROOT, "profiles", f"tc_gemm_pair_kernel_{workload}_dram.md")
    if not os.path.exists(p):
        return None
    vals = {}
    for ln in open(p):
        if ln.startswith("- ") and ":" in ln:
            k, v = ln[2:].split(":", 1)
            vals[k.strip()] = v.strip().strip("`")
    if vals.get("kernel_source_sha256_16") != kernel_source_hash():
        return None
    try:
        return {"bytes_per_launch": float(vals["dram_bytes_per_launch"]), "source": os.path.relpath(p, ROOT)}
    except (KeyError, ValueError):
        return None


# ---------------------------------------------------------------- CPU oracle

def oracle_sample(d, n_rows, Wf64=None):
    """Run the float64 oracle on the first n_rows tokens: the full per-token work
    (logits over V, loss, grad_X rows, their grad_W contribution). Returns seconds."""
    import numpy as np
    import oracle

    n_valid = oracle.count_valid(d["target"], d["V"])
    X = d["X"][:n_rows].astype(np.float64)
    t0 = time.perf_counter()
    oracle.flce(X, Wf64, d["target"][:n_rows], n_valid=n_valid)
    return time.perf_counter() - t0


def blas_threads():
    try:
        from threadpoolctl import threadpool_info

        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:  # noqa: BLE001
        return os.cpu_count()


def cpu_model():
    try:
        for ln in open("/proc/cpuinfo"):
            if ln.startswith("model name"):
                return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def calibrate_rows(d, Wf, target_s, cap):
    """Rows whose oracle call takes about target_s: the call has a fixed cost
    (the [V, H] float64 grad_W it allocates and fills) plus a per-row cost, so
    both are measured (8 and 40 rows) before extrapolating."""
    t8 = oracle_sample(d, 8, Wf)
    t40 = oracle_sample(d, 40, Wf)
    per_row = max((t40 - t8) / 32, 1e-6)
    fixed = max(t8 - 8 * per_row, 0.0)
    return int(min(cap, max(8, (target_s - fixed) / per_row)))


def cpu_baseline(d, target_s):
    import numpy as np

    Wf = d["W"].astype(np.float64)
    rows = calibrate_rows(d, Wf, target_s, min(4096, d["BT"]))
    t = oracle_sample(d, rows, Wf)
    return {"value": rows / t, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": f"first {rows} tokens of the workload, full fwd+bwd per token in float64 NumPy "
                      f"({t:.1f} s), on {cpu_model()}",
            "seconds": t}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import numpy as np

    from linear_cross_entropy_04_b200.inputs import WORKLOADS, make_inputs

    w = workload(args)
    d = make_inputs(w)
    Wf = d["W"].astype(np.float64)
    rows = calibrate_rows(d, Wf, 150.0 / max(1, args.steps + args.warmup), min(4096, d["BT"]))
    for _ in range(args.warmup):
        oracle_sample(d, rows, Wf)
    tot = 0.0
    for _ in range(args.steps):
        tot += oracle_sample(d, rows, Wf)
    value = rows * args.steps / tot
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": w.name, "BT": w.BT, "H": w.H, "V": w.V,
                                            "sample_tokens_per_step": rows},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                             "sample": f"each step: the first {rows} tokens, full fwd+bwd in float64 NumPy, "
                                       f"on {cpu_model()}"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- logits-given CE

def run_ce(args):
    """Cross-entropy of given logits [BT, V] (the paper review's CrossEntropy
    kernel: online softmax, gradient written over the logits) against the
    plain PyTorch cross_entropy + backward on the same bf16 logits."""
    import torch
    import torch.nn.functional as F

    import linear_cross_entropy_04_b200 as flce
    from linear_cross_entropy_04_b200.inputs import WORKLOADS, draw_targets

    import numpy as np

    w = workload(args)
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev).manual_seed(0)
    z0 = (torch.randn(w.BT, w.V, device=dev, generator=g) * 1.28).to(torch.bfloat16)
    t = torch.from_numpy(draw_targets(np.random.default_rng(0), w.BT, w.V, w.targets, w.ignore_frac)).to(dev)
    z = z0.clone()

    def ours():
        flce.cross_entropy(z, t, inplace=True)

    def torch_ce():
        zz = z0.detach().requires_grad_(True)
        F.cross_entropy(zz, t, ignore_index=-100).backward()
        return zz.grad

    res = {}
    for name, fn in (("ours", ours), ("torch", torch_ce)):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        base = torch.cuda.memory_allocated(dev)
        torch.cuda.reset_peak_memory_stats(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with ClockSampler(0) as clk:
            time.sleep(0.3)
            clk.mark_start()
            e0.record()
            for _ in range(args.steps):
                fn()
            e1.record()
            torch.cuda.synchronize()
            clk.mark_end()
        ms = e0.elapsed_time(e1) / args.steps
        res[name] = {"ms_per_step": ms, "tokens_per_s": w.BT / (ms / 1e3),
                     "peak_extra_bytes": torch.cuda.max_memory_allocated(dev) - base, "clocks": clk.summary()}
    # the library's CE workspace (taken from its own pool, invisible to torch's counters).
    # One-pass cluster kernel (bf16, V <= 16 * 32768): N and the per-row losses.
    # Multi-pass kernels: also per-row lse / target logit and per-(1024-column
    # tile, row) max and sum-exp.
    a256 = lambda n: (n + 255) // 256 * 256  # noqa: E731
    one_pass = w.dtype == "bf16" and w.V <= 16 * 32768 and os.environ.get("FLCE_CE") != "multipass"
    if one_pass:
        lib_ws = a256(8) + a256(4 * w.BT)
    else:
        ntile, ldp = -(-w.V // 1024), -(-w.BT // 32) * 32
        lib_ws = a256(8) + 3 * a256(4 * w.BT) + 2 * a256(4 * ntile * ldp)
    res["ours"]["peak_extra_bytes"] += lib_ws
    res["ours"]["library_workspace_bytes"] = lib_ws
    # algorithmic HBM bytes: read z once, write dz once (the one-pass kernel moves
    # exactly these; the multi-pass kernels read z a second time on top)
    bytes_moved = 2 * w.BT * w.V * 2
    line = {"metric": "CE (logits given) fwd+bwd tokens/s and peak extra memory", "value": res["ours"]["tokens_per_s"],
            "unit": "tokens/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": res["ours"]["ms_per_step"], "higher_is_better": True, "dtype": "bf16",
            "data": "synthetic", "config": {"workload": f"{w.name} logits", "BT": w.BT, "V": w.V},
            "speedup_vs_torch": res["torch"]["ms_per_step"] / res["ours"]["ms_per_step"],
            "kernel_path": "one-pass cluster kernel" if one_pass else "partials + combine + gradient kernels",
            "memory_ratio_torch_over_ours": res["torch"]["peak_extra_bytes"] / max(res["ours"]["peak_extra_bytes"], 1),
            "ours": res["ours"], "torch": res["torch"], "clocks": res["ours"]["clocks"],
            "roofline": {"bound": "hbm", "achieved": bytes_moved / (res["ours"]["ms_per_step"] / 1e3) / 1e9,
                         "peak": load_peaks()["hbm_gbs"], "unit": "GB/s",
                         "frac": bytes_moved / (res["ours"]["ms_per_step"] / 1e3) / 1e9 / load_peaks()["hbm_gbs"],
                         "traffic": None, "algorithmic_bytes": bytes_moved}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- preference losses

def run_preference(args):
    """One fused-linear preference-loss step (loss, grad_x, grad_weight) on the
    lm_head shapes of the workload: its BT tokens form BT / seq_len sequences
    (chosen rows first, then rejected), the first quarter of each sequence is
    prompt (ignore_index). Timed against the same loss in plain PyTorch on
    materialised logits (bf16 matmul, fp32 log-softmax, autograd)."""
    import numpy as np
    import torch

    import linear_cross_entropy_04_b200 as flce
    from linear_cross_entropy_04_b200.inputs import IGNORE_INDEX, WORKLOADS, make_inputs
    from linear_cross_entropy_04_b200.preference import fused_linear_preference_loss, preference_loss_from_logps

    w = workload(args)
    T = args.seq_len
    n_seq = w.BT // T
    assert n_seq >= 2 and n_seq % 2 == 0, "BT / seq_len must be an even number of sequences"
    d = make_inputs(w, BT=n_seq * T)
    dev = torch.device("cuda", 0)
    X = torch.from_numpy(d["X"]).to(torch.bfloat16).to(dev)
    W = torch.from_numpy(d["W"]).to(torch.bfloat16).to(dev)
    t = d["target"].reshape(n_seq, T).copy()
    t[:, : T // 4] = IGNORE_INDEX
    t = torch.from_numpy(t).to(dev)
    rng = np.random.default_rng(5)
    ref = torch.from_numpy(rng.standard_normal(n_seq) * 5.0 - 3000.0).to(dev)
    des = torch.from_numpy((np.arange(n_seq) % 2).astype(np.float64)).to(dev)
    kw = dict(ref_logps=ref) if args.kind == "dpo" else dict(desirable=des) if args.kind == "kto" else {}

    def ours():
        return fused_linear_preference_loss(args.kind, W, X, t, **kw)

    def torch_ref():
        Xr = X.detach().requires_grad_(True)
        Wr = W.detach().requires_grad_(True)
        logits = (Xr @ Wr.t()).float()
        tt = t.reshape(-1)
        valid = tt != IGNORE_INDEX
        lp_tok = torch.log_softmax(logits, -1).gather(1, tt.clamp(min=0)[:, None])[:, 0] * valid
        row_loss = -lp_tok
        lp = lp_tok.reshape(n_seq, T).double().sum(1)
        cnt = valid.reshape(n_seq, T).double().sum(1)
        nll_sum_chosen = row_loss.reshape(n_seq, T)[: n_seq // 2].double().sum()
        loss = preference_loss_from_logps(args.kind, lp, cnt, nll_sum_chosen,
                                          ref_logps=kw.get("ref_logps"), desirable=kw.get("desirable"))
        loss.backward()
        return loss, Xr.grad, Wr.grad

    res = {}
    for name, fn in (("ours", ours), ("torch", torch_ref)):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        # peak memory of one step, outputs included, with no earlier step's outputs alive
        base = torch.cuda.memory_allocated(dev)
        torch.cuda.reset_peak_memory_stats(dev)
        out = fn()
        torch.cuda.synchronize()
        peak = torch.cuda.max_memory_allocated(dev) - base
        loss_val = float(out[0])
        del out
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with ClockSampler(0) as clk:
            time.sleep(0.3)
            clk.mark_start()
            e0.record()
            for _ in range(args.steps):
                fn()
            e1.record()
            torch.cuda.synchronize()
            clk.mark_end()
        ms = e0.elapsed_time(e1) / args.steps
        res[name] = {"ms_per_step": ms, "tokens_per_s": n_seq * T / (ms / 1e3), "peak_extra_bytes": peak,
                     "loss": loss_val, "clocks": clk.summary()}
    BT = n_seq * T
    useful = 6.0 * BT * w.H * w.V
    peaks = load_peaks()
    rel = abs(res["ours"]["loss"] - res["torch"]["loss"]) / max(abs(res["torch"]["loss"]), 1e-30)
    line = {"metric": f"fused-linear {args.kind.upper()} loss fwd+bwd tokens/s", "value": res["ours"]["tokens_per_s"],
            "unit": "tokens/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": res["ours"]["ms_per_step"], "higher_is_better": True, "dtype": "bf16",
            "data": "synthetic (seeded; random-init lm_head weights; prompt quarter of each sequence ignored)",
            "config": {"workload": f"{w.name} as {n_seq} sequences of {T}", "BT": BT, "H": w.H, "V": w.V,
                       "kind": args.kind},
            "speedup_vs_torch": res["torch"]["ms_per_step"] / res["ours"]["ms_per_step"],
            "memory_ratio_torch_over_ours": res["torch"]["peak_extra_bytes"] / max(res["ours"]["peak_extra_bytes"], 1),
            "loss_rel_diff_vs_torch": rel, "ours": res["ours"], "torch": res["torch"],
            "roofline": {"bound": "tensor", "achieved": useful / (res["ours"]["ms_per_step"] / 1e3) / 1e12,
                         "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": useful / (res["ours"]["ms_per_step"] / 1e3) / 1e12 / peaks["bf16_tflops"],
                         "traffic": None, "algorithmic_flops": useful,
                         "peak_kind": f"{peaks['source']} burst bf16",
                         "frac_of_sustained_peak": useful / (res["ours"]["ms_per_step"] / 1e3) / 1e12
                         / peaks["bf16_tflops_sustained"],
                         "note": "useful 6*BT*H*V; the single-pass schedule executes exactly these, the "
                                 "two-pass one (batches whose store exceeds the keep budget) 8*BT*H*V"},
            "clocks": res["ours"]["clocks"]}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- GPU arm

def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if args.path == "ce":
        return run_ce(args)
    if args.path == "preference":
        return run_preference(args)

    import torch
    import torch.distributed as dist

    import linear_cross_entropy_04_b200 as flce
    from linear_cross_entropy_04_b200 import _binding as B
    from linear_cross_entropy_04_b200.inputs import WORKLOADS, make_inputs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dp = world > 1 or args.dp  # the data-parallel code path, collectives included
    if dp:
        import datetime

        if world == 1:
            os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
            os.environ.setdefault("MASTER_PORT", "29531")
            os.environ.setdefault("RANK", "0")
            os.environ.setdefault("WORLD_SIZE", "1")
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    w = workload(args)
    d = make_inputs(w, seed=w.seed + rank)
    dev = torch.device("cuda", local)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    X = torch.from_numpy(d["X"]).to(dt).to(dev)
    W = torch.from_numpy(d["W"]).to(dt).to(dev)
    t = torch.from_numpy(d["target"]).to(dev)
    loss = torch.empty((), dtype=torch.float32, device=dev)
    gX = torch.empty_like(X)
    gW = torch.empty_like(W)
    nvalid = torch.empty((), dtype=torch.int64, device=dev)
    kw = dict(chunk_rows=args.chunk_rows, grad_w_accum=args.grad_w_accum, schedule=args.schedule,
              workspace_limit_bytes=args.workspace_limit_mib << 20)

    from linear_cross_entropy_04_b200.dp import dp_fused_linear_cross_entropy

    exchange = grad_w_exchange(args, w.V, world)

    def step(flags=0):
        if exchange == "fused":
            # data-parallel step, grad_W reduce-scattered by the grad_W GEMM's epilogue
            dp_fused_linear_cross_entropy(X, W, t, fused_grad_W=True, flags=flags, **kw)
        elif exchange is not None:
            # data-parallel step: all-reduce N before the loss, then the loss and grad_W
            # (reduce-scattered by rows, or all-reduced)
            dp_fused_linear_cross_entropy(X, W, t, out=(loss, gX, gW), shard_grad_W=exchange == "reduce_scatter",
                                          flags=flags, **kw)
        else:
            flce.fused_linear_cross_entropy(X, W, t, out=(loss, gX, gW), flags=flags, **kw)

    # launch count and workspace of one step (untimed; every rank does the same)
    st = flce.fused_linear_cross_entropy(X, W, t, out=(loss, gX, gW), return_stats=True, **kw)[3]
    launches_per_step = st["kernel_launches"] + (1 if dp else 0)  # the data-parallel path counts N itself

    mem0 = torch.cuda.memory_allocated(dev)
    torch.cuda.reset_peak_memory_stats(dev)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if flce.device_error() != 0:
        raise RuntimeError("device error word set during warm-up")
    peak_extra_torch = torch.cuda.max_memory_allocated(dev) - mem0
    flce.phase_times(reset=True)

    stream = torch.cuda.current_stream()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dp:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        time.sleep(0.3)
        clk.mark_start()
        ev0.record(stream)
        for _ in range(args.steps):
            step(flags=B.FLAG_TIME_PHASES)
        ev1.record(stream)
        torch.cuda.synchronize()
        clk.mark_end()
    if dp:
        dist.barrier()
    ms = ev0.elapsed_time(ev1)
    if dp:
        mt = torch.tensor([ms], device=dev, dtype=torch.float64)
        dist.all_reduce(mt, op=dist.ReduceOp.MAX)
        ms = float(mt.item())
    phases = flce.phase_times(reset=True)
    err = flce.device_error()

    ms_step = ms / args.steps
    tokens = w.BT * world * args.steps
    value = tokens / (ms / 1e3)
    tflops = w.useful_flops * world * args.steps / (ms / 1e3) / 1e12
    peaks = load_peaks()

    # Roofline of the dominant kernel: tc_gemm_pair_kernel, launched for the
    # logits GEMM and the grad_X / grad_W GEMMs of every chunk; its algorithmic
    # work per step is the 6*BT*H*V useful FLOPs, timed by the CUDA events the
    # library records around those launches on the launching stream.
    gemm_phases = ("logits_gemm_softmax", "grad_gemms")
    gemm_ms = sum(phases[k][0] for k in gemm_phases)
    gemm_launches = sum(phases[k][1] for k in gemm_phases)
    achieved = w.useful_flops * args.steps / (gemm_ms / 1e3) / 1e12
    # the timed region is well under the seconds-long loop the sustained figure
    # was measured over, so the kernel is scored against the burst peak; the
    # sustained fraction is reported beside it
    peak = peaks["bf16_tflops"]
    traffic = recorded_traffic(w.name)
    roof = {"kernel": "tc_gemm_pair_kernel (logits, grad_X, grad_W launches)", "bound": "tensor",
            "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
            "traffic": traffic["bytes_per_launch"] if traffic else None,
            "traffic_source": traffic["source"] if traffic else "no capture of the current kernel source",
            "algorithmic_flops_per_launch": w.useful_flops * args.steps / max(gemm_launches, 1),
            "peak_kind": f"{peaks['source']} burst bf16 (timed region {ms / 1e3:.2f} s)",
            "frac_of_sustained_peak": achieved / peaks["bf16_tflops_sustained"],
            "launches": gemm_launches, "avg_launch_ms": gemm_ms / max(gemm_launches, 1),
            # HBM GB/s of the GEMM launches: the recorded per-launch DRAM bytes over this run's launch time
            "hbm_gbs": (traffic["bytes_per_launch"] / (gemm_ms / max(gemm_launches, 1) / 1e3) / 1e9
                        if traffic else None),
            # the recompute schedule executes 8*BT*H*V tensor FLOPs for the 6 that count
            "executed_tflops": achieved * (8.0 if args.schedule == "recompute" else 6.0) / 6.0}
    all_ms = sum(v[0] for v in phases.values())

    # end to end through the public API with host buffers: every step copies
    # X, W and target in from pinned host memory and loss, grad_X and grad_W
    # back out; HostPipeline overlaps step i's upload with step i-1's compute
    # and step i-2's download on separate streams (wall clock, both ends synced)
    e2e = None
    if exchange is None and args.e2e_steps > 0:
        from linear_cross_entropy_04_b200.pipeline import HostPipeline

        Xh = X.cpu().pin_memory()
        Wh = W.cpu().pin_memory()
        th = t.cpu().pin_memory()
        del gX, gW
        torch.cuda.empty_cache()
        houts = [(torch.empty((), dtype=torch.float32).pin_memory(), torch.empty_like(Xh).pin_memory(),
                  torch.empty_like(Wh).pin_memory()) for _ in range(2)]
        pipe = HostPipeline(w.BT, w.H, w.V, dtype=dt, slots=args.e2e_slots, **kw)
        for i in range(2):
            pipe.submit(Xh, Wh, th, houts[i % 2])
        pipe.synchronize()
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        for i in range(args.e2e_steps):
            pipe.submit(Xh, Wh, th, houts[i % 2])
        pipe.synchronize()
        wall = time.perf_counter() - t0
        h2d = Xh.numel() * Xh.element_size() + Wh.numel() * Wh.element_size() + th.numel() * 8
        d2h = 4 + houts[0][1].numel() * houts[0][1].element_size() + houts[0][2].numel() * houts[0][2].element_size()
        e2e = {"value": w.BT * args.e2e_steps / wall, "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": 1e3 * wall / args.e2e_steps, "slots": args.e2e_slots,
               "how": "public API (HostPipeline): pinned host X, W, target copied in and loss, grad_X, grad_W "
                      "copied back every step; copies overlap compute across steps (wall clock, the "
                      "pipeline's fill and drain included)"}
        del pipe
        # the copies' own bound: one step's uploads and downloads issued together on
        # two streams (PCIe carries both directions at once), no compute
        up = [torch.empty_like(Xh, device=dev), torch.empty_like(Wh, device=dev), torch.empty_like(th, device=dev)]
        dn = [torch.empty_like(houts[0][1], device=dev), torch.empty_like(houts[0][2], device=dev)]
        s1, s2 = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        best = float("inf")
        for _ in range(4):
            torch.cuda.synchronize()
            t0 = time.perf_counter()
            with torch.cuda.stream(s1):
                for d_, h_ in zip(up, (Xh, Wh, th)):
                    d_.copy_(h_, non_blocking=True)
            with torch.cuda.stream(s2):
                houts[0][1].copy_(dn[0], non_blocking=True)
                houts[0][2].copy_(dn[1], non_blocking=True)
            torch.cuda.synchronize()
            best = min(best, time.perf_counter() - t0)
        e2e["pcie_bound"] = {"value": w.BT / best, "unit": UNIT, "ms_per_step": 1e3 * best,
                             "frac": e2e["value"] / (w.BT / best),
                             "how": "one step's host-to-device and device-to-host copies issued together "
                                    "on two streams, best of 4 (wall clock)"}
        del up, dn, Xh, Wh, th, houts

    # several ranks: the data-parallel call itself, end to end, through the same
    # host pipeline. Every step each rank copies its X, W and target in from pinned
    # host memory, runs the step (the collectives included) and copies the loss,
    # its grad_X and its grad_W rows back out; uploads, compute and downloads of
    # consecutive steps overlap on three streams. CUDA events from the first
    # upload to the last download, max over ranks.
    if exchange in ("reduce_scatter", "all_reduce") and args.e2e_steps > 0:
        try:
            from linear_cross_entropy_04_b200.pipeline import HostPipeline

            Xh, Wh, th = X.cpu().pin_memory(), W.cpu().pin_memory(), t.cpu().pin_memory()
            gw_rows = w.V // world if exchange == "reduce_scatter" else w.V
            del gX, gW
            torch.cuda.empty_cache()
            houts = [(torch.empty((), dtype=torch.float32).pin_memory(), torch.empty_like(Xh).pin_memory(),
                      torch.empty((gw_rows, w.H), dtype=dt).pin_memory()) for _ in range(2)]

            def dp_step(Xs, Ws, ts, out):
                return dp_fused_linear_cross_entropy(Xs, Ws, ts, out=out, shard_grad_W=exchange == "reduce_scatter",
                                                     **kw)

            pipe = HostPipeline(w.BT, w.H, w.V, dtype=dt, slots=args.e2e_slots, step=dp_step, **kw)
            for i in range(2):
                pipe.submit(Xh, Wh, th, houts[i % 2])
            pipe.synchronize()
            torch.cuda.synchronize()
            dist.barrier()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(pipe.s_in)
            for i in range(args.e2e_steps):
                pipe.submit(Xh, Wh, th, houts[i % 2])
            e1.record(pipe.s_out)
            pipe.synchronize()
            torch.cuda.synchronize()
            et = torch.tensor([e0.elapsed_time(e1)], device=dev, dtype=torch.float64)
            dist.all_reduce(et, op=dist.ReduceOp.MAX)
            ems = float(et.item())
            h2d = Xh.numel() * Xh.element_size() + Wh.numel() * Wh.element_size() + th.numel() * 8
            d2h = 4 + houts[0][1].numel() * houts[0][1].element_size() + houts[0][2].numel() * houts[0][2].element_size()
            e2e = {"value": w.BT * world * args.e2e_steps / (ems / 1e3), "unit": UNIT,
                   "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ems / args.e2e_steps,
                   "slots": args.e2e_slots,
                   "how": "per rank, the public data-parallel call (dp_fused_linear_cross_entropy) through "
                          "HostPipeline: pinned host X, W, target copied in and loss, grad_X and this rank's "
                          "grad_W rows copied back every step, copies overlapping compute across steps; CUDA "
                          "events from the first upload to the last download, max over ranks; bytes are per rank"}
            del pipe
        except Exception as exc:  # the device-timed line above stands without it
            e2e = {"unavailable": f"{type(exc).__name__}: {exc}"[:300]}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(d, args.cpu_seconds)

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic (seeded; random-init lm_head weights)",
        "config": {"workload": w.name, "BT": w.BT, "H": w.H, "V": w.V, "global_batch": w.BT * world,
                   "seq_len": w.BT, "parallelism": f"dp{world}",
                   "grad_w_exchange": EXCHANGE_NAMES.get(exchange),
                   "l2": "inputs larger than L2 (W alone is %.2f GB)" % (w.V * w.H * 2 / 1e9),
                   "chunk_rows": st["chunk_rows"], "n_chunks": st["n_chunks"],
                   "grad_w_accum": args.grad_w_accum, "schedule": args.schedule},
        "tflops": tflops,
        "frac_of_bf16_peak": tflops / peaks["bf16_tflops"],
        "frac_of_bf16_sustained_peak": tflops / peaks["bf16_tflops_sustained"],
        "peak_workspace_bytes": st["workspace_bytes"],
        "peak_extra_torch_bytes": peak_extra_torch,
        "materialized_logits_bytes": st["materialized_logits_bytes"],
        "workspace_vs_materialized": st["workspace_bytes"] / st["materialized_logits_bytes"],
        "phases_ms_per_step": {k: v[0] / args.steps for k, v in phases.items()},
        "gemm_share_of_step": gemm_ms / max(all_ms, 1e-9),
        "roofline": roof,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk.summary(),
        "device_error": err,
        "peaks": peaks,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dp:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
