"""Seeded synthetic inputs for fused linear cross-entropy.

This module only draws random numbers and rounds them to the storage dtype.
It holds none of the loss arithmetic, so both the CUDA path (tests, bench)
and the float64 CPU oracle can be fed from it without sharing any method code.

Workloads are the lm_head shapes of the model families that "Liger-Kernel
項目詳細介紹" lists under 支持的模型架構 (LLaMA 3, Qwen2), plus a tiny fp32 case
and a wide-vocabulary stress case. No dataset items are used: the pages'
fine-tuning runs (Alpaca) are stood in for by these synthetic draws.

Recipe (one numpy PCG64 generator per call, draws in this order):
  1. X ~ N(0, 1), shape [BT, H]           (float32 draw, then rounded to dtype)
  2. W ~ N(0, w_std), shape [V, H]        (standard deviation w_std)
  3. targets: uniform integers in [0, V), or Zipf(s) over ranks 1..V truncated
     to the vocabulary and sampled by inverse CDF, token id = rank - 1
  4. exactly round(ignore_frac * BT) positions, chosen by a seeded permutation,
     are set to ignore_index (-100)
Rounding to bf16 is round-to-nearest-even (torch's CPU cast). The float32
arrays returned hold exactly the rounded values, so upcasting them to float64
gives the oracle the very numbers the GPU reads.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

IGNORE_INDEX = -100


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    BT: int
    H: int
    V: int
    dtype: str            # "f32" or "bf16"
    w_std: float
    targets: str          # "uniform" or "zipf"
    ignore_frac: float
    zipf_s: float = 1.1
    seed: int = 0

    @property
    def useful_flops(self) -> float:
        """6*BT*H*V: the three BT x H x V contractions (logits, grad_X, grad_W)."""
        return 6.0 * self.BT * self.H * self.V

    @property
    def logits_bytes_bf16(self) -> int:
        """Size of the fully materialised BT x V logits at 2 bytes per element."""
        return self.BT * self.V * 2


WORKLOADS = {
    "tiny": Workload("tiny", 512, 256, 4096, "f32", 0.02, "uniform", 0.05),
    "llama3_8b_seq": Workload("llama3_8b_seq", 4096, 4096, 128256, "bf16", 0.02, "uniform", 0.10),
    "qwen2_7b": Workload("qwen2_7b", 16384, 3584, 152064, "bf16", 0.02, "zipf", 0.05),
    "llama3_8b_train": Workload("llama3_8b_train", 32768, 4096, 128256, "bf16", 0.02, "zipf", 0.10),
    "large_vocab_stress": Workload("large_vocab_stress", 16384, 2048, 256000, "bf16", 0.05, "uniform", 0.30),
}


def round_to_dtype(a: np.ndarray, dtype: str) -> np.ndarray:
    """Round float32 values to the storage dtype and return them as float32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    if dtype == "f32":
        return a
    if dtype == "bf16":
        import torch

        return torch.from_numpy(a).to(torch.bfloat16).to(torch.float32).numpy()
    raise ValueError(f"unknown dtype {dtype!r}")


def draw_targets(rng: np.random.Generator, BT: int, V: int, kind: str,
                 ignore_frac: float, zipf_s: float = 1.1,
                 ignore_index: int = IGNORE_INDEX) -> np.ndarray:
    if kind == "uniform":
        t = rng.integers(0, V, size=BT, dtype=np.int64)
    elif kind == "zipf":
        ranks = np.arange(1, V + 1, dtype=np.float64)
        cdf = np.cumsum(ranks ** (-zipf_s))
        cdf /= cdf[-1]
        u = rng.random(BT)
        t = np.minimum(np.searchsorted(cdf, u, side="right"), V - 1).astype(np.int64)
    else:
        raise ValueError(f"unknown target distribution {kind!r}")
    n_ign = int(round(ignore_frac * BT))
    if n_ign:
        t[rng.permutation(BT)[:n_ign]] = ignore_index
    return t


def make_inputs(w: Workload, BT: Optional[int] = None, H: Optional[int] = None,
                V: Optional[int] = None, seed: Optional[int] = None,
                w_zero: bool = False) -> dict:
    """Draw (X, W, target) for a workload; sizes may be overridden for small cases.

    Returns float32 arrays X [BT,H], W [V,H] holding exactly the dtype-rounded
    values, int64 target [BT], and the workload's dtype string.
    """
    BT = w.BT if BT is None else BT
    H = w.H if H is None else H
    V = w.V if V is None else V
    rng = np.random.Generator(np.random.PCG64(w.seed if seed is None else seed))
    X = rng.standard_normal((BT, H), dtype=np.float32)
    if w_zero:
        W = np.zeros((V, H), dtype=np.float32)
    else:
        W = rng.standard_normal((V, H), dtype=np.float32)
        W *= np.float32(w.w_std)
    target = draw_targets(rng, BT, V, w.targets, w.ignore_frac, w.zipf_s)
    return {
        "X": round_to_dtype(X, w.dtype),
        "W": W if w_zero else round_to_dtype(W, w.dtype),  # zeros are exact in every dtype
        "target": target,
        "dtype": w.dtype,
        "BT": BT, "H": H, "V": V,
    }


def sample_rows(BT: int, n: int = 256, seed: int = 1) -> np.ndarray:
    """Rows checked one by one on full-size workloads: n distinct rows, sorted."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return np.sort(rng.choice(BT, size=min(n, BT), replace=False)).astype(np.int64)
