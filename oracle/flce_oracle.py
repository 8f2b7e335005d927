"""Float64 CPU oracle for fused linear cross-entropy (FLCE).

TEST INFRASTRUCTURE. Only tests/, __graft_entry__.smoke() and bench.py's CPU
baseline / reference arm may import this module. The CUDA library never calls
it, and it shares no code with the CUDA path: it reads plain arrays and
computes the textbook definition in float64 with NumPy.

What it computes. "Liger Kernel: Efficient Triton Kernels for LLM Training"
(paper review, 提案手法) describes a chunked fused Linear+CrossEntropy that
computes lm_head logits over a large vocabulary without keeping them, and
"Liger-Kernel 項目詳細介紹" (核心特性 > 技術實現) states that the kernels make no
approximation. So the result the fused method must reach is the plain one:

    z      = X W^T                                   (BT x V)
    lse_i  = m_i + log sum_v exp(z_iv - m_i),  m_i = max_v z_iv
    l_i    = lse_i - z_{i,t_i}        for rows with t_i != ignore_index, else 0
    loss   = sum_i l_i / N  (mean, N = number of non-ignored rows)  or sum_i l_i
    dz_i   = (softmax(z_i) - onehot(t_i)) * s,   s = 1/N (mean) or 1 (sum);
             dz_i = 0 for ignored rows
    grad_X = dz W,      grad_W = dz^T X

The call shape follows the low-level API of "Liger-Kernel 項目詳細介紹"
(使用方法 > 3. 低級 API 方式): loss_fn(weight [V,H], input [BT,H], target [BT]).

Readings where the pages are silent:
  * mean divides by N, the count of non-ignored rows;
  * 'none' returns the per-row losses (0 for ignored rows), as the torch loss
    modules the pages' low-level API mirrors do; with an upstream gradient
    per row, each dlogits row is scaled by it;
  * N = 0 (every row ignored) gives loss 0 and zero gradients, not NaN;
  * a target outside [0, V) that is not ignore_index is an error (ValueError);
  * a row whose target equals ignore_index is ignored even if ignore_index is
    inside [0, V).

The only blocking is over independent rows (block_rows) so that full-size
vocabularies fit in host memory; it changes no arithmetic except the order in
which grad_W's per-row contributions are summed, in float64.

Parity pins: every function here is pinned in tests/test_oracle.py against
closed forms, invariants, finite differences and a pure-Python brute force.
"""
from __future__ import annotations

import math
from typing import Optional, Sequence

import numpy as np

__all__ = [
    "valid_mask",
    "count_valid",
    "logits",
    "row_logsumexp",
    "dlogits",
    "flce",
    "flce_rows",
    "flce_grad_W_rows",
    "flce_brute_force",
    "cross_entropy",
]


def _f64(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


def valid_mask(target: np.ndarray, V: int, ignore_index: int = -100) -> np.ndarray:
    """Rows that take part in the loss: target != ignore_index.

    Raises ValueError for a target outside [0, V) that is not ignore_index.
    """
    target = np.asarray(target, dtype=np.int64)
    valid = target != ignore_index
    bad = valid & ((target < 0) | (target >= V))
    if bad.any():
        raise ValueError(f"target out of range at rows {np.nonzero(bad)[0][:8].tolist()}")
    return valid


def count_valid(target: np.ndarray, V: int, ignore_index: int = -100) -> int:
    """N, the mean-reduction denominator: the number of non-ignored rows."""
    return int(valid_mask(target, V, ignore_index).sum())


def logits(X: np.ndarray, W: np.ndarray) -> np.ndarray:
    """z = X W^T, the lm_head projection (X is [BT,H], W is [V,H])."""
    return _f64(X) @ _f64(W).T


def row_logsumexp(z: np.ndarray) -> np.ndarray:
    """lse_i = m_i + log sum_v exp(z_iv - m_i) with m_i the row maximum."""
    z = _f64(z)
    m = z.max(axis=1)
    return m + np.log(np.exp(z - m[:, None]).sum(axis=1))


def _scale(reduction: str, n_valid: int) -> float:
    if reduction == "mean":
        return 0.0 if n_valid == 0 else 1.0 / n_valid
    if reduction in ("sum", "none"):
        return 1.0
    raise ValueError(f"unknown reduction {reduction!r}")


def _target_logits(z: np.ndarray, rows: np.ndarray, target: np.ndarray) -> np.ndarray:
    """z_{i, t_i} for the given rows."""
    return z[rows, target[rows]]


def _softmax_minus_onehot(z: np.ndarray, lse: np.ndarray, target: np.ndarray,
                          valid: np.ndarray, s: float) -> np.ndarray:
    """dz_i = (exp(z_i - lse_i) - onehot(t_i)) * s for valid rows, 0 otherwise."""
    dz = np.exp(z - lse[:, None])
    rows = np.nonzero(valid)[0]
    dz[rows, target[rows]] -= 1.0
    dz *= s
    dz[~valid] = 0.0
    return dz


def _grad_X(dz: np.ndarray, W: np.ndarray) -> np.ndarray:
    """grad_X = dz W  ([rows,V] x [V,H])."""
    return dz @ W


def _grad_W(dz: np.ndarray, X: np.ndarray) -> np.ndarray:
    """grad_W contribution dz^T X  ([V,rows] x [rows,H])."""
    return dz.T @ X


def dlogits(z: np.ndarray, target: np.ndarray, ignore_index: int = -100,
            reduction: str = "mean", n_valid: Optional[int] = None) -> np.ndarray:
    """dloss/dz for the rows of z: (softmax(z_i) - onehot(t_i)) * scale, 0 if ignored.

    n_valid overrides the mean denominator (needed when z holds a subset of
    the rows of a larger batch).
    """
    z = _f64(z)
    target = np.asarray(target, dtype=np.int64)
    valid = valid_mask(target, z.shape[1], ignore_index)
    N = int(valid.sum()) if n_valid is None else int(n_valid)
    return _softmax_minus_onehot(z, row_logsumexp(z), target, valid, _scale(reduction, N))


def flce(X, W, target, ignore_index: int = -100, reduction: str = "mean",
         n_valid: Optional[int] = None, want_grad_X: bool = True,
         want_grad_W: bool = True, block_rows: int = 4096, row_grad=None) -> dict:
    """Loss, per-row losses, lse and both gradients of FLCE in float64.

    reduction 'none' returns the per-row losses as `loss`. row_grad [BT]
    (default all ones) is an upstream gradient per row: the gradients are
    those of sum_i row_grad_i * l_i * s, s = 1/N (mean) or 1 (sum, none).
    Returns a dict with keys loss (float, or [BT] for 'none'), row_loss [BT],
    lse [BT], n_valid, grad_X [BT,H] (or None) and grad_W [V,H] (or None).
    """
    X = _f64(X)
    W = _f64(W)
    target = np.asarray(target, dtype=np.int64)
    BT, H = X.shape
    V = W.shape[0]
    valid = valid_mask(target, V, ignore_index)
    N = int(valid.sum()) if n_valid is None else int(n_valid)
    s = _scale(reduction, N)
    g = np.ones(BT) if row_grad is None else _f64(row_grad).reshape(BT)

    row_loss = np.zeros(BT)
    lse = np.zeros(BT)
    grad_X = np.zeros((BT, H)) if want_grad_X else None
    grad_W = np.zeros((V, H)) if want_grad_W else None
    for r0 in range(0, BT, max(1, block_rows)):
        r1 = min(BT, r0 + block_rows)
        z = logits(X[r0:r1], W)
        lse_b = row_logsumexp(z)
        lse[r0:r1] = lse_b
        vb = valid[r0:r1]
        tb = target[r0:r1]
        rows = np.nonzero(vb)[0]
        row_loss[r0 + rows] = lse_b[rows] - _target_logits(z, rows, tb)
        dz = _softmax_minus_onehot(z, lse_b, tb, vb, s) * g[r0:r1, None]
        if want_grad_X:
            grad_X[r0:r1] = _grad_X(dz, W)
        if want_grad_W:
            grad_W += _grad_W(dz, X[r0:r1])
    total = float(row_loss.sum())
    if reduction == "none":
        loss = row_loss.copy()
    else:
        loss = total * s if reduction == "mean" else total
    return {"loss": loss, "row_loss": row_loss, "lse": lse, "n_valid": N,
            "grad_X": grad_X, "grad_W": grad_W}


def flce_rows(X, W, target, rows: Sequence[int], n_valid: int,
              ignore_index: int = -100, reduction: str = "mean") -> dict:
    """Per-row loss and grad_X rows for a subset of a larger batch.

    Rows are independent except for the mean denominator, which the caller
    passes as n_valid (the count over the whole batch).
    """
    rows = np.asarray(rows, dtype=np.int64)
    out = flce(_f64(X)[rows], W, np.asarray(target)[rows], ignore_index=ignore_index,
               reduction=reduction, n_valid=n_valid, want_grad_W=False)
    return {"row_loss": out["row_loss"], "lse": out["lse"], "grad_X": out["grad_X"]}


def flce_grad_W_rows(X, W, target, vocab_rows: Sequence[int], ignore_index: int = -100,
                     reduction: str = "mean", n_valid: Optional[int] = None) -> np.ndarray:
    """grad_W[v, :] = sum_i dz[i, v] X_i for the listed vocabulary rows only.

    Every row's lse still needs all V logits; only the final contraction is
    restricted to the requested rows of grad_W.
    """
    X = _f64(X)
    target = np.asarray(target, dtype=np.int64)
    z = logits(X, W)
    valid = valid_mask(target, z.shape[1], ignore_index)
    N = int(valid.sum()) if n_valid is None else int(n_valid)
    dz = _softmax_minus_onehot(z, row_logsumexp(z), target, valid, _scale(reduction, N))
    return _grad_W(dz[:, np.asarray(vocab_rows, dtype=np.int64)], X)


def flce_brute_force(X, W, target, ignore_index: int = -100,
                     reduction: str = "mean") -> dict:
    """The same definition written as plain Python loops over scalars.

    For tiny inputs only; it cross-checks the vectorised flce().
    """
    X = [[float(v) for v in row] for row in np.asarray(X, dtype=np.float64)]
    W = [[float(v) for v in row] for row in np.asarray(W, dtype=np.float64)]
    t = [int(v) for v in np.asarray(target)]
    BT, H, V = len(X), len(X[0]) if X else 0, len(W)
    valid = []
    for i in range(BT):
        if t[i] == ignore_index:
            valid.append(False)
        elif 0 <= t[i] < V:
            valid.append(True)
        else:
            raise ValueError("target out of range")
    N = sum(valid)
    s = _scale(reduction, N)
    total = 0.0
    grad_X = [[0.0] * H for _ in range(BT)]
    grad_W = [[0.0] * H for _ in range(V)]
    for i in range(BT):
        if not valid[i]:
            continue
        z = [sum(X[i][k] * W[v][k] for k in range(H)) for v in range(V)]
        m = max(z)
        lse = m + math.log(sum(math.exp(zv - m) for zv in z))
        total += lse - z[t[i]]
        for v in range(V):
            g = (math.exp(z[v] - lse) - (1.0 if v == t[i] else 0.0)) * s
            for k in range(H):
                grad_X[i][k] += g * W[v][k]
                grad_W[v][k] += g * X[i][k]
    loss = total * s if reduction == "mean" else total
    return {"loss": loss, "grad_X": np.array(grad_X).reshape(BT, H),
            "grad_W": np.array(grad_W).reshape(V, H), "n_valid": N}


def cross_entropy(z, target, ignore_index: int = -100, reduction: str = "mean") -> dict:
    """Cross-entropy of given logits z [BT,V]: loss, per-row losses, dz.

    This is the logits-given CrossEntropy of "Liger Kernel: Efficient Triton
    Kernels for LLM Training" (paper review, 主な発見: online softmax with
    in-place gradient replacement); its result is the same textbook formula.
    """
    z = _f64(z)
    target = np.asarray(target, dtype=np.int64)
    V = z.shape[1]
    valid = valid_mask(target, V, ignore_index)
    N = int(valid.sum())
    s = _scale(reduction, N)
    lse = row_logsumexp(z)
    rows = np.nonzero(valid)[0]
    row_loss = np.zeros(z.shape[0])
    row_loss[rows] = lse[rows] - _target_logits(z, rows, target)
    total = float(row_loss.sum())
    loss = total * s if reduction == "mean" else total
    return {"loss": loss, "row_loss": row_loss, "lse": lse, "n_valid": N,
            "dz": _softmax_minus_onehot(z, lse, target, valid, s)}
