"""Float64 CPU oracle for the fused-linear preference losses (test infrastructure).

Only tests/ import this module. It restates each loss from its published
definition (DPO: Rafailov et al. 2023; ORPO: Hong et al. 2024; CPO: Xu et al.
2024; SimPO: Meng et al. 2024; KTO: Ethayarajh et al. 2024) in NumPy, with the
gradient of the loss with respect to every per-token loss derived by hand,
then obtains grad_X and grad_W from flce() with those per-row weights.

Conventions (readings; the pages name the losses and show only their call,
"Liger-Kernel 項目詳細介紹", 使用方法 > 4. 後訓練損失使用示例):
  * sequences are rows of target [N, T]; prompt / padding tokens carry
    ignore_index; lp = sum of log p over a sequence's other tokens, c = count;
  * pairs: rows 0..B-1 chosen, B..2B-1 rejected (N = 2B);
  * NLL(chosen) = sum of chosen token losses / number of chosen tokens;
  * pair terms are averaged over the B pairs, KTO terms over the N sequences,
    and KTO's reference point z0 = max(0, mean(lp - ref)) is held constant.

Pins (tests/test_oracle.py): closed forms for identical chosen / rejected
sequences, central finite differences, and torch float64 autograd.
"""
from __future__ import annotations

import numpy as np

from .flce_oracle import flce


def _sigmoid(u):
    return 1.0 / (1.0 + np.exp(-u))


def _logsig(u):
    return -np.logaddexp(0.0, -u)


def sequence_logps(row_loss, target, n_seq, ignore_index=-100):
    valid = (np.asarray(target).reshape(n_seq, -1) != ignore_index).astype(np.float64)
    lp = -(np.asarray(row_loss, dtype=np.float64).reshape(n_seq, -1) * valid).sum(1)
    return lp, valid.sum(1), valid


def loss_and_token_grad(kind, row_loss, target, n_seq, ignore_index=-100, beta=0.1, gamma=0.5, lam=0.1,
                        ref_logps=None, desirable=None):
    """(loss, dloss/drow_loss [N*T]) for per-token losses row_loss."""
    lp, c, valid = sequence_logps(row_loss, target, n_seq, ignore_index)
    dlp = np.zeros(n_seq)  # dL/dlp per sequence
    dS = 0.0               # dL/d(sum of chosen token losses)
    if kind == "kto":
        ref = np.zeros(n_seq) if ref_logps is None else np.asarray(ref_logps, dtype=np.float64)
        r = lp - ref
        z0 = max(0.0, float(r.mean()))
        s = np.asarray(desirable, dtype=np.float64) * 2.0 - 1.0
        v = beta * s * (r - z0)
        loss = float((1.0 - _sigmoid(v)).mean())
        dlp = -_sigmoid(v) * (1.0 - _sigmoid(v)) * beta * s / n_seq
    else:
        B = n_seq // 2
        lw, ll, cw, cl = lp[:B], lp[B:], c[:B], c[B:]
        Cw = max(float(cw.sum()), 1.0)
        S = float((np.asarray(row_loss, dtype=np.float64).reshape(n_seq, -1)[:B] * valid[:B]).sum())
        if kind == "dpo":
            ref = np.zeros(n_seq) if ref_logps is None else np.asarray(ref_logps, dtype=np.float64)
            u = beta * ((lw - ref[:B]) - (ll - ref[B:]))
            loss = float(-_logsig(u).mean())
            dlp[:B] = -_sigmoid(-u) * beta / B
            dlp[B:] = _sigmoid(-u) * beta / B
        elif kind == "cpo":
            u = beta * (lw - ll)
            loss = float(-_logsig(u).mean()) + S / Cw
            dlp[:B] = -_sigmoid(-u) * beta / B
            dlp[B:] = _sigmoid(-u) * beta / B
            dS = 1.0 / Cw
        elif kind == "simpo":
            cwc, clc = np.maximum(cw, 1.0), np.maximum(cl, 1.0)
            u = beta * (lw / cwc - ll / clc) - gamma
            loss = float(-_logsig(u).mean())
            dlp[:B] = -_sigmoid(-u) * beta / (cwc * B)
            dlp[B:] = _sigmoid(-u) * beta / (clc * B)
        elif kind == "orpo":
            cwc, clc = np.maximum(cw, 1.0), np.maximum(cl, 1.0)
            aw, al = lw / cwc, ll / clc
            u = (aw - np.log1p(-np.exp(aw))) - (al - np.log1p(-np.exp(al)))
            loss = S / Cw + lam * float(-_logsig(u).mean())
            dlp[:B] = -lam * _sigmoid(-u) / B / (1.0 - np.exp(aw)) / cwc
            dlp[B:] = lam * _sigmoid(-u) / B / (1.0 - np.exp(al)) / clc
            dS = 1.0 / Cw
        else:
            raise ValueError(kind)
    # l_t enters lp with a minus sign; chosen tokens also enter S
    g = -dlp[:, None] * valid
    if dS:
        g[: n_seq // 2] += dS * valid[: n_seq // 2]
    return loss, g.reshape(-1)


def preference(kind, X, W, target, ignore_index=-100, **kw):
    """Loss, grad_X [N*T, H] and grad_W of a preference loss, in float64."""
    target = np.asarray(target)
    n_seq = target.shape[0]
    t = target.reshape(-1)
    base = flce(X, W, t, ignore_index=ignore_index, reduction="none", want_grad_X=False, want_grad_W=False)
    loss, g = loss_and_token_grad(kind, base["row_loss"], target, n_seq, ignore_index, **kw)
    r = flce(X, W, t, ignore_index=ignore_index, reduction="none", row_grad=g)
    return {"loss": loss, "grad_X": r["grad_X"], "grad_W": r["grad_W"], "token_grad": g}
