"""Chunked fused-linear preference losses on top of the fused CE path.

"Liger-Kernel 項目詳細介紹" lists post-training losses built the same way as the
fused linear cross-entropy (支持的模型和操作 > 後訓練內核: DPO, ORPO, CPO, SimPO,
KTO) and shows the call `orpo_loss(lm_head.weight, x, target)` (使用方法 > 4).
The pages give no formulas; each loss here restates its published definition:

  DPO   (Rafailov et al., 2023): -log sigmoid(beta * ((lp_w - ref_w) - (lp_l - ref_l)))
  ORPO  (Hong et al., 2024):     NLL(chosen) + lam * -log sigmoid(log_odds_w - log_odds_l),
                                 log_odds = a - log(1 - exp(a)), a = mean token log-prob
  CPO   (Xu et al., 2024):       -log sigmoid(beta * (lp_w - lp_l)) + NLL(chosen)
  SimPO (Meng et al., 2024):     -log sigmoid(beta * (lp_w / |y_w| - lp_l / |y_l|) - gamma)
  KTO   (Ethayarajh et al., 2024): w_i * (1 - sigmoid(beta * s_i * (r_i - z0))),
                                 r = lp - ref, s = +1 desirable / -1 undesirable,
                                 z0 = max(0, mean r) held constant

lp is a sequence's summed token log-probability over its non-ignored tokens,
|y| its count of such tokens, NLL(chosen) the mean token loss over the chosen
sequences' tokens; pair terms are averaged over pairs (KTO over sequences).

Layout (a reading; the pages show only the call): x is [2B, T, H] (or
[2B*T, H] with seq_len T), target [2B, T]; rows 0..B-1 are the chosen
responses and rows B..2B-1 the rejected ones of the same prompts. Prompt and
padding positions carry ignore_index. KTO takes [N, T] sequences and a 0/1
`desirable` vector instead of pairs.

Every loss depends on the logits only through the per-token losses l_t. The
CUDA path gives l_t (reduction 'none'), O(batch) tensor work gives the loss and
g_t = dLoss/dl_t, and the gradients are those of sum_t g_t * l_t (row_grad).
Two schedules:
  single pass (default while the batch's chunk store fits keep_limit_bytes):
    forward_keep keeps the bf16 store of the whole batch, and backward_from_kept
    takes the gradients from it: 6*BT*H*V tensor FLOPs;
  two passes: a forward pass, then the chunked fused path again with row_grad:
    8*BT*H*V tensor FLOPs, with the chunked path's memory.
The fp32 logits are never materialised in either.
"""
from __future__ import annotations

from typing import Optional

import torch

from .api import backward_from_kept, forward_keep, fused_linear_cross_entropy, keep_workspace_bytes

KINDS = ("dpo", "orpo", "cpo", "simpo", "kto")


def sequence_stats(row_loss: torch.Tensor, target: torch.Tensor, n_seq: int, ignore_index: int = -100):
    """Per-sequence summed log-prob and token count from per-token losses [n_seq*T]."""
    valid = (target.reshape(n_seq, -1) != ignore_index).to(row_loss.dtype)
    lp = -(row_loss.reshape(n_seq, -1) * valid).sum(1)
    return lp, valid.sum(1)


def preference_loss_from_logps(kind: str, lp: torch.Tensor, count: torch.Tensor, nll_sum_chosen: torch.Tensor,
                               beta: float = 0.1, gamma: float = 0.5, lam: float = 0.1,
                               ref_logps: Optional[torch.Tensor] = None,
                               desirable: Optional[torch.Tensor] = None) -> torch.Tensor:
    """The scalar loss from per-sequence log-probs (differentiable in lp and nll_sum_chosen)."""
    logsig = torch.nn.functional.logsigmoid
    if kind == "kto":
        ref = ref_logps if ref_logps is not None else torch.zeros_like(lp)
        r = lp - ref
        z0 = torch.clamp(r.detach().mean(), min=0.0)
        s = desirable.to(lp.dtype) * 2.0 - 1.0
        return (1.0 - torch.sigmoid(beta * s * (r - z0))).mean()
    B = lp.shape[0] // 2
    lw, ll = lp[:B], lp[B:]
    cw, cl = count[:B], count[B:]
    nll_chosen = nll_sum_chosen / torch.clamp(cw.sum(), min=1.0)
    if kind == "dpo":
        ref = ref_logps if ref_logps is not None else torch.zeros_like(lp)
        return -logsig(beta * ((lw - ref[:B]) - (ll - ref[B:]))).mean()
    if kind == "cpo":
        return -logsig(beta * (lw - ll)).mean() + nll_chosen
    if kind == "simpo":
        return -logsig(beta * (lw / torch.clamp(cw, min=1.0) - ll / torch.clamp(cl, min=1.0)) - gamma).mean()
    if kind == "orpo":
        aw = lw / torch.clamp(cw, min=1.0)
        al = ll / torch.clamp(cl, min=1.0)
        log_odds_w = aw - torch.log1p(-torch.exp(aw))
        log_odds_l = al - torch.log1p(-torch.exp(al))
        return nll_chosen + lam * -logsig(log_odds_w - log_odds_l).mean()
    raise ValueError(f"unknown preference loss {kind!r}")


def fused_linear_preference_loss(kind: str, weight: torch.Tensor, x: torch.Tensor, target: torch.Tensor,
                                 ignore_index: int = -100, beta: float = 0.1, gamma: float = 0.5, lam: float = 0.1,
                                 ref_logps: Optional[torch.Tensor] = None, desirable: Optional[torch.Tensor] = None,
                                 want_grad_X: bool = True, want_grad_W: bool = True, single_pass="auto",
                                 keep_limit_bytes: int = 2 << 30, **kw):
    """(loss, grad_x, grad_weight) of a preference loss over lm_head logits x weight^T.

    x [N, T, H] or [N*T, H] with target [N, T]; N = 2B (pairs) or the KTO
    sequence count. Returns grads shaped like x and weight.
    single_pass: True, False, or "auto" (when the batch's store fits
    keep_limit_bytes and the batch is at most 32768 tokens).
    """
    if kind not in KINDS:
        raise ValueError(f"kind must be one of {KINDS}")
    n_seq = target.shape[0]
    X = x.reshape(-1, x.shape[-1])
    t = target.reshape(-1)
    if single_pass == "auto":
        single_pass = (not kw and X.shape[0] <= 32768 and
                       keep_workspace_bytes(X.shape[0], X.shape[1], weight.shape[0],
                                            "bf16" if X.dtype == torch.bfloat16 else "f32") <= keep_limit_bytes)
    kept = None
    if single_pass:
        row_loss, kept = forward_keep(X, weight, t, ignore_index=ignore_index, reduction="none")
    else:
        row_loss, _, _ = fused_linear_cross_entropy(X, weight, t, ignore_index=ignore_index, reduction="none",
                                                    want_grad_X=False, want_grad_W=False, **kw)
    # O(batch) sequence-level part: loss and its gradient w.r.t. each token's loss
    # (grad mode is forced on: autograd.Function.forward runs with it off)
    with torch.enable_grad():
        rl = row_loss.detach().double().requires_grad_(True)
        lp, count = sequence_stats(rl, t, n_seq, ignore_index)
        B = n_seq // 2
        chosen_valid = (t.reshape(n_seq, -1)[:B] != ignore_index).to(rl.dtype)
        nll_sum_chosen = (rl.reshape(n_seq, -1)[:B] * chosen_valid).sum()
        loss = preference_loss_from_logps(kind, lp, count, nll_sum_chosen, beta=beta, gamma=gamma, lam=lam,
                                          ref_logps=None if ref_logps is None else ref_logps.double(),
                                          desirable=desirable)
        (g,) = torch.autograd.grad(loss, rl)
    if kept is not None:
        gX, gW = backward_from_kept(kept, reduction="none", row_grad=g.float(), want_grad_X=want_grad_X,
                                    want_grad_W=want_grad_W)
    else:
        _, gX, gW = fused_linear_cross_entropy(X, weight, t, ignore_index=ignore_index, reduction="none",
                                               row_grad=g.float(), want_grad_X=want_grad_X,
                                               want_grad_W=want_grad_W, **kw)
    return loss.detach().float(), (gX.reshape(x.shape) if gX is not None else None), gW


class _PrefFunction(torch.autograd.Function):
    @staticmethod
    def forward(ctx, weight, x, target, kind, ignore_index, beta, gamma, lam, ref_logps, desirable):
        loss, gX, gW = fused_linear_preference_loss(kind, weight, x, target, ignore_index=ignore_index, beta=beta,
                                                    gamma=gamma, lam=lam, ref_logps=ref_logps,
                                                    desirable=desirable, want_grad_X=ctx.needs_input_grad[1],
                                                    want_grad_W=ctx.needs_input_grad[0])
        ctx.save_for_backward(gX if gX is not None else torch.empty(0), gW if gW is not None else torch.empty(0))
        ctx.has = (gX is not None, gW is not None)
        return loss

    @staticmethod
    def backward(ctx, grad_out):
        gX, gW = ctx.saved_tensors
        hx, hw = ctx.has
        dX = gX * grad_out.to(gX.dtype) if hx else None
        dW = gW * grad_out.to(gW.dtype) if hw else None
        return dW, dX, None, None, None, None, None, None, None, None


class FusedLinearPreferenceLoss(torch.nn.Module):
    """loss_fn(lm_head.weight, x, target[, ref_logps | desirable]) for one preference loss kind."""

    def __init__(self, kind: str, ignore_index: int = -100, beta: float = 0.1, gamma: float = 0.5,
                 lam: float = 0.1):
        super().__init__()
        if kind not in KINDS:
            raise ValueError(f"kind must be one of {KINDS}")
        self.kind, self.ignore_index, self.beta, self.gamma, self.lam = kind, ignore_index, beta, gamma, lam

    def forward(self, weight, x, target, ref_logps=None, desirable=None):
        return _PrefFunction.apply(weight, x, target, self.kind, self.ignore_index, self.beta, self.gamma,
                                   self.lam, ref_logps, desirable)


def FusedLinearDPOLoss(**kw):
    return FusedLinearPreferenceLoss("dpo", **kw)


def FusedLinearORPOLoss(**kw):
    return FusedLinearPreferenceLoss("orpo", **kw)


def FusedLinearCPOLoss(**kw):
    return FusedLinearPreferenceLoss("cpo", **kw)


def FusedLinearSimPOLoss(**kw):
    return FusedLinearPreferenceLoss("simpo", **kw)


def FusedLinearKTOLoss(**kw):
    return FusedLinearPreferenceLoss("kto", **kw)
