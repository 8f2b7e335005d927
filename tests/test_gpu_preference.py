"""Fused-linear preference losses on the CUDA path vs the float64 oracle."""
import numpy as np
import pytest
import torch

from oracle import preference_oracle as po
from linear_cross_entropy_04_b200.inputs import WORKLOADS, make_inputs, IGNORE_INDEX
from flce_testlib import need_gpu, rel_err, assert_grad_close

pytestmark = pytest.mark.gpu

KINDS = ["dpo", "orpo", "cpo", "simpo", "kto"]


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()


def _case(B=4, T=48, H=256, V=3000):
    N = 2 * B
    d = make_inputs(WORKLOADS["llama3_8b_seq"], BT=N * T, H=H, V=V)
    t = d["target"].reshape(N, T).copy()
    t[t == IGNORE_INDEX] = 0
    t[:, :8] = IGNORE_INDEX  # prompt tokens
    t[1, -5:] = IGNORE_INDEX  # padding
    t[N - 2, -11:] = IGNORE_INDEX
    return d["X"], d["W"], t


@pytest.mark.parametrize("single_pass", [True, False])
@pytest.mark.parametrize("kind", KINDS)
def test_preference_loss_parity(kind, single_pass):
    from linear_cross_entropy_04_b200.preference import fused_linear_preference_loss

    X, W, t = _case()
    N, T = t.shape
    rng = np.random.default_rng(4)
    kw = {}
    if kind in ("dpo", "kto"):
        kw["ref_logps"] = rng.standard_normal(N) * 3 - 100
    if kind == "kto":
        kw["desirable"] = np.array([1, 0, 1, 1, 0, 0, 1, 0])
    ref = po.preference(kind, X, W, t, beta=0.1, gamma=0.5, lam=0.1, **kw)
    dkw = {k: torch.from_numpy(np.asarray(v)).cuda() for k, v in kw.items()}
    Xd = torch.from_numpy(X).to(torch.bfloat16).cuda().reshape(N, T, -1)
    Wd = torch.from_numpy(W).to(torch.bfloat16).cuda()
    loss, gX, gW = fused_linear_preference_loss(kind, Wd, Xd, torch.from_numpy(t).cuda(), beta=0.1, gamma=0.5,
                                                lam=0.1, single_pass=single_pass, **dkw)
    torch.cuda.synchronize()
    assert rel_err(loss.item(), ref["loss"]) <= 1e-3, (loss.item(), ref["loss"])
    assert_grad_close(gX.reshape(N * T, -1), ref["grad_X"], "bf16", f"{kind} grad_X")
    assert_grad_close(gW, ref["grad_W"], "bf16", f"{kind} grad_W")


def test_preference_module_matches_function():
    from linear_cross_entropy_04_b200.preference import FusedLinearORPOLoss

    X, W, t = _case(B=2, T=32, H=128, V=1000)
    N, T = t.shape
    Xd = torch.from_numpy(X).to(torch.bfloat16).cuda().reshape(N, T, -1).requires_grad_(True)
    Wd = torch.from_numpy(W).to(torch.bfloat16).cuda().requires_grad_(True)
    loss = FusedLinearORPOLoss(lam=0.2)(Wd, Xd, torch.from_numpy(t).cuda())
    loss.backward()
    ref = po.preference("orpo", X, W, t, lam=0.2)
    assert rel_err(loss.item(), ref["loss"]) <= 1e-3
    assert_grad_close(Xd.grad.reshape(N * T, -1), ref["grad_X"], "bf16", "orpo module grad_X")
    assert_grad_close(Wd.grad, ref["grad_W"], "bf16", "orpo module grad_W")


def test_single_pass_matches_two_pass():
    """The kept-store schedule and the recompute schedule give the same loss and
    gradients up to the order of grad_W's chunk additions."""
    from linear_cross_entropy_04_b200.preference import fused_linear_preference_loss

    X, W, t = _case(B=8, T=64, H=256, V=5000)  # 1024 tokens: two chunks in the recompute schedule
    N, T = t.shape
    Xd = torch.from_numpy(X).to(torch.bfloat16).cuda().reshape(N, T, -1)
    Wd = torch.from_numpy(W).to(torch.bfloat16).cuda()
    td = torch.from_numpy(t).cuda()
    l1, x1, w1 = fused_linear_preference_loss("simpo", Wd, Xd, td, single_pass=True)
    l2, x2, w2 = fused_linear_preference_loss("simpo", Wd, Xd, td, single_pass=False, chunk_rows=512)
    torch.cuda.synchronize()
    assert l1.item() == l2.item()
    assert torch.equal(x1, x2)  # grad_X rows do not depend on the chunking
    d = (w1.float() - w2.float()).abs().max().item()
    assert d <= 2 ** -7 * w2.float().abs().max().item(), d
