"""Pins for the float64 oracle, each independent of the oracle's own code.

The pages print no worked FLCE example, so the oracle is pinned by what the
mathematics fixes: closed forms (a hand-derived case, W = 0, V = 2), exact
invariants, central finite differences, a pure-Python brute force, and an
independent library routine (torch's float64 cross_entropy with autograd).
test_mutants_are_caught plants plausible mistakes in the oracle and checks
that at least one pin fails for each.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import flce_oracle as fo
from linear_cross_entropy_04_b200.inputs import WORKLOADS, make_inputs, sample_rows, IGNORE_INDEX


def _rand_case(BT=7, H=5, V=11, seed=3, ignore=(1,), scale=1.0):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((BT, H)) * scale
    W = rng.standard_normal((V, H)) * scale
    t = rng.integers(0, V, BT)
    for i in ignore:
        t[i] = IGNORE_INDEX
    return X, W, t


# ---------------------------------------------------------------- pin helpers
# Each pin takes an implementation impl(X, W, target, ignore_index, reduction)
# returning a dict with loss, grad_X, grad_W, and raises AssertionError on
# disagreement with what the mathematics fixes.

def pin_hand_case(impl):
    """z = [ln2, ln3, 0] for row 0 (target 2), row 1 ignored: loss = ln 6.

    softmax = [1/3, 1/2, 1/6] so dz_0 = [1/3, 1/2, -5/6] (N = 1), and with
    W = [[1,0],[0,1],[0,0]]: grad_X_0 = [1/3, 1/2], grad_W = dz_0^T X_0.
    """
    a, b = math.log(2.0), math.log(3.0)
    X = np.array([[a, b], [7.0, -3.0]])
    W = np.array([[1.0, 0.0], [0.0, 1.0], [0.0, 0.0]])
    t = np.array([2, IGNORE_INDEX])
    r = impl(X, W, t, IGNORE_INDEX, "mean")
    assert abs(r["loss"] - math.log(6.0)) < 1e-14
    np.testing.assert_allclose(r["grad_X"], [[1 / 3, 1 / 2], [0.0, 0.0]], rtol=0, atol=1e-15)
    dz = np.array([1 / 3, 1 / 2, -5 / 6])
    np.testing.assert_allclose(r["grad_W"], np.outer(dz, [a, b]), rtol=0, atol=1e-15)
    r = impl(X, W, t, IGNORE_INDEX, "sum")
    assert abs(r["loss"] - math.log(6.0)) < 1e-14


def pin_w_zero(impl):
    """W = 0: every logit is 0, so l_i = ln V, grad_X = 0 and
    grad_W[v] = (1/N) * ((1/V) * sum_valid X_i - sum_{valid, t_i = v} X_i)."""
    X, _, t = _rand_case(BT=13, H=4, V=9, ignore=(0, 5))
    W = np.zeros((9, 4))
    r = impl(X, W, t, IGNORE_INDEX, "mean")
    assert abs(r["loss"] - math.log(9)) < 1e-13
    assert np.all(r["grad_X"] == 0.0)
    valid = t != IGNORE_INDEX
    N = valid.sum()
    expect = np.tile(X[valid].sum(0) / 9.0, (9, 1))
    for i in np.nonzero(valid)[0]:
        expect[t[i]] -= X[i]
    np.testing.assert_allclose(r["grad_W"], expect / N, rtol=0, atol=1e-14)


def pin_v2_logistic(impl):
    """V = 2 reduces to the logistic loss log(1 + exp(-(z_t - z_o)))."""
    X, W, t = _rand_case(BT=6, H=3, V=2, ignore=())
    r = impl(X, W, t, IGNORE_INDEX, "sum")
    total = 0.0
    for i in range(6):
        zt = float(X[i] @ W[t[i]])
        zo = float(X[i] @ W[1 - t[i]])
        total += math.log1p(math.exp(-(zt - zo)))
    assert abs(r["loss"] - total) < 1e-12


def pin_torch_float64(impl):
    """torch's float64 cross_entropy of X W^T, differentiated by autograd."""
    for reduction in ("mean", "sum"):
        X, W, t = _rand_case(BT=9, H=6, V=13, ignore=(2, 3), seed=11)
        r = impl(X, W, t, IGNORE_INDEX, reduction)
        Xt = torch.tensor(X, requires_grad=True)
        Wt = torch.tensor(W, requires_grad=True)
        loss = torch.nn.functional.cross_entropy(Xt @ Wt.T, torch.tensor(t),
                                                 ignore_index=IGNORE_INDEX, reduction=reduction)
        loss.backward()
        assert abs(r["loss"] - loss.item()) < 1e-12 * max(1.0, abs(loss.item()))
        np.testing.assert_allclose(r["grad_X"], Xt.grad.numpy(), rtol=1e-10, atol=1e-14)
        np.testing.assert_allclose(r["grad_W"], Wt.grad.numpy(), rtol=1e-10, atol=1e-14)


def pin_finite_differences(impl):
    """Central differences, h = 1e-6, on a tiny float64 case with one ignored row."""
    X, W, t = _rand_case(BT=5, H=3, V=7, ignore=(1,), seed=5)
    for reduction in ("mean", "sum"):
        r = impl(X, W, t, IGNORE_INDEX, reduction)
        h = 1e-6

        def L(Xp, Wp):
            return impl(Xp, Wp, t, IGNORE_INDEX, reduction)["loss"]

        for M, g, other_first in ((X, r["grad_X"], True), (W, r["grad_W"], False)):
            num = np.zeros_like(M)
            for idx in np.ndindex(*M.shape):
                Mp, Mm = M.copy(), M.copy()
                Mp[idx] += h
                Mm[idx] -= h
                lp = L(Mp, W) if other_first else L(X, Mp)
                lm = L(Mm, W) if other_first else L(X, Mm)
                num[idx] = (lp - lm) / (2 * h)
            np.testing.assert_allclose(g, num, rtol=1e-6, atol=1e-9)


PINS = [pin_hand_case, pin_w_zero, pin_v2_logistic, pin_torch_float64, pin_finite_differences]


def _oracle_impl(X, W, t, ignore_index, reduction):
    return oracle.flce(X, W, t, ignore_index=ignore_index, reduction=reduction)


def _brute_impl(X, W, t, ignore_index, reduction):
    return oracle.flce_brute_force(X, W, t, ignore_index=ignore_index, reduction=reduction)


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_oracle_pins(pin):
    pin(_oracle_impl)


@pytest.mark.parametrize("pin", [pin_hand_case, pin_w_zero, pin_v2_logistic, pin_torch_float64],
                         ids=lambda p: p.__name__)
def test_brute_force_pins(pin):
    pin(_brute_impl)


# ------------------------------------------------------------ direct checks

def test_brute_force_matches_vectorised():
    for seed in range(4):
        X, W, t = _rand_case(BT=6, H=4, V=8, seed=seed, ignore=(seed % 6,))
        for red in ("mean", "sum"):
            a = oracle.flce(X, W, t, reduction=red)
            b = oracle.flce_brute_force(X, W, t, reduction=red)
            assert abs(a["loss"] - b["loss"]) < 1e-12
            np.testing.assert_allclose(a["grad_X"], b["grad_X"], rtol=0, atol=1e-12)
            np.testing.assert_allclose(a["grad_W"], b["grad_W"], rtol=0, atol=1e-12)


def test_dlogits_rows_sum_to_zero_and_ignored_rows_are_zero():
    X, W, t = _rand_case(BT=20, H=8, V=31, ignore=(0, 7, 19))
    dz = oracle.dlogits(oracle.logits(X, W), t)
    valid = t != IGNORE_INDEX
    assert np.all(np.abs(dz[valid].sum(1)) < 1e-15)
    assert np.all(dz[~valid] == 0.0)
    # the target entry is the only negative one in each valid row
    for i in np.nonzero(valid)[0]:
        assert dz[i, t[i]] < 0 and np.all(np.delete(dz[i], t[i]) > 0)


def test_ignored_rows_do_not_touch_grad_W_and_get_zero_grad_X():
    X, W, t = _rand_case(BT=12, H=6, V=10, ignore=(2, 9))
    a = oracle.flce(X, W, t)
    Xg = X.copy()
    Xg[[2, 9]] = 1e30 * np.random.default_rng(0).standard_normal((2, 6))
    b = oracle.flce(Xg, W, t)
    assert a["loss"] == b["loss"]
    np.testing.assert_array_equal(a["grad_W"], b["grad_W"])
    assert np.all(b["grad_X"][[2, 9]] == 0.0)


def test_invariances():
    X, W, t = _rand_case(BT=10, H=5, V=12, ignore=(4,), seed=9)
    base = oracle.flce(X, W, t)
    rng = np.random.default_rng(1)
    # row shift: W -> W + 1 c^T changes every logit of row i by X_i . c
    c = rng.standard_normal(5)
    r = oracle.flce(X, W + c[None, :], t)
    assert abs(r["loss"] - base["loss"]) < 1e-12
    np.testing.assert_allclose(r["grad_X"], base["grad_X"], atol=1e-12)
    # vocabulary permutation permutes grad_W rows only
    perm = rng.permutation(12)
    inv = np.argsort(perm)
    t2 = np.where(t == IGNORE_INDEX, t, inv[np.maximum(t, 0)])
    r = oracle.flce(X, W[perm], t2)
    assert abs(r["loss"] - base["loss"]) < 1e-12
    np.testing.assert_allclose(r["grad_W"], base["grad_W"][perm], atol=1e-14)
    np.testing.assert_allclose(r["grad_X"], base["grad_X"], atol=1e-14)
    # row permutation permutes grad_X rows only
    rp = rng.permutation(10)
    r = oracle.flce(X[rp], W, t[rp])
    assert abs(r["loss"] - base["loss"]) < 1e-12
    np.testing.assert_allclose(r["grad_X"], base["grad_X"][rp], atol=1e-14)
    np.testing.assert_allclose(r["grad_W"], base["grad_W"], atol=1e-14)
    # sum = N * mean
    s = oracle.flce(X, W, t, reduction="sum")
    N = base["n_valid"]
    assert abs(s["loss"] - N * base["loss"]) < 1e-12
    np.testing.assert_allclose(s["grad_W"], N * base["grad_W"], atol=1e-13)
    # sum of grad_W over the vocabulary is 0 (each dz row sums to 0)
    assert np.all(np.abs(base["grad_W"].sum(0)) < 1e-14)


def test_all_rows_ignored_reading():
    X, W, _ = _rand_case(BT=4, H=3, V=5)
    t = np.full(4, IGNORE_INDEX)
    r = oracle.flce(X, W, t)
    assert r["loss"] == 0.0 and r["n_valid"] == 0
    assert np.all(r["grad_X"] == 0) and np.all(r["grad_W"] == 0)


def test_target_range_and_in_range_ignore_index():
    X, W, t = _rand_case(BT=4, H=3, V=5, ignore=())
    bad = t.copy()
    bad[2] = 5
    with pytest.raises(ValueError):
        oracle.flce(X, W, bad)
    bad[2] = -1
    with pytest.raises(ValueError):
        oracle.flce(X, W, bad)
    # ignore_index inside [0, V): rows equal to it are ignored
    ii = int(t[0])
    r = oracle.flce(X, W, t, ignore_index=ii)
    keep = t != ii
    r2 = oracle.flce(X[keep], W, t[keep], ignore_index=IGNORE_INDEX)
    assert abs(r["loss"] - r2["loss"]) < 1e-14


def test_row_logsumexp_library_and_overflow():
    from scipy.special import logsumexp

    z = np.random.default_rng(2).standard_normal((6, 50)) * 30
    np.testing.assert_allclose(oracle.row_logsumexp(z), logsumexp(z, axis=1), rtol=1e-15, atol=1e-12)
    big = np.full((2, 4), 1000.0)
    np.testing.assert_allclose(oracle.row_logsumexp(big), 1000.0 + math.log(4.0), rtol=1e-15)


def test_logits_is_the_plain_dot_product():
    X, W, _ = _rand_case(BT=3, H=4, V=5)
    z = oracle.logits(X, W)
    for i in range(3):
        for v in range(5):
            assert abs(z[i, v] - sum(X[i, k] * W[v, k] for k in range(4))) < 1e-14


def test_block_rows_does_not_change_the_result():
    X, W, t = _rand_case(BT=37, H=6, V=19, ignore=(3, 30))
    a = oracle.flce(X, W, t, block_rows=4096)
    b = oracle.flce(X, W, t, block_rows=5)
    assert abs(a["loss"] - b["loss"]) < 1e-14
    np.testing.assert_allclose(a["grad_X"], b["grad_X"], atol=1e-15)
    np.testing.assert_allclose(a["grad_W"], b["grad_W"], atol=1e-14)


def test_flce_rows_matches_full_batch():
    X, W, t = _rand_case(BT=30, H=5, V=17, ignore=(1, 2, 20))
    full = oracle.flce(X, W, t)
    rows = np.array([0, 2, 5, 29])
    r = oracle.flce_rows(X, W, t, rows, n_valid=full["n_valid"])
    np.testing.assert_allclose(r["row_loss"], full["row_loss"][rows], atol=1e-14)
    np.testing.assert_allclose(r["grad_X"], full["grad_X"][rows], atol=1e-15)


def test_flce_grad_W_rows_matches_full():
    X, W, t = _rand_case(BT=25, H=4, V=19, ignore=(3,))
    full = oracle.flce(X, W, t)
    for red in ("mean", "sum"):
        full = oracle.flce(X, W, t, reduction=red)
        vr = np.array([0, 4, 18, int(t[0])])
        np.testing.assert_allclose(oracle.flce_grad_W_rows(X, W, t, vr, reduction=red),
                                   full["grad_W"][vr], atol=1e-15)


def test_cross_entropy_matches_torch_and_flce():
    X, W, t = _rand_case(BT=9, H=4, V=15, ignore=(0,))
    z = oracle.logits(X, W)
    ce = oracle.cross_entropy(z, t)
    zt = torch.tensor(z, requires_grad=True)
    loss = torch.nn.functional.cross_entropy(zt, torch.tensor(t), ignore_index=IGNORE_INDEX)
    loss.backward()
    assert abs(ce["loss"] - loss.item()) < 1e-13
    np.testing.assert_allclose(ce["dz"], zt.grad.numpy(), atol=1e-15)
    assert abs(ce["loss"] - oracle.flce(X, W, t)["loss"]) < 1e-14
    assert oracle.count_valid(t, 15) == 8


# ------------------------------------------------------------- mutation tests

def _mutants():
    """Plausible mistakes, each planted in one step of the oracle."""
    def lse_drops_max(z):
        z = np.asarray(z, dtype=np.float64)
        m = z.max(axis=1)
        return np.log(np.exp(z - m[:, None]).sum(axis=1))

    def onehot_sign(z, lse, target, valid, s):
        dz = np.exp(z - lse[:, None])
        rows = np.nonzero(valid)[0]
        dz[rows, target[rows]] += 1.0
        dz *= s
        dz[~valid] = 0.0
        return dz

    def ignored_not_zeroed(z, lse, target, valid, s):
        dz = np.exp(z - lse[:, None])
        rows = np.nonzero(valid)[0]
        dz[rows, target[rows]] -= 1.0
        return dz * s

    def target_off_by_one(z, rows, target):
        return z[rows, (target[rows] + 1) % z.shape[1]]

    def grad_X_transposed(dz, W):
        return (dz @ W[:, ::-1])

    def grad_W_wrong_operand(dz, X):
        return dz.T @ (X * 0.5)

    def scale_bt(reduction, n_valid):
        return 1.0 / (n_valid + 1) if reduction == "mean" else 1.0

    def logits_transposed(X, W):
        X = np.asarray(X, dtype=np.float64)
        W = np.asarray(W, dtype=np.float64)
        return X @ W[::-1].T

    return [
        ("row_logsumexp", lse_drops_max),
        ("_softmax_minus_onehot", onehot_sign),
        ("_softmax_minus_onehot", ignored_not_zeroed),
        ("_target_logits", target_off_by_one),
        ("_grad_X", grad_X_transposed),
        ("_grad_W", grad_W_wrong_operand),
        ("_scale", scale_bt),
        ("logits", logits_transposed),
    ]


@pytest.mark.parametrize("name,fn", _mutants(), ids=lambda x: x if isinstance(x, str) else x.__name__)
def test_mutants_are_caught(monkeypatch, name, fn):
    monkeypatch.setattr(fo, name, fn)
    caught = []
    for pin in PINS:
        try:
            pin(_oracle_impl)
        except (AssertionError, ValueError, IndexError):
            caught.append(pin.__name__)
    assert caught, f"no pin caught the planted mistake in {name} ({fn.__name__})"


# -------------------------------------------------------------- input recipe

def test_input_recipe():
    w = WORKLOADS["tiny"]
    a = make_inputs(w)
    b = make_inputs(w)
    np.testing.assert_array_equal(a["X"], b["X"])
    t = a["target"]
    assert (t == IGNORE_INDEX).sum() == round(0.05 * w.BT)
    assert t[t != IGNORE_INDEX].min() >= 0 and t.max() < w.V
    assert abs(a["W"].std() - 0.02) < 1e-3 and abs(a["X"].std() - 1.0) < 1e-2
    # bf16 rounding is exact: values survive a bf16 round trip unchanged
    z = make_inputs(WORKLOADS["qwen2_7b"], BT=300, H=64, V=1000)
    np.testing.assert_array_equal(
        z["X"], torch.from_numpy(z["X"]).to(torch.bfloat16).float().numpy())
    tz = z["target"][z["target"] != IGNORE_INDEX]
    assert np.mean(tz == 0) > 0.05  # Zipf: rank 1 is the most frequent token
    assert (z["target"] == IGNORE_INDEX).sum() == round(0.05 * 300)
    rows = sample_rows(4096)
    assert len(set(rows.tolist())) == 256 and rows.max() < 4096


def test_golden_tiny_regression():
    """The oracle still reproduces the values make_golden.py stored from it."""
    import json
    import os

    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "tiny_flce.json")))
    d = make_inputs(WORKLOADS["tiny"])
    for red in ("mean", "sum"):
        r = oracle.flce(d["X"], d["W"], d["target"], reduction=red)
        assert r["n_valid"] == g[red]["n_valid"]
        assert abs(r["loss"] - g[red]["loss"]) <= 1e-12 * abs(g[red]["loss"])
        np.testing.assert_allclose(r["row_loss"][:16], g[red]["row_loss_first16"], rtol=1e-12)
        np.testing.assert_allclose(r["grad_W"][:4, :8], g[red]["grad_W_rows0to3_first8"], rtol=1e-9, atol=1e-18)
    # loss of a near-uniform softmax over 4096 classes sits near ln 4096
    assert abs(g["mean"]["loss"] - math.log(4096)) < 0.3


def test_none_reduction_and_row_grad_against_torch():
    """reduction 'none' with an upstream gradient per row: torch float64 autograd."""
    X, W, t = _rand_case(BT=11, H=5, V=9, ignore=(2, 7), seed=21)
    g = np.random.default_rng(5).standard_normal(11)
    r = oracle.flce(X, W, t, reduction="none", row_grad=g)
    Xt = torch.tensor(X, requires_grad=True)
    Wt = torch.tensor(W, requires_grad=True)
    rows = torch.nn.functional.cross_entropy(Xt @ Wt.T, torch.tensor(t), ignore_index=IGNORE_INDEX,
                                             reduction="none")
    rows.backward(torch.tensor(g))
    np.testing.assert_allclose(r["loss"], rows.detach().numpy(), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(r["grad_X"], Xt.grad.numpy(), rtol=1e-10, atol=1e-14)
    np.testing.assert_allclose(r["grad_W"], Wt.grad.numpy(), rtol=1e-10, atol=1e-14)
    # weights of 1 give back the 'sum' gradients; weights 1/N the 'mean' ones
    s = oracle.flce(X, W, t, reduction="sum")
    n1 = oracle.flce(X, W, t, reduction="none", row_grad=np.ones(11))
    np.testing.assert_allclose(n1["grad_W"], s["grad_W"], atol=1e-15)
    m = oracle.flce(X, W, t, reduction="mean")
    nm = oracle.flce(X, W, t, reduction="sum", row_grad=np.full(11, 1.0 / m["n_valid"]))
    np.testing.assert_allclose(nm["grad_X"], m["grad_X"], atol=1e-15)


# ------------------------------------------------------------ preference losses

from oracle import preference_oracle as po  # noqa: E402

PREF = ["dpo", "orpo", "cpo", "simpo", "kto"]


def _pref_case(seed=0, B=2, T=4, H=3, V=6):
    rng = np.random.default_rng(seed)
    N = 2 * B
    X = rng.standard_normal((N * T, H))
    W = rng.standard_normal((V, H)) * 0.7
    t = rng.integers(0, V, (N, T))
    t[:, 0] = IGNORE_INDEX  # a prompt position in every sequence
    t[1, 3] = IGNORE_INDEX  # padding
    kw = {}
    return X, W, t, kw


def _pref_kw(kind, N, rng):
    if kind == "dpo":
        return {"ref_logps": rng.standard_normal(N)}
    if kind == "kto":
        return {"ref_logps": rng.standard_normal(N), "desirable": np.array([1, 0, 1, 1])}
    return {}


@pytest.mark.parametrize("kind", PREF)
def test_preference_finite_differences(kind):
    X, W, t, _ = _pref_case()
    kw = _pref_kw(kind, 4, np.random.default_rng(1))
    r = po.preference(kind, X, W, t, beta=0.7, **kw)
    h = 1e-6
    for M, g in ((X, r["grad_X"]), (W, r["grad_W"])):
        num = np.zeros_like(M)
        for idx in np.ndindex(*M.shape):
            Mp, Mm = M.copy(), M.copy()
            Mp[idx] += h
            Mm[idx] -= h
            args_p = (Mp, W) if M is X else (X, Mp)
            args_m = (Mm, W) if M is X else (X, Mm)
            lp = po.preference(kind, *args_p, t, beta=0.7, **kw)["loss"]
            lm = po.preference(kind, *args_m, t, beta=0.7, **kw)["loss"]
            num[idx] = (lp - lm) / (2 * h)
        np.testing.assert_allclose(g, num, rtol=1e-5, atol=1e-9)


def test_preference_closed_forms_for_identical_pairs():
    """Chosen == rejected: DPO/CPO pair term = log 2, SimPO = log(1 + e^gamma),
    ORPO = NLL + lam * log 2, KTO at r = z0 = 0.5."""
    X, W, t, _ = _pref_case(seed=3)
    N, T = t.shape
    B = N // 2
    X = X.reshape(N, T, -1)
    X[B:] = X[:B]
    t[B:] = t[:B]
    X = X.reshape(N * T, -1)
    base = oracle.flce(X, W, t.reshape(-1), reduction="none")
    valid = (t[:B] != IGNORE_INDEX)
    nll = base["row_loss"].reshape(N, T)[:B][valid].sum() / valid.sum()
    assert abs(po.preference("dpo", X, W, t)["loss"] - math.log(2)) < 1e-12
    assert abs(po.preference("cpo", X, W, t)["loss"] - (math.log(2) + nll)) < 1e-12
    g = 0.3
    assert abs(po.preference("simpo", X, W, t, gamma=g)["loss"] - math.log1p(math.exp(g))) < 1e-12
    assert abs(po.preference("orpo", X, W, t, lam=0.25)["loss"] - (nll + 0.25 * math.log(2))) < 1e-12
    # KTO: with ref = lp every r = 0 = z0, so every term is 1 - sigmoid(0)
    lp, _, _ = po.sequence_logps(base["row_loss"], t, N)
    assert abs(po.preference("kto", X, W, t, ref_logps=lp, desirable=np.array([1, 0, 1, 0]))["loss"] - 0.5) < 1e-12


@pytest.mark.parametrize("kind", PREF)
def test_preference_against_torch_float64(kind):
    X, W, t, _ = _pref_case(seed=5, B=3, T=5, H=4, V=7)
    rng = np.random.default_rng(2)
    kw = {"ref_logps": rng.standard_normal(6)} if kind in ("dpo", "kto") else {}
    if kind == "kto":
        kw["desirable"] = np.array([1, 1, 0, 1, 0, 0])
    r = po.preference(kind, X, W, t, beta=0.5, gamma=0.2, lam=0.3, **kw)
    Xt = torch.tensor(X, requires_grad=True)
    Wt = torch.tensor(W, requires_grad=True)
    rows = torch.nn.functional.cross_entropy(Xt @ Wt.T, torch.tensor(t.reshape(-1)), ignore_index=IGNORE_INDEX,
                                             reduction="none").reshape(6, 5)
    valid = torch.tensor(t != IGNORE_INDEX, dtype=torch.float64)
    lp = -(rows * valid).sum(1)
    c = valid.sum(1)
    ls = torch.nn.functional.logsigmoid
    if kind == "kto":
        rr = lp - torch.tensor(kw["ref_logps"])
        z0 = torch.clamp(rr.detach().mean(), min=0.0)
        s = torch.tensor(kw["desirable"], dtype=torch.float64) * 2 - 1
        L = (1 - torch.sigmoid(0.5 * s * (rr - z0))).mean()
    else:
        lw, ll, cw, cl = lp[:3], lp[3:], c[:3], c[3:]
        nll = (rows[:3] * valid[:3]).sum() / cw.sum()
        if kind == "dpo":
            ref = torch.tensor(kw["ref_logps"])
            L = -ls(0.5 * ((lw - ref[:3]) - (ll - ref[3:]))).mean()
        elif kind == "cpo":
            L = -ls(0.5 * (lw - ll)).mean() + nll
        elif kind == "simpo":
            L = -ls(0.5 * (lw / cw - ll / cl) - 0.2).mean()
        else:
            aw, al = lw / cw, ll / cl
            L = nll + 0.3 * -ls((aw - torch.log1p(-torch.exp(aw))) - (al - torch.log1p(-torch.exp(al)))).mean()
    L.backward()
    assert abs(r["loss"] - L.item()) < 1e-12
    np.testing.assert_allclose(r["grad_X"], Xt.grad.numpy(), rtol=1e-9, atol=1e-14)
    np.testing.assert_allclose(r["grad_W"], Wt.grad.numpy(), rtol=1e-9, atol=1e-14)


# ------------------------------------------------ preference-oracle mutations

def _pref_pins():
    def finite_differences():
        for k in PREF:
            test_preference_finite_differences(k)

    def closed_forms():
        test_preference_closed_forms_for_identical_pairs()

    def torch_float64():
        for k in PREF:
            test_preference_against_torch_float64(k)

    return [finite_differences, closed_forms, torch_float64]


def _pref_mutants():
    """Plausible mistakes in the preference oracle, each planted in one helper."""
    real_seq = po.sequence_logps
    real_ltg = po.loss_and_token_grad

    def logps_unmasked(row_loss, target, n_seq, ignore_index=-100):
        _, _, valid = real_seq(row_loss, target, n_seq, ignore_index)
        ones = np.ones_like(valid)
        return -np.asarray(row_loss, dtype=np.float64).reshape(n_seq, -1).sum(1), ones.sum(1), ones

    def logsig_sign(u):
        return -np.logaddexp(0.0, u)

    def sigmoid_flipped(u):
        return 1.0 / (1.0 + np.exp(u))

    def token_grad_sign(*a, **k):
        loss, g = real_ltg(*a, **k)
        return loss, -g

    def token_grad_halved(*a, **k):
        loss, g = real_ltg(*a, **k)
        return loss, 0.5 * g

    return [("sequence_logps", logps_unmasked), ("_logsig", logsig_sign), ("_sigmoid", sigmoid_flipped),
            ("loss_and_token_grad", token_grad_sign), ("loss_and_token_grad", token_grad_halved)]


@pytest.mark.parametrize("name,fn", _pref_mutants(), ids=lambda x: x if isinstance(x, str) else x.__name__)
def test_preference_mutants_are_caught(monkeypatch, name, fn):
    monkeypatch.setattr(po, name, fn)
    caught = []
    for pin in _pref_pins():
        try:
            pin()
        except (AssertionError, ValueError, IndexError, FloatingPointError):
            caught.append(pin.__name__)
    assert caught, f"no preference pin caught the planted mistake in {name} ({fn.__name__})"
