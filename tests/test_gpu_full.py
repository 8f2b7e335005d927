"""Full-size workloads, in the launch configuration bench.py times.

What is compared, element by element, at the stated tolerances (loss: relative
error <= 1e-3; grad_X, grad_W: max |gpu - ref| <= 2e-2 * max |ref|):

  * the bench workload (Llama-3-8B lm_head, 4096 x 4096 x 128256) whole: the
    loss, every per-row loss and every element of grad_X and grad_W against
    the float64 oracle over the whole batch, on the stored-chunk schedule and
    on the recompute schedule (2 and 16 vocabulary chunks);
  * the four large workloads at full size with W = 0, in both grad_W
    accumulation modes: loss = ln V, grad_X = 0 exactly, and every element of
    grad_W against its closed form ((1/V) sum_valid X_i - sum_{valid, t_i = v}
    X_i) / N. This runs the full-size chunking of grad_W (2 to 16 chunks of
    2048 rows, each adding into the result) on every vocabulary row;
  * the four large workloads at full size: per-row loss and grad_X on a seeded
    sample of 256 rows (seed 1) against the oracle with the whole batch's N;
    ignored rows of grad_X are exactly 0; the loss is the mean of the per-row
    losses;
  * each large workload's recipe cut to its first 1024 tokens (same H, V,
    distribution and seed): loss, every row of grad_X and every vocabulary row
    of grad_W against the oracle;
  * the 16-chunk workload's recipe on 2048 tokens split into 16 chunks of 128
    rows, both accumulation modes: every element of grad_W against the oracle,
    with real (non-zero) weights.
"""
import numpy as np
import pytest
import torch

import oracle
from linear_cross_entropy_04_b200.inputs import WORKLOADS, make_inputs, sample_rows, IGNORE_INDEX
from flce_testlib import need_gpu, to_dev, rel_err, assert_grad_close, TOL

pytestmark = pytest.mark.gpu

FULL = ["llama3_8b_seq", "qwen2_7b", "llama3_8b_train", "large_vocab_stress"]


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()


def L():
    import linear_cross_entropy_04_b200 as lib

    return lib


def assert_close_blockwise(gpu, ref, name, tol=TOL["bf16"]["grad"], block=8192):
    """max |gpu - ref| <= tol * max |ref| for a device tensor against a host
    float64 array, moved to the host a block of rows at a time."""
    scale = float(np.abs(ref).max())
    err = 0.0
    for r0 in range(0, ref.shape[0], block):
        g = gpu[r0:r0 + block].double().cpu().numpy()
        err = max(err, float(np.abs(g - ref[r0:r0 + block]).max()))
    assert err <= tol * max(scale, 1e-30), f"{name}: max|err| {err:.3e} > {tol * scale:.3e} (max|ref| {scale:.3e})"
    return err / max(scale, 1e-30)


def test_bench_workload_whole_batch_against_the_oracle():
    """Every output of the bench workload, in its default plan (2 chunks of 2048 rows)."""
    w = WORKLOADS["llama3_8b_seq"]
    d = make_inputs(w)
    X, W, t = to_dev(d)
    row_loss = torch.empty(w.BT, dtype=torch.float32, device="cuda")
    loss, gX, gW, st = L().fused_linear_cross_entropy(X, W, t, row_loss=row_loss, return_stats=True)
    torch.cuda.synchronize()
    assert L().device_error() == 0
    assert st["n_chunks"] == 2 and st["chunk_rows"] == 2048
    ref = oracle.flce(d["X"], d["W"], d["target"], block_rows=1024)
    assert rel_err(loss.item(), ref["loss"]) <= 1e-3, (loss.item(), ref["loss"])
    np.testing.assert_allclose(row_loss.cpu().numpy(), ref["row_loss"], rtol=1e-3, atol=1e-3)
    assert_close_blockwise(gX, ref["grad_X"], "grad_X")
    assert_close_blockwise(gW, ref["grad_W"], "grad_W")
    # the recompute schedule on the same batch: its default (2 vocabulary chunks of
    # 65536 columns) and a 64 MiB store (16 chunks of 8192)
    for budget, n in ((0, 2), (64 << 20, 16)):
        loss, gX, gW, st = L().fused_linear_cross_entropy(X, W, t, row_loss=row_loss, schedule="recompute",
                                                           workspace_limit_bytes=budget, return_stats=True)
        torch.cuda.synchronize()
        assert L().device_error() == 0
        assert st["n_chunks"] == n
        assert rel_err(loss.item(), ref["loss"]) <= 1e-3, (loss.item(), ref["loss"])
        np.testing.assert_allclose(row_loss.cpu().numpy(), ref["row_loss"], rtol=1e-3, atol=1e-3)
        assert_close_blockwise(gX, ref["grad_X"], f"grad_X (recompute, {n} chunks)")
        assert_close_blockwise(gW, ref["grad_W"], f"grad_W (recompute, {n} chunks)")


_x_cache = {}


def _w_zero_inputs(name):
    """X and targets of the workload's recipe (the W draw is skipped: W = 0)."""
    if name not in _x_cache:
        _x_cache.clear()
        _x_cache[name] = make_inputs(WORKLOADS[name], w_zero=True)
    return _x_cache[name]


def _w_zero_grad_W(X, target, V, ignore_index=IGNORE_INDEX):
    """Closed form of grad_W at W = 0 (every logit 0, softmax uniform 1/V):
    grad_W[v] = ((1/V) * sum_valid X_i - sum_{valid, t_i = v} X_i) / N, in float64."""
    Xt = torch.from_numpy(X).double()
    tt = torch.from_numpy(target)
    valid = tt != ignore_index
    N = int(valid.sum())
    Xv = Xt[valid]
    ref = (Xv.sum(0) / V).expand(V, X.shape[1]).clone()
    ref.index_add_(0, tt[valid], Xv, alpha=-1.0)
    ref /= N
    return ref.numpy()


@pytest.mark.parametrize("accum", ["output", "fp32"])
@pytest.mark.parametrize("name", FULL)
def test_full_size_w_zero_closed_form(name, accum):
    w = WORKLOADS[name]
    d = _w_zero_inputs(name)
    X = torch.from_numpy(d["X"]).to(torch.bfloat16).cuda()
    t = torch.from_numpy(d["target"]).cuda()
    W = torch.zeros(w.V, w.H, dtype=torch.bfloat16, device="cuda")
    loss, gX, gW, st = L().fused_linear_cross_entropy(X, W, t, grad_w_accum=accum, return_stats=True)
    torch.cuda.synchronize()
    assert L().device_error() == 0
    assert st["n_chunks"] == -(-w.BT // 2048) and st["chunk_rows"] == 2048
    assert rel_err(loss.item(), np.log(w.V)) <= 1e-3, (loss.item(), np.log(w.V))
    assert torch.count_nonzero(gX).item() == 0
    del X, gX
    ref = _w_zero_grad_W(d["X"], d["target"], w.V)
    assert_close_blockwise(gW, ref, f"{name} grad_W (W = 0, {accum})")


@pytest.mark.parametrize("name", FULL)
def test_full_size_sampled(name):
    w = WORKLOADS[name]
    d = make_inputs(w)
    X, W, t = to_dev(d)
    row_loss = torch.empty(w.BT, dtype=torch.float32, device="cuda")
    loss, gX, gW = L().fused_linear_cross_entropy(X, W, t, row_loss=row_loss)
    torch.cuda.synchronize()
    assert L().device_error() == 0
    del gW
    N = oracle.count_valid(d["target"], w.V)
    rl = row_loss.cpu().numpy().astype(np.float64)
    assert rel_err(loss.item(), rl.sum() / N) <= 1e-5
    ign = torch.from_numpy(d["target"] == IGNORE_INDEX).cuda()
    assert torch.all(gX[ign] == 0)
    rows = sample_rows(w.BT)
    Wf = d["W"].astype(np.float64)
    ref = oracle.flce_rows(d["X"], Wf, d["target"], rows, n_valid=N)
    np.testing.assert_allclose(rl[rows], ref["row_loss"], rtol=1e-3, atol=1e-3)
    assert_grad_close(gX[torch.from_numpy(rows).cuda()], ref["grad_X"], "bf16", f"{name} grad_X sample")
    del X, gX
    torch.cuda.empty_cache()
    # the first 1024 tokens, whole: every row of grad_X, every vocabulary row of grad_W
    n = 1024
    Xs = torch.from_numpy(d["X"][:n]).to(torch.bfloat16).cuda()
    ts = torch.from_numpy(d["target"][:n]).cuda()
    ls, gXs, gWs = L().fused_linear_cross_entropy(Xs, W, ts)
    torch.cuda.synchronize()
    assert L().device_error() == 0
    refs = oracle.flce(d["X"][:n], Wf, d["target"][:n], block_rows=512)
    assert rel_err(ls.item(), refs["loss"]) <= 1e-3, (ls.item(), refs["loss"])
    assert_close_blockwise(gXs, refs["grad_X"], f"{name} grad_X (1024 tokens)")
    assert_close_blockwise(gWs, refs["grad_W"], f"{name} grad_W (1024 tokens)")


def test_sixteen_chunks_with_real_weights():
    """The 16-chunk workload's recipe on 2048 tokens in 16 chunks of 128 rows:
    grad_W accumulates 16 chunk sums, in bf16 and in the fp32 accumulator."""
    w = WORKLOADS["llama3_8b_train"]
    d = make_inputs(w, BT=2048)
    X, W, t = to_dev(d)
    ref = oracle.flce(d["X"], d["W"], d["target"], block_rows=512)
    for accum in ("output", "fp32"):
        loss, gX, gW, st = L().fused_linear_cross_entropy(X, W, t, chunk_rows=128, grad_w_accum=accum,
                                                           return_stats=True)
        torch.cuda.synchronize()
        assert L().device_error() == 0
        assert st["n_chunks"] == 16
        assert rel_err(loss.item(), ref["loss"]) <= 1e-3
        assert_close_blockwise(gX, ref["grad_X"], f"grad_X (16 chunks, {accum})")
        assert_close_blockwise(gW, ref["grad_W"], f"grad_W (16 chunks, {accum})")
