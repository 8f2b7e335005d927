"""Data-parallel exchange logic on CPU ranks (gloo, world size 2).

The per-rank compute is the float64 oracle, injected into
dp_fused_linear_cross_entropy by these tests only; the library's own path
computes on the GPU. Each rank holds a replica of W and its own rows; the
result must equal the oracle on the whole batch.
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _case(case):
    rng = np.random.default_rng(7)
    BT, H, V = 37, 6, 20
    X = rng.standard_normal((BT, H))
    W = rng.standard_normal((V, H)) * 0.5
    t = rng.integers(0, V, BT)
    t[[3, 9, 30]] = -100
    split = 12  # uneven: rank 0 gets 12 rows, rank 1 gets 25
    if case == "rank0_all_ignored":
        t[:split] = -100
    return X, W, t, split


def _oracle_fns():
    import oracle

    def count_fn(t, V, ii):
        return torch.tensor(oracle.count_valid(t.numpy(), V, ii), dtype=torch.int64)

    def flce_fn(X, W, t, ii, red, nv, want_gx, want_gw):
        r = oracle.flce(X.numpy(), W.numpy(), t.numpy(), ignore_index=ii, reduction=red,
                        n_valid=None if nv is None else int(nv))
        return (torch.tensor(r["loss"], dtype=torch.float64), torch.from_numpy(r["grad_X"]) if want_gx else None,
                torch.from_numpy(r["grad_W"]) if want_gw else None)

    return count_fn, flce_fn


def _worker(rank, world, port, case, reduction, shard, q):
    import sys

    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    from linear_cross_entropy_04_b200.dp import dp_fused_linear_cross_entropy

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=30))
    try:
        X, W, t, split = _case(case)
        sl = slice(0, split) if rank == 0 else slice(split, None)
        count_fn, flce_fn = _oracle_fns()
        loss, gX, gW = dp_fused_linear_cross_entropy(
            torch.from_numpy(X[sl]), torch.from_numpy(W), torch.from_numpy(t[sl]), reduction=reduction,
            shard_grad_W=shard, count_fn=count_fn, flce_fn=flce_fn)
        q.put((rank, float(loss), gX.numpy(), gW.numpy()))
    finally:
        dist.destroy_process_group()


def _run(case, reduction, shard=False):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_worker, args=(r, 2, port, case, reduction, shard, q)) for r in range(2)]
    for p in ps:
        p.start()
    out = {}
    for _ in range(2):
        r, loss, gX, gW = q.get(timeout=120)
        out[r] = (loss, gX, gW)
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    return out


@pytest.mark.parametrize("case", ["plain", "rank0_all_ignored"])
@pytest.mark.parametrize("reduction", ["mean", "sum"])
def test_dp_matches_single_process_oracle(case, reduction):
    import oracle

    X, W, t, split = _case(case)
    ref = oracle.flce(X, W, t, reduction=reduction)
    out = _run(case, reduction)
    for r in range(2):
        assert abs(out[r][0] - ref["loss"]) < 1e-12 * max(1.0, abs(ref["loss"]))
        np.testing.assert_allclose(out[r][2], ref["grad_W"], atol=1e-14)
    np.testing.assert_allclose(np.concatenate([out[0][1], out[1][1]]), ref["grad_X"], atol=1e-15)


def test_dp_sharded_grad_W():
    import oracle

    X, W, t, split = _case("plain")
    ref = oracle.flce(X, W, t)
    out = _run("plain", "mean", shard=True)
    np.testing.assert_allclose(np.concatenate([out[0][2], out[1][2]]), ref["grad_W"], atol=1e-14)


def _dying_worker(rank, world, port, q):
    import sys

    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    from linear_cross_entropy_04_b200.dp import dp_fused_linear_cross_entropy

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=4))
    if rank == 1:
        os._exit(3)  # this rank fails before its first collective
    X, W, t, split = _case("plain")
    count_fn, flce_fn = _oracle_fns()
    try:
        dp_fused_linear_cross_entropy(torch.from_numpy(X[:split]), torch.from_numpy(W), torch.from_numpy(t[:split]),
                                      count_fn=count_fn, flce_fn=flce_fn)
        q.put("no error")
    except Exception as e:  # noqa: BLE001 - the collective must fail, not hang
        q.put("error: " + type(e).__name__)


def test_a_dead_rank_makes_the_next_collective_fail_instead_of_hanging():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_dying_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    msg = q.get(timeout=90)
    for p in ps:
        p.join(timeout=30)
        if p.is_alive():
            p.kill()
    assert msg.startswith("error"), msg
