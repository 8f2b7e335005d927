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
    BT, H, V = 37, 6, (70 if case == "wide" else 20)
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


# ---- fused grad_W reduce-scatter: the host logic (shard sizes, zeroing, the two
# barriers, the slice each rank keeps), with CPU shards in shared memory standing
# in for symmetric memory and the oracle standing in for the device call, whose
# per-box adds into the owner shards are emulated under a lock (in L2 they are
# atomic element-wise adds).

def test_shard_sizes():
    from linear_cross_entropy_04_b200.dp import owned_rows, shard_rows_for

    assert shard_rows_for(128256, 8) == 16032 and shard_rows_for(70, 2) == 64 and shard_rows_for(20, 2) == 32
    for V, world in ((128256, 8), (152064, 3), (70, 2), (20, 2), (33, 4)):
        S = shard_rows_for(V, world)
        assert S % 32 == 0 and S * world >= V
        assert sum(owned_rows(V, S, r) for r in range(world)) == V


def test_none_reduction_is_refused_before_any_collective():
    """'none' has no global loss; the call fails at once, with no process group at all."""
    import torch

    from linear_cross_entropy_04_b200.dp import dp_fused_linear_cross_entropy

    X, W, t = torch.zeros(4, 8), torch.zeros(10, 8), torch.zeros(4, dtype=torch.int64)
    for fused in (False, True):
        with pytest.raises(ValueError, match="reduction"):
            dp_fused_linear_cross_entropy(X, W, t, reduction="none", fused_grad_W=fused)


class _CpuShards:
    """Shards in shared memory. The emulated device call adds into them from a
    background thread (device work is asynchronous); barrier() first waits for
    this rank's pending adds, as a device-side barrier orders after the work
    already on its stream, then meets the other ranks."""

    def __init__(self, bufs, rank, shard_rows):
        self.buf, self.peers, self.shard_rows, self.rank = bufs[rank], bufs, shard_rows, rank
        self.pending = []

    def barrier(self):
        import torch.distributed as dist

        for th in self.pending:
            th.join()
        self.pending.clear()
        dist.barrier()


def _bf16_chunked_grad_W(Xr, Wr, tr, ii, red, nv, n_chunks):
    """This rank's grad_W rounded as the device rounds it: each chunk's float64
    sum rounded to bf16; the chunks before the last added into a local bf16 sum
    (one rounding per add); the last chunk's box rounded, then the local sum
    added and the total rounded again."""
    import oracle

    X, W, t = Xr.numpy(), Wr.numpy(), tr.numpy()
    bf = lambda a: torch.from_numpy(np.asarray(a)).to(torch.bfloat16)  # noqa: E731
    bounds = np.linspace(0, X.shape[0], n_chunks + 1).astype(int)
    local = None
    for c in range(n_chunks):
        sl = slice(bounds[c], bounds[c + 1])
        g = bf(oracle.flce(X[sl], W, t[sl], ignore_index=ii, reduction=red, n_valid=nv, want_grad_X=False)["grad_W"])
        if c == n_chunks - 1:
            return g if local is None else (g.float() + local.float()).to(torch.bfloat16)
        local = g if local is None else (local.float() + g.float()).to(torch.bfloat16)


def _fused_worker(rank, world, port, reduction, bufs, lock, q, bf16=False):
    import sys
    import time

    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import oracle
    from linear_cross_entropy_04_b200.dp import dp_fused_linear_cross_entropy, owned_rows

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=30))
    try:
        X, W, t, split = _case("wide")
        V = W.shape[0]
        sl = slice(0, split) if rank == 0 else slice(split, None)
        count_fn, _ = _oracle_fns()

        shards = _CpuShards(bufs, rank, bufs[0].shape[0])

        def flce_fn(Xr, Wr, tr, ii, red, nv, want_gx, want_gw, grad_w_shards=None, shard_rows=0):
            import threading

            r = oracle.flce(Xr.numpy(), Wr.numpy(), tr.numpy(), ignore_index=ii, reduction=red,
                            n_valid=None if nv is None else int(nv))
            nvi = None if nv is None else int(nv)
            g = _bf16_chunked_grad_W(Xr, Wr, tr, ii, red, nvi, 4) if bf16 else torch.from_numpy(r["grad_W"])

            def adds():
                if rank == 1:
                    time.sleep(0.5)  # a slow rank: its adds land late
                with lock:
                    for k, shard in enumerate(grad_w_shards):
                        n = owned_rows(V, shard_rows, k)
                        # bf16 shards: the add is done in fp32 and rounded once, as the owner's L2 does
                        shard[:n] = (shard[:n].double() + g[k * shard_rows:k * shard_rows + n].double()).to(shard.dtype)

            th = threading.Thread(target=adds)
            th.start()
            shards.pending.append(th)
            return torch.tensor(r["loss"], dtype=torch.float64), torch.from_numpy(r["grad_X"]), None

        if rank == 1:
            time.sleep(0.5)  # late to zero its shard: rank 0 must not add into it before
        loss, gX, gW = dp_fused_linear_cross_entropy(
            torch.from_numpy(X[sl]), torch.from_numpy(W), torch.from_numpy(t[sl]), reduction=reduction,
            fused_grad_W=True, shards=shards, count_fn=count_fn, flce_fn=flce_fn)
        res = (rank, float(loss), gX.numpy(), gW.clone().double().numpy())
        for th in shards.pending:
            th.join()
        q.put(res)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("bf16", [False, True])
@pytest.mark.parametrize("reduction", ["mean", "sum"])
def test_dp_fused_grad_W_reduce_scatter_host_logic(reduction, bf16):
    """float64 shards: the exchange logic exactly (zeroing, both barriers, what each
    rank keeps). bf16 shards: the same with the device's roundings (4 chunks per
    rank summed locally in bf16, the last chunk's boxes plus that sum added into
    the owner's bf16 shard, ranks in either order), within the bf16 tolerance."""
    import oracle
    from linear_cross_entropy_04_b200.dp import shard_rows_for

    X, W, t, split = _case("wide")
    V, H = W.shape
    S = shard_rows_for(V, 2)
    ctx = mp.get_context("spawn")
    dt = torch.bfloat16 if bf16 else torch.float64
    bufs = [torch.full((S, H), float("nan"), dtype=dt).share_memory_() for _ in range(2)]
    lock = ctx.Lock()
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_fused_worker, args=(r, 2, port, reduction, bufs, lock, q, bf16)) for r in range(2)]
    for p in ps:
        p.start()
    out = {}
    for _ in range(2):
        r, loss, gX, gW = q.get(timeout=120)
        out[r] = (loss, gX, gW)
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    ref = oracle.flce(X, W, t, reduction=reduction)
    assert out[0][2].shape == (S, H) and out[1][2].shape == (V - S, H)
    for r in range(2):
        assert abs(out[r][0] - ref["loss"]) < 1e-12 * max(1.0, abs(ref["loss"]))
    joined = np.concatenate([out[0][2], out[1][2]])
    if bf16:
        assert np.isfinite(joined).all()
        err = np.abs(joined - ref["grad_W"]).max()
        assert err <= 2e-2 * np.abs(ref["grad_W"]).max(), err
    else:
        np.testing.assert_allclose(joined, ref["grad_W"], atol=1e-14)
    np.testing.assert_allclose(np.concatenate([out[0][1], out[1][1]]), ref["grad_X"], atol=1e-15)
