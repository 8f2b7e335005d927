"""The data-parallel paths on one rank, for real on one GPU: the fused grad_W
path's symmetric-memory calls (buffer, rendezvous, peer view, device barrier)
and the collective path's NCCL all-reduces and reduce-scatter.

With one rank the owner of every grad_W row is this rank, so the shard it
keeps must equal the plain path's grad_W bit for bit (the first chunk's adds
into the zeroed shard are exact, as the plain path's first store is), and the
loss and grad_X must be identical. Runs in a spawned child so the process
group does not outlive the test.
"""
import datetime
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _child(port, q):
    import sys

    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    from linear_cross_entropy_04_b200 import fused_linear_cross_entropy
    from linear_cross_entropy_04_b200.dp import dp_fused_linear_cross_entropy
    from linear_cross_entropy_04_b200.inputs import WORKLOADS, make_inputs

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        d = make_inputs(WORKLOADS["llama3_8b_seq"], BT=700, H=256, V=3000)
        X = torch.from_numpy(d["X"]).to(torch.bfloat16).cuda()
        W = torch.from_numpy(d["W"]).to(torch.bfloat16).cuda()
        t = torch.from_numpy(d["target"]).cuda()
        l1, x1, w1 = fused_linear_cross_entropy(X, W, t, chunk_rows=256)
        l2, x2, w2 = dp_fused_linear_cross_entropy(X, W, t, fused_grad_W=True, chunk_rows=256)
        # the collective path (NCCL all-reduces, and the reduce-scatter of sharded grad_W)
        l3, x3, w3 = dp_fused_linear_cross_entropy(X, W, t, chunk_rows=256)
        l4, x4, w4 = dp_fused_linear_cross_entropy(X, W, t, shard_grad_W=True, chunk_rows=256)
        ls, _, ws = fused_linear_cross_entropy(X, W, t, reduction="sum", chunk_rows=256)
        l5, _, w5 = dp_fused_linear_cross_entropy(X, W, t, reduction="sum", chunk_rows=256)
        torch.cuda.synchronize()
        collective = (float(l3) == float(l1) and torch.equal(x3, x1) and torch.equal(w3, w1) and
                      float(l4) == float(l1) and torch.equal(w4, w1) and
                      float(l5) == float(ls) and torch.equal(w5, ws))
        q.put(("ok", float(l1), float(l2), bool(torch.equal(x1, x2)), tuple(w2.shape), bool(torch.equal(w1, w2)),
               bool(collective)))
    except Exception as e:  # noqa: BLE001 - report, do not hang the parent
        q.put(("error", f"{type(e).__name__}: {e}"))
    finally:
        dist.destroy_process_group()


def test_data_parallel_paths_on_one_rank():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    p = ctx.Process(target=_child, args=(_free_port(), q))
    p.start()
    res = q.get(timeout=300)
    p.join(timeout=60)
    assert res[0] == "ok", res
    _, l1, l2, same_x, shape, same_w, collective = res
    assert l1 == l2 and same_x
    assert shape == (3000, 256) and same_w
    assert collective  # all-reduce and reduce-scatter paths equal the single-process call
    assert p.exitcode == 0


@pytest.mark.parametrize("exchange", ["reduce_scatter", "all_reduce", "fused"])
def test_bench_data_parallel_path_on_one_rank(exchange):
    """`bench.py --dp` takes the multi-GPU code path (process group, collectives,
    the chosen grad_W exchange, and, for the NCCL exchanges, the end-to-end run
    through HostPipeline with the data-parallel call) on one rank, and prints a
    complete line. A small workload keeps it short."""
    import json
    import subprocess
    import sys

    env = dict(os.environ, MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()), RANK="0", WORLD_SIZE="1",
               LOCAL_RANK="0")
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--dp", "--grad-w-exchange", exchange, "--BT", "2048",
           "--V", "32768", "--steps", "3", "--warmup", "3", "--no-cpu-baseline", "--e2e-steps", "3"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["n_gpus"] == 1 and line["device_error"] == 0 and line["value"] > 0
    assert line["config"]["grad_w_exchange"].startswith(
        {"reduce_scatter": "NCCL reduce-scatter", "all_reduce": "NCCL all-reduce", "fused": "fused"}[exchange])
    if exchange == "fused":
        assert line["e2e"] is None
    else:
        e2e = line["e2e"]
        assert "unavailable" not in e2e and e2e["value"] > 0
        assert e2e["h2d_bytes_per_step"] > 0 and e2e["d2h_bytes_per_step"] > 0
