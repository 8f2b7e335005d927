"""Data-parallel fused linear cross-entropy over torch.distributed.

Each rank holds a replica of W and its own rows of X and targets (the FSDP /
DeepSpeed data-parallel setting the pages benchmark, "Liger-Kernel 項目詳細介紹",
性能基準測試: FSDP1 on 8 GPUs). Rows are independent except for three
exchanges, done with the process group's collectives (NCCL over NVLink on GPUs):

  1. all_reduce(N)      the mean denominator counts non-ignored rows of every
                        rank, and the in-place dlogits already divide by it;
  2. all_reduce(grad_W) (or reduce_scatter of its rows, for sharded grad_W);
                        on GPUs it starts on a side stream as soon as grad_W
                        is complete and overlaps the step's last grad_X GEMM;
  3. all_reduce(loss)   each rank's loss is its rows' sum / N, so the sum over
                        ranks is the global mean.

grad_X stays local. With fused_grad_W the third exchange disappears: the
grad_W GEMM adds each output box into the owner rank's shard itself (NVLink,
torch symmetric memory). The per-rank compute is the CUDA library; `count_fn`,
`flce_fn` and `shards` exist so that host-side tests can run the exchange
logic on CPU ranks with a stand-in compute.
"""
from __future__ import annotations

from typing import Callable, Optional

import torch
import torch.distributed as dist


def _lib_count(target, V, ignore_index):
    from .api import count_valid

    return count_valid(target, V, ignore_index)


def _lib_flce(X, W, target, ignore_index, reduction, n_valid, want_grad_X, want_grad_W, **kw):
    from .api import fused_linear_cross_entropy

    return fused_linear_cross_entropy(X, W, target, ignore_index=ignore_index, reduction=reduction,
                                      n_valid=n_valid, want_grad_X=want_grad_X, want_grad_W=want_grad_W, **kw)


def shard_rows_for(V: int, world: int) -> int:
    """Rows of grad_W each rank owns: V / world rounded up to a multiple of 32,
    so that no 32-row output box of the grad_W GEMM straddles two owners."""
    return ((-(-V // world)) + 31) // 32 * 32


def owned_rows(V: int, shard_rows: int, rank: int) -> int:
    """How many of rank's shard_rows are real grad_W rows (the last owners may hold fewer, or none)."""
    return max(0, min(shard_rows, V - rank * shard_rows))


class _PeerShards:
    """This rank's grad_W shard in symmetric memory and every rank's shard mapped
    here (buf, peers, shard_rows, rank, barrier(): the interface the fused path uses)."""

    def __init__(self, V, H, dtype, device, group):
        import torch.distributed._symmetric_memory as symm_mem

        world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.shard_rows = shard_rows_for(V, world)
        self.buf = symm_mem.empty(self.shard_rows, H, dtype=dtype, device=device)
        self.hdl = symm_mem.rendezvous(self.buf, group if group is not None else dist.group.WORLD)
        self.peers = [self.hdl.get_buffer(r, (self.shard_rows, H), dtype) for r in range(world)]
        self.V = V

    def barrier(self):
        self.hdl.barrier()  # device-side, on the current stream


_shards_cache = {}


def _peer_shards(V, H, dtype, device, group):
    key = (V, H, dtype, str(device), id(group))
    if key not in _shards_cache:
        _shards_cache[key] = _PeerShards(V, H, dtype, device, group)
    return _shards_cache[key]


def dp_fused_linear_cross_entropy(X: torch.Tensor, W: torch.Tensor, target: torch.Tensor,
                                  ignore_index: int = -100, reduction: str = "mean",
                                  group: Optional[dist.ProcessGroup] = None,
                                  want_grad_X: bool = True, want_grad_W: bool = True,
                                  shard_grad_W: bool = False, fused_grad_W: bool = False, shards=None,
                                  count_fn: Callable = _lib_count, flce_fn: Callable = _lib_flce, **kw):
    """Global loss, this rank's grad_X, and grad_W summed over ranks.

    reduction 'mean' divides by the non-ignored rows of all ranks; 'sum' sums
    over all ranks. With shard_grad_W, grad_W is reduce-scattered by rows and
    this rank gets rows [r*V/P, (r+1)*V/P) (V must divide by the world size).
    With fused_grad_W (GPUs only), the reduce-scatter happens inside the
    grad_W GEMM: each output tile is added, over NVLink, into the shard of the
    rank that owns its rows (torch symmetric memory), and this rank gets its
    shard, rows [r*S, (r+1)*S) with S = V/world rounded up to 32. The shards
    are zeroed before and read after a barrier across ranks. `shards` may
    supply them (buf, peers, shard_rows, rank, barrier()); by default they are
    symmetric-memory buffers.
    Every rank takes the same collective steps in the same order.
    reduction 'none' is refused (ValueError) before any collective: its
    per-row losses stay with their rank and there is no global loss to reduce.
    """
    if reduction not in ("mean", "sum"):
        raise ValueError(f"data-parallel reduction must be 'mean' or 'sum', not {reduction!r}")
    if fused_grad_W:
        return _dp_fused_grad_w(X, W, target, ignore_index, reduction, group, want_grad_X, shards, count_fn,
                                flce_fn, **kw)
    world = dist.get_world_size(group)
    if want_grad_W and shard_grad_W and W.shape[0] % world:
        raise ValueError("shard_grad_W needs V divisible by the world size")
    n_valid = None
    if reduction == "mean":
        n_valid = count_fn(target, W.shape[0], ignore_index).to(torch.int64).reshape(())
        dist.all_reduce(n_valid, group=group)
    # On GPUs the grad_W exchange starts as soon as grad_W is complete: the library
    # records an event there (the last chunk runs its grad_W GEMM before its grad_X
    # GEMM), and the collective runs on a side stream behind it, overlapping the
    # last grad_X GEMM. It is issued before the loss all-reduce, so every rank
    # issues the two in the same order and the loss's does not hold it back.
    overlap = (want_grad_W and flce_fn is _lib_flce and X.is_cuda and dist.get_backend(group) == "nccl"
               and kw.get("grad_w_shards") is None)
    ev = None
    if overlap:
        ev = torch.cuda.Event()
        kw = dict(kw, grad_w_ready_event=ev)
    loss, gX, gW = flce_fn(X, W, target, ignore_index, reduction, n_valid, want_grad_X, want_grad_W, **kw)
    loss = loss.reshape(())
    if want_grad_W:
        if overlap:
            main = torch.cuda.current_stream(X.device) if kw.get("stream") is None else kw["stream"]
            side = _side_stream(X.device)
            side.wait_event(ev)
            gW.record_stream(side)  # read by the collective on the side stream
            with torch.cuda.stream(side):
                gW = _exchange_grad_w(gW, shard_grad_W, group)
            main.wait_stream(side)
            gW.record_stream(main)
        else:
            gW = _exchange_grad_w(gW, shard_grad_W, group)
    dist.all_reduce(loss, group=group)
    return loss, gX, gW


_side_streams = {}


def _side_stream(device):
    key = str(device)
    if key not in _side_streams:
        _side_streams[key] = torch.cuda.Stream(device)
    return _side_streams[key]


def _exchange_grad_w(gW, shard_grad_W, group):
    """grad_W summed over ranks: all of it, or (shard_grad_W) this rank's V/world rows."""
    if not shard_grad_W:
        dist.all_reduce(gW, group=group)
        return gW
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    V = gW.shape[0]
    if dist.get_backend(group) == "gloo":
        # gloo has no reduce_scatter of one tensor: reduce all rows, keep ours
        dist.all_reduce(gW, group=group)
        return gW[rank * (V // world):(rank + 1) * (V // world)].clone()
    out = torch.empty_like(gW[: V // world])
    dist.reduce_scatter_tensor(out, gW.contiguous(), group=group)
    return out


def _dp_fused_grad_w(X, W, target, ignore_index, reduction, group, want_grad_X, shards, count_fn, flce_fn, **kw):
    V, H = W.shape
    sh = shards if shards is not None else _peer_shards(V, H, W.dtype, W.device, group)
    n_valid = None
    if reduction == "mean":
        n_valid = count_fn(target, V, ignore_index).to(torch.int64).reshape(())
        dist.all_reduce(n_valid, group=group)
    sh.buf.zero_()
    sh.barrier()  # every rank's shard is zero before any rank adds into it
    loss, gX, _ = flce_fn(X, W, target, ignore_index, reduction, n_valid, want_grad_X, False,
                          grad_w_shards=sh.peers, shard_rows=sh.shard_rows, **kw)
    sh.barrier()  # every rank's additions into this rank's shard have landed
    dist.all_reduce(loss, group=group)
    return loss, gX, sh.buf[:owned_rows(V, sh.shard_rows, sh.rank)]
