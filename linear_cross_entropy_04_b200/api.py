"""Public Python API over the C ABI (argument marshalling only).

fused_linear_cross_entropy(X, W, target) runs the whole path (loss, grad_X,
grad_W) in the CUDA library in one call. FusedLinearCrossEntropyLoss mirrors
the low-level API of "Liger-Kernel 項目詳細介紹" (使用方法 > 3. 低級 API 方式):
loss_fn(lm_head.weight, input, target) followed by loss.backward().
"""
from __future__ import annotations

import contextlib
import ctypes
from typing import Optional

import torch

from . import _binding as B

_RED = {"mean": B.MEAN, "sum": B.SUM, "none": B.NONE}
_ACC = {"output": B.GRADW_ACCUM_OUTPUT, "fp32": B.GRADW_ACCUM_FP32}


_SCHED = {"stored": 0, "recompute": B.FLAG_RECOMPUTE}


def _check_reduction(reduction):
    if reduction not in _RED:
        raise ValueError(f"reduction must be one of {sorted(_RED)}, not {reduction!r}")


def _schedule_flag(schedule):
    if schedule not in _SCHED:
        raise ValueError(f"schedule must be one of {sorted(_SCHED)}, not {schedule!r}")
    return _SCHED[schedule]


def _options(chunk_rows=0, workspace_limit_bytes=0, grad_w_accum="output", flags=0,
             n_valid=None, row_loss=None, lse=None, workspace=None, row_grad=None):
    o = B.FlceOptions()
    B.lib().flce_options_init(ctypes.byref(o))
    o.chunk_rows = int(chunk_rows)
    o.workspace_limit_bytes = int(workspace_limit_bytes)
    if grad_w_accum not in _ACC:
        raise ValueError(f"grad_w_accum must be one of {sorted(_ACC)}, not {grad_w_accum!r}")
    o.grad_w_accum = _ACC[grad_w_accum]
    o.flags = int(flags)
    o.n_valid = None if n_valid is None else n_valid.data_ptr()
    o.row_loss = None if row_loss is None else row_loss.data_ptr()
    o.lse = None if lse is None else lse.data_ptr()
    o.row_grad = None if row_grad is None else row_grad.data_ptr()
    if workspace is not None:
        o.workspace = workspace.data_ptr()
        o.workspace_bytes = workspace.numel() * workspace.element_size()
    return o


def fused_linear_cross_entropy(X: torch.Tensor, W: torch.Tensor, target: torch.Tensor,
                               ignore_index: int = -100, reduction: str = "mean",
                               want_grad_X: bool = True, want_grad_W: bool = True,
                               chunk_rows: int = 0, workspace_limit_bytes: int = 0,
                               grad_w_accum: str = "output", n_valid: Optional[torch.Tensor] = None,
                               row_loss: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                               row_grad: Optional[torch.Tensor] = None, grad_w_shards=None,
                               shard_rows: int = 0, schedule: str = "stored",
                               flags: int = 0, stream=None, out=None, host_out=None,
                               return_stats: bool = False, grad_w_ready_event=None):
    """Loss, grad_X and grad_W of cross-entropy over X W^T in one call.

    X [BT, H] and W [V, H] (bf16 or fp32, CUDA), target [BT] int64.
    reduction 'mean' | 'sum' | 'none' ('none': loss is the [BT] per-row losses).
    row_grad [BT] fp32 scales each row's contribution to the gradients (the
    upstream gradient of the per-row losses); default all ones.
    grad_w_shards: a list of bf16 [shard_rows, H] tensors (local or mapped
    from peer GPUs); shard k owns grad_W rows [k*shard_rows, (k+1)*shard_rows)
    and each grad_W tile is added into its owner shard as it is produced
    (no grad_W tensor is returned then). The caller zeroes the shards first.
    Tensors on the host are staged to the current CUDA device and the
    results copied back (the end-to-end path); nothing runs on the CPU.
    host_out = (loss, grad_X, grad_W) pinned host tensors receive them then.
    out = (loss, grad_X, grad_W) preallocated device tensors may be given.
    The library's workspace is taken from torch's caching allocator.
    schedule 'stored' (default) chunks the rows and keeps each chunk's logits
    store (6*BT*H*V tensor FLOPs); 'recompute' chunks the vocabulary, computes
    every row's logsumexp first and rebuilds the logits per vocabulary chunk
    (8*BT*H*V tensor FLOPs; the store is [BT, chunk_rows] with chunk_rows read
    as vocabulary columns, or sized from workspace_limit_bytes).
    grad_w_ready_event (a torch.cuda.Event) is recorded on the call's stream as
    soon as grad_W is complete: in the row-chunked schedule the last chunk runs
    its grad_W GEMM before its grad_X GEMM, so that work queued on another stream
    behind the event (a grad_W reduction across ranks) overlaps the grad_X GEMM.
    Returns (loss [scalar fp32], grad_X or None, grad_W or None[, stats]).
    """
    _check_reduction(reduction)
    flags = int(flags) | _schedule_flag(schedule)
    host = not X.is_cuda
    if host:
        dev = torch.device("cuda", torch.cuda.current_device())
        X = X.to(dev, non_blocking=True)
        W = W.to(dev, non_blocking=True)
        target = target.to(dev, non_blocking=True)
    if out is not None:
        loss, gX, gW = out
    else:
        loss = torch.empty((X.shape[0],) if reduction == "none" else (), dtype=torch.float32, device=X.device)
        gX = torch.empty_like(X) if want_grad_X else None
        gW = torch.empty_like(W) if want_grad_W and grad_w_shards is None else None
    if row_grad is not None:
        row_grad = row_grad.to(device=X.device, dtype=torch.float32).contiguous()
    o = _options(chunk_rows, workspace_limit_bytes, grad_w_accum, flags, n_valid, row_loss, lse,
                 row_grad=row_grad)
    if grad_w_ready_event is not None:
        if not grad_w_ready_event.cuda_event:  # torch creates its CUDA event at the first record
            grad_w_ready_event.record(torch.cuda.current_stream(X.device) if stream is None else stream)
        o.grad_w_ready_event = grad_w_ready_event.cuda_event
    if grad_w_shards is not None:
        shard_ptrs = (ctypes.c_void_p * len(grad_w_shards))(*[t_.data_ptr() for t_ in grad_w_shards])
        o.grad_w_shards = ctypes.cast(shard_ptrs, ctypes.POINTER(ctypes.c_void_p))
        o.n_shards = len(grad_w_shards)
        o.shard_rows = int(shard_rows)
        o.grad_w_shard_ld = grad_w_shards[0].stride(0)
    st = B.FlceStats()
    B.check(B.lib().flce_plan(X.shape[0], X.shape[1], W.shape[0], B.dtype_code(X),
                              int(gW is not None or grad_w_shards is not None),
                              ctypes.byref(o), ctypes.byref(st)), "flce_plan")
    ws = None
    if st.workspace_bytes > 0:
        ws = torch.empty(st.workspace_bytes, dtype=torch.uint8, device=X.device)
        o.workspace = ws.data_ptr()
        o.workspace_bytes = st.workspace_bytes
    tX, tW, tt, tl = B.tensor(X), B.tensor(W), B.tensor(target), B.tensor(loss)
    tgX = B.tensor(gX) if gX is not None else None
    tgW = B.tensor(gW) if gW is not None else None
    rc = B.lib().flce_fwd_bwd_ex(ctypes.byref(tX), ctypes.byref(tW), ctypes.byref(tt), int(ignore_index),
                                 _RED[reduction], ctypes.byref(tl),
                                 ctypes.byref(tgX) if tgX is not None else None,
                                 ctypes.byref(tgW) if tgW is not None else None,
                                 B.stream_handle(stream), ctypes.byref(o), ctypes.byref(st))
    B.check(rc, "flce_fwd_bwd_ex")
    if ws is not None and stream is not None:
        ws.record_stream(stream)  # allocated on the current stream, used on `stream`
    if host:
        if host_out is not None:
            hl, hx, hw = host_out
            hl.copy_(loss, non_blocking=True)
            if gX is not None:
                hx.copy_(gX, non_blocking=True)
            if gW is not None:
                hw.copy_(gW, non_blocking=True)
            torch.cuda.current_stream().synchronize()
            loss, gX, gW = hl, (hx if gX is not None else None), (hw if gW is not None else None)
        else:
            loss = loss.to("cpu", non_blocking=False)
            gX = gX.cpu() if gX is not None else None
            gW = gW.cpu() if gW is not None else None
    res = (loss, gX, gW)
    return res + (st.as_dict(),) if return_stats else res


class KeptLogits:
    """What forward_keep leaves for backward_from_kept: the device workspace that
    holds the batch's store of exp(z - m_tile), its tile maxima and row lse,
    with the inputs it was computed from. Nothing else may use the workspace
    until the gradients are taken."""

    def __init__(self, X, W, target, ignore_index, workspace, n_valid):
        self.X, self.W, self.target = X, W, target
        self.ignore_index = ignore_index
        self.workspace = workspace
        self.n_valid = n_valid


def keep_workspace_bytes(BT: int, H: int, V: int, dtype: str = "bf16", want_grad_W: bool = True) -> int:
    """Workspace a forward_keep / backward_from_kept pair needs (the whole batch as one chunk)."""
    o = _options(flags=B.FLAG_KEEP_LOGITS)
    st = B.FlceStats()
    B.check(B.lib().flce_plan(BT, H, V, B.BF16 if dtype == "bf16" else B.F32, int(want_grad_W),
                              ctypes.byref(o), ctypes.byref(st)), "flce_plan")
    return st.workspace_bytes


def forward_keep(X: torch.Tensor, W: torch.Tensor, target: torch.Tensor, ignore_index: int = -100,
                 reduction: str = "mean", n_valid: Optional[torch.Tensor] = None,
                 lse: Optional[torch.Tensor] = None, stream=None):
    """Loss of cross-entropy over X W^T with the batch's chunk store kept for
    backward_from_kept (FLCE_FLAG_KEEP_LOGITS). Returns (loss, KeptLogits)."""
    _check_reduction(reduction)
    loss = torch.empty((X.shape[0],) if reduction == "none" else (), dtype=torch.float32, device=X.device)
    o = _options(flags=B.FLAG_KEEP_LOGITS, n_valid=n_valid, lse=lse)
    st = B.FlceStats()
    B.check(B.lib().flce_plan(X.shape[0], X.shape[1], W.shape[0], B.dtype_code(X), 1, ctypes.byref(o),
                              ctypes.byref(st)), "flce_plan")
    ws = torch.empty(max(st.workspace_bytes, 256), dtype=torch.uint8, device=X.device)
    o.workspace = ws.data_ptr()
    o.workspace_bytes = ws.numel()
    tX, tW, tt, tl = B.tensor(X), B.tensor(W), B.tensor(target), B.tensor(loss)
    B.check(B.lib().flce_fwd_bwd_ex(ctypes.byref(tX), ctypes.byref(tW), ctypes.byref(tt), int(ignore_index),
                                    _RED[reduction], ctypes.byref(tl), None, None, B.stream_handle(stream),
                                    ctypes.byref(o), None), "flce_fwd_bwd_ex (keep)")
    if stream is not None:
        ws.record_stream(stream)  # allocated on the current stream, used on `stream`
    return loss, KeptLogits(X, W, target, ignore_index, ws, n_valid)


def backward_from_kept(kept: KeptLogits, reduction: str = "mean", row_grad: Optional[torch.Tensor] = None,
                       want_grad_X: bool = True, want_grad_W: bool = True, stream=None):
    """grad_X, grad_W from a forward_keep (FLCE_FLAG_FROM_KEPT): the gradients
    of sum_i row_grad_i * l_i * (1/N or 1) without running the logits GEMM again.
    The kept workspace is released afterwards."""
    _check_reduction(reduction)
    X, W, t = kept.X, kept.W, kept.target
    if kept.workspace is None:
        raise RuntimeError("the kept logits were already used")
    gX = torch.empty_like(X) if want_grad_X else None
    gW = torch.empty_like(W) if want_grad_W else None
    if row_grad is not None:
        row_grad = row_grad.to(device=X.device, dtype=torch.float32).contiguous()
    o = _options(flags=B.FLAG_FROM_KEPT, n_valid=kept.n_valid, workspace=kept.workspace, row_grad=row_grad)
    dummy = torch.empty((X.shape[0],) if reduction == "none" else (), dtype=torch.float32, device=X.device)
    tX, tW, tt, tl = B.tensor(X), B.tensor(W), B.tensor(t), B.tensor(dummy)
    tgX = B.tensor(gX) if gX is not None else None
    tgW = B.tensor(gW) if gW is not None else None
    B.check(B.lib().flce_fwd_bwd_ex(ctypes.byref(tX), ctypes.byref(tW), ctypes.byref(tt), int(kept.ignore_index),
                                    _RED[reduction], ctypes.byref(tl),
                                    ctypes.byref(tgX) if tgX is not None else None,
                                    ctypes.byref(tgW) if tgW is not None else None,
                                    B.stream_handle(stream), ctypes.byref(o), None), "flce_fwd_bwd_ex (from kept)")
    # the workspace was allocated on the forward's stream; keep the allocator
    # from reusing it before this call's kernels, possibly on another stream, finish
    kept.workspace.record_stream(stream if stream is not None else torch.cuda.current_stream(X.device))
    kept.workspace = None
    return gX, gW


def cross_entropy(logits: torch.Tensor, target: torch.Tensor, ignore_index: int = -100,
                  reduction: str = "mean", want_grad: bool = True, inplace: bool = False,
                  n_valid: Optional[torch.Tensor] = None, row_loss: Optional[torch.Tensor] = None,
                  lse: Optional[torch.Tensor] = None, row_grad: Optional[torch.Tensor] = None, stream=None):
    """Cross-entropy of given logits [BT, V]; the gradient may replace the logits in place.

    The kernels read and write rows in 16-byte vectors. Logits whose rows are
    not 16-byte aligned (a contiguous [BT, V] with V not a multiple of 8 for
    bf16, of 4 for fp32) are staged through a copy with padded rows, and an
    in-place gradient is copied back into them."""
    _check_reduction(reduction)
    caller_logits = None
    if logits.dim() == 2 and logits.shape[0] > 0 and not _rows_16b_aligned(logits):
        caller_logits = logits if (want_grad and inplace) else None
        per = 16 // logits.element_size()
        V = logits.shape[1]
        buf = torch.empty((logits.shape[0], V + (-V) % per), dtype=logits.dtype, device=logits.device)
        with torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext():
            buf[:, :V].copy_(logits)
        logits = buf[:, :V]
    loss = torch.empty((logits.shape[0],) if reduction == "none" else (), dtype=torch.float32,
                       device=logits.device)
    grad = None
    if want_grad:
        grad = logits if inplace else torch.empty_strided(logits.size(), logits.stride(), dtype=logits.dtype,
                                                          device=logits.device)
    if row_grad is not None:
        row_grad = row_grad.to(device=logits.device, dtype=torch.float32).contiguous()
    o = _options(n_valid=n_valid, row_loss=row_loss, lse=lse, row_grad=row_grad)
    tz, tt, tl = B.tensor(logits), B.tensor(target), B.tensor(loss)
    tg = B.tensor(grad) if grad is not None else None
    rc = B.lib().flce_cross_entropy(ctypes.byref(tz), ctypes.byref(tt), int(ignore_index), _RED[reduction],
                                    ctypes.byref(tl), ctypes.byref(tg) if tg is not None else None,
                                    B.stream_handle(stream), ctypes.byref(o))
    B.check(rc, "flce_cross_entropy")
    if caller_logits is not None:
        with torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext():
            caller_logits.copy_(grad)
        grad = caller_logits
    return loss, grad


def _rows_16b_aligned(t: torch.Tensor) -> bool:
    return t.data_ptr() % 16 == 0 and (t.stride(0) * t.element_size()) % 16 == 0 and t.stride(-1) == 1


def count_valid(target: torch.Tensor, V: int, ignore_index: int = -100, stream=None) -> torch.Tensor:
    """N (int64 device scalar): rows whose target is not ignore_index."""
    n = torch.empty((), dtype=torch.int64, device=target.device)
    tt = B.tensor(target)
    B.check(B.lib().flce_count_valid(ctypes.byref(tt), int(V), int(ignore_index), B.ptr(n),
                                     B.stream_handle(stream)), "flce_count_valid")
    return n


def gemm_bf16(A: torch.Tensor, Bm: torch.Tensor, M: int, N: int, K: int, a_mn_major: bool,
              b_mn_major: bool, stream=None) -> torch.Tensor:
    """C[M,N] fp32 = sum_k A(m,k) B(n,k) on the tcgen05 engine (a test hook)."""
    C = torch.empty((M, N), dtype=torch.float32, device=A.device)
    rc = B.lib().flce_gemm_bf16(B.ptr(A), B.ptr(Bm), B.ptr(C), M, N, K, A.stride(0), Bm.stride(0),
                                C.stride(0), int(a_mn_major), int(b_mn_major), B.stream_handle(stream))
    B.check(rc, "flce_gemm_bf16")
    return C


def scale_grad_(t: torch.Tensor, scale: torch.Tensor, stream=None) -> torch.Tensor:
    """t *= scale in place, scale a one-element fp32 device tensor; nothing is
    read or written when it is exactly 1, and the host never waits for it."""
    if scale.dtype != torch.float32 or scale.device != t.device or scale.numel() != 1:
        scale = scale.to(device=t.device, dtype=torch.float32)
    scale = scale.reshape(())
    tt = B.tensor(t)
    B.check(B.lib().flce_scale_grad(ctypes.byref(tt), B.ptr(scale), B.stream_handle(stream)), "flce_scale_grad")
    return t


def plan(BT: int, H: int, V: int, dtype: str = "bf16", want_grad_W: bool = True,
         chunk_rows: int = 0, workspace_limit_bytes: int = 0, grad_w_accum: str = "output",
         schedule: str = "stored") -> dict:
    """Chunk rows (vocabulary columns for schedule 'recompute'), chunk count and
    workspace bytes for a shape (host only)."""
    o = _options(chunk_rows, workspace_limit_bytes, grad_w_accum, flags=_schedule_flag(schedule))
    st = B.FlceStats()
    rc = B.lib().flce_plan(BT, H, V, B.BF16 if dtype == "bf16" else B.F32, int(want_grad_W),
                           ctypes.byref(o), ctypes.byref(st))
    B.check(rc, "flce_plan")
    return st.as_dict()


def device_error(stream=None) -> int:
    """Read and clear the device error word (synchronises the stream)."""
    e = ctypes.c_uint32(0)
    B.check(B.lib().flce_get_device_error(B.stream_handle(stream), ctypes.byref(e)), "flce_get_device_error")
    return e.value


def phase_times(reset: bool = True) -> dict:
    """{phase name: (milliseconds, launches)} for calls made with FLAG_TIME_PHASES."""
    ms = (ctypes.c_double * B.NUM_PHASES)()
    cnt = (ctypes.c_int32 * B.NUM_PHASES)()
    B.check(B.lib().flce_phase_times(ms, cnt, B.NUM_PHASES, int(reset)), "flce_phase_times")
    return {B.PHASE_NAMES[i]: (ms[i], cnt[i]) for i in range(B.NUM_PHASES)}


class _FLCEFunction(torch.autograd.Function):
    """'mean' / 'sum': the forward computes the loss and both gradients at
    once, and backward hands them back scaled by the upstream gradient, in
    place and on the device (flce_scale_grad), so backward never waits for the
    GPU. The saved gradients are handed out once: a second backward through
    the same graph raises instead of scaling them a second time.
    'none': the forward computes only the per-row losses; backward runs the
    fused path again with the per-row upstream gradient (row_grad), so the
    logits GEMM is done twice in exchange for never storing dlogits. With
    keep_logits the forward keeps the batch's bf16 store instead (held until
    backward) and backward takes the gradients from it."""

    @staticmethod
    def forward(ctx, weight, inp, target, ignore_index, reduction, grad_w_accum, keep_logits=False):
        shape = inp.shape
        X = inp.reshape(-1, shape[-1])
        if X.stride(-1) != 1 or (X.stride(0) % 8 and X.dtype == torch.bfloat16):
            X = X.contiguous()
        t = target.reshape(-1)
        ctx.shape = shape
        ctx.reduction = reduction
        ctx.ignore_index = ignore_index
        ctx.grad_w_accum = grad_w_accum
        if reduction == "none":
            ctx.need = (ctx.needs_input_grad[1], ctx.needs_input_grad[0])
            ctx.kept = None
            if keep_logits:
                loss, ctx.kept = forward_keep(X, weight, t, ignore_index=ignore_index, reduction="none")
                return loss.reshape(shape[:-1])
            loss, _, _ = fused_linear_cross_entropy(X, weight, t, ignore_index=ignore_index, reduction="none",
                                                    want_grad_X=False, want_grad_W=False)
            ctx.save_for_backward(X, weight, t)
            return loss.reshape(shape[:-1])
        loss, gX, gW = fused_linear_cross_entropy(
            X, weight, t, ignore_index=ignore_index, reduction=reduction,
            want_grad_X=ctx.needs_input_grad[1], want_grad_W=ctx.needs_input_grad[0],
            grad_w_accum=grad_w_accum)
        ctx.save_for_backward(gX if gX is not None else torch.empty(0), gW if gW is not None else torch.empty(0))
        ctx.has = (gX is not None, gW is not None)
        return loss

    @staticmethod
    def backward(ctx, grad_out):
        if ctx.reduction == "none":
            want_x, want_w = ctx.need
            if ctx.kept is not None:
                gX, gW = backward_from_kept(ctx.kept, reduction="none", row_grad=grad_out.reshape(-1),
                                            want_grad_X=want_x, want_grad_W=want_w)
                ctx.kept = None
            else:
                X, W, t = ctx.saved_tensors
                _, gX, gW = fused_linear_cross_entropy(X, W, t, ignore_index=ctx.ignore_index, reduction="none",
                                                       row_grad=grad_out.reshape(-1), want_grad_X=want_x,
                                                       want_grad_W=want_w, grad_w_accum=ctx.grad_w_accum)
            return gW, (gX.reshape(ctx.shape) if gX is not None else None), None, None, None, None, None
        if getattr(ctx, "consumed", False):
            raise RuntimeError("fused linear cross-entropy: its gradients were computed in the forward pass and "
                               "were already scaled in place by an earlier backward through this graph")
        ctx.consumed = True
        gX, gW = ctx.saved_tensors
        hx, hw = ctx.has
        dX = scale_grad_(gX, grad_out).reshape(ctx.shape) if hx else None
        dW = scale_grad_(gW, grad_out) if hw else None
        return dW, dX, None, None, None, None, None


class FusedLinearCrossEntropyLoss(torch.nn.Module):
    """loss_fn(lm_head.weight, input, target) -> scalar loss with autograd.

    input may be [BT, H] or [B, T, H]; target has the matching leading shape.
    reduction 'none' returns the per-row losses with the leading shape; with
    keep_logits=True its forward keeps the batch's bf16 store until backward
    (BT * V * 2 bytes held, 6 rather than 8 * BT * H * V tensor FLOPs).
    """

    def __init__(self, ignore_index: int = -100, reduction: str = "mean", grad_w_accum: str = "output",
                 keep_logits: bool = False):
        super().__init__()
        if reduction not in _RED:
            raise ValueError("reduction must be 'mean', 'sum' or 'none'")
        self.ignore_index = ignore_index
        self.reduction = reduction
        self.grad_w_accum = grad_w_accum
        self.keep_logits = keep_logits

    def forward(self, weight, input, target):  # noqa: A002 - mirrors the pages' call
        return _FLCEFunction.apply(weight, input, target, self.ignore_index, self.reduction, self.grad_w_accum,
                                   self.keep_logits)
