"""CUDA path vs the float64 oracle, element by element, at sizes the oracle
finishes in seconds (several tiles, ragged tails), plus the edge cases."""
import numpy as np
import pytest
import torch

import oracle
from linear_cross_entropy_04_b200.inputs import WORKLOADS, make_inputs, IGNORE_INDEX
from flce_testlib import need_gpu, to_dev, rel_err, assert_grad_close, TOL

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()


def L():
    import linear_cross_entropy_04_b200 as lib

    return lib


def run_case(d, reduction="mean", chunk_rows=0, grad_w_accum="output", ignore_index=IGNORE_INDEX,
             want_grad_X=True, want_grad_W=True, **kw):
    X, W, t = to_dev(d)
    row_loss = torch.empty(d["BT"], dtype=torch.float32, device="cuda")
    loss, gX, gW, st = L().fused_linear_cross_entropy(
        X, W, t, ignore_index=ignore_index, reduction=reduction, chunk_rows=chunk_rows,
        grad_w_accum=grad_w_accum, row_loss=row_loss, want_grad_X=want_grad_X, want_grad_W=want_grad_W,
        return_stats=True, **kw)
    torch.cuda.synchronize()
    assert L().device_error() == 0
    ref = oracle.flce(d["X"], d["W"], d["target"], ignore_index=ignore_index, reduction=reduction)
    tol = TOL[d["dtype"]]
    assert rel_err(loss.item(), ref["loss"]) <= tol["loss"], (loss.item(), ref["loss"])
    np.testing.assert_allclose(row_loss.cpu().numpy(), ref["row_loss"], rtol=tol["loss"], atol=tol["loss"])
    if want_grad_X:
        assert_grad_close(gX, ref["grad_X"], d["dtype"], "grad_X")
        ign = d["target"] == ignore_index
        if ign.any():
            assert torch.all(gX[torch.from_numpy(ign).cuda()] == 0), "ignored rows must get exactly 0"
    if want_grad_W:
        assert_grad_close(gW, ref["grad_W"], d["dtype"], "grad_W")
    return st


# ------------------------------------------------------------ tcgen05 engine alone

@pytest.mark.parametrize("a_mn,b_mn", [(0, 0), (0, 1), (1, 0), (1, 1)])
@pytest.mark.parametrize("M,N,K", [(128, 256, 64), (300, 520, 200), (1024, 768, 2048), (129, 8, 4099)])
def test_engine_gemm_matches_torch(a_mn, b_mn, M, N, K):
    g = torch.Generator().manual_seed(M * 7 + N + K)
    A = torch.randn(M, K, generator=g).to(torch.bfloat16)
    Bm = torch.randn(N, K, generator=g).to(torch.bfloat16)
    ref = A.float() @ Bm.float().T
    # the engine wants leading dimensions that are multiples of 8 elements
    def lay(T, mn):
        S = T.T.contiguous() if mn else T.contiguous()
        cols = S.shape[1]
        pad = (-cols) % 8
        return torch.nn.functional.pad(S, (0, pad)).cuda()[:, :cols]
    Ad, Bd = lay(A, a_mn), lay(Bm, b_mn)
    C = L().gemm_bf16(Ad, Bd, M, N, K, bool(a_mn), bool(b_mn))
    torch.cuda.synchronize()
    assert L().device_error() == 0
    err = (C.cpu() - ref).abs().max().item()
    assert err <= 1e-3 * ref.abs().max().item() + 1e-3, err


# ------------------------------------------------------------ FLCE parity

def test_tiny_fp32_config():
    d = make_inputs(WORKLOADS["tiny"])
    st = run_case(d)
    assert st["path"] == 0 and st["n_chunks"] >= 2


@pytest.mark.parametrize("reduction", ["mean", "sum"])
def test_tiny_fp32_sum_and_chunks(reduction):
    d = make_inputs(WORKLOADS["tiny"], BT=300, V=1000)
    run_case(d, reduction=reduction, chunk_rows=128)


@pytest.mark.parametrize("BT,H,V", [(512, 256, 4096), (300, 192, 1000), (129, 192, 4099), (1000, 512, 3000),
                                    (64, 8, 300)])
def test_bf16_small_shapes(BT, H, V):
    d = make_inputs(WORKLOADS["llama3_8b_seq"], BT=BT, H=H, V=V)
    run_case(d)


@pytest.mark.parametrize("accum", ["output", "fp32"])
def test_bf16_many_chunks_ragged(accum):
    d = make_inputs(WORKLOADS["qwen2_7b"], BT=700, H=256, V=2000)
    st = run_case(d, chunk_rows=256, grad_w_accum=accum)
    assert st["n_chunks"] == 3


def test_bf16_sum_reduction_and_wide_logits():
    d = make_inputs(WORKLOADS["large_vocab_stress"], BT=400, H=512, V=5000)
    run_case(d, reduction="sum")


def test_bf16_ignore_index_inside_vocab():
    d = make_inputs(WORKLOADS["llama3_8b_seq"], BT=200, H=64, V=700)
    ii = int(d["target"][d["target"] >= 0][0])
    d["target"][d["target"] == IGNORE_INDEX] = ii  # -100 would now be out of range
    run_case(d, ignore_index=ii)


def test_bf16_only_one_gradient():
    d = make_inputs(WORKLOADS["llama3_8b_seq"], BT=300, H=128, V=900)
    run_case(d, want_grad_X=False)
    run_case(d, want_grad_W=False)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_all_rows_ignored(dtype):
    w = WORKLOADS["tiny"] if dtype == "f32" else WORKLOADS["llama3_8b_seq"]
    d = make_inputs(w, BT=150, H=64, V=500)
    d["target"][:] = IGNORE_INDEX
    X, W, t = to_dev(d)
    loss, gX, gW = L().fused_linear_cross_entropy(X, W, t)
    torch.cuda.synchronize()
    assert loss.item() == 0.0
    assert torch.all(gX == 0) and torch.all(gW == 0)


def test_empty_batch_zeroes_grad_W():
    W = torch.randn(300, 64, device="cuda").to(torch.bfloat16)
    X = torch.empty(0, 64, device="cuda", dtype=torch.bfloat16)
    t = torch.empty(0, dtype=torch.int64, device="cuda")
    gW = torch.full_like(W, 7.0)
    loss = torch.full((), 3.0, device="cuda")
    L().fused_linear_cross_entropy(X, W, t, out=(loss, None, gW))
    torch.cuda.synchronize()
    assert loss.item() == 0.0 and torch.all(gW == 0)


def test_w_zero_closed_form_bf16():
    d = make_inputs(WORKLOADS["llama3_8b_seq"], BT=500, H=256, V=3000, w_zero=True)
    X, W, t = to_dev(d)
    loss, gX, gW = L().fused_linear_cross_entropy(X, W, t)
    torch.cuda.synchronize()
    assert rel_err(loss.item(), np.log(3000)) <= 1e-3
    assert torch.all(gX == 0)
    ref = oracle.flce(d["X"], d["W"], d["target"])["grad_W"]
    assert_grad_close(gW, ref, "bf16", "grad_W (W=0)")


def test_out_of_range_target_sets_the_error_word():
    d = make_inputs(WORKLOADS["llama3_8b_seq"], BT=64, H=64, V=300)
    d["target"][5] = 300
    X, W, t = to_dev(d)
    L().fused_linear_cross_entropy(X, W, t)
    assert L().device_error() & 0x1
    assert L().device_error() == 0  # reading clears it


def test_deterministic():
    d = make_inputs(WORKLOADS["llama3_8b_seq"], BT=600, H=256, V=3000)
    X, W, t = to_dev(d)
    a = L().fused_linear_cross_entropy(X, W, t, chunk_rows=256)
    b = L().fused_linear_cross_entropy(X, W, t, chunk_rows=256)
    torch.cuda.synchronize()
    assert a[0].item() == b[0].item()
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("inplace", [False, True])
def test_cross_entropy_logits_given(dtype, inplace):
    rng = np.random.default_rng(4)
    BT, V = 300, 5003
    z = (rng.standard_normal((BT, V)) * 3).astype(np.float32)
    t = rng.integers(0, V, BT)
    t[::7] = IGNORE_INDEX
    zt = torch.from_numpy(z).to(torch.bfloat16 if dtype == "bf16" else torch.float32)
    z64 = zt.double().numpy()
    ref = oracle.cross_entropy(z64, t)
    # rows of 5003 elements are not 16-byte aligned: pad the row pitch
    pitch = 5008
    buf = torch.zeros(BT, pitch, dtype=zt.dtype)
    buf[:, :V] = zt
    zd = buf.cuda()[:, :V]
    loss, g = L().cross_entropy(zd, torch.from_numpy(t).cuda(), inplace=inplace)
    torch.cuda.synchronize()
    assert rel_err(loss.item(), ref["loss"]) <= TOL[dtype]["loss"]
    assert_grad_close(g, ref["dz"], dtype, "dz")
    if inplace:
        assert g.data_ptr() == zd.data_ptr()


def test_module_autograd_matches_oracle():
    d = make_inputs(WORKLOADS["llama3_8b_seq"], BT=256, H=128, V=1000)
    X, W, t = to_dev(d)
    X = X.reshape(2, 128, 128).clone().requires_grad_(True)
    W = W.clone().requires_grad_(True)
    loss = L().FusedLinearCrossEntropyLoss()(W, X, t.reshape(2, 128))
    (2.5 * loss).backward()
    ref = oracle.flce(d["X"], d["W"], d["target"])
    assert rel_err(loss.item(), ref["loss"]) <= 1e-3
    assert_grad_close(X.grad.reshape(256, 128), 2.5 * ref["grad_X"], "bf16", "module grad_X")
    assert_grad_close(W.grad, 2.5 * ref["grad_W"], "bf16", "module grad_W")


def test_module_backward_does_not_wait_for_the_gpu():
    """backward applies the upstream gradient on the device: with the stream kept
    busy by a long spin kernel, backward returns before that kernel ends, and the
    gradients still come out scaled (1 leaves them untouched, 0.5 halves them)."""
    d = make_inputs(WORKLOADS["llama3_8b_seq"], BT=256, H=128, V=1000)
    ref = oracle.flce(d["X"], d["W"], d["target"])
    # the same sequence untimed first: under lazy module loading the first launch of any
    # kernel in the process (torch's own included, such as the multiply's backward) may
    # block the host once
    for factor in (1.0, 0.5):
        X, W, t = to_dev(d)
        loss = L().FusedLinearCrossEntropyLoss()(W.requires_grad_(True), X.requires_grad_(True), t)
        (loss * factor).backward()
    torch.cuda.synchronize()
    for factor in (1.0, 0.5):
        X, W, t = to_dev(d)
        X.requires_grad_(True)
        W.requires_grad_(True)
        loss = L().FusedLinearCrossEntropyLoss()(W, X, t)
        torch.cuda.synchronize()
        torch.cuda._sleep(2_000_000_000)  # about a second of spinning ahead of backward's work
        (loss * factor).backward()
        busy = not torch.cuda.current_stream().query()
        torch.cuda.synchronize()
        assert busy, "backward waited for the GPU"
        assert_grad_close(X.grad, factor * ref["grad_X"], "bf16", f"grad_X x{factor}")
        assert_grad_close(W.grad, factor * ref["grad_W"], "bf16", f"grad_W x{factor}")
        with pytest.raises(RuntimeError, match="already scaled"):
            loss2 = L().FusedLinearCrossEntropyLoss()(W.detach().requires_grad_(True), X.detach(), t)
            loss2.backward(retain_graph=True)
            loss2.backward()


def test_scale_grad_layouts():
    """flce_scale_grad on vector and element paths, strided rows, both dtypes."""
    g = torch.Generator(device="cuda").manual_seed(3)
    for dt in (torch.bfloat16, torch.float32):
        for shape, cols in (((300, 264), 264), ((64, 101), 101), ((7,), None)):
            base = torch.randn(*shape, generator=g, device="cuda").to(dt)
            if cols == 264:
                big = torch.randn(300, 272, generator=g, device="cuda").to(dt)
                base = big[:, :264]  # row pitch 272
            ref = base.float() * 0.3
            s = torch.tensor(0.3, device="cuda")
            L().scale_grad_(base, s)
            tol = 2 ** -8 if dt == torch.bfloat16 else 1e-6
            assert torch.allclose(base.float(), ref, rtol=tol, atol=0)
            before = base.clone()
            L().scale_grad_(base, torch.tensor(1.0, device="cuda"))
            assert torch.equal(base, before)


def test_host_buffers_end_to_end():
    d = make_inputs(WORKLOADS["llama3_8b_seq"], BT=256, H=128, V=1000)
    X = torch.from_numpy(d["X"]).to(torch.bfloat16).pin_memory()
    W = torch.from_numpy(d["W"]).to(torch.bfloat16).pin_memory()
    t = torch.from_numpy(d["target"]).pin_memory()
    loss, gX, gW = L().fused_linear_cross_entropy(X, W, t)
    assert not loss.is_cuda and not gW.is_cuda
    ref = oracle.flce(d["X"], d["W"], d["target"])
    assert rel_err(loss.item(), ref["loss"]) <= 1e-3
    assert_grad_close(gW, ref["grad_W"], "bf16", "grad_W")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_none_reduction_with_row_grad(dtype):
    w = WORKLOADS["tiny"] if dtype == "f32" else WORKLOADS["llama3_8b_seq"]
    d = make_inputs(w, BT=300, H=128, V=2000)
    g = np.random.default_rng(3).standard_normal(300).astype(np.float32)
    X, W, t = to_dev(d)
    loss, gX, gW = L().fused_linear_cross_entropy(X, W, t, reduction="none", row_grad=torch.from_numpy(g).cuda(),
                                                  chunk_rows=128)
    torch.cuda.synchronize()
    ref = oracle.flce(d["X"], d["W"], d["target"], reduction="none", row_grad=g)
    assert loss.shape == (300,)
    np.testing.assert_allclose(loss.cpu().numpy(), ref["loss"], rtol=TOL[dtype]["loss"], atol=TOL[dtype]["loss"])
    assert_grad_close(gX, ref["grad_X"], dtype, "grad_X (none)")
    assert_grad_close(gW, ref["grad_W"], dtype, "grad_W (none)")


def test_cross_entropy_none_reduction():
    rng = np.random.default_rng(8)
    BT, V = 200, 3000
    z = torch.from_numpy((rng.standard_normal((BT, V)) * 2).astype(np.float32)).to(torch.bfloat16)
    t = rng.integers(0, V, BT)
    t[::9] = IGNORE_INDEX
    g = rng.standard_normal(BT).astype(np.float32)
    z64 = z.double().numpy()
    ref_rows = oracle.cross_entropy(z64, t, reduction="none")["row_loss"]
    ref_dz = oracle.dlogits(z64, t, reduction="sum") * g[:, None]
    loss, dz = L().cross_entropy(z.cuda(), torch.from_numpy(t).cuda(), reduction="none",
                                 row_grad=torch.from_numpy(g).cuda())
    torch.cuda.synchronize()
    np.testing.assert_allclose(loss.cpu().numpy(), ref_rows, rtol=1e-3, atol=1e-3)
    assert_grad_close(dz, ref_dz, "bf16", "dz (none)")


def test_module_none_reduction_backward():
    d = make_inputs(WORKLOADS["llama3_8b_seq"], BT=256, H=128, V=1000)
    X, W, t = to_dev(d)
    X = X.reshape(2, 128, 128).clone().requires_grad_(True)
    W = W.clone().requires_grad_(True)
    rows = L().FusedLinearCrossEntropyLoss(reduction="none")(W, X, t.reshape(2, 128))
    assert rows.shape == (2, 128)
    g = torch.randn(2, 128, device="cuda", generator=torch.Generator(device="cuda").manual_seed(1))
    rows.backward(g)
    ref = oracle.flce(d["X"], d["W"], d["target"], reduction="none", row_grad=g.reshape(-1).cpu().numpy())
    np.testing.assert_allclose(rows.detach().reshape(-1).cpu().numpy(), ref["loss"], rtol=1e-3, atol=1e-3)
    assert_grad_close(X.grad.reshape(256, 128), ref["grad_X"], "bf16", "module grad_X (none)")
    assert_grad_close(W.grad, ref["grad_W"], "bf16", "module grad_W (none)")


def test_host_pipeline_matches_device_call():
    from linear_cross_entropy_04_b200.pipeline import HostPipeline

    d = make_inputs(WORKLOADS["llama3_8b_seq"], BT=384, H=128, V=1500)
    X, W, t = to_dev(d)
    ref = L().fused_linear_cross_entropy(X, W, t)
    Xh, Wh, th = X.cpu().pin_memory(), W.cpu().pin_memory(), t.cpu().pin_memory()
    outs = [(torch.empty((), dtype=torch.float32).pin_memory(), torch.empty_like(Xh).pin_memory(),
             torch.empty_like(Wh).pin_memory()) for _ in range(3)]
    pipe = HostPipeline(384, 128, 1500)
    for o in outs:
        pipe.submit(Xh, Wh, th, o)
    pipe.synchronize()
    for o in outs:
        assert o[0].item() == ref[0].item()
        assert torch.equal(o[1], ref[1].cpu()) and torch.equal(o[2], ref[2].cpu())


def test_grad_w_ready_event_marks_a_complete_grad_W_before_the_end():
    """grad_w_ready_event: the library records it as soon as grad_W is complete. A
    copy queued on another stream behind it sees the final grad_W; the grad_X GEMM
    of the last chunk (launched after grad_W when the event is given) still runs
    after it; and the results equal the call without the event bit for bit. The
    recompute schedule records it at the end."""
    d = make_inputs(WORKLOADS["llama3_8b_seq"], BT=4096, H=4096, V=32768)
    X, W, t = to_dev(d)
    ref = L().fused_linear_cross_entropy(X, W, t)
    side = torch.cuda.Stream()
    for schedule in ("stored", "recompute"):
        ref_s = ref if schedule == "stored" else L().fused_linear_cross_entropy(X, W, t, schedule=schedule)
        ev = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        loss, gX, gW = L().fused_linear_cross_entropy(X, W, t, grad_w_ready_event=ev, schedule=schedule)
        end.record()
        side.wait_event(ev)
        with torch.cuda.stream(side):
            snap = gW.clone()
        torch.cuda.synchronize()
        assert L().device_error() == 0
        assert torch.equal(snap, ref_s[2]) and torch.equal(gW, ref_s[2]) and torch.equal(gX, ref_s[1])
        assert loss.item() == ref_s[0].item()
        gap = ev.elapsed_time(end)
        if schedule == "stored":
            assert gap > 0.05, gap  # the last grad_X GEMM (4096 x 2048 x 32768) ran after the event
        else:
            assert gap >= 0.0
    # grad_W only, and grad_X with grad_W in one launch: recorded after the last grad_W launch
    small = make_inputs(WORKLOADS["llama3_8b_seq"], BT=700, H=256, V=3000)
    Xs, Ws, ts = to_dev(small)
    for kw in ({"want_grad_X": False}, {"flags": 0, "chunk_rows": 256}):
        ref_k = L().fused_linear_cross_entropy(Xs, Ws, ts, **kw)
        ev = torch.cuda.Event()
        lo, gx, gw = L().fused_linear_cross_entropy(Xs, Ws, ts, grad_w_ready_event=ev, **kw)
        side.wait_event(ev)
        with torch.cuda.stream(side):
            snap = gw.clone()
        torch.cuda.synchronize()
        assert torch.equal(snap, ref_k[2]) and torch.equal(gw, ref_k[2]), kw


def test_host_pipeline_runs_a_caller_step():
    """HostPipeline(step=...) runs the given step on its compute stream and copies
    back the tensors the step returns, here a freshly allocated slice of grad_W
    (as the data-parallel call returns this rank's rows), over several steps
    whose slots are reused."""
    from linear_cross_entropy_04_b200.pipeline import HostPipeline

    d = make_inputs(WORKLOADS["llama3_8b_seq"], BT=384, H=128, V=1500)
    X, W, t = to_dev(d)
    ref = L().fused_linear_cross_entropy(X, W, t)
    rows = 700

    def step(Xs, Ws, ts, out):
        lo, gx, gw = L().fused_linear_cross_entropy(Xs, Ws, ts, out=out)
        return lo, gx, gw[:rows].clone()

    Xh, Wh, th = X.cpu().pin_memory(), W.cpu().pin_memory(), t.cpu().pin_memory()
    outs = [(torch.empty((), dtype=torch.float32).pin_memory(), torch.empty_like(Xh).pin_memory(),
             torch.empty((rows, 128), dtype=Wh.dtype).pin_memory()) for _ in range(4)]
    pipe = HostPipeline(384, 128, 1500, step=step)
    for o in outs:
        pipe.submit(Xh, Wh, th, o)
    pipe.synchronize()
    for o in outs:
        assert o[0].item() == ref[0].item()
        assert torch.equal(o[1], ref[1].cpu()) and torch.equal(o[2], ref[2][:rows].cpu())


@pytest.mark.parametrize("every_chunk", [False, True])
@pytest.mark.parametrize("n_shards,shard_rows,BT,chunk", [(3, 1024, 700, 256), (4, 800, 700, 256),
                                                         (4, 768, 1100, 128)])
def test_grad_W_shard_routing(n_shards, shard_rows, BT, chunk, every_chunk):
    """grad_W added tile by tile into shards (the data-parallel reduce-scatter path), with every
    shard on this GPU: shard k must hold rows [k*shard_rows, ...) of the plain grad_W, bit for
    bit, whether the chunks before the last accumulate locally (the default) or every chunk's
    boxes are routed (FLAG_ROUTE_EVERY_CHUNK); and match the oracle. The last case runs
    9 chunks into 4 shards."""
    from linear_cross_entropy_04_b200 import _binding as B

    d = make_inputs(WORKLOADS["llama3_8b_seq"], BT=BT, H=256, V=3000)
    X, W, t = to_dev(d)
    loss, gX, gW = L().fused_linear_cross_entropy(X, W, t, chunk_rows=chunk)
    shards = [torch.zeros(shard_rows, 256, dtype=torch.bfloat16, device="cuda") for _ in range(n_shards)]
    flags = B.FLAG_ROUTE_EVERY_CHUNK if every_chunk else 0
    loss2, gX2, gW2, st = L().fused_linear_cross_entropy(X, W, t, chunk_rows=chunk, grad_w_shards=shards,
                                                         shard_rows=shard_rows, flags=flags, return_stats=True)
    torch.cuda.synchronize()
    assert L().device_error() == 0
    assert st["n_chunks"] == -(-BT // chunk)
    plain = L().plan(BT, 256, 3000, chunk_rows=chunk)["workspace_bytes"]
    local = 0 if every_chunk else 3000 * 256 * 2  # the earlier chunks' local bf16 sum
    assert st["workspace_bytes"] - plain == local
    assert gW2 is None and loss2.item() == loss.item() and torch.equal(gX2, gX)
    joined = torch.cat(shards)[:3000]
    assert torch.equal(joined, gW)  # same roundings in the same order
    assert torch.all(torch.cat(shards)[3000:] == 0)
    ref = oracle.flce(d["X"], d["W"], d["target"])
    assert_grad_close(joined, ref["grad_W"], "bf16", "sharded grad_W")


def _ce_inputs(seed, BT, V, ignore_every=6):
    rng = np.random.default_rng(seed)
    z = torch.from_numpy((rng.standard_normal((BT, V)) * 3).astype(np.float32)).to(torch.bfloat16)
    t = rng.integers(0, V, BT)
    t[::ignore_every] = IGNORE_INDEX
    return z, t


# V spans one-pass clusters of 1, 2, 6, 10 and 12 CTAs (the shared-memory
# kernel's rule: ceil(V / 25600) CTAs up to 16, else up to 32768 columns each),
# and a V past 16 CTAs of 32768 columns (and not a multiple of 8) that takes the
# multi-pass kernels.
@pytest.mark.parametrize("V", [1000, 16385, 50000, 128256, 152064, 256000, 300007, 600011])
@pytest.mark.parametrize("mode", ["mean_inplace", "sum", "none_rowgrad", "loss_only"])
def test_cross_entropy_across_cluster_sizes(V, mode):
    BT = 48
    z, t = _ce_inputs(V % 97, BT, V)
    z64 = z.double().numpy()
    pitch = V + (-V) % 8
    buf = torch.zeros(BT, pitch, dtype=torch.bfloat16)
    buf[:, :V] = z
    zd = buf.cuda()[:, :V]
    td = torch.from_numpy(t).cuda()
    if mode == "none_rowgrad":
        g = np.random.default_rng(1).standard_normal(BT).astype(np.float32)
        loss, dz = L().cross_entropy(zd, td, reduction="none", row_grad=torch.from_numpy(g).cuda())
        ref_rows = oracle.cross_entropy(z64, t, reduction="none")["row_loss"]
        torch.cuda.synchronize()
        np.testing.assert_allclose(loss.cpu().numpy(), ref_rows, rtol=1e-3, atol=1e-3)
        assert_grad_close(dz, oracle.dlogits(z64, t, reduction="sum") * g[:, None], "bf16", "dz (none)")
        return
    red = "sum" if mode == "sum" else "mean"
    lse = torch.full((BT,), float("nan"), dtype=torch.float32, device="cuda")
    loss, dz = L().cross_entropy(zd, td, reduction=red, inplace=mode == "mean_inplace",
                                 want_grad=mode != "loss_only", lse=lse)
    torch.cuda.synchronize()
    ref = oracle.cross_entropy(z64, t, reduction=red)
    assert rel_err(loss.item(), ref["loss"]) <= TOL["bf16"]["loss"], (loss.item(), ref["loss"])
    ref_lse = np.log(np.exp(z64 - z64.max(1, keepdims=True)).sum(1)) + z64.max(1)
    np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, rtol=1e-5, atol=1e-4)
    if mode == "loss_only":
        assert dz is None
        return
    assert_grad_close(dz, ref["dz"], "bf16", f"dz ({mode})")
    ign = t == IGNORE_INDEX
    assert torch.all(dz[torch.from_numpy(ign).cuda()] == 0)  # ignored rows exactly 0
    if mode == "mean_inplace":
        assert dz.data_ptr() == zd.data_ptr()


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("inplace", [False, True])
def test_cross_entropy_unaligned_rows_are_staged(dtype, inplace):
    """Contiguous logits whose rows are not 16-byte aligned (V = 50257) go through a
    padded copy in the binding: results match the oracle, and an in-place gradient
    lands in the caller's tensor."""
    BT, V = 96, 50257
    z, t = _ce_inputs(5, BT, V)
    zt = z if dtype == "bf16" else z.float()
    zd = zt.cuda()
    assert (zd.stride(0) * zd.element_size()) % 16 != 0
    loss, dz = L().cross_entropy(zd, torch.from_numpy(t).cuda(), inplace=inplace)
    torch.cuda.synchronize()
    assert L().device_error() == 0
    ref = oracle.cross_entropy(zt.double().numpy(), t)
    assert rel_err(loss.item(), ref["loss"]) <= TOL[dtype]["loss"]
    assert_grad_close(dz, ref["dz"], dtype, "dz (unaligned rows)")
    if inplace:
        assert dz.data_ptr() == zd.data_ptr()


def test_cross_entropy_one_pass_edge_rows():
    """All rows ignored (loss 0, dz 0), one row, and -inf logits (masked vocabulary)."""
    V = 50000
    z, t = _ce_inputs(3, 5, V)
    t[:] = IGNORE_INDEX
    loss, dz = L().cross_entropy(z.cuda(), torch.from_numpy(t).cuda())
    torch.cuda.synchronize()
    assert loss.item() == 0.0 and torch.all(dz == 0)
    z, t = _ce_inputs(4, 1, V)
    z[0, 20000:40000] = float("-inf")  # two whole CTA slices and parts of others are masked
    t[0] = 5
    z64 = z.double().numpy()
    loss, dz = L().cross_entropy(z.cuda(), torch.from_numpy(t).cuda())
    torch.cuda.synchronize()
    ref = oracle.cross_entropy(z64, t)
    assert np.isfinite(loss.item()) and rel_err(loss.item(), ref["loss"]) <= TOL["bf16"]["loss"]
    assert torch.all(dz[0, 20000:40000] == 0)
    assert_grad_close(dz, ref["dz"], "bf16", "dz (-inf)")


@pytest.mark.parametrize("V", [128256, 50021, 16391, 7])
def test_cross_entropy_one_pass_matches_multipass(monkeypatch, V):
    """The one-pass kernels agree with the oracle and with the partials + combine +
    grad kernels: the shared-memory kernel with its default CTA count and with
    16384-column slices (FLCE_CE_SLICE), and the register kernel (FLCE_CE=regs). With
    the same 16384-column slices the shared-memory and register kernels take the
    same arithmetic in the same order, so they agree bit for bit. Ragged V leaves a
    tail of fewer than 8 columns in the last CTA's slice; rows are padded to 16
    bytes and the padding columns must stay untouched."""
    import ctypes

    from linear_cross_entropy_04_b200 import _binding as B

    Vp = V + (-V) % 8
    z, t = _ce_inputs(9, 256, V)
    zp = torch.full((256, Vp), -1.0, dtype=torch.bfloat16)
    zp[:, :V] = z
    zd, td = zp.cuda()[:, :V], torch.from_numpy(t).cuda()
    assert zd.stride(0) == Vp
    gp = torch.full((256, Vp), 7.0, dtype=torch.bfloat16, device="cuda")
    out = {}
    for mode, env in (("default", {}), ("slice16384", {"FLCE_CE_SLICE": "16384"}), ("regs", {"FLCE_CE": "regs"}),
                      ("multipass", {"FLCE_CE": "multipass"})):
        monkeypatch.delenv("FLCE_CE", raising=False)
        monkeypatch.delenv("FLCE_CE_SLICE", raising=False)
        for k, v in env.items():
            monkeypatch.setenv(k, v)
        g = gp[:, :V]
        loss = torch.empty((), dtype=torch.float32, device="cuda")
        tz, tt, tl, tg = B.tensor(zd), B.tensor(td), B.tensor(loss), B.tensor(g)
        B.check(B.lib().flce_cross_entropy(ctypes.byref(tz), ctypes.byref(tt), -100, 0, ctypes.byref(tl),
                                           ctypes.byref(tg), B.stream_handle(), None), "flce_cross_entropy")
        torch.cuda.synchronize()
        assert L().device_error() == 0
        assert torch.all(gp[:, V:] == 7.0), "padding columns must stay untouched"
        out[mode] = (loss.item(), g.clone())
    ref = oracle.cross_entropy(z.double().numpy(), t)
    for mode, (lv, g) in out.items():
        assert rel_err(lv, ref["loss"]) <= TOL["bf16"]["loss"], mode
        assert_grad_close(g, ref["dz"], "bf16", f"dz ({mode})")
    assert out["slice16384"][0] == out["regs"][0] and torch.equal(out["slice16384"][1], out["regs"][1])
    for mode in ("default", "slice16384"):
        assert rel_err(out[mode][0], out["multipass"][0]) <= 1e-5
        d = (out[mode][1].float() - out["multipass"][1].float()).abs().max().item()
        assert d <= 2 ** -8 * out["multipass"][1].float().abs().max().item(), (mode, d)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("reduction", ["mean", "none"])
def test_keep_then_gradients_from_kept(dtype, reduction):
    """forward_keep + backward_from_kept (the logits GEMM once) against the oracle
    and against the one-call path with the same row_grad."""
    w = WORKLOADS["tiny"] if dtype == "f32" else WORKLOADS["llama3_8b_seq"]
    d = make_inputs(w, BT=700, H=256, V=3000)
    X, W, t = to_dev(d)
    g = np.random.default_rng(2).standard_normal(700).astype(np.float32)
    rg = torch.from_numpy(g).cuda() if reduction == "none" else None
    lse = torch.empty(700, dtype=torch.float32, device="cuda")
    loss, kept = L().forward_keep(X, W, t, reduction=reduction, lse=lse)
    gX, gW = L().backward_from_kept(kept, reduction=reduction, row_grad=rg)
    torch.cuda.synchronize()
    ref = oracle.flce(d["X"], d["W"], d["target"], reduction=reduction, row_grad=g if rg is not None else None)
    tol = TOL[dtype]
    if reduction == "none":
        np.testing.assert_allclose(loss.cpu().numpy(), ref["loss"], rtol=tol["loss"], atol=tol["loss"])
    else:
        assert rel_err(loss.item(), ref["loss"]) <= tol["loss"]
    assert_grad_close(gX, ref["grad_X"], dtype, "grad_X (kept)")
    assert_grad_close(gW, ref["grad_W"], dtype, "grad_W (kept)")
    z = d["X"].astype(np.float64) @ d["W"].astype(np.float64).T
    ref_lse = np.log(np.exp(z - z.max(1, keepdims=True)).sum(1)) + z.max(1)
    np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, rtol=1e-4, atol=1e-3)
    # the one-call path with the same reduction and row_grad: same dz, same grad_X rows
    l2, gX2, gW2 = L().fused_linear_cross_entropy(X, W, t, reduction=reduction, row_grad=rg, chunk_rows=768)
    torch.cuda.synchronize()
    assert torch.equal(gX, gX2)
    assert torch.allclose(loss, l2, rtol=1e-6, atol=0)
    with pytest.raises(RuntimeError, match="already used"):
        L().backward_from_kept(kept)


def test_module_none_keep_logits():
    d = make_inputs(WORKLOADS["llama3_8b_seq"], BT=256, H=128, V=1000)
    X, W, t = to_dev(d)
    X = X.reshape(2, 128, 128).clone().requires_grad_(True)
    W = W.clone().requires_grad_(True)
    rows = L().FusedLinearCrossEntropyLoss(reduction="none", keep_logits=True)(W, X, t.reshape(2, 128))
    g = torch.randn(2, 128, device="cuda", generator=torch.Generator(device="cuda").manual_seed(1))
    rows.backward(g)
    ref = oracle.flce(d["X"], d["W"], d["target"], reduction="none", row_grad=g.reshape(-1).cpu().numpy())
    assert_grad_close(X.grad.reshape(256, 128), ref["grad_X"], "bf16", "module keep grad_X")
    assert_grad_close(W.grad, ref["grad_W"], "bf16", "module keep grad_W")


@pytest.mark.parametrize("V,BT", [(50000, 1000), (128256, 400), (152064, 300)])
@pytest.mark.parametrize("want_lse", [False, True])
def test_cross_entropy_many_rows_in_place(V, BT, want_lse):
    """Hundreds of rows (many clusters per SM over the launch), ignored rows
    interleaved and in runs, in place, with and without the lse output."""
    z, t = _ce_inputs(V % 89, BT, V, ignore_every=3)
    t[5:9] = IGNORE_INDEX
    td = torch.from_numpy(t).cuda()
    zd = z.cuda()
    lse = torch.empty(BT, dtype=torch.float32, device="cuda") if want_lse else None
    loss, g = L().cross_entropy(zd, td, inplace=True, lse=lse)
    torch.cuda.synchronize()
    z64 = z.double().numpy()
    ref = oracle.cross_entropy(z64, t)
    assert rel_err(loss.item(), ref["loss"]) <= TOL["bf16"]["loss"]
    assert_grad_close(g, ref["dz"], "bf16", "dz (many rows)")
    assert g.data_ptr() == zd.data_ptr()
    if want_lse:
        ref_lse = np.log(np.exp(z64 - z64.max(1, keepdims=True)).sum(1)) + z64.max(1)
        np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, rtol=1e-5, atol=1e-4)


# The engine's alternative paths, each forced by its switch: the single-CTA
# engine, grad_X and grad_W in one launch or two, and grad_X split over K
# (few output tiles, a long K: 2 x 2 tiles over K = 9000 / 64 blocks).
@pytest.mark.parametrize("env", [{"FLCE_ENGINE": "1sm"}, {"FLCE_GRAD_LAUNCH": "combined"},
                                 {"FLCE_GRAD_LAUNCH": "split"}, {"FLCE_GRADX_SPLITK": "1"},
                                 {"FLCE_ENGINE": "1sm", "FLCE_GRAD_LAUNCH": "combined"}],
                         ids=["1sm", "combined", "split", "splitk", "1sm-combined"])
def test_engine_variants_match_oracle(monkeypatch, env):
    for k, v in env.items():
        monkeypatch.setenv(k, v)
    d = make_inputs(WORKLOADS["llama3_8b_seq"], BT=500, H=512, V=9000)
    X, W, t = to_dev(d)
    loss, gX, gW = L().fused_linear_cross_entropy(X, W, t, chunk_rows=384)
    torch.cuda.synchronize()
    assert L().device_error() == 0
    ref = oracle.flce(d["X"], d["W"], d["target"])
    assert rel_err(loss.item(), ref["loss"]) <= TOL["bf16"]["loss"]
    assert_grad_close(gX, ref["grad_X"], "bf16", f"grad_X {env}")
    assert_grad_close(gW, ref["grad_W"], "bf16", f"grad_W {env}")


# grad_X on the pair engine's 256 x 512 tiles, forced on and off: a ragged last
# 512-column tile (H = 264, 776: the second half of the last tile lies partly or
# wholly outside), several waves of wide tiles on 74 pairs (BT = 4200 in one
# chunk, H = 2560: 17 x 5 tiles), and chunk rows that are not a tile multiple.
@pytest.mark.parametrize("tile", ["wide", "narrow"])
@pytest.mark.parametrize("BT,H,V,chunk", [(500, 264, 3000, 384), (300, 776, 2000, 0), (4200, 2560, 1000, 4224),
                                          (700, 512, 9000, 256)])
def test_gradx_tile_width_matches_oracle(monkeypatch, tile, BT, H, V, chunk):
    monkeypatch.setenv("FLCE_GRADX_TILE", tile)
    d = make_inputs(WORKLOADS["llama3_8b_seq"], BT=BT, H=H, V=V)
    X, W, t = to_dev(d)
    loss, gX, gW = L().fused_linear_cross_entropy(X, W, t, chunk_rows=chunk)
    gX_only = L().fused_linear_cross_entropy(X, W, t, chunk_rows=chunk, want_grad_W=False)[1]
    torch.cuda.synchronize()
    assert L().device_error() == 0
    assert torch.equal(gX, gX_only)
    ref = oracle.flce(d["X"], d["W"], d["target"])
    assert rel_err(loss.item(), ref["loss"]) <= TOL["bf16"]["loss"]
    assert_grad_close(gX, ref["grad_X"], "bf16", f"grad_X ({tile})")
    assert_grad_close(gW, ref["grad_W"], "bf16", f"grad_W ({tile})")


# Degenerate shapes of the method: a one-class vocabulary (every row's loss and
# gradient are exactly 0), two classes (the logistic loss), a single row, and
# the smallest hidden size with an odd vocabulary.
@pytest.mark.parametrize("wl,BT,H,V", [("llama3_8b_seq", 1, 64, 100), ("llama3_8b_seq", 40, 64, 2),
                                       ("llama3_8b_seq", 5, 8, 7), ("tiny", 1, 16, 2), ("tiny", 9, 8, 3)])
def test_degenerate_shapes(wl, BT, H, V):
    run_case(make_inputs(WORKLOADS[wl], BT=BT, H=H, V=V))


@pytest.mark.parametrize("wl", ["llama3_8b_seq", "tiny"])
def test_one_class_vocabulary_is_exactly_zero(wl):
    d = make_inputs(WORKLOADS[wl], BT=40, H=64, V=1)
    d["target"][d["target"] != IGNORE_INDEX] = 0
    X, W, t = to_dev(d)
    loss, gX, gW = L().fused_linear_cross_entropy(X, W, t)
    torch.cuda.synchronize()
    assert loss.item() == 0.0
    assert torch.all(gX == 0) and torch.all(gW == 0)
    # logits given: rows padded to 16 bytes, as the ABI requires; the one-pass
    # kernel's exp2(z*log2e - max*log2e) leaves the rounding of z*log2e, so the
    # result is 0 to fp32 precision rather than exactly
    buf = torch.zeros(7, 8, dtype=X.dtype)
    buf[:, 0] = torch.randn(7).to(X.dtype)
    z = buf.cuda()[:, :1]
    lz, dz = L().cross_entropy(z, torch.zeros(7, dtype=torch.int64, device="cuda"))
    torch.cuda.synchronize()
    assert abs(lz.item()) <= 1e-6 and dz.float().abs().max().item() <= 1e-6


def test_nvtx_ranges_per_phase_and_chunk(tmp_path):
    """With an NVTX tool attached, a call shows as one range holding a range per
    phase launch, named with its row chunk, in launch order."""
    from test_abi import run_with_nvtx

    code = ("import torch\n"
            "import linear_cross_entropy_04_b200 as flce\n"
            "X = torch.randn(700, 256, device='cuda').to(torch.bfloat16)\n"
            "W = (torch.randn(3000, 256, device='cuda') * 0.02).to(torch.bfloat16)\n"
            "t = torch.randint(0, 3000, (700,), device='cuda')\n"
            "flce.fused_linear_cross_entropy(X, W, t, chunk_rows=256)\n"
            "torch.cuda.synchronize()\n")
    lines = run_with_nvtx(tmp_path, code)
    depth = 0
    for ln in lines:
        depth += 1 if ln.startswith("push") else -1
        assert depth >= 0
    assert depth == 0
    pushes = [ln[5:] for ln in lines if ln.startswith("push")]
    assert pushes[0] == "flce_fwd_bwd"
    assert pushes[1] == "flce count_valid" and pushes[-1] == "flce loss_reduce"
    body = [p for p in pushes[2:-1]]
    expect = []
    for c in range(3):
        expect += [f"flce logits_gemm_softmax chunk {c}", f"flce row_combine chunk {c}",
                   f"flce dlogits_inplace chunk {c}"]
        grads = [p for p in body if p == f"flce grad_gemms chunk {c}"]
        assert 1 <= len(grads) <= 2
        expect += grads
    assert body == expect


# ------------------------------------------------------------ recompute schedule
@pytest.mark.parametrize("BT,H,V,vc", [(700, 256, 3000, 512), (129, 192, 4099, 256), (1000, 512, 3000, 0),
                                       (300, 8, 1000, 256), (513, 264, 9000, 2048)])
def test_recompute_schedule_matches_oracle(BT, H, V, vc):
    """The vocabulary-outer schedule against the oracle: several vocabulary chunks
    with ragged last chunks, row tails, H = 8, and the default chunk from the budget."""
    st = run_case(make_inputs(WORKLOADS["llama3_8b_seq"], BT=BT, H=H, V=V), chunk_rows=vc, schedule="recompute")
    expect_vc = min(-(-V // 256) * 256, -(-vc // 256) * 256) if vc else -(-V // 256) * 256
    assert st["chunk_rows"] == expect_vc and st["n_chunks"] == -(-V // expect_vc)


@pytest.mark.parametrize("reduction", ["sum", "none"])
def test_recompute_schedule_reductions_and_row_grad(reduction):
    d = make_inputs(WORKLOADS["llama3_8b_seq"], BT=600, H=128, V=2000)
    X, W, t = to_dev(d)
    g = np.random.default_rng(4).standard_normal(600).astype(np.float32)
    loss, gX, gW = L().fused_linear_cross_entropy(X, W, t, reduction=reduction, row_grad=torch.from_numpy(g).cuda(),
                                                  chunk_rows=512, schedule="recompute")
    torch.cuda.synchronize()
    assert L().device_error() == 0
    ref = oracle.flce(d["X"], d["W"], d["target"], reduction=reduction, row_grad=g)
    if reduction == "none":
        np.testing.assert_allclose(loss.cpu().numpy(), ref["loss"], rtol=1e-3, atol=1e-3)
    else:
        assert rel_err(loss.item(), ref["loss"]) <= 1e-3
    assert_grad_close(gX, ref["grad_X"], "bf16", "grad_X (recompute)")
    assert_grad_close(gW, ref["grad_W"], "bf16", "grad_W (recompute)")


def test_recompute_schedule_edge_cases():
    """ignore_index inside the vocabulary, one gradient only, every row ignored,
    and W = 0 (loss ln V, grad_X exactly 0), on the recompute schedule."""
    d = make_inputs(WORKLOADS["llama3_8b_seq"], BT=300, H=64, V=1500)
    d["target"][d["target"] == IGNORE_INDEX] = 5  # -100 would be an out-of-range target with ignore_index 5
    d["target"][::7] = 5
    run_case(d, ignore_index=5, chunk_rows=256, schedule="recompute")
    d = make_inputs(WORKLOADS["llama3_8b_seq"], BT=300, H=64, V=1500)
    run_case(d, want_grad_X=False, chunk_rows=256, schedule="recompute")
    run_case(d, want_grad_W=False, chunk_rows=256, schedule="recompute")
    d2 = make_inputs(WORKLOADS["llama3_8b_seq"], BT=200, H=64, V=1000)
    d2["target"][:] = IGNORE_INDEX
    X, W, t = to_dev(d2)
    loss, gX, gW = L().fused_linear_cross_entropy(X, W, t, chunk_rows=256, schedule="recompute")
    torch.cuda.synchronize()
    assert loss.item() == 0.0 and torch.all(gX == 0) and torch.all(gW == 0)
    d3 = make_inputs(WORKLOADS["llama3_8b_seq"], BT=500, H=256, V=3000, w_zero=True)
    X, W, t = to_dev(d3)
    loss, gX, gW = L().fused_linear_cross_entropy(X, W, t, chunk_rows=1024, schedule="recompute")
    torch.cuda.synchronize()
    assert rel_err(loss.item(), np.log(3000)) <= 1e-3
    assert torch.all(gX == 0)
    assert_grad_close(gW, oracle.flce(d3["X"], d3["W"], d3["target"])["grad_W"], "bf16", "grad_W (W=0, recompute)")
