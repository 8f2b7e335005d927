"""The cross-entropy entry point that allocates nothing.

flce_cross_entropy_noalloc serves callers that cannot allocate device memory
where they compute the loss (for example while a CUDA graph is captured around
them, or inside a host that owns all device memory through its own allocator).
It keeps its scratch in a fixed device array inside the library instead.

This test calls it through the C ABI twice in a row, with different inputs so
that the second call runs over the scratch the first one left behind, and
checks each result against the allocating entry point flce_cross_entropy on
the same inputs, within the tolerances the other GPU tests use. It also
checks small cases of both dtypes against the float64 oracle directly (the
two entry points share kernels, so agreeing with each other alone would not
catch a fault in those), that a call leaves the device's free memory
unchanged, that the largest problem the fixed array holds runs and the next
size up is refused before any GPU work, and that reduction 'none' is refused.
The file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from flce_testlib import need_gpu, rel_err, TOL, assert_grad_close

pytestmark = pytest.mark.gpu


def _ce_case(seed, BT, V, dtype):
    rng = np.random.default_rng(seed)
    z = torch.from_numpy((rng.standard_normal((BT, V)) * 2.5).astype(np.float32)).to(dtype).cuda()
    t = rng.integers(0, V, BT)
    t[rng.permutation(BT)[: BT // 10]] = -100
    return z, torch.from_numpy(t).cuda()


def _call(fn, z, t, reduction, grad):
    from linear_cross_entropy_04_b200 import _binding as B

    loss = torch.full((), float("nan"), dtype=torch.float32, device="cuda")
    tz, tt, tl = B.tensor(z), B.tensor(t), B.tensor(loss)
    tg = B.tensor(grad) if grad is not None else None
    args = [ctypes.byref(tz), ctypes.byref(tt), -100, reduction, ctypes.byref(tl),
            ctypes.byref(tg) if tg is not None else None, B.stream_handle()]
    if fn == "flce_cross_entropy":
        args.append(None)
    rc = getattr(B.lib(), fn)(*args)
    return rc, loss


@pytest.mark.parametrize("dtype,name", [(torch.bfloat16, "bf16"), (torch.float32, "f32")])
def test_noalloc_matches_the_allocating_entry_point_on_two_calls(dtype, name):
    need_gpu()
    from linear_cross_entropy_04_b200 import _binding as B

    cases = [(11, 2048, 128256 // 4, B.MEAN), (12, 777, 50021 - 5, B.SUM)]
    for seed, BT, V, red in cases:
        V8 = V + (-V) % 8  # 16-byte aligned rows
        z, t = _ce_case(seed, BT, V8, dtype)
        g_ref = torch.empty_like(z)
        g_new = torch.full_like(z, float("nan"))
        rc_ref, l_ref = _call("flce_cross_entropy", z, t, red, g_ref)
        rc_new, l_new = _call("flce_cross_entropy_noalloc", z, t, red, g_new)
        torch.cuda.synchronize()
        assert rc_ref == 0 and rc_new == 0, (rc_ref, rc_new)
        assert rel_err(l_new.item(), l_ref.item()) <= TOL[name]["loss"], (l_new.item(), l_ref.item())
        gr = g_ref.float()
        err = (g_new.float() - gr).abs().max().item()
        assert err <= TOL[name]["grad"] * gr.abs().max().item(), err
    from linear_cross_entropy_04_b200 import device_error

    assert device_error() == 0


def test_noalloc_refuses_problems_larger_than_its_scratch():
    need_gpu()
    from linear_cross_entropy_04_b200 import _binding as B

    # 9000 rows x 128256 columns needs ~9 MiB of scratch, more than the fixed 8 MiB
    z = torch.empty((9000, 128256), dtype=torch.bfloat16, device="cuda")
    t = torch.zeros(9000, dtype=torch.int64, device="cuda")
    rc, loss = _call("flce_cross_entropy_noalloc", z, t, B.MEAN, None)
    assert rc == 6  # FLCE_ERR_WORKSPACE_TOO_SMALL
    assert torch.isnan(loss).item()  # nothing was enqueued


@pytest.mark.parametrize("dtype,name", [(torch.bfloat16, "bf16"), (torch.float32, "f32")])
@pytest.mark.parametrize("red", [0, 1])
def test_noalloc_matches_the_oracle(dtype, name, red):
    """Element by element against the float64 oracle, at the stated tolerances."""
    need_gpu()
    z, t = _ce_case(21 + red, 300, 5000, dtype)
    g = torch.full_like(z, float("nan"))
    rc, loss = _call("flce_cross_entropy_noalloc", z, t, red, g)
    torch.cuda.synchronize()
    assert rc == 0
    ref = oracle.cross_entropy(z.double().cpu().numpy(), t.cpu().numpy(), reduction=("mean", "sum")[red])
    assert rel_err(loss.item(), ref["loss"]) <= TOL[name]["loss"], (loss.item(), ref["loss"])
    assert_grad_close(g, ref["dz"], name, "dz")


def test_noalloc_allocates_no_device_memory():
    """After a first call has set up the device, further calls leave the free device memory as it was."""
    need_gpu()
    from linear_cross_entropy_04_b200 import _binding as B

    z, t = _ce_case(31, 1024, 32000, torch.bfloat16)
    g = torch.empty_like(z)
    _call("flce_cross_entropy_noalloc", z, t, B.MEAN, g)
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(3):
        rc, _ = _call("flce_cross_entropy_noalloc", z, t, B.MEAN, g)
        assert rc == 0
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0


def test_noalloc_size_limit_is_exact_at_the_boundary():
    """At V = 128256 the 8 MiB array holds exactly 8192 rows: that call runs and
    matches the allocating entry point; 8193 rows are refused before any work."""
    need_gpu()
    from linear_cross_entropy_04_b200 import _binding as B

    z, t = _ce_case(41, 8192, 128256, torch.bfloat16)
    g_ref = torch.empty_like(z)
    rc_ref, l_ref = _call("flce_cross_entropy", z, t, B.MEAN, g_ref)
    g_new = torch.empty_like(z)
    rc_new, l_new = _call("flce_cross_entropy_noalloc", z, t, B.MEAN, g_new)
    torch.cuda.synchronize()
    assert rc_ref == 0 and rc_new == 0
    assert rel_err(l_new.item(), l_ref.item()) <= TOL["bf16"]["loss"]
    assert (g_new.float() - g_ref.float()).abs().max().item() <= TOL["bf16"]["grad"] * g_ref.float().abs().max().item()
    del z, g_ref, g_new
    z = torch.empty((8193, 128256), dtype=torch.bfloat16, device="cuda")
    t = torch.zeros(8193, dtype=torch.int64, device="cuda")
    rc, loss = _call("flce_cross_entropy_noalloc", z, t, B.MEAN, None)
    assert rc == 6  # FLCE_ERR_WORKSPACE_TOO_SMALL
    assert torch.isnan(loss).item()


def test_noalloc_refuses_reduction_none():
    need_gpu()
    from linear_cross_entropy_04_b200 import _binding as B

    z, t = _ce_case(51, 64, 1000, torch.bfloat16)
    rc, loss = _call("flce_cross_entropy_noalloc", z, t, B.NONE, None)
    assert rc == 1  # FLCE_ERR_INVALID_ARG
    assert torch.isnan(loss).item()
