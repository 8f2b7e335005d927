"""Failure detection on the GPU, without faulting it.

Every wait inside the library's kernels is bounded. flce_gemm_bf16_wait_test
makes one of them run out on purpose: the MMA issuer of every CTA pair waits,
before a chosen output tile, on a barrier that nothing arrives on. The test
checks that the kernel returns by itself after the wait limit, that the host
reads FLCE_DEVERR_TIMEOUT from the device error word, that the tiles finished
before the stall are intact, and that the context stays usable: the next
calls run normally and match their references.
"""
import ctypes
import time

import numpy as np
import pytest
import torch

import oracle
from linear_cross_entropy_04_b200.inputs import WORKLOADS, make_inputs
from flce_testlib import need_gpu, to_dev, rel_err, assert_grad_close

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("stall_tile", [0, 1])
def test_wait_timeout_is_reported_and_the_context_recovers(stall_tile):
    need_gpu()
    import linear_cross_entropy_04_b200 as flce
    from linear_cross_entropy_04_b200 import _binding as B

    assert flce.device_error() == 0
    # 8 x 19 = 152 output tiles of 256 x 256 on 74 pairs: every pair has at least two
    M, N, K = 2048, 19 * 256, 512
    g = torch.Generator(device="cuda").manual_seed(9)
    A = torch.randn(M, K, generator=g, device="cuda").to(torch.bfloat16)
    Bm = torch.randn(N, K, generator=g, device="cuda").to(torch.bfloat16)
    C = torch.full((M, N), float("nan"), device="cuda")
    t0 = time.time()
    rc = B.lib().flce_gemm_bf16_wait_test(A.data_ptr(), Bm.data_ptr(), C.data_ptr(), M, N, K, K, K, N, stall_tile,
                                          B.stream_handle())
    assert rc == 0
    err = flce.device_error()  # waits for the kernel
    elapsed = time.time() - t0
    assert err & B.DEVERR_TIMEOUT, err
    assert 1.0 < elapsed < 60.0, elapsed  # the wait ran out at its limit (about 2 s), no sooner
    ref = A.float() @ Bm.float().t()
    if stall_tile == 1:
        # each pair's first tile (tiles 0..73, m fastest: all 8 row tiles of the first 9 column tiles
        # and 2 of the tenth) was finished before the stall
        torch.testing.assert_close(C[:, : 9 * 256], ref[:, : 9 * 256], rtol=1e-3, atol=1e-2)
    # the context is usable: the same GEMM without the stall, then a full fused call
    C2 = flce.gemm_bf16(A, Bm, M, N, K, False, False)
    torch.testing.assert_close(C2, ref, rtol=1e-3, atol=1e-2)
    d = make_inputs(WORKLOADS["llama3_8b_seq"], BT=300, H=128, V=2000)
    X, W, t = to_dev(d)
    loss, gX, gW = flce.fused_linear_cross_entropy(X, W, t)
    torch.cuda.synchronize()
    assert flce.device_error() == 0
    ref = oracle.flce(d["X"], d["W"], d["target"])
    assert rel_err(loss.item(), ref["loss"]) <= 1e-3
    assert_grad_close(gX, ref["grad_X"], "bf16", "grad_X after a timeout")
    assert_grad_close(gW, ref["grad_W"], "bf16", "grad_W after a timeout")
