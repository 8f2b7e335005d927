"""Shared helpers for the GPU tests: device staging and the parity bars.

Tolerances are the ones the task states for this path:
  loss: relative error <= 1e-3 (bf16) / 1e-4 (fp32);
  grad_X, grad_W: max |gpu - ref| <= 2e-2 * max |ref| (bf16) / 1e-4 * max |ref| (fp32).
"""
import numpy as np
import pytest
import torch

TOL = {"bf16": {"loss": 1e-3, "grad": 2e-2}, "f32": {"loss": 1e-4, "grad": 1e-4}}
TDT = {"bf16": torch.bfloat16, "f32": torch.float32}


def need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    major, minor = torch.cuda.get_device_capability()
    if (major, minor) != (10, 0):
        pytest.skip("needs sm_100 (B200)")
    from linear_cross_entropy_04_b200 import build

    build.build()


def to_dev(d, dtype=None):
    dt = TDT[dtype or d["dtype"]]
    X = torch.from_numpy(d["X"]).to(dt).cuda()
    W = torch.from_numpy(d["W"]).to(dt).cuda()
    t = torch.from_numpy(d["target"]).cuda()
    return X, W, t


def rel_err(a, b):
    return abs(float(a) - float(b)) / max(abs(float(b)), 1e-30)


def assert_grad_close(gpu, ref, dtype, name):
    g = gpu.float().cpu().numpy().astype(np.float64) if isinstance(gpu, torch.Tensor) else gpu
    scale = float(np.abs(ref).max())
    err = float(np.abs(g - ref).max())
    bound = TOL[dtype]["grad"] * max(scale, 1e-30)
    assert err <= bound, f"{name}: max|err| {err:.3e} > {bound:.3e} (max|ref| {scale:.3e})"
    return err / max(scale, 1e-30)
