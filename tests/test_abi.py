"""Host-side checks of the C ABI: the library loads, exports every declared
entry point, and rejects bad arguments before touching a GPU."""
import ctypes
import os
import re

import pytest

from linear_cross_entropy_04_b200 import _binding as B
from linear_cross_entropy_04_b200 import build as build_mod

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "flce.h")


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return B.lib()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"FLCE_API\s+[\w\s\*]+?\b(flce_\w+)\s*\(", text)))


def exported_symbols():
    import subprocess

    out = subprocess.run(["nm", "-D", "--defined-only", B.LIB_PATH], capture_output=True, text=True).stdout
    return {ln.split()[-1] for ln in out.splitlines() if " T " in ln}


def test_every_declared_entry_point_is_exported(lib):
    decl = declared_functions()
    assert len(decl) >= 11
    exported = exported_symbols()
    missing = [d for d in decl if d not in exported]
    assert not missing, missing
    for d in decl:
        assert hasattr(lib, d)


def test_binding_signatures_cover_the_header():
    assert set(declared_functions()) == set(B._SIGS)


def test_version_and_status_strings(lib):
    assert lib.flce_version() == 120
    assert lib.flce_status_string(0) == b"ok"
    assert b"unsupported device" in lib.flce_status_string(3)
    assert lib.flce_status_string(99) == b"unknown status"


def _t(ptr, dtype, shape, stride=None):
    d = B.FlceTensor()
    d.data = ptr
    d.dtype = dtype
    d.ndim = len(shape)
    for i, n in enumerate(shape):
        d.shape[i] = n
    if stride is None:
        stride = [1] * len(shape)
        for i in range(len(shape) - 2, -1, -1):
            stride[i] = stride[i + 1] * shape[i + 1]
    for i, s in enumerate(stride):
        d.stride[i] = s
    return d


FAKE = 0x10000  # never dereferenced: validation fails before any device work


def _call(lib, X, W, tg, loss, gX=None, gW=None, reduction=0):
    ref = lambda t: ctypes.byref(t) if t is not None else None  # noqa: E731
    return lib.flce_fwd_bwd(ref(X), ref(W), ref(tg), -100, reduction, ref(loss), ref(gX), ref(gW), None)


@pytest.mark.parametrize("case", ["null_X", "null_loss", "dtype_mix", "bad_dtype", "shape_H", "target_len",
                                  "target_dtype", "stride", "bad_reduction", "bf16_H_mod8", "bf16_misaligned",
                                  "grad_shape", "loss_shape"])
def test_invalid_arguments_are_rejected_on_the_host(lib, case):
    X = _t(FAKE, B.BF16, (64, 128))
    W = _t(FAKE, B.BF16, (1000, 128))
    tg = _t(FAKE, B.I64, (64,))
    loss = _t(FAKE, B.F32, ())
    gX, gW, red = None, None, 0
    expect = 1
    if case == "null_X":
        X = None
    elif case == "null_loss":
        loss = None
    elif case == "dtype_mix":
        W = _t(FAKE, B.F32, (1000, 128))
        expect = 2
    elif case == "bad_dtype":
        X = _t(FAKE, B.I64, (64, 128))
        expect = 2
    elif case == "shape_H":
        W = _t(FAKE, B.BF16, (1000, 120))
    elif case == "target_len":
        tg = _t(FAKE, B.I64, (63,))
    elif case == "target_dtype":
        tg = _t(FAKE, B.F32, (64,))
    elif case == "stride":
        X = _t(FAKE, B.BF16, (64, 128), stride=(128, 2))
    elif case == "bad_reduction":
        red = 7
    elif case == "bf16_H_mod8":
        X = _t(FAKE, B.BF16, (64, 100))
        W = _t(FAKE, B.BF16, (1000, 100))
    elif case == "bf16_misaligned":
        X = _t(FAKE + 2, B.BF16, (64, 128))
    elif case == "grad_shape":
        gW = _t(FAKE, B.BF16, (999, 128))
    elif case == "loss_shape":
        loss = _t(FAKE, B.F32, (2,))
    assert _call(lib, X, W, tg, loss, gX, gW, red) == expect


def test_other_entry_points_validate(lib):
    assert lib.flce_gemm_bf16(None, None, None, 1, 1, 1, 8, 8, 4, 0, 0, None) == 1
    assert lib.flce_gemm_bf16(FAKE, FAKE, FAKE, 16, 16, 16, 12, 16, 16, 0, 0, None) == 1  # lda % 8
    assert lib.flce_count_valid(None, 10, -100, None, None) == 1
    z = _t(FAKE, B.BF16, (4, 100))
    tg = _t(FAKE, B.I64, (3,))
    loss = _t(FAKE, B.F32, ())
    assert lib.flce_cross_entropy(ctypes.byref(z), ctypes.byref(tg), -100, 0, ctypes.byref(loss), None, None,
                                  None) == 1
    assert lib.flce_get_device_error(None, None) == 1
    assert lib.flce_phase_times(None, None, -1, 0) == 1
    g = _t(FAKE, B.BF16, (4, 100))
    assert lib.flce_scale_grad(None, FAKE, None) == 1                    # no tensor
    assert lib.flce_scale_grad(ctypes.byref(g), None, None) == 1         # no scale
    assert lib.flce_scale_grad(ctypes.byref(tg), FAKE, None) == 2        # int64 is not a gradient
    bad = _t(FAKE, B.BF16, (4, 100), stride=(50, 1))                     # rows overlap
    assert lib.flce_scale_grad(ctypes.byref(bad), FAKE, None) == 1
    empty = _t(None, B.F32, (0, 8))
    assert lib.flce_scale_grad(ctypes.byref(empty), FAKE, None) == 0     # nothing to scale, no device needed


def test_plan_is_host_only_and_bounded(lib):
    from linear_cross_entropy_04_b200.inputs import WORKLOADS
    from linear_cross_entropy_04_b200 import plan

    for w in WORKLOADS.values():
        p = plan(w.BT, w.H, w.V, w.dtype)
        assert p["n_chunks"] >= 2, w.name  # the logits of the whole batch are never held
        assert p["chunk_rows"] % 128 == 0 and p["chunk_rows"] * (p["n_chunks"] - 1) < w.BT
        if w.dtype == "bf16":
            # at most 512 MiB of chunk store, or the 2048-row floor's store when that is larger
            store_2048 = 2048 * (-(-w.V // 64) * 64) * 2
            assert p["workspace_bytes"] <= max(512 << 20, store_2048) + (64 << 20)
            assert p["chunk_rows"] >= min(2048, -(-w.BT // 2))
            assert p["workspace_bytes"] < 0.55 * w.BT * w.V * 2
    p = plan(4096, 4096, 128256, chunk_rows=1000)
    assert p["chunk_rows"] == 1024 and p["n_chunks"] == 4
    p = plan(4096, 4096, 128256, workspace_limit_bytes=300 << 20)
    assert p["workspace_bytes"] <= (300 << 20) + (8 << 20)
    acc = plan(4096, 4096, 128256, grad_w_accum="fp32")
    assert acc["workspace_bytes"] - plan(4096, 4096, 128256)["workspace_bytes"] >= 128256 * 4096 * 4
    st = B.FlceStats()
    assert lib.flce_plan(10, 0, 10, B.BF16, 1, None, ctypes.byref(st)) == 1
    assert lib.flce_plan(10, 8, 10, B.I64, 1, None, ctypes.byref(st)) == 2


def test_missing_library_fails_loudly(monkeypatch):
    monkeypatch.setattr(B, "_lib", None)
    monkeypatch.setattr(B, "LIB_PATH", "/nonexistent/libflce.so")
    with pytest.raises(RuntimeError, match="not built"):
        B.lib()


def test_plain_c_caller(tmp_path, lib):
    """The ABI works from C: compile tests/c/abi_smoke.c against include/flce.h."""
    import shutil
    import subprocess

    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    exe = tmp_path / "abi_smoke"
    libdir = os.path.dirname(B.LIB_PATH)
    r = subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                        os.path.join(ROOT, "tests", "c", "abi_smoke.c"), "-o", str(exe),
                        "-L", libdir, "-l:libflce.so", f"-Wl,-rpath,{libdir}"], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.strip().endswith("ok")


def test_grad_W_shard_options_are_validated(lib):
    X = _t(FAKE, B.BF16, (64, 128))
    W = _t(FAKE, B.BF16, (1000, 128))
    tg = _t(FAKE, B.I64, (64,))
    loss = _t(FAKE, B.F32, ())
    ptrs = (ctypes.c_void_p * 2)(FAKE, FAKE)
    for rows, n, ld in ((500, 2, 128), (512, 1, 128), (512, 2, 100)):  # rows % 32, n*rows < V, ld < H
        o = B.FlceOptions()
        lib.flce_options_init(ctypes.byref(o))
        o.grad_w_shards = ctypes.cast(ptrs, ctypes.POINTER(ctypes.c_void_p))
        o.n_shards, o.shard_rows, o.grad_w_shard_ld = n, rows, ld
        st = B.FlceStats()
        rc = lib.flce_fwd_bwd_ex(ctypes.byref(X), ctypes.byref(W), ctypes.byref(tg), -100, 0, ctypes.byref(loss),
                                 None, None, None, ctypes.byref(o), ctypes.byref(st))
        assert rc == 1, (rows, n, ld)


def test_keep_flags_are_validated(lib):
    X = _t(FAKE, B.BF16, (64, 128))
    W = _t(FAKE, B.BF16, (1000, 128))
    tg = _t(FAKE, B.I64, (64,))
    loss = _t(FAKE, B.F32, ())
    gW = _t(FAKE, B.BF16, (1000, 128))

    def call(flags, workspace, grad_W=None, X=X, tg=tg):
        o = B.FlceOptions()
        lib.flce_options_init(ctypes.byref(o))
        o.flags = flags
        if workspace:
            o.workspace, o.workspace_bytes = FAKE * 256, 1 << 40
        return lib.flce_fwd_bwd_ex(ctypes.byref(X), ctypes.byref(W), ctypes.byref(tg), -100, 0,
                                   ctypes.byref(loss), None, ctypes.byref(grad_W) if grad_W else None, None,
                                   ctypes.byref(o), None)

    assert call(B.FLAG_KEEP_LOGITS, False) == 1                      # the store needs a caller workspace
    assert call(B.FLAG_FROM_KEPT, False) == 1
    assert call(B.FLAG_KEEP_LOGITS | B.FLAG_FROM_KEPT, True) == 1    # one phase at a time
    assert call(B.FLAG_KEEP_LOGITS, True, grad_W=gW) == 1            # the forward phase takes no gradients
    big_X, big_t = _t(FAKE, B.BF16, (40000, 128)), _t(FAKE, B.I64, (40000,))
    assert call(B.FLAG_KEEP_LOGITS, True, X=big_X, tg=big_t) == 1    # more rows than one chunk holds
    st = B.FlceStats()
    o = B.FlceOptions()
    lib.flce_options_init(ctypes.byref(o))
    o.flags = B.FLAG_KEEP_LOGITS
    assert lib.flce_plan(4096, 4096, 128256, B.BF16, 1, ctypes.byref(o), ctypes.byref(st)) == 0
    assert st.n_chunks == 1 and st.chunk_rows == 4096
    assert st.workspace_bytes >= 4096 * 128256 * 2


def test_workspace_bytes_matches_the_plan(lib):
    """flce_workspace_bytes is flce_plan's workspace figure with grad_W requested."""
    for BT, H, V, dt in ((4096, 4096, 128256, B.BF16), (512, 256, 4096, B.F32), (16384, 2048, 256000, B.BF16)):
        st = B.FlceStats()
        assert lib.flce_plan(BT, H, V, dt, 1, None, ctypes.byref(st)) == 0
        assert lib.flce_workspace_bytes(BT, H, V, dt, None) == st.workspace_bytes > 0
    o = B.FlceOptions()
    lib.flce_options_init(ctypes.byref(o))
    o.grad_w_accum = B.GRADW_ACCUM_FP32
    st = B.FlceStats()
    assert lib.flce_plan(4096, 4096, 128256, B.BF16, 1, ctypes.byref(o), ctypes.byref(st)) == 0
    assert lib.flce_workspace_bytes(4096, 4096, 128256, B.BF16, ctypes.byref(o)) == st.workspace_bytes
    assert lib.flce_workspace_bytes(0, 4096, 128256, B.BF16, None) == 0          # empty batch
    invalid = ctypes.c_size_t(-1).value
    assert lib.flce_workspace_bytes(10, 0, 10, B.BF16, None) == invalid          # H = 0
    assert lib.flce_workspace_bytes(10, 8, 10, B.I64, None) == invalid           # not a float dtype


def test_python_api_rejects_bad_option_strings():
    """Bad option strings fail in Python with a clear error, before any device work."""
    import torch

    from linear_cross_entropy_04_b200 import api

    X, W, t = torch.zeros(4, 8), torch.zeros(10, 8), torch.zeros(4, dtype=torch.int64)
    with pytest.raises(ValueError, match="reduction"):
        api.fused_linear_cross_entropy(X, W, t, reduction="avg")
    with pytest.raises(ValueError, match="reduction"):
        api.cross_entropy(torch.zeros(4, 10), t, reduction="total")
    with pytest.raises(ValueError, match="reduction"):
        api.forward_keep(X, W, t, reduction="mean_")
    with pytest.raises(ValueError, match="grad_w_accum"):
        api.plan(4, 8, 10, grad_w_accum="fp16")


def test_build_dependencies_cover_every_source(tmp_path, monkeypatch):
    """Every file under csrc/ and every public header counts for up_to_date():
    touching any one of them makes the built library stale."""
    srcs = set(os.listdir(os.path.join(build_mod.PKG, "csrc")))
    deps = build_mod.deps()
    assert {os.path.basename(d) for d in deps if os.sep + "csrc" + os.sep in d} == srcs
    assert HEADER in deps
    # a fake library newer than every source is up to date until one source is newer
    fake = tmp_path / "libflce.so"
    fake.write_bytes(b"")
    newest = max(os.path.getmtime(d) for d in deps)
    os.utime(fake, (newest + 10, newest + 10))
    monkeypatch.setattr(build_mod, "OUT", str(fake))
    assert build_mod.up_to_date()
    os.utime(fake, (newest - 1, newest - 1))
    assert not build_mod.up_to_date()


def test_chunk_rows_environment_override(lib, monkeypatch):
    """FLCE_CHUNK_ROWS sets the chunk rows when the options leave them at 0; an
    explicit option wins, and values that are not positive integers are ignored."""
    def plan(opt_rows=0):
        o = B.FlceOptions()
        lib.flce_options_init(ctypes.byref(o))
        o.chunk_rows = opt_rows
        st = B.FlceStats()
        assert lib.flce_plan(4096, 4096, 128256, B.BF16, 1, ctypes.byref(o), ctypes.byref(st)) == 0
        return st.chunk_rows, st.n_chunks

    monkeypatch.delenv("FLCE_CHUNK_ROWS", raising=False)
    default = plan()
    assert default == (2048, 2)
    monkeypatch.setenv("FLCE_CHUNK_ROWS", "1000")
    assert plan() == (1024, 4)          # rounded up to 128
    assert plan(opt_rows=512) == (512, 8)
    for bad in ("", "abc", "-5", "0", "12x"):
        monkeypatch.setenv("FLCE_CHUNK_ROWS", bad)
        assert plan() == default, bad


def _nvtx_recorder(tmp_path):
    """Build tests/c/nvtx_record.c, a minimal NVTX tool that logs range pushes and pops."""
    import shutil
    import subprocess

    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    so = tmp_path / "nvtx_record.so"
    r = subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-shared", "-fPIC", "-I", "/usr/local/cuda/include",
                        os.path.join(ROOT, "tests", "c", "nvtx_record.c"), "-o", str(so)],
                       capture_output=True, text=True)
    if r.returncode != 0 and "nvToolsExt.h" in r.stderr:
        pytest.skip("NVTX 3 headers not found")
    assert r.returncode == 0, r.stderr
    return so


def run_with_nvtx(tmp_path, code):
    """Run `code` in a fresh Python with the NVTX recorder injected; return the logged lines."""
    import subprocess
    import sys

    so = _nvtx_recorder(tmp_path)
    log = tmp_path / "nvtx.log"
    env = dict(os.environ, NVTX_INJECTION64_PATH=str(so), FLCE_NVTX_LOG=str(log), PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    return log.read_text().splitlines() if log.exists() else []


def test_nvtx_range_around_each_call(tmp_path, lib):
    """Every compute entry point opens an NVTX range for its call, closed on
    every return path (here: an argument error, found before any device work)."""
    code = ("from linear_cross_entropy_04_b200 import _binding as B\n"
            "L = B.lib()\n"
            "assert L.flce_fwd_bwd(None, None, None, -100, 0, None, None, None, None) == 1\n"
            "assert L.flce_cross_entropy(None, None, -100, 0, None, None, None, None) == 1\n")
    assert run_with_nvtx(tmp_path, code) == ["push flce_fwd_bwd", "pop", "push flce_cross_entropy", "pop"]


def test_recompute_schedule_plan(lib):
    """The recompute schedule's workspace: the [BT, Vc] store with Vc from the
    option or the budget, plus per-row lse / losses and one row block's partials;
    it refuses f32, the two-phase flags and grad_W shards on the host."""
    from linear_cross_entropy_04_b200.api import plan

    a256 = lambda n: (n + 255) // 256 * 256  # noqa: E731
    BT, H, V = 4096, 4096, 128256
    p = plan(BT, H, V, schedule="recompute", chunk_rows=1000)
    assert p["chunk_rows"] == 1024 and p["n_chunks"] == -(-V // 1024)
    ntile = -(-V // 256)
    expect = a256(8) + a256(4 * BT) + a256(4 * 4096) + 2 * a256(4 * ntile * 4096) + a256(BT * 1024 * 2) + a256(4 * BT)
    assert p["workspace_bytes"] == expect
    q = plan(BT, H, V, schedule="recompute", workspace_limit_bytes=64 << 20)
    assert q["chunk_rows"] == (64 << 20) // (BT * 2) // 256 * 256 == 8192
    d = plan(BT, H, V, schedule="recompute")
    assert d["chunk_rows"] == 65536 and d["n_chunks"] == 2   # 512 MiB over 4096 rows
    tiny = plan(BT, H, V, schedule="recompute", chunk_rows=1)
    assert tiny["chunk_rows"] == 256 and tiny["workspace_bytes"] < plan(BT, H, V)["workspace_bytes"] / 8
    whole = plan(100, 64, 1000, schedule="recompute", chunk_rows=5000)
    assert whole["chunk_rows"] == 1024 and whole["n_chunks"] == 1  # capped at V rounded up to 256
    st = B.FlceStats()
    for flags, dt, code in ((B.FLAG_RECOMPUTE, B.F32, 2), (B.FLAG_RECOMPUTE | B.FLAG_KEEP_LOGITS, B.BF16, 1),
                            (B.FLAG_RECOMPUTE | B.FLAG_FROM_KEPT, B.BF16, 1)):
        o = B.FlceOptions()
        lib.flce_options_init(ctypes.byref(o))
        o.flags = flags
        assert lib.flce_plan(BT, H, V, dt, 1, ctypes.byref(o), ctypes.byref(st)) == code, (flags, dt)
    o = B.FlceOptions()
    lib.flce_options_init(ctypes.byref(o))
    o.flags = B.FLAG_RECOMPUTE
    o.n_shards, o.shard_rows = 2, 64128
    assert lib.flce_plan(BT, H, V, B.BF16, 1, ctypes.byref(o), ctypes.byref(st)) == 1
    with pytest.raises(ValueError, match="schedule"):
        plan(BT, H, V, schedule="vocab")


def test_wait_test_hook_validates(lib, monkeypatch):
    """flce_gemm_bf16_wait_test refuses, on the host, what flce_gemm_bf16 refuses, a
    negative stall tile, and the single-CTA engine (the hook lives in the pair engine)."""
    assert lib.flce_gemm_bf16_wait_test(None, None, None, 1, 1, 1, 8, 8, 4, 0, None) == 1
    assert lib.flce_gemm_bf16_wait_test(FAKE, FAKE, FAKE, 16, 16, 16, 16, 16, 16, -1, None) == 1
    monkeypatch.setenv("FLCE_ENGINE", "1sm")
    assert lib.flce_gemm_bf16_wait_test(FAKE, FAKE, FAKE, 256, 256, 64, 64, 64, 256, 0, None) == 1


def test_options_struct_matches_the_header():
    """The ctypes mirror of flce_options ends with grad_w_ready_event, as the header
    does, and has the C struct's size (compiled with gcc from the header)."""
    import ctypes
    import shutil
    import subprocess
    import tempfile

    from linear_cross_entropy_04_b200 import _binding as B

    names = [f for f, _ in B.FlceOptions._fields_]
    assert names[-1] == "grad_w_ready_event"
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no gcc")
    with tempfile.TemporaryDirectory() as d:
        src = os.path.join(d, "sz.c")
        with open(src, "w") as f:
            f.write('#include <stdio.h>\n#include <stddef.h>\n#include "flce.h"\n'
                    'int main(void) { printf("%zu %zu\\n", sizeof(flce_options), '
                    'offsetof(flce_options, grad_w_ready_event)); return 0; }\n')
        exe = os.path.join(d, "sz")
        r = subprocess.run([gcc, "-std=c99", "-I", os.path.join(ROOT, "include"), src, "-o", exe],
                           capture_output=True, text=True)
        assert r.returncode == 0, r.stderr
        size, off = map(int, subprocess.run([exe], capture_output=True, text=True).stdout.split())
    assert size == ctypes.sizeof(B.FlceOptions)
    assert off == B.FlceOptions.grad_w_ready_event.offset
