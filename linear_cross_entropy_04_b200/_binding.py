"""ctypes binding to libflce.so: argument marshalling only.

Every step of the computation runs in the CUDA library; this module turns
torch tensors into flce_tensor descriptors (pointer, dtype, shape, strides),
allocates outputs with torch (device memory plumbing) and checks status codes.
There is no fallback: if the library is missing or the device is not a B200,
the call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

PKG = os.path.dirname(os.path.abspath(__file__))
# FLCE_LIBRARY may name another build of the same library (e.g. a tuning variant)
LIB_PATH = os.environ.get("FLCE_LIBRARY") or os.path.join(PKG, "libflce.so")

F32, BF16, I64 = 0, 1, 2
MEAN, SUM, NONE = 0, 1, 2
FLAG_SYNC_CHECK, FLAG_TIME_PHASES, FLAG_KEEP_LOGITS, FLAG_FROM_KEPT = 0x1, 0x2, 0x4, 0x8
FLAG_ROUTE_EVERY_CHUNK, FLAG_RECOMPUTE = 0x10, 0x20
GRADW_ACCUM_OUTPUT, GRADW_ACCUM_FP32 = 0, 1
DEVERR_TARGET_RANGE, DEVERR_TIMEOUT = 0x1, 0x2
NUM_PHASES = 6
PHASE_NAMES = ["count_valid", "logits_gemm_softmax", "row_combine", "dlogits_inplace",
               "grad_gemms", "loss_reduce"]

STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported dtype", 3: "unsupported device",
          4: "workspace allocation failed", 5: "CUDA error", 6: "workspace too small"}


class FlceTensor(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("ndim", ctypes.c_int32),
                ("shape", ctypes.c_int64 * 2), ("stride", ctypes.c_int64 * 2)]


class FlceOptions(ctypes.Structure):
    _fields_ = [("chunk_rows", ctypes.c_int64), ("workspace_limit_bytes", ctypes.c_int64),
                ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_int64),
                ("grad_w_accum", ctypes.c_int32), ("flags", ctypes.c_int32),
                ("n_valid", ctypes.c_void_p), ("row_loss", ctypes.c_void_p), ("lse", ctypes.c_void_p),
                ("row_grad", ctypes.c_void_p), ("grad_w_shards", ctypes.POINTER(ctypes.c_void_p)),
                ("n_shards", ctypes.c_int32), ("shard_rows", ctypes.c_int64), ("grad_w_shard_ld", ctypes.c_int64),
                ("grad_w_ready_event", ctypes.c_void_p)]


class FlceStats(ctypes.Structure):
    _fields_ = [("chunk_rows", ctypes.c_int64), ("n_chunks", ctypes.c_int64),
                ("workspace_bytes", ctypes.c_int64), ("materialized_logits_bytes", ctypes.c_int64),
                ("kernel_launches", ctypes.c_int32), ("path", ctypes.c_int32)]

    def as_dict(self):
        return {f: getattr(self, f) for f, _ in self._fields_}


class FlceError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, 'unknown status')} ({status})")


_lock = threading.Lock()
_lib = None

_P = ctypes.POINTER
_SIGS = {
    "flce_options_init": (None, [_P(FlceOptions)]),
    "flce_fwd_bwd": (ctypes.c_int, [_P(FlceTensor), _P(FlceTensor), _P(FlceTensor), ctypes.c_int64,
                                    ctypes.c_int32, _P(FlceTensor), _P(FlceTensor), _P(FlceTensor),
                                    ctypes.c_void_p]),
    "flce_fwd_bwd_ex": (ctypes.c_int, [_P(FlceTensor), _P(FlceTensor), _P(FlceTensor), ctypes.c_int64,
                                       ctypes.c_int32, _P(FlceTensor), _P(FlceTensor), _P(FlceTensor),
                                       ctypes.c_void_p, _P(FlceOptions), _P(FlceStats)]),
    "flce_plan": (ctypes.c_int, [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int32,
                                 ctypes.c_int32, _P(FlceOptions), _P(FlceStats)]),
    "flce_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int32,
                                               _P(FlceOptions)]),
    "flce_count_valid": (ctypes.c_int, [_P(FlceTensor), ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p,
                                        ctypes.c_void_p]),
    "flce_cross_entropy": (ctypes.c_int, [_P(FlceTensor), _P(FlceTensor), ctypes.c_int64, ctypes.c_int32,
                                          _P(FlceTensor), _P(FlceTensor), ctypes.c_void_p, _P(FlceOptions)]),
    "flce_cross_entropy_noalloc": (ctypes.c_int, [_P(FlceTensor), _P(FlceTensor), ctypes.c_int64, ctypes.c_int32,
                                                  _P(FlceTensor), _P(FlceTensor), ctypes.c_void_p]),
    "flce_gemm_bf16": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                      ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                      ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p]),
    "flce_gemm_bf16_wait_test": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                                ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                                ctypes.c_int64, ctypes.c_int32, ctypes.c_void_p]),
    "flce_scale_grad": (ctypes.c_int, [_P(FlceTensor), ctypes.c_void_p, ctypes.c_void_p]),
    "flce_get_device_error": (ctypes.c_int, [ctypes.c_void_p, _P(ctypes.c_uint32)]),
    "flce_phase_times": (ctypes.c_int, [_P(ctypes.c_double), _P(ctypes.c_int32), ctypes.c_int32,
                                        ctypes.c_int32]),
    "flce_status_string": (ctypes.c_char_p, [ctypes.c_int32]),
    "flce_version": (ctypes.c_int32, []),
}


def lib():
    """Load libflce.so (built in-tree) once; raise if it is missing."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is not built; run `python -m linear_cross_entropy_04_b200.build`")
            L = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in _SIGS.items():
                fn = getattr(L, name)
                fn.restype = res
                fn.argtypes = args
            _lib = L
        return _lib


def check(status, where):
    if status != 0:
        raise FlceError(status, where)


def dtype_code(t) -> int:
    import torch

    return {torch.float32: F32, torch.bfloat16: BF16, torch.int64: I64}[t.dtype]


def tensor(t) -> FlceTensor:
    """Describe a torch tensor (rank 0-2) without copying it."""
    if t.dim() > 2:
        raise ValueError("flce tensors have rank <= 2")
    d = FlceTensor()
    d.data = t.data_ptr() if t.numel() > 0 or t.data_ptr() else None
    d.dtype = dtype_code(t)
    d.ndim = t.dim()
    for i in range(t.dim()):
        d.shape[i] = t.shape[i]
        d.stride[i] = t.stride(i)
    return d


def ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def stream_handle(stream=None):
    import torch

    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)
