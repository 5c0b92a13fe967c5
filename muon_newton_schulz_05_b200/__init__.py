"""Python binding of libmuonb200.so (B200 / sm_100a Muon optimizer step).

Argument marshalling only: every step of the optimizer runs in the library's
CUDA kernels. PyTorch provides device memory and streams; the C ABI takes raw
pointers (``tensor.data_ptr()``) and a ``cudaStream_t`` (the current torch
stream unless one is given). Importing this module fails if the compiled
library is missing; build it with ``python muon_newton_schulz_05_b200/build.py``.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass, field
from typing import List, Optional, Sequence, Tuple

_PKG = os.path.dirname(os.path.abspath(__file__))
# MUON_B200_CHECK=1 selects the debug build with device-side bounds checks
# (`build.py --check`); the default is the release library.
LIB_PATH = os.path.join(_PKG, "libmuonb200_check.so" if os.environ.get("MUON_B200_CHECK") == "1"
                        else "libmuonb200.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python muon_newton_schulz_05_b200/build.py"
        f"{' --check' if LIB_PATH.endswith('_check.so') else ''}` "
        "(this package has no fallback implementation)")

_lib = ctypes.CDLL(LIB_PATH)

MAX_NS_STEPS = 16
MAX_BANKS = 8
F32, BF16 = 0, 1

STATUS_NAMES = {
    0: "MUON_OK", 1: "MUON_ERR_NULL", 2: "MUON_ERR_SHAPE", 3: "MUON_ERR_DTYPE",
    4: "MUON_ERR_ALIGN", 5: "MUON_ERR_HPARAM", 6: "MUON_ERR_WORKSPACE", 7: "MUON_ERR_CUDA",
    8: "MUON_ERR_TIMEOUT", 9: "MUON_ERR_ALIAS", 10: "MUON_ERR_BOUNDS",
}

EXPORTED = ("muon_abi_version", "muon_status_string", "muon_workspace_size", "muon_step",
            "anvil_step", "muon_orthogonalize", "ema_update", "readout_blend",
            "muon_device_status", "muon_set_debug", "muon_set_ns_events",
            "muon_orthogonalize_static", "muon_chain_plan")


class MuonError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {status_string(code)}")


class CBank(ctypes.Structure):
    _fields_ = [("count", ctypes.c_int64), ("rows", ctypes.c_int64), ("cols", ctypes.c_int64),
                ("param", ctypes.c_void_p), ("param_dtype", ctypes.c_int32),
                ("grad_dtype", ctypes.c_int32), ("grad", ctypes.c_void_p),
                ("momentum", ctypes.c_void_p), ("momentum_slow", ctypes.c_void_p),
                ("ema", ctypes.c_void_p)]


class CHparams(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_float), ("mu", ctypes.c_float),
                ("weight_decay", ctypes.c_float), ("eps", ctypes.c_float),
                ("nesterov", ctypes.c_int32), ("ns_steps", ctypes.c_int32),
                ("coeffs", ctypes.c_float * (3 * MAX_NS_STEPS)), ("ema_beta", ctypes.c_float),
                ("beta_fast", ctypes.c_float), ("beta_slow", ctypes.c_float),
                ("sgd_momentum", ctypes.c_int32)]


_vp, _i32, _i64, _sz, _f = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
_sig = {
    "muon_abi_version": (_i32, []),
    "muon_status_string": (ctypes.c_char_p, [_i32]),
    "muon_workspace_size": (_sz, [ctypes.POINTER(CBank), _i32]),
    "muon_step": (_i32, [ctypes.POINTER(CBank), _i32, ctypes.POINTER(CHparams), _vp, _sz, _vp]),
    "anvil_step": (_i32, [ctypes.POINTER(CBank), _i32, ctypes.POINTER(CHparams), _vp, _sz, _vp]),
    "muon_orthogonalize": (_i32, [_vp, _i32, _vp, _i32, _i64, _i64, _i64,
                                  ctypes.POINTER(CHparams), _vp, _sz, _vp]),
    "ema_update": (_i32, [ctypes.POINTER(CBank), _i32, _f, _vp]),
    "readout_blend": (_i32, [_vp, _i32, _vp, _vp, _i32, _i64, _f, _vp]),
    "muon_device_status": (_i32, [_vp, _sz, _vp, _i32]),
    "muon_set_debug": (_i32, [_i32, ctypes.c_double]),
    "muon_set_ns_events": (_i32, [_vp, _vp]),
    "muon_chain_plan": (_i64, [ctypes.POINTER(_i64), _i32, _i32, ctypes.POINTER(_i32), _i64]),
    "muon_orthogonalize_static": (_i32, [_vp, _i32, _vp, _i32, _i64, _i64, _i64,
                                         ctypes.POINTER(CHparams), _vp]),
}
for _name, (_res, _args) in _sig.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


def status_string(code: int) -> str:
    return _lib.muon_status_string(int(code)).decode()


def abi_version() -> int:
    return int(_lib.muon_abi_version())


def _check(code: int, what: str) -> None:
    if code != 0:
        raise MuonError(code, what)


# ---------------------------------------------------------------- data types
@dataclass
class Bank:
    """A bank of same-shape matrices: tensors [count, rows, cols] on one device.

    param: bf16 or fp32; grad: bf16 or fp32; momentum (M or ANVIL's M_fast),
    momentum_slow and ema: fp32 (the last two optional)."""
    param: "object"
    grad: "object"
    momentum: "object"
    momentum_slow: Optional["object"] = None
    ema: Optional["object"] = None

    @property
    def shape(self) -> Tuple[int, int, int]:
        s = tuple(self.param.shape)
        return (1, s[0], s[1]) if len(s) == 2 else s  # type: ignore[return-value]


@dataclass
class Hparams:
    lr: float = 0.02
    mu: float = 0.95
    weight_decay: float = 0.0
    eps: float = 1e-7
    nesterov: bool = True
    coeffs: Sequence[Sequence[float]] = field(default_factory=lambda: [(3.4445, -4.7750, 2.0315)] * 5)
    ema_beta: float = 0.99
    beta_fast: float = 0.9
    beta_slow: float = 0.99
    sgd_momentum: bool = False

    @classmethod
    def from_dict(cls, d: dict) -> "Hparams":
        keys = {k: d[k] for k in ("lr", "mu", "weight_decay", "eps", "nesterov", "coeffs",
                                  "ema_beta", "beta_fast", "beta_slow", "sgd_momentum") if k in d}
        return cls(**keys)

    def to_c(self) -> CHparams:
        h = CHparams()
        h.lr, h.mu, h.weight_decay, h.eps = self.lr, self.mu, self.weight_decay, self.eps
        h.nesterov = 1 if self.nesterov else 0
        h.ns_steps = len(self.coeffs)  # range checked by the library (MUON_ERR_HPARAM)
        for i, (a, b, c) in enumerate(list(self.coeffs)[:MAX_NS_STEPS]):
            h.coeffs[3 * i], h.coeffs[3 * i + 1], h.coeffs[3 * i + 2] = a, b, c
        h.ema_beta, h.beta_fast, h.beta_slow = self.ema_beta, self.beta_fast, self.beta_slow
        h.sgd_momentum = 1 if self.sgd_momentum else 0
        return h


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    return 99  # rejected by the library with MUON_ERR_DTYPE


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to the library must be contiguous")
    return t.data_ptr()


def _cbanks(banks: Sequence[Bank]):
    arr = (CBank * max(1, len(banks)))()
    for i, b in enumerate(banks):
        cnt, r, c = b.shape
        arr[i].count, arr[i].rows, arr[i].cols = cnt, r, c
        arr[i].param = _ptr(b.param)
        arr[i].param_dtype = _dtype_code(b.param)
        arr[i].grad = _ptr(b.grad)
        arr[i].grad_dtype = _dtype_code(b.grad)
        arr[i].momentum = _ptr(b.momentum)
        arr[i].momentum_slow = _ptr(b.momentum_slow)
        arr[i].ema = _ptr(b.ema)
        for t in (b.momentum, b.momentum_slow, b.ema):
            if t is not None and _dtype_code(t) != F32:
                raise ValueError("momentum buffers and the EMA must be float32")
    return arr


def _stream_handle(stream) -> Optional[int]:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


# ---------------------------------------------------------------- entry points
def workspace_size(banks_or_shapes) -> int:
    """Bytes of workspace for a list of Banks or (count, rows, cols) tuples."""
    shapes = [b.shape if isinstance(b, Bank) else tuple(b) for b in banks_or_shapes]
    arr = (CBank * max(1, len(shapes)))()
    for i, (cnt, r, c) in enumerate(shapes):
        arr[i].count, arr[i].rows, arr[i].cols = cnt, r, c
    return int(_lib.muon_workspace_size(arr, len(shapes)))


def alloc_workspace(banks_or_shapes, device="cuda"):
    """A zero-filled uint8 workspace tensor of the right size."""
    import torch
    n = workspace_size(banks_or_shapes)
    if n == 0:
        raise MuonError(2, "workspace_size")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def muon_step(banks: Sequence[Bank], hp: Hparams, workspace, stream=None) -> None:
    arr = _cbanks(banks)
    h = hp.to_c()
    _check(_lib.muon_step(arr, len(banks), ctypes.byref(h), _ptr(workspace),
                          workspace.numel() * workspace.element_size(), _stream_handle(stream)),
           "muon_step")


def anvil_step(banks: Sequence[Bank], hp: Hparams, workspace, stream=None) -> None:
    arr = _cbanks(banks)
    h = hp.to_c()
    _check(_lib.anvil_step(arr, len(banks), ctypes.byref(h), _ptr(workspace),
                           workspace.numel() * workspace.element_size(), _stream_handle(stream)),
           "anvil_step")


def orthogonalize(x, out, hp: Hparams, workspace, stream=None) -> None:
    """out = NS(x / (||x||_F + eps)) per matrix; x, out: [count, rows, cols]."""
    s = tuple(x.shape)
    cnt, r, c = (1, s[0], s[1]) if len(s) == 2 else s
    h = hp.to_c()
    _check(_lib.muon_orthogonalize(_ptr(x), _dtype_code(x), _ptr(out), _dtype_code(out), cnt, r, c,
                                   ctypes.byref(h), _ptr(workspace),
                                   workspace.numel() * workspace.element_size(),
                                   _stream_handle(stream)), "muon_orthogonalize")


def ema_update(banks: Sequence[Bank], beta: float, stream=None) -> None:
    arr = _cbanks(banks)
    _check(_lib.ema_update(arr, len(banks), beta, _stream_handle(stream)), "ema_update")


def checkpoint_average_betas(weights: Sequence[float]) -> List[float]:
    """The beta of each ema_update call that turns the EMA recurrence into a
    weighted checkpoint average sum_i w_i theta_i / sum_i w_i: checkpoint n
    uses beta_n = 1 - w_n / (w_1 + ... + w_n) (so beta_1 = 0: the average
    starts at the first checkpoint). A checkpoint with weight 0 gets beta = 1,
    which ema_update rejects: skip its call instead. Host scalars only; the
    averaging itself is ema_update's kernel."""
    out, total = [], 0.0
    for w in weights:
        w = float(w)
        if w < 0.0:
            raise ValueError("checkpoint weights must be non-negative")
        total += w
        if total <= 0.0:
            raise ValueError("the first checkpoint needs a positive weight")
        out.append(1.0 - w / total)
    return out


def readout_blend(theta, ema, out, w_final: float = 0.35, stream=None) -> None:
    _check(_lib.readout_blend(_ptr(theta), _dtype_code(theta), _ptr(ema), _ptr(out),
                              _dtype_code(out), theta.numel(), w_final, _stream_handle(stream)),
           "readout_blend")


def device_status(workspace, stream=None, clear: bool = False) -> int:
    """Synchronises the stream and returns the workspace's device status code."""
    return int(_lib.muon_device_status(_ptr(workspace), workspace.numel() * workspace.element_size(),
                                       _stream_handle(stream), 1 if clear else 0))


def set_debug(fault_mode: int = 0, wait_limit_seconds: float = 0.0) -> None:
    _check(_lib.muon_set_debug(fault_mode, wait_limit_seconds), "muon_set_debug")


def set_ns_events(before, after) -> None:
    """The next step call records these torch.cuda.Events around its
    Newton-Schulz launches (instrumentation for the benchmark)."""
    _check(_lib.muon_set_ns_events(before.cuda_event if before is not None else None,
                                   after.cuda_event if after is not None else None),
           "muon_set_ns_events")


def raw_library():
    """The ctypes handle (used by tests that call the C ABI directly)."""
    return _lib


def loaded_library_path() -> str:
    return LIB_PATH


__all__: List[str] = ["Bank", "Hparams", "MuonError", "workspace_size", "alloc_workspace",
                      "muon_step", "anvil_step", "orthogonalize", "ema_update", "readout_blend",
                      "checkpoint_average_betas",
                      "device_status", "set_debug", "set_ns_events", "status_string", "abi_version",
                      "raw_library", "CBank", "CHparams", "EXPORTED", "F32", "BF16"]
