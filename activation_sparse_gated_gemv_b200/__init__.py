"""Activation-sparse gated FFN inference for B200 (sm_100a).

A thin ctypes binding over the C ABI in ``include/sffn.h`` (``libsffn.so``,
built in-tree by ``build.py``).  The functions ``sffn_*`` below carry the C
names and only marshal arguments; every step of the computation runs in the
library's CUDA kernels.  PyTorch is used for device memory and streams only.

    y = W_down^T ( act(x W_gate) (*) (x W_up) )

with the gate evaluated first (dense, or LoPA's rank-r ``A B``), channels
selected by a threshold (``z > tau``, act = ``z - tau``), per-token top-K of
``SiLU(z)``, or per-token top-p of the softmax mass of z, and only the active
channels' ``W_up``/``W_down`` rows read ("Model Casting and Low-Parameter
Gating", abstract; "Mixture-of-Channels", sections "Dentro il mixture" and
"Dentro MoC"; "PrunePath", abstract).

There is no fallback: importing this package builds ``libsffn.so`` if it is
missing and fails if it cannot, and every call that needs a GPU fails if there
is none.
"""
from __future__ import annotations

import ctypes
import os
from typing import List, Optional, Tuple

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsffn.so")

SFFN_OK = 0
SFFN_ERR_INVALID_ARG = 1
SFFN_ERR_NOT_READY = 2
SFFN_ERR_UNSUPPORTED = 3
SFFN_ERR_CUDA = 4
SFFN_ERR_OOM = 5
SFFN_ERR_TIMEOUT = 6
SFFN_ERR_DEVICE_CHECK = 7

SFFN_BF16, SFFN_F32 = 0, 1
SFFN_GATE_DENSE, SFFN_GATE_LOPA = 0, 1
SFFN_SELECT_THRESHOLD, SFFN_SELECT_TOPK, SFFN_SELECT_TOPP = 0, 1, 2
SFFN_INJECT_WAIT_TIMEOUT, SFFN_INJECT_BAD_LIST_ENTRY = 1, 2


class sffn_config(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int32), ("d_ff", ctypes.c_int32), ("lopa_rank", ctypes.c_int32),
                ("max_tokens", ctypes.c_int32), ("wdtype", ctypes.c_int32), ("device", ctypes.c_int32)]


class sffn_select(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("tau", ctypes.c_float), ("k", ctypes.c_int32), ("p", ctypes.c_float)]


from . import build as _build  # noqa: E402

if not _build.up_to_date():
    # a fresh checkout, or sources newer than the library: compile it in-tree
    # first (nvcc, sm_100a); if that fails the import fails with it
    _build.build()
_lib = ctypes.CDLL(LIB_PATH)

_P, _I = ctypes.c_void_p, ctypes.c_int
_sigs = {
    "sffn_create": ([ctypes.POINTER(ctypes.c_void_p), ctypes.POINTER(sffn_config)], _I),
    "sffn_set_weights": ([_P, _P, _P, _P, _P, _P, _I, _P], _I),
    "sffn_forward": ([_P, _P, _I, _I, ctypes.POINTER(sffn_select), _P, _P], _I),
    "sffn_forward_dense": ([_P, _P, _I, _I, ctypes.POINTER(sffn_select), _P, _P], _I),
    "sffn_forward_host": ([_P, _P, _I, _I, ctypes.POINTER(sffn_select), _P, _P], _I),
    "sffn_get_active": ([_P, _P, _P, _P], _I),
    "sffn_set_stage_events": ([_P, ctypes.POINTER(ctypes.c_void_p), _I], _I),
    "sffn_last_launches": ([_P, _P], _I),
    "sffn_check_status": ([_P], _I),
    "sffn_destroy": ([_P], _I),
    "sffn_strerror": ([_I], ctypes.c_char_p),
    "sffn_last_error": ([], ctypes.c_char_p),
    "sffn_forward_noalloc": ([_P, _P, _P, _I, _I, _I, _P, _I, ctypes.c_float, _P, _P], _I),
    "sffn_last_kernel_name": ([_P, _I], ctypes.c_char_p),
    "sffn_set_hot": ([_P, _P, _I], _I),
    "sffn_get_union": ([_P, _P, _I], _I),
    "sffn_debug_inject": ([_P, _I, ctypes.c_longlong], _I),
    "sffn_noalloc_check_status": ([], _I),
}
for _name, (_args, _res) in _sigs.items():
    _f = getattr(_lib, _name)
    _f.argtypes = _args
    _f.restype = _res

# The C entry points under their own names.
sffn_create = _lib.sffn_create
sffn_set_weights = _lib.sffn_set_weights
sffn_forward = _lib.sffn_forward
sffn_forward_dense = _lib.sffn_forward_dense
sffn_forward_host = _lib.sffn_forward_host
sffn_get_active = _lib.sffn_get_active
sffn_set_stage_events = _lib.sffn_set_stage_events
sffn_last_launches = _lib.sffn_last_launches
sffn_check_status = _lib.sffn_check_status
sffn_destroy = _lib.sffn_destroy
sffn_strerror = _lib.sffn_strerror
sffn_last_error = _lib.sffn_last_error
sffn_forward_noalloc = _lib.sffn_forward_noalloc
sffn_last_kernel_name = _lib.sffn_last_kernel_name
sffn_set_hot = _lib.sffn_set_hot
sffn_get_union = _lib.sffn_get_union
sffn_debug_inject = _lib.sffn_debug_inject
sffn_noalloc_check_status = _lib.sffn_noalloc_check_status

EXPORTED = tuple(_sigs)


class SFFNError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        msg = sffn_strerror(code).decode()
        detail = sffn_last_error().decode()
        super().__init__(f"{where}: {msg} ({code}){': ' + detail if detail else ''}")


def check(code: int, where: str) -> None:
    if code != SFFN_OK:
        raise SFFNError(code, where)


def _torch():
    import torch
    return torch


def _stream_ptr(stream) -> Optional[int]:
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def make_select(select: str = "threshold", tau: float = 0.0, k: int = 0, p: float = 0.0) -> sffn_select:
    kind = {"threshold": SFFN_SELECT_THRESHOLD, "topk": SFFN_SELECT_TOPK, "topp": SFFN_SELECT_TOPP}[select]
    return sffn_select(kind, float(tau), int(k), float(p))


def gate_code(gate: str) -> int:
    return {"dense": SFFN_GATE_DENSE, "lopa": SFFN_GATE_LOPA}[gate]


class SparseFFN:
    """One FFN layer's weights on one GPU, behind an ``sffn_handle``."""

    def __init__(self, d: int, d_ff: int, lopa_rank: int = 0, max_tokens: int = 1,
                 dtype: str = "bf16", device: int = 0):
        self.d, self.d_ff, self.r = d, d_ff, lopa_rank
        self.max_tokens = max_tokens
        self.dtype = dtype
        self.device = device
        self._h = ctypes.c_void_p()
        cfg = sffn_config(d, d_ff, lopa_rank, max_tokens, SFFN_BF16 if dtype == "bf16" else SFFN_F32, device)
        check(sffn_create(ctypes.byref(self._h), ctypes.byref(cfg)), "sffn_create")

    @property
    def handle(self):
        return self._h

    def _tdtype(self):
        torch = _torch()
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    def set_weights(self, w_gate=None, A=None, B=None, w_up=None, w_down=None, stream=None) -> None:
        """Row-major tensors (all on the CPU, or all on this GPU) in the handle's dtype."""
        ts = [t for t in (w_gate, A, B, w_up, w_down) if t is not None]
        on_dev = ts[0].is_cuda
        keep = []

        def ptr(t):
            if t is None:
                return None
            if t.dtype != self._tdtype() or t.is_cuda != on_dev:
                raise TypeError("weights must share the handle's dtype and one memory kind")
            t = t.contiguous()
            keep.append(t)
            return t.data_ptr()

        args = [ptr(t) for t in (w_gate, A, B, w_up, w_down)]
        check(sffn_set_weights(self._h, *args, 1 if on_dev else 0,
                               _stream_ptr(stream) if on_dev else None), "sffn_set_weights")

    def forward(self, x, gate: str = "dense", select: str = "threshold", tau: float = 0.0, k: int = 0,
                out=None, stream=None, dense: bool = False, p: float = 0.0):
        """y for device tokens x (n x d); asynchronous on the stream."""
        torch = _torch()
        n = x.shape[0]
        if out is None:
            out = torch.empty((n, self.d), dtype=x.dtype, device=x.device)
        sel = make_select(select, tau, k, p)
        fn = sffn_forward_dense if dense else sffn_forward
        check(fn(self._h, x.data_ptr(), n, gate_code(gate), ctypes.byref(sel), out.data_ptr(),
                 _stream_ptr(stream)), "sffn_forward_dense" if dense else "sffn_forward")
        return out

    def forward_host(self, x, gate: str = "dense", select: str = "threshold", tau: float = 0.0, k: int = 0,
                     out=None, stream=None, p: float = 0.0):
        """y for host tokens x (n x d, CPU tensor; pinned for async copies); synchronous."""
        torch = _torch()
        n = x.shape[0]
        if out is None:
            out = torch.empty((n, self.d), dtype=x.dtype, pin_memory=x.is_pinned())
        sel = make_select(select, tau, k, p)
        check(sffn_forward_host(self._h, x.data_ptr(), n, gate_code(gate), ctypes.byref(sel),
                                out.data_ptr(), _stream_ptr(stream)), "sffn_forward_host")
        return out

    def active(self, n: int) -> Tuple[List[np.ndarray], int]:
        """(per-token ascending active channel lists, union size) of the last forward."""
        idx = np.zeros((n, self.d_ff), np.int32)
        cnt = np.zeros(n, np.int32)
        uni = ctypes.c_int32(0)
        check(sffn_get_active(self._h, idx.ctypes.data_as(ctypes.c_void_p),
                              cnt.ctypes.data_as(ctypes.c_void_p), ctypes.byref(uni)), "sffn_get_active")
        return [idx[t, :cnt[t]].copy() for t in range(n)], int(uni.value)

    def union_bits(self) -> np.ndarray:
        """The union bitmap (uint32 words, bit k = channel k) the last
        tensor-core forward's up and down kernels read their active blocks from."""
        words = (self.d_ff + 31) // 32
        bits = np.zeros(words, np.uint32)
        check(sffn_get_union(self._h, bits.ctypes.data_as(ctypes.c_void_p), words), "sffn_get_union")
        return bits

    def debug_inject(self, what: int, arg: int = 0) -> None:
        """Arm a one-shot host-side failure injection (SFFN_INJECT_*)."""
        check(sffn_debug_inject(self._h, int(what), int(arg)), "sffn_debug_inject")

    def set_hot(self, channels) -> None:
        """Heavy-hitter channels (any int sequence; empty clears the set): the
        fused decode kernel takes their up dots before the gate selects them.
        y and the active lists do not change."""
        a64 = np.asarray(channels, dtype=np.int64).reshape(-1)
        if a64.size and (a64.min() < -2**31 or a64.max() >= 2**31):
            raise SFFNError(SFFN_ERR_INVALID_ARG, "sffn_set_hot")
        arr = np.ascontiguousarray(a64.astype(np.int32))
        check(sffn_set_hot(self._h, arr.ctypes.data_as(ctypes.c_void_p) if arr.size else None, int(arr.size)),
              "sffn_set_hot")

    def set_stage_events(self, events) -> None:
        arr = (ctypes.c_void_p * max(1, len(events)))(*[e.cuda_event for e in events])
        check(sffn_set_stage_events(self._h, arr, len(events)), "sffn_set_stage_events")

    def last_launches(self) -> int:
        v = ctypes.c_int32(0)
        check(sffn_last_launches(self._h, ctypes.byref(v)), "sffn_last_launches")
        return int(v.value)

    def last_kernel_names(self) -> List[str]:
        return [sffn_last_kernel_name(self._h, i).decode() for i in range(self.last_launches())]

    def check_status(self) -> None:
        check(sffn_check_status(self._h), "sffn_check_status")

    def close(self) -> None:
        if self._h:
            sffn_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
