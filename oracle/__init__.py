"""CPU oracle for the activation-sparse gated FFN -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The library (the CUDA path) never does
and shares no code with it.

It is a thin ctypes wrapper around ``sffn_oracle.c``: plain fp64 loops that
restate the method,

    y = W_down^T ( act(x W_gate) (*) (x W_up) ),

with the gate evaluated first ("Model Casting and Low-Parameter Gating",
abstract), the gate either dense or LoPA's low-rank product ``A B`` (same
abstract), the active channels chosen by a threshold (``z > tau``,
``act = z - tau``) or per token by top-K of ``SiLU(z)`` ("Mixture-of-Channels",
sections "Dentro il mixture" and "Dentro MoC"), and only the active channels'
``W_up`` columns and ``W_down`` rows used.  The FLOP and byte counters below
follow the same definitions.

Pins (tests/test_oracle_*.py): brute-force enumeration of all masks on tiny
inputs with exact rational arithmetic, the dense special cases K = d_ff and
tau below every gate value against an independent matrix-product chain, the
LoPA identity (x A) B = x (A B), the closed-form active count of a Gaussian
gate, the bitwise sparse == dense invariant, the empty cases, and the page's
3x FLOP cap for a full-size gate.  The published speedups (3.2x FLOPs, 3.31x
GPU, about 1.38x per MoC layer) depend on trained models and unstated
hardware: parity unpinned for those.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass
from typing import List, Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sffn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

ODT_BF16, ODT_F32, ODT_F64 = 0, 1, 2
SEL_THRESHOLD, SEL_TOPK, SEL_TOPP = 0, 1, 2

_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (OpenMP, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fPIC",
                               "-shared", "-std=c11", "-Wall", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    P, I, L, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
    lib.oracle_vecmat.argtypes = [P, I, P, I, L, L, L, P]
    lib.oracle_gate_dense.argtypes = [P, I, P, I, L, L, L, P]
    lib.oracle_gate_lopa.argtypes = [P, I, P, P, I, L, L, L, L, P, P]
    lib.oracle_gate_values.argtypes = [P, L, L, P, P, I, D, P]
    lib.oracle_select_threshold.argtypes = [P, L, L, D, P, P, P]
    lib.oracle_select_topk.argtypes = [P, L, L, L, P, P, P]
    lib.oracle_select_topk.restype = I
    lib.oracle_select_topp.argtypes = [P, L, L, D, P, P, P]
    lib.oracle_select_topp.restype = I
    lib.oracle_sparse_ffn.argtypes = [P, I, P, P, I, L, L, L, P, P, P, P, P]
    lib.oracle_dense_ffn.argtypes = [P, I, P, P, I, L, L, L, P, P]
    lib.oracle_num_threads.restype = I
    lib.oracle_set_threads.argtypes = [I]
    _lib = lib
    return lib


def num_threads() -> int:
    return _load().oracle_num_threads()


def set_threads(n: int) -> None:
    _load().oracle_set_threads(int(n))


def _arr(a):
    """(contiguous numpy array, dtype code) of a torch tensor or numpy array.

    bf16 tensors are passed as their raw 16-bit patterns; nothing is rounded."""
    try:
        import torch
        if isinstance(a, torch.Tensor):
            a = a.detach().cpu().contiguous()
            if a.dtype == torch.bfloat16:
                return a.view(torch.int16).numpy().view(np.uint16), ODT_BF16
            a = a.numpy()
    except ImportError:  # pragma: no cover
        pass
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return a, ODT_BF16
    if a.dtype == np.float32:
        return a, ODT_F32
    if a.dtype == np.float64:
        return a, ODT_F64
    return np.ascontiguousarray(a, dtype=np.float64), ODT_F64


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _same_w_dtype(*ws):
    codes = {c for _, c in ws}
    if len(codes) != 1:
        raise TypeError("all weight matrices must share one storage dtype")
    return codes.pop()


def vecmat(inp, M) -> np.ndarray:
    """out = inp M with inp n x rows, M rows x cols, ascending-order fp64 sums."""
    a, adt = _arr(inp)
    m, mdt = _arr(M)
    n, rows = a.shape
    assert m.shape[0] == rows
    out = np.empty((n, m.shape[1]), np.float64)
    _load().oracle_vecmat(_ptr(a), adt, _ptr(m), mdt, n, rows, m.shape[1], _ptr(out))
    return out


def gate_dense(x, w_gate) -> np.ndarray:
    """z = x W_gate, n x d_ff."""
    a, adt = _arr(x)
    w, wdt = _arr(w_gate)
    n, d = a.shape
    d_ff = w.shape[1]
    z = np.empty((n, d_ff), np.float64)
    _load().oracle_gate_dense(_ptr(a), adt, _ptr(w), wdt, n, d, d_ff, _ptr(z))
    return z


def gate_lopa(x, A, B):
    """(u, z): u = x A (n x r, fp64) and z = u B (n x d_ff)."""
    a, adt = _arr(x)
    A_, B_ = _arr(A), _arr(B)
    wdt = _same_w_dtype(A_, B_)
    n, d = a.shape
    r, d_ff = B_[0].shape
    u = np.empty((n, r), np.float64)
    z = np.empty((n, d_ff), np.float64)
    _load().oracle_gate_lopa(_ptr(a), adt, _ptr(A_[0]), _ptr(B_[0]), wdt, n, d, r, d_ff,
                             _ptr(u), _ptr(z))
    return u, z


def _lists(idx: np.ndarray, cnt: np.ndarray) -> List[np.ndarray]:
    return [idx[t, :cnt[t]].copy() for t in range(idx.shape[0])]


def _packed(sets: Sequence[np.ndarray], d_ff: int):
    n = len(sets)
    idx = np.zeros((n, max(d_ff, 1)), np.int32)
    cnt = np.zeros(n, np.int32)
    for t, s in enumerate(sets):
        s = np.asarray(s, np.int32)
        idx[t, :len(s)] = s
        cnt[t] = len(s)
    return idx, cnt


def select_threshold(z: np.ndarray, tau: float):
    """(sets, g): S_t = {k : z[t,k] > tau} ascending, g = z - tau on S_t, else 0."""
    z = np.ascontiguousarray(z, np.float64)
    n, d_ff = z.shape
    idx = np.zeros((n, max(d_ff, 1)), np.int32)
    cnt = np.zeros(n, np.int32)
    g = np.empty((n, d_ff), np.float64)
    _load().oracle_select_threshold(_ptr(z), n, d_ff, float(tau), _ptr(idx), _ptr(cnt), _ptr(g))
    return _lists(idx, cnt), g


def select_topk(z: np.ndarray, k: int):
    """(sets, g): the k channels of largest SiLU(z) per token (ties: lower index),
    listed ascending; g = SiLU(z) on S_t, else 0."""
    z = np.ascontiguousarray(z, np.float64)
    n, d_ff = z.shape
    idx = np.zeros((n, max(d_ff, 1)), np.int32)
    cnt = np.zeros(n, np.int32)
    g = np.empty((n, d_ff), np.float64)
    if _load().oracle_select_topk(_ptr(z), n, d_ff, int(k), _ptr(idx), _ptr(cnt), _ptr(g)) != 0:
        raise ValueError(f"bad top-K k={k} for d_ff={d_ff}")
    return _lists(idx, cnt), g


def select_topp(z: np.ndarray, p: float):
    """(sets, g): per token the shortest prefix of channels by descending z
    (ties: lower index) whose softmax mass reaches p, listed ascending;
    g = SiLU(z) on S_t, else 0."""
    z = np.ascontiguousarray(z, np.float64)
    n, d_ff = z.shape
    idx = np.zeros((n, max(d_ff, 1)), np.int32)
    cnt = np.zeros(n, np.int32)
    g = np.empty((n, d_ff), np.float64)
    if _load().oracle_select_topp(_ptr(z), n, d_ff, float(p), _ptr(idx), _ptr(cnt), _ptr(g)) != 0:
        raise ValueError(f"bad top-p p={p}")
    return _lists(idx, cnt), g


def gate_values(z: np.ndarray, sets: Sequence[np.ndarray], kind: str, tau: float = 0.0):
    """g = act(z) on the given per-token sets (z - tau or SiLU(z)), 0 elsewhere."""
    z = np.ascontiguousarray(z, np.float64)
    n, d_ff = z.shape
    idx, cnt = _packed(sets, d_ff)
    g = np.empty((n, d_ff), np.float64)
    code = {"threshold": SEL_THRESHOLD, "topk": SEL_TOPK, "topp": SEL_TOPP}[kind]
    _load().oracle_gate_values(_ptr(z), n, d_ff, _ptr(idx), _ptr(cnt), code, float(tau), _ptr(g))
    return g


def sparse_ffn(x, w_up, w_down, sets: Sequence[np.ndarray], g: np.ndarray, want_u: bool = False):
    """y (n x d): sum over each token's listed channels, ascending, of
    g * <x, W_up[:,k]> * W_down[k,:]."""
    a, adt = _arr(x)
    U, D = _arr(w_up), _arr(w_down)
    wdt = _same_w_dtype(U, D)
    n, d = a.shape
    d_ff = U[0].shape[1]
    idx, cnt = _packed(sets, d_ff)
    g = np.ascontiguousarray(g, np.float64)
    y = np.empty((n, d), np.float64)
    u = np.empty((n, d_ff), np.float64) if want_u else None
    _load().oracle_sparse_ffn(_ptr(a), adt, _ptr(U[0]), _ptr(D[0]), wdt, n, d, d_ff, _ptr(idx),
                              _ptr(cnt), _ptr(g), _ptr(y), _ptr(u) if want_u else None)
    return (y, u) if want_u else y


def dense_ffn(x, w_up, w_down, g: np.ndarray):
    """y (n x d) over all d_ff channels with g given densely (0 off the sets)."""
    a, adt = _arr(x)
    U, D = _arr(w_up), _arr(w_down)
    wdt = _same_w_dtype(U, D)
    n, d = a.shape
    d_ff = U[0].shape[1]
    g = np.ascontiguousarray(g, np.float64)
    y = np.empty((n, d), np.float64)
    _load().oracle_dense_ffn(_ptr(a), adt, _ptr(U[0]), _ptr(D[0]), wdt, n, d, d_ff, _ptr(g),
                             _ptr(y))
    return y


@dataclass
class Result:
    z: np.ndarray                 # n x d_ff gate pre-activation
    sets: List[np.ndarray]        # per-token ascending active channels
    g: np.ndarray                 # n x d_ff activation, 0 off the sets
    y: np.ndarray                 # n x d output
    u_lopa: Optional[np.ndarray] = None


def gate(x, weights: dict, gate_mode: str = "dense"):
    if gate_mode == "dense":
        return gate_dense(x, weights["w_gate"]), None
    u, z = gate_lopa(x, weights["A"], weights["B"])
    return z, u


def forward(x, weights: dict, gate_mode: str, select: str, tau: float = 0.0, k: int = 0,
            dense: bool = False, p: float = 0.0) -> Result:
    """The whole path: gate, select, then the sparse (or the dense) FFN."""
    z, u = gate(x, weights, gate_mode)
    if select == "threshold":
        sets, g = select_threshold(z, tau)
    elif select == "topk":
        sets, g = select_topk(z, k)
    else:
        sets, g = select_topp(z, p)
    if dense:
        y = dense_ffn(x, weights["w_up"], weights["w_down"], g)
    else:
        y = sparse_ffn(x, weights["w_up"], weights["w_down"], sets, g)
    return Result(z, sets, g, y, u)


def forward_hybrid(x, weights: dict, gate_mode: str, tau: float, hot) -> Result:
    """The heavy-hitter split with threshold selection (an abstract in the "FFN
    modules" paper listing: a few FFN neurons carry a large output for every
    input while the others fire sparsely, so the FFN is split into a part for
    those neurons and a sparse rest):

        y = dense FFN over the hot channels H, act = ReLU(z - tau)
          + sparse FFN over each token's selected channels outside H.

    The active sets are the threshold sets, whatever H is."""
    z, u = gate(x, weights, gate_mode)
    sets, g = select_threshold(z, tau)
    d_ff = z.shape[1]
    in_h = np.zeros(d_ff, bool)
    in_h[np.asarray(hot, dtype=np.int64).reshape(-1)] = True
    g_hot = np.where(in_h[None, :], np.maximum(z - float(tau), 0.0), 0.0)
    y_hot = dense_ffn(x, weights["w_up"], weights["w_down"], g_hot)
    rest = [s[~in_h[s]] for s in sets]
    y_rest = sparse_ffn(x, weights["w_up"], weights["w_down"], rest, np.where(in_h[None, :], 0.0, g))
    return Result(z, sets, g, y_hot + y_rest, u)


def forward_on_sets(x, weights: dict, gate_mode: str, select: str, sets, tau: float = 0.0):
    """The sparse FFN with the oracle's own gate values on caller-given sets."""
    z, _ = gate(x, weights, gate_mode)
    g = gate_values(z, sets, select, tau)
    return sparse_ffn(x, weights["w_up"], weights["w_down"], sets, g)


# ---------------------------------------------------------------------------
# FLOP and byte counters ("Model Casting and Low-Parameter Gating", abstract:
# gate-first evaluation skips the two other matrices on inactive channels, so
# with a full-size gate the FLOP count falls by at most 3x; LoPA shrinks the
# gate to lift that cap).

def flops(n: int, d: int, d_ff: int, active_total: int, r: int = 0) -> int:
    """Sparse-path FLOPs: gate (2 n d d_ff, or 2 n r (d + d_ff) for LoPA) plus
    2 d for the up dot and 2 d for the down update per active (token, channel)."""
    gate_f = 2 * n * r * (d + d_ff) if r else 2 * n * d * d_ff
    return gate_f + 4 * d * int(active_total)


def dense_flops(n: int, d: int, d_ff: int) -> int:
    """Dense FFN with a full-size gate: three d x d_ff products per token."""
    return 6 * n * d * d_ff


def bytes_moved(n: int, d: int, d_ff: int, union: int, w_bytes: int, x_bytes: int,
                r: int = 0) -> int:
    """Algorithmic HBM bytes of one sparse forward: the gate weights, the union's
    W_up and W_down rows (each read once for all tokens), x read and y written."""
    gate_b = r * (d + d_ff) * w_bytes if r else d * d_ff * w_bytes
    return gate_b + 2 * int(union) * d * w_bytes + 2 * n * d * x_bytes


def dense_bytes(n: int, d: int, d_ff: int, w_bytes: int, x_bytes: int) -> int:
    return 3 * d * d_ff * w_bytes + 2 * n * d * x_bytes


def union_size(sets: Sequence[np.ndarray]) -> int:
    if not sets:
        return 0
    return int(np.unique(np.concatenate([np.asarray(s) for s in sets])).size)
