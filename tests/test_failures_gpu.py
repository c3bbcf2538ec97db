"""Failure handling through the C ABI, with every failure planted on the host.

* A bounded device wait that runs out: the fused decode kernel's final grid
  barrier is armed to expect one arrival more than its grid makes, with a 1 ms
  limit.  The kernel gives up, records the timeout in the handle's status word
  and returns; the context stays usable.
* A bad list entry: the host overwrites a gate list entry and a segment count
  between the gate and the down kernel; the down kernel's own checks skip both
  and record them.
* Allocation and copy failures in sffn_create / sffn_set_weights, through the
  SFFN_FAULT environment variable: the call fails cleanly, frees what it took,
  and the handle stays usable.

No test here makes a kernel fault, trap or hang.
"""
import os

import pytest
import torch

import workloads
from parity import check_forward

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sffn(cuda_device):
    from activation_sparse_gated_gemv_b200 import build
    build.build()
    import activation_sparse_gated_gemv_b200 as m
    return m


def _handle(sffn, d=256, d_ff=2048, r=0, n=1, dtype="bf16", seed=11):
    w = workloads.ffn_weights(d, d_ff, dtype, seed=seed, gate="both" if r else "dense", r=r)
    ffn = sffn.SparseFFN(d, d_ff, r, n, dtype)
    ffn.set_weights(**w)
    return ffn, w


def test_timed_out_grid_barrier_is_reported_and_sticky(sffn):
    ffn, w = _handle(sffn)
    tau = workloads.tau_for_sparsity(0.9)
    x = workloads.tokens(1, 256, "bf16", seed=12)
    check_forward(ffn, w, x, "dense", "threshold", tau=tau)          # a clean forward first
    assert ffn.last_kernel_names() == ["decode_fused"]
    ffn.debug_inject(sffn.SFFN_INJECT_WAIT_TIMEOUT, 1_000_000)       # 1 ms, then a barrier no one completes
    ffn.forward(x.cuda(), tau=tau)                                   # asynchronous: returns OK
    torch.cuda.synchronize()
    with pytest.raises(sffn.SFFNError) as e:
        ffn.check_status()
    assert e.value.code == sffn.SFFN_ERR_TIMEOUT
    # the next calls see it without synchronising, and launch nothing
    for call in (lambda: ffn.forward(x.cuda(), tau=tau), lambda: ffn.forward(x.cuda(), tau=tau, dense=True),
                 lambda: ffn.forward_host(x.pin_memory(), tau=tau), lambda: ffn.active(1)):
        with pytest.raises(sffn.SFFNError) as e:
            call()
        assert e.value.code == sffn.SFFN_ERR_TIMEOUT
    ffn.close()
    # the context is still usable: a new handle runs and matches the oracle
    ffn2, w2 = _handle(sffn, seed=13)
    check_forward(ffn2, w2, x, "dense", "threshold", tau=tau)
    ffn2.close()


def test_bad_list_entry_is_caught_by_the_down_kernel(sffn):
    # fp32 top-K runs gate (z) -> top-K -> selected up -> down as separate kernels
    d, d_ff, n = 64, 500, 3
    ffn, w = _handle(sffn, d=d, d_ff=d_ff, n=n, dtype="f32", seed=14)
    x = workloads.tokens(n, d, "f32", seed=15)
    check_forward(ffn, w, x, "dense", "topk", k=d_ff // 8)
    assert ffn.last_kernel_names()[-1] == "down"
    ffn.debug_inject(sffn.SFFN_INJECT_BAD_LIST_ENTRY)
    ffn.forward(x.cuda(), select="topk", k=d_ff // 8)
    torch.cuda.synchronize()
    with pytest.raises(sffn.SFFNError) as e:
        ffn.check_status()
    assert e.value.code == sffn.SFFN_ERR_DEVICE_CHECK
    with pytest.raises(sffn.SFFNError) as e:
        ffn.forward(x.cuda(), select="topk", k=d_ff // 8)
    assert e.value.code == sffn.SFFN_ERR_DEVICE_CHECK
    ffn.close()


def test_inject_rejects_bad_arguments(sffn):
    ffn, _ = _handle(sffn, d=64, d_ff=128)
    for what, arg in ((sffn.SFFN_INJECT_WAIT_TIMEOUT, 10), (sffn.SFFN_INJECT_WAIT_TIMEOUT, 10**10), (99, 0)):
        with pytest.raises(sffn.SFFNError) as e:
            ffn.debug_inject(what, arg)
        assert e.value.code == sffn.SFFN_ERR_INVALID_ARG
    ffn.close()


def _with_fault(spec, fn):
    os.environ["SFFN_FAULT"] = spec
    try:
        return fn()
    finally:
        del os.environ["SFFN_FAULT"]


@pytest.mark.parametrize("n", [1, 2])
def test_create_fails_cleanly_on_allocation_failure(sffn, n):
    """alloc:1 is the workspace, alloc:2 the host-mapped status mirror."""
    import ctypes
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    h = ctypes.c_void_p()
    cfg = sffn.sffn_config(256, 2048, 0, 4, sffn.SFFN_BF16, 0)
    rc = _with_fault(f"alloc:{n}", lambda: sffn.sffn_create(ctypes.byref(h), ctypes.byref(cfg)))
    assert rc == sffn.SFFN_ERR_OOM and not h.value
    torch.cuda.synchronize()
    assert abs(torch.cuda.mem_get_info()[0] - free0) < 8 << 20
    # without the fault the same call works
    assert sffn.sffn_create(ctypes.byref(h), ctypes.byref(cfg)) == sffn.SFFN_OK
    sffn.sffn_destroy(h)


@pytest.mark.parametrize("spec,code", [("alloc:1", "OOM"), ("alloc:3", "OOM"), ("alloc:5", "OOM"),
                                       ("copy:1", "CUDA"), ("copy:2", "CUDA"), ("copy:3", "CUDA")])
def test_set_weights_fails_cleanly_and_recovers(sffn, spec, code):
    d, d_ff, r = 1024, 4096, 64                # 8 MB per weight matrix: a kept one shows
    w = workloads.ffn_weights(d, d_ff, "bf16", seed=16, gate="both", r=r)
    ffn = sffn.SparseFFN(d, d_ff, r, 1, "bf16")
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    with pytest.raises(sffn.SFFNError) as e:
        _with_fault(spec, lambda: ffn.set_weights(**w))
    assert e.value.code == getattr(sffn, f"SFFN_ERR_{code}")
    torch.cuda.synchronize()
    assert abs(torch.cuda.mem_get_info()[0] - free0) < 4 << 20       # nothing it took is kept
    x = workloads.tokens(1, d, "bf16", seed=17)
    with pytest.raises(sffn.SFFNError) as e:
        ffn.forward(x.cuda())
    assert e.value.code == sffn.SFFN_ERR_NOT_READY
    ffn.set_weights(**w)                                             # recovers
    check_forward(ffn, w, x, "lopa", "threshold", tau=workloads.tau_for_sparsity(0.9))
    ffn.close()


def test_status_is_clean_after_normal_forwards(sffn):
    ffn, w = _handle(sffn, r=64, n=8)
    tau = workloads.tau_for_sparsity(0.9)
    for n, gate, select in ((1, "dense", "threshold"), (1, "lopa", "threshold"), (8, "dense", "topk"),
                            (8, "lopa", "threshold"), (2, "dense", "topp")):
        x = workloads.tokens(n, 256, "bf16", seed=18 + n)
        ffn.forward(x.cuda(), gate=gate, select=select, tau=tau, k=256, p=0.5)
    ffn.check_status()
    ffn.close()
