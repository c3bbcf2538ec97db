"""sffn_forward_noalloc: the forward for callers that cannot allocate device
memory while they run (a runtime that owns all device memory through its own
pool, or latency-critical code where an allocation may stall the device).
It takes the caller's channel-major weights and keeps its scratch in a
file-scope device array, so it needs no handle.

Checked against the CPU oracle directly and against the handle-based
sffn_forward on the same weights and tokens, on two calls in a row (the second
finds the first call's leftovers in the shared scratch), with the tolerance of
the parity tests; one case sits at the documented limits (d = 8192, 8 tokens,
the 70B-shaped d_ff).  After the calls the no-alloc status word must be clean.
This file is named to run last so that a run stopping at the first failure has
run the rest.
"""
import pytest
import torch

import oracle
import workloads
from parity import YTOL, assert_y, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sffn(cuda_device):
    from activation_sparse_gated_gemv_b200 import build
    build.build()
    import activation_sparse_gated_gemv_b200 as m
    return m


CASES = [
    # d, d_ff, n, dtype, tau, oracle tokens
    (4096, 11008, 1, "bf16", workloads.tau_for_sparsity(0.9), [0]),
    (512, 3000, 5, "bf16", workloads.tau_for_sparsity(0.8), None),
    (256, 1024, 4, "f32", 1.2816, None),
    (8192, 28672, 8, "bf16", workloads.tau_for_sparsity(0.9), [0, 7]),   # at the limits
]


@pytest.mark.parametrize("d,d_ff,n,dtype,tau,tokens", CASES)
def test_noalloc_matches_oracle_and_handle_forward_twice(sffn, d, d_ff, n, dtype, tau, tokens):
    w = workloads.ffn_weights(d, d_ff, dtype, seed=d_ff + 1)
    x_cpu = workloads.tokens(n, d, dtype, seed=d_ff + 2)
    x = x_cpu.cuda()
    ffn = sffn.SparseFFN(d, d_ff, 0, n, dtype)
    ffn.set_weights(**w)
    y_ref = ffn.forward(x, gate="dense", select="threshold", tau=tau)
    torch.cuda.synchronize()
    ffn.close()

    # The caller's weights, already in the kernels' channel-major layout.
    wg_cm = w["w_gate"].t().contiguous().cuda()
    wu_cm = w["w_up"].t().contiguous().cuda()
    wd = w["w_down"].cuda()
    code = sffn.SFFN_BF16 if dtype == "bf16" else sffn.SFFN_F32
    stream = torch.cuda.current_stream().cuda_stream
    outs = [torch.full_like(x, float("nan")) for _ in range(2)]
    for out in outs:
        rc = sffn.sffn_forward_noalloc(wg_cm.data_ptr(), wu_cm.data_ptr(), wd.data_ptr(), d, d_ff, code,
                                       x.data_ptr(), n, tau, out.data_ptr(), stream)
        assert rc == sffn.SFFN_OK
        torch.cuda.synchronize()
    assert sffn.sffn_noalloc_check_status() == sffn.SFFN_OK
    tok = list(range(n)) if tokens is None else tokens
    ref = oracle.forward(x_cpu[tok], w, "dense", "threshold", tau=tau)
    for i, out in enumerate(outs):
        assert_y(to_np(out), to_np(y_ref), YTOL, f"call {i + 1} vs the handle forward")
        assert_y(to_np(out)[tok], ref.y, YTOL, f"call {i + 1} vs the oracle")
    del wg_cm, wu_cm, wd


def test_noalloc_rejects_sizes_beyond_its_limits(sffn):
    t = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    p = t.data_ptr()
    for d, d_ff, n in ((8200, 1024, 1), (4096, 32769, 1), (4096, 1024, 9), (12, 1024, 1)):
        rc = sffn.sffn_forward_noalloc(p, p, p, d, d_ff, sffn.SFFN_BF16, p, n, 1.0, p, None)
        assert rc == sffn.SFFN_ERR_INVALID_ARG, (d, d_ff, n)
    assert sffn.sffn_noalloc_check_status() == sffn.SFFN_OK
