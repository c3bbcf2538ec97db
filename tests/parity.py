"""Comparison rules between the CUDA path and the oracle (test helper).

* Active sets: identical per token, except channels whose oracle gate value
  lies within EXEMPT of the decision boundary (tau for threshold, the K-th
  largest SiLU value for top-K), where fp32 and fp64 rounding may disagree;
  for top-p, channels whose cumulative softmax mass lies within EXEMPT of the
  budget (the kernel sums the masses in fixed point).
* Outputs: per token, max |y_gpu - y_ref| <= YTOL * max |y_ref| with y_ref the
  oracle evaluated on the GPU's own sets (and, for threshold, on its own sets
  too: the activation z - tau is continuous at the boundary).  A token whose
  reference is all zeros must come back exactly zero.
"""
import numpy as np
import torch

import oracle

EXEMPT = 1e-3
YTOL = 2e-2


def silu(z):
    return z / (1.0 + np.exp(-z))


def to_np(t):
    return t.detach().to("cpu", torch.float64).numpy()


def topp_exempt(z, p, tol=EXEMPT):
    """Channels the top-p decision may flip: where the oracle's cumulative
    softmax mass (descending z, ties to the lower index) before or after the
    channel lies within tol of the budget p, or whose z is within EXEMPT of
    the boundary channel's."""
    z = np.asarray(z, np.float64)
    order = np.lexsort((np.arange(z.size), -z))
    w = np.exp(z[order] - z.max())
    total = w.sum()
    cum_after = np.cumsum(w) / total
    cum_before = cum_after - w / total
    near = (np.abs(cum_before - p) <= tol) | (np.abs(cum_after - p) <= tol)
    q = int(np.searchsorted(cum_after, p * (1 - 1e-12)))
    zb = z[order[min(q, z.size - 1)]]
    return set(order[near].tolist()) | set(np.nonzero(np.abs(z - zb) <= EXEMPT)[0].tolist())


def assert_sets(gpu_sets, ref, select, tau=0.0, k=0, tokens=None, p=0.0):
    tokens = range(len(gpu_sets)) if tokens is None else tokens
    for i, t in enumerate(tokens):
        gs = np.asarray(gpu_sets[i])
        assert np.all(np.diff(gs) > 0), f"token {t}: list not strictly ascending"
        a, b = set(gs.tolist()), set(np.asarray(ref.sets[i]).tolist())
        diff = sorted(a ^ b)
        z = ref.z[i]
        if select == "threshold":
            bad = [c for c in diff if abs(z[c] - tau) > EXEMPT]
        elif select == "topp":
            ex = topp_exempt(z, p) if diff else set()
            bad = [c for c in diff if c not in ex]
        else:
            assert len(gs) == k, f"token {t}: {len(gs)} selected, expected {k}"
            s = silu(z)
            gk = np.sort(s)[::-1][k - 1] if k > 0 else np.inf
            bad = [c for c in diff if abs(s[c] - gk) > EXEMPT]
        assert not bad, f"token {t}: {len(bad)} channels differ outside the exempt band: {bad[:8]}"


def assert_y(y_gpu, y_ref, tol=YTOL, what=""):
    y_gpu = np.asarray(y_gpu, np.float64)
    y_ref = np.asarray(y_ref, np.float64)
    assert y_gpu.shape == y_ref.shape
    assert np.all(np.isfinite(y_gpu)), what
    for t in range(y_ref.shape[0]):
        m = np.abs(y_ref[t]).max()
        err = np.abs(y_gpu[t] - y_ref[t]).max()
        if m == 0:
            assert err == 0, f"{what} token {t}: expected zeros, max |y| = {err}"
        else:
            assert err <= tol * m, f"{what} token {t}: max err {err:.3e} > {tol} * {m:.3e}"


def check_forward(ffn, w, x_cpu, gate, select, tau=0.0, k=0, dense=False, tokens=None, tol=YTOL, p=0.0):
    """Run the CUDA path on all of x, compare the tokens listed (default all)
    with the oracle; returns (y_gpu, gpu_sets, union)."""
    x_dev = x_cpu.cuda()
    y = ffn.forward(x_dev, gate=gate, select=select, tau=tau, k=k, dense=dense, p=p)
    torch.cuda.synchronize()
    ffn.check_status()
    sets, union = ffn.active(x_cpu.shape[0])
    tok = list(range(x_cpu.shape[0])) if tokens is None else list(tokens)
    xs = x_cpu[tok]
    ref = oracle.forward(xs, w, gate, select, tau=tau, k=k, p=p)
    gsets = [sets[t] for t in tok]
    assert_sets(gsets, ref, select, tau, k, tokens=tok, p=p)
    yg = to_np(y)[tok]
    y_on_gpu_sets = oracle.forward_on_sets(xs, w, gate, select, gsets, tau=tau)
    assert_y(yg, y_on_gpu_sets, tol, "vs oracle on the GPU's sets")
    if select == "threshold":
        assert_y(yg, ref.y, tol, "vs oracle on its own sets")
    return y, sets, union
