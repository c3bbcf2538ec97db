"""Pins for the CPU oracle: each check holds it to something other than itself.

* brute force over every mask on tiny inputs, in exact rational arithmetic;
* special cases that reduce to a plain matrix-product chain (numpy): top-K with
  K = d_ff is the dense SwiGLU FFN, a threshold below every gate value is an
  affine-gated (bilinear) FFN, LoPA's two stages equal x (A B);
* the closed-form active count of a Gaussian gate;
* the sparse == dense invariant behind gate-first evaluation ("Model Casting
  and Low-Parameter Gating", abstract);
* the empty cases (tau = +inf, K = 0);
* the page's 3x FLOP cap for a full-size gate and its lifting by LoPA.
"""
import itertools
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _np64(t):
    return t.to(torch.float64).numpy()


def _silu_np(z):
    return z / (1.0 + np.exp(-z))


def _tiny_weights(d, d_ff, n, seed, dtype="bf16", r=0):
    gate = "both" if r else "dense"
    w = workloads.ffn_weights(d, d_ff, dtype, seed=seed, gate=gate, r=r)
    x = workloads.tokens(n, d, dtype, seed=seed)
    return w, x


# --------------------------------------------------------------------------
# brute force

def _exact(t):
    return [[Fraction(float(v)) for v in row] for row in t.to(torch.float64).tolist()]


@pytest.mark.parametrize("seed,d,d_ff,n", [(1, 3, 8, 2), (2, 5, 10, 2), (3, 8, 12, 1)])
def test_threshold_set_and_y_by_brute_force(seed, d, d_ff, n):
    w, x = _tiny_weights(d, d_ff, n, seed)
    tau = 0.1234567
    X, WG, WU, WD = _exact(x), _exact(w["w_gate"]), _exact(w["w_up"]), _exact(w["w_down"])
    T = Fraction(tau)
    res = oracle.forward(x, w, "dense", "threshold", tau=tau)
    for t in range(n):
        z = [sum(X[t][j] * WG[j][k] for j in range(d)) for k in range(d_ff)]
        assert all(zk != T for zk in z)
        best, best_mask = None, None
        for mask in itertools.product((0, 1), repeat=d_ff):
            s = sum((z[k] - T) for k in range(d_ff) if mask[k])
            if best is None or s > best:
                best, best_mask = s, mask
        S = [k for k in range(d_ff) if best_mask[k]]
        assert list(res.sets[t]) == S
        u = [sum(X[t][j] * WU[j][k] for j in range(d)) for k in range(d_ff)]
        for j in range(d):
            terms = [(z[k] - T) * u[k] * WD[k][j] for k in S]
            exact = sum(terms, Fraction(0))
            scale = float(sum(abs(v) for v in terms)) + 1e-300
            assert abs(res.y[t, j] - float(exact)) <= 1e-13 * scale


@pytest.mark.parametrize("seed,d,d_ff,K", [(4, 4, 10, 3), (5, 6, 12, 5), (6, 3, 9, 8)])
def test_topk_set_by_brute_force(seed, d, d_ff, K):
    n = 2
    w, x = _tiny_weights(d, d_ff, n, seed)
    res = oracle.forward(x, w, "dense", "topk", k=K)
    X, WG = _exact(x), _exact(w["w_gate"])
    for t in range(n):
        z = [float(sum(X[t][j] * WG[j][k] for j in range(d))) for k in range(d_ff)]
        g = [zk / (1.0 + math.exp(-zk)) for zk in z]
        best, best_set = None, None
        for S in itertools.combinations(range(d_ff), K):   # lexicographic order
            s = math.fsum(g[k] for k in S)
            if best is None or s > best:
                best, best_set = s, S
        assert tuple(res.sets[t]) == best_set
        for k in range(d_ff):
            expect = g[k] if k in best_set else 0.0
            assert res.g[t, k] == pytest.approx(expect, rel=1e-13, abs=1e-300)


def test_topk_ties_go_to_lower_index():
    z = np.array([[0.5, 2.0, 1.0, 2.0, 1.0, 1.0, -3.0]])
    sets, g = oracle.select_topk(z, 4)
    assert list(sets[0]) == [1, 2, 3, 4]
    sets, _ = oracle.select_topk(z, 3)
    assert list(sets[0]) == [1, 2, 3]


def test_topk_ranks_by_silu_not_by_z():
    # SiLU is not monotone below its minimum near z = -1.278: -6 outranks -1.3.
    z = np.array([[-1.3, -6.0, 0.2]])
    sets, _ = oracle.select_topk(z, 2)
    assert list(sets[0]) == [1, 2]


# top-p ("PrunePath", abstract: a softmax-normalised routing distribution and a
# cumulative-mass threshold, i.e. a per-token probability budget)

def _softmax_exact(z):
    m = max(z)
    w = [math.exp(v - m) for v in z]
    tot = math.fsum(w)
    return [v / tot for v in w]


@pytest.mark.parametrize("seed,d,d_ff,p", [(7, 4, 9, 0.5), (8, 6, 11, 0.8), (9, 3, 12, 0.3), (10, 5, 10, 0.95)])
def test_topp_set_by_brute_force(seed, d, d_ff, p):
    """The kept set is the smallest set of channels whose softmax mass reaches
    p, and among sets of that size the one of largest mass (found over every
    subset)."""
    n = 2
    w, x = _tiny_weights(d, d_ff, n, seed)
    res = oracle.forward(x, w, "dense", "topp", p=p)
    X, WG = _exact(x), _exact(w["w_gate"])
    for t in range(n):
        z = [float(sum(X[t][j] * WG[j][k] for j in range(d))) for k in range(d_ff)]
        P = _softmax_exact(z)
        best_size, best, best_set = None, None, None
        for size in range(1, d_ff + 1):
            for S in itertools.combinations(range(d_ff), size):
                mass = math.fsum(P[k] for k in S)
                if mass >= p * (1 - 1e-12) and (best is None or mass > best):
                    best, best_set = mass, S
            if best_set is not None:
                best_size = size
                break
        assert tuple(res.sets[t]) == best_set and len(best_set) == best_size
        for k in range(d_ff):
            expect = z[k] / (1.0 + math.exp(-z[k])) if k in best_set else 0.0
            assert res.g[t, k] == pytest.approx(expect, rel=1e-12, abs=1e-300)


@pytest.mark.parametrize("d_ff,p", [(10, 0.35), (64, 0.5001), (1000, 0.9004), (37, 0.01)])
def test_topp_uniform_gate_keeps_ceil_p_dff_lowest(d_ff, p):
    """Equal gate values: every channel carries 1/d_ff, so exactly ceil(p d_ff)
    channels are kept, the lowest indices first (ties to the lower index)."""
    z = np.full((1, d_ff), 0.25)
    sets, _ = oracle.select_topp(z, p)
    m = math.ceil(p * d_ff)
    assert list(sets[0]) == list(range(m))


def test_topp_extremes_and_monotone():
    rng = np.random.default_rng(3)
    z = rng.standard_normal((3, 200))
    for t in range(3):
        top = int(np.argmax(z[t]))
        assert list(oracle.select_topp(z[t:t + 1], 1e-9)[0][0]) == [top]      # tiny budget: the arg max
    assert all(len(s) == 0 for s in oracle.select_topp(z, 0.0)[0])             # no budget: nothing
    assert all(len(s) == 200 for s in oracle.select_topp(z, 1.0)[0])           # the whole mass: all
    prev = [set() for _ in range(3)]
    for p in (0.1, 0.3, 0.5, 0.7, 0.9, 0.99):                                   # nested as p grows
        sets, _ = oracle.select_topp(z, p)
        for t in range(3):
            cur = set(sets[t].tolist())
            assert prev[t] <= cur
            prev[t] = cur


def test_topp_equals_topk_by_z_of_the_same_size():
    """For positive gate values SiLU orders like z, so the kept set is the
    top-K set of the same size."""
    rng = np.random.default_rng(4)
    z = np.abs(rng.standard_normal((2, 300))) + 0.1
    sets, _ = oracle.select_topp(z, 0.6)
    for t in range(2):
        ks, _ = oracle.select_topk(z[t:t + 1], len(sets[t]))
        assert list(ks[0]) == list(sets[t])


# --------------------------------------------------------------------------
# special cases against an independent numpy product chain

@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_topk_all_channels_is_dense_swiglu(dtype):
    d, d_ff, n = 48, 80, 3
    w, x = _tiny_weights(d, d_ff, n, 7, dtype)
    res = oracle.forward(x, w, "dense", "topk", k=d_ff)
    X, WG, WU, WD = (_np64(t) for t in (x, w["w_gate"], w["w_up"], w["w_down"]))
    y_ref = (_silu_np(X @ WG) * (X @ WU)) @ WD
    np.testing.assert_allclose(res.y, y_ref, rtol=1e-11, atol=1e-12 * np.abs(y_ref).max())
    assert all(len(s) == d_ff for s in res.sets)


def test_threshold_below_all_gates_is_affine_glu():
    d, d_ff, n = 40, 72, 2
    w, x = _tiny_weights(d, d_ff, n, 8)
    tau = -50.0
    res = oracle.forward(x, w, "dense", "threshold", tau=tau)
    X, WG, WU, WD = (_np64(t) for t in (x, w["w_gate"], w["w_up"], w["w_down"]))
    y_ref = ((X @ WG - tau) * (X @ WU)) @ WD
    np.testing.assert_allclose(res.y, y_ref, rtol=1e-11, atol=1e-12 * np.abs(y_ref).max())


def test_lopa_gate_equals_product_gate():
    d, d_ff, r, n = 64, 96, 16, 3
    w, x = _tiny_weights(d, d_ff, n, 9, r=r)
    u, z = oracle.gate_lopa(x, w["A"], w["B"])
    X, A, B = _np64(x), _np64(w["A"]), _np64(w["B"])
    np.testing.assert_allclose(u, X @ A, rtol=1e-12, atol=1e-13)
    zr = X @ (A @ B)
    assert np.abs(z - zr).max() <= 1e-12 * np.abs(zr).max()


def test_dense_gate_against_matmul():
    d, d_ff, n = 33, 70, 4
    w, x = _tiny_weights(d, d_ff, n, 10, "f32")
    z = oracle.gate_dense(x, w["w_gate"])
    np.testing.assert_allclose(z, _np64(x) @ _np64(w["w_gate"]), rtol=1e-12, atol=1e-13)


# --------------------------------------------------------------------------
# invariants

@pytest.mark.parametrize("select", ["threshold", "topk"])
def test_sparse_equals_dense_bitwise(select):
    wl = workloads.tiny()
    w, x = wl.weights(), wl.x()
    kw = dict(tau=wl.tau) if select == "threshold" else dict(k=wl.d_ff // 8)
    sp = oracle.forward(x, w, "dense", select, **kw)
    de = oracle.forward(x, w, "dense", select, dense=True, **kw)
    assert np.array_equal(sp.y, de.y)      # == treats -0.0 and +0.0 as equal


def test_empty_selection_gives_zero():
    d, d_ff, n = 16, 24, 3
    w, x = _tiny_weights(d, d_ff, n, 11)
    for kw in (dict(select="threshold", tau=float("inf")), dict(select="topk", k=0)):
        res = oracle.forward(x, w, "dense", **kw)
        assert all(len(s) == 0 for s in res.sets)
        assert not res.y.any()
        assert not res.g.any()


def test_gate_values_on_given_sets():
    z = np.array([[0.3, 2.0, -1.0], [1.5, 0.0, 4.0]])
    g = oracle.gate_values(z, [np.array([1]), np.array([0, 2])], "threshold", 1.0)
    np.testing.assert_array_equal(g, [[0.0, 1.0, 0.0], [0.5, 0.0, 3.0]])
    g = oracle.gate_values(z, [np.array([0]), np.array([])], "topk")
    assert g[0, 0] == pytest.approx(0.3 / (1 + math.exp(-0.3)), rel=1e-15) and g.sum() == g[0, 0]


# --------------------------------------------------------------------------
# closed forms

def _phi(v):
    return 0.5 * math.erfc(-v / math.sqrt(2.0))


@pytest.mark.parametrize("s", [0.5, 0.8, 0.9, 0.99])
def test_active_count_matches_gaussian_closed_form(s):
    d, d_ff, n = 256, 4096, 4
    w, x = _tiny_weights(d, d_ff, n, 12, "f32")
    tau = workloads.tau_for_sparsity(s)
    res = oracle.forward(x, w, "dense", "threshold", tau=tau)
    X = _np64(x)
    var_w = float(_np64(w["w_gate"]).var())
    for t in range(n):
        sigma = math.sqrt(float(X[t] @ X[t]) * var_w)
        p = 1.0 - _phi(tau / sigma)
        m = len(res.sets[t])
        assert abs(m - d_ff * p) <= 4.0 * math.sqrt(d_ff * p * (1 - p)) + 1, (t, m, d_ff * p)


def test_lopa_active_count_matches_gaussian_closed_form():
    d, d_ff, r, n = 512, 4096, 32, 3
    w, x = _tiny_weights(d, d_ff, n, 13, "f32", r=r)
    tau = workloads.tau_for_sparsity(0.9)
    res = oracle.forward(x, w, "lopa", "threshold", tau=tau)
    U = _np64(x) @ _np64(w["A"])
    var_b = float(_np64(w["B"]).var())
    for t in range(n):
        sigma = math.sqrt(float(U[t] @ U[t]) * var_b)
        p = 1.0 - _phi(tau / sigma)
        m = len(res.sets[t])
        assert abs(m - d_ff * p) <= 4.0 * math.sqrt(d_ff * p * (1 - p)) + 1


def test_topk_count_is_exactly_k():
    wl = workloads.moc_topk(n=3)
    w = workloads.ffn_weights(256, 704, "bf16", seed=3)
    x = workloads.tokens(3, 256, "bf16", seed=3)
    res = oracle.forward(x, w, "dense", "topk", k=88)
    for t in range(3):
        S = res.sets[t]
        assert len(S) == 88 and np.all(np.diff(S) > 0)
        sil = _silu_np(res.z[t])
        chosen = np.zeros(704, bool)
        chosen[S] = True
        assert sil[chosen].min() >= sil[~chosen].max()
    assert wl.k == wl.d_ff // 8


def _claims():
    out = {}
    with open(os.path.join(GOLDEN, "page_claims.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            name, value, pinned, _src = [p.strip() for p in line.split("|", 3)]
            out[name] = (float(value), pinned == "yes")
    return out


def test_flop_ratio_closed_form_and_page_cap():
    claims = _claims()
    cap, pinned = claims["dense_gate_flop_cap"]
    assert pinned
    d, d_ff, n = 4096, 11008, 1
    for m in (0, 1, 110, 1101, 5504, 11008):
        rho = Fraction(m, n * d_ff)
        ratio = Fraction(oracle.dense_flops(n, d, d_ff), oracle.flops(n, d, d_ff, m))
        assert ratio == 3 / (1 + 2 * rho)
        assert ratio <= cap
    assert Fraction(oracle.dense_flops(n, d, d_ff), oracle.flops(n, d, d_ff, 0)) == cap
    # LoPA r = 256 at 90 % sparsity: 3 d d_ff / (r (d + d_ff) + 2 rho d d_ff)
    lifts, pinned = claims["lopa_lifts_cap"]
    assert pinned and lifts == 1
    m, r = 1101, 256
    ratio = Fraction(oracle.dense_flops(n, d, d_ff), oracle.flops(n, d, d_ff, m, r=r))
    assert ratio == Fraction(3 * d * d_ff, r * (d + d_ff) + 2 * m * d)
    assert ratio > cap


def test_byte_counter_counts_an_enumerated_row_list():
    """The byte counters against the reads of one forward listed one by one on a
    tiny case: every gate column (LoPA: every column of A and of B), each union
    channel's W_up column and W_down row once for all tokens, each token's x
    row read and y row written (dense FFN: every W_up column and W_down row)."""
    d, d_ff, n, r = 16, 40, 3, 8
    for dtype, wb in (("bf16", 2), ("f32", 4)):
        w = workloads.ffn_weights(d, d_ff, dtype, seed=9, gate="both", r=r)
        x = workloads.tokens(n, d, dtype, seed=9)
        for gate in ("dense", "lopa"):
            ref = oracle.forward(x, w, gate, "threshold", tau=0.3)
            touched = sorted({int(k) for s in ref.sets for k in s})
            assert 0 < len(touched) < d_ff
            reads = []                                   # (what, index, elements)
            if gate == "dense":
                reads += [("W_gate column", k, d) for k in range(d_ff)]
            else:
                reads += [("A column", j, d) for j in range(r)] + [("B column", k, r) for k in range(d_ff)]
            for k in touched:
                reads += [("W_up column", k, d), ("W_down row", k, d)]
            reads += [("x row", t, d) for t in range(n)] + [("y row", t, d) for t in range(n)]
            assert len({(m, i) for m, i, _ in reads}) == len(reads)      # nothing listed twice
            total = sum(e for _, _, e in reads) * wb
            assert oracle.bytes_moved(n, d, d_ff, len(touched), wb, wb, r=r if gate == "lopa" else 0) == total
            assert oracle.union_size(ref.sets) == len(touched)
        dense = [("W_gate column", k, d) for k in range(d_ff)] + [("W_up column", k, d) for k in range(d_ff)]
        dense += [("W_down row", k, d) for k in range(d_ff)] + [("x row", t, d) for t in range(n)]
        dense += [("y row", t, d) for t in range(n)]
        assert oracle.dense_bytes(n, d, d_ff, wb, wb) == sum(e for _, _, e in dense) * wb


def test_thread_count_does_not_change_results():
    wl = workloads.tiny()
    w, x = wl.weights(), wl.x()
    n0 = oracle.num_threads()
    try:
        oracle.set_threads(1)
        a = oracle.forward(x, w, "dense", "threshold", tau=wl.tau)
        oracle.set_threads(max(2, n0))
        b = oracle.forward(x, w, "dense", "threshold", tau=wl.tau)
    finally:
        oracle.set_threads(n0)
    assert np.array_equal(a.y, b.y) and np.array_equal(a.z, b.z)


# --------------------------------------------------------------------------
# heavy-hitter split (the heavy-hitter abstract in the "FFN modules" paper
# listing: a dense part for the neurons that fire for every input, a sparse
# rest)

def test_hybrid_split_regroups_the_sparse_sum():
    wl = workloads.tiny()
    w, x = wl.weights(), wl.x()
    sp = oracle.forward(x, w, "dense", "threshold", tau=wl.tau)
    for frac, seed in ((0.05, 3), (0.5, 4)):
        hot = workloads.hot_channels(wl.d_ff, frac, seed=seed).numpy()
        hy = oracle.forward_hybrid(x, w, "dense", wl.tau, hot)
        assert all(np.array_equal(a, b) for a, b in zip(hy.sets, sp.sets))
        # the same terms, grouped as (hot channels, dense) + (the rest, sparse)
        np.testing.assert_allclose(hy.y, sp.y, rtol=0, atol=1e-12 * np.abs(sp.y).max())
        assert not np.array_equal(hy.y, oracle.forward_on_sets(
            x, w, "dense", "threshold", [s[~np.isin(s, hot)] for s in sp.sets], tau=wl.tau))


def test_hybrid_extremes_reduce_to_sparse_and_dense():
    wl = workloads.tiny()
    w, x = wl.weights(), wl.x()
    sp = oracle.forward(x, w, "dense", "threshold", tau=wl.tau)
    de = oracle.forward(x, w, "dense", "threshold", tau=wl.tau, dense=True)
    assert np.array_equal(oracle.forward_hybrid(x, w, "dense", wl.tau, []).y, sp.y)
    assert np.array_equal(oracle.forward_hybrid(x, w, "dense", wl.tau, np.arange(wl.d_ff)).y, de.y)


def test_hybrid_lopa_gate_matches_sparse():
    wl = workloads.lopa7b()
    d, d_ff, r = 64, 256, 16
    w = workloads.ffn_weights(d, d_ff, "f32", 5, "lopa", r)
    x = workloads.tokens(3, d, "f32", 5)
    tau = wl.tau
    sp = oracle.forward(x, w, "lopa", "threshold", tau=tau)
    hy = oracle.forward_hybrid(x, w, "lopa", tau, workloads.hot_channels(d_ff, 0.1, 6).numpy())
    np.testing.assert_allclose(hy.y, sp.y, rtol=0, atol=1e-12 * np.abs(sp.y).max())


def test_heavy_hitter_workload_structure():
    wl = workloads.heavy7b(n=4)
    w, x = wl.weights(), wl.x()
    z = oracle.gate_dense(x, w["w_gate"])
    hot = wl.hot().numpy()
    assert len(hot) == round(0.02 * wl.d_ff)
    # hot channels: mean tau + 3 from the outlier feature, so active almost surely
    assert (z[:, hot] > wl.tau).mean() >= 0.99
    # the rest: z ~ N(0, |x|^2 / d) given x, the Gaussian closed form of the active count
    rest = np.setdiff1d(np.arange(wl.d_ff), hot)
    xs = x.double().numpy()
    for t in range(wl.n):
        sig = math.sqrt(float((xs[t] ** 2).sum()) / wl.d)
        pr = 1.0 - _phi(wl.tau / sig)
        m = int((z[t, rest] > wl.tau).sum())
        assert abs(m - pr * len(rest)) <= 4.0 * math.sqrt(len(rest) * pr * (1 - pr))


def test_topp_exempt_band_is_narrow_on_the_moc_shape():
    """The top-p parity band (channels whose cumulative softmax mass lies within
    1e-3 of the budget) covers at most 2 % of each token's selection on the
    MoC top-K shape (d=2048, d_ff=5632, 16 tokens): 5-6 channels at p = 0.3,
    about 13 at p = 0.7, about 26 at p = 0.9."""
    import sys
    sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
    from parity import topp_exempt
    wl = workloads.moc_topk()
    w, x = wl.weights(), wl.x()
    for p, cap in ((0.3, 8), (0.7, 16), (0.9, 32)):
        r = oracle.forward(x, w, "dense", "topp", p=p)
        for t, s in enumerate(r.sets):
            ex = topp_exempt(r.z[t], p)
            assert len(ex) <= cap and len(ex) <= 0.02 * len(s), (p, t, len(ex), len(s))
