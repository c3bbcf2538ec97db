"""CUDA path vs the CPU oracle, through the C ABI, on the pages' workload
shapes (seeded synthetic stand-ins), small ragged shapes and edge cases."""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import EXEMPT, YTOL, assert_sets, assert_y, check_forward, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sffn(cuda_device):
    from activation_sparse_gated_gemv_b200 import build
    build.build()
    import activation_sparse_gated_gemv_b200 as m
    return m


def _ffn(sffn, wl, max_tokens=None, weights=None, device_src=False):
    w = weights if weights is not None else wl.weights()
    ffn = sffn.SparseFFN(wl.d, wl.d_ff, wl.r, max_tokens or wl.n, wl.dtype)
    if device_src:
        ffn.set_weights(**{k: v.cuda() for k, v in w.items()})
    else:
        ffn.set_weights(**w)
    return ffn, w


# --------------------------------------------------------------------------
# the pages' workload shapes

def test_tiny_relu_fp32(sffn):
    wl = workloads.tiny()
    ffn, w = _ffn(sffn, wl)
    x = wl.x()
    y, sets, union = check_forward(ffn, w, x, "dense", "threshold", tau=wl.tau)
    # fp32 weights and accumulation: far inside the bf16 bar
    ref = oracle.forward_on_sets(x, w, "dense", "threshold", sets, tau=wl.tau)
    assert_y(to_np(y), ref, 1e-4, "fp32")
    assert union == oracle.union_size(sets)
    ffn.close()


def test_llama7b_decode_dense_gate_90(sffn):
    wl = workloads.llama7b_decode(0.9)
    ffn, w = _ffn(sffn, wl)
    x = wl.x()
    _, sets, _ = check_forward(ffn, w, x, "dense", "threshold", tau=wl.tau)
    frac = len(sets[0]) / wl.d_ff
    assert 0.05 < frac < 0.15
    ffn.close()


@pytest.fixture(scope="module")
def lopa7b_model(sffn):
    wl = workloads.lopa7b(0.9)
    w = workloads.ffn_weights(wl.d, wl.d_ff, wl.dtype, seed=wl.seed, gate="both", r=wl.r)
    ffn = sffn.SparseFFN(wl.d, wl.d_ff, wl.r, 8, wl.dtype)
    ffn.set_weights(**w)
    yield wl, ffn, w
    ffn.close()


@pytest.mark.parametrize("sparsity", workloads.LOPA_SPARSITIES)
def test_lopa7b_sweep(lopa7b_model, sparsity):
    wl, ffn, w = lopa7b_model
    tau = workloads.tau_for_sparsity(sparsity)
    x = wl.x()
    _, sets, _ = check_forward(ffn, w, x, "lopa", "threshold", tau=tau)
    assert abs(len(sets[0]) / wl.d_ff - (1 - sparsity)) < 0.05


def test_lopa7b_dense_gate_on_same_handle(lopa7b_model):
    wl, ffn, w = lopa7b_model
    check_forward(ffn, w, wl.x(n=3, tag="b"), "dense", "threshold", tau=wl.tau)


def test_moc_topk_16_tokens(sffn):
    wl = workloads.moc_topk()
    ffn, w = _ffn(sffn, wl)
    x = wl.x()
    _, sets, union = check_forward(ffn, w, x, "dense", "topk", k=wl.k)
    assert all(len(s) == wl.k for s in sets)
    assert union == oracle.union_size(sets)
    ffn.close()


@pytest.fixture(scope="module")
def llama70b_model(sffn):
    wl = workloads.llama70b(64, "dense", 0.9)
    w = workloads.ffn_weights(wl.d, wl.d_ff, wl.dtype, seed=wl.seed, gate="both", r=512)
    ffn = sffn.SparseFFN(wl.d, wl.d_ff, 512, 64, wl.dtype)
    ffn.set_weights(**w)
    yield wl, ffn, w
    ffn.close()


@pytest.mark.parametrize("gate", ["dense", "lopa"])
@pytest.mark.parametrize("n", workloads.SWEEP_70B_BATCHES)
def test_llama70b_batches(llama70b_model, gate, n):
    wl, ffn, w = llama70b_model
    x = wl.x(n=n)
    tokens = range(n) if n <= 4 else [0, n // 2, n - 1]       # oracle on sampled tokens
    _, sets, union = check_forward(ffn, w, x, gate, "threshold", tau=wl.tau, tokens=tokens)
    assert union == len(set(np.concatenate(sets).tolist()))


@pytest.mark.parametrize("gate", ["dense", "lopa"])
@pytest.mark.parametrize("sparsity", workloads.SWEEP_70B_SPARSITIES)
def test_llama70b_sparsity_sweep_one_token(llama70b_model, gate, sparsity):
    wl, ffn, w = llama70b_model
    _, sets, _ = check_forward(ffn, w, wl.x(n=1, tag="s"), gate, "threshold",
                               tau=workloads.tau_for_sparsity(sparsity))
    assert ffn.last_kernel_names() == ["decode_fused"]
    assert abs(len(sets[0]) / wl.d_ff - (1 - sparsity)) < 0.05


# Every batch of the 70B-shaped sweep at sparsities other than 90 %, both
# gates, on the tensor-core path (oracle on sampled tokens; the union is
# checked against the oracle's at block granularity).
@pytest.mark.parametrize("gate", ["dense", "lopa"])
@pytest.mark.parametrize("n,sparsity", [(4, 0.7), (16, 0.5), (16, 0.99), (64, 0.8), (64, 0.95), (4, 0.99)])
def test_llama70b_batches_other_sparsities(llama70b_model, gate, n, sparsity):
    wl, ffn, w = llama70b_model
    tau = workloads.tau_for_sparsity(sparsity)
    x = wl.x(n=n, tag=f"b{sparsity}")
    tokens = range(n) if n <= 4 else [0, n // 3, n - 1]
    _, sets, union = check_forward(ffn, w, x, gate, "threshold", tau=tau, tokens=tokens)
    assert "tc_gate" in ffn.last_kernel_names()
    _check_union(ffn, sets, union)


def _check_union(ffn, sets, union):
    """The tensor-core kernels' union bitmap is exactly the OR of the per-token
    selections the kernels made (which the parity checks compared with the
    oracle up to the exempt band), and so are its active 128-channel blocks."""
    bits = ffn.union_bits()
    mask = np.zeros(ffn.d_ff, bool)
    for s in sets:
        mask[s] = True
    got = ((bits[np.arange(ffn.d_ff) >> 5] >> (np.arange(ffn.d_ff) & 31).astype(np.uint32)) & 1).astype(bool)
    assert np.array_equal(got, mask)
    assert union == int(mask.sum())
    nblk = (ffn.d_ff + 127) // 128
    blk_got = np.zeros(nblk, bool)
    blk_got[np.nonzero(got)[0] >> 7] = True
    blk_want = np.zeros(nblk, bool)
    blk_want[np.nonzero(mask)[0] >> 7] = True
    assert np.array_equal(blk_got, blk_want)


def _check_union_vs_oracle(ffn, w, x, gate, select, tau=0.0, k=0, p=0.0):
    """Union bitmap against the oracle's union over all tokens: equal except
    for channels inside the exempt band of the token that flips them; at block
    granularity, equal except blocks whose only differences are such channels."""
    from parity import silu, topp_exempt
    ref = oracle.forward(x, w, gate, select, tau=tau, k=k, p=p)
    bits = ffn.union_bits()
    ch = np.arange(ffn.d_ff)
    got = ((bits[ch >> 5] >> (ch & 31).astype(np.uint32)) & 1).astype(bool)
    want = np.zeros(ffn.d_ff, bool)
    exempt = np.zeros(ffn.d_ff, bool)
    for t, s in enumerate(ref.sets):
        want[s] = True
        z = ref.z[t]
        if select == "threshold":
            exempt |= np.abs(z - tau) <= EXEMPT
        elif select == "topk":
            sv = silu(z)
            gk = np.sort(sv)[::-1][k - 1] if k > 0 else np.inf
            exempt |= np.abs(sv - gk) <= EXEMPT
        else:
            exempt[list(topp_exempt(z, p))] = True
    diff = got ^ want
    assert not np.any(diff & ~exempt), np.nonzero(diff & ~exempt)[0][:8]
    nblk = (ffn.d_ff + 127) // 128
    bg, bw = np.zeros(nblk, bool), np.zeros(nblk, bool)
    bg[np.nonzero(got)[0] >> 7] = True
    bw[np.nonzero(want)[0] >> 7] = True
    for b in np.nonzero(bg ^ bw)[0]:
        assert np.all(exempt[b * 128:(b + 1) * 128][diff[b * 128:(b + 1) * 128]]), f"block {b}"


@pytest.mark.parametrize("select", ["threshold", "topk", "topp"])
@pytest.mark.parametrize("n,sparsity", [(5, 0.999), (16, 0.995), (64, 0.9)])
def test_union_bitmap_matches_oracle(sffn, select, n, sparsity):
    # sparse enough that some 128-channel blocks stay inactive at small n
    d, d_ff = 256, 4000
    w = workloads.ffn_weights(d, d_ff, "bf16", seed=61, gate="dense")
    x = workloads.tokens(n, d, "bf16", seed=62)
    ffn = sffn.SparseFFN(d, d_ff, 0, n, "bf16")
    ffn.set_weights(**w)
    tau = workloads.tau_for_sparsity(sparsity)
    k = max(1, int(round(d_ff * (1 - sparsity))))
    _, sets, union = check_forward(ffn, w, x, "dense", select, tau=tau, k=k, p=0.3)
    assert "tc_gate" in ffn.last_kernel_names()
    _check_union(ffn, sets, union)
    _check_union_vs_oracle(ffn, w, x, "dense", select, tau=tau, k=k, p=0.3)
    if select == "threshold" and n == 5:
        nact = len({c >> 7 for s in sets for c in s})
        assert nact < (d_ff + 127) // 128              # the case does skip blocks
    ffn.close()


# --------------------------------------------------------------------------
# small ragged shapes: several gate CTAs, ragged tails, token tiles

SMALL = [
    # d, d_ff, r, n, dtype, gate, select
    (64, 1000, 0, 1, "bf16", "dense", "threshold"),
    (64, 777, 0, 3, "f32", "dense", "threshold"),
    (136, 4100, 0, 5, "bf16", "dense", "threshold"),
    (136, 4100, 16, 5, "bf16", "lopa", "threshold"),
    (256, 2048, 24, 17, "bf16", "lopa", "threshold"),
    (512, 3000, 0, 9, "f32", "dense", "topk"),
    (64, 1000, 8, 2, "bf16", "lopa", "topk"),
    (1032, 1536, 0, 4, "bf16", "dense", "topk"),
    (8, 300, 8, 1, "f32", "lopa", "threshold"),
    (64, 256, 0, 1024, "bf16", "dense", "threshold"),    # the largest token count
    # batched tensor-core path (bf16, 5 <= n <= 128): ragged row tiles and k-blocks
    (136, 4100, 0, 64, "bf16", "dense", "threshold"),
    (520, 3000, 64, 33, "bf16", "lopa", "threshold"),
    (264, 1000, 0, 16, "bf16", "dense", "topk"),
    (264, 1000, 32, 128, "bf16", "lopa", "topk"),
    (64, 300, 8, 6, "bf16", "lopa", "topk"),
    (1024, 640, 0, 100, "bf16", "dense", "threshold"),
    # top-p: the batched path and the one-token path, dense and LoPA gates
    (264, 1000, 0, 16, "bf16", "dense", "topp"),
    (136, 4100, 0, 1, "bf16", "dense", "topp"),
    (520, 3000, 64, 33, "bf16", "lopa", "topp"),
    (512, 3000, 0, 9, "f32", "dense", "topp"),
    (64, 1000, 8, 2, "bf16", "lopa", "topp"),
]


@pytest.mark.parametrize("d,d_ff,r,n,dtype,gate,select", SMALL)
def test_small_ragged(sffn, d, d_ff, r, n, dtype, gate, select):
    w = workloads.ffn_weights(d, d_ff, dtype, seed=d + d_ff + n, gate="both" if r else "dense", r=r)
    x = workloads.tokens(n, d, dtype, seed=d_ff)
    ffn = sffn.SparseFFN(d, d_ff, r, n, dtype)
    ffn.set_weights(**w)
    tau = workloads.tau_for_sparsity(0.85)
    k = max(1, d_ff // 8)
    tokens = None if n <= 32 else [0, 1, n // 2, n - 1]
    check_forward(ffn, w, x, gate, select, tau=tau, k=k, tokens=tokens, p=0.7)
    ffn.close()


@pytest.mark.parametrize("n", [3, 20])
@pytest.mark.parametrize("select", ["threshold", "topk"])
@pytest.mark.parametrize("gate", ["dense", "lopa"])
def test_dense_path_matches_oracle_and_sparse(sffn, gate, select, n):
    d, d_ff, r = 128, 1500, 16
    w = workloads.ffn_weights(d, d_ff, "bf16", seed=5, gate="both", r=r)
    x = workloads.tokens(n, d, "bf16", seed=5)
    ffn = sffn.SparseFFN(d, d_ff, r, n, "bf16")
    ffn.set_weights(**w)
    tau, k = workloads.tau_for_sparsity(0.9), d_ff // 8
    yd, _, union = check_forward(ffn, w, x, gate, select, tau=tau, k=k, dense=True)
    ys, _, _ = check_forward(ffn, w, x, gate, select, tau=tau, k=k)
    assert_y(to_np(yd), to_np(ys), 1e-2, "dense vs sparse")
    ffn.close()


# --------------------------------------------------------------------------
# edge cases

def _small(sffn, n=4, r=8, dtype="bf16", d=64, d_ff=500):
    w = workloads.ffn_weights(d, d_ff, dtype, seed=77, gate="both", r=r)
    ffn = sffn.SparseFFN(d, d_ff, r, max(n, 1), dtype)
    ffn.set_weights(**w)
    return ffn, w, workloads.tokens(n, d, dtype, seed=78)


def test_tau_inf_and_k_zero_give_zero(sffn):
    ffn, w, x = _small(sffn)
    for gate in ("dense", "lopa"):
        y = ffn.forward(x.cuda(), gate=gate, select="threshold", tau=math.inf)
        assert not to_np(y).any()
        sets, union = ffn.active(4)
        assert union == 0 and all(len(s) == 0 for s in sets)
        y = ffn.forward(x.cuda(), gate=gate, select="topk", k=0)
        assert not to_np(y).any()
    ffn.close()


@pytest.mark.parametrize("n", [1, 6])
def test_topp_extremes(sffn, n):
    """p = 0 keeps nothing (y = 0); p = 1 keeps every channel with mass (the
    dense SwiGLU FFN); a tiny p keeps each token's largest gate value."""
    ffn, w, x = _small(sffn, n=n, d_ff=300)
    y = ffn.forward(x.cuda(), gate="dense", select="topp", p=0.0)
    assert not to_np(y).any()
    sets, union = ffn.active(n)
    assert union == 0
    check_forward(ffn, w, x, "dense", "topp", p=1.0)
    _, sets, _ = check_forward(ffn, w, x, "dense", "topp", p=1e-6)
    z = oracle.forward(x, w, "dense", "topp", p=1e-6).z
    assert [list(s) for s in sets] == [[int(np.argmax(z[t]))] for t in range(n)]
    ffn.close()


@pytest.mark.parametrize("p", [0.3, 0.9])
def test_moc_shape_topp(sffn, p):
    wl = workloads.moc_topk()
    ffn, w = _ffn(sffn, wl)
    check_forward(ffn, w, wl.x(), "dense", "topp", p=p)
    ffn.close()


@pytest.mark.parametrize("n,d_ff", [(1, 1000), (6, 1000), (6, 5632)])
def test_topk_and_topp_ties_go_to_the_lower_channel(sffn, n, d_ff):
    """W_gate with every column equal gives every channel the same z (each dot
    product is summed in the same order), so the whole row ties: top-K must
    keep channels 0..K-1 and top-p the first ceil(p d_ff) channels (equal
    masses).  Then half the columns equal: the ties at the boundary are ranked
    by channel index."""
    d = 64
    w = workloads.ffn_weights(d, d_ff, "bf16", seed=71)
    col = w["w_gate"][:, :1].clone()
    w["w_gate"] = col.expand(d, d_ff).contiguous()
    ffn = sffn.SparseFFN(d, d_ff, 0, n, "bf16")
    ffn.set_weights(**w)
    x = workloads.tokens(n, d, "bf16", seed=72)
    k = d_ff * 3 // 10 + 1
    ffn.forward(x.cuda(), select="topk", k=k)
    sets, _ = ffn.active(n)
    assert all(np.array_equal(s, np.arange(k)) for s in sets)
    ffn.forward(x.cuda(), select="topp", p=0.25)
    sets, _ = ffn.active(n)
    m = math.ceil(0.25 * d_ff)
    assert all(abs(len(s) - m) <= 1 and np.array_equal(s, np.arange(len(s))) for s in sets)
    # half the channels tie (equal columns at the odd channels), the rest are distinct
    wg = workloads.ffn_weights(d, d_ff, "bf16", seed=73)["w_gate"].clone()
    wg[:, 1::2] = wg[:, 1:2]
    w["w_gate"] = wg.contiguous()
    ffn.set_weights(**w)
    check_forward(ffn, w, x, "dense", "topk", k=k)
    sets, _ = ffn.active(n)
    tied = np.arange(1, d_ff, 2)
    for t in range(n):
        got = np.intersect1d(sets[t], tied)
        # which tied channels are kept is fixed: the lowest ones
        assert np.array_equal(got, tied[:len(got)])
    ffn.close()


def test_k_equals_d_ff_is_dense_swiglu(sffn):
    ffn, w, x = _small(sffn, d_ff=300)
    y = ffn.forward(x.cuda(), gate="dense", select="topk", k=300)
    X, WG, WU, WD = (t.to(torch.float64).numpy() for t in (x, w["w_gate"], w["w_up"], w["w_down"]))
    z = X @ WG
    ref = (z / (1 + np.exp(-z)) * (X @ WU)) @ WD
    assert_y(to_np(y), ref, YTOL, "K = d_ff")
    ffn.close()


def test_all_channels_active(sffn):
    ffn, w, x = _small(sffn)
    check_forward(ffn, w, x, "dense", "threshold", tau=-40.0)
    sets, union = ffn.active(4)
    assert union == 500
    ffn.close()


def test_zero_tokens_is_a_noop(sffn):
    ffn, w, _ = _small(sffn)
    x = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    y = ffn.forward(x)
    assert y.shape == (0, 64)
    ffn.close()


def test_deterministic_bitwise(sffn):
    wl = workloads.moc_topk(n=5)
    ffn, w = _ffn(sffn, wl)
    x = wl.x().cuda()
    a = ffn.forward(x, select="topk", k=wl.k).clone()
    b = ffn.forward(x, select="topk", k=wl.k).clone()
    assert torch.equal(a, b)
    tau = workloads.tau_for_sparsity(0.9)
    a = ffn.forward(x, select="threshold", tau=tau).clone()
    b = ffn.forward(x, select="threshold", tau=tau).clone()
    assert torch.equal(a, b)
    ffn.close()


def test_paths_alternate_on_one_handle(sffn):
    """One handle takes the fused decode kernel (grid-barrier counters), the
    unfused top-K path (per-forward tickets), the tensor-core path and the
    fused LoPA kernel in turn; every forward still matches the oracle."""
    d, d_ff, r = 256, 2048, 64
    w = workloads.ffn_weights(d, d_ff, "bf16", seed=31, gate="both", r=r)
    ffn = sffn.SparseFFN(d, d_ff, r, 8, "bf16")
    ffn.set_weights(**w)
    tau, k = workloads.tau_for_sparsity(0.9), d_ff // 8
    plan = [(1, "dense", "threshold"), (1, "dense", "topk"), (8, "dense", "threshold"), (1, "lopa", "threshold"),
            (2, "dense", "topp"), (1, "dense", "threshold"), (8, "lopa", "topk"), (2, "lopa", "threshold")]
    for i, (n, gate, select) in enumerate(plan * 2):
        x = workloads.tokens(n, d, "bf16", seed=100 + i)
        check_forward(ffn, w, x, gate, select, tau=tau, k=k, p=0.6)
    ffn.close()


def test_forward_host_matches_device_forward(sffn):
    ffn, w, x = _small(sffn)
    tau = workloads.tau_for_sparsity(0.8)
    yd = ffn.forward(x.cuda(), gate="lopa", tau=tau).cpu()
    yh = ffn.forward_host(x.pin_memory(), gate="lopa", tau=tau)
    assert torch.equal(yd, yh)
    ffn.close()


@pytest.mark.parametrize("n,pinned_x,pinned_out", [(1, True, True), (1, False, True), (1, True, False),
                                                   (2, True, True), (2, False, False), (5, True, True)])
def test_forward_host_buffer_kinds(sffn, n, pinned_x, pinned_out):
    """One or two tokens with page-locked buffers: the decode kernel pulls x in
    from host memory and stores y there itself; pageable buffers, or a batch,
    go through copies.  Either way y is bitwise the device forward's, call
    after call (the kernel's x arrival counter never resets)."""
    d, d_ff = 512, 3000
    w = workloads.ffn_weights(d, d_ff, "bf16", seed=91)
    ffn = sffn.SparseFFN(d, d_ff, 0, 8, "bf16")
    ffn.set_weights(**w)
    tau = workloads.tau_for_sparsity(0.9)
    out = torch.full((n, d), float("nan"), dtype=torch.bfloat16)
    if pinned_out:
        out = out.pin_memory()
    for i in range(3):
        x = workloads.tokens(n, d, "bf16", seed=92 + i)
        yd = ffn.forward(x.cuda(), tau=tau).cpu()
        xh = x.pin_memory() if pinned_x else x.clone()
        yh = ffn.forward_host(xh, tau=tau, out=out)
        assert torch.equal(yd, yh), i
        out.fill_(float("nan"))
    ffn.check_status()
    ffn.close()


def test_forward_host_mixed_calls(sffn):
    """Host forwards of every kind in one handle, interleaved with device
    forwards and LoPA: each matches the device forward bitwise, and the status
    stays clean (a miscounted x arrival would time out)."""
    d, d_ff, r = 512, 3000, 64
    w = workloads.ffn_weights(d, d_ff, "bf16", seed=93, gate="both", r=r)
    ffn = sffn.SparseFFN(d, d_ff, r, 8, "bf16")
    ffn.set_weights(**w)
    tau = workloads.tau_for_sparsity(0.9)
    for i, (n, gate, pinned) in enumerate([(1, "dense", True), (2, "lopa", True), (1, "dense", False), (4, "dense", True),
                                           (1, "lopa", True), (2, "dense", True), (1, "dense", True)]):
        x = workloads.tokens(n, d, "bf16", seed=94 + i)
        yd = ffn.forward(x.cuda(), gate=gate, tau=tau).cpu()
        yh = ffn.forward_host(x.pin_memory() if pinned else x.clone(), gate=gate, tau=tau)
        assert torch.equal(yd, yh), (i, n, gate, pinned)
    ffn.check_status()
    ffn.close()


def test_device_source_weights(sffn):
    wl = workloads.tiny()
    ffn, w = _ffn(sffn, wl, device_src=True)
    check_forward(ffn, w, wl.x(), "dense", "threshold", tau=wl.tau)
    ffn.close()


def test_errors(sffn):
    import ctypes
    ffn = sffn.SparseFFN(64, 128, 0, 2, "bf16")
    x = torch.zeros((2, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(sffn.SFFNError) as e:
        ffn.forward(x)
    assert e.value.code == sffn.SFFN_ERR_NOT_READY
    w = workloads.ffn_weights(64, 128, "bf16", seed=1)
    ffn.set_weights(**w)
    with pytest.raises(sffn.SFFNError) as e:
        ffn.forward(x, gate="lopa")
    assert e.value.code == sffn.SFFN_ERR_UNSUPPORTED
    for kw in (dict(select="threshold", tau=float("nan")), dict(select="threshold", tau=-math.inf),
               dict(select="topk", k=-1), dict(select="topk", k=129)):
        with pytest.raises(sffn.SFFNError) as e:
            ffn.forward(x, **kw)
        assert e.value.code == sffn.SFFN_ERR_INVALID_ARG
    with pytest.raises(sffn.SFFNError) as e:
        ffn.forward(torch.zeros((3, 64), dtype=torch.bfloat16, device="cuda"))
    assert e.value.code == sffn.SFFN_ERR_INVALID_ARG
    # misaligned device pointer
    buf = torch.zeros(2 * 64 + 1, dtype=torch.bfloat16, device="cuda")
    sel = sffn.make_select("threshold", 1.0)
    out = torch.zeros((2, 64), dtype=torch.bfloat16, device="cuda")
    rc = sffn.sffn_forward(ffn.handle, buf.data_ptr() + 2, 2, 0, ctypes.byref(sel), out.data_ptr(), None)
    assert rc == sffn.SFFN_ERR_INVALID_ARG
    ffn.close()


# --------------------------------------------------------------------------
# heavy-hitter channels (sffn_set_hot)

@pytest.mark.parametrize("n", [1, 2])
def test_heavy_hitter_workload_matches_hybrid_oracle(sffn, n):
    wl = workloads.heavy7b(n=n)
    ffn, w = _ffn(sffn, wl)
    x = wl.x()
    hot = wl.hot().numpy()
    y0 = ffn.forward(x.cuda(), tau=wl.tau).clone()
    ffn.set_hot(hot)
    y, sets, _ = check_forward(ffn, w, x, "dense", "threshold", tau=wl.tau)
    assert ffn.last_kernel_names() == ["decode_fused"]
    assert torch.equal(y, y0)                  # the set moves reads, not results
    assert_y(to_np(y), oracle.forward_hybrid(x, w, "dense", wl.tau, hot).y, YTOL, "vs the hybrid oracle")
    assert all(np.isin(hot, s).mean() >= 0.99 for s in sets)
    ffn.set_hot([])
    assert torch.equal(ffn.forward(x.cuda(), tau=wl.tau), y0)
    ffn.close()


@pytest.mark.parametrize("gate,dtype", [("dense", "bf16"), ("lopa", "bf16"), ("dense", "f32")])
def test_hot_set_leaves_results_bitwise_unchanged(sffn, gate, dtype):
    d, d_ff, r = 256, 2000, 64                 # d_ff not a multiple of 32: a ragged last bit word
    w = workloads.ffn_weights(d, d_ff, dtype, seed=41, gate="both", r=r)
    ffn = sffn.SparseFFN(d, d_ff, r, 8, dtype)
    ffn.set_weights(**w)
    hot = np.union1d(workloads.hot_channels(d_ff, 0.1, seed=7).numpy(), [0, 1, d_ff - 1])
    tau = workloads.tau_for_sparsity(0.9)
    plan = [(1, "threshold"), (2, "threshold"), (1, "topk")] + ([(8, "threshold")] if dtype == "bf16" else [])
    for i, (n, select) in enumerate(plan):
        x = workloads.tokens(n, d, dtype, seed=200 + i)
        kw = dict(gate=gate, select=select, tau=tau, k=d_ff // 8)
        ffn.set_hot([])
        a = ffn.forward(x.cuda(), **kw).clone()
        ffn.set_hot(hot)
        b, _, _ = check_forward(ffn, w, x, gate, select, tau=tau, k=d_ff // 8)
        assert torch.equal(a, b)
        if select == "threshold":
            assert_y(to_np(b), oracle.forward_hybrid(x, w, gate, tau, hot).y, YTOL, "vs the hybrid oracle")
    ffn.close()


def test_hot_set_errors(sffn):
    ffn = sffn.SparseFFN(64, 100, 0, 1, "bf16")
    for bad in ([100], [-1], [5, 3, 1000]):
        with pytest.raises(sffn.SFFNError) as e:
            ffn.set_hot(bad)
        assert e.value.code == sffn.SFFN_ERR_INVALID_ARG
    ffn.set_hot([0, 99, 99])                   # duplicates are fine
    ffn.set_hot([])
    ffn.close()


# --------------------------------------------------------------------------
# batches above one pass: one tensor-core pass per 256 tokens (128 with LoPA)

@pytest.mark.parametrize("gate,select", [("dense", "threshold"), ("lopa", "threshold"), ("dense", "topk"),
                                         ("lopa", "topp")])
def test_batch_above_128_tokens_in_passes(sffn, gate, select):
    d, d_ff, r, n = 256, 2000, 64, 300         # passes of 128, 128 and 44 tokens
    w = workloads.ffn_weights(d, d_ff, "bf16", seed=51, gate="both", r=r)
    ffn = sffn.SparseFFN(d, d_ff, r, n, "bf16")
    ffn.set_weights(**w)
    x = workloads.tokens(n, d, "bf16", seed=52)
    tau, k = workloads.tau_for_sparsity(0.9), d_ff // 8
    edges = [0, 1, 127, 128, 129, 255, 256, 257, 299]
    check_forward(ffn, w, x, gate, select, tau=tau, k=k, p=0.7, tokens=edges)
    # passes of 256 tokens (128 with LoPA, whose u enters the gate as hi/lo pairs)
    assert ffn.last_kernel_names().count("tc_gate") == (3 if gate == "lopa" else 2)
    ffn.close()


def test_dense_ffn_above_128_tokens(sffn):
    d, d_ff, n = 256, 1024, 200
    w = workloads.ffn_weights(d, d_ff, "bf16", seed=53)
    ffn = sffn.SparseFFN(d, d_ff, 0, n, "bf16")
    ffn.set_weights(**w)
    x = workloads.tokens(n, d, "bf16", seed=54)
    tau = workloads.tau_for_sparsity(0.9)
    yd, _, _ = check_forward(ffn, w, x, "dense", "threshold", tau=tau, dense=True, tokens=[0, 127, 128, 199])
    ys = ffn.forward(x.cuda(), tau=tau)
    assert_y(to_np(ys), to_np(yd), YTOL, "sparse vs dense")
    ffn.close()
