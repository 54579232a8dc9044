"""Pins of the RoLA gradient oracle against things other than itself: central
finite differences of the forward oracle (the derivative's definition), and
library autograd of scaled dot-product attention where RoLA reduces to it."""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import rola_backward_oracle as rbo
from oracle import rola_oracle as ro

GRID = (2, 3, 5)   # N = 30 tokens: blocks of 8 -> 4 blocks, the last one ragged (6 valid)
BS, D, R = 8, 8, 6  # r = 6 splits 2 / 2 / 2 over (t, y, x)


def _case(seed, k_b, g=0.7, nb=4):
    rng = np.random.default_rng(seed)
    N = int(np.prod(GRID))
    q, k, v, dO = (rng.standard_normal((N, D)) for _ in range(4))
    P = rng.standard_normal((D, R)) / np.sqrt(D)
    idx = np.stack([np.sort(rng.choice(nb, size=k_b, replace=False)) for _ in range(nb)])
    return dict(q=q, k=k, v=v, P=P, g=g, dO=dO, idx=idx)


def _loss(c, **over):
    x = {**c, **over}
    res = ro.rola_head(x["q"], x["k"], x["v"], x["P"], x["g"], bs=BS, k_b=x["idx"].shape[1],
                       grid=GRID, rope_base=10000.0, idx=x["idx"])
    N = x["q"].shape[0]
    return sum(float((x["dO"][slice(*ro.block_range(a, BS, N))] * o).sum()) for a, o in res.o.items())


def _grads(c):
    return rbo.rola_head_backward(c["q"], c["k"], c["v"], c["P"], c["g"], c["dO"], bs=BS,
                                  idx=c["idx"], grid=GRID)


def _directional_fd(c, name, direction, eps=1e-5):
    plus = _loss(c, **{name: c[name] + eps * direction})
    minus = _loss(c, **{name: c[name] - eps * direction})
    return (plus - minus) / (2 * eps)


@pytest.mark.parametrize("seed,k_b", [(0, 1), (1, 2), (2, 3)])
def test_gradients_match_central_differences(seed, k_b):
    c = _case(seed, k_b)
    G = _grads(c)
    rng = np.random.default_rng(100 + seed)
    for name, grad in (("q", G.dq), ("k", G.dk), ("v", G.dv), ("P", G.dP)):
        for _ in range(3):
            direction = rng.standard_normal(c[name].shape)
            fd = _directional_fd(c, name, direction)
            an = float((grad * direction).sum())
            assert abs(fd - an) <= 1e-7 * max(1.0, abs(fd)), (name, fd, an)
    fd_g = (_loss(c, g=c["g"] + 1e-5) - _loss(c, g=c["g"] - 1e-5)) / 2e-5
    assert abs(fd_g - G.dg) <= 1e-7 * max(1.0, abs(fd_g))


def test_single_entries_of_the_projection():
    """P_h reaches the output through both the query and the key features."""
    c = _case(3, 2)
    G = _grads(c)
    for (i, j) in [(0, 0), (3, 5), (7, 2)]:
        e = np.zeros_like(c["P"])
        e[i, j] = 1.0
        fd = _directional_fd(c, "P", e)
        assert abs(fd - G.dP[i, j]) <= 1e-7 * max(1.0, abs(fd))


def _torch_sdpa_grads(c, mask=None):
    q, k, v = (torch.tensor(c[n], dtype=torch.float64, requires_grad=True) for n in ("q", "k", "v"))
    o = F.scaled_dot_product_attention(q[None, None], k[None, None], v[None, None],
                                       attn_mask=None if mask is None else torch.tensor(mask))
    (o[0, 0] * torch.tensor(c["dO"])).sum().backward()
    return q.grad.numpy(), k.grad.numpy(), v.grad.numpy()


def test_dense_limit_matches_library_autograd():
    """Every block kept: no linear branch, RoLA is exact attention."""
    c = _case(4, 4)
    G = _grads(c)
    dq, dk, dv = _torch_sdpa_grads(c)
    for ours, ref in ((G.dq, dq), (G.dk, dk), (G.dv, dv)):
        assert np.allclose(ours, ref, rtol=1e-10, atol=1e-12)
    assert np.all(G.dP == 0) and G.dg == 0.0


def test_gate_zero_matches_masked_library_autograd():
    """g = 0: only the block-sparse softmax reaches the output; the gate's own
    gradient is the linear branch's output against dO."""
    c = _case(5, 2, g=0.0)
    G = _grads(c)
    N = c["q"].shape[0]
    mask = np.zeros((N, N), dtype=bool)
    for a in range(c["idx"].shape[0]):
        lo, hi = ro.block_range(a, BS, N)
        mask[lo:hi, ro.kept_tokens(c["idx"][a], BS, N)] = True
    dq, dk, dv = _torch_sdpa_grads(c, mask)
    for ours, ref in ((G.dq, dq), (G.dk, dk), (G.dv, dv)):
        assert np.allclose(ours, ref, rtol=1e-10, atol=1e-12)
    assert np.all(G.dP == 0)
    res = ro.rola_head(c["q"], c["k"], c["v"], c["P"], 0.0, bs=BS, k_b=2, grid=GRID,
                       rope_base=10000.0, idx=c["idx"])
    want = sum(float((c["dO"][slice(*ro.block_range(a, BS, N))] * o).sum()) for a, o in res.o_lin.items())
    assert abs(G.dg - want) <= 1e-12 * max(1.0, abs(want))


def test_a_planted_mistake_is_caught(monkeypatch):
    """Dropping the feature map's derivative (a plausible slip) breaks the
    finite-difference pin: the pin is sensitive to the linear branch."""
    c = _case(6, 2)
    monkeypatch.setattr(rbo, "phi_grad", lambda u: np.ones_like(u))
    G = _grads(c)
    rng = np.random.default_rng(7)
    direction = rng.standard_normal(c["q"].shape)
    fd = _directional_fd(c, "q", direction)
    assert abs(fd - float((G.dq * direction).sum())) > 1e-4 * max(1.0, abs(fd))


def test_transposed_mask_lists_every_keeping_query_block():
    idx = np.array([[0, 2], [1, 2], [0, 3], [2, 3]])
    offsets, rows = rbo.transposed_mask(idx, 4)
    got = [rows[offsets[j]:offsets[j + 1]].tolist() for j in range(4)]
    assert got == [[0, 2], [1], [0, 1, 3], [2, 3]]
    # on a random mask: membership both ways, ascending, total = nb * k_b
    rng = np.random.default_rng(9)
    nb, kb = 37, 5
    idx = np.stack([np.sort(rng.choice(nb, size=kb, replace=False)) for _ in range(nb)])
    offsets, rows = rbo.transposed_mask(idx, nb)
    assert offsets[-1] == nb * kb
    for j in range(nb):
        lst = rows[offsets[j]:offsets[j + 1]]
        assert np.all(np.diff(lst) > 0)
        assert set(lst.tolist()) == {a for a in range(nb) if j in idx[a]}


def test_forward_stats_against_library_logsumexp():
    from scipy.special import logsumexp
    c = _case(8, 2)
    lse, den = rbo.forward_stats(c["q"], c["k"], c["v"], c["P"], bs=BS, idx=c["idx"], grid=GRID)
    N = c["q"].shape[0]
    for a in range(c["idx"].shape[0]):
        lo, hi = ro.block_range(a, BS, N)
        J = ro.kept_tokens(c["idx"][a], BS, N)
        s = c["q"][lo:hi] @ c["k"][J].T / np.sqrt(D)
        assert np.allclose(lse[lo:hi], logsumexp(s, axis=1), rtol=0, atol=1e-12)
    assert np.all(den > 0)
    # the saved statistics reproduce the forward: o_sp = exp(s - lse) v, o_lin = num / den
    res = ro.rola_head(c["q"], c["k"], c["v"], c["P"], c["g"], bs=BS, k_b=2, grid=GRID,
                       rope_base=10000.0, idx=c["idx"])
    for a, o_sp in res.o_sp.items():
        lo, hi = ro.block_range(a, BS, N)
        J = ro.kept_tokens(c["idx"][a], BS, N)
        p = np.exp(c["q"][lo:hi] @ c["k"][J].T / np.sqrt(D) - lse[lo:hi, None])
        assert np.allclose(p @ c["v"][J], o_sp, rtol=1e-12, atol=1e-12)
    _, dense = rbo.forward_stats(c["q"], c["k"], c["v"], c["P"], bs=BS,
                                 idx=np.tile(np.arange(4), (4, 1)), grid=GRID)
    assert np.all(np.isnan(dense))
