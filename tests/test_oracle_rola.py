"""Pins for the fp64 RoLA oracle, checked against things other than itself:
hand-built cases with known answers, brute force on tiny inputs, library
routines (torch SDPA and elu in float64), closed-form special cases and
invariants of the rotary embedding."""
import math
import os

import numpy as np
import pytest
import torch

from oracle import rola_oracle as ro
from sparse_linear_attention_mean_b200 import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


# ---------------------------------------------------------------- kept blocks

def test_kept_blocks_integer_rule_matches_golden():
    rows = [l.split() for l in open(os.path.join(GOLD, "kept_blocks.txt")) if l.strip() and not l.startswith("#")]
    assert rows
    for nb, s, kb in rows:
        assert ro.kb_from_sparsity(int(nb), int(s)) == int(kb), (nb, s, kb)
    # the floating-point ceiling would keep 4 of 100 blocks at 97 %
    assert math.ceil((1 - 0.97) * 100) == 4


def test_workload_table_kb_consistent():
    for w in synth.WORKLOADS.values():
        assert ro.kb_from_sparsity(w.n_blocks, w.sparsity_permille) == w.k_b


# ---------------------------------------------------------------- selector

def test_pool_uses_valid_tokens_only():
    x = _rand((21, 3), 1)          # 21 tokens, blocks of 8 -> last block has 5
    got = ro.pool_blocks(x, 8)
    for b in range(3):
        toks = range(b * 8, min(21, b * 8 + 8))
        for c in range(3):
            want = sum(x[t, c] for t in toks) / len(toks)
            assert abs(got[b, c] - want) < 1e-14


def test_selector_hand_built_known_topk():
    # 6 key blocks of 4 tokens whose pooled vectors are (b+1) e_b, and query
    # blocks whose pooled vectors weight those axes -> scores known by hand.
    d, bs, nb = 8, 4, 6
    k = np.zeros((nb * bs, d))
    for b in range(nb):
        k[b * bs:(b + 1) * bs, b] = b + 1
    w = np.array([[6, 5, 4, 3, 2, 1],       # scores 6,10,12,12,10,6 -> ties
                  [0, 0, 0, 0, 0, 1],       # only block 5 positive
                  [1, 1, 1, 1, 1, 1],       # scores 1..6 increasing
                  [-1, -2, -3, -4, -5, -6],  # all negative, least negative first
                  [0, 0, 0, 0, 0, 0],       # all zero -> lowest indices
                  [3, 0, 0, 0, 0, 0]], dtype=float)
    q = np.zeros((nb * bs, d))
    for a in range(nb):
        q[a * bs:(a + 1) * bs, :nb] = w[a]
    sig = ro.block_scores(ro.pool_blocks(q, bs), ro.pool_blocks(k, bs))
    np.testing.assert_allclose(sig[0] * math.sqrt(d), [6, 10, 12, 12, 10, 6])
    idx = ro.select_topk(sig, 3)
    expected = [[1, 2, 3],    # 12, 12, then 10 @ 1 beats 10 @ 4
                [0, 1, 5],    # 6 > 0 = 0 = ...: ties at 0 go to 0, 1
                [3, 4, 5],
                [0, 1, 2],
                [0, 1, 2],
                [0, 1, 2]]    # 3 > 0 = 0 ...
    assert idx.tolist() == expected


def test_selector_bruteforce_python():
    bs, N, d, kb = 5, 37, 6, 3          # ragged: last block has 2 tokens
    q, k = _rand((N, d), 2), _rand((N, d), 3)
    nb = -(-N // bs)
    idx = ro.select_topk(ro.block_scores(ro.pool_blocks(q, bs), ro.pool_blocks(k, bs)), kb)
    def mean(x, b):
        toks = [t for t in range(b * bs, (b + 1) * bs) if t < N]
        return [sum(x[t][c] for t in toks) / len(toks) for c in range(d)]
    qb = [mean(q.tolist(), b) for b in range(nb)]
    kbar = [mean(k.tolist(), b) for b in range(nb)]
    for a in range(nb):
        sc = [(sum(qb[a][c] * kbar[b][c] for c in range(d)) / math.sqrt(d), b) for b in range(nb)]
        best = sorted(sc, key=lambda t: (-t[0], t[1]))[:kb]
        assert sorted(b for _, b in best) == idx[a].tolist()


def test_near_tie_detection():
    sig = np.array([[5.0, 4.0, 4.0 * (1 + 1e-7), 1.0],
                    [5.0, 4.0, 3.0, 1.0]])
    assert ro.near_ties(sig, 2) == [0]
    assert ro.near_ties(sig, 4) == []


# ---------------------------------------------------------------- sparse branch

def _sdpa64(q, k, v, mask=None):
    """torch's scaled_dot_product_attention in float64 on [N, d] operands."""
    Q, K, V = (torch.from_numpy(np.ascontiguousarray(t))[None, None] for t in (q, k, v))
    m = None if mask is None else torch.from_numpy(mask)[None, None]
    return torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=m)[0, 0].numpy()


def test_sparse_branch_equals_masked_dense_sdpa():
    bs, N, d = 8, 45, 16               # 6 blocks, last has 5 tokens
    q, k, v = _rand((N, d), 4), _rand((N, d), 5), _rand((N, d), 6)
    nb = -(-N // bs)
    kept = {a: sorted(np.random.default_rng(7 + a).choice(nb, 2, replace=False).tolist()) for a in range(nb)}
    mask = np.zeros((N, N), dtype=bool)
    for a in range(nb):
        for b in kept[a]:
            mask[a * bs:(a + 1) * bs, b * bs:min(N, (b + 1) * bs)] = True
    ref = _sdpa64(q, k, v, mask)
    for a in range(nb):
        got = ro.sparse_branch_block(q, k, v, a, kept[a], bs)
        np.testing.assert_allclose(got, ref[a * bs:min(N, (a + 1) * bs)], rtol=1e-12, atol=1e-12)


def test_dense_limit_s0_is_sdpa_and_gate_zero_is_sparse():
    w = synth.custom_workload(synth.WORKLOADS[0], H=1, T=2, Hg=8, W=9, block=16,
                              sparsity_permille=0, k_b=ro.kb_from_sparsity(9, 0))
    inp = synth.make_inputs(w)
    assert w.k_b == w.n_blocks
    res = ro.rola_forward(inp, bs=w.block, k_b=w.k_b, grid=(w.T, w.Hg, w.W))[(0, 0)]
    q, k, v, _ = ro.head_slices(inp, 0, 0)
    ref = _sdpa64(q, k, v)
    for a, o in res.o.items():
        lo, hi = ro.block_range(a, w.block, w.N)
        assert np.all(res.o_lin[a] == 0.0)
        np.testing.assert_allclose(o, ref[lo:hi], rtol=1e-12, atol=1e-12)
    # g = 0: output is exactly the block-sparse branch
    w2 = synth.custom_workload(synth.WORKLOADS[0], H=1, gate_const=0.0)
    inp2 = synth.make_inputs(w2)
    r2 = ro.rola_forward(inp2, bs=w2.block, k_b=w2.k_b, grid=(w2.T, w2.Hg, w2.W))[(0, 0)]
    for a in r2.o:
        assert np.array_equal(r2.o[a], r2.o_sp[a])
        assert np.abs(r2.o_lin[a]).max() > 0


# ---------------------------------------------------------------- linear branch

def test_rope_split_and_hand_rotation():
    assert ro.rope_split(32) == (12, 10, 10)
    assert ro.rope_split(16) == (8, 4, 4)
    assert ro.rope_split(6) == (2, 2, 2)
    # r = 6: one pair per axis, frequency 1 -> angle equals (t, y, x)
    T, Hg, W = 3, 4, 5
    th = ro.rope_angles(T * Hg * W, T, Hg, W, 6, 10000.0)
    n = 2 * Hg * W + 3 * W + 4             # (t, y, x) = (2, 3, 4)
    psi = np.array([1.0, 0.0, 1.0, 0.0, 1.0, 0.0])
    got = ro.rotate(psi, th[n])
    want = [math.cos(2), math.sin(2), math.cos(3), math.sin(3), math.cos(4), math.sin(4)]
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-15)
    # second t pair at r = 32 turns by t * 10000^(-2/12)
    th32 = ro.rope_angles(T * Hg * W, T, Hg, W, 32, 10000.0)
    assert abs(th32[n, 1] - 2 * 10000 ** (-2 / 12)) < 1e-15
    assert abs(th32[n, 6] - 3.0) < 1e-15 and abs(th32[n, 11] - 4.0) < 1e-15


def test_rope_is_orthogonal_and_relative():
    T, Hg, W, r = 3, 5, 7, 12
    N = T * Hg * W
    psi_a, psi_b = _rand((N, r), 8), _rand((N, r), 9)
    th = ro.rope_angles(N, T, Hg, W, r, 10000.0)
    ra, rb = ro.rotate(psi_a, th), ro.rotate(psi_b, th)
    np.testing.assert_allclose(np.linalg.norm(ra, axis=1), np.linalg.norm(psi_a, axis=1), rtol=1e-13)
    # shifting every position by the same offset leaves rho_n . rho_j unchanged
    t, y, x = ro.token_coords(N, T, Hg, W)
    th_shift = np.zeros_like(th)
    p = 0
    for pos, ra_ in zip((t + 5, y + 2, x + 11), ro.rope_split(r)):
        for m in range(ra_ // 2):
            th_shift[:, p] = pos * 10000.0 ** (-2.0 * m / ra_)
            p += 1
    G = ra @ rb.T
    Gs = ro.rotate(psi_a, th_shift) @ ro.rotate(psi_b, th_shift).T
    np.testing.assert_allclose(Gs, G, rtol=1e-10, atol=1e-10)


def test_feature_map_matches_torch_elu():
    u = np.linspace(-8, 8, 1001)
    want = torch.nn.functional.elu(torch.from_numpy(u)).numpy() + 1.0
    np.testing.assert_allclose(ro.phi(u), want, rtol=1e-15, atol=2e-16)
    assert np.all(ro.phi(u) > 0)


def test_state_identity_global_minus_kept():
    w = synth.custom_workload(synth.WORKLOADS[0], H=1)
    inp = synth.make_inputs(w)
    q, k, v, P = ro.head_slices(inp, 0, 0)
    th = ro.rope_angles(w.N, w.T, w.Hg, w.W, w.r, w.rope_base)
    S_blk, z_blk, S, z = ro.block_states(k, v, P, th, w.block)
    for kept in ([0, 3, 7, 15], [1], list(range(15))):
        a1, b1 = ro.complement_state(S_blk, z_blk, S, z, kept)
        a2, b2 = ro.complement_state_direct(S_blk, z_blk, kept)
        assert np.abs(a1 - a2).max() <= 1e-12 * np.abs(S).max()
        assert np.abs(b1 - b2).max() <= 1e-12 * np.abs(z).max()


def test_linear_special_case_is_plain_elu_linear_attention():
    # r = d, P = I, zero angles: the branch must reduce to elu+1 linear
    # attention over the complement tokens, computed here with torch's elu.
    bs, N, d = 4, 26, 6
    q, k, v = _rand((N, d), 10), _rand((N, d), 11), _rand((N, d), 12)
    P = np.eye(d)
    th = np.zeros((N, d // 2))
    S_blk, z_blk, S, z = ro.block_states(k, v, P, th, bs)
    kept = [1, 4]
    S_U, z_U = ro.complement_state(S_blk, z_blk, S, z, kept)
    got = ro.linear_branch_block(q, P, th, 2, bs, S_U, z_U, empty=False)
    fq = torch.nn.functional.elu(torch.from_numpy(q)).numpy() + 1
    fk = torch.nn.functional.elu(torch.from_numpy(k)).numpy() + 1
    U = [j for j in range(N) if j // bs not in kept]
    for i, n in enumerate(range(8, 12)):
        wts = fk[U] @ fq[n]
        np.testing.assert_allclose(got[i], (wts @ v[U]) / wts.sum(), rtol=1e-12)


def _bruteforce_token_level(q, k, v, P, g, kept_blocks, bs, grid, base, n):
    """Full RoLA output for query token n by explicit loops over key tokens:
    softmax over the kept blocks' tokens; linear attention with per-pair
    math.cos/math.sin rotation over every other valid token."""
    N, d = q.shape
    T, Hg, W = grid
    r = P.shape[1]
    rt, rh, rw = ro.rope_split(r)

    def angles(j):
        t, y, x = j // (Hg * W), (j // W) % Hg, j % W
        out = []
        for pos, ra in ((t, rt), (y, rh), (x, rw)):
            out += [pos * base ** (-2.0 * m / ra) for m in range(ra // 2)]
        return out

    def feat(vec, j):
        u = [sum(vec[c] * P[c, e] for c in range(d)) for e in range(r)]
        psi = [x + 1.0 if x > 0 else math.exp(x) for x in u]
        rho = []
        for p, a in enumerate(angles(j)):
            x0, x1 = psi[2 * p], psi[2 * p + 1]
            rho += [x0 * math.cos(a) - x1 * math.sin(a), x0 * math.sin(a) + x1 * math.cos(a)]
        return psi, rho

    keep = [j for j in range(N) if j // bs in kept_blocks]
    rest = [j for j in range(N) if j // bs not in kept_blocks]
    s = [sum(q[n, c] * k[j, c] for c in range(d)) / math.sqrt(d) for j in keep]
    m = max(s)
    p = [math.exp(x - m) for x in s]
    o_sp = [sum(p[i] * v[j, e] for i, j in enumerate(keep)) / sum(p) for e in range(d)]
    if not rest:
        return np.array(o_sp)
    psi_n, rho_n = feat(q[n], n)
    num = [0.0] * d
    den = 0.0
    for j in rest:
        psi_j, rho_j = feat(k[j], j)
        wn = sum(a * b for a, b in zip(rho_n, rho_j))
        den += sum(a * b for a, b in zip(psi_n, psi_j))
        for e in range(d):
            num[e] += wn * v[j, e]
    return np.array(o_sp) + g * np.array(num) / den


@pytest.mark.parametrize("grid,bs,r,kb", [((2, 5, 7), 16, 6, 2), ((3, 4, 5), 8, 16, 3)])
def test_full_forward_bruteforce_ragged(grid, bs, r, kb):
    T, Hg, W = grid
    N, d = T * Hg * W, 8
    w = synth.Workload("t", 1, 2, d, T, Hg, W, bs, 0, kb, r, seed=21, gate_const=None)
    inp = synth.make_inputs(w)
    res = ro.rola_forward(inp, bs=bs, k_b=kb, grid=grid)
    for h in range(2):
        q, k, v, P = ro.head_slices(inp, 0, h)
        g = float(inp["gate"][h])
        out = res[(0, h)]
        nb = -(-N // bs)
        for n in (0, bs + 3, N - 1):
            a = n // bs
            want = _bruteforce_token_level(q, k, v, P, g, set(out.idx[a].tolist()), bs, grid, 10000.0, n)
            got = out.o[a][n - a * bs]
            np.testing.assert_allclose(got, want, rtol=1e-10, atol=1e-12)
        assert out.idx.shape == (nb, kb)


def test_generator_is_deterministic_and_bf16():
    w = synth.WORKLOADS[0]
    a, b = synth.make_inputs(w), synth.make_inputs(w)
    for key in ("q", "k", "v", "P", "gate"):
        assert np.array_equal(a[key], b[key])
    assert a["q"].dtype == np.uint16 and a["q"].shape == (1, 1024, 2, 64)
    q = ro.bf16_to_f64(a["q"])
    # structured q and k share the positional field: strongly correlated
    k = ro.bf16_to_f64(a["k"])
    assert np.corrcoef(q.ravel(), k.ravel())[0, 1] > 0.6


def test_per_head_selection_is_nested_and_brute_force():
    """Head-adaptive counts: each head's kept set is the brute-force top
    kb_per_head[h] by (score desc, index asc), the unused entries are -1, and
    the sets are nested in the count (keeping one more block adds one)."""
    rng = np.random.default_rng(21)
    B, N, H, d, bs = 1, 160, 3, 8, 16
    inp = {"q": (rng.standard_normal((B, N, H, d)) * 4).astype(np.float32),
           "k": (rng.standard_normal((B, N, H, d)) * 4).astype(np.float32)}
    # bf16 bit patterns of the draws (truncated: any bf16 values will do here)
    inp = {kk: (vv.view(np.uint32) >> 16).astype(np.uint16) for kk, vv in inp.items()}
    kbh = [1, 4, 7]
    idx, sig = ro.select_all_per_head(inp, bs, kbh, 7)
    nb = N // bs
    for h, kh in enumerate(kbh):
        assert (idx[0, h, :, kh:] == -1).all()
        for a in range(nb):
            order = sorted(range(nb), key=lambda j: (-sig[0, h, a, j], j))
            assert sorted(order[:kh]) == idx[0, h, a, :kh].tolist()
    for kh in range(1, nb):
        small, _ = ro.select_all_per_head(inp, bs, [kh] * H, nb)
        big, _ = ro.select_all_per_head(inp, bs, [kh + 1] * H, nb)
        for h in range(H):
            for a in range(nb):
                s1, s2 = set(small[0, h, a, :kh].tolist()), set(big[0, h, a, :kh + 1].tolist())
                assert s1 < s2 and len(s2 - s1) == 1
