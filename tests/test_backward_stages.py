"""The staged form of the RoLA gradient that a kernel implementation follows,
checked against the gradient oracle: a query-major pass that forms the query
side of the linear branch (dS_U, dz_U per query block, and o_lin again), D =
dO . o - g dO . o_lin from the layer output, the softmax from the saved per-row
log-sum-exp, and dQ; the transposed
block mask; per key block, dS_b = (sum of all dS_U) - (those of the query blocks
that keep b), the mirror of the forward's global-minus-kept states; and a
key-major pass over the keeping query blocks for dK, dV and the key side of
the linear branch.  Every step uses only saved statistics and the mask."""
import math

import numpy as np
import pytest

from oracle import rola_backward_oracle as rbo
from oracle import rola_oracle as ro


def staged_backward(q, k, v, P, g, dO, bs, idx, grid):
    N, d = q.shape
    r = P.shape[1]
    nb = -(-N // bs)
    sc = 1 / math.sqrt(d)
    theta = ro.rope_angles(N, *grid, r, 10000.0)
    lse, den = rbo.forward_stats(q, k, v, P, bs=bs, idx=idx, grid=grid)
    S_blk, z_blk, S, z = ro.block_states(k, v, P, theta, bs)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    dP = np.zeros_like(P)
    dg = 0.0
    D = np.zeros(N)
    dSU, dzU = {}, {}

    # the layer output, as the forward wrote it
    res = ro.rola_head(q, k, v, P, g, bs=bs, k_b=idx.shape[1], grid=grid, rope_base=10000.0, idx=idx)

    # query-major pass: the query side of the linear branch first (it recomputes
    # o_lin), then D = dO . o - g dO . o_lin = dO . o_sp, the softmax from the
    # saved log-sum-exp, and dQ
    for a in range(nb):
        lo, hi = ro.block_range(a, bs, N)
        o_lin = np.zeros((hi - lo, d))
        if not np.isnan(den[lo]):  # NaN: every block kept, no linear branch
            S_U, z_U = ro.complement_state(S_blk, z_blk, S, z, idx[a])
            u = q[lo:hi] @ P
            psi = ro.phi(u)
            rho = ro.rotate(psi, theta[lo:hi])
            o_lin = rho @ S_U / den[lo:hi, None]
            dg += (dO[lo:hi] * o_lin).sum()
            dnum = g * dO[lo:hi] / den[lo:hi, None]
            dden = -(g * dO[lo:hi] * o_lin).sum(1) / den[lo:hi]
            dpsi = dden[:, None] * z_U + ro.rotate(dnum @ S_U.T, -theta[lo:hi])
            du = dpsi * rbo.phi_grad(u)
            dq[lo:hi] += du @ P.T
            dP += q[lo:hi].T @ du
            dSU[a] = rho.T @ dnum
            dzU[a] = (dden[:, None] * psi).sum(0)
        D[lo:hi] = (dO[lo:hi] * res.o[a]).sum(1) - g * (dO[lo:hi] * o_lin).sum(1)
        J = ro.kept_tokens(idx[a], bs, N)
        p = np.exp(q[lo:hi] @ k[J].T * sc - lse[lo:hi, None])
        ds = p * (dO[lo:hi] @ v[J].T - D[lo:hi, None])
        dq[lo:hi] += ds @ k[J] * sc

    # block-state gradients: all query blocks' dS_U minus those that keep the block
    off, rows = rbo.transposed_mask(idx, nb)
    tot_S = sum(dSU.values(), np.zeros((r, d)))
    tot_z = sum(dzU.values(), np.zeros(r))

    # key-major pass over the query blocks that keep each key block, and the
    # key side of the linear branch
    uk = k @ P
    rhok = ro.rotate(ro.phi(uk), theta)
    for j in range(nb):
        lo, hi = ro.block_range(j, bs, N)
        keepers = [int(a) for a in rows[off[j]:off[j + 1]]]
        dS_b = tot_S - sum((dSU[a] for a in keepers if a in dSU), np.zeros((r, d)))
        dz_b = tot_z - sum((dzU[a] for a in keepers if a in dzU), np.zeros(r))
        for a in keepers:
            qlo, qhi = ro.block_range(a, bs, N)
            p = np.exp(q[qlo:qhi] @ k[lo:hi].T * sc - lse[qlo:qhi, None])
            ds = p * (dO[qlo:qhi] @ v[lo:hi].T - D[qlo:qhi, None])
            dk[lo:hi] += ds.T @ q[qlo:qhi] * sc
            dv[lo:hi] += p.T @ dO[qlo:qhi]
        dv[lo:hi] += rhok[lo:hi] @ dS_b
        dpsi = dz_b + ro.rotate(v[lo:hi] @ dS_b.T, -theta[lo:hi])
        du = dpsi * rbo.phi_grad(uk[lo:hi])
        dk[lo:hi] += du @ P.T
        dP += k[lo:hi].T @ du
    return dq, dk, dv, dP, dg


@pytest.mark.parametrize("kb", [1, 4, 9])
def test_staged_backward_equals_the_oracle(kb):
    rng = np.random.default_rng(kb)
    grid, bs, d, r = (3, 4, 6), 8, 16, 12   # 72 tokens, 9 blocks of 8; r = 12 -> 4 / 4 / 4
    N = int(np.prod(grid))
    nb = -(-N // bs)
    q, k, v, dO = (rng.standard_normal((N, d)) for _ in range(4))
    P = rng.standard_normal((d, r)) / math.sqrt(d)
    idx = np.stack([np.sort(rng.choice(nb, size=kb, replace=False)) for _ in range(nb)])
    G = rbo.rola_head_backward(q, k, v, P, 0.6, dO, bs=bs, idx=idx, grid=grid)
    got = staged_backward(q, k, v, P, 0.6, dO, bs, idx, grid)
    for a, b in zip(got, (G.dq, G.dk, G.dv, G.dP, G.dg)):
        assert np.max(np.abs(np.asarray(a) - np.asarray(b))) < 1e-10
