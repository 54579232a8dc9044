"""fp64 CPU oracle for the gradients of RoLA attention, one (batch, head) at a time.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this module:
only ``tests/`` may use it.  It shares no code with the CUDA library.

Why a backward: the SparkDiffusion write-up (「首次定义“高稀疏陷阱”」, 0539edu.com
news page, section 05) and the project blog ("A simple staging principle",
item 1) train the RoLA module for a short sparse warm-up, so that the dense
pretrained model adapts to 97 % sparsity; that needs the gradients of the
RoLA output with respect to q, k, v, the low-rank projection P_h and the gate.
The pages print no backward; the gradient here is the exact derivative of the
forward in ``rola_oracle.rola_head`` with the block mask held fixed (selection
is a discrete choice and passes no gradient), taken by the chain rule through
the forward's steps in reverse order:

4. combine ``o = o_sp + g o_lin``: ``do_sp = dO``, ``do_lin = g dO``,
   ``dg = sum dO . o_lin``.
3. linear branch of query block ``a`` (rows n):
   ``num_n = rho_n^T S_U``, ``den_n = psi_n . z_U``, ``o_lin = num / den``;
   ``dnum = do_lin / den``, ``dden = -(do_lin . o_lin) / den``;
   ``drho_n = S_U dnum_n``, ``dpsi_n = dden_n z_U + R^T drho_n``;
   ``dS_U = sum_n rho_n dnum_n^T``, ``dz_U = sum_n dden_n psi_n``.
   The complement ``S_U = S - sum_{b in K_a} S_b`` with ``S = sum_b S_b`` sends
   ``+dS_U`` to every block state and ``-dS_U`` to the kept ones (likewise z).
   Block states ``S_b = sum_j rho_j v_j^T``, ``z_b = sum_j psi_j``:
   ``drho_j = dS_b v_j``, ``dv_j += dS_b^T rho_j``, ``dpsi_j = dz_b + R^T drho_j``.
   Features ``psi = phi(u)``, ``u = x P_h``: ``du = dpsi phi'(u)`` with
   ``phi'(u) = 1`` for ``u > 0`` and ``e^u`` otherwise; ``dx += du P_h^T``,
   ``dP_h += x^T du`` (x is q for the query side, k for the key side).
2. sparse branch (softmax over the kept blocks' valid keys, scale 1/sqrt(d)):
   ``dp = dO v_J^T``, ``ds = p (dp - rowsum(dO . o_sp))``,
   ``dq += ds k_J / sqrt(d)``, ``dk_J += ds^T q / sqrt(d)``, ``dv_J += p^T dO``.

Parity pins (tests/test_oracle_rola_backward.py): central finite differences of
the forward oracle along random directions for every input; the dense limit
(every block kept) against library autograd of scaled dot-product attention;
the gate-zero case against library autograd of masked attention; a planted
slip that the finite differences catch.  ``transposed_mask`` is checked by
membership both ways, ``forward_stats`` against the library log-sum-exp and by
rebuilding the forward's sparse output from it.
"""
from __future__ import annotations

import math

import numpy as np

from oracle.rola_oracle import (block_range, block_states, complement_state, kept_tokens, phi,
                                rope_angles, rotate)


def phi_grad(u: np.ndarray) -> np.ndarray:
    """Derivative of elu(u) + 1: 1 for u > 0, e^u otherwise."""
    return np.where(u > 0, 1.0, np.exp(np.minimum(u, 0.0)))


class HeadGrads:
    def __init__(self, N: int, d: int, r: int):
        self.dq = np.zeros((N, d))
        self.dk = np.zeros((N, d))
        self.dv = np.zeros((N, d))
        self.dP = np.zeros((d, r))
        self.dg = 0.0
        self.dS_blk = None   # gradient reaching each block state [nb, r, d]
        self.dz_blk = None   # [nb, r]


def rola_head_backward(q, k, v, P_h, g_h: float, dO, *, bs: int, idx, grid,
                       rope_base: float = 10000.0) -> HeadGrads:
    """Gradients of sum(dO * o) for one (batch, head): q, k, v, dO [N, d] float64
    over the valid tokens, P_h [d, r], idx [nb, k_b] the (fixed) kept blocks."""
    N, d = q.shape
    r = P_h.shape[1]
    nb = -(-N // bs)
    T, Hg, W = grid
    idx = np.asarray(idx, dtype=np.int64)
    theta = rope_angles(N, T, Hg, W, r, rope_base)
    G = HeadGrads(N, d, r)
    S_blk, z_blk, S, z = block_states(k, v, P_h, theta, bs)
    dS_blk = np.zeros_like(S_blk)
    dz_blk = np.zeros_like(z_blk)
    scale = 1.0 / math.sqrt(d)

    for a in range(nb):
        lo, hi = block_range(a, bs, N)
        kept = idx[a]
        dOa = dO[lo:hi]
        qa = q[lo:hi]
        # 2. sparse branch
        J = kept_tokens(kept, bs, N)
        s = (qa @ k[J].T) * scale
        s -= s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p /= p.sum(axis=1, keepdims=True)
        o_sp = p @ v[J]
        dp = dOa @ v[J].T
        ds = p * (dp - (dOa * o_sp).sum(axis=1, keepdims=True))
        G.dq[lo:hi] += (ds @ k[J]) * scale
        G.dk[J] += (ds.T @ qa) * scale
        G.dv[J] += p.T @ dOa
        # 3. linear branch (nothing when every block is kept)
        if len(set(kept.tolist())) >= nb:
            continue
        S_U, z_U = complement_state(S_blk, z_blk, S, z, kept)
        uq = qa @ P_h
        psiq = phi(uq)
        rhoq = rotate(psiq, theta[lo:hi])
        den = psiq @ z_U
        o_lin = (rhoq @ S_U) / den[:, None]
        G.dg += float((dOa * o_lin).sum())
        dlin = g_h * dOa
        dnum = dlin / den[:, None]
        dden = -(dlin * o_lin).sum(axis=1) / den
        drhoq = dnum @ S_U.T
        dpsiq = dden[:, None] * z_U[None, :] + rotate(drhoq, -theta[lo:hi])
        duq = dpsiq * phi_grad(uq)
        G.dq[lo:hi] += duq @ P_h.T
        G.dP += qa.T @ duq
        dS_U = rhoq.T @ dnum
        dz_U = (dden[:, None] * psiq).sum(axis=0)
        # S_U = S - sum_kept S_b and S = sum_b S_b
        dS_blk += dS_U[None]
        dz_blk += dz_U[None]
        dS_blk[kept] -= dS_U[None]
        dz_blk[kept] -= dz_U[None]

    # block states back to k, v and P_h
    uk = k @ P_h
    rhok = rotate(phi(uk), theta)
    for b in range(nb):
        lo, hi = block_range(b, bs, N)
        drho = v[lo:hi] @ dS_blk[b].T
        G.dv[lo:hi] += rhok[lo:hi] @ dS_blk[b]
        dpsi = dz_blk[b][None, :] + rotate(drho, -theta[lo:hi])
        duk = dpsi * phi_grad(uk[lo:hi])
        G.dk[lo:hi] += duk @ P_h.T
        G.dP += k[lo:hi].T @ duk
    G.dS_blk, G.dz_blk = dS_blk, dz_blk
    return G


def transposed_mask(idx, nb: int):
    """For each key block j, the ascending query blocks a whose kept list holds
    j, in compressed form: ``rows[offsets[j]:offsets[j+1]]``.  The key-major
    side of the backward walks these lists."""
    idx = np.asarray(idx, dtype=np.int64)
    lists = [[] for _ in range(nb)]
    for a in range(idx.shape[0]):
        for j in sorted(set(idx[a].tolist())):
            lists[j].append(a)
    offsets = np.zeros(nb + 1, dtype=np.int64)
    offsets[1:] = np.cumsum([len(x) for x in lists])
    rows = np.array([a for x in lists for a in x], dtype=np.int32)
    return offsets, rows


def forward_stats(q, k, v, P_h, *, bs: int, idx, grid, rope_base: float = 10000.0):
    """Per-row quantities a forward saves for the backward: the natural-log
    log-sum-exp of the scaled scores over the kept keys, and the linear
    branch's denominator psi_q . z_U (NaN for query blocks whose complement is
    empty, where the linear branch is zero)."""
    N, d = q.shape
    nb = -(-N // bs)
    T, Hg, W = grid
    idx = np.asarray(idx, dtype=np.int64)
    theta = rope_angles(N, T, Hg, W, P_h.shape[1], rope_base)
    S_blk, z_blk, S, z = block_states(k, v, P_h, theta, bs)
    lse = np.empty(N)
    den = np.full(N, np.nan)
    for a in range(nb):
        lo, hi = block_range(a, bs, N)
        J = kept_tokens(idx[a], bs, N)
        s = (q[lo:hi] @ k[J].T) / math.sqrt(d)
        m = s.max(axis=1)
        lse[lo:hi] = m + np.log(np.exp(s - m[:, None]).sum(axis=1))
        if len(set(idx[a].tolist())) < nb:
            _, z_U = complement_state(S_blk, z_blk, S, z, idx[a])
            den[lo:hi] = phi(q[lo:hi] @ P_h) @ z_U
    return lse, den
