"""fp64 CPU oracle for RoLA hybrid block-sparse + rotary low-rank linear attention.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this module:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may use it.  It shares no code with
the CUDA library; both sides consume the same seeded bf16 bytes.

What it computes, and where it comes from
-----------------------------------------
The method is RoLA as described in the SparkDiffusion write-up
(「首次定义“高稀疏陷阱”」, 0539edu.com news page, section 05 "RoLA: keeping
global information at extreme sparsity"): a block-sparse softmax branch keeps
the high-energy query-key block interactions, and a rotary-positioned
low-rank linear branch restores the global context that sparsification
dropped.  The arXiv listing of the SparkDiffusion paper (montaan.com,
"Sources") names the sibling idea "3D RoPE-driven Sparse-LowRank Attention",
hence a 3-D rotary embedding.  The pages give no formula; this library fixes
one concrete form, written out step by step below in the order the method
applies it:

1. selector: mean-pool q and k over each block's *valid* tokens, score
   ``sigma_ab = qbar_a . kbar_b / sqrt(d)``, keep the ``k_b`` largest per query
   block, ties to the lower block index, emitted ascending.
   ``k_b = ceil((1000 - s_permille) * n_blocks / 1000)`` in integers.
2. sparse branch: exact softmax over the tokens of the kept blocks (padded
   tokens excluded), scale ``1/sqrt(d)``.
3. linear branch: ``psi(x) = phi(x P_h)`` with ``phi = elu + 1``;
   ``rho = R(t, y, x) psi`` (feature map first, then rotation);
   per-block states ``S_b = sum_j rho_j v_j^T`` (r x d) and
   ``z_b = sum_j psi_j`` over the block's valid keys; global ``S, z`` are their
   sums; the complement state of query block ``a`` is ``S - sum_{b in K_a} S_b``
   (likewise ``z``); ``o_lin = rho_q^T S_U / (psi_q^T z_U)`` -- rotation in the
   numerator only -- and ``o_lin = 0`` when the complement is empty.
4. combine: ``o = o_sp + g_h o_lin``.

Readings taken where the pages are silent (each repeated where it is used):
valid-token pooling; integer k_b; no forced diagonal/sink block; one
projection per head shared by q and k; phi before rotation; denominator
unrotated; 3-D rotary split ``r_t = r - 4 floor(r/6)``, ``r_h = r_w = 2 floor(r/6)``
with interleaved pairs and angle ``pos * base**(-2m / r_axis)``; empty
complement gives zero; padded keys excluded from both branches.
"""
from __future__ import annotations

import math

import numpy as np


# ---------------------------------------------------------------------------
# scalars and helpers
# ---------------------------------------------------------------------------

def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to float64."""
    return (np.asarray(bits).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def kb_from_sparsity(n_blocks: int, sparsity_permille: int) -> int:
    """Kept blocks per query block: ceil((1 - s) * n_blocks), in integers so that
    97 % of 100 blocks keeps exactly 3 (floating point would give 4)."""
    keep = (1000 - sparsity_permille) * n_blocks
    return -(-keep // 1000)


def token_coords(N: int, T: int, Hg: int, W: int):
    """Frame-major raster order: token n -> (t, y, x)."""
    n = np.arange(N, dtype=np.int64)
    return n // (Hg * W), (n // W) % Hg, n % W


def rope_split(r: int):
    """Rank split over (t, h, w): r_t = r - 4 floor(r/6), r_h = r_w = 2 floor(r/6)."""
    rh = 2 * (r // 6)
    return r - 2 * rh, rh, rh


def rope_angles(N: int, T: int, Hg: int, W: int, r: int, base: float) -> np.ndarray:
    """theta[n, p] for the r/2 rotation pairs: the t-axis pairs first, then h,
    then w; pair m of an axis with r_axis dims turns by pos * base^(-2m/r_axis)."""
    t, y, x = token_coords(N, T, Hg, W)
    theta = np.zeros((N, r // 2), dtype=np.float64)
    p = 0
    for pos, ra in zip((t, y, x), rope_split(r)):
        for m in range(ra // 2):
            theta[:, p] = pos.astype(np.float64) * base ** (-2.0 * m / ra)
            p += 1
    return theta


def phi(u: np.ndarray) -> np.ndarray:
    """elu(u) + 1: u + 1 for u > 0, exp(u) otherwise (strictly positive)."""
    return np.where(u > 0, u + 1.0, np.exp(np.minimum(u, 0.0)))


def rotate(psi: np.ndarray, theta: np.ndarray) -> np.ndarray:
    """Apply the block-diagonal rotation R(theta) to interleaved pairs (2p, 2p+1)."""
    c, s = np.cos(theta), np.sin(theta)
    a, b = psi[..., 0::2], psi[..., 1::2]
    out = np.empty_like(psi)
    out[..., 0::2] = a * c - b * s
    out[..., 1::2] = a * s + b * c
    return out


def block_range(blk: int, bs: int, N: int):
    return blk * bs, min(N, (blk + 1) * bs)


# ---------------------------------------------------------------------------
# 1. selector
# ---------------------------------------------------------------------------

def pool_blocks(x: np.ndarray, bs: int) -> np.ndarray:
    """Mean of each block's valid tokens; x is [N, d] for one (batch, head)."""
    N = x.shape[0]
    nb = -(-N // bs)
    out = np.empty((nb, x.shape[1]), dtype=np.float64)
    for b in range(nb):
        lo, hi = block_range(b, bs, N)
        out[b] = x[lo:hi].sum(axis=0) / (hi - lo)
    return out


def block_scores(qbar: np.ndarray, kbar: np.ndarray) -> np.ndarray:
    d = qbar.shape[1]
    return (qbar @ kbar.T) / math.sqrt(d)


def select_topk(sigma: np.ndarray, k_b: int) -> np.ndarray:
    """Per row, the k_b block indices that come first when sorted by
    (-sigma, index); returned ascending.  No block is forced in."""
    nb = sigma.shape[1]
    ids = np.arange(nb)
    out = np.empty((sigma.shape[0], k_b), dtype=np.int32)
    for a in range(sigma.shape[0]):
        order = np.lexsort((ids, -sigma[a]))
        out[a] = np.sort(order[:k_b])
    return out


def near_ties(sigma: np.ndarray, k_b: int, rel: float = 1e-5):
    """Rows whose k-th and (k+1)-th largest scores lie within ``rel`` of each
    other (relative to the larger magnitude): the mask there is decided by
    rounding, so a GPU mask may legitimately differ in that row."""
    nb = sigma.shape[1]
    if k_b >= nb:
        return []
    rows = []
    for a in range(sigma.shape[0]):
        s = np.sort(sigma[a])[::-1]
        hi, lo = s[k_b - 1], s[k_b]
        if abs(hi - lo) <= rel * max(abs(hi), abs(lo)):
            rows.append(a)
    return rows


# ---------------------------------------------------------------------------
# 2. sparse branch
# ---------------------------------------------------------------------------

def kept_tokens(kept_blocks, bs: int, N: int) -> np.ndarray:
    return np.concatenate([np.arange(*block_range(int(b), bs, N)) for b in kept_blocks])


def sparse_branch_block(q: np.ndarray, k: np.ndarray, v: np.ndarray, a: int,
                        kept_blocks, bs: int) -> np.ndarray:
    """Softmax attention of query block a's valid rows over the valid tokens of
    its kept key blocks; scale 1/sqrt(d), max subtracted."""
    N, d = q.shape
    lo, hi = block_range(a, bs, N)
    J = kept_tokens(kept_blocks, bs, N)
    s = (q[lo:hi] @ k[J].T) / math.sqrt(d)
    s -= s.max(axis=1, keepdims=True)
    p = np.exp(s)
    return (p @ v[J]) / p.sum(axis=1, keepdims=True)


# ---------------------------------------------------------------------------
# 3. linear branch
# ---------------------------------------------------------------------------

def features(x: np.ndarray, P_h: np.ndarray, theta: np.ndarray):
    """psi = phi(x P_h) and rho = R(theta) psi for rows x [n, d]."""
    psi = phi(x @ P_h)
    return psi, rotate(psi, theta)


def block_states(k: np.ndarray, v: np.ndarray, P_h: np.ndarray, theta: np.ndarray, bs: int):
    """S_b = sum_j rho_j v_j^T ([nb, r, d]) and z_b = sum_j psi_j ([nb, r]) over each
    block's valid keys, plus their totals S [r, d] and z [r]."""
    N = k.shape[0]
    nb = -(-N // bs)
    psi, rho = features(k, P_h, theta)
    r, d = P_h.shape[1], v.shape[1]
    S_blk = np.empty((nb, r, d))
    z_blk = np.empty((nb, r))
    for b in range(nb):
        lo, hi = block_range(b, bs, N)
        S_blk[b] = rho[lo:hi].T @ v[lo:hi]
        z_blk[b] = psi[lo:hi].sum(axis=0)
    return S_blk, z_blk, S_blk.sum(axis=0), z_blk.sum(axis=0)


def complement_state(S_blk, z_blk, S, z, kept_blocks):
    """Global state minus the kept blocks' states (the form the method uses)."""
    kept = np.asarray(kept_blocks, dtype=np.int64)
    return S - S_blk[kept].sum(axis=0), z - z_blk[kept].sum(axis=0)


def complement_state_direct(S_blk, z_blk, kept_blocks):
    """Sum over the blocks that were not kept (for the identity check)."""
    mask = np.ones(S_blk.shape[0], dtype=bool)
    mask[np.asarray(kept_blocks, dtype=np.int64)] = False
    return S_blk[mask].sum(axis=0), z_blk[mask].sum(axis=0)


def linear_branch_block(q: np.ndarray, P_h: np.ndarray, theta: np.ndarray, a: int, bs: int,
                        S_U: np.ndarray, z_U: np.ndarray, empty: bool) -> np.ndarray:
    """o_lin = rho_q^T S_U / (psi_q^T z_U) for query block a's valid rows; 0 when
    the complement holds no block."""
    N = q.shape[0]
    lo, hi = block_range(a, bs, N)
    if empty:
        return np.zeros((hi - lo, S_U.shape[1]))
    psi, rho = features(q[lo:hi], P_h, theta[lo:hi])
    return (rho @ S_U) / (psi @ z_U)[:, None]


# ---------------------------------------------------------------------------
# whole forward, one (batch, head) at a time
# ---------------------------------------------------------------------------

class HeadResult:
    def __init__(self):
        self.idx = None        # [nb, k_b] int32
        self.sigma = None      # [nb, nb]
        self.S_blk = self.z_blk = self.S = self.z = None
        self.o = {}            # query block -> [rows, d]
        self.o_sp = {}
        self.o_lin = {}


def rola_head(q, k, v, P_h, g_h: float, *, bs: int, k_b: int, grid, rope_base: float,
              idx=None, qblocks=None) -> HeadResult:
    """RoLA forward for one (batch, head).  q, k, v are [N, d] float64, P_h [d, r].
    ``idx`` overrides the selector (to check the attention given a mask);
    ``qblocks`` restricts which query blocks are evaluated."""
    N, d = q.shape
    T, Hg, W = grid
    nb = -(-N // bs)
    res = HeadResult()
    res.sigma = block_scores(pool_blocks(q, bs), pool_blocks(k, bs))
    res.idx = select_topk(res.sigma, k_b) if idx is None else np.asarray(idx, dtype=np.int32)
    theta = rope_angles(N, T, Hg, W, P_h.shape[1], rope_base)
    res.S_blk, res.z_blk, res.S, res.z = block_states(k, v, P_h, theta, bs)
    for a in (range(nb) if qblocks is None else qblocks):
        kept = res.idx[a]
        o_sp = sparse_branch_block(q, k, v, a, kept, bs)
        S_U, z_U = complement_state(res.S_blk, res.z_blk, res.S, res.z, kept)
        o_lin = linear_branch_block(q, P_h, theta, a, bs, S_U, z_U, empty=len(set(kept.tolist())) >= nb)
        res.o_sp[a], res.o_lin[a] = o_sp, o_lin
        res.o[a] = o_sp + g_h * o_lin
    return res


def head_slices(inputs: dict, b: int, h: int):
    """float64 [N, d] views of one (batch, head) of bf16 [B, N, H, d] inputs,
    and the head's projection [d, r]."""
    q = bf16_to_f64(inputs["q"][b, :, h, :])
    k = bf16_to_f64(inputs["k"][b, :, h, :])
    v = bf16_to_f64(inputs["v"][b, :, h, :])
    return q, k, v, bf16_to_f64(inputs["P"][h])


def select_all(inputs: dict, bs: int, k_b: int):
    """Selector over every (batch, head): idx [B, H, nb, k_b] and sigma."""
    B, N, H, d = inputs["q"].shape
    nb = -(-N // bs)
    idx = np.empty((B, H, nb, k_b), dtype=np.int32)
    sig = np.empty((B, H, nb, nb))
    for b in range(B):
        for h in range(H):
            qb = pool_blocks(bf16_to_f64(inputs["q"][b, :, h, :]), bs)
            kb = pool_blocks(bf16_to_f64(inputs["k"][b, :, h, :]), bs)
            sig[b, h] = block_scores(qb, kb)
            idx[b, h] = select_topk(sig[b, h], k_b)
    return idx, sig


def rola_forward(inputs: dict, *, bs: int, k_b: int, grid, rope_base: float = 10000.0,
                 idx=None, heads=None, qblocks=None, kb_per_head=None):
    """RoLA forward over (batch, head) pairs; returns {(b, h): HeadResult}.
    ``kb_per_head`` (length H): head h keeps kb_per_head[h] blocks, and a
    given ``idx`` holds them in the first kb_per_head[h] entries of each row."""
    B, N, H, d = inputs["q"].shape
    out = {}
    for b in range(B):
        for h in (range(H) if heads is None else heads):
            q, k, v, P_h = head_slices(inputs, b, h)
            kh = k_b if kb_per_head is None else int(kb_per_head[h])
            out[(b, h)] = rola_head(q, k, v, P_h, float(inputs["gate"][h]), bs=bs, k_b=kh,
                                    grid=grid, rope_base=rope_base,
                                    idx=None if idx is None else idx[b, h][:, :kh], qblocks=qblocks)
    return out


def select_all_per_head(inputs: dict, bs: int, kb_per_head, k_b_max: int):
    """Selector with a kept count per head (head-adaptive sparsity): head h
    keeps its kb_per_head[h] best blocks per query block; rows have k_b_max
    entries, the unused ones -1.  Returns idx [B, H, nb, k_b_max] and sigma."""
    B, N, H, d = inputs["q"].shape
    nb = -(-N // bs)
    idx = np.full((B, H, nb, k_b_max), -1, dtype=np.int32)
    sig = np.empty((B, H, nb, nb))
    for b in range(B):
        for h in range(H):
            qb = pool_blocks(bf16_to_f64(inputs["q"][b, :, h, :]), bs)
            kb = pool_blocks(bf16_to_f64(inputs["k"][b, :, h, :]), bs)
            sig[b, h] = block_scores(qb, kb)
            kh = int(kb_per_head[h])
            idx[b, h, :, :kh] = select_topk(sig[b, h], kh)
    return idx, sig


def assemble_output(results: dict, B: int, N: int, H: int, d: int, bs: int) -> np.ndarray:
    """Dense [B, N, H, d] float64 output from per-head results (NaN where a
    query block was not evaluated)."""
    o = np.full((B, N, H, d), np.nan)
    for (b, h), res in results.items():
        for a, rows in res.o.items():
            lo, hi = block_range(a, bs, N)
            o[b, lo:hi, h, :] = rows
    return o
