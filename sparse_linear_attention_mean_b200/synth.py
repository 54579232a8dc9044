"""Seeded synthetic inputs for RoLA hybrid attention on Wan-DiT attention shapes.

This module only draws numbers: it holds none of the attention arithmetic, so
both the fp64 oracle (under ``oracle/``) and the CUDA path consume exactly the
bytes produced here.  Everything is NumPy (PCG64 via ``default_rng``) and
deterministic in the workload id and seed.

Shapes follow the SparkDiffusion write-up (0539edu.com news page, section 07,
Figure 7 caption: 81 frames, 480P = 480x832, 720P = 720x1280) mapped onto the
Wan latent grid (21 frames x 30x52 or 45x80 patches); sparsity settings follow
the SparkDiffusion project blog, "Results" (97 % at 720P, 90 % for the 1.3B
480P model).

Input recipe (the pages give none, so this is a stated choice):

* A smooth positional field per (head, channel):
  ``F(t,y,x) = sum_{m<8} a_m sin(2 pi (f_t t/T + f_y y/Hg + f_x x/W) + phi_m)``
  with ``a_m ~ N(0, 0.25)``, ``f_t ~ U{0,1,2}``, ``f_y, f_x ~ U{0..3}``,
  ``phi_m ~ U(0, 2 pi)``.  The same F enters q and k, which gives the
  positional locality that block selection exploits in video DiTs.
* ``q = F + 0.5 eps_q``, ``k = F + 0.5 eps_k``, ``v = eps_v`` with
  ``eps ~ N(0, 1)`` (drawn as float32, added in float64).
* Projections ``P ~ N(0, 1/d)`` of shape ``[H, d, r]``; gate ``g_h``: 0.5 for
  the tiny workload, ``U(0.2, 1)`` per head otherwise.
* Everything is rounded float64 -> float32 -> bfloat16 (round to nearest even).
* The full-block workload adds ``x ~ N(0, 1)`` ``[N, 5120]`` and four
  ``5120 x 5120`` float32 weights ``~ N(0, 1/5120)``; its FFN weights are
  ``W1 [13824, 5120] ~ N(0, 1/5120)`` and ``W2 [5120, 13824] ~ N(0, 1/13824)``.

Tokens are in frame-major raster order: token ``n`` sits at
``t = n // (Hg*W)``, ``y = (n // W) % Hg``, ``x = n % W``.
"""
from __future__ import annotations

import dataclasses
import math
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_CHUNK = 2048  # tokens per independently seeded noise chunk

# stream ids (entropy words) -- one independent PCG64 stream per draw kind
_S_FIELD, _S_PROJ, _S_GATE = 1, 2, 3
_S_NOISE = {"q": 10, "k": 11, "v": 12}
_S_X, _S_WQKV, _S_WO = 20, 21, 22
_S_W1, _S_W2 = 23, 24

# FFN hidden width of the 14B model (the pages give none; the Wan2.1-14B
# transformer's feed-forward width is taken as the stated reading)
FFN_HIDDEN_14B = 13824


@dataclasses.dataclass(frozen=True)
class Workload:
    """One attention workload.  ``k_b`` is listed explicitly (the value the
    integer ceiling of ``(1000 - sparsity_permille) * n_blocks / 1000`` gives);
    tests check both implementations of that rule against it."""

    name: str
    B: int
    H: int
    d: int
    T: int
    Hg: int
    W: int
    block: int
    sparsity_permille: int
    k_b: int
    r: int
    seed: int
    gate_const: float | None = None  # None -> U(0.2, 1) per head
    rope_base: float = 10000.0
    full_block: bool = False  # wrap the attention in W8A8 FP8 projections
    model_dim: int = 0

    @property
    def N(self) -> int:
        return self.T * self.Hg * self.W

    @property
    def n_blocks(self) -> int:
        return -(-self.N // self.block)

    def sparse_flops(self) -> float:
        """FLOPs of the kept query-key block pairs (QK^T and PV), counting a
        full block x block tile per kept pair, including the padded tail."""
        pairs = self.B * self.H * self.n_blocks * self.k_b
        return 4.0 * self.block * self.block * self.d * pairs


WORKLOADS = {
    0: Workload("tiny-4x16x16", 1, 2, 64, 4, 16, 16, 64, 750, 4, 16, 0, gate_const=0.5),
    1: Workload("wan1.3b-480p-s90", 1, 12, 128, 21, 30, 52, 128, 900, 26, 32, 1),
    2: Workload("wan14b-480p-s97", 1, 40, 128, 21, 30, 52, 128, 970, 8, 32, 2),
    3: Workload("wan14b-720p-s97", 1, 40, 128, 21, 45, 80, 128, 970, 18, 32, 3),
    4: Workload("wan14b-720p-s97-fp8block", 1, 40, 128, 21, 45, 80, 128, 970, 18, 32, 4,
                full_block=True, model_dim=5120),
}


def custom_workload(base: Workload, **kw) -> Workload:
    return dataclasses.replace(base, **kw)


# --------------------------------------------------------------------------
# bf16 helpers (storage only)
# --------------------------------------------------------------------------

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest, ties to even); returns uint16 bits.
    Inputs here are finite."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> 16) & 1
    return ((u + np.uint32(0x7FFF) + lsb) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32)


def _rng(*words: int) -> np.random.Generator:
    return np.random.default_rng([int(w) for w in words])


# --------------------------------------------------------------------------
# positional field
# --------------------------------------------------------------------------

def _field_coefficients(w: Workload):
    """Coefficients of F in the separable sin/cos basis over the 48 possible
    integer frequency triples (f_t, f_y, f_x)."""
    g = _rng(w.seed, _S_FIELD)
    C = w.H * w.d
    a = g.normal(0.0, 0.5, size=(C, 8))
    ft = g.integers(0, 3, size=(C, 8))
    fy = g.integers(0, 4, size=(C, 8))
    fx = g.integers(0, 4, size=(C, 8))
    ph = g.uniform(0.0, 2.0 * math.pi, size=(C, 8))
    combo = (ft * 4 + fy) * 4 + fx  # 0..47
    coef = np.zeros((96, C), dtype=np.float64)
    cols = np.broadcast_to(np.arange(C)[:, None], combo.shape)
    # sin(theta + phi) = sin(theta) cos(phi) + cos(theta) sin(phi)
    np.add.at(coef, (2 * combo, cols), a * np.cos(ph))
    np.add.at(coef, (2 * combo + 1, cols), a * np.sin(ph))
    return coef


def _field_basis(w: Workload, n0: int, n1: int) -> np.ndarray:
    n = np.arange(n0, n1, dtype=np.int64)
    t = n // (w.Hg * w.W)
    y = (n // w.W) % w.Hg
    x = n % w.W
    basis = np.empty((n1 - n0, 96), dtype=np.float64)
    for ft in range(3):
        for fy in range(4):
            for fx in range(4):
                c = (ft * 4 + fy) * 4 + fx
                th = 2.0 * math.pi * (ft * t / w.T + fy * y / w.Hg + fx * x / w.W)
                basis[:, 2 * c] = np.sin(th)
                basis[:, 2 * c + 1] = np.cos(th)
    return basis


def _noise(w: Workload, stream: int, chunk: int, rows: int, cols: int) -> np.ndarray:
    return _rng(w.seed, stream, chunk).standard_normal((rows, cols), dtype=np.float32)


def _chunks(N: int):
    for c, n0 in enumerate(range(0, N, _CHUNK)):
        yield c, n0, min(N, n0 + _CHUNK)


def make_qkv(w: Workload, threads: int = 8):
    """Structured q, k and plain v as bf16 bit arrays of shape [B, N, H, d].
    The batch index is folded into the noise streams (b * 1_000_000 + chunk)."""
    coef = _field_coefficients(w)
    C = w.H * w.d
    out = {nm: np.empty((w.B, w.N, C), dtype=np.uint16) for nm in ("q", "k", "v")}

    def work(job):
        b, c, n0, n1 = job
        F = _field_basis(w, n0, n1) @ coef
        for nm in ("q", "k"):
            e = _noise(w, _S_NOISE[nm], b * 1_000_000 + c, n1 - n0, C)
            out[nm][b, n0:n1] = f32_to_bf16_bits((F + 0.5 * e.astype(np.float64)).astype(np.float32))
        e = _noise(w, _S_NOISE["v"], b * 1_000_000 + c, n1 - n0, C)
        out["v"][b, n0:n1] = f32_to_bf16_bits(e)

    jobs = [(b, c, n0, n1) for b in range(w.B) for c, n0, n1 in _chunks(w.N)]
    with ThreadPoolExecutor(max_workers=max(1, threads)) as ex:
        list(ex.map(work, jobs))
    return tuple(out[nm].reshape(w.B, w.N, w.H, w.d) for nm in ("q", "k", "v"))


def make_projection(w: Workload) -> np.ndarray:
    """P ~ N(0, 1/d), shape [H, d, r], bf16 bits."""
    g = _rng(w.seed, _S_PROJ)
    P = g.normal(0.0, 1.0 / math.sqrt(w.d), size=(w.H, w.d, w.r))
    return f32_to_bf16_bits(P.astype(np.float32))


def make_gate(w: Workload) -> np.ndarray:
    if w.gate_const is not None:
        return np.full(w.H, w.gate_const, dtype=np.float32)
    g = _rng(w.seed, _S_GATE)
    return g.uniform(0.2, 1.0, size=w.H).astype(np.float32)


def make_inputs(w: Workload, threads: int = 8) -> dict:
    """All attention inputs of a workload (bf16 as uint16 bits, gate float32)."""
    q, k, v = make_qkv(w, threads)
    return {"q": q, "k": k, "v": v, "P": make_projection(w), "gate": make_gate(w)}


def make_block_inputs(w: Workload, threads: int = 8) -> dict:
    """Inputs of the full attention block: activations x [B*N, D] (bf16 bits)
    and float32 weights W_q, W_k, W_v, W_o [D, D] (out x in)."""
    D = w.model_dim
    M = w.B * w.N
    x = np.empty((M, D), dtype=np.uint16)

    def work(job):
        c, n0, n1 = job
        x[n0:n1] = f32_to_bf16_bits(_noise(w, _S_X, c, n1 - n0, D))

    with ThreadPoolExecutor(max_workers=max(1, threads)) as ex:
        list(ex.map(work, list(_chunks(M))))
    g = _rng(w.seed, _S_WQKV)
    sd = 1.0 / math.sqrt(D)
    Wqkv = (g.standard_normal((3 * D, D), dtype=np.float32) * np.float32(sd))
    Wo = (_rng(w.seed, _S_WO).standard_normal((D, D), dtype=np.float32) * np.float32(sd))
    return {"x": x, "Wq": Wqkv[:D], "Wk": Wqkv[D:2 * D], "Wv": Wqkv[2 * D:], "Wo": Wo,
            "P": make_projection(w), "gate": make_gate(w)}


def make_ffn_weights(w: Workload, hidden: int = FFN_HIDDEN_14B) -> dict:
    """float32 FFN weights of the full block: W1 [hidden, D] ~ N(0, 1/D) (up
    projection) and W2 [D, hidden] ~ N(0, 1/hidden) (down projection)."""
    D = w.model_dim
    W1 = _rng(w.seed, _S_W1).standard_normal((hidden, D), dtype=np.float32) * np.float32(1.0 / math.sqrt(D))
    W2 = _rng(w.seed, _S_W2).standard_normal((D, hidden), dtype=np.float32) * np.float32(1.0 / math.sqrt(hidden))
    return {"W1": W1, "W2": W2}


def make_uniform(shape, seed: int, lo: float, hi: float) -> np.ndarray:
    """Plain uniform float32 draws for ad-hoc test inputs."""
    return _rng(seed, 99).uniform(lo, hi, size=shape).astype(np.float32)


def make_normal_bf16(shape, seed: int, stream: int, mean: float = 0.0, std: float = 1.0) -> np.ndarray:
    """Plain normal bf16 bits for ad-hoc test inputs."""
    e = _rng(seed, 100 + stream).standard_normal(shape, dtype=np.float32)
    return f32_to_bf16_bits((e.astype(np.float64) * std + mean).astype(np.float32))
