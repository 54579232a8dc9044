"""CPU oracle for the W8A8 FP8 E4M3 projections.

TEST INFRASTRUCTURE ONLY (same rule as ``rola_oracle``): used by ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU legs, never by the product
path, and sharing no code with the CUDA library.

The SparkDiffusion write-up (「首次定义“高稀疏陷阱”」, 0539edu.com news page,
section 07 "From algorithmic subtraction to real GPU speed-up") quantises the
linear projections of attention and FFN to W8A8 FP8 E4M3 and fuses the
activation scaling and type conversion into the kernels.  The pages fix no
scaling granularity; this library takes per-output-channel weight scales and
per-token dynamic activation scales:

* ``s[m] = amax_m / 448`` (1 when the row is all zero);
* ``q[m, k] = E4M3(x[m, k] * (448 / amax_m))`` with the reciprocal and the
  product each rounded to float32 -- the quantised code is an integer decided
  by floating point, so both sides make that decision in float32;
* ``y[m, n] = (sum_k dec(q_x[m, k]) dec(q_w[n, k])) * s_x[m] * s_w[n]``, in float64.

The FFN of the transformer block (the write-up's "FFN projections", section 07)
is ``y = W2 gelu(W1 x)`` with both projections in W8A8.  The pages fix neither
the hidden width nor the activation; this library takes the tanh form of GELU
and, for the 14B model, a hidden width of 13824 (see ``ffn_w8a8``).  The hidden
activation is stored in bf16 between the two projections, as a GPU
implementation keeps it.

The E4M3 codec follows the OCP 8-bit floating point specification (OFP8):
1 sign, 4 exponent (bias 7) and 3 mantissa bits; exponent field 0 is
subnormal (m/8 * 2^-6); S.1111.111 is NaN; there is no infinity; the largest
finite magnitude is 1.75 * 2^8 = 448.  Conversion rounds to nearest, ties to
even, and saturates to +-448 (the "satfinite" mode).
"""
from __future__ import annotations

import math

import numpy as np

E4M3_MAX = 448.0


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """Value of each E4M3 byte, float64 (NaN for the two NaN codes)."""
    c = np.asarray(codes).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    mag = np.where((e == 15) & ((c & 7) == 7), np.nan, mag)
    return sign * mag


def e4m3_round(x: np.ndarray) -> np.ndarray:
    """Nearest E4M3 value (ties to even mantissa), saturated to +-448; float64."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    _, ex = np.frexp(a)                     # a = f * 2^ex, f in [0.5, 1)
    e = np.clip(ex - 1, -6, 8)              # binade exponent, subnormals share -6
    quantum = np.exp2(e.astype(np.float64) - 3.0)
    r = np.rint(a / quantum) * quantum      # np.rint rounds half to even
    r = np.minimum(r, E4M3_MAX)
    return np.copysign(r, x)


def e4m3_encode(v: np.ndarray) -> np.ndarray:
    """Byte of an exactly representable E4M3 value (as produced by e4m3_round)."""
    v = np.asarray(v, dtype=np.float64)
    sign = (np.signbit(v)).astype(np.int64) << 7
    a = np.abs(v)
    _, ex = np.frexp(a)
    e = ex - 1
    normal = a >= 2.0 ** -6
    efield = np.where(normal, e + 7, 0)
    mant = np.where(normal, a / np.exp2(e.astype(np.float64)) - 1.0, a / 2.0 ** -6) * 8.0
    code = sign | (efield.astype(np.int64) << 3) | np.rint(mant).astype(np.int64)
    return np.where(a == 0, sign, code).astype(np.uint8)


def quantize_rows(x: np.ndarray):
    """Per-row (per-token or per-output-channel) E4M3 quantisation of a float32
    matrix [M, K]: returns (codes uint8 [M, K], scale float32 [M])."""
    x = np.asarray(x, dtype=np.float32)
    amax = np.abs(x).max(axis=1)
    nz = amax > 0
    safe = np.where(nz, amax, np.float32(1.0)).astype(np.float32)
    scale = np.where(nz, safe / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    inv = (np.float32(E4M3_MAX) / safe).astype(np.float32)
    xs = (x * inv[:, None]).astype(np.float32)       # one float32 rounding
    codes = e4m3_encode(e4m3_round(xs.astype(np.float64)))
    return codes, scale


def gemm_w8a8(x_codes, x_scale, w_codes, w_scale) -> np.ndarray:
    """y = (dec(x_q) dec(w_q)^T) * s_x[:, None] * s_w[None, :], float64."""
    a = e4m3_decode(x_codes)
    b = e4m3_decode(w_codes)
    return (a @ b.T) * np.asarray(x_scale, np.float64)[:, None] * np.asarray(w_scale, np.float64)[None, :]


def linear_w8a8(x_f32: np.ndarray, w_codes, w_scale) -> np.ndarray:
    """Activation quantisation followed by the scaled FP8 product."""
    xq, sx = quantize_rows(x_f32)
    return gemm_w8a8(xq, sx, w_codes, w_scale)


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Nearest bfloat16 value (ties to even) of float64 values, as float64:
    first to float32 (nearest), then the 16 low bits of the float32 pattern
    rounded away to nearest even.  Finite inputs."""
    u = np.ascontiguousarray(np.asarray(x, dtype=np.float64).astype(np.float32)).view(np.uint32)
    u = u.astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return r.astype(np.uint32).view(np.float32).astype(np.float64)


def gelu_tanh(u: np.ndarray) -> np.ndarray:
    """GELU in its tanh form: 0.5 u (1 + tanh(sqrt(2/pi) (u + 0.044715 u^3)))."""
    u = np.asarray(u, dtype=np.float64)
    return 0.5 * u * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (u + 0.044715 * u ** 3)))


def ffn_w8a8(x_f32: np.ndarray, w1_codes, w1_scale, w2_codes, w2_scale):
    """The block's FFN with both projections in W8A8, in the order the method
    applies the steps: per-token quantisation of x, the up projection
    (hidden = W1 x), GELU, the hidden activation stored as bf16, per-token
    quantisation of that activation, the down projection.  Returns
    (h, y): h the bf16 hidden activation [M, F] as float64, y [M, D] float64."""
    hidden = linear_w8a8(x_f32, w1_codes, w1_scale)
    h = round_bf16(gelu_tanh(hidden))
    y = linear_w8a8(h.astype(np.float32), w2_codes, w2_scale)
    return h, y
