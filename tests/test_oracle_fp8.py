"""Pins for the FP8 E4M3 oracle: hand-derived code values from the OCP FP8
format definition, torch's own float8_e4m3fn casts (an independent library),
rounding-mode and saturation cases, and exactness of the scaled product on
exactly representable operands."""
import os

import numpy as np
import torch

from oracle import fp8_oracle as fo

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def test_decode_golden_values():
    for line in open(os.path.join(GOLD, "e4m3_values.txt")):
        if not line.strip() or line.startswith("#"):
            continue
        code, val = line.split()
        got = fo.e4m3_decode(np.array([int(code, 16)]))[0]
        want = float(val)
        if np.isnan(want):
            assert np.isnan(got)
        else:
            assert got == want and np.signbit(got) == np.signbit(want), (code, got, want)


def test_decode_all_codes_match_torch():
    codes = np.arange(256, dtype=np.uint8)
    tv = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ov = fo.e4m3_decode(codes)
    assert np.array_equal(np.isnan(tv), np.isnan(ov))
    ok = ~np.isnan(tv)
    assert np.array_equal(tv[ok], ov[ok])


def test_encode_roundtrip_all_finite_codes():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    vals = fo.e4m3_decode(codes)
    assert np.array_equal(fo.e4m3_encode(vals), codes)
    assert np.array_equal(fo.e4m3_round(vals), vals)


def test_round_matches_torch_in_range_and_on_midpoints():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(200000) * 60, rng.standard_normal(20000) * 0.01])
    x = np.clip(x, -448, 448)
    pos = np.unique(fo.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8)))
    mids = (pos[:-1] + pos[1:]) / 2             # exact ties -> even mantissa
    x = np.concatenate([x, mids, -mids])
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(fo.e4m3_round(x), want)
    # a tie between 1.0 (m=0) and 1.125 (m=1) goes to 1.0
    assert fo.e4m3_round(np.array([1.0625]))[0] == 1.0
    assert fo.e4m3_round(np.array([1.1875]))[0] == 1.25


def test_saturation_to_448():
    x = np.array([448.0, 463.9, 464.0, 470.0, 1e9, -500.0, -1e30])
    assert fo.e4m3_round(x).tolist() == [448.0, 448.0, 448.0, 448.0, 448.0, -448.0, -448.0]


def test_quantize_rows_scale_and_error_bound():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal((64, 300)) * rng.uniform(0.01, 100, size=(64, 1))).astype(np.float32)
    x[5] = 0.0
    codes, scale = fo.quantize_rows(x)
    assert scale.dtype == np.float32 and scale[5] == 1.0 and np.all(codes[5] == 0)
    deq = fo.e4m3_decode(codes) * scale[:, None].astype(np.float64)
    for m in range(64):
        if m == 5:
            continue
        amax = np.abs(x[m]).max()
        # the row maximum lands on +-448 (times a float32 rounding of the scale)
        assert np.abs(fo.e4m3_decode(codes[m])).max() == 448.0
        assert scale[m] == np.float32(amax) / np.float32(448.0)
        # relative error of normal-range values is at most 2^-4 (+ float32 slack)
        big = np.abs(x[m]) >= amax * 2.0 ** -6 / 448.0 * 2
        rel = np.abs(deq[m][big] - x[m][big]) / np.abs(x[m][big])
        assert rel.max() <= 2.0 ** -4 + 1e-6


def test_gemm_exact_on_representable_operands():
    rng = np.random.default_rng(2)
    vals = fo.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8))
    a = rng.choice(vals, size=(16, 32)) * rng.choice([-1, 1], size=(16, 32))
    b = rng.choice(vals, size=(8, 32)) * rng.choice([-1, 1], size=(8, 32))
    a[:, 0] = 448.0
    b[:, 0] = 448.0                       # amax = 448 -> scale 1, codes exact
    qa, sa = fo.quantize_rows(a.astype(np.float32))
    qb, sb = fo.quantize_rows(b.astype(np.float32))
    assert np.all(sa == 1.0) and np.all(sb == 1.0)
    np.testing.assert_array_equal(fo.gemm_w8a8(qa, sa, qb, sb), a @ b.T)


def test_round_bf16_matches_torch():
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.standard_normal(100000) * 10.0 ** rng.integers(-6, 6, 100000),
                        [0.0, -0.0, 1.0, 1.00390625, 1.005859375, 3.0e38]])
    want = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(fo.round_bf16(x.astype(np.float32).astype(np.float64)), want)
    # ties between bf16 neighbours go to the even mantissa
    assert fo.round_bf16(np.array([1.00390625]))[0] == 1.0          # 1 + 2^-8: tie, 1.0 is even
    assert fo.round_bf16(np.array([1.01171875]))[0] == 1.015625     # 1 + 3*2^-8: tie, up to even


def test_gelu_tanh_matches_torch_and_limits():
    u = np.linspace(-12.0, 12.0, 4001)
    want = torch.nn.functional.gelu(torch.from_numpy(u), approximate="tanh").numpy()
    np.testing.assert_allclose(fo.gelu_tanh(u), want, rtol=1e-13, atol=1e-15)
    assert fo.gelu_tanh(np.array([0.0]))[0] == 0.0
    big = np.array([30.0, -30.0])
    np.testing.assert_allclose(fo.gelu_tanh(big), [30.0, 0.0], atol=1e-300)
    # GELU is not odd: gelu(u) - gelu(-u) = u
    np.testing.assert_allclose(fo.gelu_tanh(u) - fo.gelu_tanh(-u), u, atol=1e-12)


def test_ffn_matches_an_independent_library_chain():
    """The FFN composition against the same steps taken with torch's own
    float8_e4m3fn casts, float64 matmuls, GELU and bfloat16 rounding: a wrong
    step order (GELU after the bf16 rounding, a missing scale, the scales of
    the wrong operand) fails it."""
    rng = np.random.default_rng(4)
    M, D, F = 24, 64, 96
    x = (rng.standard_normal((M, D)) * 2).astype(np.float32)
    W1 = (rng.standard_normal((F, D)) / 8).astype(np.float32)
    W2 = (rng.standard_normal((D, F)) / 10).astype(np.float32)
    c1, s1 = fo.quantize_rows(W1)
    c2, s2 = fo.quantize_rows(W2)
    h, y = fo.ffn_w8a8(x, c1, s1, c2, s2)

    def tq(a):  # torch: per-row E4M3 quantisation, reciprocal and product in float32
        a = torch.from_numpy(a)
        amax = a.abs().amax(dim=1)
        inv = (448.0 / amax).to(torch.float32)
        q = (a * inv[:, None]).to(torch.float8_e4m3fn).to(torch.float64)
        return q, (amax / 448.0).to(torch.float64)

    qx, sx = tq(x)
    qw1, sw1 = tq(W1)
    qw2, sw2 = tq(W2)
    hid = (qx @ qw1.T) * sx[:, None] * sw1[None, :]
    ht = torch.nn.functional.gelu(hid, approximate="tanh").to(torch.bfloat16)
    qh, sh = tq(ht.to(torch.float32).numpy())
    yt = (qh @ qw2.T) * sh[:, None] * sw2[None, :]
    np.testing.assert_array_equal(h, ht.to(torch.float64).numpy())
    np.testing.assert_allclose(y, yt.numpy(), rtol=1e-12, atol=1e-12)
