"""GPU parity of the W8A8 FP8 E4M3 projections against the oracle, through the
C ABI (SparkDiffusion write-up, section 07).

* quantisation: E4M3 codes and float32 scales bit-exact (the oracle rounds
  the reciprocal and the product to float32 as the kernel does);
* GEMM: relative Frobenius error <= 1e-2 against the oracle's float64 product
  of the same codes; per element within 1e-2 |ref| plus 1e-3 of the row's
  largest magnitude (bf16 output rounding, fp32 accumulation order).
"""
import numpy as np
import pytest
import torch

from oracle import fp8_oracle as fo
from sparse_linear_attention_mean_b200 import binding as rb
from sparse_linear_attention_mean_b200 import synth

pytestmark = pytest.mark.gpu

FROB = 1e-2


def _bf16_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits)).view(torch.bfloat16).cuda()


def _bf16_f32(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32)


def _check_gemm(y_dev, ref, what):
    y = y_dev.float().cpu().numpy().astype(np.float64)
    fro = np.linalg.norm(y - ref) / max(np.linalg.norm(ref), 1e-300)
    assert fro <= FROB, f"{what}: relative Frobenius {fro:.3g}"
    bound = 1e-2 * np.abs(ref) + 1e-3 * np.abs(ref).max(axis=1, keepdims=True)
    bad = np.abs(y - ref) > bound
    assert not bad.any(), f"{what}: {int(bad.sum())} elements out of tolerance"
    return fro


@pytest.mark.parametrize("M,K", [(1, 16), (37, 80), (256, 5120), (300, 1040)])
def test_quantize_rows_bitexact(M, K):
    bits = synth.make_normal_bf16((M, K), seed=M * 7 + K, stream=1, std=3.0)
    if M > 2:
        bits[2] = 0          # an all-zero row takes scale 1
        bits[1, 5] = 0x4380  # 256.0: a large outlier in one row
    xq, xs = rb.fp8_quantize_rows(_bf16_dev(bits))
    codes, scale = fo.quantize_rows(_bf16_f32(bits))
    torch.cuda.synchronize()
    assert np.array_equal(xq.cpu().numpy(), codes)
    assert np.array_equal(xs.cpu().numpy(), scale)


@pytest.mark.parametrize("N,K", [(96, 48), (512, 5120)])
def test_quantize_weight_bitexact(N, K):
    w = (synth.make_normal_bf16((N, K), seed=N + K, stream=2).astype(np.uint32) << 16).view(np.float32)
    w = np.ascontiguousarray(w * np.float32(0.013))
    wq, ws = rb.fp8_quantize_weight(torch.from_numpy(w).cuda())
    codes, scale = fo.quantize_rows(w)
    torch.cuda.synchronize()
    assert np.array_equal(wq.cpu().numpy(), codes)
    assert np.array_equal(ws.cpu().numpy(), scale)


def _random_codes(shape, seed):
    """Finite E4M3 codes (0x7f / 0xff are NaN and never produced by the cast)."""
    g = np.random.default_rng(seed)
    c = g.integers(0, 256, size=shape, dtype=np.uint8)
    return np.where((c & 0x7f) == 0x7f, c ^ 0x01, c).astype(np.uint8)


@pytest.mark.parametrize("M,N,K", [
    (1, 32, 16),        # single row, one 32-column chunk, K inside one slice
    (200, 96, 80),      # ragged M tile, partial N tile, K tail
    (128, 256, 128),    # exactly one tile
    (1000, 768, 1024),  # several tiles in both directions, several K slices
    (333, 544, 2064),   # ragged everything, more tiles than one pass of the CTAs
])
def test_gemm_small(M, N, K):
    xq = _random_codes((M, K), 11 + M)
    wq = _random_codes((N, K), 13 + N)
    g = np.random.default_rng(M + N + K)
    xs = g.uniform(0.001, 0.02, size=M).astype(np.float32)
    ws = g.uniform(0.001, 0.02, size=N).astype(np.float32)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = rb.fp8_gemm(torch.from_numpy(xq).cuda(), torch.from_numpy(xs).cuda(),
                    torch.from_numpy(wq).cuda(), torch.from_numpy(ws).cuda(), dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    _check_gemm(y, fo.gemm_w8a8(xq, xs, wq, ws), f"gemm {M}x{N}x{K}")


@pytest.mark.parametrize("M,N,K", [(200, 96, 80), (333, 544, 2064), (1000, 768, 1024)])
def test_gemm_gelu_small(M, N, K):
    """The GELU epilogue (the FFN's up projection): y = bf16(gelu(product))."""
    xq = _random_codes((M, K), 21 + M)
    wq = _random_codes((N, K), 23 + N)
    g = np.random.default_rng(M * N + K)
    # scales that put the products in GELU's curved range (|u| up to ~6)
    ones_m, ones_n = np.ones(M, np.float32), np.ones(N, np.float32)
    raw = np.abs(fo.gemm_w8a8(xq, ones_m, wq, ones_n)).max(axis=1)
    xs = (6.0 / np.maximum(raw, 1.0) * g.uniform(0.3, 1.0, size=M)).astype(np.float32)
    ws = g.uniform(0.5, 1.0, size=N).astype(np.float32)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = rb.fp8_gemm(torch.from_numpy(xq).cuda(), torch.from_numpy(xs).cuda(), torch.from_numpy(wq).cuda(),
                    torch.from_numpy(ws).cuda(), dev_err=err, act=rb.ACT_GELU_TANH)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    prod = fo.gemm_w8a8(xq, xs, wq, ws)
    assert np.abs(prod).max() > 2.0 and (prod < -0.5).mean() > 0.02
    _check_gemm(y, fo.gelu_tanh(prod), f"gemm+gelu {M}x{N}x{K}")


def test_gemm_rejects_bad_shapes():
    xq = torch.zeros((4, 64), dtype=torch.uint8, device="cuda")
    xs = torch.ones(4, device="cuda")
    for N, K in ((40, 64), (64, 24)):  # N % 32, K % 16
        wq = torch.zeros((N, K), dtype=torch.uint8, device="cuda")
        with pytest.raises(rb.RolaError):
            rb.fp8_gemm(torch.zeros((4, K), dtype=torch.uint8, device="cuda"), xs, wq,
                        torch.ones(N, device="cuda"))


_BLOCK = {}


def _block_inputs():
    if not _BLOCK:
        w = synth.WORKLOADS[4]
        _BLOCK["w"] = w
        _BLOCK["inp"] = synth.make_block_inputs(w)
    return _BLOCK["w"], _BLOCK["inp"]


def test_linear_full_size_sampled():
    """Full 14B-720P projection (x [75600, 5120] -> [75600, 5120]) in the
    launch configuration the benchmark times; the oracle checks sampled rows,
    including the ragged last tile, against every output column."""
    w, inp = _block_inputs()
    D = w.model_dim
    x = _bf16_dev(inp["x"])
    Wq = np.ascontiguousarray(inp["Wq"])
    wq, ws = rb.fp8_quantize_weight(torch.from_numpy(Wq).cuda())
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = rb.fp8_linear(x, wq, ws, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    M = x.shape[0]
    rows = np.unique(np.concatenate([np.arange(0, 8), np.arange(M - 80, M, 9), [M - 1],
                                     np.random.default_rng(5).integers(0, M, 24)]))
    xs_codes, xs_scale = fo.quantize_rows(_bf16_f32(inp["x"][rows]))
    w_codes, w_scale = fo.quantize_rows(Wq)
    assert np.array_equal(wq.cpu().numpy(), w_codes)
    ref = fo.gemm_w8a8(xs_codes, xs_scale, w_codes, w_scale)
    _check_gemm(y[torch.from_numpy(rows).cuda()], ref, "linear 75600x5120x5120")
    # the fused call equals quantisation followed by the GEMM
    xq, xsc = rb.fp8_quantize_rows(x)
    y2 = rb.fp8_gemm(xq, xsc, wq, ws)
    torch.cuda.synchronize()
    assert torch.equal(y, y2)
    assert D == 5120


def _oracle_head_projections(x_bits, Ws, heads, d, chunk=4096):
    """The oracle's W8A8 projections of x by each weight of `Ws`, restricted to
    the output columns of `heads` and rounded to bf16 as the projections'
    outputs are; a list of uint16 bit arrays [M, len(heads), d]."""
    cols = np.concatenate([np.arange(h * d, (h + 1) * d) for h in heads])
    wd, wsc = [], []
    for W in Ws:
        w_codes, w_scale = fo.quantize_rows(np.ascontiguousarray(W))
        wd.append(fo.e4m3_decode(w_codes[cols]))
        wsc.append(w_scale[cols].astype(np.float64))
    wd, wsc = np.concatenate(wd), np.concatenate(wsc)
    out = np.empty((x_bits.shape[0], wd.shape[0]), dtype=np.float64)

    def rows(m0):
        xc, xs = fo.quantize_rows(_bf16_f32(x_bits[m0:m0 + chunk]))
        out[m0:m0 + chunk] = (fo.e4m3_decode(xc) @ wd.T) * xs[:, None].astype(np.float64) * wsc[None, :]

    from concurrent.futures import ThreadPoolExecutor
    with ThreadPoolExecutor(max_workers=8) as ex:
        list(ex.map(rows, range(0, x_bits.shape[0], chunk)))
    bits = synth.f32_to_bf16_bits(out.astype(np.float32))
    n = len(cols)
    return [bits[:, i * n:(i + 1) * n].reshape(x_bits.shape[0], len(heads), d).copy()
            for i in range(len(Ws))]


def test_attention_block_chain():
    """The full 14B-720P attention block: FP8 QKV projections -> RoLA layer ->
    FP8 output projection, all on the GPU.  The oracle runs the same chain for
    two heads from x on its own (projection of those heads' columns, mask,
    attention at sampled query blocks, given the oracle's mask)."""
    from oracle import rola_oracle as ro
    from helpers import check_close, mask_mismatch
    w, inp = _block_inputs()
    D, H, d = w.model_dim, w.H, w.d
    shape = rb.Shape.of(w)
    x = _bf16_dev(inp["x"])
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    proj = {}
    for nm in ("Wq", "Wk", "Wv"):
        wq, ws = rb.fp8_quantize_weight(torch.from_numpy(np.ascontiguousarray(inp[nm])).cuda())
        proj[nm] = rb.fp8_linear(x, wq, ws, dev_err=err).view(w.B, w.N, H, d)
    P = torch.from_numpy(np.ascontiguousarray(inp["P"])).view(torch.bfloat16).cuda()
    gate = torch.from_numpy(inp["gate"]).cuda()
    q, k, v = proj["Wq"], proj["Wk"], proj["Wv"]
    idx_gpu = rb.select_blocks(shape, q, k)
    heads = [0, H - 1]
    oq, ok_, ov = _oracle_head_projections(inp["x"], [inp["Wq"], inp["Wk"], inp["Wv"]], heads, d)
    sub = {"q": oq[None], "k": ok_[None], "v": ov[None],
           "P": np.ascontiguousarray(inp["P"][heads]), "gate": inp["gate"][heads]}
    idx_ref, sig = ro.select_all(sub, w.block, w.k_b)
    torch.cuda.synchronize()
    # the GPU's own mask from its own projections: near-tie rows may differ
    ties, bad = mask_mismatch(idx_gpu[:, heads].cpu().numpy(), idx_ref, sig, w.k_b)
    assert not bad, f"mask rows differ outside near-ties: {bad[:5]}"
    # attention given the oracle's mask for the checked heads
    idx_full = idx_gpu.clone()
    idx_full[:, heads] = torch.from_numpy(idx_ref).cuda()
    states = rb.block_states(shape, k, v, P)
    o = rb.attention_fwd(shape, q, k, v, idx_full, P, states, gate, dev_err=err)
    nb = w.n_blocks
    qblocks = [0, nb // 2, nb - 1]
    res = ro.rola_forward(sub, bs=w.block, k_b=w.k_b, grid=(w.T, w.Hg, w.W), rope_base=w.rope_base,
                          idx=idx_ref, qblocks=qblocks)
    wo_q, wo_s = rb.fp8_quantize_weight(torch.from_numpy(np.ascontiguousarray(inp["Wo"])).cuda())
    y = rb.fp8_linear(o.view(w.B * w.N, D), wo_q, wo_s, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    o64 = o.float().cpu().numpy().astype(np.float64)
    for (b, j), r in res.items():
        for a, rows in r.o.items():
            lo, hi = ro.block_range(a, w.block, w.N)
            check_close(o64[b, lo:hi, heads[j], :], rows, what=f"head {heads[j]} block {a}")
    # the output projection on sampled rows: the oracle's W8A8 product of the
    # GPU's attention output (its own quantisation of those rows and of W_o)
    M = w.B * w.N
    rows = np.unique(np.concatenate([np.arange(0, 4), np.arange(M - 80, M, 19), [M - 1],
                                     np.random.default_rng(8).integers(0, M, 24)]))
    o_rows = o.view(M, D)[torch.from_numpy(rows).cuda()].float().cpu().numpy()
    w_codes, w_scale = fo.quantize_rows(np.ascontiguousarray(inp["Wo"]))
    assert np.array_equal(wo_q.cpu().numpy(), w_codes)
    ref_y = fo.linear_w8a8(o_rows, w_codes, w_scale)
    _check_gemm(y[torch.from_numpy(rows).cuda()], ref_y, "output projection 75600x5120x5120")


def test_ffn_full_size_sampled():
    """The full 14B-720P FFN in W8A8 (x [75600, 5120] -> GELU(x W1^T) [75600,
    13824] -> [75600, 5120]), the benchmark's launch configuration.  The fused
    entry equals the step-by-step chain bit for bit; on sampled rows the hidden
    activation matches the oracle's GELU of the W8A8 product, and the output
    matches the oracle's W8A8 product of the GPU's hidden activation (its own
    quantisation of those rows)."""
    w, inp = _block_inputs()
    ffw = synth.make_ffn_weights(w)
    M, D, F = w.B * w.N, w.model_dim, ffw["W1"].shape[0]
    x = _bf16_dev(inp["x"])
    w1q, w1s = rb.fp8_quantize_weight(torch.from_numpy(ffw["W1"]).cuda())
    w2q, w2s = rb.fp8_quantize_weight(torch.from_numpy(ffw["W2"]).cuda())
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = rb.fp8_ffn(x, w1q, w1s, w2q, w2s, dev_err=err)
    xq, xsc = rb.fp8_quantize_rows(x)
    h = rb.fp8_gemm(xq, xsc, w1q, w1s, dev_err=err, act=rb.ACT_GELU_TANH)
    hq, hsc = rb.fp8_quantize_rows(h)
    y2 = rb.fp8_gemm(hq, hsc, w2q, w2s, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert torch.equal(y, y2)
    rows = np.unique(np.concatenate([np.arange(0, 4), np.arange(M - 80, M, 19), [M - 1],
                                     np.random.default_rng(9).integers(0, M, 24)]))
    rows_d = torch.from_numpy(rows).cuda()
    w1_codes, w1_scale = fo.quantize_rows(ffw["W1"])
    w2_codes, w2_scale = fo.quantize_rows(ffw["W2"])
    assert np.array_equal(w1q.cpu().numpy(), w1_codes) and np.array_equal(w2q.cpu().numpy(), w2_codes)
    x_codes, x_scale = fo.quantize_rows(_bf16_f32(inp["x"][rows]))
    h_ref = fo.gelu_tanh(fo.gemm_w8a8(x_codes, x_scale, w1_codes, w1_scale))
    _check_gemm(h[rows_d], h_ref, "FFN up projection + GELU 75600x13824x5120")
    h_rows = h[rows_d].float().cpu().numpy()
    y_ref = fo.linear_w8a8(h_rows, w2_codes, w2_scale)
    _check_gemm(y[rows_d], y_ref, "FFN down projection 75600x5120x13824")


def test_ffn_small_matches_oracle_chain():
    """A small ragged FFN through the fused entry against the oracle's whole
    chain (its own quantisation, GELU and bf16 hidden activation)."""
    g = np.random.default_rng(12)
    M, D, F = 300, 256, 608
    x_bits = synth.make_normal_bf16((M, D), seed=12, stream=3, std=1.0)
    W1 = (g.standard_normal((F, D)) / np.sqrt(D)).astype(np.float32)
    W2 = (g.standard_normal((D, F)) / np.sqrt(F)).astype(np.float32)
    w1q, w1s = rb.fp8_quantize_weight(torch.from_numpy(W1).cuda())
    w2q, w2s = rb.fp8_quantize_weight(torch.from_numpy(W2).cuda())
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = rb.fp8_ffn(_bf16_dev(x_bits), w1q, w1s, w2q, w2s, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    _, y_ref = fo.ffn_w8a8(_bf16_f32(x_bits), *fo.quantize_rows(W1), *fo.quantize_rows(W2))
    _check_gemm(y, y_ref, "FFN 300x256x608")
