"""GPU parity of the RoLA backward against the fp64 gradient oracle, through
the C ABI.

* the training forward's output equals the plain forward's bit for bit; its
  saved log-sum-exp and linear denominator match the oracle's statistics;
* dq, dk, dv (bf16): |err| <= 1e-2 + 1e-2 |ref| per element;
* dP_h and dgate (sums over every row): relative error <= 1e-2 (Frobenius);
* two calls give bit-identical gradients (no atomics).
The block mask is the oracle's selection; dout is seeded N(0, 1) bf16.
"""
import numpy as np
import pytest
import torch

from oracle import rola_backward_oracle as rbo
from oracle import rola_oracle as ro
from sparse_linear_attention_mean_b200 import binding as rb
from sparse_linear_attention_mean_b200 import synth

from helpers import bf16_to_f64, check_close, dev_bf16, dev_inputs

pytestmark = pytest.mark.gpu

FROB = 1e-2


def _run(w, inp, gate_scale=1.0, idx_ref=None):
    shape = rb.Shape.of(w)
    q, k, v, P, gate = dev_inputs(inp)
    gate = gate * gate_scale
    if idx_ref is None:
        idx_ref, _ = ro.select_all(inp, w.block, w.k_b)
    idx = torch.from_numpy(idx_ref).cuda()
    states = rb.block_states(shape, k, v, P)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, out_lo, lse, den = rb.attention_fwd_train(shape, q, k, v, idx, P, states, gate, dev_err=err)
    dout_bits = synth.make_normal_bf16((w.B, w.N, w.H, w.d), seed=w.seed + 50, stream=7)
    dout = dev_bf16(dout_bits)
    grads = rb.attention_bwd(shape, q, k, v, idx, P, states, gate, out, out_lo, lse, den, dout, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return dict(shape=shape, q=q, k=k, v=v, P=P, gate=gate, idx=idx, idx_ref=idx_ref, states=states, out=out,
                out_lo=out_lo, lse=lse, den=den, dout=dout, dout_bits=dout_bits, grads=grads)


def _frob(got, ref):
    return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))


def _check_heads(w, inp, r, heads, gate_scale=1.0):
    dq, dk, dv, dP, dg = (t.cpu().numpy().astype(np.float64) if t.dtype != torch.bfloat16 else bf16_to_f64(t)
                          for t in r["grads"])
    worst = 0.0
    for h in heads:
        q, k, v, P_h = ro.head_slices(inp, 0, h)
        g = float(inp["gate"][h]) * gate_scale
        dO = ro.bf16_to_f64(r["dout_bits"][0, :, h, :])
        G = rbo.rola_head_backward(q, k, v, P_h, g, dO, bs=w.block, idx=r["idx_ref"][0, h],
                                   grid=(w.T, w.Hg, w.W), rope_base=w.rope_base)
        for nm, got, ref in (("dq", dq[0, :, h], G.dq), ("dk", dk[0, :, h], G.dk), ("dv", dv[0, :, h], G.dv)):
            worst = max(worst, check_close(got, ref, what=f"{nm} head {h}"))
        assert _frob(dP[h], G.dP) <= FROB, (h, _frob(dP[h], G.dP))
        assert abs(dg[h] - G.dg) <= FROB * abs(G.dg) + 1e-6, (h, dg[h], G.dg)
    return worst


def test_forward_stats_match_the_oracle():
    w = synth.custom_workload(synth.WORKLOADS[2], H=2)
    inp = synth.make_inputs(w)
    r = _run(w, inp)
    plain = rb.attention_fwd(r["shape"], r["q"], r["k"], r["v"], r["idx"], r["P"], r["states"], r["gate"])
    torch.cuda.synchronize()
    lse, den = r["lse"].cpu().numpy(), r["den"].cpu().numpy()
    # the training forward takes P as bf16 hi + lo in P.V; out_lo is the
    # rounding residual of its output (at most half a bf16 step of out); both
    # forwards meet the output bound, and out + out_lo is several times closer
    # to the oracle than the inference forward's bf16-P output
    o_hi, o_lo = bf16_to_f64(r["out"]), bf16_to_f64(r["out_lo"])
    res = ro.rola_forward(inp, bs=w.block, k_b=w.k_b, grid=(w.T, w.Hg, w.W), rope_base=w.rope_base,
                          idx=r["idx_ref"])
    ref = ro.assemble_output(res, w.B, w.N, w.H, w.d, w.block)
    check_close(o_hi, ref, what="training forward")
    check_close(bf16_to_f64(plain), ref, what="inference forward")
    assert np.all(np.abs(o_lo) <= 2.0 ** -8 * np.abs(o_hi))
    assert np.abs(o_hi + o_lo - ref).mean() <= 0.5 * np.abs(bf16_to_f64(plain) - ref).mean()
    for h in range(w.H):
        q, k, v, P_h = ro.head_slices(inp, 0, h)
        l_ref, d_ref = rbo.forward_stats(q, k, v, P_h, bs=w.block, idx=r["idx_ref"][0, h],
                                         grid=(w.T, w.Hg, w.W), rope_base=w.rope_base)
        np.testing.assert_allclose(lse[0, h], l_ref, rtol=0, atol=2e-3)
        np.testing.assert_allclose(den[0, h], d_ref, rtol=2e-3, atol=0)


@pytest.mark.parametrize("T,Hg,W,kb,r_", [
    (2, 16, 20, 2, 32),   # 640 tokens: 5 full blocks
    (3, 9, 10, 1, 16),    # 270 tokens: 3 blocks, ragged last (14 valid), r = 16
    (2, 15, 21, 2, 32),   # 630 tokens: 5 blocks, ragged last (118 valid)
])
@pytest.mark.parametrize("gate_scale", [1.0, 1000.0])
def test_backward_small_all_rows(T, Hg, W, kb, r_, gate_scale):
    """Small d = 128 shapes, every row of every head; at 1000x the gate the
    linear branch's gradients carry the result."""
    w = synth.Workload("bwd-small", 1, 3, 128, T, Hg, W, 128, 0, kb, r_, seed=13)
    inp = synth.make_inputs(w)
    r = _run(w, inp, gate_scale)
    worst = _check_heads(w, inp, r, range(w.H), gate_scale)
    print(f"{T}x{Hg}x{W} k_b {kb} r {r_} gate x{gate_scale:g}: worst err/bound {worst:.3f}")


def test_backward_dense_limit_every_block_kept():
    """s = 0: every block kept, the linear branch is exactly zero, and the
    gradients are those of dense softmax attention (library autograd)."""
    w = synth.Workload("bwd-dense", 1, 2, 128, 2, 16, 20, 128, 0, 5, 32, seed=17)
    inp = synth.make_inputs(w)
    r = _run(w, inp)
    dq, dk, dv, dP, dg = r["grads"]
    q, k, v = (torch.from_numpy(ro.bf16_to_f64(inp[x])).permute(0, 2, 1, 3).requires_grad_(True)
               for x in ("q", "k", "v"))
    o = torch.nn.functional.scaled_dot_product_attention(q, k, v)
    dO = torch.from_numpy(ro.bf16_to_f64(r["dout_bits"])).permute(0, 2, 1, 3)
    (o * dO).sum().backward()
    for nm, got, ref in (("dq", dq, q.grad), ("dk", dk, k.grad), ("dv", dv, v.grad)):
        check_close(bf16_to_f64(got), ref.permute(0, 2, 1, 3).numpy(), what=f"dense {nm}")
    assert torch.all(dP == 0) and torch.all(dg == 0)


@pytest.mark.parametrize("cfg,heads,gate_scale", [(1, [0, 11], 1.0), (2, [39], 1.0), (3, [0], 1.0), (3, [7], 1000.0)])
def test_backward_workloads(cfg, heads, gate_scale):
    """Wan2.1-1.3B 480P (all rows of two heads), 14B 480P (all rows of the
    last head) and 14B 720P (all rows of head 0) at the nominal gate, and
    all rows of a 720P head at 1000x the gate, where the linear branch's
    gradients (state gather, complement, 720P rotary table) carry the result."""
    w = synth.WORKLOADS[cfg]
    inp = synth.make_inputs(w)
    idx_ref, _ = ro.select_all(inp, w.block, w.k_b)
    r = _run(w, inp, gate_scale, idx_ref=idx_ref)
    worst = _check_heads(w, inp, r, heads, gate_scale)
    print(f"workload {cfg}: heads {heads}, gate x{gate_scale:g}, worst err/bound {worst:.3f}")


def test_backward_is_deterministic():
    w = synth.custom_workload(synth.WORKLOADS[2], H=2)
    inp = synth.make_inputs(w)
    r = _run(w, inp)
    again = rb.attention_bwd(r["shape"], r["q"], r["k"], r["v"], r["idx"], r["P"], r["states"], r["gate"],
                             r["out"], r["out_lo"], r["lse"], r["den"], r["dout"])
    torch.cuda.synchronize()
    for a, b in zip(r["grads"], again):
        assert torch.equal(a, b)
