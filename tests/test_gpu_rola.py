"""GPU parity of the RoLA path against the fp64 oracle, through the C ABI.

* block masks: bit-exact; rows whose k-th and (k+1)-th scores lie within 1e-5
  (relative) are reported and are the only rows allowed to differ;
* states S_blk, z_blk, S, z: within 1e-4 relative (plus 1e-4 of the block's
  largest magnitude);
* attention output given the oracle's mask: |err| <= 1e-2 + 1e-2 |ref|.
"""
import numpy as np
import pytest
import torch

from oracle import rola_oracle as ro
from sparse_linear_attention_mean_b200 import binding as rb
from sparse_linear_attention_mean_b200 import synth

from helpers import bf16_to_f64, check_close, dev_bf16, dev_inputs, mask_mismatch

pytestmark = pytest.mark.gpu

_CACHE = {}


def workload_inputs(i):
    if i not in _CACHE:
        w = synth.WORKLOADS[i]
        _CACHE.clear()
        _CACHE[i] = (w, synth.make_inputs(w))
    return _CACHE[i]


def _grid(w):
    return (w.T, w.Hg, w.W)


def _states_check(w, inp, states, heads):
    S_blk, z_blk, S_glb, z_glb = (t.cpu().numpy().astype(np.float64) for t in states)
    for h in heads:
        q, k, v, P = ro.head_slices(inp, 0, h)
        th = ro.rope_angles(w.N, w.T, w.Hg, w.W, w.r, w.rope_base)
        Sb, zb, S, z = ro.block_states(k, v, P, th, w.block)
        scale = np.abs(Sb).max(axis=(1, 2), keepdims=True)
        err = np.abs(S_blk[0, h] - Sb)
        assert np.all(err <= 1e-4 * scale + 1e-4 * np.abs(Sb)), (h, float((err / (scale + 1e-30)).max()))
        assert np.all(np.abs(z_blk[0, h] - zb) <= 1e-4 * np.abs(zb) + 1e-6), h
        assert np.all(np.abs(S_glb[0, h] - S) <= 1e-4 * np.abs(S).max() + 1e-4 * np.abs(S)), h
        assert np.all(np.abs(z_glb[0, h] - z) <= 1e-5 * np.abs(z)), h


@pytest.mark.parametrize("cfg", [0, 1, 2, 3])
def test_select_blocks_bitexact(cfg):
    w, inp = workload_inputs(cfg)
    shape = rb.Shape.of(w)
    q, k, v, P, gate = dev_inputs(inp)
    idx_gpu, sc_gpu = rb.select_blocks(shape, q, k, scores=True)
    idx_ref, sig = ro.select_all(inp, w.block, w.k_b)
    idx_gpu = idx_gpu.cpu().numpy()
    ties, bad = mask_mismatch(idx_gpu, idx_ref, sig, w.k_b)
    assert not bad, f"mask rows differ outside near-ties: {bad[:5]}"
    # scores agree to float64 rounding
    np.testing.assert_allclose(sc_gpu.cpu().numpy(), sig, rtol=1e-12, atol=1e-12 * np.abs(sig).max())
    n_ties = sum(len(ro.near_ties(sig[0, h], w.k_b)) for h in range(w.H))
    print(f"workload {cfg}: {idx_ref.size // w.k_b} rows, near-tie rows {n_ties}, differing tie rows {len(ties)}")
    # every row strictly ascending and in range
    assert (np.diff(idx_gpu, axis=-1) > 0).all() and idx_gpu.min() >= 0 and idx_gpu.max() < w.n_blocks


@pytest.mark.parametrize("T,Hg,W,kb", [
    (4, 40, 40, 32),   # 100 blocks of 64: largest k_b of the candidate path
    (4, 40, 40, 33),   # k_b above 32: arg-max rounds
    (4, 60, 80, 7),    # 300 blocks: more lanes' worth of scores per lane
])
def test_select_kb_paths(T, Hg, W, kb):
    w = synth.Workload("sel", 1, 3, 64, T, Hg, W, 64, 0, kb, 16, seed=5)
    inp = synth.make_inputs(w)
    q, k, v, P, gate = dev_inputs(inp)
    idx_gpu = rb.select_blocks(rb.Shape.of(w), q, k).cpu().numpy()
    idx_ref, sig = ro.select_all(inp, w.block, w.k_b)
    ties, bad = mask_mismatch(idx_gpu, idx_ref, sig, w.k_b)
    assert not bad, f"mask rows differ outside near-ties: {bad[:5]}"


@pytest.mark.parametrize("T,Hg,W,kb", [(4, 40, 40, 5), (4, 60, 80, 5), (4, 60, 80, 40)])
def test_select_all_scores_equal(T, Hg, W, kb):
    """q = 0 makes every score 0: ties go to the lower block index, so each
    row keeps blocks 0 .. k_b - 1 (300 blocks exceed the candidate buffer)."""
    w = synth.Workload("ties", 1, 2, 64, T, Hg, W, 64, 0, kb, 16, seed=6)
    inp = synth.make_inputs(w)
    inp["q"] = np.zeros_like(inp["q"])
    q, k, v, P, gate = dev_inputs(inp)
    idx_gpu = rb.select_blocks(rb.Shape.of(w), q, k).cpu().numpy()
    idx_ref, _ = ro.select_all(inp, w.block, w.k_b)
    assert np.array_equal(idx_ref, np.broadcast_to(np.arange(kb, dtype=np.int32), idx_ref.shape))
    assert np.array_equal(idx_gpu, idx_ref)


@pytest.mark.parametrize("cfg,heads", [(0, [0, 1]), (1, [0, 11]), (3, [0, 39])])
def test_block_states(cfg, heads):
    w, inp = workload_inputs(cfg)
    shape = rb.Shape.of(w)
    q, k, v, P, gate = dev_inputs(inp)
    states = rb.block_states(shape, k, v, P)
    torch.cuda.synchronize()
    _states_check(w, inp, states, heads)


def _attention_case(w, inp, heads, qblocks, gate_scale=1.0, idx_ref=None):
    shape = rb.Shape.of(w)
    q, k, v, P, gate = dev_inputs(inp)
    gate = gate * gate_scale
    if idx_ref is None:
        idx_ref, _ = ro.select_all(inp, w.block, w.k_b)
    idx = torch.from_numpy(idx_ref).cuda()
    states = rb.block_states(shape, k, v, P)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = rb.attention_fwd(shape, q, k, v, idx, P, states, gate, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    o = bf16_to_f64(out)
    inp2 = dict(inp)
    inp2["gate"] = (inp["gate"].astype(np.float64) * gate_scale)
    res = ro.rola_forward(inp2, bs=w.block, k_b=w.k_b, grid=_grid(w), rope_base=w.rope_base,
                          idx=idx_ref, heads=heads, qblocks=qblocks)
    worst = 0.0
    for (b, h), r in res.items():
        for a, rows in r.o.items():
            lo, hi = ro.block_range(a, w.block, w.N)
            worst = max(worst, check_close(o[b, lo:hi, h, :], rows, what=f"head {h} block {a}"))
    return worst, out


@pytest.mark.parametrize("cfg", [0, 1])
def test_attention_all_rows(cfg):
    w, inp = workload_inputs(cfg)
    worst, out = _attention_case(w, inp, heads=None, qblocks=None)
    print(f"workload {cfg}: worst err/bound {worst:.3f}")
    # padded rows are never written: the buffer beyond N does not exist, and
    # every valid row is finite
    assert torch.isfinite(out.float()).all()


@pytest.mark.parametrize("cfg", [2, 3])
def test_attention_sampled(cfg):
    w, inp = workload_inputs(cfg)
    nb = w.n_blocks
    qblocks = [0, 1, nb // 2, nb - 2, nb - 1]
    worst, _ = _attention_case(w, inp, heads=[0, w.H - 1], qblocks=qblocks)
    print(f"workload {cfg}: worst err/bound {worst:.3f}")


def _spread_heads(H, n):
    return sorted({round(i * (H - 1) / (n - 1)) for i in range(n)})


@pytest.mark.parametrize("cfg", [2, 3])
def test_layer_full_heads(cfg):
    """The layer entry point (the benchmark's path: fused pass over q, k, v for
    block means and states, selector, state totals, two-tile attention) on
    every query block of ten heads spread over the 40, at the nominal gate and
    at 1000x the gate, where the linear branch (state gather, global-minus-kept
    complement, rotary table up to the grid's last positions) carries the
    output.  The GPU's mask must equal the oracle's outside reported near-ties;
    the oracle then evaluates the attention given the GPU's mask."""
    w, inp = workload_inputs(cfg)
    shape = rb.Shape.of(w)
    q, k, v, P, gate = dev_inputs(inp)
    layer = rb.Layer(shape)
    idx = torch.empty((1, w.H, w.n_blocks, w.k_b), dtype=torch.int32, device="cuda")
    out = layer(q, k, v, P, gate, idx_out=idx)
    out_lin = layer(q, k, v, P, gate * 1000.0)
    torch.cuda.synchronize()
    assert int(layer.dev_err.item()) == 0
    idx_gpu = idx.cpu().numpy()
    heads = _spread_heads(w.H, 10)
    o, o_lin = bf16_to_f64(out), bf16_to_f64(out_lin)
    worst = [0.0, 0.0]
    n_ties = 0
    for h in heads:
        qh, kh, vh, Ph = ro.head_slices(inp, 0, h)
        g = float(inp["gate"][h])
        r = ro.rola_head(qh, kh, vh, Ph, g, bs=w.block, k_b=w.k_b, grid=_grid(w),
                         rope_base=w.rope_base, idx=idx_gpu[0, h])
        # the GPU's mask against the oracle's own selection (same scores)
        ref_idx = ro.select_topk(r.sigma, w.k_b)
        ties = set(ro.near_ties(r.sigma, w.k_b))
        n_ties += len(ties)
        diff = np.nonzero((ref_idx != idx_gpu[0, h]).any(axis=1))[0]
        assert set(diff.tolist()) <= ties, f"head {h}: mask rows differ outside near-ties"
        for a in range(w.n_blocks):
            lo, hi = ro.block_range(a, w.block, w.N)
            worst[0] = max(worst[0], check_close(o[0, lo:hi, h, :], r.o[a], what=f"head {h} block {a}"))
            ref_l = r.o_sp[a] + 1000.0 * g * r.o_lin[a]
            worst[1] = max(worst[1], check_close(o_lin[0, lo:hi, h, :], ref_l,
                                                 what=f"gate x1000 head {h} block {a}"))
    print(f"workload {cfg}: heads {heads}, all {w.n_blocks} query blocks; worst err/bound "
          f"{worst[0]:.3f} (gate) {worst[1]:.3f} (gate x1000); near-tie rows {n_ties}")


@pytest.mark.parametrize("cfg", [0, 1])
def test_attention_linear_branch_dominant(cfg):
    # o_lin of zero-mean v is ~1e-3; a gate of 1e3 makes the linear branch
    # carry the output so that its parity is visible at the same tolerance.
    w, inp = workload_inputs(cfg)
    worst, _ = _attention_case(w, inp, heads=[0, w.H - 1], qblocks=None, gate_scale=1000.0)
    print(f"workload {cfg} gate x1000: worst err/bound {worst:.3f}")


def test_attention_gate_zero_is_block_sparse():
    w = synth.custom_workload(synth.WORKLOADS[0], gate_const=0.0)
    inp = synth.make_inputs(w)
    worst, _ = _attention_case(w, inp, heads=None, qblocks=None)


@pytest.mark.parametrize("T,Hg,W,block,d,r,kb", [
    (2, 8, 9, 64, 64, 16, 3),      # 144 tokens: ragged last block of 16
    (3, 5, 7, 64, 64, 32, 1),      # 105 tokens, one kept block
    (2, 8, 9, 128, 128, 32, 2),    # 2 blocks of 128, last has 16 valid
    (3, 9, 10, 128, 64, 16, 2),    # d = 64 with 128-token blocks
])
def test_attention_ragged_small(T, Hg, W, block, d, r, kb):
    w = synth.Workload("ragged", 1, 3, d, T, Hg, W, block, 0, kb, r, seed=7)
    inp = synth.make_inputs(w)
    worst, _ = _attention_case(w, inp, heads=None, qblocks=None)
    worst_l, _ = _attention_case(w, inp, heads=None, qblocks=None, gate_scale=1000.0)


@pytest.mark.parametrize("block,d,r", [(64, 64, 16), (128, 128, 32)])
def test_dense_limit_s0(block, d, r):
    T, Hg, W = (2, 8, 16) if block == 64 else (2, 16, 20)
    N = T * Hg * W
    nb = -(-N // block)
    w = synth.Workload("dense", 1, 2, d, T, Hg, W, block, 0, nb, r, seed=11)
    inp = synth.make_inputs(w)
    worst, out = _attention_case(w, inp, heads=None, qblocks=None, gate_scale=1000.0)
    # with every block kept, o_lin is exactly 0: the output is plain softmax attention
    q, k, v = (torch.from_numpy(ro.bf16_to_f64(inp[x])).permute(0, 2, 1, 3) for x in ("q", "k", "v"))
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v).permute(0, 2, 1, 3).numpy()
    check_close(bf16_to_f64(out), ref, what="dense limit vs SDPA")


@pytest.mark.parametrize("base", ["tiny", "128"])
def test_batch_two_matches_single(base):
    """B = 2 through the selector, the states and the attention: the 64-token
    workload (one-tile kernel) and a 128-token-block one (two-tile kernel,
    fused prep pass on the layer path)."""
    if base == "tiny":
        w = synth.custom_workload(synth.WORKLOADS[0], B=2)
    else:
        w = synth.Workload("batch2-128", 2, 3, 128, 2, 16, 20, 128, 0, 2, 32, seed=9)
    inp = synth.make_inputs(w)
    idx_ref, _ = ro.select_all(inp, w.block, w.k_b)
    shape = rb.Shape.of(w)
    q, k, v, P, gate = dev_inputs(inp)
    idx_gpu = rb.select_blocks(shape, q, k).cpu().numpy()
    assert np.array_equal(idx_gpu, idx_ref)
    _attention_case(w, inp, heads=None, qblocks=None)
    # the whole layer: the same mask, and the output matches the oracle
    layer = rb.Layer(shape)
    idx_l = torch.empty_like(torch.from_numpy(idx_ref)).cuda()
    out = layer(q, k, v, P, gate, idx_out=idx_l)
    torch.cuda.synchronize()
    assert int(layer.dev_err.item()) == 0
    assert np.array_equal(idx_l.cpu().numpy(), idx_ref)
    res = ro.rola_forward(inp, bs=w.block, k_b=w.k_b, grid=_grid(w), rope_base=w.rope_base, idx=idx_ref)
    check_close(bf16_to_f64(out), ro.assemble_output(res, w.B, w.N, w.H, w.d, w.block), what="layer, B = 2")


def test_bad_index_reported_not_trapped():
    w, inp = workload_inputs(0)
    shape = rb.Shape.of(w)
    q, k, v, P, gate = dev_inputs(inp)
    idx_ref, _ = ro.select_all(inp, w.block, w.k_b)
    bad = idx_ref.copy()
    bad[0, 0, 3, 1] = 999            # out of range
    bad[0, 1, 5, 2] = bad[0, 1, 5, 1]  # duplicate (not ascending)
    states = rb.block_states(shape, k, v, P)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = rb.attention_fwd(shape, q, k, v, torch.from_numpy(bad).cuda(), P, states, gate, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & rb.DEVERR_BAD_INDEX
    assert not (int(err.item()) & rb.DEVERR_TIMEOUT)
    # untouched rows still match the oracle
    o = bf16_to_f64(out)
    res = ro.rola_forward(inp, bs=w.block, k_b=w.k_b, grid=_grid(w), idx=idx_ref, heads=[0], qblocks=[0, 1])
    for a, rows in res[(0, 0)].o.items():
        lo, hi = ro.block_range(a, w.block, w.N)
        check_close(o[0, lo:hi, 0, :], rows)


@pytest.mark.parametrize("cfg", [0, 1, 3])
def test_layer_entry_points(cfg):
    w, inp = workload_inputs(cfg)
    shape = rb.Shape.of(w)
    q, k, v, P, gate = dev_inputs(inp)
    idx = torch.empty((1, w.H, w.n_blocks, w.k_b), dtype=torch.int32, device="cuda")
    layer = rb.Layer(shape)
    out = layer(q, k, v, P, gate, idx_out=idx)
    torch.cuda.synchronize()
    assert int(layer.dev_err.item()) == 0
    idx_ref, sig = ro.select_all(inp, w.block, w.k_b)
    ties, bad = mask_mismatch(idx.cpu().numpy(), idx_ref, sig, w.k_b)
    assert not bad
    # same as the three calls in sequence
    idx2 = rb.select_blocks(shape, q, k)
    out2 = rb.attention_fwd(shape, q, k, v, idx2, P, rb.block_states(shape, k, v, P), gate)
    torch.cuda.synchronize()
    assert torch.equal(out, out2)
    # host-buffer variant: pinned host tensors in, host tensor out
    host = [t.cpu().pin_memory() for t in (q, k, v, P, gate)]
    out_h = torch.empty(out.shape, dtype=torch.bfloat16).pin_memory()
    hl = rb.HostLayer(shape)
    hl(*host, out_h)
    torch.cuda.synchronize()
    assert torch.equal(out_h, out.cpu())
    # timed variant (three and five events): same result, ordered stage times
    for n in (3, 5):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        out3 = layer(q, k, v, P, gate, events=ev)
        torch.cuda.synchronize()
        assert torch.equal(out3, out)
        assert all(ev[i].elapsed_time(ev[i + 1]) >= 0 for i in range(n - 1))
        assert ev[0].elapsed_time(ev[n - 1]) > 0
    assert rb.layer_launches(shape) in (5, 6)


def test_attention_output_alignment_16_bytes():
    """The output may be 16-byte aligned only (the epilogue then stores 16
    bytes at a time instead of 32): same result either way."""
    w = synth.custom_workload(synth.WORKLOADS[2], H=2)
    inp = synth.make_inputs(w)
    shape = rb.Shape.of(w)
    q, k, v, P, gate = dev_inputs(inp)
    idx = rb.select_blocks(shape, q, k)
    states = rb.block_states(shape, k, v, P)
    ref = rb.attention_fwd(shape, q, k, v, idx, P, states, gate)
    n = ref.numel()
    raw = torch.empty(n + 64, dtype=torch.bfloat16, device="cuda")
    base = raw.data_ptr()
    off = ((32 - base % 32) % 32 + 16) // 2  # elements to a 16-mod-32 address
    out = raw[off:off + n].view(ref.shape)
    assert out.data_ptr() % 32 == 16
    rb.attention_fwd(shape, q, k, v, idx, P, states, gate, out=out)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)


def test_attention_states_16_byte_aligned():
    """Block states that are 16- but not 32-byte aligned take the one-tile
    kernel (the two-tile kernel reads them 32 bytes at a time).  That kernel's
    output at d = 128 with 128-token blocks is compared with the oracle on
    every query block of both heads, at the nominal gate and at 1000x."""
    w = synth.custom_workload(synth.WORKLOADS[2], H=2)
    inp = synth.make_inputs(w)
    shape = rb.Shape.of(w)
    q, k, v, P, gate = dev_inputs(inp)
    idx_ref, _ = ro.select_all(inp, w.block, w.k_b)
    idx = torch.from_numpy(idx_ref).cuda()
    S_blk, z_blk, S_glb, z_glb = rb.block_states(shape, k, v, P)
    raw = torch.empty(S_blk.numel() + 16, dtype=torch.float32, device="cuda")
    off = ((32 - raw.data_ptr() % 32) % 32 + 16) // 4
    S16 = raw[off:off + S_blk.numel()].view(S_blk.shape)
    S16.copy_(S_blk)
    assert S16.data_ptr() % 32 == 16
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = rb.attention_fwd(shape, q, k, v, idx, P, (S16, z_blk, S_glb, z_glb), gate, dev_err=err)
    out_l = rb.attention_fwd(shape, q, k, v, idx, P, (S16, z_blk, S_glb, z_glb), gate * 1000.0, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    res = ro.rola_forward(inp, bs=w.block, k_b=w.k_b, grid=_grid(w), rope_base=w.rope_base, idx=idx_ref)
    o, o_l = bf16_to_f64(out), bf16_to_f64(out_l)
    for (b, h), r in res.items():
        g = float(inp["gate"][h])
        for a in r.o:
            lo, hi = ro.block_range(a, w.block, w.N)
            check_close(o[b, lo:hi, h, :], r.o[a], what=f"one-tile head {h} block {a}")
            check_close(o_l[b, lo:hi, h, :], r.o_sp[a] + 1000.0 * g * r.o_lin[a],
                        what=f"one-tile gate x1000 head {h} block {a}")


def test_bad_index_two_tile_kernel():
    """Bad kept-block entries on the d = 128, 128-token-block shape (the
    persistent two-tile kernel): reported through ROLA_DEVERR_BAD_INDEX, never
    trapped, and every query block without a bad entry still matches the
    oracle."""
    w = synth.custom_workload(synth.WORKLOADS[2], H=2)
    inp = synth.make_inputs(w)
    shape = rb.Shape.of(w)
    q, k, v, P, gate = dev_inputs(inp)
    idx_ref, _ = ro.select_all(inp, w.block, w.k_b)
    bad = idx_ref.copy()
    bad[0, 0, 3, 1] = 999                 # out of range
    bad[0, 1, 40, 2] = bad[0, 1, 40, 1]   # duplicate (not ascending)
    bad[0, 1, 255, 0] = -5                # negative, in the ragged last block's row
    touched = {(0, 3), (1, 40), (1, 255)}
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    states = rb.block_states(shape, k, v, P)
    out = rb.attention_fwd(shape, q, k, v, torch.from_numpy(bad).cuda(), P, states, gate, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & rb.DEVERR_BAD_INDEX
    assert not (int(err.item()) & rb.DEVERR_TIMEOUT)
    o = bf16_to_f64(out)
    res = ro.rola_forward(inp, bs=w.block, k_b=w.k_b, grid=_grid(w), rope_base=w.rope_base, idx=idx_ref)
    checked = 0
    for (b, h), r in res.items():
        for a, rows in r.o.items():
            if (h, a) in touched:
                continue
            lo, hi = ro.block_range(a, w.block, w.N)
            check_close(o[b, lo:hi, h, :], rows, what=f"head {h} block {a}")
            checked += 1
    assert checked == 2 * w.n_blocks - len(touched)


@pytest.mark.parametrize("which", ["one-tile", "two-tile"])
def test_wait_timeout_reported_and_recovered(which):
    """The bounded-wait timeout path, without any fault: with a wait bound of
    0 ns every pipeline wait that finds its stage not ready gives up, so the
    kernel stops, drains its copies and MMAs, frees tensor memory and sets
    ROLA_DEVERR_TIMEOUT.  The call returns, and a normal call afterwards in the
    same process reproduces the earlier output bit for bit (itself checked
    against the oracle)."""
    if which == "one-tile":
        w = synth.WORKLOADS[0]
    else:
        w = synth.custom_workload(synth.WORKLOADS[2], H=2)
    inp = synth.make_inputs(w)
    shape = rb.Shape.of(w)
    q, k, v, P, gate = dev_inputs(inp)
    idx_ref, _ = ro.select_all(inp, w.block, w.k_b)
    idx = torch.from_numpy(idx_ref).cuda()
    states = rb.block_states(shape, k, v, P)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ref = rb.attention_fwd(shape, q, k, v, idx, P, states, gate, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    res = ro.rola_forward(inp, bs=w.block, k_b=w.k_b, grid=_grid(w), rope_base=w.rope_base, idx=idx_ref,
                          heads=[0], qblocks=[0, 1, w.n_blocks - 1])
    for a, rows in res[(0, 0)].o.items():
        lo, hi = ro.block_range(a, w.block, w.N)
        check_close(bf16_to_f64(ref)[0, lo:hi, 0, :], rows, what=f"reference block {a}")
    out = torch.zeros_like(ref)
    rb.attention_fwd(shape, q, k, v, idx, P, states, gate, out=out, dev_err=err, wait_limit_ns=0)
    torch.cuda.synchronize()
    assert int(err.item()) & rb.DEVERR_TIMEOUT
    assert not (int(err.item()) & rb.DEVERR_BAD_INDEX)
    err.zero_()
    again = rb.attention_fwd(shape, q, k, v, idx, P, states, gate, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert torch.equal(again, ref)
    # an ample bound behaves like the default one
    bounded = rb.attention_fwd(shape, q, k, v, idx, P, states, gate, dev_err=err, wait_limit_ns=10**9)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert torch.equal(bounded, ref)


def _per_head_counts(w):
    return np.array([1 + (h * 7) % w.k_b for h in range(w.H)], dtype=np.int32)


@pytest.mark.parametrize("cfg", [0, 1, 2])
def test_layer_per_head_kept_counts(cfg):
    """Head-adaptive sparsity through the layer entry: each head keeps its own
    number of blocks; the mask is bit-exact against the oracle's per-head
    selection (outside near-ties), unused entries are -1, and the output
    matches the oracle given that mask (all query blocks of two heads)."""
    w, inp = workload_inputs(cfg)
    shape = rb.Shape.of(w)
    q, k, v, P, gate = dev_inputs(inp)
    kbh = _per_head_counts(w)
    layer = rb.Layer(shape)
    idx = torch.empty((1, w.H, w.n_blocks, w.k_b), dtype=torch.int32, device="cuda")
    out = layer.run_ex(q, k, v, P, gate, idx, kb_per_head=torch.from_numpy(kbh).cuda())
    out_l = layer.run_ex(q, k, v, P, gate * 1000.0, idx, kb_per_head=torch.from_numpy(kbh).cuda())
    torch.cuda.synchronize()
    assert int(layer.dev_err.item()) == 0
    got = idx.cpu().numpy()
    ref, sig = ro.select_all_per_head(inp, w.block, kbh, w.k_b)
    for h in range(w.H):
        kh = int(kbh[h])
        assert (got[0, h, :, kh:] == -1).all()
        ties = set(ro.near_ties(sig[0, h], kh))
        diff = np.nonzero((got[0, h, :, :kh] != ref[0, h, :, :kh]).any(axis=1))[0]
        assert set(diff.tolist()) <= ties, f"head {h}: mask rows differ outside near-ties"
    heads = [0, w.H - 1]
    res = ro.rola_forward(inp, bs=w.block, k_b=w.k_b, grid=_grid(w), rope_base=w.rope_base, idx=got,
                          heads=heads, kb_per_head=kbh)
    o, o_l = bf16_to_f64(out), bf16_to_f64(out_l)
    for (b, h), r in res.items():
        g = float(inp["gate"][h])
        for a in r.o:
            lo, hi = ro.block_range(a, w.block, w.N)
            check_close(o[b, lo:hi, h, :], r.o[a], what=f"head {h} (k_b {kbh[h]}) block {a}")
            check_close(o_l[b, lo:hi, h, :], r.o_sp[a] + 1000.0 * g * r.o_lin[a],
                        what=f"gate x1000 head {h} block {a}")


def test_layer_per_head_count_out_of_range_reported():
    w, inp = workload_inputs(1)
    shape = rb.Shape.of(w)
    q, k, v, P, gate = dev_inputs(inp)
    kbh = _per_head_counts(w)
    kbh[3] = 0
    kbh[5] = w.k_b + 9
    layer = rb.Layer(shape)
    idx = torch.empty((1, w.H, w.n_blocks, w.k_b), dtype=torch.int32, device="cuda")
    layer.run_ex(q, k, v, P, gate, idx, kb_per_head=torch.from_numpy(kbh).cuda())
    torch.cuda.synchronize()
    assert int(layer.dev_err.item()) & rb.DEVERR_BAD_INDEX
    assert not (int(layer.dev_err.item()) & rb.DEVERR_TIMEOUT)
    got = idx.cpu().numpy()
    assert (got[0, 3, :, 1:] == -1).all() and (got[0, 3, :, 0] >= 0).all()   # clamped to 1
    assert (got[0, 5] >= 0).all()                                            # clamped to k_b


@pytest.mark.parametrize("cfg", [0, 2])
def test_layer_mask_reuse_across_steps(cfg):
    """Cross-step reuse of the sparsity pattern: a layer call that takes the
    mask of an earlier step runs no selection and gives the attention of the
    new step's q, k, v under that mask -- bit-identical to selecting the same
    mask, and to the three separate calls with it; checked against the oracle
    on sampled query blocks (also with per-head counts)."""
    w, inp = workload_inputs(cfg)
    shape = rb.Shape.of(w)
    q, k, v, P, gate = dev_inputs(inp)
    layer = rb.Layer(shape)
    idx = torch.empty((1, w.H, w.n_blocks, w.k_b), dtype=torch.int32, device="cuda")
    out1 = layer.run_ex(q, k, v, P, gate, idx)
    idx1 = idx.clone()
    out2 = layer.run_ex(q, k, v, P, gate, idx1, reuse_mask=True)
    torch.cuda.synchronize()
    assert int(layer.dev_err.item()) == 0
    assert torch.equal(out1, out2) and torch.equal(idx1, idx)
    # the next step: other activations (another seed of the same shape), the old mask
    inp2 = synth.make_inputs(synth.custom_workload(w, seed=w.seed + 100))
    q2, k2, v2, _, _ = dev_inputs(inp2)
    out3 = layer.run_ex(q2, k2, v2, P, gate, idx1, reuse_mask=True)
    sep = rb.attention_fwd(shape, q2, k2, v2, idx1, P, rb.block_states(shape, k2, v2, P), gate)
    torch.cuda.synchronize()
    assert int(layer.dev_err.item()) == 0
    assert torch.equal(out3, sep)
    assert torch.equal(idx1, idx)  # the reused mask is read, not written
    inp2["P"], inp2["gate"] = inp["P"], inp["gate"]
    qb = [0, 1, w.n_blocks // 2, w.n_blocks - 1]
    heads = [0, w.H - 1]
    res = ro.rola_forward(inp2, bs=w.block, k_b=w.k_b, grid=_grid(w), rope_base=w.rope_base,
                          idx=idx1.cpu().numpy(), heads=heads, qblocks=qb)
    o3 = bf16_to_f64(out3)
    for (b, h), r in res.items():
        for a, rows in r.o.items():
            lo, hi = ro.block_range(a, w.block, w.N)
            check_close(o3[b, lo:hi, h, :], rows, what=f"reused mask head {h} block {a}")
    # per-head counts with a reused mask
    kbh = torch.from_numpy(_per_head_counts(w)).cuda()
    idx_h = torch.empty_like(idx)
    out4 = layer.run_ex(q, k, v, P, gate, idx_h, kb_per_head=kbh)
    out5 = layer.run_ex(q, k, v, P, gate, idx_h.clone(), kb_per_head=kbh, reuse_mask=True)
    torch.cuda.synchronize()
    assert int(layer.dev_err.item()) == 0
    assert torch.equal(out4, out5)
