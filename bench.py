"""Benchmark of the RoLA attention layer on B200.

One step = one RoLA attention layer (block selection, linear-branch states,
fused sparse + linear attention) over the Wan2.1-14B 720P attention shape at
97 % block sparsity: B=1, H=40, d=128, 21x45x80 latent grid (N=75600 tokens,
591 blocks of 128, 18 kept per query block), rank 32.  Inputs are the seeded
synthetic tensors of ``synth`` (2.3 GB of q/k/v, larger than the 126 MB L2,
so no flush is needed between steps).

Printed (rank 0, one JSON line): effective TFLOP/s over the computed blocks
(4 * 128^2 * d per kept block pair, QK^T and PV) for the whole job, ms per
layer, per-kernel times, the roofline of the dominant kernel, an end-to-end
figure through the host-buffer entry point, the fp64 oracle timed on the host
cores on a bounded sample, and the SM clocks seen during the timed region.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

With N > 1 (under torchrun) every rank runs an independent replica of the
layer; the whole-job figure is N x work / (max over ranks of the time).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "RoLA attn fwd ms/layer & effective TFLOPS (% B200 BF16 peak), Wan-14B 720P 97%"
UNIT = "TFLOP/s"
WORKLOAD_ID = 3


def workload_config(w) -> dict:
    return {"workload": w.name, "B": w.B, "H": w.H, "d": w.d,
            "grid_thw": [w.T, w.Hg, w.W], "N": w.N, "block": w.block,
            "n_blocks": w.n_blocks, "sparsity_permille": w.sparsity_permille, "k_b": w.k_b,
            "rank": w.r, "flop_per_layer": w.sparse_flops(),
            "l2": "inputs 2.3 GB > 126 MB L2, no flush between steps"}


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while running."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=2)

    def summary(self) -> dict | None:
        rows = []
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                rows.append((float(parts[0]), float(parts[1]), parts[4:8]))
            except ValueError:
                continue
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, fl in rows for i, x in enumerate(fl) if x.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "samples": len(rows), "reasons": reasons}


# ---------------------------------------------------------------- CPU oracle

def oracle_sample(w, inp, heads=(0,), qblocks=None):
    """Runs the fp64 oracle on a bounded sample; returns (seconds, flop, text)."""
    from oracle import rola_oracle as ro
    nb = w.n_blocks
    qb = list(range(nb)) if qblocks is None else list(qblocks)
    t0 = time.perf_counter()
    ro.rola_forward(inp, bs=w.block, k_b=w.k_b, grid=(w.T, w.Hg, w.W), rope_base=w.rope_base,
                    heads=list(heads), qblocks=qb)
    dt = time.perf_counter() - t0
    flop = 4.0 * w.block * w.block * w.d * w.k_b * len(qb) * len(heads)
    text = (f"fp64 oracle on {len(heads)} head(s) x {len(qb)} of {nb} query blocks "
            f"(selection and states over the whole head included)")
    return dt, flop, text


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def cpu_baseline(w, inp) -> dict:
    # several seconds of host work: every query block of four heads
    heads = tuple(sorted({0, w.H // 3, (2 * w.H) // 3, w.H - 1}))
    dt, flop, text = oracle_sample(w, inp, heads=heads, qblocks=range(w.n_blocks))
    return {"value": flop / dt / 1e12, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": text + f"; {dt:.1f} s"}


# ---------------------------------------------------------------- replicas

def max_over_ranks(x: float) -> float:
    """Max of a per-rank scalar over the process group (the value itself when
    there is none): multi-GPU times are the slowest rank's."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(flop_per_step: float, steps: int, world: int, total_ms: float) -> float:
    """Whole-job TFLOP/s of `world` replicas that each ran `steps` steps of
    `flop_per_step`, timed by the slowest rank's `total_ms`."""
    return world * flop_per_step * steps / (total_ms * 1e-3) / 1e12


# ---------------------------------------------------------------- reference arm

def run_reference(args) -> int:
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from sparse_linear_attention_mean_b200 import synth
    w = synth.WORKLOADS[WORKLOAD_ID]
    inp = synth.make_inputs(w)
    qblocks = range(w.n_blocks)           # bounded sample per step: every query block of one head
    for _ in range(args.warmup):
        oracle_sample(w, inp, heads=(0,), qblocks=qblocks)
    times, flop, text = [], 0.0, ""
    for s in range(args.steps):
        dt, flop, text = oracle_sample(w, inp, heads=(s % w.H,), qblocks=qblocks)
        times.append(dt)
    tot = sum(times)
    value = flop * len(times) / tot / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / len(times),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(w),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                             "sample": text + " per step"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


# ---------------------------------------------------------------- GPU arm

def run_gpu(args) -> int:
    import torch
    import torch.distributed as dist

    from sparse_linear_attention_mean_b200 import binding as rb
    from sparse_linear_attention_mean_b200 import synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))

    w = synth.WORKLOADS[args.workload]
    if args.heads:
        w = synth.custom_workload(w, H=args.heads)
    shape = rb.Shape.of(w)
    inp = synth.make_inputs(w)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).view(torch.bfloat16).cuda()
    q, k, v, P = dev(inp["q"]), dev(inp["k"]), dev(inp["v"]), dev(inp["P"])
    gate = torch.from_numpy(inp["gate"]).cuda()
    stream = torch.cuda.current_stream()

    # the layer's own entry point
    layer = rb.Layer(shape)
    out = torch.empty((w.B, w.N, w.H, w.d), dtype=torch.bfloat16, device="cuda")
    # five events: the q/k/v pass (block means + states), scores + top-k,
    # state totals, attention
    stage_names = ("prep", "score+topk", "state_totals", "attention")
    launches_per_step = rb.layer_launches(shape)

    for _ in range(args.warmup):
        layer(q, k, v, P, gate, out=out, stream=stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()

    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(K)]
    with ClockSampler(local) as clk:
        time.sleep(0.3)
        for s in range(K):
            layer(q, k, v, P, gate, out=out, stream=stream, events=ev[s])
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    err = int(layer.dev_err.item())
    assert err == 0, f"device error flag {err}"

    per_stage = {nm: [ev[s][i].elapsed_time(ev[s][i + 1]) for s in range(K)]
                 for i, nm in enumerate(stage_names)}
    total_ms = max_over_ranks(ev[0][0].elapsed_time(ev[K - 1][4]))
    ms_step = total_ms / K
    flop = w.sparse_flops()
    value = job_tflops(flop, K, world, total_ms)

    # the same layer with the mask of an earlier step reused (cross-step
    # pattern reuse: no selection kernels; block states and attention as usual)
    idx_keep = torch.empty((w.B, w.H, w.n_blocks, w.k_b), dtype=torch.int32, device="cuda")
    layer.run_ex(q, k, v, P, gate, idx_keep, out=out, stream=stream)
    for _ in range(args.warmup):
        layer.run_ex(q, k, v, P, gate, idx_keep, reuse_mask=True, out=out, stream=stream)
    torch.cuda.synchronize()
    ev_r = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(K)]
    for s_ in range(K):
        layer.run_ex(q, k, v, P, gate, idx_keep, reuse_mask=True, out=out, stream=stream, events=ev_r[s_])
    torch.cuda.synchronize()
    assert int(layer.dev_err.item()) == 0
    reuse_ms = statistics.mean(e[0].elapsed_time(e[4]) for e in ev_r)
    reuse = {"ms_per_layer": reuse_ms, "tflops": flop / (reuse_ms * 1e-3) / 1e12,
             "stages_ms": {nm: statistics.mean(e[i].elapsed_time(e[i + 1]) for e in ev_r)
                           for i, nm in enumerate(stage_names)},
             "selection_ms_when_selecting": statistics.mean(per_stage["score+topk"])}

    # one FP8 W8A8 projection of the full attention block (x [N, 5120] ->
    # [N, 5120]: quantisation + tcgen05 GEMM), timed on its own after the layer
    fp8 = None
    if not args.no_fp8 and w.H * w.d == 5120:
        fp8 = fp8_projection(w.B * w.N, w.H * w.d, stream)

    # end to end through the host-buffer entry point (pinned host memory)
    e2e = None
    if not args.no_e2e:
        host = [x.cpu().pin_memory() for x in (q, k, v, P, gate)]
        out_h = torch.empty(out.shape, dtype=torch.bfloat16).pin_memory()
        hl = rb.HostLayer(shape)
        for _ in range(max(1, args.warmup)):
            hl(*host, out_h)
        torch.cuda.synchronize()
        K2 = max(2, min(K, 5))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(K2):
            hl(*host, out_h)
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1) / K2)
        e2e = {"value": job_tflops(flop, 1, world, e2e_ms), "unit": UNIT, "ms_per_step": e2e_ms,
               "h2d_bytes_per_step": sum(x.numel() * x.element_size() for x in host),
               "d2h_bytes_per_step": out_h.numel() * out_h.element_size()}

    if rank == 0:
        peaks = measured_peaks()
        att_ms = statistics.mean(per_stage["attention"])
        achieved = flop / (att_ms * 1e-3) / 1e12
        traffic = None
        prof = os.path.join(ROOT, "profiles", "attention_traffic.json")
        if os.path.exists(prof):
            with open(prof) as f:
                tr = json.load(f)
            if tr.get("kernel_hash") == kernel_hash():
                traffic = tr.get("bytes_per_launch")
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {**workload_config(w), "parallelism": f"replicas x{world}"},
            "kernels_ms": {nm: statistics.mean(x) for nm, x in per_stage.items()},
            "hbm": hbm_report(w, {nm: statistics.mean(x) for nm, x in per_stage.items()}, peaks),
            "attention_tflops": achieved,
            "layer_frac_of_bf16_peak": value / world / peaks["bf16_tflops"],
            "roofline": {"bound": "tensor", "kernel": "rola_attn_pair_kernel", "achieved": achieved,
                         "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": achieved / peaks["bf16_tflops"], "traffic": traffic,
                         "peak_source": peaks["source"] + " bf16 burst"},
            "e2e": e2e,
            "fp8_projection": fp8,
            "mask_reuse": reuse,
            "gpu_launches": K * launches_per_step,
            "clocks": clk.summary(),
        }
        if args.per_config and world == 1:
            flush = L2Flush()
            line["per_config"] = {str(i): config_report(i, stream, peaks, flush, 10, 50)
                                  for i in (0, 1, 2, 3)}
            line["per_config"]["4"] = block_report(stream, peaks, flush, 3, 10)
            line["training"] = backward_report(args.workload, stream, peaks, flush, 3, 10)
        if not args.no_cpu_baseline and world == 1:
            # the host-core oracle is timed at one GPU only (the multi-GPU
            # lines keep the other ranks waiting as little as possible)
            line["cpu_baseline"] = cpu_baseline(w, inp)
        print(json.dumps(line))
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def hbm_report(w, stage_ms: dict, peaks: dict) -> dict:
    """Achieved HBM bandwidth of the HBM-bound stages from their algorithmic
    bytes: the pass over q, k, v (reads q, k, v; writes the block states and
    the float64 block means) and the state totals (read the block states)."""
    act = 2.0 * w.B * w.N * w.H * w.d
    states = 4.0 * w.B * w.H * w.n_blocks * w.r * (w.d + 1)
    means = 2.0 * 8 * w.B * w.H * w.n_blocks * w.d
    out = {"peak_gbs": peaks["hbm_gbs"], "peak_source": peaks["source"] + " copy bandwidth"}
    for nm, nbytes in (("prep", 3 * act + states + means), ("state_totals", states)):
        if nm in stage_ms and stage_ms[nm] > 0:
            gbs = nbytes / (stage_ms[nm] * 1e-3) / 1e9
            out[nm] = {"bytes": nbytes, "achieved_gbs": gbs, "frac": gbs / peaks["hbm_gbs"]}
    return out


# ---------------------------------------------------------------- per-config report

def _pct(xs, q):
    return float(np.percentile(np.asarray(xs, dtype=np.float64), q))


class L2Flush:
    """Writes a 256 MB buffer (twice the 126 MB L2) so that a timed rep starts
    with nothing of its inputs in L2."""

    def __init__(self):
        import torch
        self.buf = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")

    def __call__(self, stream):
        import torch
        with torch.cuda.stream(stream):
            self.buf.fill_(1)


def _timed_reps(fn, stream, flush, warmup: int, reps: int, n_events: int = 2):
    """Runs fn(events) warmup + reps times with an L2 flush before each rep;
    returns the per-rep lists of the intervals between consecutive events."""
    import torch
    for _ in range(warmup):
        flush(stream)
        fn([torch.cuda.Event(enable_timing=True) for _ in range(n_events)])
    torch.cuda.synchronize()
    evs = []
    for _ in range(reps):
        flush(stream)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(n_events)]
        fn(ev)
        evs.append(ev)
    torch.cuda.synchronize()
    return [[ev[i].elapsed_time(ev[i + 1]) for i in range(n_events - 1)] for ev in evs]


def unit_overlap(idx: np.ndarray) -> dict:
    """Mean size of the union and of the intersection of the kept lists of the
    two query blocks (2p, 2p + 1) that the attention kernel pairs in a unit
    (padding entries -1 ignored)."""
    B, H, nb, _ = idx.shape
    uni, inter = [], []
    for b in range(B):
        for h in range(H):
            for p in range(0, nb, 2):
                a = set(int(x) for x in idx[b, h, p] if x >= 0)
                c = set(int(x) for x in idx[b, h, p + 1] if x >= 0) if p + 1 < nb else set()
                uni.append(len(a | c))
                inter.append(len(a & c))
    return {"units": len(uni), "union_mean": float(np.mean(uni)), "shared_mean": float(np.mean(inter))}


def config_report(wid: int, stream, peaks: dict, flush, warmup: int, reps: int) -> dict:
    """One attention workload through the layer entry point: ms per layer and
    per stage (p50 / p95), effective TFLOP/s of the layer and of the attention
    kernel against the bf16 peak, HBM rate of the pass over q, k, v and of the
    state totals, and the mask against the oracle's selection (mismatching rows
    outside near-ties, near-tie rows)."""
    import torch
    from oracle import rola_oracle as ro
    from sparse_linear_attention_mean_b200 import binding as rb
    from sparse_linear_attention_mean_b200 import synth
    w = synth.WORKLOADS[wid]
    shape = rb.Shape.of(w)
    inp = synth.make_inputs(w)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).view(torch.bfloat16).cuda()
    q, k, v, P = dev(inp["q"]), dev(inp["k"]), dev(inp["v"]), dev(inp["P"])
    gate = torch.from_numpy(inp["gate"]).cuda()
    layer = rb.Layer(shape)
    out = torch.empty_like(q)
    idx = torch.empty((w.B, w.H, w.n_blocks, w.k_b), dtype=torch.int32, device="cuda")
    fused = rb.layer_launches(shape) == 5
    n_ev = 5 if fused else 3
    per = _timed_reps(lambda ev: layer(q, k, v, P, gate, out=out, idx_out=idx, stream=stream, events=ev),
                      stream, flush, warmup, reps, n_ev)
    assert int(layer.dev_err.item()) == 0
    layer_ms = [sum(x) for x in per]
    att_ms = [x[-1] for x in per]
    flop = w.sparse_flops()
    rep = {"workload": w.name, "H": w.H, "d": w.d, "grid_thw": [w.T, w.Hg, w.W], "block": w.block,
           "n_blocks": w.n_blocks, "k_b": w.k_b, "rank": w.r, "flop": flop, "reps": reps, "warmup": warmup,
           "l2": "256 MB flush before each rep",
           "layer_ms_p50": _pct(layer_ms, 50), "layer_ms_p95": _pct(layer_ms, 95),
           "attention_ms_p50": _pct(att_ms, 50), "attention_ms_p95": _pct(att_ms, 95)}
    rep["layer_tflops"] = flop / (rep["layer_ms_p50"] * 1e-3) / 1e12
    rep["attention_tflops"] = flop / (rep["attention_ms_p50"] * 1e-3) / 1e12
    rep["layer_frac_of_bf16_peak"] = rep["layer_tflops"] / peaks["bf16_tflops"]
    rep["attention_frac_of_bf16_peak"] = rep["attention_tflops"] / peaks["bf16_tflops"]
    if fused:
        names = ("prep", "score+topk", "state_totals", "attention")
        rep["stages_ms_p50"] = {nm: _pct([x[i] for x in per], 50) for i, nm in enumerate(names)}
        rep["hbm"] = hbm_report(w, rep["stages_ms_p50"], peaks)
    else:
        rep["stages_ms_p50"] = {"select+states": _pct([x[0] for x in per], 50),
                                "attention": _pct([x[1] for x in per], 50)}
    idx_ref, sig = ro.select_all(inp, w.block, w.k_b)
    got = idx.cpu().numpy()
    ties = bad = n_tie_rows = 0
    for b in range(w.B):
        for h in range(w.H):
            tie_rows = set(ro.near_ties(sig[b, h], w.k_b))
            n_tie_rows += len(tie_rows)
            for a in np.nonzero((got[b, h] != idx_ref[b, h]).any(axis=1))[0]:
                if int(a) in tie_rows:
                    ties += 1
                else:
                    bad += 1
    rep["mask"] = {"rows": int(w.B * w.H * w.n_blocks), "mismatch_outside_near_ties": bad,
                   "near_tie_rows": n_tie_rows, "differing_near_tie_rows": ties}
    rep["unit_lists"] = unit_overlap(got)
    del q, k, v, out, layer
    torch.cuda.empty_cache()
    return rep


def backward_report(wid: int, stream, peaks: dict, flush, warmup: int, reps: int, heads: int = 0) -> dict:
    """Training on one attention workload: the training forward (which also
    saves the output residual, log-sum-exp and linear denominator) and the
    backward (transposed mask, query-major and key-major tcgen05 passes,
    fixed-order reductions), each timed alone with an L2 flush before every
    rep.  TFLOP/s count the kept pairs' contractions as the usual dense
    accounting does: 2 per pair forward, 5 backward (S recomputed, dP, dQ,
    dK, dV); the two-pass backward executes 7 (S and dP in both passes)."""
    import ctypes

    import torch
    from sparse_linear_attention_mean_b200 import binding as rb
    from sparse_linear_attention_mean_b200 import synth
    w = synth.WORKLOADS[wid]
    if heads:
        w = synth.custom_workload(w, H=heads)
    shape = rb.Shape.of(w)
    inp = synth.make_inputs(w)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).view(torch.bfloat16).cuda()
    q, k, v, P = dev(inp["q"]), dev(inp["k"]), dev(inp["v"]), dev(inp["P"])
    gate = torch.from_numpy(inp["gate"]).cuda()
    dout = dev(synth.make_normal_bf16((w.B, w.N, w.H, w.d), seed=w.seed + 50, stream=7))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    idx = rb.select_blocks(shape, q, k, stream=stream)
    states = rb.block_states(shape, k, v, P, stream=stream)
    fwd = rb.attention_fwd_train(shape, q, k, v, idx, P, states, gate, dev_err=err, stream=stream)
    grads = rb.attention_bwd(shape, q, k, v, idx, P, states, gate, *fwd, dout, dev_err=err, stream=stream)
    ws = torch.empty(rb.lib().rola_attention_bwd_workspace_bytes(ctypes.byref(shape.c())),
                     dtype=torch.uint8, device="cuda")

    def f_fwd(ev):
        ev[0].record(stream)
        rb.attention_fwd_train(shape, q, k, v, idx, P, states, gate, dev_err=err, stream=stream)
        ev[1].record(stream)

    def f_bwd(ev):
        ev[0].record(stream)
        rb.attention_bwd(shape, q, k, v, idx, P, states, gate, *fwd, dout, dev_err=err, stream=stream,
                         workspace=ws, grads=grads)
        ev[1].record(stream)

    t_f = [x[0] for x in _timed_reps(f_fwd, stream, flush, warmup, reps)]
    t_b = [x[0] for x in _timed_reps(f_bwd, stream, flush, warmup, reps)]
    assert int(err.item()) == 0
    flop_fwd = w.sparse_flops()
    rep = {"workload": w.name, "H": w.H, "reps": reps, "warmup": warmup, "l2": "256 MB flush before each rep",
           "train_forward_ms_p50": _pct(t_f, 50), "train_forward_ms_p95": _pct(t_f, 95),
           "backward_ms_p50": _pct(t_b, 50), "backward_ms_p95": _pct(t_b, 95)}
    rep["train_forward_tflops"] = flop_fwd / (rep["train_forward_ms_p50"] * 1e-3) / 1e12
    rep["backward_tflops"] = 2.5 * flop_fwd / (rep["backward_ms_p50"] * 1e-3) / 1e12
    rep["backward_tflops_executed"] = 3.5 * flop_fwd / (rep["backward_ms_p50"] * 1e-3) / 1e12
    rep["backward_frac_of_bf16_peak"] = rep["backward_tflops"] / peaks["bf16_tflops"]
    del q, k, v, P, dout, fwd, grads, ws, states, idx
    torch.cuda.empty_cache()
    return rep


def block_report(stream, peaks: dict, flush, warmup: int, reps: int) -> dict:
    """The full 14B-720P attention block (x [75600, 5120]): per-token
    quantisation + the Q, K, V W8A8 projections, the RoLA layer, quantisation
    + the output projection; and the block's FFN (5120 -> 13824 -> 5120, W8A8,
    GELU).  ms p50 / p95 per part, the GEMMs' effective TFLOP/s against the
    FP8 peak (2 x the measured bf16 peak, the nominal ratio)."""
    import torch
    from sparse_linear_attention_mean_b200 import binding as rb
    from sparse_linear_attention_mean_b200 import synth
    w = synth.WORKLOADS[4]
    inp = synth.make_block_inputs(w)
    M, D = w.B * w.N, w.model_dim
    x = torch.from_numpy(np.ascontiguousarray(inp["x"])).view(torch.bfloat16).cuda()
    wts = {nm: rb.fp8_quantize_weight(torch.from_numpy(np.ascontiguousarray(inp[nm])).cuda())
           for nm in ("Wq", "Wk", "Wv", "Wo")}
    P = torch.from_numpy(np.ascontiguousarray(inp["P"])).view(torch.bfloat16).cuda()
    gate = torch.from_numpy(inp["gate"]).cuda()
    shape = rb.Shape.of(w)
    layer = rb.Layer(shape)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    qkv = {nm: torch.empty((M, D), dtype=torch.bfloat16, device="cuda") for nm in ("Wq", "Wk", "Wv")}
    o = torch.empty((M, D), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((M, D), dtype=torch.bfloat16, device="cuda")
    xq = torch.empty((M, D), dtype=torch.uint8, device="cuda")
    xs = torch.empty((M,), dtype=torch.float32, device="cuda")
    lib = rb.lib()
    import ctypes
    P_ = lambda t: ctypes.c_void_p(t.data_ptr())
    cs = ctypes.c_void_p(stream.cuda_stream)

    def quant(src):
        assert lib.fp8_quantize_rows_bf16(M, D, P_(src), P_(xq), P_(xs), cs) == 0

    def gemm(wq, ws, dst):
        assert lib.fp8_gemm_w8a8(M, D, D, P_(xq), P_(xs), P_(wq), P_(ws), P_(dst), P_(err), cs) == 0

    idx = torch.empty((w.B, w.H, w.n_blocks, w.k_b), dtype=torch.int32, device="cuda")

    def step(ev):
        ev[0].record(stream)
        quant(x)
        for nm in ("Wq", "Wk", "Wv"):
            gemm(*wts[nm], qkv[nm])
        ev[1].record(stream)
        layer(qkv["Wq"].view(w.B, w.N, w.H, w.d), qkv["Wk"].view(w.B, w.N, w.H, w.d),
              qkv["Wv"].view(w.B, w.N, w.H, w.d), P, gate, out=o.view(w.B, w.N, w.H, w.d), idx_out=idx,
              stream=stream)
        ev[2].record(stream)
        quant(o)
        gemm(*wts["Wo"], y)
        ev[3].record(stream)

    per = _timed_reps(step, stream, flush, warmup, reps, 4)
    assert int(err.item()) == 0 and int(layer.dev_err.item()) == 0
    fp8_peak = 2.0 * peaks["bf16_tflops"]
    gflop = 2.0 * M * D * D
    names = ("quant+qkv_gemms", "rola_layer", "quant+out_gemm")
    rep = {"workload": w.name, "reps": reps, "warmup": warmup, "l2": "256 MB flush before each rep",
           "fp8_peak_tflops": fp8_peak,
           "fp8_peak_source": peaks["source"] + " bf16 burst x 2 (nominal fp8:bf16 ratio)"}
    for i, nm in enumerate(names):
        rep[nm + "_ms_p50"] = _pct([x[i] for x in per], 50)
        rep[nm + "_ms_p95"] = _pct([x[i] for x in per], 95)
    tot = [sum(x) for x in per]
    rep["block_ms_p50"], rep["block_ms_p95"] = _pct(tot, 50), _pct(tot, 95)
    rep["qkv_tflops"] = 3 * gflop / (rep["quant+qkv_gemms_ms_p50"] * 1e-3) / 1e12
    rep["qkv_frac_of_fp8_peak"] = rep["qkv_tflops"] / fp8_peak
    rep["out_tflops"] = gflop / (rep["quant+out_gemm_ms_p50"] * 1e-3) / 1e12
    rep["out_frac_of_fp8_peak"] = rep["out_tflops"] / fp8_peak
    rep["unit_lists"] = unit_overlap(idx.cpu().numpy())
    del qkv, o, layer, idx
    torch.cuda.empty_cache()
    # the block's FFN
    ffw = synth.make_ffn_weights(w)
    F = ffw["W1"].shape[0]
    w1q, w1s = rb.fp8_quantize_weight(torch.from_numpy(ffw["W1"]).cuda())
    w2q, w2s = rb.fp8_quantize_weight(torch.from_numpy(ffw["W2"]).cuda())
    ws_ffn = torch.empty(lib.fp8_ffn_workspace_bytes(M, D, F), dtype=torch.uint8, device="cuda")

    def ffn(ev):
        ev[0].record(stream)
        rb.fp8_ffn(x, w1q, w1s, w2q, w2s, out=y, workspace=ws_ffn, dev_err=err, stream=stream)
        ev[1].record(stream)

    per = _timed_reps(ffn, stream, flush, max(1, warmup // 2), max(3, reps // 3), 2)
    assert int(err.item()) == 0
    ffn_ms = [x[0] for x in per]
    ffn_flop = 2 * 2.0 * M * D * F
    rep["ffn"] = {"shape_m_d_f": [M, D, F], "activation": "gelu_tanh",
                  "ms_p50": _pct(ffn_ms, 50), "ms_p95": _pct(ffn_ms, 95),
                  "tflops": ffn_flop / (_pct(ffn_ms, 50) * 1e-3) / 1e12}
    rep["ffn"]["frac_of_fp8_peak"] = rep["ffn"]["tflops"] / fp8_peak
    del ws_ffn
    torch.cuda.empty_cache()
    return rep


def fp8_projection(M: int, D: int, stream, reps: int = 5) -> dict:
    """Times fp8_linear_w8a8 (per-token quantisation + W8A8 GEMM) for x [M, D]
    bf16 ~ N(0, 1) and W [D, D] ~ N(0, 1/D), and the GEMM alone."""
    import torch
    from sparse_linear_attention_mean_b200 import binding as rb
    g = torch.Generator(device="cuda")
    g.manual_seed(4)
    x = torch.randn((M, D), generator=g, device="cuda").to(torch.bfloat16)
    W = torch.randn((D, D), generator=g, device="cuda") / D ** 0.5
    wq, ws = rb.fp8_quantize_weight(W)
    xq, xs = rb.fp8_quantize_rows(x)
    y = torch.empty((M, D), dtype=torch.bfloat16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws_buf = torch.empty(rb.lib().fp8_linear_workspace_bytes(M, D), dtype=torch.uint8, device="cuda")

    def timed(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    gemm_ms = timed(lambda: rb.fp8_gemm(xq, xs, wq, ws, out=y, dev_err=err, stream=stream))
    lin_ms = timed(lambda: rb.fp8_linear(x, wq, ws, out=y, workspace=ws_buf, dev_err=err, stream=stream))
    assert int(err.item()) == 0
    flop = 2.0 * M * D * D
    peaks = measured_peaks()
    fp8_peak = 2.0 * peaks["bf16_tflops"]
    return {"shape_mnk": [M, D, D], "gemm_ms": gemm_ms, "linear_ms": lin_ms,
            "gemm_tflops": flop / gemm_ms / 1e9, "linear_tflops": flop / lin_ms / 1e9,
            "fp8_peak_tflops": fp8_peak,
            "peak_source": peaks["source"] + " bf16 burst x 2 (nominal fp8:bf16 ratio)",
            "gemm_frac": flop / gemm_ms / 1e9 / fp8_peak}


def kernel_hash() -> str:
    """Hash of the attention kernel's source code with comments and blank
    lines removed: it changes when the code does, not when a comment does."""
    import hashlib
    import re
    h = hashlib.sha1()
    for nm in ("rola_attention.cu", "rola_attention_pair.cu", "rola_common.cuh"):
        with open(os.path.join(ROOT, "sparse_linear_attention_mean_b200", "csrc", nm)) as f:
            src = f.read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        code = "\n".join(line.rstrip() for line in src.splitlines() if line.strip())
        h.update(code.encode())
    return h.hexdigest()[:12]


def main() -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer pass (profiling runs)")
    ap.add_argument("--no-fp8", action="store_true", help="skip the FP8 projection timing")
    ap.add_argument("--per-config", dest="per_config", action="store_true", default=True,
                    help="add the per-workload report (default at one GPU)")
    ap.add_argument("--no-per-config", dest="per_config", action="store_false")
    ap.add_argument("--fp8-only", action="store_true",
                    help="time only the FP8 projection (x [rows, 5120] -> [rows, 5120]); profiling captures")
    ap.add_argument("--fp8-rows", type=int, default=75600, help="rows of x for --fp8-only")
    ap.add_argument("--training-only", action="store_true",
                    help="time only the training forward and the backward of --workload; profiling captures")
    ap.add_argument("--heads", type=int, default=0,
                    help="override the head count (per-head work unchanged; for profiling captures)")
    ap.add_argument("--workload", type=int, default=WORKLOAD_ID,
                    help="attention workload id of synth.WORKLOADS (profiling of smaller cases)")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.fp8_only:
        import torch
        print(json.dumps({"fp8_projection": fp8_projection(args.fp8_rows, 5120, torch.cuda.current_stream())}))
        return 0
    if args.training_only:
        import torch
        stream = torch.cuda.current_stream()
        print(json.dumps({"training": backward_report(args.workload, stream, measured_peaks(), L2Flush(),
                                                      args.warmup, args.steps, args.heads)}))
        return 0
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
