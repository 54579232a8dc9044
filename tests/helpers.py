"""Shared test plumbing: moving seeded inputs to the device and comparing
GPU results with the oracle under the stated tolerances."""
import numpy as np
import torch

from oracle import rola_oracle as ro
from sparse_linear_attention_mean_b200 import binding as rb
from sparse_linear_attention_mean_b200 import synth

# attention outputs: |err| <= ATOL + RTOL * |ref| per element (bf16 in,
# fp32 accumulate, bf16 out)
ATOL = 1e-2
RTOL = 1e-2


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits)).view(torch.bfloat16).cuda()


def dev_inputs(inp: dict):
    return (dev_bf16(inp["q"]), dev_bf16(inp["k"]), dev_bf16(inp["v"]), dev_bf16(inp["P"]),
            torch.from_numpy(inp["gate"]).cuda())


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def check_close(got: np.ndarray, ref: np.ndarray, atol=ATOL, rtol=RTOL, what=""):
    err = np.abs(got - ref)
    bound = atol + rtol * np.abs(ref)
    bad = ~(err <= bound)
    if bad.any():
        i = np.unravel_index(np.argmax(np.where(bad, err / bound, 0)), err.shape)
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} elements out of tolerance; worst at "
                             f"{i}: got {got[i]!r} ref {ref[i]!r} (bound {bound[i]:.3g})")
    return float((err / bound).max()) if err.size else 0.0


def mask_mismatch(idx_gpu: np.ndarray, idx_ref: np.ndarray, sigma: np.ndarray, k_b: int):
    """Rows whose kept sets differ, split into (allowed near-tie rows, other rows)."""
    B, H, nb, _ = idx_ref.shape
    tie_rows, bad_rows = [], []
    for b in range(B):
        for h in range(H):
            diff = np.nonzero((idx_gpu[b, h] != idx_ref[b, h]).any(axis=1))[0]
            if len(diff) == 0:
                continue
            ties = set(ro.near_ties(sigma[b, h], k_b))
            for a in diff:
                (tie_rows if a in ties else bad_rows).append((b, h, int(a)))
    return tie_rows, bad_rows
