"""The selector entry point without a caller workspace
(rola_select_blocks_noalloc), through the C ABI.  Collected last, so that it
runs both alone and after every other test in the session: its scratch is a
fixed device array that earlier calls of other entry points never touch."""
import ctypes

import numpy as np
import pytest
import torch

from sparse_linear_attention_mean_b200 import binding as rb
from sparse_linear_attention_mean_b200 import synth

from helpers import dev_inputs

ROLA_ERR_WORKSPACE = 3


def test_noalloc_rejects_shapes_beyond_its_scratch():
    """Host-side check, no GPU needed: the 14B-720P selector needs ~160 MB of
    scratch, far over the fixed 16 MiB."""
    cs = rb.Shape.of(synth.WORKLOADS[3]).c()
    ok = ctypes.c_void_p(4096)
    assert rb.lib().rola_select_blocks_noalloc(ctypes.byref(cs), ok, ok, ok, None) == ROLA_ERR_WORKSPACE


@pytest.mark.gpu
@pytest.mark.parametrize("cfg", [0, 1])
def test_noalloc_matches_workspace_entry(cfg):
    w = synth.WORKLOADS[cfg]
    inp = synth.make_inputs(w)
    shape = rb.Shape.of(w)
    q, k, v, P, gate = dev_inputs(inp)
    ref = rb.select_blocks(shape, q, k)  # the workspace entry point
    cs = shape.c()
    stream = torch.cuda.current_stream()
    for call in range(2):  # the first call sets up, the second reuses the scratch
        idx = torch.full((w.B, w.H, w.n_blocks, w.k_b), -7, dtype=torch.int32, device="cuda")
        st = rb.lib().rola_select_blocks_noalloc(ctypes.byref(cs), ctypes.c_void_p(q.data_ptr()),
                                                 ctypes.c_void_p(k.data_ptr()),
                                                 ctypes.c_void_p(idx.data_ptr()),
                                                 ctypes.c_void_p(stream.cuda_stream))
        assert st == 0, rb.lib().rola_status_string(st)
        torch.cuda.synchronize()
        assert torch.equal(idx, ref), f"call {call}"
    # different inputs through the same scratch: still the workspace result
    q2 = torch.flip(q, dims=[1]).contiguous()
    ref2 = rb.select_blocks(shape, q2, k)
    idx2 = torch.empty_like(ref2)
    st = rb.lib().rola_select_blocks_noalloc(ctypes.byref(cs), ctypes.c_void_p(q2.data_ptr()),
                                             ctypes.c_void_p(k.data_ptr()), ctypes.c_void_p(idx2.data_ptr()),
                                             ctypes.c_void_p(stream.cuda_stream))
    assert st == 0
    torch.cuda.synchronize()
    assert torch.equal(idx2, ref2)
    assert not np.array_equal(ref2.cpu().numpy(), ref.cpu().numpy())
