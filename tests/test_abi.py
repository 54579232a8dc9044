"""The C ABI: the library loads without a GPU, exports every entry point the
header declares, and rejects bad arguments on the host before any launch."""
import ctypes
import os
import re

import pytest

from sparse_linear_attention_mean_b200 import binding as rb
from sparse_linear_attention_mean_b200 import build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "rola.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return rb.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b([a-z][a-z0-9_]*)\s*\(", text)) - {"defined"})


def test_header_declares_binding_exports():
    assert declared_functions() == sorted(rb.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings_and_kb_rule(lib):
    for s in range(6):
        assert lib.rola_status_string(s)
    assert rb.kb_from_sparsity(100, 970) == 3
    assert rb.kb_from_sparsity(591, 970) == 18
    assert rb.kb_from_sparsity(256, 900) == 26
    assert rb.kb_from_sparsity(16, 750) == 4
    assert rb.kb_from_sparsity(0, 970) == -1
    assert rb.kb_from_sparsity(10, 1000) == -1


def test_num_blocks_and_workspace_sizes(lib):
    s = rb.Shape(1, 40, 128, 21, 45, 80, 128, 18, 32)
    assert rb.num_blocks(s) == 591
    cs = s.c()
    assert lib.rola_layer_workspace_bytes(ctypes.byref(cs)) > lib.rola_select_workspace_bytes(ctypes.byref(cs)) > 0
    assert lib.rola_workspace_bytes(ctypes.byref(cs)) == lib.rola_select_workspace_bytes(ctypes.byref(cs))
    # pooled q and k means and the scores, float64, each rounded up to 256 bytes
    r256 = lambda n: -(-n // 256) * 256
    assert lib.rola_select_workspace_bytes(ctypes.byref(cs)) == r256(2 * 40 * 591 * 128 * 8) + r256(40 * 591 * 591 * 8)
    bad = rb.Shape(1, 40, 128, 21, 45, 80, 128, 592, 32).c()   # k_b > n_blocks
    assert lib.rola_layer_workspace_bytes(ctypes.byref(bad)) == 0
    assert lib.rola_workspace_bytes(ctypes.byref(bad)) == 0


@pytest.mark.parametrize("field,value,status", [
    ("N", 123, 1),          # N != T*Hg*W
    ("B", 0, 1),            # empty batch
    ("H", 0, 1),            # no heads
    ("T", 0, 1),            # empty grid
    ("W", -4, 1),
    ("k_b", 0, 1),
    ("k_b", 10_000, 1),
    ("r", 3, 1),            # odd rank
    ("d", 96, 2),           # valid but no kernel
    ("block", 32, 2),
    ("rope_base", -1.0, 1),
])
def test_bad_shapes_rejected_on_host(lib, field, value, status):
    cs = rb.Shape(1, 2, 64, 4, 16, 16, 64, 4, 16).c()
    setattr(cs, field, value)
    dummy = ctypes.c_void_p(256)
    st = lib.rola_block_states(ctypes.byref(cs), dummy, dummy, dummy, dummy, dummy, dummy, dummy, None)
    assert st == status


def test_null_and_misaligned_pointers_rejected(lib):
    cs = rb.Shape(1, 2, 64, 4, 16, 16, 64, 4, 16).c()
    ok = ctypes.c_void_p(4096)
    assert lib.rola_block_states(ctypes.byref(cs), None, ok, ok, ok, ok, ok, ok, None) == 1
    odd = ctypes.c_void_p(4097)
    assert lib.rola_block_states(ctypes.byref(cs), odd, ok, ok, ok, ok, ok, ok, None) == 5
    assert lib.rola_select_blocks(ctypes.byref(cs), ok, ok, ok, None, None, 0, None) == 3  # no workspace
    assert lib.fp8_quantize_rows_bf16(4, 15, ok, ok, ok, None) == 1                          # K % 16


def test_bounded_attention_arguments_rejected_on_host(lib):
    """The attention entry with an explicit wait bound checks its arguments
    like the default one before any launch."""
    cs = rb.Shape(1, 2, 64, 4, 16, 16, 64, 4, 16).c()
    ok = ctypes.c_void_p(4096)
    odd = ctypes.c_void_p(4097)
    fn = lib.rola_attention_fwd_bounded
    args = [ok] * 12
    assert fn(ctypes.byref(cs), *args[:3], None, *args[4:], ctypes.c_uint64(0), None) == 1  # null idx
    assert fn(ctypes.byref(cs), odd, *args[1:], ctypes.c_uint64(0), None) == 5               # misaligned q
    bad = rb.Shape(1, 2, 64, 4, 16, 16, 64, 17, 16).c()                                      # k_b > n_blocks
    assert fn(ctypes.byref(bad), *args, ctypes.c_uint64(10**9), None) == 1


def test_fp8_gemm_arguments_rejected_on_host(lib):
    ok = ctypes.c_void_p(4096)
    odd = ctypes.c_void_p(4104)  # 8-byte aligned only
    gemm = lib.fp8_gemm_w8a8
    assert gemm(64, 40, 64, ok, ok, ok, ok, ok, None, None) == 1    # N % 32
    assert gemm(64, 64, 24, ok, ok, ok, ok, ok, None, None) == 1    # K % 16
    assert gemm(0, 64, 64, ok, ok, ok, ok, ok, None, None) == 1     # empty M
    assert gemm(64, 64, 64, None, ok, ok, ok, ok, None, None) == 1  # null operand
    assert gemm(64, 64, 64, odd, ok, ok, ok, ok, None, None) == 5   # misaligned codes
    assert gemm(64, 64, 64, ok, ok, ok, odd, ok, None, None) == 5   # misaligned w_scale
    assert lib.fp8_linear_w8a8(64, 64, 64, ok, ok, ok, ok, None, 0, None, None) == 3  # no workspace
    act = lib.fp8_gemm_w8a8_act
    assert act(64, 64, 64, ok, ok, ok, ok, 2, ok, None, None) == 1       # unknown activation
    assert act(64, 40, 64, ok, ok, ok, ok, 1, ok, None, None) == 1       # N % 32
    ffn = lib.fp8_ffn_w8a8
    assert ffn(64, 64, 96, ok, ok, ok, ok, ok, ok, None, 0, None, None) == 3    # no workspace
    assert ffn(64, 64, 100, ok, ok, ok, ok, ok, ok, ok, 1 << 30, None, None) == 1  # F % 32
    assert ffn(64, 64, 96, ok, ok, ok, None, ok, ok, ok, 1 << 30, None, None) == 1  # null w2
    r256 = lambda n: -(-n // 256) * 256
    M, D, F = 75600, 5120, 13824
    assert lib.fp8_ffn_workspace_bytes(M, D, F) == (r256(M * D) + r256(4 * M) + r256(2 * M * F)
                                                    + r256(M * F) + r256(4 * M))


def test_timed_layer_event_count_checked_on_host(lib):
    cs = rb.Shape(1, 2, 64, 4, 16, 16, 64, 4, 16).c()
    ok = ctypes.c_void_p(4096)
    ev = (ctypes.c_void_p * 4)(4096, 4096, 4096, 4096)
    st = lib.rola_layer_fwd_timed(ctypes.byref(cs), ok, ok, ok, ok, ok, ok, None, ok, 1 << 30, None, None, ev, 4)
    assert st == 1  # ROLA_ERR_INVALID_ARG: three or five events


@pytest.mark.parametrize("H,d,r,block,T,Hg,W,kb", [
    (40, 128, 32, 128, 21, 45, 80, 18),   # 5 groups of 8 heads
    (12, 128, 32, 128, 21, 30, 52, 26),   # 8 + 4 heads
    (2, 64, 16, 64, 4, 16, 16, 4),        # one group of 2 heads (d = 64 groups hold 16)
])
def test_host_workspace_is_two_group_slots(lib, H, d, r, block, T, Hg, W, kb):
    """The host-buffer layer stages P and gate of all heads, two slots of
    q, k, v, out for one head group (2 KB of each token row), and the layer
    workspace of one group."""
    r256 = lambda n: -(-n // 256) * 256
    s = rb.Shape(1, H, d, T, Hg, W, block, kb, r)
    hc = min(H, -(-2048 // (2 * d)))
    g = rb.Shape(1, hc, d, T, Hg, W, block, kb, r)
    act = r256(s.N * hc * d * 2)
    want = (r256(H * d * r * 2) + r256(H * 4) + 8 * act
            + lib.rola_layer_workspace_bytes(ctypes.byref(g.c())))
    assert lib.rola_layer_host_workspace_bytes(ctypes.byref(s.c())) == want


def test_binding_constants_match_the_header():
    text = open(HEADER).read()
    enum = dict((int(v), n) for n, v in re.findall(r"\b(ROLA_(?:OK|ERR_\w+))\s*=\s*(\d+)", text))
    assert sorted(enum) == sorted(rb.STATUS)
    defines = dict(re.findall(r"#define\s+ROLA_DEVERR_(\w+)\s+(0x[0-9a-fA-F]+)", text))
    assert int(defines["BAD_INDEX"], 16) == rb.DEVERR_BAD_INDEX
    assert int(defines["TIMEOUT"], 16) == rb.DEVERR_TIMEOUT
    acts = dict(re.findall(r"#define\s+ROLA_ACT_(\w+)\s+(\d+)", text))
    assert int(acts["NONE"]) == rb.ACT_NONE and int(acts["GELU_TANH"]) == rb.ACT_GELU_TANH
