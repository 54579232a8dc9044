"""Thin ctypes binding of librola.so (declared in include/rola.h).

Argument marshalling only: every step of the computation runs in the
library's CUDA kernels.  torch supplies device memory and the current stream.
There is no fallback: if librola.so is missing or a call fails, this raises.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "librola.so")

STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported shape", 3: "workspace",
          4: "CUDA error", 5: "alignment"}
DEVERR_BAD_INDEX = 0x1
DEVERR_TIMEOUT = 0x2
ACT_NONE = 0
ACT_GELU_TANH = 1

EXPORTS = [
    "rola_status_string", "rola_num_blocks", "rola_kb_from_sparsity",
    "rola_select_workspace_bytes", "rola_workspace_bytes", "rola_select_blocks", "rola_select_blocks_noalloc",
    "rola_block_states",
    "rola_attention_fwd", "rola_attention_fwd_bounded", "rola_layer_workspace_bytes", "rola_layer_fwd", "rola_layer_fwd_timed",
    "rola_layer_kernel_launches", "rola_layer_fwd_ex",
    "rola_attention_fwd_train", "rola_attention_bwd_workspace_bytes", "rola_attention_bwd",
    "rola_layer_host_workspace_bytes", "rola_layer_fwd_host",
    "fp8_quantize_rows_bf16", "fp8_quantize_weight", "fp8_gemm_w8a8", "fp8_gemm_w8a8_act",
    "fp8_linear_workspace_bytes", "fp8_linear_w8a8", "fp8_ffn_workspace_bytes", "fp8_ffn_w8a8",
]


class LayerOpts(ctypes.Structure):
    _fields_ = [("kb_per_head", ctypes.c_void_p), ("reuse_mask", ctypes.c_int32)]


class RolaShape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("d", ctypes.c_int32),
                ("N", ctypes.c_int32), ("T", ctypes.c_int32), ("Hg", ctypes.c_int32),
                ("W", ctypes.c_int32), ("block", ctypes.c_int32), ("k_b", ctypes.c_int32),
                ("r", ctypes.c_int32), ("rope_base", ctypes.c_float)]


@dataclasses.dataclass(frozen=True)
class Shape:
    B: int
    H: int
    d: int
    T: int
    Hg: int
    W: int
    block: int
    k_b: int
    r: int
    rope_base: float = 10000.0

    @property
    def N(self) -> int:
        return self.T * self.Hg * self.W

    @property
    def n_blocks(self) -> int:
        return -(-self.N // self.block)

    def c(self) -> RolaShape:
        return RolaShape(self.B, self.H, self.d, self.N, self.T, self.Hg, self.W, self.block,
                         self.k_b, self.r, self.rope_base)

    @staticmethod
    def of(w) -> "Shape":
        """From any object with the workload fields (B, H, d, T, Hg, W, block, k_b, r)."""
        return Shape(w.B, w.H, w.d, w.T, w.Hg, w.W, w.block, w.k_b, w.r,
                     float(getattr(w, "rope_base", 10000.0)))


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m sparse_linear_attention_mean_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
        sp = ctypes.POINTER(RolaShape)
        L.rola_status_string.restype = ctypes.c_char_p
        L.rola_status_string.argtypes = [ctypes.c_int]
        L.rola_num_blocks.restype = i32
        L.rola_num_blocks.argtypes = [sp]
        L.rola_kb_from_sparsity.restype = i32
        L.rola_kb_from_sparsity.argtypes = [i32, i32]
        for nm in ("rola_select_workspace_bytes", "rola_workspace_bytes", "rola_layer_workspace_bytes",
                   "rola_layer_host_workspace_bytes"):
            getattr(L, nm).restype = sz
            getattr(L, nm).argtypes = [sp]
        L.rola_select_blocks.restype = ctypes.c_int
        L.rola_select_blocks.argtypes = [sp, vp, vp, vp, vp, vp, sz, vp]
        L.rola_select_blocks_noalloc.restype = ctypes.c_int
        L.rola_select_blocks_noalloc.argtypes = [sp, vp, vp, vp, vp]
        L.rola_block_states.restype = ctypes.c_int
        L.rola_block_states.argtypes = [sp, vp, vp, vp, vp, vp, vp, vp, vp]
        L.rola_attention_fwd.restype = ctypes.c_int
        L.rola_attention_fwd.argtypes = [sp] + [vp] * 12 + [vp]
        L.rola_attention_fwd_bounded.restype = ctypes.c_int
        L.rola_attention_fwd_bounded.argtypes = [sp] + [vp] * 12 + [ctypes.c_uint64, vp]
        L.rola_layer_fwd.restype = ctypes.c_int
        L.rola_layer_fwd.argtypes = [sp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp, vp]
        L.rola_layer_fwd_timed.restype = ctypes.c_int
        L.rola_layer_fwd_timed.argtypes = [sp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp, vp,
                                           ctypes.POINTER(ctypes.c_void_p), i32]
        L.rola_layer_fwd_ex.restype = ctypes.c_int
        L.rola_layer_fwd_ex.argtypes = [sp, ctypes.POINTER(LayerOpts), vp, vp, vp, vp, vp, vp, vp, vp, sz, vp,
                                        vp, ctypes.POINTER(ctypes.c_void_p), i32]
        L.rola_attention_fwd_train.restype = ctypes.c_int
        L.rola_attention_fwd_train.argtypes = [sp] + [vp] * 15 + [vp]
        L.rola_attention_bwd_workspace_bytes.restype = sz
        L.rola_attention_bwd_workspace_bytes.argtypes = [sp]
        L.rola_attention_bwd.restype = ctypes.c_int
        L.rola_attention_bwd.argtypes = [sp] + [vp] * 20 + [vp, sz, vp, vp]
        L.rola_layer_kernel_launches.restype = ctypes.c_int
        L.rola_layer_kernel_launches.argtypes = [sp]
        L.rola_layer_fwd_host.restype = ctypes.c_int
        L.rola_layer_fwd_host.argtypes = [sp, vp, vp, vp, vp, vp, vp, vp, sz, vp, vp]
        L.fp8_quantize_rows_bf16.restype = ctypes.c_int
        L.fp8_quantize_rows_bf16.argtypes = [i32, i32, vp, vp, vp, vp]
        L.fp8_quantize_weight.restype = ctypes.c_int
        L.fp8_quantize_weight.argtypes = [i32, i32, vp, vp, vp, vp]
        L.fp8_gemm_w8a8.restype = ctypes.c_int
        L.fp8_gemm_w8a8.argtypes = [i32, i32, i32, vp, vp, vp, vp, vp, vp, vp]
        L.fp8_linear_workspace_bytes.restype = sz
        L.fp8_linear_workspace_bytes.argtypes = [i32, i32]
        L.fp8_linear_w8a8.restype = ctypes.c_int
        L.fp8_linear_w8a8.argtypes = [i32, i32, i32, vp, vp, vp, vp, vp, sz, vp, vp]
        L.fp8_gemm_w8a8_act.restype = ctypes.c_int
        L.fp8_gemm_w8a8_act.argtypes = [i32, i32, i32, vp, vp, vp, vp, i32, vp, vp, vp]
        L.fp8_ffn_workspace_bytes.restype = sz
        L.fp8_ffn_workspace_bytes.argtypes = [i32, i32, i32]
        L.fp8_ffn_w8a8.restype = ctypes.c_int
        L.fp8_ffn_w8a8.argtypes = [i32, i32, i32, vp, vp, vp, vp, vp, vp, vp, sz, vp, vp]
        _lib = L
    return _lib


class RolaError(RuntimeError):
    pass


def _check(status: int, what: str):
    if status != 0:
        msg = lib().rola_status_string(status).decode()
        raise RolaError(f"{what}: {msg} (status {status})")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need(t: torch.Tensor, dtype, shape, name: str):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")


def _ws(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(1, nbytes), dtype=torch.uint8, device=device)


def num_blocks(shape: Shape) -> int:
    return int(lib().rola_num_blocks(ctypes.byref(shape.c())))


def kb_from_sparsity(n_blocks: int, sparsity_permille: int) -> int:
    return int(lib().rola_kb_from_sparsity(n_blocks, sparsity_permille))


# ------------------------------------------------------------------ RoLA

def select_blocks(shape: Shape, q, k, *, scores: bool = False, stream=None):
    """Kept key blocks per query block, int32 [B, H, n_blocks, k_b] ascending
    (and the float64 block scores if ``scores``)."""
    act = (shape.B, shape.N, shape.H, shape.d)
    _need(q, torch.bfloat16, act, "q")
    _need(k, torch.bfloat16, act, "k")
    nb = shape.n_blocks
    idx = torch.empty((shape.B, shape.H, nb, shape.k_b), dtype=torch.int32, device=q.device)
    sc = torch.empty((shape.B, shape.H, nb, nb), dtype=torch.float64, device=q.device) if scores else None
    cs = shape.c()
    ws_bytes = lib().rola_select_workspace_bytes(ctypes.byref(cs))
    ws = _ws(ws_bytes, q.device)
    _check(lib().rola_select_blocks(ctypes.byref(cs), _ptr(q), _ptr(k), _ptr(idx), _ptr(sc),
                                    _ptr(ws), ws_bytes, _stream(stream)), "rola_select_blocks")
    return (idx, sc) if scores else idx


def block_states(shape: Shape, k, v, P, *, stream=None):
    """(S_blk [B,H,nb,r,d], z_blk [B,H,nb,r], S_glb [B,H,r,d], z_glb [B,H,r]) fp32."""
    act = (shape.B, shape.N, shape.H, shape.d)
    _need(k, torch.bfloat16, act, "k")
    _need(v, torch.bfloat16, act, "v")
    _need(P, torch.bfloat16, (shape.H, shape.d, shape.r), "P")
    nb, dev = shape.n_blocks, k.device
    S_blk = torch.empty((shape.B, shape.H, nb, shape.r, shape.d), dtype=torch.float32, device=dev)
    z_blk = torch.empty((shape.B, shape.H, nb, shape.r), dtype=torch.float32, device=dev)
    S_glb = torch.empty((shape.B, shape.H, shape.r, shape.d), dtype=torch.float32, device=dev)
    z_glb = torch.empty((shape.B, shape.H, shape.r), dtype=torch.float32, device=dev)
    _check(lib().rola_block_states(ctypes.byref(shape.c()), _ptr(k), _ptr(v), _ptr(P), _ptr(S_blk),
                                   _ptr(z_blk), _ptr(S_glb), _ptr(z_glb), _stream(stream)),
           "rola_block_states")
    return S_blk, z_blk, S_glb, z_glb


def attention_fwd(shape: Shape, q, k, v, idx, P, states, gate, *, out=None, dev_err=None,
                  stream=None, wait_limit_ns=None):
    """RoLA attention output bf16 [B, N, H, d] for a given block mask.
    ``wait_limit_ns`` bounds each pipeline wait of the kernel (default 1 s;
    0 gives up at the first wait that is not ready, for tests of the timeout
    path)."""
    act = (shape.B, shape.N, shape.H, shape.d)
    for t, nm in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.bfloat16, act, nm)
    nb = shape.n_blocks
    _need(idx, torch.int32, (shape.B, shape.H, nb, shape.k_b), "idx")
    _need(P, torch.bfloat16, (shape.H, shape.d, shape.r), "P")
    _need(gate, torch.float32, (shape.H,), "gate")
    S_blk, z_blk, S_glb, z_glb = states
    _need(S_blk, torch.float32, (shape.B, shape.H, nb, shape.r, shape.d), "S_blk")
    _need(z_blk, torch.float32, (shape.B, shape.H, nb, shape.r), "z_blk")
    _need(S_glb, torch.float32, (shape.B, shape.H, shape.r, shape.d), "S_glb")
    _need(z_glb, torch.float32, (shape.B, shape.H, shape.r), "z_glb")
    if out is None:
        out = torch.empty(act, dtype=torch.bfloat16, device=q.device)
    _need(out, torch.bfloat16, act, "out")
    args = (ctypes.byref(shape.c()), _ptr(q), _ptr(k), _ptr(v), _ptr(idx), _ptr(P), _ptr(S_blk),
            _ptr(z_blk), _ptr(S_glb), _ptr(z_glb), _ptr(gate), _ptr(out), _ptr(dev_err))
    if wait_limit_ns is None:
        _check(lib().rola_attention_fwd(*args, _stream(stream)), "rola_attention_fwd")
    else:
        _check(lib().rola_attention_fwd_bounded(*args, ctypes.c_uint64(int(wait_limit_ns)), _stream(stream)),
               "rola_attention_fwd_bounded")
    return out


def attention_fwd_train(shape: Shape, q, k, v, idx, P, states, gate, *, dev_err=None, stream=None):
    """Forward that also returns what the backward reads: (out, out_lo bf16
    [B, N, H, d], lse float [B, H, N], den float [B, H, N])."""
    act = (shape.B, shape.N, shape.H, shape.d)
    S_blk, z_blk, S_glb, z_glb = states
    out = torch.empty(act, dtype=torch.bfloat16, device=q.device)
    out_lo = torch.empty_like(out)
    lse = torch.empty((shape.B, shape.H, shape.N), dtype=torch.float32, device=q.device)
    den = torch.empty_like(lse)
    _check(lib().rola_attention_fwd_train(ctypes.byref(shape.c()), _ptr(q), _ptr(k), _ptr(v), _ptr(idx), _ptr(P),
                                          _ptr(S_blk), _ptr(z_blk), _ptr(S_glb), _ptr(z_glb), _ptr(gate),
                                          _ptr(out), _ptr(out_lo), _ptr(lse), _ptr(den), _ptr(dev_err),
                                          _stream(stream)),
           "rola_attention_fwd_train")
    return out, out_lo, lse, den


def attention_bwd(shape: Shape, q, k, v, idx, P, states, gate, out, out_lo, lse, den, dout, *, dev_err=None,
                  stream=None, workspace=None, grads=None):
    """Gradients (dq, dk, dv bf16 [B, N, H, d], dP float [H, d, r], dgate
    float [H]) of sum(dout * out) for the forward of attention_fwd_train.
    `grads`, if given, is that tuple preallocated (every element is written)."""
    act = (shape.B, shape.N, shape.H, shape.d)
    for t, nm in ((q, "q"), (k, "k"), (v, "v"), (out, "out"), (out_lo, "out_lo"), (dout, "dout")):
        _need(t, torch.bfloat16, act, nm)
    S_blk, z_blk, S_glb, z_glb = states
    if grads is None:
        dq, dk, dv = (torch.empty(act, dtype=torch.bfloat16, device=q.device) for _ in range(3))
        dP = torch.empty((shape.H, shape.d, shape.r), dtype=torch.float32, device=q.device)
        dgate = torch.empty((shape.H,), dtype=torch.float32, device=q.device)
    else:
        dq, dk, dv, dP, dgate = grads
        for t, nm in ((dq, "dq"), (dk, "dk"), (dv, "dv")):
            _need(t, torch.bfloat16, act, nm)
        _need(dP, torch.float32, (shape.H, shape.d, shape.r), "dP")
        _need(dgate, torch.float32, (shape.H,), "dgate")
    c = shape.c()
    nbytes = lib().rola_attention_bwd_workspace_bytes(ctypes.byref(c))
    if nbytes == 0:
        raise RolaError("rola_attention_bwd: unsupported shape")
    if workspace is None or workspace.numel() < nbytes:
        workspace = _ws(nbytes, q.device)
    _check(lib().rola_attention_bwd(ctypes.byref(c), _ptr(q), _ptr(k), _ptr(v), _ptr(idx), _ptr(P), _ptr(S_blk),
                                    _ptr(z_blk), _ptr(S_glb), _ptr(z_glb), _ptr(gate), _ptr(out), _ptr(out_lo),
                                    _ptr(lse), _ptr(den), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dP), _ptr(dgate),
                                    _ptr(workspace), nbytes, _ptr(dev_err), _stream(stream)),
           "rola_attention_bwd")
    return dq, dk, dv, dP, dgate


class Layer:
    """One RoLA attention layer with its workspace allocated once."""

    def __init__(self, shape: Shape, device="cuda"):
        self.shape = shape
        self.c = shape.c()
        self.ws_bytes = lib().rola_layer_workspace_bytes(ctypes.byref(self.c))
        if self.ws_bytes == 0:
            raise RolaError("invalid or unsupported shape")
        self.ws = _ws(self.ws_bytes, device)
        self.dev_err = torch.zeros(1, dtype=torch.int32, device=device)

    def __call__(self, q, k, v, P, gate, *, out=None, idx_out=None, stream=None, events=None):
        """events: optional three or five torch.cuda.Event(enable_timing=True):
        three are recorded before the layer, after selection + states and after
        the attention; five also split the first stage into the pass over q, k,
        v, the scores + top-k and the state totals."""
        s = self.shape
        act = (s.B, s.N, s.H, s.d)
        for t, nm in ((q, "q"), (k, "k"), (v, "v")):
            _need(t, torch.bfloat16, act, nm)
        _need(P, torch.bfloat16, (s.H, s.d, s.r), "P")
        _need(gate, torch.float32, (s.H,), "gate")
        if out is None:
            out = torch.empty(act, dtype=torch.bfloat16, device=q.device)
        if idx_out is not None:
            _need(idx_out, torch.int32, (s.B, s.H, s.n_blocks, s.k_b), "idx_out")
        if events is None:
            _check(lib().rola_layer_fwd(ctypes.byref(self.c), _ptr(q), _ptr(k), _ptr(v), _ptr(P),
                                        _ptr(gate), _ptr(out), _ptr(idx_out), _ptr(self.ws),
                                        self.ws_bytes, _ptr(self.dev_err), _stream(stream)),
                   "rola_layer_fwd")
        else:
            if len(events) not in (3, 5):
                raise ValueError("events: three or five torch.cuda.Event")
            for e in events:
                if not e.cuda_event:  # torch creates the handle on first record
                    e.record(stream if stream is not None else torch.cuda.current_stream())
            ev = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
            _check(lib().rola_layer_fwd_timed(ctypes.byref(self.c), _ptr(q), _ptr(k), _ptr(v), _ptr(P),
                                              _ptr(gate), _ptr(out), _ptr(idx_out), _ptr(self.ws),
                                              self.ws_bytes, _ptr(self.dev_err), _stream(stream), ev,
                                              len(events)),
                   "rola_layer_fwd_timed")
        return out


    def run_ex(self, q, k, v, P, gate, idx, *, kb_per_head=None, reuse_mask=False, out=None,
               stream=None, events=None):
        """The layer with options: ``kb_per_head`` (int32 [H] on the device,
        each in 1..k_b) keeps a different number of blocks per head;
        ``reuse_mask`` takes ``idx`` (int32 [B, H, n_blocks, k_b]) as the mask
        instead of selecting one (else the selected mask is written to it)."""
        s = self.shape
        act = (s.B, s.N, s.H, s.d)
        for t, nm in ((q, "q"), (k, "k"), (v, "v")):
            _need(t, torch.bfloat16, act, nm)
        _need(P, torch.bfloat16, (s.H, s.d, s.r), "P")
        _need(gate, torch.float32, (s.H,), "gate")
        _need(idx, torch.int32, (s.B, s.H, s.n_blocks, s.k_b), "idx")
        if kb_per_head is not None:
            _need(kb_per_head, torch.int32, (s.H,), "kb_per_head")
        if out is None:
            out = torch.empty(act, dtype=torch.bfloat16, device=q.device)
        opts = LayerOpts(None if kb_per_head is None else kb_per_head.data_ptr(), 1 if reuse_mask else 0)
        ev, n_ev = None, 0
        if events is not None:
            if len(events) not in (3, 5):
                raise ValueError("events: three or five torch.cuda.Event")
            for e in events:
                if not e.cuda_event:
                    e.record(stream if stream is not None else torch.cuda.current_stream())
            ev, n_ev = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events]), len(events)
        _check(lib().rola_layer_fwd_ex(ctypes.byref(self.c), ctypes.byref(opts), _ptr(q), _ptr(k), _ptr(v),
                                       _ptr(P), _ptr(gate), _ptr(out), _ptr(idx), _ptr(self.ws), self.ws_bytes,
                                       _ptr(self.dev_err), _stream(stream), ev, n_ev),
               "rola_layer_fwd_ex")
        return out


def layer_launches(shape: Shape) -> int:
    """Kernels one layer call launches for `shape`."""
    c = shape.c()
    n = lib().rola_layer_kernel_launches(ctypes.byref(c))
    if n <= 0:
        raise RolaError("invalid or unsupported shape")
    return n


class HostLayer:
    """The layer on HOST tensors (pinned for asynchronous copies): the library
    copies the inputs in by head groups, runs the layer on each group while the
    next one is copied in, and copies each group's output back meanwhile; the
    given (or current) stream waits for the last copy."""

    def __init__(self, shape: Shape, device="cuda"):
        self.shape = shape
        self.c = shape.c()
        self.ws_bytes = lib().rola_layer_host_workspace_bytes(ctypes.byref(self.c))
        if self.ws_bytes == 0:
            raise RolaError("invalid or unsupported shape")
        self.ws = _ws(self.ws_bytes, device)
        self.dev_err = torch.zeros(1, dtype=torch.int32, device=device)

    def __call__(self, q, k, v, P, gate, out, *, stream=None):
        for t in (q, k, v, P, gate, out):
            if t.is_cuda or not t.is_contiguous():
                raise ValueError("HostLayer takes contiguous host tensors")
        _check(lib().rola_layer_fwd_host(ctypes.byref(self.c), _ptr(q), _ptr(k), _ptr(v), _ptr(P),
                                         _ptr(gate), _ptr(out), _ptr(self.ws), self.ws_bytes,
                                         _ptr(self.dev_err), _stream(stream)),
               "rola_layer_fwd_host")
        return out


# ------------------------------------------------------------------ FP8 W8A8

def fp8_quantize_rows(x, *, stream=None):
    """Per-row E4M3 codes (uint8 [M, K]) and float32 scales [M] of bf16 x."""
    M, K = x.shape
    _need(x, torch.bfloat16, (M, K), "x")
    xq = torch.empty((M, K), dtype=torch.uint8, device=x.device)
    sc = torch.empty((M,), dtype=torch.float32, device=x.device)
    _check(lib().fp8_quantize_rows_bf16(M, K, _ptr(x), _ptr(xq), _ptr(sc), _stream(stream)),
           "fp8_quantize_rows_bf16")
    return xq, sc


def fp8_quantize_weight(w, *, stream=None):
    N, K = w.shape
    _need(w, torch.float32, (N, K), "w")
    wq = torch.empty((N, K), dtype=torch.uint8, device=w.device)
    sc = torch.empty((N,), dtype=torch.float32, device=w.device)
    _check(lib().fp8_quantize_weight(N, K, _ptr(w), _ptr(wq), _ptr(sc), _stream(stream)),
           "fp8_quantize_weight")
    return wq, sc


def fp8_gemm(xq, xs, wq, ws, *, out=None, dev_err=None, stream=None, act=ACT_NONE):
    """y = bf16(act((x_q w_q^T) x_scale w_scale)); act ACT_NONE or ACT_GELU_TANH."""
    M, K = xq.shape
    N = wq.shape[0]
    _need(xq, torch.uint8, (M, K), "x_q")
    _need(wq, torch.uint8, (N, K), "w_q")
    _need(xs, torch.float32, (M,), "x_scale")
    _need(ws, torch.float32, (N,), "w_scale")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=xq.device)
    _need(out, torch.bfloat16, (M, N), "y")
    if act == ACT_NONE:
        _check(lib().fp8_gemm_w8a8(M, N, K, _ptr(xq), _ptr(xs), _ptr(wq), _ptr(ws), _ptr(out),
                                   _ptr(dev_err), _stream(stream)), "fp8_gemm_w8a8")
    else:
        _check(lib().fp8_gemm_w8a8_act(M, N, K, _ptr(xq), _ptr(xs), _ptr(wq), _ptr(ws), act, _ptr(out),
                                       _ptr(dev_err), _stream(stream)), "fp8_gemm_w8a8_act")
    return out


def fp8_linear(x, wq, ws, *, out=None, workspace=None, dev_err=None, stream=None):
    M, K = x.shape
    N = wq.shape[0]
    _need(x, torch.bfloat16, (M, K), "x")
    _need(wq, torch.uint8, (N, K), "w_q")
    _need(ws, torch.float32, (N,), "w_scale")
    nbytes = lib().fp8_linear_workspace_bytes(M, K)
    if workspace is None or workspace.numel() < nbytes:
        workspace = _ws(nbytes, x.device)
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    _check(lib().fp8_linear_w8a8(M, N, K, _ptr(x), _ptr(wq), _ptr(ws), _ptr(out), _ptr(workspace),
                                 nbytes, _ptr(dev_err), _stream(stream)), "fp8_linear_w8a8")
    return out


def fp8_ffn(x, w1q, w1s, w2q, w2s, *, out=None, workspace=None, dev_err=None, stream=None):
    """y = W2 gelu_tanh(W1 x) with both projections in W8A8 FP8: x bf16 [M, D],
    w1q uint8 [F, D], w2q uint8 [D, F], per-output-channel float32 scales."""
    M, D = x.shape
    F = w1q.shape[0]
    _need(x, torch.bfloat16, (M, D), "x")
    _need(w1q, torch.uint8, (F, D), "w1_q")
    _need(w1s, torch.float32, (F,), "w1_scale")
    _need(w2q, torch.uint8, (D, F), "w2_q")
    _need(w2s, torch.float32, (D,), "w2_scale")
    nbytes = lib().fp8_ffn_workspace_bytes(M, D, F)
    if workspace is None or workspace.numel() < nbytes:
        workspace = _ws(nbytes, x.device)
    if out is None:
        out = torch.empty((M, D), dtype=torch.bfloat16, device=x.device)
    _need(out, torch.bfloat16, (M, D), "y")
    _check(lib().fp8_ffn_w8a8(M, D, F, _ptr(x), _ptr(w1q), _ptr(w1s), _ptr(w2q), _ptr(w2s), _ptr(out),
                              _ptr(workspace), nbytes, _ptr(dev_err), _stream(stream)), "fp8_ffn_w8a8")
    return out
