"""MoE token dispatch and combine on one B200 (sm_100a CUDA kernels behind a C ABI).

Dispatch groups each token's hidden vector by its top-k routed experts into
contiguous per-expert (and per-virtual-rank) receive buffers, optionally as fp8
e4m3 with one scale per 128 columns; combine gathers the experts' output rows
back and returns each token's routing-weighted sum ("Enabling
trillion-parameter models on AWS EFA", sections "Introdução", "Buffers de Envio
e Recebimento" and "Despacho e Combinação").

This module only marshals arguments: torch allocates device memory and
provides the stream, ctypes calls ``libmoe_b200.so``, and every step runs in
that library's kernels.  There is no CPU fallback: without the built library,
importing this package raises.

    import combine_route_meta_b200 as moe
    d = moe.dispatch(x, topk_idx, topk_w, num_experts=256, num_virtual_ranks=8, fp8=True)
    y = moe.combine(d.handle, expert_out)
"""
from __future__ import annotations

import ctypes
import os
from typing import NamedTuple, Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python combine_route_meta_b200/build.py` "
        "(there is no fallback implementation)")

# ---- C ABI mirror (include/moe_dispatch_combine.h) -----------------------------

FP8 = 1
PAD128 = 2
INPUTS_READY = 4

OK = 0
ERR_INVALID_ARG = -1
ERR_UNSUPPORTED = -2
ERR_CUDA = -3
ERR_DEVICE = -4
ERR_TOO_LARGE = -5

DEV_BAD_INDEX = 1
DEV_CAPACITY = 2
DEV_TIMEOUT = 4
DEV_BAD_SLOT = 8

MAX_EXPERTS = 2048
MAX_TOPK = 64
SCORE_SOFTMAX = 0
SCORE_SIGMOID = 1
NO_ALLOC_SCRATCH_BYTES = 1 << 20


class moe_config(ctypes.Structure):
    _fields_ = [("H", ctypes.c_int32), ("k", ctypes.c_int32), ("E", ctypes.c_int32),
                ("R", ctypes.c_int32), ("flags", ctypes.c_int32)]


class moe_dispatch_out(ctypes.Structure):
    _fields_ = [("recv_x", ctypes.c_void_p), ("recv_scale", ctypes.c_void_p),
                ("expert_count", ctypes.c_void_p), ("expert_offset", ctypes.c_void_p),
                ("rank_offset", ctypes.c_void_p), ("recv_src", ctypes.c_void_p),
                ("rows_cap", ctypes.c_int64)]


class moe_handle(ctypes.Structure):
    _fields_ = [("cfg", moe_config), ("T", ctypes.c_int32), ("slot", ctypes.c_void_p),
                ("topk_w", ctypes.c_void_p), ("rows_cap", ctypes.c_int64)]


class moe_dispatch_sizes(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in
                ("recv_x", "recv_scale", "expert_count", "expert_offset", "rank_offset",
                 "recv_src", "slot")]


def _declare(lib):
    P, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    cfgp = ctypes.POINTER(moe_config)
    lib.moe_version.argtypes, lib.moe_version.restype = [], ctypes.c_int
    lib.moe_status_string.argtypes, lib.moe_status_string.restype = [ctypes.c_int], ctypes.c_char_p
    lib.moe_rows_capacity.argtypes, lib.moe_rows_capacity.restype = [cfgp, i32], i64
    lib.moe_workspace_bytes.argtypes, lib.moe_workspace_bytes.restype = [cfgp, i32], ctypes.c_size_t
    lib.moe_dispatch_sizes_for.argtypes = [cfgp, i32, i64, ctypes.POINTER(moe_dispatch_sizes)]
    lib.moe_dispatch_sizes_for.restype = ctypes.c_int
    lib.moe_dispatch.argtypes = [cfgp, i32, P, P, P, ctypes.POINTER(moe_dispatch_out), P, P,
                                 ctypes.c_size_t, P, P, ctypes.POINTER(moe_handle)]
    lib.moe_dispatch.restype = ctypes.c_int
    lib.moe_dispatch_layout.argtypes = [cfgp, i32, P, ctypes.POINTER(moe_dispatch_out), P, P,
                                        ctypes.c_size_t, P, P]
    lib.moe_dispatch_layout.restype = ctypes.c_int
    lib.moe_dispatch_payload.argtypes = [cfgp, i32, P, P, ctypes.POINTER(moe_dispatch_out), P, P]
    lib.moe_dispatch_payload.restype = ctypes.c_int
    lib.moe_dispatch_no_alloc.argtypes = [cfgp, i32, P, P, P, ctypes.POINTER(moe_dispatch_out), P,
                                          P, P, ctypes.POINTER(moe_handle)]
    lib.moe_dispatch_no_alloc.restype = ctypes.c_int
    lib.moe_combine.argtypes = [ctypes.POINTER(moe_handle), P, P, P, P]
    lib.moe_combine.restype = ctypes.c_int
    lib.moe_selftest_bounded_wait.argtypes = [P, ctypes.c_uint64, P]
    lib.moe_selftest_bounded_wait.restype = ctypes.c_int
    lib.moe_combine_rank_partial.argtypes = [ctypes.POINTER(moe_handle), P, P, P, P, P, P, P, P]
    lib.moe_combine_rank_partial.restype = ctypes.c_int
    lib.moe_silu_quant.argtypes = [i64, i32, P, P, P, P, P, i32, P]
    lib.moe_silu_quant.restype = ctypes.c_int
    lib.moe_silu_mul.argtypes = [i64, P, P, P, P, i32, P]
    lib.moe_silu_mul.restype = ctypes.c_int
    lib.moe_router_topk.argtypes = [i32, i32, i32, P, i32, i32, i32, i32, P, P, P]
    lib.moe_router_topk.restype = ctypes.c_int
    lib.moe_route_dispatch.argtypes = [cfgp, i32, P, P, i32, i32, i32, i32, P, P,
                                       ctypes.POINTER(moe_dispatch_out), P, P, ctypes.c_size_t, P, P,
                                       ctypes.POINTER(moe_handle)]
    lib.moe_route_dispatch.restype = ctypes.c_int
    lib.moe_ep_rows_capacity.argtypes, lib.moe_ep_rows_capacity.restype = [cfgp, i32], i64
    lib.moe_ep_layout.argtypes = [cfgp, i32, i32, P, P, P, P, i64, P, P, P, P, P]
    lib.moe_ep_layout.restype = ctypes.c_int
    lib.moe_ep_dispatch_payload.argtypes = [cfgp, i32, P, P, P, ctypes.POINTER(P), ctypes.POINTER(P),
                                            i64, i32, ctypes.POINTER(P), P, P, P, P]
    lib.moe_ep_dispatch_payload.restype = ctypes.c_int
    lib.moe_ep_signal.argtypes = [i32, i32, ctypes.POINTER(P), P, P]
    lib.moe_ep_signal.restype = ctypes.c_int
    lib.moe_ep_wait.argtypes = [i32, P, P, ctypes.c_uint64, P, P]
    lib.moe_ep_wait.restype = ctypes.c_int
    lib.moe_ep_combine.argtypes = [cfgp, i32, P, P, P, ctypes.POINTER(P), i64, P, P, P]
    lib.moe_ep_combine.restype = ctypes.c_int
    lib.moe_check.argtypes = [P, P, ctypes.POINTER(ctypes.c_int32)]
    lib.moe_check.restype = ctypes.c_int
    return lib


lib = _declare(ctypes.CDLL(LIB_PATH))

# C names, callable directly with ctypes arguments.
moe_version = lib.moe_version
moe_status_string = lib.moe_status_string
moe_rows_capacity = lib.moe_rows_capacity
moe_workspace_bytes = lib.moe_workspace_bytes
moe_dispatch_sizes_for = lib.moe_dispatch_sizes_for
moe_dispatch = lib.moe_dispatch
moe_dispatch_no_alloc = lib.moe_dispatch_no_alloc
moe_dispatch_layout = lib.moe_dispatch_layout
moe_dispatch_payload = lib.moe_dispatch_payload
moe_combine = lib.moe_combine
moe_check = lib.moe_check
moe_selftest_bounded_wait = lib.moe_selftest_bounded_wait
moe_combine_rank_partial = lib.moe_combine_rank_partial
moe_silu_quant = lib.moe_silu_quant
moe_silu_mul = lib.moe_silu_mul
moe_router_topk = lib.moe_router_topk
moe_route_dispatch = lib.moe_route_dispatch
moe_ep_rows_capacity = lib.moe_ep_rows_capacity
moe_ep_layout = lib.moe_ep_layout
moe_ep_dispatch_payload = lib.moe_ep_dispatch_payload
moe_ep_combine = lib.moe_ep_combine
moe_ep_signal = lib.moe_ep_signal
moe_ep_wait = lib.moe_ep_wait


class MoeError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        msg = lib.moe_status_string(status).decode()
        super().__init__(f"{what}: {msg} ({status})" if what else f"{msg} ({status})")
        self.status = status


def _ok(status: int, what: str):
    if status != OK:
        raise MoeError(status, what)


# ---- torch-level helpers ------------------------------------------------------

def make_config(H: int, k: int, num_experts: int, num_virtual_ranks: int,
                fp8: bool, pad128: bool = False, inputs_ready: bool = False) -> moe_config:
    """inputs_ready: MOE_INPUTS_READY (see the C header)."""
    return moe_config(H, k, num_experts, num_virtual_ranks,
                      (FP8 if fp8 else 0) | (PAD128 if pad128 else 0) | (INPUTS_READY if inputs_ready else 0))


def rows_capacity(cfg: moe_config, T: int) -> int:
    r = lib.moe_rows_capacity(ctypes.byref(cfg), T)
    if r < 0:
        raise MoeError(ERR_INVALID_ARG, "moe_rows_capacity")
    return int(r)


def workspace_bytes(cfg: moe_config, T: int) -> int:
    return int(lib.moe_workspace_bytes(ctypes.byref(cfg), T))


def _stream_ptr(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


_err_words: dict[int, torch.Tensor] = {}


def error_word(device=None) -> torch.Tensor:
    """The per-device int32 word the kernels OR error bits into."""
    dev = torch.device("cuda", torch.cuda.current_device() if device is None else
                       torch.device(device).index or 0)
    w = _err_words.get(dev.index)
    if w is None:
        w = torch.zeros(1, dtype=torch.int32, device=dev)
        _err_words[dev.index] = w
    return w


def check(stream: Optional[torch.cuda.Stream] = None, device=None) -> int:
    """Waits for the stream, returns and clears the device error bits."""
    bits = ctypes.c_int32(0)
    st = lib.moe_check(ctypes.c_void_p(error_word(device).data_ptr()),
                       ctypes.c_void_p(_stream_ptr(stream)), ctypes.byref(bits))
    if st not in (OK, ERR_DEVICE):
        raise MoeError(st, "moe_check")
    return int(bits.value)


class Handle:
    """Routing state combine needs: the C handle plus the tensors it points to."""

    def __init__(self, c: moe_handle, slot: torch.Tensor, topk_w: torch.Tensor):
        self.c = c
        self.slot = slot
        self.topk_w = topk_w


class DispatchResult(NamedTuple):
    recv_x: torch.Tensor           # [rows_cap, H] bf16 or float8_e4m3fn
    recv_scale: Optional[torch.Tensor]  # [rows_cap, H/128] float32 (fp8) or None
    expert_count: torch.Tensor     # [E] int32
    expert_offset: torch.Tensor    # [E+1] int32
    rank_offset: torch.Tensor      # [R+1] int32
    recv_src: torch.Tensor         # [rows_cap] int32
    handle: Handle


class Buffers:
    """Preallocated dispatch/combine buffers for one (config, T) on one device."""

    def __init__(self, cfg: moe_config, T: int, device, rows_cap: Optional[int] = None):
        device = torch.device(device)
        self.cfg, self.T, self.device = cfg, T, device
        self.rows_cap = rows_capacity(cfg, T) if rows_cap is None else int(rows_cap)
        fp8 = bool(cfg.flags & FP8)
        e = dict(device=device)
        self.recv_x = torch.empty((self.rows_cap, cfg.H),
                                  dtype=torch.float8_e4m3fn if fp8 else torch.bfloat16, **e)
        self.recv_scale = (torch.empty((self.rows_cap, cfg.H // 128), dtype=torch.float32, **e)
                           if fp8 else None)
        self.expert_count = torch.empty(cfg.E, dtype=torch.int32, **e)
        self.expert_offset = torch.empty(cfg.E + 1, dtype=torch.int32, **e)
        self.rank_offset = torch.empty(cfg.R + 1, dtype=torch.int32, **e)
        self.recv_src = torch.empty(self.rows_cap, dtype=torch.int32, **e)
        self.slot = torch.empty((T, cfg.k), dtype=torch.int32, **e)
        nws = workspace_bytes(cfg, T)
        self.workspace = torch.empty(max(nws, 1), dtype=torch.uint8, **e)
        self.workspace_bytes = nws
        self.out = moe_dispatch_out(
            self.recv_x.data_ptr(),
            self.recv_scale.data_ptr() if fp8 else None,
            self.expert_count.data_ptr(), self.expert_offset.data_ptr(),
            self.rank_offset.data_ptr(), self.recv_src.data_ptr(), self.rows_cap)
        self.handle_c = moe_handle()
        self.err = error_word(device)


def _check_tensor(t: torch.Tensor, name: str, dtype, ndim: int):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {ndim}-D tensor")


def dispatch_into(buf: Buffers, x: torch.Tensor, topk_idx: torch.Tensor, topk_w: torch.Tensor,
                  stream: Optional[torch.cuda.Stream] = None) -> None:
    """moe_dispatch into preallocated buffers (no allocation, no host sync)."""
    st = lib.moe_dispatch(ctypes.byref(buf.cfg), buf.T, ctypes.c_void_p(x.data_ptr()),
                          ctypes.c_void_p(topk_idx.data_ptr()), ctypes.c_void_p(topk_w.data_ptr()),
                          ctypes.byref(buf.out), ctypes.c_void_p(buf.slot.data_ptr()),
                          ctypes.c_void_p(buf.workspace.data_ptr()), buf.workspace_bytes,
                          ctypes.c_void_p(buf.err.data_ptr()), ctypes.c_void_p(_stream_ptr(stream)),
                          ctypes.byref(buf.handle_c))
    _ok(st, "moe_dispatch")


def dispatch_layout_into(buf: Buffers, topk_idx: torch.Tensor,
                         stream: Optional[torch.cuda.Stream] = None) -> None:
    """moe_dispatch_layout: counts, offsets, slots and recv_src only."""
    st = lib.moe_dispatch_layout(ctypes.byref(buf.cfg), buf.T, ctypes.c_void_p(topk_idx.data_ptr()),
                                 ctypes.byref(buf.out), ctypes.c_void_p(buf.slot.data_ptr()),
                                 ctypes.c_void_p(buf.workspace.data_ptr()), buf.workspace_bytes,
                                 ctypes.c_void_p(buf.err.data_ptr()),
                                 ctypes.c_void_p(_stream_ptr(stream)))
    _ok(st, "moe_dispatch_layout")


def dispatch_payload_into(buf: Buffers, x: torch.Tensor, slot: Optional[torch.Tensor] = None,
                          stream: Optional[torch.cuda.Stream] = None) -> None:
    """moe_dispatch_payload: the rows of x to the slots (buf.slot by default)."""
    slot = buf.slot if slot is None else slot
    st = lib.moe_dispatch_payload(ctypes.byref(buf.cfg), buf.T, ctypes.c_void_p(x.data_ptr()),
                                  ctypes.c_void_p(slot.data_ptr()), ctypes.byref(buf.out),
                                  ctypes.c_void_p(buf.err.data_ptr()),
                                  ctypes.c_void_p(_stream_ptr(stream)))
    _ok(st, "moe_dispatch_payload")


def combine_into(handle_c: moe_handle, expert_out: torch.Tensor, y: torch.Tensor,
                 err: torch.Tensor, stream: Optional[torch.cuda.Stream] = None) -> None:
    """moe_combine into a preallocated y (no allocation, no host sync)."""
    st = lib.moe_combine(ctypes.byref(handle_c), ctypes.c_void_p(expert_out.data_ptr()),
                         ctypes.c_void_p(y.data_ptr()), ctypes.c_void_p(err.data_ptr()),
                         ctypes.c_void_p(_stream_ptr(stream)))
    _ok(st, "moe_combine")


def dispatch(x: torch.Tensor, topk_idx: torch.Tensor, topk_w: torch.Tensor,
             num_experts: int, num_virtual_ranks: int, fp8: bool, pad128: bool = False, *,
             rows_cap: Optional[int] = None,
             stream: Optional[torch.cuda.Stream] = None) -> DispatchResult:
    """Dispatch x[T,H] (bf16) by topk_idx[T,k] into per-expert receive buffers.

    topk_idx may be int32 or int64 (converted); topk_w is float32 and is kept
    by the returned handle for combine.
    """
    if topk_idx.dtype == torch.int64:
        topk_idx = topk_idx.to(torch.int32)
    _check_tensor(x, "x", torch.bfloat16, 2)
    _check_tensor(topk_idx, "topk_idx", torch.int32, 2)
    _check_tensor(topk_w, "topk_w", torch.float32, 2)
    T, H = x.shape
    k = topk_idx.shape[1]
    if topk_idx.shape[0] != T or tuple(topk_w.shape) != (T, k):
        raise ValueError("x, topk_idx and topk_w disagree on shape")
    cfg = make_config(H, k, num_experts, num_virtual_ranks, fp8, pad128)
    buf = Buffers(cfg, T, x.device, rows_cap)
    dispatch_into(buf, x, topk_idx, topk_w, stream)
    handle = Handle(buf.handle_c, buf.slot, topk_w)
    return DispatchResult(buf.recv_x, buf.recv_scale, buf.expert_count, buf.expert_offset,
                          buf.rank_offset, buf.recv_src, handle)


def combine(handle: Handle, expert_out: torch.Tensor, *,
            stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """y[T,H] bf16: each token's routing-weighted sum of its rows of expert_out."""
    _check_tensor(expert_out, "expert_out", torch.bfloat16, 2)
    c = handle.c
    if expert_out.shape[0] < c.rows_cap or expert_out.shape[1] != c.cfg.H:
        raise ValueError("expert_out must be [rows_cap, H] in the receive layout")
    y = torch.empty((c.T, c.cfg.H), dtype=torch.bfloat16, device=expert_out.device)
    combine_into(c, expert_out, y, error_word(expert_out.device), stream)
    return y


def combine_rank_partial_into(handle_c: moe_handle, rank_offset: torch.Tensor,
                              expert_out: torch.Tensor, partial: torch.Tensor,
                              partial_rank: torch.Tensor, npart: torch.Tensor, y: torch.Tensor,
                              err: torch.Tensor, stream: Optional[torch.cuda.Stream] = None) -> None:
    """moe_combine_rank_partial into preallocated buffers."""
    P = ctypes.c_void_p
    st = lib.moe_combine_rank_partial(ctypes.byref(handle_c), P(rank_offset.data_ptr()),
                                      P(expert_out.data_ptr()), P(partial.data_ptr()),
                                      P(partial_rank.data_ptr()), P(npart.data_ptr()),
                                      P(y.data_ptr()), P(err.data_ptr()), P(_stream_ptr(stream)))
    _ok(st, "moe_combine_rank_partial")


def combine_rank_partial(handle: Handle, rank_offset: torch.Tensor, expert_out: torch.Tensor, *,
                         stream: Optional[torch.cuda.Stream] = None):
    """(y, partial, partial_rank, npart): combine with per-rank partial sums (see the C header)."""
    c = handle.c
    dev = expert_out.device
    partial = torch.empty((c.T, c.cfg.k, c.cfg.H), dtype=torch.bfloat16, device=dev)
    partial_rank = torch.full((c.T, c.cfg.k), -1, dtype=torch.int32, device=dev)
    npart = torch.empty(c.T, dtype=torch.int32, device=dev)
    y = torch.empty((c.T, c.cfg.H), dtype=torch.bfloat16, device=dev)
    combine_rank_partial_into(c, rank_offset, expert_out, partial, partial_rank, npart, y,
                              error_word(dev), stream)
    return y, partial, partial_rank, npart


def silu_quant_into(gate_up: torch.Tensor, recv_src: torch.Tensor, rows_in_use: torch.Tensor,
                    act: torch.Tensor, act_scale: torch.Tensor, col_major: bool = False,
                    stream: Optional[torch.cuda.Stream] = None) -> None:
    """moe_silu_quant into preallocated act (float8_e4m3fn) and act_scale (float32)."""
    P = ctypes.c_void_p
    rows_cap, two_i = gate_up.shape
    st = lib.moe_silu_quant(rows_cap, two_i // 2, P(gate_up.data_ptr()), P(recv_src.data_ptr()),
                            P(rows_in_use.data_ptr()), P(act.data_ptr()), P(act_scale.data_ptr()),
                            1 if col_major else 0, P(_stream_ptr(stream)))
    _ok(st, "moe_silu_quant")


def silu_quant(gate_up: torch.Tensor, recv_src: torch.Tensor, rows_in_use: torch.Tensor, *,
               col_major: bool = False, stream: Optional[torch.cuda.Stream] = None):
    """(act, act_scale): block-fp8 SiLU(gate) * up of the populated rows (see the C header)."""
    rows_cap, two_i = gate_up.shape
    I = two_i // 2
    act = torch.zeros((rows_cap, I), dtype=torch.float8_e4m3fn, device=gate_up.device)
    shape = (I // 128, rows_cap) if col_major else (rows_cap, I // 128)
    act_scale = torch.zeros(shape, dtype=torch.float32, device=gate_up.device)
    silu_quant_into(gate_up, recv_src, rows_in_use, act, act_scale, col_major, stream)
    return act, act_scale


def silu_mul(gate: torch.Tensor, up: torch.Tensor, *, exact_only: bool = False,
             with_fast_value: bool = False, stream: Optional[torch.cuda.Stream] = None):
    """The activations of moe_silu_quant alone (see moe_silu_mul in the C header):
    float32 tensor shaped like gate, and with with_fast_value the fp64 values of
    the kernel's first tier."""
    g, u = gate.contiguous(), up.contiguous()
    act = torch.empty(g.shape, dtype=torch.float32, device=g.device)
    fast = torch.empty(g.shape, dtype=torch.float64, device=g.device) if with_fast_value else None
    P = ctypes.c_void_p
    st = lib.moe_silu_mul(g.numel(), P(g.data_ptr()), P(u.data_ptr()), P(act.data_ptr()),
                          P(fast.data_ptr() if fast is not None else 0), 1 if exact_only else 0,
                          P(_stream_ptr(stream)))
    _ok(st, "moe_silu_mul")
    return (act, fast) if with_fast_value else act


def router_topk_into(logits: torch.Tensor, k: int, topk_idx: torch.Tensor, topk_w: torch.Tensor, *,
                     score_fn: str = "softmax", n_group: int = 1, topk_group: int = 1,
                     renormalize: bool = True, stream: Optional[torch.cuda.Stream] = None) -> None:
    """moe_router_topk into preallocated topk_idx (int32) and topk_w (float32)."""
    T, E = logits.shape
    P = ctypes.c_void_p
    st = lib.moe_router_topk(T, E, k, P(logits.data_ptr()),
                             {"softmax": SCORE_SOFTMAX, "sigmoid": SCORE_SIGMOID}[score_fn],
                             n_group, topk_group, 1 if renormalize else 0,
                             P(topk_idx.data_ptr()), P(topk_w.data_ptr()), P(_stream_ptr(stream)))
    _ok(st, "moe_router_topk")


def router_topk(logits: torch.Tensor, k: int, **kw):
    """(topk_idx, topk_w) of group-limited top-k routing (see the C header)."""
    T = logits.shape[0]
    idx = torch.empty((T, k), dtype=torch.int32, device=logits.device)
    w = torch.empty((T, k), dtype=torch.float32, device=logits.device)
    router_topk_into(logits.contiguous().float(), k, idx, w, **kw)
    return idx, w


def route_dispatch_into(buf: Buffers, x: torch.Tensor, logits: torch.Tensor, topk_idx: torch.Tensor,
                        topk_w: torch.Tensor, *, score_fn: str = "softmax", n_group: int = 1,
                        topk_group: int = 1, renormalize: bool = True,
                        stream: Optional[torch.cuda.Stream] = None) -> None:
    """moe_route_dispatch into preallocated buffers: the routing writes topk_idx
    and topk_w and the dispatch reads them (one launch at decode sizes)."""
    P = ctypes.c_void_p
    st = lib.moe_route_dispatch(ctypes.byref(buf.cfg), buf.T, P(x.data_ptr()), P(logits.data_ptr()),
                                {"softmax": SCORE_SOFTMAX, "sigmoid": SCORE_SIGMOID}[score_fn],
                                n_group, topk_group, 1 if renormalize else 0,
                                P(topk_idx.data_ptr()), P(topk_w.data_ptr()), ctypes.byref(buf.out),
                                P(buf.slot.data_ptr()), P(buf.workspace.data_ptr()), buf.workspace_bytes,
                                P(buf.err.data_ptr()), P(_stream_ptr(stream)), ctypes.byref(buf.handle_c))
    _ok(st, "moe_route_dispatch")


def route_dispatch(x: torch.Tensor, logits: torch.Tensor, k: int, num_experts: int,
                   num_virtual_ranks: int, fp8: bool, pad128: bool = False, *,
                   stream: Optional[torch.cuda.Stream] = None, **router_kw):
    """Router top-k on logits[T,E] (float32), then dispatch of x[T,H] (bf16).

    Returns (DispatchResult, topk_idx, topk_w); the handle keeps topk_w."""
    _check_tensor(x, "x", torch.bfloat16, 2)
    _check_tensor(logits, "logits", torch.float32, 2)
    T, H = x.shape
    if logits.shape != (T, num_experts):
        raise ValueError("logits must be [T, num_experts]")
    cfg = make_config(H, k, num_experts, num_virtual_ranks, fp8, pad128)
    buf = Buffers(cfg, T, x.device)
    idx = torch.empty((T, k), dtype=torch.int32, device=x.device)
    w = torch.empty((T, k), dtype=torch.float32, device=x.device)
    route_dispatch_into(buf, x, logits, idx, w, stream=stream, **router_kw)
    handle = Handle(buf.handle_c, buf.slot, w)
    return (DispatchResult(buf.recv_x, buf.recv_scale, buf.expert_count, buf.expert_offset,
                           buf.rank_offset, buf.recv_src, handle), idx, w)


# ---- expert parallelism across ranks (see the C header) ------------------------------

def ep_rows_capacity(cfg: moe_config, T: int) -> int:
    """Rows of one rank's receive buffer when every rank dispatches up to T tokens."""
    n = lib.moe_ep_rows_capacity(ctypes.byref(cfg), T)
    if n < 0:
        raise MoeError(ERR_INVALID_ARG, "moe_ep_rows_capacity")
    return int(n)


def _ptr_table(bufs):
    """A ctypes array of device pointers from tensors (or ints, or None)."""
    if bufs is None:
        return None
    vals = [b if isinstance(b, int) else (None if b is None else b.data_ptr()) for b in bufs]
    return (ctypes.c_void_p * len(vals))(*vals)


def ep_layout_into(cfg: moe_config, rank: int, topk_idx: torch.Tensor, local_slot: torch.Tensor,
                   local_offset: torch.Tensor, counts_all: torch.Tensor, rows_cap: int,
                   dst_row: torch.Tensor, recv_count: torch.Tensor, recv_offset: torch.Tensor,
                   err: Optional[torch.Tensor] = None, stream: Optional[torch.cuda.Stream] = None) -> None:
    """moe_ep_layout into preallocated int32 tensors."""
    P = ctypes.c_void_p
    err = error_word(topk_idx.device) if err is None else err
    st = lib.moe_ep_layout(ctypes.byref(cfg), rank, topk_idx.shape[0], P(topk_idx.data_ptr()),
                           P(local_slot.data_ptr()), P(local_offset.data_ptr()), P(counts_all.data_ptr()),
                           rows_cap, P(dst_row.data_ptr()), P(recv_count.data_ptr()),
                           P(recv_offset.data_ptr()), P(err.data_ptr()), P(_stream_ptr(stream)))
    _ok(st, "moe_ep_layout")


def ep_dispatch_payload_into(cfg: moe_config, x: torch.Tensor, topk_idx: torch.Tensor,
                             dst_row: torch.Tensor, peer_recv_x, peer_recv_scale, rows_cap: int,
                             err: Optional[torch.Tensor] = None,
                             stream: Optional[torch.cuda.Stream] = None, signal=None) -> None:
    """moe_ep_dispatch_payload; the peer tables are W tensors or device addresses.
    signal = (rank, peer_flags, epoch, done_count) makes the kernel signal the
    "rows in place" event (see the C header); None signals nothing."""
    P = ctypes.c_void_p
    err = error_word(x.device) if err is None else err
    rank, flags, epoch, done = (0, None, None, None) if signal is None else signal
    st = lib.moe_ep_dispatch_payload(ctypes.byref(cfg), x.shape[0], P(x.data_ptr()),
                                     P(topk_idx.data_ptr()), P(dst_row.data_ptr()),
                                     _ptr_table(peer_recv_x), _ptr_table(peer_recv_scale), rows_cap,
                                     rank, _ptr_table(flags),
                                     P(0 if epoch is None else epoch.data_ptr()),
                                     P(0 if done is None else done.data_ptr()),
                                     P(err.data_ptr()), P(_stream_ptr(stream)))
    _ok(st, "moe_ep_dispatch_payload")


def ep_signal_into(rank: int, peer_flags, epoch: torch.Tensor,
                   stream: Optional[torch.cuda.Stream] = None) -> None:
    """moe_ep_signal: publish this rank's next epoch of an event in every peer's flags."""
    P = ctypes.c_void_p
    st = lib.moe_ep_signal(len(peer_flags), rank, _ptr_table(peer_flags), P(epoch.data_ptr()),
                           P(_stream_ptr(stream)))
    _ok(st, "moe_ep_signal")


def ep_wait_into(flags: torch.Tensor, epoch: torch.Tensor, limit_ns: int = 1_000_000_000,
                 err: Optional[torch.Tensor] = None, stream: Optional[torch.cuda.Stream] = None) -> None:
    """moe_ep_wait: the stream waits (bounded) until every sender's flag reaches *epoch."""
    P = ctypes.c_void_p
    err = error_word(flags.device) if err is None else err
    st = lib.moe_ep_wait(flags.numel(), P(flags.data_ptr()), P(epoch.data_ptr()), int(limit_ns),
                         P(err.data_ptr()), P(_stream_ptr(stream)))
    _ok(st, "moe_ep_wait")


def ep_combine_into(cfg: moe_config, topk_idx: torch.Tensor, dst_row: torch.Tensor,
                    topk_w: torch.Tensor, peer_expert_out, rows_cap: int, y: torch.Tensor,
                    err: Optional[torch.Tensor] = None,
                    stream: Optional[torch.cuda.Stream] = None) -> None:
    """moe_ep_combine into y[T, H] (bf16)."""
    P = ctypes.c_void_p
    err = error_word(y.device) if err is None else err
    st = lib.moe_ep_combine(ctypes.byref(cfg), topk_idx.shape[0], P(topk_idx.data_ptr()),
                            P(dst_row.data_ptr()), P(topk_w.data_ptr()), _ptr_table(peer_expert_out),
                            rows_cap, P(y.data_ptr()), P(err.data_ptr()), P(_stream_ptr(stream)))
    _ok(st, "moe_ep_combine")
