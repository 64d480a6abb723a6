"""CPU oracle for MoE token dispatch and combine -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the bench's CPU-baseline leg
may import this package.  The product path (``combine_route_meta_b200``) never
does, and the two share no code.

The arithmetic lives in ``moe_oracle.c`` (plain, single-threaded C, compiled
with gcc without fast-math or FMA contraction, so float operations are IEEE
binary32/binary64 with round-to-nearest).  This module only builds that file
and passes NumPy arrays to it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

BAD_INDEX = 1
CAPACITY = 2

GCC_FLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
             "-ffp-contract=off", "-fno-finite-math-only"]


def build(force: bool = False) -> str:
    """Compile moe_oracle.c into liboracle.so next to it (if missing or stale)."""
    with _lock:
        stale = (not os.path.exists(_LIB)
                 or os.path.getmtime(_LIB) < os.path.getmtime(_SRC))
        if force or stale:
            tmp = _LIB + f".tmp{os.getpid()}"
            subprocess.check_call(["gcc", *GCC_FLAGS, "-o", tmp, _SRC, "-lquadmath", "-lm"])
            os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i32, i64 = ctypes.c_int32, ctypes.c_int64
        lib.oracle_e4m3_from_float.argtypes = [ctypes.c_float]
        lib.oracle_e4m3_from_float.restype = ctypes.c_uint8
        lib.oracle_dispatch.argtypes = [i32, i32, i32, i32, i32, i32, i32, i64,
                                        P, P, P, P, P, P, P, P, P]
        lib.oracle_dispatch.restype = i32
        lib.oracle_dispatch_layout.argtypes = [i32, i32, i32, i32, i32, i64, P, P, P, P, P, P]
        lib.oracle_dispatch_layout.restype = i32
        lib.oracle_dispatch_payload_rows.argtypes = [i32, i32, i32, i32, i32, P, P, P, P]
        lib.oracle_dispatch_payload_rows.restype = None
        lib.oracle_combine.argtypes = [i32, i32, i32, P, P, P, P]
        lib.oracle_combine.restype = None
        lib.oracle_combine_rank_partial.argtypes = [i32, i32, i32, i32, i32, P, P, P, P, P, P, P, P]
        lib.oracle_combine_rank_partial.restype = None
        lib.oracle_silu_mul.argtypes = [ctypes.c_float, ctypes.c_float]
        lib.oracle_silu_mul.restype = ctypes.c_float
        lib.oracle_silu_mul_many.argtypes = [i64, P, P, P]
        lib.oracle_silu_mul_many.restype = None
        lib.oracle_silu_quant.argtypes = [i64, i32, P, P, i64, P, P, i32]
        lib.oracle_silu_quant.restype = None
        lib.oracle_router_topk.argtypes = [i32, i32, i32, P, i32, i32, i32, i32, P, P]
        lib.oracle_router_topk.restype = None
        lib.oracle_quantise_row_fp8.argtypes = [P, i32, P, P]
        lib.oracle_quantise_row_fp8.restype = None
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def e4m3_from_float(v: float) -> int:
    """e4m3 code of one float: nearest, ties to even, saturated to +-448."""
    return int(_load().oracle_e4m3_from_float(float(np.float32(v))))


def quantise_row_fp8(x_bf16: np.ndarray):
    """(codes uint8[H], scales float32[H/128]) of one bf16 row."""
    x = _c(x_bf16, np.uint16)
    H = x.shape[0]
    if H % 128:
        raise ValueError("fp8 block quantisation needs H % 128 == 0")
    codes = np.zeros(H, np.uint8)
    scales = np.zeros(H // 128, np.float32)
    _load().oracle_quantise_row_fp8(_ptr(x), H, _ptr(codes), _ptr(scales))
    return codes, scales


def rows_capacity(T: int, k: int, E: int, pad128: bool) -> int:
    """Worst-case receive rows.

    Unpadded: T*k.  Padded: the most 128-row blocks S = T*k entries can fill when
    split over at most m = min(E, S) experts is reached by m-1 experts with one
    entry each and the rest in one expert: (m-1) + ceil((S-m+1)/128) blocks,
    which equals floor((S + 127*m) / 128).
    """
    S = T * k
    if not pad128:
        return S
    used = min(E, S)
    return (S + 127 * used) // 128 * 128


def dispatch(x_bf16, topk_idx, *, E: int, R: int, fp8: bool, pad128: bool = False,
             rows_cap: int | None = None, recv_fill: int = 0):
    """Run the oracle dispatch.  Returns a dict of NumPy arrays plus 'err'.

    recv_x / recv_scale rows that receive no entry keep ``recv_fill`` bytes.
    """
    x = _c(x_bf16, np.uint16)
    idx = _c(topk_idx, np.int32)
    T, H = x.shape
    k = idx.shape[1] if idx.ndim == 2 else 0
    if idx.shape[0] != T:
        raise ValueError("x and topk_idx disagree on T")
    if R <= 0 or E <= 0 or E % R:
        raise ValueError("E must be a positive multiple of R")
    if fp8 and H % 128:
        raise ValueError("fp8 dispatch needs H % 128 == 0")
    if rows_cap is None:
        rows_cap = rows_capacity(T, k, E, pad128)
    nb = H // 128
    if fp8:
        recv_x = np.full((rows_cap, H), recv_fill, np.uint8)
        recv_scale = np.full((rows_cap, nb), 0, np.float32)
        if recv_fill:
            recv_scale.view(np.uint8)[:] = recv_fill
    else:
        recv_x = np.full((rows_cap, H), recv_fill * 0x0101, np.uint16)
        recv_scale = np.zeros((0, 0), np.float32)
    out = dict(
        recv_x=recv_x,
        recv_scale=recv_scale,
        expert_count=np.zeros(E, np.int32),
        expert_offset=np.zeros(E + 1, np.int32),
        rank_offset=np.zeros(R + 1, np.int32),
        recv_src=np.zeros(rows_cap, np.int32),
        slot=np.zeros((T, k), np.int32),
    )
    err = _load().oracle_dispatch(
        T, H, k, E, R, int(bool(fp8)), int(bool(pad128)), rows_cap,
        _ptr(x), _ptr(idx), _ptr(out["recv_x"]), _ptr(out["recv_scale"]),
        _ptr(out["expert_count"]), _ptr(out["expert_offset"]), _ptr(out["rank_offset"]),
        _ptr(out["recv_src"]), _ptr(out["slot"]))
    out["err"] = int(err)
    out["rows_cap"] = rows_cap
    return out


def _ranges(T: int, parts: int):
    step = (T + parts - 1) // parts if T else 0
    return [(a, min(T, a + step)) for a in range(0, T, step)] if step else []


def dispatch_parallel(x_bf16, topk_idx, *, E: int, R: int, fp8: bool, pad128: bool = False,
                      rows_cap: int | None = None, threads: int = 1):
    """dispatch() with its payload step split over `threads` host threads by
    token range (the layout stays one serial walk).  The same C functions run on
    disjoint tokens, so the result is bitwise that of dispatch(); the C calls
    release the interpreter lock, so the ranges run on separate cores."""
    from concurrent.futures import ThreadPoolExecutor
    x = _c(x_bf16, np.uint16)
    idx = _c(topk_idx, np.int32)
    T, H = x.shape
    k = idx.shape[1] if idx.ndim == 2 else 0
    if rows_cap is None:
        rows_cap = rows_capacity(T, k, E, pad128)
    nb = H // 128
    recv_x = np.zeros((rows_cap, H), np.uint8 if fp8 else np.uint16)
    recv_scale = np.zeros((rows_cap, nb), np.float32) if fp8 else np.zeros((0, 0), np.float32)
    out = dict(recv_x=recv_x, recv_scale=recv_scale, expert_count=np.zeros(E, np.int32),
               expert_offset=np.zeros(E + 1, np.int32), rank_offset=np.zeros(R + 1, np.int32),
               recv_src=np.zeros(rows_cap, np.int32), slot=np.zeros((T, k), np.int32))
    lib = _load()
    out["err"] = int(lib.oracle_dispatch_layout(
        T, k, E, R, int(bool(pad128)), rows_cap, _ptr(idx), _ptr(out["expert_count"]),
        _ptr(out["expert_offset"]), _ptr(out["rank_offset"]), _ptr(out["recv_src"]), _ptr(out["slot"])))
    with ThreadPoolExecutor(max(1, threads)) as ex:
        list(ex.map(lambda r: lib.oracle_dispatch_payload_rows(
            r[0], r[1], H, k, int(bool(fp8)), _ptr(x), _ptr(out["slot"]), _ptr(recv_x), _ptr(recv_scale)),
            _ranges(T, max(1, threads))))
    out["rows_cap"] = rows_cap
    return out


def combine_parallel(slot, topk_w, expert_out_bf16, threads: int = 1) -> np.ndarray:
    """combine() over `threads` host threads by token range; bitwise the same."""
    from concurrent.futures import ThreadPoolExecutor
    slot = _c(slot, np.int32)
    w = _c(topk_w, np.float32)
    eo = _c(expert_out_bf16, np.uint16)
    T = slot.shape[0]
    k = slot.shape[1] if slot.ndim == 2 else 0
    H = eo.shape[1]
    y = np.zeros((T, H), np.float64)
    lib = _load()
    with ThreadPoolExecutor(max(1, threads)) as ex:
        list(ex.map(lambda r: lib.oracle_combine(r[1] - r[0], H, k, _ptr(slot[r[0]:r[1]]), _ptr(w[r[0]:r[1]]),
                                                 _ptr(eo), _ptr(y[r[0]:r[1]])),
                    _ranges(T, max(1, threads))))
    return y


def combine(slot, topk_w, expert_out_bf16, tokens=None) -> np.ndarray:
    """fp64 routing-weighted sum y[t,:] = sum_j w[t,j] * expert_out[slot[t,j],:].

    With ``tokens`` given, only those rows of y are computed (in that order).
    """
    slot = _c(slot, np.int32)
    w = _c(topk_w, np.float32)
    eo = _c(expert_out_bf16, np.uint16)
    if tokens is not None:
        tokens = np.asarray(tokens, dtype=np.int64)
        slot = np.ascontiguousarray(slot[tokens])
        w = np.ascontiguousarray(w[tokens])
    T = slot.shape[0]
    k = slot.shape[1] if slot.ndim == 2 else 0
    H = eo.shape[1]
    if slot.size and slot.max() >= eo.shape[0]:
        raise ValueError("slot points past expert_out")
    y = np.zeros((T, H), np.float64)
    _load().oracle_combine(T, H, k, _ptr(slot), _ptr(w), _ptr(eo), _ptr(y))
    return y


def combine_rank_partial(topk_idx, slot, topk_w, expert_out_bf16, *, E: int, R: int):
    """Sender-side (per-rank) partial combine.  Returns dict with partial
    (uint16 [T,k,H], bf16 bits), partial_rank [T,k], npart [T], y (fp64 [T,H])."""
    idx = _c(topk_idx, np.int32)
    slot = _c(slot, np.int32)
    w = _c(topk_w, np.float32)
    eo = _c(expert_out_bf16, np.uint16)
    T = slot.shape[0]
    k = slot.shape[1] if slot.ndim == 2 else 0
    H = eo.shape[1]
    out = dict(partial=np.zeros((T, k, H), np.uint16), partial_rank=np.full((T, k), -1, np.int32),
               npart=np.zeros(T, np.int32), y=np.zeros((T, H), np.float64))
    _load().oracle_combine_rank_partial(T, H, k, E, R, _ptr(idx), _ptr(slot), _ptr(w), _ptr(eo),
                                        _ptr(out["partial"]), _ptr(out["partial_rank"]),
                                        _ptr(out["npart"]), _ptr(out["y"]))
    return out


def silu_mul(g: float, u: float = 1.0) -> float:
    """The activation silu(g) * u: the binary32 value nearest the real one (see moe_oracle.c)."""
    return float(_load().oracle_silu_mul(float(np.float32(g)), float(np.float32(u))))


def silu_mul_bits(g_bf16, u_bf16) -> np.ndarray:
    """silu_mul over arrays of bf16 bit patterns; float32 results of the same shape."""
    g = _c(g_bf16, np.uint16)
    u = _c(np.broadcast_to(u_bf16, g.shape), np.uint16)
    out = np.empty(g.shape, np.float32)
    _load().oracle_silu_mul_many(g.size, _ptr(g), _ptr(u), _ptr(out))
    return out


def silu_quant(gate_up_bf16, recv_src, rows_in_use: int, *, col_major: bool = False,
               fill: int = 0):
    """(act uint8 [rows_cap, I], scale float32) of the expert-side SiLU + block quantiser.
    Rows that are not written keep `fill` bytes."""
    gu = _c(gate_up_bf16, np.uint16)
    src = _c(recv_src, np.int32)
    rows_cap, two_i = gu.shape
    I = two_i // 2
    if I % 128:
        raise ValueError("I must be a multiple of 128")
    act = np.full((rows_cap, I), fill, np.uint8)
    shape = (I // 128, rows_cap) if col_major else (rows_cap, I // 128)
    scale = np.zeros(shape, np.float32)
    if fill:
        scale.view(np.uint8)[:] = fill
    _load().oracle_silu_quant(rows_cap, I, _ptr(gu), _ptr(src), int(rows_in_use), _ptr(act),
                              _ptr(scale), int(bool(col_major)))
    return act, scale


def router_topk(logits, k: int, *, score_fn: str = "softmax", n_group: int = 1,
                topk_group: int = 1, renormalize: bool = True):
    """(topk_idx int32 [T,k], topk_w float32 [T,k]) of group-limited top-k routing."""
    l = _c(logits, np.float32)
    T, E = l.shape
    if k > 64 or E % n_group or not (1 <= topk_group <= n_group) or k > topk_group * (E // n_group):
        raise ValueError("unsupported router shape")
    idx = np.zeros((T, k), np.int32)
    w = np.zeros((T, k), np.float32)
    _load().oracle_router_topk(T, E, k, _ptr(l), {"softmax": 0, "sigmoid": 1}[score_fn], n_group,
                               topk_group, int(bool(renormalize)), _ptr(idx), _ptr(w))
    return idx, w
