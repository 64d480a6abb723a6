"""Seeded synthetic inputs for MoE token dispatch and combine.

This module only draws random numbers and shapes them into the inputs of the
dispatch/combine path: hidden vectors, router choices and routing weights, and
the experts' output rows.  It holds none of the dispatch or combine arithmetic,
so both the CUDA path and the CPU oracle can take their inputs from here.

The workloads stand in for the settings that "Enabling trillion-parameter
models on AWS EFA" (section "Avaliação" / Evaluation) measures on: DeepSeek-V3
and Kimi-K2 style MoE layers with hidden size 7168, decode batches of 128 tokens
and prefill batches of 4096 tokens.  No dataset or trained weights are used:
hidden vectors and expert outputs are N(0,1) rounded to bf16, and the routing is
drawn from the distributions below.

Every array is a plain NumPy array.  bf16 data is carried as uint16 bit
patterns (the top half of an IEEE binary32).
"""
from __future__ import annotations

import dataclasses

import numpy as np

# Rows of a bf16 payload are drawn in blocks of this many rows, each block from
# its own seeded stream, so any row can be regenerated on its own.
ROW_BLOCK = 256

# Sub-stream ids of one workload seed.
_STREAM_X = 1
_STREAM_ROUTING = 2
_STREAM_EXPERT_OUT = 3


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape and routing recipe of one synthetic dispatch/combine problem."""

    name: str
    T: int            # tokens
    H: int            # hidden size
    E: int            # experts
    R: int            # virtual ranks; rank r hosts experts [r*E/R, (r+1)*E/R)
    k: int            # experts per token
    routing: str      # "softmax_topk" | "sigmoid_topk" | "uniform_dirichlet" | "zipf_softmax"
    fp8: bool         # dispatch payload quantised to fp8 e4m3 with per-128 scales
    pad128: bool      # per-expert receive segments padded to a multiple of 128 rows
    identity_experts: bool  # combine input is the dispatched bf16 payload itself
    zipf_s: float = 1.2
    seed: int = 0
    note: str = ""


WORKLOADS: dict[str, Workload] = {
    w.name: w
    for w in [
        Workload("tiny", T=16, H=256, E=8, R=2, k=2, routing="softmax_topk",
                 fp8=False, pad128=False, identity_experts=True,
                 note="top-2 of softmax(N(0,1) logits), renormalised weights"),
        Workload("dsv3_decode", T=128, H=7168, E=256, R=8, k=8, routing="sigmoid_topk",
                 fp8=True, pad128=False, identity_experts=False,
                 note="DeepSeek-V3-shaped decode: top-8 of sigmoid(N(0,1)), weights sum to 1"),
        Workload("kimi_decode", T=128, H=7168, E=384, R=16, k=8, routing="uniform_dirichlet",
                 fp8=True, pad128=False, identity_experts=False,
                 note="Kimi-K2-shaped decode: 8 uniform distinct experts, Dirichlet(1) weights"),
        Workload("prefill_zipf", T=4096, H=7168, E=256, R=32, k=8, routing="zipf_softmax",
                 fp8=False, pad128=False, identity_experts=False,
                 note="prefill with load imbalance: Zipf(1.2) over a seeded expert permutation"),
    ]
    + [
        Workload(f"sweep_{T}", T=T, H=7168, E=256, R=32, k=8, routing="uniform_dirichlet",
                 fp8=True, pad128=True, identity_experts=False,
                 note="batch sweep: uniform routing, Dirichlet(1) weights, fp8, PAD128")
        for T in (256, 1024, 4096, 16384)
    ]
}


def _rng(seed: int, *stream: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([seed, *stream]))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); return uint16 bits.

    Inputs here are finite, so no NaN handling is needed.
    """
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    bias = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + bias) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def normal_bf16_rows(seed: int, stream: int, row0: int, nrows: int, H: int) -> np.ndarray:
    """Rows [row0, row0+nrows) of an N(0,1) bf16 matrix with H columns.

    Row blocks of ROW_BLOCK rows come from independent seeded streams, so the
    result for a row does not depend on which range it was requested in.
    """
    out = np.empty((nrows, H), dtype=np.uint16)
    if nrows == 0:
        return out
    b0, b1 = row0 // ROW_BLOCK, (row0 + nrows - 1) // ROW_BLOCK
    for b in range(b0, b1 + 1):
        blk = _rng(seed, stream, b).standard_normal((ROW_BLOCK, H), dtype=np.float32)
        lo = max(row0, b * ROW_BLOCK)
        hi = min(row0 + nrows, (b + 1) * ROW_BLOCK)
        out[lo - row0:hi - row0] = f32_to_bf16_bits(blk[lo - b * ROW_BLOCK:hi - b * ROW_BLOCK])
    return out


def _topk_desc(scores: np.ndarray, k: int) -> np.ndarray:
    # Highest score first; equal scores keep ascending expert id (stable sort).
    return np.argsort(-scores, axis=1, kind="stable")[:, :k].astype(np.int32)


def make_router_logits(w: Workload) -> np.ndarray:
    """The N(0,1) router logits[T,E] (float64) behind the softmax / sigmoid workloads."""
    if w.routing not in ("softmax_topk", "sigmoid_topk"):
        raise ValueError(f"{w.name} draws its routing without logits")
    return _rng(w.seed, _STREAM_ROUTING).standard_normal((w.T, w.E))


def make_routing(w: Workload) -> tuple[np.ndarray, np.ndarray]:
    """Router choices topk_idx[T,k] (int32) and weights topk_w[T,k] (float32)."""
    rng = _rng(w.seed, _STREAM_ROUTING)
    T, E, k = w.T, w.E, w.k
    if w.routing == "softmax_topk":
        logits = rng.standard_normal((T, E))
        p = np.exp(logits - logits.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        idx = _topk_desc(p, k)
        sel = np.take_along_axis(p, idx, axis=1)
        wts = sel / sel.sum(axis=1, keepdims=True)
    elif w.routing == "sigmoid_topk":
        logits = rng.standard_normal((T, E))
        s = 1.0 / (1.0 + np.exp(-logits))
        idx = _topk_desc(s, k)
        sel = np.take_along_axis(s, idx, axis=1)
        wts = sel / sel.sum(axis=1, keepdims=True)
    elif w.routing == "uniform_dirichlet":
        idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
        wts = rng.dirichlet(np.ones(k), size=T)
    elif w.routing == "zipf_softmax":
        perm = rng.permutation(E)
        p = np.empty(E)
        p[perm] = (np.arange(E) + 1.0) ** (-w.zipf_s)
        p /= p.sum()
        idx = np.stack([rng.choice(E, k, replace=False, p=p) for _ in range(T)]).astype(np.int32)
        logits = rng.standard_normal((T, k))
        e = np.exp(logits - logits.max(axis=1, keepdims=True))
        wts = e / e.sum(axis=1, keepdims=True)
    else:
        raise ValueError(f"unknown routing {w.routing!r}")
    return np.ascontiguousarray(idx, dtype=np.int32), np.ascontiguousarray(wts, dtype=np.float32)


def make_x(w: Workload) -> np.ndarray:
    """Hidden vectors x[T,H] as bf16 bits, N(0,1)."""
    return normal_bf16_rows(w.seed, _STREAM_X, 0, w.T, w.H)


def make_expert_out(w: Workload, nrows: int, row0: int = 0) -> np.ndarray:
    """Rows [row0, row0+nrows) of the experts' bf16 output, N(0,1).

    The combine input has the receive-buffer layout; its row count is the
    receive capacity chosen by the caller.
    """
    return normal_bf16_rows(w.seed, _STREAM_EXPERT_OUT, row0, nrows, w.H)


def make_inputs(name_or_workload, **overrides):
    """(workload, x, topk_idx, topk_w) for a named workload."""
    w = WORKLOADS[name_or_workload] if isinstance(name_or_workload, str) else name_or_workload
    if overrides:
        w = dataclasses.replace(w, **overrides)
    idx, wts = make_routing(w)
    return w, make_x(w), idx, wts


def random_problem(seed: int, T: int, H: int, E: int, k: int, *, distinct: bool = True):
    """A small random problem for parity sweeps: uniform routing, Dirichlet weights."""
    rng = _rng(seed, 7)
    if distinct:
        idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]) if T else np.zeros((0, k))
    else:
        idx = rng.integers(0, E, size=(T, k))
    wts = rng.dirichlet(np.ones(k), size=T) if T else np.zeros((0, k))
    x = f32_to_bf16_bits(rng.standard_normal((T, H), dtype=np.float32))
    return (x, np.ascontiguousarray(idx, dtype=np.int32),
            np.ascontiguousarray(wts, dtype=np.float32))
