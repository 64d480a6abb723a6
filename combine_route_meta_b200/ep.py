"""Expert-parallel dispatch and combine of one rank in a torch.distributed group.

"Enabling trillion-parameter models on AWS EFA", sections "Buffers de Envio e
Recebimento" and "Despacho e Combinação": the ranks first exchange their
per-expert counts; from them each sender computes, for every peer, the range
its rows take in that peer's receive buffer, and writes them there itself (one
receive buffer per rank, no per-sender space).  A receiver uses its buffer once
every sender has signalled that its writes are complete.  On one node the
receive and expert-output buffers of the peers, and their completion flags, are
opened through CUDA IPC, and the library's kernels store to and load from them
directly (plain accesses over NVLink, no TMA, no multicast).

Ordering between ranks is on the device: the payload kernel of each sender
signals "rows in place" to every peer when its last CTA finishes, and a bounded
wait kernel on each receiver holds its stream until every sender has signalled;
after the experts, each rank signals "outputs ready" and waits for every peer's
signal before its combine reads their outputs.  The host never blocks, so a
layer's exchange can be captured in a CUDA graph (the count exchange is an NCCL
all-gather, which graphs capture too).  A wait that runs out of time sets the
device error bit MOE_DEV_TIMEOUT; check() reads and clears the error word.

This module only marshals; every step runs in the library's kernels or in the
group's collectives.
"""
from __future__ import annotations

import ctypes
from typing import Optional

import torch
import torch.distributed as dist

from . import (MoeError, ERR_DEVICE, _ok, _stream_ptr, ep_combine_into, ep_dispatch_payload_into,
               ep_layout_into, ep_rows_capacity, ep_signal_into, ep_wait_into, lib, make_config,
               moe_dispatch_out, workspace_bytes)


def exchange_counts(counts: torch.Tensor, group=None, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Every rank's per-expert counts, [W, E], gathered on every rank (into `out` if given)."""
    W = dist.get_world_size(group)
    if out is None:
        out = torch.empty((W, counts.numel()), dtype=counts.dtype, device=counts.device)
    dist.all_gather_into_tensor(out.view(-1), counts.contiguous().view(-1), group=group)
    return out


def share_buffers(tensors, group=None):
    """For each local CUDA tensor, every rank's tensor of the same role (this
    rank's own at its index), the others opened through CUDA IPC."""
    from torch.multiprocessing.reductions import reduce_tensor
    rank, W = dist.get_rank(group), dist.get_world_size(group)
    if W == 1:
        return [[t] for t in tensors]
    handles = [None] * W
    dist.all_gather_object(handles, [reduce_tensor(t) for t in tensors], group=group)
    out = []
    for i, t in enumerate(tensors):
        row = []
        for r in range(W):
            if r == rank:
                row.append(t)
            else:
                rebuild, args = handles[r][i]
                row.append(rebuild(*args))
        out.append(row)
    return out


def check_batch(T: int, T_max: int) -> None:
    """The receive buffers hold every rank's T_max tokens at most: a larger batch
    would overflow them, so it is refused before anything is launched."""
    if T < 0 or T > T_max:
        raise ValueError(f"batch of {T} tokens outside [0, T_max={T_max}] of this ExpertParallel")


class ExpertParallel:
    """One rank of expert-parallel dispatch/combine over a group of W ranks.

    H, k, E (global experts; rank d hosts [d E/W, (d+1) E/W)), fp8, pad128.
    T_max: the most tokens any rank dispatches at once (sizes the buffers).
    wait_limit_s: how long a device wait for the peers may take before it gives
    up with MOE_DEV_TIMEOUT.

    Per layer, on one stream:  dst_row = dispatch(x, topk_idx);  the experts read
    recv_x (recv_count / recv_offset give their segments) and write expert_out;
    experts_done();  y = combine(topk_idx, dst_row, topk_w).  check() reports
    device errors (bad ids, timeouts).
    """

    def __init__(self, H: int, k: int, E: int, fp8: bool, pad128: bool, T_max: int,
                 group=None, device=None, wait_limit_s: float = 1.0):
        self.group = group
        self.W, self.rank = dist.get_world_size(group), dist.get_rank(group)
        self.device = torch.device("cuda", torch.cuda.current_device()) if device is None \
            else torch.device(device)
        self.T_max = int(T_max)
        self.wait_limit_ns = int(wait_limit_s * 1e9)
        self.cfg = make_config(H, k, E, self.W, fp8, pad128)
        self.local_cfg = make_config(H, k, E, 1, False, False)
        self.rows_cap = ep_rows_capacity(self.cfg, self.T_max)
        e = dict(device=self.device)
        i32 = dict(dtype=torch.int32, device=self.device)
        self.recv_x = torch.empty((self.rows_cap, H), dtype=torch.float8_e4m3fn if fp8 else torch.bfloat16, **e)
        self.recv_scale = torch.empty((self.rows_cap, H // 128), dtype=torch.float32, **e) if fp8 else None
        self.expert_out = torch.empty((self.rows_cap, H), dtype=torch.bfloat16, **e)
        El = E // self.W
        self.recv_count = torch.empty(El, **i32)
        self.recv_offset = torch.empty(El + 1, **i32)
        # completion: one flag per sender for "rows in place" and for "outputs
        # ready"; this rank's epochs of the two events; the payload's CTA count
        self.flags_rows = torch.zeros(self.W, **i32)
        self.flags_out = torch.zeros(self.W, **i32)
        self.epochs = torch.zeros(2, **i32)
        self.done = torch.zeros(1, **i32)
        self.counts_all = torch.empty((self.W, E), **i32)
        bufs = [self.recv_x, self.recv_scale, self.expert_out, self.flags_rows, self.flags_out]
        shared = share_buffers([t for t in bufs if t is not None], group)
        self.peer_recv_x = shared[0]
        self.peer_recv_scale = shared[1] if fp8 else None
        self.peer_expert_out = shared[-3]
        self.peer_flags_rows = shared[-2]
        self.peer_flags_out = shared[-1]
        self.err = torch.zeros(1, **i32)
        # every rank's flags are zero and mapped before any rank signals
        torch.cuda.synchronize(self.device)
        dist.barrier(group=group)

    def _local_layout(self, topk_idx: torch.Tensor, stream):
        """This rank's one-rank unpadded layout: counts, offsets and slots."""
        T, k = topk_idx.shape
        e = dict(dtype=torch.int32, device=self.device)
        E = self.cfg.E
        count, offset, rank_off = torch.empty(E, **e), torch.empty(E + 1, **e), torch.empty(2, **e)
        src, slot = torch.empty(max(T * k, 1), **e), torch.empty((T, k), **e)
        nws = workspace_bytes(self.local_cfg, T)
        ws = torch.empty(max(nws, 1), dtype=torch.uint8, device=self.device)
        out = moe_dispatch_out(None, None, count.data_ptr(), offset.data_ptr(), rank_off.data_ptr(),
                               src.data_ptr(), T * k)
        P = ctypes.c_void_p
        st = lib.moe_dispatch_layout(ctypes.byref(self.local_cfg), T, P(topk_idx.data_ptr()),
                                     ctypes.byref(out), P(slot.data_ptr()), P(ws.data_ptr()), nws,
                                     P(self.err.data_ptr()), P(_stream_ptr(stream)))
        _ok(st, "moe_dispatch_layout")
        return count, offset, slot

    def dispatch(self, x: torch.Tensor, topk_idx: torch.Tensor,
                 stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
        """Writes this rank's rows into the hosting ranks' buffers and returns
        dst_row[T, k] for the combine.  Work after this call on the same stream
        sees every sender's rows in this rank's recv_x."""
        check_batch(topk_idx.shape[0], self.T_max)
        if topk_idx.dtype == torch.int64:
            topk_idx = topk_idx.to(torch.int32)
        s = stream if stream is not None else torch.cuda.current_stream(self.device)
        with torch.cuda.stream(s):
            count, offset, slot = self._local_layout(topk_idx, s)
            exchange_counts(count, self.group, out=self.counts_all)
            dst_row = torch.empty_like(slot)
            ep_layout_into(self.cfg, self.rank, topk_idx, slot, offset, self.counts_all, self.rows_cap,
                           dst_row, self.recv_count, self.recv_offset, self.err, s)
            ep_dispatch_payload_into(self.cfg, x, topk_idx, dst_row, self.peer_recv_x,
                                     self.peer_recv_scale, self.rows_cap, self.err, s,
                                     signal=(self.rank, self.peer_flags_rows, self.epochs[0:1], self.done))
            ep_wait_into(self.flags_rows, self.epochs[0:1], self.wait_limit_ns, self.err, s)
        return dst_row

    def experts_done(self, stream: Optional[torch.cuda.Stream] = None) -> None:
        """Signals every peer that this rank's expert_out is written (call after
        the experts' kernels, on their stream)."""
        ep_signal_into(self.rank, self.peer_flags_out, self.epochs[1:2], stream)

    def combine(self, topk_idx: torch.Tensor, dst_row: torch.Tensor, topk_w: torch.Tensor,
                stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
        """y[T, H] from the hosting ranks' expert outputs, once every peer has
        signalled experts_done()."""
        if topk_idx.dtype == torch.int64:
            topk_idx = topk_idx.to(torch.int32)
        ep_wait_into(self.flags_out, self.epochs[1:2], self.wait_limit_ns, self.err, stream)
        y = torch.empty((topk_idx.shape[0], self.cfg.H), dtype=torch.bfloat16, device=self.device)
        ep_combine_into(self.cfg, topk_idx, dst_row, topk_w, self.peer_expert_out, self.rows_cap, y,
                        self.err, stream)
        return y

    def check(self, stream: Optional[torch.cuda.Stream] = None) -> None:
        """Synchronises the stream, reads and clears the device error word, and
        raises MoeError if a kernel reported a bad id, a capacity overflow or a
        wait that ran out of time."""
        bits = ctypes.c_int32(0)
        P = ctypes.c_void_p
        lib.moe_check(P(self.err.data_ptr()), P(_stream_ptr(stream)), ctypes.byref(bits))
        if bits.value:
            raise MoeError(ERR_DEVICE, f"expert-parallel device error bits {bits.value}")
