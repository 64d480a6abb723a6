"""Expert-parallel dispatch and combine of one rank in a torch.distributed group.

"Enabling trillion-parameter models on AWS EFA", sections "Buffers de Envio e
Recebimento" and "Despacho e Combinação": the ranks first exchange their
per-expert counts; from them each sender computes, for every peer, the range
its rows take in that peer's receive buffer, and writes them there itself (one
receive buffer per rank, no per-sender space).  On one node the receive and
expert-output buffers of the peers are opened through CUDA IPC, and the
library's kernels store to and load from them directly (plain 16-byte
accesses over NVLink, no TMA, no multicast).

Ordering between ranks is a stream synchronisation and a group barrier: after
every rank's payload (before the experts read their buffers) and after the
experts (before the combine reads the peers' outputs).  This module only
marshals; every step runs in the library's kernels or in the group's
collectives.
"""
from __future__ import annotations

import ctypes
from typing import Optional

import torch
import torch.distributed as dist

from . import (_ok, _stream_ptr, ep_combine_into, ep_dispatch_payload_into,
               ep_layout_into, ep_rows_capacity, error_word, lib, make_config, moe_dispatch_out,
               workspace_bytes)


def exchange_counts(counts: torch.Tensor, group=None) -> torch.Tensor:
    """Every rank's per-expert counts, [W, E], gathered on every rank."""
    W = dist.get_world_size(group)
    parts = [torch.empty_like(counts) for _ in range(W)]
    dist.all_gather(parts, counts.contiguous(), group=group)
    return torch.stack(parts)


def share_buffers(tensors, group=None):
    """For each local CUDA tensor, every rank's tensor of the same role (this
    rank's own at its index), the others opened through CUDA IPC."""
    from torch.multiprocessing.reductions import reduce_tensor
    rank, W = dist.get_rank(group), dist.get_world_size(group)
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


class ExpertParallel:
    """One rank of expert-parallel dispatch/combine over a group of W ranks.

    cfg: H, k, E (global experts; rank d hosts [d E/W, (d+1) E/W)), fp8, pad128.
    T_max: the most tokens any rank dispatches at once (sizes the buffers).
    """

    def __init__(self, H: int, k: int, E: int, fp8: bool, pad128: bool, T_max: int,
                 group=None, device=None):
        self.group = group
        self.W, self.rank = dist.get_world_size(group), dist.get_rank(group)
        self.device = torch.device("cuda", torch.cuda.current_device()) if device is None \
            else torch.device(device)
        self.cfg = make_config(H, k, E, self.W, fp8, pad128)
        self.local_cfg = make_config(H, k, E, 1, False, False)
        self.rows_cap = ep_rows_capacity(self.cfg, T_max)
        e = dict(device=self.device)
        self.recv_x = torch.empty((self.rows_cap, H), dtype=torch.float8_e4m3fn if fp8 else torch.bfloat16, **e)
        self.recv_scale = torch.empty((self.rows_cap, H // 128), dtype=torch.float32, **e) if fp8 else None
        self.expert_out = torch.empty((self.rows_cap, H), dtype=torch.bfloat16, **e)
        El = E // self.W
        self.recv_count = torch.empty(El, dtype=torch.int32, **e)
        self.recv_offset = torch.empty(El + 1, dtype=torch.int32, **e)
        shared = share_buffers([t for t in (self.recv_x, self.recv_scale, self.expert_out)
                                if t is not None], group)
        self.peer_recv_x = shared[0]
        self.peer_recv_scale = shared[1] if fp8 else None
        self.peer_expert_out = shared[-1]
        self.err = error_word(self.device)

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
        """Writes this rank's rows into the hosting ranks' buffers; returns
        dst_row[T, k] for the combine.  On return every rank's rows are in place
        (the group has passed the barrier)."""
        if topk_idx.dtype == torch.int64:
            topk_idx = topk_idx.to(torch.int32)
        count, offset, slot = self._local_layout(topk_idx, stream)
        counts_all = exchange_counts(count, self.group)
        dst_row = torch.empty_like(slot)
        ep_layout_into(self.cfg, self.rank, topk_idx, slot, offset, counts_all, self.rows_cap,
                       dst_row, self.recv_count, self.recv_offset, self.err, stream)
        ep_dispatch_payload_into(self.cfg, x, topk_idx, dst_row, self.peer_recv_x,
                                 self.peer_recv_scale, self.rows_cap, self.err, stream)
        torch.cuda.synchronize(self.device)
        dist.barrier(group=self.group)
        return dst_row

    def combine(self, topk_idx: torch.Tensor, dst_row: torch.Tensor, topk_w: torch.Tensor,
                stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
        """y[T, H] from the hosting ranks' expert outputs; call once every rank's
        experts have written expert_out (this waits for the group first)."""
        if topk_idx.dtype == torch.int64:
            topk_idx = topk_idx.to(torch.int32)
        torch.cuda.synchronize(self.device)
        dist.barrier(group=self.group)
        y = torch.empty((topk_idx.shape[0], self.cfg.H), dtype=torch.bfloat16, device=self.device)
        ep_combine_into(self.cfg, topk_idx, dst_row, topk_w, self.peer_expert_out, self.rows_cap, y,
                        self.err, stream)
        return y
