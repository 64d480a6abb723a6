"""Expert-parallel dispatch/combine, checked on one GPU.

W virtual ranks run their layout, payload and combine one after another on one
device; the "peer" buffer table holds W separate local buffers, so the kernels'
addressing is exactly that of W GPUs writing into each other's buffers.  Rank
d's buffer must equal rows [rank_offset[d], rank_offset[d+1]) of the oracle's
single-GPU dispatch of all ranks' batches concatenated in rank order (R = W),
and each rank's combine must equal, bit for bit, the single-GPU combine of the
concatenated batch for its tokens.  The ranks' completion flags are exercised
in the one stream (all payloads, which signal, before all waits).  A one-rank
NCCL group runs the host orchestration (count exchange, buffer sharing,
device-side completion, graph capture) end to end.
"""
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch

import oracle
from tests._lib import bf16_from_dev, bf16_to_dev, to_dev
from workloads import normal_bf16_rows, random_problem

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import combine_route_meta_b200 as moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
POISON = 0xA5


def _poisoned(rows, cols, dtype):
    """A [rows, cols] tensor of `dtype` whose bytes all hold POISON."""
    esize = torch.empty((), dtype=dtype).element_size()
    t = torch.full((rows, cols * esize), POISON, dtype=torch.uint8, device="cuda").view(dtype)
    assert t.shape == (rows, cols)
    return t


def _local_layout(H, k, E, idx_dev):
    cfg1 = moe.make_config(H, k, E, 1, False, False)
    buf = moe.Buffers(cfg1, idx_dev.shape[0], "cuda")
    moe.dispatch_layout_into(buf, idx_dev)
    return buf.expert_count, buf.expert_offset, buf.slot


def _signals(W):
    """Every virtual rank's completion state: its "rows" flags (one per sender),
    its epoch of the event and its payload's CTA count, all zero."""
    z = lambda n: torch.zeros(n, dtype=torch.int32, device="cuda")
    return dict(flags=[z(W) for _ in range(W)], epoch=[z(1) for _ in range(W)], done=[z(1) for _ in range(W)])


def _run_ep(W, E, k, H, Ts, fp8, pad, seed, bad_ids=False, rows_cap=None, layers=1):
    batches = [random_problem(seed + r, T, H, E, k) for r, T in enumerate(Ts)]
    if bad_ids:
        batches[0][1][0, 0] = E          # out of range
        batches[-1][1][-1, k - 1] = -3
    cfg = moe.make_config(H, k, E, W, fp8, pad)
    cap = moe.ep_rows_capacity(cfg, max(Ts)) if rows_cap is None else rows_cap
    xs = [bf16_to_dev(b[0]) for b in batches]
    idxs = [to_dev(b[1]) for b in batches]
    ws = [to_dev(b[2]) for b in batches]
    locals_ = [_local_layout(H, k, E, i) for i in idxs]
    counts_all = torch.stack([c for c, _, _ in locals_])
    recv_x = [_poisoned(cap, H, torch.uint8 if fp8 else torch.int16) for _ in range(W)]
    recv_sc = [_poisoned(cap, H // 128, torch.float32) for _ in range(W)] if fp8 else None
    El = E // W
    sig = _signals(W)
    for layer in range(layers):
        dst, rcount, roff = [], [], []
        # every sender's payload signals "rows in place" in every rank's flags;
        # the waits come after all payloads in the one stream, so none waits
        # on a kernel that has not run
        for r in range(W):
            d = torch.empty_like(locals_[r][2])
            rc = torch.empty(El, dtype=torch.int32, device="cuda")
            ro = torch.empty(El + 1, dtype=torch.int32, device="cuda")
            moe.ep_layout_into(cfg, r, idxs[r], locals_[r][2], locals_[r][1], counts_all, cap, d, rc, ro)
            moe.ep_dispatch_payload_into(cfg, xs[r], idxs[r], d, recv_x, recv_sc, cap,
                                         signal=(r, sig["flags"], sig["epoch"][r], sig["done"][r]))
            dst.append(d)
            rcount.append(rc)
            roff.append(ro)
        for r in range(W):
            moe.ep_wait_into(sig["flags"][r], sig["epoch"][r], 1_000_000_000)
        torch.cuda.synchronize()
        for r in range(W):
            assert sig["flags"][r].cpu().tolist() == [layer + 1] * W
            assert int(sig["epoch"][r].item()) == layer + 1 and int(sig["done"][r].item()) == 0
    return dict(batches=batches, cfg=cfg, cap=cap, xs=xs, idxs=idxs, ws=ws, dst=dst, rcount=rcount,
                roff=roff, recv_x=recv_x, recv_sc=recv_sc)


@pytest.mark.parametrize("W,E,k,H,Ts,fp8,pad,bad", [
    (2, 16, 4, 512, [300, 200], False, False, False),
    (4, 32, 8, 1024, [100, 0, 37, 250], True, True, False),    # an empty rank, padding
    (8, 256, 8, 7168, [128] * 8, True, False, False),          # DeepSeek-V3-shaped decode on 8 ranks
    (3, 12, 2, 256, [1000, 999, 1], False, True, True),        # bad ids dropped on two ranks
    (2, 64, 6, 2048, [3000, 2500], True, False, False),        # tiled local layouts
])
def test_ep_matches_the_concatenated_single_gpu_dispatch(W, E, k, H, Ts, fp8, pad, bad):
    moe.check()
    run = _run_ep(W, E, k, H, Ts, fp8, pad, seed=W * 100 + E, bad_ids=bad, layers=2)
    assert moe.check() == (moe.DEV_BAD_INDEX if bad else 0)
    X = np.concatenate([b[0] for b in run["batches"]])
    IDX = np.concatenate([b[1] for b in run["batches"]])
    WT = np.concatenate([b[2] for b in run["batches"]])
    o = oracle.dispatch(X, IDX, E=E, R=W, fp8=fp8, pad128=pad, recv_fill=POISON)
    ro = o["rank_offset"]
    El = E // W
    starts = np.cumsum([0] + Ts)
    for r in range(W):
        # this rank's rows in the hosting ranks' buffers
        slot_g = o["slot"][starts[r]:starts[r + 1]]
        host = np.where(IDX[starts[r]:starts[r + 1]] >= 0, IDX[starts[r]:starts[r + 1]], 0) // El
        want = np.where(slot_g >= 0, slot_g - ro[np.minimum(host, W - 1)], -1)
        np.testing.assert_array_equal(run["dst"][r].cpu().numpy(), want)
        # this rank as a host: its experts' totals and offsets in its buffer
        np.testing.assert_array_equal(run["rcount"][r].cpu().numpy(), o["expert_count"][r * El:(r + 1) * El])
        np.testing.assert_array_equal(run["roff"][r].cpu().numpy(),
                                      o["expert_offset"][r * El:(r + 1) * El + 1] - ro[r])
    for d in range(W):
        n = ro[d + 1] - ro[d]
        got = run["recv_x"][d].view(torch.uint8).cpu().numpy().reshape(run["cap"], -1)
        ref = o["recv_x"].view(np.uint8).reshape(o["recv_x"].shape[0], -1)[ro[d]:ro[d + 1]]
        np.testing.assert_array_equal(got[:n], ref)
        assert np.all(got[n:] == POISON)             # nothing past the rank's part
        if fp8:
            gs = run["recv_sc"][d].view(torch.uint8).cpu().numpy().reshape(run["cap"], -1)
            rs = o["recv_scale"].view(np.uint8).reshape(o["recv_scale"].shape[0], -1)[ro[d]:ro[d + 1]]
            np.testing.assert_array_equal(gs[:n], rs)
    # combine: each rank reads its rows from the hosting ranks' expert outputs,
    # after every rank signalled "outputs ready" and waited for the others
    out_sig = _signals(W)
    for r in range(W):
        moe.ep_signal_into(r, out_sig["flags"], out_sig["epoch"][r])
    for r in range(W):
        moe.ep_wait_into(out_sig["flags"][r], out_sig["epoch"][r], 1_000_000_000)
    rows_g = o["recv_x"].shape[0]
    eo_g = normal_bf16_rows(5, 3, 0, rows_g, H)
    eo = []
    for d in range(W):
        part = np.zeros((run["cap"], H), np.uint16)
        part[:ro[d + 1] - ro[d]] = eo_g[ro[d]:ro[d + 1]]
        eo.append(bf16_to_dev(part))
    single = moe.dispatch(bf16_to_dev(X), to_dev(IDX), to_dev(WT), E, W, fp8, pad)
    y_single = bf16_from_dev(moe.combine(single.handle, bf16_to_dev(
        np.concatenate([eo_g, np.zeros((max(0, single.recv_x.shape[0] - rows_g), H), np.uint16)]))))
    moe.check()
    for r in range(W):
        if Ts[r] == 0:
            continue
        y = torch.empty((Ts[r], H), dtype=torch.bfloat16, device="cuda")
        moe.ep_combine_into(run["cfg"], run["idxs"][r], run["dst"][r], run["ws"][r], eo, run["cap"], y)
        np.testing.assert_array_equal(bf16_from_dev(y), y_single[starts[r]:starts[r + 1]])
    assert moe.check() == 0


def test_ep_capacity_overflow_stays_inside_the_buffers():
    # per-rank buffers too small for the batch: rows past the end are dropped and
    # flagged, and the guard rows after each buffer's end keep their pattern
    W, E, k, H, Ts = 2, 8, 4, 256, [400, 400]
    cfg = moe.make_config(H, k, E, W, False, False)
    cap = 500
    moe.check()
    run = _run_ep(W, E, k, H, Ts, False, False, seed=11, rows_cap=cap + 64)
    # re-run the payload against buffers that claim only `cap` rows
    for r in range(W):
        d = torch.empty_like(run["dst"][r])
        _, off, slot = _local_layout(H, k, E, run["idxs"][r])
        counts_all = torch.stack([_local_layout(H, k, E, i)[0] for i in run["idxs"]])
        rc = torch.empty(E // W, dtype=torch.int32, device="cuda")
        ro = torch.empty(E // W + 1, dtype=torch.int32, device="cuda")
        bufs = [_poisoned(cap + 64, H, torch.int16) for _ in range(W)]
        moe.ep_layout_into(cfg, r, run["idxs"][r], slot, off, counts_all, cap, d, rc, ro)
        moe.ep_dispatch_payload_into(cfg, run["xs"][r], run["idxs"][r], d, bufs, None, cap)
        torch.cuda.synchronize()
        assert int(d.max().item()) < cap
        for b in bufs:
            assert np.all(b.view(torch.uint8).cpu().numpy().reshape(cap + 64, -1)[cap:] == POISON)
    assert moe.check() & moe.DEV_CAPACITY


def test_ep_wait_gives_up_on_a_flag_nothing_sets():
    # a sender that never signals: the wait runs out after its limit, sets the
    # timeout bit and returns, and the stream and context stay usable
    moe.check()
    flags = torch.zeros(4, dtype=torch.int32, device="cuda")
    flags[:3] = 1                                    # sender 3 never signals
    epoch = torch.ones(1, dtype=torch.int32, device="cuda")
    moe.ep_wait_into(flags, epoch, 2_000_000)        # 2 ms
    assert moe.check() == moe.DEV_TIMEOUT
    flags[3] = 1
    moe.ep_wait_into(flags, epoch, 2_000_000)
    assert moe.check() == 0
    x, idx, w = random_problem(1, 64, 256, 8, 2)     # ordinary work afterwards
    d = moe.dispatch(bf16_to_dev(x), to_dev(idx), to_dev(w), 8, 2, False)
    o = oracle.dispatch(x, idx, E=8, R=2, fp8=False)
    np.testing.assert_array_equal(d.handle.slot.cpu().numpy(), o["slot"])
    assert moe.check() == 0


def test_ep_signal_wraps_its_epoch_comparison():
    # epochs compare wrap-safe: a flag one past the int32 maximum still counts
    flags = torch.tensor([-2**31, 2**31 - 1], dtype=torch.int32, device="cuda")
    epoch = torch.tensor([2**31 - 1], dtype=torch.int32, device="cuda")
    moe.check()
    moe.ep_wait_into(flags, epoch, 2_000_000)
    assert moe.check() == 0
    flags[1] = 2**31 - 2
    moe.ep_wait_into(flags, epoch, 2_000_000)
    assert moe.check() == moe.DEV_TIMEOUT


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


ONE_RANK = r"""
import datetime, sys
import numpy as np, torch, torch.distributed as dist
sys.path.insert(0, {root!r})
torch.cuda.set_device(0)
dist.init_process_group("nccl", init_method="tcp://127.0.0.1:{port}", rank=0, world_size=1,
                        timeout=datetime.timedelta(seconds=60))
import combine_route_meta_b200 as moe
from combine_route_meta_b200.ep import ExpertParallel
import oracle
from tests._lib import bf16_from_dev, bf16_to_dev, to_dev
from workloads import normal_bf16_rows, random_problem
x, idx, w = random_problem(3, 200, 1024, 16, 4)
ep = ExpertParallel(1024, 4, 16, True, True, 200)
dst = ep.dispatch(bf16_to_dev(x), to_dev(idx))
o = oracle.dispatch(x, idx, E=16, R=1, fp8=True, pad128=True)
assert np.array_equal(dst.cpu().numpy(), o["slot"])
n = int(o["expert_offset"][16])
valid = o["recv_src"][:n] >= 0
got = ep.recv_x.view(torch.uint8).cpu().numpy()[:n]
assert np.array_equal(got[valid], o["recv_x"][:n][valid])
eo = normal_bf16_rows(4, 3, 0, ep.rows_cap, 1024)
ep.expert_out.copy_(bf16_to_dev(eo))
ep.experts_done()
y = ep.combine(to_dev(idx), dst, to_dev(w))
ref = oracle.combine(o["slot"], w, eo[:o["recv_x"].shape[0]])
yf = bf16_from_dev(y).astype(np.uint32) << 16
err = np.abs(yf.view(np.float32).astype(np.float64) - ref)
assert np.all(err <= 1e-2 + 4e-3 * np.abs(ref))
ep.check()
# the whole layer (layout, count exchange, payload, waits, signals, combine)
# captured in a CUDA graph and replayed: the same result, epochs advancing
xd, idd, wd = bf16_to_dev(x), to_dev(idx), to_dev(w)
s = torch.cuda.Stream()
s.wait_stream(torch.cuda.current_stream())
with torch.cuda.stream(s):
    for _ in range(2):   # warm-up outside capture
        dd = ep.dispatch(xd, idd); ep.experts_done(); yy = ep.combine(idd, dd, wd)
torch.cuda.current_stream().wait_stream(s)
torch.cuda.synchronize()
e0 = ep.epochs.cpu().tolist()
g = torch.cuda.CUDAGraph()
with torch.cuda.graph(g):
    dg = ep.dispatch(xd, idd)
    ep.experts_done()
    yg = ep.combine(idd, dg, wd)
for _ in range(3):
    g.replay()
torch.cuda.synchronize()
assert ep.epochs.cpu().tolist() == [e0[0] + 3, e0[1] + 3]     # capture records, replays run
assert np.array_equal(bf16_from_dev(yg), bf16_from_dev(y))
ep.check()
del g
# a batch above T_max is refused on the host; a bad id is reported by check()
try:
    ep.dispatch(bf16_to_dev(np.zeros((201, 1024), np.uint16)), to_dev(np.zeros((201, 4), np.int32)))
    raise AssertionError("T > T_max accepted")
except ValueError:
    pass
bad = idx.copy(); bad[0, 0] = 99
ep.dispatch(xd, to_dev(bad)); ep.experts_done(); ep.combine(to_dev(bad), dst, wd)
try:
    ep.check()
    raise AssertionError("bad id not reported")
except moe.MoeError:
    pass
del ep
dist.destroy_process_group()
print("ONE RANK OK")
"""


def test_expert_parallel_host_flow_on_a_one_rank_group():
    code = ONE_RANK.format(root=ROOT, port=_free_port())
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True,
                       timeout=300)
    assert "ONE RANK OK" in r.stdout, r.stdout[-2000:] + r.stderr[-4000:]


def test_bench_expert_parallel_mode_on_one_rank():
    # `bench.py --parallelism ep` as a one-rank group: the graph-replayed EP step
    # runs, checks the device error word and prints its JSON line
    import json
    r = subprocess.run([sys.executable, "bench.py", "--parallelism", "ep", "--workload", "dsv3_decode",
                        "--steps", "5", "--warmup", "3"], cwd=ROOT, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["config"]["parallelism"] == "ep x1" and line["value"] > 0 and line["steps"] == 5
