"""Tensor-parallel vocabulary sampling, host side (no GPU): shard bounds, and
the exchange protocol on two gloo ranks.

Each rank builds, from the oracle's perturbed scores of its vocabulary shard,
the documented packed key (order-preserving score bits << 32 | ~token, then
XOR 2^63 so that signed order is key order), the ranks reduce with an int64
MAX all-reduce, and the decoded token must equal the oracle's flat sample
(abstract: argmax decomposes over a partition)."""
import datetime
import os
import socket
import time

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from lm_head_exact_fmms_b200 import synth
from lm_head_exact_fmms_b200.tp import reduce_keys, shard_bounds


@pytest.mark.parametrize("V,world", [(1, 1), (7, 2), (8, 2), (151936, 8), (128256, 3), (4097, 5),
                                     (20, 8)])
def test_shard_bounds(V, world):
    b = shard_bounds(V, world)
    assert len(b) == world and b[0][0] == 0 and b[-1][1] == V
    for (lo, hi), (lo2, _) in zip(b, b[1:]):
        assert hi == lo2
    assert all(lo % 8 == 0 and lo <= hi for lo, hi in b)
    sizes = [hi - lo for lo, hi in b[:-1]]
    if sizes:
        assert max(sizes) - min(sizes) <= 8


def _order_bits(s):
    f = np.float32(s).view(np.uint32).astype(np.uint64)
    return np.where(f >> 31, (~f) & 0xFFFFFFFF, f | 0x80000000)


def encode(scores, offset):
    """Best key of a shard's scores (row-wise), signed encoding; -inf = masked."""
    B, n = scores.shape
    out = np.zeros(B, dtype=np.int64)
    for b in range(B):
        best = 0
        for j in range(n):
            if scores[b, j] == -np.inf:
                continue
            k = int(_order_bits(scores[b, j])) << 32 | (0xFFFFFFFF - (offset + j))
            best = max(best, k)
        out[b] = np.int64(np.uint64(best ^ (1 << 63)).view(np.int64))
    return out


def decode(keys):
    u = keys.view(np.uint64) ^ np.uint64(1 << 63)
    hi = u >> np.uint64(32)
    tok = (np.uint64(0xFFFFFFFF) - (u & np.uint64(0xFFFFFFFF))).astype(np.int64)
    return np.where(hi == 0, -1, tok)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank(rank, world, port, scores, results):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    V = scores.shape[1]
    lo, hi = shard_bounds(V, world)[rank]
    keys = torch.from_numpy(encode(scores[:, lo:hi], lo))
    reduce_keys(keys)
    results[rank] = decode(keys.numpy()).tolist()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_two_rank_exchange_matches_flat_oracle(oracle, world):
    B, d, V = 6, 32, 203
    H = synth.make_hidden(B, d, seed=5)
    W = synth.make_weight(V, d, 0.4, seed=6)
    allowed = torch.rand(B, V, generator=torch.Generator().manual_seed(2)) < 0.6
    allowed[1] = False                       # fully masked row -> -1
    allowed[2] = False
    allowed[2, V - 1] = True                 # only the last shard has a token
    mask = synth.mask_from_bool(allowed)
    scores = oracle.scores(H, W, T=0.9, seed=3, step=4, mask=mask)
    flat, _, _ = oracle.sample(H, W, T=0.9, seed=3, step=4, mask=mask)
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    results = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, scores, results)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    for r in range(world):
        assert results[r] == flat.tolist()
    assert flat[1] == -1 and flat[2] == V - 1


def _handles_rank(rank, world, port, results):
    import torch.distributed as dist
    from lm_head_exact_fmms_b200.tp import exchange_handles
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    mine = bytes([rank + 1]) * 64
    results[rank] = exchange_handles(mine)
    dist.destroy_process_group()


def test_exchange_handles_in_rank_order():
    """The fused exchange's only host collective: every rank receives every
    rank's 64-byte IPC handle, in rank order (gloo, three ranks)."""
    world = 3
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    results = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_handles_rank, args=(r, world, port, results))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    want = [bytes([r + 1]) * 64 for r in range(world)]
    for r in range(world):
        assert list(results[r]) == want


# ------------------------------------------------ failure detection on the host
def _monitor_rank(rank, world, port, plan, results):
    """Runs six calls' check-ins; `plan[rank]` = (what, at_call) makes this
    rank exit without a word, raise, or leave the group before that call."""
    import torch.distributed as dist
    from lm_head_exact_fmms_b200.tp import PeerLost, PeerMonitor
    store = dist.TCPStore("127.0.0.1", port, None, False, timeout=datetime.timedelta(seconds=30))
    mon = PeerMonitor(store, rank, world, timeout_s=3.0)
    what, at = plan.get(rank, ("ok", -1))
    log = []
    for seq in range(6):
        if seq == at:
            results[rank] = log
            if what == "exit":
                os._exit(0)
            if what == "raise":
                raise RuntimeError("planted failure on rank %d" % rank)
            if what == "leave":
                mon.leave()
                return
        t0 = time.monotonic()
        try:
            mon.check_in(seq)
        except PeerLost as e:
            log.append(("lost", e.seq, e.missing, e.left, time.monotonic() - t0))
            break
        log.append(("ok", seq))
    results[rank] = log


def _run_monitor(world, plan):
    import torch.distributed as dist
    server = dist.TCPStore("127.0.0.1", 0, None, True, timeout=datetime.timedelta(seconds=30),
                           wait_for_workers=False)
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    results = mgr.dict()
    procs = [ctx.Process(target=_monitor_rank, args=(r, world, server.port, plan, results))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    codes = [p.exitcode for p in procs]
    out = {r: list(results.get(r, [])) for r in range(world)}
    return server, codes, out


def test_peer_monitor_all_ranks_present():
    """Three ranks through six calls: every check-in passes, and each rank
    keeps only its latest call's key in the store."""
    server, codes, out = _run_monitor(3, {})
    assert codes == [0, 0, 0]
    for r in range(3):
        assert out[r] == [("ok", s) for s in range(6)]
    assert server.num_keys() <= 3 + 1   # one live key per rank (+ the store's own counter)


@pytest.mark.parametrize("what", ["exit", "raise"])
def test_peer_monitor_reports_a_rank_that_died(what):
    """A rank that exits without a word or raises before call 2: the others
    get PeerLost for call 2, naming it, after the 3 s limit and before
    launching anything."""
    _, codes, out = _run_monitor(3, {2: (what, 2)})
    assert codes[:2] == [0, 0] and codes[2] == (0 if what == "exit" else 1)
    for r in (0, 1):
        assert out[r][:2] == [("ok", 0), ("ok", 1)]
        kind, seq, missing, left, waited = out[r][2]
        assert (kind, seq, missing, left) == ("lost", 2, [2], [])
        assert 2.9 <= waited < 30


def test_peer_monitor_sees_a_leave_at_once():
    """A rank that leaves on purpose before call 3 is reported within a poll
    interval or so, not after the time limit."""
    _, codes, out = _run_monitor(2, {1: ("leave", 3)})
    assert codes == [0, 0]
    assert out[1] == [("ok", 0), ("ok", 1), ("ok", 2)]
    kind, seq, missing, left, waited = out[0][3]
    assert (kind, seq, missing, left) == ("lost", 3, [1], [1])
    assert waited < 2.0


def _collective_rank(rank, world, port, results):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=3))
    keys = torch.full((4,), rank, dtype=torch.int64)
    reduce_keys(keys)                                  # call 0: both ranks
    if rank == 1:
        time.sleep(8)                                  # alive, but skips call 1
        results[rank] = "skipped"
        return
    t0 = time.monotonic()
    try:
        reduce_keys(keys)
        results[rank] = "returned"
    except RuntimeError:
        results[rank] = ("error", time.monotonic() - t0)


def test_key_all_reduce_ends_with_an_error_when_a_peer_skips_it():
    """The all-reduce exchange: a rank that is alive but never joins call 1
    makes the other rank's collective end with an error after the process
    group's 3 s timeout, not hang."""
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    results = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_collective_rank, args=(r, 2, port, results)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert results[1] == "skipped"
    kind, waited = results[0]
    assert kind == "error" and waited < 30


class _FakeBinding:
    """Records the exchange's library calls (no GPU): areas are integers."""

    def __init__(self, rank, log):
        self.rank, self.log = rank, log

    def fs_tp_area_create(self):
        return 1000 + self.rank

    def fs_ipc_handle(self, area):
        return bytes([area - 1000 + 1]) * 64

    def fs_ipc_open(self, handle):
        return 2000 + handle[0] - 1

    def fs_ipc_close(self, area):
        self.log.append(("ipc_close", area))

    def fs_tp_area_destroy(self, area):
        self.log.append(("destroy", area))

    def fs_sample_tp(self, H, W, off, V, areas, seq, *args, **kw):
        self.log.append(("sample", seq, tuple(areas)))

    def fs_tp_wait(self, area, B, seq, out_idx=None, device=None, stream=None, timeout_us=None):
        self.log.append(("wait", seq, area, timeout_us))
        return out_idx


def _fused_host_rank(rank, world, port, store_port, results):
    import torch.distributed as dist
    from lm_head_exact_fmms_b200 import tp
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=20))
    log = []
    tp.binding = _FakeBinding(rank, log)
    torch.cuda.synchronize = lambda *a, **k: None     # no device here
    store = dist.TCPStore("127.0.0.1", store_port, None, False,
                          timeout=datetime.timedelta(seconds=30))
    kw = {} if rank == 1 else {"timeout_us": 123_456}   # rank 1 keeps the default limit
    ex = tp.FusedExchange(monitor=tp.PeerMonitor(store, rank, world, timeout_s=2.0), **kw)
    H = torch.zeros(4, 8)
    outcome = "done"
    for call in range(4):
        if rank == 1 and call == 2:
            results[rank] = (log, "exited")
            os._exit(0)                                  # dies between calls, without a word
        try:
            ex.sample(H, None, 0, 100, out_idx=torch.zeros(4, dtype=torch.int32))
        except tp.PeerLost as e:
            outcome = ("lost", e.seq, e.missing)
            break
    results[rank] = (log, outcome, ex.areas)


def test_fused_exchange_stops_before_launching_when_a_peer_died():
    """FusedExchange on two gloo ranks with the library calls recorded: the
    areas are the own one plus the peers' opened handles, in rank order; each
    call checks in, samples with the call number and waits with the given
    limit; when rank 1 dies before call 2, rank 0 gets PeerLost for call 2
    and has enqueued nothing for it."""
    import torch.distributed as dist
    server = dist.TCPStore("127.0.0.1", 0, None, True, timeout=datetime.timedelta(seconds=30),
                           wait_for_workers=False)
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    results = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_fused_host_rank, args=(r, 2, port, server.port, results))
             for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert [p.exitcode for p in procs] == [0, 0]
    log0, outcome0, areas0 = results[0]
    assert areas0 == [1000, 2001]                        # own area, then rank 1's opened handle
    assert outcome0 == ("lost", 2, [1])
    assert log0 == [("sample", 0, (1000, 2001)), ("wait", 0, 1000, 123_456),
                    ("sample", 1, (1000, 2001)), ("wait", 1, 1000, 123_456)]
    log1, outcome1 = results[1]
    assert outcome1 == "exited" and [e[1] for e in log1 if e[0] == "sample"] == [0, 1]
    from lm_head_exact_fmms_b200 import tp
    assert tp.DEFAULT_WAIT_US == 3_000_000
    assert [e[3] for e in log1 if e[0] == "wait"] == [tp.DEFAULT_WAIT_US] * 2
