"""Tensor-parallel vocabulary sampling, host side (no GPU): shard bounds, and
the exchange protocol on two gloo ranks.

Each rank builds, from the oracle's perturbed scores of its vocabulary shard,
the documented packed key (order-preserving score bits << 32 | ~token, then
XOR 2^63 so that signed order is key order), the ranks reduce with an int64
MAX all-reduce, and the decoded token must equal the oracle's flat sample
(abstract: argmax decomposes over a partition)."""
import os
import socket

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
