"""Tensor-parallel vocabulary sampling across GPUs.

The LM head's vocabulary rows are split over the ranks of a process group;
each rank samples its shard with global token indices (so noise, mask and
tie-breaking are those of the full head), producing one packed
(score, token) key per row, and the maximum over ranks picks the winner
(readus.org page, "distributed FlashSampling": each GPU is one group and
sends only its winning index and score; abstract: argmax decomposes over a
partition).  The tokens equal single-GPU sampling bit for bit.

Two ways to exchange the keys:
  * FusedExchange: the kernel's last CTA writes the keys straight into every
    rank's exchange area over NVLink and the rank completing an area decodes
    it (fs_sample_tp); the stream then waits on the area's flag.  Only the
    IPC handles of the areas go through torch.distributed, once.
  * tp_sample: an int64 MAX all-reduce of 8 bytes per row through
    torch.distributed (NCCL) after the kernel, then a decode kernel.
"""
import time

import torch
import torch.distributed as dist

from . import binding

GRANULE = 8   # shard boundaries are multiples of 8 tokens (the kernel's noise layout)


def shard_bounds(V, world, granule=GRANULE):
    """[(lo, hi)] for each rank: contiguous, balanced to within one granule,
    every lo a multiple of `granule`."""
    if V < 1 or world < 1:
        raise ValueError("V and world must be positive")
    ngran = (V + granule - 1) // granule
    cuts = [min(V, granule * ((r * ngran) // world)) for r in range(world + 1)]
    cuts[-1] = V
    return [(cuts[r], cuts[r + 1]) for r in range(world)]


def reduce_keys(keys, group=None):
    """In-place int64 MAX all-reduce of per-row keys across the group."""
    dist.all_reduce(keys, op=dist.ReduceOp.MAX, group=group)
    return keys


def tp_sample(H, W_shard, vocab_offset, V_total, temperature=1.0, seed=0, row_seeds=None, step=0,
              mask_bits=None, group=None, workspace=None, stream=None):
    """Samples B rows of a vocabulary-sharded head; every rank gets all tokens."""
    keys = binding.fs_sample_shard_keys(H, W_shard, vocab_offset, V_total, temperature, seed,
                                        row_seeds, step, mask_bits, workspace=workspace,
                                        stream=stream)
    reduce_keys(keys, group)
    return binding.fs_keys_to_tokens(keys, stream=stream)


def exchange_handles(handle, group=None):
    """All ranks' IPC handles (bytes), in rank order, via an all-gather."""
    world = dist.get_world_size(group)
    out = [None] * world
    dist.all_gather_object(out, bytes(handle), group=group)
    return out


class PeerLost(RuntimeError):
    """A rank of the group did not reach a call in time, or left the group."""

    def __init__(self, seq, missing, left):
        self.seq, self.missing, self.left = seq, sorted(missing), sorted(left)
        super().__init__("call %d: rank(s) %s did not check in%s" % (
            seq, self.missing, (" (left the group: %s)" % self.left) if self.left else ""))


class PeerMonitor:
    """Host-side liveness of the ranks of a group, checked before each launch
    whose completion depends on the peers (the fused exchange's kernel and
    stream wait): every rank posts the number of the call it is about to
    launch in a key-value store (a torch.distributed Store) and waits, for at
    most `timeout_s`, until every other rank has posted it.  A rank that
    raised, exited or never arrived is reported here, as PeerLost, before
    this rank enqueues anything that would wait for it; a rank that leaves on
    purpose calls leave(), which the others see within one poll interval.
    Each rank keeps one key per call alive at a time."""

    def __init__(self, store, rank, world, timeout_s=10.0, poll_s=0.05, prefix="fmms/peers"):
        self.store, self.rank, self.world = store, rank, world
        self.timeout_s, self.poll_s, self.prefix = timeout_s, poll_s, prefix
        self._posted = None

    def _key(self, seq, r):
        return "%s/%d/%d" % (self.prefix, seq, r)

    def _left_key(self, r):
        return "%s/left/%d" % (self.prefix, r)

    def check_in(self, seq):
        """Posts call `seq` and returns once every rank has posted it;
        raises PeerLost otherwise."""
        self.store.set(self._key(seq, self.rank), b"1")
        others = [r for r in range(self.world) if r != self.rank]
        deadline = time.monotonic() + self.timeout_s
        pending = list(others)
        while True:
            pending = [r for r in pending if not self.store.check([self._key(seq, r)])]
            if not pending:
                break
            left = [r for r in pending if self.store.check([self._left_key(r)])]
            if left or time.monotonic() >= deadline:
                raise PeerLost(seq, pending, left)
            time.sleep(self.poll_s)
        # Every rank has posted `seq`, so none still waits for call seq-1.
        if self._posted is not None:
            self.store.delete_key(self._key(self._posted, self.rank))
        self._posted = seq

    def leave(self):
        """Tells the other ranks that this one takes no further calls."""
        self.store.set(self._left_key(self.rank), b"1")


# Default limit of each fused call's wait for its tokens.  The sampling
# kernel's own bounded waits give up after 2e9 SM cycles (about 1.0 s at the
# top clock, 1.7 s at the 1.2 GHz a power-capped board can fall to), and a
# call whose kernel gave up still completes the exchange, marked as failed;
# 3 s keeps that report ahead of the wait's own limit while a peer that died
# with its kernel in flight stalls this rank's stream for seconds, not tens
# of seconds.
DEFAULT_WAIT_US = 3_000_000


class FusedExchange:
    """The exchange areas of a process group for fs_sample_tp: this rank's
    own area and its peers', mapped here by CUDA IPC.  Every rank calls
    sample() in the same order (the call sequence number is kept here).
    timeout_us: the limit of each call's wait for its tokens (after it, the
    tokens read -1 and fs_tp_failed names the call)."""

    def __init__(self, group=None, monitor=None, timeout_us=DEFAULT_WAIT_US):
        self.group = group
        self.monitor = monitor    # an optional PeerMonitor, checked before every call
        self.timeout_us = timeout_us  # limit of each call's wait for its tokens
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        self.mine = binding.fs_tp_area_create()
        handles = exchange_handles(binding.fs_ipc_handle(self.mine), group)
        self._opened = []
        self.areas = []
        for r, h in enumerate(handles):
            if r == self.rank:
                self.areas.append(self.mine)
            else:
                a = binding.fs_ipc_open(h)
                self._opened.append(a)
                self.areas.append(a)
        self.seq = 0

    def sample(self, H, W_shard, vocab_offset, V_total, temperature=1.0, seed=0, row_seeds=None,
               step=0, mask_bits=None, out_idx=None, workspace=None, stream=None):
        """Samples B <= 256 rows of the sharded head; every rank gets all tokens.
        With a monitor, raises PeerLost (having enqueued nothing) when a peer
        did not reach this call."""
        if self.monitor is not None:
            self.monitor.check_in(self.seq)
        binding.fs_sample_tp(H, W_shard, vocab_offset, V_total, self.areas, self.seq, temperature,
                             seed, row_seeds, step, mask_bits, workspace=workspace, stream=stream)
        out = binding.fs_tp_wait(self.mine, H.shape[0], self.seq, out_idx, device=H.device,
                                 stream=stream, timeout_us=self.timeout_us)
        self.seq += 1
        return out

    def close(self):
        """Unmaps the peers' areas and frees this rank's, once every rank is
        done with the exchange.  With a monitor, first tells the peers that
        this rank takes no further calls."""
        if self.monitor is not None:
            self.monitor.leave()
        torch.cuda.synchronize()
        dist.barrier(group=self.group)
        for a in self._opened:
            binding.fs_ipc_close(a)
        self._opened = []
        dist.barrier(group=self.group)
        binding.fs_tp_area_destroy(self.mine)
        self.mine = None


class LocalExchange:
    """`world` shards on one GPU, each with its own exchange area in this
    process: the same kernels and protocol as FusedExchange, with the ranks'
    calls issued one after another on one stream (no call waits for a later
    one, so nothing waits for a kernel that has not run)."""

    def __init__(self, world):
        self.world = world
        self.areas = [binding.fs_tp_area_create() for _ in range(world)]
        self.seq = 0

    def sample(self, H, shards, V_total, temperature=1.0, seed=0, row_seeds=None, step=0,
               mask_bits=None, workspaces=None, stream=None):
        """shards: [(W_shard, vocab_offset)] per rank.  Returns each rank's tokens."""
        for r, (Ws, off) in enumerate(shards):
            ws = workspaces[r] if workspaces is not None else None
            binding.fs_sample_tp(H, Ws, off, V_total, self.areas, self.seq, temperature, seed,
                                 row_seeds, step, mask_bits, workspace=ws, stream=stream)
        outs = [binding.fs_tp_wait(a, H.shape[0], self.seq, device=H.device, stream=stream)
                for a in self.areas]
        self.seq += 1
        return outs

    def close(self):
        torch.cuda.synchronize()
        for a in self.areas:
            binding.fs_tp_area_destroy(a)
        self.areas = []
