"""Tensor-parallel vocabulary sampling across GPUs.

The LM head's vocabulary rows are split over the ranks of a process group;
each rank samples its shard with global token indices (so noise, mask and
tie-breaking are those of the full head), producing one packed
(score, token) key per row, and a single int64 MAX all-reduce of 8 bytes per
row picks the winner (readus.org page, "distributed FlashSampling": each GPU
is one group and sends only its winning index and score; abstract: argmax
decomposes over a partition).  The tokens equal single-GPU sampling bit for
bit.  torch.distributed (NCCL) carries the exchange; the sampling itself runs
in the library's kernels.
"""
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
