"""Small and ragged shapes run through the debug build of the library.

Run by tests/test_gpu_debug_build.py in a child process with
FMMS_LIBRARY=debug, so that the binding loads libfmms_debug.so, whose kernels
check their global, shared and tensor-memory indices and record
FS_ERR_DEVICE_BOUNDS in the status word instead of trapping.  For every shape
(B in {1, 3, 17}, V in {1, 7, 129, 4097}, d in {8, 24}) and every kind of call
(flat with mask and row seeds, on single CTAs and CTA pairs; grouped; several
samples; unfused; top-k; vocabulary shards), and for 250 and 256 rows (CTA
pairs whose partial tiles run transposed; V up to 18952) with the flat,
grouped, multi-sample and shard calls, the status word must read FS_OK
and the tokens must match the oracle under the stated tie rule.  Prints one
line per shape and exits non-zero on the first failure.
"""
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from lm_head_exact_fmms_b200 import binding, synth  # noqa: E402
from lm_head_exact_fmms_b200.tp import shard_bounds  # noqa: E402

TIE_REL = 2e-3


def parity(got, idx, best, second, what):
    got = np.asarray(got).ravel()
    idx, best, second = np.ravel(idx), np.ravel(best), np.ravel(second)
    bad = got != idx
    tie = (best - second) <= TIE_REL * (1.0 + np.abs(best))
    assert not np.any(bad & ~tie), "%s: gpu %s oracle %s" % (what, got[bad & ~tie][:8],
                                                            idx[bad & ~tie][:8])


def status_ok(what):
    torch.cuda.synchronize()
    st = binding.fs_device_status(None)
    assert st == 0, "%s: device status %s" % (what, binding.fs_status_string(st))


def main():
    assert binding.library_path().endswith("libfmms_debug.so"), binding.library_path()
    binding.load_library()
    dev = torch.device("cuda:0")
    n = 0
    for d in (8, 24):
        for V in (1, 7, 129, 4097):
            for B in (1, 3, 17):
                seed = 1000 * d + 10 * V + B
                H = synth.make_hidden(B, d, seed=seed)
                W = synth.make_weight(V, d, 0.5, seed=seed + 1)
                Hd, Wd = H.to(dev), W.to(dev)
                rs = synth.make_row_seeds(B)
                mask = synth.make_mask(B, V, 0.5, seed=seed + 2)
                rsd, md = rs.to(dev), mask.to(dev)
                what = "B=%d d=%d V=%d" % (B, d, V)
                ref = oracle.sample(H, W, T=0.9, seed=3, row_seeds=rs, step=1, mask=mask)
                for policy in (0, 1):
                    binding.fs_set_cta_pairs(policy)
                    try:
                        got = binding.fs_sample_ex(Hd, Wd, temperature=0.9, seed=3, row_seeds=rsd,
                                                   step=1, mask_bits=md)
                        status_ok(what + " flat pairs=%d" % policy)
                        parity(got.cpu().numpy(), *ref, what + " flat pairs=%d" % policy)
                        G = min(3, V)
                        g = binding.fs_sample_grouped(Hd, Wd, G, temperature=0.9, seed=3,
                                                      row_seeds=rsd, step=1, mask_bits=md)
                        status_ok(what + " grouped pairs=%d" % policy)
                        gi, gs, gm = oracle.sample_grouped(H, W, G, T=0.9, seed=3, row_seeds=rs,
                                                           step=1, mask=mask)
                        gg = g.cpu().numpy()
                        for b in np.flatnonzero(gg != gi):
                            scale = TIE_REL * (1 + abs(gs[b, :, 0].max()))
                            assert gm[b, 0] <= scale or gm[b, 1] <= scale, (what, "grouped", b)
                    finally:
                        binding.fs_set_cta_pairs(-1)
                got = binding.fs_sample_multi(Hd, Wd, 2, temperature=0.9, seed=3, row_seeds=rsd,
                                              step=1, mask_bits=md)
                status_ok(what + " multi")
                parity(got.cpu().numpy(), *oracle.sample_multi(H, W, 2, T=0.9, seed=3,
                                                               row_seeds=rs, step=1, mask=mask),
                       what + " multi")
                got = binding.fs_sample_unfused(Hd, Wd, temperature=0.9, seed=3, row_seeds=rsd,
                                                step=1, mask_bits=md)
                status_ok(what + " unfused")
                parity(got.cpu().numpy(), *ref, what + " unfused")
                K = min(5, V)
                got = binding.fs_sample_topk(Hd, Wd, K, temperature=0.9, seed=3, row_seeds=rsd,
                                             step=1, mask_bits=md)
                status_ok(what + " top-k")
                parity(got.cpu().numpy(), *oracle.sample_topk(H, W, K, T=0.9, seed=3,
                                                              row_seeds=rs, step=1, mask=mask),
                       what + " top-k")
                keys = [binding.fs_sample_shard_keys(Hd, Wd[lo:hi].contiguous(), lo, V,
                                                     temperature=0.9, seed=3, row_seeds=rsd,
                                                     step=1, mask_bits=md)
                        for lo, hi in shard_bounds(V, 2) if hi > lo]
                got = binding.fs_keys_to_tokens(torch.stack(keys).max(dim=0).values.contiguous())
                status_ok(what + " shards")
                parity(got.cpu().numpy(), *ref, what + " shards")
                n += 1
                print("ok", what, flush=True)
    # 241-256 rows: CTA pairs with a 256-row batch tile, whose partial tiles
    # run transposed (every unit's range is a single partial tile for the
    # small vocabularies, an 8-row one beside whole tiles for V = 18952).
    for V in (1, 7, 129, 4097, 18952):
        for B in (250, 256):
            d = 24
            seed = 7000 + 10 * V + B
            H = synth.make_hidden(B, d, seed=seed)
            W = synth.make_weight(V, d, 0.5, seed=seed + 1)
            Hd, Wd = H.to(dev), W.to(dev)
            rs = synth.make_row_seeds(B)
            mask = synth.make_mask(B, V, 0.5, seed=seed + 2)
            rsd, md = rs.to(dev), mask.to(dev)
            what = "B=%d d=%d V=%d" % (B, d, V)
            assert binding.fs_uses_cta_pairs(B), what
            ref = oracle.sample(H, W, T=0.9, seed=3, row_seeds=rs, step=1, mask=mask)
            got = binding.fs_sample_ex(Hd, Wd, temperature=0.9, seed=3, row_seeds=rsd, step=1,
                                       mask_bits=md)
            status_ok(what + " flat")
            parity(got.cpu().numpy(), *ref, what + " flat")
            G = min(3, V)
            g = binding.fs_sample_grouped(Hd, Wd, G, temperature=0.9, seed=3, row_seeds=rsd,
                                          step=1, mask_bits=md)
            status_ok(what + " grouped")
            gi, gs, gm = oracle.sample_grouped(H, W, G, T=0.9, seed=3, row_seeds=rs, step=1,
                                               mask=mask)
            gg = g.cpu().numpy()
            for b in np.flatnonzero(gg != gi):
                scale = TIE_REL * (1 + abs(gs[b, :, 0].max()))
                assert gm[b, 0] <= scale or gm[b, 1] <= scale, (what, "grouped", b)
            got = binding.fs_sample_multi(Hd, Wd, 2, temperature=0.9, seed=3, row_seeds=rsd,
                                          step=1, mask_bits=md)
            status_ok(what + " multi")
            parity(got.cpu().numpy(), *oracle.sample_multi(H, W, 2, T=0.9, seed=3, row_seeds=rs,
                                                           step=1, mask=mask), what + " multi")
            keys = [binding.fs_sample_shard_keys(Hd, Wd[lo:hi].contiguous(), lo, V,
                                                 temperature=0.9, seed=3, row_seeds=rsd, step=1,
                                                 mask_bits=md)
                    for lo, hi in shard_bounds(V, 2) if hi > lo]
            got = binding.fs_keys_to_tokens(torch.stack(keys).max(dim=0).values.contiguous())
            status_ok(what + " shards")
            parity(got.cpu().numpy(), *ref, what + " shards")
            n += 1
            print("ok", what, flush=True)
    print("debug build: %d shapes, every call FS_OK and oracle parity" % n, flush=True)


if __name__ == "__main__":
    main()
