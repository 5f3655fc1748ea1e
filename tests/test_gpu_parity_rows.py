"""Every row of the LM-head workloads at full size against the CPU oracle, in
the launch configuration the benchmark times (CTA pairs from 97 rows,
several 256-row launches for B=512, flat steps issued back to back): 2,048 rows in all,
over several steps.
Same tolerance as test_gpu_parity: a token may differ from the oracle's only
at a near tie of the oracle's two best perturbed scores; at most one such row
is allowed here (the expected count is about 0.02).  (Runs for about a
minute and a half, mostly oracle time.)"""
import numpy as np
import pytest
import torch

from lm_head_exact_fmms_b200 import binding, synth
from tests.test_gpu_parity import TIE_REL, assert_parity, dev  # noqa: F401  (fixture)

pytestmark = pytest.mark.gpu

# (workload, B, steps): the flat heads at their largest batch of one launch
# and at the headline B = 64, and the grouped + masked head at B = 512 (two
# launches).
CASES = [("qwen3-8b", 256, 3), ("qwen3-8b", 64, 2), ("qwen3-1.7b", 64, 4), ("large", 64, 2),
         ("large", 256, 1), ("grouped-masked", 512, 1)]


def test_every_row_of_full_size_workloads(dev, oracle):
    total = mism = 0
    for name, B, steps in CASES:
        wl = synth.WORKLOADS[name]
        Wd = synth.make_weight(wl.V, wl.d, wl.w_std, device=dev)
        W = Wd.cpu()
        Hd = synth.make_hidden(B, wl.d, device=dev)
        H = Hd.cpu()
        rs = synth.make_row_seeds(B) if wl.per_row_seeds else None
        mask = synth.make_mask(B, wl.V, wl.mask_allowed) if wl.mask_allowed else None
        for step in range(steps):
            kw = dict(temperature=wl.temperature, seed=11, step=step,
                      row_seeds=rs.to(dev) if rs is not None else None,
                      mask_bits=mask.to(dev) if mask is not None else None)
            if wl.groups:
                got = binding.fs_sample_grouped(Hd, Wd, wl.groups, **kw).cpu().numpy()
                idx, summ, margin = oracle.sample_grouped(H, W, wl.groups, T=wl.temperature,
                                                          seed=11, row_seeds=rs, step=step,
                                                          mask=mask)
                bad = got != idx
                for b in np.flatnonzero(bad):
                    scale = TIE_REL * (1 + abs(summ[b, :, 0].max()))
                    assert margin[b, 0] <= scale or margin[b, 1] <= scale, (name, step, b)
                mism += int(bad.sum())
            else:
                # The steps go out back to back with no synchronisation (each
                # launch of up to 128 rows a programmatic dependent of the one
                # before, as in the benchmark) and are checked afterwards.
                if step == 0:
                    outs = [binding.fs_sample_ex(Hd, Wd, **dict(kw, step=s))
                            for s in range(steps)]
                    torch.cuda.synchronize()
                got = outs[step].cpu().numpy()
                idx, best, second = oracle.sample(H, W, T=wl.temperature, seed=11,
                                                  row_seeds=rs, step=step, mask=mask)
                mism += assert_parity(got, idx, best, second, "%s B=%d step %d" % (name, B, step))
            total += B
        del Wd, Hd
        torch.cuda.empty_cache()
    assert total == sum(B * steps for _, B, steps in CASES) == 2048
    assert mism <= 1, (mism, total)
