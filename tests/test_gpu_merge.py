"""Merged 8-row partial tiles (fs_set_partial_merge): a CTA whose range starts
with an 8-row partial tile multiplies it in the stages of its first whole
tile instead of as a tile of its own.  Every mode that runs single CTAs of
up to 64 batch rows must give the same result either way, bit for bit, and
the merged variant must follow the oracle."""
import numpy as np
import pytest
import torch

from lm_head_exact_fmms_b200 import binding, synth
from tests.test_gpu_parity import assert_parity, dev, rand_inputs  # noqa: F401  (fixture)

pytestmark = pytest.mark.gpu

# 148 CTAs x 136 rows: every CTA has one whole tile and an 8-row partial tile;
# 148 x 264 + 5: two whole tiles and an 8-row partial, the last CTA ragged.
SHAPES = [(1, 64, 148 * 136), (16, 128, 148 * 264 + 5), (33, 96, 148 * 136), (64, 64, 148 * 264 + 5)]


def both(fn):
    out = []
    for policy in (0, 1):
        binding.fs_set_partial_merge(policy)
        try:
            out.append(fn())
        finally:
            binding.fs_set_partial_merge(-1)
    return out


@pytest.mark.parametrize("B,d,V", SHAPES)
def test_flat_merged_equals_unmerged_and_oracle(dev, oracle, B, d, V):
    H, W, Hd, Wd = rand_inputs(B, d, V, seed=B + V)
    rs = synth.make_row_seeds(B)
    mask = synth.make_mask(B, V, 0.6, seed=B)
    kw = dict(temperature=0.8, seed=3, row_seeds=rs.to(dev), step=2, mask_bits=mask.to(dev))
    t0, t1 = both(lambda: binding.fs_sample_ex(Hd, Wd, **kw).cpu())
    assert torch.equal(t0, t1)
    idx, best, second = oracle.sample(H, W, T=0.8, seed=3, row_seeds=rs, step=2, mask=mask)
    assert_parity(t1.numpy(), idx, best, second, "merged flat")


@pytest.mark.parametrize("B,d,V", SHAPES[:2])
def test_logits_and_multi_sample_merged_equal_unmerged(dev, B, d, V):
    _, _, Hd, Wd = rand_inputs(B, d, V, seed=7 * B + 1)

    def logits():
        lg = torch.empty(B, V, dtype=torch.float32, device=dev)
        binding.fs_sample_unfused(Hd, Wd, temperature=1.0, logits=lg)
        return lg.cpu()
    l0, l1 = both(logits)
    assert torch.equal(l0.view(torch.int32), l1.view(torch.int32))
    m0, m1 = both(lambda: binding.fs_sample_multi(Hd, Wd, 4, temperature=0.9, seed=5, step=1).cpu())
    assert torch.equal(m0, m1)


@pytest.mark.parametrize("B,d,V,G", [(20, 64, 148 * 136, 3), (64, 128, 148 * 264 + 5, 8)])
def test_grouped_merged_equals_unmerged(dev, B, d, V, G):
    _, _, Hd, Wd = rand_inputs(B, d, V, seed=G + B)
    md = synth.make_mask(B, V, 0.5, seed=G).to(dev)

    def call():
        summ = torch.empty(B, G, 3, dtype=torch.float32, device=dev)
        tok = binding.fs_sample_grouped(Hd, Wd, G, temperature=0.8, seed=12, step=2,
                                        mask_bits=md, out_summary=summ)
        return tok.cpu(), summ.cpu()
    (t0, s0), (t1, s1) = both(call)
    assert torch.equal(s0[:, :, :2].contiguous().view(torch.int32),
                       s1[:, :, :2].contiguous().view(torch.int32))
    l0, l1 = s0[:, :, 2].numpy(), s1[:, :, 2].numpy()
    fin = np.isfinite(l0)
    assert np.array_equal(fin, np.isfinite(l1))
    assert np.allclose(l0[fin], l1[fin], rtol=1e-5, atol=1e-5)
    assert torch.equal(t0, t1)


def test_full_size_head_automatic_choice(dev):
    """The Qwen3-8B head: the automatic policy merges (48 of 148 CTAs have an
    8-row partial tile) and gives the unmerged tokens at B = 1 and 64."""
    wl = synth.WORKLOADS["qwen3-8b"]
    Wd = synth.make_weight(wl.V, wl.d, wl.w_std, device=dev)
    try:
        for B in (1, 64):
            Hd = synth.make_hidden(B, wl.d, device=dev)
            rs = synth.make_row_seeds(B).to(dev)
            auto = binding.fs_sample_ex(Hd, Wd, temperature=wl.temperature, row_seeds=rs,
                                        step=3).cpu()
            t0, t1 = both(lambda: binding.fs_sample_ex(Hd, Wd, temperature=wl.temperature,
                                                       row_seeds=rs, step=3).cpu())
            assert torch.equal(auto, t1) and torch.equal(t0, t1)
    finally:
        del Wd
        torch.cuda.empty_cache()


def test_policy_argument_checked(dev):
    with pytest.raises(binding.FmmsError):
        binding.fs_set_partial_merge(2)
    binding.fs_set_partial_merge(-1)
