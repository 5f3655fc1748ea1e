"""Transposed pair tiles against the CPU oracle.

On CTA pairs with a 256-row batch tile, a segment's partial tile (at most 240
vocabulary rows) is multiplied as logits^T: the pair's 256 batch rows are the
MMA's M operand and the tile's vocabulary rows, rounded up to n = 16 .. 240,
its N operand; an epilogue thread then owns one batch row.  The vocabularies
below give the pairs' partial tiles every width n from 16 to 240 (each row
of VOCAB_OF_WIDTH is a vocabulary whose split over 74 pairs yields that width), and the
flat, ragged, masked, grouped, multi-sample and vocabulary-shard paths
are all put through them, every row compared with the oracle under the
tolerance of test_gpu_parity (a token may differ only at a near tie of the
oracle's two best scores).
"""
import numpy as np
import pytest
import torch

from lm_head_exact_fmms_b200 import binding, synth
from tests.test_gpu_parity import TIE_REL, assert_parity, dev, rand_inputs  # noqa: F401

pytestmark = pytest.mark.gpu

# n -> a vocabulary whose partial tiles on 74 CTA pairs are n columns wide
VOCAB_OF_WIDTH = {16: 18952, 32: 2000, 48: 2370, 64: 3554, 80: 4738, 96: 5922, 112: 7106,
                  128: 8290, 144: 9474, 160: 10658, 176: 11842, 192: 13026, 208: 14210,
                  224: 15394, 240: 16578}


@pytest.fixture(scope="module")
def pairs_on_148(dev):
    """The widths above assume 74 pairs, i.e. 148 SMs."""
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    if sms != 148:
        pytest.skip("the vocabulary table assumes 148 SMs, this device has %d" % sms)
    assert binding.fs_uses_cta_pairs(256)
    return dev


@pytest.mark.parametrize("n", sorted(VOCAB_OF_WIDTH))
def test_flat_every_width(pairs_on_148, oracle, n):
    V = VOCAB_OF_WIDTH[n]
    d = 96 if n % 32 == 0 else 128  # 96: the last K block half filled
    B = 256
    H, W, Hd, Wd = rand_inputs(B, d, V, seed=n)
    got = binding.fs_sample_ex(Hd, Wd, temperature=0.8, seed=5, step=n).cpu().numpy()
    idx, best, second = oracle.sample(H, W, T=0.8, seed=5, step=n)
    mism = assert_parity(got, idx, best, second, "n=%d V=%d" % (n, V))
    assert mism <= 1


@pytest.mark.parametrize("B,V", [(250, 12345), (241, 16578), (256, 30011)])
def test_flat_ragged_masked_row_seeds(pairs_on_148, oracle, B, V):
    """Batches of 241-256 rows run on the 256-row pair tile; the rows past B
    hold nothing, masked tokens are never drawn, fully masked rows give -1."""
    d = 192
    H, W, Hd, Wd = rand_inputs(B, d, V, seed=B)
    rs = synth.make_row_seeds(B)
    mask = synth.make_mask(B, V, 0.4, seed=B)
    mask[3] = 0  # a row with no allowed token
    for step in range(2):
        got = binding.fs_sample_ex(Hd, Wd, temperature=1.1, seed=9, row_seeds=rs.to(pairs_on_148),
                                   step=step, mask_bits=mask.to(pairs_on_148)).cpu().numpy()
        idx, best, second = oracle.sample(H, W, T=1.1, seed=9, row_seeds=rs, step=step, mask=mask)
        assert got[3] == -1 and idx[3] == -1
        assert assert_parity(got, idx, best, second, "B=%d V=%d step %d" % (B, V, step)) <= 1


@pytest.mark.parametrize("V,G", [(12345, 7), (5000, 3), (16578, 5), (30011, 8)])
def test_grouped_masked(pairs_on_148, oracle, V, G):
    """Group boundaries cut the pairs' ranges into segments whose partial
    tiles have many widths; each segment's (key, max, sum) over its
    transposed tile joins the running state of the chunks that follow."""
    B, d = 256, 128
    H, W, Hd, Wd = rand_inputs(B, d, V, seed=V + G)
    mask = synth.make_mask(B, V, 0.5, seed=G)
    got = binding.fs_sample_grouped(Hd, Wd, G, temperature=0.9, seed=2, step=1,
                                    mask_bits=mask.to(pairs_on_148)).cpu().numpy()
    idx, summ, margin = oracle.sample_grouped(H, W, G, T=0.9, seed=2, step=1, mask=mask)
    bad = got != idx
    for b in np.flatnonzero(bad):
        scale = TIE_REL * (1 + abs(summ[b, :, 0].max()))
        assert margin[b, 0] <= scale or margin[b, 1] <= scale, (V, G, b, got[b], idx[b])
    assert int(bad.sum()) <= 1


def test_multi_sample(pairs_on_148, oracle):
    B, d, V, S = 256, 128, 9474, 3
    H, W, Hd, Wd = rand_inputs(B, d, V, seed=31)
    rs = synth.make_row_seeds(B)
    got = binding.fs_sample_multi(Hd, Wd, S, temperature=0.7, seed=1, row_seeds=rs.to(pairs_on_148),
                                  step=4).cpu().numpy()
    idx, best, second = oracle.sample_multi(H, W, S, T=0.7, seed=1, row_seeds=rs, step=4)
    assert assert_parity(got.ravel(), idx.ravel(), best.ravel(), second.ravel(), "multi") <= 1


def test_vocab_shards(pairs_on_148, oracle):
    """Shards at vocabulary offsets (multiples of 8): the noise, the mask and
    the packed tokens of a transposed tile use global token indices."""
    from lm_head_exact_fmms_b200.tp import shard_bounds
    B, d, V, world = 256, 128, 30011, 3
    H, W, Hd, Wd = rand_inputs(B, d, V, seed=77)
    mask = synth.make_mask(B, V, 0.6, seed=77)
    keys = [binding.fs_sample_shard_keys(Hd, Wd[lo:hi].contiguous(), lo, V, temperature=0.9,
                                         seed=4, step=3, mask_bits=mask.to(pairs_on_148))
            for lo, hi in shard_bounds(V, world)]
    got = binding.fs_keys_to_tokens(torch.stack(keys).max(dim=0).values.contiguous()).cpu().numpy()
    idx, best, second = oracle.sample(H, W, T=0.9, seed=4, step=3, mask=mask)
    assert assert_parity(got, idx, best, second, "shards") <= 1


@pytest.mark.parametrize("V", [18952, 16578, 5000])
def test_pairs_match_single_ctas(pairs_on_148, V):
    """The same flat calls on single CTAs, where every tile runs the usual
    way: the tokens are the same bit for bit (the contract of
    fs_set_cta_pairs), masked, over several steps.  (Grouped tokens may
    differ at near ties of the group log-sum-exps, which the two kernels
    merge in different orders; test_gpu_pairs covers that relation.)"""
    B, d = 256, 256
    _, _, Hd, Wd = rand_inputs(B, d, V, seed=5)
    mask = synth.make_mask(B, V, 0.5, seed=V).to(pairs_on_148)

    def calls():
        out = []
        for step in range(3):
            out.append(binding.fs_sample_ex(Hd, Wd, temperature=1.0, seed=3, step=step,
                                            mask_bits=mask).cpu())
        return out

    a = calls()
    binding.fs_set_cta_pairs(0)
    try:
        b = calls()
    finally:
        binding.fs_set_cta_pairs(-1)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
