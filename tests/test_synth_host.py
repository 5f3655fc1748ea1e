"""The seeded input recipe (CPU): what the generators draw is what the
recipe states -- shapes, bf16 values of the stated normal scales, the mask's
bit layout and allowed fraction, the row seeds -- and the same seed gives the
same bytes."""
import numpy as np
import pytest
import torch

from lm_head_exact_fmms_b200 import synth


def test_same_seed_same_bytes_and_seeds_differ():
    a = synth.make_weight(1000, 64, 0.02, seed=9)
    b = synth.make_weight(1000, 64, 0.02, seed=9)
    c = synth.make_weight(1000, 64, 0.02, seed=10)
    assert a.dtype == torch.bfloat16 and a.shape == (1000, 64)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert not torch.equal(a, c)
    h = synth.make_hidden(8, 64)
    assert torch.equal(h, synth.make_hidden(8, 64, seed=synth.H_SEED_BASE + 8))


def test_weight_chunking_is_part_of_the_recipe():
    """Rows drawn in 16384-row chunks from one generator: the first chunk of a
    larger head equals a head of exactly that many rows."""
    big = synth.make_weight(20000, 16, 0.5, chunk_rows=16384)
    small = synth.make_weight(16384, 16, 0.5)
    assert torch.equal(big[:16384], small)


@pytest.mark.parametrize("std", [0.02, 0.015, 1.0 / 16.0])
def test_weight_scale_and_bf16_values(std):
    W = synth.make_weight(20000, 64, std).float().numpy()
    assert abs(W.mean()) < 5 * std / np.sqrt(W.size)
    assert abs(W.std() / std - 1.0) < 0.01
    # every value is a bf16 number: the low 16 bits of its fp32 pattern are 0
    assert np.all((W.view(np.uint32) & 0xFFFF) == 0)


def test_hidden_states_are_standard_normal():
    H = synth.make_hidden(64, 4096).float().numpy()
    assert abs(H.mean()) < 5 / np.sqrt(H.size)
    assert abs(H.std() - 1.0) < 0.01


def test_mask_layout_and_fraction():
    """Bit (v & 31) of word [b, v >> 5]; about the stated fraction allowed;
    bits past V are 0; mask_from_bool packs the same layout."""
    B, V = 5, 1000
    m = synth.make_mask(B, V, 0.5)
    assert m.dtype == torch.int32 and m.shape == (B, (V + 31) // 32)
    words = m.numpy().view(np.uint32)
    bits = np.array([[(words[b, v >> 5] >> (v & 31)) & 1 for v in range(32 * words.shape[1])]
                     for b in range(B)])
    assert np.all(bits[:, V:] == 0)
    assert abs(bits[:, :V].mean() - 0.5) < 0.03
    again = synth.mask_from_bool(torch.from_numpy(bits[:, :V].astype(bool)))
    assert torch.equal(again, m)


def test_row_seeds_and_workload_table():
    assert synth.make_row_seeds(4).tolist() == [1000, 1001, 1002, 1003]
    w = synth.WORKLOADS
    assert (w["qwen3-8b"].d, w["qwen3-8b"].V, w["qwen3-8b"].temperature) == (4096, 151936, 0.7)
    assert w["qwen3-8b"].per_row_seeds and tuple(w["qwen3-8b"].batches) == (1, 8, 32, 64, 128, 256)
    assert (w["qwen3-1.7b"].d, w["qwen3-1.7b"].V) == (2048, 151936)
    assert (w["large"].d, w["large"].V, w["large"].w_std) == (8192, 128256, 0.015)
    g = w["grouped-masked"]
    assert (g.groups, g.mask_allowed, g.temperature, tuple(g.batches)) == (8, 0.5, 0.8, (1, 64, 512))
    assert (w["tiny"].d, w["tiny"].V, w["tiny"].w_std) == (256, 4096, 1.0 / 16.0)
