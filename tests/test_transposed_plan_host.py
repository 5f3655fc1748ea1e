"""The pair schedule's partial tiles, on the CPU, through the library's host
schedule query.

A launch on CTA pairs splits the vocabulary over the pair units exactly as
single CTAs split it over SMs (fs_plan_tiles with num_sms = the number of
units gives each unit's segments), and walks each segment in 256-row pair
tiles, its partial tile first: the segment's length from its first token
rounded down to a multiple of 8, modulo 256, rounded up to 8 rows.  With a
256-row batch tile a partial tile of at most 240 rows is multiplied
transposed, as n = its rows rounded up to 16 columns.  These checks pin the
vocabulary table of the GPU test of those tiles (each vocabulary yields its
width on 74 pairs) and the tile passes of the busiest unit on the LM heads.
"""
import numpy as np
import pytest

from lm_head_exact_fmms_b200 import binding
from tests.test_gpu_transposed import VOCAB_OF_WIDTH

UNITS = 74  # CTA pairs on 148 SMs


def segments(V, G, units):
    """[(unit, first token, end)] of every segment, from the host query."""
    _, n = binding.fs_plan_tiles(V, G, units, 0)
    out = []
    for u in range(n):
        tiles, _ = binding.fs_plan_tiles(V, G, units, u)
        for slot in np.unique(tiles[:, 3]):
            t = tiles[tiles[:, 3] == slot]
            out.append((u, int(t[:, 1].min()), int(t[:, 2].max())))
    return out, n


def pair_tile_costs(V, G, units=UNITS):
    """Per unit: (tile passes with the partial tiles transposed, tile passes
    without, the transposed widths)."""
    segs, n = segments(V, G, units)
    cost_t = np.zeros(n)
    cost_plain = np.zeros(n)
    widths = [[] for _ in range(n)]
    for u, lo, hi in segs:
        start = lo & ~7
        rem = (hi - start) % 256
        whole = (hi - start) // 256
        cost_t[u] += whole
        cost_plain[u] += whole
        if rem:
            rows = min(hi, start + ((rem + 7) & ~7)) - start
            width = (rows + 15) & ~15
            cost_plain[u] += 1
            if width < 256:
                cost_t[u] += width / 256
                widths[u].append(width)
            else:
                cost_t[u] += 1
    return cost_t, cost_plain, widths


@pytest.mark.parametrize("n", sorted(VOCAB_OF_WIDTH))
def test_each_vocabulary_gives_its_width(n):
    V = VOCAB_OF_WIDTH[n]
    _, _, widths = pair_tile_costs(V, 1)
    found = sorted({w for ws in widths for w in ws})
    assert n in found, (n, V, found)
    assert all(16 <= w <= 240 and w % 16 == 0 for w in found)


def test_every_width_from_16_to_240_is_covered():
    assert sorted(VOCAB_OF_WIDTH) == list(range(16, 241, 16))


@pytest.mark.parametrize("V,G,before,after", [
    (151936, 1, 9.0, 8.0625),    # Qwen3 heads: 48 of 74 units own 8 rows past 8 whole tiles
    (151936, 8, 9.0, 8.0625),    # the grouped + masked head: the group cuts add no partial tile
])
def test_busiest_unit_on_the_qwen3_heads(V, G, before, after):
    cost_t, cost_plain, widths = pair_tile_costs(V, G)
    assert cost_plain.max() == before
    assert cost_t.max() == pytest.approx(after)
    assert sum(len(w) for w in widths) == 48
    assert cost_t.sum() == pytest.approx(V / 256 + 48 * (16 - 8) / 256, rel=1e-3)


def test_busiest_unit_on_the_d8192_head():
    """V = 128256: every unit's partial tile holds 192-208 rows."""
    cost_t, cost_plain, widths = pair_tile_costs(128256, 1)
    assert cost_plain.max() == 7
    assert {w for ws in widths for w in ws} <= {192, 208}
    assert 6.75 < cost_t.max() < 6.82
