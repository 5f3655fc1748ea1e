"""Pins of the CPU oracle against facts fixed outside the oracle itself.

Each test checks the oracle against something independent of its own code:
another implementation of the published Philox4x32-10 algorithm (Triton's,
run on the CPU interpreter), high-precision decimal arithmetic, a library
matmul / logsumexp, closed forms, exact softmax probabilities (chi-square),
and brute force over partitions.  The method statements pinned are those of
FlashSampling (arXiv:2603.15854): the abstract ("argmax decomposes over a
partition", "grouped variants ... exact by hierarchical factorization") and
the readus.org page (Gumbel-Max theorem, Group Gumbel Max, masking with -inf,
the uniform mapping u = (r+1)/(2^32+1), reproducibility under a fixed seed).
"""
import decimal
import itertools
import math

import numpy as np
import pytest
import torch

from lm_head_exact_fmms_b200 import synth

pytestmark = pytest.mark.filterwarnings("ignore::DeprecationWarning")


# --------------------------------------------------------------------------
# Philox4x32-10
# --------------------------------------------------------------------------

def _triton_philox(keys, ctrs):
    """Philox4x32-10 via Triton's own implementation on the CPU interpreter."""
    import os
    os.environ["TRITON_INTERPRET"] = "1"
    triton = pytest.importorskip("triton")
    import triton.language as tl

    @triton.jit
    def _kern(key_ptr, c_ptr, o_ptr, n: tl.constexpr):
        i = tl.arange(0, n)
        klo = tl.load(key_ptr + 2 * i + 0).to(tl.uint64)
        khi = tl.load(key_ptr + 2 * i + 1).to(tl.uint64)
        seed = (khi << 32) | klo
        c0 = tl.load(c_ptr + 4 * i + 0)
        c1 = tl.load(c_ptr + 4 * i + 1)
        c2 = tl.load(c_ptr + 4 * i + 2)
        c3 = tl.load(c_ptr + 4 * i + 3)
        a, b, c, d = tl.philox(seed, c0, c1, c2, c3)
        tl.store(o_ptr + 4 * i + 0, a)
        tl.store(o_ptr + 4 * i + 1, b)
        tl.store(o_ptr + 4 * i + 2, c)
        tl.store(o_ptr + 4 * i + 3, d)

    n = ctrs.shape[0]
    k = torch.from_numpy(keys.astype(np.int64)).to(torch.uint32)
    c = torch.from_numpy(ctrs.astype(np.int64)).to(torch.uint32)
    o = torch.zeros(n, 4, dtype=torch.uint32)
    _kern[(1,)](k, c, o, n)
    return o.to(torch.int64).numpy().astype(np.uint32)


def test_philox_matches_independent_implementation(oracle):
    """Bitwise agreement with Triton's Philox (same published algorithm, written
    independently), over random keys and counters including edge words."""
    rng = np.random.default_rng(7)
    n = 256
    keys = rng.integers(0, 2 ** 32, size=(n, 2), dtype=np.uint64).astype(np.uint32)
    ctrs = rng.integers(0, 2 ** 32, size=(n, 4), dtype=np.uint64).astype(np.uint32)
    ctrs[0] = 0
    keys[0] = 0
    ctrs[1] = 0xFFFFFFFF
    keys[1] = 0xFFFFFFFF
    ref = _triton_philox(keys, ctrs)
    got = oracle.philox4x32_10(ctrs, keys)
    assert np.array_equal(got, ref)


def test_noise_word_layout(oracle):
    """Noise word for (seed, step, row, v, tag) is word v&3 of
    Philox(key=(seed lo, seed hi), counter=(v>>2, row, step, tag))."""
    rng = np.random.default_rng(11)
    cases = []
    for _ in range(64):
        seed = int(rng.integers(0, 2 ** 63)) * 2 + int(rng.integers(0, 2))
        step = int(rng.integers(0, 2 ** 32))
        row = int(rng.integers(0, 2 ** 20))
        v = int(rng.integers(0, 2 ** 24))
        tag = int(rng.integers(0, 2))
        cases.append((seed, step, row, v, tag))
    keys = np.array([[s & 0xFFFFFFFF, s >> 32] for s, *_ in cases], dtype=np.uint32)
    ctrs = np.array([[v >> 2, row, step, tag] for _, step, row, v, tag in cases], dtype=np.uint32)
    ref = _triton_philox(keys, ctrs)
    for i, (seed, step, row, v, tag) in enumerate(cases):
        assert oracle.noise_word(seed, step, row, v, tag) == int(ref[i, v & 3])


def test_philox_bit_balance_and_bytes(oracle):
    """4M consecutive-counter words: every bit is 1 about half the time and the
    byte histogram is uniform (chi-square, 255 dof)."""
    from scipy import stats
    n = 1 << 20
    ctrs = np.zeros((n, 4), dtype=np.uint32)
    ctrs[:, 0] = np.arange(n, dtype=np.uint32)
    ctrs[:, 1] = 3
    out = oracle.philox4x32_10(ctrs, np.array([12345, 678], dtype=np.uint32)).ravel()
    bits = np.unpackbits(out.view(np.uint8)).reshape(-1, 8)
    ones = bits.sum(axis=0) / bits.shape[0]
    sigma = 0.5 / math.sqrt(bits.shape[0])
    assert np.all(np.abs(ones - 0.5) < 6 * sigma)
    hist = np.bincount(out.view(np.uint8), minlength=256)
    chi2 = ((hist - hist.mean()) ** 2 / hist.mean()).sum()
    assert stats.chi2.sf(chi2, 255) > 1e-4
    # neighbouring counters must not share words
    assert len(np.unique(out)) > 0.999 * out.size



def test_philox_digest_definition(oracle):
    """The digest helper equals its definition written out over the oracle's
    own words (word 0 of the counter wrapping past 2^32), and a change of one
    word in one counter changes it."""
    n = 5000
    c0 = (0xFFFFFFFF - 1234, 77, 0xDEADBEEF, 2)
    seed = 0x0123456789ABCDEF
    ctrs = np.empty((n, 4), dtype=np.uint32)
    ctrs[:, 0] = (np.arange(n, dtype=np.uint64) + c0[0]).astype(np.uint32)
    ctrs[:, 1:] = c0[1:]
    words = oracle.philox4x32_10(ctrs, np.array([seed & 0xFFFFFFFF, seed >> 32], dtype=np.uint32))
    weights = np.arange(1, 4 * n + 1, dtype=object).reshape(n, 4)
    want = int((words.astype(object) * weights).sum()) % (1 << 64)
    assert oracle.philox_digest(c0, seed, n) == want
    assert oracle.philox_digest(c0, seed ^ 1, n) != want
    assert oracle.philox_digest((c0[0], c0[1], c0[2], 3), seed, n) != want
    assert oracle.philox_digest(c0, seed, n - 1) != want


# --------------------------------------------------------------------------
# Gumbel transform g(r) = -log(-log((r+1)/(2^32+1)))
# --------------------------------------------------------------------------

def _gumbel_decimal(r):
    ctx = decimal.Context(prec=50)
    u = ctx.divide(decimal.Decimal(r + 1), decimal.Decimal(2 ** 32 + 1))
    t = -ctx.ln(u)
    return float(-ctx.ln(t))


def test_gumbel_high_precision(oracle):
    """fp64 g(r) agrees with 50-digit decimal arithmetic across both branches,
    the branch boundary and both ends of the u32 range."""
    rng = np.random.default_rng(3)
    rs = [0, 1, 2, 255, 2 ** 20, 2 ** 31 - 2, 2 ** 31 - 1, 2 ** 31, 2 ** 31 + 1,
          2 ** 32 - 2 ** 20, 2 ** 32 - 257, 2 ** 32 - 256, 2 ** 32 - 3, 2 ** 32 - 2, 2 ** 32 - 1]
    rs += [int(x) for x in rng.integers(0, 2 ** 32, size=200, dtype=np.uint64)]
    got = oracle.gumbel(np.array(rs, dtype=np.uint32))
    for r, g in zip(rs, got):
        ref = _gumbel_decimal(r)
        assert abs(g - ref) <= 4e-15 * max(1.0, abs(ref)), (r, g, ref)


def test_gumbel_closed_form_ends(oracle):
    """u never reaches 0 or 1 (readus.org page, floating point precision), so
    g is finite at both ends: g(0) = -log(log(2^32+1)), and at r = 2^32-1
    -log u = log1p(1/2^32) so g = -log(log1p(2^-32))."""
    g = oracle.gumbel(np.array([0, 2 ** 32 - 1], dtype=np.uint32))
    assert g[0] == pytest.approx(-math.log(math.log(2 ** 32 + 1)), rel=1e-15)
    assert g[1] == pytest.approx(-math.log(math.log1p(2.0 ** -32)), rel=1e-15)
    assert -3.1 < g[0] < -3.09 and 22.18 < g[1] < 22.19


def test_gumbel_tails_finite_and_monotone(oracle):
    """Exhaustive over both 2^20-wide tails and a stratified sample of the
    middle: g is finite and non-decreasing in r (u rises with r)."""
    lo = np.arange(0, 2 ** 20, dtype=np.uint32)
    hi = np.arange(2 ** 32 - 2 ** 20, 2 ** 32, dtype=np.uint64).astype(np.uint32)
    mid = np.linspace(2 ** 20, 2 ** 32 - 2 ** 20 - 1, 2 ** 20).astype(np.uint64).astype(np.uint32)
    r = np.concatenate([lo, mid, hi])
    g = oracle.gumbel(r)
    assert np.all(np.isfinite(g))
    assert np.all(np.diff(g) >= 0)


def test_gumbel_is_standard_gumbel(oracle):
    """Over uniformly spread r, the Gumbel CDF exp(-exp(-g)) recovers u, i.e.
    g is the Gumbel(0, 1) quantile of u (not, say, an exponential one)."""
    r = np.linspace(0, 2 ** 32 - 1, 100001).astype(np.uint64)
    g = oracle.gumbel(r.astype(np.uint32))
    u = (r.astype(np.float64) + 1.0) / (2.0 ** 32 + 1.0)
    assert np.allclose(np.exp(-np.exp(-g)), u, rtol=1e-12, atol=0)


# --------------------------------------------------------------------------
# Logits
# --------------------------------------------------------------------------

def _bf16_to_f64(x):
    return x.to(torch.float64).numpy()


def test_logits_match_library_matmul(oracle):
    H = synth.make_hidden(5, 96, seed=1)
    W = synth.make_weight(300, 96, 0.3, seed=2)
    got = oracle.logits(H, W)
    ref = _bf16_to_f64(H) @ _bf16_to_f64(W).T
    assert np.allclose(got, ref, rtol=1e-13, atol=1e-13)


def test_logits_one_hot_rows_are_exact(oracle):
    """W rows that are one-hot select entries of h exactly."""
    d, V = 64, 64
    H = synth.make_hidden(3, d, seed=9)
    W = torch.eye(V, d, dtype=torch.bfloat16)
    got = oracle.logits(H, W)
    assert np.array_equal(got, _bf16_to_f64(H)[:, :V])


# --------------------------------------------------------------------------
# Gumbel-Max = softmax (Theorem 2.1 as narrated on the readus.org page)
# --------------------------------------------------------------------------

def _softmax(x):
    z = x - x.max()
    e = np.exp(z)
    return e / e.sum()


def _chi2_pvalue(counts, probs):
    from scipy import stats
    n = counts.sum()
    exp = probs * n
    order = np.argsort(exp)
    # merge the smallest expected bins until each merged bin expects >= 5
    obs_b, exp_b, acc_o, acc_e = [], [], 0.0, 0.0
    for i in order:
        acc_o += counts[i]
        acc_e += exp[i]
        if acc_e >= 5:
            obs_b.append(acc_o)
            exp_b.append(acc_e)
            acc_o = acc_e = 0.0
    if acc_e > 0:
        obs_b[-1] += acc_o
        exp_b[-1] += acc_e
    obs_b, exp_b = np.array(obs_b), np.array(exp_b)
    chi2 = ((obs_b - exp_b) ** 2 / exp_b).sum()
    return stats.chi2.sf(chi2, len(obs_b) - 1)


@pytest.mark.parametrize("G", [0, 3])
def test_histogram_counts_the_sampler_draws(oracle, G):
    """The draw-counting helper that the distribution pins use returns the
    bincount of the samplers' own tokens over the same steps (flat, and
    grouped with uneven groups), masked tokens and row seeds included -- so
    what those pins show about it holds for the samplers."""
    V, d, B, row, T, N, step0 = 61, 32, 3, 1, 0.8, 300, 100
    H = synth.make_hidden(B, d, seed=131)
    W = synth.make_weight(V, d, 0.35, seed=132)
    rs = synth.make_row_seeds(B)
    allowed = torch.from_numpy(np.random.default_rng(133).random((B, V)) < 0.6)
    mask = synth.mask_from_bool(allowed)
    counts = oracle.histogram(H, W, row=row, nsteps=N, G=G, T=T, row_seeds=rs, mask=mask,
                              step0=step0)
    rows = np.array([row], dtype=np.int32)
    want = np.zeros(V + 1, dtype=np.int64)
    for step in range(step0, step0 + N):
        if G:
            idx, _, _ = oracle.sample_grouped(H, W, G, T=T, row_seeds=rs, step=step, mask=mask,
                                              rows=rows)
        else:
            idx, _, _ = oracle.sample(H, W, T=T, row_seeds=rs, step=step, mask=mask, rows=rows)
        want[V if idx[0] < 0 else idx[0]] += 1
    assert np.array_equal(counts, want)


@pytest.mark.parametrize("T", [0.7, 1.0, 2.0])
def test_gumbel_max_matches_softmax(oracle, T):
    """10^6 draws of one row (V=64, d=32) with step = 0 .. 10^6 - 1 follow the
    exact softmax of l / T (chi-square), and not the softmax of l."""
    V, d, N = 64, 32, 1_000_000
    H = synth.make_hidden(1, d, seed=21)
    W = synth.make_weight(V, d, 0.35, seed=22)
    counts = oracle.histogram(H, W, row=0, nsteps=N, T=T, seed=5)
    l = oracle.logits(H, W)[0]
    p = _softmax(l / T)
    assert counts[V] == 0
    assert _chi2_pvalue(counts[:V], p) > 1e-3
    # the same test must reject the temperature-free distribution
    if T != 1.0:
        assert _chi2_pvalue(counts[:V], _softmax(l)) < 1e-6


def test_masked_tokens_never_drawn_and_rest_is_softmax(oracle):
    V, d, N = 64, 32, 400_000
    H = synth.make_hidden(1, d, seed=31)
    W = synth.make_weight(V, d, 0.35, seed=32)
    allowed = torch.rand(1, V, generator=torch.Generator().manual_seed(3)) < 0.5
    mask = synth.mask_from_bool(allowed)
    counts = oracle.histogram(H, W, row=0, nsteps=N, T=1.0, seed=6, mask=mask)
    a = allowed[0].numpy()
    assert counts[:V][~a].sum() == 0 and counts[V] == 0
    l = oracle.logits(H, W)[0]
    p = _softmax(l[a])
    assert _chi2_pvalue(counts[:V][a], p) > 1e-3


def test_mask_edge_cases(oracle):
    V, d, B = 100, 16, 4
    H = synth.make_hidden(B, d, seed=41)
    W = synth.make_weight(V, d, 1.0, seed=42)
    allowed = torch.zeros(B, V, dtype=torch.bool)
    allowed[0, 37] = True          # single allowed token
    allowed[1, :] = False          # everything masked
    allowed[2, :] = True
    allowed[3, 99] = True
    allowed[3, 0] = True
    mask = synth.mask_from_bool(allowed)
    for step in range(20):
        idx, best, second = oracle.sample(H, W, seed=1, step=step, mask=mask)
        assert idx[0] == 37 and second[0] == -np.inf
        assert idx[1] == -1 and best[1] == -np.inf
        assert 0 <= idx[2] < V
        assert idx[3] in (0, 99)


# --------------------------------------------------------------------------
# Argmax decomposes over a partition (abstract)
# --------------------------------------------------------------------------

def _reduce_parts(s, parts):
    """Per-part argmax (first index on ties), then argmax over the part winners
    with ties broken toward the smaller vocab index."""
    best_v, best_s = -1, -np.inf
    for part in parts:
        part = np.sort(np.asarray(part))
        sv = s[part]
        if np.all(sv == -np.inf):
            continue
        v = int(part[int(np.argmax(sv))])
        if best_v < 0 or s[v] > best_s or (s[v] == best_s and v < best_v):
            best_v, best_s = v, s[v]
    return best_v


def test_partition_argmax_equals_global_small(oracle):
    V, d = 12, 16
    H = synth.make_hidden(3, d, seed=51)
    W = synth.make_weight(V, d, 1.0, seed=52)
    s_all = oracle.scores(H, W, seed=8, step=4)
    idx, _, _ = oracle.sample(H, W, seed=8, step=4)
    rng = np.random.default_rng(0)
    for b in range(3):
        s = s_all[b]
        for cuts in itertools.product([0, 1], repeat=V - 1):   # all 2^11 contiguous partitions
            bounds = [0] + [i + 1 for i, c in enumerate(cuts) if c] + [V]
            parts = [range(bounds[i], bounds[i + 1]) for i in range(len(bounds) - 1)]
            assert _reduce_parts(s, parts) == idx[b]
        for _ in range(200):                                     # random set partitions
            labels = rng.integers(0, rng.integers(1, V + 1), size=V)
            parts = [np.flatnonzero(labels == k) for k in np.unique(labels)]
            assert _reduce_parts(s, parts) == idx[b]


def test_partition_argmax_every_tile_size(oracle):
    V, d = 4096, 32
    H = synth.make_hidden(1, d, seed=61)
    W = synth.make_weight(V, d, 0.5, seed=62)
    s = oracle.scores(H, W, seed=9, step=0)[0]
    idx, _, _ = oracle.sample(H, W, seed=9, step=0)
    for t in range(1, V + 1):
        n = -(-V // t)
        padded = np.full(n * t, -np.inf)
        padded[:V] = s
        tiles = padded.reshape(n, t)
        winners = tiles.argmax(axis=1) + np.arange(n) * t
        ws = padded[winners]
        m = ws.max()
        assert winners[ws == m].min() == idx[0]


def test_tie_rule_smallest_index():
    """Reduction rule on planted exact ties: the smallest vocab index wins at
    every level."""
    s = np.array([1.0, 3.0, 2.0, 3.0, -np.inf, 3.0])
    for t in range(1, 7):
        parts = [range(i, min(6, i + t)) for i in range(0, 6, t)]
        assert _reduce_parts(s, parts) == 1


def test_oracle_argmax_scan_ties_to_the_smallest_index(oracle):
    """The oracle's own argmax scan (the one every sampler runs) on scores
    drawn from a handful of values, so exact ties are everywhere, with -inf
    (masked) entries mixed in: the index is numpy's argmax, whose documented
    rule is the first occurrence of the maximum; the best score is the
    maximum and the second-best is the second entry of the sorted finite
    scores (equal to the best on a tie); all -inf gives -1."""
    rng = np.random.default_rng(12)
    for n in (1, 2, 3, 7, 64, 1000):
        for _ in range(200):
            s = rng.integers(0, 4, size=n).astype(np.float64) - 1.5
            s[rng.random(n) < 0.3] = -np.inf
            idx, best, second = oracle.argmax(s)
            fin = np.sort(s[np.isfinite(s)])
            if fin.size == 0:
                assert idx == -1 and best == -np.inf and second == -np.inf
                continue
            assert idx == int(np.argmax(s)), (s, idx)
            assert best == fin[-1]
            assert second == (fin[-2] if fin.size > 1 else -np.inf)
    assert oracle.argmax(np.array([2.0, 5.0, 5.0, 5.0]))[0] == 1
    assert oracle.argmax(np.full(9, -np.inf))[0] == -1


# --------------------------------------------------------------------------
# Group-Gumbel-Max
# --------------------------------------------------------------------------

def test_grouped_single_group_is_flat(oracle):
    V, d, B = 200, 32, 16
    H = synth.make_hidden(B, d, seed=71)
    W = synth.make_weight(V, d, 0.5, seed=72)
    for step in range(5):
        flat, _, _ = oracle.sample(H, W, T=0.9, seed=3, step=step)
        grp, _, _ = oracle.sample_grouped(H, W, 1, T=0.9, seed=3, step=step)
        assert np.array_equal(flat, grp)


@pytest.mark.parametrize("G", [2, 3, 7, 8])
def test_grouped_summary_identities(oracle, G):
    """(1) lse_g is the log-sum-exp of l/T over the group's allowed tokens;
    (2) the argmax over groups of (max s in g) is the flat sample, bitwise."""
    from scipy.special import logsumexp
    V, d, B, T = 301, 32, 8, 0.8
    H = synth.make_hidden(B, d, seed=81)
    W = synth.make_weight(V, d, 0.5, seed=82)
    allowed = torch.rand(B, V, generator=torch.Generator().manual_seed(4)) < 0.6
    allowed[0] = False
    mask = synth.mask_from_bool(allowed)
    flat, _, _ = oracle.sample(H, W, T=T, seed=4, step=2, mask=mask)
    _, summ, _ = oracle.sample_grouped(H, W, G, T=T, seed=4, step=2, mask=mask)
    l = oracle.logits(H, W)
    a = allowed.numpy()
    for b in range(B):
        best_v, best_s = -1, -np.inf
        for g in range(G):
            lo, hi = (g * V) // G, ((g + 1) * V) // G
            sel = a[b, lo:hi]
            ref = logsumexp(l[b, lo:hi][sel] / T) if sel.any() else -np.inf
            assert summ[b, g, 2] == pytest.approx(ref, rel=1e-12, abs=1e-12)
            gs, gv = summ[b, g, 0], int(summ[b, g, 1])
            if gv >= 0 and (best_v < 0 or gs > best_s or (gs == best_s and gv < best_v)):
                best_v, best_s = gv, gs
        assert best_v == flat[b]


@pytest.mark.parametrize("G", [1, 2, 3, 8])
def test_grouped_summary_and_margins_match_the_scores(oracle, G):
    """The grouped sampler's per-group (max score, argmax) and its margins,
    which the GPU tests' tie rule relies on, against the separately pinned
    perturbed scores: each group's maximum and first maximiser over its range;
    the token lies in a group; the within-group margin is the gap between the
    top two scores of the token's group (+inf with one allowed token); the
    group-key margin is positive, and +inf with a single group."""
    V, d, B, T = 211, 24, 12, 0.9
    H = synth.make_hidden(B, d, seed=91)
    W = synth.make_weight(V, d, 0.5, seed=92)
    allowed = torch.rand(B, V, generator=torch.Generator().manual_seed(5)) < 0.5
    allowed[1] = False
    allowed[2] = False
    allowed[2, 17] = True
    mask = synth.mask_from_bool(allowed)
    rs = synth.make_row_seeds(B)
    idx, summ, margin = oracle.sample_grouped(H, W, G, T=T, seed=6, row_seeds=rs, step=3,
                                              mask=mask)
    sc = oracle.scores(H, W, T=T, seed=6, row_seeds=rs, step=3, mask=mask)
    for b in range(B):
        for g in range(G):
            lo, hi = (g * V) // G, ((g + 1) * V) // G
            seg = sc[b, lo:hi]
            if np.isfinite(seg).any():
                assert summ[b, g, 0] == seg.max()
                assert int(summ[b, g, 1]) == lo + int(np.argmax(seg))
            else:
                assert summ[b, g, 0] == -np.inf and int(summ[b, g, 1]) == -1
        if idx[b] < 0:
            assert not np.isfinite(sc[b]).any()
            continue
        g = next(g for g in range(G) if (g * V) // G <= idx[b] < ((g + 1) * V) // G)
        assert idx[b] == int(summ[b, g, 1])
        seg = np.sort(sc[b, (g * V) // G:((g + 1) * V) // G])
        want = seg[-1] - seg[-2] if np.isfinite(seg[-2]) else np.inf
        assert margin[b, 1] == want
        assert margin[b, 0] > 0
        if G == 1:
            assert margin[b, 0] == np.inf
    assert idx[1] == -1 and idx[2] == 17


@pytest.mark.parametrize("G", [2, 3, 8, 64])
def test_grouped_matches_softmax(oracle, G):
    V, d, N, T = 64, 32, 200_000, 1.3
    H = synth.make_hidden(1, d, seed=91)
    W = synth.make_weight(V, d, 0.35, seed=92)
    counts = oracle.histogram(H, W, row=0, nsteps=N, G=G, T=T, seed=12)
    p = _softmax(oracle.logits(H, W)[0] / T)
    assert counts[V] == 0
    assert _chi2_pvalue(counts[:V], p) > 1e-3


def _two_sample_pvalue(a, b, min_count=10):
    """Chi-square test that two count vectors come from one distribution;
    bins with fewer than `min_count` draws in total are pooled."""
    from scipy import stats
    keep = (a + b) >= min_count
    table = [np.append(a[keep], a[~keep].sum()), np.append(b[keep], b[~keep].sum())]
    table = np.array(table)
    table = table[:, table.sum(axis=0) > 0]
    return stats.chi2_contingency(table, correction=False)[1]


@pytest.mark.parametrize("G", [3, 8])
def test_grouped_and_flat_draws_agree(oracle, G):
    """Grouped draws and flat draws, with independent noise, follow one
    distribution (two-sample chi-square); the same test tells apart flat
    draws at two temperatures."""
    V, d, N, T = 64, 32, 200_000, 1.3
    H = synth.make_hidden(1, d, seed=93)
    W = synth.make_weight(V, d, 0.35, seed=94)
    flat = oracle.histogram(H, W, row=0, nsteps=N, T=T, seed=13)[:V]
    grouped = oracle.histogram(H, W, row=0, nsteps=N, G=G, T=T, seed=14)[:V]
    assert _two_sample_pvalue(flat, grouped) > 1e-3
    other_T = oracle.histogram(H, W, row=0, nsteps=N, T=1.0, seed=15)[:V]
    assert _two_sample_pvalue(flat, other_T) < 1e-6


def test_constant_rows_sample_the_noise_argmax(oracle):
    """With every row of W equal, all logits of a row are equal, so the token
    is the allowed index of the largest Gumbel value alone: the sampler's
    noise must be word v&3 of Philox(row seed, (v>>2, row, step, 0)), the
    layout pinned above, and ties go to the smaller index."""
    V, d, B = 1000, 16, 4
    H = synth.make_hidden(B, d, seed=121)
    w = synth.make_weight(1, d, 0.5, seed=122)
    W = w.expand(V, d).contiguous()
    rs = synth.make_row_seeds(B)
    allowed = torch.from_numpy(np.random.default_rng(123).random((B, V)) < 0.5)
    mask = synth.mask_from_bool(allowed)
    for step in (0, 1, 77):
        idx, _, _ = oracle.sample(H, W, T=0.9, row_seeds=rs, step=step, mask=mask)
        for b in range(B):
            words = np.array([oracle.noise_word(int(rs[b]), step, b, v) for v in range(V)],
                             dtype=np.uint32)
            g = np.where(allowed[b].numpy(), oracle.gumbel(words), -np.inf)
            assert idx[b] == int(np.argmax(g)), (step, b)


def test_grouped_masked_groups(oracle):
    V, d, B, G = 64, 16, 3, 4
    H = synth.make_hidden(B, d, seed=101)
    W = synth.make_weight(V, d, 1.0, seed=102)
    allowed = torch.zeros(B, V, dtype=torch.bool)
    allowed[0, 40] = True                 # one group has one allowed token
    allowed[2, :16] = True                # only group 0 allowed
    mask = synth.mask_from_bool(allowed)
    for step in range(10):
        idx, summ, _ = oracle.sample_grouped(H, W, G, seed=2, step=step, mask=mask)
        assert idx[0] == 40
        assert idx[1] == -1
        assert 0 <= idx[2] < 16
        assert np.all(summ[2, 1:, 2] == -np.inf)


# --------------------------------------------------------------------------
# Reproducibility (readus.org page, seed management)
# --------------------------------------------------------------------------

def test_sample_steps_equals_one_call_per_step(oracle):
    """The many-steps helper (logits computed once) returns, bit for bit, what
    one sampling call per step returns, masks and row seeds included."""
    V, d, B, n0, N = 333, 48, 7, 1000, 6
    H = synth.make_hidden(B, d, seed=171)
    W = synth.make_weight(V, d, 0.3, seed=172)
    rs = synth.make_row_seeds(B)
    allowed = torch.from_numpy(np.random.default_rng(173).random((B, V)) < 0.4)
    allowed[3] = False
    mask = synth.mask_from_bool(allowed)
    idx, best, second = oracle.sample_steps(H, W, N, T=0.6, row_seeds=rs, step0=n0, mask=mask)
    for n in range(N):
        i1, b1, s1 = oracle.sample(H, W, T=0.6, row_seeds=rs, step=n0 + n, mask=mask)
        assert np.array_equal(idx[n], i1) and np.array_equal(best[n], b1)
        assert np.array_equal(second[n], s1)
    assert np.all(idx[:, 3] == -1)


def test_same_seed_same_tokens_and_steps_differ(oracle):
    V, d, B = 500, 64, 32
    H = synth.make_hidden(B, d, seed=111)
    W = synth.make_weight(V, d, 0.3, seed=112)
    rs = synth.make_row_seeds(B)
    a, _, _ = oracle.sample(H, W, T=0.7, row_seeds=rs, step=17)
    b, _, _ = oracle.sample(H, W, T=0.7, row_seeds=rs, step=17)
    c, _, _ = oracle.sample(H, W, T=0.7, row_seeds=rs, step=18)
    assert np.array_equal(a, b)
    assert not np.array_equal(a, c)
    rows = np.array([5, 0, 31], dtype=np.int32)
    sub, _, _ = oracle.sample(H, W, T=0.7, row_seeds=rs, step=17, rows=rows)
    assert np.array_equal(sub, a[rows])


# --------------------------------------------------------------------------
# Several samples per row (readus.org page, API: number of samples)
# --------------------------------------------------------------------------

def test_multi_sample_first_is_single_sample(oracle):
    B, d, V = 12, 32, 300
    H = synth.make_hidden(B, d, seed=121)
    W = synth.make_weight(V, d, 0.5, seed=122)
    single, b1, s1 = oracle.sample(H, W, T=0.8, seed=5, step=3)
    multi, mb, ms = oracle.sample_multi(H, W, 6, T=0.8, seed=5, step=3)
    assert np.array_equal(multi[:, 0], single) and np.array_equal(mb[:, 0], b1)
    assert np.array_equal(ms[:, 0], s1)      # the runner-up the tie rule uses, too
    # the samples use distinct noise: they are not all equal
    assert (multi != multi[:, :1]).any()


def test_multi_samples_are_softmax_draws(oracle):
    """All S samples of one row over many steps follow the exact softmax."""
    V, d, S, steps = 64, 32, 16, 4000
    H = synth.make_hidden(1, d, seed=131)
    W = synth.make_weight(V, d, 0.35, seed=132)
    counts = np.zeros(V, dtype=np.int64)
    for step in range(0, steps, 1):
        idx, _, _ = oracle.sample_multi(H, W, S, T=1.2, seed=9, step=step)
        counts += np.bincount(idx.ravel(), minlength=V)
    p = _softmax(oracle.logits(H, W)[0] / 1.2)
    assert _chi2_pvalue(counts, p) > 1e-3


# --------------------------------------------------------------------------
# Top-k (readus.org page, "Top-K and masking": prefilter, then exact Gumbel-max)
# --------------------------------------------------------------------------

def test_topk_degenerate_cases(oracle):
    B, d, V = 10, 32, 257
    H = synth.make_hidden(B, d, seed=141)
    W = synth.make_weight(V, d, 0.5, seed=142)
    for step in range(4):
        flat, fb, fs = oracle.sample(H, W, T=0.9, seed=2, step=step)
        all_k, ab, asec = oracle.sample_topk(H, W, V, T=0.9, seed=2, step=step)
        more, _, _ = oracle.sample_topk(H, W, 10 * V, T=0.9, seed=2, step=step)
        assert np.array_equal(all_k, flat) and np.array_equal(ab, fb) and np.array_equal(more, flat)
        assert np.array_equal(asec, fs)     # the runner-up the tie rule uses, too
        one, _, _ = oracle.sample_topk(H, W, 1, T=0.9, seed=2, step=step)
        assert np.array_equal(one, np.argmax(oracle.logits(H, W), axis=1))   # greedy


def test_topk_respects_mask_and_set(oracle):
    B, d, V, K = 6, 32, 300, 7
    H = synth.make_hidden(B, d, seed=151)
    W = synth.make_weight(V, d, 0.5, seed=152)
    allowed = torch.rand(B, V, generator=torch.Generator().manual_seed(8)) < 0.5
    allowed[0] = False
    mask = synth.mask_from_bool(allowed)
    l = oracle.logits(H, W)
    for step in range(8):
        idx, _, _ = oracle.sample_topk(H, W, K, seed=3, step=step, mask=mask)
        assert idx[0] == -1
        for b in range(1, B):
            a = np.flatnonzero(allowed[b].numpy())
            top = a[np.lexsort((a, -l[b, a]))][:K]
            assert idx[b] in top


def test_topk_all_logits_tied_keeps_the_smallest_indices(oracle):
    """Every W row equal, so every logit of a row ties: the k candidates are
    the k smallest allowed indices, and the token is the largest Gumbel value
    among them (noise from the separately pinned noise-word function)."""
    V, d, B, K = 300, 16, 3, 37
    H = synth.make_hidden(B, d, seed=161)
    W = synth.make_weight(1, d, 0.5, seed=162).expand(V, d).contiguous()
    allowed = torch.from_numpy(np.random.default_rng(163).random((B, V)) < 0.7)
    mask = synth.mask_from_bool(allowed)
    for step in (0, 9):
        idx, _, _ = oracle.sample_topk(H, W, K, T=1.1, seed=77, step=step, mask=mask)
        for b in range(B):
            cand = np.flatnonzero(allowed[b].numpy())[:K]
            words = np.array([oracle.noise_word(77, step, b, int(v)) for v in cand],
                             dtype=np.uint32)
            assert idx[b] == int(cand[np.argmax(oracle.gumbel(words))]), (step, b)


def test_topk_matches_truncated_softmax(oracle):
    V, d, K, N, T = 64, 32, 9, 200_000, 1.1
    H = synth.make_hidden(1, d, seed=161)
    W = synth.make_weight(V, d, 0.35, seed=162)
    l = oracle.logits(H, W)[0]
    counts = np.zeros(V, dtype=np.int64)
    # 2000 rows of the same hidden state, 100 steps: 200k draws
    Hr = H.repeat(2000, 1)
    for step in range(N // 2000):
        idx, _, _ = oracle.sample_topk(Hr, W, K, T=T, seed=4, step=step)
        counts += np.bincount(idx, minlength=V)
    top = np.argsort(-l, kind="stable")[:K]
    assert counts[np.setdiff1d(np.arange(V), top)].sum() == 0
    p = _softmax(l[top] / T)
    assert _chi2_pvalue(counts[top], p) > 1e-3
