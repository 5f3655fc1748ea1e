"""The flat kernel on CTA pairs (two SMs sharing one M = 256 tcgen05 MMA),
and pipeline stages of one or two 64-wide K sub-blocks.

The pair kernel is a B200 design choice, not part of the method, so the
sampled tokens must be those of the single-CTA kernel bit for bit, and both
must match the oracle within the stated tie tolerance.  Every batch tile
(16..256 rows), ragged batches and vocabularies (pair tiles of 256 rows
whose odd half is partly or wholly empty), masks, per-row seeds, several
samples per row, vocabulary shards and the bounded-wait failure path are
covered with the pair kernel forced on.
"""
import time

import numpy as np
import pytest
import torch

from lm_head_exact_fmms_b200 import binding, synth

pytestmark = pytest.mark.gpu

TIE_REL = 2e-3


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from lm_head_exact_fmms_b200 import build
    build.build()
    binding.load_library()
    yield torch.device("cuda:0")
    binding.fs_set_cta_pairs(-1)


def with_policy(policy, fn):
    binding.fs_set_cta_pairs(policy)
    try:
        out = fn()
        torch.cuda.synchronize()
        return out
    finally:
        binding.fs_set_cta_pairs(-1)


def both(fn):
    """(single-CTA result, pair result) of the same call."""
    return with_policy(0, fn), with_policy(1, fn)


def assert_parity(gpu, o_idx, o_best, o_second, what=""):
    gpu = np.asarray(gpu)
    bad = gpu != o_idx
    if bad.any():
        tie = (o_best - o_second) <= TIE_REL * (1.0 + np.abs(o_best))
        hard = bad & ~tie
        assert not hard.any(), "%s: rows %s gpu %s oracle %s" % (
            what, np.flatnonzero(hard)[:8], gpu[hard][:8], o_idx[hard][:8])


def rand_inputs(B, d, V, seed, w_std=None):
    H = synth.make_hidden(B, d, device="cpu", seed=seed)
    W = synth.make_weight(V, d, w_std if w_std is not None else 1.0 / np.sqrt(d), device="cpu",
                          seed=seed + 1)
    return H, W, H.cuda(), W.cuda()


def test_policy_argument_checked(dev):
    with pytest.raises(binding.FmmsError):
        binding.fs_set_cta_pairs(2)
    with pytest.raises(binding.FmmsError):
        binding.fs_set_cta_pairs(-2)
    binding.fs_set_cta_pairs(-1)


@pytest.mark.parametrize("B,d,V", [
    (1, 256, 4096), (8, 64, 300), (9, 128, 5000), (16, 64, 129), (17, 96, 4097),
    (33, 128, 777), (64, 256, 12345), (65, 64, 2000), (100, 128, 256), (128, 64, 8),
    (129, 192, 3001), (200, 64, 9000), (256, 256, 4096), (257, 64, 1500), (300, 40, 640),
    # K not a multiple of the stage's two 64-wide sub-blocks (last stage half
    # full), and a K tail shorter than one sub-block
    (40, 192, 3000), (100, 200, 2500), (120, 72, 999), (50, 8, 100),
])
def test_pairs_equal_single_and_oracle(dev, oracle, B, d, V):
    H, W, Hd, Wd = rand_inputs(B, d, V, seed=3 * B + V)
    single, pair = both(lambda: binding.fs_sample(Hd, Wd, temperature=0.9, seed=21, step=2))
    assert torch.equal(single, pair), (B, d, V)
    assert_parity(pair.cpu().numpy(), *oracle.sample(H, W, T=0.9, seed=21, step=2),
                  "B=%d d=%d V=%d" % (B, d, V))


def test_pairs_masks_row_seeds_and_fully_masked_rows(dev, oracle):
    B, d, V = 70, 128, 6001
    H, W, Hd, Wd = rand_inputs(B, d, V, seed=17)
    rs = synth.make_row_seeds(B)
    allowed = torch.rand(B, V, generator=torch.Generator().manual_seed(8)) < 0.3
    allowed[5] = False                        # no allowed token: -1
    allowed[6] = False
    allowed[6, V - 1] = True                  # one allowed token: always it
    mask = synth.mask_from_bool(allowed)
    for step in (0, 7):
        single, pair = both(lambda: binding.fs_sample_ex(
            Hd, Wd, temperature=0.7, seed=3, row_seeds=rs.cuda(), step=step,
            mask_bits=mask.cuda()))
        assert torch.equal(single, pair)
        got = pair.cpu().numpy()
        assert got[5] == -1 and got[6] == V - 1
        assert_parity(got, *oracle.sample(H, W, T=0.7, seed=3, row_seeds=rs, step=step,
                                          mask=mask), "masked step %d" % step)


def test_pairs_multi_sample_and_shards(dev, oracle):
    from lm_head_exact_fmms_b200.tp import shard_bounds
    B, d, V, S = 96, 128, 7003, 3
    H, W, Hd, Wd = rand_inputs(B, d, V, seed=29)
    single, pair = both(lambda: binding.fs_sample_multi(Hd, Wd, S, temperature=1.1, seed=6,
                                                        step=4))
    assert torch.equal(single, pair)
    idx, best, second = oracle.sample_multi(H, W, S, T=1.1, seed=6, step=4)
    assert_parity(pair.cpu().numpy().ravel(), idx.ravel(), best.ravel(), second.ravel(), "multi")

    def shards():
        keys = [binding.fs_sample_shard_keys(Hd, Wd[lo:hi].contiguous(), lo, V, temperature=1.1,
                                             seed=6, step=4)
                for lo, hi in shard_bounds(V, 3)]
        return binding.fs_keys_to_tokens(torch.stack(keys).max(dim=0).values.contiguous())
    ref = with_policy(0, lambda: binding.fs_sample(Hd, Wd, temperature=1.1, seed=6, step=4))
    assert torch.equal(with_policy(1, shards), ref)


@pytest.mark.parametrize("B", [128, 256])
def test_pairs_full_size_head(dev, oracle, B):
    """The Qwen3-8B-shaped head the benchmark times: pair and single kernels
    agree on every row; the oracle checks sampled rows."""
    wl = synth.WORKLOADS["qwen3-8b"]
    Wd = synth.make_weight(wl.V, wl.d, wl.w_std, device=dev)
    Hd = synth.make_hidden(B, wl.d, device=dev)
    rs = synth.make_row_seeds(B)
    single, pair = both(lambda: binding.fs_sample_ex(Hd, Wd, temperature=wl.temperature, seed=0,
                                                     row_seeds=rs.to(dev), step=0))
    assert torch.equal(single, pair)
    rows = np.array([0, B // 3, B - 1], dtype=np.int32)
    idx, best, second = oracle.sample(Hd.cpu(), Wd.cpu(), T=wl.temperature, seed=0, row_seeds=rs,
                                      step=0, rows=rows)
    assert_parity(pair.cpu().numpy()[rows], idx, best, second, "qwen3-8b B=%d" % B)
    del Wd, Hd
    torch.cuda.empty_cache()


def test_pairs_wait_timeout_is_reported_and_context_survives(dev, oracle):
    """No loads are issued, so the even CTA's MMA wait and then every
    epilogue wait of both CTAs of each pair run out; the kernel records
    FS_ERR_DEVICE_TIMEOUT and exits, and the context samples correctly after."""
    B, d, V = 160, 64, 4096
    H = synth.make_hidden(B, d, seed=13)
    W = synth.make_weight(V, d, 0.125, seed=14)
    Hd, Wd = H.to(dev), W.to(dev)
    ws = torch.zeros(binding.fs_workspace_bytes(B, V, 0), dtype=torch.uint8, device=dev)
    t0 = time.time()
    with_policy(1, lambda: binding.fs_test_stalled_sample(Hd, Wd, ws))
    status = binding.fs_device_status(ws)
    assert status == 5, binding.fs_status_string(status)
    assert time.time() - t0 < 120
    got = with_policy(1, lambda: binding.fs_sample_ex(Hd, Wd, temperature=1.0, seed=2, step=1,
                                                      workspace=ws))
    assert_parity(got.cpu().numpy(), *oracle.sample(H, W, T=1.0, seed=2, step=1), "after")
    assert binding.fs_device_status(ws) == 0


@pytest.mark.parametrize("B,d,V,G,masked", [
    (20, 64, 6007, 3, True), (70, 128, 9001, 8, True), (130, 64, 5000, 1, False),
    (160, 96, 12000, 64, False), (256, 128, 8192, 8, True), (300, 64, 3000, 1000, True),
])
def test_pairs_grouped(dev, oracle, B, d, V, G, masked):
    """Group-Gumbel-Max on CTA pairs: per-group maxima and their tokens equal
    the single-CTA kernel's bit for bit; the group log-sum-exps (merged in
    another order) agree to float rounding; the tokens follow the oracle."""
    H, W, Hd, Wd = rand_inputs(B, d, V, seed=B + G)
    mask = synth.make_mask(B, V, 0.5, seed=G) if masked else None
    md = mask.to(dev) if masked else None

    def call():
        summ = torch.empty(B, G, 3, dtype=torch.float32, device=dev)
        tok = binding.fs_sample_grouped(Hd, Wd, G, temperature=0.8, seed=12, step=2,
                                        mask_bits=md, out_summary=summ)
        return tok, summ

    (t0, s0), (t1, s1) = both(call)
    a0, a1 = s0.cpu(), s1.cpu()
    # max score and argmax, bitwise (argmax -1 of an all-masked group reads as NaN)
    assert torch.equal(a0[:, :, :2].contiguous().view(torch.int32),
                       a1[:, :, :2].contiguous().view(torch.int32))
    l0, l1 = a0[:, :, 2].numpy(), a1[:, :, 2].numpy()
    fin = np.isfinite(l0)
    assert np.array_equal(fin, np.isfinite(l1))
    assert np.allclose(l0[fin], l1[fin], rtol=1e-6, atol=1e-5)
    idx, o_summ, margin = oracle.sample_grouped(H, W, G, T=0.8, seed=12, step=2, mask=mask)
    got = t1.cpu().numpy()
    # Both kernels' tokens follow the oracle; where they differ from it (or
    # from each other, the log-sum-exps being merged in another order), the
    # oracle's group keys or the chosen group's top two scores are a near tie.
    for name, toks in (("single", t0.cpu().numpy()), ("pair", got)):
        for b in np.flatnonzero(toks != idx):
            scale = TIE_REL * (1 + abs(o_summ[b, :, 0].max()))
            assert margin[b, 0] <= scale or margin[b, 1] <= scale, (name, b, toks[b], idx[b])
    if G == 1:
        flat = with_policy(1, lambda: binding.fs_sample_ex(Hd, Wd, temperature=0.8, seed=12,
                                                           step=2, mask_bits=md))
        assert torch.equal(flat, t1)


def test_pairs_grouped_full_size_head(dev, oracle):
    """The grouped-masked workload at B = 512 (two pair launches): pair and
    single kernels agree on every row; the oracle checks sampled rows."""
    wl = synth.WORKLOADS["grouped-masked"]
    B = 512
    Wd = synth.make_weight(wl.V, wl.d, wl.w_std, device=dev)
    Hd = synth.make_hidden(B, wl.d, device=dev)
    mask = synth.make_mask(B, wl.V, wl.mask_allowed)
    single, pair = both(lambda: binding.fs_sample_grouped(Hd, Wd, wl.groups,
                                                          temperature=wl.temperature, seed=0,
                                                          step=0, mask_bits=mask.to(dev)))
    s_np, p_np = single.cpu().numpy(), pair.cpu().numpy()
    # sampled rows (launch edges) and every row where the two kernels differ
    rows = np.union1d([0, 255, 256, B - 1], np.flatnonzero(s_np != p_np)).astype(np.int32)
    assert rows.size <= 4 + 5   # differences only at rare near ties
    idx, summ, margin = oracle.sample_grouped(Hd.cpu(), Wd.cpu(), wl.groups, T=wl.temperature,
                                              seed=0, step=0, mask=mask, rows=rows)
    for name, toks in (("single", s_np[rows]), ("pair", p_np[rows])):
        for i in np.flatnonzero(toks != idx):
            scale = TIE_REL * (1 + abs(summ[i, :, 0].max()))
            assert margin[i, 0] <= scale or margin[i, 1] <= scale, (name, rows[i], toks[i], idx[i])
    del Wd, Hd
    torch.cuda.empty_cache()


@pytest.mark.parametrize("B,grouped", [(48, False), (200, False), (130, True)])
def test_cuda_graph_replay(dev, B, grouped):
    """Calls captured into a CUDA graph (single-CTA and CTA-pair launches,
    the latter with a cluster launch attribute) replay to the eager tokens.
    The first eager call sizes the library workspace, so capture allocates
    nothing."""
    d, V, G = 128, 9000, 4
    _, _, Hd, Wd = rand_inputs(B, d, V, seed=B + 7)
    rs = synth.make_row_seeds(B).to(dev)
    outs = [torch.empty(B, dtype=torch.int32, device=dev) for _ in range(3)]

    def call(i):
        if grouped:
            binding.fs_sample_grouped(Hd, Wd, G, temperature=0.9, seed=3, row_seeds=rs, step=i,
                                      out_idx=outs[i], stream=torch.cuda.current_stream())
        else:
            binding.fs_sample_ex(Hd, Wd, temperature=0.9, seed=3, row_seeds=rs, step=i,
                                 out_idx=outs[i], stream=torch.cuda.current_stream())

    for i in range(3):
        call(i)
    torch.cuda.synchronize()
    eager = [o.clone() for o in outs]
    for o in outs:
        o.fill_(-7)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for i in range(3):
            call(i)
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    for i in range(3):
        assert torch.equal(outs[i], eager[i]), i
    del g


@pytest.mark.parametrize("B", [1, 16, 40, 64, 100, 200])
@pytest.mark.parametrize("d", [320, 384, 448, 576])
def test_partial_last_stage(dev, oracle, B, d):
    """K lengths (d / 64 = 5, 6, 7, 9 sub-blocks) that leave the last stage
    partly filled for every stage shape the kernel picks: four sub-blocks per
    stage at 16 rows, two at 32, three at 64 and on pairs at 128, one on
    pairs at 256; flat and grouped."""
    V = 3001
    H, W, Hd, Wd = rand_inputs(B, d, V, seed=B * 7 + d)
    got = binding.fs_sample(Hd, Wd, temperature=0.9, seed=4, step=1).cpu().numpy()
    assert_parity(got, *oracle.sample(H, W, T=0.9, seed=4, step=1), "B=%d d=%d" % (B, d))
    G = 5
    tok = binding.fs_sample_grouped(Hd, Wd, G, temperature=0.9, seed=4, step=1).cpu().numpy()
    idx, summ, margin = oracle.sample_grouped(H, W, G, T=0.9, seed=4, step=1)
    for b in np.flatnonzero(tok != idx):
        scale = TIE_REL * (1 + abs(summ[b, :, 0].max()))
        assert margin[b, 0] <= scale or margin[b, 1] <= scale, (b, tok[b], idx[b])


def test_programmatic_launch_back_to_back_equals_plain_order(dev, oracle):
    """Back-to-back calls on one stream with no synchronisation between them,
    sharing the library workspace -- flat calls of several batch sizes (single
    CTAs and CTA pairs), grouped calls (fused kernel + merge) and several
    samples per row, interleaved -- give the same tokens bit for bit with the
    fused kernel launched as a programmatic dependent of the kernel ahead
    (its workspace accesses and H loads waiting for it) as in plain stream
    order, and match the oracle."""
    d, V = 256, 20011
    W = synth.make_weight(V, d, 1.0 / 16.0, device="cpu", seed=77)
    Wd = W.cuda()
    Bs = [1, 64, 130, 256, 17, 200]
    Hs = {B: synth.make_hidden(B, d, device="cpu", seed=78 + B) for B in Bs}
    Hd = {B: h.cuda() for B, h in Hs.items()}

    def run():
        outs = []
        for step in range(4):
            for B in Bs:
                outs.append(binding.fs_sample(Hd[B], Wd, temperature=0.9, seed=5, step=step))
            outs.append(binding.fs_sample_grouped(Hd[130], Wd, 5, temperature=0.9, seed=5,
                                                  step=step))
            outs.append(binding.fs_sample_multi(Hd[64], Wd, 3, temperature=0.9, seed=5,
                                                step=step))
        torch.cuda.synchronize()
        return outs
    try:
        binding.fs_set_programmatic_launch(0)
        plain = run()
        binding.fs_set_programmatic_launch(1)
        pdl = run()
    finally:
        binding.fs_set_programmatic_launch(1)
    for a, b in zip(plain, pdl):
        assert torch.equal(a, b)
    for step in range(4):
        for i, B in enumerate(Bs):
            got = pdl[step * (len(Bs) + 2) + i].cpu().numpy()
            assert_parity(got, *oracle.sample(Hs[B], W, T=0.9, seed=5, step=step),
                          "B=%d step %d" % (B, step))
