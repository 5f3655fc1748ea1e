"""The allocation-free entry point returns the same tokens as fs_sample_ex.

fs_sample_noalloc is for callers that may not call cudaMalloc, such as a
serving engine that owns all device memory through its own pool and gives a
plug-in only its inputs and outputs.  Instead of a workspace it uses a fixed
scratch array inside the library.  This test calls it through the C ABI twice
in a row and compares each result with the regular entry point's tokens for
the same inputs (the kernels are the same, so the tokens must be identical),
then checks that a batch above its 256-row limit is refused and that a call
whose kernel gave up on a bounded wait is reported by fs_noalloc_status (the
array's own status word, which later calls keep until it is read).  It lives
in its own file so that pytest collects it last.
"""
import pytest
import torch

from lm_head_exact_fmms_b200 import binding, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from lm_head_exact_fmms_b200 import build
    build.build()
    binding.load_library()
    return torch.device("cuda:0")


@pytest.mark.parametrize("B", [1, 2, 96, 256])
def test_noalloc_matches_fs_sample_ex_on_two_calls(dev, B):
    """1 and 2 rows, 96 rows (single CTAs) and 256 rows (CTA pairs, whose
    ticket counts both CTAs of every pair)."""
    d, V = 256, 20011
    H = synth.make_hidden(B, d, device="cpu", seed=7).to(dev)
    W = synth.make_weight(V, d, 1.0 / 16.0, device="cpu", seed=8).to(dev)
    seeds = synth.make_row_seeds(B).to(dev)
    mask = synth.make_mask(B, V, 0.6, seed=9).to(dev)
    for step in (3, 4):
        ref = binding.fs_sample_ex(H, W, temperature=0.8, seed=1, row_seeds=seeds, step=step,
                                   mask_bits=mask)
        first = binding.fs_sample_noalloc(H, W, temperature=0.8, seed=1, row_seeds=seeds,
                                          step=step, mask_bits=mask)
        second = binding.fs_sample_noalloc(H, W, temperature=0.8, seed=1, row_seeds=seeds,
                                           step=step, mask_bits=mask)
        torch.cuda.synchronize()
        assert torch.equal(first, ref)
        assert torch.equal(second, ref)


def test_noalloc_refuses_batches_above_its_limit(dev):
    B, d, V = 257, 64, 1000
    H = synth.make_hidden(B, d, device="cpu", seed=10).to(dev)
    W = synth.make_weight(V, d, 0.125, device="cpu", seed=11).to(dev)
    with pytest.raises(binding.FmmsError) as err:
        binding.fs_sample_noalloc(H, W)
    assert err.value.status == 2   # FS_ERR_UNSUPPORTED


def test_noalloc_reports_a_kernel_that_gave_up(dev):
    """With the failure-detection switch on, the load warp issues nothing and
    the kernel's bounded waits run out (about a second): fs_noalloc_status
    then reports FS_ERR_DEVICE_TIMEOUT, also after a later good call, and
    reads 0 once cleared; the calls after it match fs_sample_ex again."""
    B, d, V = 24, 128, 5003
    H = synth.make_hidden(B, d, device="cpu", seed=12).to(dev)
    W = synth.make_weight(V, d, 0.125, device="cpu", seed=13).to(dev)
    assert binding.fs_noalloc_status() == 0
    binding.fs_test_stall_loads(True)
    try:
        binding.fs_sample_noalloc(H, W, temperature=0.9, seed=5, step=0)
    finally:
        binding.fs_test_stall_loads(False)
    ref = binding.fs_sample_ex(H, W, temperature=0.9, seed=5, step=1)
    got = binding.fs_sample_noalloc(H, W, temperature=0.9, seed=5, step=1)
    torch.cuda.synchronize()
    assert torch.equal(got, ref)
    assert binding.fs_noalloc_status() == 5    # FS_ERR_DEVICE_TIMEOUT, kept until read
    assert binding.fs_noalloc_status() == 0
    again = binding.fs_sample_noalloc(H, W, temperature=0.9, seed=5, step=1)
    torch.cuda.synchronize()
    assert torch.equal(again, ref)
    assert binding.fs_noalloc_status() == 0
