"""Device-side failure detection without a GPU fault.

Every wait in the fused kernel has a time limit (about one second).  The
test entry point fs_test_stalled_sample tells the load-issuing warp to issue
nothing, so the MMA warp's wait for data runs out: each CTA records
FS_ERR_DEVICE_TIMEOUT in the workspace status word, drains, frees its tensor
memory and exits.  The host reads the status with fs_device_status, and the
same context and workspace then sample correctly again.
"""
import time

import numpy as np
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


def test_wait_timeout_is_reported_and_context_survives(dev, oracle):
    B, d, V = 8, 64, 2048
    H = synth.make_hidden(B, d, seed=3)
    W = synth.make_weight(V, d, 0.125, seed=4)
    Hd, Wd = H.to(dev), W.to(dev)
    ws = torch.zeros(binding.fs_workspace_bytes(B, V, 0), dtype=torch.uint8, device=dev)
    t0 = time.time()
    binding.fs_test_stalled_sample(Hd, Wd, ws)
    status = binding.fs_device_status(ws)
    elapsed = time.time() - t0
    assert status == 5, binding.fs_status_string(status)      # FS_ERR_DEVICE_TIMEOUT
    assert 0.2 < elapsed < 60
    assert int(ws.count_nonzero()) == 0                        # re-zeroed for reuse
    assert binding.fs_device_status(ws) == 0
    got = binding.fs_sample_ex(Hd, Wd, temperature=1.0, seed=2, step=1, workspace=ws)
    torch.cuda.synchronize()
    idx, best, second = oracle.sample(H, W, T=1.0, seed=2, step=1)
    bad = got.cpu().numpy() != idx
    assert not np.any(bad & ((best - second) > 2e-3 * (1 + np.abs(best))))
    assert binding.fs_device_status(ws) == 0
