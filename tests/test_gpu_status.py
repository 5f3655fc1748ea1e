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


def test_injected_host_faults_leave_the_library_usable(dev, oracle):
    """Host-side fault injection (fs_test_inject_fault, or FS_FAULT in the
    environment): with "launch" every sampling call fails with FS_ERR_CUDA
    and enqueues nothing (the output keeps its sentinel); with "alloc" every
    call that needs new device memory fails the same way; once cleared, the
    same calls on the same context sample the oracle's tokens."""
    B, d, V = 16, 64, 3001
    H = synth.make_hidden(B, d, seed=30)
    W = synth.make_weight(V, d, 0.125, seed=31)
    Hd, Wd = H.to(dev), W.to(dev)
    out = torch.full((B,), -7, dtype=torch.int32, device=dev)
    keys = torch.zeros(B, dtype=torch.int64, device=dev)
    torch.cuda.synchronize()
    binding.fs_test_inject_fault("launch")
    try:
        for call in (lambda: binding.fs_sample_ex(Hd, Wd, seed=2, step=1, out_idx=out),
                     lambda: binding.fs_sample_grouped(Hd, Wd, 4, seed=2, step=1, out_idx=out),
                     lambda: binding.fs_sample_noalloc(Hd, Wd, seed=2, step=1, out_idx=out),
                     lambda: binding.fs_keys_to_tokens(keys, out_idx=out)):
            with pytest.raises(binding.FmmsError) as err:
                call()
            assert err.value.status == 3                          # FS_ERR_CUDA
    finally:
        binding.fs_test_inject_fault("none")
    torch.cuda.synchronize()
    assert (out == -7).all()                                       # nothing ran
    # 4 MiB of H: more than any host-entry staging buffer the other tests grew
    Hh = synth.make_hidden(64, 32768, seed=32).pin_memory()
    W2 = synth.make_weight(64, 32768, 0.01, seed=33).to(dev)
    binding.fs_test_inject_fault("alloc")
    try:
        with pytest.raises(binding.FmmsError) as err:
            binding.fs_tp_area_create()
        assert err.value.status == 3
        with pytest.raises(binding.FmmsError) as err:
            binding.fs_sample_host(Hh, W2, seed=1)
        assert err.value.status == 3
    finally:
        binding.fs_test_inject_fault("none")
    got = binding.fs_sample_ex(Hd, Wd, seed=2, step=1, out_idx=out)
    torch.cuda.synchronize()
    idx, best, second = oracle.sample(H, W, T=1.0, seed=2, step=1)
    bad = got.cpu().numpy() != idx
    assert not np.any(bad & ((best - second) > 2e-3 * (1 + np.abs(best))))
    host = binding.fs_sample_host(Hh, W2, seed=1)
    ref = binding.fs_sample(Hh.to(dev), W2, seed=1)
    torch.cuda.synchronize()
    assert torch.equal(host.to(dev), ref)
    area = binding.fs_tp_area_create()
    binding.fs_tp_area_destroy(area)


def test_forced_unfused_path_gives_the_fused_tokens(dev, oracle):
    """FS_FORCE_PATH=unfused (a child process): fs_sample_ex runs the two-kernel
    mode (fp32 logits through HBM, then the sampler) and returns the tokens
    of the fused kernel bit for bit, for one and for two 256-row launches, with
    mask and row seeds; the tokens match the oracle."""
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    shapes = [(5, 128, 3001), (300, 64, 2048)]
    code = """
import json, sys, torch
sys.path.insert(0, %r)
from lm_head_exact_fmms_b200 import binding, synth
assert binding.fs_get_policies()["unfused"] == 1
res = []
for B, d, V in %r:
    H = synth.make_hidden(B, d, seed=B).cuda()
    W = synth.make_weight(V, d, 0.125, seed=V).cuda()
    rs = synth.make_row_seeds(B).cuda()
    mask = synth.make_mask(B, V, 0.5, seed=3).cuda()
    t = binding.fs_sample_ex(H, W, temperature=0.8, seed=2, row_seeds=rs, step=4, mask_bits=mask)
    torch.cuda.synchronize()
    assert binding.fs_device_status(None) == 0
    res.append(t.cpu().tolist())
print(json.dumps(res))
""" % (root, shapes)
    env = dict(os.environ, FS_FORCE_PATH="unfused")
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, env=env,
                         cwd=root, timeout=600)
    assert out.returncode == 0, out.stdout[-2000:] + out.stderr[-2000:]
    forced = json.loads(out.stdout.strip().splitlines()[-1])
    for (B, d, V), toks in zip(shapes, forced):
        H = synth.make_hidden(B, d, seed=B)
        W = synth.make_weight(V, d, 0.125, seed=V)
        rs = synth.make_row_seeds(B)
        mask = synth.make_mask(B, V, 0.5, seed=3)
        fused = binding.fs_sample_ex(H.to(dev), W.to(dev), temperature=0.8, seed=2,
                                     row_seeds=rs.to(dev), step=4, mask_bits=mask.to(dev))
        torch.cuda.synchronize()
        assert fused.cpu().tolist() == toks, (B, d, V)
        idx, best, second = oracle.sample(H, W, T=0.8, seed=2, row_seeds=rs, step=4, mask=mask)
        bad = np.asarray(toks) != idx
        assert not np.any(bad & ((best - second) > 2e-3 * (1 + np.abs(best))))


def test_two_kernel_reduction_gives_the_last_cta_tokens(dev, oracle):
    """FS_FORCE_PATH=twokernel (a child process): flat calls leave the per-row
    maxima for a second, decoding kernel instead of the fused kernel's last
    CTA; single- and several-sample calls, one and two 256-row launches, and
    shard keys give the default path's results bit for bit."""
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

    def runs(binding, synth, torch):
        out = []
        for B, d, V in [(5, 128, 3001), (300, 64, 2048)]:
            H = synth.make_hidden(B, d, seed=B).cuda()
            W = synth.make_weight(V, d, 0.125, seed=V).cuda()
            rs = synth.make_row_seeds(B).cuda()
            t = binding.fs_sample_ex(H, W, temperature=0.8, seed=2, row_seeds=rs, step=4)
            m = binding.fs_sample_multi(H, W, 3, temperature=0.8, seed=2, step=4)
            k = binding.fs_sample_shard_keys(H, W[:1024].contiguous(), 0, V, temperature=0.8,
                                             seed=2, step=4)
            torch.cuda.synchronize()
            assert binding.fs_device_status(None) == 0
            out.append([t.cpu().tolist(), m.cpu().tolist(), k.cpu().tolist()])
        return out

    import inspect
    import textwrap
    src = textwrap.dedent(inspect.getsource(runs))
    code = "import json, sys, torch\nsys.path.insert(0, %r)\n" % root + \
        "from lm_head_exact_fmms_b200 import binding, synth\n" + src + \
        "assert binding.fs_get_policies()['two_kernel_reduce'] == 1\n" + \
        "print(json.dumps(runs(binding, synth, torch)))\n"
    env = dict(os.environ, FS_FORCE_PATH="twokernel")
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, env=env,
                         cwd=root, timeout=600)
    assert out.returncode == 0, out.stdout[-2000:] + out.stderr[-2000:]
    forced = json.loads(out.stdout.strip().splitlines()[-1])
    assert binding.fs_get_policies()["two_kernel_reduce"] == 0
    assert runs(binding, synth, torch) == forced
