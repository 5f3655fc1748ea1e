"""Host-side checks of the C ABI that need no GPU: the library loads and
exports every symbol include/fmms.h declares, arguments are validated before
anything touches CUDA, and the split-V schedule the kernels walk covers the
vocabulary exactly once with tiles that never cross a group boundary."""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

from lm_head_exact_fmms_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fmms.h")


@pytest.fixture(scope="module")
def lib():
    from lm_head_exact_fmms_b200 import build
    build.build()
    return binding.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fs_\w+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 12
    for name in names:
        assert hasattr(lib, name), name
    assert set(names) == set(binding.EXPORTED)


def test_status_strings(lib):
    for code, name in binding._STATUS.items():
        assert binding.fs_status_string(code) == name


FAKE = ctypes.c_void_p(0x10000)      # never dereferenced: validation fails first
FAKE_ODD = ctypes.c_void_p(0x10008)  # not 16-byte aligned


def _sample(lib, H=FAKE, W=FAKE, B=4, d=64, V=100, T=1.0, out=FAKE):
    return lib.fs_sample(H, W, B, d, V, T, 0, 0, None, out, None)


@pytest.mark.parametrize("kw", [
    dict(H=None), dict(W=None), dict(out=None), dict(B=0), dict(V=0), dict(d=0), dict(d=4),
    dict(d=12), dict(T=0.0), dict(T=-1.0), dict(T=float("nan")), dict(T=float("inf")),
    dict(H=FAKE_ODD), dict(W=FAKE_ODD),
])
def test_invalid_arguments_rejected_on_host(lib, kw):
    assert _sample(lib, **kw) == 1


def test_grouped_and_unfused_validation(lib):
    g = lambda G: lib.fs_sample_grouped(FAKE, FAKE, 4, 64, 100, G, 1.0, 0, None, 0, None, FAKE,
                                        None, None, 0, None)
    assert g(0) == 1 and g(101) == 1 and g(-3) == 1
    assert lib.fs_sample_unfused(FAKE, FAKE, 4, 64, 100, 1.0, 0, None, 0, None, FAKE, None, None,
                                 0, None) == 1
    assert lib.fs_sample_host(None, FAKE, 4, 64, 100, 1.0, 0, None, 0, None, FAKE, None) == 1
    assert lib.fs_philox4x32_10(None, None, None, 5, None) == 1
    assert lib.fs_test_stalled_sample(None, FAKE, 4, 64, 100, FAKE, None, 0, None) == 1
    assert lib.fs_sample_noalloc(FAKE, FAKE, 4, 64, 100, 0.0, 0, None, 0, None, FAKE, None) == 1
    assert lib.fs_gumbel(None, None, -1, None) == 1


@pytest.mark.parametrize("B,kind,want", [
    (1, "flat", (1, 16, 0)), (16, "flat", (1, 16, 0)), (17, "flat", (1, 32, 0)),
    (64, "flat", (1, 64, 0)), (96, "flat", (1, 96, 0)), (97, "flat", (1, 112, 1)),
    (112, "flat", (1, 112, 1)), (113, "flat", (1, 128, 1)),
    (200, "flat", (1, 208, 1)), (256, "flat", (1, 256, 1)), (257, "flat", (2, 256, 1)),
    (1, "grouped", (1, 16, 0)), (512, "grouped", (2, 256, 1)), (100, "grouped", (1, 112, 1)),
    (90, "grouped", (1, 96, 0)),
    (256, "logits", (1, 256, 0)), (300, "logits", (2, 256, 0)),
])
def test_plan_batch_automatic_choice(lib, B, kind, want):
    """The launch plan of a call: one fused launch per 256 rows, the batch
    tile rounded up to 16 rows, and CTA pairs (automatic policy) from a
    112-row tile up, never in logits mode."""
    binding.fs_set_cta_pairs(-1)
    assert binding.fs_plan_batch(B, kind) == want


def test_plan_batch_follows_the_pair_policy(lib):
    try:
        binding.fs_set_cta_pairs(0)
        assert binding.fs_plan_batch(256)[2] == 0
        binding.fs_set_cta_pairs(1)
        assert binding.fs_plan_batch(1)[2] == 1 and binding.fs_plan_batch(1, "grouped")[2] == 1
        assert binding.fs_plan_batch(1, "logits")[2] == 0
    finally:
        binding.fs_set_cta_pairs(-1)
    n = ctypes.c_int(0)
    assert lib.fs_plan_batch(0, 0, ctypes.byref(n), None, None) == 1
    assert lib.fs_plan_batch(4, 3, ctypes.byref(n), None, None) == 1
    assert lib.fs_plan_batch(4, 0, None, None, None) == 1


def test_fault_injection_switch(lib):
    """fs_test_inject_fault sets and reports the kind; invalid kinds are
    refused; with "launch" set a sampling call with valid arguments fails with
    FS_ERR_CUDA before touching any device."""
    assert binding.fs_test_inject_fault("launch") == "none"
    try:
        assert binding.fs_test_inject_fault() == "launch"
        assert _sample(lib) == 3
        assert lib.fs_sample_noalloc(FAKE, FAKE, 4, 64, 100, 1.0, 0, None, 0, None, FAKE,
                                     None) == 3
        assert binding.fs_test_inject_fault("alloc") == "launch"
        area = ctypes.c_void_p(0)
        assert lib.fs_tp_area_create(ctypes.byref(area)) in (2, 3)
        assert area.value is None
    finally:
        binding.fs_test_inject_fault("none")
    prev = ctypes.c_int(0)
    assert lib.fs_test_inject_fault(3, ctypes.byref(prev)) == 1
    assert lib.fs_test_inject_fault(-2, None) == 1


@pytest.mark.parametrize("env,kind", [("alloc", "alloc"), ("launch", "launch"), ("", "none"),
                                      ("bogus", "none")])
def test_fault_injection_reads_the_environment(env, kind):
    """FS_FAULT sets the initial kind, read at the first call (a fresh
    process per value)."""
    import subprocess
    import sys
    code = ("from lm_head_exact_fmms_b200 import binding; "
            "print(binding.fs_test_inject_fault())")
    envd = dict(os.environ, FS_FAULT=env)
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True,
                         env=envd, cwd=ROOT, timeout=300)
    assert out.returncode == 0, out.stderr[-1000:]
    assert out.stdout.strip().splitlines()[-1] == kind


def _all_tiles(V, G, sms):
    _, nc = binding.fs_plan_tiles(V, G, sms, 0)
    return nc, [binding.fs_plan_tiles(V, G, sms, c)[0] for c in range(nc)]


@pytest.mark.parametrize("V,G,sms", [
    (1, 0, 148), (7, 1, 148), (12, 3, 148), (129, 0, 148), (4096, 0, 148), (4097, 5, 148),
    (151936, 0, 148), (151936, 8, 148), (151937, 8, 148), (128256, 0, 148), (1000, 1000, 148),
    (64, 64, 148), (5003, 7, 13), (100000, 97, 148),
])
def test_schedule_covers_vocab_once(lib, V, G, sms):
    nc, per_cta = _all_tiles(V, G, sms)
    Geff = max(G, 1)
    assert nc == min(sms, (V + 7) // 8)
    bounds = [(g * V) // Geff for g in range(Geff + 1)]
    owner = np.full(V, -1)
    slots = set()
    rows_per_cta = []
    for c, tiles in enumerate(per_cta):
        assert len(tiles) > 0
        rows = 0
        for i, (start, lo, hi, slot, last) in enumerate(tiles):
            assert start % 8 == 0 and start <= lo < hi <= start + 128
            g = np.searchsorted(bounds, lo, side="right") - 1
            assert bounds[g] <= lo and hi <= bounds[g + 1], "tile crosses a group boundary"
            assert slot == c + g and slot < nc + Geff - 1
            assert np.all(owner[lo:hi] == -1), "token covered twice"
            owner[lo:hi] = c
            rows += hi - lo
            nxt = tiles[i + 1] if i + 1 < len(tiles) else None
            assert last == (1 if nxt is None or nxt[3] != slot else 0)
            slots.add((c, g, slot))
        rows_per_cta.append(rows)
    assert np.all(owner >= 0), "token never covered"
    assert np.all(np.diff(owner) >= 0), "CTA ranges are not contiguous and ordered"
    assert len({s for _, _, s in slots}) == len(slots), "slot reused by two segments"
    # balance: every CTA streams the same number of rows to within one granule
    full = rows_per_cta[:-1] if V % 8 else rows_per_cta
    if full:
        assert max(full) - min(full) <= 8
    # the grouped merge enumerates exactly the CTAs that met the group
    if G >= 1:
        for g in range(Geff):
            first, last = binding.fs_plan_group_ctas(V, G, sms, g)
            met = sorted({c for c, gg, _ in slots if gg == g})
            assert met == list(range(first, last + 1))


@pytest.mark.parametrize("V,G,sms", [
    (151936, 0, 148), (151936, 8, 148), (151937, 8, 148), (128256, 0, 148), (4097, 5, 148),
    (5003, 7, 13), (100000, 97, 148), (12, 3, 148), (1000, 1000, 148),
])
def test_merged_schedule_is_the_schedule_with_pairs_fused(lib, V, G, sms):
    """The schedule of the merged-partial kernel variant: expanding each merged
    8-row partial into a tile of its own, just before its tile and with its
    slot, gives exactly the plain schedule; a merged partial is an 8-row tile
    directly followed by a whole tile of the same segment."""
    nc, per_cta = _all_tiles(V, G, sms)
    merged_ctas = 0
    for c in range(nc):
        merged, _ = binding.fs_plan_tiles_merged(V, G, sms, c)
        expanded = []
        any_merged = False
        for start, lo, hi, slot, last, pstart, plo, phi in merged:
            if pstart >= 0:
                any_merged = True
                assert pstart + 8 == start and pstart <= plo < phi <= pstart + 8
                assert hi - lo == 128 or last == 1
                expanded.append((pstart, plo, phi, slot, 0))
            else:
                assert (plo, phi) == (0, 0)
            expanded.append((start, lo, hi, slot, last))
        assert [tuple(t) for t in per_cta[c]] == expanded
        merged_ctas += any_merged
    _, merges = binding.fs_plan_tiles_merged(V, G, sms, 0)
    assert merges == (merged_ctas * 10 >= nc)


def test_merge_choice_on_the_benchmarked_heads(lib):
    """The automatic choice: 48 of the 148 CTAs of a 151936-token head start
    with an 8-row partial tile, so it merges; the 128256-token head has none
    worth it."""
    _, nc = binding.fs_plan_tiles(151936, 0, 148, 0)
    with_partial = sum(bool((binding.fs_plan_tiles_merged(151936, 0, 148, c)[0][:, 5] >= 0).any())
                       for c in range(nc))
    assert (nc, with_partial) == (148, 48)
    assert binding.fs_plan_tiles_merged(151936, 0, 148, 0)[1] is True
    assert binding.fs_plan_tiles_merged(128256, 0, 148, 0)[1] is False


def test_flagship_schedule_balance(lib):
    """Qwen3 heads: 148 CTAs stream 1026-1027 rows each (8.02 tiles), not 8 or 9 tiles."""
    nc, per_cta = _all_tiles(151936, 0, 148)
    rows = [int(sum(t[2] - t[1] for t in tiles)) for tiles in per_cta]
    assert nc == 148 and min(rows) >= 1024 and max(rows) <= 1032


def test_fused_exchange_validation(lib):
    """fs_sample_tp and its helpers reject bad arguments before any CUDA call."""
    areas = (ctypes.c_void_p * 2)(0x100000, 0x200000)          # 256-byte aligned, never touched
    odd = (ctypes.c_void_p * 2)(0x100000, 0x200008)

    def tp(H=FAKE, B=4, V_shard=100, off=0, V_total=200, table=areas, world=2):
        return lib.fs_sample_tp(H, FAKE, B, 64, V_shard, off, V_total, 1.0, 0, None, 0, None,
                                table, world, 0, None, 0, None)
    assert tp(H=None) == 1
    assert tp(B=257) == 2                     # more than one launch's rows
    assert tp(off=4) == 1                     # shard offsets are multiples of 8
    assert tp(off=104) == 1                   # shard beyond V_total
    assert tp(table=None) == 1
    assert tp(world=0) == 1 and tp(world=17) == 1
    assert tp(table=odd) == 1                 # areas are 256-byte aligned
    assert lib.fs_tp_wait(None, 4, 0, FAKE, 1000, None) == 1
    assert lib.fs_tp_wait(FAKE, 0, 0, FAKE, 1000, None) == 1
    assert lib.fs_tp_wait(FAKE, 257, 0, FAKE, 1000, None) == 1
    assert lib.fs_tp_wait(FAKE, 4, 0, None, 1000, None) == 1
    assert lib.fs_tp_wait(FAKE, 4, 0, FAKE, 0, None) == 1            # no time to wait
    assert lib.fs_tp_wait(FAKE, 4, 0, FAKE, 60_000_001, None) == 1   # longer than a minute
    assert lib.fs_ipc_handle(None, None) == 1
    assert lib.fs_ipc_open(None, None) == 1
    assert lib.fs_tp_area_create(None) == 1
    assert lib.fs_tp_area_destroy(None) == 0 and lib.fs_ipc_close(None) == 0
    # the area holds two halves of 256 keys and 256 tokens plus its header
    assert binding.fs_tp_area_bytes() >= 2 * 256 * (8 + 4) + 32
    assert binding.fs_tp_area_bytes() % 256 == 0


class _DeviceTensorStandIn:
    """Just enough of a CUDA bf16 tensor for the binding's argument checks."""
    dtype = torch.bfloat16
    is_cuda = True
    device = torch.device("cuda", 0)

    def __init__(self, *shape):
        self.shape = shape

    def dim(self):
        return len(self.shape)

    def is_contiguous(self):
        return True


def test_host_entry_binding_rejects_mismatched_operands(lib):
    """fs_sample_host's binding refuses, before any library call, a W whose
    inner dimension differs from H's (the C ABI cannot see W's real shape,
    and the kernel would read past its end) and an unusable token buffer."""
    H = torch.zeros(4, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match=r"\[B, d\]"):
        binding.fs_sample_host(H, _DeviceTensorStandIn(100, 32))
    for bad in (torch.zeros(4, dtype=torch.int64), torch.zeros(3, dtype=torch.int32),
                torch.zeros(8, dtype=torch.int32)[::2]):
        with pytest.raises(ValueError, match="out_idx_host"):
            binding.fs_sample_host(H, _DeviceTensorStandIn(100, 64), out_idx_host=bad)


C_CALLER = r"""
#include <stdio.h>
#include "fmms.h"
int main(void) {
  int32_t tiles[8 * 64];
  int n = 0, nc = 0, merges = -1;
  if (fs_plan_tiles(151936, 0, 148, 5, tiles, 64, &n, &nc) != FS_OK) return 1;
  printf("plain %d %d %d %d\n", n, nc, tiles[0], tiles[2]);
  if (fs_plan_tiles_merged(151936, 0, 148, 5, tiles, 64, &n, &merges) != FS_OK) return 2;
  printf("merged %d %d %d\n", n, merges, tiles[5]);
  printf("area %zu\n", fs_tp_area_bytes());
  printf("status %d %s\n",
         (int)fs_sample(NULL, NULL, 1, 64, 100, 1.0f, 0, 0, NULL, NULL, NULL),
         fs_status_string(FS_ERR_INVALID_ARG));
  return 0;
}
"""


def test_c_program_links_and_calls_the_abi(lib):
    """A plain C99 program that includes only include/fmms.h links against
    libfmms.so and gets, from host-only calls, what the Python binding gets."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    work = os.path.join(ROOT, "_build", "c_abi")
    os.makedirs(work, exist_ok=True)
    src, exe = os.path.join(work, "caller.c"), os.path.join(work, "caller")
    with open(src, "w") as f:
        f.write(C_CALLER)
    libdir = os.path.dirname(binding.library_path())
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), src,
                    "-L", libdir, "-lfmms", "-Wl,-rpath," + libdir, "-o", exe], check=True)
    out = subprocess.run([exe], capture_output=True, text=True, timeout=120, check=True).stdout
    lines = dict(line.split(" ", 1) for line in out.strip().splitlines())
    tiles, nc = binding.fs_plan_tiles(151936, 0, 148, 5)
    assert lines["plain"].split() == [str(len(tiles)), str(nc), str(tiles[0][0]), str(tiles[0][2])]
    merged, merges = binding.fs_plan_tiles_merged(151936, 0, 148, 5)
    assert lines["merged"].split() == [str(len(merged)), str(int(merges)), str(merged[0][5])]
    assert int(lines["area"]) == binding.fs_tp_area_bytes()
    assert lines["status"] == "1 FS_ERR_INVALID_ARG"


def test_debug_build_exports_the_same_symbols():
    """libfmms_debug.so (device-side bounds checks, selected with
    FMMS_LIBRARY=debug) exports every symbol the header declares."""
    from lm_head_exact_fmms_b200 import build
    path = build.build(debug=True)
    dbg = ctypes.CDLL(path)
    for name in declared_functions():
        assert hasattr(dbg, name), name
    assert dbg.fs_status_string is not None
    dbg.fs_status_string.restype = ctypes.c_char_p
    assert dbg.fs_status_string(6) == b"FS_ERR_DEVICE_BOUNDS"


def test_programmatic_launch_switch_validates(lib):
    assert lib.fs_set_programmatic_launch(2) == 1
    assert lib.fs_set_programmatic_launch(-1) == 1
    assert lib.fs_set_programmatic_launch(0) == 0
    assert lib.fs_set_programmatic_launch(1) == 0


@pytest.mark.parametrize("env,want,pairs256", [
    (None, {"cta_pairs": -1, "partial_merge": -1, "programmatic": 1, "unfused": 0,
            "two_kernel_reduce": 0}, 1),
    ("single,nomerge,plain,unfused,twokernel",
     {"cta_pairs": 0, "partial_merge": 0, "programmatic": 0, "unfused": 1,
      "two_kernel_reduce": 1}, 0),
    ("pairs,merge,bogus,fused,twokernel,lastcta",
     {"cta_pairs": 1, "partial_merge": 1, "programmatic": 1, "unfused": 0,
      "two_kernel_reduce": 0}, 1),
])
def test_force_path_environment(env, want, pairs256):
    """FS_FORCE_PATH sets the initial execution-path choices (read once, in a
    fresh process per value); fs_plan_batch follows them."""
    import subprocess
    import sys
    code = ("from lm_head_exact_fmms_b200 import binding; import json; "
            "print(json.dumps([binding.fs_get_policies(), binding.fs_plan_batch(256)[2]]))")
    envd = dict(os.environ)
    envd.pop("FS_FORCE_PATH", None)
    if env is not None:
        envd["FS_FORCE_PATH"] = env
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True,
                         env=envd, cwd=ROOT, timeout=300)
    assert out.returncode == 0, out.stderr[-1000:]
    import json
    pol, pairs = json.loads(out.stdout.strip().splitlines()[-1])
    assert pol == want and pairs == pairs256


def test_setters_override_the_environment():
    import subprocess
    import sys
    code = ("from lm_head_exact_fmms_b200 import binding; binding.fs_set_cta_pairs(1); "
            "print(binding.fs_get_policies()['cta_pairs'])")
    envd = dict(os.environ, FS_FORCE_PATH="single")
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True,
                         env=envd, cwd=ROOT, timeout=300)
    assert out.returncode == 0, out.stderr[-1000:]
    assert out.stdout.strip().splitlines()[-1] == "1"
