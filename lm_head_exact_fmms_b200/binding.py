"""Thin ctypes binding of libfmms.so (include/fmms.h).

Argument marshalling only: tensors are checked for dtype, device, shape and
contiguity and passed as raw pointers; every step of the sampling path runs in
the library's CUDA kernels.  torch supplies device memory and the current
stream.  There is no fallback: if the library is missing, every call raises.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# FMMS_LIBRARY=debug selects the debug build (device-side bounds checks that
# report FS_ERR_DEVICE_BOUNDS through fs_device_status).
_LIB_PATH = os.path.join(_HERE, "libfmms_debug.so" if os.environ.get("FMMS_LIBRARY") == "debug"
                         else "libfmms.so")

FS_OK = 0
_STATUS = {0: "FS_OK", 1: "FS_ERR_INVALID_ARG", 2: "FS_ERR_UNSUPPORTED", 3: "FS_ERR_CUDA",
           4: "FS_ERR_WORKSPACE", 5: "FS_ERR_DEVICE_TIMEOUT", 6: "FS_ERR_DEVICE_BOUNDS"}

# Every symbol include/fmms.h declares.
EXPORTED = ("fs_sample", "fs_sample_ex", "fs_sample_grouped", "fs_sample_unfused",
            "fs_sample_host", "fs_workspace_bytes", "fs_device_status", "fs_status_string",
            "fs_philox4x32_10", "fs_gumbel", "fs_plan_tiles", "fs_plan_group_ctas",
            "fs_sample_noalloc", "fs_test_stalled_sample", "fs_sample_shard_keys",
            "fs_keys_to_tokens", "fs_sample_multi", "fs_workspace_bytes_multi",
            "fs_summarize_group", "fs_merge_groups", "fs_workspace_bytes_summary",
            "fs_sample_topk", "fs_set_cta_pairs", "fs_tp_area_bytes", "fs_tp_area_create",
            "fs_tp_area_destroy", "fs_ipc_handle", "fs_ipc_open", "fs_ipc_close", "fs_sample_tp",
            "fs_tp_wait", "fs_tp_failed", "fs_test_stall_loads", "fs_set_partial_merge",
            "fs_plan_tiles_merged", "fs_plan_batch", "fs_noalloc_status",
            "fs_test_inject_fault", "fs_set_programmatic_launch", "fs_get_policies")

FS_IPC_HANDLE_BYTES = 64


class FmmsError(RuntimeError):
    def __init__(self, status, what):
        super().__init__("%s failed: %s" % (what, _STATUS.get(status, str(status))))
        self.status = status


class GroupSummary(ctypes.Structure):
    _fields_ = [("max_score", ctypes.c_float), ("argmax", ctypes.c_int32), ("lse", ctypes.c_float)]


_lib = None


def library_path() -> str:
    return _LIB_PATH


def load_library():
    """Loads libfmms.so (once).  Raises FmmsError if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise FmmsError(-1, "loading %s (build it with python -m lm_head_exact_fmms_b200.build)"
                        % _LIB_PATH)
    lib = ctypes.CDLL(_LIB_PATH)
    vp, i32, u32, u64, f32, sz = (ctypes.c_void_p, ctypes.c_int, ctypes.c_uint32, ctypes.c_uint64,
                                  ctypes.c_float, ctypes.c_size_t)
    common = [vp, vp, i32, i32, i32]
    lib.fs_sample.argtypes = common + [f32, u64, u32, vp, vp, vp]
    lib.fs_sample_ex.argtypes = common + [f32, u64, vp, u32, vp, vp, vp, sz, vp]
    lib.fs_sample_grouped.argtypes = common + [i32, f32, u64, vp, u32, vp, vp, vp, vp, sz, vp]
    lib.fs_sample_unfused.argtypes = common + [f32, u64, vp, u32, vp, vp, vp, vp, sz, vp]
    lib.fs_sample_host.argtypes = common + [f32, u64, vp, u32, vp, vp, vp]
    lib.fs_sample_noalloc.argtypes = common + [f32, u64, vp, u32, vp, vp, vp]
    lib.fs_test_stalled_sample.argtypes = common + [vp, vp, sz, vp]
    lib.fs_sample_shard_keys.argtypes = common + [i32, i32, f32, u64, vp, u32, vp, vp, vp, sz, vp]
    lib.fs_keys_to_tokens.argtypes = [vp, i32, vp, vp]
    lib.fs_sample_multi.argtypes = common + [i32, f32, u64, vp, u32, vp, vp, vp, sz, vp]
    lib.fs_workspace_bytes_multi.argtypes = [i32, i32, i32]
    lib.fs_workspace_bytes_multi.restype = sz
    lib.fs_summarize_group.argtypes = common + [i32, i32, f32, u64, vp, u32, vp, vp, vp, sz, vp]
    lib.fs_merge_groups.argtypes = [vp, i32, i32, u64, vp, u32, vp, vp]
    lib.fs_workspace_bytes_summary.argtypes = [i32, i32]
    lib.fs_workspace_bytes_summary.restype = sz
    lib.fs_sample_topk.argtypes = common + [i32, f32, u64, vp, u32, vp, vp, vp, vp, sz, vp]
    lib.fs_tp_area_bytes.argtypes = []
    lib.fs_tp_area_bytes.restype = sz
    lib.fs_tp_area_create.argtypes = [ctypes.POINTER(ctypes.c_void_p)]
    lib.fs_tp_area_destroy.argtypes = [vp]
    lib.fs_ipc_handle.argtypes = [vp, vp]
    lib.fs_ipc_open.argtypes = [vp, ctypes.POINTER(ctypes.c_void_p)]
    lib.fs_ipc_close.argtypes = [vp]
    lib.fs_sample_tp.argtypes = common + [i32, i32, f32, u64, vp, u32, vp, vp, i32, u32, vp, sz,
                                          vp]
    lib.fs_tp_wait.argtypes = [vp, i32, u32, vp, u32, vp]
    lib.fs_tp_failed.argtypes = [vp, ctypes.POINTER(ctypes.c_uint32)]
    lib.fs_test_stall_loads.argtypes = [i32]
    lib.fs_set_partial_merge.argtypes = [i32]
    lib.fs_workspace_bytes.argtypes = [i32, i32, i32]
    lib.fs_workspace_bytes.restype = sz
    lib.fs_device_status.argtypes = [vp, sz, vp]
    lib.fs_status_string.argtypes = [i32]
    lib.fs_status_string.restype = ctypes.c_char_p
    lib.fs_philox4x32_10.argtypes = [vp, vp, vp, ctypes.c_int64, vp]
    lib.fs_gumbel.argtypes = [vp, vp, ctypes.c_int64, vp]
    lib.fs_plan_tiles.argtypes = [i32, i32, i32, i32, vp, i32, ctypes.POINTER(ctypes.c_int),
                                  ctypes.POINTER(ctypes.c_int)]
    lib.fs_plan_group_ctas.argtypes = [i32, i32, i32, i32, ctypes.POINTER(ctypes.c_int),
                                       ctypes.POINTER(ctypes.c_int)]
    lib.fs_plan_tiles_merged.argtypes = [i32, i32, i32, i32, vp, i32,
                                         ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int)]
    lib.fs_plan_batch.argtypes = [i32, i32, ctypes.POINTER(ctypes.c_int),
                                  ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int)]
    lib.fs_noalloc_status.argtypes = [vp]
    lib.fs_test_inject_fault.argtypes = [i32, ctypes.POINTER(ctypes.c_int)]
    lib.fs_set_programmatic_launch.argtypes = [i32]
    lib.fs_get_policies.argtypes = [ctypes.POINTER(ctypes.c_int)] * 5
    for name in EXPORTED:
        if name not in ("fs_workspace_bytes", "fs_workspace_bytes_multi",
                        "fs_workspace_bytes_summary", "fs_status_string", "fs_tp_area_bytes"):
            getattr(lib, name).restype = ctypes.c_int
    _lib = lib
    return lib


# ------------------------------------------------------------------ helpers
def _check(status, what):
    if status != FS_OK:
        raise FmmsError(status, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check_operands(H, W):
    if H.dtype != torch.bfloat16 or W.dtype != torch.bfloat16:
        raise TypeError("H and W must be bfloat16")
    if H.dim() != 2 or W.dim() != 2 or H.shape[1] != W.shape[1]:
        raise ValueError("H must be [B, d] and W [V, d]")
    if not (H.is_cuda and W.is_cuda) or H.device != W.device:
        raise ValueError("H and W must be CUDA tensors on the same device")
    if not (H.is_contiguous() and W.is_contiguous()):
        raise ValueError("H and W must be contiguous")
    return H.shape[0], H.shape[1], W.shape[0]


def _opt_dev(t, dtype, n, name, device):
    if t is None:
        return None
    if t.dtype != dtype or not t.is_cuda or t.device != device or not t.is_contiguous():
        raise ValueError("%s must be a contiguous %s CUDA tensor on %s" % (name, dtype, device))
    if t.numel() < n:
        raise ValueError("%s has %d elements, needs %d" % (name, t.numel(), n))
    return t


def _out(out, B, device):
    if out is None:
        return torch.empty(B, dtype=torch.int32, device=device)
    _opt_dev(out, torch.int32, B, "out_idx", device)
    return out


def _seed(seed):
    return ctypes.c_uint64(int(seed) & 0xFFFFFFFFFFFFFFFF)


# ------------------------------------------------------------- entry points
def fs_sample(H, W, temperature=1.0, seed=0, step=0, mask_bits=None, out_idx=None, stream=None):
    """Flat FMMS sample (scalar seed, library workspace).  Returns out_idx [B] int32."""
    lib = load_library()
    B, d, V = _check_operands(H, W)
    mask_bits = _opt_dev(mask_bits, torch.int32, B * ((V + 31) // 32), "mask_bits", H.device)
    out_idx = _out(out_idx, B, H.device)
    _check(lib.fs_sample(_ptr(H), _ptr(W), B, d, V, float(temperature), _seed(seed), int(step),
                         _ptr(mask_bits), _ptr(out_idx), _stream(stream)), "fs_sample")
    return out_idx


def fs_sample_ex(H, W, temperature=1.0, seed=0, row_seeds=None, step=0, mask_bits=None,
                 out_idx=None, workspace=None, stream=None):
    """Flat FMMS sample with optional per-row seeds ([B] int64) and caller workspace (uint8)."""
    lib = load_library()
    B, d, V = _check_operands(H, W)
    row_seeds = _opt_dev(row_seeds, torch.int64, B, "row_seeds", H.device)
    mask_bits = _opt_dev(mask_bits, torch.int32, B * ((V + 31) // 32), "mask_bits", H.device)
    out_idx = _out(out_idx, B, H.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.fs_sample_ex(_ptr(H), _ptr(W), B, d, V, float(temperature), _seed(seed),
                            _ptr(row_seeds), int(step), _ptr(mask_bits), _ptr(out_idx),
                            _ptr(workspace), ws_bytes, _stream(stream)), "fs_sample_ex")
    return out_idx


def fs_sample_grouped(H, W, G, temperature=1.0, seed=0, row_seeds=None, step=0, mask_bits=None,
                      out_idx=None, out_summary=None, workspace=None, stream=None):
    """Group-Gumbel-Max sample.  out_summary, if given, is a float32 CUDA tensor
    [B, G, 3] receiving (max score, argmax bits as int32, lse)."""
    lib = load_library()
    B, d, V = _check_operands(H, W)
    row_seeds = _opt_dev(row_seeds, torch.int64, B, "row_seeds", H.device)
    mask_bits = _opt_dev(mask_bits, torch.int32, B * ((V + 31) // 32), "mask_bits", H.device)
    out_idx = _out(out_idx, B, H.device)
    if out_summary is not None:
        _opt_dev(out_summary, torch.float32, B * G * 3, "out_summary", H.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.fs_sample_grouped(_ptr(H), _ptr(W), B, d, V, int(G), float(temperature),
                                 _seed(seed), _ptr(row_seeds), int(step), _ptr(mask_bits),
                                 _ptr(out_idx), _ptr(out_summary), _ptr(workspace), ws_bytes,
                                 _stream(stream)), "fs_sample_grouped")
    return out_idx


def fs_sample_unfused(H, W, temperature=1.0, seed=0, row_seeds=None, step=0, mask_bits=None,
                      out_idx=None, logits=None, workspace=None, stream=None):
    """Unfused two-kernel mode (measurement only): fp32 logits [B, V] go through HBM."""
    lib = load_library()
    B, d, V = _check_operands(H, W)
    row_seeds = _opt_dev(row_seeds, torch.int64, B, "row_seeds", H.device)
    mask_bits = _opt_dev(mask_bits, torch.int32, B * ((V + 31) // 32), "mask_bits", H.device)
    out_idx = _out(out_idx, B, H.device)
    if logits is None:
        logits = torch.empty(B, V, dtype=torch.float32, device=H.device)
    _opt_dev(logits, torch.float32, B * V, "logits", H.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.fs_sample_unfused(_ptr(H), _ptr(W), B, d, V, float(temperature), _seed(seed),
                                 _ptr(row_seeds), int(step), _ptr(mask_bits), _ptr(out_idx),
                                 _ptr(logits), _ptr(workspace), ws_bytes, _stream(stream)),
           "fs_sample_unfused")
    return out_idx


def fs_sample_host(H_host, W, temperature=1.0, seed=0, row_seeds=None, step=0, mask_bits=None,
                   out_idx_host=None, stream=None):
    """End-to-end call with host buffers: H_host (pinned CPU bf16 [B, d]) in,
    out_idx_host (pinned CPU int32 [B]) out, asynchronous on the stream."""
    lib = load_library()
    if H_host.dtype != torch.bfloat16 or H_host.is_cuda or not H_host.is_contiguous():
        raise ValueError("H_host must be a contiguous CPU bfloat16 tensor")
    if W.dtype != torch.bfloat16 or not W.is_cuda or not W.is_contiguous():
        raise ValueError("W must be a contiguous CUDA bfloat16 tensor")
    if H_host.dim() != 2 or W.dim() != 2 or H_host.shape[1] != W.shape[1]:
        raise ValueError("H_host must be [B, d] and W [V, d]")
    B, d = H_host.shape
    V = W.shape[0]
    row_seeds = _opt_dev(row_seeds, torch.int64, B, "row_seeds", W.device)
    mask_bits = _opt_dev(mask_bits, torch.int32, B * ((V + 31) // 32), "mask_bits", W.device)
    if out_idx_host is None:
        out_idx_host = torch.empty(B, dtype=torch.int32, pin_memory=True)
    elif (out_idx_host.dtype != torch.int32 or out_idx_host.is_cuda
          or not out_idx_host.is_contiguous() or out_idx_host.numel() < B):
        raise ValueError("out_idx_host must be a contiguous CPU int32 tensor of at least B elements")
    _check(lib.fs_sample_host(_ptr(H_host), _ptr(W), B, d, V, float(temperature), _seed(seed),
                              _ptr(row_seeds), int(step), _ptr(mask_bits), _ptr(out_idx_host),
                              _stream(stream)), "fs_sample_host")
    return out_idx_host


def fs_workspace_bytes(B, V, G=0):
    return int(load_library().fs_workspace_bytes(int(B), int(V), int(G)))


def fs_device_status(workspace=None, stream=None):
    lib = load_library()
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    return int(lib.fs_device_status(_ptr(workspace), ws_bytes, _stream(stream)))


def fs_status_string(status):
    return load_library().fs_status_string(int(status)).decode()


def fs_philox4x32_10(ctr, key, stream=None):
    """Device Philox4x32-10 of int32-viewed [n, 4] counters with [n, 2] keys."""
    lib = load_library()
    n = ctr.shape[0]
    out = torch.empty_like(ctr)
    _check(lib.fs_philox4x32_10(_ptr(ctr), _ptr(key), _ptr(out), n, _stream(stream)),
           "fs_philox4x32_10")
    return out


def fs_gumbel(r, stream=None):
    """Device fp32 Gumbel transform of int32-viewed u32 words."""
    lib = load_library()
    out = torch.empty(r.shape, dtype=torch.float32, device=r.device)
    _check(lib.fs_gumbel(_ptr(r), _ptr(out), r.numel(), _stream(stream)), "fs_gumbel")
    return out


def fs_plan_tiles(V, G, num_sms, cta, max_tiles=4096):
    """Host-only schedule query: (tiles int32 [n, 5], num_ctas)."""
    import numpy as np
    lib = load_library()
    buf = np.zeros((max_tiles, 5), dtype=np.int32)
    n = ctypes.c_int(0)
    nc = ctypes.c_int(0)
    _check(lib.fs_plan_tiles(int(V), int(G), int(num_sms), int(cta),
                             buf.ctypes.data_as(ctypes.c_void_p), max_tiles, ctypes.byref(n),
                             ctypes.byref(nc)), "fs_plan_tiles")
    return buf[: min(n.value, max_tiles)].copy(), nc.value


def fs_plan_tiles_merged(V, G, num_sms, cta, max_tiles=4096):
    """Host-only query of the merged-partial schedule: (tiles int32 [n, 8],
    whether the automatic choice merges for this split)."""
    import numpy as np
    lib = load_library()
    buf = np.zeros((max_tiles, 8), dtype=np.int32)
    n = ctypes.c_int(0)
    merges = ctypes.c_int(0)
    _check(lib.fs_plan_tiles_merged(int(V), int(G), int(num_sms), int(cta),
                                    buf.ctypes.data_as(ctypes.c_void_p), max_tiles,
                                    ctypes.byref(n), ctypes.byref(merges)),
           "fs_plan_tiles_merged")
    return buf[: min(n.value, max_tiles)].copy(), bool(merges.value)


_PLAN_KINDS = {"flat": 0, "grouped": 1, "logits": 2}


def fs_plan_batch(B, kind="flat"):
    """Host-only query of how a call of B rows launches: (fused launches,
    first launch's batch tile, 1 if the current policy runs it on CTA pairs)."""
    lib = load_library()
    n, bn, pairs = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_int(0)
    _check(lib.fs_plan_batch(int(B), _PLAN_KINDS[kind], ctypes.byref(n), ctypes.byref(bn),
                             ctypes.byref(pairs)), "fs_plan_batch")
    return n.value, bn.value, pairs.value


def fs_uses_cta_pairs(B, kind="flat"):
    return bool(fs_plan_batch(B, kind)[2])


def fs_fused_launches(B, kind="flat"):
    return fs_plan_batch(B, kind)[0]


def plan_num_ctas(V, G, num_sms):
    lib = load_library()
    n = ctypes.c_int(0)
    nc = ctypes.c_int(0)
    _check(lib.fs_plan_tiles(int(V), int(G), int(num_sms), 0, None, 0, ctypes.byref(n),
                             ctypes.byref(nc)), "fs_plan_tiles")
    return nc.value


def fs_plan_group_ctas(V, G, num_sms, g):
    """Host-only: (first, last) CTA whose range meets group g."""
    lib = load_library()
    a = ctypes.c_int(0)
    z = ctypes.c_int(0)
    _check(lib.fs_plan_group_ctas(int(V), int(G), int(num_sms), int(g), ctypes.byref(a),
                                  ctypes.byref(z)), "fs_plan_group_ctas")
    return a.value, z.value


def fs_sample_noalloc(H, W, temperature=1.0, seed=0, row_seeds=None, step=0, mask_bits=None,
                      out_idx=None, stream=None):
    """Allocation-free flat sample (B <= 256) for callers that may not allocate
    device memory: the library keeps the scratch in a fixed device array.
    Calls on one device share that array, so they must not overlap on the GPU."""
    lib = load_library()
    B, d, V = _check_operands(H, W)
    row_seeds = _opt_dev(row_seeds, torch.int64, B, "row_seeds", H.device)
    mask_bits = _opt_dev(mask_bits, torch.int32, B * ((V + 31) // 32), "mask_bits", H.device)
    out_idx = _out(out_idx, B, H.device)
    _check(lib.fs_sample_noalloc(_ptr(H), _ptr(W), B, d, V, float(temperature), _seed(seed),
                                 _ptr(row_seeds), int(step), _ptr(mask_bits), _ptr(out_idx),
                                 _stream(stream)), "fs_sample_noalloc")
    return out_idx


def fs_noalloc_status(stream=None):
    """Reads and clears the status word of fs_sample_noalloc's fixed array:
    0 (FS_OK) or 5 (FS_ERR_DEVICE_TIMEOUT: a call gave up on a bounded wait)."""
    return int(load_library().fs_noalloc_status(_stream(stream)))


FAULT_KINDS = {"none": 0, "alloc": 1, "launch": 2}


def fs_test_inject_fault(kind=None):
    """Sets the host-side fault injection ("none", "alloc" or "launch"; None
    leaves it unchanged) and returns the kind in force before the call."""
    lib = load_library()
    prev = ctypes.c_int(0)
    k = -1 if kind is None else FAULT_KINDS[kind]
    _check(lib.fs_test_inject_fault(k, ctypes.byref(prev)), "fs_test_inject_fault")
    return {v: n for n, v in FAULT_KINDS.items()}[prev.value]


def fs_test_stalled_sample(H, W, workspace, out_idx=None, stream=None):
    """Failure-detection test hook: launches a sampling kernel whose waits run
    out (about one second); the workspace then holds FS_ERR_DEVICE_TIMEOUT."""
    lib = load_library()
    B, d, V = _check_operands(H, W)
    out_idx = _out(out_idx, B, H.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib.fs_test_stalled_sample(_ptr(H), _ptr(W), B, d, V, _ptr(out_idx), _ptr(workspace),
                                      ws_bytes, _stream(stream)), "fs_test_stalled_sample")
    return out_idx


def fs_set_cta_pairs(policy):
    """Kernel choice for flat-mode calls: -1 automatic, 0 single-CTA kernel
    only, 1 CTA-pair (cta_group::2) kernel whenever possible.  Process-wide."""
    _check(load_library().fs_set_cta_pairs(int(policy)), "fs_set_cta_pairs")


def fs_set_programmatic_launch(on):
    """1: launch the fused kernel as a programmatic dependent of the kernel
    ahead of it in the stream (the default); 0: plain stream order."""
    _check(load_library().fs_set_programmatic_launch(int(on)), "fs_set_programmatic_launch")


def fs_get_policies():
    """The execution-path choices in force (FS_FORCE_PATH, then the fs_set_*
    calls): {"cta_pairs", "partial_merge", "programmatic", "unfused",
    "two_kernel_reduce"}."""
    v = [ctypes.c_int(0) for _ in range(5)]
    _check(load_library().fs_get_policies(*[ctypes.byref(x) for x in v]), "fs_get_policies")
    return dict(zip(("cta_pairs", "partial_merge", "programmatic", "unfused",
                     "two_kernel_reduce"), (x.value for x in v)))


def fs_sample_shard_keys(H, W_shard, vocab_offset, V_total, temperature=1.0, seed=0,
                         row_seeds=None, step=0, mask_bits=None, out_keys=None, workspace=None,
                         stream=None):
    """Packed (score, global token) keys [B] int64 of one vocabulary shard;
    their int64 maximum over shards is the full head's key."""
    lib = load_library()
    B, d, Vs = _check_operands(H, W_shard)
    row_seeds = _opt_dev(row_seeds, torch.int64, B, "row_seeds", H.device)
    mask_bits = _opt_dev(mask_bits, torch.int32, B * ((V_total + 31) // 32), "mask_bits",
                         H.device)
    if out_keys is None:
        out_keys = torch.empty(B, dtype=torch.int64, device=H.device)
    _opt_dev(out_keys, torch.int64, B, "out_keys", H.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.fs_sample_shard_keys(_ptr(H), _ptr(W_shard), B, d, Vs, int(vocab_offset),
                                    int(V_total), float(temperature), _seed(seed), _ptr(row_seeds),
                                    int(step), _ptr(mask_bits), _ptr(out_keys), _ptr(workspace),
                                    ws_bytes, _stream(stream)), "fs_sample_shard_keys")
    return out_keys


def fs_tp_area_bytes():
    return int(load_library().fs_tp_area_bytes())


def fs_tp_area_create():
    """A zeroed exchange area on the current device; returns its address (int)."""
    lib = load_library()
    p = ctypes.c_void_p()
    _check(lib.fs_tp_area_create(ctypes.byref(p)), "fs_tp_area_create")
    return int(p.value)


def fs_tp_area_destroy(area):
    _check(load_library().fs_tp_area_destroy(ctypes.c_void_p(area)), "fs_tp_area_destroy")


def fs_ipc_handle(area):
    """The IPC handle (bytes) of an area made by fs_tp_area_create."""
    buf = ctypes.create_string_buffer(FS_IPC_HANDLE_BYTES)
    _check(load_library().fs_ipc_handle(ctypes.c_void_p(area), buf), "fs_ipc_handle")
    return buf.raw


def fs_ipc_open(handle):
    """Maps a peer's area from its handle; returns the address here (int)."""
    if len(handle) != FS_IPC_HANDLE_BYTES:
        raise ValueError("an IPC handle has %d bytes" % FS_IPC_HANDLE_BYTES)
    p = ctypes.c_void_p()
    _check(load_library().fs_ipc_open(ctypes.create_string_buffer(bytes(handle),
                                                                  FS_IPC_HANDLE_BYTES),
                                      ctypes.byref(p)), "fs_ipc_open")
    return int(p.value)


def fs_ipc_close(area):
    _check(load_library().fs_ipc_close(ctypes.c_void_p(area)), "fs_ipc_close")


def fs_sample_tp(H, W_shard, vocab_offset, V_total, areas, seq, temperature=1.0, seed=0,
                 row_seeds=None, step=0, mask_bits=None, workspace=None, stream=None):
    """One rank's shard with the exchange fused into the kernel; `areas` are
    the addresses of every rank's exchange area as mapped here."""
    lib = load_library()
    B, d, Vs = _check_operands(H, W_shard)
    row_seeds = _opt_dev(row_seeds, torch.int64, B, "row_seeds", H.device)
    mask_bits = _opt_dev(mask_bits, torch.int32, B * ((V_total + 31) // 32), "mask_bits",
                         H.device)
    table = (ctypes.c_void_p * len(areas))(*[ctypes.c_void_p(a) for a in areas])
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.fs_sample_tp(_ptr(H), _ptr(W_shard), B, d, Vs, int(vocab_offset), int(V_total),
                            float(temperature), _seed(seed), _ptr(row_seeds), int(step),
                            _ptr(mask_bits), table, len(areas), int(seq) & 0xFFFFFFFF,
                            _ptr(workspace), ws_bytes, _stream(stream)), "fs_sample_tp")


def fs_tp_wait(area, B, seq, out_idx=None, device=None, stream=None, timeout_us=10_000_000):
    """Tokens of call `seq` once they reach `area`, waiting on the stream for
    at most timeout_us (then -1 tokens, and fs_tp_failed reports the call)."""
    lib = load_library()
    dev = device if device is not None else torch.device("cuda", torch.cuda.current_device())
    out_idx = _out(out_idx, B, dev)
    _check(lib.fs_tp_wait(ctypes.c_void_p(area), int(B), int(seq) & 0xFFFFFFFF, _ptr(out_idx),
                          int(timeout_us), _stream(stream)), "fs_tp_wait")
    return out_idx


def fs_tp_failed(area):
    v = ctypes.c_uint32()
    _check(load_library().fs_tp_failed(ctypes.c_void_p(area), ctypes.byref(v)), "fs_tp_failed")
    return int(v.value)


def fs_set_partial_merge(policy):
    """-1 automatic, 0 never, 1 always: merged 8-row partial tiles (single CTAs)."""
    _check(load_library().fs_set_partial_merge(int(policy)), "fs_set_partial_merge")


def fs_test_stall_loads(on):
    """Test switch: fused kernels issue no loads, so their waits time out."""
    _check(load_library().fs_test_stall_loads(1 if on else 0), "fs_test_stall_loads")


def fs_keys_to_tokens(keys, out_idx=None, stream=None):
    """Tokens [B] int32 from reduced keys [B] int64."""
    lib = load_library()
    B = keys.numel()
    out_idx = _out(out_idx, B, keys.device)
    _check(lib.fs_keys_to_tokens(_ptr(keys), B, _ptr(out_idx), _stream(stream)),
           "fs_keys_to_tokens")
    return out_idx


def fs_sample_multi(H, W, num_samples, temperature=1.0, seed=0, row_seeds=None, step=0,
                    mask_bits=None, out_idx=None, workspace=None, stream=None):
    """num_samples exact draws per row from one pass over W: int32 [B, num_samples]."""
    lib = load_library()
    B, d, V = _check_operands(H, W)
    row_seeds = _opt_dev(row_seeds, torch.int64, B, "row_seeds", H.device)
    mask_bits = _opt_dev(mask_bits, torch.int32, B * ((V + 31) // 32), "mask_bits", H.device)
    if out_idx is None:
        out_idx = torch.empty(B, int(num_samples), dtype=torch.int32, device=H.device)
    _opt_dev(out_idx, torch.int32, B * int(num_samples), "out_idx", H.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.fs_sample_multi(_ptr(H), _ptr(W), B, d, V, int(num_samples), float(temperature),
                               _seed(seed), _ptr(row_seeds), int(step), _ptr(mask_bits),
                               _ptr(out_idx), _ptr(workspace), ws_bytes, _stream(stream)),
           "fs_sample_multi")
    return out_idx


def fs_workspace_bytes_multi(B, V, num_samples):
    return int(load_library().fs_workspace_bytes_multi(int(B), int(V), int(num_samples)))


def fs_summarize_group(H, W_g, vocab_offset, V_total, temperature=1.0, seed=0, row_seeds=None,
                     step=0, mask_bits=None, out_summary=None, workspace=None, stream=None):
    """Summary of one group (rows [vocab_offset, vocab_offset + V_g) of the head):
    float32 [B, 3] records (max score, argmax as int32 bits, lse)."""
    lib = load_library()
    B, d, Vg = _check_operands(H, W_g)
    row_seeds = _opt_dev(row_seeds, torch.int64, B, "row_seeds", H.device)
    mask_bits = _opt_dev(mask_bits, torch.int32, B * ((V_total + 31) // 32), "mask_bits",
                         H.device)
    if out_summary is None:
        out_summary = torch.empty(B, 3, dtype=torch.float32, device=H.device)
    _opt_dev(out_summary, torch.float32, B * 3, "out_summary", H.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.fs_summarize_group(_ptr(H), _ptr(W_g), B, d, Vg, int(vocab_offset), int(V_total),
                                float(temperature), _seed(seed), _ptr(row_seeds), int(step),
                                _ptr(mask_bits), _ptr(out_summary), _ptr(workspace), ws_bytes,
                                _stream(stream)), "fs_summarize_group")
    return out_summary


def fs_merge_groups(summaries, seed=0, row_seeds=None, step=0, out_idx=None, stream=None):
    """Tokens [B] from group summaries [G, B, 3] (float32 records)."""
    lib = load_library()
    G, B = summaries.shape[0], summaries.shape[1]
    row_seeds = _opt_dev(row_seeds, torch.int64, B, "row_seeds", summaries.device)
    out_idx = _out(out_idx, B, summaries.device)
    _check(lib.fs_merge_groups(_ptr(summaries.contiguous()), int(G), int(B), _seed(seed),
                               _ptr(row_seeds), int(step), _ptr(out_idx), _stream(stream)),
           "fs_merge_groups")
    return out_idx


def fs_workspace_bytes_summary(B, V_g):
    return int(load_library().fs_workspace_bytes_summary(int(B), int(V_g)))


def fs_sample_topk(H, W, K, temperature=1.0, seed=0, row_seeds=None, step=0, mask_bits=None,
                   out_idx=None, logits=None, workspace=None, stream=None):
    """Top-k sample: Gumbel-max over each row's K largest allowed logits."""
    lib = load_library()
    B, d, V = _check_operands(H, W)
    row_seeds = _opt_dev(row_seeds, torch.int64, B, "row_seeds", H.device)
    mask_bits = _opt_dev(mask_bits, torch.int32, B * ((V + 31) // 32), "mask_bits", H.device)
    out_idx = _out(out_idx, B, H.device)
    if logits is None:
        logits = torch.empty(B, V, dtype=torch.float32, device=H.device)
    _opt_dev(logits, torch.float32, B * V, "logits", H.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.fs_sample_topk(_ptr(H), _ptr(W), B, d, V, int(K), float(temperature), _seed(seed),
                              _ptr(row_seeds), int(step), _ptr(mask_bits), _ptr(out_idx),
                              _ptr(logits), _ptr(workspace), ws_bytes, _stream(stream)),
           "fs_sample_topk")
    return out_idx
