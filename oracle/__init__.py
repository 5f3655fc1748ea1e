"""CPU oracle for the FlashSampling fused matmul-sample (FMMS) step.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py``, never by
the product package.  It shares no code with the CUDA path.

The arithmetic lives in ``fmms_oracle.c`` (plain C, fp64, OpenMP over
independent entries); this module only marshals numpy arrays into it.
Every function follows the plain definition stated in the C file's header:
Gumbel-max over ``h W^T / T`` with Philox4x32-10 noise keyed on
(seed, step, row, vocab index), and Group-Gumbel-Max for the grouped variant
(FlashSampling, arXiv:2603.15854, abstract; readus.org page, sections
"Gumbel Max Trick", "Group Gumbel Max", "Top-K and masking", "floating point
precision").
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None

_u16p = ctypes.POINTER(ctypes.c_uint16)
_u32p = ctypes.POINTER(ctypes.c_uint32)
_u64p = ctypes.POINTER(ctypes.c_uint64)
_i32p = ctypes.POINTER(ctypes.c_int32)
_i64p = ctypes.POINTER(ctypes.c_int64)
_f64p = ctypes.POINTER(ctypes.c_double)


def _load():
    global _lib
    if _lib is not None:
        return _lib
    path = _build.build()
    lib = ctypes.CDLL(path)
    lib.oracle_philox4x32_10.argtypes = [_u32p, _u32p, _u32p]
    lib.oracle_philox_batch.argtypes = [_u32p, _u32p, _u32p, ctypes.c_int64]
    lib.oracle_philox_digest.argtypes = [ctypes.c_uint32] * 4 + [ctypes.c_uint64, ctypes.c_int64]
    lib.oracle_philox_digest.restype = ctypes.c_uint64
    lib.oracle_noise_word.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint32,
                                      ctypes.c_uint32, ctypes.c_uint32]
    lib.oracle_noise_word.restype = ctypes.c_uint32
    lib.oracle_gumbel_from_u32.argtypes = [ctypes.c_uint32]
    lib.oracle_gumbel_from_u32.restype = ctypes.c_double
    lib.oracle_gumbel_batch.argtypes = [_u32p, _f64p, ctypes.c_int64]
    common = [_u16p, _u16p, ctypes.c_int, ctypes.c_int, ctypes.c_int]
    lib.oracle_logits.argtypes = common + [_i32p, ctypes.c_int, _f64p]
    sample_args = [ctypes.c_double, ctypes.c_uint64, _u64p, ctypes.c_uint32, _u32p,
                   _i32p, ctypes.c_int]
    lib.oracle_scores.argtypes = common + sample_args + [_f64p]
    lib.oracle_sample.argtypes = common + sample_args + [_i32p, _f64p, _f64p]
    lib.oracle_sample_steps.argtypes = common + [ctypes.c_double, ctypes.c_uint64, _u64p,
                                                 ctypes.c_uint32, ctypes.c_int, _u32p, _i32p,
                                                 _f64p, _f64p]
    lib.oracle_sample_grouped.argtypes = common + [ctypes.c_int] + sample_args + [_i32p, _f64p, _f64p]
    lib.oracle_sample_multi.argtypes = common + [ctypes.c_int] + sample_args + [_i32p, _f64p, _f64p]
    lib.oracle_sample_topk.argtypes = common + [ctypes.c_int] + sample_args + [_i32p, _f64p, _f64p]
    lib.oracle_histogram.argtypes = common + [ctypes.c_int, ctypes.c_double, ctypes.c_uint64, _u64p,
                                              ctypes.c_int, _u32p, ctypes.c_uint32, ctypes.c_int64,
                                              _i64p]
    lib.oracle_argmax.argtypes = [_f64p, ctypes.c_int, _f64p, _f64p]
    lib.oracle_argmax.restype = ctypes.c_int
    lib.oracle_num_threads.restype = ctypes.c_int
    _lib = lib
    return lib


def _ptr(a, typ):
    if a is None:
        return ctypes.cast(None, typ)
    return a.ctypes.data_as(typ)


def _as_u16(x):
    """bf16 payload as a contiguous uint16 numpy array (torch bf16 tensors and
    uint16 arrays are both accepted)."""
    if hasattr(x, "view") and hasattr(x, "dtype") and str(x.dtype) == "torch.bfloat16":
        import torch
        x = x.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    return np.ascontiguousarray(x, dtype=np.uint16)


def _opt(x, dtype):
    if x is None:
        return None
    if hasattr(x, "cpu"):
        x = x.cpu().numpy()
    return np.ascontiguousarray(x, dtype=dtype)


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def philox4x32_10(ctr, key):
    """Philox4x32-10 of one or more counters.  ctr: [..., 4] u32, key: [..., 2] u32."""
    lib = _load()
    ctr = np.ascontiguousarray(ctr, dtype=np.uint32)
    key = np.ascontiguousarray(np.broadcast_to(key, ctr.shape[:-1] + (2,)), dtype=np.uint32)
    out = np.empty_like(ctr)
    n = ctr.size // 4
    lib.oracle_philox_batch(_ptr(ctr, _u32p), _ptr(key, _u32p), _ptr(out, _u32p), n)
    return out


def philox_digest(ctr0, seed, n) -> int:
    """Digest of the Philox words of the n counters (ctr0[0] + i mod 2^32,
    ctr0[1], ctr0[2], ctr0[3]) under `seed`: sum of word j of counter i times
    (4 i + j + 1), mod 2^64."""
    c = [int(x) & 0xFFFFFFFF for x in ctr0]
    return int(_load().oracle_philox_digest(c[0], c[1], c[2], c[3], int(seed) % (1 << 64), int(n)))


def noise_word(seed, step, row, index, tag=0) -> int:
    return int(_load().oracle_noise_word(seed, step, row, index, tag))


def gumbel(r):
    """fp64 Gumbel transform g(r) = -log(-log((r+1)/(2^32+1))) of u32 words."""
    lib = _load()
    r = np.ascontiguousarray(r, dtype=np.uint32)
    out = np.empty(r.shape, dtype=np.float64)
    lib.oracle_gumbel_batch(_ptr(r, _u32p), _ptr(out, _f64p), r.size)
    return out


def argmax(s):
    """The samplers' argmax scan over a 1-D fp64 score array: returns (index,
    best, second); -inf entries (masked tokens) never win, the smallest index
    wins ties, and the index is -1 when every entry is -inf."""
    lib = _load()
    s = np.ascontiguousarray(s, dtype=np.float64)
    b1 = ctypes.c_double()
    b2 = ctypes.c_double()
    i = lib.oracle_argmax(_ptr(s, _f64p), int(s.size), ctypes.byref(b1), ctypes.byref(b2))
    return int(i), b1.value, b2.value


def _rows(rows, B):
    if rows is None:
        rows = np.arange(B, dtype=np.int32)
    return np.ascontiguousarray(rows, dtype=np.int32)


def logits(H, W, rows=None):
    """fp64 logits l[rows, :] = H[rows] W^T."""
    lib = _load()
    H16, W16 = _as_u16(H), _as_u16(W)
    B, d = H16.shape
    V = W16.shape[0]
    rows = _rows(rows, B)
    out = np.empty((rows.size, V), dtype=np.float64)
    lib.oracle_logits(_ptr(H16, _u16p), _ptr(W16, _u16p), B, d, V, _ptr(rows, _i32p), rows.size,
                      _ptr(out, _f64p))
    return out


def _sample_common(H, W, T, seed, row_seeds, step, mask, rows):
    H16, W16 = _as_u16(H), _as_u16(W)
    B, d = H16.shape
    V = W16.shape[0]
    rs = _opt(row_seeds, np.uint64)
    mk = _opt(mask, np.uint32)
    rows = _rows(rows, B)
    return H16, W16, B, d, V, rs, mk, rows


def scores(H, W, T=1.0, seed=0, row_seeds=None, step=0, mask=None, rows=None):
    """Perturbed scores s[rows, :] = l/T + g (or -inf where masked), fp64."""
    lib = _load()
    H16, W16, B, d, V, rs, mk, rows = _sample_common(H, W, T, seed, row_seeds, step, mask, rows)
    out = np.empty((rows.size, V), dtype=np.float64)
    lib.oracle_scores(_ptr(H16, _u16p), _ptr(W16, _u16p), B, d, V, float(T), int(seed),
                      _ptr(rs, _u64p), int(step), _ptr(mk, _u32p), _ptr(rows, _i32p), rows.size,
                      _ptr(out, _f64p))
    return out


def sample(H, W, T=1.0, seed=0, row_seeds=None, step=0, mask=None, rows=None):
    """Flat FMMS sample of the listed rows.

    Returns (idx int32 [n], best f64 [n], second f64 [n]): the sampled token
    (-1 if every token is masked), its perturbed score and the runner-up's."""
    lib = _load()
    H16, W16, B, d, V, rs, mk, rows = _sample_common(H, W, T, seed, row_seeds, step, mask, rows)
    idx = np.empty(rows.size, dtype=np.int32)
    best = np.empty(rows.size, dtype=np.float64)
    second = np.empty(rows.size, dtype=np.float64)
    lib.oracle_sample(_ptr(H16, _u16p), _ptr(W16, _u16p), B, d, V, float(T), int(seed),
                      _ptr(rs, _u64p), int(step), _ptr(mk, _u32p), _ptr(rows, _i32p), rows.size,
                      _ptr(idx, _i32p), _ptr(best, _f64p), _ptr(second, _f64p))
    return idx, best, second


def sample_steps(H, W, nsteps, T=1.0, seed=0, row_seeds=None, step0=0, mask=None):
    """Flat FMMS sample of every row at steps step0 .. step0+nsteps-1 (the
    logits computed once).  Returns (idx int32 [nsteps, B], best, second f64
    [nsteps, B]), equal to `sample` called at each step."""
    lib = _load()
    H16, W16, B, d, V, rs, mk, _ = _sample_common(H, W, T, seed, row_seeds, step0, mask, None)
    idx = np.empty((nsteps, B), dtype=np.int32)
    best = np.empty((nsteps, B), dtype=np.float64)
    second = np.empty((nsteps, B), dtype=np.float64)
    lib.oracle_sample_steps(_ptr(H16, _u16p), _ptr(W16, _u16p), B, d, V, float(T), int(seed),
                            _ptr(rs, _u64p), int(step0), int(nsteps), _ptr(mk, _u32p),
                            _ptr(idx, _i32p), _ptr(best, _f64p), _ptr(second, _f64p))
    return idx, best, second


def sample_multi(H, W, S, T=1.0, seed=0, row_seeds=None, step=0, mask=None, rows=None):
    """S samples per row (sample k uses token-noise tag 2k).

    Returns (idx int32 [n, S], best f64 [n, S], second f64 [n, S])."""
    lib = _load()
    H16, W16, B, d, V, rs, mk, rows = _sample_common(H, W, T, seed, row_seeds, step, mask, rows)
    idx = np.empty((rows.size, S), dtype=np.int32)
    best = np.empty((rows.size, S), dtype=np.float64)
    second = np.empty((rows.size, S), dtype=np.float64)
    lib.oracle_sample_multi(_ptr(H16, _u16p), _ptr(W16, _u16p), B, d, V, int(S), float(T),
                            int(seed), _ptr(rs, _u64p), int(step), _ptr(mk, _u32p),
                            _ptr(rows, _i32p), rows.size, _ptr(idx, _i32p), _ptr(best, _f64p),
                            _ptr(second, _f64p))
    return idx, best, second


def sample_topk(H, W, K, T=1.0, seed=0, row_seeds=None, step=0, mask=None, rows=None):
    """Top-k sample of the listed rows: Gumbel-max over each row's k allowed
    tokens with the largest logits (ties toward the smaller index).

    Returns (idx int32 [n], best f64 [n], second f64 [n])."""
    lib = _load()
    H16, W16, B, d, V, rs, mk, rows = _sample_common(H, W, T, seed, row_seeds, step, mask, rows)
    idx = np.empty(rows.size, dtype=np.int32)
    best = np.empty(rows.size, dtype=np.float64)
    second = np.empty(rows.size, dtype=np.float64)
    lib.oracle_sample_topk(_ptr(H16, _u16p), _ptr(W16, _u16p), B, d, V, int(K), float(T),
                           int(seed), _ptr(rs, _u64p), int(step), _ptr(mk, _u32p),
                           _ptr(rows, _i32p), rows.size, _ptr(idx, _i32p), _ptr(best, _f64p),
                           _ptr(second, _f64p))
    return idx, best, second


def sample_grouped(H, W, G, T=1.0, seed=0, row_seeds=None, step=0, mask=None, rows=None):
    """Group-Gumbel-Max sample of the listed rows.

    Returns (idx int32 [n], summary f64 [n, G, 3] = (max s, argmax, lse) per
    group, margin f64 [n, 2] = (group-key gap, within-group gap))."""
    lib = _load()
    H16, W16, B, d, V, rs, mk, rows = _sample_common(H, W, T, seed, row_seeds, step, mask, rows)
    idx = np.empty(rows.size, dtype=np.int32)
    summ = np.empty((rows.size, G, 3), dtype=np.float64)
    margin = np.empty((rows.size, 2), dtype=np.float64)
    lib.oracle_sample_grouped(_ptr(H16, _u16p), _ptr(W16, _u16p), B, d, V, int(G), float(T),
                              int(seed), _ptr(rs, _u64p), int(step), _ptr(mk, _u32p),
                              _ptr(rows, _i32p), rows.size, _ptr(idx, _i32p), _ptr(summ, _f64p),
                              _ptr(margin, _f64p))
    return idx, summ, margin


def histogram(H, W, row, nsteps, G=0, T=1.0, seed=0, row_seeds=None, mask=None, step0=0):
    """Counts of sampled tokens of row ``row`` over steps step0..step0+nsteps-1.

    Returns int64 [V+1]; the last entry counts rows with no allowed token."""
    lib = _load()
    H16, W16 = _as_u16(H), _as_u16(W)
    B, d = H16.shape
    V = W16.shape[0]
    rs = _opt(row_seeds, np.uint64)
    mk = _opt(mask, np.uint32)
    counts = np.zeros(V + 1, dtype=np.int64)
    lib.oracle_histogram(_ptr(H16, _u16p), _ptr(W16, _u16p), B, d, V, int(G), float(T), int(seed),
                         _ptr(rs, _u64p), int(row), _ptr(mk, _u32p), int(step0), int(nsteps),
                         _ptr(counts, _i64p))
    return counts
