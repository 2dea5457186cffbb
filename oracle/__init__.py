"""CPU fp64 attention oracle -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The CUDA
library never imports it and shares no code with it.

The arithmetic lives in ``attention_oracle.c`` (plain fp64 C, OpenMP over
independent problems); this module only marshals numpy arrays into it.  See
that file's header for the definitions it follows and for which page passage
each one cites.  ``brute.py`` is a second, fully independent pure-Python
implementation for tiny shapes.  ``columns.py`` holds the key-column sampler
(dK, dV of selected key rows at sizes where the full backward is too slow),
written with fp64 torch matrix products on the CPU.
"""
import ctypes
import os

import numpy as np

from . import build as _build
from .columns import attention_cols  # noqa: F401  (key-column sampler, torch fp64)

_lib = None


def load_library(path):
    """Open a compiled oracle library and declare its signatures."""
    lib = ctypes.CDLL(path)
    dp = ctypes.POINTER(ctypes.c_double)
    ip = ctypes.POINTER(ctypes.c_int)
    lp = ctypes.POINTER(ctypes.c_long)
    common = [ctypes.c_int] * 5 + [ctypes.c_double, ctypes.c_int, ip, ctypes.c_int]
    lib.oracle_attention_fwd.argtypes = [dp, dp, dp, dp, dp] + common
    lib.oracle_attention_fwd.restype = ctypes.c_int
    lib.oracle_attention_bwd.argtypes = [dp] * 10 + common
    lib.oracle_attention_bwd.restype = ctypes.c_int
    lib.oracle_attention_rows.argtypes = [dp, dp, dp, dp, lp, ctypes.c_long,
                                          dp, dp, dp, dp] + common
    lib.oracle_attention_rows.restype = ctypes.c_int
    lib.oracle_attention_fwd_streaming.argtypes = [dp, dp, dp, dp, dp, ctypes.c_int,
                                                   ctypes.c_int, ctypes.c_double,
                                                   ctypes.c_int, ctypes.c_int, ip]
    lib.oracle_attention_fwd_streaming.restype = ctypes.c_int
    bp = ctypes.POINTER(ctypes.c_ubyte)
    maskc = [ctypes.c_int] * 5 + [ctypes.c_double, ctypes.c_int, bp, ctypes.c_long,
                                  ctypes.c_long, ctypes.c_int]
    lib.oracle_attention_fwd_blockmask.argtypes = [dp, dp, dp, dp, dp] + maskc
    lib.oracle_attention_fwd_blockmask.restype = ctypes.c_int
    lib.oracle_attention_bwd_blockmask.argtypes = [dp] * 10 + maskc
    lib.oracle_attention_bwd_blockmask.restype = ctypes.c_int
    lib.oracle_softmax_rows.argtypes = [dp, ctypes.c_long, ctypes.c_int, ctypes.c_double,
                                        ctypes.c_int, dp, dp, ctypes.c_int]
    lib.oracle_softmax_rows.restype = ctypes.c_int
    lib.oracle_num_threads.argtypes = []
    lib.oracle_num_threads.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = load_library(_build.build())
    return _lib


class use_library:
    """Context manager: route this module's calls to another compiled copy
    of the oracle (the tests use it to run the pins on planted mistakes)."""

    def __init__(self, path):
        self.path = path

    def __enter__(self):
        global _lib
        self._saved = _lib
        _lib = load_library(self.path)
        return _lib

    def __exit__(self, *exc):
        global _lib
        _lib = self._saved
        return False


def _f64(a):
    a = np.ascontiguousarray(np.asarray(a, dtype=np.float64))
    return a


def _dptr(a):
    if a is None:
        return ctypes.POINTER(ctypes.c_double)()
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _cu(cu_seqlens):
    if cu_seqlens is None:
        return None, ctypes.POINTER(ctypes.c_int)()
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
    return cu, cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int))


def _dims(q, k, cu_seqlens):
    """(B, Hq, Hkv, N, d) from the arrays' shapes.

    dense: q [B, N, Hq, d], k [B, N, Hkv, d]; varlen: q [total, Hq, d]."""
    if cu_seqlens is None:
        B, N, Hq, d = q.shape
        Hkv = k.shape[2]
    else:
        _, Hq, d = q.shape
        Hkv = k.shape[1]
        cu = np.asarray(cu_seqlens)
        B = len(cu) - 1
        N = int(np.max(np.diff(cu))) if B > 0 else 0
    return B, Hq, Hkv, N, d


def num_threads():
    return _load().oracle_num_threads()


def attention_fwd(q, k, v, scale, causal, cu_seqlens=None, nthreads=0):
    """O and LSE by the materialised three-pass definition (fp64).

    Returns (o, lse): o shaped like q; lse [B, Hq, N] (dense) or
    [Hq, total] (varlen)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, Hkv, N, d = _dims(q, k, cu_seqlens)
    cu, cup = _cu(cu_seqlens)
    o = np.zeros(q.shape, dtype=np.float64)
    if cu_seqlens is None:
        lse = np.zeros((B, Hq, N), dtype=np.float64)
    else:
        lse = np.zeros((Hq, q.shape[0]), dtype=np.float64)
    rc = _load().oracle_attention_fwd(_dptr(q), _dptr(k), _dptr(v), _dptr(o), _dptr(lse),
                                      B, Hq, Hkv, N, d, float(scale), int(bool(causal)),
                                      cup, int(nthreads))
    if rc != 0:
        raise RuntimeError("oracle_attention_fwd failed: %d" % rc)
    return o, lse


def attention_bwd(q, k, v, dout, scale, causal, cu_seqlens=None, nthreads=0):
    """dQ, dK, dV (plus O, LSE, D as by-products), fp64, from scratch.

    Returns dict with keys dq, dk, dv, o, lse, D."""
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, Hq, Hkv, N, d = _dims(q, k, cu_seqlens)
    cu, cup = _cu(cu_seqlens)
    dq = np.zeros(q.shape, dtype=np.float64)
    dk = np.zeros(k.shape, dtype=np.float64)
    dv = np.zeros(v.shape, dtype=np.float64)
    o = np.zeros(q.shape, dtype=np.float64)
    if cu_seqlens is None:
        lse = np.zeros((B, Hq, N), dtype=np.float64)
    else:
        lse = np.zeros((Hq, q.shape[0]), dtype=np.float64)
    D = np.zeros_like(lse)
    rc = _load().oracle_attention_bwd(_dptr(q), _dptr(k), _dptr(v), _dptr(dout),
                                      _dptr(dq), _dptr(dk), _dptr(dv),
                                      _dptr(o), _dptr(lse), _dptr(D),
                                      B, Hq, Hkv, N, d, float(scale), int(bool(causal)),
                                      cup, int(nthreads))
    if rc != 0:
        raise RuntimeError("oracle_attention_bwd failed: %d" % rc)
    return {"dq": dq, "dk": dk, "dv": dv, "o": o, "lse": lse, "D": D}


def attention_rows(q, k, v, dout, rows, scale, causal, cu_seqlens=None, nthreads=0):
    """O, LSE, D, dQ of selected query rows.

    rows: int array [R, 3] of (sequence, query head, row within sequence).
    dout may be None (then D and dQ are not computed)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    dout = None if dout is None else _f64(dout)
    B, Hq, Hkv, N, d = _dims(q, k, cu_seqlens)
    cu, cup = _cu(cu_seqlens)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
    R = rows.shape[0]
    o = np.zeros((R, d), dtype=np.float64)
    lse = np.zeros((R,), dtype=np.float64)
    D = np.zeros((R,), dtype=np.float64)
    dq = np.zeros((R, d), dtype=np.float64)
    rc = _load().oracle_attention_rows(_dptr(q), _dptr(k), _dptr(v), _dptr(dout),
                                       rows.ctypes.data_as(ctypes.POINTER(ctypes.c_long)), R,
                                       _dptr(o), _dptr(lse), _dptr(D), _dptr(dq),
                                       B, Hq, Hkv, N, d, float(scale), int(bool(causal)),
                                       cup, int(nthreads))
    if rc != 0:
        raise RuntimeError("oracle_attention_rows failed: %d" % rc)
    out = {"o": o, "lse": lse}
    if dout is not None:
        out["D"] = D
        out["dq"] = dq
    return out


def attention_fwd_streaming(q, k, v, scale, causal, tile, tile_order=None):
    """Online-softmax forward of one [n, d] problem (tiles of `tile` keys,
    visited in `tile_order`)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    n, d = q.shape
    o = np.zeros((n, d), dtype=np.float64)
    lse = np.zeros((n,), dtype=np.float64)
    if tile_order is None:
        order_p = ctypes.POINTER(ctypes.c_int)()
        order = None
    else:
        order = np.ascontiguousarray(np.asarray(tile_order, dtype=np.int32))
        order_p = order.ctypes.data_as(ctypes.POINTER(ctypes.c_int))
    rc = _load().oracle_attention_fwd_streaming(_dptr(q), _dptr(k), _dptr(v), _dptr(o),
                                                _dptr(lse), n, d, float(scale),
                                                int(bool(causal)), int(tile), order_p)
    if rc != 0:
        raise RuntimeError("oracle_attention_fwd_streaming failed: %d" % rc)
    return o, lse


def softmax_rows(s, scale, causal, nthreads=0):
    """Row softmax of score matrices s [..., n, n] (raw q.k products): the
    middle step of standard attention.  Row i of each n x n matrix is query
    i; the logits are scale * s, with j > i masked when causal.  Returns
    (p, lse), p shaped like s, lse shaped like s[..., 0]."""
    s = _f64(s)
    n = s.shape[-1]
    if s.ndim < 2 or s.shape[-2] != n:
        raise ValueError("s must be [..., n, n]")
    rows = s.size // n
    p = np.zeros(s.shape, dtype=np.float64)
    lse = np.zeros(s.shape[:-1], dtype=np.float64)
    rc = _load().oracle_softmax_rows(_dptr(s), rows, n, float(scale), int(bool(causal)),
                                     _dptr(p), _dptr(lse), int(nthreads))
    if rc != 0:
        raise RuntimeError("oracle_softmax_rows failed: %d" % rc)
    return p, lse


def _mask(block_mask):
    """uint8 [Bm, Hm, nt, nt] with Bm in {1, B} and Hm in {1, Hkv}: returns
    the array and its (sequence, head) strides in elements (0 broadcasts)."""
    bm = np.ascontiguousarray(np.asarray(block_mask, dtype=np.uint8))
    if bm.ndim != 4 or bm.shape[2] != bm.shape[3]:
        raise ValueError("block mask must be [Bm, Hm, nt, nt]")
    nt = bm.shape[2]
    sb = 0 if bm.shape[0] == 1 else bm.shape[1] * nt * nt
    sh = 0 if bm.shape[1] == 1 else nt * nt
    return bm, sb, sh


def attention_fwd_blockmask(q, k, v, scale, causal, block_mask, nthreads=0):
    """O and LSE of block-sparse attention (dense layout): the definition with
    every (query, key) pair whose 128 x 128 tile is not allowed by the block
    mask of its key/value head removed.  block_mask: [Bm, Hm, nt, nt] with
    nt = ceil(N / 128), Bm in {1, B}, Hm in {1, Hkv} (1 broadcasts)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    bm, sb, sh = _mask(block_mask)
    if bm.shape[2] != (N + 127) // 128 or bm.shape[0] not in (1, B) or bm.shape[1] not in (1, Hkv):
        raise ValueError("block mask shape %s does not fit B=%d Hkv=%d N=%d" % (bm.shape, B, Hkv, N))
    o = np.zeros(q.shape, dtype=np.float64)
    lse = np.zeros((B, Hq, N), dtype=np.float64)
    rc = _load().oracle_attention_fwd_blockmask(
        _dptr(q), _dptr(k), _dptr(v), _dptr(o), _dptr(lse), B, Hq, Hkv, N, d, float(scale),
        int(bool(causal)), bm.ctypes.data_as(ctypes.POINTER(ctypes.c_ubyte)), sb, sh,
        int(nthreads))
    if rc != 0:
        raise RuntimeError("oracle_attention_fwd_blockmask failed: %d" % rc)
    return o, lse


def attention_bwd_blockmask(q, k, v, dout, scale, causal, block_mask, nthreads=0):
    """dQ, dK, dV (plus O, LSE, D) of block-sparse attention; see
    attention_fwd_blockmask."""
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    bm, sb, sh = _mask(block_mask)
    if bm.shape[2] != (N + 127) // 128 or bm.shape[0] not in (1, B) or bm.shape[1] not in (1, Hkv):
        raise ValueError("block mask shape %s does not fit B=%d Hkv=%d N=%d" % (bm.shape, B, Hkv, N))
    dq, dk, dv = (np.zeros(t.shape, dtype=np.float64) for t in (q, k, v))
    o = np.zeros(q.shape, dtype=np.float64)
    lse = np.zeros((B, Hq, N), dtype=np.float64)
    D = np.zeros_like(lse)
    rc = _load().oracle_attention_bwd_blockmask(
        _dptr(q), _dptr(k), _dptr(v), _dptr(dout), _dptr(dq), _dptr(dk), _dptr(dv), _dptr(o),
        _dptr(lse), _dptr(D), B, Hq, Hkv, N, d, float(scale), int(bool(causal)),
        bm.ctypes.data_as(ctypes.POINTER(ctypes.c_ubyte)), sb, sh, int(nthreads))
    if rc != 0:
        raise RuntimeError("oracle_attention_bwd_blockmask failed: %d" % rc)
    return {"dq": dq, "dk": dk, "dv": dv, "o": o, "lse": lse, "D": D}
