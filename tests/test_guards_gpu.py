"""Out-of-bounds protection: guard bands around every output, and a corrupt
cu_seqlens (GPU).

Each output is written in place into the middle of a larger buffer whose
two guard bands hold a canary pattern; after the call the bands must be
untouched.  A corrupt cu_seqlens (not starting at 0, decreasing, past the
allocation, a sequence longer than N) must leave every access inside the
caller's buffers -- the kernels clamp the ranges they derive from it -- and
fa_validate_cu_seqlens must name the broken rule.  The corrupt values stay
within a few hundred rows of the real ones and the guard bands are
thousands of rows wide, so even a missing clamp would land in a band (and
be caught) rather than outside the allocation.
"""
import ctypes

import numpy as np
import pytest
import torch

from exact_io_aware_67_b200 import ops, workloads
import parity

pytestmark = pytest.mark.gpu

PAD_ROWS = 4096


def _banded(shape, fill, dtype):
    """A view of `shape` inside a buffer with PAD_ROWS rows of `fill` on both
    sides (rows along dim 0)."""
    row = int(np.prod(shape[1:])) if len(shape) > 1 else 1
    buf = torch.full((shape[0] + 2 * PAD_ROWS,) + tuple(shape[1:]), fill, dtype=dtype,
                     device="cuda")
    return buf, buf[PAD_ROWS:PAD_ROWS + shape[0]]


def _bands_intact(buf, fill):
    return bool((buf[:PAD_ROWS] == fill).all()) and bool((buf[-PAD_ROWS:] == fill).all())


def _run_banded(dev, inp, cu, N, total):
    w = inp.workload
    Hq, Hkv, d = w.Hq, w.Hkv, w.d
    bufs = {}
    bufs["o"], o = _banded((total, Hq, d), 7.0, torch.bfloat16)
    bufs["o_lo"], o_lo = _banded((total, Hq, d), 5.0, torch.bfloat16)
    bufs["lse"], lse = _banded((Hq, total), -3.0, torch.float32)
    bufs["dq"], dq = _banded((total, Hq, d), 9.0, torch.bfloat16)
    bufs["dk"], dk = _banded((total, Hkv, d), 11.0, torch.bfloat16)
    bufs["dv"], dv = _banded((total, Hkv, d), 13.0, torch.bfloat16)
    ops.attention_fwd(dev["q"], dev["k"], dev["v"], w.scale, w.causal, cu, N, out=o, lse=lse,
                      o_lo=o_lo)
    ops.attention_bwd(dev["q"], dev["k"], dev["v"], o, lse, dev["dout"], w.scale, w.causal, cu,
                      N, dq=dq, dk=dk, dv=dv, o_lo=o_lo)
    torch.cuda.synchronize()
    fills = {"o": 7.0, "o_lo": 5.0, "lse": -3.0, "dq": 9.0, "dk": 11.0, "dv": 13.0}
    for nm, buf in bufs.items():
        assert _bands_intact(buf, fills[nm]), "%s: a guard band was overwritten" % nm
    return o, lse, dq, dk, dv


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
def test_fwd_bwd_guard_bands_varlen(causal, d):
    inp = workloads.from_lengths("guard", [5, 200, 1, 333, 128], 4, 2, d, causal)
    dev = parity.to_dev(inp)
    total = inp.q.shape[0]
    o, lse, dq, dk, dv = _run_banded(dev, inp, dev["cu"], 333, total)
    parity.no_device_error()
    parity.check_fwd(inp, o, lse)
    ref = parity.oracle_bwd(inp)
    for nm, t in (("dQ", dq), ("dK", dk), ("dV", dv)):
        parity.assert_close(nm, parity.f64(t), ref[nm.lower()])


def test_bwd_guard_bands_dense():
    inp = workloads.generate(workloads.custom("gd", 2, 4, 2, 300, 128, True))
    dev = parity.to_dev(inp)
    w = inp.workload
    o, lse = parity.gpu_fwd(inp, dev)
    bq, dq = _banded(tuple(dev["q"].shape), 9.0, torch.bfloat16)
    bk, dk = _banded(tuple(dev["k"].shape), 11.0, torch.bfloat16)
    bv, dv = _banded(tuple(dev["v"].shape), 13.0, torch.bfloat16)
    ops.attention_bwd(dev["q"], dev["k"], dev["v"], o, lse, dev["dout"], w.scale, True,
                      dq=dq, dk=dk, dv=dv, o_lo=dev["o_lo"])
    torch.cuda.synchronize()
    parity.no_device_error()
    assert _bands_intact(bq, 9.0) and _bands_intact(bk, 11.0) and _bands_intact(bv, 13.0)
    ref = parity.oracle_bwd(inp)
    parity.assert_close("dK", parity.f64(dk), ref["dk"])


def test_decode_guard_bands():
    B, Hq, Hkv, L, d = 3, 8, 2, 700, 128
    rng = torch.Generator().manual_seed(5)
    q = torch.randn(B, Hq, d, generator=rng).to(torch.bfloat16).cuda()
    kc = torch.randn(B, L, Hkv, d, generator=rng).to(torch.bfloat16).cuda()
    vc = torch.randn(B, L, Hkv, d, generator=rng).to(torch.bfloat16).cuda()
    lens = torch.tensor([700, 1, 333], dtype=torch.int32).cuda()
    bo, o = _banded((B, Hq, d), 7.0, torch.bfloat16)
    bl, lse = _banded((B, Hq), -3.0, torch.float32)
    ops.decode(q, kc, vc, lens, out=o, lse=lse)
    torch.cuda.synchronize()
    parity.no_device_error()
    assert _bands_intact(bo, 7.0) and _bands_intact(bl, -3.0)
    assert bool(torch.isfinite(o.float()).all())


def _validate(cu_list, B, N, total):
    cu = torch.tensor(cu_list, dtype=torch.int32).cuda()
    ops.fa_clear_device_error()
    st = ops.fa_validate_cu_seqlens(ctypes.c_void_p(cu.data_ptr()), B, N, total, ops._stream())
    assert st == 0, ops.fa_status_string(st)
    torch.cuda.synchronize()
    code = ops.fa_device_error()
    ops.fa_clear_device_error()
    return code


def test_validate_cu_seqlens_codes():
    assert _validate([0, 5, 205, 206, 539], 4, 333, 539) == 0
    assert _validate([0], 0, 1, 0) == 0                       # no sequences
    assert _validate([3, 5, 205, 206, 539], 4, 333, 539) == 0x501
    assert _validate([0, 205, 100, 539], 3, 333, 539) == 0x502
    assert _validate([0, 5, 405, 539], 3, 333, 539) == 0x503
    assert _validate([0, 5, 205, 600], 3, 400, 539) == 0x504
    # the lowest failing rule is reported
    assert _validate([1, 205, 100, 900], 3, 333, 539) == 0x501


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("cu_bad", [
    [0, 205, 100, 839],          # decreasing, last offset 300 rows past the allocation
    [-50, 5, 205, 206, 700],     # negative start, end past the allocation
    [0, 5, 500, 501, 539],       # a sequence longer than the stated N
])
def test_corrupt_cu_seqlens_stays_in_bounds(causal, cu_bad):
    inp = workloads.from_lengths("corrupt", [5, 200, 1, 333], 4, 2, 128, causal)
    dev = parity.to_dev(inp)
    total = inp.q.shape[0]                     # 539
    cu = torch.tensor(cu_bad, dtype=torch.int32).cuda()
    ops.fa_clear_device_error()
    _run_banded(dev, inp, cu, 333, total)
    parity.no_device_error()
    B = len(cu_bad) - 1
    st = ops.fa_validate_cu_seqlens(ctypes.c_void_p(cu.data_ptr()), B, 333, total, ops._stream())
    assert st == 0
    torch.cuda.synchronize()
    assert ops.fa_device_error() != 0
    ops.fa_clear_device_error()
