"""Helpers for the GPU parity tests: run the CUDA path through the C ABI,
run the oracle on the same seeded bf16 inputs (upcast to fp64), compare.

Tolerances (fixed by the project's acceptance bar): O, dQ, dK, dV max-abs
error <= 2e-2 and mean-abs error <= 2e-3 against the fp64 oracle; LSE
max-abs error <= 1e-3.
"""
import numpy as np
import torch

import oracle
from exact_io_aware_67_b200 import ops

TOL_MAX = 2e-2
TOL_MEAN = 2e-3
TOL_LSE = 1e-3


def f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def to_dev(inp):
    dev = {}
    for nm in ("q", "k", "v", "dout"):
        t = getattr(inp, nm)
        dev[nm] = None if t is None else t.cuda().contiguous()
    dev["cu"] = None if inp.cu_seqlens is None else inp.cu_seqlens.cuda()
    return dev


def max_seqlen(inp):
    w = inp.workload
    if inp.cu_seqlens is None:
        return w.N
    return max(inp.lengths) if inp.lengths else 1


def gpu_fwd(inp, dev=None):
    dev = dev or to_dev(inp)
    w = inp.workload
    o, lse = ops.attention_fwd(dev["q"], dev["k"], dev["v"], w.scale, w.causal, dev["cu"],
                               max_seqlen(inp) if dev["cu"] is not None else None)
    torch.cuda.synchronize()
    return o, lse


def gpu_bwd(inp, o, lse, dev=None):
    dev = dev or to_dev(inp)
    w = inp.workload
    dq, dk, dv = ops.attention_bwd(dev["q"], dev["k"], dev["v"], o, lse, dev["dout"], w.scale,
                                   w.causal, dev["cu"],
                                   max_seqlen(inp) if dev["cu"] is not None else None)
    torch.cuda.synchronize()
    return dq, dk, dv


def oracle_fwd(inp):
    w = inp.workload
    return oracle.attention_fwd(f64(inp.q), f64(inp.k), f64(inp.v), w.scale, w.causal,
                                None if inp.cu_seqlens is None else inp.cu_seqlens.numpy())


def oracle_bwd(inp):
    w = inp.workload
    return oracle.attention_bwd(f64(inp.q), f64(inp.k), f64(inp.v), f64(inp.dout), w.scale,
                                w.causal,
                                None if inp.cu_seqlens is None else inp.cu_seqlens.numpy())


def errors(got, ref):
    d = np.abs(np.asarray(got, dtype=np.float64) - np.asarray(ref, dtype=np.float64))
    if d.size == 0:
        return 0.0, 0.0
    return float(d.max()), float(d.mean())


def assert_close(name, got, ref, tol_max=TOL_MAX, tol_mean=TOL_MEAN):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), "%s has non-finite values" % name
    mx, mn = errors(got, ref)
    assert mx <= tol_max, "%s max-abs error %.3e > %.1e (mean %.3e)" % (name, mx, tol_max, mn)
    if tol_mean is not None:
        assert mn <= tol_mean, "%s mean-abs error %.3e > %.1e" % (name, mn, tol_mean)
    return mx, mn


def bf16_floor(ref):
    """Max error of rounding the fp64 reference itself to bf16: the best any
    bf16 output can do."""
    r = torch.from_numpy(np.ascontiguousarray(ref, dtype=np.float64))
    return float((r - r.to(torch.bfloat16).double()).abs().max()) if r.numel() else 0.0


def check_fwd(inp, o, lse, ref=None):
    ref_o, ref_lse = ref if ref is not None else oracle_fwd(inp)
    eo = assert_close("O", f64(o), ref_o)
    el = assert_close("LSE", f64(lse), ref_lse, tol_max=TOL_LSE, tol_mean=None)
    return eo, el


def no_device_error():
    err = ops.fa_device_error()
    assert err == 0, "device error word 0x%x" % err
