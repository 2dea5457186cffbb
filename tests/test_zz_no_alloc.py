"""fa_bwd_noalloc: the backward for callers that cannot allocate device
memory at call time (a strict memory pool, a no-cudaMalloc hot path).  It
runs the same kernels as fa_bwd with the library's fixed scratch array as
workspace.

This file is named to be collected last, so that a run that stops at its
first failure has already run every other test; it passes both alone in a
fresh process and after the rest of the suite.
"""
import ctypes

import pytest
import torch

from exact_io_aware_67_b200 import ops, workloads
import parity


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def test_noalloc_rejects_problems_beyond_capacity():
    # host-side check, no device work: B=64, Hq=64, N=4096, d=128 needs far
    # more than the fixed scratch
    need = ops.fa_bwd_workspace_size(64, 64, 4096, 128, 64 * 4096)
    assert need > ops.FA_BWD_NOALLOC_SCRATCH_BYTES
    fake = ctypes.c_void_p(4096)
    st = ops.fa_bwd_noalloc(*([fake] * 5), None, *([fake] * 4), 64, 64, 64, 4096, 128, 0.088, 1,
                            None, 0, None)
    assert st == 3   # FA_ERR_WORKSPACE


@pytest.mark.gpu
@pytest.mark.parametrize("varlen", [False, True])
def test_noalloc_matches_workspace_entry_point_twice(varlen):
    if varlen:
        inp = workloads.from_lengths("na", [300, 1, 517, 128], 8, 2, 128, True)
        B, N, total = 4, 517, inp.q.shape[0]
    else:
        inp = workloads.generate(workloads.custom("na", 2, 8, 2, 640, 64, True))
        B, N, total = 2, 640, 2 * 640
    w = inp.workload
    assert ops.fa_bwd_workspace_size(B, w.Hq, N, w.d, total) <= ops.FA_BWD_NOALLOC_SCRATCH_BYTES
    dev = parity.to_dev(inp)
    o, lse = parity.gpu_fwd(inp, dev)
    ref_dq, ref_dk, ref_dv = parity.gpu_bwd(inp, o, lse, dev)
    stream = ops._stream()
    for call in range(2):
        dq = torch.full_like(dev["q"], float("nan"))
        dk = torch.full_like(dev["k"], float("nan"))
        dv = torch.full_like(dev["v"], float("nan"))
        st = ops.fa_bwd_noalloc(_p(dev["q"]), _p(dev["k"]), _p(dev["v"]), _p(o), _p(lse),
                                _p(dev["o_lo"]), _p(dev["dout"]), _p(dq), _p(dk), _p(dv), B, w.Hq,
                                w.Hkv, N, w.d, w.scale, w.causal, _p(dev["cu"]), total, stream)
        assert st == 0, ops.fa_status_string(st)
        torch.cuda.synchronize()
        parity.no_device_error()
        for nm, got, ref in (("dQ", dq, ref_dq), ("dK", dk, ref_dk), ("dV", dv, ref_dv)):
            parity.assert_close("%s (call %d)" % (nm, call + 1), parity.f64(got), parity.f64(ref))
