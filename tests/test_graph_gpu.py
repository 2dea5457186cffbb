"""The forward and backward launch path inside a CUDA graph.

A captured fa_fwd + fa_bwd step must replay with the results of the same
calls made eagerly, and must pick up new input values written into the
captured buffers.  This holds because the library makes no host
synchronisation, no allocation and no device-to-host read on the launch
path: launch parameters come from the host arguments, variable-length
boundaries stay on the device (cu_seqlens), and the workspace is the
caller's.  The one-time set-up (the driver entry point for tensor-map
encoding, the kernels' shared-memory attribute) happens in the eager warm-up
call, as is usual before a capture.
"""
import pytest
import torch

from exact_io_aware_67_b200 import ops, workloads
import parity

pytestmark = pytest.mark.gpu


def _inputs(varlen, seed):
    if varlen:
        return workloads.from_lengths("graph", [300, 1, 517, 128], 8, 2, 128, True, seed=seed)
    return workloads.generate(workloads.custom("graph", 2, 8, 2, 640, 64, True, seed=seed))


def _step(dev, inp, ws):
    w = inp.workload
    ms = parity.max_seqlen(inp) if dev["cu"] is not None else None
    o_lo = torch.empty_like(dev["q"])
    o, lse = ops.attention_fwd(dev["q"], dev["k"], dev["v"], w.scale, w.causal, dev["cu"], ms,
                               o_lo=o_lo)
    dq, dk, dv = ops.attention_bwd(dev["q"], dev["k"], dev["v"], o, lse, dev["dout"], w.scale,
                                   w.causal, dev["cu"], ms, workspace=ws, o_lo=o_lo)
    return o, lse, dq, dk, dv


@pytest.mark.parametrize("varlen", [False, True])
def test_captured_step_replays_eager_results_and_new_inputs(varlen):
    inp = _inputs(varlen, seed=0)
    dev = parity.to_dev(inp)
    ms = parity.max_seqlen(inp) if dev["cu"] is not None else None
    ws = ops.workspace_for(dev["q"], dev["k"], dev["cu"], ms)

    eager = _step(dev, inp, ws)           # warm-up, outside the capture
    torch.cuda.synchronize()
    eager = [t.clone() for t in eager]

    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(g):
            out = _step(dev, inp, ws)
    torch.cuda.current_stream().wait_stream(side)

    g.replay()
    torch.cuda.synchronize()
    parity.no_device_error()
    names = ("O", "LSE", "dQ", "dK", "dV")
    for nm, a, b in zip(names, out, eager):
        if nm == "dQ":
            # dQ is reduced with fp32 atomics in no fixed order
            parity.assert_close("replayed dQ", parity.f64(a), parity.f64(b), tol_max=1e-2,
                                tol_mean=1e-4)
        else:
            assert torch.equal(a, b), "replayed %s differs from the eager call" % nm

    # new values in the captured input buffers; the replay must use them
    inp2 = _inputs(varlen, seed=1)
    for nm in ("q", "k", "v", "dout"):
        dev[nm].copy_(getattr(inp2, nm))
    g.replay()
    torch.cuda.synchronize()
    parity.no_device_error()
    o, lse, dq, dk, dv = out
    parity.check_fwd(inp2, o, lse)
    ref = parity.oracle_bwd(inp2)
    parity.assert_close("dQ", parity.f64(dq), ref["dq"])
    parity.assert_close("dK", parity.f64(dk), ref["dk"])
    parity.assert_close("dV", parity.f64(dv), ref["dv"])
    del g
