"""Backward parity: dQ, dK, dV from the CUDA path (fa_fwd then fa_bwd through
the C ABI) vs the fp64 oracle's from-scratch gradients on the same seeded
bf16 inputs; plus gradient invariants checked on the GPU outputs and the
autograd wrapper."""
import numpy as np
import pytest
import torch

from exact_io_aware_67_b200 import ops, workloads
import parity

pytestmark = pytest.mark.gpu

CASES = [
    ("c1", lambda: workloads.WORKLOADS["single_head_n128_d64"]),
    ("n512_d128", lambda: workloads.custom("n512_d128", 1, 2, 2, 512, 128, False)),
    ("n512_d128_causal", lambda: workloads.custom("n512_d128_c", 1, 2, 2, 512, 128, True)),
    ("n300_d64_causal", lambda: workloads.custom("n300_d64_c", 2, 3, 3, 300, 64, True)),
    ("n300_d128", lambda: workloads.custom("n300_d128", 2, 3, 3, 300, 128, False)),
    ("n1_d64", lambda: workloads.custom("n1_d64", 2, 2, 1, 1, 64, True)),
    ("n1_d128", lambda: workloads.custom("n1_d128", 1, 1, 1, 1, 128, False)),
    ("n129_d128_causal", lambda: workloads.custom("n129", 1, 2, 2, 129, 128, True)),
    ("gqa4_n384_d128_causal", lambda: workloads.custom("gqa", 2, 8, 2, 384, 128, True)),
    ("gqa8_n640_d64", lambda: workloads.custom("gqa8", 1, 8, 1, 640, 64, False)),
    ("x8row_n1024_d128", lambda: workloads.custom("x8", 1, 4, 4, 1024, 128, True, x8_row=True)),
]


def _check_grads(inp, dq, dk, dv, ref=None):
    g = ref if ref is not None else parity.oracle_bwd(inp)
    out = {}
    for nm, t in (("dQ", dq), ("dK", dk), ("dV", dv)):
        out[nm] = parity.assert_close(nm, parity.f64(t), g[nm.lower()])
    return out


def _run(inp):
    dev = parity.to_dev(inp)
    o, lse = parity.gpu_fwd(inp, dev)
    dq, dk, dv = parity.gpu_bwd(inp, o, lse, dev)
    parity.no_device_error()
    return o, lse, dq, dk, dv


@pytest.mark.parametrize("name,mk", CASES, ids=[c[0] for c in CASES])
def test_bwd_matches_oracle(name, mk):
    inp = workloads.generate(mk())
    ops.fa_clear_device_error()
    o, lse, dq, dk, dv = _run(inp)
    _check_grads(inp, dq, dk, dv)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_bwd_varlen_edge_lengths(d, causal):
    inp = workloads.from_lengths("vl", [1, 129, 300, 0, 517, 128, 64, 255, 256, 257], 4, 2, d,
                                 causal)
    o, lse, dq, dk, dv = _run(inp)
    _check_grads(inp, dq, dk, dv)


@pytest.mark.parametrize("wname", ["gpt2_small_causal_b8_h12_n1024_d64",
                                   "bert_large_varlen_32x128to512_h16_d64"])
def test_bwd_full_config(wname):
    inp = workloads.generate(workloads.WORKLOADS[wname])
    o, lse, dq, dk, dv = _run(inp)
    _check_grads(inp, dq, dk, dv)


def test_o_residual_is_the_rounding_error_of_o():
    """The forward's optional second output is O's bf16 rounding residual:
    at most half a bf16 spacing of o, and o + o_lo is at least as close to
    the oracle's O as o alone (the rest is the bf16 rounding of P in P V)."""
    inp = workloads.generate(workloads.custom("res", 1, 4, 4, 1024, 128, True, x8_row=True))
    dev = parity.to_dev(inp)
    o, lse = parity.gpu_fwd(inp, dev)
    parity.no_device_error()
    of, lof = o.float(), dev["o_lo"].float()
    assert bool((lof.abs() <= of.abs() * 2.0 ** -8).all())
    ref_o, _ = parity.oracle_fwd(inp)
    e_hi = np.abs(parity.f64(o) - ref_o)
    e_sum = np.abs(parity.f64(o) + parity.f64(dev["o_lo"]) - ref_o)
    assert e_sum.max() <= e_hi.max() and e_sum.mean() < e_hi.mean()
    # without the residual the backward still runs (D from bf16 O alone)
    dq, dk, dv = ops.attention_bwd(dev["q"], dev["k"], dev["v"], o, lse, dev["dout"],
                                   inp.workload.scale, True)
    torch.cuda.synchronize()
    parity.no_device_error()
    g = parity.oracle_bwd(inp)
    parity.assert_close("dV without residual", parity.f64(dv), g["dv"])


def test_bwd_invariants_on_gpu_outputs():
    """sum_j dK_j = 0 and sum_j dV_j = sum over the group of sum_i dO_i hold
    for the GPU's gradients up to bf16 rounding."""
    w = workloads.custom("inv", 2, 8, 2, 700, 128, True)
    inp = workloads.generate(w)
    o, lse, dq, dk, dv = _run(inp)
    dk64, dv64 = parity.f64(dk), parity.f64(dv)
    do64 = parity.f64(inp.dout)
    sk = dk64.sum(axis=1)
    assert np.abs(sk).max() <= 0.05 * np.abs(dk64).max() * np.sqrt(700) / 10
    grp = do64.reshape(2, 700, 2, 4, 128).sum(axis=(1, 3))
    np.testing.assert_allclose(dv64.sum(axis=1), grp, atol=0.5)


def test_dk_dv_deterministic():
    inp = workloads.generate(workloads.custom("det", 1, 4, 2, 640, 64, True))
    dev = parity.to_dev(inp)
    o, lse = parity.gpu_fwd(inp, dev)
    a = parity.gpu_bwd(inp, o, lse, dev)
    b = parity.gpu_bwd(inp, o, lse, dev)
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])
    # dQ is summed by fp32 atomics: any difference stays far below bf16 ulp
    assert float((a[0].float() - b[0].float()).abs().max()) <= 2e-2


def test_autograd_wrapper():
    inp = workloads.generate(workloads.custom("ag", 1, 4, 4, 256, 64, True))
    q = inp.q.cuda().requires_grad_(True)
    k = inp.k.cuda().requires_grad_(True)
    v = inp.v.cuda().requires_grad_(True)
    o = ops.attention(q, k, v, causal=True)
    o.backward(inp.dout.cuda())
    g = parity.oracle_bwd(inp)
    parity.assert_close("O", parity.f64(o), g["o"])
    parity.assert_close("dQ", parity.f64(q.grad), g["dq"])
    parity.assert_close("dK", parity.f64(k.grad), g["dk"])
    parity.assert_close("dV", parity.f64(v.grad), g["dv"])


def test_calls_from_another_host_thread():
    """The C entry points work from a thread other than the one that first
    touched the device (autograd runs backward on its own thread)."""
    import threading
    inp = workloads.generate(workloads.custom("thr", 1, 2, 2, 256, 64, True))
    dev = parity.to_dev(inp)
    o, lse = parity.gpu_fwd(inp, dev)
    box = {}

    def work():
        try:
            box["g"] = parity.gpu_bwd(inp, o, lse, dev)
        except Exception as e:  # reported below
            box["e"] = e

    th = threading.Thread(target=work)
    th.start()
    th.join()
    assert "e" not in box, box.get("e")
    g = parity.oracle_bwd(inp)
    parity.assert_close("dQ", parity.f64(box["g"][0]), g["dq"])


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_x8_key_row_relative(d, causal):
    """One key row per (batch, kv head) scaled by 8 draws weight from about
    half the query rows, so dV and dK on that row reach magnitudes where
    bf16 rounding alone exceeds the absolute bar; such a case is judged by
    relative error: every output within 1e-2 of its largest oracle
    magnitude, and the mean error within 1e-3 of it."""
    inp = workloads.generate(workloads.custom("x8k", 1, 4, 2, 1024, d, causal, x8_key_row=True))
    ops.fa_clear_device_error()
    o, lse, dq, dk, dv = _run(inp)
    g = parity.oracle_bwd(inp)
    # the scaled rows carry the largest dV entries, as the case intends
    kr = inp.x8_key_rows.numpy()
    dv_ref = np.abs(g["dv"])
    assert all(dv_ref[0, kr[0, h], h].max() >= 0.5 * dv_ref[0, :, h].max() for h in range(2))
    for nm, got, ref in (("O", o, g["o"]), ("dQ", dq, g["dq"]), ("dK", dk, g["dk"]),
                         ("dV", dv, g["dv"])):
        err = np.abs(parity.f64(got) - ref)
        scale = np.abs(ref).max()
        assert err.max() <= 1e-2 * scale, "%s: max error %.3e, max |ref| %.3e" % (
            nm, err.max(), scale)
        assert err.mean() <= 1e-3 * scale, "%s: mean error %.3e" % (nm, err.mean())
    np.testing.assert_allclose(parity.f64(lse), g["lse"], atol=parity.TOL_LSE, rtol=0)
