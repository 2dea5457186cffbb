"""Block-sparse attention (fa_fwd_blockmask, fa_bwd_blockmask) against the
oracle's block-mask definition, on the same seeded inputs, at the project's
tolerances.  The cases cover random masks of per-(sequence, kv head) tiles,
GQA groups sharing their kv head's mask, causal and not, d = 64 and 128, a
ragged last tile, query rows left with no key, K/V tiles met by no query
tile, and CTAs whose whole tile list is empty."""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_67_b200 import ops, workloads
import parity

pytestmark = pytest.mark.gpu


def _mask(Bm, Hm, nt, density, seed, diag=None):
    rng = np.random.default_rng(seed)
    m = (rng.random((Bm, Hm, nt, nt)) < density).astype(np.uint8)
    if diag is not None:
        m[:, :, np.arange(nt), np.arange(nt)] = diag
    return m


def _run(inp, bm, causal):
    w = inp.workload
    dev = parity.to_dev(inp)
    bmd = torch.from_numpy(bm).cuda()
    o_lo = torch.empty_like(dev["q"])
    o, lse = ops.attention_fwd_blockmask(dev["q"], dev["k"], dev["v"], bmd, w.scale, causal,
                                         o_lo=o_lo)
    dq, dk, dv = ops.attention_bwd_blockmask(dev["q"], dev["k"], dev["v"], o, lse, dev["dout"],
                                             bmd, w.scale, causal, o_lo=o_lo)
    torch.cuda.synchronize()
    parity.no_device_error()
    return o, lse, dq, dk, dv


def _check(inp, bm, causal, outs):
    w = inp.workload
    o, lse, dq, dk, dv = outs
    f = lambda t: t.double().numpy()
    ref = oracle.attention_bwd_blockmask(f(inp.q), f(inp.k), f(inp.v), f(inp.dout), w.scale,
                                         causal, bm)
    got_lse = parity.f64(lse)
    empty = np.isneginf(ref["lse"])
    assert np.array_equal(np.isneginf(got_lse), empty), "rows without keys differ"
    got_o = parity.f64(o)
    # rows without keys: O = 0 and dQ = 0 exactly
    e_rows = np.transpose(empty, (0, 2, 1))           # [B, N, Hq]
    assert np.all(got_o[e_rows] == 0.0)
    assert np.all(parity.f64(dq)[e_rows] == 0.0)
    parity.assert_close("O", got_o, ref["o"])
    parity.assert_close("LSE", got_lse[~empty], ref["lse"][~empty], tol_max=parity.TOL_LSE,
                        tol_mean=None, bf16_out=False)
    parity.assert_close("dQ", parity.f64(dq), ref["dq"])
    parity.assert_close("dK", parity.f64(dk), ref["dk"])
    parity.assert_close("dV", parity.f64(dv), ref["dv"])


@pytest.mark.parametrize("B,Hq,Hkv,N,d,causal,density,per_head", [
    (1, 2, 2, 600, 64, False, 0.5, True),     # ragged last tile, per-head masks
    (2, 4, 2, 640, 128, True, 0.6, True),     # GQA: the group shares its kv head's mask
    (2, 8, 2, 1024, 64, True, 0.4, False),    # one mask for every head of a sequence
    (1, 4, 1, 900, 128, False, 0.3, True),    # sparse: rows and K/V tiles without partners
])
def test_blockmask_matches_oracle(B, Hq, Hkv, N, d, causal, density, per_head):
    inp = workloads.generate(workloads.custom("bm", B, Hq, Hkv, N, d, causal, seed=N + d))
    nt = (N + 127) // 128
    bm = _mask(B, Hkv if per_head else 1, nt, density, seed=N)
    _check(inp, bm, causal, _run(inp, bm, causal))


def test_blockmask_all_allowed_equals_dense():
    inp = workloads.generate(workloads.custom("bm1", 2, 4, 2, 700, 128, False, seed=3))
    nt = (700 + 127) // 128
    bm = np.ones((1, 1, nt, nt), dtype=np.uint8)
    o, lse, dq, dk, dv = _run(inp, bm, False)
    dev = parity.to_dev(inp)
    o2, lse2 = parity.gpu_fwd(inp, dev)
    dq2, dk2, dv2 = parity.gpu_bwd(inp, o2, lse2, dev)
    assert torch.equal(o, o2) and torch.equal(lse, lse2)
    assert torch.equal(dk, dk2) and torch.equal(dv, dv2)
    parity.assert_close("dQ vs dense", parity.f64(dq), parity.f64(dq2), tol_max=1e-2,
                        tol_mean=1e-4)


def test_blockmask_empty_lists():
    # query tiles 2-3 (one forward CTA) see nothing; K/V tile 4 is met by no
    # query tile; everything else allowed
    N, nt = 640, 5
    inp = workloads.generate(workloads.custom("bm2", 1, 2, 1, N, 64, False, seed=4))
    bm = np.ones((1, 1, nt, nt), dtype=np.uint8)
    bm[0, 0, 2:4, :] = 0
    bm[0, 0, :, 4] = 0
    outs = _run(inp, bm, False)
    _check(inp, bm, False, outs)
    o, lse, dq, dk, dv = outs
    assert torch.all(dk[:, 512:] == 0) and torch.all(dv[:, 512:] == 0)


def test_blockmask_band_long_sequence():
    # a causal band of 4 tiles (sliding window of 512 keys) at N = 4096: every
    # output against the oracle on the first and last query heads' rows is
    # covered by the full check of a small head count
    N, nt = 4096, 32
    inp = workloads.generate(workloads.custom("band", 1, 2, 1, N, 128, True, seed=6))
    i = np.arange(nt)
    bm = ((i[:, None] - i[None, :] >= 0) & (i[:, None] - i[None, :] < 4)).astype(np.uint8)
    bm = bm[None, None]
    _check(inp, bm, True, _run(inp, bm, True))


@pytest.mark.parametrize("name", sorted(workloads.BLOCKSPARSE_WORKLOADS))
def test_blocksparse_workloads_first_group(name):
    # the benchmark's block-sparse workloads at full size; the oracle checks
    # every output of kv head 0's query heads (and kv head 0's dK, dV)
    bw = workloads.BLOCKSPARSE_WORKLOADS[name]
    w = bw.base
    inp = workloads.generate(w)
    bm = workloads.block_mask(bw)
    o, lse, dq, dk, dv = _run(inp, bm, w.causal)
    g = w.Hq // w.Hkv
    f = lambda t: t.double().numpy()
    sub = lambda t, n: np.ascontiguousarray(f(t)[:, :, :n])
    ref = oracle.attention_bwd_blockmask(sub(inp.q, g), sub(inp.k, 1), sub(inp.v, 1),
                                         sub(inp.dout, g), w.scale, w.causal, bm[:, :1])
    parity.assert_close("O", parity.f64(o[:, :, :g]), ref["o"])
    parity.assert_close("LSE", parity.f64(lse[:, :g]), ref["lse"], tol_max=parity.TOL_LSE,
                        tol_mean=None, bf16_out=False)
    parity.assert_close("dQ", parity.f64(dq[:, :, :g]), ref["dq"])
    parity.assert_close("dK", parity.f64(dk[:, :, :1]), ref["dk"])
    parity.assert_close("dV", parity.f64(dv[:, :, :1]), ref["dv"])
