"""Parity at the full sizes of the benchmark workloads, in the launch
configuration the benchmark times (dense layout, default wait limit).

The oracle cannot afford every element at these sizes, so each workload is
checked four ways:
  * whole key/value groups (all their query heads) element by element where
    the fp64 oracle finishes in seconds or tens of seconds (N = 4096, and
    heads 0 and 15 at N = 16384);
  * sampled query rows on every head -- O, LSE and dQ of a row depend only
    on that row, so the oracle computes them one by one (O(N d) per row);
    the rows scaled by 8 are always in the sample;
  * sampled key rows on every key/value head -- dK and dV of a key row
    depend on every query row's LSE and D, so the oracle's column sampler
    computes those row statistics by the definition and then the sampled
    columns; the sample always holds the first and last key rows, keys in
    the diagonal tile of each x8 query row and the keys that row weighs most;
  * gradient invariants on every head: sum_j dK_j = 0 (each row of dS sums
    to 0) and sum_j dV_j = sum over the group of sum_i dO_i (each row of P
    sums to 1), up to the bf16 rounding of the outputs.
"""
import concurrent.futures as cf

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_67_b200 import workloads
import parity

pytestmark = pytest.mark.gpu


def _run_gpu(inp):
    dev = parity.to_dev(inp)
    o, lse = parity.gpu_fwd(inp, dev)
    dq, dk, dv = parity.gpu_bwd(inp, o, lse, dev)
    parity.no_device_error()
    return o, lse, dq, dk, dv


def _head(t, b, h):
    """[N, 1, 1, d] fp64 slice of a dense [B, N, H, d] tensor."""
    return t[b:b + 1, :, h:h + 1].float().numpy().astype(np.float64)


def _group_reference(inp, b, hk):
    """Oracle O, LSE, dQ of the group's query heads and dK, dV of the kv
    head, one single-head oracle call per query head, run concurrently; dK
    and dV are the sums of the per-head contributions."""
    w = inp.workload
    g = w.Hq // w.Hkv
    heads = list(range(hk * g, (hk + 1) * g))
    k, v = _head(inp.k, b, hk), _head(inp.v, b, hk)

    # one head per pool thread; a lone head gets all the oracle's threads
    nth = 1 if len(heads) > 1 else 0

    def one(h):
        return oracle.attention_bwd(_head(inp.q, b, h), k, v, _head(inp.dout, b, h), w.scale,
                                    w.causal, nthreads=nth)

    with cf.ThreadPoolExecutor(len(heads)) as ex:
        res = list(ex.map(one, heads))
    return heads, res


def _check_group(inp, outs, b, hk, dk_tol):
    o, lse, dq, dk, dv = outs
    heads, res = _group_reference(inp, b, hk)
    for h, r in zip(heads, res):
        parity.assert_close("O b%d h%d" % (b, h), parity.f64(o[b, :, h]), r["o"][0, :, 0])
        parity.assert_close("LSE b%d h%d" % (b, h), parity.f64(lse[b, h]), r["lse"][0, 0],
                            tol_max=parity.TOL_LSE, tol_mean=None, bf16_out=False)
        parity.assert_close("dQ b%d h%d" % (b, h), parity.f64(dq[b, :, h]), r["dq"][0, :, 0])
    ref_dk = sum(r["dk"][0, :, 0] for r in res)
    ref_dv = sum(r["dv"][0, :, 0] for r in res)
    parity.assert_close("dK b%d kv%d" % (b, hk), parity.f64(dk[b, :, hk]), ref_dk, tol_max=dk_tol)
    parity.assert_close("dV b%d kv%d" % (b, hk), parity.f64(dv[b, :, hk]), ref_dv)


# seeded query rows per head checked through the oracle's row sampler (on
# top of the first and last rows and the x8 row)
ROWS_PER_HEAD = 256


def _check_rows(inp, outs, nrows, seed=0):
    """O, LSE, dQ of sampled rows on every head (plus every x8 row)."""
    o, lse, dq, dk, dv = outs
    w = inp.workload
    rng = np.random.default_rng(seed)
    g = w.Hq // w.Hkv
    for b in range(w.B):
        for hk in range(w.Hkv):
            k, v = _head(inp.k, b, hk), _head(inp.v, b, hk)
            for h in range(hk * g, (hk + 1) * g):
                rows = set(int(x) for x in rng.integers(0, w.N, nrows))
                rows |= {0, w.N - 1}
                if inp.x8_rows is not None:
                    rows.add(int(inp.x8_rows[b, h]))
                rows = sorted(rows)
                sel = np.array([[0, 0, i] for i in rows])
                ref = oracle.attention_rows(_head(inp.q, b, h), k, v, _head(inp.dout, b, h), sel,
                                            w.scale, w.causal)
                parity.assert_close("O rows b%d h%d" % (b, h), parity.f64(o[b, rows, h]), ref["o"])
                parity.assert_close("LSE rows b%d h%d" % (b, h), parity.f64(lse[b, h, rows]),
                                    ref["lse"], tol_max=parity.TOL_LSE, tol_mean=None,
                                    bf16_out=False)
                parity.assert_close("dQ rows b%d h%d" % (b, h), parity.f64(dq[b, rows, h]),
                                    ref["dq"])


def _key_sample(inp, b, hk, nrand, rng):
    """Key rows of (sequence b, kv head hk) to check: first and last rows,
    tile edges, seeded random rows, and for each x8 query row i of the group
    the keys of its diagonal tile up to i plus the keys it weighs most (the
    largest q_i . k_j over j <= i), where its dS is largest."""
    w = inp.workload
    N = w.N
    keys = {0, 1, 127, 128, N // 2, N - 1}
    keys |= set(int(x) for x in rng.integers(0, N, nrand))
    if inp.x8_rows is not None:
        g = w.Hq // w.Hkv
        kf = inp.k[b, :, hk].float()
        for h in range(hk * g, (hk + 1) * g):
            i = int(inp.x8_rows[b, h])
            t0 = 128 * (i // 128)
            keys |= {t0, i, (t0 + i) // 2}
            lim = i + 1 if w.causal else N
            logit = kf[:lim] @ inp.q[b, i, h].float()
            keys |= set(int(x) for x in torch.topk(logit, min(3, lim)).indices)
    return sorted(keys)


def _check_cols(inp, outs, nrand, seed=0):
    """dK and dV of sampled key rows on every kv head against the oracle's
    column sampler (summed over each group's query heads)."""
    o, lse, dq, dk, dv = outs
    w = inp.workload
    rng = np.random.default_rng(seed)
    g = w.Hq // w.Hkv
    for b in range(w.B):
        for hk in range(w.Hkv):
            keys = _key_sample(inp, b, hk, nrand, rng)
            heads = slice(hk * g, (hk + 1) * g)
            f = lambda t, hs: t[b:b + 1, :, hs].float().numpy().astype(np.float64)
            cols = np.array([[0, 0, j] for j in keys])
            ref = oracle.attention_cols(f(inp.q, heads), f(inp.k, slice(hk, hk + 1)),
                                        f(inp.v, slice(hk, hk + 1)), f(inp.dout, heads), cols,
                                        w.scale, w.causal)
            parity.assert_close("dK cols b%d kv%d" % (b, hk), parity.f64(dk[b, keys, hk]),
                                ref["dk"])
            parity.assert_close("dV cols b%d kv%d" % (b, hk), parity.f64(dv[b, keys, hk]),
                                ref["dv"])


def _to_host(outs):
    """Copy the GPU outputs to host memory and release the device copies."""
    host = tuple(t.cpu() for t in outs)
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return host


def _check_invariants(inp, outs):
    o, lse, dq, dk, dv = outs
    w = inp.workload
    g = w.Hq // w.Hkv
    dk64 = dk.double()
    dv64 = dv.double()
    do64 = inp.dout.cuda().double()
    # sum over keys of dK vanishes; bound: bf16 rounding of every summand
    sk = dk64.sum(dim=1).abs()
    bound_k = 2.0 ** -8 * dk64.abs().sum(dim=1) + 1e-2
    assert bool((sk <= bound_k).all()), float((sk - bound_k).max())
    grp = do64.view(w.B, w.N, w.Hkv, g, w.d).sum(dim=(1, 3))
    sv = (dv64.sum(dim=1) - grp).abs()
    bound_v = 2.0 ** -8 * dv64.abs().sum(dim=1) + 1e-2
    assert bool((sv <= bound_v).all()), float((sv - bound_v).max())


def test_gqa_causal_b2_hq32_hkv8_n4096_d128():
    inp = workloads.generate(workloads.WORKLOADS["gqa_causal_b2_hq32_hkv8_n4096_d128"])
    outs = _run_gpu(inp)
    _check_group(inp, outs, 0, 0, parity.TOL_MAX)
    _check_group(inp, outs, 1, 7, parity.TOL_MAX)
    _check_rows(inp, outs, nrows=ROWS_PER_HEAD)
    _check_invariants(inp, outs)


@pytest.mark.parametrize("d", [64, 128])
def test_long_causal_n4096_x8row(d):
    inp = workloads.generate(workloads.WORKLOADS["long_causal_b1_h16_n4096_d%d_x8row" % d])
    outs = _run_gpu(inp)
    for hk in (0, 15):
        _check_group(inp, outs, 0, hk, parity.TOL_MAX)
    _check_rows(inp, outs, nrows=ROWS_PER_HEAD)
    _check_invariants(inp, outs)


@pytest.mark.parametrize("d", [64, 128])
def test_long_causal_n16384_x8row(d):
    inp = workloads.generate(workloads.WORKLOADS["long_causal_b1_h16_n16384_d%d_x8row" % d])
    outs = _run_gpu(inp)
    _check_invariants(inp, outs)
    outs = _to_host(outs)
    for hk in (0, 15):
        _check_group(inp, outs, 0, hk, parity.TOL_MAX)
    _check_rows(inp, outs, nrows=ROWS_PER_HEAD)
    _check_cols(inp, outs, nrand=8)


@pytest.mark.parametrize("d", [64, 128])
def test_long_causal_n65536_x8row(d):
    inp = workloads.generate(workloads.WORKLOADS["long_causal_b1_h16_n65536_d%d_x8row" % d])
    outs = _run_gpu(inp)
    _check_invariants(inp, outs)
    outs = _to_host(outs)
    _check_rows(inp, outs, nrows=ROWS_PER_HEAD)
    _check_cols(inp, outs, nrand=6)
