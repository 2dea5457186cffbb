"""Decode attention over a KV cache (fa_decode) against the oracle.

The oracle computes each (sequence, query head) as row 0 of a non-causal
attention problem whose keys and values are the sequence's first L_b cache
rows: that row's output and LSE depend only on its own query and on every
key and value, which is exactly the decode step.  Tolerances are the
project's bar: O max-abs 2e-2 (+ the bf16 rounding distance of the oracle
value) and mean-abs 2e-3, LSE max-abs 1e-3.
"""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_67_b200 import ops, workloads
import parity

pytestmark = pytest.mark.gpu


def _oracle_decode(inp, batches=None):
    """o [B', Hq, d] and lse [B', Hq] of the selected sequences (fp64)."""
    w = inp.workload
    lens = inp.lengths
    batches = range(w.B) if batches is None else batches
    os_, ls_ = [], []
    for b in batches:
        L = lens[b]
        if L == 0:
            os_.append(np.zeros((w.Hq, w.d)))
            ls_.append(np.full((w.Hq,), -np.inf))
            continue
        qf = np.zeros((1, L, w.Hq, w.d))
        qf[0, 0] = inp.q[b].double().numpy()
        kb = inp.k[b:b + 1, :L].double().numpy()
        vb = inp.v[b:b + 1, :L].double().numpy()
        rows = np.array([[0, h, 0] for h in range(w.Hq)])
        r = oracle.attention_rows(qf, kb, vb, None, rows, w.scale, False)
        os_.append(r["o"])
        ls_.append(r["lse"])
    return np.stack(os_), np.stack(ls_)


def _run(inp, poison_tail=False):
    w = inp.workload
    q, k, v = inp.q.cuda(), inp.k.cuda(), inp.v.cuda()
    sl = None if inp.seqlens is None else inp.seqlens.cuda()
    if poison_tail:
        # cache rows past each sequence's length may hold anything
        for b, L in enumerate(inp.lengths):
            k[b, L:] = float("nan")
            v[b, L:] = float("inf")
    o, lse = ops.decode(q, k, v, sl, w.scale)
    torch.cuda.synchronize()
    parity.no_device_error()
    return o, lse


def _check(inp, o, lse, batches=None):
    ref_o, ref_l = _oracle_decode(inp, batches)
    sel = list(range(inp.workload.B)) if batches is None else list(batches)
    got_o = parity.f64(o[sel])
    got_l = parity.f64(lse[sel])
    empty = np.array([inp.lengths[b] == 0 for b in sel])
    if empty.any():
        assert np.all(got_o[empty] == 0.0) and np.all(np.isneginf(got_l[empty]))
    keep = ~empty
    parity.assert_close("O", got_o[keep], ref_o[keep])
    parity.assert_close("LSE", got_l[keep], ref_l[keep], tol_max=parity.TOL_LSE, tol_mean=None,
                        bf16_out=False)


def _custom(B, Hq, Hkv, Lmax, d, lengths=None, seed=0):
    w = workloads.DecodeWorkload(name="t", B=B, Hq=Hq, Hkv=Hkv, Lmax=Lmax, d=d,
                                 scale=d ** -0.5, seed=seed)
    inp = workloads.generate_decode(w)
    if lengths is not None:
        inp.seqlens = torch.tensor(lengths, dtype=torch.int32)
    return inp


@pytest.mark.parametrize("B,Hq,Hkv,Lmax,d,lengths", [
    (3, 4, 4, 300, 64, [300, 1, 129]),         # ragged tiles, one key
    (2, 8, 2, 1024, 128, None),                 # GQA 4, full caches, several chunks
    (1, 16, 1, 2000, 128, None),                # 16 query heads per kv head
    (2, 6, 2, 777, 64, [777, 500]),             # 3 heads per kv head (padded group)
    (2, 2, 2, 640, 128, [0, 640]),              # an empty cache
    (40, 8, 8, 200, 64, None),                  # enough CTAs for a single chunk
    (2, 4, 1, 5000, 64, [4999, 3000]),          # one kv head, long ragged caches
    (2, 4, 1, 1280, 64, [1280, 1]),             # more CTAs than tiles: empty ranges
    (3, 8, 8, 4096, 128, [0, 3000, 0]),         # empty sequences around a long one
])
def test_decode_matches_oracle(B, Hq, Hkv, Lmax, d, lengths):
    inp = _custom(B, Hq, Hkv, Lmax, d, lengths, seed=Lmax)
    o, lse = _run(inp)
    _check(inp, o, lse)


def test_decode_ignores_cache_rows_past_the_length():
    inp = _custom(3, 8, 2, 1000, 128, [1000, 333, 17], seed=9)
    o, lse = _run(inp, poison_tail=True)
    assert torch.isfinite(o.float()).all()
    _check(inp, o, lse)


@pytest.mark.parametrize("name", sorted(workloads.DECODE_WORKLOADS))
def test_decode_workloads_sampled(name):
    w = workloads.DECODE_WORKLOADS[name]
    inp = workloads.generate_decode(w)
    o, lse = _run(inp)
    # every head of three sequences (first, last, longest), against the oracle
    lens = inp.lengths
    sel = sorted({0, w.B - 1, int(np.argmax(lens))})
    _check(inp, o, lse, sel)
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
