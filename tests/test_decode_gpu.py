"""Decode attention over a KV cache (fa_decode) against the oracle.

The oracle computes each (sequence, query head) as row 0 of a non-causal
attention problem whose keys and values are the sequence's first L_b cache
rows: that row's output and LSE depend only on its own query and on every
key and value, which is exactly the decode step.  Tolerances are the
project's bar: O max-abs 2e-2 and mean-abs 2e-3, LSE max-abs 1e-3 (an O
entry whose oracle value is itself farther than 2e-2 from every bf16 number
would be held to 2e-2 plus that distance and reported; see parity.py).
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


def _run(inp, poison_tail=False, workspace=None):
    w = inp.workload
    q, k, v = inp.q.cuda(), inp.k.cuda(), inp.v.cuda()
    sl = None if inp.seqlens is None else inp.seqlens.cuda()
    if poison_tail:
        # cache rows past each sequence's length may hold anything
        for b, L in enumerate(inp.lengths):
            k[b, L:] = float("nan")
            v[b, L:] = float("inf")
    o, lse = ops.decode(q, k, v, sl, w.scale, workspace=workspace)
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
    (64, 4, 4, 100, 128, None),                 # one tile per pair: no partials at all
    (1, 16, 1, 40000, 128, None),               # one pair over every CTA: 148 partials
    (1, 1, 1, 20000, 64, None),                 # a single query head over every CTA
    (1, 4, 1, 512, 64, [256]),                  # 3 slots, the middle CTA empty
    (2, 8, 2, 512, 128, [300, 0]),              # 6 slots with empty CTAs, an empty sequence
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


@pytest.mark.parametrize("device_lengths", [False, True])
def test_decode_reuses_one_workspace(device_lengths):
    # back-to-back calls on one workspace (uninitialised: every call sets
    # up what it reads), alternating lengths, each checked
    lens = ([3000, 17, 2999, 1500], [129, 3000, 0, 640]) if device_lengths else (None, None)
    a = _custom(4, 8, 2, 3000, 128, lens[0], seed=3)
    b = _custom(4, 8, 2, 3000, 128, lens[1], seed=4)
    need = ops.fa_decode_workspace_size(4, 8, 3000, 128)
    ws = torch.full((need,), 0xFF, dtype=torch.uint8, device="cuda")
    for inp in (a, b, a, b):
        o, lse = _run(inp, workspace=ws)
        _check(inp, o, lse)


def test_decode_back_to_back_calls_without_host_waits():
    # Many calls queued on one stream with no synchronisation in between,
    # each into its own outputs, alternating two problems on one workspace:
    # a call's kernels start while the previous call's finish (programmatic
    # dependent launches), so each must wait before touching memory.
    a = _custom(4, 8, 2, 2000, 64, [2000, 1, 777, 1500], seed=5)
    b = _custom(4, 8, 2, 2000, 64, [640, 2000, 0, 129], seed=6)
    dev = []
    for inp in (a, b):
        dev.append((inp.q.cuda(), inp.k.cuda(), inp.v.cuda(), inp.seqlens.cuda(),
                    inp.workload.scale))
    ws = torch.empty(ops.fa_decode_workspace_size(4, 8, 2000, 64), dtype=torch.uint8,
                     device="cuda")
    outs = []
    for i in range(12):
        q, k, v, sl, sc = dev[i % 2]
        outs.append(ops.decode(q, k, v, sl, sc, workspace=ws))
    torch.cuda.synchronize()
    parity.no_device_error()
    for i in (0, 1):
        _check((a, b)[i], *outs[i])
    for i in range(2, 12):
        o0, l0 = outs[i % 2]
        o, l = outs[i]
        assert bool(((o.double() - o0.double()).abs() <=
                     o0.double().abs() * 2.0 ** -7 + 1e-6).all())
        fin = torch.isfinite(l0)
        assert torch.equal(fin, torch.isfinite(l))
        assert float((l[fin] - l0[fin]).abs().max()) <= 1e-5


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


@pytest.mark.parametrize("lengths", [None, [900, 1, 0, 640]])
def test_decode_captured_in_a_graph(lengths):
    # The decode launch path ([prefix,] split and merge kernels, the last two
    # programmatic dependent launches) captured once: a replay gives the eager
    # results, and picks up new queries and new device-side cache lengths
    # written into the captured buffers.  Equal up to summation order: a
    # CTA's eight warps add their states with shared-memory atomics, so the
    # fp32 sums may differ in the last bits (o by one bf16 rounding step).
    inp = _custom(4, 8, 2, 1000, 64, lengths, seed=21)
    w = inp.workload
    q, k, v = inp.q.cuda(), inp.k.cuda(), inp.v.cuda()
    sl = None if inp.seqlens is None else inp.seqlens.cuda()
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device="cuda")
    ws = torch.empty(ops.fa_decode_workspace_size(w.B, w.Hq, w.Lmax, w.d), dtype=torch.uint8,
                     device="cuda")
    step = lambda: ops.decode(q, k, v, sl, w.scale, out=o, lse=lse, workspace=ws)
    step()
    torch.cuda.synchronize()
    eager_o, eager_l = o.clone(), lse.clone()
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(g):
            step()
    torch.cuda.current_stream().wait_stream(side)
    o.zero_()
    g.replay()
    torch.cuda.synchronize()
    parity.no_device_error()
    d_o = (o.double() - eager_o.double()).abs()
    assert bool((d_o <= eager_o.double().abs() * 2.0 ** -7 + 1e-6).all()), float(d_o.max())
    finite = torch.isfinite(eager_l)
    assert torch.equal(finite, torch.isfinite(lse))
    assert torch.equal(lse[~finite], eager_l[~finite])
    assert float((lse[finite] - eager_l[finite]).abs().max()) <= 1e-5

    inp2 = _custom(4, 8, 2, 1000, 64, None if lengths is None else [17, 1000, 333, 0], seed=22)
    inp2.k, inp2.v = inp.k, inp.v           # same cache, new queries (and lengths)
    q.copy_(inp2.q)
    if sl is not None:
        sl.copy_(inp2.seqlens)
    g.replay()
    torch.cuda.synchronize()
    parity.no_device_error()
    _check(inp2, o, lse)
    del g
