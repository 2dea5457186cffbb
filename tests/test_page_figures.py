"""The FLOP / byte accounting reproduces the figures the pages print.

Fixture: tests/golden/page_figures.json (each entry cites its page and
section).  CPU only.
"""
import json
import os

import pytest

from exact_io_aware_67_b200 import flops, workloads

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_figures.json")))


def _parse(s, binary):
    num, unit = s.split()
    if binary:
        return float(num) * {"MB": 2 ** 20, "GB": 2 ** 30}[unit]
    return float(num) * {"MB": 1e6, "GB": 1e9}[unit]


@pytest.mark.parametrize("row", GOLD["standard_attention_table"]["rows"])
def test_flop_column(row):
    d = GOLD["standard_attention_table"]["d"]
    f = flops.standard_attention_flops(row["N"], d)
    # the page rounds to 2-3 significant digits
    assert abs(f / 1e9 - row["gflops"]) <= 0.006 * row["gflops"] + 0.005


@pytest.mark.parametrize("row", GOLD["standard_attention_table"]["rows"])
def test_traffic_and_memory_columns(row):
    d = GOLD["standard_attention_table"]["d"]
    N = row["N"]
    # traffic column: 4N^2 + 4Nd elements at one byte each (the page's own
    # arithmetic), i.e. half of our fp16 byte count
    t = flops.standard_attention_hbm_bytes(N, d, elem_bytes=1)
    assert abs(t / _parse(row["traffic"], binary=False) - 1) < 0.065
    # intermediate column: S and P of N^2 fp16 values each = 4 N^2 bytes
    assert abs(4.0 * N * N / _parse(row["intermediate"], binary=True) - 1) < 1e-9


def test_page1_io_example():
    ex = GOLD["io_example"]
    N, d = ex["N"], ex["d"]
    assert abs(3 * N * d * 2 / 2 ** 20 - 3.0) < 1e-9
    assert abs(N * N * 2 / 2 ** 20 - 32.0) < 1e-9


def test_workload_flop_counts():
    w = workloads.WORKLOADS["gqa_causal_b2_hq32_hkv8_n4096_d128"]
    assert flops.fwd_flops(w) == 0.5 * 4 * 2 * 32 * 4096 ** 2 * 128
    assert abs(flops.fwd_flops(w) / 1e9 - 274.9) < 0.1
    assert flops.bwd_flops(w) == 2.5 * flops.fwd_flops(w)
    w2 = workloads.WORKLOADS["gpt2_small_causal_b8_h12_n1024_d64"]
    assert abs(flops.fwd_flops(w2) / 1e9 - 12.88) < 0.01
    w4 = workloads.WORKLOADS["long_causal_b1_h16_n65536_d128_x8row"]
    assert abs(flops.fwd_flops(w4) / 1e9 - 17592) < 1
    wv = workloads.WORKLOADS["bert_large_varlen_32x128to512_h16_d64"]
    lens = [128, 512]
    assert flops.fwd_flops(wv, lens) == 4 * 16 * 64 * (128 ** 2 + 512 ** 2)


def test_generator_is_deterministic_and_ordered():
    w = workloads.custom("t", 1, 2, 1, 16, 8, True, x8_row=True)
    a = workloads.generate(w)
    b = workloads.generate(w)
    for x, y in ((a.q, b.q), (a.k, b.k), (a.v, b.v), (a.dout, b.dout)):
        assert (x.float() == y.float()).all()
    assert a.x8_rows.shape == (1, 2)
    # the key-row variant draws the same Q, K, V, dO and scales exactly one K
    # row per (batch, kv head) by 8, leaving the query rows alone
    wk = workloads.custom("tk", 2, 4, 2, 16, 8, True, x8_key_row=True)
    ck = workloads.generate(wk)
    c0 = workloads.generate(workloads.custom("tk", 2, 4, 2, 16, 8, True))
    assert (ck.q.float() == c0.q.float()).all() and (ck.v.float() == c0.v.float()).all()
    ratio_rows = (ck.k.float() != c0.k.float()).any(dim=-1)      # [B, N, Hkv]
    for bb in range(2):
        for h in range(2):
            r = int(ck.x8_key_rows[bb, h])
            assert ratio_rows[bb, :, h].nonzero().flatten().tolist() in ([r], [])
            assert (ck.k[bb, r, h].float() == 8 * c0.k[bb, r, h].float()).all()
    wv = workloads.WORKLOADS["bert_large_varlen_32x128to512_h16_d64"]
    iv = workloads.generate(wv)
    assert len(iv.lengths) == 32 and all(128 <= L <= 512 for L in iv.lengths)
    assert int(iv.cu_seqlens[-1]) == sum(iv.lengths) == iv.q.shape[0]


# ------------------------------------------------- block-sparse accounting

@pytest.mark.parametrize("N,causal,seed", [(300, False, 1), (300, True, 2), (1024, True, 3),
                                           (1000, False, 4)])
def test_blocksparse_pairs_match_brute_force(N, causal, seed):
    # allowed (query, key) pairs of a block mask, counted element by element
    import numpy as np
    nt = (N + 127) // 128
    rng = np.random.default_rng(seed)
    m = rng.random((nt, nt)) < 0.5
    el = np.repeat(np.repeat(m, 128, axis=0), 128, axis=1)[:N, :N]
    if causal:
        el &= np.tril(np.ones((N, N), dtype=bool))
    assert flops.blocksparse_pairs(N, causal, m) == int(el.sum())


def test_blocksparse_flops_all_allowed_equals_dense_count():
    # with every tile allowed and no mask, 4 d per pair over all N^2 pairs is
    # the dense forward count
    import numpy as np
    bw = workloads.BlockSparseWorkload(
        "t", workloads.custom("t", 2, 4, 2, 512, 64, False), density=1.0)
    mask = np.ones((1, 2, 4, 4), dtype=np.uint8)
    assert flops.blocksparse_fwd_flops(bw, mask) == flops.fwd_flops(bw.base)
