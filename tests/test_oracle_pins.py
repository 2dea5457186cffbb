"""Pins of the CPU oracle to things other than itself (CPU only).

Each test checks the oracle against something the pages or the mathematics
fix: a fully independent pure-Python brute force, closed forms, the online
softmax recurrence of "FlashAttention优化" 3.2.1-3.2.2, central finite
differences of the gradients, structural invariants, and a library routine
(PyTorch's fp64 CPU scaled_dot_product_attention with autograd).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import brute

RNG = np.random.default_rng(12345)


def rand(*shape, rng=RNG):
    return rng.standard_normal(shape)


def to_lists(a):
    return a.tolist()


# ---------------------------------------------------------------- brute force

@pytest.mark.parametrize("n", [1, 2, 3, 4])
@pytest.mark.parametrize("Hq,Hkv", [(1, 1), (2, 1), (2, 2)])
@pytest.mark.parametrize("causal", [False, True])
def test_brute_force_matches(n, Hq, Hkv, causal):
    d = 3 if n % 2 else 2
    rng = np.random.default_rng(n * 100 + Hq * 10 + Hkv + causal)
    q = rand(1, n, Hq, d, rng=rng)
    k = rand(1, n, Hkv, d, rng=rng)
    v = rand(1, n, Hkv, d, rng=rng)
    do = rand(1, n, Hq, d, rng=rng)
    scale = 0.7
    o, lse = oracle.attention_fwd(q, k, v, scale, causal)
    g = oracle.attention_bwd(q, k, v, do, scale, causal)
    bo, blse = brute.forward(to_lists(q[0]), to_lists(k[0]), to_lists(v[0]), scale, causal)
    bdq, bdk, bdv = brute.backward(to_lists(q[0]), to_lists(k[0]), to_lists(v[0]),
                                   to_lists(do[0]), scale, causal)
    np.testing.assert_allclose(o[0], np.array(bo), rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse[0], np.array(blse), rtol=0, atol=1e-13)
    np.testing.assert_allclose(g["dq"][0], np.array(bdq), rtol=0, atol=1e-12)
    np.testing.assert_allclose(g["dk"][0], np.array(bdk), rtol=0, atol=1e-12)
    np.testing.assert_allclose(g["dv"][0], np.array(bdv), rtol=0, atol=1e-12)
    np.testing.assert_allclose(g["o"], o, rtol=0, atol=1e-14)
    np.testing.assert_allclose(g["lse"], lse, rtol=0, atol=1e-14)


# ---------------------------------------------------------------- closed forms

@pytest.mark.parametrize("causal", [False, True])
def test_uniform_v_gives_v(causal):
    """Every P row sums to 1, so equal V rows give O_i = v exactly."""
    B, N, H, d = 2, 33, 3, 8
    q, k = rand(B, N, H, d), rand(B, N, H, d)
    row = rand(d)
    v = np.broadcast_to(row, (B, N, H, d)).copy()
    o, _ = oracle.attention_fwd(q, k, v, 0.35, causal)
    np.testing.assert_allclose(o, np.broadcast_to(row, o.shape), rtol=0, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_identical_keys_give_uniform_weights(causal):
    """Identical keys: every allowed logit equals s_i, so P is uniform over the
    allowed keys, O_i is the mean of those V rows and LSE_i = s_i + ln(count)."""
    B, N, H, d = 1, 21, 2, 5
    q = rand(B, N, H, d)
    krow = rand(d)
    k = np.broadcast_to(krow, (B, N, H, d)).copy()
    v = rand(B, N, H, d)
    scale = 0.4
    o, lse = oracle.attention_fwd(q, k, v, scale, causal)
    for h in range(H):
        for i in range(N):
            cnt = i + 1 if causal else N
            np.testing.assert_allclose(o[0, i, h], v[0, :cnt, h].mean(axis=0), atol=1e-13)
            s = scale * float(q[0, i, h] @ krow)
            assert abs(lse[0, h, i] - (s + math.log(cnt))) < 1e-13


def test_causal_first_row():
    """Causal row 0 sees only key 0: O_0 = V_0 and LSE_0 = scale q_0 . k_0."""
    B, N, H, d = 2, 17, 2, 6
    q, k, v = rand(B, N, H, d), rand(B, N, H, d), rand(B, N, H, d)
    o, lse = oracle.attention_fwd(q, k, v, 0.9, True)
    np.testing.assert_allclose(o[:, 0], v[:, 0], rtol=0, atol=1e-14)
    for b in range(B):
        for h in range(H):
            assert abs(lse[b, h, 0] - 0.9 * float(q[b, 0, h] @ k[b, 0, h])) < 1e-13


def test_single_key_gradients():
    """N = 1: P = [1], O = V, so dV = dO, dQ = 0 and dK = 0."""
    q, k, v, do = rand(1, 1, 2, 4), rand(1, 1, 2, 4), rand(1, 1, 2, 4), rand(1, 1, 2, 4)
    g = oracle.attention_bwd(q, k, v, do, 0.5, False)
    np.testing.assert_allclose(g["dv"], do, atol=1e-15)
    np.testing.assert_allclose(g["dq"], 0.0, atol=1e-15)
    np.testing.assert_allclose(g["dk"], 0.0, atol=1e-15)


# ---------------------------------------------------------------- online softmax

@pytest.mark.parametrize("tile", [1, 3, 64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_streaming_order_matches_three_pass(tile, causal):
    """Online softmax ("FlashAttention优化" 3.2.1) over any tile size and any
    tile order equals the three-pass result (3.2.2)."""
    n, d = 200, 16
    rng = np.random.default_rng(tile + 7 * causal)
    q = rng.standard_normal((n, d)) * 2.0
    k = rng.standard_normal((n, d))
    v = rng.standard_normal((n, d))
    q[17] *= 8.0   # one large row so that the running max moves a lot
    ntiles = (n + tile - 1) // tile
    o_ref, lse_ref = oracle.attention_fwd(q[None, :, None], k[None, :, None],
                                          v[None, :, None], 0.25, causal)
    for order in (None, rng.permutation(ntiles), np.arange(ntiles)[::-1].copy()):
        o, lse = oracle.attention_fwd_streaming(q, k, v, 0.25, causal, tile, order)
        np.testing.assert_allclose(o, o_ref[0, :, 0], rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse, lse_ref[0, 0], rtol=0, atol=1e-12)


# ---------------------------------------------------------------- finite differences

def _loss(q, k, v, do, scale, causal):
    o, _ = oracle.attention_fwd(q, k, v, scale, causal)
    return float(np.sum(o * do))


@pytest.mark.parametrize("N,d,Hq,Hkv,causal", [
    (9, 4, 2, 1, False), (9, 4, 2, 1, True), (16, 8, 2, 2, True), (13, 8, 4, 2, False)])
def test_finite_difference_gradients(N, d, Hq, Hkv, causal):
    rng = np.random.default_rng(N * d + Hq + causal)
    q = rng.standard_normal((1, N, Hq, d))
    k = rng.standard_normal((1, N, Hkv, d))
    v = rng.standard_normal((1, N, Hkv, d))
    do = rng.standard_normal((1, N, Hq, d))
    scale = 1.0 / math.sqrt(d)
    g = oracle.attention_bwd(q, k, v, do, scale, causal)
    h = 1e-6
    for name, arr in (("dq", q), ("dk", k), ("dv", v)):
        idx = [tuple(rng.integers(0, s) for s in arr.shape) for _ in range(12)]
        for ix in idx:
            a0 = arr[ix]
            arr[ix] = a0 + h
            lp = _loss(q, k, v, do, scale, causal)
            arr[ix] = a0 - h
            lm = _loss(q, k, v, do, scale, causal)
            arr[ix] = a0
            fd = (lp - lm) / (2 * h)
            an = g[name][ix]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, ix, fd, an)


# ---------------------------------------------------------------- invariants

@pytest.mark.parametrize("causal", [False, True])
def test_gradient_invariants(causal):
    """Each row of dS sums to 0 and each row of P sums to 1, so
    sum_j dK_j = 0 and sum_j dV_j = sum_{h in group} sum_i dO_i; also
    D_i = dO_i . O_i and max_j S_ij <= LSE_i <= max_j S_ij + ln(count)."""
    B, N, Hq, Hkv, d = 2, 40, 4, 2, 8
    q, k, v = rand(B, N, Hq, d), rand(B, N, Hkv, d), rand(B, N, Hkv, d)
    do = rand(B, N, Hq, d)
    scale = 0.3
    g = oracle.attention_bwd(q, k, v, do, scale, causal)
    np.testing.assert_allclose(g["dk"].sum(axis=1), 0.0, atol=1e-12)
    grp = do.reshape(B, N, Hkv, Hq // Hkv, d).sum(axis=(1, 3))
    np.testing.assert_allclose(g["dv"].sum(axis=1), grp, atol=1e-12)
    np.testing.assert_allclose(g["D"], np.einsum("bnhd,bnhd->bhn", do, g["o"]), atol=1e-12)
    kk = np.repeat(k, Hq // Hkv, axis=2)
    S = scale * np.einsum("bihd,bjhd->bhij", q, kk)
    if causal:
        S = np.where(np.tril(np.ones((N, N), bool)), S, -np.inf)
    mx = S.max(axis=-1)
    cnt = (np.arange(N) + 1) if causal else np.full(N, N)
    assert np.all(g["lse"] >= mx - 1e-12)
    assert np.all(g["lse"] <= mx + np.log(cnt) + 1e-12)


def test_permuting_keys_values_jointly():
    B, N, H, d = 1, 30, 2, 4
    q, k, v = rand(B, N, H, d), rand(B, N, H, d), rand(B, N, H, d)
    perm = RNG.permutation(N)
    o1, l1 = oracle.attention_fwd(q, k, v, 0.5, False)
    o2, l2 = oracle.attention_fwd(q, k[:, perm], v[:, perm], 0.5, False)
    np.testing.assert_allclose(o1, o2, atol=1e-13)
    np.testing.assert_allclose(l1, l2, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_equals_independent_sequences(causal):
    lengths = [5, 1, 12, 0, 7]
    Hq, Hkv, d = 4, 2, 6
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    T = int(cu[-1])
    q, k, v, do = rand(T, Hq, d), rand(T, Hkv, d), rand(T, Hkv, d), rand(T, Hq, d)
    o, lse = oracle.attention_fwd(q, k, v, 0.4, causal, cu_seqlens=cu)
    g = oracle.attention_bwd(q, k, v, do, 0.4, causal, cu_seqlens=cu)
    for s, L in enumerate(lengths):
        a, b = cu[s], cu[s + 1]
        if L == 0:
            continue
        os_, ls_ = oracle.attention_fwd(q[None, a:b], k[None, a:b], v[None, a:b], 0.4, causal)
        gs = oracle.attention_bwd(q[None, a:b], k[None, a:b], v[None, a:b], do[None, a:b],
                                  0.4, causal)
        np.testing.assert_allclose(o[a:b], os_[0], atol=1e-14)
        np.testing.assert_allclose(lse[:, a:b], ls_[0], atol=1e-14)
        for nm in ("dq", "dk", "dv"):
            np.testing.assert_allclose(g[nm][a:b], gs[nm][0], atol=1e-13)


def test_gqa_equals_repeated_heads():
    """Grouped-query attention equals multi-head attention on K, V repeated
    along the head axis (contiguous groups), with dK, dV summed over copies."""
    B, N, Hq, Hkv, d = 1, 19, 6, 2, 4
    g = Hq // Hkv
    q, k, v, do = rand(B, N, Hq, d), rand(B, N, Hkv, d), rand(B, N, Hkv, d), rand(B, N, Hq, d)
    kr, vr = np.repeat(k, g, axis=2), np.repeat(v, g, axis=2)
    a = oracle.attention_bwd(q, k, v, do, 0.6, True)
    b = oracle.attention_bwd(q, kr, vr, do, 0.6, True)
    np.testing.assert_allclose(a["o"], b["o"], atol=1e-14)
    np.testing.assert_allclose(a["dq"], b["dq"], atol=1e-13)
    np.testing.assert_allclose(a["dk"], b["dk"].reshape(B, N, Hkv, g, d).sum(3), atol=1e-13)
    np.testing.assert_allclose(a["dv"], b["dv"].reshape(B, N, Hkv, g, d).sum(3), atol=1e-13)


def test_row_sample_matches_full():
    B, N, Hq, Hkv, d = 2, 50, 4, 2, 8
    q, k, v, do = rand(B, N, Hq, d), rand(B, N, Hkv, d), rand(B, N, Hkv, d), rand(B, N, Hq, d)
    full = oracle.attention_bwd(q, k, v, do, 0.35, True)
    rows = np.array([[0, 0, 0], [1, 3, 49], [0, 2, 17], [1, 1, 31]])
    r = oracle.attention_rows(q, k, v, do, rows, 0.35, True)
    for t, (b, h, i) in enumerate(rows):
        np.testing.assert_allclose(r["o"][t], full["o"][b, i, h], atol=1e-14)
        assert abs(r["lse"][t] - full["lse"][b, h, i]) < 1e-14
        assert abs(r["D"][t] - full["D"][b, h, i]) < 1e-13
        np.testing.assert_allclose(r["dq"][t], full["dq"][b, i, h], atol=1e-13)


# ---------------------------------------------------------------- key-column sampler

def _all_cols(B, Hkv, N):
    return np.array([[b, h, j] for b in range(B) for h in range(Hkv) for j in range(N)])


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,N,Hq,Hkv,d", [(2, 300, 4, 2, 16), (1, 517, 2, 1, 64),
                                          (1, 700, 3, 3, 8)])
def test_cols_match_full_backward(B, N, Hq, Hkv, d, causal):
    """Every key row's dK, dV from the column sampler (torch fp64 products)
    equals the C oracle's full backward; N spans several of its row blocks."""
    rng = np.random.default_rng(B * N + d + causal)
    q, k = rng.standard_normal((B, N, Hq, d)), rng.standard_normal((B, N, Hkv, d))
    v, do = rng.standard_normal((B, N, Hkv, d)), rng.standard_normal((B, N, Hq, d))
    full = oracle.attention_bwd(q, k, v, do, d ** -0.5, causal)
    cols = _all_cols(B, Hkv, N)
    got = oracle.attention_cols(q, k, v, do, cols, d ** -0.5, causal)
    np.testing.assert_allclose(got["dk"], full["dk"][cols[:, 0], cols[:, 2], cols[:, 1]],
                               rtol=0, atol=1e-12)
    np.testing.assert_allclose(got["dv"], full["dv"][cols[:, 0], cols[:, 2], cols[:, 1]],
                               rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_cols_varlen_match_full_backward(causal):
    lengths = [5, 600, 1, 130]
    Hq, Hkv, d = 4, 2, 8
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    T = int(cu[-1])
    rng = np.random.default_rng(7 + causal)
    q, k, v, do = (rng.standard_normal((T, H, d)) for H in (Hq, Hkv, Hkv, Hq))
    full = oracle.attention_bwd(q, k, v, do, 0.3, causal, cu_seqlens=cu)
    cols = np.array([[s, h, j] for s, L in enumerate(lengths) for h in range(Hkv)
                     for j in range(L)])
    got = oracle.attention_cols(q, k, v, do, cols, 0.3, causal, cu_seqlens=cu)
    tok = cu[cols[:, 0]] + cols[:, 2]
    np.testing.assert_allclose(got["dk"], full["dk"][tok, cols[:, 1]], rtol=0, atol=1e-12)
    np.testing.assert_allclose(got["dv"], full["dv"][tok, cols[:, 1]], rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_cols_match_brute_force(causal):
    n, Hq, Hkv, d = 4, 2, 1, 3
    rng = np.random.default_rng(31 + causal)
    q, k = rng.standard_normal((1, n, Hq, d)), rng.standard_normal((1, n, Hkv, d))
    v, do = rng.standard_normal((1, n, Hkv, d)), rng.standard_normal((1, n, Hq, d))
    _, bdk, bdv = brute.backward(to_lists(q[0]), to_lists(k[0]), to_lists(v[0]),
                                 to_lists(do[0]), 0.8, causal)
    got = oracle.attention_cols(q, k, v, do, _all_cols(1, Hkv, n), 0.8, causal)
    np.testing.assert_allclose(got["dk"], np.array(bdk)[:, 0], rtol=0, atol=1e-13)
    np.testing.assert_allclose(got["dv"], np.array(bdv)[:, 0], rtol=0, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_cols_finite_differences(causal):
    """Central differences of L = sum(O o dO) (O from the C oracle's forward)
    with respect to sampled K and V entries match the column sampler."""
    N, Hq, Hkv, d = 11, 4, 2, 4
    rng = np.random.default_rng(99 + causal)
    q, k = rng.standard_normal((1, N, Hq, d)), rng.standard_normal((1, N, Hkv, d))
    v, do = rng.standard_normal((1, N, Hkv, d)), rng.standard_normal((1, N, Hq, d))
    scale = 0.5
    cols = np.array([[0, 0, 0], [0, 1, 5], [0, 1, 10], [0, 0, 7]])
    got = oracle.attention_cols(q, k, v, do, cols, scale, causal)
    h = 1e-6
    for t, (_, hk, j) in enumerate(cols):
        for name, arr in (("dk", k), ("dv", v)):
            for c in range(d):
                a0 = arr[0, j, hk, c]
                arr[0, j, hk, c] = a0 + h
                lp = _loss(q, k, v, do, scale, causal)
                arr[0, j, hk, c] = a0 - h
                lm = _loss(q, k, v, do, scale, causal)
                arr[0, j, hk, c] = a0
                fd = (lp - lm) / (2 * h)
                an = got[name][t, c]
                assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, t, c, fd, an)


# ---------------------------------------------------------------- library routine

def _torch_reference(q, k, v, do, scale, causal):
    """PyTorch fp64 CPU SDPA with autograd, layout [B, N, H, d]."""
    Hq, Hkv = q.shape[2], k.shape[2]
    tq = torch.tensor(q, dtype=torch.float64, requires_grad=True)
    tk = torch.tensor(k, dtype=torch.float64, requires_grad=True)
    tv = torch.tensor(v, dtype=torch.float64, requires_grad=True)
    kk = tk.repeat_interleave(Hq // Hkv, dim=2)
    vv = tv.repeat_interleave(Hq // Hkv, dim=2)
    o = torch.nn.functional.scaled_dot_product_attention(
        tq.transpose(1, 2), kk.transpose(1, 2), vv.transpose(1, 2),
        is_causal=causal, scale=scale).transpose(1, 2)
    o.backward(torch.tensor(do, dtype=torch.float64))
    return o.detach().numpy(), tq.grad.numpy(), tk.grad.numpy(), tv.grad.numpy()


@pytest.mark.parametrize("N,Hq,Hkv,causal", [(37, 4, 2, True), (64, 2, 2, False),
                                             (130, 8, 2, True)])
def test_matches_torch_sdpa_fp64(N, Hq, Hkv, causal):
    B, d = 2, 16
    rng = np.random.default_rng(N)
    q = rng.standard_normal((B, N, Hq, d))
    k = rng.standard_normal((B, N, Hkv, d))
    v = rng.standard_normal((B, N, Hkv, d))
    do = rng.standard_normal((B, N, Hq, d))
    scale = 1.0 / math.sqrt(d)
    o_t, dq_t, dk_t, dv_t = _torch_reference(q, k, v, do, scale, causal)
    o, _ = oracle.attention_fwd(q, k, v, scale, causal)
    g = oracle.attention_bwd(q, k, v, do, scale, causal)
    np.testing.assert_allclose(o, o_t, atol=1e-12)
    np.testing.assert_allclose(g["dq"], dq_t, atol=1e-11)
    np.testing.assert_allclose(g["dk"], dk_t, atol=1e-11)
    np.testing.assert_allclose(g["dv"], dv_t, atol=1e-11)


# ------------------------------------------------- softmax step of standard attention

@pytest.mark.parametrize("n,causal", [(1, False), (5, True), (7, False), (16, True)])
def test_softmax_rows_matches_brute_force(n, causal):
    rng = np.random.default_rng(100 + n)
    s = rng.standard_normal((3, n, n)) * 4.0
    scale = 0.3
    p, lse = oracle.softmax_rows(s, scale, causal)
    for h in range(3):
        for i in range(n):
            row = [-math.inf if (causal and j > i) else scale * float(s[h, i, j])
                   for j in range(n)]
            bp, bl = brute._softmax(row)
            np.testing.assert_allclose(p[h, i], bp, rtol=0, atol=1e-15)
            assert abs(lse[h, i] - bl) < 1e-13


@pytest.mark.parametrize("causal", [False, True])
def test_softmax_rows_constant_rows(causal):
    # every allowed logit equal: P uniform over the allowed keys and
    # LSE = scale * c + ln(count)
    n, c, scale = 9, 2.5, 0.7
    p, lse = oracle.softmax_rows(np.full((2, n, n), c), scale, causal)
    for i in range(n):
        cnt = i + 1 if causal else n
        np.testing.assert_allclose(p[:, i, :cnt], 1.0 / cnt, atol=1e-15)
        assert np.all(p[:, i, cnt:] == 0.0)
        np.testing.assert_allclose(lse[:, i], scale * c + math.log(cnt), atol=1e-14)


@pytest.mark.parametrize("causal", [False, True])
def test_softmax_rows_matches_torch_softmax(causal):
    rng = np.random.default_rng(7)
    n, scale = 33, 0.125
    s = rng.standard_normal((4, n, n)) * 8.0
    x = torch.tensor(s, dtype=torch.float64) * scale
    if causal:
        x = x.masked_fill(torch.ones(n, n, dtype=torch.bool).triu(1), float("-inf"))
    p, lse = oracle.softmax_rows(s, scale, causal)
    np.testing.assert_allclose(p, torch.softmax(x, dim=-1).numpy(), atol=1e-15)
    np.testing.assert_allclose(lse, torch.logsumexp(x, dim=-1).numpy(), atol=1e-13)


def test_standard_pipeline_equals_attention():
    # S materialised, softmax step, then P V: the same O and LSE as the
    # attention definition (one head per [n, n] matrix)
    rng = np.random.default_rng(11)
    N, H, d, scale = 40, 3, 8, 0.35
    q, k, v = (rng.standard_normal((1, N, H, d)) for _ in range(3))
    o_ref, lse_ref = oracle.attention_fwd(q, k, v, scale, True)
    s = np.einsum("nhc,mhc->hnm", q[0], k[0])
    p, lse = oracle.softmax_rows(s, scale, True)
    o = np.einsum("hnm,mhc->nhc", p, v[0])
    np.testing.assert_allclose(o, o_ref[0], atol=1e-13)
    np.testing.assert_allclose(lse, lse_ref[0], atol=1e-13)


# ------------------------------------------------------------------ block masks

def _bm_problem(B=1, N=300, Hq=4, Hkv=2, d=8, seed=21):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, N, Hq, d))
    k = rng.standard_normal((B, N, Hkv, d))
    v = rng.standard_normal((B, N, Hkv, d))
    do = rng.standard_normal((B, N, Hq, d))
    return q, k, v, do


@pytest.mark.parametrize("causal", [False, True])
def test_blockmask_all_allowed_equals_unmasked(causal):
    q, k, v, do = _bm_problem()
    nt = 3
    bm = np.ones((1, 1, nt, nt), dtype=np.uint8)
    o, lse = oracle.attention_fwd_blockmask(q, k, v, 0.3, causal, bm)
    o_ref, lse_ref = oracle.attention_fwd(q, k, v, 0.3, causal)
    assert np.array_equal(o, o_ref) and np.array_equal(lse, lse_ref)
    g = oracle.attention_bwd_blockmask(q, k, v, do, 0.3, causal, bm)
    r = oracle.attention_bwd(q, k, v, do, 0.3, causal)
    for nm in ("dq", "dk", "dv"):
        assert np.array_equal(g[nm], r[nm])


def test_blockmask_diagonal_equals_independent_sequences():
    # only the diagonal 128 x 128 tiles allowed, non-causal: every 128-token
    # block attends to itself alone, which is varlen attention over
    # sequences of 128, 128, ..., the rest (a different indexing path)
    q, k, v, do = _bm_problem(N=3 * 128 + 50)
    N = q.shape[1]
    nt = 4
    bm = np.eye(nt, dtype=np.uint8)[None, None]
    o, lse = oracle.attention_fwd_blockmask(q, k, v, 0.35, False, bm)
    g = oracle.attention_bwd_blockmask(q, k, v, do, 0.35, False, bm)
    cu = np.array([0, 128, 256, 384, N], dtype=np.int32)
    o_v, lse_v = oracle.attention_fwd(q[0], k[0], v[0], 0.35, False, cu)
    r = oracle.attention_bwd(q[0], k[0], v[0], do[0], 0.35, False, cu)
    np.testing.assert_allclose(o[0], o_v, atol=1e-14)
    np.testing.assert_allclose(lse[0], lse_v, atol=1e-14)
    for nm in ("dq", "dk", "dv"):
        np.testing.assert_allclose(g[nm][0], r[nm], atol=1e-13)


def _sdpa_masked(q, k, v, do, scale, causal, bm):
    """PyTorch fp64 SDPA with the block mask expanded to a boolean element
    mask (per key/value head, repeated over its query heads)."""
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    g = Hq // Hkv
    el = np.repeat(np.repeat(bm, 128, axis=2), 128, axis=3)[:, :, :N, :N].astype(bool)
    el = np.broadcast_to(el, (B, Hkv, N, N))
    if causal:
        el = el & np.tril(np.ones((N, N), dtype=bool))
    mask = torch.tensor(np.repeat(el, g, axis=1).copy())
    tq = torch.tensor(q, requires_grad=True)
    tk = torch.tensor(k, requires_grad=True)
    tv = torch.tensor(v, requires_grad=True)
    kk = tk.repeat_interleave(g, dim=2)
    vv = tv.repeat_interleave(g, dim=2)
    o = torch.nn.functional.scaled_dot_product_attention(
        tq.transpose(1, 2), kk.transpose(1, 2), vv.transpose(1, 2), attn_mask=mask,
        scale=scale).transpose(1, 2)
    return o, tq, tk, tv, mask


@pytest.mark.parametrize("causal", [False, True])
def test_blockmask_matches_torch_sdpa_with_element_mask(causal):
    q, k, v, do = _bm_problem(B=2, N=300, Hq=4, Hkv=2, seed=5)
    rng = np.random.default_rng(9)
    bm = (rng.random((2, 2, 3, 3)) < 0.6).astype(np.uint8)
    bm[:, :, np.arange(3), np.arange(3)] = 1          # every row keeps a key
    o_t, tq, tk, tv, _ = _sdpa_masked(q, k, v, do, 0.3, causal, bm)
    o_t.backward(torch.tensor(do))
    o, _ = oracle.attention_fwd_blockmask(q, k, v, 0.3, causal, bm)
    g = oracle.attention_bwd_blockmask(q, k, v, do, 0.3, causal, bm)
    np.testing.assert_allclose(o, o_t.detach().numpy(), atol=1e-12)
    np.testing.assert_allclose(g["dq"], tq.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(g["dk"], tk.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(g["dv"], tv.grad.numpy(), atol=1e-11)


def test_blockmask_rows_without_keys():
    # query tile 1 allowed nowhere: its rows get O = 0, LSE = -inf, dQ = 0
    # and contribute nothing to dK, dV
    q, k, v, do = _bm_problem(N=300)
    bm = np.ones((1, 1, 3, 3), dtype=np.uint8)
    bm[0, 0, 1, :] = 0
    o, lse = oracle.attention_fwd_blockmask(q, k, v, 0.3, False, bm)
    g = oracle.attention_bwd_blockmask(q, k, v, do, 0.3, False, bm)
    assert np.all(o[:, 128:256] == 0.0) and np.all(np.isneginf(lse[:, :, 128:256]))
    assert np.all(g["dq"][:, 128:256] == 0.0)
    # the other rows are the unmasked problem with those query rows removed:
    # zeroing dO on them leaves dK and dV of the full problem unchanged
    do2 = do.copy()
    do2[:, 128:256] = 0.0
    r = oracle.attention_bwd(q, k, v, do2, 0.3, False)
    np.testing.assert_allclose(g["dk"], r["dk"], atol=1e-12)
    np.testing.assert_allclose(g["dv"], r["dv"], atol=1e-12)
    np.testing.assert_allclose(o[:, :128], r["o"][:, :128], atol=1e-14)


def test_blockmask_finite_differences():
    q, k, v, do = _bm_problem(N=140, Hq=2, Hkv=1, d=4, seed=3)
    bm = np.array([[[[1, 0], [1, 1]]]], dtype=np.uint8)
    bm[0, 0, 1, 0] = 0                                 # row tile 1 sees only tile 1
    scale, causal = 0.5, True
    g = oracle.attention_bwd_blockmask(q, k, v, do, scale, causal, bm)

    def loss():
        o, _ = oracle.attention_fwd_blockmask(q, k, v, scale, causal, bm)
        return float(np.sum(o * do))

    h = 1e-6
    for nm, arr, ixs in (("dq", q, [(0, 3, 1, 2), (0, 131, 0, 1)]),
                         ("dk", k, [(0, 2, 0, 3), (0, 135, 0, 0)]),
                         ("dv", v, [(0, 5, 0, 1), (0, 139, 0, 2)])):
        for ix in ixs:
            a0 = arr[ix]
            arr[ix] = a0 + h
            lp = loss()
            arr[ix] = a0 - h
            lm = loss()
            arr[ix] = a0
            fd = (lp - lm) / (2 * h)
            assert abs(fd - g[nm][ix]) <= 1e-6 * max(1.0, abs(g[nm][ix])), (nm, ix, fd, g[nm][ix])
