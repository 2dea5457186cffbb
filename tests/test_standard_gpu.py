"""The standard-attention comparator on the GPU: its softmax step
(fa_std_softmax) against the oracle's row softmax, and the whole
materialised pipeline (library GEMM, fa_std_softmax, library GEMM) against
the oracle's attention.

Tolerances follow from the comparator's arithmetic:
  * fa_std_softmax reads bf16 S and writes bf16 P; everything in between is
    fp32.  P may differ from the fp64 softmax of the same S by its own bf16
    rounding plus fp32 error (1e-5 here); LSE by fp32 error.
  * The pipeline stores S as bf16, as the pages' standard attention stores
    16-bit S ("注意力机制基础" 2.2.2).  Rounding S_ij moves logit ij by at
    most delta_i = scale * max_j |S_ij| * 2^-8, which moves LSE_i by at most
    delta_i and P_i. by at most (e^(2 delta_i) - 1) in total; P is then
    rounded to bf16 (2^-8 relative).  So
        |dO_ic| <= max_j |V_jc| ((e^(2 delta_i) - 1) + 2^-7) + rounding(O),
        |dLSE_i| <= delta_i,
    plus 1e-3 for fp32 accumulation.  The mean bar of 2e-3 is kept.
"""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_67_b200 import ops
import parity

pytestmark = pytest.mark.gpu


def _bf16_scores(BH, N, seed, sigma=6.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn((BH, N, N), generator=g) * sigma).to(torch.bfloat16)


@pytest.mark.parametrize("BH,N,causal", [(3, 8, True), (2, 264, False), (2, 1024, True),
                                         (2, 1032, False), (1, 4096, True),
                                         (1, 8192, False)])
def test_std_softmax_matches_oracle(BH, N, causal):
    s = _bf16_scores(BH, N, seed=N)
    scale = 0.125
    s_dev = s.cuda()
    p = torch.full_like(s_dev, float("nan"))
    lse = torch.full((BH, N), float("nan"), dtype=torch.float32, device="cuda")
    st = ops.fa_std_softmax(ops._ptr(s_dev), ops._ptr(p), ops._ptr(lse), BH, N, scale, causal,
                            ops._stream())
    assert st == 0, ops.fa_status_string(st)
    torch.cuda.synchronize()
    ref_p, ref_lse = oracle.softmax_rows(s.double().numpy(), scale, causal)
    got_p = parity.f64(p)
    parity.assert_close("P", got_p, ref_p, tol_max=1e-5, tol_mean=None)
    # on average P is as far from the fp64 softmax as bf16 rounding puts it
    assert np.abs(got_p - ref_p).mean() <= parity.rounding_distance(ref_p).mean() + 1e-6
    parity.assert_close("LSE", parity.f64(lse), ref_lse, tol_max=1e-4, tol_mean=None,
                        bf16_out=False)
    if causal:
        assert torch.all(p.float().triu(1) == 0)


def test_std_softmax_largest_rows_invariants():
    # N = 32768, the largest row the kernel takes: per-row properties that
    # hold at any size (the oracle pins them): P rows sum to 1 up to bf16
    # rounding, masked entries are 0, and max_j x_ij <= LSE_i <= max_j x_ij
    # + ln(allowed keys)
    BH, N, scale = 1, 32768, 0.08
    s = _bf16_scores(BH, N, seed=5).cuda()
    p = torch.empty_like(s)
    lse = torch.empty((BH, N), dtype=torch.float32, device="cuda")
    st = ops.fa_std_softmax(ops._ptr(s), ops._ptr(p), ops._ptr(lse), BH, N, scale, True,
                            ops._stream())
    assert st == 0
    torch.cuda.synchronize()
    rows = torch.arange(N, device="cuda")
    sums = p[0].double().sum(dim=1)
    assert float((sums - 1).abs().max()) <= 2.0 ** -8
    for i in (0, 1, 777, N // 2, N - 1):
        assert torch.all(p[0, i, i + 1:] == 0)
    x = s[0].double() * scale
    x = x.masked_fill(rows[None, :] > rows[:, None], float("-inf"))
    mx = x.max(dim=1).values
    l = lse[0].double()
    assert bool((l >= mx - 1e-4).all())
    assert bool((l <= mx + torch.log(rows.double() + 1) + 1e-4).all())


@pytest.mark.parametrize("B,H,N,d,causal", [(1, 2, 264, 64, True), (2, 2, 1024, 128, False),
                                            (1, 2, 2048, 64, True)])
def test_standard_attention_matches_oracle(B, H, N, d, causal):
    g = torch.Generator().manual_seed(N + d)
    q, k, v = ((torch.randn((B, N, H, d), generator=g)).to(torch.bfloat16) for _ in range(3))
    scale = d ** -0.5
    hm = lambda t: t.transpose(1, 2).contiguous().cuda()   # [B, H, N, d]
    o, lse = ops.standard_attention_fwd(hm(q), hm(k), hm(v), scale, causal)
    torch.cuda.synchronize()
    ref_o, ref_lse = oracle.attention_fwd(q.double().numpy(), k.double().numpy(),
                                          v.double().numpy(), scale, causal)
    got_o = parity.f64(o.transpose(1, 2))                  # [B, N, H, d]
    # error bound from the 16-bit S (module docstring)
    s64 = np.einsum("bnhc,bmhc->bhnm", q.double().numpy(), k.double().numpy())
    if causal:
        s64 = np.where(np.triu(np.ones((N, N), dtype=bool), 1), 0.0, s64)
    delta = scale * np.abs(s64).max(axis=-1) * 2.0 ** -8            # [B, H, N]
    vmax = np.abs(v.double().numpy()).max(axis=1)                   # [B, H, d]
    bound = (vmax[:, None, :, :] * (np.expm1(2 * delta).transpose(0, 2, 1)[..., None]
                                     + 2.0 ** -7)
             + parity.rounding_distance(ref_o) + 1e-3)
    err = np.abs(got_o - ref_o)
    assert np.all(err <= bound), float((err - bound).max())
    assert err.mean() <= parity.TOL_MEAN, err.mean()
    err_l = np.abs(parity.f64(lse) - ref_lse)
    assert np.all(err_l <= delta + 1e-3), float((err_l - delta).max())
