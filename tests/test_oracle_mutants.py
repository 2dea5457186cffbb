"""The pins catch plausible mistakes (CPU only).

Each case plants one mistake in a temporary copy of the oracle's C source
(a flipped sign, a dropped factor, a wrong head index, an off-by-one mask, a
transposed operand, a dropped rescale, a dropped term), compiles it, and runs
a compact battery of the same pins as test_oracle_pins.py against it.  At
least one pin must fail for every mutant, and none may fail for the
unmodified source.
"""
import math
import os
import subprocess

import numpy as np
import pytest

import oracle
from oracle import brute

SRC = os.path.join(os.path.dirname(oracle.__file__), "attention_oracle.c")

MUTANTS = {
    "ds_sign": ("const double ds = p * (dP[j] - Di);", "const double ds = p * (dP[j] + Di);"),
    "dk_drop_scale": ("dkj[c] += scale * ds * qi[c];", "dkj[c] += ds * qi[c];"),
    "kv_head_index": ("const int hk = h / sh->g;\n    const double* qi",
                      "const int hk = h % sh->Hkv;\n    const double* qi"),
    "causal_off_by_one": ("if (sh->causal && j > i) {", "if (sh->causal && j >= i && i > 0) {"),
    "dv_transposed": ("dvj[c] += p * doi[c];", "dvj[c] += p * qi[c];"),
    "stream_no_rescale": ("for (int c = 0; c < d; ++c) acc[c] *= alpha;",
                          "for (int c = 0; c < d; ++c) acc[c] *= 1.0;"),
    "lse_drop_max": ("return m + log(l);", "return log(l);"),
    "o_missing_normalise": ("for (int j = 0; j < len; ++j) prow[j] /= l;",
                            "for (int j = 0; j < len; ++j) prow[j] /= 1.0;"),
}


def _compile(tmp_path, name, src_text):
    c = tmp_path / (name + ".c")
    so = tmp_path / ("lib" + name + ".so")
    c.write_text(src_text)
    subprocess.run(["gcc", "-O1", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o",
                    str(so), str(c), "-lm"], check=True)
    return str(so)


def _battery():
    """Returns the list of failed pin names for the currently loaded oracle."""
    failed = []
    rng = np.random.default_rng(7)

    # brute force, GQA, causal and not
    for causal in (False, True):
        n, Hq, Hkv, d = 4, 4, 2, 3
        q = rng.standard_normal((1, n, Hq, d))
        k = rng.standard_normal((1, n, Hkv, d))
        v = rng.standard_normal((1, n, Hkv, d))
        do = rng.standard_normal((1, n, Hq, d))
        o, lse = oracle.attention_fwd(q, k, v, 0.7, causal)
        g = oracle.attention_bwd(q, k, v, do, 0.7, causal)
        bo, bl = brute.forward(q[0].tolist(), k[0].tolist(), v[0].tolist(), 0.7, causal)
        bq, bk, bv = brute.backward(q[0].tolist(), k[0].tolist(), v[0].tolist(),
                                    do[0].tolist(), 0.7, causal)
        for nm, a, b in (("o", o[0], bo), ("lse", lse[0], bl), ("dq", g["dq"][0], bq),
                         ("dk", g["dk"][0], bk), ("dv", g["dv"][0], bv)):
            if not np.allclose(a, np.array(b), atol=1e-11, rtol=0):
                failed.append("brute_%s_causal%d" % (nm, causal))

    # uniform V
    q = rng.standard_normal((1, 9, 2, 4))
    k = rng.standard_normal((1, 9, 2, 4))
    row = rng.standard_normal(4)
    v = np.broadcast_to(row, (1, 9, 2, 4)).copy()
    o, _ = oracle.attention_fwd(q, k, v, 0.5, True)
    if not np.allclose(o, np.broadcast_to(row, o.shape), atol=1e-12):
        failed.append("uniform_v")

    # causal first row
    v = rng.standard_normal((1, 9, 2, 4))
    o, lse = oracle.attention_fwd(q, k, v, 0.5, True)
    if not np.allclose(o[:, 0], v[:, 0], atol=1e-13):
        failed.append("causal_row0")
    if abs(lse[0, 0, 0] - 0.5 * float(q[0, 0, 0] @ k[0, 0, 0])) > 1e-12:
        failed.append("causal_row0_lse")

    # streaming recurrence vs three-pass
    n, d = 50, 4
    qs = rng.standard_normal((n, d)) * 3
    ks, vs = rng.standard_normal((n, d)), rng.standard_normal((n, d))
    o_ref, l_ref = oracle.attention_fwd(qs[None, :, None], ks[None, :, None],
                                        vs[None, :, None], 0.5, False)
    o_s, l_s = oracle.attention_fwd_streaming(qs, ks, vs, 0.5, False, 7,
                                              rng.permutation((n + 6) // 7))
    if not (np.allclose(o_s, o_ref[0, :, 0], atol=1e-11) and np.allclose(l_s, l_ref[0, 0], atol=1e-11)):
        failed.append("streaming")

    # finite differences (GQA g=2, causal)
    N, Hq, Hkv, d = 6, 2, 1, 4
    q = rng.standard_normal((1, N, Hq, d))
    k = rng.standard_normal((1, N, Hkv, d))
    v = rng.standard_normal((1, N, Hkv, d))
    do = rng.standard_normal((1, N, Hq, d))
    g = oracle.attention_bwd(q, k, v, do, 0.5, True)

    def loss():
        o, _ = oracle.attention_fwd(q, k, v, 0.5, True)
        return float(np.sum(o * do))

    h = 1e-6
    for nm, arr in (("dq", q), ("dk", k), ("dv", v)):
        ok = True
        for ix in [(0, 3, 0, 1), (0, 5, 0, 2)] if nm != "dq" else [(0, 3, 1, 1), (0, 5, 0, 2)]:
            a0 = arr[ix]
            arr[ix] = a0 + h
            lp = loss()
            arr[ix] = a0 - h
            lm = loss()
            arr[ix] = a0
            if abs((lp - lm) / (2 * h) - g[nm][ix]) > 1e-5 * max(1, abs(g[nm][ix])):
                ok = False
        if not ok:
            failed.append("fd_" + nm)
    return failed


def test_unmodified_oracle_passes_battery():
    assert _battery() == []


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(tmp_path, name):
    src = open(SRC).read()
    old, new = MUTANTS[name]
    assert src.count(old) >= 1, "mutation anchor not found: %s" % name
    so = _compile(tmp_path, name, src.replace(old, new, 1))
    with oracle.use_library(so):
        failed = _battery()
    assert failed, "planted mistake %s was not caught by any pin" % name
