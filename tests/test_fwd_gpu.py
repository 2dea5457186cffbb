"""Forward parity: CUDA path (through the C ABI) vs the fp64 oracle on the
same seeded bf16 inputs, over sizes that span several tiles and ragged tails,
plus edge cases (N = 1, empty and length-1 sequences, GQA, causal tile
boundaries) and guard-band canaries around the outputs."""
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
    ("n300_d64", lambda: workloads.custom("n300_d64", 2, 3, 3, 300, 64, False)),
    ("n300_d64_causal", lambda: workloads.custom("n300_d64_c", 2, 3, 3, 300, 64, True)),
    ("n300_d128_causal", lambda: workloads.custom("n300_d128_c", 2, 3, 3, 300, 128, True)),
    ("n1_d64", lambda: workloads.custom("n1_d64", 2, 2, 1, 1, 64, True)),
    ("n1_d128", lambda: workloads.custom("n1_d128", 1, 1, 1, 1, 128, False)),
    ("n129_d64_causal", lambda: workloads.custom("n129", 1, 2, 2, 129, 64, True)),
    ("gqa4_n384_d128_causal", lambda: workloads.custom("gqa", 2, 8, 2, 384, 128, True)),
    ("gqa8_n640_d64", lambda: workloads.custom("gqa8", 1, 8, 1, 640, 64, False)),
    ("x8row_n1024_d64", lambda: workloads.custom("x8", 1, 4, 4, 1024, 64, True, x8_row=True)),
]


@pytest.mark.parametrize("name,mk", CASES, ids=[c[0] for c in CASES])
def test_fwd_matches_oracle(name, mk):
    inp = workloads.generate(mk())
    ops.fa_clear_device_error()
    o, lse = parity.gpu_fwd(inp)
    parity.no_device_error()
    parity.check_fwd(inp, o, lse)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_fwd_varlen_edge_lengths(d, causal):
    inp = workloads.from_lengths("vl", [1, 129, 300, 0, 517, 128, 64, 255, 256, 257], 4, 2, d,
                                 causal)
    o, lse = parity.gpu_fwd(inp)
    parity.no_device_error()
    parity.check_fwd(inp, o, lse)


@pytest.mark.parametrize("wname", ["gpt2_small_causal_b8_h12_n1024_d64",
                                   "bert_large_varlen_32x128to512_h16_d64"])
def test_fwd_full_config(wname):
    inp = workloads.generate(workloads.WORKLOADS[wname])
    o, lse = parity.gpu_fwd(inp)
    parity.no_device_error()
    parity.check_fwd(inp, o, lse)


def test_fwd_guard_bands_untouched():
    """Outputs are written in place inside larger buffers; the bytes around
    them must keep their canary pattern (no out-of-bounds writes)."""
    inp = workloads.from_lengths("canary", [5, 200, 1, 333], 4, 2, 128, True)
    dev = parity.to_dev(inp)
    total, H, d = inp.q.shape
    pad = 4096
    obuf = torch.full((total * H * d + 2 * pad,), 7.0, dtype=torch.bfloat16, device="cuda")
    lbuf = torch.full((total * H + 2 * pad,), -3.0, dtype=torch.float32, device="cuda")
    o = obuf[pad:pad + total * H * d].view(total, H, d)
    lse = lbuf[pad:pad + total * H].view(H, total)
    ops.attention_fwd(dev["q"], dev["k"], dev["v"], inp.workload.scale, True, dev["cu"], 333,
                      out=o, lse=lse)
    torch.cuda.synchronize()
    parity.no_device_error()
    assert bool((obuf[:pad] == 7.0).all()) and bool((obuf[-pad:] == 7.0).all())
    assert bool((lbuf[:pad] == -3.0).all()) and bool((lbuf[-pad:] == -3.0).all())
    parity.check_fwd(inp, o, lse)


def test_fwd_repeatable():
    inp = workloads.generate(workloads.custom("rep", 1, 2, 1, 700, 128, True))
    dev = parity.to_dev(inp)
    o1, l1 = parity.gpu_fwd(inp, dev)
    o2, l2 = parity.gpu_fwd(inp, dev)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_watchdog_gives_up_and_reports():
    """A wait on an mbarrier nothing arrives on must time out, record its
    code and return; afterwards the context still works."""
    ops.fa_clear_device_error()
    ops.fa_set_wait_limit_ns(2_000_000)   # 2 ms
    try:
        st = ops.fa_watchdog_selftest(ops._stream())
        assert st == 0
        torch.cuda.synchronize()
        assert ops.fa_device_error() == 0x301
    finally:
        ops.fa_set_wait_limit_ns(2_000_000_000)
        ops.fa_clear_device_error()
    inp = workloads.generate(workloads.WORKLOADS["single_head_n128_d64"])
    o, lse = parity.gpu_fwd(inp)
    parity.no_device_error()
    parity.check_fwd(inp, o, lse)
