"""Standard attention against the tiled forward, on one GPU.

Standard attention ("注意力机制基础" 2.1, 2.2.2) writes S = Q K^T to device
memory, reads it back for the row softmax, writes P, and reads P again for
O = P V: 2 (4 N^2 + 4 N d) bytes per head at 16-bit elements, against
about 2 (4 N d) for the tiled forward, which keeps S and P on chip
("FlashAttention优化" 3.1, 4.1; paper review 方法 item 1).  This module times
both on the same inputs and prints one JSON line per (N, d):

    python -m exact_io_aware_67_b200.compare_standard [--sizes 1024,4096,16384]
        [--dims 64,128] [--heads 16] [--causal] [--steps 10] [--warmup 3]
        [--only both|standard|flash]

Besides the times, each side's device memory beyond its inputs is measured
(the peak the allocator saw during one call): S and P make it grow as N^2
for standard attention, against O and LSE, linear in N, for the tiled
forward (paper review 结果; "注意力机制基础" 2.2.2's memory column).  When
S and P (2 heads N^2 bf16) exceed the free device memory less a 4 GiB
margin, the standard side is skipped and reports the bytes it would need,
so that no allocation is ever made to fail; the tiled side still runs.

Times are CUDA events on the launching stream, after warm-up.  Between timed
iterations the L2 cache is flushed by writing a buffer larger than it, so
that small problems do not run from L2.  The standard pipeline is
ops.standard_attention_fwd (two library GEMMs around fa_std_softmax); its
softmax kernel is also timed alone, against the HBM roofline of its
4 N^2 bytes per head.  The flash side is fa_fwd.  Inputs are seeded N(0,1)
bf16.
"""
import argparse
import json
import os

import torch

from . import ops
from .flops import standard_attention_hbm_bytes

L2_FLUSH_BYTES = 256 << 20


def _peaks():
    p = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                     "MEASURED_PEAKS.json")
    try:
        return json.load(open(p))
    except (OSError, ValueError):
        return {}


def _time(fn, steps, warmup, flush):
    for _ in range(warmup):
        fn()
    start = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    end = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    for i in range(steps):
        flush.zero_()
        start[i].record()
        fn()
        end[i].record()
    torch.cuda.synchronize()
    ts = sorted(s.elapsed_time(e) for s, e in zip(start, end))
    return ts[len(ts) // 2]


def _extra_bytes(fn):
    """Peak device memory one call of fn allocates beyond what was live."""
    torch.cuda.synchronize()
    base = torch.cuda.memory_allocated()
    torch.cuda.reset_peak_memory_stats()
    r = fn()
    torch.cuda.synchronize()
    peak = torch.cuda.max_memory_allocated() - base
    del r
    return peak


def run(N, d, heads, causal, steps, warmup, only, flush):
    g = torch.Generator(device="cuda").manual_seed(N * 1000 + d)
    q, k, v = (torch.randn((1, heads, N, d), generator=g, device="cuda").to(torch.bfloat16)
               for _ in range(3))
    scale = d ** -0.5
    out = {"N": N, "d": d, "heads": heads, "batch": 1, "causal": bool(causal)}
    if only in ("both", "standard"):
        need = 2 * heads * N * N * 2          # S and P, bf16
        free, _ = torch.cuda.mem_get_info()
        if need > free - (4 << 30):
            out["standard_skipped_bytes_needed"] = need
            out["device_free_bytes"] = free
            only = "flash"
        else:
            out["standard_extra_bytes"] = _extra_bytes(
                lambda: ops.standard_attention_fwd(q, k, v, scale, causal))
    if only in ("both", "standard"):
        ms = _time(lambda: ops.standard_attention_fwd(q, k, v, scale, causal), steps, warmup,
                   flush)
        out["standard_ms"] = ms
        model = heads * standard_attention_hbm_bytes(N, d)
        out["standard_model_bytes"] = model
        out["standard_model_gbs"] = model / (ms * 1e-3) / 1e9
        # the softmax step alone (S already in memory)
        s = torch.matmul(q, k.transpose(-1, -2))
        p = torch.empty_like(s)
        lse = torch.empty((1, heads, N), dtype=torch.float32, device="cuda")

        def softmax():
            st = ops.fa_std_softmax(ops._ptr(s), ops._ptr(p), ops._ptr(lse), heads, N, scale,
                                    causal, ops._stream())
            if st != 0:
                raise ops.FAError("fa_std_softmax", st)

        sms = _time(softmax, steps, warmup, flush)
        sbytes = heads * 4 * N * N
        out["softmax_ms"] = sms
        out["softmax_bytes"] = sbytes
        out["softmax_gbs"] = sbytes / (sms * 1e-3) / 1e9
        hbm = _peaks().get("hbm_gbs")
        if hbm:
            out["softmax_frac_of_measured_hbm"] = out["softmax_gbs"] / hbm
        del s, p, lse
    if only in ("both", "flash"):
        qt, kt, vt = (t.transpose(1, 2).contiguous() for t in (q, k, v))   # [1, N, H, d]
        out["flash_extra_bytes"] = _extra_bytes(lambda: ops.attention_fwd(qt, kt, vt, scale,
                                                                          causal))
        fms = _time(lambda: ops.attention_fwd(qt, kt, vt, scale, causal), steps, warmup, flush)
        out["flash_fwd_ms"] = fms
        out["flash_model_bytes"] = heads * 2 * (4 * N * d) + heads * 4 * N
        if "standard_ms" in out:
            out["speedup"] = out["standard_ms"] / fms
    return out


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--sizes", default="1024,4096,16384")
    ap.add_argument("--dims", default="64,128")
    ap.add_argument("--heads", type=int, default=16)
    ap.add_argument("--causal", action="store_true")
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--only", default="both", choices=["both", "standard", "flash"])
    a = ap.parse_args(argv)
    if not torch.cuda.is_available():
        raise SystemExit("compare_standard needs a CUDA device")
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    for N in (int(x) for x in a.sizes.split(",")):
        for d in (int(x) for x in a.dims.split(",")):
            r = run(N, d, a.heads, a.causal, a.steps, a.warmup, a.only, flush)
            print(json.dumps(r), flush=True)
            torch.cuda.empty_cache()


if __name__ == "__main__":
    main()
