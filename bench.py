"""Benchmark: exact attention forward + backward on B200 (TFLOP/s and % of
dense BF16 tensor peak).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl {b200,reference}] [--no-cpu-baseline] [--no-e2e]

One step = fa_fwd (O, LSE) + fa_bwd (dQ, dK, dV) over one batch of the
workload, all through the C ABI of libfa.so.  FLOPs: forward 4 B H N^2 d
(halved for causal), backward 2.5x forward.  Prints ONE JSON line (rank 0).

A decode workload (``--workload decode_*``) times one decode step over a
KV cache instead (fa_decode: split-KV attention of one new token per
sequence); it is bound by HBM bandwidth, so that line reports GB/s of the
algorithmic bytes (the valid K and V cache rows, q, o, lse) against the
measured copy bandwidth.

Multi-GPU (torchrun, one process per GPU): the path partitions into
independent (sequence, kv-head group) problems, so each rank runs its own
batch of the same shape (weak scaling) with no data-path collective; the
host-side barrier and a max-reduction of the elapsed time are the only
communication.  ``--impl reference`` times the CPU fp64 oracle instead (the
reference arm; rank 0 only).
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = ("attention fwd+bwd TFLOP/s (bf16, 1×B200) and % of dense BF16 tensor peak")
DECODE_METRIC = "decode attention over a KV cache: GB/s of K/V cache read (bf16, 1×B200)"
SPARSE_METRIC = ("block-sparse attention fwd+bwd TFLOP/s on the allowed (query, key) pairs "
                 "(bf16, 1×B200) and % of dense BF16 tensor peak")
L2_FLUSH_BYTES = 256 << 20
DEFAULT_WORKLOAD = "long_causal_b1_h16_n65536_d128_x8row"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# SM clock at which the measured sustained bf16 figure was taken, when the
# peaks file does not record it (1342 MHz under the 1000 W cap)
SUSTAINED_PEAK_MHZ = 1342.0


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(values, device=None):
    """Element-wise max of a list of floats over all ranks of the default
    process group (identity without one).  The only cross-rank traffic of the
    benchmark besides barriers."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.cpu()]


def weak_scaling_value(world_size, flops_per_step_per_rank, steps, ms_max):
    """Whole-job TFLOP/s: every rank processed `steps` steps of its own batch;
    the job took as long as the slowest rank."""
    return world_size * flops_per_step_per_rank * steps / (ms_max / 1e3) / 1e12


def rank_workload(w, rank):
    """Rank r's batch: same shape, its own seed (the ranks hold disjoint
    independent problems, so nothing is exchanged)."""
    from exact_io_aware_67_b200 import workloads
    return workloads.Workload(**{**w.__dict__, "seed": w.seed + rank})


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi sampled every 200 ms during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append(dict(sm=float(parts[1]), smax=float(parts[2]),
                                 power=float(parts[3]) if parts[3] not in ("[N/A]", "") else None,
                                 hw=parts[5], hwt=parts[6], swt=parts[7], swp=parts[8]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        load = [r for r in rows if r["power"] is None or r["power"] > 300] or rows
        reasons = set()
        for r in load:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("swp", "sw_power_cap")):
                if r[key].lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in load),
                "sm_max_mhz": max(r["smax"] for r in rows),
                "reasons": sorted(reasons), "samples": len(rows), "samples_under_load": len(load)}


# ------------------------------------------------------------------ CPU oracle
_INPUTS = {}


def _inputs(w):
    """The workload's seeded inputs, drawn once per process."""
    from exact_io_aware_67_b200 import workloads
    key = (w.name, w.seed)
    if key not in _INPUTS:
        _INPUTS.clear()
        _INPUTS[key] = workloads.generate(w)
    return _INPUTS[key]


def cpu_rows_sample(w, nrows, nthreads, seed=0, problems=2):
    """fp64 oracle on `nrows` query rows of workload w at seeded positions,
    split over `problems` (batch, query head) problems (the first and the
    last, then evenly spaced ones): O, LSE, D and dQ of each row (the
    oracle's row sampler; those outputs depend on the row alone).  Each
    problem's rows go to the oracle in one call, so its threads share them.
    Returns (seconds, flops, description).  FLOPs count the work the
    definition does for those rows: 2 d per allowed key for each of S,
    O = P V, dP and dQ, i.e. 8 d per allowed key."""
    import numpy as np
    import oracle
    inp = _inputs(w)
    g = w.Hq // w.Hkv
    rng = np.random.default_rng(seed)
    total = w.B * w.Hq
    npb = max(1, min(problems, total))
    picks = sorted(set(int(round(x)) for x in np.linspace(0, total - 1, npb)))
    secs, flops, used = 0.0, 0.0, 0
    for n, u in enumerate(picks):
        b, h = divmod(u, w.Hq)
        take = nrows // len(picks) + (1 if n < nrows % len(picks) else 0)
        if inp.cu_seqlens is None:
            sl = lambda t, hh: t[b, :, hh]
            L = w.N
        else:
            st = int(inp.cu_seqlens[b])
            L = int(inp.cu_seqlens[b + 1]) - st
            sl = lambda t, hh: t[st:st + L, hh]
        if L == 0 or take == 0:
            continue
        one = lambda t, hh: sl(t, hh)[None, :, None, :].float().numpy().astype(np.float64)
        q, k, v, do = one(inp.q, h), one(inp.k, h // g), one(inp.v, h // g), one(inp.dout, h)
        rows = rng.integers(0, L, take)
        sel = np.stack([np.zeros_like(rows), np.zeros_like(rows), rows], axis=1)
        t0 = time.perf_counter()
        oracle.attention_rows(q, k, v, do, sel, w.scale, w.causal, nthreads=nthreads)
        secs += time.perf_counter() - t0
        keys = (rows + 1) if w.causal else np.full_like(rows, L)
        flops += 8.0 * w.d * float(keys.sum())
        used += take
    desc = ("%d query rows of %s at seeded positions in %d (batch, query head) problems: fp64 "
            "oracle O, LSE, D and dQ of each row; FLOPs = 8 d per allowed key" %
            (used, w.name, len(picks)))
    return secs, flops, desc


def cpu_model():
    """The host CPU's model name (first processor in /proc/cpuinfo)."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def rows_for_seconds(w, seconds, nthreads):
    """Rows that take the oracle about `seconds` on `nthreads` threads,
    calibrated on a short probe of the same workload."""
    probe = max(64, nthreads * 16)
    dt, _, _ = cpu_rows_sample(w, probe, nthreads, seed=12345)
    rate = probe / max(dt, 1e-6)
    return max(nthreads, int(rate * seconds))


def cpu_per_core(w):
    """TFLOP/s of the oracle's row sampler on one thread (a few rows of the
    same workload): the per-core figure beside the all-cores one."""
    dt, f, _ = cpu_rows_sample(w, 8, 1, seed=777, problems=1)
    return f / max(dt, 1e-9) / 1e12


def run_reference(args, w):
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    cores = len(os.sched_getaffinity(0))
    # each step is a bounded sample (about 3 s of oracle time, less when
    # many steps are asked for), so that the whole --steps/--warmup run stays
    # within about three minutes
    per_step_s = min(3.0, max(0.1, 150.0 / max(1, args.steps + args.warmup)))
    nrows = rows_for_seconds(w, per_step_s, cores)
    for it in range(args.warmup):
        cpu_rows_sample(w, nrows, cores, seed=1000 + it)
    times, flops, desc = [], [], ""
    for it in range(args.steps):
        dt, f, desc = cpu_rows_sample(w, nrows, cores, seed=it)
        times.append(dt)
        flops.append(f)
    tot = sum(times)
    value = sum(flops) / tot / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
            "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * tot / len(times), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, **w.describe()},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores,
                             "kind": "oracle", "sample": "per step: " + desc,
                             "cpu_model": cpu_model(), "per_core_value": cpu_per_core(w)},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def peak_for_clock(peaks, clk):
    """The dense bf16 peak that applies to a run at the clocks it was sampled
    at: the measured sustained cuBLAS figure scaled from the SM clock it was
    measured at to this run's median SM clock, capped at the burst figure
    (the cap applies whenever the run held its clock).  Returns (peak,
    source note)."""
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    sus = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    sus_mhz = None
    for key, val in peaks.items():
        kl = key.lower()
        if "sustained" in kl and ("mhz" in kl or "clock" in kl):
            try:
                sus_mhz = float(val)
                break
            except (TypeError, ValueError):
                continue
    if sus_mhz is None:
        sus_mhz = SUSTAINED_PEAK_MHZ
    mhz = clk.get("sm_mhz")
    if not mhz:
        return burst, "bf16_tflops (burst; no clock samples)"
    scaled = sus * float(mhz) / sus_mhz
    if scaled >= burst:
        return burst, "bf16_tflops (burst; clock-scaled sustained figure %.0f is higher)" % scaled
    return scaled, ("bf16_tflops_sustained %.1f at %.0f MHz scaled to the run's median %.0f MHz"
                    % (sus, sus_mhz, mhz))


# ------------------------------------------------------------------ GPU arm
def run_b200(args, w):
    import torch
    import torch.distributed as dist
    from exact_io_aware_67_b200 import flops, ops, workloads

    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    if ws > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    # each rank draws its own batch of the same shape (weak scaling)
    wr = rank_workload(w, rank)
    inp = workloads.generate(wr)
    lengths = inp.lengths
    q, k, v, do = (t.to(dev) for t in (inp.q, inp.k, inp.v, inp.dout))
    cu = None if inp.cu_seqlens is None else inp.cu_seqlens.to(dev)
    maxlen = (max(lengths) if lengths else w.N) if cu is not None else None
    o = torch.empty_like(q)
    o_lo = torch.empty_like(q)      # O's rounding residual, read back by the backward
    lse = torch.empty((w.B, w.Hq, w.N) if cu is None else (w.Hq, q.shape[0]),
                      dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws_buf = ops.workspace_for(q, k, cu, maxlen)
    fwd_f = flops.fwd_flops(w, lengths)
    bwd_f = flops.bwd_flops(w, lengths)
    step_f = fwd_f + bwd_f
    stream = torch.cuda.current_stream()

    def step():
        ops.attention_fwd(q, k, v, w.scale, w.causal, cu, maxlen, out=o, lse=lse, o_lo=o_lo)
        ops.attention_bwd(q, k, v, o, lse, do, w.scale, w.causal, cu, maxlen,
                          workspace=ws_buf, dq=dq, dk=dk, dv=dv, o_lo=o_lo)

    ops.fa_clear_device_error()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    # per-kernel events: forward kernel and backward main kernel of every step
    # (recorded by the library around those kernels), then the whole backward
    # call (preprocess, main and dQ-convert kernels) on the same stream
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
    for row in ev:
        for e in row:
            e.record(stream)
    torch.cuda.synchronize()
    t_begin = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_begin.record(stream)
    for s in range(args.steps):
        ops.fa_set_profile_events(ev[s][0], ev[s][1])
        ops.attention_fwd(q, k, v, w.scale, w.causal, cu, maxlen, out=o, lse=lse, o_lo=o_lo)
        ops.fa_set_profile_events(ev[s][2], ev[s][3])
        ev[s][4].record(stream)
        ops.attention_bwd(q, k, v, o, lse, do, w.scale, w.causal, cu, maxlen,
                          workspace=ws_buf, dq=dq, dk=dk, dv=dv, o_lo=o_lo)
        ev[s][5].record(stream)
    ops.fa_set_profile_events(None, None)
    t_end.record(stream)
    torch.cuda.synchronize()
    if ws > 1:
        dist.barrier()
    clk = clocks.stop()
    ms = t_begin.elapsed_time(t_end)
    fwd_ms = [ev[s][0].elapsed_time(ev[s][1]) for s in range(args.steps)]
    bwd_ms = [ev[s][2].elapsed_time(ev[s][3]) for s in range(args.steps)]
    bwd_all_ms = [ev[s][4].elapsed_time(ev[s][5]) for s in range(args.steps)]
    err = ops.fa_device_error()
    if err != 0:
        raise RuntimeError("device error word 0x%x during the timed region" % err)

    # ---------------------------------------------------------------- e2e
    # Every step copies its inputs in from pinned host memory and its results
    # (O, dQ, dK, dV) out.  Two device buffer sets and three streams (copy-in,
    # compute, copy-out) let step s+1's inputs upload and step s-1's results
    # download while step s computes, as a training loop would overlap them;
    # the time runs from the first upload to the last download (CUDA events).
    e2e = None
    if not args.no_e2e:
        hq = [t.pin_memory() for t in (inp.q, inp.k, inp.v, inp.dout)]
        hout = [[torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in (o, dq, dk, dv)]
                for _ in range(2)]
        din = [[q, k, v, do], [torch.empty_like(t) for t in (q, k, v, do)]]
        dout_ = [[o, dq, dk, dv], [torch.empty_like(t) for t in (o, dq, dk, dv)]]
        lses = [lse, torch.empty_like(lse)]
        olos = [o_lo, torch.empty_like(o_lo)]
        wss = [ws_buf, torch.empty_like(ws_buf)]
        h2d = sum(t.numel() * t.element_size() for t in hq)
        d2h = sum(t.numel() * t.element_size() for t in hout[0])
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_cmp = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]
        for e_ in ev_cmp + ev_out:
            e_.record(stream)

        def e2e_step(it):
            x = it & 1
            qq, kk, vv, dd = din[x]
            oo, gq, gk, gv = dout_[x]
            with torch.cuda.stream(s_in):
                s_in.wait_event(ev_cmp[x])          # step it-2 done reading these inputs
                for dst, src in zip(din[x], hq):
                    dst.copy_(src, non_blocking=True)
                ev_in[x].record(s_in)
            stream.wait_event(ev_in[x])
            stream.wait_event(ev_out[x])             # step it-2's results downloaded
            ops.attention_fwd(qq, kk, vv, w.scale, w.causal, cu, maxlen, out=oo, lse=lses[x],
                              o_lo=olos[x])
            ops.attention_bwd(qq, kk, vv, oo, lses[x], dd, w.scale, w.causal, cu, maxlen,
                              workspace=wss[x], dq=gq, dk=gk, dv=gv, o_lo=olos[x])
            ev_cmp[x].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_cmp[x])
                for dst, src in zip(hout[x], dout_[x]):
                    dst.copy_(src, non_blocking=True)
                ev_out[x].record(s_out)

        e2e_steps = min(args.steps, 50)
        for it in range(2):                          # warm-up of the pipeline
            e2e_step(it)
        torch.cuda.synchronize()
        if ws > 1:
            dist.barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(s_in)
        for it in range(e2e_steps):
            e2e_step(it)
        e1.record(s_out)
        torch.cuda.synchronize()
        e2e_ms = e0.elapsed_time(e1)
        e2e = {"ms": e2e_ms * args.steps / e2e_steps, "h2d": h2d, "d2h": d2h}

    # ---------------------------------------------------------------- reduce
    ms_max, e2e_max = max_over_ranks([ms, e2e["ms"] if e2e else 0.0], device=dev)
    if ws > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0

    peaks, peaks_src = load_peaks()
    value = weak_scaling_value(ws, step_f, args.steps, ms_max)
    fwd_avg = sum(fwd_ms) / len(fwd_ms)
    bwd_avg = sum(bwd_ms) / len(bwd_ms)
    fwd_tf = fwd_f / (fwd_avg / 1e3) / 1e12
    bwd_tf = bwd_f / (bwd_avg / 1e3) / 1e12
    bwd_all_tf = bwd_f / (sum(bwd_all_ms) / len(bwd_all_ms) / 1e3) / 1e12
    peak, peak_kind = peak_for_clock(peaks, clk)
    peak_burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    # dominant kernel: the one with the larger share of the step
    if bwd_avg >= fwd_avg:
        dom, dom_ms, dom_f = "bwd_main_kernel", bwd_avg, bwd_f
    else:
        dom, dom_ms, dom_f = "fwd_kernel", fwd_avg, fwd_f
    achieved = dom_f / (dom_ms / 1e3) / 1e12
    traffic = load_traffic(dom, w.name)
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16 inputs of the workload's shape)",
        "config": {"workload": w.name, **w.describe(),
                   "l2": "inputs larger than L2 (%.0f MB touched per step)" %
                         (bytes_per_step(q, k, v, o, do, dq, dk, dv, ws_buf) / 1e6),
                   "parallelism": "independent batches per GPU" if ws > 1 else "1 GPU"},
        "pct_of_peak": 100.0 * value / ws / peak,
        "fwd_tflops": fwd_tf, "bwd_tflops": bwd_tf,
        "fwd_pct_of_peak": 100.0 * fwd_tf / peak, "bwd_pct_of_peak": 100.0 * bwd_tf / peak,
        # the whole backward call: preprocess + main + dQ-convert kernels
        "bwd_all_tflops": bwd_all_tf, "bwd_all_pct_of_peak": 100.0 * bwd_all_tf / peak,
        "peak_tflops": peak, "peak_source": "%s %s" % (peaks_src, peak_kind),
        "roofline": {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": peak,
                     "unit": "TFLOP/s", "frac": achieved / peak,
                     "frac_of_burst_peak": achieved / peak_burst,
                     "traffic": traffic,
                     "algorithmic_flops_per_launch": dom_f, "avg_launch_ms": dom_ms},
        "gpu_launches": 5 * args.steps,
        "clocks": clk,
    }
    if e2e:
        line["e2e"] = {"value": weak_scaling_value(ws, step_f, args.steps, e2e_max),
                       "unit": "TFLOP/s", "h2d_bytes_per_step": e2e["h2d"],
                       "d2h_bytes_per_step": e2e["d2h"],
                       "ms_per_step": e2e_max / args.steps}
    if not args.no_cpu_baseline and ws == 1:
        # a bounded sample of the same workload: about 15 s of oracle time
        cores = len(os.sched_getaffinity(0))
        nrows = rows_for_seconds(w, 15.0, cores)
        dt, f, desc = cpu_rows_sample(w, nrows, cores)
        line["cpu_baseline"] = {
            "value": f / dt / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "seconds": dt, "sample": desc, "cpu_model": cpu_model(),
            "per_core_value": cpu_per_core(w)}
    print(json.dumps(line), flush=True)
    return 0


def bytes_per_step(*ts):
    return sum(t.numel() * t.element_size() for t in ts)


def load_traffic(kernel, workload):
    """DRAM bytes per launch from a committed ncu summary, if one exists for
    this kernel and workload and the kernel sources are unchanged since."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        d = json.load(open(p))
        ent = d.get(kernel, {}).get(workload)
        if not ent:
            return None
        if kernel not in KERNEL_SOURCES or ent.get("source_sha") != source_sha(kernel):
            return None
        return ent.get("dram_bytes_per_launch")
    except Exception:
        return None


# the sources a kernel's DRAM traffic depends on: its own header, the shared
# helpers, and the host file that sets its launch configuration
KERNEL_SOURCES = {
    "fwd_kernel": ("fa_fwd.cuh", "fa_common.cuh", "sm100.cuh", "fa_api.cu"),
    "bwd_main_kernel": ("fa_bwd.cuh", "fa_common.cuh", "sm100.cuh", "fa_api.cu"),
}


def source_sha(kernel):
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "exact_io_aware_67_b200", "csrc")
    for f in KERNEL_SOURCES[kernel]:
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


# ------------------------------------------------------------------ block-sparse
def run_blocksparse(args, bw):
    """fa_fwd_blockmask + fa_bwd_blockmask on one GPU; FLOPs counted on the
    allowed (query, key) pairs only (what the kernels must compute)."""
    import torch
    from exact_io_aware_67_b200 import flops, ops, workloads
    ws, rank, local = dist_env()
    if ws > 1 or args.impl == "reference":
        if rank == 0:
            print(json.dumps({"impl": args.impl, "metric": SPARSE_METRIC,
                              "unavailable": "block-sparse workloads run on one GPU, b200 arm only"}))
        return 0
    torch.cuda.set_device(local)
    w = bw.base
    inp = workloads.generate(w)
    mask = workloads.block_mask(bw)
    q, k, v, do = (t.cuda() for t in (inp.q, inp.k, inp.v, inp.dout))
    bm = torch.from_numpy(mask).cuda()
    lse = torch.empty((w.B, w.Hq, w.N), dtype=torch.float32, device="cuda")
    o = torch.empty_like(q)
    o_lo = torch.empty_like(q)
    wsb = torch.empty(ops.fa_bwd_workspace_size(w.B, w.Hq, w.N, w.d, w.B * w.N),
                      dtype=torch.uint8, device="cuda")
    fwd_f = flops.blocksparse_fwd_flops(bw, mask)
    bwd_f = 2.5 * fwd_f
    stream = torch.cuda.current_stream()

    def step(evs=None):
        if evs:
            ops.fa_set_profile_events(evs[0], evs[1])
        ops.attention_fwd_blockmask(q, k, v, bm, w.scale, w.causal, out=o, lse=lse, o_lo=o_lo)
        if evs:
            ops.fa_set_profile_events(evs[2], evs[3])
        ops.attention_bwd_blockmask(q, k, v, o, lse, do, bm, w.scale, w.causal, workspace=wsb,
                                    o_lo=o_lo)
        if evs:
            ops.fa_set_profile_events(None, None)

    ops.fa_clear_device_error()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    for row in ev:   # the library records them later; torch must know they exist
        for e in row:
            e.record(stream)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    torch.cuda.synchronize()
    t0.record(stream)
    for s_ in range(args.steps):
        step(ev[s_])
    t1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    if ops.fa_device_error() != 0:
        raise RuntimeError("device error word 0x%x" % ops.fa_device_error())
    ms = t0.elapsed_time(t1)
    fwd_ms = sum(e[0].elapsed_time(e[1]) for e in ev) / args.steps
    bwd_ms = sum(e[2].elapsed_time(e[3]) for e in ev) / args.steps
    peaks, src = load_peaks()
    peak, peak_kind = peak_for_clock(peaks, clk)
    fwd_tf = fwd_f / (fwd_ms / 1e3) / 1e12
    bwd_tf = bwd_f / (bwd_ms / 1e3) / 1e12
    dom, dom_ms, dom_f = (("bwd_main_kernel", bwd_ms, bwd_f) if bwd_ms >= fwd_ms
                          else ("fwd_kernel", fwd_ms, fwd_f))
    value = (fwd_f + bwd_f) * args.steps / (ms / 1e3) / 1e12
    line = {"metric": SPARSE_METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) bf16 inputs of the workload's shape)",
            "config": {"workload": bw.name, **bw.describe(),
                       "allowed_tile_fraction": float(mask.mean()),
                       "l2": "inputs larger than L2", "parallelism": "1 GPU"},
            "fwd_tflops": fwd_tf, "bwd_tflops": bwd_tf,
            "fwd_pct_of_peak": 100 * fwd_tf / peak, "bwd_pct_of_peak": 100 * bwd_tf / peak,
            "roofline": {"bound": "tensor", "kernel": dom,
                         "achieved": dom_f / (dom_ms / 1e3) / 1e12, "peak": peak,
                         "unit": "TFLOP/s", "frac": dom_f / (dom_ms / 1e3) / 1e12 / peak,
                         "traffic": None, "algorithmic_flops_per_launch": dom_f,
                         "avg_launch_ms": dom_ms, "peak_source": "%s %s" % (src, peak_kind)},
            "gpu_launches": 5 * args.steps, "clocks": clk}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ decode
def decode_bytes(w, lengths):
    """Algorithmic bytes of one decode step: every valid K and V cache row
    read once, q read, o written (bf16) and lse written (fp32)."""
    kv = sum(lengths) * w.Hkv * w.d * 2 * 2
    return kv + w.B * w.Hq * w.d * 2 * 2 + w.B * w.Hq * 4


def decode_cpu_sample(w, inp, nthreads, seqs=1):
    """The oracle on `seqs` sequences of the decode step (every query head):
    returns (seconds, algorithmic bytes of that sample)."""
    import numpy as np
    import oracle
    lens = inp.lengths
    t0 = time.perf_counter()
    nbytes = 0
    for b in range(seqs):
        L = lens[b]
        qf = np.zeros((1, L, w.Hq, w.d))
        qf[0, 0] = inp.q[b].double().numpy()
        rows = np.array([[0, h, 0] for h in range(w.Hq)])
        oracle.attention_rows(qf, inp.k[b:b + 1, :L].double().numpy(),
                              inp.v[b:b + 1, :L].double().numpy(), None, rows, w.scale, False,
                              nthreads=nthreads)
        nbytes += L * w.Hkv * w.d * 4 + w.Hq * w.d * 4 + w.Hq * 4
    return time.perf_counter() - t0, nbytes


def run_decode(args, w, impl):
    import torch
    import torch.distributed as dist
    from exact_io_aware_67_b200 import ops, workloads

    ws, rank, local = dist_env()
    cores = len(os.sched_getaffinity(0))
    if impl == "reference":
        if rank != 0:
            return 0
        inp = workloads.generate_decode(w)
        for _ in range(args.warmup):
            decode_cpu_sample(w, inp, cores)
        tot_t, tot_b = 0.0, 0
        for _ in range(args.steps):
            dt, nb = decode_cpu_sample(w, inp, cores)
            tot_t += dt
            tot_b += nb
        value = tot_b / tot_t / 1e9
        sample = "1 sequence (all %d query heads, %d cached keys) of %s per step, fp64 oracle" % (
            w.Hq, inp.lengths[0], w.name)
        print(json.dumps({
            "impl": "reference", "metric": DECODE_METRIC, "value": value, "unit": "GB/s",
            "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * tot_t / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, **w.describe()},
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}), flush=True)
        return 0

    torch.cuda.set_device(local)
    if ws > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    wr = workloads.DecodeWorkload(**{**w.__dict__, "seed": w.seed + rank})
    inp = workloads.generate_decode(wr)
    lengths = inp.lengths
    q, k, v = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev)
    sl = None if inp.seqlens is None else inp.seqlens.to(dev)
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device=dev)
    wsb = torch.empty(ops.fa_decode_workspace_size(w.B, w.Hq, w.Lmax, w.d), dtype=torch.uint8,
                      device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    step_bytes = decode_bytes(w, lengths)
    # a cache of more than twice the L2 (126 MB) evicts itself between steps;
    # a smaller one is flushed by writing a buffer larger than the L2
    flush_l2 = step_bytes < 2 * 126e6

    def step():
        ops.decode(q, k, v, sl, w.scale, out=o, lse=lse, workspace=wsb)

    ops.fa_clear_device_error()
    for _ in range(args.warmup):
        if flush_l2:
            flush.zero_()
        step()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    for s in range(args.steps):
        if flush_l2:
            flush.zero_()                  # L2 flushed between timed steps
        ev[s][0].record(stream)
        step()
        ev[s][1].record(stream)
    torch.cuda.synchronize()
    if ws > 1:
        dist.barrier()
    clk = clocks.stop()
    ms = sum(a.elapsed_time(b) for a, b in ev)
    err = ops.fa_device_error()
    if err != 0:
        raise RuntimeError("device error word 0x%x during the timed region" % err)

    # e2e: the new token's q, k and v from pinned host memory (k and v written
    # into the cache at each sequence's last position), o and lse back
    e2e = None
    if not args.no_e2e:
        hq = inp.q.pin_memory()
        last = [max(L - 1, 0) for L in lengths]
        hk = torch.stack([inp.k[b, last[b]] for b in range(w.B)]).pin_memory()
        hv = torch.stack([inp.v[b, last[b]] for b in range(w.B)]).pin_memory()
        dk, dv = torch.empty_like(hk, device=dev), torch.empty_like(hv, device=dev)
        ho = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
        hl = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
        bidx = torch.arange(w.B, device=dev)
        lidx = torch.tensor(last, device=dev)
        h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv))
        d2h = ho.numel() * ho.element_size() + hl.numel() * hl.element_size()
        n_e2e = min(args.steps, 200)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        for it in range(1 + n_e2e):
            if it == 1:
                torch.cuda.synchronize()
                e0.record(stream)
            q.copy_(hq, non_blocking=True)
            dk.copy_(hk, non_blocking=True)
            dv.copy_(hv, non_blocking=True)
            k[bidx, lidx] = dk
            v[bidx, lidx] = dv
            step()
            ho.copy_(o, non_blocking=True)
            hl.copy_(lse, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        e2e = {"ms": e0.elapsed_time(e1) * args.steps / n_e2e, "h2d": h2d, "d2h": d2h}

    ms_max, e2e_max = max_over_ranks([ms, e2e["ms"] if e2e else 0.0], device=dev)
    if ws > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0
    peaks, peaks_src = load_peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    value = ws * step_bytes * args.steps / (ms_max / 1e3) / 1e9
    avg_ms = ms / args.steps
    achieved = step_bytes / (avg_ms / 1e3) / 1e9
    line = {
        "metric": DECODE_METRIC, "value": value, "unit": "GB/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16 q and cache of the workload's shape)",
        "config": {"workload": w.name, **w.describe(),
                   "l2": ("flushed between timed steps (256 MB write)" if flush_l2 else
                          "cache larger than twice the L2 (%.0f MB per step)" % (step_bytes / 1e6)),
                   "parallelism": "independent batches per GPU" if ws > 1 else "1 GPU"},
        "roofline": {"bound": "hbm",
                     "kernel": ("decode_split_kernel + decode_merge_kernel" if sl is None else
                                "decode_prefix_kernel + decode_split_kernel + decode_merge_kernel"),
                     "achieved": achieved, "peak": hbm, "unit": "GB/s",
                     "frac": achieved / hbm, "traffic": None,
                     "algorithmic_bytes_per_launch": step_bytes, "avg_launch_ms": avg_ms,
                     "peak_source": "%s hbm_gbs" % peaks_src},
        # split + merge, after a prefix kernel when the lengths live on the device
        "gpu_launches": (2 if sl is None else 3) * args.steps,
        "clocks": clk,
    }
    if e2e:
        line["e2e"] = {"value": ws * step_bytes * args.steps / (e2e_max / 1e3) / 1e9,
                       "unit": "GB/s", "h2d_bytes_per_step": e2e["h2d"],
                       "d2h_bytes_per_step": e2e["d2h"], "ms_per_step": e2e_max / args.steps}
    if not args.no_cpu_baseline and ws == 1:
        dt, nb = decode_cpu_sample(w, inp, cores)
        line["cpu_baseline"] = {
            "value": nb / dt / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
            "seconds": dt,
            "sample": "1 sequence (all %d query heads, %d cached keys), fp64 oracle" % (
                w.Hq, lengths[0])}
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=60)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="b200", choices=["b200", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    args = ap.parse_args()
    from exact_io_aware_67_b200 import workloads
    if args.workload in workloads.DECODE_WORKLOADS:
        return run_decode(args, workloads.DECODE_WORKLOADS[args.workload], args.impl)
    if args.workload in workloads.BLOCKSPARSE_WORKLOADS:
        return run_blocksparse(args, workloads.BLOCKSPARSE_WORKLOADS[args.workload])
    w = workloads.WORKLOADS[args.workload]
    if args.warmup < 3 and args.impl == "b200":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        return run_reference(args, w)
    return run_b200(args, w)


if __name__ == "__main__":
    sys.exit(main())
