"""C ABI: libfa.so loads, exports every entry point include/fa.h declares, and
rejects bad arguments on the host before touching the device (CPU only)."""
import ctypes
import os
import re
import subprocess
import sys

import pytest

from exact_io_aware_67_b200 import build, ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    txt = open(os.path.join(ROOT, "include", "fa.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    names = re.findall(r"\b(fa_[a-z_]+)\s*\(", txt)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    return ops.load()


def test_header_declares_expected_entry_points():
    assert set(_declared()) == set(ops.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for name in _declared():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for code, name in ops.STATUS.items():
        assert ops.fa_status_string(code) == name


def _fwd(**kw):
    a = dict(q=ctypes.c_void_p(4096), k=ctypes.c_void_p(4096), v=ctypes.c_void_p(4096),
             o=ctypes.c_void_p(4096), lse=ctypes.c_void_p(4096), o_lo=None, B=1, Hq=2, Hkv=1,
             N=128, d=64, scale=0.125, causal=0, cu_seqlens=None, total_tokens=0, stream=None)
    a.update(kw)
    return ops.fa_fwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["o_lo"], a["B"], a["Hq"],
                      a["Hkv"], a["N"], a["d"], a["scale"], a["causal"], a["cu_seqlens"],
                      a["total_tokens"], a["stream"])


@pytest.mark.parametrize("kw,expect", [
    (dict(d=96), 2), (dict(d=256), 2), (dict(Hq=3, Hkv=2), 1), (dict(Hkv=0), 1),
    (dict(N=0), 1), (dict(B=-1), 1), (dict(scale=0.0), 1), (dict(scale=float("nan")), 1),
    (dict(q=None), 1), (dict(o=ctypes.c_void_p(4100)), 1),
    (dict(o_lo=ctypes.c_void_p(4100)), 1),                        # misaligned residual
    (dict(o_lo=ctypes.c_void_p(4096)), 1),                        # residual aliasing o
    (dict(cu_seqlens=ctypes.c_void_p(4096), total_tokens=-1), 1),
])
def test_fwd_rejects_bad_arguments(lib, kw, expect):
    assert _fwd(**kw) == expect


def test_fwd_empty_batch_is_a_no_op(lib):
    # B = 0 and an empty varlen batch need no launch at all
    assert _fwd(B=0) == 0
    assert _fwd(cu_seqlens=ctypes.c_void_p(4096), total_tokens=0) == 0


def test_bwd_workspace_checks(lib):
    need = ops.fa_bwd_workspace_size(2, 4, 256, 128, 512)
    assert need >= 512 * 4 * 128 * 4 + 512 * 4 * 4
    assert ops.fa_bwd_workspace_size(1, 1, 1, 96, 1) == 0
    p = ctypes.c_void_p(4096)
    args = [p] * 5 + [None] + [p] * 4     # no residual of O
    st = ops.fa_bwd(*args, ctypes.c_void_p(4096), 1024, 2, 4, 4, 256, 128, 0.1, 1, None, 0,
                    None)
    assert st == 3
    st = ops.fa_bwd(*args, None, need, 2, 4, 4, 256, 128, 0.1, 1, None, 0, None)
    assert st == 3
    st = ops.fa_bwd(*args, ctypes.c_void_p(4096 + 16), need, 2, 4, 4, 256, 128, 0.1, 1, None, 0,
                    None)
    assert st == 3   # workspace must be 256-byte aligned
    # a misaligned optional residual is rejected before the workspace check
    st = ops.fa_bwd(*([p] * 5), ctypes.c_void_p(4104), *([p] * 4), ctypes.c_void_p(4096), need,
                    2, 4, 4, 256, 128, 0.1, 1, None, 0, None)
    assert st == 1


def test_build_command_targets_sm100a():
    cmd = build.nvcc_command("x.so")
    assert "arch=compute_100a,code=sm_100a" in cmd
    assert "-lineinfo" in cmd


@pytest.mark.parametrize("kw,expect", [
    (dict(N=12), 2), (dict(N=32776), 2), (dict(BH=-1), 1), (dict(N=0), 1),
    (dict(scale=0.0), 1), (dict(scale=float("inf")), 1), (dict(s=None), 1),
    (dict(p=ctypes.c_void_p(4104)), 1), (dict(BH=1 << 20, N=4096), 1), (dict(BH=0), 0),
])
def test_std_softmax_rejects_bad_arguments(lib, kw, expect):
    a = dict(s=ctypes.c_void_p(4096), p=ctypes.c_void_p(8192), lse=ctypes.c_void_p(12288), BH=2,
             N=64, scale=0.125, causal=1)
    a.update(kw)
    assert ops.fa_std_softmax(a["s"], a["p"], a["lse"], a["BH"], a["N"], a["scale"],
                              a["causal"], None) == expect


def test_decode_rejects_bad_arguments(lib):
    # host-side checks need no device work; sizes as for a valid call
    p = ctypes.c_void_p(4096)
    need = ops.fa_decode_workspace_size(2, 8, 512, 64)
    ws = ctypes.c_void_p(4096)
    args = lambda **kw: dict(dict(q=p, k=p, v=p, o=p, lse=p, sl=None, B=2, Hq=8, Hkv=2, L=512,
                                  d=64, scale=0.125, ws=ws, wsb=need), **kw)

    def call(a):
        return ops.fa_decode(a["q"], a["k"], a["v"], a["o"], a["lse"], a["sl"], a["B"], a["Hq"],
                             a["Hkv"], a["L"], a["d"], a["scale"], a["ws"], a["wsb"], None)
    assert call(args(d=96)) == 2
    assert call(args(Hq=34, Hkv=2)) == 2          # 17 query heads per kv head
    assert call(args(Hq=7)) == 1
    assert call(args(L=0)) == 1
    assert call(args(scale=0.0)) == 1
    assert call(args(wsb=need - 1)) == 3
    assert call(args(ws=ctypes.c_void_p(4096 + 16))) == 3
    assert call(args(q=ctypes.c_void_p(4100))) == 1
    assert call(args(B=0)) == 0


def test_blockmask_rejects_bad_arguments(lib):
    p = ctypes.c_void_p(4096)
    m = ctypes.c_void_p(8192)
    f = lambda **kw: ops.fa_fwd_blockmask(*([p] * 5), None, kw.get("B", 1), 2, 2, kw.get("N", 256),
                                          kw.get("d", 64), 0.125, 0, kw.get("m", m),
                                          kw.get("sb", 0), kw.get("sh", 0), None)
    assert f(m=None) == 1
    assert f(N=65537) == 2          # more tiles than the per-CTA lists hold
    assert f(d=96) == 2
    assert f(sb=-1) == 1
    assert f(B=0) == 0
    need = ops.fa_bwd_workspace_size(1, 2, 256, 64, 256)
    g = ops.fa_bwd_blockmask(*([p] * 5), None, *([p] * 4), p, need, 1, 2, 2, 256, 64, 0.125, 1,
                             None, 0, 0, None)
    assert g == 1


def _run_python(code, env_extra=None):
    env = dict(os.environ)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env,
                          capture_output=True, text=True, timeout=300)


def test_missing_library_fails_loudly():
    # no fallback: without the CUDA library the binding raises
    r = _run_python("from exact_io_aware_67_b200 import ops\n"
                    "try:\n"
                    "    ops.load()\n"
                    "except RuntimeError as e:\n"
                    "    print('raised', e)\n",
                    {"FA_LIBRARY_PATH": "/nonexistent/libfa.so"})
    assert r.returncode == 0, r.stderr
    assert r.stdout.startswith("raised"), r.stdout


def test_product_path_does_not_import_the_oracle():
    # the package and its binding never load the oracle (test infrastructure)
    r = _run_python("import sys\n"
                    "import exact_io_aware_67_b200\n"
                    "from exact_io_aware_67_b200 import ops, workloads, flops\n"
                    "ops.load()\n"
                    "print(sorted(m for m in sys.modules if m == 'oracle' or m.startswith('oracle.')))\n")
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == "[]", r.stdout
