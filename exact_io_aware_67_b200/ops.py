"""Python binding of libfa.so -- argument marshalling only.

The functions named ``fa_*`` mirror the C entry points of ``include/fa.h``
one to one (plain integers and device pointers).  ``attention_fwd`` and
``attention_bwd`` are conveniences that take torch CUDA tensors, allocate the
outputs and the workspace with torch, and call the C entry points on the
current torch stream.  Every step of the computation runs in the CUDA
kernels of libfa.so; there is no other implementation behind this module,
and it raises if the library cannot be loaded.
"""
import ctypes
import os

import torch

from . import build as _build

_lib = None

FA_OK = 0
STATUS = {0: "FA_OK", 1: "FA_ERR_INVALID_ARG", 2: "FA_ERR_UNSUPPORTED",
          3: "FA_ERR_WORKSPACE", 4: "FA_ERR_CUDA"}

EXPORTED = ["fa_fwd", "fa_bwd", "fa_bwd_workspace_size", "fa_device_error",
            "fa_clear_device_error", "fa_set_wait_limit_ns", "fa_watchdog_selftest",
            "fa_status_string", "fa_last_cuda_error", "fa_set_profile_events",
            "fa_bwd_noalloc", "fa_std_softmax", "fa_decode", "fa_decode_workspace_size",
            "fa_fwd_blockmask", "fa_bwd_blockmask", "fa_validate_cu_seqlens"]

# capacity of the fixed scratch behind fa_bwd_noalloc (include/fa.h)
FA_BWD_NOALLOC_SCRATCH_BYTES = 64 << 20


class FAError(RuntimeError):
    def __init__(self, fn, status):
        msg = "%s failed: %s" % (fn, STATUS.get(status, status))
        if status == 4:
            msg += " (cudaError %d)" % fa_last_cuda_error()
        super().__init__(msg)
        self.status = status


def lib_path():
    return _build.LIB


def load(build_if_missing=True):
    """Load libfa.so (building it first if it is missing or stale)."""
    global _lib
    if _lib is not None:
        return _lib
    # FA_LIBRARY_PATH selects another build of libfa.so (e.g. to compare two
    # builds in one process tree); by default the in-tree build is used
    path = os.environ.get("FA_LIBRARY_PATH") or _build.LIB
    if build_if_missing and not os.environ.get("FA_LIBRARY_PATH"):
        path = _build.build()
    if not os.path.exists(path):
        raise RuntimeError("libfa.so not found at %s; run python -m exact_io_aware_67_b200.build"
                           % path)
    lib = ctypes.CDLL(path)
    vp, ip, c_int, c_float = ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_float
    lib.fa_fwd.argtypes = [vp] * 6 + [c_int] * 5 + [c_float, c_int, vp, c_int, vp]
    lib.fa_fwd.restype = c_int
    lib.fa_bwd.argtypes = [vp] * 11 + [ctypes.c_size_t] + [c_int] * 5 + \
        [c_float, c_int, vp, c_int, vp]
    lib.fa_bwd.restype = c_int
    lib.fa_bwd_noalloc.argtypes = [vp] * 10 + [c_int] * 5 + [c_float, c_int, vp, c_int, vp]
    lib.fa_bwd_noalloc.restype = c_int
    cl = ctypes.c_long
    lib.fa_fwd_blockmask.argtypes = [vp] * 6 + [c_int] * 5 + [c_float, c_int, vp, cl, cl, vp]
    lib.fa_fwd_blockmask.restype = c_int
    lib.fa_bwd_blockmask.argtypes = [vp] * 11 + [ctypes.c_size_t] + [c_int] * 5 + \
        [c_float, c_int, vp, cl, cl, vp]
    lib.fa_bwd_blockmask.restype = c_int
    lib.fa_decode.argtypes = [vp] * 6 + [c_int] * 5 + [c_float, vp, ctypes.c_size_t, vp]
    lib.fa_decode.restype = c_int
    lib.fa_decode_workspace_size.argtypes = [c_int] * 4
    lib.fa_decode_workspace_size.restype = ctypes.c_size_t
    lib.fa_std_softmax.argtypes = [vp, vp, vp, c_int, c_int, c_float, c_int, vp]
    lib.fa_std_softmax.restype = c_int
    lib.fa_bwd_workspace_size.argtypes = [c_int] * 5
    lib.fa_bwd_workspace_size.restype = ctypes.c_size_t
    lib.fa_validate_cu_seqlens.argtypes = [vp, c_int, c_int, c_int, vp]
    lib.fa_validate_cu_seqlens.restype = c_int
    lib.fa_device_error.argtypes = []
    lib.fa_device_error.restype = c_int
    lib.fa_clear_device_error.argtypes = []
    lib.fa_clear_device_error.restype = c_int
    lib.fa_set_wait_limit_ns.argtypes = [ctypes.c_ulonglong]
    lib.fa_set_wait_limit_ns.restype = None
    lib.fa_watchdog_selftest.argtypes = [vp]
    lib.fa_watchdog_selftest.restype = c_int
    lib.fa_set_profile_events.argtypes = [vp, vp]
    lib.fa_set_profile_events.restype = None
    lib.fa_last_cuda_error.argtypes = []
    lib.fa_last_cuda_error.restype = c_int
    lib.fa_status_string.argtypes = [c_int]
    lib.fa_status_string.restype = ctypes.c_char_p
    if os.environ.get("FA_WAIT_LIMIT_NS"):
        lib.fa_set_wait_limit_ns(int(os.environ["FA_WAIT_LIMIT_NS"]))
    _lib = lib
    return lib


# ------------------------------------------------------------ raw C entry points

def fa_fwd(q, k, v, o, lse, o_lo, B, Hq, Hkv, N, d, scale, causal, cu_seqlens, total_tokens,
           stream):
    return load().fa_fwd(q, k, v, o, lse, o_lo, B, Hq, Hkv, N, d, scale, int(causal), cu_seqlens,
                         total_tokens, stream)


def fa_bwd(q, k, v, o, lse, o_lo, dO, dq, dk, dv, workspace, workspace_bytes, B, Hq, Hkv, N, d,
           scale, causal, cu_seqlens, total_tokens, stream):
    return load().fa_bwd(q, k, v, o, lse, o_lo, dO, dq, dk, dv, workspace, workspace_bytes, B, Hq,
                         Hkv, N, d, scale, int(causal), cu_seqlens, total_tokens, stream)


def fa_bwd_noalloc(q, k, v, o, lse, o_lo, dO, dq, dk, dv, B, Hq, Hkv, N, d, scale, causal,
                   cu_seqlens, total_tokens, stream):
    """Backward through the library's fixed scratch array (no allocation by
    the library or by this binding); see include/fa.h for its limits."""
    return load().fa_bwd_noalloc(q, k, v, o, lse, o_lo, dO, dq, dk, dv, B, Hq, Hkv, N, d, scale,
                                 int(causal), cu_seqlens, total_tokens, stream)


def fa_fwd_blockmask(q, k, v, o, lse, o_lo, B, Hq, Hkv, N, d, scale, causal, block_mask, mask_bs,
                     mask_hs, stream):
    return load().fa_fwd_blockmask(q, k, v, o, lse, o_lo, B, Hq, Hkv, N, d, scale, int(causal),
                                   block_mask, mask_bs, mask_hs, stream)


def fa_bwd_blockmask(q, k, v, o, lse, o_lo, dO, dq, dk, dv, workspace, workspace_bytes, B, Hq,
                     Hkv, N, d, scale, causal, block_mask, mask_bs, mask_hs, stream):
    return load().fa_bwd_blockmask(q, k, v, o, lse, o_lo, dO, dq, dk, dv, workspace,
                                   workspace_bytes, B, Hq, Hkv, N, d, scale, int(causal),
                                   block_mask, mask_bs, mask_hs, stream)


def fa_decode(q, k_cache, v_cache, o, lse, cache_seqlens, B, Hq, Hkv, Lmax, d, scale, workspace,
              workspace_bytes, stream):
    return load().fa_decode(q, k_cache, v_cache, o, lse, cache_seqlens, B, Hq, Hkv, Lmax, d,
                            scale, workspace, workspace_bytes, stream)


def fa_decode_workspace_size(B, Hq, Lmax, d):
    return load().fa_decode_workspace_size(B, Hq, Lmax, d)


def fa_std_softmax(s, p, lse, BH, N, scale, causal, stream):
    """Softmax step of standard attention over a materialised S (comparator
    only); see include/fa.h."""
    return load().fa_std_softmax(s, p, lse, BH, N, scale, int(causal), stream)


def fa_bwd_workspace_size(B, Hq, N, d, total_tokens):
    return load().fa_bwd_workspace_size(B, Hq, N, d, total_tokens)


def fa_validate_cu_seqlens(cu_seqlens, B, N, total_tokens, stream):
    """Enqueue the device-side check of a cu_seqlens array; its result is
    read with fa_device_error() after a synchronise (see include/fa.h)."""
    return load().fa_validate_cu_seqlens(cu_seqlens, B, N, total_tokens, stream)


def fa_device_error():
    return load().fa_device_error()


def fa_clear_device_error():
    return load().fa_clear_device_error()


def fa_set_wait_limit_ns(ns):
    load().fa_set_wait_limit_ns(int(ns))


def fa_watchdog_selftest(stream):
    return load().fa_watchdog_selftest(stream)


def fa_set_profile_events(main_begin, main_end):
    """main_begin / main_end: torch.cuda.Event objects (or None to stop)."""
    b = None if main_begin is None else ctypes.c_void_p(main_begin.cuda_event)
    e = None if main_end is None else ctypes.c_void_p(main_end.cuda_event)
    load().fa_set_profile_events(b, e)


def fa_last_cuda_error():
    return load().fa_last_cuda_error()


def fa_status_string(s):
    return load().fa_status_string(int(s)).decode()


# ------------------------------------------------------------ torch conveniences

def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _shape(q, k, cu_seqlens, max_seqlen):
    if cu_seqlens is None:
        B, N, Hq, d = q.shape
        Hkv = k.shape[2]
        total = B * N
    else:
        total, Hq, d = q.shape
        Hkv = k.shape[1]
        B = cu_seqlens.numel() - 1
        if max_seqlen is None:
            raise ValueError("varlen inputs need max_seqlen (no device->host read is made)")
        N = int(max_seqlen)
    return B, Hq, Hkv, N, d, total


def _check(t, name, dtype=torch.bfloat16):
    if not t.is_cuda or t.dtype != dtype or not t.is_contiguous():
        raise ValueError("%s must be a contiguous CUDA %s tensor" % (name, dtype))


def attention_fwd(q, k, v, scale=None, causal=False, cu_seqlens=None, max_seqlen=None,
                  out=None, lse=None, o_lo=None):
    """O, LSE = fa_fwd(q, k, v).  Dense [B, N, H, d] or varlen [total, H, d].
    o_lo: optional bf16 tensor shaped like q that receives O's rounding
    residual (pass it to attention_bwd for an fp32-accurate D)."""
    for t, nm in ((q, "q"), (k, "k"), (v, "v")):
        _check(t, nm)
    B, Hq, Hkv, N, d, total = _shape(q, k, cu_seqlens, max_seqlen)
    if scale is None:
        scale = d ** -0.5
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, N) if cu_seqlens is None else (Hq, total),
                          dtype=torch.float32, device=q.device)
    if cu_seqlens is not None:
        _check(cu_seqlens, "cu_seqlens", torch.int32)
    if o_lo is not None:
        _check(o_lo, "o_lo")
        if o_lo.shape != q.shape:
            raise ValueError("o_lo must have q's shape")
    st = fa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(o_lo), B, Hq, Hkv, N, d,
                float(scale), causal, _ptr(cu_seqlens), total, _stream())
    if st != FA_OK:
        raise FAError("fa_fwd", st)
    return out, lse


def workspace_for(q, k, cu_seqlens=None, max_seqlen=None):
    """A torch-allocated workspace of fa_bwd_workspace_size() bytes."""
    B, Hq, _, N, d, total = _shape(q, k, cu_seqlens, max_seqlen)
    nbytes = fa_bwd_workspace_size(B, Hq, N, d, total)
    return torch.empty(nbytes, dtype=torch.uint8, device=q.device)


def attention_bwd(q, k, v, out, lse, dout, scale=None, causal=False, cu_seqlens=None,
                  max_seqlen=None, workspace=None, dq=None, dk=None, dv=None, o_lo=None):
    """dQ, dK, dV = fa_bwd(...), recomputing P from the forward's LSE.
    o_lo: the forward's rounding residual of O, if it was written."""
    for t, nm in ((q, "q"), (k, "k"), (v, "v"), (out, "out"), (dout, "dout")):
        _check(t, nm)
    if o_lo is not None:
        _check(o_lo, "o_lo")
    _check(lse, "lse", torch.float32)
    B, Hq, Hkv, N, d, total = _shape(q, k, cu_seqlens, max_seqlen)
    if scale is None:
        scale = d ** -0.5
    if workspace is None:
        workspace = torch.empty(fa_bwd_workspace_size(B, Hq, N, d, total), dtype=torch.uint8,
                                device=q.device)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    st = fa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(o_lo), _ptr(dout), _ptr(dq),
                _ptr(dk), _ptr(dv), _ptr(workspace), workspace.numel(), B, Hq, Hkv, N, d,
                float(scale), causal, _ptr(cu_seqlens), total, _stream())
    if st != FA_OK:
        raise FAError("fa_bwd", st)
    return dq, dk, dv


class Attention(torch.autograd.Function):
    """Autograd wrapper: forward saves Q, K, V, O, O's rounding residual and
    LSE (O(N) memory) and the backward recomputes P in fa_bwd."""

    @staticmethod
    def forward(ctx, q, k, v, scale, causal, cu_seqlens, max_seqlen):
        o_lo = torch.empty_like(q)
        o, lse = attention_fwd(q, k, v, scale, causal, cu_seqlens, max_seqlen, o_lo=o_lo)
        ctx.save_for_backward(q, k, v, o, lse, o_lo, cu_seqlens)
        ctx.scale, ctx.causal, ctx.max_seqlen = scale, causal, max_seqlen
        return o

    @staticmethod
    def backward(ctx, do):
        q, k, v, o, lse, o_lo, cu = ctx.saved_tensors
        dq, dk, dv = attention_bwd(q, k, v, o, lse, do.contiguous(), ctx.scale, ctx.causal,
                                   cu, ctx.max_seqlen, o_lo=o_lo)
        return dq, dk, dv, None, None, None, None


def attention(q, k, v, scale=None, causal=False, cu_seqlens=None, max_seqlen=None):
    return Attention.apply(q, k, v, scale if scale is not None else q.shape[-1] ** -0.5,
                           causal, cu_seqlens, max_seqlen)


# ------------------------------------------------------------ block-sparse

def _mask_strides(block_mask, B, Hkv, N):
    _check(block_mask, "block_mask", torch.uint8)
    nt = (N + 127) // 128
    if block_mask.dim() != 4 or block_mask.shape[2:] != (nt, nt) or \
            block_mask.shape[0] not in (1, B) or block_mask.shape[1] not in (1, Hkv):
        raise ValueError("block_mask must be [1 or B, 1 or Hkv, %d, %d] uint8" % (nt, nt))
    sb = 0 if block_mask.shape[0] == 1 else block_mask.shape[1] * nt * nt
    sh = 0 if block_mask.shape[1] == 1 else nt * nt
    return sb, sh


def attention_fwd_blockmask(q, k, v, block_mask, scale=None, causal=False, out=None, lse=None,
                            o_lo=None):
    """O, LSE of block-sparse attention (fa_fwd_blockmask): dense [B, N, H, d]
    inputs; block_mask [1 or B, 1 or Hkv, nt, nt] uint8 on the device,
    nt = ceil(N / 128), nonzero = the 128 x 128 tile is computed."""
    for t, nm in ((q, "q"), (k, "k"), (v, "v")):
        _check(t, nm)
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    sb, sh = _mask_strides(block_mask, B, Hkv, N)
    if scale is None:
        scale = d ** -0.5
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device) if lse is None else lse
    if o_lo is not None:
        _check(o_lo, "o_lo")
    st = fa_fwd_blockmask(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(o_lo), B, Hq, Hkv,
                          N, d, float(scale), causal, _ptr(block_mask), sb, sh, _stream())
    if st != FA_OK:
        raise FAError("fa_fwd_blockmask", st)
    return out, lse


def attention_bwd_blockmask(q, k, v, out, lse, dout, block_mask, scale=None, causal=False,
                            workspace=None, o_lo=None):
    """dQ, dK, dV of block-sparse attention (fa_bwd_blockmask)."""
    for t, nm in ((q, "q"), (k, "k"), (v, "v"), (out, "out"), (dout, "dout")):
        _check(t, nm)
    _check(lse, "lse", torch.float32)
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    sb, sh = _mask_strides(block_mask, B, Hkv, N)
    if scale is None:
        scale = d ** -0.5
    if workspace is None:
        workspace = torch.empty(fa_bwd_workspace_size(B, Hq, N, d, B * N), dtype=torch.uint8,
                                device=q.device)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    if o_lo is not None:
        _check(o_lo, "o_lo")
    st = fa_bwd_blockmask(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(o_lo), _ptr(dout),
                          _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace), workspace.numel(), B,
                          Hq, Hkv, N, d, float(scale), causal, _ptr(block_mask), sb, sh,
                          _stream())
    if st != FA_OK:
        raise FAError("fa_bwd_blockmask", st)
    return dq, dk, dv


# ------------------------------------------------------------ decode

def decode(q, k_cache, v_cache, cache_seqlens=None, scale=None, out=None, lse=None,
           workspace=None):
    """One decode step over a KV cache (fa_decode): q [B, Hq, d], caches
    [B, Lmax, Hkv, d], cache_seqlens int32 [B] on the device or None (every
    cache full).  Returns o [B, Hq, d] and lse [B, Hq]."""
    for t, nm in ((q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _check(t, nm)
    B, Hq, d = q.shape
    _, Lmax, Hkv, _ = k_cache.shape
    if v_cache.shape != k_cache.shape or k_cache.shape[0] != B or k_cache.shape[3] != d:
        raise ValueError("cache shapes must be [B, Lmax, Hkv, d] and match q")
    if cache_seqlens is not None:
        _check(cache_seqlens, "cache_seqlens", torch.int32)
    if scale is None:
        scale = d ** -0.5
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device) if lse is None else lse
    if workspace is None:
        workspace = torch.empty(fa_decode_workspace_size(B, Hq, Lmax, d), dtype=torch.uint8,
                                device=q.device)
    st = fa_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(out), _ptr(lse),
                   _ptr(cache_seqlens), B, Hq, Hkv, Lmax, d, float(scale), _ptr(workspace),
                   workspace.numel(), _stream())
    if st != FA_OK:
        raise FAError("fa_decode", st)
    return out, lse


# ------------------------------------------------------------ comparator

def standard_attention_fwd(q, k, v, scale=None, causal=False):
    """Standard attention with S and P materialised in device memory, for
    comparison with fa_fwd ("注意力机制基础" 2.1 and 2.2.2): S = Q K^T and
    O = P V are library GEMMs (cuBLAS through torch.matmul, bf16 in, bf16
    out), and the row softmax between them is fa_std_softmax.  Inputs are
    head-major [B, H, N, d] bf16 with the same number of heads (the layout
    of the pages' per-head matrices); returns O [B, H, N, d] and LSE
    [B, H, N].  Device memory: two B*H*N*N bf16 matrices."""
    for t, nm in ((q, "q"), (k, "k"), (v, "v")):
        _check(t, nm)
    B, H, N, d = q.shape
    if k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must have the same [B, H, N, d] shape")
    if scale is None:
        scale = d ** -0.5
    s = torch.matmul(q, k.transpose(-1, -2))            # [B, H, N, N]
    p = torch.empty_like(s)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    st = fa_std_softmax(_ptr(s), _ptr(p), _ptr(lse), B * H, N, float(scale), causal, _stream())
    if st != FA_OK:
        raise FAError("fa_std_softmax", st)
    del s
    return torch.matmul(p, v), lse
