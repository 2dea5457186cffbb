"""Seeded synthetic inputs for the attention workloads.

This module only draws random numbers and packs them; it contains none of
the attention arithmetic, so both the CUDA path and the CPU oracle can be fed
from it without sharing any of the method.

Recipe (one CPU ``torch.Generator`` per workload, seeded with ``seed``):
  1. varlen lengths: integers uniform in [lo, hi] (inclusive), one per
     sequence, packed in draw order into int32 ``cu_seqlens``;
  2. Q, then K, then V, then dO: i.i.d. N(0, 1) drawn in fp32, rounded to
     bf16 (round-to-nearest-even);
  3. optionally one query row per (batch, head) scaled by 8: the row index is
     drawn uniformly in [0, N) after dO.  Multiplying by 8 is exact in bf16.
Dense layout is [B, N, H, d] (d contiguous); varlen layout is [total, H, d].

The named workloads mirror the shapes of the five benchmark configurations:
GPT-2-small-shaped causal attention, BERT-large-shaped padding-free varlen
attention, a long-sequence causal sweep, and grouped-query causal attention.
These shapes stand in for the datasets and models of the experiments the
pages describe; only the shapes are taken.
"""
import math
from dataclasses import dataclass, field
from typing import Optional

import torch


@dataclass
class Workload:
    name: str
    B: int              # batch size, or number of sequences when varlen
    Hq: int
    Hkv: int
    N: int              # sequence length, or the maximum length when varlen
    d: int
    causal: bool
    scale: float
    varlen: Optional[tuple] = None   # (lo, hi) inclusive length range
    x8_row: bool = False             # scale one query row per head by 8
    x8_key_row: bool = False         # scale one key row per kv head by 8
    seed: int = 0
    note: str = ""

    def describe(self):
        out = dict(B=self.B, Hq=self.Hq, Hkv=self.Hkv, N=self.N, d=self.d,
                   causal=self.causal, scale=self.scale)
        if self.varlen:
            out["varlen_lengths"] = list(self.varlen)
        if self.x8_row:
            out["x8_query_row_per_head"] = True
        if self.x8_key_row:
            out["x8_key_row_per_kv_head"] = True
        return out


def _w(name, B, H, N, d, causal, Hkv=None, **kw):
    return Workload(name=name, B=B, Hq=H, Hkv=H if Hkv is None else Hkv, N=N, d=d,
                    causal=causal, scale=1.0 / math.sqrt(d), **kw)


WORKLOADS = {
    "single_head_n128_d64": _w("single_head_n128_d64", 1, 1, 128, 64, False),
    "gpt2_small_causal_b8_h12_n1024_d64": _w("gpt2_small_causal_b8_h12_n1024_d64",
                                             8, 12, 1024, 64, True),
    "bert_large_varlen_32x128to512_h16_d64": _w("bert_large_varlen_32x128to512_h16_d64",
                                                32, 16, 512, 64, False, varlen=(128, 512)),
    "gqa_causal_b2_hq32_hkv8_n4096_d128": _w("gqa_causal_b2_hq32_hkv8_n4096_d128",
                                             2, 32, 4096, 128, True, Hkv=8),
}
for _d in (64, 128):
    for _n in (4096, 16384, 65536):
        _name = "long_causal_b1_h16_n%d_d%d_x8row" % (_n, _d)
        WORKLOADS[_name] = _w(_name, 1, 16, _n, _d, True, x8_row=True)


@dataclass
class Inputs:
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    dout: torch.Tensor
    cu_seqlens: Optional[torch.Tensor]
    workload: Workload
    x8_rows: Optional[torch.Tensor] = None   # [B, Hq] row index scaled by 8
    lengths: Optional[list] = field(default=None)
    x8_key_rows: Optional[torch.Tensor] = None   # [B, Hkv] key row index scaled by 8

    @property
    def total(self):
        return self.q.shape[0] if self.cu_seqlens is not None else self.q.shape[0] * self.q.shape[1]


def generate(w: Workload, with_dout: bool = True) -> Inputs:
    """Draw the inputs of workload ``w`` on the CPU (bf16 tensors)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed)
    cu = None
    lengths = None
    if w.varlen:
        lo, hi = w.varlen
        lens = torch.randint(lo, hi + 1, (w.B,), generator=g, dtype=torch.int64)
        lengths = [int(x) for x in lens]
        cu = torch.zeros(w.B + 1, dtype=torch.int32)
        cu[1:] = torch.cumsum(lens, 0).to(torch.int32)
        total = int(cu[-1])
        qshape, kshape = (total, w.Hq, w.d), (total, w.Hkv, w.d)
    else:
        qshape, kshape = (w.B, w.N, w.Hq, w.d), (w.B, w.N, w.Hkv, w.d)
    q = torch.randn(qshape, generator=g, dtype=torch.float32)
    k = torch.randn(kshape, generator=g, dtype=torch.float32)
    v = torch.randn(kshape, generator=g, dtype=torch.float32)
    dout = torch.randn(qshape, generator=g, dtype=torch.float32) if with_dout else None
    x8 = None
    if w.x8_row:
        if w.varlen:
            raise ValueError("x8 rows are defined for dense workloads only")
        x8 = torch.randint(0, w.N, (w.B, w.Hq), generator=g, dtype=torch.int64)
        for b in range(w.B):
            for h in range(w.Hq):
                q[b, int(x8[b, h]), h, :] *= 8.0
    x8k = None
    if w.x8_key_row:
        if w.varlen:
            raise ValueError("x8 rows are defined for dense workloads only")
        x8k = torch.randint(0, w.N, (w.B, w.Hkv), generator=g, dtype=torch.int64)
        for b in range(w.B):
            for h in range(w.Hkv):
                k[b, int(x8k[b, h]), h, :] *= 8.0
    bf = torch.bfloat16
    return Inputs(q=q.to(bf), k=k.to(bf), v=v.to(bf),
                  dout=None if dout is None else dout.to(bf),
                  cu_seqlens=cu, workload=w, x8_rows=x8, lengths=lengths, x8_key_rows=x8k)


def custom(name, B, Hq, Hkv, N, d, causal, scale=None, varlen=None, x8_row=False, seed=0,
           x8_key_row=False):
    """An ad-hoc workload (tests use this for edge shapes)."""
    return Workload(name=name, B=B, Hq=Hq, Hkv=Hkv, N=N, d=d, causal=causal,
                    scale=(1.0 / math.sqrt(d)) if scale is None else scale,
                    varlen=varlen, x8_row=x8_row, x8_key_row=x8_key_row, seed=seed)


def from_lengths(name, lengths, Hq, Hkv, d, causal, seed=0):
    """Varlen inputs with explicitly given sequence lengths (edge cases such
    as 0, 1 and 129); the values follow the same Q, K, V, dO draw order."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    lens = torch.tensor(lengths, dtype=torch.int64)
    cu = torch.zeros(len(lengths) + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(lens, 0).to(torch.int32)
    total = int(cu[-1])
    q = torch.randn((total, Hq, d), generator=g, dtype=torch.float32)
    k = torch.randn((total, Hkv, d), generator=g, dtype=torch.float32)
    v = torch.randn((total, Hkv, d), generator=g, dtype=torch.float32)
    dout = torch.randn((total, Hq, d), generator=g, dtype=torch.float32)
    w = Workload(name=name, B=len(lengths), Hq=Hq, Hkv=Hkv,
                 N=max(lengths) if lengths else 0, d=d, causal=causal,
                 scale=1.0 / math.sqrt(d), varlen=(min(lengths), max(lengths)) if lengths else (0, 0),
                 seed=seed)
    bf = torch.bfloat16
    return Inputs(q=q.to(bf), k=k.to(bf), v=v.to(bf), dout=dout.to(bf), cu_seqlens=cu,
                  workload=w, lengths=list(lengths))


# ------------------------------------------------------------ decode over a KV cache

@dataclass
class DecodeWorkload:
    """One decode step: B sequences, each with one new query token and a
    cache of L_b keys and values (L_b = Lmax, or drawn uniformly in
    ``lengths`` = (lo, hi) inclusive)."""
    name: str
    B: int
    Hq: int
    Hkv: int
    Lmax: int
    d: int
    scale: float
    lengths: Optional[tuple] = None
    seed: int = 0

    def describe(self):
        out = dict(B=self.B, Hq=self.Hq, Hkv=self.Hkv, Lmax=self.Lmax, d=self.d,
                   scale=self.scale)
        if self.lengths:
            out["cache_lengths"] = list(self.lengths)
        return out


def _dw(name, B, Hq, Hkv, Lmax, d, lengths=None, seed=0):
    return DecodeWorkload(name=name, B=B, Hq=Hq, Hkv=Hkv, Lmax=Lmax, d=d,
                          scale=1.0 / math.sqrt(d), lengths=lengths, seed=seed)


DECODE_WORKLOADS = {
    # the tutorial's inference case study: batch 4, 8 heads of d = 64, a
    # 2048-token prompt plus 512 generated tokens in the cache
    "decode_b4_h8_l2560_d64": _dw("decode_b4_h8_l2560_d64", 4, 8, 8, 2560, 64),
    # grouped-query decode of a long context, the shape of the GQA config
    "decode_gqa_b8_hq32_hkv8_l8192_d128": _dw("decode_gqa_b8_hq32_hkv8_l8192_d128",
                                              8, 32, 8, 8192, 128),
    # a serving batch of mixed cache lengths
    "decode_gqa_b16_hq32_hkv8_l1024to16384_d128": _dw(
        "decode_gqa_b16_hq32_hkv8_l1024to16384_d128", 16, 32, 8, 16384, 128,
        lengths=(1024, 16384)),
}


@dataclass
class DecodeInputs:
    q: torch.Tensor          # [B, Hq, d]
    k: torch.Tensor          # [B, Lmax, Hkv, d]
    v: torch.Tensor          # [B, Lmax, Hkv, d]
    seqlens: Optional[torch.Tensor]   # int32 [B] or None (all Lmax)
    workload: DecodeWorkload

    @property
    def lengths(self):
        w = self.workload
        return [w.Lmax] * w.B if self.seqlens is None else [int(x) for x in self.seqlens]


def generate_decode(w: DecodeWorkload) -> DecodeInputs:
    """Draw a decode step's inputs on the CPU: cache lengths (if drawn), then
    q, then the K cache, then the V cache, i.i.d. N(0, 1) rounded to bf16.
    Cache rows past a sequence's length are drawn like the rest (a real
    cache holds stale values there); the kernels must not use them."""
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed)
    seqlens = None
    if w.lengths:
        lo, hi = w.lengths
        seqlens = torch.randint(lo, hi + 1, (w.B,), generator=g, dtype=torch.int64).to(torch.int32)
    q = torch.randn((w.B, w.Hq, w.d), generator=g, dtype=torch.float32)
    k = torch.randn((w.B, w.Lmax, w.Hkv, w.d), generator=g, dtype=torch.float32)
    v = torch.randn((w.B, w.Lmax, w.Hkv, w.d), generator=g, dtype=torch.float32)
    bf = torch.bfloat16
    return DecodeInputs(q=q.to(bf), k=k.to(bf), v=v.to(bf), seqlens=seqlens, workload=w)


# ------------------------------------------------------------ block-sparse masks

@dataclass
class BlockSparseWorkload:
    """A dense workload plus a block mask of 128 x 128 tiles: ``band`` = w
    keeps the w tiles on and left of the diagonal (a sliding window of 128 w
    keys), ``density`` = r keeps each tile with probability r (per kv head,
    drawn from the workload's seed after its inputs), the diagonal always."""
    name: str
    base: Workload
    band: Optional[int] = None
    density: Optional[float] = None

    def describe(self):
        out = dict(self.base.describe())
        if self.band is not None:
            out["block_mask"] = "band of %d tiles (%d keys)" % (self.band, 128 * self.band)
        else:
            out["block_mask"] = "random tiles, density %.2f per kv head, diagonal kept" % self.density
        return out


def block_mask(bw: BlockSparseWorkload):
    """uint8 [1, 1 or Hkv, nt, nt] mask of the workload."""
    import numpy as np
    w = bw.base
    nt = (w.N + 127) // 128
    i = np.arange(nt)
    if bw.band is not None:
        m = ((i[:, None] - i[None, :] >= 0) & (i[:, None] - i[None, :] < bw.band))
        return m.astype(np.uint8)[None, None]
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed + 1000003)
    m = (torch.rand((1, w.Hkv, nt, nt), generator=g) < bw.density).numpy()
    m[:, :, i, i] = True
    return m.astype(np.uint8)


BLOCKSPARSE_WORKLOADS = {
    # a causal sliding window of 1024 keys over a 16384-token sequence
    "blocksparse_band8_causal_b1_h16_n16384_d128": BlockSparseWorkload(
        "blocksparse_band8_causal_b1_h16_n16384_d128",
        _w("blocksparse_band8_causal_b1_h16_n16384_d128", 1, 16, 16384, 128, True), band=8),
    # random half of the tiles of a non-causal 8192-token problem, GQA 4
    "blocksparse_random50_b1_hq16_hkv4_n8192_d64": BlockSparseWorkload(
        "blocksparse_random50_b1_hq16_hkv4_n8192_d64",
        _w("blocksparse_random50_b1_hq16_hkv4_n8192_d64", 1, 16, 8192, 64, False, Hkv=4),
        density=0.5),
}
