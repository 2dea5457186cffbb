"""FLOP and byte accounting for the attention path.

Forward FLOPs follow the standard-attention count of "注意力机制基础"
section 2.2.1: QK^T is 2 N^2 d and PV is 2 N^2 d, so 4 N^2 d per (batch,
head); softmax and mask work is not counted.  Causal attention counts exactly
half of that (N^2 / 2 score entries), variable-length batches sum 4 L_s^2 d
over their sequences, and grouped-query attention counts every query head.
The backward counts 2.5x the forward (five products of 2 N^2 d each: S, dP,
dV, dK, dQ).

Byte counts are the algorithmic HBM traffic of one pass: every input read
once and every output written once; key/value tiles are read once per
key/value head, intermediates never reach HBM.
"""


def seq_lengths(w, lengths=None):
    if w.varlen:
        if lengths is None:
            raise ValueError("varlen workload needs its drawn lengths")
        return list(lengths)
    return [w.N] * w.B


def fwd_flops(w, lengths=None):
    f = 0.0
    for L in seq_lengths(w, lengths):
        f += 4.0 * w.Hq * float(L) * float(L) * w.d
    return f * (0.5 if w.causal else 1.0)


def bwd_flops(w, lengths=None):
    return 2.5 * fwd_flops(w, lengths)


def standard_attention_flops(N, d):
    """4 N^2 d for one head ("注意力机制基础" 2.2.1)."""
    return 4.0 * N * N * d


def standard_attention_hbm_bytes(N, d, elem_bytes=2):
    """Reads of Q, K, S, S, P, V and writes of S, P, O for one head
    ("注意力机制基础" 2.2.2): 4 N^2 + 4 N d elements."""
    return elem_bytes * (4.0 * N * N + 4.0 * N * d)


def fwd_bytes(w, lengths=None):
    """Q read, K and V read once per kv head, O written (bf16), LSE (fp32)."""
    tot = sum(seq_lengths(w, lengths))
    e = 2
    return tot * (2 * w.Hq * w.d * e + 2 * w.Hkv * w.d * e + 4 * w.Hq)


def bwd_bytes(w, lengths=None):
    """Q, K, V, O, dO read, LSE read, dQ, dK, dV written (bf16), plus the fp32
    D vector and one fp32 dQ accumulator written, read back and converted."""
    tot = sum(seq_lengths(w, lengths))
    e = 2
    qh = w.Hq * w.d
    kh = w.Hkv * w.d
    return tot * (e * (3 * qh + 2 * kh)        # q, o, dO read; k, v read
                  + e * (qh + 2 * kh)          # dq, dk, dv written
                  + 4 * w.Hq * 2               # lse read, D written
                  + 4 * qh * 3)                # dq_acc zero, reduce, read


def blocksparse_pairs(N, causal, mask_row):
    """(query, key) pairs a block mask allows in one head: the sum over the
    allowed 128 x 128 tiles of their element count, cut at N, and with only
    j <= i kept on diagonal tiles when causal (off-diagonal allowed tiles
    below it count whole; tiles above it are never allowed)."""
    import numpy as np
    m = np.asarray(mask_row, dtype=bool)
    nt = m.shape[0]
    sizes = np.minimum(128, N - 128 * np.arange(nt))
    total = 0
    for qt in range(nt):
        for kt in range(nt):
            if not m[qt, kt] or (causal and kt > qt):
                continue
            if causal and kt == qt:
                r = int(sizes[qt])
                total += r * (r + 1) // 2
            else:
                total += int(sizes[qt]) * int(sizes[kt])
    return total


def blocksparse_fwd_flops(bw, mask):
    """4 d per allowed (query, key) pair, summed over query heads (each uses
    its key/value head's mask row)."""
    w = bw.base
    g = w.Hq // w.Hkv
    tot = 0
    for hk in range(w.Hkv):
        row = mask[0, hk if mask.shape[1] > 1 else 0]
        tot += g * blocksparse_pairs(w.N, w.causal, row)
    return 4.0 * w.d * tot * w.B
