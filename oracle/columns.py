"""Key-column sampler of the fp64 oracle -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU legs may
use the ``oracle`` package; the CUDA library never imports it.

dK_j and dV_j of one key row j depend on every query row i that may attend
to it, through that row's P_ij = exp(S_ij - LSE_i) and D_i = dO_i . O_i.
So this sampler first computes, for every query row of the (sequence,
query head) problems that share key/value head hk, the row statistics by the
plain definition, then the sampled key rows' gradients:

  per query row i ("注意力机制基础" 2.1; "FlashAttention优化" 2.2, three
  passes over a materialised score row):
      S_ij  = scale q_i . k_j   (j > i set to -inf when causal)
      m_i   = max_j S_ij
      l_i   = sum_j exp(S_ij - m_i)
      P_ij  = exp(S_ij - m_i) / l_i
      O_i   = sum_j P_ij v_j,  LSE_i = m_i + ln l_i,  D_i = dO_i . O_i
  per sampled key row j (the derivative of the definition, as in
  ``attention_oracle.c``), summed over the group's query heads:
      dV_j = sum_i P_ij dO_i
      dS_ij = P_ij (dO_i . v_j - D_i)
      dK_j = scale sum_i dS_ij q_i

The score rows are materialised a block of rows at a time (memory only) and
the products over keys and over the head dimension are fp64 matrix
multiplications (a library primitive, torch on the CPU).  It shares no code
with the CUDA library and none with the C oracle; the tests pin it against
the C oracle's full backward, against central finite differences and
against the pure-Python brute force.
"""
import numpy as np
import torch

ROW_BLOCK = 512


def _seq(t, cu, b, h):
    """[L, d] fp64 tensor of sequence b, head h (dense [B, N, H, d] or
    varlen [total, H, d])."""
    if cu is None:
        return t[b, :, h]
    return t[int(cu[b]):int(cu[b + 1]), h]


def _row_stats(q, k, v, do, scale, causal):
    """LSE_i and D_i of every query row of one problem (q, k, v, do: [L, d]
    fp64), by the three-pass definition over materialised score rows."""
    L = q.shape[0]
    lse = torch.empty(L, dtype=torch.float64)
    D = torch.empty(L, dtype=torch.float64)
    for r0 in range(0, L, ROW_BLOCK):
        r1 = min(L, r0 + ROW_BLOCK)
        keys = r1 if causal else L          # keys beyond the block's last row are all masked
        S = scale * (q[r0:r1] @ k[:keys].T)
        if causal:
            rows = torch.arange(r0, r1).unsqueeze(1)
            cols = torch.arange(keys).unsqueeze(0)
            S.masked_fill_(cols > rows, float("-inf"))
        m = S.max(dim=1, keepdim=True).values          # pass 1: row max
        E = torch.exp(S - m)                            # pass 2: exponentials and sum
        l = E.sum(dim=1, keepdim=True)
        P = E / l                                       # pass 3: normalise
        O = P @ v[:keys]
        lse[r0:r1] = (m + torch.log(l)).squeeze(1)
        D[r0:r1] = (do[r0:r1] * O).sum(dim=1)
    return lse, D


def attention_cols(q, k, v, dout, cols, scale, causal, cu_seqlens=None, nthreads=0):
    """dK and dV of selected key rows.

    q, dout: [B, N, Hq, d] (dense) or [total, Hq, d] (varlen, with
    cu_seqlens); k, v: the same with Hkv heads.  cols: int array [C, 3] of
    (sequence, key/value head, key row within the sequence).  Returns
    {"dk": [C, d], "dv": [C, d]} (fp64): each the sum over the query heads
    h with h // (Hq / Hkv) == the key/value head."""
    cols = np.asarray(cols, dtype=np.int64).reshape(-1, 3)
    t64 = lambda a: torch.from_numpy(np.ascontiguousarray(np.asarray(a, dtype=np.float64)))
    q, k, v, dout = t64(q), t64(k), t64(v), t64(dout)
    cu = None if cu_seqlens is None else np.asarray(cu_seqlens, dtype=np.int64)
    Hq = q.shape[-2]
    Hkv = k.shape[-2]
    g = Hq // Hkv
    d = q.shape[-1]
    old_threads = torch.get_num_threads()
    if nthreads > 0:
        torch.set_num_threads(nthreads)
    try:
        dk = np.zeros((cols.shape[0], d))
        dv = np.zeros((cols.shape[0], d))
        groups = {}
        for n, (b, hk, j) in enumerate(cols):
            groups.setdefault((int(b), int(hk)), []).append((n, int(j)))
        for (b, hk), members in groups.items():
            kk, vv = _seq(k, cu, b, hk), _seq(v, cu, b, hk)
            L = kk.shape[0]
            idx = [n for n, _ in members]
            js = torch.tensor([j for _, j in members], dtype=torch.int64)
            if int(js.min()) < 0 or int(js.max()) >= L:
                raise ValueError("key row outside its sequence")
            acc_k = torch.zeros(len(members), d, dtype=torch.float64)
            acc_v = torch.zeros(len(members), d, dtype=torch.float64)
            for h in range(hk * g, (hk + 1) * g):
                qq, dd = _seq(q, cu, b, h), _seq(dout, cu, b, h)
                lse, D = _row_stats(qq, kk, vv, dd, scale, causal)
                # [L, C] blocks of P_ij and dS_ij for the sampled keys j
                S = scale * (qq @ kk[js].T)
                if causal:
                    S.masked_fill_(torch.arange(L).unsqueeze(1) < js.unsqueeze(0), float("-inf"))
                P = torch.exp(S - lse.unsqueeze(1))
                dP = dd @ vv[js].T
                dS = P * (dP - D.unsqueeze(1))
                acc_v += P.T @ dd
                acc_k += scale * (dS.T @ qq)
            dk[idx] = acc_k.numpy()
            dv[idx] = acc_v.numpy()
        return {"dk": dk, "dv": dv}
    finally:
        torch.set_num_threads(old_threads)
