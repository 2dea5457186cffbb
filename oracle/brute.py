"""Pure-Python brute-force attention for tiny shapes -- TEST INFRASTRUCTURE.

A second implementation of the same definition as ``attention_oracle.c``,
written independently (nested Python lists, ``math.fsum`` for every sum) so
that an index or sign slip in the C oracle cannot hide behind a shared helper.

Definition ("注意力机制基础" section 2.1): S = scale * Q K^T, causal mask sets
key j > i to -inf, P = softmax over each row, O = P V.  The backward routes
the upstream gradient through the full softmax Jacobian
dP_ik/dS_ij = P_ik (delta_kj - P_ij) explicitly (no shortcut through D), then
through the two products.  Grouped-query reading: query head h reads
key/value head h // (Hq // Hkv).

Inputs are nested lists: q[n][h][c] for one sequence (n tokens), k/v with
Hkv heads.  Sizes are meant for n <= 4, d <= 4.
"""
import math


def _scores(q, k, h, hk, scale, causal):
    n = len(q)
    d = len(q[0][0])
    S = [[0.0] * n for _ in range(n)]
    for i in range(n):
        for j in range(n):
            if causal and j > i:
                S[i][j] = -math.inf
            else:
                S[i][j] = scale * math.fsum(q[i][h][c] * k[j][hk][c] for c in range(d))
    return S


def _softmax(row):
    m = max(row)
    e = [0.0 if x == -math.inf else math.exp(x - m) for x in row]
    z = math.fsum(e)
    return [x / z for x in e], m + math.log(z)


def forward(q, k, v, scale, causal):
    """Returns (o[n][Hq][d], lse[Hq][n])."""
    n, Hq, d = len(q), len(q[0]), len(q[0][0])
    Hkv = len(k[0])
    g = Hq // Hkv
    o = [[[0.0] * d for _ in range(Hq)] for _ in range(n)]
    lse = [[0.0] * n for _ in range(Hq)]
    for h in range(Hq):
        hk = h // g
        S = _scores(q, k, h, hk, scale, causal)
        for i in range(n):
            p, lse[h][i] = _softmax(S[i])
            for c in range(d):
                o[i][h][c] = math.fsum(p[j] * v[j][hk][c] for j in range(n))
    return o, lse


def backward(q, k, v, dout, scale, causal):
    """Gradients of L = sum(O * dout).  Returns (dq, dk, dv) shaped like
    q, k, v."""
    n, Hq, d = len(q), len(q[0]), len(q[0][0])
    Hkv = len(k[0])
    g = Hq // Hkv
    dq = [[[0.0] * d for _ in range(Hq)] for _ in range(n)]
    dk_terms = [[[[] for _ in range(d)] for _ in range(Hkv)] for _ in range(n)]
    dv_terms = [[[[] for _ in range(d)] for _ in range(Hkv)] for _ in range(n)]
    for h in range(Hq):
        hk = h // g
        S = _scores(q, k, h, hk, scale, causal)
        P = [_softmax(S[i])[0] for i in range(n)]
        for i in range(n):
            # upstream gradient w.r.t. P_ik: dO_i . V_k
            gP = [math.fsum(dout[i][h][c] * v[kk][hk][c] for c in range(d)) for kk in range(n)]
            # gradient w.r.t. S_ij through the softmax Jacobian
            gS = []
            for j in range(n):
                terms = []
                for kk in range(n):
                    jac = P[i][kk] * ((1.0 if kk == j else 0.0) - P[i][j])
                    terms.append(gP[kk] * jac)
                gS.append(math.fsum(terms))
            for c in range(d):
                dq[i][h][c] = math.fsum(scale * gS[j] * k[j][hk][c] for j in range(n))
            for j in range(n):
                for c in range(d):
                    dk_terms[j][hk][c].append(scale * gS[j] * q[i][h][c])
                    dv_terms[j][hk][c].append(P[i][j] * dout[i][h][c])
    dk = [[[math.fsum(dk_terms[j][hk][c]) for c in range(d)] for hk in range(Hkv)]
          for j in range(n)]
    dv = [[[math.fsum(dv_terms[j][hk][c]) for c in range(d)] for hk in range(Hkv)]
          for j in range(n)]
    return dq, dk, dv
