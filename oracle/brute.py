"""Pure-Python brute-force attention on tiny inputs -- TEST INFRASTRUCTURE ONLY.

A second restatement of the definition, independent of ``attn_oracle.c``:
nested lists of Python floats, ``math.fsum`` for every sum (correctly rounded
sums), and each query row's softmax written from the formula
P_j = exp(s_j) / sum_j' exp(s_j') with the largest score factored out.
Use it for shapes with at most a few hundred score entries.

Semantics (shared with the C oracle because they are the definition, not
code): kv head h // (Hq // Hkv); causal keeps j <= i + Sk - Sq (bottom-right
alignment, mxflashattn 1.4.0 ``prefill_chunked_reference``); a row with no
visible key gives O = 0 and LSE = -inf.
"""
from __future__ import annotations

import math


def attention_rows(q, k, v, scale, causal):
    """One sequence, one head pair.  q: Sq x D lists; k: Sk x D; v: Sk x Dv.
    Returns (O as Sq x Dv lists, LSE list)."""
    sq, sk = len(q), len(k)
    out, lse = [], []
    for i in range(sq):
        vis = [j for j in range(sk) if (not causal) or j <= i + sk - sq]
        if not vis:
            out.append([0.0] * (len(v[0]) if v else 0))
            lse.append(-math.inf)
            continue
        s = {j: scale * math.fsum(a * b for a, b in zip(q[i], k[j])) for j in vis}
        m = max(s.values())
        e = {j: math.exp(s[j] - m) for j in vis}
        z = math.fsum(e.values())
        out.append([math.fsum(e[j] / z * v[j][d] for j in vis) for d in range(len(v[0]))])
        lse.append(m + math.log(z))
    return out, lse


def attention_packed(q, k, v, cu_q, cu_k, scale, causal):
    """Packed layout: q [total_q][Hq][D], k [total_k][Hkv][D], v [total_k][Hkv][Dv]
    as nested lists; cu_q / cu_k cumulative lengths.  Returns O [total_q][Hq][Dv]
    and LSE [total_q][Hq]."""
    hq, hkv = len(q[0]) if q else 0, len(k[0]) if k else 1
    group = hq // hkv if hkv else 1
    total_q = len(q)
    dv = len(v[0][0]) if v else 0
    out = [[[0.0] * dv for _ in range(hq)] for _ in range(total_q)]
    lse = [[-math.inf] * hq for _ in range(total_q)]
    for b in range(len(cu_q) - 1):
        q0, q1, k0, k1 = cu_q[b], cu_q[b + 1], cu_k[b], cu_k[b + 1]
        for h in range(hq):
            g = h // group
            qs = [q[t][h] for t in range(q0, q1)]
            ks = [k[t][g] for t in range(k0, k1)]
            vs = [v[t][g] for t in range(k0, k1)]
            if not qs:
                continue
            if not ks:
                for t in range(q0, q1):
                    out[t][h] = [0.0] * dv
                    lse[t][h] = -math.inf
                continue
            o, l = attention_rows(qs, ks, vs, scale, causal)
            for r, t in enumerate(range(q0, q1)):
                out[t][h] = o[r]
                lse[t][h] = l[r]
    return out, lse
