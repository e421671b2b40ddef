"""Pure-Python loop evaluations for tiny inputs (TEST INFRASTRUCTURE ONLY).

These restate the same definitions in a different form from
``gecko_oracle`` so that each pins the other:
  * SCA as full attention over the whole sequence with a banded mask
    mask(t, u) = (u <= t) and (u // c >= t // c - 1)
    (Gecko digest, paper.rainbus.top, method step 3; paperlayer.ai summary,
    section 3.2: each chunk attends to itself and the preceding chunk).
  * AWM in its un-normalised, token-by-token form.  Multiplying the chunk
    update by z^{s-1} gives U_s = z^{s-1} (.) M'_s with
      U_{s+1} = U_s + sum_{i in chunk s} exp(km_i)^T (v_i - psi(km_i) M'_s),
    where every z^s is recomputed from scratch as a plain scalar sum over all
    tokens of chunks 1..s (digest, 核心方法 / core method).  No ratio of
    denominators and no log space appear here.
Scalars only: lists of floats and math.exp, no vectorised library code.
"""
from __future__ import annotations

import math


def sca_banded(q, k, v, c):
    """q, k, v: lists of T rows (lists of floats).  Returns list of rows."""
    T = len(q)
    out = []
    for t in range(T):
        keys = [u for u in range(T) if u <= t and u // c >= t // c - 1]
        sc = [sum(q[t][f] * k[u][f] for f in range(len(q[t]))) for u in keys]
        m = max(sc)
        w = [math.exp(x - m) for x in sc]
        tot = sum(w)
        out.append([sum(w[n] * v[u][j] for n, u in enumerate(keys)) / tot
                    for j in range(len(v[0]))])
    return out


def _psi_row(x):
    m = max(x)
    e = [math.exp(a - m) for a in x]
    tot = sum(e)
    return [a / tot for a in e]


def awm_tokenwise(qm, km, v, c):
    """Returns (out_mem rows, [M'_1 .. M'_{S+1}] as nested lists, z^S list)."""
    T, d, dv = len(km), len(km[0]), len(v[0])
    S = T // c

    def z_upto(s):  # z^s per feature, straight sum over tokens of chunks 1..s
        return [sum(math.exp(km[t][f]) for t in range(s * c)) for f in range(d)]

    Ms = {0: [[0.0] * dv for _ in range(d)], 1: [[0.0] * dv for _ in range(d)]}
    for s in range(1, S + 1):
        z_prev = z_upto(s - 1) if s > 1 else [0.0] * d
        z_cur = z_upto(s)
        M = Ms[s]
        U = [[z_prev[f] * M[f][j] for j in range(dv)] for f in range(d)]
        for t in range((s - 1) * c, s * c):
            ps = _psi_row(km[t])
            ret = [sum(ps[g] * M[g][j] for g in range(d)) for j in range(dv)]
            for f in range(d):
                ek = math.exp(km[t][f])
                for j in range(dv):
                    U[f][j] += ek * (v[t][j] - ret[j])
        Ms[s + 1] = [[U[f][j] / z_cur[f] for j in range(dv)] for f in range(d)]
    out = []
    for t in range(T):
        s = t // c + 1
        M = Ms[s - 1]
        pq = _psi_row(qm[t])
        out.append([sum(pq[f] * M[f][j] for f in range(d)) for j in range(dv)])
    z_last = z_upto(S)
    return out, [Ms[s] for s in range(1, S + 2)], z_last
