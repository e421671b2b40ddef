"""Plain fp64 CPU oracle for the gradients of the Gecko hot path: Sliding
Chunk Attention (SCA) and the Adaptive Working Memory (AWM) recurrence.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU legs of ``bench.py`` may import this module.  The product path never calls
it and shares no code with it.

What is differentiated is the forward of ``oracle.gecko_oracle`` (the
definitions of the Gecko pages: paper.rainbus.top digest, 核心方法 and 方法步骤详情
steps 3-5; paperlayer.ai summary, sections 3.2-3.3 and Appendix A), under the
readings R1-R7 stated there.  The pages print no backward pass for this
path; the paperlayer.ai summary reports pretraining (section 4, pretraining
results) and, in appendix B.1 (backward pass), rematerialisation that keeps
only chunk-boundary states from the forward and rebuilds the rest while
differentiating.  The gradients below are reverse-mode differentiation of that forward, written out
step by step in the forward's notation:

SCA, chunk s with key window w (reading R2), P = softmax_rows(Q_s K_w^T):
    dP = dO_s V_w^T,  D = rowsum(dO_s * O_s) = rowsum(P * dP),
    dS = P * (dP - D),  dQ_s = dS K_w,  dK_w += dS^T Q_s,  dV_w += P^T dO_s.

AWM, 1-based chunks, M'_s the state read by chunk s + 1:
    forward  M'_{s+1} = r_s (.) M'_s + Phi_s^T (V_s - Psi_s M'_s),
             O_m,s = Psiq_s M'_{s-1},
    reverse  G_s = dL/dM'_s, starting from G_{S+1} (the final-state gradient):
             G_{s-1} += Psiq_s^T dO_m,s,         dPsiq_s = dO_m,s M'_{s-1}^T,
             R = V_s - Psi_s M'_s,  dR = Phi_s G_{s+1},
             dPhi_s = R G_{s+1}^T,  dV_s += dR,  dPsi_s = -dR M'_s^T,
             dr_s = rowsum(G_{s+1} * M'_s),  G_s += r_s (.) G_{s+1} - Psi_s^T dR,
then through the log-space denominators (L_s = log z^s, l_s = log e_s):
             Phi_s = exp(Km_s - L_s):  dKm_s += dPhi_s * Phi_s,
                                        dL_s -= colsum(dPhi_s * Phi_s),
             r_s = exp(L_{s-1} - L_s): dL_{s-1} += dr_s r_s,  dL_s -= dr_s r_s,
             L_s = logaddexp(L_{s-1}, l_s), taken in reverse order:
                 dl_s = dL_s exp(l_s - L_s),  dL_{s-1} += dL_s exp(L_{s-1} - L_s),
             l_s = logsumexp_i Km_s[i]:      dKm_s[i] += dl_s exp(Km_s[i] - l_s),
and through the feature softmaxes Psi = softmax_rows(Km_s), Psiq = softmax_rows(Qm_s):
             dX = Y * (dY - rowsum(dY * Y)).
All arithmetic is float64.
"""
from __future__ import annotations

import numpy as np

from . import gecko_oracle as F

__all__ = ["sca_lse", "sca_head_backward", "sca_query_rows_backward", "sca_key_rows_backward",
           "awm_head_backward", "backward"]


def _softmax_backward(y: np.ndarray, dy: np.ndarray) -> np.ndarray:
    """Gradient through y = softmax_rows(x)."""
    return y * (dy - (dy * y).sum(axis=-1, keepdims=True))


def sca_lse(q: np.ndarray, k: np.ndarray, c: int) -> np.ndarray:
    """Natural-log sum of exp of each query row's visible scores (the SCA
    normaliser a training forward keeps for the backward) -> [T]."""
    T = q.shape[0]
    out = np.empty(T)
    for t in range(T):
        lo = F.window_lo(t, c)
        sc = F.SCA_SCALE * (k[lo:t + 1] @ q[t])
        m = sc.max()
        out[t] = m + np.log(np.exp(sc - m).sum())
    return out


def sca_head_backward(q, k, v, c: int, dout):
    """(dq, dk, dv) of the SCA output of one head; all [T, d] float64."""
    T = q.shape[0]
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for s0 in range(T // c):
        a, b = s0 * c, (s0 + 1) * c
        lo = F.window_lo(a, c)
        t = np.arange(a, b)[:, None]
        u = np.arange(lo, b)[None, :]
        P = F._masked_softmax_rows(F.SCA_SCALE * (q[a:b] @ k[lo:b].T), u <= t)
        O = P @ v[lo:b]
        dP = dout[a:b] @ v[lo:b].T
        D = (dout[a:b] * O).sum(axis=1, keepdims=True)
        dS = P * (dP - D) * F.SCA_SCALE
        dq[a:b] = dS @ k[lo:b]
        dk[lo:b] += dS.T @ q[a:b]
        dv[lo:b] += P.T @ dout[a:b]
    return dq, dk, dv


def _row_softmax(q_t, k_w):
    sc = F.SCA_SCALE * (k_w @ q_t)
    p = np.exp(sc - sc.max())
    return p / p.sum()


def sca_query_rows_backward(q, k, v, dout, c: int, rows):
    """dq of selected query rows, each from its own window (the same
    definition row by row; used for sampled checks of full-size runs)."""
    out = np.empty((len(rows), q.shape[1]))
    for n, t in enumerate(rows):
        t = int(t)
        lo = F.window_lo(t, c)
        p = _row_softmax(q[t], k[lo:t + 1])
        o = p @ v[lo:t + 1]
        ds = p * (v[lo:t + 1] @ dout[t] - dout[t] @ o) * F.SCA_SCALE
        out[n] = ds @ k[lo:t + 1]
    return out


def sca_key_rows_backward(q, k, v, dout, c: int, keys):
    """(dk, dv) of selected key rows: every query that sees the key (from
    the key itself to the end of the next chunk), each with the softmax of
    its own window."""
    T = q.shape[0]
    dk = np.zeros((len(keys), k.shape[1]))
    dv = np.zeros((len(keys), v.shape[1]))
    for n, u in enumerate(keys):
        u = int(u)
        for t in range(u, min(T, (u // c + 2) * c)):
            lo = F.window_lo(t, c)
            p = _row_softmax(q[t], k[lo:t + 1])
            o = p @ v[lo:t + 1]
            pu = p[u - lo]
            dv[n] += pu * dout[t]
            dk[n] += pu * (dout[t] @ v[u] - dout[t] @ o) * F.SCA_SCALE * q[t]
    return dk, dv


def awm_head_backward(qm, km, v, c: int, dout_mem, dM_final=None, dlogz_final=None):
    """(dqm, dkm, dv) of the AWM part of one head for the output gradient
    dout_mem [T, dv] and optional gradients of the exported state
    (dM_final [d, dv] for M'_{S+1}, dlogz_final [d] for log z^S)."""
    T, d = km.shape
    S = T // c
    _, M, L = F.awm_head(qm, km, v, c)            # M[s] = M'_s, s = 0..S+1; L[s-1] = log z^s
    l = F.chunk_log_exp_sums(km, c)               # l[s-1] = log e_s
    G = [np.zeros((d, v.shape[1])) for _ in range(S + 2)]
    if dM_final is not None:
        G[S + 1] = G[S + 1] + dM_final
    dqm = np.zeros_like(qm)
    dkm = np.zeros_like(km)
    dv = np.zeros_like(v)
    dL = np.zeros((S, d))
    if dlogz_final is not None:
        dL[S - 1] += dlogz_final
    rows = [slice((s - 1) * c, s * c) for s in range(S + 1)]   # rows[s] for 1-based s
    # readout O_m,s = Psiq_s M'_{s-1}
    for s in range(1, S + 1):
        Pq = F.psi(qm[rows[s]])
        G[s - 1] += Pq.T @ dout_mem[rows[s]]
        dqm[rows[s]] = _softmax_backward(Pq, dout_mem[rows[s]] @ M[s - 1].T)
    # carry M'_{s+1} = r_s (.) M'_s + Phi_s^T (V_s - Psi_s M'_s), in reverse
    for s in range(S, 0, -1):
        g = G[s + 1]
        ks = km[rows[s]]
        Phi = F.phi(ks, L[s - 1])
        Psi = F.psi(ks)
        r = F.z_ratio(L, s)
        R = v[rows[s]] - Psi @ M[s]
        dR = Phi @ g
        dv[rows[s]] += dR
        dPhi = R @ g.T
        dPsi = -dR @ M[s].T
        dr = (g * M[s]).sum(axis=1)
        G[s] = G[s] + r[:, None] * g - Psi.T @ dR
        t = dPhi * Phi
        dkm[rows[s]] += t + _softmax_backward(Psi, dPsi)
        dL[s - 1] -= t.sum(axis=0)
        if s >= 2:
            dL[s - 2] += dr * r
            dL[s - 1] -= dr * r
    return dqm, dkm + _log_z_backward(km, c, l, L, dL), dv


def _log_z_backward(km, c: int, l, L, dL):
    """K_m gradient routed through the denominators: L_s = logaddexp(L_{s-1}, l_s)
    with L_1 = l_1 (taken in reverse), then l_s = logsumexp over the chunk."""
    S = km.shape[0] // c
    dL = dL.copy()
    dkm = np.zeros_like(km)
    for s in range(S, 0, -1):
        rows = slice((s - 1) * c, s * c)
        dl = dL[s - 1] * np.exp(l[s - 1] - L[s - 1])
        if s >= 2:
            dL[s - 2] += dL[s - 1] * np.exp(L[s - 2] - L[s - 1])
        dkm[rows] = dl[None, :] * np.exp(km[rows] - l[s - 1][None, :])
    return dkm


def backward(q, k, v, qm, km, c: int, dout_sca, dout_mem):
    """Gradients of the whole path on [B, H, T, d] arrays for the output
    gradients dout_sca, dout_mem.  Returns (dq, dk, dv, dqm, dkm); dv sums the
    SCA and AWM contributions (V feeds both)."""
    q, k, v, qm, km, dos, dom = (np.asarray(x, dtype=np.float64)
                                 for x in (q, k, v, qm, km, dout_sca, dout_mem))
    B, H = q.shape[:2]
    dq, dk, dv = np.empty_like(q), np.empty_like(k), np.empty_like(v)
    dqm, dkm = np.empty_like(qm), np.empty_like(km)
    for b in range(B):
        for h in range(H):
            dq[b, h], dk[b, h], dv1 = sca_head_backward(q[b, h], k[b, h], v[b, h], c, dos[b, h])
            dqm[b, h], dkm[b, h], dv2 = awm_head_backward(qm[b, h], km[b, h], v[b, h], c, dom[b, h])
            dv[b, h] = dv1 + dv2
    return dq, dk, dv, dqm, dkm
