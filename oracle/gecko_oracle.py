"""Plain fp64 CPU oracle for the Gecko forward hot path: Sliding Chunk Attention
(SCA) and the Adaptive Working Memory (AWM) chunk recurrence.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  The product path
(the CUDA library and its Python binding) never calls it, and it shares no
code with that path.

Sources (two web pages on "Gecko: An Efficient Neural Architecture Inherently
Processing Sequences with Arbitrary Lengths", arXiv 2601.06463):
  [digest]  paper.rainbus.top Chinese digest, sections 核心方法 (core method:
            the online-softmax kernel phi^s, the cumulative denominator z^s,
            the feature softmax psi) and 方法步骤详情 (method step details:
            steps 3-5, SCA, the M'_s update, the readout, the output sum).
  [summary] paperlayer.ai summary, section 3.2 Sliding Chunk Attention,
            section 3.3 Adaptive Working Memory (tau_s = 1), Appendix A
            (delta rule; M_0 = 0; M'_1 = 0 with sliding chunks).

Readings taken where the pages are silent or garbled (each is listed in the
design notes with its reasoning):
  R1  SCA scale is 1 (the SCA formula in [digest] step 3 prints no 1/sqrt(d)).
  R2  inside the current chunk the mask is causal (key u <= query t); all c
      keys of the previous chunk are visible; chunk 1 attends only to itself.
  R3  the delta term is phi^{s-1}(K_{s-1})^T (V_{s-1} - psi(K_{s-1}) M'_{s-1}),
      the only form of the printed update that is a d x d matrix for c != d.
  R4  phi, psi and z use the memory keys K_m; the readout uses Q_m; V is the
      SCA value tensor.  z^s is a per-feature vector.
  R5  the z-ratio scales row f (key feature f) of M'.  z^0 = 0, so the ratio
      is 0 at s = 2 where it multiplies M'_1 = 0.
  R6  chunk s reads M'_{s-1} (which holds chunks <= s-2); M'_0 := 0, so chunks
      1 and 2 read zero.
  R7  the exported state is (M'_{S+1}, log z^S).
All arithmetic is float64.  Chunks are 1-based in the docstrings (chunk s
covers tokens (s-1)c .. sc-1, 0-based); arrays are 0-based.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "window_lo", "sca_head", "sca_rows", "chunk_log_exp_sums", "log_z",
    "phi", "psi", "z_ratio", "carry_step", "readout", "awm_head",
    "forward", "awm_propagate",
]


# --------------------------------------------------------------------------
# SCA: [digest] step 3, O_s = softmax(Q_s [K_{s-1}; K_s]^T) [V_{s-1}; V_s];
# [summary] 3.2 "attention over each current chunk and its preceding chunk".
# --------------------------------------------------------------------------

def window_lo(t: int, c: int) -> int:
    """First key index visible to query t: the first token of the previous
    chunk, or 0 in chunk 1 (reading R2)."""
    return max(0, (t // c - 1) * c)


def _masked_softmax_rows(scores: np.ndarray, allowed: np.ndarray) -> np.ndarray:
    """Row softmax over the allowed entries (max-subtracted exp)."""
    s = np.where(allowed, scores, -np.inf)
    m = s.max(axis=1, keepdims=True)
    p = np.exp(s - m)
    return p / p.sum(axis=1, keepdims=True)


SCA_SCALE = 1.0  # reading R1


def sca_head(q: np.ndarray, k: np.ndarray, v: np.ndarray, c: int) -> np.ndarray:
    """SCA output for one head; q, k, v are [T, d] float64, T % c == 0."""
    T = q.shape[0]
    out = np.empty((T, v.shape[1]), dtype=np.float64)
    for s0 in range(T // c):
        a, b = s0 * c, (s0 + 1) * c
        lo = window_lo(a, c)
        scores = SCA_SCALE * (q[a:b] @ k[lo:b].T)
        t = np.arange(a, b)[:, None]
        u = np.arange(lo, b)[None, :]
        out[a:b] = _masked_softmax_rows(scores, u <= t) @ v[lo:b]
    return out


def sca_rows(q, k, v, c: int, rows) -> np.ndarray:
    """SCA output of selected query rows only (same definition, row by row);
    used for sampled checks of full-size runs."""
    out = np.empty((len(rows), v.shape[1]), dtype=np.float64)
    for n, t in enumerate(rows):
        lo = window_lo(int(t), c)
        sc = SCA_SCALE * (k[lo:t + 1] @ q[t])
        p = np.exp(sc - sc.max())
        out[n] = (p / p.sum()) @ v[lo:t + 1]
    return out


# --------------------------------------------------------------------------
# AWM: [digest] 核心方法: phi^s(k_{s,t}) = exp(k_{s,t}) / z^s,
# z^s = sum_{t<=s} sum_{i<=c} exp(k_{t,i}),  psi(q) = exp(q) / sum_j exp(q_j).
# [digest] step 4: M'_s = (z^{s-2}/z^{s-1}) (.) M'_{s-1} + phi^{s-1}(K_{s-1})^T V_{s-1}
#                          - psi(K_{s-1}) M'_{s-1}   (read as R3).
# [digest] step 5: O_m = psi(Q_m) M'_{s-1}; output = SCA output + AWM output.
# [summary] Appendix A: delta rule, M'_1 = 0.
# --------------------------------------------------------------------------

def chunk_log_exp_sums(km: np.ndarray, c: int) -> np.ndarray:
    """log e_s[f] = log sum_{i in chunk s} exp(km[i, f]) -> [S, d]."""
    S = km.shape[0] // c
    kc = km.reshape(S, c, -1)
    mx = kc.max(axis=1)
    return mx + np.log(np.exp(kc - mx[:, None, :]).sum(axis=1))


def log_z(km: np.ndarray, c: int) -> np.ndarray:
    """log z^s for s = 1..S (row s-1), z^s = sum_{t<=s} e_t, in log space so
    that long sequences cannot overflow."""
    return np.logaddexp.accumulate(chunk_log_exp_sums(km, c), axis=0)


def phi(km_s: np.ndarray, logz_s: np.ndarray) -> np.ndarray:
    """phi^s(K_s) = exp(K_s) / z^s, per feature (reading R4)."""
    return np.exp(km_s - logz_s[None, :])


def psi(x: np.ndarray) -> np.ndarray:
    """Softmax along the feature dimension, row by row."""
    m = x.max(axis=-1, keepdims=True)
    e = np.exp(x - m)
    return e / e.sum(axis=-1, keepdims=True)


def z_ratio(logz: np.ndarray, s: int) -> np.ndarray:
    """z^{s-1} / z^s per feature for 1-based chunk s (0 for s = 1, R5)."""
    if s == 1:
        return np.zeros(logz.shape[1])
    return np.exp(logz[s - 2] - logz[s - 1])


def carry_step(M_s, km_s, v_s, logz, s: int, delta: bool = True) -> np.ndarray:
    """M'_{s+1} from M'_s and chunk s (the printed update with s -> s+1):
    M'_{s+1} = (z^{s-1}/z^s) (.) M'_s + phi^s(K_s)^T (V_s - psi(K_s) M'_s)."""
    Phi = phi(km_s, logz[s - 1])
    corr = psi(km_s) @ M_s if delta else 0.0
    return z_ratio(logz, s)[:, None] * M_s + Phi.T @ (v_s - corr)


def readout(qm_s: np.ndarray, M_prev: np.ndarray) -> np.ndarray:
    """O_m for chunk s = psi(Q_m,s) M'_{s-1} (R6)."""
    return psi(qm_s) @ M_prev


def awm_head(qm, km, v, c: int, delta: bool = True, keep_states: bool = True):
    """AWM for one head.  Returns (out_mem [T, dv], states, logz [S, d]) where
    states[s] = M'_s for s = 0..S+1 (states[0] = M'_0 := 0, states[1] = M'_1 = 0)
    if keep_states, else only [M'_S, M'_{S+1}]."""
    T, d = km.shape
    dv = v.shape[1]
    S = T // c
    lz = log_z(km, c)
    zero = np.zeros((d, dv))
    prev, cur = zero, zero                # M'_{s-1}, M'_s at s = 1
    states = [zero, zero]
    out = np.empty((T, dv))
    for s in range(1, S + 1):
        rows = slice((s - 1) * c, s * c)
        out[rows] = readout(qm[rows], prev)
        nxt = carry_step(cur, km[rows], v[rows], lz, s, delta)
        prev, cur = cur, nxt
        if keep_states:
            states.append(nxt)
    if not keep_states:
        states = [prev, cur]
    return out, states, lz


def forward(q, k, v, qm, km, c: int):
    """Whole path on [B, H, T, d] arrays (any float dtype; computed in fp64).
    Returns out_sca [B,H,T,d], out_mem [B,H,T,d], M [B,H,d,d] = M'_{S+1},
    logz [B,H,d] = log z^S (R7).  The layer output is out_sca + out_mem."""
    q, k, v, qm, km = (np.asarray(x, dtype=np.float64) for x in (q, k, v, qm, km))
    B, H, T, d = q.shape
    out_sca = np.empty((B, H, T, v.shape[-1]))
    out_mem = np.empty_like(out_sca)
    M = np.empty((B, H, d, v.shape[-1]))
    lz = np.empty((B, H, d))
    for b in range(B):
        for h in range(H):
            out_sca[b, h] = sca_head(q[b, h], k[b, h], v[b, h], c)
            om, st, l = awm_head(qm[b, h], km[b, h], v[b, h], c, keep_states=False)
            out_mem[b, h] = om
            M[b, h] = st[-1]
            lz[b, h] = l[-1]
    return out_sca, out_mem, M, lz


def awm_propagate(km_chunks, v_chunks, qm_chunks, c: int, want_chunks=()):
    """Streaming AWM for one head over chunk iterables (for long sequences).

    km_chunks / v_chunks / qm_chunks yield [c, d] arrays for s = 1..S in order.
    Returns ({s: out_mem of chunk s for s in want_chunks}, M'_{S+1}, log z^S).
    Same steps as awm_head, with z accumulated in log space chunk by chunk."""
    want = set(int(s) for s in want_chunks)
    got = {}
    prev = cur = None
    lz_prev = None
    s = 0
    for km_s, v_s, qm_s in zip(km_chunks, v_chunks, qm_chunks):
        s += 1
        km_s = np.asarray(km_s, dtype=np.float64)
        v_s = np.asarray(v_s, dtype=np.float64)
        if cur is None:
            prev = cur = np.zeros((km_s.shape[1], v_s.shape[1]))
        if s in want:
            got[s] = readout(np.asarray(qm_s, dtype=np.float64), prev)
        le = chunk_log_exp_sums(km_s, c)[0]
        lz_s = le if lz_prev is None else np.logaddexp(lz_prev, le)
        lz2 = np.stack([lz_prev if lz_prev is not None else lz_s, lz_s])
        if lz_prev is None:
            nxt = phi(km_s, lz_s).T @ (v_s - psi(km_s) @ cur)
        else:
            nxt = carry_step(cur, km_s, v_s, lz2, 2)
        prev, cur, lz_prev = cur, nxt, lz_s
    return got, cur, lz_prev
