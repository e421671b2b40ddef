"""Where the bf16 gradient bar comes from (oracle only, no GPU): a backward
that receives the forward's output rounded to bf16 (as every caller that
keeps its activations in bf16 supplies it) computes the SCA row term
delta = rowsum(dO * O) from the rounded O.  Evaluated entirely in the fp64
oracle, that rounding alone moves dq by several 1e-3 in rel-L2 on the
Z'-affine workloads, more than the forward's 5e-3 bar leaves room for, and
well inside the 1e-2 the GPU gradient tests use."""
import numpy as np
import torch

from long_context_sequence_sca_b200.inputs import Workload, make_inputs
from oracle import gecko_oracle as F


def _dq(q, k, v, do, c, round_o):
    dq = np.zeros_like(q)
    for s0 in range(q.shape[0] // c):
        a, b = s0 * c, (s0 + 1) * c
        lo = F.window_lo(a, c)
        t = np.arange(a, b)[:, None]
        u = np.arange(lo, b)[None, :]
        P = F._masked_softmax_rows(q[a:b] @ k[lo:b].T, u <= t)
        O = P @ v[lo:b]
        if round_o:
            O = torch.tensor(O).bfloat16().double().numpy()
        delta = (do[a:b] * O).sum(axis=1, keepdims=True)
        dq[a:b] = (P * (do[a:b] @ v[lo:b].T - delta)) @ k[lo:b]
    return dq


def test_bf16_output_rounding_floor_of_dq():
    w = Workload("floor", 71, "bf16", 1, 1, 2048, 64, 256)
    x = make_inputs(w, device="cpu")
    q, k, v = (x[n][0, 0].double().numpy() for n in ("q", "k", "v"))
    do = torch.randn(q.shape, generator=torch.Generator().manual_seed(1)).bfloat16().double().numpy()
    exact = _dq(q, k, v, do, w.c, False)
    rounded = _dq(q, k, v, do, w.c, True)
    rel = np.linalg.norm(rounded - exact) / np.linalg.norm(exact)
    assert 2e-3 < rel < 1e-2, rel
