"""Context parallelism on the CPU: 2 and 3 gloo ranks run cp.cp_forward (the
same orchestration as on GPUs: halo send/receive, the two all-gathers, the
composition of segment maps) with a backend made of oracle steps in fp64, and
each rank's outputs must equal the oracle's forward over the whole sequence.
A backend with a plausible slip (maps composed in the wrong order) must fail."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from long_context_sequence_sca_b200 import cp
from oracle import gecko_oracle as F


def _lse(x, axis):
    return np.logaddexp.reduce(x, axis=axis)


class OracleBackend:
    """Each phase computed with the oracle's steps (fp64 CPU tensors)."""

    reverse_compose = False   # planted slip for the negative test

    def segment_logsum(self, seg, c):
        km = seg["km"].numpy()
        out = np.array([[_lse(F.chunk_log_exp_sums(km[b, h], c), 0) for h in range(km.shape[1])]
                        for b in range(km.shape[0])])
        return torch.from_numpy(out)

    def cp_logz(self, lsum_all, rank):
        a = lsum_all.numpy()
        out = np.full(a.shape[1:], -np.inf) if rank == 0 else _lse(a[:rank], 0)
        return torch.from_numpy(out)

    def segment_maps(self, seg, logz_in, c):
        km, v = seg["km"].numpy(), seg["v"].numpy()
        B, H, T, d = km.shape
        out = np.empty((B, H, 4, d, d))
        for b in range(B):
            for h in range(H):
                lz = logz_in.numpy()[b, h]
                A, bb = np.eye(d), np.zeros((d, d))
                A2, b2 = np.eye(d), np.zeros((d, d))
                for s in range(T // c):
                    rows = slice(s * c, (s + 1) * c)
                    le = F.chunk_log_exp_sums(km[b, h, rows], c)[0]
                    lzn = np.logaddexp(lz, le)
                    r = np.exp(lz - lzn)
                    Phi, Psi = F.phi(km[b, h, rows], lzn), F.psi(km[b, h, rows])
                    As = np.diag(r) - Phi.T @ Psi
                    bs = Phi.T @ v[b, h, rows]
                    A2, b2 = A, bb
                    A, bb = As @ A, As @ bb + bs
                    lz = lzn
                out[b, h] = A, bb, A2, b2
        return torch.from_numpy(out)

    def cp_state(self, lsum_all, maps_all, rank):
        maps = maps_all.numpy()
        lz = self.cp_logz(lsum_all, rank).numpy()
        B, H, _, d, _ = maps.shape[1:]
        state = np.zeros((B, H, 2 * d * d + d))
        order = range(rank - 1, -1, -1) if self.reverse_compose else range(rank)
        for b in range(B):
            for h in range(H):
                M = np.zeros((d, d))
                Mprev = np.zeros((d, d))
                for j in order:
                    A, bb, A2, b2 = maps[j, b, h]
                    if j == rank - 1:
                        Mprev = A2 @ M + b2
                    M = A @ M + bb
                state[b, h] = np.concatenate([Mprev.ravel(), M.ravel(), lz[b, h]])
        return torch.from_numpy(state)

    def forward(self, seg, c, halo, state_in):
        q, k, v, qm, km = (seg[n].numpy() for n in ("q", "k", "v", "qm", "km"))
        B, H, T, d = q.shape
        out_sca, out_mem = np.empty_like(q), np.empty_like(q)
        for b in range(B):
            for h in range(H):
                if halo is None:
                    out_sca[b, h] = F.sca_head(q[b, h], k[b, h], v[b, h], c)
                else:
                    hk, hv = halo.numpy()[:, b, h]
                    qx = np.concatenate([np.zeros((c, d)), q[b, h]])
                    o = F.sca_head(qx, np.concatenate([hk, k[b, h]]), np.concatenate([hv, v[b, h]]), c)
                    out_sca[b, h] = o[c:]
                if state_in is None:
                    prev = cur = np.zeros((d, d))
                    lz = None
                else:
                    st = state_in.numpy()[b, h]
                    prev, cur, lz = st[:d * d].reshape(d, d), st[d * d:2 * d * d].reshape(d, d), st[2 * d * d:]
                for s in range(T // c):
                    rows = slice(s * c, (s + 1) * c)
                    out_mem[b, h, rows] = F.psi(qm[b, h, rows]) @ prev
                    le = F.chunk_log_exp_sums(km[b, h, rows], c)[0]
                    lzn = le if lz is None else np.logaddexp(lz, le)
                    r = np.zeros(d) if lz is None else np.exp(lz - lzn)
                    Phi = F.phi(km[b, h, rows], lzn)
                    nxt = r[:, None] * cur + Phi.T @ (v[b, h, rows] - F.psi(km[b, h, rows]) @ cur)
                    prev, cur, lz = cur, nxt, lzn
        return torch.from_numpy(out_sca), torch.from_numpy(out_mem)


def _inputs(P, B=1, H=2, S_per=3, c=4, d=3, seed=0):
    rng = np.random.default_rng(seed)
    T = P * S_per * c
    x = {n: rng.normal(size=(B, H, T, d)) * (1.0 if n == "v" else 0.8) for n in ("q", "k", "v", "qm", "km")}
    return x, T


def _worker(rank, P, port, c, reverse, errq):
    try:
        os.environ["MASTER_ADDR"] = "127.0.0.1"
        os.environ["MASTER_PORT"] = str(port)
        dist.init_process_group("gloo", rank=rank, world_size=P)
        x, T = _inputs(P)
        Tr = T // P
        seg = {n: torch.from_numpy(a[:, :, rank * Tr:(rank + 1) * Tr].copy()) for n, a in x.items()}
        be = OracleBackend()
        be.reverse_compose = reverse
        o_sca, o_mem = cp.cp_forward(seg, c, backend=be)
        want_sca, want_mem, _, _ = F.forward(x["q"], x["k"], x["v"], x["qm"], x["km"], c)
        ok_sca = np.allclose(o_sca.numpy(), want_sca[:, :, rank * Tr:(rank + 1) * Tr], rtol=1e-10, atol=1e-12)
        ok_mem = np.allclose(o_mem.numpy(), want_mem[:, :, rank * Tr:(rank + 1) * Tr], rtol=1e-10, atol=1e-12)
        errq.put((rank, bool(ok_sca), bool(ok_mem)))
        dist.barrier()
        dist.destroy_process_group()
    except Exception as e:  # pragma: no cover - reported to the parent
        errq.put((rank, repr(e), None))


def _worker_groups(rank, port, errq):
    """Four ranks in two process groups of two, each group running the
    context-parallel forward of its own sequence: the halo peers and the
    gathers must stay inside the group (group ranks mapped to global ones)."""
    try:
        os.environ["MASTER_ADDR"] = "127.0.0.1"
        os.environ["MASTER_PORT"] = str(port)
        dist.init_process_group("gloo", rank=rank, world_size=4)
        groups = [dist.new_group([0, 1]), dist.new_group([2, 3])]
        seq = rank // 2
        grp = groups[seq]
        r = dist.get_rank(grp)
        x, T = _inputs(2, seed=10 + seq)
        Tr = T // 2
        seg = {n: torch.from_numpy(a[:, :, r * Tr:(r + 1) * Tr].copy()) for n, a in x.items()}
        o_sca, o_mem = cp.cp_forward(seg, 4, group=grp, backend=OracleBackend())
        want_sca, want_mem, _, _ = F.forward(x["q"], x["k"], x["v"], x["qm"], x["km"], 4)
        ok_sca = np.allclose(o_sca.numpy(), want_sca[:, :, r * Tr:(r + 1) * Tr], rtol=1e-10, atol=1e-12)
        ok_mem = np.allclose(o_mem.numpy(), want_mem[:, :, r * Tr:(r + 1) * Tr], rtol=1e-10, atol=1e-12)
        errq.put((rank, bool(ok_sca), bool(ok_mem)))
        dist.barrier()
        dist.destroy_process_group()
    except Exception as e:  # pragma: no cover - reported to the parent
        errq.put((rank, repr(e), None))


class FailingBackend(OracleBackend):
    """A rank whose first phase fails on the host: it raises, or it stalls
    (sleeps past the group's timeout before going on)."""

    def __init__(self, mode):
        self.mode = mode

    def segment_logsum(self, seg, c):
        if self.mode == "raise":
            raise RuntimeError("injected failure")
        import time
        time.sleep(8)
        return super().segment_logsum(seg, c)


def _worker_fail(rank, P, port, fail_rank, mode, errq):
    """Every rank runs cp_forward under a 3 s process-group timeout; rank
    `fail_rank` fails in its first phase.  Each rank reports how its call
    ended, then exits without tearing the group down (a peer may be gone)."""
    from datetime import timedelta
    try:
        os.environ["MASTER_ADDR"] = "127.0.0.1"
        os.environ["MASTER_PORT"] = str(port)
        dist.init_process_group("gloo", rank=rank, world_size=P, timeout=timedelta(seconds=3))
        x, T = _inputs(P)
        Tr = T // P
        seg = {n: torch.from_numpy(a[:, :, rank * Tr:(rank + 1) * Tr].copy()) for n, a in x.items()}
        be = FailingBackend(mode) if rank == fail_rank else OracleBackend()
        try:
            cp.cp_forward(seg, 4, backend=be)
            errq.put((rank, "completed"))
        except Exception as e:
            errq.put((rank, f"{type(e).__name__}: {e}"[:300]))
    except Exception as e:  # pragma: no cover - reported to the parent
        errq.put((rank, f"setup {e!r}"))
    errq.close()
    errq.join_thread()
    os._exit(0)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _run(P, reverse=False, groups=False):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    if groups:
        procs = [ctx.Process(target=_worker_groups, args=(r, port, q)) for r in range(P)]
    else:
        procs = [ctx.Process(target=_worker, args=(r, P, port, 4, reverse, q)) for r in range(P)]
    for p in procs:
        p.start()
    res = []
    try:
        for _ in range(P):   # a rank stuck in a collective ends the test here
            res.append(q.get(timeout=120))
    finally:
        for p in procs:
            p.join(timeout=10)
            if p.is_alive():
                p.kill()
    return sorted(res, key=lambda t: t[0])


@pytest.mark.parametrize("P", [2, 3])
def test_context_parallel_equals_whole_sequence(P):
    res = _run(P)
    for rank, ok_sca, ok_mem in res:
        assert ok_sca is True and ok_mem is True, res


def test_wrong_composition_order_is_caught():
    res = _run(3, reverse=True)
    assert res[0][1] is True and res[0][2] is True   # rank 0 needs no state
    assert not all(r[2] is True for r in res)


def test_two_sequences_in_two_process_groups():
    res = _run(4, groups=True)
    for rank, ok_sca, ok_mem in res:
        assert ok_sca is True and ok_mem is True, res


@pytest.mark.parametrize("fail_rank,mode", [(0, "raise"), (1, "raise"), (1, "stall")])
def test_a_failed_rank_ends_the_others_calls(fail_rank, mode):
    """Failure detection on the host: when one rank of a context-parallel
    forward fails before its collectives (raises and leaves, or stalls past
    the group's timeout), the other ranks' calls end with an error (the
    gather's peer closed, or the timeout) instead of waiting for good."""
    import time
    P = 3
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker_fail, args=(r, P, port, fail_rank, mode, q)) for r in range(P)]
    t0 = time.time()
    for p in procs:
        p.start()
    res = []
    try:
        for _ in range(P):
            res.append(q.get(timeout=120))
    finally:
        for p in procs:
            p.join(timeout=30)
            if p.is_alive():
                p.kill()
    res = dict(res)
    if mode == "raise":
        assert "injected failure" in res[fail_rank], res
    for r in range(P):
        if r != fail_rank:
            assert res[r] != "completed" and not res[r].startswith("setup"), res
    assert time.time() - t0 < 100
