"""Context parallelism: one sequence split into P consecutive segments, one
per rank, with outputs equal to a single forward over the whole sequence (up
to rounding).

What crosses ranks (the only exchange steps of the method):
  * SCA: the previous segment's last chunk of K and V (a halo of c rows,
    sent from rank r to rank r + 1), because every chunk attends its
    predecessor (Gecko digest, paper.rainbus.top, method step details,
    step 3).
  * AWM: the carry M'_{s+1} = A_s M'_s + b_s is affine in the state once
    log z is known, and log z is a prefix of per-chunk exp-sums (core method;
    step 4).  So two all-gathers suffice: every rank's log-exp-sum (d values
    per head), from which each rank gets the log z entering its segment, and
    then every rank's segment maps (A, b, A', b'), d x d each per head,
    computed with that log z; composing the maps of the ranks before it gives
    a rank its incoming state.  Each rank then runs the streaming forward of
    its segment from that state.

The arithmetic of every step runs in the library's CUDA kernels
(`GpuBackend`); this module only moves tensors between ranks.  The phases
are separate functions so that the same steps run under torch.distributed
(`cp_forward`, one process per GPU; NCCL on GPUs) or for all segments in one
process (`cp_forward_emulated`).
"""
from __future__ import annotations

import torch

from . import lib as L


class GpuBackend:
    """The library's entry points for each phase (CUDA tensors)."""

    def segment_logsum(self, seg, c):
        return L.awm_segment_logsum(seg["km"], c)

    def cp_logz(self, lsum_all, rank):
        return L.awm_cp_logz(lsum_all, rank)

    def segment_maps(self, seg, logz_in, c):
        return L.awm_segment_maps(seg["km"], seg["v"], logz_in, c)

    def cp_state(self, lsum_all, maps_all, rank):
        return L.awm_cp_state(lsum_all, maps_all, rank)

    def forward(self, seg, c, halo, state_in):
        """(out_sca, out_mem) of one segment; halo [2, B, H, c, d] is the
        previous segment's last chunk of K and V (None for the first)."""
        if state_in is None:
            return L.sca_awm_forward(seg["q"], seg["k"], seg["v"], seg["qm"], seg["km"], c)
        k = torch.cat([halo[0], seg["k"]], dim=2).contiguous()
        v = torch.cat([halo[1], seg["v"]], dim=2).contiguous()
        out_sca, out_mem, _ = L.sca_awm_forward_segment(seg["q"], k, v, seg["qm"], seg["km"], c, state_in=state_in)
        return out_sca, out_mem


def halo_of(seg, c):
    """The last chunk of K and V of a segment, [2, B, H, c, d]."""
    return torch.stack([seg["k"][:, :, -c:], seg["v"][:, :, -c:]]).contiguous()


def phase_logsum(seg, c, backend):
    return backend.segment_logsum(seg, c)


def phase_maps(seg, c, lsum_all, rank, backend):
    return backend.segment_maps(seg, backend.cp_logz(lsum_all, rank), c)


def phase_forward(seg, c, rank, halo, lsum_all, maps_all, backend):
    state = backend.cp_state(lsum_all, maps_all, rank) if rank > 0 else None
    return backend.forward(seg, c, halo if rank > 0 else None, state)


def _check_segment(seg, c):
    T = seg["q"].shape[2]
    if T % c != 0:
        raise ValueError(f"segment length {T} is not a multiple of the chunk size {c}")


def cp_forward(seg, c: int, group=None, backend=None):
    """This rank's (out_sca, out_mem) for its segment `seg` (dict of q, k, v,
    qm, km, [B, H, T, d], T % c == 0) of a sequence split over the ranks of
    `group` in rank order."""
    import torch.distributed as dist
    backend = backend or GpuBackend()
    _check_segment(seg, c)
    rank, P = dist.get_rank(group), dist.get_world_size(group)

    def peer(r):
        return dist.get_global_rank(group, r) if group is not None else r

    # SCA halo: send the last chunk to the next rank, receive the previous one
    send = halo_of(seg, c)
    recv = torch.empty_like(send)
    ops = []
    if rank + 1 < P:
        ops.append(dist.P2POp(dist.isend, send, peer(rank + 1), group))
    if rank > 0:
        ops.append(dist.P2POp(dist.irecv, recv, peer(rank - 1), group))
    reqs = dist.batch_isend_irecv(ops) if ops else []

    # AWM: log-sums, then segment maps under the right log z
    lsum = phase_logsum(seg, c, backend)
    parts = [torch.empty_like(lsum) for _ in range(P)]
    dist.all_gather(parts, lsum.contiguous(), group=group)
    lsum_all = torch.stack(parts)
    maps = phase_maps(seg, c, lsum_all, rank, backend)
    parts = [torch.empty_like(maps) for _ in range(P)]
    dist.all_gather(parts, maps.contiguous(), group=group)
    maps_all = torch.stack(parts)

    for r in reqs:
        r.wait()
    return phase_forward(seg, c, rank, recv, lsum_all, maps_all, backend)


def cp_forward_emulated(segments, c: int, backend=None):
    """The same phases for all P segments in one process (the exchanges
    become list indexing).  Returns [(out_sca, out_mem)] per segment."""
    backend = backend or GpuBackend()
    for seg in segments:
        _check_segment(seg, c)
    lsum_all = torch.stack([phase_logsum(seg, c, backend) for seg in segments])
    maps_all = torch.stack([phase_maps(seg, c, lsum_all, r, backend) for r, seg in enumerate(segments)])
    halos = [None] + [halo_of(seg, c) for seg in segments[:-1]]
    return [phase_forward(seg, c, r, halos[r], lsum_all, maps_all, backend) for r, seg in enumerate(segments)]
