"""Host logic of bench.py: the algorithmic work counts and the multi-rank
aggregation (world size 2 over gloo on CPU)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from long_context_sequence_sca_b200.inputs import Workload


def test_sca_pair_count_matches_mask_enumeration():
    for c, S in ((4, 1), (4, 3), (8, 5)):
        w = Workload("t", 0, "bf16", 1, 1, c * S, 64, c)
        n = sum(1 for t in range(w.T) for u in range(w.T) if u <= t and u // c >= t // c - 1)
        assert bench.sca_pairs(w) == n


def test_flops_and_bytes_headline():
    w = bench.WORKLOADS["bf16_h32_c4096"]
    f = bench.flops(w)
    assert abs(f["sca"] / 1e12 - 3.024) < 0.01
    assert abs(f["awm"] / 1e9 - 120.3) < 0.5
    assert bench.io_bytes(w) == 7 * 32 * 32768 * 128 * 2


def test_awm_plan_and_launch_count():
    """The plan bench.py assumes when it counts launches (the library's own
    rule: k CTAs per chunk when that saves a quarter of waves x (tiles per
    CTA + 2), the statistics fused only with one CTA per chunk)."""
    sms = 148
    # 256 chunks fill one wave of two CTAs per SM: one CTA per chunk, fused
    # statistics (first-tile pass, redo pass, prefix, carry, readout, SCA)
    assert bench.awm_plan(bench.WORKLOADS["bf16_h32_c4096"], sms) == (True, 1)
    # 32 chunks of 64 tiles: nine CTAs each (288 CTAs, 7-8 tiles, one wave)
    assert bench.awm_plan(bench.WORKLOADS["bf16_h4_c4096"], sms) == (False, 9)
    # c = 256 has 4 tiles per chunk: never split
    assert bench.awm_plan(bench.WORKLOADS["bf16_many_chunks"], sms) == (True, 1)
    # fp32 takes the CUDA-core kernels: separate statistics pass
    assert bench.awm_plan(bench.WORKLOADS["fp32_small"], sms) == (False, 1)
    # one wave with P CTAs per chunk costs (n + 2P) / P against n + 2 for one
    w = bench.WORKLOADS["bf16_h4_c4096"]
    n = w.c // 64
    assert (n + 2 * 9) / 9 <= 0.75 * (n + 2)
    if not torch.cuda.is_available():   # the counts below assume 148 SMs
        # fused: chunk pass, redo pass, prefix, carry, readout, SCA
        assert bench.forward_launches(bench.WORKLOADS["bf16_h32_c4096"]) == 6
        # split: partial + combine + prefix, chunk, Cm image, carry, readout, SCA
        assert bench.forward_launches(bench.WORKLOADS["bf16_h4_c4096"]) == 8


def test_secondary_rooflines_at_the_bench_workload():
    """HBM and SFU bounds: 1.88 GB in 3.44 ms is 546 GB/s; 5.91e9
    exponentials in 2.97 ms at 1965 MHz against 16 per clock on 148 SMs
    (4653 G/s) is 0.43 of the SFU rate."""
    w = bench.WORKLOADS["bf16_h32_c4096"]
    r = bench.secondary_rooflines(w, 3.44, 2.97, 1965, 6545.3)
    assert abs(r["hbm"]["achieved_gbs"] - 7 * 32 * 32768 * 128 * 2 / 3.44e-3 / 1e9) < 0.1
    assert r["sfu"]["exps_per_launch"] == 32 * (8 * 4096 * 4097 // 2 + 7 * 4096 * 4096)
    assert abs(r["sfu"]["peak_gexp_s"] - 16 * 148 * 1.965) < 0.1
    assert 0.42 < r["sfu"]["frac"] < 0.44
    assert "sfu" not in bench.secondary_rooflines(w, 3.44, 2.97, None, 6545.3)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, ws, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws)
    try:
        agg = bench.aggregate(ms_local=2.0 + rank, tokens_local=1000, ws=ws)
        q.put((rank, agg))
    finally:
        dist.destroy_process_group()


def test_aggregate_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    got = dict(q.get(timeout=120) for _ in ps)
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in (0, 1):
        assert got[r]["ms_per_step"] == 3.0
        assert abs(got[r]["value"] - 2000 / 3e-3) < 1e-6


def test_clock_rejection_rules():
    assert bench.clocks_rejected({"samples": 5, "reasons": ["hw_slowdown"], "sm_mhz": 1800, "sm_max_mhz": 1965})
    assert not bench.clocks_rejected({"samples": 5, "reasons": ["sw_power_cap"], "sm_mhz": 1300, "sm_max_mhz": 1965})
    assert bench.clocks_rejected({"samples": 5, "reasons": [], "sm_mhz": 600, "sm_max_mhz": 1965})
