#!/usr/bin/env python
"""Throughput of the fused Gecko SCA + AWM forward (tokens/s, bf16).

Default workload: the 7B-layer-shaped case B=1, H=32, d=128, c=4096,
T=32768 (8 chunks), synthetic inputs from the seeded generator, all resident
in HBM (1.34 GB of inputs, larger than the 126 MB L2, so no L2 flush is
needed between steps).  One step = one forward through the C ABI
(AWM statistics, chunk products, carry, readout, SCA).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl gecko|reference]

N > 1 runs under torchrun, one rank per GPU, each rank a full replica of the
workload on its own inputs (weak scaling; the heads and batches of the method
are independent, so there is no data-path collective).  The timed region is
bracketed by a barrier and a device synchronise; the step time is the max
over ranks; rank 0 prints one JSON line.

`--impl reference` times the CPU oracle (fp64 NumPy, the host's cores) on
bounded samples of the same workload instead.

`--op backward` measures gecko_sca_awm_backward on the same workload (the
gradients of q, k, v, qm, km for N(0,1) output gradients); its roofline is
the SCA dK/dV kernel against the bf16 tensor peak.
`--op cp` runs the forward as context-parallel segments (--segments, every
rank's phases emulated in one process on one GPU) and reports the whole-
sequence forward of the same run beside it.
`--op tdnorm` measures timestep decay normalisation on the same x shape
(HBM roofline).  `--op cema` measures the CEMA recurrence (gecko_cema_forward) instead, on
x [1, 32768, 4096] bf16 with h = 16, and prints its own JSON line (an FP32
ALU-bound kernel: roofline against the FP32 FMA rate of 148 SMs x 128 lanes
at the sampled SM clock).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from long_context_sequence_sca_b200.inputs import (  # noqa: E402
    CEMA_WORKLOADS, NORM_WORKLOADS, WORKLOADS, CemaWorkload, NormWorkload, Workload, make_cema_inputs, make_inputs,
    make_norm_inputs)

DEFAULT_WORKLOAD = "bf16_h32_c4096"
METRIC = "tokens/s fused SCA+AWM fwd (bf16,H=32,d=128,c=4096); % bf16 TC peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
SCA_PROFILE = os.path.join(ROOT, "profiles", "sca_tc_traffic_bf16_h32_c4096.md")


# ------------------------------------------------------- algorithmic work --

def sca_pairs(w: Workload) -> int:
    """(query, key) pairs the SCA must score per (b, h): chunk 1 is causal over
    itself; every later chunk sees all c previous keys plus its causal part."""
    S, c = w.S, w.c
    return S * c * (c + 1) // 2 + (S - 1) * c * c


def flops(w: Workload) -> dict:
    """Algorithmic FLOPs (2 per multiply-add) of one forward."""
    BH, c, d, S = w.B * w.H, w.c, w.d, w.S
    f_sca = 4 * d * sca_pairs(w) * BH                    # QK^T and PV
    # AWM: chunk products Phi^T V (all S) and Phi^T Psi (S-1 needed), the
    # d x d carry product C M' (S-1), and the readout of chunks 3..S.
    f_awm = (2 * c * d * d + (S - 1) * 6 * c * d * d + max(S - 2, 0) * 2 * c * d * d) * BH
    return {"sca": f_sca, "awm": f_awm, "total": f_sca + f_awm}


def io_bytes(w: Workload) -> int:
    """Algorithmic HBM bytes: five inputs read once, two outputs written once."""
    esz = 2 if w.dtype == "bf16" else 4
    return 7 * w.B * w.H * w.T * w.d * esz


def awm_plan(w: Workload, sms: int = 148) -> tuple:
    """(fused, parts) as the library chooses them for a forward: `parts` CTAs
    per chunk of the tensor-core chunk kernel (several when the chunks are
    too few to fill two CTAs per SM), and whether the chunk kernel computes
    each chunk's K_m statistics itself (one CTA per chunk) instead of a
    separate statistics pass."""
    if not (w.dtype == "bf16" and w.c % 128 == 0):
        return False, 1
    ctas, slots, n = w.B * w.H * w.S, 2 * sms, w.c // 64

    def cost(P):   # waves x (tiles per CTA + 2), times P
        return -(-ctas * P // slots) * (n + 2 * P)

    best = 1
    for P in range(2, min(n // 4, 16) + 1):
        if cost(P) * best < cost(best) * P:
            best = P
    parts = best if best > 1 and 4 * cost(best) <= 3 * cost(1) * best else 1
    return parts == 1, parts


def _sms() -> int:
    try:
        return torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    except Exception:
        return 148


def fused_stats(w: Workload) -> bool:
    """The chunk kernel computes each chunk's K_m statistics itself (no
    separate pass over K_m)."""
    return awm_plan(w, _sms())[0]


def forward_launches(w: Workload) -> int:
    """Kernels of one forward: [statistics partial + combine] or nothing,
    chunk products, [the fix-up pass of the fused statistics (its CTAs
    return at once unless their chunk outgrew the first tile's reference)],
    [Cm image when several CTAs share a chunk at d = 128], prefix, carry,
    readout, SCA."""
    fused, parts = awm_plan(w, _sms())
    return (1 if fused else 2) + 1 + (1 if parts > 1 and w.d == 128 else 0) + 4


def stage_bytes(w: Workload) -> dict:
    """Algorithmic HBM bytes of each timed stage that moves the inputs or
    outputs: the statistics read K_m (a stage of its own unless the chunk
    kernel computes them), the chunk products read K_m and V, the readout
    reads Q_m and writes out_mem, SCA reads Q, K, V and writes out_sca.  The
    carry and the prefix over chunks only touch the O(S d) and O(S d^2)
    workspace."""
    esz = 2 if w.dtype == "bf16" else 4
    t = w.B * w.H * w.T * w.d * esz
    out = {"awm_chunk": 2 * t, "awm_readout": 2 * t, "sca": 4 * t}
    if not fused_stats(w):
        out["awm_stats"] = t
    return out


def hbm_bound(w: Workload, pk: dict) -> bool:
    """Arithmetic intensity of the step below the ridge of the measured peaks."""
    return flops(w)["total"] / io_bytes(w) < pk["bf16_tflops"] * 1e12 / (pk["hbm_gbs"] * 1e9)


# exp2 results per clock per SM of the special-function units (the public
# arithmetic-throughput table's figure for compute capability 10.0)
SFU_EXP_PER_CLK_SM = 16
N_SM = 148
L2_BYTES = 126 * 1024 * 1024


def secondary_rooflines(w: Workload, ms_per_step: float, sca_ms: float, sm_mhz, hbm_gbs: float) -> dict:
    """The two other bounds of the forward: the step's algorithmic HBM bytes
    over its time against the measured copy bandwidth, and the SCA kernel's
    exponentials (one per visible (query, key) pair) over its launch time
    against the SFU issue rate at the sampled SM clock."""
    gbs = io_bytes(w) / (ms_per_step / 1e3) / 1e9
    exps = sca_pairs(w) * w.B * w.H
    out = {"hbm": {"algorithmic_bytes_per_step": io_bytes(w), "achieved_gbs": round(gbs, 1),
                   "peak_gbs": hbm_gbs, "frac": round(gbs / hbm_gbs, 4)}}
    if sm_mhz:
        g_exp = exps / (sca_ms / 1e3) / 1e9
        peak = SFU_EXP_PER_CLK_SM * N_SM * sm_mhz / 1e3
        out["sfu"] = {"kernel": "sca_tc_kernel", "exps_per_launch": exps, "achieved_gexp_s": round(g_exp, 1),
                      "peak_gexp_s": round(peak, 1), "frac": round(g_exp / peak, 4),
                      "clock": f"{sm_mhz} MHz (sampled)"}
    return out


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------- clocks --

class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML (read-only) in a
    background thread while the timed region runs."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.ok = False
        self.samples = []
        self.period = period_s
        try:
            import pynvml as nv
            nv.nvmlInit()
            self.nv = nv
            self.h = self._handle(device_index)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # pragma: no cover - depends on the machine
            self.err = repr(e)

    def _handle(self, idx):
        nv = self.nv
        props = torch.cuda.get_device_properties(idx)
        uuid = getattr(props, "uuid", None)
        if uuid is not None:
            s = str(uuid)
            for cand in (s if s.startswith("GPU-") else "GPU-" + s,):
                try:
                    return nv.nvmlDeviceGetHandleByUUID(cand)
                except Exception:
                    pass
        bus = getattr(props, "pci_bus_id", None)
        dom = getattr(props, "pci_domain_id", 0)
        dev = getattr(props, "pci_device_id", 0)
        if bus is not None:
            return nv.nvmlDeviceGetHandleByPciBusId(f"{dom:08x}:{bus:02x}:{dev:02x}.0")
        return nv.nvmlDeviceGetHandleByIndex(idx)

    def _reasons(self):
        nv = self.nv
        fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
        return int(fn(self.h))

    def _loop(self):
        while not self._stop.is_set():
            try:
                self.samples.append((self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM),
                                     self._reasons()))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        self.samples = []
        if not self.ok:
            return
        self._stop = threading.Event()
        self._t = threading.Thread(target=self._loop, daemon=True)
        self._t.start()

    def stop(self) -> dict:
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "error": getattr(self, "err", "nvml unavailable")}
        self._stop.set()
        self._t.join()
        mhz = [m for m, _ in self.samples]
        bits = 0
        for _, r in self.samples:
            bits |= r
        reasons = sorted(name for b, name in self.REASONS.items() if bits & b)
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(mhz), "source": "nvml"}


BAD_REASONS = {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"}


def clocks_rejected(ck: dict) -> bool:
    if not ck.get("samples"):
        return False
    if BAD_REASONS & set(ck["reasons"]):
        return True
    # stuck well below max with no reason: a leftover clock lock
    return bool(ck["sm_mhz"] and ck["sm_max_mhz"] and not ck["reasons"]
                and ck["sm_mhz"] < 0.6 * ck["sm_max_mhz"])


# ------------------------------------------------------------ multi-rank --

def dist_setup():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, ws: int) -> float:
    """Max of a per-rank scalar (the step time) over all ranks."""
    if ws == 1:
        return float(x)
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(ms_local: float, tokens_local: int, ws: int) -> dict:
    """Whole-job throughput: all ranks' tokens over the slowest rank's time."""
    ms = max_over_ranks(ms_local, ws)
    return {"ms_per_step": ms, "value": tokens_local * ws / (ms / 1e3)}


# ------------------------------------------------------------ CPU oracle --

def oracle_sample(w: Workload, n_chunks: int, head: int = 0):
    """A bounded sample of the workload for the CPU oracle: the first
    n_chunks chunks of one (b, h) head, drawn by the same generator recipe
    (shapes, c, d and distributions of the workload)."""
    sw = w.with_(B=1, H=1, T=n_chunks * w.c, dtype="f32", name=w.name + "_sample", wid=w.wid * 10 + head)
    x = make_inputs(sw, device="cpu")
    return {k_: v_.to(torch.bfloat16).double().numpy() if w.dtype == "bf16" else v_.double().numpy()
            for k_, v_ in x.items()}, sw.T


def time_oracle(w: Workload, n_chunks: int, reps: int = 1, head: int = 0):
    from oracle import gecko_oracle as G
    tot_s, tot_tok = 0.0, 0
    for r in range(reps):
        x, tok = oracle_sample(w, n_chunks, head + r)
        t0 = time.perf_counter()
        G.forward(x["q"], x["k"], x["v"], x["qm"], x["km"], w.c)
        tot_s += time.perf_counter() - t0
        tot_tok += tok
    return tot_tok / tot_s, tot_s, tot_tok


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


# --------------------------------------------------------- traffic record --

def source_hash(files=("sca_tc.cu", "common.cuh")) -> str:
    h = hashlib.sha1()
    for f in files:
        with open(os.path.join(ROOT, "long_context_sequence_sca_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:12]


def sca_source_hash() -> str:
    return source_hash(("sca_tc.cu", "common.cuh"))


CEMA_PROFILE = os.path.join(ROOT, "profiles", "cema_bf16_7b_32k.md")
NORM_PROFILE = os.path.join(ROOT, "profiles", "tdnorm_bf16_7b_32k.md")


def norm_source_hash() -> str:
    return source_hash(("tdnorm.cu", "common.cuh"))


def cema_source_hash() -> str:
    return source_hash(("cema.cu", "common.cuh"))


def recorded_traffic(w: Workload, path: str = SCA_PROFILE, src_hash=None):
    """DRAM bytes per launch from a committed ncu summary, or None if the
    summary is missing, for another workload, or older than the kernel
    source.  The summary carries `key: value` lines for workload,
    source_hash and dram_bytes_per_launch."""
    if not os.path.exists(path):
        return None
    src_hash = src_hash or sca_source_hash()
    rec = {}
    with open(path) as f:
        for line in f:
            if ":" in line and not line.startswith(("#", "|", " ")):
                k_, v_ = line.split(":", 1)
                rec[k_.strip()] = v_.strip()
    if rec.get("source_hash") != src_hash or rec.get("workload") != w.name:
        return None
    try:
        return int(rec["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


# ------------------------------------------------------------------ arms --

def run_gecko(args, w: Workload, ws: int, rank: int, local: int) -> dict:
    from long_context_sequence_sca_b200 import lib as L
    L.load()
    x = make_inputs(w, device="cuda", seed_offset=1000 * rank)
    o_sca = torch.empty_like(x["q"])
    o_mem = torch.empty_like(x["q"])
    stream = torch.cuda.current_stream()

    def step():
        L.sca_awm_forward(x["q"], x["k"], x["v"], x["qm"], x["km"], w.c, o_sca, o_mem, stream)

    # The timed steps run without per-stage events; a separate pass with
    # stage timing on gives the per-stage times and the SCA launch time for
    # the roofline.
    L.timing_enable(False)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if L.device_status() != 0:
        raise RuntimeError("device status reported a timed-out wait during warm-up")

    sampler = ClockSampler(local)
    # inputs that fit in L2 would be served from it on the next step: write a
    # buffer of twice the L2 size between timed steps and time each step alone
    in_bytes = sum(x[n].numel() * x[n].element_size() for n in ("q", "k", "v", "qm", "km"))
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device="cuda") if in_bytes <= L2_BYTES else None

    def timed():
        barrier(ws)
        torch.cuda.synchronize()
        sampler.start()
        if flush is None:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(args.steps):
                step()
            e1.record(stream)
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1) / args.steps
        else:
            evs = []
            for _ in range(args.steps):
                flush.fill_(1.0)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                step()
                e1.record(stream)
                evs.append((e0, e1))
            torch.cuda.synchronize()
            ms = sum(a.elapsed_time(b) for a, b in evs) / args.steps
        ck = sampler.stop()
        barrier(ws)
        return ms, ck

    ms_local, ck = timed()
    note = None
    if clocks_rejected(ck):
        note = f"re-measured once: first run saw clocks {ck}"
        ms_local, ck = timed()
    # per-stage times: the same steps with stage timing on
    L.timing_enable(True)
    n_stage = max(3, min(args.steps, 10))
    for _ in range(2):
        step()
    torch.cuda.synchronize()
    L.timing_read()
    for _ in range(n_stage):
        if flush is not None:
            flush.fill_(1.0)
        step()
    torch.cuda.synchronize()
    stage_tot, n = L.timing_read()
    L.timing_enable(False)
    stages = {k_: v_ / max(n, 1) for k_, v_ in stage_tot.items()}
    serial_ms = sum(stages.values())
    if L.device_status() != 0:
        raise RuntimeError("device status reported a timed-out wait")
    tokens = w.B * w.T
    agg = aggregate(ms_local, tokens, ws)
    fl = flops(w)
    pk, pk_kind = peaks()

    # dominant kernel: the SCA launch (one per step), timed on its stream
    sca_ms = max_over_ranks(stages["sca"], ws)
    achieved = fl["sca"] / (sca_ms / 1e3) / 1e12
    sb = stage_bytes(w)
    stage_hbm = {}
    for k_, b_ in sb.items():
        ms_ = max_over_ranks(stages[k_], ws)
        gbs = b_ / (ms_ / 1e3) / 1e9 if ms_ > 0 else 0.0
        stage_hbm[k_] = {"algorithmic_bytes": b_, "ms": round(ms_, 4), "achieved_gbs": round(gbs, 1),
                         "frac": round(gbs / pk["hbm_gbs"], 4)}
    if hbm_bound(w, pk):
        # below the ridge the kernels are bounded by HBM: the dominant one is
        # the stage with the longest time
        top = max(sb, key=lambda k_: stage_hbm[k_]["ms"])
        roofline = {"bound": "hbm", "kernel": top, "achieved": stage_hbm[top]["achieved_gbs"],
                    "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": stage_hbm[top]["frac"],
                    "peak_kind": f"{pk_kind} HBM copy",
                    "traffic": recorded_traffic(w) if top == "sca" else None,
                    "launch_ms": stage_hbm[top]["ms"], "algorithmic_bytes_per_launch": sb[top]}
    else:
        roofline = {"bound": "tensor", "kernel": "sca_tc_kernel", "achieved": round(achieved, 2),
                    "peak": pk["bf16_tflops"], "unit": "TFLOP/s", "frac": round(achieved / pk["bf16_tflops"], 4),
                    "peak_kind": f"{pk_kind} bf16 dense (burst)",
                    "frac_of_sustained": round(achieved / pk["bf16_tflops_sustained"], 4),
                    "traffic": recorded_traffic(w), "launch_ms": round(sca_ms, 4),
                    "algorithmic_flop_per_launch": fl["sca"]}

    out = {
        "metric": METRIC, "value": round(agg["value"], 1), "unit": "tokens/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(agg["ms_per_step"], 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic (seeded Z'-affine generator; no dataset)",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "T": w.T, "d": w.d, "c": w.c,
                   "tokens_per_step_per_gpu": tokens,
                   "l2": (f"inputs larger than L2 ({in_bytes / 1e9:.2f} GB), no flush" if flush is None else
                          f"inputs {in_bytes / 1e6:.1f} MB fit in L2: {2 * L2_BYTES / 1e6:.0f} MB written between "
                          f"timed steps, each step timed alone"),
                   "parallelism": f"replicas x{ws} (heads/batches independent)"},
        "tflops": round(ws * fl["total"] / (agg["ms_per_step"] / 1e3) / 1e12, 2),
        "pct_bf16_peak": round(100 * fl["total"] / (agg["ms_per_step"] / 1e3) / 1e12 / pk["bf16_tflops"], 2),
        "stage_ms": {k_: round(v_, 4) for k_, v_ in stages.items()},
        "stage_note": (f"stages timed in a separate pass of {n_stage} steps with CUDA events between the stages "
                       f"(sum {serial_ms:.4f} ms)" +
                       ("; the chunk kernel computes the K_m statistics and awm_chunk includes the prefix over "
                        "chunks" if fused_stats(w) else "")),
        "stage_hbm": stage_hbm,
        "roofline": roofline,
        "other_bounds": secondary_rooflines(w, agg["ms_per_step"], sca_ms, ck.get("sm_mhz"), pk["hbm_gbs"]),
        "clocks": ck,
        "gpu_launches": forward_launches(w) * args.steps,
    }
    if note:
        out["note"] = note
    if not args.no_e2e:
        out["e2e"] = run_e2e(args, w, x, ws, stream, L)
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(w)
    return out


def run_e2e(args, w, x, ws, stream, L) -> dict:
    """Same metric through the public API with host buffers: every step copies
    its five inputs from pinned host memory and reads both outputs back.
    Steps are pipelined the way a caller streaming batches would run them:
    two device buffer sets, uploads on one stream, the forward on the
    compute stream and downloads on a third, ordered by events, so step
    k + 1's uploads and step k - 1's downloads overlap step k's compute.  The
    timed region runs from the first upload to the last download."""
    names = ("q", "k", "v", "qm", "km")
    host_in = {n: x[n].cpu().pin_memory() for n in names}
    host_out = [[torch.empty(x["q"].shape, dtype=x["q"].dtype).pin_memory() for _ in range(2)] for _ in range(2)]
    dev_in = [{n: torch.empty_like(x[n]) for n in names} for _ in range(2)]
    dev_out = [[torch.empty_like(x["q"]) for _ in range(2)] for _ in range(2)]
    s_up, s_down = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()
    in_ready, computed, out_read = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    steps = max(1, min(args.steps, 10))

    def run(n_steps):
        for k in range(n_steps):
            i = k % 2
            if k >= 2:
                s_up.wait_event(computed[i])         # the forward of step k - 2 has read this set
            with torch.cuda.stream(s_up):
                for n in names:
                    dev_in[i][n].copy_(host_in[n], non_blocking=True)
                in_ready[i].record(s_up)
            stream.wait_event(in_ready[i])
            if k >= 2:
                stream.wait_event(out_read[i])       # step k - 2's outputs have been read back
            L.sca_awm_forward(*(dev_in[i][n] for n in names), w.c, dev_out[i][0], dev_out[i][1], stream)
            computed[i].record(stream)
            s_down.wait_event(computed[i])
            with torch.cuda.stream(s_down):
                host_out[i][0].copy_(dev_out[i][0], non_blocking=True)
                host_out[i][1].copy_(dev_out[i][1], non_blocking=True)
                out_read[i].record(s_down)

    run(2)
    torch.cuda.synchronize()
    barrier(ws)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_up)
    run(steps)
    e1.record(s_down)
    torch.cuda.synchronize()
    barrier(ws)
    L.timing_read()
    agg = aggregate(e0.elapsed_time(e1) / steps, w.B * w.T, ws)
    nb = x["q"].numel() * x["q"].element_size()
    return {"value": round(agg["value"], 1), "unit": "tokens/s", "h2d_bytes_per_step": 5 * nb,
            "d2h_bytes_per_step": 2 * nb, "steps": steps, "ms_per_step": round(agg["ms_per_step"], 3),
            "pipelining": "uploads, forward and downloads of consecutive steps overlap (2 buffer sets, 3 streams)"}


def cpu_baseline(w: Workload) -> dict:
    n_chunks = 3 if w.S >= 3 else w.S
    tok_s, secs, tok = time_oracle(w, n_chunks, reps=10)
    return {"value": round(tok_s, 2), "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"fp64 oracle forward on the first {n_chunks} chunks of 10 heads "
                      f"({tok} tokens, c={w.c}, d={w.d}) in {secs:.1f} s"}


def run_reference(args, w: Workload) -> dict:
    """The CPU oracle as the reference arm: every step is one bounded sample
    (the first chunks of one head), timed with perf_counter."""
    n_chunks = 2 if w.S >= 2 else 1
    for i in range(args.warmup):
        time_oracle(w, n_chunks, head=i)
    tot_s, tot_tok = 0.0, 0
    for i in range(args.steps):
        _, s, t = time_oracle(w, n_chunks, head=100 + i)
        tot_s += s
        tot_tok += t
    val = tot_tok / tot_s
    sample = (f"per step: fp64 oracle forward on the first {n_chunks} chunks of one head "
              f"({n_chunks * w.c} tokens, c={w.c}, d={w.d})")
    return {
        "metric": METRIC, "value": round(val, 2), "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(1e3 * tot_s / args.steps, 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded generator)",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "T": w.T, "d": w.d, "c": w.c},
        "impl": "reference", "host": "CPU oracle on the host's cores (no GPU work)",
        "cpu_baseline": {"value": round(val, 2), "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(val, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ------------------------------------------------------------------ CEMA --

CEMA_METRIC = "tokens/s CEMA fwd (bf16, D=4096, h=16, 32K tokens)"
CEMA_FLOP_PER_ELEMENT = 12 * 16   # per hidden: complex q*h (6) + alpha beta x (1) + add (1) + Re(eta h) and sum (4)
SM_COUNT, FP32_LANES = 148, 128


def cema_oracle_sample(w: CemaWorkload, x, n_feat: int):
    """Time the fp64 CEMA oracle on the first n_feat features of every token."""
    from oracle import cema_oracle as C
    f = slice(0, n_feat)
    xs = x["x"][:, :, f].double().cpu().numpy()
    prm = {k: x[k][f].double().cpu().numpy() for k in ("alpha", "delta", "theta", "beta")}
    e = x["eta"][f].double().cpu().numpy()
    t0 = time.perf_counter()
    C.cema_forward(xs, prm["alpha"], prm["delta"], prm["theta"], prm["beta"], e[..., 0] + 1j * e[..., 1])
    secs = time.perf_counter() - t0
    return w.B * w.L * n_feat / w.D / secs, secs


def run_cema(args, ws: int, rank: int, local: int) -> dict:
    from long_context_sequence_sca_b200 import lib as L
    L.load()
    w = CEMA_WORKLOADS["cema_bf16_7b_32k"]
    x = make_cema_inputs(w, device="cuda", seed_offset=1000 * rank)
    y = torch.empty_like(x["x"])
    stream = torch.cuda.current_stream()
    prm = (x["alpha"], x["delta"], x["theta"], x["beta"], x["eta"])

    def step(xin, yout):
        L.cema_forward(xin, *prm, reset=x["reset"], y=yout, stream=stream)

    for _ in range(args.warmup):
        step(x["x"], y)
    torch.cuda.synchronize()
    sampler = ClockSampler(local)

    def timed():
        barrier(ws)
        torch.cuda.synchronize()
        sampler.start()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            step(x["x"], y)
        e1.record(stream)
        torch.cuda.synchronize()
        ck = sampler.stop()
        barrier(ws)
        return e0.elapsed_time(e1) / args.steps, ck

    ms_local, ck = timed()
    note = None
    if clocks_rejected(ck):
        note = f"re-measured once: first run saw clocks {ck}"
        ms_local, ck = timed()
    tokens = w.B * w.L
    agg = aggregate(ms_local, tokens, ws)
    op_ms = max_over_ranks(ms_local, ws)
    flop = CEMA_FLOP_PER_ELEMENT * w.B * w.L * w.D
    mhz = ck.get("sm_mhz") or ck.get("sm_max_mhz") or 1965
    peak = SM_COUNT * FP32_LANES * 2 * mhz * 1e6 / 1e12
    achieved = flop / (op_ms / 1e3) / 1e12
    nb = x["x"].numel() * x["x"].element_size()
    out = {
        "metric": CEMA_METRIC, "value": round(agg["value"], 1), "unit": "tokens/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(agg["ms_per_step"], 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded generator; no dataset)",
        "config": {"workload": w.name, "B": w.B, "L": w.L, "D": w.D, "h": w.h,
                   "l2": f"x larger than L2 ({nb / 1e9:.2f} GB), no flush",
                   "parallelism": f"replicas x{ws}"},
        "roofline": {"bound": "alu", "kernel": "cema_local_tma_kernel + cema_carry_kernel + cema_out_tma_kernel (one op)",
                     "achieved": round(achieved, 2), "peak": round(peak, 1), "unit": "TFLOP/s",
                     "frac": round(achieved / peak, 4),
                     "peak_kind": f"derived: {SM_COUNT} SMs x {FP32_LANES} FP32 FMA/clk x 2 flop x {mhz} MHz",
                     "traffic": recorded_traffic(w, CEMA_PROFILE, cema_source_hash()), "launch_ms": round(op_ms, 4),
                     "algorithmic_flop_per_launch": flop},
        "clocks": ck,
        "gpu_launches": 3 * args.steps,
    }
    if note:
        out["note"] = note
    if not args.no_e2e:
        hx = x["x"].cpu().pin_memory()
        hy = torch.empty_like(hx).pin_memory()
        dx = torch.empty_like(x["x"])
        steps = max(1, min(args.steps, 10))

        def e2e_step():
            dx.copy_(hx, non_blocking=True)
            step(dx, y)
            hy.copy_(y, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        barrier(ws)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(ws)
        ea = aggregate(e0.elapsed_time(e1) / steps, tokens, ws)
        out["e2e"] = {"value": round(ea["value"], 1), "unit": "tokens/s", "h2d_bytes_per_step": nb,
                      "d2h_bytes_per_step": nb, "steps": steps, "ms_per_step": round(ea["ms_per_step"], 3)}
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        n_feat = 1024
        val, secs = cema_oracle_sample(w, x, n_feat)
        out["cpu_baseline"] = {"value": round(val, 2), "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                               "sample": f"fp64 CEMA oracle on the first {n_feat} of {w.D} features of all "
                                         f"{w.L} tokens in {secs:.1f} s (tokens scaled by {n_feat}/{w.D})"}
    return out


# ------------------------------------------------ timestep decay norm --

NORM_METRIC = "tokens/s timestep-decay norm fwd (bf16, D=4096, G=32, 32K tokens)"


def time_steps(args, ws, local, step, stream, drain=None):
    """Warm up, then time args.steps calls of step() between CUDA events on
    `stream` (barriers and synchronisation on both sides), sampling clocks;
    re-measure once if the clocks are rejected.  `drain` (e.g. a read of the
    library's stage log) runs right before the timed region, so what it
    discards is the warm-up.  Returns (ms, clocks, note)."""
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    sampler = ClockSampler(local)

    def timed():
        barrier(ws)
        torch.cuda.synchronize()
        if drain is not None:
            drain()
        sampler.start()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
        ck = sampler.stop()
        barrier(ws)
        return e0.elapsed_time(e1) / args.steps, ck

    ms, ck = timed()
    note = None
    if clocks_rejected(ck):
        note = f"re-measured once: first run saw clocks {ck}"
        ms, ck = timed()
    return ms, ck, note


def run_tdnorm(args, ws: int, rank: int, local: int) -> dict:
    from long_context_sequence_sca_b200 import lib as L
    from oracle import tdnorm_oracle as N
    L.load()
    w = NORM_WORKLOADS["tdnorm_bf16_7b_32k"]
    x = make_norm_inputs(w, device="cuda", seed_offset=1000 * rank)
    y = torch.empty_like(x["x"])
    stream = torch.cuda.current_stream()

    def step(xin=x["x"]):
        L.tdnorm_forward(xin, x["gamma"], x["bias"], w.G, w.beta1, w.beta2, w.eps, y=y, stream=stream)

    ms_local, ck, note = time_steps(args, ws, local, step, stream)
    tokens = w.B * w.L
    agg = aggregate(ms_local, tokens, ws)
    op_ms = max_over_ranks(ms_local, ws)
    nb = x["x"].numel() * x["x"].element_size()
    pk, pk_kind = peaks()
    achieved = 2 * nb / (op_ms / 1e3) / 1e9
    out = {
        "metric": NORM_METRIC, "value": round(agg["value"], 1), "unit": "tokens/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(agg["ms_per_step"], 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded generator; no dataset)",
        "config": {"workload": w.name, "B": w.B, "L": w.L, "D": w.D, "G": w.G, "beta1": w.beta1, "beta2": w.beta2,
                   "l2": f"x larger than L2 ({nb / 1e9:.2f} GB), no flush", "parallelism": f"replicas x{ws}"},
        "roofline": {"bound": "hbm", "kernel": "tdnorm_stats_kernel + tdnorm_scan_kernel + tdnorm_apply_kernel (one op)",
                     "achieved": round(achieved, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                     "frac": round(achieved / pk["hbm_gbs"], 4), "peak_kind": f"{pk_kind} HBM copy",
                     "traffic": recorded_traffic(w, NORM_PROFILE, norm_source_hash()), "launch_ms": round(op_ms, 4),
                     "algorithmic_bytes_per_launch": 2 * nb},
        "clocks": ck,
        "gpu_launches": 3 * args.steps,
    }
    if note:
        out["note"] = note
    if not args.no_e2e:
        hx = x["x"].cpu().pin_memory()
        hy = torch.empty_like(hx).pin_memory()
        dx = torch.empty_like(x["x"])

        def e2e_step():
            dx.copy_(hx, non_blocking=True)
            step(dx)
            hy.copy_(y, non_blocking=True)

        e_args = argparse.Namespace(steps=max(1, min(args.steps, 10)), warmup=3)
        ems, _, _ = time_steps(e_args, ws, local, e2e_step, stream)
        ea = aggregate(ems, tokens, ws)
        out["e2e"] = {"value": round(ea["value"], 1), "unit": "tokens/s", "h2d_bytes_per_step": nb,
                      "d2h_bytes_per_step": nb, "steps": e_args.steps, "ms_per_step": round(ea["ms_per_step"], 3)}
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        groups = 4
        gs = w.D // w.G
        xs = x["x"][:, :, :groups * gs].double().cpu().numpy()
        g = x["gamma"][:groups * gs].double().cpu().numpy()
        b = x["bias"][:groups * gs].double().cpu().numpy()
        t0 = time.perf_counter()
        N.tdnorm_forward(xs, groups, w.beta1, w.beta2, w.eps, g, b)
        secs = time.perf_counter() - t0
        out["cpu_baseline"] = {"value": round(tokens * groups / w.G / secs, 2), "unit": "tokens/s",
                               "cores": blas_threads(), "kind": "oracle",
                               "sample": f"fp64 oracle on the first {groups} of {w.G} groups of all {w.L} tokens "
                                         f"in {secs:.1f} s (tokens scaled by {groups}/{w.G})"}
    return out


BWD_METRIC = "tokens/s fused SCA+AWM backward (bf16,H=32,d=128,c=4096); % bf16 TC peak"
BWD_PROFILE = os.path.join(ROOT, "profiles", "sca_bwd_tc_bf16_h32_c4096.md")
# launches of one backward: AWM rebuild (lse partial, combine, prefix, chunk,
# carry), AWM reverse pass (E, carry, dl, chunk, readout), SCA delta, SCA
# dK/dV, SCA dQ
BWD_LAUNCHES = 13


def bwd_source_hash() -> str:
    return source_hash(("sca_bwd_tc.cu", "common.cuh"))


def run_backward(args, ws: int, rank: int, local: int) -> dict:
    """One step = one gecko_sca_awm_backward on the bench workload (the
    forward's outputs and row statistics prepared once, outside the timed
    region; output gradients seeded N(0, 1))."""
    from long_context_sequence_sca_b200 import lib as L
    L.load()
    w = WORKLOADS[DEFAULT_WORKLOAD]
    x = make_inputs(w, device="cuda", seed_offset=1000 * rank)
    names = ("q", "k", "v", "qm", "km")
    g = torch.Generator(device="cuda").manual_seed(77 + rank)
    dos = torch.randn(x["q"].shape, generator=g, device="cuda").to(x["q"].dtype)
    dom = torch.randn(x["q"].shape, generator=g, device="cuda").to(x["q"].dtype)
    stream = torch.cuda.current_stream()
    out_sca, _, lse, lo = L.sca_awm_forward_train(*(x[n] for n in names), w.c, stream=stream)
    grads = [None]

    def step():
        grads[0] = L.sca_awm_backward(*(x[n] for n in names), out_sca, lse, dos, dom, w.c, out_sca_lo=lo,
                                      stream=stream)

    L.timing_enable(True)
    ms_local, ck, note = time_steps(args, ws, local, step, stream, drain=L.timing_read_backward)
    stage_tot, n_calls = L.timing_read_backward()
    L.timing_enable(False)
    stage_ms = {k: v / max(n_calls, 1) for k, v in stage_tot.items()}
    tokens = w.B * w.T
    agg = aggregate(ms_local, tokens, ws)
    f = flops(w)
    kv_ms = max_over_ranks(stage_ms["sca_dkdv"], ws)
    pk, pk_kind = peaks()
    f_kv = 2 * f["sca"]            # S^T, dP^T, dV and dK: four products of the SCA pair count
    f_bwd = 5 * f["sca"] // 2      # the minimal SCA backward: recomputed S, dP, dV, dK, dQ
    achieved = f_kv / (kv_ms / 1e3) / 1e12
    out = {
        "metric": BWD_METRIC, "value": round(agg["value"], 1), "unit": "tokens/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(agg["ms_per_step"], 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded Z'-affine generator, output gradients N(0,1); no dataset)",
        "config": {"workload": w.name + "_backward", "B": w.B, "H": w.H, "T": w.T, "d": w.d, "c": w.c,
                   "tokens_per_step_per_gpu": tokens,
                   "l2": "inputs larger than L2 (2.7 GB incl. output gradients), no flush",
                   "parallelism": f"replicas x{ws} (heads/batches independent)"},
        "tflops_sca_algorithmic": round(f_bwd / (agg["ms_per_step"] / 1e3) / 1e12, 2),
        "stage_ms": {k: round(v, 4) for k, v in stage_ms.items()},
        "roofline": {"bound": "tensor", "kernel": "sca_bwd_tc_kernel<128, false> (dK/dV)",
                     "achieved": round(achieved, 2), "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": round(achieved / pk["bf16_tflops"], 4),
                     "peak_kind": f"{pk_kind} bf16 dense (burst)",
                     "frac_of_sustained": round(achieved / pk.get("bf16_tflops_sustained", pk["bf16_tflops"]), 4),
                     "traffic": recorded_traffic(WORKLOADS[DEFAULT_WORKLOAD], BWD_PROFILE, bwd_source_hash()),
                     "launch_ms": round(kv_ms, 4), "algorithmic_flop_per_launch": f_kv},
        "clocks": ck,
        "gpu_launches": BWD_LAUNCHES * args.steps,
    }
    if note:
        out["note"] = note
    if not args.no_e2e:
        dev_in = [x[n] for n in names] + [out_sca, lse, dos, dom, lo]
        host_in = [t.cpu().pin_memory() for t in dev_in]
        host_out = [torch.empty_like(x["q"], device="cpu").pin_memory() for _ in range(5)]
        staged = [torch.empty_like(t) for t in dev_in]

        def e2e_step():
            for d_, h_ in zip(staged, host_in):
                d_.copy_(h_, non_blocking=True)
            gr = L.sca_awm_backward(*staged[:5], staged[5], staged[6], staged[7], staged[8], w.c,
                                    out_sca_lo=staged[9], stream=stream)
            for h_, d_ in zip(host_out, gr):
                h_.copy_(d_, non_blocking=True)

        e_args = argparse.Namespace(steps=max(1, min(args.steps, 5)), warmup=3)
        ems, _, _ = time_steps(e_args, ws, local, e2e_step, stream)
        ea = aggregate(ems, tokens, ws)
        out["e2e"] = {"value": round(ea["value"], 1), "unit": "tokens/s",
                      "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in dev_in),
                      "d2h_bytes_per_step": sum(t.numel() * t.element_size() for t in host_out),
                      "steps": e_args.steps, "ms_per_step": round(ea["ms_per_step"], 3),
                      "pipelining": "none (copy in, backward, copy out in one stream)"}
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        from oracle import gecko_backward_oracle as GB
        n_ch = 2
        rows = slice(0, n_ch * w.c)
        xs = [x[n][0, 0, rows].double().cpu().numpy() for n in names]
        do_s = dos[0, 0, rows].double().cpu().numpy()
        do_m = dom[0, 0, rows].double().cpu().numpy()
        t0 = time.perf_counter()
        GB.sca_head_backward(xs[0], xs[1], xs[2], w.c, do_s)
        GB.awm_head_backward(xs[3], xs[4], xs[2], w.c, do_m)
        secs = time.perf_counter() - t0
        out["cpu_baseline"] = {"value": round(n_ch * w.c / w.H / secs, 2), "unit": "tokens/s", "cores": blas_threads(),
                               "kind": "oracle",
                               "sample": f"fp64 gradient oracle on the first {n_ch} chunks of 1 of {w.H} heads "
                                         f"({n_ch * w.c} rows, c={w.c}, d={w.d}) in {secs:.1f} s; tokens counted "
                                         f"as rows / H (a token carries all H heads)"}
    return out


CP_METRIC = "tokens/s SCA+AWM fwd, sequence split into context-parallel segments (bf16,H=32,d=128,c=4096)"


def run_cp(args, ws: int, rank: int, local: int) -> dict:
    """Context parallelism on one GPU: the bench sequence is split into
    --segments segments and every rank's phases (log-sums, cp log z, segment
    maps, composed states, continued forwards) run in this process, so the
    line measures the work context parallelism adds per rank.  The
    whole-sequence forward is timed in the same run for comparison."""
    from long_context_sequence_sca_b200 import cp
    from long_context_sequence_sca_b200 import lib as L
    L.load()
    w = WORKLOADS[DEFAULT_WORKLOAD]
    P = args.segments
    if w.T % (P * w.c) != 0:
        raise SystemExit(f"T={w.T} does not split into {P} segments of whole chunks (c={w.c})")
    x = make_inputs(w, device="cuda", seed_offset=1000 * rank)
    names = ("q", "k", "v", "qm", "km")
    Tr = w.T // P
    segs = [{n: x[n][:, :, r * Tr:(r + 1) * Tr].contiguous() for n in names} for r in range(P)]
    stream = torch.cuda.current_stream()

    def step():
        cp.cp_forward_emulated(segs, w.c)

    L.timing_enable(True)
    ms_local, ck, note = time_steps(args, ws, local, step, stream, drain=L.timing_read)
    stage_tot, n_calls = L.timing_read()
    L.timing_enable(False)
    # the library logs every segment forward of the timed steps: P per step
    sca_ms = stage_tot["sca"] / max(n_calls / P, 1)

    # what one rank does on its own GPU, phase by phase (no exchange time)
    def timed(fn, reps=5):
        fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    seg = segs[min(1, P - 1)]
    lz = L.awm_segment_logsum(seg["km"], w.c)
    lsum_all = torch.stack([L.awm_segment_logsum(sg["km"], w.c) for sg in segs])
    maps_all = torch.stack([L.awm_segment_maps(sg["km"], sg["v"], L.awm_cp_logz(lsum_all, r), w.c)
                            for r, sg in enumerate(segs)])
    state = L.awm_cp_state(lsum_all, maps_all, 1)
    halo = cp.halo_of(segs[0], w.c)
    k1 = torch.cat([halo[0], seg["k"]], dim=2).contiguous()
    v1 = torch.cat([halo[1], seg["v"]], dim=2).contiguous()
    rank_phases = {
        "segment_logsum": timed(lambda: L.awm_segment_logsum(seg["km"], w.c)),
        "cp_logz": timed(lambda: L.awm_cp_logz(lsum_all, 1)),
        "segment_maps": timed(lambda: L.awm_segment_maps(seg["km"], seg["v"], lz, w.c)),
        "cp_state": timed(lambda: L.awm_cp_state(lsum_all, maps_all, 1)),
        "continued_forward": timed(lambda: L.sca_awm_forward_segment(seg["q"], k1, v1, seg["qm"], seg["km"], w.c,
                                                                     state_in=state)),
    }

    def whole():
        L.sca_awm_forward(*(x[n] for n in names), w.c)

    whole_ms, _, _ = time_steps(args, ws, local, whole, stream)
    tokens = w.B * w.T
    agg = aggregate(ms_local, tokens, ws)
    f = flops(w)
    pk, pk_kind = peaks()
    achieved = f["sca"] / (max_over_ranks(sca_ms, ws) / 1e3) / 1e12
    out = {
        "metric": CP_METRIC, "value": round(agg["value"], 1), "unit": "tokens/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(agg["ms_per_step"], 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded Z'-affine generator; no dataset)",
        "config": {"workload": f"{w.name}_cp{P}", "B": w.B, "H": w.H, "T": w.T, "d": w.d, "c": w.c,
                   "segments": P, "ranks": f"{P} emulated on one GPU (exchanges are tensor indexing)",
                   "l2": "inputs larger than L2 (1.34 GB), no flush",
                   "parallelism": f"replicas x{ws}"},
        "whole_sequence_ms": round(whole_ms, 4),
        "cp_overhead_ms": round(ms_local - whole_ms, 4),
        "one_rank_phase_ms": {k: round(v, 4) for k, v in rank_phases.items()},
        "roofline": {"bound": "tensor", "kernel": "sca_tc_kernel (the P segment launches of a step)",
                     "achieved": round(achieved, 2), "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": round(achieved / pk["bf16_tflops"], 4), "peak_kind": f"{pk_kind} bf16 dense (burst)",
                     "traffic": None, "launch_ms": round(sca_ms / P, 4),
                     "algorithmic_flop_per_launch": f["sca"] // P},
        "clocks": ck,
        # per segment: log-sum 3, maps 7, cp log z 1, forward 7; cp state 2 for every segment but the first
        "gpu_launches": (18 * P + 2 * (P - 1)) * args.steps,
    }
    if note:
        out["note"] = note
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        # the segmented outputs equal the whole-sequence forward, so the
        # oracle's forward on a bounded sample is the CPU baseline
        out["cpu_baseline"] = cpu_baseline(w)
    return out


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("gecko", "reference"), default="gecko")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--op", choices=("sca_awm", "backward", "cp", "cema", "tdnorm"), default="sca_awm",
                    help="sca_awm: the fused SCA + AWM forward (default); backward: its gradients; "
                         "cp: the forward as context-parallel segments (emulated ranks on one GPU); "
                         "cema: the CEMA recurrence; tdnorm: timestep decay normalisation")
    ap.add_argument("--segments", type=int, default=4, help="segments of --op cp")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    w = WORKLOADS[args.workload]

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args, w)), flush=True)
        return 0

    ws, rank, local = dist_setup()
    if ws != args.gpus and rank == 0:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {ws}", file=sys.stderr)
    try:
        runner = {"cema": lambda: run_cema(args, ws, rank, local), "tdnorm": lambda: run_tdnorm(args, ws, rank, local),
                  "backward": lambda: run_backward(args, ws, rank, local),
                  "cp": lambda: run_cp(args, ws, rank, local)}
        out = runner[args.op]() if args.op in runner else run_gecko(args, w, ws, rank, local)
        if rank == 0:
            print(json.dumps(out), flush=True)
    finally:
        if ws > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
