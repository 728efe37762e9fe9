#!/usr/bin/env python3
"""Benchmark of the sparse chunked-prefill hot path of one attention layer.

One step = the whole path for one layer over the synthetic workload: for every
32K-query chunk, estimation (last 64 queries against the growing KV), top-k
vertical/slash selection with refinement by attention recall where the workload
has a threshold, and the sparse attention of the chunk's rows (with DCA
positions where the workload uses DCA). Inputs are resident in HBM when the
timed region starts; L2 is flushed between steps. The `e2e` figure repeats the
step through the same public API from pinned host buffers, host<->device copies
of the inputs and of the output inside the timed region.

Multi-GPU (torchrun): every rank prefills its own independent layer (seed
offset by rank), no collective on the data path; value = all tokens / max rank
time ("weak" scaling).

--impl reference: the CPU oracle (oracle/) timed on a bounded sample of the same
workload, extrapolated to the layer.
"""
from __future__ import annotations

import argparse
import faulthandler
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time
from dataclasses import replace

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from workloads import WORKLOADS, generate_head, structure  # noqa: E402

METRIC = "sparse-prefill tokens/s per layer; executed TFLOP/s and % of B200 BF16 peak"
FLOP_PER_TILE = 4 * 128 * 128 * 128  # QK^T and PV of one executed 128-query x 128-key tile
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# NVIDIA's published dense BF16 tensor figure for one B200 (the 4.5 PFLOP/s of the
# datasheet is with 2:4 sparsity); reported beside the measured peaks, never as the
# roofline denominator.
DATASHEET_BF16_TFLOPS = 2250.0
# DRAM bytes (read + write) of one attention-kernel launch, from one ncu capture per
# workload (the launch-list summaries under profiles/), valid only for the kernel sources they were
# taken on: a sha256 prefix over attn.cu, sm100.cuh and internal.cuh. A changed
# kernel reports null until it is captured again.
ATTN_TRAFFIC = {
    # one step's 32 launches averaged (the 1-pass launch list of the whole step)
    "cfg5_14b_n1m_dca256k_refine": ("a9347671274814d5", 23130152608),
    "cfg9_14b_n1m_dca256k_refine_structured": ("a9347671274814d5", 13509399688),
}


def attn_traffic(workload: str):
    import hashlib

    rec = ATTN_TRAFFIC.get(workload)
    if rec is None:
        return None
    h = hashlib.sha256()
    for f in ("attn.cu", "sm100.cuh", "internal.cuh"):
        with open(os.path.join(ROOT, "sparse_attention_estimate_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return rec[1] if h.hexdigest().startswith(rec[0]) else None


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def parse():
    p = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=5)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--config", type=int, default=5, choices=sorted(WORKLOADS),
                   help="workload (default 5: 40/8 heads, 1M tokens in 32 chunks, DCA 262144, refinement 0.9)")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--max-iters", type=int, default=19)
    p.add_argument("--seq-len", type=int, default=None,
                   help="prefill only the first SEQ_LEN tokens of the workload (profiling cases)")
    p.add_argument("--calibrate", action="store_true",
                   help="offline refinement: per-head budgets calibrated once (outside the timed region) on "
                        "another sequence of the same workload (seed + 7919); the timed steps select with them")
    p.add_argument("--refine-positions", choices=["continuous", "dca"], default="continuous",
                   help="dca: refinement's recall from the estimation rows' attention at DCA positions "
                        "(DCA workloads)")
    p.add_argument("--shard", choices=["layers", "heads"], default="layers",
                   help="N > 1: layers = an independent layer per rank (weak scaling); heads = one layer's "
                        "KV groups split over the ranks (strong scaling)")
    p.add_argument("--mask", choices=["selected", "full"], default="selected",
                   help="full: the dense causal baseline through the same attention kernel (every key "
                        "of [0, e) selected; no estimation or selection)")
    return p.parse_args()


def select_workload(args):
    w = WORKLOADS[args.config]
    if args.seq_len is not None and args.seq_len < w.seq_len:
        w = replace(w, seq_len=args.seq_len, name=f"{w.name}_first{args.seq_len}")
    return w


def rank_workload(w, rank: int):
    """Rank r > 0 prefills an independent layer: same shapes, seed offset by 1000 r."""
    return w if rank == 0 else replace(w, seed=w.seed + 1000 * rank)


def shard_heads(w, rank: int, world: int):
    """KV-group sharding of one layer (no data crosses KV groups on the path): rank r
    takes KV heads [r G, (r + 1) G) with G = hkv / world, and their query heads.
    Returns the rank's workload (same seed, local head counts) and the global index
    of its first query head and first KV head; the per-head generators make the
    rank's heads bit-identical to the same heads of the whole layer."""
    if w.hkv % world:
        raise ValueError(f"{w.hkv} KV heads do not split over {world} ranks")
    gk = w.hkv // world
    local = replace(w, hq=w.group * gk, hkv=gk, name=f"{w.name}_kvshard{rank}of{world}")
    return local, rank * w.group * gk, rank * gk


def max_over_ranks(x: float, world: int, device) -> float:
    """Largest value over the ranks (the job's time is its slowest rank's)."""
    if world == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(seq_len: int, steps: int, world: int, total_ms: float) -> float:
    """Whole-job tokens/s: every rank prefilled `steps` layers of seq_len tokens."""
    return seq_len * steps * world / (total_ms / 1e3)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------------------- clocks
_NVML_LOOP = r"""
import sys, time
import pynvml as nv
nv.nvmlInit()
bus, idx = sys.argv[1], int(sys.argv[2])
h = nv.nvmlDeviceGetHandleByPciBusId(bus) if bus else nv.nvmlDeviceGetHandleByIndex(idx)
bits = (nv.nvmlClocksEventReasonHwSlowdown, nv.nvmlClocksEventReasonHwThermalSlowdown,
        nv.nvmlClocksEventReasonSwThermalSlowdown, nv.nvmlClocksEventReasonSwPowerCap)
mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
print("ready", flush=True)
while True:
    sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
    r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
    pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
    print(", ".join([str(sm), str(mx), f"{pw:.1f}"] + ["Active" if r & b else "Not Active" for b in bits]), flush=True)
    time.sleep(0.005)
"""


class ClockSampler:
    """Samples the SM clock and the clock-event (throttle) reasons during the timed
    region, in a child process (read-only queries): NVML every 5 ms when its Python
    bindings load, else nvidia-smi every 200 ms."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None
        self.lines = []
        self.source = None

    def __enter__(self):
        try:  # the device's PCI address, domain:bus:device.function, as NVML and nvidia-smi take it
            pr = torch.cuda.get_device_properties(self.idx)
            bus = f"{int(pr.pci_domain_id):08x}:{int(pr.pci_bus_id):02x}:{int(pr.pci_device_id):02x}.0"
        except Exception:
            bus = ""
        try:  # NVML loop in a child process; it prints "ready" once it samples
            p = subprocess.Popen([sys.executable, "-c", _NVML_LOOP, bus, str(self.idx)],
                                 stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            import select

            ready, _, _ = select.select([p.stdout], [], [], 15.0)
            first = p.stdout.readline().strip() if ready else ""
            if first == "ready":
                self.proc, self.source = p, "nvml, 5 ms"
            else:
                p.kill()
        except Exception:
            self.proc = None
        if self.proc is None:
            sel = ["--id=" + bus] if bus else ["-i", str(self.idx)]
            try:
                self.proc = subprocess.Popen(["nvidia-smi", *sel, "--query-gpu=" + self.FIELDS,
                                              "--format=csv,noheader,nounits", "-lms", "200"],
                                             stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
                self.source = "nvidia-smi, 200 ms"
            except Exception:
                self.proc = None
        if self.proc is not None:
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm), "source": self.source}


# ----------------------------------------------------------------------------- the GPU path
class Layer:
    """One layer's inputs on the device, the library context and per-chunk buffers."""

    def __init__(self, w, device, max_iters, full_mask=False, q0=0, k0=0, refine_dca=False):
        import sparse_attention_estimate_b200 as vsb

        self.vsb = vsb
        self.w = w
        self.full_mask = full_mask
        self.calibrated = False
        self.dev = device
        self.max_iters = max_iters
        st = structure(w)
        t0 = time.time()
        self.q = torch.empty(w.hq, w.seq_len, 128, dtype=torch.bfloat16, device=device)
        self.k = torch.empty(w.hkv, w.seq_len, 128, dtype=torch.bfloat16, device=device)
        self.v = torch.empty(w.hkv, w.seq_len, 128, dtype=torch.bfloat16, device=device)
        self.h0 = {"q": q0, "k": k0, "v": k0}  # global index of the first local head
        for name, t, nh in (("q", self.q, w.hq), ("k", self.k, w.hkv), ("v", self.v, w.hkv)):
            for h in range(nh):
                t[h].copy_(generate_head(w, name, self.h0[name] + h, st=st))
        log(f"[bench] generated {w.name} in {time.time() - t0:.1f}s")
        self.out = torch.empty_like(self.q)
        self.lse = torch.empty(w.hq, w.seq_len, dtype=torch.float32, device=device)
        C = w.dca_chunk
        cfg = vsb.Config(hq=w.hq, hkv=w.hkv, rope_base=w.rope_base, last_q=w.last_q, dca_chunk=C,
                         dca_window=w.dca_window if C else None, softmax_scale=w.softmax_scale,
                         refine_dca_positions=refine_dca)
        self.ctx = vsb.Context(cfg, max_seq=w.seq_len, max_chunk=min(w.chunk, w.seq_len), device=device)
        e_max = w.seq_len
        self.vert = torch.empty(w.hq, e_max, dtype=torch.float32, device=device)
        self.slash = torch.empty_like(self.vert)
        self.lse_est = torch.empty(w.hq, 64, dtype=torch.float32, device=device)
        self.base_v = torch.full((w.hq,), w.kv_budget, dtype=torch.int32, device=device)
        self.base_s = torch.full((w.hq,), w.ks_budget, dtype=torch.int32, device=device)
        self.kv = torch.empty_like(self.base_v)
        self.ks = torch.empty_like(self.base_s)
        self.recall = torch.empty(w.hq, dtype=torch.float32, device=device)
        self.sets = (torch.empty(w.hq, e_max, dtype=torch.int32, device=device),
                     torch.empty(w.hq, dtype=torch.int32, device=device),
                     torch.empty(w.hq, e_max, dtype=torch.int32, device=device),
                     torch.empty(w.hq, dtype=torch.int32, device=device))
        self.chunks = [w.chunk_bounds(c) for c in range(w.n_chunks)]
        self.cal_summary = None
        if full_mask:  # every column of [0, e) is a selected vertical: the dense causal mask
            self.sets[0].copy_(torch.arange(e_max, dtype=torch.int32, device=device).expand(w.hq, e_max))
            self.sets[3].zero_()

    def step(self, attn_events=None, stats=None, q=None, k=None, v=None):
        """One pass of the whole hot path. attn_events: list of (start, stop) per
        chunk, recorded around the attention kernel; stats: list receiving the
        (executed tiles, useful pairs) of each chunk (synchronises)."""
        w, ctx = self.w, self.ctx
        q = self.q if q is None else q
        k = self.k if k is None else k
        v = self.v if v is None else v
        ctx.reset()  # every step rotates its keys again
        for ci, (cs, e) in enumerate(self.chunks):
            vert, slash = self.vert[:, :e], self.slash[:, :e]
            if self.full_mask:
                self.sets[1].fill_(e)
                self._attend(ci, cs, e, q, k, v, attn_events, stats)
                continue
            ctx.estimate(q, cs, k, e, out=(self.vert, self.slash, self.lse_est), full=True)
            self.kv.copy_(self.base_v)
            self.ks.copy_(self.base_s)
            if w.refine_tau is None or self.calibrated:
                ctx.select(self.vert, self.slash, e, self.kv, self.ks, sets=self.sets)
            else:
                ctx.refine(q, cs, k, e, self.vert, self.slash, self.lse_est, w.refine_tau, self.kv, self.ks,
                           max_iters=self.max_iters, sets=self.sets, recall=self.recall, full=True)
            self._attend(ci, cs, e, q, k, v, attn_events, stats)
            del vert, slash

    def calibrate(self):
        """Per-head budgets from another sequence of the same workload (seed + 7919),
        generated into the q / k buffers and regenerated afterwards."""
        w = self.w
        wc = replace(w, seed=w.seed + 7919)
        st = structure(wc)
        for name, t, nh in (("q", self.q, w.hq), ("k", self.k, w.hkv)):
            for h in range(nh):
                t[h].copy_(generate_head(wc, name, self.h0[name] + h, st=st))
        self.ctx.reset()
        log(f"[bench] calibrating on {wc.name} seed {wc.seed}")
        kv, ks = self.vsb.calibrate(self.ctx, self.q, self.k, chunk=w.chunk, kv_budget=w.kv_budget,
                                    ks_budget=w.ks_budget, tau=w.refine_tau, max_iters=self.max_iters)
        self.base_v.copy_(kv)
        self.base_s.copy_(ks)
        st = structure(w)
        for name, t, nh in (("q", self.q, w.hq), ("k", self.k, w.hkv)):
            for h in range(nh):
                t[h].copy_(generate_head(w, name, self.h0[name] + h, st=st))
        self.ctx.reset()
        self.calibrated = True
        kvh, ksh = kv.cpu().tolist(), ks.cpu().tolist()
        self.cal_summary = {"kv": [min(kvh), int(statistics.median(kvh)), max(kvh)],
                            "ks": [min(ksh), int(statistics.median(ksh)), max(ksh)],
                            "of": "min / median / max over heads", "sequence": f"seed {wc.seed}"}

    def _attend(self, ci, cs, e, q, k, v, attn_events, stats):
        ctx = self.ctx
        if attn_events is not None:
            ctx.set_prefill_events(*attn_events[ci])
        ctx.sparse_prefill(q, cs, e, k, v, self.sets, out=self.out, lse=self.lse, full=True)
        if attn_events is not None:
            ctx.set_prefill_events(None, None)
        if stats is not None:
            stats.append(ctx.prefill_stats())


def job_workloads(args, rank: int, world: int):
    """(this rank's workload, the job's workload, layers the job prefills): one layer's
    KV groups over the ranks with --shard heads, else an independent layer per rank."""
    if args.shard == "heads" and world > 1:
        return shard_heads(select_workload(args), rank, world), select_workload(args), 1
    w = rank_workload(select_workload(args), rank)
    return (w, 0, 0), w, world


def workload_config(args, w, wj, world: int, job_layers: int, cal_summary=None) -> dict:
    """The JSON line's `config`: the workload, the same for both arms of the bench."""
    return {
        "workload": wj.name + ("_fullmask" if args.mask == "full" else ""), "seq_len": w.seq_len,
        "hq": wj.hq, "hkv": wj.hkv, "head_dim": 128, "mask": args.mask, "q_scale": w.q_scale,
        "softmax_scale": round(w.softmax_scale, 6),
        "chunk": w.chunk, "n_chunks": w.n_chunks, "dca": [w.dca_chunk, w.dca_window] if w.dca_chunk else None,
        "budgets": [w.kv_budget, w.ks_budget], "refine_tau": w.refine_tau,
        "calibrated_budgets": cal_summary, "refine_positions": args.refine_positions,
        "parallelism": ("single GPU" if world == 1 else f"KV groups of one layer over {world} GPUs"
                        if job_layers == 1 else f"independent layer per GPU x{world}"),
        "l2": "flushed between steps (256 MiB write)",
    }


def flush_l2(buf):
    buf.zero_()


def run_ours(args, rank, world, device):
    import sparse_attention_estimate_b200 as vsb
    from sparse_attention_estimate_b200 import build as vsbuild

    vsbuild.build()
    vsb.load_library()
    (w, q0, k0), wj, job_layers = job_workloads(args, rank, world)
    lay = Layer(w, device, args.max_iters, full_mask=args.mask == "full", q0=q0, k0=k0,
                refine_dca=args.refine_positions == "dca")
    lay.job_layers = job_layers
    if args.calibrate:
        if w.refine_tau is None or args.mask == "full":
            raise SystemExit("--calibrate needs a workload with a refinement threshold and --mask selected")
        lay.calibrate()
    l2 = torch.empty(256 << 20, dtype=torch.uint8, device=device)  # > 126 MB L2
    nchunks = len(lay.chunks)

    def new_events():
        evs = []
        for _ in range(nchunks):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            b.record()
            evs.append((a, b))
        return evs

    for _ in range(args.warmup):
        flush_l2(l2)
        lay.step()
    torch.cuda.synchronize()
    assert lay.ctx.status() == vsb.VS_OK, "device error during warm-up"
    # executed tiles / useful pairs of one step (untimed; reads counters per chunk)
    stats = []
    lay.step(stats=stats)
    executed = sum(s[0] for s in stats)
    useful = sum(s[1] for s in stats)
    # ---------------------------------------------------------------- timed region
    step_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
    attn_ev = [new_events() for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    n0 = vsb.kernel_launches()
    with ClockSampler(device.index or 0) as clk:
        for i in range(args.steps):
            flush_l2(l2)
            step_ev[i][0].record()
            lay.step(attn_events=attn_ev[i])
            step_ev[i][1].record()
        torch.cuda.synchronize()
    launches = vsb.kernel_launches() - n0
    if world > 1:
        torch.distributed.barrier()
    assert lay.ctx.status() == vsb.VS_OK, "device error in the timed region"
    step_ms = [a.elapsed_time(b) for a, b in step_ev]
    attn_ms = [sum(a.elapsed_time(b) for a, b in evs) for evs in attn_ev]
    tot_ms = max_over_ranks(sum(step_ms), world, device)
    ms_per_step = tot_ms / args.steps
    value = job_throughput(w.seq_len, args.steps, lay.job_layers, tot_ms)
    attn_ms_step = sum(attn_ms) / args.steps
    exec_flops = executed * FLOP_PER_TILE
    useful_flops = useful * 4 * 128
    pk, pk_src = peaks()
    long_step = ms_per_step > 1000.0
    peak = pk["bf16_tflops_sustained"] if long_step else pk["bf16_tflops"]
    attn_tflops = exec_flops / (attn_ms_step / 1e3) / 1e12
    res = {
        "metric": METRIC,
        "value": round(value, 1),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 3),
        "higher_is_better": True,
        "scaling": "strong" if lay.job_layers == 1 and world > 1 else "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": ("synthetic (seeded generator: N(0,1) Q/K/V" + (f", Q's N(0,1) part x{w.q_scale:g}" if w.q_scale != 1
                 else "") + ", planted verticals, 64-aligned band)"),
        "config": workload_config(args, w, wj, world, lay.job_layers, lay.cal_summary),
        "executed_tflops": round(exec_flops / (ms_per_step / 1e3) / 1e12, 2),
        "attn_executed_tflops": round(attn_tflops, 2),
        "pct_bf16_peak": round(100 * attn_tflops / peak, 2),
        "pct_bf16_peak_of": f"{pk_src} {'sustained' if long_step else 'burst'} {peak} TFLOP/s",
        "pct_bf16_datasheet_peak": round(100 * attn_tflops / DATASHEET_BF16_TFLOPS, 2),
        "useful_tflops": round(useful_flops / (ms_per_step / 1e3) / 1e12, 2),
        "density_useful_over_executed": round(useful_flops / exec_flops, 4) if exec_flops else None,
        "attn_ms_per_step": round(attn_ms_step, 3),
        "roofline": {
            "bound": "tensor", "kernel": "attn_kernel",
            "achieved": round(attn_tflops, 2), "peak": peak, "unit": "TFLOP/s",
            "frac": round(attn_tflops / peak, 4), "traffic": attn_traffic(w.name),
            "traffic_unit": "DRAM bytes per launch (ncu)",
            "peak_kind": f"{pk_src} {'sustained' if long_step else 'burst'} bf16",
            "flop_per_launch": round(exec_flops / nchunks),
        },
        "gpu_launches": int(launches),
        "clocks": clk.summary(),
    }
    # ---------------------------------------------------------------- end to end (host buffers)
    if not args.no_e2e:
        res["e2e"] = run_e2e(args, lay, l2, world, device, ms_per_step)
    return res, w, lay


def run_e2e(args, lay, l2, world, device, ms_per_step):
    """Same step through the public API from pinned host memory: H2D of q, k, v
    and D2H of the output inside the timed region. With the selected mask the step
    is HostStreamedPrefill (uploads, compute and downloads of work units overlapped
    on three streams): units of (chunk, KV head) for a single-chunk layer, whole
    chunks otherwise (each chunk's attention then fills the GPU in one launch);
    with --mask full, copies then the step. Seconds-long steps time fewer e2e steps
    (about 40 s in all, at least 2); the line gives the count."""
    hq_h = lay.q.cpu().pin_memory()
    hk_h = lay.k.cpu().pin_memory()
    hv_h = lay.v.cpu().pin_memory()
    out_h = torch.empty(lay.out.shape, dtype=lay.out.dtype).pin_memory()
    w = lay.w
    if not lay.full_mask:
        tau = None if (w.refine_tau is None or lay.calibrated) else w.refine_tau
        per_unit = 1 if w.n_chunks == 1 else w.hkv
        sp = lay.vsb.HostStreamedPrefill(lay.ctx.cfg, w.seq_len, w.chunk, lay.base_v, lay.base_s, tau,
                                         max_iters=lay.max_iters, kv_heads_per_unit=per_unit, device=device)
        mode = ("streamed: (chunk, KV head) units" if per_unit == 1 else "streamed: chunk units") + \
            ", uploads and downloads overlapped with compute"

        def e2e_step():
            sp.run(hq_h, hk_h, hv_h, out_h)
    else:
        dq, dk, dv = torch.empty_like(lay.q), torch.empty_like(lay.k), torch.empty_like(lay.v)
        mode = "serial: inputs uploaded, step, output downloaded"

        def e2e_step():
            dq.copy_(hq_h, non_blocking=True)
            dk.copy_(hk_h, non_blocking=True)
            dv.copy_(hv_h, non_blocking=True)
            lay.step(q=dq, k=dk, v=dv)
            out_h.copy_(lay.out, non_blocking=True)

    long_step = ms_per_step > 2000.0
    n_steps = max(2, min(args.steps, int(40000.0 // max(ms_per_step, 1e-3))))
    for _ in range(1 if long_step else 2):
        e2e_step()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_steps)]
    if world > 1:
        torch.distributed.barrier()
    for i in range(n_steps):
        flush_l2(l2)
        evs[i][0].record()
        e2e_step()
        evs[i][1].record()
    torch.cuda.synchronize()
    tot = max_over_ranks(sum(a.elapsed_time(b) for a, b in evs), world, device)
    h2d = (hq_h.numel() + hk_h.numel() + hv_h.numel()) * 2
    d2h = out_h.numel() * 2
    return {"value": round(job_throughput(lay.w.seq_len, n_steps, lay.job_layers, tot), 1), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(tot / n_steps, 3),
            "steps": n_steps, "mode": mode}


# ----------------------------------------------------------------------------- the CPU oracle
def oracle_sample(w, budget_s=15.0, n_rows=64, seed=0):
    """Times the oracle on a bounded sample of workload w and extrapolates to the
    layer. Work units are (head, chunk) pairs: the chunk's estimation, selection
    and refinement for that head, plus the attention of n_rows sampled query rows
    of the chunk. Chunks are taken from a spread over the sequence (first, last and
    up to three between), smallest first, heads in turn; a unit whose predicted
    cost (the per-key rates measured so far times its key count) exceeds the time
    left is skipped, so one sample stays near budget_s even where one unit at the
    longest chunk would take longer. Each unit's cost is taken as linear in its key
    count e (estimation and per-row attention both are), so the measured per-key
    rates extrapolate to every chunk, row and head. Returns (tokens/s, seconds
    spent, description)."""
    import oracle.vs_oracle as vo

    st = structure(w)
    rng = np.random.default_rng(seed)
    dca = (w.dca_chunk, w.dca_window) if w.dca_chunk else None
    scale = w.softmax_scale
    spread = sorted(set(int(round(x)) for x in np.linspace(0, w.n_chunks - 1, min(w.n_chunks, 5))))
    units = [((r * len(spread) + i) % w.hq, c) for r in range(w.hq) for i, c in enumerate(spread)]
    fixed_per_key, row_per_key = [], []  # seconds per key of e: per chunk, and per row and chunk
    cache = _ORACLE_INPUTS.setdefault(w, {})  # generated heads, kept across samples
    spent = 0.0  # oracle time only: generating the inputs is not part of the sample
    wall0 = time.time()
    done, chunks_seen = 0, set()
    for h, c in units:
        left = budget_s - spent
        if done and (left <= 0 or time.time() - wall0 > 4 * budget_s):
            break
        cs, e = w.chunk_bounds(c)
        nrow = min(n_rows, e - cs)
        if done and (np.mean(fixed_per_key) + nrow * np.mean(row_per_key)) * e > left:
            continue  # predicted to overrun the budget
        hk = h // w.group
        if ("k", hk) not in cache:
            cache = {k: v for k, v in cache.items() if k[0] != "k" and k[0] != "v"}
            cache[("k", hk)] = generate_head(w, "k", hk, st=st).float().double().numpy()
            cache[("v", hk)] = generate_head(w, "v", hk, st=st).float().double().numpy()
        if ("q", h) not in cache:
            cache = {k: v for k, v in cache.items() if k[0] != "q"}
            cache[("q", h)] = generate_head(w, "q", h, st=st).float().double().numpy()
        kf, vf, qf = cache[("k", hk)], cache[("v", hk)], cache[("q", h)]
        nr = min(w.last_q, e - cs)
        t0 = time.time()
        _, vert, slash, a = vo.estimate(qf[e - nr : e], kf, e, w.rope_base, scale)
        if w.refine_tau is None:
            V, S = vo.select(vert, slash, w.kv_budget, w.ks_budget)
        else:
            _, _, V, S, _, _ = vo.refine(a, np.arange(e - nr, e), vert, slash, w.kv_budget, w.ks_budget,
                                         w.refine_tau)
        t1 = time.time()
        rows = np.sort(rng.choice(np.arange(cs, e), size=nrow, replace=False))
        inV, inS = vo.membership(e, V), vo.membership(e, S)
        # two-point fit: one row (the call's fixed cost, e.g. rotating the keys) and all rows
        vo.attention_rows(qf[rows[-1:]], rows[-1:], kf, vf, e, inV, inS, w.rope_base, scale, dca)
        t2 = time.time()
        vo.attention_rows(qf[rows], rows, kf, vf, e, inV, inS, w.rope_base, scale, dca)
        t3 = time.time()
        per_row = max(t3 - t2 - (t2 - t1), 0.0) / max(len(rows) - 1, 1)
        fixed = max((t2 - t1) - per_row, 0.0)
        fixed_per_key.append(((t1 - t0) + fixed) / e)
        row_per_key.append(per_row / e)
        spent += t3 - t0
        done += 1
        chunks_seen.add(c)
    fk, rk = float(np.mean(fixed_per_key)), float(np.mean(row_per_key))
    layer_s = 0.0
    for c in range(w.n_chunks):
        cs, e = w.chunk_bounds(c)
        layer_s += w.hq * (fk * e + rk * e * (e - cs))
    desc = (f"{done} (head, chunk) units of {w.hq * w.n_chunks} (chunks {sorted(chunks_seen)}), each the chunk's "
            f"estimation+selection{'+refinement' if w.refine_tau else ''} for one head and up to {n_rows} sampled "
            f"query rows of its attention; per-key rates extrapolated to every row, chunk and head")
    return w.seq_len / layer_s, spent, desc


_ORACLE_INPUTS: dict = {}


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count()


def run_reference(args, world: int = 1):
    w = select_workload(args)
    (wr, _, _), wj, job_layers = job_workloads(args, 0, world)
    for _ in range(args.warmup):
        oracle_sample(w, budget_s=2.0, n_rows=16, seed=99)
    vals, walls = [], []
    for i in range(args.steps):
        v, spent, desc = oracle_sample(w, budget_s=8.0, n_rows=32, seed=i)
        vals.append(v)
        walls.append(spent)
    value = statistics.median(vals)
    cb = {"value": round(value, 3), "unit": "tokens/s", "cores": cpu_cores(), "kind": "oracle", "sample": desc}
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(w.seq_len / value * 1e3, 1),
        # a step is a bounded sample: ms_per_step is the layer time extrapolated from it
        "extrapolated": True, "timed_wall_s_per_step": round(statistics.mean(walls), 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded generator)",
        "config": workload_config(args, wr, wj, world, job_layers),
        "cpu_baseline": cb,
        "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ----------------------------------------------------------------------------- main
def main():
    faulthandler.enable()  # a native crash prints the Python stack to stderr
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, world)), flush=True)
        return 0
    if not torch.cuda.is_available():
        print(json.dumps({"metric": METRIC, "error": "no CUDA device"}))
        return 1
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime

        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=device)
    res, w, lay = run_ours(args, rank, world, device)
    if rank == 0 and world == 1 and not args.no_cpu_baseline and args.mask == "selected":
        v, spent, desc = oracle_sample(w, budget_s=15.0, n_rows=64)
        res["cpu_baseline"] = {"value": round(v, 3), "unit": "tokens/s", "cores": cpu_cores(), "kind": "oracle",
                               "sample": desc, "seconds": round(spent, 1)}
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
