"""Benchmark of one Veda sparse-attention layer on B200.

python bench.py [--gpus N] [--steps K] [--warmup W] [--workload single] [--impl veda|reference]
               [--path auto|gathered|direct]

A step is one whole layer with the tile plan cached (as the pages' layout cache does). On the default
path (the layer's choice: gather-free wherever every head group's layout has a box form, which holds for
every published configuration) a step is pool Q and K, score, select, and the attend reading the tiles
as TMA boxes of the packed tensors with the scatter fused; on the tile-order path (``--path gathered``)
it is gather+pool Q and K, score, select, gather V, attend. Inputs are seeded synthetic bf16 tensors of
the workload's shape, resident in HBM when the timed region starts; they total more than the 126 MB
L2, so no flush is needed between steps. With N GPUs each rank runs its own layer (independent
problems, weak scaling) and the time is the max over ranks.

Rank 0 prints one JSON line. ``value`` is ms per layer for the whole job (step time / layers per step
over all ranks), lower is better. ``--impl reference`` times the CPU oracle on the host cores on a
bounded sample of the same layer, extrapolated to ms per layer.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import veda_synth as V  # noqa: E402

METRIC = "ms per sparse attention layer (104k tok, 10% kept); kept-tile TFLOP/s vs peak"
UNIT = "ms/layer"


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sustained=d["bf16_tflops_sustained"],
                    source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


def attend_source_hash():
    h = hashlib.sha256()
    for f in ("attend.cuh", "attend_pair.cuh", "ptx.cuh"):
        h.update(open(os.path.join(ROOT, "learned_block_sparse_tile_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(workload, dim):
    """DRAM bytes per attend launch from the committed ncu summary, when it was taken on this kernel."""
    p = os.path.join(ROOT, "profiles", "attend_traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    e = d.get(workload)
    if not e or e.get("attend_source") != attend_source_hash():
        return None
    return e.get("bytes_per_launch")


class Clocks:
    """SM clock and clock-event reasons of this rank's GPU, sampled every ~10 ms by a thread during the
    timed region (NVML reads only; nvidia-smi at 200 ms where NVML is missing). Nothing is changed."""

    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4), ("hw_power_brake_slowdown", 0x80))

    def __init__(self, device_index, period_s=0.01):
        self.index, self.period = device_index, period_s
        self.rows, self.proc, self.thread = [], None, None

    def _handle(self, nv):
        try:
            pr = torch.cuda.get_device_properties(self.index)
            bus = f"{pr.pci_domain_id:08X}:{pr.pci_bus_id:02X}:{pr.pci_device_id:02X}.0"
            return nv.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return nv.nvmlDeviceGetHandleByIndex(self.index)

    def __enter__(self):
        import threading
        try:
            import pynvml as nv
            nv.nvmlInit()
            h = self._handle(nv)
            self.sm_max = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
        except Exception:
            nv = None
        if nv is None:
            return self._start_smi()
        self.stop = threading.Event()

        def poll():
            while not self.stop.is_set():
                try:
                    sm = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                    bits = int(nv.nvmlDeviceGetCurrentClocksEventReasons(h))
                    watts = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                    self.rows.append((sm, bits, watts))
                except Exception:
                    pass
                self.stop.wait(self.period)

        self.thread = threading.Thread(target=poll, daemon=True)
        self.thread.start()
        return self

    def _start_smi(self):
        q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
             "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
             "clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.thread is not None:
            self.stop.set()
            self.thread.join(timeout=5)
            return
        if self.proc is None:
            return
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) >= 7:
                try:
                    bits = sum(b for (_, b), v in zip(self.REASONS[:4], f[3:7]) if v.lower() == "active")
                    self.rows.append((float(f[0]), bits, float(f[2])))
                    self.sm_max = float(f[1])
                except ValueError:
                    pass

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        sm = [r[0] for r in self.rows]
        reasons = sorted({name for _, bits, _ in self.rows for name, b in self.REASONS if bits & b})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": getattr(self, "sm_max", None), "reasons": reasons,
                "samples": len(self.rows), "power_w_max": round(max(r[2] for r in self.rows), 1),
                "source": "nvml, 10 ms" if self.thread is not None else "nvidia-smi, 200 ms"}


def max_over_ranks(value, world, device):
    """The largest of every rank's ``value`` (a time), as a float; collective only over the timings."""
    if world <= 1:
        return float(value)
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def flops_per_pair(dim):
    return 4.0 * 128 * 128 * dim


def stage_bytes(layer, wl):
    """Algorithmic HBM bytes per launch of each stage, summed over head groups."""
    D, S = wl.dim, wl.seq_len
    out = {"gather_qk": 0, "pool_qk": 0, "score": 0, "select": 0, "gather_v": 0, "attend": 0}
    for g in layer.groups:
        lay, n = g["layout"], len(g["heads_list"])
        real = n * S * D * 2
        slots = n * lay.n_slots * D * 2
        feats = n * lay.n_video * 3 * D * 4
        # the FP8 Q/K variant writes e4m3 codes (1 byte per element) and per-tile scales instead of bf16
        eight_bit = layer.fp8_qk or layer.int8_qk
        tiles_out = slots // 2 + n * lay.n_tiles * 4 if eight_bit else slots
        if layer.direct:  # Q and K are read once for the pooled features; no tile-order copies
            out["pool_qk"] += 2 * (real + feats)
        else:
            out["gather_qk"] += 2 * (real + tiles_out + feats)
            out["gather_v"] += real + slots
        sc = n * lay.n_video * lay.n_video * 4
        proj = 2 * n * 3 * D * D * 4
        hat = 2 * n * lay.n_video * D * 4
        out["score"] += 2 * feats + proj + 2 * hat + sc
        kept = int(g["kept_cnt"].sum())
        out["select"] += sc + 4 * (kept + n * lay.n_video)
        # Q, K and V each read once per head (re-reads of a kept K/V tile are L2 hits), O written once,
        # the kept lists read
        qk_in = slots // 2 if eight_bit else real if layer.direct else slots
        v_in = real if layer.direct else slots
        out["attend"] += 2 * qk_in + v_in + real + 4 * (kept + n * lay.n_video)
    return out


def run_veda(args, rank, world, local):
    import torch.distributed as dist
    from learned_block_sparse_tile_b200 import HostPipeline, VedaLayer, _lib as L

    torch.cuda.set_device(local)
    L.veda_device_check()
    wl = V.workload(args.workload)
    q, k, v = V.make_qkv(wl)
    pq, pk = V.make_projections(wl)
    layer = VedaLayer(wl.seq_len, wl.ref_spans, wl.target, wl.head_shapes, (wl.generated, wl.reference),
                      wl.heads, wl.dim, device=f"cuda:{local}", fp8_qk=wl.fp8_qk, int8_qk=wl.int8_qk,
                      direct={"auto": None, "gathered": False, "direct": True}[args.path],
                      logit_bound=args.logit_bound == "on", paired=args.paired == "on")
    direct = layer.direct
    layer.set_projections(pq, pk)
    dq, dk, dv = q.cuda(), k.cuda(), v.cuda()
    out = torch.empty_like(dq)
    stream = torch.cuda.current_stream()

    def step(ev=None):
        layer.forward(dq, dk, dv, out, stream=stream, events=ev)

    for _ in range(args.warmup):
        step()
    if L.veda_sync_status(stream) != L.VEDA_OK:
        raise RuntimeError(L.veda_last_error())

    # timed region: K whole layers, attend launches bracketed by events on the same stream
    stage_ev = {}
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with Clocks(local) as clk:
        t0.record(stream)
        for _ in range(args.steps):
            step(stage_ev)
        t1.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    rc = L.veda_sync_status(stream)
    if rc != L.VEDA_OK:
        raise RuntimeError(L.veda_last_error())
    ms_total = t0.elapsed_time(t1)
    stage_ms = {name: sum(a.elapsed_time(b) for a, b in evs) / args.steps for name, evs in stage_ev.items()}
    attend_launch_ms = stage_ms["attend"] / len(layer.groups)
    ms_step = max_over_ranks(ms_total / args.steps, world, f"cuda:{local}")

    # end to end through the public API: every step uploads its Q/K/V from pinned host memory and downloads
    # its output; HostPipeline overlaps step i's kernels with step i + 1's upload and step i - 1's download
    # (independent layer calls), so a step costs about the slowest of the three
    hq, hk, hv = (x.pin_memory() for x in (q, k, v))
    hout = torch.empty_like(hq).pin_memory()
    e2e_steps = max(1, min(args.steps, 8))
    pipe = HostPipeline(layer, wl.seq_len, wl.heads, wl.dim, device=f"cuda:{local}")
    pipe.run([(hq, hk, hv)] * 2, [hout] * 2, stream=stream)  # warm-up of the pipeline's streams
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    pipe.run([(hq, hk, hv)] * e2e_steps, [hout] * e2e_steps, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize()
    if L.veda_sync_status(stream) != L.VEDA_OK:
        raise RuntimeError(L.veda_last_error())
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, world, f"cuda:{local}")

    work = layer.work_tiles()
    pairs = layer.attended_tile_pairs()
    kept_flops = flops_per_pair(wl.dim) * work
    pk_ = peaks()
    achieved_tflops = kept_flops / (attend_launch_ms * len(layer.groups)) / 1e9
    # the denominator: the burst cuBLAS figure for a timed region shorter than a second (the GPU has not
    # settled at its power cap), the sustained one for a seconds-long loop
    sustained = ms_total >= 1000.0
    peak = pk_["bf16_sustained"] if sustained else pk_["bf16"]
    peak_kind = (f"{pk_['source']} " + ("sustained cuBLAS bf16 (timed region of a second or more)" if sustained
                                        else "burst cuBLAS bf16 (timed region under a second)"))
    sbytes = stage_bytes(layer, wl)
    stages = {}
    for name, ms in stage_ms.items():
        gbs = sbytes[name] / (ms * 1e-3) / 1e9 if ms > 0 else None
        stages[name] = {"ms": round(ms, 4), "bytes": sbytes[name], "gb_s": round(gbs, 1) if gbs else None,
                        "hbm_frac": round(gbs / pk_["hbm"], 3) if gbs else None}
    traffic = recorded_traffic(args.workload + ("/direct" if direct else "") + ("/paired" if layer.paired else ""),
                               wl.dim)
    kernel = (f"attend_pair_kernel<{wl.dim}> (with its list merge and redo pass)" if layer.paired
              else f"attend_kernel<{wl.dim}>")
    dense_pairs = wl.heads * (wl.seq_len / 128.0) ** 2
    res = {
        "metric": METRIC, "value": round(ms_step / world, 4), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3 Q/K, bf16 P/V" if wl.fp8_qk else "int8 Q/K, bf16 P/V" if wl.int8_qk else "bf16",
        "data": "synthetic (seeded N(0,1) bf16 Q/K/V with a low-rank locality bias; random predictor projections)",
        "config": {"workload": f"{wl.name}: {wl.note}", "seq_len": wl.seq_len, "heads": wl.heads,
                   "head_dim": wl.dim, "budget": {"generated": wl.generated, "reference": wl.reference},
                   "head_groups": [list(g["box"]) for g in layer.groups],
                   "attend_path": ("gather-free: Q/K pooled in place, tiles loaded as TMA boxes of the packed tensors"
                                   if direct else "tile-order copies of Q/K/V (gather), then attend"),
                   "logit_bound": layer.logit_bound, "paired": layer.paired,
                   "parallelism": f"replicas x{world} (one layer per rank)",
                   "l2": "no flush: per-step inputs and outputs (2.6 GB at 104k tokens) exceed the 126 MB L2"},
        "kept_tile_tflops": round(achieved_tflops, 1),
        "kept_tile_work": work, "attended_tile_pairs": pairs,
        "work_share_of_dense": round(work / dense_pairs, 4),
        "stages": stages,
        "roofline": {"bound": "tensor", "kernel": kernel, "achieved": round(achieved_tflops, 1),
                     "peak": peak, "unit": "TFLOP/s", "frac": round(achieved_tflops / peak, 3),
                     "peak_kind": peak_kind, "timed_region_s": round(ms_total / 1e3, 3),
                     "frac_of_burst_peak": round(achieved_tflops / pk_["bf16"], 3),
                     "frac_of_sustained_peak": round(achieved_tflops / pk_["bf16_sustained"], 3),
                     "traffic": traffic,
                     "algorithmic_flops_per_launch": kept_flops / len(layer.groups),
                     "launch_ms": round(attend_launch_ms, 4)},
        "e2e": {"value": round(e2e_ms / world, 4), "unit": UNIT,
                "h2d_bytes_per_step": 3 * q.numel() * q.element_size(),
                "d2h_bytes_per_step": out.numel() * out.element_size(),
                "steps": e2e_steps, "overlap": "uploads, kernels and downloads of consecutive steps on three streams"},
        "gpu_launches": layer.launches * args.steps,
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(wl, args.cpu_budget_s)
    return res


def cpu_baseline(wl, budget_s):
    """The oracle as it stands, on the host cores, on a bounded sample of the layer (extrapolated)."""
    from oracle import timing
    return timing.time_layer(wl, budget_s)


def launch_ranks(n, argv, port=None):
    """Runs this script with ``argv`` as ``n`` local ranks (torch.distributed.run, rendezvous on 127.0.0.1);
    returns the launcher's exit status."""
    import socket
    if port is None:
        with socket.socket() as sk:
            sk.bind(("127.0.0.1", 0))
            port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr=127.0.0.1", f"--master-port={port}", os.path.abspath(__file__), *argv]
    return subprocess.call(cmd)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="single")
    ap.add_argument("--path", default="auto", choices=["auto", "gathered", "direct"],
                    help="attend on tile-order copies (gathered), on the packed tensors as TMA boxes (direct), "
                         "or the layer's choice (auto: direct where every layout has a box form)")
    ap.add_argument("--logit-bound", default="on", choices=["on", "off"],
                    help="attend with the Cauchy-Schwarz logit bound (later tiles of an item may skip the row max; "
                         "the same softmax) or with the exact row max on every tile")
    ap.add_argument("--paired", default="on", choices=["on", "off"],
                    help="with the logit bound: the paired attend (two query tiles per work item) or the single-tile one")
    ap.add_argument("--impl", default="veda", choices=["veda", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget-s", type=float, default=20.0)
    args = ap.parse_args()
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        # --gpus N without a launcher: start N ranks of this same command under torch.distributed.run
        sys.exit(launch_ranks(args.gpus, sys.argv[1:]))
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local = int(os.environ.get("LOCAL_RANK", 0))
    if world != args.gpus:
        raise SystemExit(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}; launch one rank per GPU")
    if args.impl == "reference":
        if rank != 0:
            return
        from oracle import timing
        res = timing.reference_arm(V.workload(args.workload), args.steps, args.warmup, METRIC, UNIT, world)
        print(json.dumps(res), flush=True)
        return
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device(f"cuda:{local}"))
    try:
        res = run_veda(args, rank, world, local)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
