"""Timing of the CPU oracle on a bounded sample of one layer (test infrastructure: the bench's
``cpu_baseline`` and ``--impl reference`` legs only; both use the one procedure below).

One sample is, for each head group: ``SAMPLE_HEADS`` heads through the pre-attention pipeline (gather of
Q, K and V, pooling, logits, selection, tile mask), then exact float64 attention of one of those heads on
``SAMPLE_TILES`` seeded query tiles. The tile plan is built once per geometry outside the timed sample
(the GPU path caches it too, as the pages' layout cache does). The sample is extrapolated linearly to the
whole layer: pre-attention time per head x heads, plus attention time per attended tile pair x the
layer's attended pairs. A figure is the median of several samples.
"""
from __future__ import annotations

import os
import statistics
import time

import numpy as np

from . import veda as O

SAMPLE_HEADS = 2   # heads per head group through the pre-attention stages
SAMPLE_TILES = 32  # query tiles per head group through exact attention


def _threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


class _Layer:
    """Inputs and the cached per-group plans of one workload."""

    def __init__(self, wl):
        import veda_synth as V
        self.wl = wl
        self.q, self.k, self.v = (x.float().numpy() for x in V.make_qkv(wl))
        self.pq, self.pk = (x.numpy().astype(np.float64) for x in V.make_projections(wl))
        tile_refs = not O.keeps_all(wl.reference)
        lps = O.least_padding_shape(wl.target[1])
        groups = {}
        for h, s in enumerate(wl.head_shapes):
            groups.setdefault(tuple(lps if s is None else s), []).append(h)
        self.groups = []
        for shape, heads in sorted(groups.items()):
            lay = O.build_layout(O.layer_spans(wl.ref_spans, (wl.target[0], wl.target[1], shape), tile_refs),
                                 wl.seq_len)
            self.groups.append((heads, lay))


def _sample(layer, seed, heads_per_group=SAMPLE_HEADS, tiles_per_group=SAMPLE_TILES):
    """One timed sample; returns (extrapolated ms per layer, CPU seconds spent, heads, tile pairs)."""
    wl = layer.wl
    rng = np.random.default_rng(seed)
    t_pre = t_att = 0.0
    heads_done = pairs_sampled = 0
    pairs_layer = 0.0
    for heads, lay in layer.groups:
        sub = sorted(rng.choice(heads, size=min(heads_per_group, len(heads)), replace=False).tolist())
        t0 = time.perf_counter()
        qt, kt, vt = O.gather(layer.q, lay, sub), O.gather(layer.k, lay, sub), O.gather(layer.v, lay, sub)
        scores = O.logits(O.pool(qt, lay), O.pool(kt, lay), layer.pq[sub], layer.pk[sub])
        kept = O.select(scores.astype(np.float32), lay, O.column_blocks(lay, wl.generated, wl.reference))
        mask = O.block_mask(kept, lay)
        t_pre += time.perf_counter() - t0
        heads_done += len(sub)
        counts = mask.sum(-1)  # [len(sub), n_tiles]
        pairs_layer += counts.mean(0).sum() * len(heads)
        pick = rng.choice(lay.n_tiles, size=min(tiles_per_group, lay.n_tiles), replace=False)
        t0 = time.perf_counter()
        O.attend_tiles(qt[:, :1], kt[:, :1], vt[:, :1], lay, lambda hh, i: np.flatnonzero(mask[0, i]), q_tiles=pick)
        t_att += time.perf_counter() - t0
        pairs_sampled += int(counts[0, pick].sum())
    ms = 1e3 * (t_pre / heads_done * wl.heads + t_att / max(pairs_sampled, 1) * pairs_layer)
    return ms, t_pre + t_att, heads_done, pairs_sampled


def _describe(layer, n):
    g = len(layer.groups)
    return (f"per sample: {SAMPLE_HEADS} heads of each of the {g} head group(s) through gather/pool/logits/"
            f"select/mask and exact float64 attention of one head on {SAMPLE_TILES} seeded query tiles per "
            f"group, extrapolated linearly to the whole layer (plan built once, outside the samples); "
            f"median of {n} samples")


def time_layer(wl, budget_s=20.0):
    """The ``cpu_baseline`` leg: samples (at least three) until about ``budget_s`` seconds of CPU work."""
    layer = _Layer(wl)
    _sample(layer, seed=1000, heads_per_group=1, tiles_per_group=2)  # warm-up (thread pools, first touches)
    vals, spent_all = [], 0.0
    seed = 0
    while len(vals) < 3 or spent_all < budget_s:
        ms, spent, _, _ = _sample(layer, seed)
        vals.append(ms)
        spent_all += spent
        seed += 1
    return {"value": round(statistics.median(vals), 1), "unit": "ms/layer", "cores": _threads(), "kind": "oracle",
            "sample": _describe(layer, len(vals)) + f" ({spent_all:.1f} s of CPU work)"}


def reference_arm(wl, steps, warmup, metric, unit, n_gpus=1):
    """``bench.py --impl reference``: one sample per step (the same sample as ``time_layer``), median."""
    layer = _Layer(wl)
    for i in range(warmup):
        _sample(layer, seed=1000 + i, heads_per_group=1, tiles_per_group=2)
    vals, spent_all = [], 0.0
    for i in range(steps):
        ms, spent, _, _ = _sample(layer, seed=i)
        vals.append(ms)
        spent_all += spent
    value = float(statistics.median(vals)) if vals else float("nan")
    cores = _threads()
    return {"impl": "reference", "metric": metric, "value": round(value, 1), "unit": unit, "n_gpus": n_gpus,
            "steps": steps, "warmup": warmup, "ms_per_step": round(value, 1), "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (same seeded inputs)",
            "config": {"workload": f"{wl.name}: {wl.note}", "seq_len": wl.seq_len, "heads": wl.heads,
                       "head_dim": wl.dim},
            "cpu_baseline": {"value": round(value, 1), "unit": unit, "cores": cores, "kind": "oracle",
                             "sample": _describe(layer, len(vals))},
            "e2e": {"value": round(value, 1), "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "host_seconds": round(spent_all, 1),
            "note": "each step times a bounded sample and reports the layer time extrapolated from it, so "
                    "ms_per_step x steps is not the wall time of the run"}
