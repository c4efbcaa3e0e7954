"""Timing of the CPU oracle on a bounded sample of one layer (test infrastructure: the bench's
``cpu_baseline`` and ``--impl reference`` legs only).

A sample is: for ``heads_sampled`` heads of each head group, the whole pre-attention pipeline (layout,
gather of Q, K and V, pooling, logits, selection, tile mask), plus exact attention for a seeded sample
of (head, query tile) items. The layer time is extrapolated linearly: pre-attention time per head x
heads, and attention time per attended tile pair x the layer's attended pairs.
"""
from __future__ import annotations

import os
import time

import numpy as np

from . import veda as O


def _threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def _sample_layer(wl, q, k, v, pq, pk, heads_sampled, items, seed):
    generated, reference = wl.generated, wl.reference
    tile_refs = not O.keeps_all(reference)
    lps = O.least_padding_shape(wl.target[1])
    groups = {}
    for h, s in enumerate(wl.head_shapes):
        groups.setdefault(tuple(lps if s is None else s), []).append(h)
    rng = np.random.default_rng(seed)
    t_pre = 0.0
    t_att = 0.0
    pairs_sampled = 0
    pairs_layer = 0
    heads_done = 0
    for shape, heads in sorted(groups.items()):
        sub = heads[:heads_sampled]
        t0 = time.perf_counter()
        lay = O.build_layout(O.layer_spans(wl.ref_spans, (wl.target[0], wl.target[1], shape), tile_refs),
                             wl.seq_len)
        qt, kt, vt = O.gather(q, lay, sub), O.gather(k, lay, sub), O.gather(v, lay, sub)
        scores = O.logits(O.pool(qt, lay), O.pool(kt, lay), pq[sub], pk[sub])
        kept = O.select(scores.astype(np.float32), lay, O.column_blocks(lay, generated, reference))
        mask = O.block_mask(kept, lay)
        t_pre += time.perf_counter() - t0
        heads_done += len(sub)
        counts = mask.sum(-1)  # [len(sub), n_tiles]
        pairs_layer += counts.mean(0).sum() * len(heads)
        pick = rng.choice(lay.n_tiles, size=min(items, lay.n_tiles), replace=False)
        t0 = time.perf_counter()
        O.attend_tiles(qt[:, :1], kt[:, :1], vt[:, :1], lay, lambda hh, i: np.flatnonzero(mask[0, i]), q_tiles=pick)
        t_att += time.perf_counter() - t0
        pairs_sampled += counts[0, pick].sum()
    ms = 1e3 * (t_pre / heads_done * wl.heads + t_att / max(pairs_sampled, 1) * pairs_layer)
    return ms, t_pre + t_att, heads_done, int(pairs_sampled)


def _inputs(wl):
    import veda_synth as V
    q, k, v = (x.float().numpy() for x in V.make_qkv(wl))
    pq, pk = (x.numpy().astype(np.float64) for x in V.make_projections(wl))
    return q, k, v, pq, pk


def time_layer(wl, budget_s=20.0):
    """One bounded oracle sample (about ``budget_s`` seconds of CPU work), extrapolated to ms/layer.

    The sample grows (more heads per head group, more query tiles) until the CPU work spent on the last
    sample reaches about half the budget; the estimate of the largest sample is reported."""
    q, k, v, pq, pk = _inputs(wl)
    heads_sampled, items, seed = 1, 16, 0
    total = 0.0
    while True:
        ms, spent, hs, pairs = _sample_layer(wl, q, k, v, pq, pk, heads_sampled, items, seed=seed)
        total += spent
        if spent >= budget_s / 2 or total >= budget_s or heads_sampled >= wl.heads:
            break
        grow = max(2.0, min(8.0, (budget_s / 2) / max(spent, 1e-3)))
        heads_sampled = min(wl.heads, int(round(heads_sampled * grow)))
        items = int(items * grow)
        seed += 1
    return {"value": round(ms, 1), "unit": "ms/layer", "cores": _threads(), "kind": "oracle",
            "sample": f"{hs} of {wl.heads} heads through layout/gather/pool/logits/select/mask, exact float64 "
                      f"attention on {pairs} attended tile pairs; extrapolated linearly to the whole layer "
                      f"({spent:.1f} s of CPU work in the reported sample, {total:.1f} s in all)"}


def reference_arm(wl, steps, warmup, metric, unit, n_gpus=1):
    """``bench.py --impl reference``: the oracle timed per step on a bounded sample of the layer."""
    q, k, v, pq, pk = _inputs(wl)
    for i in range(warmup):
        _sample_layer(wl, q, k, v, pq, pk, 1, 4, seed=100 + i)
    vals, spent_all = [], 0.0
    for i in range(steps):
        ms, spent, hs, pairs = _sample_layer(wl, q, k, v, pq, pk, 1, 8, seed=i)
        vals.append(ms)
        spent_all += spent
    value = float(np.median(vals))
    cores = _threads()
    sample = (f"per step: 1 head per head group through layout/gather/pool/logits/select/mask and exact float64 "
              f"attention on ~8 query tiles, extrapolated to the whole layer; median of {steps} steps")
    return {"impl": "reference", "metric": metric, "value": round(value, 1), "unit": unit, "n_gpus": n_gpus,
            "steps": steps, "warmup": warmup, "ms_per_step": round(value, 1), "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (same seeded inputs)",
            "config": {"workload": f"{wl.name}: {wl.note}", "seq_len": wl.seq_len, "heads": wl.heads,
                       "head_dim": wl.dim},
            "cpu_baseline": {"value": round(value, 1), "unit": unit, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 1), "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "host_seconds": round(spent_all, 1)}
