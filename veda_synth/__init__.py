"""Seeded synthetic inputs for the Veda sparse-attention path.

This module only draws numbers and describes workloads: the packed sequence of each workload (text
rows, reference spans, target span and their grids), the target box of each head (``None`` means
"the least-padding box", which each consumer derives for itself), the budgets, and seeded Q/K/V and
predictor projections. It holds none of the method's arithmetic and is the one module that both the
CPU oracle's tests and the CUDA path's callers use.

Recipe (fixed):

* ``torch.Generator('cpu')`` seeds: 0 -> Q, 1 -> K, 2 -> V, 3 -> proj_q, 4 -> proj_k,
  5 -> locality bias, 6 -> text-row bias directions. Everything is drawn on the host in fp32 and
  rounded to bf16; the same bytes go to the oracle and to the GPU.
* Q, K, V ~ N(0, 1).
* Locality bias (workloads with ``bias=True``): each video row at grid position ``p = (t, h, w)``
  gets ``phi(p) = [cos(w_j . p), sin(w_j . p)]_{j=1..8} / sqrt(8)`` (unit norm), with ``w_j`` a seeded
  random direction scaled to a wavelength between 4 and 32 rows; reference rows use ``t = 0``, text
  rows a seeded random unit vector. Per head ``U_h`` (``D x 16``, N(0, 1)) and
  ``Q += U_h phi``, ``K += U_h phi``, so nearby tiles score higher and the top-k is not uniform.
* Projections ``[H, 3D, D]`` ~ N(0, 1/D), rounded to bf16-representable fp32.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

SEED_Q, SEED_K, SEED_V, SEED_PQ, SEED_PK, SEED_BIAS, SEED_TEXT = range(7)


@dataclass(frozen=True)
class Workload:
    """One synthetic attention layer.

    ``ref_spans`` are ``(start, (T, H, W))``; ``target`` is ``(start, (T, H, W))``; every other row of
    the ``seq_len`` packed rows is a text/global row. ``head_shapes[h]`` is the target box of head
    ``h`` or ``None`` for the least-padding box. Budgets are ``(ratio, tiles)`` pairs with exactly one
    set. ``fp8_qk`` asks for the FP8 e4m3 Q/K variant, ``int8_qk`` for the INT8 one.
    """
    name: str
    heads: int
    dim: int
    seq_len: int
    ref_spans: tuple
    target: tuple
    head_shapes: tuple
    generated: tuple
    reference: tuple
    bias: bool
    fp8_qk: bool = False
    note: str = ""
    int8_qk: bool = False
    extra: dict = field(default_factory=dict, compare=False, hash=False)


def _ratio(r):
    return (float(r), None)


def _tiles(n):
    return (None, int(n))


_DENSE = _ratio(1.0)
_GRID_104K = (26, 48, 84)


def _mixed():
    text, ref = 512, (1, 48, 84)
    ref_rows = ref[0] * ref[1] * ref[2]
    shapes = tuple((1, 8, 16) if h % 3 == 0 else (8, 4, 4) if h % 3 == 1 else None for h in range(24))
    return Workload("mixed", 24, 128, text + ref_rows + 26 * 48 * 84, ((text, ref),),
                    (text + ref_rows, _GRID_104K), shapes, _ratio(0.10), _ratio(0.10), True,
                    note="512 text rows + reference (1,48,84) + generated (26,48,84), per-head boxes")


def workloads():
    """Every named workload: the five published configurations, the sweep points and small cases."""
    w = {}
    w["tiny"] = Workload("tiny", 2, 64, 2048, (), (0, (8, 16, 16)), ((2, 8, 8),) * 2,
                         _tiles(4), _DENSE, False, note="grid (8,16,16), box (2,8,8), 4 tiles per row")
    w["single"] = Workload("single", 24, 128, 104832, (), (0, _GRID_104K), (None,) * 24,
                           _ratio(0.10), _DENSE, True, note="grid (26,48,84) = 104,832 rows, ratio 0.10")
    w["mixed"] = _mixed()
    w["long"] = Workload("long", 24, 128, 219600, (), (0, (61, 45, 80)), (None,) * 24,
                         _ratio(0.05), _DENSE, True, note="grid (61,45,80) = 219,600 rows, ratio 0.05")
    for tag, b in (("tiles24", _tiles(24)), ("r010", _ratio(0.10)), ("r025", _ratio(0.25)),
                   ("r050", _ratio(0.50)), ("dense", _ratio(1.0))):
        w["sweep_" + tag] = Workload("sweep_" + tag, 24, 128, 104832, (), (0, _GRID_104K), (None,) * 24,
                                     b, _DENSE, True, note=f"budget sweep on (26,48,84): {tag}")
    w["sweep_fp8"] = Workload("sweep_fp8", 24, 128, 104832, (), (0, _GRID_104K), (None,) * 24,
                              _ratio(0.10), _DENSE, True, fp8_qk=True,
                              note="FP8 e4m3 Q/K with per-tile fp32 scales, ratio 0.10")
    w["sweep_int8"] = Workload("sweep_int8", 24, 128, 104832, (), (0, _GRID_104K), (None,) * 24,
                               _ratio(0.10), _DENSE, True, int8_qk=True,
                               note="INT8 Q/K with per-tile fp32 scales, ratio 0.10")
    # the 104k-token layer with 4 heads: a profiling case that still exceeds L2 (322 MB of Q/K/V)
    w["single_h4"] = Workload("single_h4", 4, 128, 104832, (), (0, _GRID_104K), (None,) * 4,
                              _ratio(0.10), _DENSE, True, note="grid (26,48,84), 4 heads, ratio 0.10 (profiling)")
    # small cases that finish in seconds on the oracle and still span several tiles and a ragged tail
    w["padded_tiny"] = Workload("padded_tiny", 2, 64, 200 + 3 * 10 * 12, (), (200, (3, 10, 12)),
                                ((2, 8, 8),) * 2, _ratio(0.5), _DENSE, True,
                                note="200 global rows + grid (3,10,12) at box (2,8,8): padding, partial tiles")
    w["small_mixed"] = Workload("small_mixed", 3, 64, 150 + 2 * 16 * 16 + 6 * 16 * 24,
                                ((150, (2, 16, 16)),), (150 + 512, (6, 16, 24)),
                                ((1, 8, 16), (8, 4, 4), None), _ratio(0.3), _ratio(0.5), True,
                                note="text + reference + target, three per-head boxes")
    w["small_dense"] = Workload("small_dense", 2, 64, 100 + 4 * 8 * 24, (), (100, (4, 8, 24)),
                                (None, (1, 8, 16)), _DENSE, _DENSE, True, note="keeps-all budget")
    w["small_d128"] = Workload("small_d128", 2, 128, 5 * 12 * 40 + 77, (), (77, (5, 12, 40)),
                               (None, (2, 8, 8)), _ratio(0.2), _DENSE, True,
                               note="head_dim 128, ragged grid, global prefix")
    return w


def workload(name):
    return workloads()[name]


def row_positions(wl):
    """``[S, 3]`` float64 grid positions (t, h, w) of every packed row and a ``[S]`` bool video flag."""
    pos = torch.zeros(wl.seq_len, 3, dtype=torch.float64)
    video = torch.zeros(wl.seq_len, dtype=torch.bool)
    spans = [(s, g, True) for s, g in wl.ref_spans] + [(wl.target[0], wl.target[1], False)]
    for start, (T, H, W), is_ref in spans:
        t, h, w = torch.meshgrid(torch.arange(T), torch.arange(H), torch.arange(W), indexing="ij")
        rows = slice(start, start + T * H * W)
        pos[rows, 0] = 0.0 if is_ref else t.reshape(-1).double()
        pos[rows, 1] = h.reshape(-1).double()
        pos[rows, 2] = w.reshape(-1).double()
        video[rows] = True
    return pos, video


def _locality_bias(wl):
    g = torch.Generator("cpu").manual_seed(SEED_BIAS)
    direction = torch.randn(8, 3, generator=g, dtype=torch.float64)
    direction /= direction.norm(dim=1, keepdim=True)
    wavelength = 4.0 + 28.0 * torch.rand(8, generator=g, dtype=torch.float64)
    omega = direction * (2.0 * math.pi / wavelength)[:, None]               # [8, 3]
    U = torch.randn(wl.heads, wl.dim, 16, generator=g, dtype=torch.float32)  # [H, D, 16]
    pos, video = row_positions(wl)
    ang = pos @ omega.T                                                      # [S, 8]
    phi = torch.cat([torch.cos(ang), torch.sin(ang)], dim=1) / math.sqrt(8.0)
    n_text = int((~video).sum())
    if n_text:
        gt = torch.Generator("cpu").manual_seed(SEED_TEXT)
        rnd = torch.randn(n_text, 16, generator=gt, dtype=torch.float64)
        phi[~video] = rnd / rnd.norm(dim=1, keepdim=True)
    return torch.einsum("hdj,sj->shd", U, phi.float())                      # [S, H, D]


def make_qkv(wl):
    """Seeded ``q, k, v`` as bf16 CPU tensors ``[S, H, D]`` (contiguous)."""
    shape = (wl.seq_len, wl.heads, wl.dim)
    out = []
    bias = _locality_bias(wl) if wl.bias else None
    for seed, biased in ((SEED_Q, True), (SEED_K, True), (SEED_V, False)):
        g = torch.Generator("cpu").manual_seed(seed)
        x = torch.randn(shape, generator=g, dtype=torch.float32)
        if bias is not None and biased:
            x += bias
        out.append(x.to(torch.bfloat16))
        del x
    return tuple(out)


def make_projections(wl):
    """Seeded predictor projections ``proj_q, proj_k`` as fp32 ``[H, 3D, D]`` ~ N(0, 1/D), each value
    rounded to the nearest bf16 (the published predictors are stored in bf16 or lower)."""
    out = []
    for seed in (SEED_PQ, SEED_PK):
        g = torch.Generator("cpu").manual_seed(seed)
        p = torch.randn(wl.heads, 3 * wl.dim, wl.dim, generator=g, dtype=torch.float32) / math.sqrt(wl.dim)
        out.append(p.to(torch.bfloat16).to(torch.float32))
    return tuple(out)


def head_groups(wl, resolve):
    """Heads grouped by target box, in ascending box order. ``resolve(None)`` must return the
    least-padding box of the target grid (each caller computes it with its own planner)."""
    groups = {}
    for h, s in enumerate(wl.head_shapes):
        shp = tuple(resolve(None) if s is None else s)
        groups.setdefault(shp, []).append(h)
    return [(shp, groups[shp]) for shp in sorted(groups)]


def sample_tiles(n_tiles, n_video, count, seed=11):
    """A seeded sample of query tile ids that always holds the first, the last video, the first and
    the last global tile (when there are any)."""
    g = torch.Generator("cpu").manual_seed(seed)
    must = {0, n_video - 1, n_tiles - 1}
    if n_tiles > n_video:
        must.add(n_video)
    rest = torch.randperm(n_tiles, generator=g)[:count].tolist()
    return sorted(set(rest) | {m for m in must if 0 <= m < n_tiles})
