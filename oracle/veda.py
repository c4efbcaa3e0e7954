"""Plain CPU restatement of Veda tile-skip sparse attention (test infrastructure only).

Source of every definition: the page ``veda_core.py`` (ComfyUI-FunPack node pack, "Veda sparse
attention, the torch half"). Citations below name that page's section and function. Where the page
is silent or ambiguous the reading adopted is stated in the docstring of the function it affects.

Conventions
-----------
* A budget is a pair ``(ratio, tiles)`` with exactly one of the two set (the other ``None``).
* A span is ``(start, (T, H, W), (st, sh, sw))``: a row-major 3D grid of packed rows starting at
  ``start``, cut into boxes of ``st*sh*sw == 128`` rows.
* Tile-ordered tensors follow the page's layout ``[N, H', D]`` with ``N = 128 * n_tiles``.
* Floating point work is float64 unless the page fixes otherwise (budget arithmetic is IEEE double
  in the page's left-to-right order; selection compares the fp32 scores it is given).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

TILE = 128

__all__ = [
    "TILE", "VedaError", "Layout", "ratio_budget", "tiles_budget", "sparsity_budget", "keeps_all",
    "row_budget", "split_budget", "extra_tile_rows", "tile_shapes", "padded_grid", "tile_count",
    "least_padding_shape", "span_tiles", "build_layout", "gather", "scatter", "pool", "logits",
    "column_blocks", "allowed_per_row", "select", "block_mask", "tile_index_list", "attend_tiles",
    "attend_dense_mask", "dense_attention", "attention_layer", "work_stats", "quantize_fp8_tiles",
    "attend_tiles_fp8", "quantize_int8_tiles", "attend_tiles_int8", "layer_spans", "grid_of",
    "describe_packed_layout",
]


class VedaError(ValueError):
    """A layout or budget the method cannot use (the page's ``VedaError``)."""


# ---------------------------------------------------------------------------------------------------
# budgets  (veda_core.py, section "budgets": sparsity_budget, keeps_all, _per_row, _split, _bresenham)
# ---------------------------------------------------------------------------------------------------

def ratio_budget(ratio):
    """A budget that keeps ``ratio`` of the key tiles (at equal kernel cost)."""
    return (float(ratio), None)


def tiles_budget(n):
    """A budget that keeps exactly ``n`` key tiles per query tile (the node's integer input)."""
    return (None, int(n))


def sparsity_budget(share):
    """Skipping a share ``s`` of the key tiles keeps the ratio ``1 - s`` (section "budgets")."""
    return (1.0 - float(share), None)


def _check_budget(budget):
    ratio, tiles = budget
    if (ratio is None) == (tiles is None):
        raise VedaError("a budget sets exactly one of ratio and tiles")


def keeps_all(budget):
    """True when the budget is a ratio of at least one and no tile count (section "budgets")."""
    _check_budget(budget)
    ratio, tiles = budget
    return tiles is None and ratio >= 1.0


def row_budget(budget, real_tokens, n_cols):
    """Fractional number of key tiles one query row keeps inside a block of ``n_cols`` tiles.

    veda_core.py, "budgets", _per_row: a tile count is used as is; a ratio is applied to the *ideal*
    tile count ``ceil(real_tokens / 128)`` of the block, squared, and spread over the padded column
    count, so a tiling with padding never receives a larger budget. The product is evaluated as
    ``((ratio * ideal) * ideal) / n_cols`` in IEEE double, the order the page writes it.
    """
    _check_budget(budget)
    ratio, tiles = budget
    if tiles is not None:
        return float(tiles)
    ideal = -(-int(real_tokens) // TILE)
    value = ratio * ideal
    value = value * ideal
    return value / n_cols


def split_budget(b, n_cols):
    """``(k_lo, k_hi, frac)`` for a fractional per-row budget ``b`` (veda_core.py, "budgets", _split).

    A budget of at least ``n_cols`` keeps the whole block: ``(n, n, 0.0)``. Otherwise
    ``k_lo = clamp(floor(b), 1, n)``, ``k_hi = min(k_lo + 1, n)`` and the fractional part
    ``b - k_lo``, clamped to [0, 1], is rounded to 12 decimals with Python's ``round``.
    """
    if b >= n_cols:
        return n_cols, n_cols, 0.0
    k_lo = math.floor(b)
    k_lo = min(max(1, k_lo), n_cols)
    k_hi = min(k_lo + 1, n_cols)
    frac = b - k_lo
    frac = min(max(frac, 0.0), 1.0)
    return k_lo, k_hi, round(frac, 12)


def extra_tile_rows(n_rows, frac):
    """Boolean ``[n_rows]``: which query rows get the one extra tile (veda_core.py, _bresenham).

    Row ``r`` gets it when ``floor((r + 1) * frac) > floor(r * frac)``, the products taken in float64.
    Over all rows exactly ``floor(n_rows * frac)`` extras are handed out (the sum telescopes).
    """
    ramp = np.floor(np.arange(n_rows + 1, dtype=np.float64) * np.float64(frac))
    return ramp[1:] > ramp[:-1]


# ---------------------------------------------------------------------------------------------------
# tiles  (veda_core.py, section "tiles": shapes, _padded, _count, least_padding_shape, span_tiles,
#         build_layout, gather, scatter_)
# ---------------------------------------------------------------------------------------------------

def tile_shapes():
    """All 36 power-of-two boxes ``(t, h, w)`` holding 128 rows, in lexicographic order."""
    found = []
    for a in range(8):
        for b in range(8 - a):
            found.append((1 << a, 1 << b, TILE >> (a + b)))
    found.sort()
    return found


def padded_grid(grid, shape):
    """Each grid axis rounded up to a multiple of the box edge on that axis."""
    return tuple(((g + s - 1) // s) * s for g, s in zip(grid, shape))


def tile_count(grid, shape):
    """Number of boxes (tiles) a grid is cut into by ``shape``."""
    tp, hp, wp = padded_grid(grid, shape)
    return (tp * hp * wp) // TILE


def least_padding_shape(grid):
    """The box that cuts ``grid`` into the fewest tiles (veda_core.py, least_padding_shape).

    Candidates are the boxes that fit inside the grid on every axis (all 36 if none fits). Ties on
    the tile count go to the most cubic box (smallest max/min edge ratio, a float), then to the
    lexicographically first.
    """
    every = tile_shapes()
    fitting = [s for s in every if s[0] <= grid[0] and s[1] <= grid[1] and s[2] <= grid[2]]
    pool_of = fitting if fitting else every
    best = None
    for s in pool_of:
        key = (tile_count(grid, s), max(s) / min(s), s)
        if best is None or key < best[0]:
            best = (key, s)
    return best[1]


def span_tiles(start, grid, shape):
    """``[n_tiles, 128]`` int64 packed row ids of one span, ``-1`` on padding (veda_core.py, span_tiles).

    The padded grid is cut into boxes; boxes are visited with the h-box index outermost, then the
    w-box, then the t-box innermost. Inside a box the cells are listed t, h, w row-major, and the
    real cells are moved (stably) in front of the padding cells, so a tile's real rows are a prefix.

    Written as a sort: every padded cell gets the key (box number, is-padding, offset in box).
    """
    T, H, W = grid
    st, sh, sw = shape
    tp, hp, wp = padded_grid(grid, shape)
    t, h, w = np.meshgrid(np.arange(tp), np.arange(hp), np.arange(wp), indexing="ij")
    t, h, w = t.ravel(), h.ravel(), w.ravel()
    n_tb, n_wb = tp // st, wp // sw
    box = ((h // sh) * n_wb + (w // sw)) * n_tb + (t // st)
    offset = ((t % st) * sh + (h % sh)) * sw + (w % sw)
    real = (t < T) & (h < H) & (w < W)
    row_id = np.where(real, start + (t * H + h) * W + w, -1)
    order = np.lexsort((offset, ~real, box))  # last key is the primary one
    return row_id[order].reshape(-1, TILE).astype(np.int64)


@dataclass
class Layout:
    """One permutation of the packed sequence into 128-row tiles (veda_core.py, build_layout)."""
    spans: list
    seq_len: int
    perm: np.ndarray          # [N] int64 packed row of each tile slot, -1 on padding
    valid_count: np.ndarray   # [n_tiles] real rows per tile (a prefix of the tile)
    n_video: int
    n_ref: int
    n_global: int
    ref_tokens: int
    target_tokens: int
    extras: dict = field(default_factory=dict)

    @property
    def n_tiles(self):
        return self.n_video + self.n_global

    @property
    def kv_ok(self):
        return self.valid_count > 0

    @property
    def slot_valid(self):
        return self.perm >= 0

    @property
    def widest(self):
        return int(self.kv_ok.sum())


def build_layout(spans, seq_len):
    """Tile every span in packed order (target last), then the uncovered ("global") rows.

    veda_core.py, build_layout: spans must come in ascending packed order without overlap and end
    inside the sequence; every row no span covers is global, and the global rows, ascending, are
    chunked into tiles after all span tiles (the last one padded with -1).
    """
    if not spans:
        raise VedaError("the target span must be tiled")
    covered = np.zeros(seq_len, dtype=bool)
    pieces = []
    end = 0
    norm = []
    for start, grid, shape in spans:
        grid = tuple(int(g) for g in grid)
        shape = tuple(int(s) for s in shape)
        rows = grid[0] * grid[1] * grid[2]
        if start < end or start + rows > seq_len:
            raise VedaError(f"span at {start} overlaps another or runs past {seq_len}")
        end = start + rows
        covered[start:end] = True
        pieces.append(span_tiles(start, grid, shape))
        norm.append((int(start), grid, shape))
    video = np.concatenate(pieces, axis=0)
    rest = np.flatnonzero(~covered)
    n_global = -(-rest.size // TILE)
    tail = np.full(n_global * TILE, -1, dtype=np.int64)
    tail[:rest.size] = rest
    perm = np.concatenate([video.ravel(), tail])
    valid = (perm.reshape(-1, TILE) >= 0).sum(axis=1).astype(np.int64)
    return Layout(
        spans=norm, seq_len=int(seq_len), perm=perm, valid_count=valid,
        n_video=int(video.shape[0]), n_ref=int(sum(p.shape[0] for p in pieces[:-1])),
        n_global=int(n_global),
        ref_tokens=int(sum(g[0] * g[1] * g[2] for _, g, _ in norm[:-1])),
        target_tokens=int(norm[-1][1][0] * norm[-1][1][1] * norm[-1][1][2]))


def gather(x, lay, heads):
    """``[S, H, D] -> [N, H', D]`` in tile order, padding slots zero (veda_core.py, gather)."""
    heads = np.asarray(heads)
    safe = np.where(lay.perm >= 0, lay.perm, 0)
    out = x[safe][:, heads, :].copy()
    out[lay.perm < 0] = 0
    return out


def scatter(out, tiled, lay, heads):
    """Tile-ordered rows back to their packed rows of ``out[S, H, D]`` (veda_core.py, scatter_).

    The page sends padding slots to a spare row ``S``; here they are simply dropped.
    """
    heads = np.asarray(heads)
    real = lay.perm >= 0
    rows = lay.perm[real]
    for j, hh in enumerate(heads):
        out[rows, hh, :] = tiled[real, j, :]
    return out


# ---------------------------------------------------------------------------------------------------
# predictor  (veda_core.py, section "predictor": pool, logits)
# ---------------------------------------------------------------------------------------------------

def pool(x_t, lay):
    """``[N, H', D]`` tile order -> ``[H', n_video, 3D]`` float64 features (veda_core.py, pool).

    For each video tile and head: the mean, the maximum and the minimum of the tile's real rows,
    concatenated as ``[mean | max | min]``; all zero for a tile without real rows. Global tiles are
    not pooled. (The page sums in fp32 and divides by the count; float64 here.)
    """
    nv = lay.n_video
    n_heads, dim = x_t.shape[1], x_t.shape[2]
    feats = np.zeros((n_heads, nv, 3 * dim), dtype=np.float64)
    for i in range(nv):
        c = int(lay.valid_count[i])
        if c == 0:
            continue
        rows = x_t[i * TILE:i * TILE + c].astype(np.float64)  # [c, H', D]
        feats[:, i, :dim] = rows.sum(axis=0) / c
        feats[:, i, dim:2 * dim] = rows.max(axis=0)
        feats[:, i, 2 * dim:] = rows.min(axis=0)
    return feats


def logits(fq, fk, pq, pk):
    """Tile-pair scores ``[H', n_q, n_k]`` (veda_core.py, logits).

    Each pooled feature row ``f`` (``3D`` wide) is projected per head, ``f @ P + f[:D]`` with
    ``P`` of shape ``[3D, D]`` (the mean part added back), and the scores are the dot products of
    projected query and key rows divided by ``sqrt(D)``. float64 here (the page uses fp32).
    """
    dim = pq.shape[-1]
    fq = np.asarray(fq, dtype=np.float64)
    fk = np.asarray(fk, dtype=np.float64)
    pq = np.asarray(pq, dtype=np.float64)
    pk = np.asarray(pk, dtype=np.float64)
    qh = np.matmul(fq, pq) + fq[..., :dim]
    kh = np.matmul(fk, pk) + fk[..., :dim]
    return np.matmul(qh, np.swapaxes(kh, 1, 2)) / math.sqrt(dim)


# ---------------------------------------------------------------------------------------------------
# selection  (veda_core.py, section "selection": column_blocks, select, block_mask, tile_index_list,
#             reference_attend)
# ---------------------------------------------------------------------------------------------------

def column_blocks(lay, generated, reference):
    """Key-column blocks ``[(start, stop, budget, real_tokens)]`` with a top-k of their own.

    veda_core.py, column_blocks: with tiled references the reference tiles ``[0, n_ref)`` form one
    block with the reference budget and the target tiles ``[n_ref, n_video)`` another with the
    generated budget; without references only the target block exists.
    """
    target = (lay.n_ref, lay.n_video, generated, lay.target_tokens)
    if lay.n_ref == 0:
        return [target]
    return [(0, lay.n_ref, reference, lay.ref_tokens), target]


def allowed_per_row(lay, block):
    """``[n_video]`` int64: how many key tiles each video query row may keep in ``block``.

    ``k_lo + extra[r]`` where the extras follow the Bresenham pattern over *all* video rows (the
    page builds it with ``n_rows = n_video``). A keeps-all block allows every column.
    """
    start, stop, budget, real = block
    n = stop - start
    if keeps_all(budget):
        return np.full(lay.n_video, n, dtype=np.int64)
    lo, _hi, frac = split_budget(row_budget(budget, real, n), n)
    return lo + extra_tile_rows(lay.n_video, frac).astype(np.int64)


def select(scores, lay, blocks):
    """Kept video key tiles, ``[H', n_video, n_video]`` bool (veda_core.py, select).

    Per head, video query row and column block: empty key tiles score -inf; the row's own tile
    scores +inf when it lies in the block; the columns are ranked by (score descending, column
    ascending) and the first ``allowed`` of them are kept unless their score is -inf. A keeps-all
    block keeps every non-empty column.

    Readings (the page is silent): equal scores are broken by the lower column index; a NaN score
    ranks as -inf and is never kept.
    """
    scores = np.asarray(scores, dtype=np.float32)
    n_heads, nv = scores.shape[0], lay.n_video
    kv_ok = lay.kv_ok
    kept = np.zeros((n_heads, nv, nv), dtype=bool)
    rows = np.arange(nv)
    for block in blocks:
        start, stop, budget, _ = block
        n = stop - start
        if keeps_all(budget):
            kept[:, :, start:stop] = kv_ok[None, None, start:stop]
            continue
        allowed = allowed_per_row(lay, block)
        s = scores[:, :, start:stop].astype(np.float64)
        s = np.where(np.isnan(s), -np.inf, s)
        s[:, :, ~kv_ok[start:stop]] = -np.inf
        mine = (rows >= start) & (rows < stop)
        s[:, rows[mine], rows[mine] - start] = np.inf
        order = np.argsort(-s, axis=-1, kind="stable")  # stable: equal scores keep column order
        rank = np.argsort(order, axis=-1)               # position of each column in that order
        keep = (rank < allowed[None, :, None]) & (s > -np.inf)
        kept[:, :, start:stop] = keep
    return kept


def block_mask(kept_video, lay):
    """``[H', n_tiles, n_tiles]`` bool tile mask, rows are query tiles (veda_core.py, block_mask).

    Video rows keep their selected video tiles plus every non-empty global tile; global rows are
    dense over every non-empty tile.
    """
    n_heads, nv, n = kept_video.shape[0], lay.n_video, lay.n_tiles
    mask = np.zeros((n_heads, n, n), dtype=bool)
    mask[:, :nv, :nv] = kept_video
    mask[:, :nv, nv:] = lay.kv_ok[None, None, nv:]
    mask[:, nv:, :] = lay.kv_ok[None, None, :]
    return mask


def tile_index_list(mask):
    """Per-row ascending kept tile ids and their count (veda_core.py, tile_index_list).

    Returns ``(index [H', n, width] int64, count [H', n] int64)``, ``width`` the widest row; entries
    past a row's count are -1 here (the page leaves them unspecified and never reads them).
    """
    count = mask.sum(axis=-1)
    width = int(count.max()) if count.size else 0
    index = np.full(mask.shape[:-1] + (width,), -1, dtype=np.int64)
    for h in range(mask.shape[0]):
        for r in range(mask.shape[1]):
            cols = np.flatnonzero(mask[h, r])
            index[h, r, :cols.size] = cols
    return index, count


def attend_tiles(q_t, k_t, v_t, lay, kept_lists, q_tiles=None, scale=None):
    """Exact block-sparse attention, float64, on tile-ordered ``[N, H', D]`` (veda_core.py,
    reference_attend).

    Query tile ``i`` of head ``h`` attends the key slots of the tiles in ``kept_lists(h, i)`` that
    hold a real row (``slot_valid``); scores are scaled by ``D**-0.5`` and soft-maxed; a row that sees
    no key gives 0 and padding query slots give 0. ``q_tiles`` restricts the work to some query tiles
    (other rows are returned as NaN). Returns float64 ``[N, H', D]``.
    """
    n_heads, dim = q_t.shape[1], q_t.shape[2]
    scale = dim ** -0.5 if scale is None else scale
    out = np.full(q_t.shape, np.nan, dtype=np.float64)
    valid = lay.slot_valid
    tiles = range(lay.n_tiles) if q_tiles is None else q_tiles
    for i in tiles:
        qs = slice(i * TILE, (i + 1) * TILE)
        for h in range(n_heads):
            cols = np.asarray(kept_lists(h, i), dtype=np.int64)
            slots = (cols[:, None] * TILE + np.arange(TILE)[None, :]).ravel() if cols.size else np.zeros(0, np.int64)
            slots = slots[valid[slots]] if slots.size else slots
            q = q_t[qs, h, :].astype(np.float64)
            res = np.zeros((TILE, dim), dtype=np.float64)
            if slots.size:
                k = k_t[slots, h, :].astype(np.float64)
                v = v_t[slots, h, :].astype(np.float64)
                z = (q @ k.T) * scale
                z = z - z.max(axis=1, keepdims=True)
                p = np.exp(z)
                res = (p @ v) / p.sum(axis=1, keepdims=True)
            res[~valid[qs]] = 0.0
            out[qs, h, :] = res
    return out


def attend_dense_mask(q_t, k_t, v_t, mask, lay):
    """The same attention from an explicit ``[H', n_tiles, n_tiles]`` tile mask, token by token.

    Builds the token-level mask (tile mask expanded to 128x128 blocks, restricted to real key slots)
    and runs a masked softmax; fully masked rows and padding rows give 0. O(N^2): tiny inputs only.
    """
    n_heads, dim = q_t.shape[1], q_t.shape[2]
    allowed = np.repeat(np.repeat(mask, TILE, axis=1), TILE, axis=2) & lay.slot_valid[None, None, :]
    q = q_t.astype(np.float64)
    k = k_t.astype(np.float64)
    v = v_t.astype(np.float64)
    z = np.einsum("qhd,khd->hqk", q, k) * dim ** -0.5
    z = np.where(allowed, z, -np.inf)
    zmax = z.max(axis=-1, keepdims=True)
    zmax = np.where(np.isfinite(zmax), zmax, 0.0)
    p = np.where(allowed, np.exp(z - zmax), 0.0)
    denom = p.sum(axis=-1, keepdims=True)
    p = np.divide(p, denom, out=np.zeros_like(p), where=denom > 0)
    out = np.einsum("hqk,khd->qhd", p, v)
    return out * lay.slot_valid[:, None, None]


def dense_attention(q, k, v):
    """Textbook softmax attention, float64, on ``[S, H, D]`` (what a keeps-all budget must equal)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    z = np.einsum("qhd,khd->hqk", q, k) / math.sqrt(q.shape[-1])
    z = z - z.max(axis=-1, keepdims=True)
    p = np.exp(z)
    p /= p.sum(axis=-1, keepdims=True)
    return np.einsum("hqk,khd->qhd", p, v)


# ---------------------------------------------------------------------------------------------------
# FP8 Q/K variant (not on the pages; the quantiser is defined by the reading written below)
# ---------------------------------------------------------------------------------------------------

E4M3_MAX = 448.0


def _round_e4m3(x):
    """Round float64 values to the nearest float8 e4m3fn value (ties to even, saturating at 448).

    e4m3fn: 1 sign, 4 exponent bits (bias 7), 3 mantissa bits, no infinities; normal numbers
    2**-6 .. 448, subnormals multiples of 2**-9.
    """
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), E4M3_MAX)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -6.0)                      # subnormal range shares the 2**-6 exponent
    quantum = np.exp2(e - 3.0)                   # spacing of representable values at that exponent
    r = np.round(a / quantum) * quantum          # numpy rounds half to even
    r = np.minimum(r, E4M3_MAX)
    return np.sign(x) * r


def quantize_fp8_tiles(x_t, lay):
    """Per (head, 128-row tile) e4m3 quantisation of tile-ordered ``[N, H', D]`` values.

    Not on the pages (their kernel quantises to INT8 by a recipe they do not print). Reading adopted:
    the scale of a tile is ``amax(|x|) over its real rows / 448`` (1.0 when that is 0); the stored
    value is ``x / scale`` rounded to nearest-even e4m3 with saturation. Returns
    ``(codes as float64 [N, H', D], scales [H', n_tiles] float64)``; the dequantised value is
    ``code * scale``. Pinned by the e4m3 rounding rule, the scale definition and exact-on-grid attention;
    that the pages' kernel used this recipe is unpinned (they do not print one).
    """
    n = lay.n_tiles
    n_heads = x_t.shape[1]
    scales = np.ones((n_heads, n), dtype=np.float64)
    codes = np.zeros(x_t.shape, dtype=np.float64)
    for i in range(n):
        c = int(lay.valid_count[i])
        blk = x_t[i * TILE:(i + 1) * TILE].astype(np.float64)
        for h in range(n_heads):
            amax = np.abs(blk[:c, h, :]).max() if c else 0.0
            s = amax / E4M3_MAX if amax > 0 else 1.0
            s = float(np.float32(s))  # the scale is stored as fp32
            scales[h, i] = s
            codes[i * TILE:(i + 1) * TILE, h, :] = _round_e4m3(blk[:, h, :] / s)
    return codes, scales


def attend_tiles_fp8(q_t, k_t, v_t, lay, kept_lists, q_tiles=None):
    """Attention with Q and K replaced by their per-tile e4m3 quantisation (dequantised exactly).

    The scores are ``(code_q * s_q) . (code_k * s_k) * D**-0.5``; V stays as given.
    """
    cq, sq = quantize_fp8_tiles(q_t, lay)
    ck, sk = quantize_fp8_tiles(k_t, lay)
    tile_of = np.arange(q_t.shape[0]) // TILE
    qd = cq * sq.T[tile_of][:, :, None]
    kd = ck * sk.T[tile_of][:, :, None]
    return attend_tiles(qd, kd, v_t, lay, kept_lists, q_tiles=q_tiles)


# ---------------------------------------------------------------------------------------------------
# INT8 Q/K variant. The pages' own kernel computes Q K^T in INT8 (a SageAttention-derived Triton
# kernel) but does not print its quantisation recipe; the reading here is the plainest symmetric one, the
# FP8 reading's twin: per (head, 128-row tile) scale amax(|x| over real rows) / 127 (1.0 when 0), kept
# as fp32; codes are x / scale rounded to the nearest integer, ties to even, saturating at +-127.
# ---------------------------------------------------------------------------------------------------

I8_MAX = 127.0


def _round_int8(x):
    """Round float64 values to the nearest integer (ties to even), saturating at +-127."""
    return np.clip(np.round(np.asarray(x, dtype=np.float64)), -I8_MAX, I8_MAX)  # numpy rounds half to even


def quantize_int8_tiles(x_t, lay):
    """Per (head, 128-row tile) INT8 quantisation of tile-ordered ``[N, H', D]`` values.

    Returns ``(codes as float64 integers [N, H', D], scales [H', n_tiles] float64)``; the dequantised
    value is ``code * scale``. Padding rows are zero and stay zero.
    """
    n = lay.n_tiles
    n_heads = x_t.shape[1]
    scales = np.ones((n_heads, n), dtype=np.float64)
    codes = np.zeros(x_t.shape, dtype=np.float64)
    for i in range(n):
        c = int(lay.valid_count[i])
        blk = x_t[i * TILE:(i + 1) * TILE].astype(np.float64)
        for h in range(n_heads):
            amax = np.abs(blk[:c, h, :]).max() if c else 0.0
            s = amax / I8_MAX if amax > 0 else 1.0
            s = float(np.float32(s))  # the scale is stored as fp32
            scales[h, i] = s
            codes[i * TILE:(i + 1) * TILE, h, :] = _round_int8(blk[:, h, :] / s)
    return codes, scales


def attend_tiles_int8(q_t, k_t, v_t, lay, kept_lists, q_tiles=None):
    """Attention with Q and K replaced by their per-tile INT8 quantisation (dequantised exactly).

    The scores are ``(code_q * s_q) . (code_k * s_k) * D**-0.5``, that is the integer dot product of
    the codes times ``s_q * s_k * D**-0.5``; V stays as given.
    """
    cq, sq = quantize_int8_tiles(q_t, lay)
    ck, sk = quantize_int8_tiles(k_t, lay)
    tile_of = np.arange(q_t.shape[0]) // TILE
    qd = cq * sq.T[tile_of][:, :, None]
    kd = ck * sk.T[tile_of][:, :, None]
    return attend_tiles(qd, kd, v_t, lay, kept_lists, q_tiles=q_tiles)


# ---------------------------------------------------------------------------------------------------
# one layer  (veda_core.py, section "one layer": attention and its stats)
# ---------------------------------------------------------------------------------------------------

# ---------------------------------------------------------------------------------------------------
# packed layouts  (veda_core.py, section "what the packed layout holds": _grid_of, describe_layout)
# ---------------------------------------------------------------------------------------------------

def grid_of(position_ids, a, b):
    """``(T, H, W)`` when rows ``a:b`` hold a row-major T x H x W grid of positions, else ``None``.

    veda_core.py, _grid_of: the distinct values of each of the three position columns give the axes;
    their sizes must multiply to the row count, and the rows must list the axes' Cartesian product in
    row-major order (t slowest, w fastest), each axis ascending.
    """
    pos = np.asarray(position_ids)[a:b]
    axes = [np.unique(pos[:, i]) for i in range(3)]
    t, h, w = (x.size for x in axes)
    if t * h * w != b - a:
        return None
    want = np.stack(np.meshgrid(*axes, indexing="ij"), axis=-1).reshape(-1, 3)
    return (t, h, w) if np.array_equal(want, pos.astype(want.dtype)) else None


def describe_packed_layout(segments, latent, seq_len, position_ids=None):
    """The spans a model's packed sequence holds (veda_core.py, describe_layout).

    ``segments`` are ``(start, stop, kind)`` row ranges; ``latent`` is the latent grid ``(lt, lh, lw)``
    of the generated video. There must be exactly one ``"video"`` segment, and it must hold
    ``lt * (lh // 2) * (lw // 2)`` rows (the target grid is ``(lt, lh // 2, lw // 2)``: two-by-two spatial
    patches). Each ``"cond"`` or ``"ref_img"`` segment becomes a reference span when its rows are a
    verified row-major grid (``grid_of`` on the position ids), and stays global otherwise (always
    correct); other kinds stay global. Returns ``(seq_len, (target start, target grid), ((ref start,
    grid), ...), (skipped notes, ...))``.
    """
    video = [(a, b) for a, b, kind in segments if kind == "video"]
    if len(video) != 1:
        raise VedaError(f"expected one target video segment, found {len(video)}")
    lt, lh, lw = (int(x) for x in latent)
    grid = (lt, lh // 2, lw // 2)
    if grid[0] * grid[1] * grid[2] != video[0][1] - video[0][0]:
        raise VedaError(f"the video segment does not match the latent grid {grid}")
    refs, skipped = [], []
    for a, b, kind in segments:
        if kind in ("cond", "ref_img"):
            g = None if position_ids is None else grid_of(position_ids, a, b)
            if g:
                refs.append((a, g))
            else:
                skipped.append(f"{kind}[{a}:{b}]")
    return int(seq_len), (video[0][0], grid), tuple(refs), tuple(skipped)


def layer_spans(ref_spans, target, tile_refs):
    """Spans of one head group: references at their least-padding box (when tiled), target last."""
    spans = [(s, g, least_padding_shape(g)) for s, g in ref_spans] if tile_refs else []
    return spans + [target]


def attention_layer(q, k, v, seq_len, ref_spans, target_start, target_grid, head_shapes, budgets,
                    proj_q, proj_k, q_tiles_sample=None):
    """One Veda layer on ``[S, H, D]`` inputs, float64 output ``[S, H, D]`` (veda_core.py, attention).

    ``head_shapes[h]`` is the target box of head ``h``; heads sharing a box share one layout and one
    pass. References are tiled at their least-padding box unless the reference budget keeps all
    (then their rows are global). Returns ``(out, info)`` where ``info`` holds per group the layout,
    the kept mask and the index lists, plus the page's work counters.
    """
    generated, reference = budgets
    tile_refs = not keeps_all(reference)
    S, H, D = q.shape
    out = np.zeros((S, H, D), dtype=np.float64)
    groups = {}
    for h, shp in enumerate(head_shapes):
        groups.setdefault(tuple(shp), []).append(h)
    info = {"groups": [], "kept": 0, "work": 0, "dense": 0.0}
    for shape in sorted(groups):
        heads = np.array(groups[shape], dtype=np.int64)
        lay = build_layout(layer_spans(ref_spans, (target_start, tuple(target_grid), shape), tile_refs),
                           seq_len)
        blocks = column_blocks(lay, generated, reference)
        q_t, k_t, v_t = gather(q, lay, heads), gather(k, lay, heads), gather(v, lay, heads)
        scores = logits(pool(q_t, lay), pool(k_t, lay), proj_q[heads], proj_k[heads])
        kept = select(scores.astype(np.float32), lay, blocks)
        mask = block_mask(kept, lay)
        o_t = attend_tiles(q_t, k_t, v_t, lay, lambda hh, i: np.flatnonzero(mask[hh, i]),
                           q_tiles=q_tiles_sample)
        o_t = np.nan_to_num(o_t, nan=0.0)
        scatter(out, o_t, lay, heads)
        n_kept = int(kept.sum())
        info["kept"] += n_kept
        info["work"] += n_kept + len(heads) * lay.n_global * (lay.n_tiles + lay.n_video)
        info["dense"] += len(heads) * (seq_len / TILE) ** 2
        info["groups"].append({"shape": shape, "heads": heads, "layout": lay, "scores": scores,
                               "kept": kept, "mask": mask})
    return out, info


def work_stats(lay, n_heads, n_kept):
    """The page's work counters for one head group (veda_core.py, attention stats):
    ``work = kept + H' * n_global * (n_tiles + n_video)`` and ``dense = H' * (S / 128)**2``."""
    work = n_kept + n_heads * lay.n_global * (lay.n_tiles + lay.n_video)
    dense = n_heads * (lay.seq_len / TILE) ** 2
    return work, dense
