"""Pins of the CPU oracle to facts fixed outside itself (brute force, closed forms, invariants, library
routines and the pages' printed values). CPU only; every test runs in seconds."""
import itertools
import math
import os

import numpy as np
import pytest
import torch

import oracle as O
import veda_synth as V

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------------------------------------ tile boxes

def test_tile_shapes_enumeration():
    # brute force: every triple of powers of two in [1, 128] whose product is 128
    pw = [1 << i for i in range(8)]
    brute = sorted(s for s in itertools.product(pw, pw, pw) if s[0] * s[1] * s[2] == 128)
    got = O.tile_shapes()
    assert got == brute
    assert len(got) == 36 and got[0] == (1, 1, 128) and got[-1] == (128, 1, 1)


def _brute_lps(grid):
    cands = [s for s in O.tile_shapes() if all(a <= b for a, b in zip(s, grid))] or O.tile_shapes()
    best = None
    for s in cands:
        n = 1
        for g, e in zip(grid, s):
            n *= math.ceil(g / e)
        key = (n, max(s) / min(s), s)
        best = key if best is None or key < best else best
    return best[2], best[0]


@pytest.mark.parametrize("grid", [(26, 48, 84), (1, 48, 84), (61, 45, 80), (8, 16, 16), (3, 10, 12),
                                  (1, 1, 1), (200, 1, 1), (5, 12, 40), (2, 16, 16), (6, 16, 24)])
def test_least_padding_shape_bruteforce(grid):
    shape, n = _brute_lps(grid)
    assert O.least_padding_shape(grid) == shape
    assert O.tile_count(grid, shape) == n


def test_least_padding_closed_forms():
    # (26,48,84) holds 819*128 rows exactly; the only zero-padding box is (2,16,4) (t | 26, h | 48, w | 84)
    assert 26 * 48 * 84 == 819 * 128
    zero_pad = [s for s in O.tile_shapes() if 26 % s[0] == 0 and 48 % s[1] == 0 and 84 % s[2] == 0]
    assert zero_pad == [(2, 16, 4)]
    assert O.least_padding_shape((26, 48, 84)) == (2, 16, 4)
    # (61,45,80): (8,1,16) and (16,1,8) tie on count (1800) and on aspect (16): lexicographic first wins
    assert O.tile_count((61, 45, 80), (8, 1, 16)) == O.tile_count((61, 45, 80), (16, 1, 8)) == 1800
    assert O.least_padding_shape((61, 45, 80)) == (8, 1, 16)
    assert O.least_padding_shape((1, 48, 84)) == (1, 16, 8) and O.tile_count((1, 48, 84), (1, 16, 8)) == 33


def _brute_span_tiles(start, grid, shape):
    """The page's words, as loops: boxes with h outermost, then w, then t; cells t,h,w row-major in a
    box; real cells first (stable)."""
    T, H, W = grid
    st, sh, sw = shape
    nt, nh, nw = -(-T // st), -(-H // sh), -(-W // sw)
    tiles = []
    for bh in range(nh):
        for bw in range(nw):
            for bt in range(nt):
                cells = []
                for dt in range(st):
                    for dh in range(sh):
                        for dw in range(sw):
                            t, h, w = bt * st + dt, bh * sh + dh, bw * sw + dw
                            cells.append(start + (t * H + h) * W + w if (t < T and h < H and w < W) else -1)
                tiles.append([c for c in cells if c >= 0] + [c for c in cells if c < 0])
    return np.array(tiles, dtype=np.int64)


@pytest.mark.parametrize("grid,shape", [((3, 10, 12), (2, 8, 8)), ((8, 16, 16), (2, 8, 8)), ((2, 3, 5), (4, 4, 8)),
                                        ((5, 7, 9), (1, 8, 16)), ((4, 4, 8), (8, 4, 4)), ((9, 2, 20), (2, 2, 32))])
def test_span_tiles_bruteforce(grid, shape):
    got = O.span_tiles(17, grid, shape)
    want = _brute_span_tiles(17, grid, shape)
    assert np.array_equal(got, want)
    real = got[got >= 0]
    assert sorted(real.tolist()) == list(range(17, 17 + grid[0] * grid[1] * grid[2]))  # bijection
    for row in got:  # real rows form a prefix
        k = int((row >= 0).sum())
        assert (row[:k] >= 0).all() and (row[k:] < 0).all()


def test_every_span_tile_is_nonempty():
    # the last box on each axis starts inside the grid, so no span tile is all padding
    for grid in [(3, 10, 12), (61, 45, 80), (1, 48, 84), (5, 7, 9)]:
        for shape in O.tile_shapes():
            t = O.span_tiles(0, grid, shape)
            assert ((t >= 0).sum(1) > 0).all()


# ------------------------------------------------------------------------------------------ layouts

def test_build_layout_errors():
    with pytest.raises(O.VedaError):
        O.build_layout([], 10)
    with pytest.raises(O.VedaError):  # overlap
        O.build_layout([(0, (1, 8, 16), (1, 8, 16)), (100, (1, 8, 16), (1, 8, 16))], 400)
    with pytest.raises(O.VedaError):  # runs past the sequence
        O.build_layout([(10, (1, 8, 16), (1, 8, 16))], 100)
    with pytest.raises(O.VedaError):  # not in packed order
        O.build_layout([(200, (1, 8, 16), (1, 8, 16)), (0, (1, 8, 16), (1, 8, 16))], 400)


def test_build_layout_global_rows_and_roundtrip():
    lay = O.build_layout([(150, (2, 16, 16), (1, 16, 8)), (662, (6, 16, 24), (8, 4, 4))], 2966 + 40)
    # uncovered rows: [0,150) and [2966, 3006), ascending, in tiles after the span tiles
    glob = lay.perm[lay.n_video * 128:]
    real = glob[glob >= 0]
    assert real.tolist() == list(range(150)) + list(range(2966, 3006))
    assert lay.n_global == -(-190 // 128)
    assert lay.n_ref == O.tile_count((2, 16, 16), (1, 16, 8))
    perm = lay.perm[lay.perm >= 0]
    assert sorted(perm.tolist()) == list(range(3006))
    x = np.random.default_rng(0).standard_normal((3006, 3, 8)).astype(np.float32)
    xt = O.gather(x, lay, [2, 0])
    assert (xt[lay.perm < 0] == 0).all()
    back = np.zeros_like(x)
    O.scatter(back, xt, lay, [2, 0])
    assert np.array_equal(back[:, [2, 0]], x[:, [2, 0]])


# ------------------------------------------------------------------------------------------ budgets

def test_budget_both_or_neither():
    with pytest.raises(O.VedaError):
        O.keeps_all((0.5, 3))
    with pytest.raises(O.VedaError):
        O.row_budget((None, None), 1000, 8)


def test_node_budget_golden():
    rows = [ln.split() for ln in open(os.path.join(GOLDEN, "node_budget.txt")) if ln.strip() and ln[0] != "#"]
    for r in rows:
        if r[0] == "sparsity":
            b = O.sparsity_budget(float(r[1]))
            assert abs(b[0] - float(r[3])) < 1e-12 and b[1] is None
        else:
            b = O.tiles_budget(int(r[1]))
            assert b == (None, int(r[3]))
        assert O.keeps_all(b) == (r[5] == "yes")


def test_split_closed_forms():
    # whole block when the budget reaches the width
    assert O.split_budget(819.0, 819) == (819, 819, 0.0)
    assert O.split_budget(1e9, 5) == (5, 5, 0.0)
    # below one tile: at least one tile, no fractional extra
    assert O.split_budget(0.3, 100) == (1, 2, 0.0)
    assert O.split_budget(0.3, 1) == (1, 1, 0.0)
    # integers keep exactly that many
    assert O.split_budget(O.row_budget(O.tiles_budget(24), 104832, 819), 819) == (24, 25, 0.0)
    # ratio 0.1 on the 819-tile grid without padding: 81.9 per row
    assert O.split_budget(O.row_budget(O.ratio_budget(0.1), 104832, 819), 819) == (81, 82, 0.9)
    # a padded tiling never gets a larger budget: the ideal count, not the padded one, is squared
    b_pad = O.row_budget(O.ratio_budget(0.05), 219600, 1800)
    assert b_pad < 0.05 * 1800 and abs(b_pad - 0.05 * 1716 ** 2 / 1800) < 1e-9


@pytest.mark.parametrize("n,frac", [(819, 0.9), (1800, 0.796), (33, 0.10303030303), (7, 0.5), (100, 0.0), (5, 1.0)])
def test_bresenham_pattern(n, frac):
    got = O.extra_tile_rows(n, frac)
    brute = [math.floor((r + 1) * frac) > math.floor(r * frac) for r in range(n)]
    assert got.tolist() == brute
    assert int(got.sum()) == math.floor(n * frac)  # the sum telescopes
    idx = np.flatnonzero(got)
    if idx.size > 2 and frac > 0:  # extras are evenly spread: gaps differ by at most one row
        gaps = np.diff(idx)
        assert gaps.max() - gaps.min() <= 1


def test_per_row_total_config_single():
    lay = O.build_layout([(0, (26, 48, 84), (2, 16, 4))], 104832)
    blk = O.column_blocks(lay, O.ratio_budget(0.1), O.ratio_budget(1.0))
    allowed = O.allowed_per_row(lay, blk[0])
    assert int(allowed.sum()) == 81 * 819 + math.floor(819 * 0.9) == 67076


# ------------------------------------------------------------------------------------------ selection

def _brute_select(scores, lay, blocks):
    H, nv = scores.shape[0], lay.n_video
    kept = np.zeros((H, nv, nv), dtype=bool)
    for (start, stop, budget, real) in blocks:
        n = stop - start
        if O.keeps_all(budget):
            kept[:, :, start:stop] = lay.kv_ok[start:stop]
            continue
        lo, hi, frac = O.split_budget(O.row_budget(budget, real, n), n)
        for h in range(H):
            for r in range(nv):
                allow = lo + (math.floor((r + 1) * frac) > math.floor(r * frac))
                cand = []
                for c in range(start, stop):
                    v = float(scores[h, r, c])
                    if math.isnan(v) or not lay.kv_ok[c]:
                        v = -math.inf
                    if c == r:
                        v = math.inf
                    cand.append((-v, c, v))
                cand.sort()
                for _, c, v in cand[:allow]:
                    if v > -math.inf:
                        kept[h, r, c] = True
    return kept


def _small_layout():
    return O.build_layout([(30, (2, 16, 16), (1, 16, 8)), (30 + 512, (3, 10, 12), (2, 8, 8))], 30 + 512 + 360 + 9)


@pytest.mark.parametrize("gen,ref", [((0.4, None), (0.3, None)), ((None, 3), (None, 1)), ((1.0, None), (0.5, None)),
                                     ((0.05, None), (None, 100))])
def test_select_bruteforce(gen, ref):
    lay = _small_layout()
    nv = lay.n_video
    rng = np.random.default_rng(1)
    scores = rng.standard_normal((2, nv, nv)).astype(np.float32)
    scores[0, 3, :] = np.round(scores[0, 3, :])  # many ties
    scores[1, 5, 2] = np.nan
    blocks = O.column_blocks(lay, gen, ref)
    got = O.select(scores, lay, blocks)
    assert np.array_equal(got, _brute_select(scores, lay, blocks))


def test_select_invariants():
    lay = _small_layout()
    nv = lay.n_video
    rng = np.random.default_rng(2)
    scores = rng.integers(-40, 40, size=(2, nv, nv)).astype(np.float32)  # integer valued: exact shifts
    blocks = O.column_blocks(lay, (0.4, None), (0.3, None))
    kept = O.select(scores, lay, blocks)
    # own tile always kept
    assert kept[:, np.arange(nv), np.arange(nv)].all()
    # per block per row: exactly k_lo + extra kept (every tile is non-empty here)
    for blk in blocks:
        s0, s1 = blk[0], blk[1]
        assert np.array_equal(kept[:, :, s0:s1].sum(-1), np.broadcast_to(O.allowed_per_row(lay, blk), (2, nv)))
    # invariant to adding a constant per row
    shift = rng.integers(-1000, 1000, size=(2, nv, 1)).astype(np.float32)
    assert np.array_equal(O.select(scores + shift, lay, blocks), kept)


def test_select_ties_go_to_lower_column():
    lay = O.build_layout([(0, (1, 8, 16 * 8), (1, 8, 16))], 1024)  # 8 tiles
    scores = np.zeros((1, 8, 8), dtype=np.float32)
    kept = O.select(scores, lay, O.column_blocks(lay, (None, 3), (1.0, None)))
    for r in range(8):
        want = {r} | set([c for c in range(8) if c != r][:2])
        assert set(np.flatnonzero(kept[0, r]).tolist()) == want


def test_select_signed_zeros_are_one_score():
    # IEEE comparison has -0.0 == +0.0: the two are the same score, so they tie and the lower column wins
    # whichever of them carries the sign bit (torch's topk on the page compares the same way)
    lay = O.build_layout([(0, (1, 8, 64), (1, 8, 16))], 512)  # 4 tiles
    z, nz = 0.0, -0.0
    s = np.array([[[5.0, nz, z, -1.0],    # own tile 0; tie of -0 (col 1) and +0 (col 2): col 1
                   [z, 3.0, nz, -1.0],    # own tile 1; tie of +0 (col 0) and -0 (col 2): col 0
                   [-1.0, nz, 9.0, z],    # own tile 2; tie of -0 (col 1) and +0 (col 3): col 1
                   [z, nz, -1.0, 2.0]]],  # own tile 3; tie of +0 (col 0) and -0 (col 1): col 0
                 dtype=np.float32)
    assert np.signbit(s[0, 0, 1]) and not np.signbit(s[0, 0, 2])
    kept = O.select(s, lay, O.column_blocks(lay, (None, 2), (1.0, None)))
    want = [{0, 1}, {0, 1}, {1, 2}, {0, 3}]
    for r in range(4):
        assert set(np.flatnonzero(kept[0, r]).tolist()) == want[r], r


def test_column_blocks_closed_form_with_unequal_budgets():
    # text rows, then a reference grid (2,16,16) = 512 rows cut at (2,8,8) into 4 tiles, then a target grid
    # (6,16,24) = 2304 rows cut at (2,8,8) into 3*2*3 = 18 tiles; reference budget 0.5, generated 0.3.
    # Everything below is worked out by hand from the page's _per_row / _split / _bresenham.
    assert O.least_padding_shape((2, 16, 16)) == (2, 8, 8)
    spans = [(150, (2, 16, 16), (2, 8, 8)), (662, (6, 16, 24), (2, 8, 8))]
    lay = O.build_layout(spans, 150 + 512 + 2304)
    assert (lay.n_ref, lay.n_video, lay.ref_tokens, lay.target_tokens) == (4, 22, 512, 2304)
    gen, ref = (0.3, None), (0.5, None)
    blocks = O.column_blocks(lay, gen, ref)
    assert blocks == [(0, 4, ref, 512), (4, 22, gen, 2304)]
    # reference block: ideal = 512/128 = 4 tiles, ((0.5 * 4) * 4) / 4 = 2.0 -> (k_lo, k_hi, frac) = (2, 3, 0):
    # every one of the 22 video rows keeps 2 reference tiles
    ref_want = np.full(22, 2)
    assert np.array_equal(O.allowed_per_row(lay, blocks[0]), ref_want)
    # target block: ideal = 18, ((0.3 * 18) * 18) / 18 is 5.4 to within an ulp -> (5, 6, 0.4); row r gets the
    # extra tile when floor(0.4 (r + 1)) > floor(0.4 r): rows 2, 4, 7, 9, 12, 14, 17, 19 (floor(22 * 0.4) = 8)
    extra = {2, 4, 7, 9, 12, 14, 17, 19}
    gen_want = np.array([5 + (r in extra) for r in range(22)])
    assert gen_want.sum() == 5 * 22 + 8
    assert np.array_equal(O.allowed_per_row(lay, blocks[1]), gen_want)
    # the selection keeps exactly those counts per block (every tile holds real rows), and the own tile of
    # each row in the block that holds it
    rng = np.random.default_rng(4)
    scores = rng.standard_normal((2, 22, 22)).astype(np.float32)
    kept = O.select(scores, lay, blocks)
    assert np.array_equal(kept[:, :, :4].sum(-1), np.broadcast_to(ref_want, (2, 22)))
    assert np.array_equal(kept[:, :, 4:].sum(-1), np.broadcast_to(gen_want, (2, 22)))
    assert kept[:, np.arange(22), np.arange(22)].all()


def test_block_mask_and_index_list():
    lay = _small_layout()
    nv, n = lay.n_video, lay.n_tiles
    rng = np.random.default_rng(3)
    kept = O.select(rng.standard_normal((2, nv, nv)).astype(np.float32), lay,
                    O.column_blocks(lay, (0.4, None), (0.3, None)))
    mask = O.block_mask(kept, lay)
    assert mask[:, nv:, :].all()             # global rows are dense (all tiles non-empty here)
    assert mask[:, :nv, nv:].all()           # video rows see every global tile
    idx, cnt = O.tile_index_list(mask)
    for h in range(2):
        for r in range(n):
            cols = idx[h, r, :cnt[h, r]]
            assert (np.diff(cols) > 0).all() and set(cols.tolist()) == set(np.flatnonzero(mask[h, r]).tolist())


# ------------------------------------------------------------------------------------------ pooling, logits

def test_pool_bruteforce():
    lay = O.build_layout([(5, (3, 10, 12), (2, 8, 8))], 5 + 360 + 3)
    rng = np.random.default_rng(4)
    x = rng.standard_normal((lay.seq_len, 2, 4)).astype(np.float32)
    xt = O.gather(x, lay, [1, 0])
    f = O.pool(xt, lay)
    for i in range(lay.n_video):
        rows = [p for p in lay.perm[i * 128:(i + 1) * 128] if p >= 0]
        for j, hh in enumerate([1, 0]):
            for d in range(4):
                vals = [float(x[p, hh, d]) for p in rows]
                assert f[j, i, 4 + d] == max(vals) and f[j, i, 8 + d] == min(vals)
                assert abs(f[j, i, d] - math.fsum(vals) / len(vals)) <= 1e-12


def test_logits_special_cases():
    rng = np.random.default_rng(5)
    H, nq, D = 2, 5, 4
    fq = rng.standard_normal((H, nq, 3 * D))
    fk = rng.standard_normal((H, nq + 2, 3 * D))
    zero = np.zeros((H, 3 * D, D))
    # no projection: the mean parts' dot products over sqrt(D)
    s = O.logits(fq, fk, zero, zero)
    assert np.allclose(s, np.einsum("hqd,hkd->hqk", fq[..., :D], fk[..., :D]) / 2.0)
    # projection picking the max part: q_hat = mean + max
    pick = np.zeros((H, 3 * D, D))
    pick[:, D:2 * D, :] = np.eye(D)
    s = O.logits(fq, fk, pick, zero)
    assert np.allclose(s, np.einsum("hqd,hkd->hqk", fq[..., :D] + fq[..., D:2 * D], fk[..., :D]) / 2.0)
    # heads are independent: swapping heads swaps outputs
    pq = rng.standard_normal((H, 3 * D, D))
    s1 = O.logits(fq, fk, pq, pq)
    s2 = O.logits(fq[::-1], fk[::-1], pq[::-1], pq[::-1])
    assert np.allclose(s1[::-1], s2)


# ------------------------------------------------------------------------------------------ attention

def _qkv(S, H, D, seed):
    rng = np.random.default_rng(seed)
    return [rng.standard_normal((S, H, D)).astype(np.float32) for _ in range(3)]


def test_keeps_all_equals_dense_attention():
    lay = O.build_layout([(40, (3, 10, 12), (2, 8, 8))], 40 + 360 + 25)
    q, k, v = _qkv(lay.seq_len, 2, 16, 6)
    heads = [0, 1]
    qt, kt, vt = (O.gather(x, lay, heads) for x in (q, k, v))
    kept = O.select(np.zeros((2, lay.n_video, lay.n_video), np.float32), lay,
                    O.column_blocks(lay, (1.0, None), (1.0, None)))
    mask = O.block_mask(kept, lay)
    ot = O.attend_tiles(qt, kt, vt, lay, lambda h, i: np.flatnonzero(mask[h, i]))
    out = np.zeros(q.shape)
    O.scatter(out, ot, lay, heads)
    assert np.abs(out - O.dense_attention(q, k, v)).max() < 1e-12


def test_sparse_matches_token_mask_in_original_order():
    lay = O.build_layout([(20, (2, 16, 16), (1, 16, 8)), (20 + 512, (3, 10, 12), (2, 8, 8))], 20 + 512 + 360 + 70)
    S, H, D = lay.seq_len, 2, 8
    q, k, v = _qkv(S, H, D, 7)
    rng = np.random.default_rng(8)
    kept = O.select(rng.standard_normal((H, lay.n_video, lay.n_video)).astype(np.float32), lay,
                    O.column_blocks(lay, (0.3, None), (None, 2)))
    mask = O.block_mask(kept, lay)
    qt, kt, vt = (O.gather(x, lay, [0, 1]) for x in (q, k, v))
    ot = O.attend_tiles(qt, kt, vt, lay, lambda h, i: np.flatnonzero(mask[h, i]))
    out = np.zeros(q.shape)
    O.scatter(out, ot, lay, [0, 1])
    # brute force in the original row order: row i sees row j iff their tiles form a kept pair
    tile_of = np.empty(S, dtype=np.int64)
    real = lay.perm >= 0
    tile_of[lay.perm[real]] = np.flatnonzero(real) // 128
    for h in range(H):
        allow = mask[h][tile_of[:, None], tile_of[None, :]]
        z = (q[:, h].astype(np.float64) @ k[:, h].astype(np.float64).T) / math.sqrt(D)
        z = np.where(allow, z, -np.inf)
        p = np.exp(z - z.max(1, keepdims=True))
        p /= p.sum(1, keepdims=True)
        assert np.abs(p @ v[:, h] - out[:, h]).max() < 1e-12
    # the tile-order path agrees with the token-mask formulation of the same layout
    assert np.nanmax(np.abs(O.attend_dense_mask(qt, kt, vt, mask, lay) - ot)) < 1e-12


def test_fully_masked_and_padding_rows_are_zero():
    lay = O.build_layout([(0, (3, 10, 12), (2, 8, 8))], 360)
    q, k, v = _qkv(360, 1, 8, 9)
    qt, kt, vt = (O.gather(x, lay, [0]) for x in (q, k, v))
    ot = O.attend_tiles(qt, kt, vt, lay, lambda h, i: [] if i == 0 else [i])
    assert (ot[:128] == 0).all()
    assert (ot[~lay.slot_valid] == 0).all()


# ------------------------------------------------------------------------------------------ FP8 reading

def test_e4m3_rounding_matches_torch():
    x = np.concatenate([np.random.default_rng(10).standard_normal(20000) * s for s in (1e-3, 0.1, 1, 30, 500)])
    x = np.concatenate([x, [0.0, 448.0, -448.0, 2 ** -9, 2 ** -10, 3 * 2 ** -11, 1.0625, 1.1875]])
    x = x[np.abs(x) <= 448.0]  # torch's cast is defined inside the finite range (it gives NaN beyond)
    want = torch.from_numpy(x.astype(np.float32)).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = O.veda._round_e4m3(x.astype(np.float32).astype(np.float64))
    assert np.array_equal(got, want)
    # beyond the range the reading saturates to +-448
    assert O.veda._round_e4m3(np.array([464.0, 1e6, -500.0])).tolist() == [448.0, 448.0, -448.0]


def test_fp8_tile_scales():
    lay = O.build_layout([(0, (3, 10, 12), (2, 8, 8))], 360)
    rng = np.random.default_rng(12)
    x = (rng.standard_normal((360, 2, 16)) * 3).astype(np.float32)
    xt = O.gather(x, lay, [0, 1])
    codes, scales = O.quantize_fp8_tiles(xt, lay)
    assert np.abs(codes).max() <= 448.0
    for i in range(lay.n_tiles):
        for h in range(2):
            c = lay.valid_count[i]
            assert np.abs(codes[i * 128:i * 128 + c, h]).max() == 448.0  # the amax lands on 448
    deq = codes * scales.T[np.arange(lay.n_tiles * 128) // 128][:, :, None]
    rel = np.abs(deq - xt)[lay.slot_valid] / (np.abs(xt)[lay.slot_valid] + 1e-3)
    assert np.median(rel) < 0.05


def test_fp8_attention_exact_on_grid_values():
    # values that are e4m3 numbers times a power-of-two step, with the tile's amax at 448 steps, quantise
    # exactly (the scale is the step, each quotient is its own e4m3 code), so the FP8 reading's attention
    # equals plain attention; different steps per tile and head catch a scale taken from the wrong tile or
    # head, and a scale without the 1/448 or applied to one side only fails as well
    lay = O.build_layout([(0, (3, 10, 12), (2, 8, 8))], 360)
    rng = np.random.default_rng(15)
    H, D = 2, 16
    qt = np.zeros((lay.n_tiles * 128, H, D))
    kt = np.zeros_like(qt)
    for arr in (qt, kt):
        for i in range(lay.n_tiles):
            c = lay.valid_count[i]
            for h in range(H):
                step = 2.0 ** -int(rng.integers(6, 12))
                e = rng.integers(-6, 9, size=(c, D)).astype(np.float64)       # normal e4m3 exponents
                m = rng.integers(0, 8, size=(c, D)).astype(np.float64)        # 3 mantissa bits
                m = np.where(e == 8, np.minimum(m, 6), m)                     # at most 448 = 1.75 * 2^8
                code = (1 + m / 8) * np.exp2(e) * np.where(rng.random((c, D)) < 0.5, -1.0, 1.0)
                code[0, 0] = 448.0 * (1 if rng.random() < 0.5 else -1)      # the tile's amax
                assert np.array_equal(O.veda._round_e4m3(code), code)
                arr[i * 128:i * 128 + c, h] = code * step
    codes, scales = O.quantize_fp8_tiles(qt, lay)
    assert set(np.unique(np.log2(scales))) <= set(range(-11, -5))
    vt = rng.standard_normal(qt.shape) * lay.slot_valid[:, None, None]
    lists = lambda hh, i: np.arange(lay.n_tiles)
    want = O.attend_tiles(qt, kt, vt, lay, lists)
    got = O.attend_tiles_fp8(qt, kt, vt, lay, lists)
    assert np.allclose(got, want, rtol=0, atol=1e-12)


# ------------------------------------------------------------------------------------------ INT8 reading

def test_int8_rounding_table():
    # nearest integer, ties to even, saturating at +-127 (values worked by hand)
    x = np.array([0.0, 0.49, 0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 3.7, -3.7, 126.5, 127.49, 127.5, 300.0, -1e9])
    want = [0.0, 0.0, 0.0, 2.0, 2.0, -0.0, -2.0, -2.0, 4.0, -4.0, 126.0, 127.0, 127.0, 127.0, -127.0]
    assert O.veda._round_int8(x).tolist() == want


def test_int8_tile_scales_and_rounding_bound():
    lay = O.build_layout([(0, (3, 10, 12), (2, 8, 8))], 360)
    rng = np.random.default_rng(13)
    x = (rng.standard_normal((360, 2, 16)) * 3).astype(np.float32)
    xt = O.gather(x, lay, [0, 1])
    codes, scales = O.quantize_int8_tiles(xt, lay)
    assert np.array_equal(codes, np.round(codes)) and np.abs(codes).max() <= 127
    tile_of = np.arange(lay.n_tiles * 128) // 128
    for i in range(lay.n_tiles):
        for h in range(2):
            c = lay.valid_count[i]
            assert np.abs(codes[i * 128:i * 128 + c, h]).max() == 127  # the amax lands on 127
            amax = np.abs(xt[i * 128:i * 128 + c, h]).max()
            assert scales[h, i] == float(np.float32(amax / 127.0))
    # a rounded code is within half a step of the value
    deq = codes * scales.T[tile_of][:, :, None]
    step = scales.T[tile_of][:, :, None] * np.ones_like(xt)
    assert np.all(np.abs(deq - xt)[lay.slot_valid] <= 0.5 * step[lay.slot_valid] * (1 + 1e-6))
    assert (codes[~lay.slot_valid] == 0).all()


def test_int8_attention_exact_on_grid_values():
    # values that are integer multiples of a power of two with the tile's amax at 127 steps quantise
    # exactly, so the INT8 reading's attention equals plain attention; different steps per tile and head
    # catch a scale taken from the wrong tile or head
    lay = O.build_layout([(0, (3, 10, 12), (2, 8, 8))], 360)
    rng = np.random.default_rng(14)
    H, D = 2, 16
    qt = np.zeros((lay.n_tiles * 128, H, D))
    kt = np.zeros_like(qt)
    for arr in (qt, kt):
        for i in range(lay.n_tiles):
            c = lay.valid_count[i]
            for h in range(H):
                step = 2.0 ** -int(rng.integers(3, 9))
                blk = rng.integers(-127, 128, size=(c, D)).astype(np.float64)
                blk[0, 0] = 127 * (1 if rng.random() < 0.5 else -1)
                arr[i * 128:i * 128 + c, h] = blk * step
    vt = rng.standard_normal(qt.shape) * lay.slot_valid[:, None, None]
    lists = lambda hh, i: np.arange(lay.n_tiles)
    want = O.attend_tiles(qt, kt, vt, lay, lists)
    got = O.attend_tiles_int8(qt, kt, vt, lay, lists)
    assert np.allclose(got, want, rtol=0, atol=1e-12)


# ------------------------------------------------------------------------------------------ work counter

def test_work_fraction_plausible_against_printed_report():
    rows = dict(ln.split() for ln in open(os.path.join(GOLDEN, "run_report.txt")) if ln.strip() and ln[0] != "#")
    printed = float(rows["attention_computed_percent"])
    wl = V.workload("mixed")
    fractions = []
    for shape in [(1, 8, 16), (8, 4, 4), (2, 16, 4)]:
        lay = O.build_layout([(512, (1, 48, 84), (1, 16, 8)), (wl.target[0], wl.target[1], shape)], wl.seq_len)
        kept = 0
        for blk in O.column_blocks(lay, wl.generated, wl.reference):
            kept += int(O.allowed_per_row(lay, blk).sum())
        work, dense = O.work_stats(lay, 1, kept)
        fractions.append(100.0 * work / dense)
    assert all(abs(f - printed) < 0.5 for f in fractions), fractions
