"""CPU checks of the C ABI: the library loads and exports every declared symbol, and the host planner
(veda_plan and friends, no GPU needed) agrees bit for bit with the oracle."""
import math
import os
import re

import numpy as np
import pytest

import oracle as O
import veda_synth as V
from learned_block_sparse_tile_b200 import _lib as L
from learned_block_sparse_tile_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    B.build()


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "veda.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(veda_[a-z_0-9]+)\s*\(", text)))


def test_every_declared_symbol_is_exported():
    lib = L.lib()
    syms = declared_symbols()
    assert len(syms) >= 14
    for s in syms:
        assert hasattr(lib, s), s
    assert set(syms) == set(L.EXPORTS)


def _plan_both(spans_o, seq_len, gen, ref):
    lay_o = O.build_layout(spans_o, seq_len)
    lay_c = L.veda_plan([(s, g, b) for s, g, b in spans_o], seq_len, gen, ref)
    return lay_o, lay_c


def _check_plan(spans_o, seq_len, gen, ref):
    lay_o, lay_c = _plan_both(spans_o, seq_len, gen, ref)
    perm, vc, allowed = L.veda_layout_export(lay_c)
    assert np.array_equal(perm, lay_o.perm)
    assert np.array_equal(vc, lay_o.valid_count)
    assert (lay_c.n_video, lay_c.n_ref, lay_c.n_global) == (lay_o.n_video, lay_o.n_ref, lay_o.n_global)
    blocks = O.column_blocks(lay_o, gen, ref)
    assert len(blocks) == len(lay_c.blocks)
    for b, blk in enumerate(blocks):
        start, stop, budget, real = blk
        cb = lay_c.blocks[b]
        assert (cb[0], cb[1], cb[2]) == (start, stop, O.keeps_all(budget))
        assert np.array_equal(allowed[b], O.allowed_per_row(lay_o, blk))
        if not O.keeps_all(budget):
            rb = O.row_budget(budget, real, stop - start)
            lo, hi, frac = O.split_budget(rb, stop - start)
            assert cb[6] == rb and (cb[3], cb[4]) == (lo, hi) and cb[5] == frac  # bit for bit
    # an upper bound on every row's kept count, and the page's own bound (non-empty tiles)
    assert lay_c.max_kept <= lay_o.widest
    return lay_o, lay_c


@pytest.mark.parametrize("name", ["tiny", "padded_tiny", "small_mixed", "small_dense", "small_d128", "single",
                                  "mixed", "long", "sweep_tiles24", "sweep_r025", "sweep_r050", "sweep_dense"])
def test_plan_matches_oracle_on_workloads(name):
    wl = V.workload(name)
    lps = O.least_padding_shape(wl.target[1])
    tile_refs = not O.keeps_all(wl.reference)
    for shape, _heads in V.head_groups(wl, lambda _: lps):
        spans = O.layer_spans(wl.ref_spans, (wl.target[0], wl.target[1], shape), tile_refs)
        _check_plan(spans, wl.seq_len, wl.generated, wl.reference)


def test_untiled_references_become_global():
    wl = V.workload("small_mixed")
    spans_c = [(s, g, None) for s, g in wl.ref_spans] + [(wl.target[0], wl.target[1], (2, 8, 8))]
    lay_c = L.veda_plan(spans_c, wl.seq_len, (0.3, None), (1.0, None))
    lay_o = O.build_layout([(wl.target[0], wl.target[1], (2, 8, 8))], wl.seq_len)
    perm, vc, _ = L.veda_layout_export(lay_c)
    assert lay_c.n_ref == 0 and np.array_equal(perm, lay_o.perm)


def test_least_padding_box_matches_oracle():
    rng = np.random.default_rng(0)
    grids = [tuple(int(x) for x in rng.integers(1, 90, 3)) for _ in range(300)]
    grids += [(26, 48, 84), (61, 45, 80), (1, 48, 84), (8, 16, 16), (1, 1, 1), (300, 2, 1)]
    for g in grids:
        assert L.veda_least_padding_box(g) == O.least_padding_shape(g), g


def test_budget_split_sweep_bit_exact():
    # many grids and budgets: the library's (k_lo, k_hi, frac, row budget) equal the oracle's bit for bit
    rng = np.random.default_rng(1)
    for _ in range(120):
        grid = tuple(int(x) for x in rng.integers(1, 40, 3))
        shape = O.tile_shapes()[int(rng.integers(0, 36))]
        start = int(rng.integers(0, 300))
        seq = start + grid[0] * grid[1] * grid[2] + int(rng.integers(0, 300))
        if rng.random() < 0.5:
            gen = (float(rng.choice([0.05, 0.1, 0.25, 0.3, 0.5, 0.75, 0.99, 1.0, 1.5, 0.001, 1 / 3])), None)
        else:
            gen = (None, int(rng.integers(0, 60)))
        _check_plan([(start, grid, shape)], seq, gen, (1.0, None))


def test_plan_errors():
    with pytest.raises(L.VedaError) as e:
        L.veda_plan([], 10, (0.1, None), (1.0, None))
    assert e.value.code == L.VEDA_ERR_INVALID
    for bad_budget in [(0.1, 3), (None, None), (-0.5, None)]:
        with pytest.raises(L.VedaError):
            L.veda_plan([(0, (1, 8, 16), None)], 128, bad_budget, (1.0, None))
    with pytest.raises(L.VedaError):  # overlap
        L.veda_plan([(0, (1, 8, 16), None), (100, (1, 8, 16), None)], 400, (0.1, None), (0.5, None))
    with pytest.raises(L.VedaError):  # past the end
        L.veda_plan([(10, (1, 8, 16), None)], 100, (0.1, None), (1.0, None))
    with pytest.raises(L.VedaError):  # not a power-of-two box of 128
        L.veda_plan([(0, (1, 8, 16), (1, 8, 15))], 128, (0.1, None), (1.0, None))
    assert "overlaps" in L.veda_last_error() or L.veda_last_error() != ""


def test_work_fraction_of_mixed_geometry():
    # the library's per-row budgets reproduce the page's work counter on the mixed workload (10.85-11.07%)
    wl = V.workload("mixed")
    for box in [(1, 8, 16), (8, 4, 4), (2, 16, 4)]:
        lay = L.veda_plan([(512, (1, 48, 84), None), (wl.target[0], wl.target[1], box)], wl.seq_len,
                          wl.generated, wl.reference)
        _, _, allowed = L.veda_layout_export(lay)
        kept = int(allowed.sum())
        work = kept + lay.n_global * (lay.n_tiles + lay.n_video)
        frac = work / (wl.seq_len / 128) ** 2
        assert 0.105 < frac < 0.112


def _expected_box_rows(start, grid, box):
    """Box origins in the pages' visiting order (h-box outermost, then w-box, then t-box) and, per box, the
    packed row of every box position (t, h, w row-major inside the box; -1 outside the grid)."""
    T, H, W = grid
    st, sh, sw = box
    out = []
    for bh in range(-(-H // sh)):
        for bw in range(-(-W // sw)):
            for bt in range(-(-T // st)):
                t0, h0, w0 = bt * st, bh * sh, bw * sw
                rows = []
                for dt in range(st):
                    for dh in range(sh):
                        for dw in range(sw):
                            t, h, w = t0 + dt, h0 + dh, w0 + dw
                            rows.append(start + (t * H + h) * W + w if t < T and h < H and w < W else -1)
                out.append(((t0, h0, w0), rows))
    return out


@pytest.mark.parametrize("name", ["tiny", "padded_tiny", "small_mixed", "small_dense", "small_d128", "mixed",
                                  "long"])
def test_box_form_of_the_layout(name):
    # the gather-free attend's boxes: every tile holds the same rows as in tile order, span tiles are the
    # grid boxes at their origins (padding in place), global tiles are runs from their first row
    wl = V.workload(name)
    lps = O.least_padding_shape(wl.target[1])
    tile_refs = not O.keeps_all(wl.reference)
    for shape, _heads in V.head_groups(wl, lambda _: lps):
        spans = O.layer_spans(wl.ref_spans, (wl.target[0], wl.target[1], shape), tile_refs)
        lay_o, lay_c = _plan_both(spans, wl.seq_len, wl.generated, wl.reference)
        box_perm, coord, mask = L.veda_layout_export_direct(lay_c)
        perm = lay_o.perm.reshape(-1, 128)
        bp = box_perm.reshape(-1, 128)
        bits = (mask.view(np.uint32)[:, :, None] >> np.arange(32, dtype=np.uint32)) & 1
        assert np.array_equal(bits.reshape(-1, 128).astype(bool), bp >= 0)
        for i in range(lay_o.n_tiles):
            assert sorted(bp[i][bp[i] >= 0].tolist()) == sorted(perm[i][perm[i] >= 0].tolist()), i
        i = 0
        for s_idx, (start, grid, box) in enumerate(spans):
            for (t0, h0, w0), rows in _expected_box_rows(start, grid, box):
                assert tuple(coord[i]) == (s_idx, w0, h0, t0), i
                assert bp[i].tolist() == rows, i
                i += 1
        assert i == lay_o.n_video
        for i in range(lay_o.n_video, lay_o.n_tiles):
            c = int(lay_o.valid_count[i])
            row0 = int(perm[i][0])
            assert tuple(coord[i]) == (-1, row0, 0, 0)
            assert bp[i].tolist() == [row0 + j if j < c else -1 for j in range(128)]


def test_box_form_needs_runs_of_global_rows():
    # two uncovered stretches that meet inside one global tile: that tile is not a run of rows
    lay = L.veda_plan([(100, (1, 8, 16), None)], 400, (0.5, None), (1.0, None))
    with pytest.raises(L.VedaError) as e:
        L.veda_layout_export_direct(lay)
    assert e.value.code == L.VEDA_ERR_UNSUPPORTED
    assert "not a run" in str(e.value)


@pytest.mark.parametrize("name", ["single", "mixed", "long", "sweep_tiles24", "sweep_r025", "sweep_r050",
                                  "sweep_dense", "single_h4"])
def test_published_configurations_take_the_gather_free_path(name):
    # every head group of the published configurations has a box form, so VedaLayer's default (and the
    # bench) runs the gather-free attend on them
    wl = V.workload(name)
    lps = L.veda_least_padding_box(wl.target[1])
    spans_ref = [(s, g, None) for s, g in wl.ref_spans]
    for shape, _heads in V.head_groups(wl, lambda _: lps):
        lay = L.veda_plan(spans_ref + [(wl.target[0], wl.target[1], shape)], wl.seq_len, wl.generated, wl.reference)
        assert L.veda_layout_has_box_form(lay), (name, shape)


@pytest.mark.parametrize("name", ["tiny", "padded_tiny", "small_d128", "single"])
@pytest.mark.parametrize("n_heads", [1, 3, 24])
def test_paired_workspace_size(name, n_heads):
    # the paired attend's workspace: per head the merged lists of ceil(n_video / 2) pairs (2 max_kept units
    # each) and their (units, units of A) counts, then a redo flag per (head, tile), the redo list's length
    # and the redo list, every region 256-byte aligned; host arithmetic only (no device)
    wl = V.workload(name)
    lps = O.least_padding_shape(wl.target[1])
    lay = L.veda_plan([(s, g, None) for s, g in wl.ref_spans] + [(wl.target[0], wl.target[1], lps)], wl.seq_len,
                      wl.generated, wl.reference)
    a256 = lambda x: (x + 255) // 256 * 256  # noqa: E731
    pairs = (lay.n_video + 1) // 2
    want = (a256(n_heads * pairs * 2 * lay.max_kept * 4) + a256(n_heads * pairs * 8) + 2 * a256(n_heads * lay.n_tiles * 4)
            + 256)
    assert L.veda_attend_paired_workspace_bytes(lay, n_heads) == want
    assert L.veda_attend_paired_workspace_bytes(lay, 0) == 0


@pytest.mark.parametrize("name,n_heads,dim", [("small_d128", 3, 128), ("single", 24, 128), ("small_d128", 2, 64)])
def test_score_workspace_size(name, n_heads, dim):
    # veda_score's workspace: per head the projected q and k features (2 n_video D floats) and both
    # projections transposed with the residual's identity block ((P + E)^T, 2 x D x 3D floats); host only
    wl = V.workload(name)
    lps = O.least_padding_shape(wl.target[1])
    lay = L.veda_plan([(s, g, None) for s, g in wl.ref_spans] + [(wl.target[0], wl.target[1], lps)], wl.seq_len,
                      wl.generated, wl.reference)
    want = n_heads * (2 * lay.n_video * dim + 2 * dim * 3 * dim) * 4
    assert L.veda_score_workspace_bytes(lay, n_heads, dim) == want
    assert L.veda_score_workspace_bytes(lay, 0, dim) == 0
