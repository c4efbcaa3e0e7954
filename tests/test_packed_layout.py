"""Packed-layout description (veda_core.py, "what the packed layout holds": _grid_of, describe_layout): the
oracle pinned by brute force and hand-worked cases, the C ABI's veda_grid_of / veda_describe_packed_layout
against the oracle, and the described spans planned by veda_plan as the oracle lays them out. CPU only."""
import itertools

import numpy as np
import pytest

import oracle as O
from learned_block_sparse_tile_b200 import _lib as L
from learned_block_sparse_tile_b200 import build as B


@pytest.fixture(scope="module", autouse=True)
def built():
    B.build()


def _grid_positions(t_vals, h_vals, w_vals):
    return np.array(list(itertools.product(t_vals, h_vals, w_vals)), dtype=np.float64)


def _brute_grid_of(pos):
    """Try every factorisation T * H * W of the row count and every axis value set, by the definition."""
    n = len(pos)
    for t in range(1, n + 1):
        for h in range(1, n // t + 1):
            if n % (t * h):
                continue
            w = n // (t * h)
            ts, hs, ws = (sorted(set(pos[:, i].tolist())) for i in range(3))
            if (len(ts), len(hs), len(ws)) != (t, h, w):
                continue
            if np.array_equal(pos, _grid_positions(ts, hs, ws)):
                return (t, h, w)
    return None


def test_grid_of_pins():
    g = _grid_positions([0, 1], [0, 2, 4], [5, 6, 7, 8])  # strided h, offset w: still a grid
    assert O.grid_of(g, 0, 24) == (2, 3, 4) == _brute_grid_of(g)
    assert O.grid_of(g[::-1], 0, 24) is None                                    # not ascending
    swapped = g.copy()
    swapped[[3, 4]] = swapped[[4, 3]]
    assert O.grid_of(swapped, 0, 24) is None and _brute_grid_of(swapped) is None  # not row-major
    assert O.grid_of(g, 0, 23) is None                                          # sizes do not multiply out
    dup = np.concatenate([g, g[:1]])
    assert O.grid_of(dup, 0, 25) is None                                        # a repeated position
    assert O.grid_of(np.concatenate([np.zeros((5, 3)), g]), 5, 29) == (2, 3, 4)  # rows a:b only
    one = _grid_positions([3], [7], list(range(10)))
    assert O.grid_of(one, 0, 10) == (1, 1, 10)


@pytest.mark.parametrize("seed", range(6))
def test_grid_of_matches_bruteforce_and_the_abi(seed):
    rng = np.random.default_rng(seed)
    t, h, w = rng.integers(1, 5, 3)
    pos = _grid_positions(np.sort(rng.choice(50, t, replace=False)), np.sort(rng.choice(50, h, replace=False)),
                          np.sort(rng.choice(50, w, replace=False)))
    if seed % 2:  # break it: move one row's w
        i = int(rng.integers(len(pos)))
        pos[i, 2] += 0.5
    want = _brute_grid_of(pos)
    assert O.grid_of(pos, 0, len(pos)) == want
    assert L.veda_grid_of(pos, 0, len(pos)) == want


def _packed(seed, verified=True):
    """A packed sequence like a video model's: text rows, a cond reference, a ref_img reference, the video."""
    rng = np.random.default_rng(seed)
    lt, lh, lw = 3, 8, 12  # latent grid: the video holds 3 x 4 x 6 = 72 rows
    text = int(rng.integers(0, 40))
    cond = (1, 4, 6)
    ref = (2, 2, 3)
    segs, pos, at = [], [], 0
    segs.append((at, at + text, "text"))
    pos.append(rng.integers(0, 9, (text, 3)).astype(np.float64))
    at += text
    for kind, g in (("cond", cond), ("ref_img", ref)):
        n = g[0] * g[1] * g[2]
        p = _grid_positions(range(g[0]), range(g[1]), range(g[2]))
        if not verified and kind == "ref_img":
            p = p[::-1].copy()
        segs.append((at, at + n, kind))
        pos.append(p)
        at += n
    segs.append((at, at + 72, "video"))
    pos.append(_grid_positions(range(lt), range(lh // 2), range(lw // 2)))
    at += 72
    return segs, (lt, lh, lw), at, np.concatenate(pos)


@pytest.mark.parametrize("verified", [True, False])
@pytest.mark.parametrize("seed", range(3))
def test_describe_packed_layout_matches_the_oracle(seed, verified):
    segs, latent, seq_len, pos = _packed(seed, verified)
    want = O.describe_packed_layout(segs, latent, seq_len, pos)
    got = L.veda_describe_packed_layout(segs, latent, seq_len, pos)
    assert got[:3] == want[:3]
    # the oracle notes skipped segments by name, the ABI by index
    assert [f"{segs[i][2]}[{segs[i][0]}:{segs[i][1]}]" for i in got[3]] == list(want[3])
    # hand-worked: the target is the last 72 rows at grid (3, 4, 6); cond is always a verified grid
    assert want[1] == (seq_len - 72, (3, 4, 6))
    assert want[2][0][1] == (1, 4, 6)
    assert len(want[2]) == (2 if verified else 1)
    # without position ids no reference can be verified: all stay global
    none = L.veda_describe_packed_layout(segs, latent, seq_len, None)
    assert none[2] == () and len(none[3]) == 2


def test_describe_packed_layout_errors():
    segs, latent, seq_len, pos = _packed(0)
    for bad in (segs + [(0, 0, "video")], [s for s in segs if s[2] != "video"]):
        with pytest.raises(O.VedaError):
            O.describe_packed_layout(bad, latent, seq_len, pos)
        with pytest.raises(L.VedaError) as e:
            L.veda_describe_packed_layout(bad, latent, seq_len, pos)
        assert e.value.code == L.VEDA_ERR_INVALID and "video segment" in str(e.value)
    with pytest.raises(O.VedaError):
        O.describe_packed_layout(segs, (3, 8, 14), seq_len, pos)
    with pytest.raises(L.VedaError) as e:
        L.veda_describe_packed_layout(segs, (3, 8, 14), seq_len, pos)
    assert "latent grid" in str(e.value)
    with pytest.raises(L.VedaError):  # a segment past the packed rows
        L.veda_describe_packed_layout(segs + [(seq_len - 2, seq_len + 5, "cond")], latent, seq_len, pos)


def test_described_spans_plan_like_the_oracle():
    # describe, then plan the target at its least-padding box with the references tiled: the C planner's
    # permutation equals the oracle's layout of the same spans
    segs, latent, seq_len, pos = _packed(1)
    _, (t0, tg), refs, _ = L.veda_describe_packed_layout(segs, latent, seq_len, pos)
    box = O.least_padding_shape(tg)
    lay = L.veda_plan([(s, g, None) for s, g in refs] + [(t0, tg, box)], seq_len, (0.5, None), (0.5, None))
    lay_o = O.build_layout(O.layer_spans(refs, (t0, tg, box), True), seq_len)
    perm, vc, _ = L.veda_layout_export(lay)
    assert np.array_equal(perm, lay_o.perm) and np.array_equal(vc, lay_o.valid_count)
