"""GPU parity of the paired attend (veda_attend_paired, veda_attend_direct_paired) against the CPU oracle:
two neighbouring query tiles per work item sharing each kept K/V tile, the softmax reference fixed by the
logit bound, and the exact redo of query tiles whose bound is too loose. Calls go through the C ABI."""
import numpy as np
import pytest
import torch

import oracle as O
from learned_block_sparse_tile_b200 import _lib as L
from learned_block_sparse_tile_b200 import build as B

from gpu_util import ATT_MAX_ABS, ATT_MEAN_ABS, Case, attention_error, f32, oracle_kept

pytestmark = pytest.mark.gpu

SMALL = ["tiny", "padded_tiny", "small_mixed", "small_dense", "small_d128"]
_cases = {}


@pytest.fixture(scope="module", autouse=True)
def built():
    B.build()
    L.veda_device_check()


def case(name):
    if name not in _cases:
        _cases[name] = Case(name)
    return _cases[name]


def norms(lay, q, k, heads, n, seq_len):
    row_sq = torch.full((n, seq_len), -1.0, device="cuda")
    max_sq = torch.full((n,), -1.0, device="cuda")
    fq = torch.empty(n, lay.n_video, 3 * q.shape[2], dtype=torch.float32, device="cuda")
    fk = torch.empty_like(fq)
    L.veda_pool(lay, q, heads, fq, row_sq=row_sq)
    L.veda_pool(lay, k, heads, fk, max_sq=max_sq)
    return row_sq, max_sq


def oracle_out(c, box, heads, res, q, k, v, want, idx=None, cnt=None):
    """Oracle attention of one group into ``want``, on the GPU's kept lists (or on idx/cnt when given)."""
    wl = c.wl
    lay_o = O.build_layout(c.spans_oracle(box), wl.seq_len)
    if idx is None:
        _, mask = oracle_kept(lay_o, f32(res["scores"]), O.column_blocks(lay_o, wl.generated, wl.reference))
        lists = lambda hh, i: np.flatnonzero(mask[hh, i])  # noqa: E731
    else:
        lists = lambda hh, i: (idx[hh, i, :cnt[hh, i]] if i < lay_o.n_video  # noqa: E731
                               else np.flatnonzero(lay_o.kv_ok))
    qt, kt, vt = (O.gather(x, lay_o, heads) for x in (q, k, v))
    O.scatter(want, O.attend_tiles(qt, kt, vt, lay_o, lists), lay_o, heads)
    return lay_o


def redo_flags(lay, n, ws):
    """The redo flags the paired launch left in its workspace ([n, n_tiles] int32 after the merged lists and
    their counts (two int32 per pair), each region 256-byte aligned), checked against the redo list that follows them: its
    length (an int32 in a 256-byte slot) and its entries (single-tile item numbers: global query tiles
    first, head-major, then video ones)."""
    a256 = lambda x: (x + 255) // 256 * 256  # noqa: E731
    pairs = (lay.n_video + 1) // 2
    off = a256(n * pairs * 2 * lay.max_kept * 4) + a256(n * pairs * 8)
    fb = a256(n * lay.n_tiles * 4)
    flags = ws[off:off + n * lay.n_tiles * 4].view(torch.int32).view(n, lay.n_tiles).cpu().numpy()
    count = int(ws[off + fb:off + fb + 4].view(torch.int32).item())
    items = ws[off + fb + 256:off + fb + 256 + 4 * count].view(torch.int32).cpu().numpy()
    want = []
    for hh in range(n):
        for t in np.flatnonzero(flags[hh]):
            want.append(hh * lay.n_global + (t - lay.n_video) if t >= lay.n_video
                        else n * lay.n_global + hh * lay.n_video + t)
    assert sorted(items.tolist()) == sorted(want), (items, want)
    return flags


@pytest.mark.parametrize("name", SMALL)
@pytest.mark.parametrize("q_scale", [1.0, 4.0, 16.0])
def test_paired_attend(name, q_scale):
    # both paired entry points against the oracle on the GPU's own kept lists: odd video tile counts (a last
    # pair of one tile), global query tiles (paired on the dense list), several head groups, head_dim 64 and
    # 128. Scaling Q (exactly, in bf16) scales the gap between each row's bound and its true maximum: at 1
    # it stays far below the redo limit (no query tile is flagged), at 4 some rows pass it and at 16 most
    # do, so the exact redo rewrites those tiles; the result matches the oracle either way
    c = case(name)
    wl = c.wl
    qs = c.dq * q_scale
    q, k, v = f32(qs), f32(c.k), f32(c.v)
    want = np.zeros((wl.seq_len, wl.heads, wl.dim), np.float64)
    out_d = torch.full((wl.seq_len, wl.heads, wl.dim), 7.0, dtype=torch.bfloat16, device="cuda")
    out_t = out_d.clone()
    for box, heads in c.groups:
        res = c.run_group(box, heads)
        lay = res["layout"]
        n = len(heads)
        row_sq, max_sq = norms(lay, qs, c.dk, res["heads"], n, wl.seq_len)
        q_t = torch.empty_like(res["q_t"])
        L.veda_gather(lay, qs, res["heads"], q_t, None)
        ws = L.paired_workspace(lay, n)
        L.veda_attend_direct_paired(lay, qs, c.dk, c.dv, res["kept_idx"], res["kept_cnt"], out_d, res["heads"],
                                    row_sq, max_sq, ws)
        assert L.veda_sync_status() == L.VEDA_OK, L.veda_last_error()
        assert q_scale != 1.0 or not redo_flags(lay, n, ws).any()
        L.veda_attend_paired(lay, q_t, res["k_t"], res["v_t"], res["kept_idx"], res["kept_cnt"], out_t,
                             res["heads"], row_sq, max_sq, ws)
        assert L.veda_sync_status() == L.VEDA_OK, L.veda_last_error()
        assert q_scale != 1.0 or not redo_flags(lay, n, ws).any()
        oracle_out(c, box, heads, res, q, k, v, want)
    for out in (out_d, out_t):
        mx, mean = attention_error(f32(out), want)
        assert mx <= ATT_MAX_ABS and mean <= ATT_MEAN_ABS, (mx, mean)


def test_paired_redo_when_the_bound_is_loose():
    # Q's dimension 0 is zeroed and one key of each head gets a spike in it: the head's largest ||k|| then
    # grows while no q . k does, so the bound overshoots every row's true maximum. Head 0 (spike 200):
    # by ~310-470 log2 units (||q|| is ~16 on this data), past the 124 the fixed reference allows, so every
    # one of its query tiles is flagged and recomputed by the exact pass. Head 1 (spike 40): by ~55-90, so
    # its rows keep the fixed reference, many with every 2^(s - m) below 1, and no redo. Both heads must match the oracle; the flags
    # must be set exactly where the rows' excess says they must and clear where it says they cannot be.
    c = case("small_d128")
    wl = c.wl
    q = c.q.clone()
    q[:, :, 0] = 0
    k = c.k.clone()
    k[5, 0, 0] = 200.0
    k[9, 1, 0] = 40.0
    dq, dk = q.cuda(), k.cuda()
    qn, kn, vn = f32(q), f32(k), f32(c.v)
    want = np.zeros((wl.seq_len, wl.heads, wl.dim), np.float64)
    out_d = torch.full((wl.seq_len, wl.heads, wl.dim), 7.0, dtype=torch.bfloat16, device="cuda")
    out_t = out_d.clone()
    scale_log2 = wl.dim ** -0.5 * np.log2(np.e)
    for box, heads in c.groups:
        res = c.run_group(box, heads)
        lay = res["layout"]
        n = len(heads)
        row_sq, max_sq = norms(lay, dq, dk, res["heads"], n, wl.seq_len)
        q_t, k_t = torch.empty_like(res["q_t"]), torch.empty_like(res["k_t"])
        L.veda_gather(lay, dq, res["heads"], q_t, None)
        L.veda_gather(lay, dk, res["heads"], k_t, None)
        ws = L.paired_workspace(lay, n)
        for direct, out in ((True, out_d), (False, out_t)):
            if direct:
                L.veda_attend_direct_paired(lay, dq, dk, c.dv, res["kept_idx"], res["kept_cnt"], out, res["heads"],
                                            row_sq, max_sq, ws)
            else:
                L.veda_attend_paired(lay, q_t, k_t, res["v_t"], res["kept_idx"], res["kept_cnt"], out,
                                     res["heads"], row_sq, max_sq, ws)
            assert L.veda_sync_status() == L.VEDA_OK, L.veda_last_error()
            flags = redo_flags(lay, n, ws)
            lay_o = O.build_layout(c.spans_oracle(box), wl.seq_len)
            _, mask = oracle_kept(lay_o, f32(res["scores"]), O.column_blocks(lay_o, wl.generated, wl.reference))
            for hh, h in enumerate(heads):
                kmax = float((kn[:, h, :].astype(np.float64) ** 2).sum(-1).max())
                n_live = 0
                for t in range(lay_o.n_tiles):
                    rows = lay_o.perm[t * 128:(t + 1) * 128]
                    rows = rows[rows >= 0]
                    keys_t = (np.flatnonzero(mask[hh, t]) if t < lay_o.n_video else np.flatnonzero(lay_o.kv_ok))
                    if len(rows) == 0 or len(keys_t) == 0:
                        assert flags[hh, t] == 0
                        continue
                    n_live += 1
                    keys = np.concatenate([lay_o.perm[j * 128:(j + 1) * 128] for j in keys_t])
                    keys = keys[keys >= 0]
                    qq = qn[rows, h, :].astype(np.float64)
                    s = qq @ kn[keys, h, :].astype(np.float64).T * scale_log2
                    bound = np.sqrt((qq ** 2).sum(-1) * kmax) * scale_log2
                    excess = bound - s.max(-1)
                    if excess.max() > 124 + np.log2(len(keys)) + 1:
                        assert flags[hh, t] == 1, (h, t, excess.max())
                    elif excess.max() < 123:
                        assert flags[hh, t] == 0, (h, t, excess.max())
                # head 0: every query tile with rows and keys; head 1: none
                assert int(flags[hh].sum()) == (n_live if h == 0 else 0), (h, int(flags[hh].sum()), n_live)
        oracle_out(c, box, heads, res, qn, kn, vn, want)
    for out in (out_d, out_t):
        mx, mean = attention_error(f32(out), want)
        assert mx <= ATT_MAX_ABS and mean <= ATT_MEAN_ABS, (mx, mean)


def test_paired_lists_of_every_shape():
    # hand-made lists for the pairs of small_d128 (27 video query tiles, the last alone): A empty / B not,
    # A / B empty, identical, disjoint, interleaved, a full row; the rows of an empty list are 0, the rest
    # match the oracle on the same lists
    c = case("small_d128")
    wl = c.wl
    box, heads = c.groups[0]
    res = c.run_group(box, heads)
    lay = res["layout"]
    n = len(heads)
    lay_o = O.build_layout(c.spans_oracle(box), wl.seq_len)
    ok = np.flatnonzero(lay_o.kv_ok)
    nv = lay_o.n_video
    rng = np.random.default_rng(3)
    idx = np.full((n, nv, lay.max_kept), -9, np.int32)
    cnt = np.zeros((n, nv), np.int32)
    for hh in range(n):
        for p in range((nv + 1) // 2):
            kind = (p + hh) % 6
            base = np.sort(rng.choice(ok, size=min(lay.max_kept, 9), replace=False))
            other = np.sort(rng.choice(ok, size=min(lay.max_kept, 7), replace=False))
            lists = {0: ([], base), 1: (base, []), 2: (base, base), 3: (base[::2], base[1::2]),
                     4: (base, other), 5: (ok[:lay.max_kept], base)}[kind]
            for r, l in zip((2 * p, 2 * p + 1), lists):
                if r < nv:
                    l = np.asarray(l, np.int32)
                    idx[hh, r, :len(l)] = l
                    cnt[hh, r] = len(l)
    didx, dcnt = torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda()
    row_sq, max_sq = norms(lay, c.dq, c.dk, res["heads"], n, wl.seq_len)
    ws = L.paired_workspace(lay, n)
    out = torch.full((wl.seq_len, wl.heads, wl.dim), 7.0, dtype=torch.bfloat16, device="cuda")
    L.veda_attend_paired(lay, res["q_t"], res["k_t"], res["v_t"], didx, dcnt, out, res["heads"], row_sq, max_sq, ws)
    assert L.veda_sync_status() == L.VEDA_OK, L.veda_last_error()
    want = np.zeros((wl.seq_len, wl.heads, wl.dim), np.float64)
    oracle_out(c, box, heads, res, f32(c.q), f32(c.k), f32(c.v), want, idx, cnt)
    rows = np.unique(lay_o.perm[lay_o.perm >= 0])
    got = f32(out)[:, heads, :][rows]
    exp = want[:, heads, :][rows]
    mx, mean = attention_error(got, exp)
    assert mx <= ATT_MAX_ABS and mean <= ATT_MEAN_ABS, (mx, mean)
    for hh in range(n):
        for r in np.flatnonzero(cnt[hh] == 0):
            pr = lay_o.perm[r * 128:(r + 1) * 128]
            assert (f32(out)[pr[pr >= 0], heads[hh]] == 0).all()


def test_paired_malformed_lists_and_bad_arguments():
    c = case("tiny")
    wl = c.wl
    box, heads = c.groups[0]
    res = c.run_group(box, heads)
    lay = res["layout"]
    n = len(heads)
    row_sq, max_sq = norms(lay, c.dq, c.dk, res["heads"], n, wl.seq_len)
    ws = L.paired_workspace(lay, n)
    out = torch.zeros((wl.seq_len, wl.heads, wl.dim), dtype=torch.bfloat16, device="cuda")
    for mutate in ("range", "order", "count"):
        idx, cnt = res["kept_idx"].clone(), res["kept_cnt"].clone()
        if mutate == "range":
            idx[0, 3, 1] = lay.n_tiles + 5
        elif mutate == "order":
            idx[1, 2, 2] = idx[1, 2, 1]
        else:
            cnt[0, 1] = lay.max_kept + 3
        L.veda_attend_paired(lay, res["q_t"], res["k_t"], res["v_t"], idx, cnt, out, res["heads"], row_sq, max_sq, ws)
        assert L.veda_sync_status() == L.VEDA_ERR_BAD_LIST, mutate
    assert L.veda_sync_status() == L.VEDA_OK
    with pytest.raises(L.VedaError):  # the norms are required
        L.veda_attend_paired(lay, res["q_t"], res["k_t"], res["v_t"], res["kept_idx"], res["kept_cnt"], out,
                             res["heads"], None, max_sq, ws)
    with pytest.raises(L.VedaError):  # workspace too small
        L.veda_attend_paired(lay, res["q_t"], res["k_t"], res["v_t"], res["kept_idx"], res["kept_cnt"], out,
                             res["heads"], row_sq, max_sq, ws[:256])
    with pytest.raises(L.VedaError):  # workspace not 256-byte aligned
        L.veda_attend_paired(lay, res["q_t"], res["k_t"], res["v_t"], res["kept_idx"], res["kept_cnt"], out,
                             res["heads"], row_sq, max_sq, torch.empty(ws.numel() + 512, dtype=torch.uint8,
                                                                       device="cuda")[16:])


@pytest.mark.parametrize("name", ["small_mixed", "small_d128", "padded_tiny"])
@pytest.mark.parametrize("ctas", [1, 3])
def test_many_items_per_cta(name, ctas):
    # with the attend launches capped at 1 or 3 CTAs each CTA walks many pair items (and the single-tile
    # kernel many query tiles) in a row, as every CTA does on a full-size layer: ring positions, barrier
    # phases and the per-item state carry across items. Both paired entry points and both single-tile ones
    # give the same output as with one CTA per item, bit for bit
    c = case(name)
    wl = c.wl
    outs = {}
    for cap in (0, ctas):
        L.veda_debug_attend_ctas(cap)
        try:
            for kind in ("paired_direct", "paired", "direct", "tile"):
                out = torch.full((wl.seq_len, wl.heads, wl.dim), 7.0, dtype=torch.bfloat16, device="cuda")
                for box, heads in c.groups:
                    res = c.run_group(box, heads)
                    lay = res["layout"]
                    n = len(heads)
                    row_sq, max_sq = norms(lay, c.dq, c.dk, res["heads"], n, wl.seq_len)
                    ws = L.paired_workspace(lay, n)
                    if kind == "paired_direct":
                        L.veda_attend_direct_paired(lay, c.dq, c.dk, c.dv, res["kept_idx"], res["kept_cnt"], out,
                                                    res["heads"], row_sq, max_sq, ws)
                    elif kind == "paired":
                        L.veda_attend_paired(lay, res["q_t"], res["k_t"], res["v_t"], res["kept_idx"], res["kept_cnt"],
                                             out, res["heads"], row_sq, max_sq, ws)
                    elif kind == "direct":
                        L.veda_attend_direct(lay, c.dq, c.dk, c.dv, res["kept_idx"], res["kept_cnt"], out,
                                             res["heads"], q_row_sq=row_sq, k_max_sq=max_sq)
                    else:
                        L.veda_attend(lay, res["q_t"], res["k_t"], res["v_t"], res["kept_idx"], res["kept_cnt"], out,
                                      res["heads"], q_row_sq=row_sq, k_max_sq=max_sq)
                    assert L.veda_sync_status() == L.VEDA_OK, (kind, cap, L.veda_last_error())
                outs[(kind, cap)] = out
        finally:
            L.veda_debug_attend_ctas(0)
    for kind in ("paired_direct", "paired", "direct", "tile"):
        assert torch.equal(outs[(kind, 0)], outs[(kind, ctas)]), kind


@pytest.mark.parametrize("fmt", ["fp8", "int8"])
@pytest.mark.parametrize("q_scale", [1.0, 16.0])
def test_paired_8bit_codes(fmt, q_scale):
    # veda_attend_fp8_paired / veda_attend_int8_paired against the oracle's 8-bit readings (bf16 tolerance)
    # on the codes of the fused 8-bit gathers, which also write the norms of the bf16 inputs (equal to
    # veda_pool's, bit for bit); q_scale 16 sends most query tiles to the exact redo. The result equals the
    # single-tile 8-bit attend's within rounding
    c = case("small_d128")
    wl = c.wl
    qs = c.dq * q_scale
    q, k, v = f32(qs), f32(c.k), f32(c.v)
    code_t = torch.int8 if fmt == "int8" else torch.uint8
    gather = L.veda_gather_int8 if fmt == "int8" else L.veda_gather_fp8
    paired = L.veda_attend_int8_paired if fmt == "int8" else L.veda_attend_fp8_paired
    single = L.veda_attend_int8 if fmt == "int8" else L.veda_attend_fp8
    reading = O.attend_tiles_int8 if fmt == "int8" else O.attend_tiles_fp8
    out_p = torch.full((wl.seq_len, wl.heads, wl.dim), 7.0, dtype=torch.bfloat16, device="cuda")
    out_s = out_p.clone()
    want = np.zeros((wl.seq_len, wl.heads, wl.dim), np.float64)
    for box, heads in c.groups:
        res = c.run_group(box, heads)
        lay = res["layout"]
        n = len(heads)
        q8 = torch.empty(n, lay.n_slots, wl.dim, dtype=code_t, device="cuda")
        k8 = torch.empty_like(q8)
        sq = torch.empty(n, lay.n_tiles, dtype=torch.float32, device="cuda")
        sk = torch.empty_like(sq)
        row_sq = torch.full((n, wl.seq_len), -1.0, device="cuda")
        max_sq = torch.full((n,), -1.0, device="cuda")
        gather(lay, qs, res["heads"], q8, sq, None, row_sq=row_sq)
        gather(lay, c.dk, res["heads"], k8, sk, None, max_sq=max_sq)
        row_sq_p, max_sq_p = norms(lay, qs, c.dk, res["heads"], n, wl.seq_len)
        assert torch.equal(row_sq, row_sq_p) and torch.equal(max_sq, max_sq_p)
        ws = L.paired_workspace(lay, n)
        paired(lay, q8, k8, sq, sk, res["v_t"], res["kept_idx"], res["kept_cnt"], out_p, res["heads"], row_sq, max_sq,
               ws)
        single(lay, q8, k8, sq, sk, res["v_t"], res["kept_idx"], res["kept_cnt"], out_s, res["heads"])
        assert L.veda_sync_status() == L.VEDA_OK, L.veda_last_error()
        assert q_scale != 1.0 or not redo_flags(lay, n, ws).any()
        lay_o = O.build_layout(c.spans_oracle(box), wl.seq_len)
        _, mask = oracle_kept(lay_o, f32(res["scores"]), O.column_blocks(lay_o, wl.generated, wl.reference))
        qt, kt, vt = (O.gather(x, lay_o, heads) for x in (q, k, v))
        O.scatter(want, reading(qt, kt, vt, lay_o, lambda hh, i: np.flatnonzero(mask[hh, i])), lay_o, heads)
    mx, mean = attention_error(f32(out_p), want)
    assert mx <= ATT_MAX_ABS and mean <= ATT_MEAN_ABS, (mx, mean)
    assert float((out_p.float() - out_s.float()).abs().max()) <= ATT_MAX_ABS
