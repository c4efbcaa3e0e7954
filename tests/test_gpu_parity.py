"""GPU parity of every stage against the CPU oracle on small workloads (several tiles, ragged tails,
padding, global rows, references, per-head boxes, head_dim 64 and 128). Calls go through the C ABI."""
import numpy as np
import pytest
import torch

import oracle as O
from learned_block_sparse_tile_b200 import _lib as L
from learned_block_sparse_tile_b200 import build as B

from gpu_util import (ATT_MAX_ABS, ATT_MEAN_ABS, POOL_ABS, POOL_REL, SCORE_REL, Case, attention_error,
                      compare_lists, f32, gpu_lists, oracle_kept, plant_signed_zero_cuts)

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


@pytest.mark.parametrize("name", SMALL)
def test_stages_match_oracle(name):
    c = case(name)
    wl = c.wl
    out = torch.full((wl.seq_len, wl.heads, wl.dim), 7.0, dtype=torch.bfloat16, device="cuda")
    want_out = np.full((wl.seq_len, wl.heads, wl.dim), np.nan)
    q, k, v = f32(c.q), f32(c.k), f32(c.v)
    for box, heads in c.groups:
        res = c.run_group(box, heads, out)
        lay_o = O.build_layout(c.spans_oracle(box), wl.seq_len)
        # gather: bit exact, head-major
        for key, x in (("q_t", q), ("k_t", k), ("v_t", v)):
            got = f32(res[key]).transpose(1, 0, 2)
            assert np.array_equal(got, O.gather(x, lay_o, heads)), key
        # pool: max/min exact, mean to fp32 rounding
        for key, x in (("fq", q), ("fk", k)):
            want = O.pool(O.gather(x, lay_o, heads), lay_o)
            got = f32(res[key]).astype(np.float64)
            D = wl.dim
            assert np.array_equal(got[..., D:], want[..., D:]), key
            assert np.all(np.abs(got[..., :D] - want[..., :D]) <= POOL_ABS + POOL_REL * np.abs(want[..., :D])), key
        # score: on the GPU's own features, against float64 logits
        fq, fk = f32(res["fq"]), f32(res["fk"])
        want_s = O.logits(fq, fk, f32(c.pq[heads]), f32(c.pk[heads]))
        got_s = f32(res["scores"])
        for h in range(len(heads)):
            assert np.abs(got_s[h] - want_s[h]).max() <= SCORE_REL * np.abs(want_s[h]).max()
        # select: bit exact on identical scores
        blocks = O.column_blocks(lay_o, wl.generated, wl.reference)
        kept, mask = oracle_kept(lay_o, got_s, blocks)
        compare_lists(res, mask, lay_o)
        # attend: the oracle on the same kept sets
        qt, kt, vt = (O.gather(x, lay_o, heads) for x in (q, k, v))
        o_t = O.attend_tiles(qt, kt, vt, lay_o, lambda hh, i: np.flatnonzero(mask[hh, i]))
        O.scatter(want_out, o_t, lay_o, heads)
    got = f32(out)
    assert not np.isnan(want_out).any()
    mx, mean = attention_error(got, want_out)
    assert mx <= ATT_MAX_ABS and mean <= ATT_MEAN_ABS, (mx, mean)


def test_keeps_all_equals_dense_attention():
    c = case("small_dense")
    wl = c.wl
    out = torch.full((wl.seq_len, wl.heads, wl.dim), 7.0, dtype=torch.bfloat16, device="cuda")
    for box, heads in c.groups:
        c.run_group(box, heads, out)
    want = O.dense_attention(f32(c.q), f32(c.k), f32(c.v))
    mx, mean = attention_error(f32(out), want)
    assert mx <= ATT_MAX_ABS and mean <= ATT_MEAN_ABS, (mx, mean)


def test_select_on_adversarial_scores():
    # ties, NaN, -inf and +inf scores through the C ABI: lists equal the oracle's bit for bit
    c = case("small_mixed")
    wl = c.wl
    box, heads = c.groups[0]
    res = c.run_group(box, heads)
    lay = res["layout"]
    lay_o = O.build_layout(c.spans_oracle(box), wl.seq_len)
    rng = np.random.default_rng(5)
    s = np.round(rng.standard_normal((len(heads), lay.n_video, lay.n_video)) * 2).astype(np.float32)
    s[0, 1, :5] = np.nan
    s[0, 2, 3] = np.inf
    s[0, 3, 4:9] = -np.inf
    s[-1, :, 0] = 3.0
    blocks = O.column_blocks(lay_o, wl.generated, wl.reference)
    # rows whose cut falls inside a run of -0.0 / +0.0 scores, in both column blocks
    plant_signed_zero_cuts(s, lay_o, blocks, rows=range(4, lay.n_video, 3))
    scores = torch.from_numpy(s).cuda()
    L.veda_select(lay, scores, res["kept_idx"], res["kept_cnt"])
    assert L.veda_sync_status() == L.VEDA_OK
    _, mask = oracle_kept(lay_o, s, blocks)
    compare_lists(res, mask, lay_o)


def test_empty_lists_give_zero_rows_and_head_order_is_free():
    c = case("padded_tiny")
    wl = c.wl
    box, heads = c.groups[0]
    res = c.run_group(box, list(reversed(heads)))  # heads [1, 0]
    lay = res["layout"]
    cnt = res["kept_cnt"].clone()
    cnt[:, 0] = 0  # video query tile 0 keeps nothing
    out = torch.full((wl.seq_len, wl.heads, wl.dim), 7.0, dtype=torch.bfloat16, device="cuda")
    L.veda_attend(lay, res["q_t"], res["k_t"], res["v_t"], res["kept_idx"], cnt, out, res["heads"])
    assert L.veda_sync_status() == L.VEDA_OK
    perm, _, _ = L.veda_layout_export(lay)
    rows0 = perm[:128][perm[:128] >= 0]
    assert (f32(out)[rows0] == 0).all()
    # every other row agrees with the normal run
    other = np.setdiff1d(np.arange(wl.seq_len), rows0)
    assert np.array_equal(f32(out)[other], f32(res["out"])[other])


def test_malformed_lists_are_reported_not_faulted():
    c = case("tiny")
    box, heads = c.groups[0]
    res = c.run_group(box, heads)
    lay = res["layout"]
    for mutate in ("range", "order", "count"):
        idx, cnt = res["kept_idx"].clone(), res["kept_cnt"].clone()
        if mutate == "range":
            idx[0, 3, 1] = lay.n_tiles + 5
        elif mutate == "order":
            idx[1, 2, 2] = idx[1, 2, 1]
        else:
            cnt[0, 0] = lay.max_kept + 3
        out = torch.zeros((c.wl.seq_len, c.wl.heads, c.wl.dim), dtype=torch.bfloat16, device="cuda")
        L.veda_attend(lay, res["q_t"], res["k_t"], res["v_t"], idx, cnt, out, res["heads"])
        assert L.veda_sync_status() == L.VEDA_ERR_BAD_LIST, mutate
    assert L.veda_sync_status() == L.VEDA_OK  # the word was cleared


def test_bad_arguments_rejected_on_host():
    c = case("tiny")
    box, heads = c.groups[0]
    res = c.run_group(box, heads)
    lay = res["layout"]
    with pytest.raises(L.VedaError):  # D stride not 1
        L.veda_gather(lay, c.dq.transpose(1, 2), res["heads"], res["q_t"], None)
    with pytest.raises(L.VedaError):  # workspace too small
        L.veda_score(lay, res["fq"], res["fk"], c.pq[heads].cuda(), c.pk[heads].cuda(),
                     torch.empty(4, device="cuda"), res["scores"])


def test_fp8_qk_variant():
    # quantiser: scales and codes equal to the oracle's reading bit for bit;
    # attention: against the oracle's FP8 reading (tight) and against unquantised attention (5e-2)
    c = case("small_d128")
    wl = c.wl
    q, k, v = f32(c.q), f32(c.k), f32(c.v)
    out = torch.full((wl.seq_len, wl.heads, wl.dim), 7.0, dtype=torch.bfloat16, device="cuda")
    want_fp8 = np.full(out.shape, np.nan)
    want_ref = np.full(out.shape, np.nan)
    for box, heads in c.groups:
        res = c.run_group(box, heads)
        lay = res["layout"]
        lay_o = O.build_layout(c.spans_oracle(box), wl.seq_len)
        n = len(heads)
        q8 = torch.empty(n, lay.n_slots, wl.dim, dtype=torch.uint8, device="cuda")
        k8 = torch.empty_like(q8)
        sq = torch.empty(n, lay.n_tiles, dtype=torch.float32, device="cuda")
        sk = torch.empty_like(sq)
        L.veda_quantize_fp8(lay, res["q_t"], q8, sq)
        L.veda_quantize_fp8(lay, res["k_t"], k8, sk)
        L.veda_attend_fp8(lay, q8, k8, sq, sk, res["v_t"], res["kept_idx"], res["kept_cnt"], out, res["heads"])
        assert L.veda_sync_status() == L.VEDA_OK, L.veda_last_error()
        qt, kt, vt = (O.gather(x, lay_o, heads) for x in (q, k, v))
        for x_t, codes, scales in ((qt, q8, sq), (kt, k8, sk)):
            want_codes, want_scales = O.quantize_fp8_tiles(x_t, lay_o)
            assert np.array_equal(f32(scales).astype(np.float64), want_scales)
            got_codes = codes.view(torch.float8_e4m3fn).float().cpu().numpy().transpose(1, 0, 2)
            assert np.array_equal(got_codes, want_codes)
        _, mask = oracle_kept(lay_o, f32(res["scores"]), O.column_blocks(lay_o, wl.generated, wl.reference))
        lists = lambda hh, i: np.flatnonzero(mask[hh, i])
        O.scatter(want_fp8, O.attend_tiles_fp8(qt, kt, vt, lay_o, lists), lay_o, heads)
        O.scatter(want_ref, O.attend_tiles(qt, kt, vt, lay_o, lists), lay_o, heads)
    got = f32(out)
    mx, mean = attention_error(got, want_fp8)
    assert mx <= ATT_MAX_ABS and mean <= ATT_MEAN_ABS, (mx, mean)
    # against unquantised attention the kernel adds nothing beyond the reading's own quantisation error
    mx, _ = attention_error(got, want_ref)
    q_err, _ = attention_error(want_fp8, want_ref)
    assert mx <= q_err + ATT_MAX_ABS, (mx, q_err)


@pytest.mark.parametrize("name", ["small_d128", "padded_tiny", "small_mixed"])
def test_fused_fp8_gather(name):
    # gather straight to e4m3 codes: codes and scales equal the two-pass path (gather, then quantise) and
    # the oracle's reading bit for bit, on head_dim 128 and 64, padded tiles and global tiles; the pooled
    # features equal the bf16 gather's
    c = case(name)
    wl = c.wl
    for box, heads in c.groups:
        res = c.run_group(box, heads)
        lay = res["layout"]
        lay_o = O.build_layout(c.spans_oracle(box), wl.seq_len)
        n = len(heads)
        for x, x_t, f_ref in ((c.dq, res["q_t"], res["fq"]), (c.dk, res["k_t"], res["fk"])):
            codes = torch.full((n, lay.n_slots, wl.dim), 0x55, dtype=torch.uint8, device="cuda")
            scales = torch.full((n, lay.n_tiles), -1.0, dtype=torch.float32, device="cuda")
            feats = torch.full_like(f_ref, float("nan"))
            L.veda_gather_fp8(lay, x, res["heads"], codes, scales, feats)
            codes2, scales2 = torch.empty_like(codes), torch.empty_like(scales)
            L.veda_quantize_fp8(lay, x_t, codes2, scales2)
            assert L.veda_sync_status() == L.VEDA_OK, L.veda_last_error()
            assert torch.equal(codes, codes2) and torch.equal(scales, scales2)
            assert torch.equal(feats, f_ref)
            want_codes, want_scales = O.quantize_fp8_tiles(O.gather(f32(x), lay_o, heads), lay_o)
            assert np.array_equal(f32(scales).astype(np.float64), want_scales)
            got = codes.view(torch.float8_e4m3fn).float().cpu().numpy().transpose(1, 0, 2)
            assert np.array_equal(got, want_codes)


def _bf16(x):
    """float64 values that are exactly bf16 -> bf16 bit patterns (uint16)."""
    b = np.asarray(x, dtype=np.float32).view(np.uint32)
    assert np.all(b & 0xFFFF == 0), "value not representable in bf16"
    return (b >> 16).astype(np.uint16)


def _midpoint_tile(rng, mode, D):
    """One 128 x D tile of bf16 bits whose quotients by the tile's fp32 scale sit on e4m3 rounding
    midpoints. mode 'near': amax has at most 6 significant bits and is not a multiple of 7, so
    amax / 448 is inexact in fp32; x = 3 amax 2^(j-9) is exact in bf16 and x / (amax / 448) is exactly the
    midpoint 2.625 2^j (and amax 2^-16 gives the subnormal midpoint 7 2^-10): the rounding of the stored
    scale alone moves x / s off the midpoint, by less than one fp32 ulp. mode 'tie': the scale is a power of
    two and every e4m3 midpoint times it is exact, so x / s is exactly a midpoint (ties to even)."""
    vals = np.array([float(v) for v in torch.arange(127, dtype=torch.uint8).view(torch.float8_e4m3fn).float()])
    mids = (vals[:-1] + vals[1:]) / 2
    if mode == "near":
        amax = float(rng.choice([13.0, 5.75, 27.5, 1.5, 0.8125, 19.0, 43.0, 2.75]))
        xs = np.concatenate([3 * amax * 2.0 ** (np.arange(-6, 8) - 9), [amax * 2.0 ** -16]])
    else:
        k = int(rng.integers(1, 6))
        amax = 448.0 * 2.0 ** -k
        xs = mids * 2.0 ** -k
    xs = xs[xs < amax]
    bits = _bf16(np.concatenate([xs, -xs]))
    tile = rng.choice(bits, size=(128, D))
    tile[0, 0] = _bf16([amax])[0]
    return tile


def test_fp8_codes_at_rounding_midpoints():
    # quotients within one fp32 ulp of (or exactly on) e4m3 rounding midpoints: the quantiser's
    # round-to-odd quotient must round like the exact quotient. Standalone quantiser and fused gather,
    # against the oracle bit for bit.
    c = case("padded_tiny")
    wl = c.wl
    box, heads = c.groups[0]
    lay = c.run_group(box, heads)["layout"]
    lay_o = O.build_layout(c.spans_oracle(box), wl.seq_len)
    D, N = wl.dim, lay.n_slots
    rng = np.random.default_rng(11)
    bits = np.zeros((N, D), dtype=np.uint16)
    for i in range(lay.n_tiles):
        tile = _midpoint_tile(rng, "near" if i % 3 else "tie", D)
        tile[int(lay_o.valid_count[i]):] = 0  # padding slots are zero
        bits[i * 128:(i + 1) * 128] = tile
    x_t = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).reshape(1, N, D).cuda()
    codes = torch.empty(1, N, D, dtype=torch.uint8, device="cuda")
    scales = torch.empty(1, lay.n_tiles, dtype=torch.float32, device="cuda")
    L.veda_quantize_fp8(lay, x_t, codes, scales)
    # the same tiles through the fused gather: scatter them back to packed rows first
    perm = lay_o.perm
    real = np.flatnonzero(perm >= 0)
    x = torch.zeros(wl.seq_len, 1, D, dtype=torch.bfloat16)
    x[torch.from_numpy(perm[real]).long(), 0] = x_t[0].cpu()[torch.from_numpy(real).long()]
    codes_g, scales_g = torch.empty_like(codes), torch.empty_like(scales)
    L.veda_gather_fp8(lay, x.cuda(), torch.zeros(1, dtype=torch.int32, device="cuda"), codes_g, scales_g)
    assert L.veda_sync_status() == L.VEDA_OK, L.veda_last_error()
    want_codes, want_scales = O.quantize_fp8_tiles(f32(x_t).transpose(1, 0, 2), lay_o)
    for cd, sc in ((codes, scales), (codes_g, scales_g)):
        assert np.array_equal(f32(sc).astype(np.float64), want_scales)
        got = cd.view(torch.float8_e4m3fn).float().cpu().numpy().transpose(1, 0, 2)
        assert np.array_equal(got, want_codes), int((got != want_codes).sum())


def test_select_two_blocks_beyond_2048_video_tiles():
    # a reference block of 1100 tiles and a target block of 1000: rows of 2100 video tiles, each block
    # narrow enough for the warp-per-row select that keeps one block in registers; cuts inside runs of
    # signed zeros and exact ties, bit for bit against the oracle
    spans = [(0, (1, 8, 16 * 1100), (1, 8, 16)), (128 * 1100, (1, 8, 16 * 1000), (1, 8, 16))]
    seq_len = 128 * 2100
    gen, ref = (0.05, None), (0.02, None)
    lay = L.veda_plan(spans, seq_len, gen, ref)
    lay_o = O.build_layout(spans, seq_len)
    assert lay.n_video == 2100 and lay.n_ref == 1100
    rng = np.random.default_rng(2100)
    s = np.round(rng.standard_normal((1, 2100, 2100)) * 3).astype(np.float32)
    s[0, ::3, rng.integers(0, 2100, 5)] = np.nan
    blocks = O.column_blocks(lay_o, gen, ref)
    plant_signed_zero_cuts(s, lay_o, blocks, rows=range(2, 2100, 23))
    idx = torch.full((1, 2100, lay.max_kept), -7, dtype=torch.int32, device="cuda")
    cnt = torch.empty(1, 2100, dtype=torch.int32, device="cuda")
    L.veda_select(lay, torch.from_numpy(s).cuda(), idx, cnt)
    assert L.veda_sync_status() == L.VEDA_OK, L.veda_last_error()
    _, mask = oracle_kept(lay_o, s, blocks)
    compare_lists(dict(kept_idx=idx, kept_cnt=cnt), mask, lay_o)


@pytest.mark.parametrize("width", [512, 513, 1024, 2048, 2049])
def test_select_block_widths(width):
    # one video span of exactly `width` tiles: the persistent warp-per-row select at the edges of its
    # register tiers (16 / 32 / 64 slots per lane) and the CTA-per-row select beyond 2048 columns; scores with
    # many ties, -inf, NaN and cuts inside runs of signed zeros, bit for bit against the oracle
    spans = [(0, (1, 8, 16 * width), (1, 8, 16))]
    seq_len = 128 * width
    gen, ref = (0.1, None), (1.0, None)
    lay = L.veda_plan(spans, seq_len, gen, ref)
    lay_o = O.build_layout(spans, seq_len)
    assert lay.n_video == width
    rng = np.random.default_rng(width)
    s = np.round(rng.standard_normal((1, width, width)) * 3).astype(np.float32)  # small integers: ties
    s[0, :, rng.integers(0, width, 7)] = -np.inf
    s[0, ::5, rng.integers(0, width, 3)] = np.nan
    # rows whose cut falls inside a run of -0.0 / +0.0 scores
    plant_signed_zero_cuts(s, lay_o, O.column_blocks(lay_o, gen, ref), rows=range(1, width, 17))
    scores = torch.from_numpy(s).cuda()
    idx = torch.full((1, width, lay.max_kept), -7, dtype=torch.int32, device="cuda")
    cnt = torch.empty(1, width, dtype=torch.int32, device="cuda")
    L.veda_select(lay, scores, idx, cnt)
    assert L.veda_sync_status() == L.VEDA_OK, L.veda_last_error()
    _, mask = oracle_kept(lay_o, s, O.column_blocks(lay_o, gen, ref))
    compare_lists(dict(kept_idx=idx, kept_cnt=cnt), mask, lay_o)


def test_int8_qk_variant():
    # quantiser (standalone and fused into the gather): scales and codes equal the oracle's INT8 reading bit
    # for bit; attention: against the oracle's INT8 reading (bf16 tolerance) and against unquantised
    # attention (no worse than the reading's own quantisation error plus that tolerance)
    c = case("small_d128")
    wl = c.wl
    q, k, v = f32(c.q), f32(c.k), f32(c.v)
    out = torch.full((wl.seq_len, wl.heads, wl.dim), 7.0, dtype=torch.bfloat16, device="cuda")
    want_i8 = np.full(out.shape, np.nan)
    want_ref = np.full(out.shape, np.nan)
    for box, heads in c.groups:
        res = c.run_group(box, heads)
        lay = res["layout"]
        lay_o = O.build_layout(c.spans_oracle(box), wl.seq_len)
        n = len(heads)
        q8 = torch.empty(n, lay.n_slots, wl.dim, dtype=torch.int8, device="cuda")
        k8, q8g = torch.empty_like(q8), torch.empty_like(q8)
        sq = torch.empty(n, lay.n_tiles, dtype=torch.float32, device="cuda")
        sk, sqg = torch.empty_like(sq), torch.empty_like(sq)
        L.veda_quantize_int8(lay, res["q_t"], q8, sq)
        L.veda_quantize_int8(lay, res["k_t"], k8, sk)
        L.veda_gather_int8(lay, c.dq, res["heads"], q8g, sqg)
        L.veda_attend_int8(lay, q8, k8, sq, sk, res["v_t"], res["kept_idx"], res["kept_cnt"], out, res["heads"])
        assert L.veda_sync_status() == L.VEDA_OK, L.veda_last_error()
        assert torch.equal(q8, q8g) and torch.equal(sq, sqg)
        qt, kt, vt = (O.gather(x, lay_o, heads) for x in (q, k, v))
        for x_t, codes, scales in ((qt, q8, sq), (kt, k8, sk)):
            want_codes, want_scales = O.quantize_int8_tiles(x_t, lay_o)
            assert np.array_equal(f32(scales).astype(np.float64), want_scales)
            assert np.array_equal(codes.cpu().numpy().astype(np.float64).transpose(1, 0, 2), want_codes)
        _, mask = oracle_kept(lay_o, f32(res["scores"]), O.column_blocks(lay_o, wl.generated, wl.reference))
        lists = lambda hh, i: np.flatnonzero(mask[hh, i])
        O.scatter(want_i8, O.attend_tiles_int8(qt, kt, vt, lay_o, lists), lay_o, heads)
        O.scatter(want_ref, O.attend_tiles(qt, kt, vt, lay_o, lists), lay_o, heads)
    got = f32(out)
    mx, mean = attention_error(got, want_i8)
    assert mx <= ATT_MAX_ABS and mean <= ATT_MEAN_ABS, (mx, mean)
    mx, _ = attention_error(got, want_ref)
    q_err, _ = attention_error(want_i8, want_ref)
    assert mx <= q_err + ATT_MAX_ABS, (mx, q_err)


def _int8_midpoint_tile(rng, mode, D):
    """Tile of bf16 bits whose quotients by the tile's fp32 scale sit on integer rounding midpoints. 'tie':
    the scale is a power of two (amax = 127 2^-k) and x = (j + 1/2) 2^-k, so x / s is exactly j + 1/2.
    'near': amax has at most 6 significant bits, so x = amax / 2 is exact in bf16 and x / (amax / 127) is
    exactly 63.5; the fp32 rounding of the stored scale alone moves x / s off it (127 is prime, so
    amax / 127 is never exact in fp32 for these amax)."""
    if mode == "tie":
        k = int(rng.integers(1, 8))
        amax = 127.0 * 2.0 ** -k
        xs = (np.arange(127) + 0.5) * 2.0 ** -k
    else:
        amax = float(rng.choice([13.0, 5.75, 27.5, 1.5, 0.8125, 19.0, 43.0, 2.75]))
        xs = np.array([amax / 2, amax / 4, 3 * amax / 8])
    bits = _bf16(np.concatenate([xs, -xs]))
    tile = rng.choice(bits, size=(128, D))
    tile[0, 0] = _bf16([amax])[0]
    return tile


def test_int8_codes_at_rounding_midpoints():
    c = case("padded_tiny")
    wl = c.wl
    box, heads = c.groups[0]
    lay = c.run_group(box, heads)["layout"]
    lay_o = O.build_layout(c.spans_oracle(box), wl.seq_len)
    D, N = wl.dim, lay.n_slots
    rng = np.random.default_rng(12)
    bits = np.zeros((N, D), dtype=np.uint16)
    for i in range(lay.n_tiles):
        tile = _int8_midpoint_tile(rng, "near" if i % 2 else "tie", D)
        tile[int(lay_o.valid_count[i]):] = 0
        bits[i * 128:(i + 1) * 128] = tile
    x_t = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).reshape(1, N, D).cuda()
    codes = torch.empty(1, N, D, dtype=torch.int8, device="cuda")
    scales = torch.empty(1, lay.n_tiles, dtype=torch.float32, device="cuda")
    L.veda_quantize_int8(lay, x_t, codes, scales)
    perm = lay_o.perm
    real = np.flatnonzero(perm >= 0)
    x = torch.zeros(wl.seq_len, 1, D, dtype=torch.bfloat16)
    x[torch.from_numpy(perm[real]).long(), 0] = x_t[0].cpu()[torch.from_numpy(real).long()]
    codes_g, scales_g = torch.empty_like(codes), torch.empty_like(scales)
    L.veda_gather_int8(lay, x.cuda(), torch.zeros(1, dtype=torch.int32, device="cuda"), codes_g, scales_g)
    assert L.veda_sync_status() == L.VEDA_OK, L.veda_last_error()
    want_codes, want_scales = O.quantize_int8_tiles(f32(x_t).transpose(1, 0, 2), lay_o)
    for cd, sc in ((codes, scales), (codes_g, scales_g)):
        assert np.array_equal(f32(sc).astype(np.float64), want_scales)
        got = cd.cpu().numpy().astype(np.float64).transpose(1, 0, 2)
        assert np.array_equal(got, want_codes), int((got != want_codes).sum())


@pytest.mark.parametrize("name", SMALL)
def test_gather_free_attend(name):
    # veda_pool gives veda_gather's features bit for bit; veda_attend_direct, on the packed tensors and the
    # same lists, matches the oracle within the bf16 tolerance and the tile-order attend within rounding
    # (identical where every tile is a full box: the keys then come in the same order)
    c = case(name)
    wl = c.wl
    groups = c.groups
    q, k, v = f32(c.q), f32(c.k), f32(c.v)
    out_t = torch.full((wl.seq_len, wl.heads, wl.dim), 7.0, dtype=torch.bfloat16, device="cuda")
    out_d = out_t.clone()
    want_out = np.zeros((wl.seq_len, wl.heads, wl.dim), np.float64)
    all_full = True
    for box, heads in groups:
        res = c.run_group(box, heads, out_t)
        lay = res["layout"]
        fq = torch.empty_like(res["fq"])
        L.veda_pool(lay, c.dq, res["heads"], fq)
        L.veda_attend_direct(lay, c.dq, c.dk, c.dv, res["kept_idx"], res["kept_cnt"], out_d, res["heads"])
        assert L.veda_sync_status() == L.VEDA_OK, L.veda_last_error()
        assert torch.equal(fq, res["fq"])
        lay_o = O.build_layout(c.spans_oracle(box), wl.seq_len)
        all_full &= bool((lay_o.valid_count == 128).all())
        _, mask = oracle_kept(lay_o, f32(res["scores"]), O.column_blocks(lay_o, wl.generated, wl.reference))
        qt, kt, vt = (O.gather(x, lay_o, heads) for x in (q, k, v))
        o_t = O.attend_tiles(qt, kt, vt, lay_o, lambda hh, i: np.flatnonzero(mask[hh, i]))
        O.scatter(want_out, o_t, lay_o, heads)
    got = f32(out_d)
    mx, mean = attention_error(got, want_out)
    assert mx <= ATT_MAX_ABS and mean <= ATT_MEAN_ABS, (mx, mean)
    diff = np.abs(got - f32(out_t)).max()
    if all_full:
        assert diff == 0.0, diff
    else:
        assert diff <= ATT_MAX_ABS, diff


def test_gather_free_attend_rejects_layouts_without_boxes():
    lay = L.veda_plan([(100, (1, 8, 16), None)], 400, (0.5, None), (1.0, None))
    x = torch.zeros(400, 1, 64, dtype=torch.bfloat16, device="cuda")
    heads = torch.zeros(1, dtype=torch.int32, device="cuda")
    idx = torch.zeros(1, 1, lay.max_kept, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(1, 1, dtype=torch.int32, device="cuda")
    with pytest.raises(L.VedaError) as e:
        L.veda_attend_direct(lay, x, x, x, idx, cnt, x.clone(), heads)
    assert e.value.code == L.VEDA_ERR_UNSUPPORTED


@pytest.mark.parametrize("name", ["small_mixed", "small_d128"])
@pytest.mark.parametrize("direct", [False, True])
def test_strided_views_match_contiguous(name, direct):
    # Q/K/V and the output as views (a head slice of a wider tensor; a head-major tensor seen as [S, H, D])
    # give bit for bit the outputs of contiguous tensors, on both attend paths; the output's other heads
    # are left untouched
    from learned_block_sparse_tile_b200 import VedaLayer
    c = case(name)
    wl = c.wl
    S, H, D = wl.seq_len, wl.heads, wl.dim
    layer = VedaLayer(S, wl.ref_spans, wl.target, wl.head_shapes, (wl.generated, wl.reference), H, D, direct=direct)
    layer.set_projections(c.pq, c.pk)
    assert layer.direct == direct
    want = torch.zeros(S, H, D, dtype=torch.bfloat16, device="cuda")
    layer.forward(c.dq, c.dk, c.dv, want)

    def wide(x):  # [S, H + 8, D] holding x in heads [0, H)
        w = torch.full((S, H + 8, D), 3.0, dtype=x.dtype, device=x.device)
        w[:, :H] = x
        return w[:, :H]

    def head_major(x):  # storage [H, S, D], viewed as [S, H, D]
        return x.permute(1, 0, 2).contiguous().permute(1, 0, 2)

    for view in (wide, head_major):
        q, k, v = view(c.dq), view(c.dk), view(c.dv)
        assert not q.is_contiguous()
        out_wide = torch.full((S, H + 8, D), 5.0, dtype=torch.bfloat16, device="cuda")
        layer.forward(q, k, v, out_wide[:, :H])
        assert L.veda_sync_status() == L.VEDA_OK, L.veda_last_error()
        assert torch.equal(out_wide[:, :H], want), view.__name__
        assert bool((out_wide[:, H:] == 5.0).all())


@pytest.mark.parametrize("name", SMALL)
@pytest.mark.parametrize("q_scale", [1.0, 16.0])
def test_logit_bound(name, q_scale):
    # veda_pool and veda_gather write ||q||^2 per packed row and the largest ||k||^2 per head (compared with
    # float64 norms of the same bf16 values); with them the attend may skip the row max on an item's later
    # tiles, which is the same softmax: both attend paths stay within the tolerance of the oracle. q_scale 16
    # (exact in bf16) widens the gap between the bound and the first tile's maxima past the limit on most
    # warps, so those take the exact per-tile maxima instead.
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
        row_sq = torch.full((n, wl.seq_len), -1.0, device="cuda")
        max_sq = torch.full((n,), -1.0, device="cuda")
        fq, fk = torch.empty_like(res["fq"]), torch.empty_like(res["fk"])
        L.veda_pool(lay, qs, res["heads"], fq, row_sq=row_sq)
        L.veda_pool(lay, c.dk, res["heads"], fk, max_sq=max_sq)
        # the tile-order path's gather writes the same norms
        q_t, k_t = torch.empty_like(res["q_t"]), torch.empty_like(res["k_t"])
        row_sq_g, max_sq_g = torch.full_like(row_sq, -1.0), torch.full_like(max_sq, -1.0)
        L.veda_gather(lay, qs, res["heads"], q_t, None, row_sq=row_sq_g)
        L.veda_gather(lay, c.dk, res["heads"], k_t, None, max_sq=max_sq_g)
        assert L.veda_sync_status() == L.VEDA_OK, L.veda_last_error()
        want_q = (q[:, heads, :].astype(np.float64) ** 2).sum(-1).T  # [n, S]
        want_k = (k[:, heads, :].astype(np.float64) ** 2).sum(-1).max(0)  # [n]
        for got in (row_sq, row_sq_g):
            assert np.allclose(f32(got), want_q, rtol=1e-5, atol=0)
        for got in (max_sq, max_sq_g):
            assert np.allclose(f32(got), want_k, rtol=1e-5, atol=0)
        assert torch.equal(row_sq, row_sq_g) and torch.equal(max_sq, max_sq_g)
        L.veda_attend_direct(lay, qs, c.dk, c.dv, res["kept_idx"], res["kept_cnt"], out_d, res["heads"],
                             q_row_sq=row_sq, k_max_sq=max_sq)
        L.veda_attend(lay, q_t, k_t, res["v_t"], res["kept_idx"], res["kept_cnt"], out_t, res["heads"],
                      q_row_sq=row_sq_g, k_max_sq=max_sq_g)
        assert L.veda_sync_status() == L.VEDA_OK, L.veda_last_error()
        lay_o = O.build_layout(c.spans_oracle(box), wl.seq_len)
        _, mask = oracle_kept(lay_o, f32(res["scores"]), O.column_blocks(lay_o, wl.generated, wl.reference))
        qt, kt, vt = (O.gather(x, lay_o, heads) for x in (q, k, v))
        O.scatter(want, O.attend_tiles(qt, kt, vt, lay_o, lambda hh, i: np.flatnonzero(mask[hh, i])), lay_o, heads)
    for out in (out_d, out_t):
        mx, mean = attention_error(f32(out), want)
        assert mx <= ATT_MAX_ABS and mean <= ATT_MEAN_ABS, (mx, mean)
