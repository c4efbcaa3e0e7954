"""Helpers shared by the GPU parity tests: run one head group through the C ABI and through the oracle."""
import numpy as np
import torch

import oracle as O
import veda_synth as V
from learned_block_sparse_tile_b200 import _lib as L

# tolerances (bf16 inputs, fp32 accumulation, compared with the float64 oracle before its bf16 cast)
ATT_MAX_ABS, ATT_MEAN_ABS = 2e-2, 2e-3
SCORE_REL = 1e-5  # |gpu - oracle| <= SCORE_REL * max|scores| per head
POOL_ABS, POOL_REL = 2e-6, 2e-6


def f32(t):
    return t.float().cpu().numpy()


class Case:
    """Inputs of one workload on the host and the device."""

    def __init__(self, name):
        self.wl = V.workload(name)
        self.q, self.k, self.v = V.make_qkv(self.wl)
        self.pq, self.pk = V.make_projections(self.wl)
        self.lps = O.least_padding_shape(self.wl.target[1])
        self.groups = V.head_groups(self.wl, lambda _: self.lps)
        self.dq, self.dk, self.dv = self.q.cuda(), self.k.cuda(), self.v.cuda()
        self.tile_refs = not O.keeps_all(self.wl.reference)

    def spans_oracle(self, box):
        return O.layer_spans(self.wl.ref_spans, (self.wl.target[0], self.wl.target[1], box), self.tile_refs)

    def run_group(self, box, heads, out=None):
        """All device stages for one group; returns a dict of host copies plus the layout."""
        wl = self.wl
        spans_c = [(s, g, None) for s, g in wl.ref_spans] + [(wl.target[0], wl.target[1], box)]
        lay = L.veda_plan(spans_c, wl.seq_len, wl.generated, wl.reference)
        n, D, dev = len(heads), wl.dim, "cuda"
        hd = torch.tensor(heads, dtype=torch.int32, device=dev)
        q_t = torch.empty(n, lay.n_slots, D, dtype=torch.bfloat16, device=dev)
        k_t, v_t = torch.empty_like(q_t), torch.empty_like(q_t)
        fq = torch.empty(n, lay.n_video, 3 * D, dtype=torch.float32, device=dev)
        fk = torch.empty_like(fq)
        L.veda_gather(lay, self.dq, hd, q_t, fq)
        L.veda_gather(lay, self.dk, hd, k_t, fk)
        L.veda_gather(lay, self.dv, hd, v_t, None)
        pq = self.pq[heads].cuda().contiguous()
        pk = self.pk[heads].cuda().contiguous()
        ws = torch.empty(L.veda_score_workspace_bytes(lay, n, D) // 4, dtype=torch.float32, device=dev)
        scores = torch.empty(n, lay.n_video, lay.n_video, dtype=torch.float32, device=dev)
        L.veda_score(lay, fq, fk, pq, pk, ws, scores)
        kept_idx = torch.full((n, lay.n_video, lay.max_kept), -7, dtype=torch.int32, device=dev)
        kept_cnt = torch.empty(n, lay.n_video, dtype=torch.int32, device=dev)
        L.veda_select(lay, scores, kept_idx, kept_cnt)
        if out is None:
            out = torch.full((wl.seq_len, wl.heads, D), 7.0, dtype=torch.bfloat16, device=dev)
        L.veda_attend(lay, q_t, k_t, v_t, kept_idx, kept_cnt, out, hd)
        rc = L.veda_sync_status()
        assert rc == L.VEDA_OK, (rc, L.veda_last_error())
        return dict(layout=lay, q_t=q_t, k_t=k_t, v_t=v_t, fq=fq, fk=fk, scores=scores, kept_idx=kept_idx,
                    kept_cnt=kept_cnt, out=out, heads=hd)


def oracle_kept(lay_o, scores_np, blocks):
    """Oracle kept mask and its per-row index lists from given fp32 scores."""
    kept = O.select(scores_np, lay_o, blocks)
    mask = O.block_mask(kept, lay_o)
    return kept, mask


def gpu_lists(res):
    idx = res["kept_idx"].cpu().numpy()
    cnt = res["kept_cnt"].cpu().numpy()
    return idx, cnt


def compare_lists(res, mask, lay_o):
    """GPU kept lists (video rows) equal the oracle's mask rows, bit for bit."""
    idx, cnt = gpu_lists(res)
    nv = lay_o.n_video
    for h in range(idx.shape[0]):
        for r in range(nv):
            want = np.flatnonzero(mask[h, r])
            got = idx[h, r, :cnt[h, r]]
            if not np.array_equal(got, want):
                raise AssertionError(f"head {h} row {r}: got {got.tolist()} want {want.tolist()}")


def plant_signed_zero_cuts(s, lay_o, blocks, rows):
    """Rewrites rows of fp32 scores ``s`` [H, n_video, n_video] in place so that, in every non-keeps-all
    column block, the selection's cut falls inside a run of zeros of alternating sign: the row keeps its
    own tile (when the block holds it), the best columns, then the lowest-column zeros. Half of the rows
    start the run with -0.0, half with +0.0, so a selection that ranks +0.0 above -0.0 keeps other columns
    than the (score desc, column asc) order on IEEE comparison."""
    for blk in blocks:
        start, stop, budget, _ = blk
        if O.keeps_all(budget):
            continue
        allowed = O.allowed_per_row(lay_o, blk)
        for r in rows:
            cols = [c for c in range(start, stop) if lay_o.kv_ok[c] and c != r]
            free = int(allowed[r]) - (1 if start <= r < stop else 0)
            if free < 1 or len(cols) < free + 4:
                continue
            z = min(2, free)
            top, zeros, rest = cols[:free - z], cols[free - z:free - z + 6], cols[free - z + 6:]
            for h in range(s.shape[0]):
                s[h, r, top] = 50.0 + np.arange(len(top), dtype=np.float32)
                first_neg = (r + h) % 2 == 0
                s[h, r, zeros] = [(-0.0 if (i % 2 == 0) == first_neg else 0.0) for i in range(len(zeros))]
                s[h, r, rest] = -10.0 - np.arange(len(rest), dtype=np.float32)
    return s


def attention_error(got, want, valid_rows=None):
    d = np.abs(got.astype(np.float64) - want)
    if valid_rows is not None:
        d = d[valid_rows]
    return float(d.max()), float(d.mean())
