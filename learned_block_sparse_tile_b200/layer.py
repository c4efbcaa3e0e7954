"""One Veda attention layer on the C ABI (veda_core.py, "one layer", attention).

For each group of heads sharing a target tile box: plan (cached), gather Q and K to tile order with
pooling (straight to e4m3 codes and per-tile scales in the FP8 Q/K variant), score, select, gather V,
attend with the scatter fused. In the gather-free mode (``direct``) Q and K are only pooled and the attend
loads every tile as a TMA box of the packed tensors, so no tile-order copy is made. PyTorch only allocates
device buffers and supplies the stream; every step runs in libveda's kernels.
"""
from __future__ import annotations

import torch

from . import _lib as L


class VedaLayer:
    """Plans and buffers for one layer geometry.

    seq_len      packed rows S
    ref_spans    [(start, (t, h, w))] reference spans in packed order (tiled at their least-padding box
                 unless the reference budget keeps all)
    target       (start, (t, h, w)) the generated span (last)
    head_shapes  per head: a (t, h, w) box or None for the target's least-padding box
    budgets      (generated, reference), each a (ratio, tiles) pair with exactly one set
    direct       gather-free attend: pool Q and K, then veda_attend_direct on the packed tensors (no
                 tile-order copies). None (default): used when Q/K are bf16 and every group's layout has a
                 box form (veda_layout_export_direct); True: required (raises otherwise); False: the
                 tile-order path (veda_gather + veda_attend), which takes every layout
    logit_bound  the pool/gather of Q also writes ||q||^2 per row and that of K the largest ||k||^2 per
                 head, and the attend takes them as its logit bound (the single bf16 attend may then skip
                 the row max on an item's later tiles; the paired attend takes its softmax reference from
                 it; same softmax). Default True
    paired       with the logit bound: the paired attend (veda_attend_paired / veda_attend_direct_paired,
                 veda_attend_fp8_paired / veda_attend_int8_paired for the 8-bit Q/K), two neighbouring query
                 tiles per work item sharing each kept K/V tile load, the softmax reference fixed by the
                 bound, and an exact redo of any query tile the bound cannot serve. Default True; False
                 keeps the single-tile attend
    """

    # tile-order path: gather q, gather k, the projections' transpose, 2 score GEMMs, select, gather v, attend
    LAUNCHES_PER_GROUP = 8
    LAUNCHES_PER_GROUP_DIRECT = 7  # gather-free path: pool q, pool k, transpose, 2 score GEMMs, select, attend
    EXTRA_LAUNCHES_PAIRED = 2  # the paired attend adds the list merge and the (usually empty) redo pass

    def __init__(self, seq_len, ref_spans, target, head_shapes, budgets, heads, dim, device="cuda", fp8_qk=False,
                 int8_qk=False, direct=None, logit_bound=True, paired=True):
        self.seq_len, self.heads, self.dim = int(seq_len), int(heads), int(dim)
        if fp8_qk and int8_qk:
            raise ValueError("VedaLayer: choose one of fp8_qk and int8_qk")
        if direct and (fp8_qk or int8_qk):
            raise ValueError("VedaLayer: the gather-free attend reads bf16 Q/K")
        self.fp8_qk, self.int8_qk = bool(fp8_qk), bool(int8_qk)
        self.device = torch.device(device)
        lps = L.veda_least_padding_box(target[1])
        groups = {}
        for h, s in enumerate(head_shapes):
            groups.setdefault(tuple(lps if s is None else s), []).append(h)
        spans_ref = [(s, g, None) for s, g in ref_spans]
        layouts = {box: L.veda_plan(spans_ref + [(target[0], target[1], box)], seq_len, budgets[0], budgets[1])
                   for box in sorted(groups)}
        if direct is None:
            direct = not (fp8_qk or int8_qk) and all(L.veda_layout_has_box_form(x) for x in layouts.values())
        elif direct:
            for x in layouts.values():
                if not L.veda_layout_has_box_form(x):
                    L.veda_layout_export_direct(x)  # raises with the reason
        self.direct = bool(direct)
        self.logit_bound = bool(logit_bound)
        self.paired = bool(paired) and self.logit_bound
        # the 8-bit single-tile attend keeps exact per-tile maxima: its norms are needed only when paired
        norms = self.logit_bound and (self.paired or not (self.fp8_qk or self.int8_qk))
        self.groups = []
        for box in sorted(groups):
            lay = layouts[box]
            hs = groups[box]
            n = len(hs)
            dev = self.device
            g = dict(box=box, heads_list=hs, layout=lay,
                     heads=torch.tensor(hs, dtype=torch.int32, device=dev),
                     feats_q=torch.empty(n, lay.n_video, 3 * dim, dtype=torch.float32, device=dev),
                     feats_k=torch.empty(n, lay.n_video, 3 * dim, dtype=torch.float32, device=dev),
                     workspace=torch.empty(L.veda_score_workspace_bytes(lay, n, dim) // 4, dtype=torch.float32,
                                           device=dev),
                     scores=torch.empty(n, lay.n_video, lay.n_video, dtype=torch.float32, device=dev),
                     kept_idx=torch.empty(n, lay.n_video, lay.max_kept, dtype=torch.int32, device=dev),
                     kept_cnt=torch.empty(n, lay.n_video, dtype=torch.int32, device=dev))
            if self.fp8_qk or self.int8_qk:  # Q and K are gathered straight to 8-bit codes with per-tile scales
                code_t = torch.int8 if self.int8_qk else torch.uint8
                g.update(q8=torch.empty(n, lay.n_slots, dim, dtype=code_t, device=dev),
                         k8=torch.empty(n, lay.n_slots, dim, dtype=code_t, device=dev),
                         sq=torch.empty(n, lay.n_tiles, dtype=torch.float32, device=dev),
                         sk=torch.empty(n, lay.n_tiles, dtype=torch.float32, device=dev))
            elif not self.direct:
                g.update(q_t=torch.empty(n, lay.n_slots, dim, dtype=torch.bfloat16, device=dev),
                         k_t=torch.empty(n, lay.n_slots, dim, dtype=torch.bfloat16, device=dev))
            if not self.direct:
                g.update(v_t=torch.empty(n, lay.n_slots, dim, dtype=torch.bfloat16, device=dev))
            if norms:
                g.update(q_row_sq=torch.empty(n, self.seq_len, dtype=torch.float32, device=dev),
                         k_max_sq=torch.empty(n, dtype=torch.float32, device=dev))
            else:
                g.update(q_row_sq=None, k_max_sq=None)
            g.update(pair_ws=L.paired_workspace(lay, n, dev) if self.paired else None)
            self.groups.append(g)
        self.launches = ((self.LAUNCHES_PER_GROUP_DIRECT if self.direct else self.LAUNCHES_PER_GROUP) +
                         (self.EXTRA_LAUNCHES_PAIRED if self.paired else 0)) * len(self.groups)
        self._side = torch.cuda.Stream(self.device)  # the V gathers

    def set_projections(self, proj_q, proj_k):
        """proj_q, proj_k: fp32 [H, 3D, D] (any device); each group keeps its heads' slices on device."""
        for g in self.groups:
            idx = torch.tensor(g["heads_list"], dtype=torch.long)
            g["proj_q"] = proj_q.index_select(0, idx).to(self.device, torch.float32).contiguous()
            g["proj_k"] = proj_k.index_select(0, idx).to(self.device, torch.float32).contiguous()

    def kept_tiles(self):
        """Total kept (video query tile, key tile) pairs of the last forward, per the page's ``kept``."""
        return sum(int(g["kept_cnt"].sum()) - g["layout"].n_global_ok * g["kept_cnt"].numel() for g in self.groups)

    def work_tiles(self):
        """The page's ``work`` counter (kept video pairs + dense global rows and columns), all groups."""
        total = 0
        for g in self.groups:
            lay = g["layout"]
            n = len(g["heads_list"])
            kept_video = int(g["kept_cnt"].sum()) - lay.n_global_ok * n * lay.n_video
            total += kept_video + n * lay.n_global * (lay.n_tiles + lay.n_video)
        return total

    def attended_tile_pairs(self):
        """Tile pairs the attend kernels process: kept lists of video rows + dense lists of global rows."""
        total = 0
        for g in self.groups:
            lay = g["layout"]
            total += int(g["kept_cnt"].sum()) + len(g["heads_list"]) * lay.n_global * lay.n_kv_ok
        return total

    def forward(self, q, k, v, out, stream=None, events=None):
        """q, k, v: bf16 [S, H, D] cuda (any strides the ABI accepts); out: bf16 [S, H, D], overwritten.

        ``events``: optional dict; CUDA event pairs recorded around each stage are appended under the stage
        names (the page's PhaseTimer): gather_qk, score, select, gather_v and attend on the tile-order path
        (gather_v runs on a second stream, concurrently with score and select; the others on ``stream``),
        pool_qk, score, select and attend on the gather-free path (all on ``stream``)."""
        st = stream if stream is not None else torch.cuda.current_stream()

        def mark(name, on):
            if events is None:
                return None
            e = torch.cuda.Event(enable_timing=True)
            e.record(on)
            events.setdefault(name, []).append([e, None])
            return name

        def done(name, on):
            if name is not None:
                e = torch.cuda.Event(enable_timing=True)
                e.record(on)
                events[name][-1][1] = e

        # V needs neither scores nor lists: its gather runs on a second stream while this stream scores and
        # selects (work bound by latency and arithmetic, not by HBM); it starts after the Q/K gathers, which
        # would otherwise share the HBM bandwidth with it, and each group's attend waits for its V
        side = self._side
        for g in self.groups:
            lay = g["layout"]
            if self.direct:
                m = mark("pool_qk", st)
                L.veda_pool(lay, q, g["heads"], g["feats_q"], st, row_sq=g["q_row_sq"])
                L.veda_pool(lay, k, g["heads"], g["feats_k"], st, max_sq=g["k_max_sq"])
                done(m, st)
                m = mark("score", st)
                L.veda_score(lay, g["feats_q"], g["feats_k"], g["proj_q"], g["proj_k"], g["workspace"], g["scores"],
                             st)
                done(m, st)
                m = mark("select", st)
                L.veda_select(lay, g["scores"], g["kept_idx"], g["kept_cnt"], st)
                done(m, st)
                m = mark("attend", st)
                if self.paired:
                    L.veda_attend_direct_paired(lay, q, k, v, g["kept_idx"], g["kept_cnt"], out, g["heads"],
                                                g["q_row_sq"], g["k_max_sq"], g["pair_ws"], st)
                else:
                    L.veda_attend_direct(lay, q, k, v, g["kept_idx"], g["kept_cnt"], out, g["heads"], st,
                                         q_row_sq=g["q_row_sq"], k_max_sq=g["k_max_sq"])
                done(m, st)
                continue
            m = mark("gather_qk", st)
            if self.fp8_qk or self.int8_qk:
                gather = L.veda_gather_int8 if self.int8_qk else L.veda_gather_fp8
                gather(lay, q, g["heads"], g["q8"], g["sq"], g["feats_q"], st, row_sq=g["q_row_sq"])
                gather(lay, k, g["heads"], g["k8"], g["sk"], g["feats_k"], st, max_sq=g["k_max_sq"])
            else:
                L.veda_gather(lay, q, g["heads"], g["q_t"], g["feats_q"], st, row_sq=g["q_row_sq"])
                L.veda_gather(lay, k, g["heads"], g["k_t"], g["feats_k"], st, max_sq=g["k_max_sq"])
            done(m, st)
            qk_done = torch.cuda.Event()
            qk_done.record(st)
            side.wait_event(qk_done)
            m = mark("gather_v", side)
            L.veda_gather(lay, v, g["heads"], g["v_t"], None, side)
            done(m, side)
            v_done = torch.cuda.Event()
            v_done.record(side)
            m = mark("score", st)
            L.veda_score(lay, g["feats_q"], g["feats_k"], g["proj_q"], g["proj_k"], g["workspace"], g["scores"], st)
            done(m, st)
            m = mark("select", st)
            L.veda_select(lay, g["scores"], g["kept_idx"], g["kept_cnt"], st)
            done(m, st)
            st.wait_event(v_done)
            m = mark("attend", st)
            if (self.fp8_qk or self.int8_qk) and self.paired:
                attend = L.veda_attend_int8_paired if self.int8_qk else L.veda_attend_fp8_paired
                attend(lay, g["q8"], g["k8"], g["sq"], g["sk"], g["v_t"], g["kept_idx"], g["kept_cnt"], out, g["heads"],
                       g["q_row_sq"], g["k_max_sq"], g["pair_ws"], st)
            elif self.fp8_qk or self.int8_qk:
                attend = L.veda_attend_int8 if self.int8_qk else L.veda_attend_fp8
                attend(lay, g["q8"], g["k8"], g["sq"], g["sk"], g["v_t"], g["kept_idx"], g["kept_cnt"], out, g["heads"], st)
            elif self.paired:
                L.veda_attend_paired(lay, g["q_t"], g["k_t"], g["v_t"], g["kept_idx"], g["kept_cnt"], out, g["heads"],
                                     g["q_row_sq"], g["k_max_sq"], g["pair_ws"], st)
            else:
                L.veda_attend(lay, g["q_t"], g["k_t"], g["v_t"], g["kept_idx"], g["kept_cnt"], out, g["heads"], st,
                              q_row_sq=g["q_row_sq"], k_max_sq=g["k_max_sq"])
            done(m, st)
        return out
