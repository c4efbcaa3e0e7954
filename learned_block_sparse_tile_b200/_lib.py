"""ctypes binding of libveda (include/veda.h): argument marshalling only.

Every function here has the name of the C entry point it calls. Device tensors are torch CUDA tensors;
their data pointers and strides are passed as plain integers. Nothing is computed in Python: when the
library is missing or the device is not an sm_100 part, calls raise instead of falling back.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

VEDA_OK, VEDA_ERR_INVALID, VEDA_ERR_CUDA, VEDA_ERR_TIMEOUT, VEDA_ERR_UNSUPPORTED, VEDA_ERR_BAD_LIST = range(6)
VEDA_BUDGET_RATIO, VEDA_BUDGET_TILES = 1, 2
TILE = 128

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libveda.so")

EXPORTS = [
    "veda_plan", "veda_layout_info", "veda_layout_export", "veda_layout_destroy", "veda_least_padding_box",
    "veda_gather", "veda_score_workspace_bytes", "veda_score", "veda_score_noalloc", "veda_select", "veda_attend",
    "veda_sync_status", "veda_last_error", "veda_device_check", "veda_set_wait_timeout_ns",
    "veda_debug_hold_next_attend", "veda_quantize_fp8", "veda_gather_fp8", "veda_attend_fp8",
    "veda_quantize_int8", "veda_gather_int8", "veda_attend_int8", "veda_layout_export_direct", "veda_pool",
    "veda_attend_direct", "veda_debug_exp2", "veda_grid_of", "veda_describe_packed_layout",
    "veda_attend_paired_workspace_bytes", "veda_attend_paired", "veda_attend_direct_paired", "veda_debug_attend_ctas",
    "veda_attend_fp8_paired", "veda_attend_int8_paired",
]

VEDA_SEG_OTHER, VEDA_SEG_VIDEO, VEDA_SEG_COND, VEDA_SEG_REF_IMG = range(4)
VEDA_MAX_PACKED_REFS = 64


class VedaError(RuntimeError):
    """A libveda call failed; ``code`` is the VEDA_ERR_* status."""

    def __init__(self, code, msg):
        super().__init__(f"[veda {code}] {msg}")
        self.code = code


class Span(C.Structure):
    _fields_ = [("start", C.c_int64), ("t", C.c_int32), ("h", C.c_int32), ("w", C.c_int32),
                ("st", C.c_int32), ("sh", C.c_int32), ("sw", C.c_int32)]


class Segment(C.Structure):
    _fields_ = [("start", C.c_int64), ("stop", C.c_int64), ("kind", C.c_int32)]


class PackedDesc(C.Structure):
    _fields_ = [("seq_len", C.c_int64), ("target_start", C.c_int64), ("target_grid", C.c_int32 * 3),
                ("n_refs", C.c_int32), ("ref_start", C.c_int64 * VEDA_MAX_PACKED_REFS),
                ("ref_grid", (C.c_int32 * 3) * VEDA_MAX_PACKED_REFS), ("n_skipped", C.c_int32),
                ("skipped", C.c_int32 * VEDA_MAX_PACKED_REFS)]


class Budget(C.Structure):
    _fields_ = [("kind", C.c_int32), ("ratio", C.c_double), ("tiles", C.c_int64)]


class BlockDesc(C.Structure):
    _fields_ = [("start", C.c_int32), ("stop", C.c_int32), ("keeps_all", C.c_int32), ("k_lo", C.c_int32),
                ("k_hi", C.c_int32), ("frac", C.c_double), ("row_budget", C.c_double)]


class LayoutDesc(C.Structure):
    _fields_ = [("seq_len", C.c_int64), ("n_slots", C.c_int64), ("n_video", C.c_int32), ("n_ref", C.c_int32),
                ("n_global", C.c_int32), ("n_tiles", C.c_int32), ("n_kv_ok", C.c_int32),
                ("n_global_ok", C.c_int32), ("max_kept", C.c_int32), ("tile_refs", C.c_int32),
                ("ref_tokens", C.c_int64), ("target_tokens", C.c_int64), ("target_box", C.c_int32 * 3),
                ("n_blocks", C.c_int32), ("blocks", BlockDesc * 2)]


_lib = None


def lib():
    """The loaded library (raises when it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise VedaError(VEDA_ERR_UNSUPPORTED, f"libveda.so is not built ({LIB_PATH}); run "
                            "`python -m learned_block_sparse_tile_b200.build`")
        L = C.CDLL(LIB_PATH)
        p, i32, i64, vp = C.c_void_p, C.c_int32, C.c_int64, C.c_void_p
        L.veda_plan.argtypes = [C.POINTER(Span), i32, i64, Budget, Budget, C.POINTER(vp)]
        L.veda_layout_info.argtypes = [vp, C.POINTER(LayoutDesc)]
        L.veda_layout_export.argtypes = [vp, p, p, p]
        L.veda_layout_export_direct.argtypes = [vp, p, p, p]
        L.veda_layout_destroy.argtypes = [vp]
        L.veda_layout_destroy.restype = None
        L.veda_least_padding_box.argtypes = [i32, i32, i32, C.POINTER(C.c_int32)]
        L.veda_gather.argtypes = [vp, p, C.POINTER(C.c_int64), i32, i32, p, i32, p, p, p, p, vp]
        L.veda_pool.argtypes = [vp, p, C.POINTER(C.c_int64), i32, i32, p, i32, p, p, p, vp]
        L.veda_attend_direct.argtypes = [vp, p, C.POINTER(C.c_int64), p, C.POINTER(C.c_int64), p,
                                         C.POINTER(C.c_int64), i32, i32, p, i32, p, p, p, C.POINTER(C.c_int64), p,
                                         p, vp]
        L.veda_attend_paired_workspace_bytes.argtypes = [vp, i32]
        L.veda_attend_paired_workspace_bytes.restype = C.c_size_t
        L.veda_attend_paired.argtypes = [vp, p, p, p, i32, i32, p, p, p, C.POINTER(C.c_int64), i32, p, p, p, p,
                                         C.c_size_t, vp]
        L.veda_attend_direct_paired.argtypes = [vp, p, C.POINTER(C.c_int64), p, C.POINTER(C.c_int64), p,
                                                C.POINTER(C.c_int64), i32, i32, p, i32, p, p, p, C.POINTER(C.c_int64),
                                                p, p, p, C.c_size_t, vp]
        L.veda_score_workspace_bytes.argtypes = [vp, i32, i32]
        L.veda_score_workspace_bytes.restype = C.c_size_t
        L.veda_score.argtypes = [vp, p, p, i32, i32, p, p, p, C.c_size_t, p, vp]
        L.veda_score_noalloc.argtypes = [vp, p, p, i32, i32, p, p, p, vp]
        L.veda_select.argtypes = [vp, p, i32, p, p, vp]
        L.veda_attend.argtypes = [vp, p, p, p, i32, i32, p, p, p, C.POINTER(C.c_int64), i32, p, p, p, vp]
        L.veda_quantize_fp8.argtypes = [vp, p, i32, i32, p, p, vp]
        L.veda_gather_fp8.argtypes = [vp, p, C.POINTER(C.c_int64), i32, i32, p, i32, p, p, p, p, p, vp]
        L.veda_quantize_int8.argtypes = [vp, p, i32, i32, p, p, vp]
        L.veda_gather_int8.argtypes = [vp, p, C.POINTER(C.c_int64), i32, i32, p, i32, p, p, p, p, p, vp]
        L.veda_attend_fp8.argtypes = [vp, p, p, p, p, p, i32, i32, p, p, p, C.POINTER(C.c_int64), i32, p, vp]
        L.veda_attend_int8.argtypes = [vp, p, p, p, p, p, i32, i32, p, p, p, C.POINTER(C.c_int64), i32, p, vp]
        for name in ("veda_attend_fp8_paired", "veda_attend_int8_paired"):
            getattr(L, name).argtypes = [vp, p, p, p, p, p, i32, i32, p, p, p, C.POINTER(C.c_int64), i32, p, p, p, p,
                                         C.c_size_t, vp]
        L.veda_sync_status.argtypes = [vp]
        L.veda_last_error.restype = C.c_char_p
        L.veda_set_wait_timeout_ns.argtypes = [C.c_uint64]
        L.veda_set_wait_timeout_ns.restype = None
        L.veda_debug_hold_next_attend.argtypes = []
        L.veda_debug_hold_next_attend.restype = None
        L.veda_debug_exp2.argtypes = [p, p, p, p, i64, vp]
        L.veda_debug_attend_ctas.argtypes = [i32]
        L.veda_debug_attend_ctas.restype = None
        L.veda_grid_of.argtypes = [p, i64, i64, C.POINTER(C.c_int32), C.POINTER(C.c_int32)]
        L.veda_describe_packed_layout.argtypes = [C.POINTER(Segment), i32, i64, C.POINTER(C.c_int32), p,
                                                  C.POINTER(PackedDesc)]
        _lib = L
    return _lib


def _check(rc):
    if rc != VEDA_OK:
        raise VedaError(rc, lib().veda_last_error().decode(errors="replace"))


def _budget(b):
    """(ratio, tiles) pair -> Budget. Exactly one must be set; the library rejects the rest."""
    ratio, tiles = b
    kind = (VEDA_BUDGET_RATIO if ratio is not None else 0) | (VEDA_BUDGET_TILES if tiles is not None else 0)
    return Budget(kind, float(ratio) if ratio is not None else 0.0, int(tiles) if tiles is not None else 0)


def _stream(stream):
    if stream is None:
        import torch
        return C.c_void_p(torch.cuda.current_stream().cuda_stream)
    return C.c_void_p(getattr(stream, "cuda_stream", stream))


def _ptr(t):
    return C.c_void_p(0 if t is None else t.data_ptr())


def _strides(t):
    return (C.c_int64 * 3)(*t.stride())


class Layout:
    """Owns a ``veda_layout*`` (freed on garbage collection)."""

    def __init__(self, handle):
        self.handle = C.c_void_p(handle)
        d = LayoutDesc()
        _check(lib().veda_layout_info(self.handle, C.byref(d)))
        self.desc = d
        self.n_video, self.n_ref, self.n_global = d.n_video, d.n_ref, d.n_global
        self.n_tiles, self.n_slots, self.max_kept = d.n_tiles, d.n_slots, d.max_kept
        self.n_kv_ok, self.n_global_ok, self.seq_len = d.n_kv_ok, d.n_global_ok, d.seq_len
        self.blocks = [(d.blocks[b].start, d.blocks[b].stop, bool(d.blocks[b].keeps_all), d.blocks[b].k_lo,
                        d.blocks[b].k_hi, d.blocks[b].frac, d.blocks[b].row_budget) for b in range(d.n_blocks)]

    def __del__(self):
        if getattr(self, "handle", None) and self.handle.value and _lib is not None:
            _lib.veda_layout_destroy(self.handle)
            self.handle = None


def veda_plan(spans, seq_len, generated, reference):
    """``spans``: [(start, (t, h, w), box or None)] references in packed order, target last."""
    arr = (Span * len(spans))()
    for i, (start, grid, box) in enumerate(spans):
        b = (0, 0, 0) if box is None else box
        arr[i] = Span(int(start), *[int(g) for g in grid], *[int(x) for x in b])
    out = C.c_void_p()
    _check(lib().veda_plan(arr, len(spans), int(seq_len), _budget(generated), _budget(reference), C.byref(out)))
    return Layout(out.value)


def veda_layout_info(layout):
    return layout.desc


def veda_layout_export(layout):
    """(perm [N], valid_count [n_tiles], allowed [n_blocks, n_video]) as int32 numpy arrays."""
    d = layout.desc
    perm = np.empty(d.n_slots, np.int32)
    vc = np.empty(d.n_tiles, np.int32)
    allowed = np.empty((d.n_blocks, d.n_video), np.int32)
    _check(lib().veda_layout_export(layout.handle, perm.ctypes.data, vc.ctypes.data, allowed.ctypes.data))
    return perm, vc, allowed


def veda_layout_export_direct(layout):
    """(box_perm [N], tile_coord [n_tiles, 4], tile_mask [n_tiles, 4]) as int32 numpy arrays: the tiles as TMA
    boxes of the packed tensors (raises VedaError with VEDA_ERR_UNSUPPORTED when the layout has no box form)."""
    d = layout.desc
    box_perm = np.empty(d.n_slots, np.int32)
    coord = np.empty((d.n_tiles, 4), np.int32)
    mask = np.empty((d.n_tiles, 4), np.int32)
    _check(lib().veda_layout_export_direct(layout.handle, box_perm.ctypes.data, coord.ctypes.data, mask.ctypes.data))
    return box_perm, coord, mask


def veda_layout_has_box_form(layout):
    """True when veda_attend_direct can take the layout (veda_layout_export_direct with no outputs)."""
    rc = lib().veda_layout_export_direct(layout.handle, None, None, None)
    if rc not in (VEDA_OK, VEDA_ERR_UNSUPPORTED):
        _check(rc)
    return rc == VEDA_OK


def veda_least_padding_box(grid):
    out = (C.c_int32 * 3)()
    _check(lib().veda_least_padding_box(int(grid[0]), int(grid[1]), int(grid[2]), out))
    return tuple(out)


def veda_gather(layout, x, heads, x_t, feats=None, stream=None, row_sq=None, max_sq=None):
    """x: bf16 [S, H, D] cuda; heads: int32 [n] cuda; x_t: bf16 [n, N, D]; feats: fp32 [n, n_video, 3D] or None;
    row_sq: fp32 [n, S] or None; max_sq: fp32 [n] or None (squared row norms for the attend's logit bound)."""
    _check(lib().veda_gather(layout.handle, _ptr(x), _strides(x), x.shape[1], x.shape[2], _ptr(heads),
                             heads.numel(), _ptr(x_t), _ptr(feats), _ptr(row_sq), _ptr(max_sq), _stream(stream)))


def veda_pool(layout, x, heads, feats, stream=None, row_sq=None, max_sq=None):
    """Pooled features only (no tile copy). x: bf16 [S, H, D] cuda; heads: int32 [n] cuda; feats: fp32
    [n, n_video, 3D]; row_sq / max_sq: optional squared row norms, as for veda_gather."""
    _check(lib().veda_pool(layout.handle, _ptr(x), _strides(x), x.shape[1], x.shape[2], _ptr(heads), heads.numel(),
                           _ptr(feats), _ptr(row_sq), _ptr(max_sq), _stream(stream)))


def veda_score_workspace_bytes(layout, n_heads, dim):
    return int(lib().veda_score_workspace_bytes(layout.handle, n_heads, dim))


def veda_score(layout, feats_q, feats_k, proj_q, proj_k, workspace, scores, stream=None):
    n_heads, dim = proj_q.shape[0], proj_q.shape[2]
    _check(lib().veda_score(layout.handle, _ptr(feats_q), _ptr(feats_k), n_heads, dim, _ptr(proj_q), _ptr(proj_k),
                            _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(scores),
                            _stream(stream)))


def veda_score_noalloc(layout, feats_q, feats_k, proj_q, proj_k, scores, stream=None):
    """veda_score without a workspace (for callers that cannot allocate): scratch is the library's own."""
    n_heads, dim = proj_q.shape[0], proj_q.shape[2]
    _check(lib().veda_score_noalloc(layout.handle, _ptr(feats_q), _ptr(feats_k), n_heads, dim, _ptr(proj_q),
                                    _ptr(proj_k), _ptr(scores), _stream(stream)))


def veda_select(layout, scores, kept_idx, kept_cnt, stream=None):
    _check(lib().veda_select(layout.handle, _ptr(scores), scores.shape[0], _ptr(kept_idx), _ptr(kept_cnt),
                             _stream(stream)))


def veda_attend(layout, q_t, k_t, v_t, kept_idx, kept_cnt, out, heads, stream=None, q_row_sq=None, k_max_sq=None):
    """q_t/k_t/v_t: bf16 [n, N, D]; out: bf16 [S, H, D] (strided ok); heads: int32 [n] cuda; q_row_sq / k_max_sq:
    the optional logit bound (row_sq of Q, max_sq of K from veda_gather or veda_pool)."""
    _check(lib().veda_attend(layout.handle, _ptr(q_t), _ptr(k_t), _ptr(v_t), q_t.shape[0], q_t.shape[2],
                             _ptr(kept_idx), _ptr(kept_cnt), _ptr(out), _strides(out), out.shape[1], _ptr(heads),
                             _ptr(q_row_sq), _ptr(k_max_sq), _stream(stream)))


def veda_attend_direct(layout, q, k, v, kept_idx, kept_cnt, out, heads, stream=None, q_row_sq=None, k_max_sq=None):
    """veda_attend on the packed tensors (no tile-order copies). q/k/v: bf16 [S, H, D] cuda (strided ok);
    out: bf16 [S, H, D]; heads: int32 [n] cuda; q_row_sq / k_max_sq: the optional logit bound."""
    _check(lib().veda_attend_direct(layout.handle, _ptr(q), _strides(q), _ptr(k), _strides(k), _ptr(v), _strides(v),
                                    q.shape[1], q.shape[2], _ptr(heads), heads.numel(), _ptr(kept_idx),
                                    _ptr(kept_cnt), _ptr(out), _strides(out), _ptr(q_row_sq), _ptr(k_max_sq),
                                    _stream(stream)))


def veda_attend_paired_workspace_bytes(layout, n_heads):
    return int(lib().veda_attend_paired_workspace_bytes(layout.handle, n_heads))


def paired_workspace(layout, n_heads, device="cuda"):
    """A device buffer for the paired attend of ``n_heads`` heads on ``layout`` (uint8, 256-byte aligned)."""
    import torch
    return torch.empty(max(veda_attend_paired_workspace_bytes(layout, n_heads), 256), dtype=torch.uint8,
                       device=device)


def veda_attend_paired(layout, q_t, k_t, v_t, kept_idx, kept_cnt, out, heads, q_row_sq, k_max_sq, workspace,
                       stream=None):
    """veda_attend two neighbouring query tiles at a time (each kept K/V tile loaded once for both), with the
    softmax reference from the logit bound; q_row_sq / k_max_sq are required, workspace from paired_workspace."""
    _check(lib().veda_attend_paired(layout.handle, _ptr(q_t), _ptr(k_t), _ptr(v_t), q_t.shape[0], q_t.shape[2],
                                    _ptr(kept_idx), _ptr(kept_cnt), _ptr(out), _strides(out), out.shape[1],
                                    _ptr(heads), _ptr(q_row_sq), _ptr(k_max_sq), _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), _stream(stream)))


def veda_attend_direct_paired(layout, q, k, v, kept_idx, kept_cnt, out, heads, q_row_sq, k_max_sq, workspace,
                              stream=None):
    """veda_attend_direct two neighbouring query tiles at a time (as veda_attend_paired)."""
    _check(lib().veda_attend_direct_paired(layout.handle, _ptr(q), _strides(q), _ptr(k), _strides(k), _ptr(v),
                                           _strides(v), q.shape[1], q.shape[2], _ptr(heads), heads.numel(),
                                           _ptr(kept_idx), _ptr(kept_cnt), _ptr(out), _strides(out), _ptr(q_row_sq),
                                           _ptr(k_max_sq), _ptr(workspace),
                                           workspace.numel() * workspace.element_size(), _stream(stream)))


def veda_gather_fp8(layout, x, heads, codes, scales, feats=None, stream=None, row_sq=None, max_sq=None):
    """x: bf16 [S, H, D] cuda; heads: int32 [n] cuda; codes: uint8 [n, N, D] (e4m3 bytes); scales: fp32
    [n, n_tiles]; feats: fp32 [n, n_video, 3D] or None; row_sq / max_sq: the bf16 norms (as veda_gather)."""
    _check(lib().veda_gather_fp8(layout.handle, _ptr(x), _strides(x), x.shape[1], x.shape[2], _ptr(heads),
                                 heads.numel(), _ptr(codes), _ptr(scales), _ptr(feats), _ptr(row_sq), _ptr(max_sq),
                                 _stream(stream)))


def veda_quantize_fp8(layout, x_t, codes, scales, stream=None):
    """x_t: bf16 [n, N, D]; codes: uint8 [n, N, D] (e4m3 bytes); scales: fp32 [n, n_tiles]."""
    _check(lib().veda_quantize_fp8(layout.handle, _ptr(x_t), x_t.shape[0], x_t.shape[2], _ptr(codes), _ptr(scales),
                                   _stream(stream)))


def veda_attend_fp8(layout, q_codes, k_codes, scales_q, scales_k, v_t, kept_idx, kept_cnt, out, heads, stream=None):
    """veda_attend with e4m3 Q/K codes (uint8 [n, N, D]) and their per-tile scales."""
    _check(lib().veda_attend_fp8(layout.handle, _ptr(q_codes), _ptr(k_codes), _ptr(scales_q), _ptr(scales_k),
                                 _ptr(v_t), v_t.shape[0], v_t.shape[2], _ptr(kept_idx), _ptr(kept_cnt), _ptr(out),
                                 _strides(out), out.shape[1], _ptr(heads), _stream(stream)))


def veda_gather_int8(layout, x, heads, codes, scales, feats=None, stream=None, row_sq=None, max_sq=None):
    """veda_gather_fp8 with int8 codes (int8 or uint8 [n, N, D])."""
    _check(lib().veda_gather_int8(layout.handle, _ptr(x), _strides(x), x.shape[1], x.shape[2], _ptr(heads),
                                  heads.numel(), _ptr(codes), _ptr(scales), _ptr(feats), _ptr(row_sq), _ptr(max_sq),
                                  _stream(stream)))


def veda_quantize_int8(layout, x_t, codes, scales, stream=None):
    """x_t: bf16 [n, N, D]; codes: int8 [n, N, D]; scales: fp32 [n, n_tiles]."""
    _check(lib().veda_quantize_int8(layout.handle, _ptr(x_t), x_t.shape[0], x_t.shape[2], _ptr(codes), _ptr(scales),
                                    _stream(stream)))


def veda_attend_int8(layout, q_codes, k_codes, scales_q, scales_k, v_t, kept_idx, kept_cnt, out, heads, stream=None):
    """veda_attend with int8 Q/K codes ([n, N, D]) and their per-tile scales."""
    _check(lib().veda_attend_int8(layout.handle, _ptr(q_codes), _ptr(k_codes), _ptr(scales_q), _ptr(scales_k),
                                  _ptr(v_t), v_t.shape[0], v_t.shape[2], _ptr(kept_idx), _ptr(kept_cnt), _ptr(out),
                                  _strides(out), out.shape[1], _ptr(heads), _stream(stream)))


def _attend_codes_paired(fn, layout, q_codes, k_codes, scales_q, scales_k, v_t, kept_idx, kept_cnt, out, heads,
                         q_row_sq, k_max_sq, workspace, stream):
    _check(fn(layout.handle, _ptr(q_codes), _ptr(k_codes), _ptr(scales_q), _ptr(scales_k), _ptr(v_t), v_t.shape[0],
              v_t.shape[2], _ptr(kept_idx), _ptr(kept_cnt), _ptr(out), _strides(out), out.shape[1], _ptr(heads),
              _ptr(q_row_sq), _ptr(k_max_sq), _ptr(workspace), workspace.numel() * workspace.element_size(),
              _stream(stream)))


def veda_attend_fp8_paired(layout, q_codes, k_codes, scales_q, scales_k, v_t, kept_idx, kept_cnt, out, heads,
                           q_row_sq, k_max_sq, workspace, stream=None):
    """veda_attend_fp8 two neighbouring query tiles at a time (as veda_attend_paired; the norms of the bf16
    inputs from veda_gather_fp8, workspace from paired_workspace)."""
    _attend_codes_paired(lib().veda_attend_fp8_paired, layout, q_codes, k_codes, scales_q, scales_k, v_t, kept_idx,
                         kept_cnt, out, heads, q_row_sq, k_max_sq, workspace, stream)


def veda_attend_int8_paired(layout, q_codes, k_codes, scales_q, scales_k, v_t, kept_idx, kept_cnt, out, heads,
                            q_row_sq, k_max_sq, workspace, stream=None):
    """veda_attend_int8 two neighbouring query tiles at a time (as veda_attend_fp8_paired)."""
    _attend_codes_paired(lib().veda_attend_int8_paired, layout, q_codes, k_codes, scales_q, scales_k, v_t, kept_idx,
                         kept_cnt, out, heads, q_row_sq, k_max_sq, workspace, stream)


def veda_sync_status(stream=None):
    """Synchronizes the stream and returns the latched kernel status code (does not raise)."""
    return int(lib().veda_sync_status(_stream(stream)))


def veda_last_error():
    return lib().veda_last_error().decode(errors="replace")


def veda_device_check():
    _check(lib().veda_device_check())


def veda_set_wait_timeout_ns(ns):
    lib().veda_set_wait_timeout_ns(int(ns))


def veda_debug_hold_next_attend():
    """Test hook: the calling thread's next veda_attend withholds its Q loads (its waits expire)."""
    lib().veda_debug_hold_next_attend()


def veda_debug_attend_ctas(n):
    """Test hook: caps the CTAs of this thread's attend launches at n (0 removes the cap)."""
    lib().veda_debug_attend_ctas(int(n))


def veda_debug_exp2(x, poly=None, mufu=None, exp2f_out=None, stream=None):
    """Test hook: the device's three forms of 2^x (attend's polynomial, the MUFU approximation, exp2f)
    for the fp32 CUDA tensor ``x``, written to the given fp32 tensors of the same size."""
    _check(lib().veda_debug_exp2(_ptr(x), _ptr(poly), _ptr(mufu), _ptr(exp2f_out), x.numel(), _stream(stream)))


_SEG_KINDS = {"video": VEDA_SEG_VIDEO, "cond": VEDA_SEG_COND, "ref_img": VEDA_SEG_REF_IMG}


def _positions(position_ids):
    return None if position_ids is None else np.ascontiguousarray(np.asarray(position_ids, dtype=np.float64))


def veda_grid_of(position_ids, a, b):
    """(T, H, W) when packed rows a:b hold a row-major grid of the [S, 3] position ids, else None."""
    pos = _positions(position_ids)
    grid, ok = (C.c_int32 * 3)(), C.c_int32()
    _check(lib().veda_grid_of(pos.ctypes.data, int(a), int(b), grid, C.byref(ok)))
    return tuple(grid) if ok.value else None


def veda_describe_packed_layout(segments, latent, seq_len, position_ids=None):
    """segments: [(start, stop, kind)] with kind "video", "cond", "ref_img" or anything else; latent: (lt, lh, lw).
    Returns (seq_len, (target start, grid), ((ref start, grid), ...), (indices of skipped segments, ...))."""
    arr = (Segment * max(1, len(segments)))()
    for i, (a, b, kind) in enumerate(segments):
        arr[i] = Segment(int(a), int(b), _SEG_KINDS.get(kind, VEDA_SEG_OTHER))
    pos = _positions(position_ids)
    lat = (C.c_int32 * 3)(*[int(x) for x in latent])
    d = PackedDesc()
    _check(lib().veda_describe_packed_layout(arr, len(segments), int(seq_len), lat,
                                             None if pos is None else pos.ctypes.data, C.byref(d)))
    refs = tuple((int(d.ref_start[i]), tuple(d.ref_grid[i])) for i in range(d.n_refs))
    return int(d.seq_len), (int(d.target_start), tuple(d.target_grid)), refs, tuple(d.skipped[:d.n_skipped])
