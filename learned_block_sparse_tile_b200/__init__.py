"""Veda tile-skip sparse attention for B200 (sm_100a): the C ABI of ``libveda.so`` and one layer on top.

``from learned_block_sparse_tile_b200 import veda_plan, veda_gather, veda_score, veda_select, veda_attend``
gives the raw entry points (same names as ``include/veda.h``); ``VedaLayer`` runs a whole layer and
``HostPipeline`` runs consecutive independent layer calls on pinned host tensors with the PCIe transfers
overlapped with the kernels.
"""
from ._lib import (  # noqa: F401
    EXPORTS, LIB_PATH, TILE, VEDA_ERR_BAD_LIST, VEDA_ERR_CUDA, VEDA_ERR_INVALID, VEDA_ERR_TIMEOUT,
    VEDA_ERR_UNSUPPORTED, VEDA_OK, Layout, VedaError, lib, veda_attend, veda_device_check, veda_gather,
    veda_last_error, veda_layout_export, veda_layout_info, veda_least_padding_box, veda_plan, veda_score,
    veda_score_noalloc, veda_score_workspace_bytes, veda_select, veda_set_wait_timeout_ns, veda_sync_status,
    veda_quantize_fp8, veda_gather_fp8, veda_attend_fp8, veda_quantize_int8, veda_gather_int8, veda_attend_int8,
    veda_layout_export_direct, veda_pool, veda_attend_direct,
)
from .layer import VedaLayer  # noqa: F401
from .pipeline import HostPipeline  # noqa: F401
