"""HostPipeline: consecutive independent layer calls on pinned host tensors, transfers overlapped with the
kernels, give exactly the outputs of the same calls run one at a time on the device."""
import pytest
import torch

import veda_synth as V
from learned_block_sparse_tile_b200 import HostPipeline, VedaLayer
from learned_block_sparse_tile_b200 import _lib as L
from learned_block_sparse_tile_b200 import build as B

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    B.build()
    L.veda_device_check()


@pytest.mark.parametrize("name", ["tiny", "small_mixed"])
def test_pipeline_matches_single_calls(name):
    wl = V.workload(name)
    q, k, v = V.make_qkv(wl)
    pq, pk = V.make_projections(wl)
    layer = VedaLayer(wl.seq_len, wl.ref_spans, wl.target, wl.head_shapes, (wl.generated, wl.reference),
                      wl.heads, wl.dim)
    layer.set_projections(pq, pk)
    # five different calls: permuted and rescaled copies of the seeded inputs
    g = torch.Generator().manual_seed(3)
    calls = []
    for i in range(5):
        p = torch.randperm(wl.seq_len, generator=g)
        calls.append(tuple((x[p] * (1.0 + 0.25 * i)).to(torch.bfloat16).pin_memory() for x in (q, k, v)))
    want = []
    for hq, hk, hv in calls:
        out = torch.empty(hq.shape, dtype=torch.bfloat16, device="cuda")
        layer.forward(hq.cuda(), hk.cuda(), hv.cuda(), out)
        want.append(out.cpu())
    assert L.veda_sync_status() == L.VEDA_OK, L.veda_last_error()
    outs = [torch.full(q.shape, 7.0, dtype=torch.bfloat16).pin_memory() for _ in calls]
    pipe = HostPipeline(layer, wl.seq_len, wl.heads, wl.dim)
    pipe.run(calls, outs)
    torch.cuda.current_stream().synchronize()
    assert L.veda_sync_status() == L.VEDA_OK, L.veda_last_error()
    for got, ref in zip(outs, want):
        assert torch.equal(got, ref)


def test_pipeline_rejects_pageable_host_memory():
    wl = V.workload("tiny")
    layer = VedaLayer(wl.seq_len, wl.ref_spans, wl.target, wl.head_shapes, (wl.generated, wl.reference),
                      wl.heads, wl.dim)
    pipe = HostPipeline(layer, wl.seq_len, wl.heads, wl.dim)
    x = torch.zeros(wl.seq_len, wl.heads, wl.dim, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        pipe.run([(x, x, x)], [x])
