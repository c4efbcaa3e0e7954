"""The allocation-free score entry point (veda_score_noalloc) agrees with veda_score.

Callers that cannot allocate device memory when they need the scores (plugins whose device memory
belongs to a pool the host application owns, real-time loops where an allocation could block on the
device) use veda_score_noalloc, which keeps its scratch in a fixed array of the library's own device
memory instead of taking a workspace. This file is collected last so that a run stopping at its first failure has already run the
other tests; it passes on its own in a fresh process as well as after them.
"""
import pytest
import torch

from learned_block_sparse_tile_b200 import _lib as L
from learned_block_sparse_tile_b200 import build as B

from gpu_util import SCORE_REL

pytestmark = pytest.mark.gpu


def _inputs(lay, n_heads, dim, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    nv = lay.n_video
    fq = torch.randn(n_heads, nv, 3 * dim, generator=g, device="cuda")
    fk = torch.randn(n_heads, nv, 3 * dim, generator=g, device="cuda")
    pq = torch.randn(n_heads, 3 * dim, dim, generator=g, device="cuda") / dim ** 0.5
    pk = torch.randn(n_heads, 3 * dim, dim, generator=g, device="cuda") / dim ** 0.5
    return fq, fk, pq, pk


def _with_workspace(lay, fq, fk, pq, pk):
    n_heads, dim = pq.shape[0], pq.shape[2]
    ws = torch.empty(L.veda_score_workspace_bytes(lay, n_heads, dim) // 4, dtype=torch.float32, device="cuda")
    out = torch.empty(n_heads, lay.n_video, lay.n_video, dtype=torch.float32, device="cuda")
    L.veda_score(lay, fq, fk, pq, pk, ws, out)
    return out


@pytest.mark.parametrize("grid,box,n_heads,dim", [
    ((26, 48, 84), (2, 16, 4), 12, 128),  # 819 tiles: one head needs 0.29 of the scratch, so 4 head chunks
    ((3, 10, 12), (2, 8, 8), 2, 64),      # a small padded grid
])
def test_noalloc_scores_match_workspace_scores(grid, box, n_heads, dim):
    B.build()
    L.veda_device_check()
    rows = grid[0] * grid[1] * grid[2]
    lay = L.veda_plan([(0, grid, box)], rows, (0.1, None), (1.0, None))
    for call in range(2):  # two calls in a row: the shared scratch keeps the previous call's contents
        fq, fk, pq, pk = _inputs(lay, n_heads, dim, seed=100 + call)
        want = _with_workspace(lay, fq, fk, pq, pk)
        got = torch.full_like(want, float("nan"))
        L.veda_score_noalloc(lay, fq, fk, pq, pk, got)
        assert L.veda_sync_status() == L.VEDA_OK, L.veda_last_error()
        for h in range(n_heads):
            tol = SCORE_REL * float(want[h].abs().max())
            assert float((got[h] - want[h]).abs().max()) <= tol, (call, h)


def test_noalloc_rejects_heads_beyond_the_scratch():
    B.build()
    L.veda_device_check()
    # (128, 64, 72) rows at a (4, 4, 8) box: 4,608 video tiles; one head would need 2 * 4608 * 128 floats
    lay = L.veda_plan([(0, (128, 64, 72), (4, 4, 8))], 128 * 64 * 72, (0.1, None), (1.0, None))
    assert lay.n_video * 2 * 128 > (1 << 20)
    one = torch.empty(16, dtype=torch.float32, device="cuda")
    proj = torch.empty(1, 3 * 128, 128, dtype=torch.float32, device="cuda")
    with pytest.raises(L.VedaError) as e:  # rejected on the host before any buffer is touched
        L.veda_score_noalloc(lay, one, one, proj, proj, one)
    assert e.value.code == L.VEDA_ERR_UNSUPPORTED and "scratch" in str(e.value)
