"""Failure detection on the GPU without a GPU fault: a wait that nothing satisfies must end in
VEDA_ERR_TIMEOUT within its limit, and the device must stay usable afterwards."""
import time

import pytest
import torch

from learned_block_sparse_tile_b200 import _lib as L
from learned_block_sparse_tile_b200 import build as B

from gpu_util import Case

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    B.build()
    L.veda_device_check()


def test_expired_wait_is_reported_and_the_device_stays_usable():
    c = Case("tiny")
    box, heads = c.groups[0]
    res = c.run_group(box, heads)
    lay = res["layout"]
    want = res["out"].clone()

    def attend(out):
        L.veda_attend(lay, res["q_t"], res["k_t"], res["v_t"], res["kept_idx"], res["kept_cnt"], out, res["heads"])
        return L.veda_sync_status()

    L.veda_set_wait_timeout_ns(20_000_000)  # 20 ms
    try:
        L.veda_debug_hold_next_attend()  # the next launch withholds its Q loads: nothing completes those waits
        t0 = time.time()
        rc = attend(torch.zeros_like(want))
        elapsed = time.time() - t0
    finally:
        L.veda_set_wait_timeout_ns(1_000_000_000)
    assert rc == L.VEDA_ERR_TIMEOUT, L.veda_last_error()
    assert elapsed < 5.0
    # the context is intact: the next launch runs normally and reproduces the earlier result
    out = torch.zeros_like(want)
    assert attend(out) == L.VEDA_OK
    assert torch.equal(out, want)
    assert L.veda_sync_status() == L.VEDA_OK


def test_expired_wait_in_the_gather_free_attend():
    # the same bounded wait on the gather-free path (its Q loads are withheld the same way)
    c = Case("padded_tiny")
    box, heads = c.groups[0]
    res = c.run_group(box, heads)
    lay = res["layout"]

    def attend(out):
        L.veda_attend_direct(lay, c.dq, c.dk, c.dv, res["kept_idx"], res["kept_cnt"], out, res["heads"])
        return L.veda_sync_status()

    want = torch.zeros_like(res["out"])
    assert attend(want) == L.VEDA_OK
    L.veda_set_wait_timeout_ns(20_000_000)  # 20 ms
    try:
        L.veda_debug_hold_next_attend()
        t0 = time.time()
        rc = attend(torch.zeros_like(want))
        elapsed = time.time() - t0
    finally:
        L.veda_set_wait_timeout_ns(1_000_000_000)
    assert rc == L.VEDA_ERR_TIMEOUT, L.veda_last_error()
    assert elapsed < 5.0
    out = torch.zeros_like(want)
    assert attend(out) == L.VEDA_OK
    assert torch.equal(out, want)


@pytest.mark.parametrize("direct", [False, True])
def test_expired_wait_in_the_paired_attend(direct):
    # the paired kernel's waits are bounded the same way; the redo pass after it then finds no flag set
    c = Case("padded_tiny")
    box, heads = c.groups[0]
    res = c.run_group(box, heads)
    lay = res["layout"]
    n = len(heads)
    row_sq = torch.empty(n, c.wl.seq_len, device="cuda")
    max_sq = torch.empty(n, device="cuda")
    fq = torch.empty_like(res["fq"])
    L.veda_pool(lay, c.dq, res["heads"], fq, row_sq=row_sq)
    L.veda_pool(lay, c.dk, res["heads"], fq, max_sq=max_sq)
    ws = L.paired_workspace(lay, n)

    def attend(out):
        if direct:
            L.veda_attend_direct_paired(lay, c.dq, c.dk, c.dv, res["kept_idx"], res["kept_cnt"], out, res["heads"],
                                        row_sq, max_sq, ws)
        else:
            L.veda_attend_paired(lay, res["q_t"], res["k_t"], res["v_t"], res["kept_idx"], res["kept_cnt"], out,
                                 res["heads"], row_sq, max_sq, ws)
        return L.veda_sync_status()

    want = torch.zeros_like(res["out"])
    assert attend(want) == L.VEDA_OK
    L.veda_set_wait_timeout_ns(20_000_000)  # 20 ms
    try:
        L.veda_debug_hold_next_attend()
        t0 = time.time()
        rc = attend(torch.zeros_like(want))
        elapsed = time.time() - t0
    finally:
        L.veda_set_wait_timeout_ns(1_000_000_000)
    assert rc == L.VEDA_ERR_TIMEOUT, L.veda_last_error()
    assert elapsed < 5.0
    out = torch.zeros_like(want)
    assert attend(out) == L.VEDA_OK
    assert torch.equal(out, want)
