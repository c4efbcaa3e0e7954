"""The attend kernel's exponentials, checked on the device through the C ABI's test hook.

The softmax takes 2^x for 2 of every 8 column pairs on the FMA pipe (Cody-Waite reduction x = n + f with
n = round(x), then a cubic for 2^f on [-1/2, 1/2] with a stated maximum relative error of 7.6e-5) and for
the rest on the MUFU. Both are compared with float64 2^x on the host and with CUDA's exp2f on the device.
"""
import numpy as np
import pytest
import torch

from learned_block_sparse_tile_b200 import _lib as L
from learned_block_sparse_tile_b200 import build as B

pytestmark = pytest.mark.gpu

POLY_REL = 7.6e-5          # the polynomial's stated bound (fitted in float64, evaluated in fp32: 7.53e-5)
EXP2F_REL = 2.0 ** -21     # CUDA's exp2f: a few ulp
MUFU_REL = 2.0 ** -20      # ex2.approx on normal results, with room


def _inputs():
    g = torch.Generator().manual_seed(3)
    parts = [torch.linspace(-125.0, 126.0, 2_000_001, dtype=torch.float64),
             # the softmax's range: x <= 8 above the running reference, most mass in [-20, 0]
             torch.rand(1_000_000, generator=g, dtype=torch.float64) * 28.0 - 20.0,
             # the reduction's edges: integers and half-integers and their fp32 neighbours
             torch.arange(-125, 127, dtype=torch.float64),
             torch.arange(-125, 126, dtype=torch.float64) + 0.5]
    x = torch.cat(parts).float()
    edges = torch.cat([torch.nextafter(x[-503:], torch.tensor(-np.inf)),
                       torch.nextafter(x[-503:], torch.tensor(np.inf))])
    return torch.cat([x, edges, torch.tensor([0.0, -0.0])])


def test_exp2_polynomial_within_its_bound():
    B.build()
    L.veda_device_check()
    x = _inputs()
    xd = x.cuda()
    poly, mufu, acc = torch.empty_like(xd), torch.empty_like(xd), torch.empty_like(xd)
    L.veda_debug_exp2(xd, poly, mufu, acc)
    assert L.veda_sync_status() == L.VEDA_OK, L.veda_last_error()
    want = np.exp2(x.double().numpy())
    p, m, a = (t.double().cpu().numpy() for t in (poly, mufu, acc))
    rel_poly = np.abs(p / want - 1.0)
    assert rel_poly.max() <= POLY_REL, (rel_poly.max(), float(x[int(rel_poly.argmax())]))
    rel_acc = np.abs(a / want - 1.0)
    assert rel_acc.max() <= EXP2F_REL, rel_acc.max()
    # against CUDA's own exp2f the polynomial stays within its bound plus exp2f's error
    assert np.abs(p / a - 1.0).max() <= POLY_REL + EXP2F_REL
    rel_mufu = np.abs(m / want - 1.0)
    assert rel_mufu.max() <= MUFU_REL, rel_mufu.max()
    # the polynomial is monotone where it matters for a softmax: no output above 2^x by more than the bound
    # and none negative
    assert (p > 0).all()


def test_exp2_polynomial_clamps_far_below():
    # inputs below -126 are taken as -126: a result no larger than 2^-125 and never negative or NaN
    B.build()
    x = torch.tensor([-126.0, -127.0, -150.0, -1000.0, -3.0e38, float("-inf")], device="cuda")
    poly = torch.empty_like(x)
    L.veda_debug_exp2(x, poly)
    assert L.veda_sync_status() == L.VEDA_OK, L.veda_last_error()
    p = poly.double().cpu().numpy()
    assert np.all(np.isfinite(p)) and np.all(p >= 0.0) and np.all(p <= 2.0 ** -125)
