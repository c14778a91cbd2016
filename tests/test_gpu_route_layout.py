"""moe_route_layout (routing with the layout's ranking folded in, the layer's
own path) against the oracle's route + layout, bit for bit: indices, counts,
offsets, row_of and src_of.  Shapes cross the routing kernel's 32-token tiles
(the decoupled look-back between tiles), reach E = 1024 and k = 16, and cover
ties, skew, empty experts and dropped slots."""
import numpy as np
import pytest
import torch

import combine_moe_route_14_b200 as moe
from combine_moe_route_14_b200 import inputs as I
from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _logits(T, E, kind, seed):
    L = I.random_f32((T, E), seed, f"rl{T}x{E}")
    if kind == "ties":
        L = torch.round(L * 2) / 2
    elif kind == "skew":
        L = L + torch.linspace(3.0, 0.0, E)
    elif kind == "sparse":  # most experts never chosen
        L[:, 4:] -= 50.0
    return L


CASES = [
    # (T, E, k, score, renorm, kind)
    (1, 8, 2, "softmax", 1, "normal"),
    (31, 8, 2, "softmax", 1, "normal"),
    (32, 8, 2, "softmax", 1, "normal"),
    (33, 8, 2, "softmax", 1, "normal"),
    (256, 8, 2, "softmax", 1, "normal"),
    (4096, 8, 2, "softmax", 1, "normal"),
    (4096, 8, 1, "softmax", 1, "skew"),
    (2000, 16, 4, "softmax", 0, "ties"),
    (8192, 256, 8, "sigmoid", 1, "normal"),
    (3000, 1024, 16, "softmax", 1, "normal"),
    (100, 64, 2, "softmax", 1, "sparse"),
    (20000, 8, 2, "sigmoid", 0, "skew"),
]


@pytest.mark.parametrize("T,E,k,score,renorm,kind", CASES)
def test_route_layout_equals_oracle(T, E, k, score, renorm, kind):
    L = _logits(T, E, kind, 31)
    idx, g, counts, offsets, row_of, src_of = moe.moe_route_layout(L.to(DEV), k, score, renorm)
    torch.cuda.synchronize()
    assert moe.moe_device_status(clear=True) == 0
    ref_idx, ref_g = O.route(L.numpy(), k, score, renorm)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    np.testing.assert_allclose(g.cpu().numpy(), ref_g, rtol=2e-6, atol=2e-7)
    rc, ro, rr, rs = O.layout(ref_idx, E)
    for name, got, ref in (("counts", counts, rc), ("offsets", offsets, ro),
                           ("row_of", row_of, rr), ("src_of", src_of, rs)):
        assert np.array_equal(got.cpu().numpy(), ref), name


@pytest.mark.parametrize("T,E,k,temp,thr", [(2000, 8, 2, 1.3, 0.15), (500, 8, 8, 1.0, 0.2),
                                            (300, 16, 4, 2.0, 0.1)])
def test_route_layout_with_dropped_slots(T, E, k, temp, thr):
    L = _logits(T, E, "normal", 32)
    sel = O.topk_order(L.numpy(), k)
    p, _ = O.gates_from_logits(L.numpy(), sel, "softmax", 0, temp, 0.0)
    ambiguous = (np.abs(p - thr) <= 1e-6 * thr).any(1)
    assert not ambiguous.any()  # every keep decision is clear of fp32 rounding
    idx, g, counts, offsets, row_of, src_of = moe.moe_route_layout(L.to(DEV), k, "softmax", 1,
                                                                   temp, thr)
    ref_idx, _ = O.route(L.numpy(), k, "softmax", 1, temp, thr)
    assert 0 < (ref_idx < 0).sum() < T * k
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    rc, ro, rr, rs = O.layout(ref_idx, E)
    for name, got, ref in (("counts", counts, rc), ("offsets", offsets, ro),
                           ("row_of", row_of, rr), ("src_of", src_of, rs)):
        assert np.array_equal(got.cpu().numpy(), ref), name


def test_route_layout_is_repeatable_and_matches_the_two_calls():
    L = _logits(5000, 32, "skew", 33).to(DEV)
    a = moe.moe_route_layout(L, 4)
    b = moe.moe_route_layout(L, 4)
    idx, g = moe.moe_route(L, 4)
    c = moe.moe_layout(idx, 32)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    assert torch.equal(a[0], idx) and torch.equal(a[1], g)
    for x, y in zip(a[2:], c):
        assert torch.equal(x, y)
