"""Pins for the CPU oracle: checks that do not reuse the oracle's own code.

Each ``check_*`` helper takes the oracle routine under test as an argument, so
the mutation tests at the bottom can hand it a deliberately broken copy (a
planted mistake, on the CPU) and show that the pin fails.

What pins what (pages: DySHARP review §1, §3.1 item 3, §3.2; GPT-4 "2%"
article §2.3, §3.1, §4.1; ThunderEP PCIe blog §1.1, §2.1):
  route   brute force over every {-1,0,1}^4 logit pattern (ties everywhere),
          torch.topk / torch.softmax / torch.sigmoid on distinct logits, closed
          forms (all-equal logits, two-expert softmax).
  layout  hand-derived golden table, O(R^2) rank count, numpy stable argsort
          (a stable counting sort is a stable sort by key), bijection.
  dispatch/combine  identity experts return X * sum(gates); one-hot gates.
  FFN     GELU textbook values and torch's exact GELU; the E=1, k=1 layer is a
          dense FFN (torch fp64); W2 = 0; linearity in W2.
  router  one-hot tokens / weights pick out columns.
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from combine_moe_route_14_b200 import inputs as I

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------
# route
# ----------------------------------------------------------------------------
def _select_by_repeated_max(row, k):
    """Independent selection: k times, take the max of what is left, lowest id on ties."""
    left = list(range(len(row)))
    out = []
    for _ in range(k):
        best = None
        for e in left:
            if best is None or row[e] > row[best]:
                best = e  # strict '>' keeps the lowest id among equals
        out.append(best)
        left.remove(best)
    return out


def check_topk_bruteforce(topk_fn):
    vals = (-1.0, 0.0, 1.0)
    pats = np.array(list(itertools.product(vals, repeat=4)), dtype=np.float32)
    for k in (1, 2, 3, 4):
        got = topk_fn(pats, k)
        for t, row in enumerate(pats):
            exp = _select_by_repeated_max(list(row), k)
            assert list(got[t]) == exp, (row, k, got[t], exp)


def check_topk_library(topk_fn):
    for (T, E, k) in ((500, 8, 2), (200, 256, 8), (300, 16, 1)):
        L = I.random_f32((T, E), 3, f"distinct{E}")
        got = topk_fn(L.numpy(), k)
        _, ref = torch.topk(L, k, dim=1, sorted=True)  # distinct values: unique answer
        assert np.array_equal(got, ref.numpy()), (T, E, k)


def check_gates_library(route_fn):
    L = I.random_f32((400, 16), 5, "gates")
    vals, _ = torch.topk(L.double(), 4, dim=1, sorted=True)
    idx, g = route_fn(L.numpy(), 4, O.SOFTMAX, 1)
    np.testing.assert_allclose(g, torch.softmax(vals, dim=1).numpy(), rtol=1e-12, atol=1e-15)
    idx, g = route_fn(L.numpy(), 4, O.SOFTMAX, 0)
    full = torch.softmax(L.double(), dim=1)
    np.testing.assert_allclose(g, torch.gather(full, 1, torch.from_numpy(idx).long()).numpy(),
                               rtol=1e-12, atol=1e-15)
    idx, g = route_fn(L.numpy(), 4, O.SIGMOID, 1)
    s = torch.sigmoid(vals)
    np.testing.assert_allclose(g, (s / s.sum(1, keepdim=True)).numpy(), rtol=1e-12, atol=1e-15)
    idx, g = route_fn(L.numpy(), 4, O.SIGMOID, 0)
    np.testing.assert_allclose(g, s.numpy(), rtol=1e-12, atol=1e-15)


def check_gates_closed_forms(route_fn):
    for E, k in ((8, 2), (256, 8), (5, 5)):
        L = np.full((3, E), 0.37, dtype=np.float32)
        idx, g = route_fn(L, k, O.SOFTMAX, 1)
        assert (idx == np.arange(k)).all()
        np.testing.assert_allclose(g, 1.0 / k, rtol=1e-15)
        idx, g = route_fn(L, k, O.SOFTMAX, 0)
        np.testing.assert_allclose(g, 1.0 / E, rtol=1e-15)
        idx, g = route_fn(np.zeros((2, E), np.float32), k, O.SIGMOID, 0)
        np.testing.assert_allclose(g, 0.5, rtol=1e-15)
    # two experts: softmax renormalised over both = logistic of the logit gap
    idx, g = route_fn(np.array([[0.0, 1.0]], np.float32), 2, O.SOFTMAX, 1)
    assert list(idx[0]) == [1, 0]
    assert abs(g[0, 0] - 0.7310585786300049) < 1e-15  # 1/(1+e^-1)
    assert abs(g[0, 1] - 0.2689414213699951) < 1e-15


def check_router_variants_library(route_fn):
    """The router of [GPT] §4.1 written with torch: softmax(L / T), top-k,
    probabilities not above the threshold masked to -1."""
    L = I.random_f32((600, 16), 13, "variants")
    for temp, thr in ((1.0, 0.0), (0.3, 0.05), (1.3, 0.1), (2.0, 0.2)):
        probs = torch.softmax(L.double() / temp, dim=1)
        vals, ids = torch.topk(probs, 4, dim=1, sorted=True)
        mask = vals > thr
        ref_idx = torch.where(mask, ids, torch.full_like(ids, -1)).numpy()
        idx, g = route_fn(L.numpy(), 4, O.SOFTMAX, 0, temp, thr)
        assert np.array_equal(idx, ref_idx), (temp, thr)
        np.testing.assert_allclose(g, torch.where(mask, vals, 0.0).numpy(), rtol=1e-12, atol=1e-15)
        idx, g = route_fn(L.numpy(), 4, O.SOFTMAX, 1, temp, thr)
        kept = torch.where(mask, vals, 0.0)
        den = kept.sum(1, keepdim=True)
        ref = torch.where(den > 0, kept / den.clamp_min(1e-300), 0.0).numpy()
        np.testing.assert_allclose(g, ref, rtol=1e-12, atol=1e-15)


def check_router_variants_closed_forms(route_fn):
    # temperature 2 on logits [0, 1]: softmax over both = logistic((1 - 0) / 2)
    idx, g = route_fn(np.array([[0.0, 1.0]], np.float32), 2, O.SOFTMAX, 1, 2.0, 0.0)
    assert list(idx[0]) == [1, 0]
    assert abs(g[0, 0] - 1.0 / (1.0 + np.exp(-0.5))) < 1e-15
    # probabilities 0.6 / 0.3 / 0.1 with threshold 0.2: the third slot is dropped
    L = np.log(np.array([[0.6, 0.3, 0.1]]))
    idx, g = route_fn(L, 3, O.SOFTMAX, 0, 1.0, 0.2)
    assert list(idx[0]) == [0, 1, -1]
    np.testing.assert_allclose(g[0], [0.6, 0.3, 0.0], rtol=1e-12, atol=1e-15)
    idx, g = route_fn(L, 3, O.SOFTMAX, 1, 1.0, 0.2)
    np.testing.assert_allclose(g[0], [2 / 3, 1 / 3, 0.0], rtol=1e-12)
    # every slot below the threshold: all dropped, all gates 0
    idx, g = route_fn(np.zeros((1, 8), np.float32), 2, O.SOFTMAX, 1, 1.0, 0.2)
    assert list(idx[0]) == [-1, -1] and (g == 0).all()


def test_router_variants_match_library():
    check_router_variants_library(O.route)


def test_router_variants_closed_forms():
    check_router_variants_closed_forms(O.route)


def test_combine_skips_dropped_slots():
    Ye = np.arange(12, dtype=np.float64).reshape(3, 4)
    row_of = np.array([0, -1, -1, -1, 2, 1], np.int32)  # T=3, k=2
    g = np.array([[0.5, 0.5], [1.0, 1.0], [0.25, 0.75]])
    Y = O.combine(Ye, row_of, g, 2)
    np.testing.assert_array_equal(Y[0], 0.5 * Ye[0])
    np.testing.assert_array_equal(Y[1], 0.0)               # every slot dropped
    np.testing.assert_array_equal(Y[2], 0.25 * Ye[2] + 0.75 * Ye[1])


def test_topk_bruteforce_ternary():
    check_topk_bruteforce(O.topk_order)


def test_topk_matches_torch_on_distinct_logits():
    check_topk_library(O.topk_order)


def test_gates_match_library_softmax_sigmoid():
    check_gates_library(O.route)


def test_gates_closed_forms():
    check_gates_closed_forms(O.route)


def test_gate_invariants():
    L = I.random_f32((1000, 64), 9, "inv").numpy()
    for score in (O.SOFTMAX, O.SIGMOID):
        idx, g = O.route(L, 6, score, 1)
        np.testing.assert_allclose(g.sum(1), 1.0, rtol=1e-12)
        assert (g >= 0).all()
        assert (np.diff(g, axis=1) <= 0).all()  # slots in descending score
        sel = np.take_along_axis(L, idx.astype(np.int64), 1)
        mask = np.ones_like(L, bool)
        np.put_along_axis(mask, idx.astype(np.int64), False, 1)
        unsel_max = np.where(mask, L, -np.inf).max(1)
        assert (sel.min(1) >= unsel_max).all()


def test_signed_zero_tie_goes_to_lower_id():
    L = np.array([[-0.0, 0.0, -1.0], [0.0, -0.0, -1.0]], np.float32)
    assert O.topk_order(L, 1).ravel().tolist() == [0, 0]


def test_route_rejects_non_finite():
    with pytest.raises(ValueError):
        O.topk_order(np.array([[np.nan, 1.0]], np.float32), 1)


# ----------------------------------------------------------------------------
# layout (AL table)
# ----------------------------------------------------------------------------
def _read_golden(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            out[key] = [int(v) for v in vals]
    return out


def check_layout_golden(layout_fn):
    gd = _read_golden("layout_small.txt")
    idx = np.array(gd["topk_idx"], np.int32).reshape(gd["T"][0], gd["k"][0])
    counts, offsets, row_of, src_of = layout_fn(idx, gd["E"][0])
    assert counts.tolist() == gd["counts"]
    assert offsets.tolist() == gd["offsets"]
    assert row_of.tolist() == gd["row_of"]
    assert src_of.tolist() == gd["src_of"]
    counts, offsets, row_of, src_of = layout_fn(idx, 4)
    assert counts.tolist() == gd["E4_counts"]
    assert offsets.tolist() == gd["E4_offsets"]
    assert row_of.tolist() == gd["row_of"]


def check_layout_dropped(layout_fn):
    gd = _read_golden("layout_small.txt")
    idx = np.array(gd["D_topk_idx"], np.int32).reshape(gd["T"][0], gd["k"][0])
    counts, offsets, row_of, src_of = layout_fn(idx, gd["E"][0])
    assert counts.tolist() == gd["D_counts"]
    assert offsets.tolist() == gd["D_offsets"]
    assert row_of.tolist() == gd["D_row_of"]
    assert src_of.tolist() == gd["D_src_of"]


def check_layout_bruteforce(layout_fn, T=37, E=6, k=3, seed=1, drop=0.0):
    idx = I.random_topk(T, E, k, seed).numpy()
    if drop:
        rng = np.random.default_rng(seed)
        idx[rng.random(idx.shape) < drop] = -1
    counts, offsets, row_of, src_of = layout_fn(idx, E)
    flat = idx.reshape(-1)
    R = flat.size
    for i in range(R):
        e = flat[i]
        if e < 0:
            assert row_of[i] == -1
            continue
        before_block = sum(1 for i2 in range(R) if 0 <= flat[i2] < e)
        before_in_block = sum(1 for i2 in range(i) if flat[i2] == e)
        assert row_of[i] == before_block + before_in_block
    kept = int((flat >= 0).sum())
    order = np.argsort(np.where(flat < 0, E, flat), kind="stable")  # dropped slots sort last
    assert np.array_equal(src_of[:kept], order[:kept])
    assert (src_of[kept:] == -1).all()


def check_layout_invariants(layout_fn, T, E, k, seed, skew=0.0):
    idx = I.random_topk(T, E, k, seed, skew=skew).numpy()
    counts, offsets, row_of, src_of = layout_fn(idx, E)
    R = T * k
    flat = idx.reshape(-1)
    assert counts.sum() == R and offsets[-1] == R and offsets[0] == 0
    assert np.array_equal(np.diff(offsets), counts)
    assert np.array_equal(np.sort(row_of), np.arange(R))      # bijection
    assert np.array_equal(src_of[row_of], np.arange(R))       # inverse
    for e in range(E):
        blk = src_of[offsets[e]:offsets[e + 1]]
        assert (flat[blk] == e).all()
        assert (np.diff(blk) > 0).all()                      # stable by token


def test_layout_golden():
    check_layout_golden(O.layout)


def test_layout_bruteforce_rank_count():
    check_layout_bruteforce(O.layout)
    check_layout_bruteforce(O.layout, T=41, E=5, k=3, seed=2, drop=0.3)


def test_layout_dropped_slots_golden():
    check_layout_dropped(O.layout)


@pytest.mark.parametrize("T,E,k,skew", [(256, 8, 2, 0.0), (1000, 64, 4, 1.2), (50, 256, 8, 0.0),
                                        (1, 1, 1, 0.0), (7, 3, 3, 0.0)])
def test_layout_invariants(T, E, k, skew):
    check_layout_invariants(O.layout, T, E, k, 11, skew)


def test_layout_rejects_bad_ids():
    with pytest.raises(ValueError):
        O.layout(np.array([[0, 3]], np.int32), 3)


# ----------------------------------------------------------------------------
# dispatch / combine
# ----------------------------------------------------------------------------
def check_identity_experts(route_fn, layout_fn, dispatch_fn, combine_fn):
    T, d, E, k = 50, 24, 6, 3
    X = O.bf16_to_f64(I.f32_to_bf16_bits(I.random_f32((T, d), 2, "X").numpy()))
    L = I.random_f32((T, E), 2, "L").numpy()
    for renorm in (1, 0):
        idx, g = route_fn(L, k, O.SOFTMAX, renorm)
        counts, offsets, row_of, src_of = layout_fn(idx, E)
        Xe = dispatch_fn(X, src_of, k)
        Y = combine_fn(Xe, row_of, g, k)  # identity experts: Ye = Xe
        np.testing.assert_allclose(Y, X * g.sum(1, keepdims=True), rtol=1e-13, atol=1e-13)


def check_one_hot_gates(layout_fn, combine_fn):
    T, d, E, k = 20, 8, 5, 2
    idx = I.random_topk(T, E, k, 4).numpy()
    counts, offsets, row_of, src_of = layout_fn(idx, E)
    Ye = np.arange(T * k * d, dtype=np.float64).reshape(T * k, d)
    for j in range(k):
        g = np.zeros((T, k))
        g[:, j] = 1.0
        Y = combine_fn(Ye, row_of, g, k)
        assert np.array_equal(Y, Ye[row_of.reshape(T, k)[:, j]])


def test_identity_experts_return_scaled_input():
    check_identity_experts(O.route, O.layout, O.dispatch, O.combine)


def test_one_hot_gates_pick_one_row():
    check_one_hot_gates(O.layout, O.combine)


def test_dispatch_copies_bf16_bits():
    X = I.f32_to_bf16_bits(I.random_f32((9, 16), 1, "X").numpy())
    idx = I.random_topk(9, 4, 2, 1).numpy()
    _, _, _, src_of = O.layout(idx, 4)
    Xe = O.dispatch(X, src_of, 2)
    assert Xe.dtype == np.uint16
    for r in range(18):
        assert np.array_equal(Xe[r], X[src_of[r] // 2])


# ----------------------------------------------------------------------------
# expert FFN
# ----------------------------------------------------------------------------
def check_gelu(gelu_fn):
    assert gelu_fn(0.0) == 0.0
    # Phi(1) = 0.8413447460685429..., GELU(x) = x * Phi(x)
    assert abs(gelu_fn(1.0) - 0.8413447460685429) < 1e-15
    assert abs(gelu_fn(-1.0) + 0.15865525393145707) < 1e-15
    assert abs(gelu_fn(2.0) - 2 * 0.9772498680518208) < 1e-14
    assert abs(gelu_fn(10.0) - 10.0) < 1e-12 and abs(gelu_fn(-10.0)) < 1e-12
    x = np.linspace(-6, 6, 1001)
    ref = torch.nn.functional.gelu(torch.from_numpy(x), approximate="none").numpy()
    np.testing.assert_allclose(gelu_fn(x), ref, rtol=1e-14, atol=1e-15)


def check_dense_special_case(layer_fn):
    """E = 1, k = 1, renormalised softmax: gate = 1 and the layer is one dense FFN."""
    T, d, f = 33, 40, 24
    X = I.f32_to_bf16_bits(I.random_f32((T, d), 7, "X").numpy())
    W1 = I.f32_to_bf16_bits(I.random_f32((1, f, d), 7, "W1", 0.2).numpy())
    W2 = I.f32_to_bf16_bits(I.random_f32((1, d, f), 7, "W2", 0.2).numpy())
    L = I.random_f32((T, 1), 7, "L").numpy()
    out = layer_fn(X, W1, W2, 1, O.SOFTMAX, 1, logits=L)
    x = torch.from_numpy(O.bf16_to_f64(X))
    w1 = torch.from_numpy(O.bf16_to_f64(W1[0]))
    w2 = torch.from_numpy(O.bf16_to_f64(W2[0]))
    ref = torch.nn.functional.gelu(x @ w1.T, approximate="none") @ w2.T
    np.testing.assert_allclose(out["Y"], ref.numpy(), rtol=1e-12, atol=1e-13)


def check_ffn_square_orientation(ffn_fn):
    """d == f with non-symmetric weights: W1 is applied as x W1^T, not x W1."""
    d = 16
    Xe = np.eye(d)[:5]                      # unit rows pick out columns of W1^T
    W1 = np.arange(d * d, dtype=np.float64).reshape(1, d, d) / 100.0
    W2 = np.eye(d).reshape(1, d, d)
    H, Ye = ffn_fn(Xe, np.array([0, 5]), W1, W2)
    np.testing.assert_allclose(H, O.gelu(W1[0][:, :5].T), rtol=1e-14)


def test_gelu_textbook_values():
    check_gelu(O.gelu)


def test_dense_ffn_special_case():
    check_dense_special_case(O.layer_forward)


def test_ffn_operand_orientation():
    check_ffn_square_orientation(O.expert_ffn)


def test_zero_w2_and_linearity():
    cfg = I.workload("tiny")
    inp = I.make_layer_inputs(cfg, 0)
    bits = lambda t: t.view(torch.int16).numpy().view(np.uint16)
    X, W1, W2 = bits(inp["X"]), bits(inp["W1"]), bits(inp["W2"])
    L = inp["logits"].numpy()
    base = O.layer_forward(X, W1, W2, cfg.k, logits=L)
    W2f = O.bf16_to_f64(W2)
    zero = O.layer_forward(X, W1, np.zeros_like(W2f), cfg.k, logits=L)
    assert np.abs(zero["Y"]).max() == 0.0
    dbl = O.layer_forward(X, W1, 2.0 * W2f, cfg.k, logits=L)
    assert np.array_equal(dbl["Y"], 2.0 * base["Y"])


def test_router_logits_one_hot():
    Wr = O.bf16_to_f64(I.f32_to_bf16_bits(I.random_f32((6, 10), 1, "Wr").numpy()))
    L = O.router_logits(np.eye(10)[:6], Wr)
    np.testing.assert_array_equal(L, Wr[:, :6].T)


def test_sampled_tokens_match_full_layer():
    cfg = I.workload("tiny")
    inp = I.make_layer_inputs(cfg, 0)
    bits = lambda t: t.view(torch.int16).numpy().view(np.uint16)
    X, W1, W2 = bits(inp["X"]), bits(inp["W1"]), bits(inp["W2"])
    full = O.layer_forward(X, W1, W2, cfg.k, logits=inp["logits"].numpy())
    toks = np.array([0, 5, 77, 255])
    Ys = O.layer_forward_tokens(X, W1, W2, full["topk_idx"], full["gates"], toks)
    np.testing.assert_allclose(Ys, full["Y"][toks], rtol=1e-12, atol=1e-14)


def test_bf16_widening_is_exact():
    bits = np.array([0x3F80, 0xC000, 0x3F81, 0x0001, 0x7F7F, 0x8000], np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    assert np.array_equal(O.bf16_to_f64(bits), ref)
    assert O.bf16_to_f64(bits)[2] == 1.0078125


# ----------------------------------------------------------------------------
# planted mistakes: each broken oracle must fail at least one pin
# ----------------------------------------------------------------------------
def _topk_ties_high(L, k):
    return np.argsort(-np.asarray(L)[:, ::-1], axis=1, kind="stable")[:, :k] * -1 + (
        np.asarray(L).shape[1] - 1)


def _topk_ascending(L, k):
    return np.argsort(np.asarray(L), axis=1, kind="stable")[:, :k].astype(np.int32)


def _route_never_renorm(L, k, score, renorm):
    return O.route(L, k, score, 0)


def _route_sigmoid_sign(L, k, score, renorm):
    idx, g = O.route(L, k, score, renorm)
    if score == O.SIGMOID:
        chosen = np.take_along_axis(np.asarray(L, np.float64), idx.astype(np.int64), 1)
        s = 1.0 / (1.0 + np.exp(chosen))
        g = s / s.sum(1, keepdims=True) if renorm else s
    return idx, g


def _layout_reverse_rows(idx, E):
    counts, offsets, row_of, src_of = O.layout(idx, E)
    flat = np.asarray(idx).reshape(-1)
    row2 = row_of.copy()
    for e in range(E):
        a, b = offsets[e], offsets[e + 1]
        row2[flat == e] = row_of[flat == e][::-1]
    src2 = np.empty_like(src_of)
    src2[row2] = np.arange(len(row2))
    return counts, offsets, row2, src2


def _layout_inclusive_offsets(idx, E):
    counts, offsets, row_of, src_of = O.layout(idx, E)
    return counts, np.concatenate([offsets[1:], offsets[-1:]]), row_of, src_of


def _gelu_tanh(x):
    x = np.asarray(x, np.float64)
    return 0.5 * x * (1 + np.tanh(np.sqrt(2 / np.pi) * (x + 0.044715 * x ** 3)))


def _ffn_untransposed(Xe, offsets, W1, W2):
    Xe = np.asarray(Xe, np.float64)
    H = O.gelu(Xe @ O._as_f64(W1[0]))
    return H, H @ O._as_f64(W2[0]).T


def _combine_no_gate(Ye, row_of, gates, k):
    return O.combine(Ye, row_of, np.ones_like(np.asarray(gates, np.float64)), k)


def _route_threshold_on_gates(L, k, score, renorm, temp=1.0, thr=0.0):
    """Plausible mistake: threshold the renormalised gates instead of the probabilities."""
    idx, g = O.route(L, k, score, renorm, temp, 0.0)
    keep = g > thr if thr > 0 else np.ones_like(g, bool)
    return np.where(keep, idx, -1).astype(np.int32), np.where(keep, g, 0.0)


def _route_temperature_multiplies(L, k, score, renorm, temp=1.0, thr=0.0):
    return O.route(L, k, score, renorm, 1.0 / temp, thr)


def _layout_drop_counts_as_expert0(idx, E):
    return O.layout(np.where(np.asarray(idx) < 0, 0, idx), E)


def _layer_with(**repl):
    def fn(*a, **kw):
        saved = {n: getattr(O, n) for n in repl}
        try:
            for n, v in repl.items():
                setattr(O, n, v)
            return O.layer_forward(*a, **kw)
        finally:
            for n, v in saved.items():
                setattr(O, n, v)
    return fn


@pytest.mark.parametrize("name,run", [
    ("ties to higher id", lambda: check_topk_bruteforce(_topk_ties_high)),
    ("ascending top-k", lambda: check_topk_library(_topk_ascending)),
    ("no renormalisation", lambda: check_gates_library(_route_never_renorm)),
    ("sigmoid sign flip", lambda: check_gates_library(_route_sigmoid_sign)),
    ("rows reversed in block", lambda: check_layout_golden(_layout_reverse_rows)),
    ("rows reversed (brute)", lambda: check_layout_bruteforce(_layout_reverse_rows)),
    ("inclusive offsets", lambda: check_layout_golden(_layout_inclusive_offsets)),
    ("tanh GELU", lambda: check_gelu(_gelu_tanh)),
    ("W1 not transposed", lambda: check_ffn_square_orientation(_ffn_untransposed)),
    ("gate dropped", lambda: check_identity_experts(O.route, O.layout, O.dispatch,
                                                    _combine_no_gate)),
    ("dense FFN with tanh GELU", lambda: check_dense_special_case(_layer_with(gelu=_gelu_tanh))),
    ("threshold on gates", lambda: check_router_variants_library(_route_threshold_on_gates)),
    ("temperature multiplies", lambda: check_router_variants_closed_forms(_route_temperature_multiplies)),
    ("dropped slot counted", lambda: check_layout_dropped(_layout_drop_counts_as_expert0)),
])
def test_planted_mistake_is_caught(name, run):
    with pytest.raises(AssertionError):
        run()
