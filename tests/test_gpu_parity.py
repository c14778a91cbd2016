"""CUDA path vs the CPU oracle, stage by stage and end to end (needs a B200).

Bars:
  * indices, counts, offsets, the permutation and dispatched rows: bit-exact;
  * floats: max|out - ref| <= 2e-2 * max|ref| + 1e-3 (bf16 I/O, fp32 accumulate),
    plus tighter per-stage bounds where the arithmetic fixes one;
  * router logits: the fp32 dot-product error bound gamma_d * sum|x w|.
Inputs are seeded (combine_moe_route_14_b200.inputs); the oracle never sees a
value produced by the CUDA path.
"""
import numpy as np
import pytest
import torch

import combine_moe_route_14_b200 as moe
from combine_moe_route_14_b200 import inputs as I
from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def f64(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return O.bf16_to_f64(bits(t))
    return t.detach().cpu().double().numpy()


def assert_close(out, ref, what, rel=2e-2, abs_=1e-3):
    out = np.asarray(out, np.float64)
    ref = np.asarray(ref, np.float64)
    assert out.shape == ref.shape, (what, out.shape, ref.shape)
    err = float(np.abs(out - ref).max()) if ref.size else 0.0
    tol = O.tolerance(ref, rel, abs_)
    assert err <= tol, f"{what}: max|err| {err:.3e} > tol {tol:.3e}"
    return err


@pytest.fixture(autouse=True)
def _status_clean(cuda_lib):
    moe.moe_device_status(clear=True)
    yield
    assert moe.moe_device_status(clear=True) == 0, "a kernel raised a device status bit"


class LazyExperts:
    """W[e] fetched from the device one expert at a time, as bf16 bits."""

    def __init__(self, W):
        self.W = W
        self.shape = tuple(W.shape)

    def __getitem__(self, e):
        return bits(self.W[e])


# ----------------------------------------------------------------------------
# route
# ----------------------------------------------------------------------------
ROUTE_CASES = [
    # (T, E, k, score, renorm, kind)
    (256, 8, 2, "softmax", 1, "normal"),
    (4096, 8, 1, "softmax", 1, "normal"),
    (8192, 256, 8, "sigmoid", 1, "normal"),
    (777, 64, 6, "softmax", 0, "normal"),
    (333, 40, 3, "sigmoid", 0, "normal"),
    (500, 8, 2, "softmax", 1, "ties"),
    (500, 256, 8, "sigmoid", 1, "ties"),
    (64, 1024, 16, "softmax", 1, "ties"),
    (64, 1024, 16, "softmax", 0, "normal"),
    (100, 5, 5, "softmax", 1, "normal"),
    (1, 1, 1, "softmax", 1, "normal"),
    (37, 33, 2, "softmax", 1, "ties"),
]


def _logits(T, E, kind, seed=0):
    L = I.random_f32((T, E), seed, f"route{T}x{E}")
    if kind == "ties":  # few distinct values, signed zeros included
        L = torch.round(L * 2) / 2
        L[L == 0] = torch.where(torch.rand(int((L == 0).sum()), generator=torch.Generator().manual_seed(1)) < 0.5,
                                torch.tensor(-0.0), torch.tensor(0.0))
    return L


@pytest.mark.parametrize("T,E,k,score,renorm,kind", ROUTE_CASES)
def test_route_parity(T, E, k, score, renorm, kind):
    L = _logits(T, E, kind)
    idx, g = moe.moe_route(L.to(DEV), k, score, renorm)
    ref_idx, ref_g = O.route(L.numpy(), k, score, renorm)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    # fp32 exp / division against float64: a few ulp of values in [0, 1]
    np.testing.assert_allclose(g.cpu().numpy(), ref_g, rtol=2e-6, atol=2e-7)


ROUTE_EX_CASES = [
    # (T, E, k, score, renorm, temperature, min_prob)
    (2000, 8, 2, "softmax", 1, 1.3, 0.05),
    (2000, 16, 4, "softmax", 0, 0.3, 0.05),
    (1000, 64, 6, "softmax", 1, 2.0, 0.02),
    (1000, 256, 8, "sigmoid", 1, 1.0, 0.6),
    (500, 8, 2, "sigmoid", 0, 0.5, 0.7),
    (300, 8, 8, "softmax", 1, 1.0, 0.2),      # most slots dropped
    (300, 1024, 16, "softmax", 1, 0.7, 0.0),  # temperature only
]


@pytest.mark.parametrize("T,E,k,score,renorm,temp,thr", ROUTE_EX_CASES)
def test_route_ex_parity(T, E, k, score, renorm, temp, thr):
    L = _logits(T, E, "normal", seed=3)
    idx, g = moe.moe_route_ex(L.to(DEV), k, score, renorm, temp, thr)
    ref_idx, ref_g = O.route(L.numpy(), k, score, renorm, temp, thr)
    # the keep decision compares a probability with the threshold: slots
    # within fp32 rounding of it may go either way on the GPU
    sel = O.topk_order(L.numpy(), k)
    gates_all, _ = O.gates_from_logits(L.numpy(), sel, score, 0, temp, 0.0)
    ambiguous = (np.abs(gates_all - thr) <= 1e-6 * max(thr, 1e-30)).any(1) if thr > 0 else np.zeros(T, bool)
    gi, gg = idx.cpu().numpy(), g.cpu().numpy()
    ok = ~ambiguous
    assert np.array_equal(gi[ok], ref_idx[ok])
    np.testing.assert_allclose(gg[ok], ref_g[ok], rtol=2e-6, atol=2e-7)
    assert ((gi == -1) == (gg == 0))[ok].all()


def test_route_masked_experts_are_never_chosen():
    """-inf logits (masked experts) are never picked; a token with fewer than k
    other experts gets its remaining slots dropped (-1, gate 0), and the kept
    gates are the softmax over the kept logits.  NaN logits only ever yield
    indices in [-1, E)."""
    T, E, k = 600, 16, 4
    L = _logits(T, E, "normal", seed=5).numpy().copy()
    rng = np.random.default_rng(5)
    n_masked = rng.integers(0, E + 1, size=T)       # 0 .. all experts masked
    for t in range(T):
        L[t, rng.permutation(E)[:n_masked[t]]] = -np.inf
    idx, g = moe.moe_route(torch.from_numpy(L).to(DEV), k, "softmax", 1)
    gi, gg = idx.cpu().numpy(), g.cpu().numpy()
    for t in range(T):
        fin = [e for e in range(E) if np.isfinite(L[t, e])]
        order = sorted(fin, key=lambda e: (-L[t, e], e))[:k]
        exp_idx = order + [-1] * (k - len(order))
        assert gi[t].tolist() == exp_idx, (t, gi[t], exp_idx)
        if order:
            z = np.exp(L[t, order].astype(np.float64) - L[t, order[0]])
            np.testing.assert_allclose(gg[t, :len(order)], z / z.sum(), rtol=2e-6, atol=2e-7)
        assert (gg[t, len(order):] == 0).all()
    Ln = L.copy()
    Ln[rng.random(Ln.shape) < 0.2] = np.nan
    idx, _ = moe.moe_route(torch.from_numpy(Ln).to(DEV), k, "softmax", 1)
    gi = idx.cpu().numpy()
    assert ((gi >= -1) & (gi < E)).all()
    assert not np.isnan(Ln[np.arange(T)[:, None].repeat(k, 1)[gi >= 0], gi[gi >= 0]]).any()


# ----------------------------------------------------------------------------
# router linear
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("T,d,E", [(4096, 4096, 8), (16, 4096, 8), (300, 136, 3), (77, 512, 40),
                                   (1, 8, 1), (100, 256, 72), (33, 4104, 130), (8, 64, 1024),
                                   (17, 72, 8),
                                   # more token tiles than resident CTAs: each CTA walks
                                   # several tiles through its ring (and, at E = 72, two
                                   # passes of expert groups per tile)
                                   (20000, 1024, 8), (5000, 2048, 72),
                                   # d too large to stage Wr in shared memory beside the ring
                                   (40, 8192, 8)])
def test_router_logits_parity(T, d, E):
    X = I.random_bf16((T, d), 1, "X")
    Wr = I.random_bf16((E, d), 1, "Wr", 0.02)
    L = moe.moe_router_logits(X.to(DEV), Wr.to(DEV)).cpu().double().numpy()
    x, w = O.bf16_to_f64(bits(X)), O.bf16_to_f64(bits(Wr))
    ref = O.router_logits(x, w)
    u = 2.0 ** -24
    gamma = d * u / (1 - d * u)
    bound = gamma * (np.abs(x) @ np.abs(w).T) + 1e-30
    assert (np.abs(L - ref) <= bound).all(), float((np.abs(L - ref) / bound).max())


# ----------------------------------------------------------------------------
# layout
# ----------------------------------------------------------------------------
LAYOUT_CASES = [
    # (T, E, k, skew)
    (256, 8, 2, 0.0),
    (4096, 8, 2, 0.0),        # 8192 slots, 8 experts: one-block path at its limit
    (4096, 8, 1, 2.5),        # skewed
    (8192, 256, 8, 0.0),      # 65536 slots: histogram + decoupled look-back, 32 tiles
    (8193, 256, 2, 0.0),      # 16386 slots: ragged last tile
    (20000, 7, 3, 1.0),       # several tiles, few experts
    (10, 256, 4, 0.0),        # mostly empty experts
    (3000, 1024, 16, 0.0),    # max experts and k, multi-block
    (50, 1024, 2, 0.0),
    (1, 1, 1, 0.0),
    (999, 1, 1, 0.0),
    (5461, 16, 3, 0.0),       # 16383 slots, E = 16: multi-block, ragged last tile
    (4096, 12, 4, 1.5),       # 16384 slots exactly, skewed
    (2731, 32, 3, 0.0),       # 8193 slots, 32 experts: just past the one-block limit
    (2048, 33, 2, 0.0),       # 4096 slots, 33 experts: one-block path at its limit
    (2049, 64, 2, 0.0),       # 4098 slots, 64 experts: just past it
    (3000, 17, 2, 0.0),       # E = 17
]


@pytest.mark.parametrize("T,E,k,skew", LAYOUT_CASES)
def test_layout_parity(T, E, k, skew):
    idx = I.random_topk(T, E, k, 5, skew=skew)
    counts, offsets, row_of, src_of = moe.moe_layout(idx.to(DEV), E)
    rc, ro, rr, rs = O.layout(idx.numpy(), E)
    assert np.array_equal(counts.cpu().numpy(), rc)
    assert np.array_equal(offsets.cpu().numpy(), ro)
    assert np.array_equal(row_of.cpu().numpy(), rr)
    assert np.array_equal(src_of.cpu().numpy(), rs)


def test_layout_repeatable_and_stable_under_reuse():
    """Same workspace twice (look-back words must be re-armed each call)."""
    T, E, k = 8192, 256, 8
    idx = I.random_topk(T, E, k, 6).to(DEV)
    ws = torch.empty(moe.moe_layout_workspace_size(T, E, k), dtype=torch.uint8, device=DEV)
    a = [x.clone() for x in moe.moe_layout(idx, E, ws=ws)]
    b = moe.moe_layout(idx, E, ws=ws)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_layout_flags_bad_expert_ids():
    idx = I.random_topk(64, 8, 2, 7)
    idx[3, 1] = 8
    idx[10, 0] = -5
    counts, offsets, row_of, src_of = moe.moe_layout(idx.to(DEV), 8)
    assert moe.moe_device_status(clear=True) & 1  # MOE_DEV_BAD_EXPERT_ID
    rc = row_of.cpu().numpy()
    assert rc[3 * 2 + 1] == -1 and rc[10 * 2] == -1
    assert counts.sum().item() == 64 * 2 - 2


@pytest.mark.parametrize("T,E,k,drop", [(256, 8, 2, 0.2), (8192, 256, 8, 0.3), (9000, 7, 3, 0.5),
                                        (40, 1024, 4, 1.0), (5000, 16, 3, 0.4)])
def test_layout_dropped_slots(T, E, k, drop):
    """-1 marks a dropped slot: no row, not counted, no flag; unused rows get src_of -1."""
    idx = I.random_topk(T, E, k, 8)
    rng = np.random.default_rng(8)
    idx[torch.from_numpy(rng.random((T, k)) < drop)] = -1
    counts, offsets, row_of, src_of = moe.moe_layout(idx.to(DEV), E)
    rc, ro, rr, rs = O.layout(idx.numpy(), E)
    assert np.array_equal(counts.cpu().numpy(), rc)
    assert np.array_equal(offsets.cpu().numpy(), ro)
    assert np.array_equal(row_of.cpu().numpy(), rr)
    assert np.array_equal(src_of.cpu().numpy(), rs)


# ----------------------------------------------------------------------------
# dispatch / combine
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("T,d,E,k", [(256, 128, 8, 2), (4096, 4096, 8, 2), (8192, 7168, 256, 8),
                                     (33, 8, 4, 3), (100, 4104, 16, 5), (5, 2056, 3, 1)])
def test_dispatch_bit_exact(T, d, E, k):
    X = I.random_bf16((T, d), 2, "X")
    idx = I.random_topk(T, E, k, 2)
    _, _, rr, rs = O.layout(idx.numpy(), E)
    Xe = moe.moe_dispatch(X.to(DEV), torch.from_numpy(rs).to(DEV), k)
    ref = O.dispatch(bits(X), rs, k)
    assert np.array_equal(bits(Xe), ref)
    # walked by token through row_of: the same bytes
    Xt = moe.moe_dispatch_by_token(X.to(DEV), torch.from_numpy(rr).to(DEV), k)
    assert np.array_equal(bits(Xt), ref)


@pytest.mark.parametrize("T,d,E,k", [(256, 128, 8, 2), (4096, 4096, 8, 2), (8192, 7168, 256, 8),
                                     (33, 8, 4, 3), (100, 4104, 16, 5), (50, 64, 16, 16),
                                     (7, 24, 12, 11), (4096, 4096, 8, 1)])
def test_combine_parity(T, d, E, k):
    Ye = I.random_bf16((T * k, d), 3, "Ye")
    idx = I.random_topk(T, E, k, 3)
    _, _, rr, _ = O.layout(idx.numpy(), E)
    L = I.random_f32((T, E), 3, "L")
    _, g = O.route(L.numpy(), k)
    g32 = torch.from_numpy(g.astype(np.float32))
    Y = moe.moe_combine(Ye.to(DEV), torch.from_numpy(rr).to(DEV), g32.to(DEV))
    ref = O.combine(O.bf16_to_f64(bits(Ye)), rr, g32.double().numpy(), k)
    out = f64(Y)
    assert_close(out, ref, "combine")
    # one bf16 rounding of an fp32 sum: |err| <= 2^-8 |ref| + fp32 slack
    slack = 1e-6 * (np.abs(g32.double().numpy()).sum(1, keepdims=True) * 8)
    assert (np.abs(out - ref) <= 2.0 ** -8 * np.abs(ref) + slack).all()


def test_dispatch_and_combine_with_dropped_slots():
    T, d, E, k = 500, 256, 8, 2
    idx = I.random_topk(T, E, k, 9)
    rng = np.random.default_rng(9)
    idx[torch.from_numpy(rng.random((T, k)) < 0.3)] = -1
    idx[7] = -1                                   # a token with every slot dropped
    _, ro, rr, rs = O.layout(idx.numpy(), E)
    kept = int(ro[-1])
    X = I.random_bf16((T, d), 9, "X")
    Xe = torch.full((T * k, d), 3.0, dtype=torch.bfloat16, device=DEV)
    moe.moe_dispatch(X.to(DEV), torch.from_numpy(rs).to(DEV), k, Xe=Xe)
    assert np.array_equal(bits(Xe[:kept]), O.dispatch(bits(X), rs, k)[:kept])
    assert (Xe[kept:] == 3.0).all()                # unused rows untouched
    Xt = torch.full((T * k, d), 3.0, dtype=torch.bfloat16, device=DEV)
    moe.moe_dispatch_by_token(X.to(DEV), torch.from_numpy(rr).to(DEV), k, Xe=Xt)
    assert np.array_equal(bits(Xt[:kept]), O.dispatch(bits(X), rs, k)[:kept])
    assert (Xt[kept:] == 3.0).all()
    Ye = I.random_bf16((T * k, d), 9, "Ye")
    Ye[kept:] = float("nan")                       # never read
    g = torch.rand((T, k), generator=torch.Generator().manual_seed(9))
    g[idx < 0] = 0.0
    Y = moe.moe_combine(Ye.to(DEV), torch.from_numpy(rr).to(DEV), g.to(DEV))
    ref = O.combine(O.bf16_to_f64(bits(Ye)), rr, g.double().numpy(), k)
    out = f64(Y)
    assert not np.isnan(out).any()
    assert (out[7] == 0).all()
    assert_close(out, ref, "combine with drops")


def test_identity_experts_return_input():
    """combine(dispatch(X)) with Ye = Xe returns X * sum(g) = X (renormalised)."""
    T, d, E, k = 1000, 256, 8, 2
    X = I.random_bf16((T, d), 4, "X").to(DEV)
    L = I.random_f32((T, E), 4, "L").to(DEV)
    idx, g = moe.moe_route(L, k)
    _, _, row_of, src_of = moe.moe_layout(idx, E)
    Y = moe.moe_combine(moe.moe_dispatch(X, src_of, k), row_of, g)
    assert_close(f64(Y), f64(X), "identity", rel=2.0 ** -7, abs_=0)


# ----------------------------------------------------------------------------
# grouped GEMM / expert FFN
# ----------------------------------------------------------------------------
def _gemm_case(counts, N, K, gelu, seed=8, std_w=0.05):
    counts = np.asarray(counts)
    E = len(counts)
    R = int(counts.sum())
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    A = I.random_bf16((max(R, 1), K), seed, "A")[:R]
    W = I.random_bf16((E, N, K), seed, "W", std_w)
    out = torch.full((R, N), float("nan"), dtype=torch.bfloat16, device=DEV)
    moe.moe_expert_gemm(A.to(DEV), torch.from_numpy(offsets).to(DEV), W.to(DEV), gelu, out=out)
    a = O.bf16_to_f64(bits(A))
    ref = np.zeros((R, N))
    for e in range(E):
        lo, hi = offsets[e], offsets[e + 1]
        if hi > lo:
            w = O.bf16_to_f64(bits(W[e]))
            ref[lo:hi] = O.expert_gemm1(a[lo:hi], w) if gelu else O.expert_gemm2(a[lo:hi], w)
    return f64(out), ref


GEMM_CASES = [
    # (counts per expert, N, K, gelu)
    ([64] * 8, 256, 128, True),                       # tiny layer, GEMM-1 shape
    ([64] * 8, 128, 256, False),                      # tiny layer, GEMM-2 shape
    ([0, 1, 15, 16, 17, 31, 33, 255, 256, 257, 300, 0], 256, 192, True),  # ragged blocks
    ([700], 384, 512, False),                         # one expert, several token blocks
    ([40, 0, 0, 90], 136, 72, True),                  # N and K tails (not multiples of 128 / 64)
    ([5, 3], 8, 8, False),                            # smallest dims
    ([128] * 3, 1024, 1024, True),
    ([1] * 64, 256, 256, False),                      # many one-row experts
    # short last token blocks (1, 16, 44, 64, 65 rows) after full ones
    ([300, 0, 513, 1, 256, 257], 512, 192, True),
    ([320, 321, 272, 576, 64], 256, 256, True),
    ([1] * 700 + [300], 256, 64, False),              # 701 experts: a large tile table in smem
    ([600, 520], 264, 128, False),                    # N tail with wide tiles
    ([1030, 990, 1024], 256, 320, True),
    ([260] * 16, 384, 64, False),                     # 16 experts just over one block
    # one CTA per tile (N <= 128) with more than 128 rows per tile: two 128-row boxes
    ([300, 0, 129, 256, 97, 128], 128, 64, True),
    ([700], 64, 200, False),
    ([1000, 3], 96, 136, True),
    # merged last blocks (a tail of at most 64 rows joins the block before it:
    # tiles of 257..320 rows) mixed with ordinary ones, enough tiles that each
    # cluster runs several in a row: the accumulator placement alternates and
    # a wide tile shares TMEM columns with its neighbour
    ([300, 256, 320, 200, 576, 17, 64, 288] * 12, 1024, 128, True),
    ([290, 260, 321, 512, 33] * 24, 512, 192, False),
]


@pytest.mark.parametrize("counts,N,K,gelu", GEMM_CASES)
def test_expert_gemm_parity(counts, N, K, gelu):
    out, ref = _gemm_case(counts, N, K, gelu)
    assert not np.isnan(out).any()
    assert_close(out, ref, "gemm")
    # bf16 output rounding plus fp32 accumulation: far inside the bar
    assert_close(out, ref, "gemm (tight)", rel=1e-2, abs_=1e-3)


def test_expert_gemm_leaves_rows_past_offsets_alone():
    counts = np.array([10, 20])
    offsets = torch.tensor([0, 10, 30], dtype=torch.int32, device=DEV)
    A = I.random_bf16((40, 64), 9, "A").to(DEV)
    W = I.random_bf16((2, 128, 64), 9, "W", 0.05).to(DEV)
    out = torch.full((40, 128), 7.0, dtype=torch.bfloat16, device=DEV)
    moe.moe_expert_gemm(A, offsets, W, True, out=out)
    assert (out[30:] == 7.0).all()


def test_expert_ffn_tiny_matches_oracle():
    cfg = I.workload("tiny")
    inp = I.make_layer_inputs(cfg, 0, device=DEV)
    Xe_bits = I.random_bf16((cfg.R, cfg.d), 0, "Xe")
    idx = I.random_topk(cfg.T, cfg.E, cfg.k, 0)
    rc, ro, _, _ = O.layout(idx.numpy(), cfg.E)
    H, Ye = moe.moe_expert_ffn(Xe_bits.to(DEV), torch.from_numpy(ro).to(DEV), inp["W1"], inp["W2"])
    rH, rYe = O.expert_ffn(O.bf16_to_f64(bits(Xe_bits)), ro, bits(inp["W1"]), bits(inp["W2"]))
    assert_close(f64(H), rH, "H")
    assert_close(f64(Ye), rYe, "Ye")


# ----------------------------------------------------------------------------
# whole layer
# ----------------------------------------------------------------------------
def _run_layer(inp, cfg):
    dev_in = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    layer = moe.MoeLayer(dev_in["W1"], dev_in["W2"], cfg.k, cfg.score, cfg.renormalize,
                         Wr=dev_in["Wr"], temperature=cfg.temperature, min_prob=cfg.min_prob)
    T = cfg.T
    idx = torch.empty((T, cfg.k), dtype=torch.int32, device=DEV)
    g = torch.empty((T, cfg.k), dtype=torch.float32, device=DEV)
    counts = torch.empty((cfg.E,), dtype=torch.int32, device=DEV)
    Y = layer(dev_in["X"], logits=dev_in["logits"], topk_idx_out=idx, gates_out=g,
              counts_out=counts)
    torch.cuda.synchronize()
    return Y, idx, g, counts, layer


def test_layer_tiny_full_parity():
    cfg = I.workload("tiny")
    inp = I.make_layer_inputs(cfg, 0, device=DEV)
    Y, idx, g, counts, _ = _run_layer(inp, cfg)
    ref = O.layer_forward(bits(inp["X"]), bits(inp["W1"]), bits(inp["W2"]), cfg.k, cfg.score,
                          cfg.renormalize, logits=inp["logits"].numpy())
    assert np.array_equal(idx.cpu().numpy(), ref["topk_idx"])
    assert np.array_equal(counts.cpu().numpy(), ref["counts"])
    np.testing.assert_allclose(g.cpu().numpy(), ref["gates"], rtol=2e-6, atol=2e-7)
    assert_close(f64(Y), ref["Y"], "Y")


def test_layer_tiny_threshold_full_parity():
    cfg = I.workload("tiny_threshold")
    inp = I.make_layer_inputs(cfg, 0, device=DEV)
    ref = O.layer_forward(bits(inp["X"]), bits(inp["W1"]), bits(inp["W2"]), cfg.k, cfg.score,
                          cfg.renormalize, logits=inp["logits"].numpy(),
                          temperature=cfg.temperature, min_prob=cfg.min_prob)
    dropped = int((ref["topk_idx"] < 0).sum())
    assert 0 < dropped < cfg.R  # the variant is exercised
    sel = O.topk_order(inp["logits"].numpy(), cfg.k)
    p, _ = O.gates_from_logits(inp["logits"].numpy(), sel, cfg.score, 0, cfg.temperature, 0.0)
    assert not (np.abs(p - cfg.min_prob) <= 1e-6 * cfg.min_prob).any()  # no ambiguous slot
    dev_in = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    layer = moe.MoeLayer(dev_in["W1"], dev_in["W2"], cfg.k, cfg.score, cfg.renormalize,
                         temperature=cfg.temperature, min_prob=cfg.min_prob)
    idx = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device=DEV)
    counts = torch.empty((cfg.E,), dtype=torch.int32, device=DEV)
    Y = layer(dev_in["X"], logits=dev_in["logits"], topk_idx_out=idx, counts_out=counts)
    assert np.array_equal(idx.cpu().numpy(), ref["topk_idx"])
    assert np.array_equal(counts.cpu().numpy(), ref["counts"])
    assert_close(f64(Y), ref["Y"], "Y (threshold)")


def test_layer_narrow_model_dim_full_tiles():
    """d = 128: GEMM-2 (N = d) runs one CTA per tile with full 256-row tiles
    (about 512 rows per expert), the case that needs two 128-row token boxes."""
    T, d, E, k, f = 1024, 128, 4, 2, 256
    X = I.random_bf16((T, d), 13, "X")
    W1 = I.random_bf16((E, f, d), 13, "W1", 0.05)
    W2 = I.random_bf16((E, d, f), 13, "W2", 0.05)
    L = I.random_f32((T, E), 13, "L")
    Y = moe.moe_layer_forward(X.to(DEV), W1.to(DEV), W2.to(DEV), k, logits=L.to(DEV))
    ref = O.layer_forward(bits(X), bits(W1), bits(W2), k, logits=L.numpy())
    assert int(ref["counts"].max()) > 256
    assert_close(f64(Y), ref["Y"], "Y (d = 128)")


def test_layer_deterministic():
    cfg = I.workload("tiny")
    inp = I.make_layer_inputs(cfg, 1, device=DEV)
    Y1 = _run_layer(inp, cfg)[0].clone()
    Y2 = _run_layer(inp, cfg)[0]
    assert torch.equal(Y1.view(torch.int16), Y2.view(torch.int16))


def _sample_tokens(T, n, seed=0):
    rng = np.random.default_rng(seed)
    pick = set([0, T - 1]) | set(rng.choice(T, size=min(T, n), replace=False).tolist())
    return np.array(sorted(pick))


def _near_ties(L, k, eps):
    """Tokens whose k-th and (k+1)-th logits lie within eps (routing there is a coin toss)."""
    if L.shape[1] <= k:
        return np.zeros(L.shape[0], bool)
    s = -np.sort(-L, axis=1)
    return (s[:, k - 1] - s[:, k]) <= eps


@pytest.mark.slow
@pytest.mark.parametrize("name,nsample", [("skewed_top1", 48), ("skewed_top1_harsh", 24),
                                          ("fine_grained", 12), ("mixtral", 32),
                                          ("mixtral_threshold", 32),
                                          ("decode_16", 16), ("decode_64", 24),
                                          ("decode_256", 24), ("decode_1024", 24)])
def test_layer_full_size_sampled(name, nsample):
    cfg = I.workload(name)
    inp = I.make_layer_inputs(cfg, 0, device=DEV)
    Y, idx, g, counts, layer = _run_layer(inp, cfg)
    X_bits = bits(inp["X"])
    gi = idx.cpu().numpy()
    if cfg.router == "weights":
        # oracle's own logits (float64 -> fp32) and routing; near-ties may differ
        Lref = O.router_logits(O.bf16_to_f64(X_bits), O.bf16_to_f64(bits(inp["Wr"]))).astype(np.float32)
        x = O.bf16_to_f64(X_bits)
        w = O.bf16_to_f64(bits(inp["Wr"]))
        eps = 2 * (cfg.d * 2.0 ** -24) * float((np.abs(x) @ np.abs(w).T).max())
        ties = _near_ties(Lref.astype(np.float64), cfg.k, eps)
    else:
        Lref = inp["logits"].numpy()
        ties = np.zeros(cfg.T, bool)
    ref_idx, ref_g = O.route(Lref, cfg.k, cfg.score, cfg.renormalize, cfg.temperature,
                             cfg.min_prob)
    if cfg.min_prob > 0:  # slots within rounding of the threshold may go either way
        sel = O.topk_order(Lref, cfg.k)
        p, _ = O.gates_from_logits(Lref, sel, cfg.score, 0, cfg.temperature, 0.0)
        ties |= (np.abs(p - cfg.min_prob) <= 1e-5 * cfg.min_prob).any(1)
    mism = np.any(gi != ref_idx, axis=1)
    assert not (mism & ~ties).any(), f"{int((mism & ~ties).sum())} tokens routed differently"
    kept = gi[gi >= 0]
    assert np.array_equal(counts.cpu().numpy(), np.bincount(kept, minlength=cfg.E))
    toks = np.array([t for t in _sample_tokens(cfg.T, nsample) if not ties[t]])
    ref = O.layer_forward_tokens(X_bits, LazyExperts(inp["W1"]), LazyExperts(inp["W2"]), ref_idx,
                                 ref_g, toks)
    assert_close(f64(Y[torch.from_numpy(toks).to(DEV)]), ref, f"{name} Y")


def test_gemm_gelu_is_exact_to_bf16():
    """Identity weights make the GEMM output GELU(x) itself.  The kernel's erf
    approximation (Abramowitz & Stegun 7.1.26, |erfc error| <= 1.5e-7) adds at
    most 0.75e-7 * |x| to the exact GELU, so the output must equal the exact
    GELU rounded to bf16 up to half an ulp plus that term (a last-place flip
    where the exact value sits next to a rounding midpoint)."""
    K = 64
    xs = torch.linspace(-9, 9, 64 * K, dtype=torch.float32).reshape(64, K)
    A = xs.to(torch.bfloat16)
    W = torch.eye(K, dtype=torch.bfloat16).reshape(1, K, K)
    offsets = torch.tensor([0, 64], dtype=torch.int32, device=DEV)
    out = moe.moe_expert_gemm(A.to(DEV), offsets, W.to(DEV), True)
    x = O.bf16_to_f64(bits(A))
    ref = O.gelu(x)
    got = f64(out)
    bound = 2.0 ** -8 * np.abs(ref) + 1e-7 * np.abs(x) + 1e-30
    assert (np.abs(got - ref) <= bound).all(), float((np.abs(got - ref) / bound).max())
    big = np.abs(ref) > 1e-3  # where bf16 resolution dominates: the rounded value itself
    ref_bits = I.f32_to_bf16_bits(ref.astype(np.float32))
    assert (bits(out)[big] == ref_bits[big]).mean() >= 0.99


@pytest.mark.parametrize("name", ["decode_16", "tiny"])
def test_layer_forward_replays_in_a_cuda_graph(name):
    """Sizes stay on the device and nothing syncs the host, so one layer forward
    captures into a CUDA graph; replays reproduce the eager output bit for bit."""
    cfg = I.workload(name)
    inp = I.make_layer_inputs(cfg, 2, device=DEV)
    X = inp["X"].to(DEV)
    L = inp["logits"].to(DEV) if inp["logits"] is not None else None
    Wr = inp["Wr"].to(DEV) if inp["Wr"] is not None else None
    layer = moe.MoeLayer(inp["W1"], inp["W2"], cfg.k, cfg.score, cfg.renormalize, Wr=Wr)
    Y = torch.empty((cfg.T, cfg.d), dtype=torch.bfloat16, device=DEV)
    s = torch.cuda.Stream(device=DEV)
    s.wait_stream(torch.cuda.current_stream(DEV))
    with torch.cuda.stream(s):
        layer(X, logits=L, Y=Y)  # first call: per-device set-up happens outside the capture
        eager = Y.clone()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            layer(X, logits=L, Y=Y)
    torch.cuda.current_stream(DEV).wait_stream(s)
    Y.zero_()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert torch.equal(Y.view(torch.int16), eager.view(torch.int16))
