"""The token-centric pipeline (DySHARP review §3.2: dispatch, GEMM-1, GEMM-2
and combine as one stream of work items, each starting once its inputs are
ready) against the oracle.

  * MOE_LAYER_FUSED_COMBINE: the gate-weighted combine in GEMM-2's epilogue
    (k <= 2).  It weights the unrounded fp32 accumulators, so it is checked
    against the oracle within the float bar, and for determinism.
  * MOE_LAYER_FUSED_DISPATCH: dispatch chunks as work items of the fused FFN
    launch.  The arithmetic is unchanged, so the output is bitwise the
    default layer's.
  * MOE_LAYER_PIPELINE: both, in one persistent launch after the routing.
Indices and counts stay bit-exact in every form.
"""
import numpy as np
import pytest
import torch

import combine_moe_route_14_b200 as moe
from combine_moe_route_14_b200 import inputs as I
from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu
DEV = "cuda:0"

VARIANTS = {
    "combine": dict(fused_combine=True),
    "combine_fused_ffn": dict(fused_ffn=True, fused_combine=True),
    "pipeline": dict(pipeline=True),
}


def bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def f64(t):
    return O.bf16_to_f64(bits(t))


def same(a, b):
    return torch.equal(a.view(torch.int16), b.view(torch.int16))


def assert_close(out, ref, what):
    err = float(np.abs(np.asarray(out) - np.asarray(ref)).max())
    tol = O.tolerance(ref)
    assert err <= tol, f"{what}: max|err| {err:.3e} > tol {tol:.3e}"


class LazyExperts:
    """W[e] fetched from the device one expert at a time, as bf16 bits."""

    def __init__(self, W):
        self.W = W
        self.shape = tuple(W.shape)

    def __getitem__(self, e):
        return bits(self.W[e])


def _layer(inp, cfg, **flags):
    dev_in = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    layer = moe.MoeLayer(dev_in["W1"], dev_in["W2"], cfg.k, cfg.score, cfg.renormalize,
                         Wr=dev_in["Wr"], temperature=cfg.temperature, min_prob=cfg.min_prob,
                         **flags)
    idx = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device=DEV)
    g = torch.empty((cfg.T, cfg.k), dtype=torch.float32, device=DEV)
    counts = torch.empty((cfg.E,), dtype=torch.int32, device=DEV)
    Y = layer(dev_in["X"], logits=dev_in["logits"], topk_idx_out=idx, gates_out=g,
              counts_out=counts)
    torch.cuda.synchronize()
    assert moe.moe_device_status(clear=True) == 0
    return Y, idx, g, counts


def _oracle(inp, cfg):
    return O.layer_forward(bits(inp["X"]), bits(inp["W1"]), bits(inp["W2"]), cfg.k, cfg.score,
                           cfg.renormalize, logits=inp["logits"].numpy(),
                           temperature=cfg.temperature, min_prob=cfg.min_prob)


@pytest.mark.parametrize("name", ["tiny", "tiny_threshold"])
@pytest.mark.parametrize("variant", sorted(VARIANTS))
def test_fused_combine_full_parity(name, variant):
    cfg = I.workload(name)
    inp = I.make_layer_inputs(cfg, 0, device=DEV)
    ref = _oracle(inp, cfg)
    Y, idx, g, counts = _layer(inp, cfg, **VARIANTS[variant])
    assert np.array_equal(idx.cpu().numpy(), ref["topk_idx"])
    assert np.array_equal(counts.cpu().numpy(), ref["counts"])
    assert_close(f64(Y), ref["Y"], f"{name} Y ({variant})")


@pytest.mark.parametrize("variant", sorted(VARIANTS))
def test_fused_combine_zeroes_tokens_with_every_slot_dropped(variant):
    """A flat router (temperature 2) and a 0.2 threshold drop both slots of
    many tokens: they have no expert row, and the routing writes their zero
    output rows (no combine kernel runs to do it)."""
    T, d, E, k, f = 300, 256, 8, 2, 256
    X, W1, W2, L = _custom(T, d, E, k, f, 23)
    temp, thr = 2.0, 0.2
    ref = O.layer_forward(bits(X), bits(W1), bits(W2), k, logits=L.numpy(), temperature=temp,
                          min_prob=thr)
    sel = O.topk_order(L.numpy(), k)
    p, _ = O.gates_from_logits(L.numpy(), sel, "softmax", 0, temp, 0.0)
    assert not (np.abs(p - thr) <= 1e-6 * thr).any()  # no slot within rounding of the threshold
    none = (ref["topk_idx"] < 0).all(1)
    assert 0 < none.sum() < T
    Y = torch.full((T, d), 7.0, dtype=torch.bfloat16, device=DEV)  # stale contents
    moe.moe_layer_forward(X.to(DEV), W1.to(DEV), W2.to(DEV), k, logits=L.to(DEV), Y=Y,
                          temperature=temp, min_prob=thr, **VARIANTS[variant])
    torch.cuda.synchronize()
    assert moe.moe_device_status(clear=True) == 0
    assert (f64(Y)[none] == 0).all()
    assert_close(f64(Y), ref["Y"], f"Y ({variant}, all-dropped tokens)")


def test_fused_combine_is_deterministic_and_the_same_in_both_forms():
    cfg = I.workload("tiny")
    inp = I.make_layer_inputs(cfg, 3, device=DEV)
    a = _layer(inp, cfg, fused_combine=True)[0].clone()
    b = _layer(inp, cfg, fused_combine=True)[0].clone()
    c = _layer(inp, cfg, pipeline=True)[0].clone()
    d = _layer(inp, cfg, fused_ffn=True, fused_combine=True)[0]
    # the two arrivals of a token are summed once (a + b), whichever comes
    # first, and the fused launch runs the same MMAs: bitwise everywhere
    assert same(a, b) and same(a, c) and same(a, d)


@pytest.mark.parametrize("name,seed", [("tiny", 4), ("tiny_threshold", 4), ("decode_64", 0),
                                       ("mixtral", 0)])
def test_fused_dispatch_is_bitwise_the_default_layer(name, seed):
    cfg = I.workload(name)
    inp = I.make_layer_inputs(cfg, seed, device=DEV)
    base = _layer(inp, cfg)[0].clone()
    fd = _layer(inp, cfg, fused_ffn=True, fused_dispatch=True)[0]
    assert same(base, fd)


def _custom(T, d, E, k, f, seed, skew=0.0):
    X = I.random_bf16((T, d), seed, "X")
    W1 = I.random_bf16((E, f, d), seed, "W1", 0.05)
    W2 = I.random_bf16((E, d, f), seed, "W2", 0.05)
    L = I.random_f32((T, E), seed, "L")
    if skew:
        L = L + torch.linspace(skew, 0, E)
    return X, W1, W2, L


@pytest.mark.parametrize("T,d,E,k,f,skew", [
    (512, 256, 8, 1, 512, 0.0),      # top-1: every token has one kept slot
    (3000, 512, 5, 2, 768, 2.0),     # many dispatch chunks, multi-block experts, skew
    (37, 136, 3, 2, 264, 0.0),       # ragged everything: N and K tails, short blocks
    (1200, 128, 4, 2, 256, 0.0),     # narrow model dim: single-CTA tiles
])
@pytest.mark.parametrize("variant", ["combine", "pipeline"])
def test_pipeline_shapes_against_the_oracle(T, d, E, k, f, skew, variant):
    X, W1, W2, L = _custom(T, d, E, k, f, 21, skew)
    Y = moe.moe_layer_forward(X.to(DEV), W1.to(DEV), W2.to(DEV), k, logits=L.to(DEV),
                              **VARIANTS[variant])
    torch.cuda.synchronize()
    assert moe.moe_device_status(clear=True) == 0
    ref = O.layer_forward(bits(X), bits(W1), bits(W2), k, logits=L.numpy())
    assert_close(f64(Y), ref["Y"], f"Y {variant} T={T} d={d} E={E} k={k}")


def test_fused_combine_is_ignored_above_top_2():
    """k > 2: the flag leaves the separate combine kernel in place (bitwise)."""
    X, W1, W2, L = _custom(400, 256, 8, 4, 256, 22)
    args = (X.to(DEV), W1.to(DEV), W2.to(DEV), 4)
    a = moe.moe_layer_forward(*args, logits=L.to(DEV)).clone()
    b = moe.moe_layer_forward(*args, logits=L.to(DEV), pipeline=True)
    assert same(a, b)
    d0 = moe.make_desc(400, 256, 8, 4, 256)
    d1 = moe.make_desc(400, 256, 8, 4, 256, pipeline=True)
    # fused FFN with its dispatch chunks: dispatch and GEMM-2 launches go, the
    # layout kernel comes back, the combine stays
    assert moe.moe_kernel_launches_per_forward(d1, False) == \
        moe.moe_kernel_launches_per_forward(d0, False) - 1


def test_pipeline_counts_one_launch_for_the_whole_ffn():
    d0 = moe.make_desc(4096, 4096, 8, 2, 14336)
    d1 = moe.make_desc(4096, 4096, 8, 2, 14336, pipeline=True)
    # dispatch, GEMM-1, GEMM-2 and combine become one launch; the pipeline
    # keeps the layout kernel (its dispatch items read src_of), which the
    # default path folds into the routing
    assert moe.moe_kernel_launches_per_forward(d1, True) == \
        moe.moe_kernel_launches_per_forward(d0, True) - 2


def test_pipeline_replays_in_a_cuda_graph():
    cfg = I.workload("decode_16")
    inp = I.make_layer_inputs(cfg, 0, device=DEV)
    dev_in = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    layer = moe.MoeLayer(dev_in["W1"], dev_in["W2"], cfg.k, cfg.score, cfg.renormalize,
                         Wr=dev_in["Wr"], pipeline=True)
    Y = torch.empty((cfg.T, cfg.d), dtype=torch.bfloat16, device=DEV)
    layer(dev_in["X"], Y=Y)
    eager = Y.clone()
    Y.zero_()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(graph, stream=s):
            layer(dev_in["X"], Y=Y, stream=s)
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    assert same(Y, eager)
    del graph


def _near_ties(L, k, eps):
    if L.shape[1] <= k:
        return np.zeros(L.shape[0], bool)
    s = -np.sort(-L, axis=1)
    return (s[:, k - 1] - s[:, k]) <= eps


@pytest.mark.slow
@pytest.mark.parametrize("name,nsample", [("mixtral", 32), ("skewed_top1", 32),
                                          ("decode_16", 16), ("decode_64", 24),
                                          ("decode_1024", 24)])
def test_pipeline_full_size_sampled(name, nsample):
    cfg = I.workload(name)
    inp = I.make_layer_inputs(cfg, 0, device=DEV)
    Y, idx, g, counts = _layer(inp, cfg, pipeline=True)
    X_bits = bits(inp["X"])
    gi = idx.cpu().numpy()
    if cfg.router == "weights":
        x = O.bf16_to_f64(X_bits)
        w = O.bf16_to_f64(bits(inp["Wr"]))
        Lref = O.router_logits(x, w).astype(np.float32)
        eps = 2 * (cfg.d * 2.0 ** -24) * float((np.abs(x) @ np.abs(w).T).max())
        ties = _near_ties(Lref.astype(np.float64), cfg.k, eps)
    else:
        Lref = inp["logits"].numpy()
        ties = np.zeros(cfg.T, bool)
    ref_idx, ref_g = O.route(Lref, cfg.k, cfg.score, cfg.renormalize)
    mism = np.any(gi != ref_idx, axis=1)
    assert not (mism & ~ties).any()
    assert np.array_equal(counts.cpu().numpy(), np.bincount(gi[gi >= 0], minlength=cfg.E))
    rng = np.random.default_rng(0)
    pick = {0, cfg.T - 1} | set(rng.choice(cfg.T, size=min(cfg.T, nsample), replace=False).tolist())
    toks = np.array(sorted(t for t in pick if not ties[t]))
    ref = O.layer_forward_tokens(X_bits, LazyExperts(inp["W1"]), LazyExperts(inp["W2"]), ref_idx,
                                 ref_g, toks)
    assert_close(f64(Y[torch.from_numpy(toks).to(DEV)]), ref, f"{name} Y (pipeline)")
