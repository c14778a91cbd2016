"""Fused FFN (GEMM-1 + GEMM-2 in one persistent kernel, the GEMM half of the
token-centric pipeline of the DySHARP review §3.2) on the GPU.

Bars: bitwise equality with the two-launch expert FFN (the same MMAs on the
same operands in the same order; only the schedule differs), and the float
bar against the oracle's FFN.  The layer with MOE_LAYER_FUSED_FFN must give
the default layer's bytes.
"""
import numpy as np
import pytest
import torch

import combine_moe_route_14_b200 as moe
from combine_moe_route_14_b200 import inputs as I
from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def f64(t):
    return O.bf16_to_f64(bits(t))


def same(a, b):
    return torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.fixture(autouse=True)
def _status_clean(cuda_lib):
    moe.moe_device_status(clear=True)
    yield
    assert moe.moe_device_status(clear=True) == 0, "a kernel raised a device status bit"


FFN_CASES = [
    # (counts per expert, d, f)
    ([64] * 8, 128, 256),                                   # tiny layer: pair off (d = 128)
    ([0, 1, 15, 16, 17, 31, 33, 255, 256, 257, 300, 0], 256, 384),  # ragged blocks, pair on
    ([700], 384, 512),                                      # one expert, several token blocks
    ([40, 0, 0, 90], 136, 264),                             # N and K tails in both GEMMs
    ([1030, 990, 1024], 256, 320),
    ([1] * 64, 256, 256),                                   # many one-row experts
    ([2048, 0, 2048, 4096], 512, 1024),                     # more token blocks than clusters
    ([500, 300, 129], 128, 256),                            # one CTA per tile, > 128 rows per tile
    ([320, 321, 272, 576], 256, 512),                       # short last token blocks (64, 65, 16 rows)
]


@pytest.mark.parametrize("counts,d,f", FFN_CASES)
def test_fused_ffn_matches_two_launches_and_oracle(counts, d, f):
    counts = np.asarray(counts)
    E, R = len(counts), int(counts.sum())
    offsets = torch.from_numpy(np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)).to(DEV)
    Xe = I.random_bf16((R, d), 31, "Xe")
    W1 = I.random_bf16((E, f, d), 31, "W1", 0.05)
    W2 = I.random_bf16((E, d, f), 31, "W2", 0.05)
    Xd, W1d, W2d = Xe.to(DEV), W1.to(DEV), W2.to(DEV)
    H1, Ye1 = moe.moe_expert_ffn(Xd, offsets, W1d, W2d)
    H2, Ye2 = moe.moe_expert_ffn_fused(Xd, offsets, W1d, W2d)
    torch.cuda.synchronize()
    assert same(H1, H2) and same(Ye1, Ye2)
    if R <= 4096:
        rH, rYe = O.expert_ffn(f64(Xe), offsets.cpu().numpy(), bits(W1), bits(W2))
        np.testing.assert_array_less(np.abs(f64(Ye2) - rYe).max(), O.tolerance(rYe))
        np.testing.assert_array_less(np.abs(f64(H2) - rH).max(), O.tolerance(rH))


def test_fused_ffn_fp8_matches_two_launches():
    counts = np.array([300, 0, 513, 1, 256, 257])
    E, R, d, f = len(counts), int(counts.sum()), 256, 512
    offsets = torch.from_numpy(np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)).to(DEV)
    X = I.random_bf16((R, d), 32, "X").to(DEV)
    W1 = I.random_bf16((E, f, d), 32, "W1", 0.05).to(DEV)
    W2 = I.random_bf16((E, d, f), 32, "W2", 0.05).to(DEV)
    Xq, xs = moe.moe_quantize_fp8(X)
    W1q, w1s = moe.moe_quantize_experts_fp8(W1)
    H1 = moe.moe_expert_gemm_fp8(Xq, xs, offsets, W1q, w1s, True)
    Ye1 = moe.moe_expert_gemm(H1, offsets, W2, False)
    H2, Ye2 = moe.moe_expert_ffn_fused_fp8(Xq, xs, offsets, W1q, w1s, W2)
    torch.cuda.synchronize()
    assert same(H1, H2) and same(Ye1, Ye2)


def test_fused_ffn_repeats_with_a_reused_workspace():
    """The readiness counters are re-zeroed by every call."""
    counts = np.array([500, 600])
    E, R, d, f = 2, 1100, 256, 512
    offsets = torch.from_numpy(np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)).to(DEV)
    Xe = I.random_bf16((R, d), 33, "Xe").to(DEV)
    W1 = I.random_bf16((E, f, d), 33, "W1", 0.05).to(DEV)
    W2 = I.random_bf16((E, d, f), 33, "W2", 0.05).to(DEV)
    ws = torch.full((moe.moe_expert_ffn_fused_workspace_size(E, R),), 0xFF, dtype=torch.uint8,
                    device=DEV)
    outs = [moe.moe_expert_ffn_fused(Xe, offsets, W1, W2, ws=ws)[1].clone() for _ in range(3)]
    torch.cuda.synchronize()
    assert same(outs[0], outs[1]) and same(outs[1], outs[2])


@pytest.mark.parametrize("name,fp8", [("tiny", False), ("tiny", True), ("tiny_threshold", False),
                                      ("decode_64", False), ("decode_64", True),
                                      ("mixtral", False), ("mixtral", True)])
def test_layer_fused_ffn_is_bitwise_the_default_layer(name, fp8):
    cfg = I.workload(name)
    inp = I.make_layer_inputs(cfg, 5, device=DEV)
    dev_in = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    outs = []
    for fused in (False, True):
        layer = moe.MoeLayer(dev_in["W1"], dev_in["W2"], cfg.k, cfg.score, cfg.renormalize,
                             Wr=dev_in["Wr"], temperature=cfg.temperature,
                             min_prob=cfg.min_prob, fp8=fp8, fused_ffn=fused)
        outs.append(layer(dev_in["X"], logits=dev_in["logits"]).clone())
        del layer
    torch.cuda.synchronize()
    assert same(outs[0], outs[1])
    if name == "tiny" and not fp8:
        ref = O.layer_forward(bits(inp["X"]), bits(inp["W1"]), bits(inp["W2"]), cfg.k, cfg.score,
                              cfg.renormalize, logits=inp["logits"].numpy())
        np.testing.assert_array_less(np.abs(f64(outs[1]) - ref["Y"]).max(), O.tolerance(ref["Y"]))


@pytest.mark.parametrize("form", ["fused", "pipeline"])
def test_fused_forms_share_the_gpu_with_another_stream(form):
    """Tiles come from an atomic ticket in dependency order, so a tile only
    waits on tiles that running clusters hold: the persistent kernel finishes
    with the right bytes, and no wait runs out, while a long, bounded stream
    of GEMMs on another stream holds SMs when it starts."""
    counts = np.array([2048, 0, 2048, 4096])
    E, R, d, f = len(counts), int(counts.sum()), 512, 1024
    offsets = torch.from_numpy(np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)).to(DEV)
    Xe = I.random_bf16((R, d), 34, "Xe").to(DEV)
    W1 = I.random_bf16((E, f, d), 34, "W1", 0.05).to(DEV)
    W2 = I.random_bf16((E, d, f), 34, "W2", 0.05).to(DEV)
    run = (lambda: moe.moe_expert_ffn_fused(Xe, offsets, W1, W2)[1]) if form == "fused" else None
    if form == "pipeline":
        cfg = I.workload("tiny")
        inp = I.make_layer_inputs(cfg, 34, device=DEV)
        dv = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
        layer = moe.MoeLayer(dv["W1"], dv["W2"], cfg.k, cfg.score, cfg.renormalize,
                             pipeline=True)
        run = lambda: layer(dv["X"], logits=dv["logits"])
    ref = run().clone()
    torch.cuda.synchronize()
    a = torch.randn(4096, 4096, device=DEV, dtype=torch.bfloat16)
    side = torch.cuda.Stream(DEV)
    outs = []
    for _ in range(3):
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            for _ in range(40):  # ~40 bounded GEMMs, a few ms in all
                a = torch.tanh(a @ a)
        outs.append(run().clone())
    torch.cuda.synchronize()
    for o in outs:
        assert same(o, ref)
