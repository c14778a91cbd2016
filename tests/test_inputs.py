"""The seeded input generator: deterministic bytes, correct bf16 rounding, recipe shapes."""
import numpy as np
import torch

from combine_moe_route_14_b200 import inputs as I


def test_bf16_rounding_matches_torch():
    a = I.random_f32((4096,), 0, "r").numpy() * np.float32(3.7)
    a[:4] = [1.0 + 2 ** -8, 1.0 + 3 * 2 ** -9, -1.0 - 2 ** -8, 0.0]  # exact halfway cases
    ours = I.f32_to_bf16_bits(a)
    ref = torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_same_seed_same_bytes():
    cfg = I.workload("tiny")
    a = I.make_layer_inputs(cfg, 3)
    b = I.make_layer_inputs(cfg, 3)
    c = I.make_layer_inputs(cfg, 4)
    for key in ("X", "W1", "W2", "logits"):
        assert torch.equal(a[key].view(torch.int16) if a[key].dtype == torch.bfloat16 else a[key],
                           b[key].view(torch.int16) if b[key].dtype == torch.bfloat16 else b[key])
    assert not torch.equal(a["X"].float(), c["X"].float())


def test_shapes_and_router_kind():
    for name, cfg in I.WORKLOADS.items():
        if cfg.d * cfg.f * cfg.E > 1 << 26:
            inp = I.make_layer_inputs(cfg, 0, with_weights=False)
        else:
            inp = I.make_layer_inputs(cfg, 0)
            assert tuple(inp["W1"].shape) == (cfg.E, cfg.f, cfg.d)
            assert tuple(inp["W2"].shape) == (cfg.E, cfg.d, cfg.f)
        assert tuple(inp["X"].shape) == (cfg.T, cfg.d) and inp["X"].dtype == torch.bfloat16
        if cfg.router == "weights":
            assert tuple(inp["Wr"].shape) == (cfg.E, cfg.d) and inp["logits"] is None
        else:
            assert tuple(inp["logits"].shape) == (cfg.T, cfg.E) and inp["Wr"] is None


def test_skewed_bias_gives_about_forty_percent():
    cfg = I.workload("skewed_top1")
    inp = I.make_layer_inputs(cfg, 0, with_weights=False)
    top = inp["logits"].argmax(1).numpy()
    share = np.bincount(top, minlength=cfg.E) / cfg.T
    assert 0.35 < share[0] < 0.45, share
    harsh = I.make_layer_inputs(I.workload("skewed_top1_harsh"), 0, with_weights=False)
    assert (np.bincount(harsh["logits"].argmax(1).numpy(), minlength=8) / cfg.T)[0] > 0.8


def test_distributions():
    inp = I.make_layer_inputs(I.workload("tiny"), 0)
    assert abs(inp["X"].float().std().item() - 1.0) < 0.02
    assert abs(inp["W1"].float().std().item() - 0.02) < 0.001
    assert abs(inp["logits"].std().item() - 1.0) < 0.05
