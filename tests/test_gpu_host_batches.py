"""moe_layer_forward_host through the C ABI: batches in host memory copied in,
run and copied out on the library's own event-ordered streams.  Every batch
must come back bitwise equal to a direct device-pointer layer call on the same
inputs, across calls that reuse the library's buffers and streams."""
import numpy as np
import pytest
import torch

import combine_moe_route_14_b200 as moe
from combine_moe_route_14_b200 import inputs as I

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(autouse=True)
def _status_clean(cuda_lib):
    moe.moe_device_status(clear=True)
    yield
    assert moe.moe_device_status(clear=True) == 0


def _same(a, b):
    return torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.parametrize("name,nb,fp8,pinned", [("tiny", 5, False, True), ("tiny", 1, False, True),
                                                ("decode_64", 4, False, True),
                                                ("tiny", 3, True, True),
                                                ("tiny_threshold", 4, False, False)])
def test_host_batches_equal_direct_calls(name, nb, fp8, pinned):
    cfg = I.workload(name)
    inp = I.make_layer_inputs(cfg, 7, device=DEV)
    Wr = inp["Wr"].to(DEV) if inp["Wr"] is not None else None
    W1, W2 = inp["W1"], inp["W2"]
    W1q, w1s = moe.moe_quantize_experts_fp8(W1) if fp8 else (None, None)
    pin = (lambda t: t.pin_memory()) if pinned else (lambda t: t)
    Xs = [pin(I.random_bf16((cfg.T, cfg.d), 200 + i, "X")) for i in range(nb)]
    Ls = ([pin(I.random_f32((cfg.T, cfg.E), 200 + i, "L")) for i in range(nb)]
          if cfg.router == "logits" else None)
    kw = dict(score=cfg.score, renormalize=cfg.renormalize, temperature=cfg.temperature,
              min_prob=cfg.min_prob)
    for call in range(2):  # a second call reuses the library's streams and buffers
        Ys = [pin(torch.full((cfg.T, cfg.d), float(call + 3), dtype=torch.bfloat16))
              for _ in range(nb)]
        moe.moe_layer_forward_host(Xs, W1q if fp8 else W1, W2, cfg.k, Ys, logits_host=Ls, Wr=Wr,
                                   w1_scale=w1s, **kw)
        torch.cuda.current_stream().synchronize()
        for i in range(nb):
            L = None if Ls is None else Ls[i].to(DEV)
            if fp8:
                ref = moe.moe_layer_forward_fp8(Xs[i].to(DEV), W1q, w1s, W2, cfg.k, logits=L,
                                                Wr=Wr if L is None else None, **kw)
            else:
                ref = moe.moe_layer_forward(Xs[i].to(DEV), W1, W2, cfg.k, logits=L,
                                            Wr=Wr if L is None else None, **kw)
            assert _same(Ys[i], ref.cpu()), f"call {call} batch {i}"
    if nb > 1:
        assert not _same(Ys[0], Ys[1])


def test_host_batches_order_after_work_on_the_stream():
    """Work enqueued on the caller's stream before the call (here: the weights
    being written) is ordered before the call's copies and forward."""
    cfg = I.workload("tiny")
    inp = I.make_layer_inputs(cfg, 8, device=DEV)
    W1 = torch.zeros_like(inp["W1"])
    s = torch.cuda.Stream()
    X = [I.random_bf16((cfg.T, cfg.d), 300, "X").pin_memory()]
    L = [I.random_f32((cfg.T, cfg.E), 300, "L").pin_memory()]
    Y = [torch.empty((cfg.T, cfg.d), dtype=torch.bfloat16).pin_memory()]
    with torch.cuda.stream(s):
        torch.cuda._sleep(20_000_000)  # keep the stream busy, then fill in the weights
        W1.copy_(inp["W1"])
        moe.moe_layer_forward_host(X, W1, inp["W2"], cfg.k, Y, logits_host=L, stream=s)
    s.synchronize()
    ref = moe.moe_layer_forward(X[0].to(DEV), inp["W1"], inp["W2"], cfg.k, logits=L[0].to(DEV))
    assert _same(Y[0], ref.cpu())
