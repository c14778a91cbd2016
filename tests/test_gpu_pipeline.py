"""HostPipeline on the GPU: host->device copies, the layer and device->host
copies of consecutive batches overlap on three streams with two device
buffers; every batch must come back exactly as a direct layer call gives it."""
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


@pytest.mark.parametrize("name,depth", [("tiny", 2), ("tiny", 3), ("decode_64", 2)])
def test_pipeline_matches_direct_calls(name, depth):
    cfg = I.workload(name)
    inp = I.make_layer_inputs(cfg, 6, device=DEV)
    Wr = inp["Wr"].to(DEV) if inp["Wr"] is not None else None
    layer = moe.MoeLayer(inp["W1"], inp["W2"], cfg.k, cfg.score, cfg.renormalize, Wr=Wr)
    nb = 5
    Xs = [I.random_bf16((cfg.T, cfg.d), 100 + i, "X").pin_memory() for i in range(nb)]
    Ls = ([I.random_f32((cfg.T, cfg.E), 100 + i, "L").pin_memory() for i in range(nb)]
          if cfg.router == "logits" else [None] * nb)
    Ys = [torch.empty((cfg.T, cfg.d), dtype=torch.bfloat16).pin_memory() for _ in range(nb)]
    pipe = moe.HostPipeline(layer, cfg.T, cfg.d, cfg.E, with_logits=Ls[0] is not None,
                            device=DEV, depth=depth)
    for i in range(nb):
        pipe.submit(Xs[i], Ys[i], Ls[i])
    pipe.synchronize()
    for i in range(nb):
        ref = layer(Xs[i].to(DEV), logits=None if Ls[i] is None else Ls[i].to(DEV)).cpu()
        torch.cuda.synchronize()
        assert torch.equal(Ys[i].view(torch.int16), ref.view(torch.int16)), f"batch {i}"
    assert not torch.equal(Ys[0].view(torch.int16), Ys[1].view(torch.int16))
