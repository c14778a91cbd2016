"""Programmatic dependent launch changes no result.

Every kernel of the library is launched as a programmatic dependent of its
stream predecessor and waits (griddepcontrol.wait) before its first global
access.  These tests run the same layers in a child process with MOE_PDL=0
(plain stream order) and compare the outputs bit for bit with this process's
(the attribute on), eagerly and replayed from a CUDA graph.
"""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import combine_moe_route_14_b200 as moe
from combine_moe_route_14_b200 import inputs as I

DEV = "cuda:0"
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import sys, numpy as np, torch
sys.path.insert(0, sys.argv[1])
import combine_moe_route_14_b200 as moe
from combine_moe_route_14_b200 import inputs as I
name, out, fp8 = sys.argv[2], sys.argv[3], sys.argv[4] == "1"
cfg = I.workload(name)
inp = I.make_layer_inputs(cfg, 3, device="cuda:0")
d = {k: (v.to("cuda:0") if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
layer = moe.MoeLayer(d["W1"], d["W2"], cfg.k, cfg.score, cfg.renormalize, Wr=d["Wr"],
                     temperature=cfg.temperature, min_prob=cfg.min_prob, fp8=fp8)
Y = layer(d["X"], logits=d["logits"])
torch.cuda.synchronize()
assert moe.moe_device_status(clear=True) == 0
np.save(out, Y.view(torch.int16).cpu().numpy())
"""


def _layer_out(name, graph, fp8):
    cfg = I.workload(name)
    inp = I.make_layer_inputs(cfg, 3, device=DEV)
    d = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    layer = moe.MoeLayer(d["W1"], d["W2"], cfg.k, cfg.score, cfg.renormalize, Wr=d["Wr"],
                         temperature=cfg.temperature, min_prob=cfg.min_prob, fp8=fp8)
    Y = torch.empty((cfg.T, cfg.d), dtype=torch.bfloat16, device=DEV)
    layer(d["X"], logits=d["logits"], Y=Y)
    if graph:
        Y.fill_(0)
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s):
                layer(d["X"], logits=d["logits"], Y=Y)
        torch.cuda.current_stream().wait_stream(s)
        g.replay()
        g.replay()
        torch.cuda.synchronize()
        del g
    torch.cuda.synchronize()
    assert moe.moe_device_status(clear=True) == 0
    return Y.view(torch.int16).cpu().numpy()


@pytest.mark.gpu
@pytest.mark.parametrize("name,fp8", [("tiny", False), ("decode_16", False),
                                      ("fine_grained_e32", False), ("tiny", True),
                                      ("fine_grained_e32", True)])
def test_programmatic_launch_is_bitwise_plain_stream_order(name, fp8, tmp_path):
    assert os.environ.get("MOE_PDL", "1") != "0", "run with the attribute on"
    out = tmp_path / "y.npy"
    env = dict(os.environ, MOE_PDL="0")
    r = subprocess.run([sys.executable, "-c", CHILD, ROOT, name, str(out), "1" if fp8 else "0"],
                       env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    plain = np.load(out)
    for graph in (False, True):
        assert np.array_equal(_layer_out(name, graph, fp8), plain), f"graph={graph}"
