"""moe_layout_static: the layout for callers that cannot allocate device memory.

Some callers have no device allocator to draw a workspace from (code running
inside another framework's callback that is handed only the tensors it works
on, or code that must not allocate after start-up).  moe_layout_static keeps
the layout's scratch in a fixed 1 MiB array inside the library instead.  These
tests call it through the C ABI and check that it returns exactly what
moe_layout returns with a caller workspace, and what the oracle's layout
returns, twice in a row (the shared array keeps the previous call's contents,
so the second call checks that the kernels re-arm it).  The file is named to
be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

import combine_moe_route_14_b200 as moe
from combine_moe_route_14_b200 import inputs as I
from oracle import moe_oracle as O

DEV = "cuda:0"


def _c_layout_static(lib, idx, E, outs, stream):
    T, k = idx.shape
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    return lib.moe_layout_static(p(idx), T, E, k, p(outs[0]), p(outs[1]), p(outs[2]), p(outs[3]),
                                 ctypes.c_void_p(stream.cuda_stream))


@pytest.mark.gpu
@pytest.mark.parametrize("T,E,k,skew", [(8192, 256, 8, 0.0),   # multi-block: uses the array
                                        (20000, 7, 3, 1.0),
                                        (3000, 1024, 16, 0.0),
                                        (256, 8, 2, 0.0)])      # one-block: no scratch
def test_static_layout_matches_workspace_layout_twice(cuda_lib, T, E, k, skew):
    lib = cuda_lib.load_library()
    stream = torch.cuda.current_stream(DEV)
    for call, seed in enumerate((11, 12)):  # two calls in a row, different routings
        idx = I.random_topk(T, E, k, seed, skew=skew).to(DEV)
        ref = moe.moe_layout(idx, E)
        R = T * k
        outs = [torch.full((E,), -7, dtype=torch.int32, device=DEV),
                torch.full((E + 1,), -7, dtype=torch.int32, device=DEV),
                torch.full((R,), -7, dtype=torch.int32, device=DEV),
                torch.full((R,), -7, dtype=torch.int32, device=DEV)]
        st = _c_layout_static(lib, idx, E, outs, stream)
        assert st == 0, lib.moe_last_error_string().decode()
        torch.cuda.synchronize()
        for name, a, b in zip(("counts", "offsets", "row_of", "src_of"), outs, ref):
            assert torch.equal(a, b), f"call {call}: {name} differs"
        # and the oracle's layout of the same routing, bit for bit
        for name, a, b in zip(("counts", "offsets", "row_of", "src_of"), outs,
                              O.layout(idx.cpu().numpy(), E)):
            assert np.array_equal(a.cpu().numpy(), b), f"call {call}: {name} differs from the oracle"
    assert moe.moe_device_status(clear=True) == 0


def test_static_layout_rejects_shapes_beyond_its_array():
    lib = moe.load_library()
    p = ctypes.c_void_p(0x10000)
    T, E, k = 1 << 20, 1024, 4  # 4M slots x 1024 experts: 2 MiB of look-back words
    assert lib.moe_layout_workspace_size(T, E, k) > (1 << 20)
    st = lib.moe_layout_static(p, T, E, k, p, p, p, p, None)
    assert st == 2  # MOE_ERR_UNSUPPORTED, before any launch
    msg = lib.moe_last_error_string().decode()
    assert "static array" in msg and "moe_layout" in msg
    assert lib.moe_layout_static(p, 4, 8, 9, p, p, p, p, None) == 1  # k > E, as moe_layout
