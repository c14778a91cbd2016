"""Gather-on-load expert GEMM on the GPU (DySHARP review §3.2: dispatch fused
into the expert GEMM) vs the CPU oracle's dispatch followed by its GEMM.

Bars: the float bar of the GEMM (max|out - ref| <= 1e-2 * max|ref| + 1e-3
against the oracle), and bitwise equality with the library's own two-step
path (dispatch, then the GEMM on the dispatched rows): both feed the tensor
cores the same operands in the same order, so any difference is a gather
bug.  Rows past offsets[E] must stay untouched.
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


def assert_close(out, ref, what, rel=1e-2, abs_=1e-3):
    err = float(np.abs(out - ref).max()) if ref.size else 0.0
    tol = O.tolerance(ref, rel, abs_)
    assert err <= tol, f"{what}: max|err| {err:.3e} > tol {tol:.3e}"


@pytest.fixture(autouse=True)
def _status_clean(cuda_lib):
    moe.moe_device_status(clear=True)
    yield
    assert moe.moe_device_status(clear=True) == 0, "a kernel raised a device status bit"


def _routing(T, E, k, seed, skew=0.0, drop=0.0):
    idx = I.random_topk(T, E, k, seed, skew=skew).numpy()
    if drop > 0:
        rng = np.random.default_rng(seed + 1)
        idx = np.where(rng.random(idx.shape) < drop, -1, idx).astype(np.int32)
    counts, offsets, row_of, src_of = O.layout(idx, E)
    return offsets.astype(np.int32), src_of.astype(np.int32)


GATHER_CASES = [
    # (T, E, k, N, K, gelu, skew, drop)
    (256, 8, 2, 256, 128, True, 0.0, 0.0),       # tiny layer GEMM-1 shape
    (300, 16, 3, 384, 320, True, 1.2, 0.0),      # skewed, ragged blocks, K tail of 64
    (1000, 4, 1, 136, 72, False, 0.0, 0.0),      # N tail, K tail (72 = 64 + 8)
    (513, 8, 2, 256, 192, True, 0.0, 0.3),       # dropped slots: R < T*k rows used
    (77, 64, 4, 128, 256, False, 0.0, 0.0),      # many small experts, pair off (N = 128)
    (2000, 2, 1, 128, 64, True, 0.0, 0.0),       # one CTA stages 256 gathered rows (64 requests)
    (3, 8, 2, 16, 16, True, 0.0, 0.0),           # tiny T
    (2048, 8, 2, 1024, 1024, True, 0.0, 0.0),    # several token blocks per expert
]


@pytest.mark.parametrize("T,E,k,N,K,gelu,skew,drop", GATHER_CASES)
def test_expert_gemm_gather_parity(T, E, k, N, K, gelu, skew, drop):
    X = I.random_bf16((T, K), 21, "X")
    W = I.random_bf16((E, N, K), 21, "W", 0.05)
    offsets, src_of = _routing(T, E, k, 21, skew, drop)
    R = T * k
    used = int(offsets[-1])
    Xd, Wd = X.to(DEV), W.to(DEV)
    off_d, src_d = torch.from_numpy(offsets).to(DEV), torch.from_numpy(src_of).to(DEV)
    out = torch.full((R, N), 3.0, dtype=torch.bfloat16, device=DEV)
    moe.moe_expert_gemm_gather(Xd, src_d, k, off_d, Wd, gelu, out=out)
    # the library's two-step path on the same inputs
    Xe = moe.moe_dispatch(Xd, src_d, k)
    ref2 = torch.full((R, N), 3.0, dtype=torch.bfloat16, device=DEV)
    moe.moe_expert_gemm(Xe, off_d, Wd, gelu, out=ref2)
    torch.cuda.synchronize()
    assert torch.equal(out[:used].view(torch.int16), ref2[:used].view(torch.int16))
    assert (out[used:] == 3.0).all()
    # the oracle: dispatch, then the per-expert GEMM
    xe = O.dispatch(f64(X), src_of, k)
    ref = np.zeros((used, N))
    for e in range(E):
        lo, hi = offsets[e], offsets[e + 1]
        if hi > lo:
            w = f64(W[e])
            ref[lo:hi] = O.expert_gemm1(xe[lo:hi], w) if gelu else O.expert_gemm2(xe[lo:hi], w)
    assert_close(f64(out[:used]), ref, "gather gemm")


def test_quantize_fp8_bit_exact():
    X = I.random_bf16((333, 160), 22, "X", 3.0)
    Xq, xs = moe.moe_quantize_fp8(X.to(DEV))
    torch.cuda.synchronize()
    q, s = O.fp8_quantize(O.bf16_to_f64(bits(X)).astype(np.float32))
    assert np.array_equal(Xq.cpu().numpy(), q)
    got = xs.cpu().numpy()
    assert got[0] == s and got[1] == np.float32(np.abs(O.bf16_to_f64(bits(X))).max())
    Z, zs = moe.moe_quantize_fp8(torch.zeros((0, 32), dtype=torch.bfloat16, device=DEV))
    torch.cuda.synchronize()
    assert zs[0].item() == 1.0 and zs[1].item() == 0.0


@pytest.mark.parametrize("T,E,k,N,K,gelu,drop", [(256, 8, 2, 256, 128, True, 0.0),
                                                 (700, 16, 3, 384, 208, True, 0.2),
                                                 (1000, 4, 1, 144, 96, False, 0.0)])
def test_expert_gemm_gather_fp8_parity(T, E, k, N, K, gelu, drop):
    X_bits = bits(I.random_bf16((T, K), 23, "X"))
    W_bits = bits(I.random_bf16((E, N, K), 23, "W", 0.05))
    offsets, src_of = _routing(T, E, k, 23, 0.0, drop)
    used = int(offsets[-1])
    # the oracle's own codes and scales are the GEMM's inputs
    xq, x_s = O.fp8_quantize(O.bf16_to_f64(X_bits).astype(np.float32))
    Wq, w_s = O.fp8_quantize_experts(W_bits)
    xq_d = torch.from_numpy(xq).to(DEV)
    xs_d = torch.tensor([x_s], dtype=torch.float32, device=DEV)
    off_d, src_d = torch.from_numpy(offsets).to(DEV), torch.from_numpy(src_of).to(DEV)
    Wq_d, ws_d = torch.from_numpy(Wq).to(DEV), torch.from_numpy(w_s).to(DEV)
    out = torch.full((T * k, N), 3.0, dtype=torch.bfloat16, device=DEV)
    moe.moe_expert_gemm_gather_fp8(xq_d, xs_d, src_d, k, off_d, Wq_d, ws_d, gelu, out=out)
    # bitwise equal to the FP8 GEMM on the dispatched codes
    xe_q = torch.from_numpy(O.dispatch(xq, src_of, k)).to(DEV)
    ref2 = torch.full((T * k, N), 3.0, dtype=torch.bfloat16, device=DEV)
    moe.moe_expert_gemm_fp8(xe_q, xs_d, off_d, Wq_d, ws_d, gelu, out=ref2)
    torch.cuda.synchronize()
    assert torch.equal(out[:used].view(torch.int16), ref2[:used].view(torch.int16))
    assert (out[used:] == 3.0).all()
    ref = np.zeros((used, N))
    xe = O.dispatch(xq, src_of, k)
    for e in range(E):
        lo, hi = offsets[e], offsets[e + 1]
        if hi > lo:
            ref[lo:hi] = (O.fp8_gemm1(xe[lo:hi], x_s, Wq[e], w_s[e]) if gelu else
                          (O.e4m3_decode(xe[lo:hi]) * float(x_s))
                          @ (O.e4m3_decode(Wq[e]) * float(w_s[e])).T)
    assert_close(f64(out[:used]), ref, "gather gemm fp8")


@pytest.mark.parametrize("name,fp8", [("tiny", False), ("tiny", True), ("tiny_threshold", False),
                                      ("tiny_threshold", True), ("decode_64", False)])
def test_layer_gather_on_load_is_bitwise_the_default_layer(name, fp8):
    """The MOE_LAYER_GATHER_ON_LOAD layer gives the default layer's bytes, which
    the oracle checks (tests/test_gpu_parity.py, tests/test_gpu_fp8.py); the
    tiny case is also checked against the oracle here directly."""
    cfg = I.workload(name)
    inp = I.make_layer_inputs(cfg, 4, device=DEV)
    dev_in = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    outs = []
    for gather in (False, True):
        layer = moe.MoeLayer(dev_in["W1"], dev_in["W2"], cfg.k, cfg.score, cfg.renormalize,
                             Wr=dev_in["Wr"], temperature=cfg.temperature,
                             min_prob=cfg.min_prob, fp8=fp8, gather_on_load=gather)
        outs.append(layer(dev_in["X"], logits=dev_in["logits"]).clone())
    torch.cuda.synchronize()
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))
    if name == "tiny" and not fp8:
        ref = O.layer_forward(bits(inp["X"]), bits(inp["W1"]), bits(inp["W2"]), cfg.k, cfg.score,
                              cfg.renormalize, logits=inp["logits"].numpy())
        assert_close(f64(outs[1]), ref["Y"], "Y (gather on load)", rel=2e-2)
