"""FP8 mode on the GPU vs the CPU oracle (ThunderEP PCIe blog §3.3, §5.2:
activations cast to E4M3 with a per-tensor dynamic scale; FP8 tensor cores).

Bars:
  * E4M3 codes and scales (weights and dispatched rows): bit-exact, since
    both sides take every quantisation step in fp32 with round to nearest
    even (the oracle emulates the fp32 products with numpy float32);
  * FP8 GEMM-1 and the FP8 layer output: the float bar of the bf16 path,
    max|out - ref| <= 2e-2 * max|ref| + 1e-3, against the oracle evaluated on
    the same codes (E4M3 products are exact; only fp32 summation and the bf16
    output rounding differ).
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
    if t.dtype == torch.bfloat16:
        return O.bf16_to_f64(bits(t))
    return t.detach().cpu().double().numpy()


def f32_of(bf16_bits):
    return O.bf16_to_f64(bf16_bits).astype(np.float32)  # exact widening


def assert_close(out, ref, what, rel=2e-2, abs_=1e-3):
    out = np.asarray(out, np.float64)
    ref = np.asarray(ref, np.float64)
    assert out.shape == ref.shape, (what, out.shape, ref.shape)
    err = float(np.abs(out - ref).max()) if ref.size else 0.0
    tol = O.tolerance(ref, rel, abs_)
    assert err <= tol, f"{what}: max|err| {err:.3e} > tol {tol:.3e}"


@pytest.fixture(autouse=True)
def _status_clean(cuda_lib):
    moe.moe_device_status(clear=True)
    yield
    assert moe.moe_device_status(clear=True) == 0, "a kernel raised a device status bit"


# ----------------------------------------------------------------------------
# quantisation: bit-exact codes and scales
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("E,rows,cols", [(3, 40, 96), (8, 256, 128), (1, 1, 16), (5, 0, 32),
                                         (2, 333, 208)])
def test_quantize_experts_bit_exact(E, rows, cols):
    W = I.random_bf16((E, rows, cols), 11, "Wq", 0.05)
    if E > 1 and rows > 0:
        W[1] = 0          # an all-zero expert: scale 1, codes 0
    if E > 2 and rows > 0:
        W[2] *= 300.0     # a wide-range expert
    Wq, s = moe.moe_quantize_experts_fp8(W.to(DEV))
    torch.cuda.synchronize()
    rq, rs = O.fp8_quantize_experts(bits(W))
    assert np.array_equal(Wq.cpu().numpy(), rq)
    assert np.array_equal(s.cpu().numpy(), rs)   # fp32 scales, bit for bit


def _crafted_tokens():
    """amax = 448 makes inv = 1, so the codes are E4M3(x) itself: ties to even,
    subnormals, signed zero and the top of the range, all bf16-representable."""
    vals = [448.0, -448.0, 1.0625, 1.1875, -1.0625, 2.0 ** -10, 3 * 2.0 ** -10, -(2.0 ** -10),
            2.0 ** -9, 7 * 2.0 ** -10, 0.0, -0.0, 240.0, 232.0, 248.0, 0.01171875, 96.5, -3.3125]
    row = np.zeros(32, np.float32)
    row[:len(vals)] = vals
    X = np.tile(row, (4, 1))
    X[1:] *= np.float32(0.5)
    X[0] = row
    return I.f32_to_bf16_bits(X)


@pytest.mark.parametrize("case", ["random", "crafted", "dropped", "empty"])
def test_dispatch_fp8_bit_exact(case):
    if case == "crafted":
        X_bits = _crafted_tokens()
        T, d = X_bits.shape
        k, E = 2, 4
    else:
        T, d, k, E = (0, 64, 2, 8) if case == "empty" else (300, 160, 3, 16)
        X_bits = bits(I.random_bf16((T, d), 12, "X", 2.5))
    idx = I.random_topk(T, E, k, 12).numpy() if T else np.zeros((0, k), np.int32)
    if case == "dropped":
        rng = np.random.default_rng(5)
        idx = np.where(rng.random(idx.shape) < 0.3, -1, idx).astype(np.int32)
    _, _, _, src_of = O.layout(idx, E)
    X = torch.from_numpy(X_bits.view(np.int16)).view(torch.bfloat16).to(DEV)
    Xeq = torch.full((T * k, d), 0xAB, dtype=torch.uint8, device=DEV)
    x_scale = torch.full((2,), -1.0, dtype=torch.float32, device=DEV)
    moe.moe_dispatch_fp8(X, torch.from_numpy(src_of.astype(np.int32)).to(DEV), k, Xeq=Xeq,
                         x_scale=x_scale)
    torch.cuda.synchronize()
    xq, s = O.fp8_quantize(f32_of(X_bits))
    amax = np.float32(np.abs(f32_of(X_bits)).max()) if T else np.float32(0)
    got_s = x_scale.cpu().numpy()
    assert got_s[0] == s and got_s[1] == amax
    got = Xeq.cpu().numpy()
    ok = src_of >= 0
    assert np.array_equal(got[ok], xq[src_of[ok] // k])
    assert (got[~ok] == 0xAB).all()  # unused rows untouched
    # walked by token through row_of: the same codes and scale
    _, _, row_of, _ = O.layout(idx, E)
    Xt = torch.full((T * k, d), 0xAB, dtype=torch.uint8, device=DEV)
    xs_t = torch.full((2,), -1.0, dtype=torch.float32, device=DEV)
    moe.moe_dispatch_fp8_by_token(X, torch.from_numpy(row_of.astype(np.int32)).to(DEV), k,
                                  Xeq=Xt, x_scale=xs_t)
    torch.cuda.synchronize()
    assert np.array_equal(Xt.cpu().numpy(), got)
    assert np.array_equal(xs_t.cpu().numpy(), got_s)
    if case == "crafted":
        # codes fixed by the format itself: 1.0625 -> 1.0 (0x38), 1.1875 -> 1.25 (0x3A),
        # 2^-10 -> +0, 3*2^-10 -> 2^-8 (0x02), 448 -> 0x7E, -0 -> 0x80
        row0 = xq[0]
        assert list(row0[[0, 1, 2, 3, 5, 6, 11]]) == [0x7E, 0xFE, 0x38, 0x3A, 0x00, 0x02, 0x80]


# ----------------------------------------------------------------------------
# FP8 grouped GEMM
# ----------------------------------------------------------------------------
def _gemm_fp8_case(counts, N, K, gelu, seed=13):
    counts = np.asarray(counts)
    E = len(counts)
    R = int(counts.sum())
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    A_bits = bits(I.random_bf16((max(R, 1), K), seed, "A"))[:R]
    W_bits = bits(I.random_bf16((E, N, K), seed, "W", 0.05))
    # inputs of the GEMM: the oracle's own codes and scales
    Aq, a_s = O.fp8_quantize(f32_of(A_bits)) if R else (np.zeros((0, K), np.uint8), np.float32(1))
    Wq, w_s = O.fp8_quantize_experts(W_bits)
    out = torch.full((R, N), float("nan"), dtype=torch.bfloat16, device=DEV)
    moe.moe_expert_gemm_fp8(torch.from_numpy(Aq).to(DEV),
                            torch.tensor([a_s], dtype=torch.float32, device=DEV),
                            torch.from_numpy(offsets).to(DEV), torch.from_numpy(Wq).to(DEV),
                            torch.from_numpy(w_s).to(DEV), gelu, out=out)
    ref = np.zeros((R, N))
    for e in range(E):
        lo, hi = offsets[e], offsets[e + 1]
        if hi > lo:
            h = (O.e4m3_decode(Aq[lo:hi]) * float(a_s)) @ (O.e4m3_decode(Wq[e]) * float(w_s[e])).T
            ref[lo:hi] = O.gelu(h) if gelu else h
    return f64(out), ref


FP8_GEMM_CASES = [
    # (counts per expert, N, K, gelu)
    ([64] * 8, 256, 128, True),                        # one K-block of 128 codes
    ([0, 1, 15, 16, 17, 31, 33, 255, 256, 257, 300, 0], 256, 384, True),  # ragged blocks
    ([700], 384, 512, False),                          # several token blocks, N tail of a pair
    ([40, 0, 0, 90], 136, 208, True),                  # N tail, K tail (208 = 128 + 80)
    ([5, 3], 16, 16, False),                           # smallest FP8 dims
    ([128] * 3, 1024, 1024, True),
    ([1] * 64, 256, 256, False),                       # many one-row experts
    ([1030, 990, 1024], 256, 320, True),
    ([300, 129, 97], 128, 256, True),                  # one CTA per tile, > 128 rows per tile
    ([320, 321, 272, 576], 256, 256, True),            # short last token blocks (64, 65, 16 rows)
    ([300, 256, 320, 200, 576, 17] * 16, 768, 256, True),  # merged blocks, several tiles per cluster
]


@pytest.mark.parametrize("counts,N,K,gelu", FP8_GEMM_CASES)
def test_expert_gemm_fp8_parity(counts, N, K, gelu):
    out, ref = _gemm_fp8_case(counts, N, K, gelu)
    assert not np.isnan(out).any()
    assert_close(out, ref, "gemm fp8")
    assert_close(out, ref, "gemm fp8 (tight)", rel=1e-2, abs_=1e-3)


def test_expert_gemm_fp8_leaves_rows_past_offsets_alone():
    offsets = torch.tensor([0, 10, 30], dtype=torch.int32, device=DEV)
    Aq = torch.full((40, 64), 0x38, dtype=torch.uint8, device=DEV)     # all 1.0
    Wq = torch.full((2, 128, 64), 0x30, dtype=torch.uint8, device=DEV)  # all 0.5
    a_s = torch.tensor([2.0], device=DEV)
    w_s = torch.tensor([1.0, 0.25], device=DEV)
    out = torch.full((40, 128), 7.0, dtype=torch.bfloat16, device=DEV)
    moe.moe_expert_gemm_fp8(Aq, a_s, offsets, Wq, w_s, False, out=out)
    # closed form: sum of 64 products 1.0 * 0.5 = 32, times a_s * w_s[e]
    assert (out[:10] == 64.0).all() and (out[10:30] == 16.0).all()
    assert (out[30:] == 7.0).all()


# ----------------------------------------------------------------------------
# FP8 layer
# ----------------------------------------------------------------------------
def _run_fp8_layer(inp, cfg):
    dev_in = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    layer = moe.MoeLayer(dev_in["W1"], dev_in["W2"], cfg.k, cfg.score, cfg.renormalize,
                         Wr=dev_in["Wr"], temperature=cfg.temperature, min_prob=cfg.min_prob,
                         fp8=True)
    idx = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device=DEV)
    g = torch.empty((cfg.T, cfg.k), dtype=torch.float32, device=DEV)
    counts = torch.empty((cfg.E,), dtype=torch.int32, device=DEV)
    Y = layer(dev_in["X"], logits=dev_in["logits"], topk_idx_out=idx, gates_out=g,
              counts_out=counts)
    torch.cuda.synchronize()
    return Y, idx, g, counts, layer


@pytest.mark.parametrize("name", ["tiny", "tiny_threshold"])
def test_layer_fp8_tiny_full_parity(name):
    cfg = I.workload(name)
    inp = I.make_layer_inputs(cfg, 0, device=DEV)
    Y, idx, g, counts, layer = _run_fp8_layer(inp, cfg)
    W1q, s_w = O.fp8_quantize_experts(bits(inp["W1"]))
    assert np.array_equal(layer.W1q.cpu().numpy(), W1q)
    assert np.array_equal(layer.w1_scale.cpu().numpy(), s_w)
    ref = O.layer_forward_fp8(bits(inp["X"]), W1q, s_w, bits(inp["W2"]), cfg.k, cfg.score,
                              cfg.renormalize, logits=inp["logits"].numpy(),
                              temperature=cfg.temperature, min_prob=cfg.min_prob)
    assert np.array_equal(idx.cpu().numpy(), ref["topk_idx"])
    assert np.array_equal(counts.cpu().numpy(), ref["counts"])
    assert_close(f64(Y), ref["Y"], f"{name} Y (fp8)")
    # FP8 stays near the bf16 layer (quantisation error of GEMM-1's operands only)
    bf = O.layer_forward(bits(inp["X"]), bits(inp["W1"]), bits(inp["W2"]), cfg.k, cfg.score,
                         cfg.renormalize, logits=inp["logits"].numpy(),
                         temperature=cfg.temperature, min_prob=cfg.min_prob)
    assert np.abs(f64(Y) - bf["Y"]).max() <= 0.1 * np.abs(bf["Y"]).max()


def test_layer_fp8_workspace_is_the_bf16_one_and_deterministic():
    cfg = I.workload("tiny")
    inp = I.make_layer_inputs(cfg, 2, device=DEV)
    Y1 = _run_fp8_layer(inp, cfg)[0].clone()
    Y2 = _run_fp8_layer(inp, cfg)[0]
    assert torch.equal(Y1.view(torch.int16), Y2.view(torch.int16))


def _expert_codes_rows(W1_dev, e, rows):
    """Oracle codes of selected rows of expert e: the scale needs the whole expert's amax."""
    full = f32_of(bits(W1_dev[e]))
    amax = np.float32(np.abs(full).max())
    q, s = O.fp8_quantize(full[rows], amax=amax)
    return q, s


@pytest.mark.slow
def test_layer_fp8_mixtral_sampled():
    """Full Mixtral-shaped layer (T=4096, d=4096, E=8, k=2, f=14336) in FP8 mode.

    Checked element by element where the oracle can afford it: sampled rows of
    every expert's W1 codes, the activation scale, sampled dispatched rows, and
    Y for sampled tokens whose two experts fall in one pair of experts (the
    oracle quantises those two experts' W1 in full)."""
    cfg = I.workload("mixtral")
    inp = I.make_layer_inputs(cfg, 0, device=DEV)
    Y, idx, g, counts, layer = _run_fp8_layer(inp, cfg)
    X_bits = bits(inp["X"])
    rng = np.random.default_rng(3)
    for e in range(cfg.E):  # weight codes: sampled rows, bit-exact
        rows = np.sort(rng.choice(cfg.f, size=24, replace=False))
        q, s = _expert_codes_rows(inp["W1"], e, rows)
        assert layer.w1_scale[e].item() == s
        assert np.array_equal(layer.W1q[e][torch.from_numpy(rows).to(DEV)].cpu().numpy(), q)
    xq, x_s = O.fp8_quantize(f32_of(X_bits))
    # the oracle's own routing (the router runs on the bf16 tokens in both modes);
    # tokens whose k-th and (k+1)-th logits lie within rounding may route either way
    x = O.bf16_to_f64(X_bits)
    wr = O.bf16_to_f64(bits(inp["Wr"]))
    Lref = O.router_logits(x, wr)
    eps = 2 * (cfg.d * 2.0 ** -24) * float((np.abs(x) @ np.abs(wr).T).max())
    srt = -np.sort(-Lref, axis=1)
    ties = (srt[:, cfg.k - 1] - srt[:, cfg.k]) <= eps
    ref_idx, ref_g = O.route(Lref.astype(np.float32), cfg.k, cfg.score, cfg.renormalize)
    gi = idx.cpu().numpy()
    mism = np.any(gi != ref_idx, axis=1)
    assert not (mism & ~ties).any()
    # dispatched rows, through the standalone call on the oracle's routing
    _, _, _, src_of = O.layout(ref_idx, cfg.E)
    Xeq, xs = moe.moe_dispatch_fp8(inp["X"].to(DEV), torch.from_numpy(src_of).to(DEV), cfg.k)
    assert xs[0].item() == x_s
    pick = np.sort(rng.choice(cfg.R, size=64, replace=False))
    assert np.array_equal(Xeq[torch.from_numpy(pick).to(DEV)].cpu().numpy(),
                          xq[src_of[pick] // cfg.k])
    # Y on tokens routed to the most common expert pair
    pairs = np.sort(ref_idx, axis=1)
    keys, cnt = np.unique(pairs, axis=0, return_counts=True)
    ea, eb = keys[int(cnt.argmax())]
    toks = np.where((pairs[:, 0] == ea) & (pairs[:, 1] == eb) & ~ties)[0][:12]
    assert len(toks) >= 4
    W1q, s_w = {}, {}
    for e in (int(ea), int(eb)):
        W1q[e], s_w[e] = O.fp8_quantize(f32_of(bits(inp["W1"][e])))
    W2 = {e: bits(inp["W2"][e]) for e in (int(ea), int(eb))}
    ref = O.layer_forward_fp8_tokens(xq, x_s, W1q, s_w, W2, ref_idx, ref_g, toks)
    assert_close(f64(Y[torch.from_numpy(toks).to(DEV)]), ref, "mixtral fp8 Y")
