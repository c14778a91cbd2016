"""Pins for the oracle's FP8 path (ThunderEP PCIe blog §3.3, §5.2: activations cast
to FP8 with a per-tensor dynamic scale).  E4M3 rounding is checked against the
format's definition (every code), torch's float8_e4m3fn cast, and closed forms."""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from combine_moe_route_14_b200 import inputs as I


def test_every_code_round_trips():
    codes = np.arange(256, dtype=np.uint8)
    vals = O.e4m3_decode(codes)
    finite = ~np.isnan(vals)
    assert finite.sum() == 254                                   # 0x7F, 0xFF are NaN
    assert np.array_equal(O.e4m3_encode(vals[finite]), codes[finite])
    assert np.nanmax(vals) == 448.0 and np.nanmin(vals) == -448.0


def test_closed_forms():
    enc = lambda v: int(O.e4m3_encode(np.array([v]))[0])
    assert enc(1.0) == 0x38 and enc(-1.0) == 0xB8
    assert enc(448.0) == 0x7E and enc(1e6) == 0x7E and enc(-500.0) == 0xFE   # saturation
    assert enc(2.0 ** -9) == 0x01                                  # smallest subnormal
    assert enc(2.0 ** -10) == 0x00                                 # halfway to 0: even code 0
    assert enc(1.0 + 1 / 16) == 0x38                               # halfway 1 .. 1.125: even
    assert enc(1.0 + 3 / 16) == 0x3A                               # halfway 1.125 .. 1.25: even
    assert enc(-0.0) == 0x80


def test_matches_torch_float8_cast_in_range():
    x = I.random_f32((20000,), 4, "fp8", 60.0).numpy()
    x = x[np.abs(x) < 440]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(O.e4m3_encode(x), ref)


def test_quantize_uses_fp32_steps_and_hits_the_range():
    x = I.random_f32((4096,), 5, "q", 3.0).numpy()
    codes, s = O.fp8_quantize(x)
    amax = np.float32(np.abs(x).max())
    assert s == np.float32(amax / np.float32(448.0))
    i = int(np.abs(x).argmax())
    assert abs(O.e4m3_decode(codes[i:i + 1])[0]) == 448.0         # the largest maps to 448
    deq = O.e4m3_decode(codes) * float(s)
    assert np.abs(deq - x).max() <= amax * 2.0 ** -4               # half an ulp at 448 scale
    zero_codes, zs = O.fp8_quantize(np.zeros(8, np.float32))
    assert (zero_codes == 0).all() and zs == 1.0


def test_fp8_layer_dense_special_case():
    """E=1, k=1: the FP8 layer is GELU(deq(Xq) deq(W1q)^T) W2^T on the dequantised values."""
    T, d, f = 24, 32, 16
    X = I.f32_to_bf16_bits(I.random_f32((T, d), 6, "X").numpy())
    W1 = I.f32_to_bf16_bits(I.random_f32((1, f, d), 6, "W1", 0.2).numpy())
    W2 = I.f32_to_bf16_bits(I.random_f32((1, d, f), 6, "W2", 0.2).numpy())
    W1q, s_w = O.fp8_quantize_experts(W1)
    out = O.layer_forward_fp8(X, W1q, s_w, W2, 1, logits=I.random_f32((T, 1), 6, "L").numpy())
    xq, s_x = O.fp8_quantize(O.bf16_to_f64(X).astype(np.float32))
    x = torch.from_numpy(O.e4m3_decode(xq) * float(s_x))
    w1 = torch.from_numpy(O.e4m3_decode(W1q[0]) * float(s_w[0]))
    w2 = torch.from_numpy(O.bf16_to_f64(W2[0]))
    ref = torch.nn.functional.gelu(x @ w1.T, approximate="none") @ w2.T
    np.testing.assert_allclose(out["Y"], ref.numpy(), rtol=1e-12, atol=1e-13)
    # and it stays close to the bf16 layer (quantisation error only)
    bf = O.layer_forward(X, W1, W2, 1, logits=I.random_f32((T, 1), 6, "L").numpy())
    assert np.abs(out["Y"] - bf["Y"]).max() <= 0.1 * np.abs(bf["Y"]).max()


def _encode_ties_away(x):
    a = np.asarray(x, np.float64)
    mag = np.abs(a)
    hi = np.searchsorted(O._E4M3_POS, mag, side="left").clip(0, 0x7E)
    lo = (hi - 1).clip(0, 0x7E)
    pick_lo = (mag - O._E4M3_POS[lo]) < (O._E4M3_POS[hi] - mag)
    return (np.where(pick_lo, lo, hi) | np.where(np.signbit(a), 0x80, 0)).astype(np.uint8)


def test_planted_rounding_mistake_is_caught():
    with pytest.raises(AssertionError):
        assert _encode_ties_away(np.array([1.0 + 1 / 16]))[0] == 0x38


def test_sampled_tokens_equal_the_whole_fp8_layer():
    T, d, E, k, f = 40, 32, 4, 2, 48
    X = I.f32_to_bf16_bits(I.random_f32((T, d), 7, "X").numpy())
    W1 = I.f32_to_bf16_bits(I.random_f32((E, f, d), 7, "W1", 0.1).numpy())
    W2 = I.f32_to_bf16_bits(I.random_f32((E, d, f), 7, "W2", 0.1).numpy())
    L = I.random_f32((T, E), 7, "L").numpy()
    W1q, s_w = O.fp8_quantize_experts(W1)
    full = O.layer_forward_fp8(X, W1q, s_w, W2, k, logits=L)
    toks = np.array([0, 3, 17, 39])
    part = O.layer_forward_fp8_tokens(full["Xq"], full["x_scale"], W1q, s_w, W2,
                                      full["topk_idx"], full["gates"], toks)
    np.testing.assert_allclose(part, full["Y"][toks], rtol=1e-12, atol=1e-14)
    # the dispatched rows are the token's codes, one per (token, slot)
    ok = full["src_of"] >= 0
    assert np.array_equal(full["Xe_q"][ok], full["Xq"][full["src_of"][ok] // k])


# ----------------------------------------------------------------------------
# per-expert weight scales (one scale per expert matrix; the pages leave weight
# quantisation open, so each expert's W1 gets its own per-tensor scale by the
# same rule the blog gives for activations, ThunderEP PCIe blog §3.3, §5.2)
# ----------------------------------------------------------------------------
# expert magnitudes x1, x10, x300: a shared scale or a shared index is far off
_MAGS = (0.02, 0.2, 6.0)


def _experts_of_mixed_magnitude(shape_rc, seed):
    rows, cols = shape_rc
    return np.stack([I.f32_to_bf16_bits(I.random_f32((rows, cols), seed, f"W{e}", m).numpy())
                     for e, m in enumerate(_MAGS)])


def _torch_quantize_one(w_bits):
    """Independent per-tensor E4M3 quantisation of one bf16 matrix with torch's
    float8_e4m3fn cast: amax, inv = 448/amax and w*inv in fp32."""
    w = torch.from_numpy(np.asarray(w_bits).view(np.int16)).view(torch.bfloat16).float()
    amax = w.abs().max()
    inv = torch.tensor(448.0, dtype=torch.float32) / amax
    codes = (w * inv).to(torch.float8_e4m3fn)
    scale = amax / torch.tensor(448.0, dtype=torch.float32)
    return codes, scale


def check_per_expert_scales(quantize_experts_fn):
    W = _experts_of_mixed_magnitude((24, 64), 11)
    codes, s = quantize_experts_fn(W)
    assert s.shape == (len(_MAGS),) and s.dtype == np.float32
    for e in range(len(_MAGS)):
        w = O.bf16_to_f64(W[e]).astype(np.float32)
        amax = np.float32(np.abs(w).max())
        assert s[e] == np.float32(amax / np.float32(448.0)), (e, s[e], amax)
        i = np.unravel_index(int(np.abs(w).argmax()), w.shape)
        assert codes[e][i] in (0x7E, 0xFE), (e, hex(codes[e][i]))   # +-448: the range is used
        ref_codes, ref_s = _torch_quantize_one(W[e])
        assert np.array_equal(codes[e], ref_codes.view(torch.uint8).numpy()), e
        assert s[e] == np.float32(ref_s.item())


def _torch_fp8_layer(X_bits, W1_bits, W2_bits, L, k):
    """The FP8 layer composed in torch (fp64 math after torch's own E4M3 casts):
    per token, the softmax top-k renormalised gates over its chosen experts,
    each expert's GELU(deq(x) deq(W1[e])^T) W2[e]^T, the gate-weighted sum."""
    X = torch.from_numpy(np.asarray(X_bits).view(np.int16)).view(torch.bfloat16).float()
    amax = X.abs().max()
    xq = (X * (torch.tensor(448.0) / amax)).to(torch.float8_e4m3fn)
    x = xq.double() * float(amax / torch.tensor(448.0))
    w1 = []
    for e in range(W1_bits.shape[0]):
        c, s = _torch_quantize_one(W1_bits[e])
        w1.append(c.double() * float(s))
    w2 = torch.from_numpy(O.bf16_to_f64(W2_bits))
    Lt = torch.from_numpy(np.asarray(L, np.float64))
    vals, idx = torch.topk(Lt, k, dim=1)               # distinct logits: order is unique
    g = torch.softmax(vals, dim=1)
    Y = torch.zeros(X.shape, dtype=torch.float64)
    for t in range(X.shape[0]):
        for j in range(k):
            e = int(idx[t, j])
            h = torch.nn.functional.gelu(x[t] @ w1[e].T, approximate="none")
            Y[t] += g[t, j] * (h @ w2[e].T)
    return Y.numpy()


def _mixed_fp8_case():
    T, d, f, k = 20, 64, 24, 2
    E = len(_MAGS)
    X = I.f32_to_bf16_bits(I.random_f32((T, d), 12, "X").numpy())
    W1 = _experts_of_mixed_magnitude((f, d), 12)
    W2 = I.f32_to_bf16_bits(I.random_f32((E, d, f), 12, "W2", 0.1).numpy())
    L = I.random_f32((T, E), 12, "L").numpy()
    return X, W1, W2, L, k


def check_fp8_layer_per_expert(layer_fn, tokens_fn=None):
    """Each expert's rows use that expert's codes and scale: the whole layer, and
    the per-token form, equal the torch composition above."""
    X, W1, W2, L, k = _mixed_fp8_case()
    W1q, s_w = O.fp8_quantize_experts(W1)
    ref = _torch_fp8_layer(X, W1, W2, L, k)
    out = layer_fn(X, W1q, s_w, W2, k, logits=L)
    assert len(set(out["topk_idx"][:, 0].tolist())) == 3   # every expert is used
    np.testing.assert_allclose(out["Y"], ref, rtol=1e-9, atol=1e-12)
    if tokens_fn is not None:
        toks = np.arange(X.shape[0])
        part = tokens_fn(out["Xq"], out["x_scale"], W1q, s_w, W2, out["topk_idx"],
                         out["gates"], toks)
        np.testing.assert_allclose(part, ref, rtol=1e-9, atol=1e-12)


def test_per_expert_weight_scales():
    check_per_expert_scales(O.fp8_quantize_experts)


def test_fp8_layer_uses_each_experts_scale():
    check_fp8_layer_per_expert(O.layer_forward_fp8, O.layer_forward_fp8_tokens)


# planted mistakes, on the CPU: each must fail the pins above
def _quantize_experts_one_global_scale(W_bits):
    W = np.asarray(W_bits)
    codes, s = O.fp8_quantize(O.bf16_to_f64(W).astype(np.float32))
    return codes, np.full(W.shape[0], s, dtype=np.float32)


def _layer_fp8_scale_of_expert0(X, W1q, s_w, W2, k, **kw):
    return O.layer_forward_fp8(X, W1q, np.full_like(s_w, s_w[0]), W2, k, **kw)


def _tokens_fp8_scale_of_expert0(Xq, x_scale, W1q, s_w, *rest):
    return O.layer_forward_fp8_tokens(Xq, x_scale, W1q, np.full_like(s_w, s_w[0]), *rest)


def _layer_fp8_codes_of_expert0(X, W1q, s_w, W2, k, **kw):
    return O.layer_forward_fp8(X, np.stack([W1q[0]] * W1q.shape[0]), s_w, W2, k, **kw)


@pytest.mark.parametrize("run", [
    lambda: check_per_expert_scales(_quantize_experts_one_global_scale),
    lambda: check_fp8_layer_per_expert(_layer_fp8_scale_of_expert0),
    lambda: check_fp8_layer_per_expert(O.layer_forward_fp8, _tokens_fp8_scale_of_expert0),
    lambda: check_fp8_layer_per_expert(_layer_fp8_codes_of_expert0),
], ids=["one-global-weight-scale", "layer-uses-w1_scale[0]", "tokens-use-w1_scale[0]",
        "layer-uses-expert0-codes"])
def test_planted_per_expert_mistake_is_caught(run):
    with pytest.raises(AssertionError):
        run()
