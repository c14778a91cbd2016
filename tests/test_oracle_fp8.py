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
