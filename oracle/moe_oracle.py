"""CPU oracle for one MoE layer: route -> layout -> dispatch -> expert FFN -> combine.

TEST INFRASTRUCTURE ONLY.  This module exists to check the CUDA library.  Only
the test-suite, the package's smoke check and the benchmark's CPU-baseline leg
may import it; the library itself never calls it, and it imports nothing from
the library (the two share no code).  It is deliberately plain and slow: numpy
in float64, per-step loops where the pages describe a per-item rule, and no
blocking, fusion or reordering beyond what each definition states.

Sources (web pages on MoE expert-parallel dispatch/combine):
  [TEP]  "ThunderEP" PCIe blog (dpshk.com), §1.1 (router scores, top-1/top-2,
         dispatch / combine), §2.1 (top-k indices and gate values travel with
         the token; combine is a gate-weighted sum), §2.2 (group tokens by
         destination expert).
  [DYS]  DySHARP review (marsggbo, "MoE 通信里一半流量是重复的"), §1 (dispatch =
         the same token sent to its k experts; combine = the k expert results
         reduced into one), §3.1 item 3 (AL table: logical i-th token -> layout
         index in a dense per-expert tensor, layout blocks allocated
         incrementally; combine looks rows up through the same table), §3.2
         (GEMM-1 -> GEMM-2 per expert).
  [GPT]  GPT-4 "1.8T parameters / 2%" article (CSDN), §2.3 (softmax with a
         temperature, then top-k), §3.1 table (expert = Linear -> GELU ->
         Linear), §4.1 (router code: logits = router_proj(h), softmax, topk).

Readings where the pages are silent (each is also listed in the design notes):
  * top-k selects on the fp32 logit (softmax and sigmoid are strictly
    increasing, so this is top-k by score) with ties broken toward the lower
    expert id; slots are ordered by descending logit.
  * gates: softmax over the chosen logits (= softmax over all experts
    renormalised over the chosen k), sigmoid scores renormalised, or, with
    renormalize=0, the plain softmax / sigmoid probability of each chosen
    expert.  No capacity limit.
  * routing variants ([GPT] §2.3, §4.1): scores use logits / temperature
    (the top-k order is unchanged for temperature > 0); with a threshold
    min_prob > 0, a chosen slot whose probability (softmax over all E, or
    sigmoid) is not above min_prob is dropped: index -1, gate 0, no layout
    row.  Renormalised gates divide by the sum over the kept slots.  Defaults
    (temperature 1, no threshold) keep every slot: R = T*k rows.
  * rows inside an expert block are in ascending (token, slot) order; blocks
    are in expert order 0..E-1.
  * GELU is the exact erf form 0.5*x*(1+erf(x/sqrt 2)).
  * everything is float64 from the same bf16 / fp32 input bytes; H and Ye
    are NOT rounded to bf16 here (the GPU does; the tolerance covers it).
  * FP8 mode ([TEP] §3.3, §5.2: activations cast to FP8 with one dynamic
    per-tensor scale before they move, cast back after): the token matrix X
    is quantised to E4M3 with inv = 448 / amax(|X|) and codes =
    E4M3(x * inv), both fp32 operations and round-to-nearest-even with
    saturation, so the codes are an integer result both sides decide in the
    same precision.  GEMM-1 then runs on the FP8 operands (the pages' FP8
    tensor-core compute); the pages do not say how the weights get to FP8,
    so each expert's W1 is quantised once with its own per-tensor scale.
    GEMM-2 and combine stay bf16.

Parity status: every function here is pinned by tests that do not reuse its
code (brute force, invariants, closed forms, library special cases).
"""
from __future__ import annotations

import numpy as np
from scipy.special import erf as _erf

SOFTMAX = "softmax"
SIGMOID = "sigmoid"


# ----------------------------------------------------------------------------
# bf16 <-> float conversion of the input bytes
# ----------------------------------------------------------------------------
def bf16_to_f64(bits) -> np.ndarray:
    """bf16 bit patterns (uint16 / int16 array) -> exact float64 values.

    bf16 is the upper half of an IEEE binary32, so widening is exact.
    """
    b = np.asarray(bits).view(np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


# ----------------------------------------------------------------------------
# a0: router linear   [GPT] §4.1 (router_proj), §3.1 table (router MLP)
# ----------------------------------------------------------------------------
def router_logits(X, Wr) -> np.ndarray:
    """L[t, e] = sum_c X[t, c] * Wr[e, c]   (float64 values; inputs float arrays)."""
    X = np.asarray(X, dtype=np.float64)
    Wr = np.asarray(Wr, dtype=np.float64)
    return X @ Wr.T


# ----------------------------------------------------------------------------
# a1: scores, top-k, gates   [GPT] §2.3, §4.1; [TEP] §1.1, §2.1
# ----------------------------------------------------------------------------
def topk_order(logits: np.ndarray, k: int) -> np.ndarray:
    """Per token, the k experts with the largest logit; ties -> lower expert id.

    A full stable sort of each row by descending logit, then the first k.
    Rejects NaN / inf (undefined for the library).
    """
    L = np.asarray(logits)
    if not np.all(np.isfinite(L)):
        raise ValueError("logits must be finite")
    T, E = L.shape
    if not (1 <= k <= E):
        raise ValueError("need 1 <= k <= E")
    # -L is exact; a stable sort keeps equal keys (including +0 / -0) in id order.
    order = np.argsort(-L, axis=1, kind="stable")
    return order[:, :k].astype(np.int32)


def gates_from_logits(logits: np.ndarray, idx: np.ndarray, score: str,
                      renormalize: int, temperature: float = 1.0,
                      min_prob: float = 0.0):
    """Gate value of each chosen slot and whether the slot is kept, float64.

    With z = logits / temperature:
    softmax:  p_e = exp(z_e - m) / sum_{e'} exp(z_e' - m)  over all E experts;
    sigmoid:  s_e = 1 / (1 + exp(-z_e)).
    A slot is kept when min_prob <= 0 or its probability exceeds min_prob.
    renormalize=1: gate = prob / sum of the kept slots' probs; else the prob.
    Dropped slots get gate 0.  Returns (gates [T,k], keep [T,k] bool).
    """
    if not temperature > 0:
        raise ValueError("temperature must be > 0")
    L = np.asarray(logits, dtype=np.float64) / float(temperature)
    T, E = L.shape
    chosen = np.take_along_axis(L, idx.astype(np.int64), axis=1)  # [T, k]
    if score == SOFTMAX:
        m = L.max(axis=1, keepdims=True)
        prob = np.exp(chosen - m) / np.exp(L - m).sum(axis=1, keepdims=True)
    elif score == SIGMOID:
        prob = 1.0 / (1.0 + np.exp(-chosen))
    else:
        raise ValueError(f"unknown score {score!r}")
    keep = np.ones_like(prob, dtype=bool) if min_prob <= 0 else prob > min_prob
    kept = np.where(keep, prob, 0.0)
    if renormalize:
        den = kept.sum(axis=1, keepdims=True)
        gates = np.divide(kept, den, out=np.zeros_like(kept), where=den > 0)
    else:
        gates = kept
    return gates, keep


def route(logits, k: int, score: str = SOFTMAX, renormalize: int = 1,
          temperature: float = 1.0, min_prob: float = 0.0):
    """(topk_idx [T,k] int32 with -1 for dropped slots, gates [T,k] float64)."""
    idx = topk_order(logits, k)
    gates, keep = gates_from_logits(logits, idx, score, renormalize, temperature, min_prob)
    return np.where(keep, idx, -1).astype(np.int32), gates


# ----------------------------------------------------------------------------
# a2 + a3: counts, offsets, AL table   [DYS] §3.1 item 3; [TEP] §2.2
# ----------------------------------------------------------------------------
def layout(topk_idx, E: int):
    """Map each logical slot i = t*k + j to its row in the dense per-expert tensor.

    Walks the slots in logical order and hands each one the next free row of
    its expert's block (the incremental layout-block allocation of the AL
    table).  Slot value -1 marks a dropped slot: it takes no row (row_of -1).
    Returns counts [E], offsets [E+1] (exclusive prefix sum, offsets[E] =
    number of kept slots), row_of [R] (logical -> layout) and src_of [R]
    (layout -> logical for rows below offsets[E], -1 above), all int32.
    """
    flat = np.asarray(topk_idx, dtype=np.int64).reshape(-1)
    R = flat.size
    if R and (flat.min() < -1 or flat.max() >= E):
        raise ValueError("expert id out of range")
    counts = np.zeros(E, dtype=np.int64)
    for e in flat:
        if e >= 0:
            counts[e] += 1
    offsets = np.zeros(E + 1, dtype=np.int64)
    for e in range(E):
        offsets[e + 1] = offsets[e] + counts[e]
    cursor = offsets[:E].copy()
    row_of = np.full(R, -1, dtype=np.int64)
    for i in range(R):
        e = flat[i]
        if e < 0:
            continue
        row_of[i] = cursor[e]
        cursor[e] += 1
    src_of = np.full(R, -1, dtype=np.int64)
    kept = row_of >= 0
    src_of[row_of[kept]] = np.arange(R)[kept]
    return (counts.astype(np.int32), offsets.astype(np.int32),
            row_of.astype(np.int32), src_of.astype(np.int32))


# ----------------------------------------------------------------------------
# a4: dispatch   [DYS] §1 (one token -> its k experts); [TEP] §1.1
# ----------------------------------------------------------------------------
def dispatch(X, src_of, k: int) -> np.ndarray:
    """Xe[r, :] = X[src_of[r] // k, :] for the layout's rows (src_of[r] >= 0); a copy,
    on any dtype (bf16 bits included).  Rows past the kept slots are returned as zeros."""
    X = np.asarray(X)
    src = np.asarray(src_of, dtype=np.int64)
    out = np.zeros((src.size,) + X.shape[1:], dtype=X.dtype)
    ok = src >= 0
    out[ok] = X[src[ok] // k]
    return out


# ----------------------------------------------------------------------------
# a5 + a6: expert FFN   [GPT] §3.1 table (Linear -> GELU -> Linear); [DYS] §3.2
# ----------------------------------------------------------------------------
def gelu(x):
    """Exact GELU: 0.5 * x * (1 + erf(x / sqrt(2)))."""
    x = np.asarray(x, dtype=np.float64)
    return 0.5 * x * (1.0 + _erf(x / np.sqrt(2.0)))


def expert_gemm1(Xe_rows, W1_e) -> np.ndarray:
    """H = GELU(Xe_rows @ W1_e^T), W1_e [f, d] (nn.Linear [out, in] layout)."""
    return gelu(np.asarray(Xe_rows, np.float64) @ np.asarray(W1_e, np.float64).T)


def expert_gemm2(H_rows, W2_e) -> np.ndarray:
    """Ye = H_rows @ W2_e^T, W2_e [d, f]."""
    return np.asarray(H_rows, np.float64) @ np.asarray(W2_e, np.float64).T


def expert_ffn(Xe, offsets, W1, W2):
    """Per expert block e (rows offsets[e]..offsets[e+1]): H = GELU(Xe W1[e]^T), Ye = H W2[e]^T.

    ``Xe`` float values [R, d]; ``W1`` [E, f, d] and ``W2`` [E, d, f] either
    float arrays or bf16 bit arrays (uint16/int16), widened per expert.
    Returns (H [R, f], Ye [R, d]) float64.
    """
    Xe = np.asarray(Xe, np.float64)
    R, d = Xe.shape
    E = len(offsets) - 1
    f = W1.shape[1]
    H = np.zeros((R, f))
    Ye = np.zeros((R, d))
    for e in range(E):
        a, b = int(offsets[e]), int(offsets[e + 1])
        if a == b:
            continue
        w1 = _as_f64(W1[e])
        w2 = _as_f64(W2[e])
        H[a:b] = expert_gemm1(Xe[a:b], w1)
        Ye[a:b] = expert_gemm2(H[a:b], w2)
    return H, Ye


def _as_f64(w):
    w = np.asarray(w)
    if w.dtype in (np.uint16, np.int16):
        return bf16_to_f64(w)
    return w.astype(np.float64)


# ----------------------------------------------------------------------------
# a7: combine   [DYS] §1 (k results reduced into one); [TEP] §1.1, §2.1
# ----------------------------------------------------------------------------
def combine(Ye, row_of, gates, k: int) -> np.ndarray:
    """Y[t, :] = sum_{j<k} gates[t, j] * Ye[row_of[t*k + j], :]  (slot order), float64.

    Dropped slots (row_of -1) contribute nothing."""
    Ye = np.asarray(Ye, np.float64)
    g = np.asarray(gates, np.float64)
    T = g.shape[0]
    rows = np.asarray(row_of, np.int64).reshape(T, k)
    Y = np.zeros((T, Ye.shape[1]))
    for j in range(k):
        kept = rows[:, j] >= 0
        Y[kept] += g[kept, j:j + 1] * Ye[rows[kept, j]]
    return Y


# ----------------------------------------------------------------------------
# the whole layer
# ----------------------------------------------------------------------------
def layer_forward(X_bits, W1_bits, W2_bits, k, score=SOFTMAX, renormalize=1,
                  logits=None, Wr_bits=None, temperature=1.0, min_prob=0.0):
    """Full layer on the CPU.  Exactly one of ``logits`` (fp32) / ``Wr_bits`` is given.

    With router weights, the logits are computed in float64 and rounded to
    fp32 before routing, so the top-k decision is taken in fp32 as on the GPU.
    Returns a dict with every intermediate.
    """
    X = bf16_to_f64(X_bits)
    T, d = X.shape
    E = W1_bits.shape[0]
    if (logits is None) == (Wr_bits is None):
        raise ValueError("give exactly one of logits / Wr_bits")
    if logits is None:
        L = router_logits(X, bf16_to_f64(Wr_bits)).astype(np.float32)
    else:
        L = np.asarray(logits, dtype=np.float32)
    idx, gates = route(L, k, score, renormalize, temperature, min_prob)
    counts, offsets, row_of, src_of = layout(idx, E)
    Xe = dispatch(X, src_of, k)
    H, Ye = expert_ffn(Xe, offsets, W1_bits, W2_bits)
    Y = combine(Ye, row_of, gates, k)
    return dict(logits=L, topk_idx=idx, gates=gates, counts=counts, offsets=offsets,
                row_of=row_of, src_of=src_of, Xe=Xe, H=H, Ye=Ye, Y=Y)


def layer_forward_tokens(X_bits, W1_bits, W2_bits, topk_idx, gates, tokens):
    """Y for a subset of tokens, each computed on its own.

    A token's output depends only on its own row of X and its own k routed
    experts (dispatch copies it, each expert applies its FFN to that row,
    combine sums the k results), so the layer can be evaluated one token at a
    time: Y[t] = sum_j gates[t,j] * W2[e_j] GELU(W1[e_j] x_t).  Used to check
    full-size runs on a sample of tokens.  Returns float64 [len(tokens), d].
    """
    tokens = np.asarray(tokens, dtype=np.int64)
    k = topk_idx.shape[1]
    X = bf16_to_f64(np.asarray(X_bits)[tokens])
    idx = np.asarray(topk_idx)[tokens]
    g = np.asarray(gates, np.float64)[tokens]
    # group the (token, slot) pairs by expert so each expert's weights are widened once
    ye = np.zeros((len(tokens), k, X.shape[1]))
    by_e = {}
    for n in range(len(tokens)):
        for j in range(k):
            if idx[n, j] >= 0:  # dropped slots contribute nothing
                by_e.setdefault(int(idx[n, j]), []).append((n, j))
    for e, pairs in sorted(by_e.items()):
        ns = np.array([p[0] for p in pairs])
        js = np.array([p[1] for p in pairs])
        ye[ns, js] = expert_gemm2(expert_gemm1(X[ns], _as_f64(W1_bits[e])), _as_f64(W2_bits[e]))
    Y = np.zeros((len(tokens), X.shape[1]))
    for j in range(k):  # slot order, as in combine()
        Y += g[:, j:j + 1] * ye[:, j]
    return Y


def tolerance(ref: np.ndarray, rel: float = 2e-2, abs_: float = 1e-3) -> float:
    """Float parity bound max|out - ref| <= rel * max|ref| + abs (bf16 I/O, fp32 accumulate)."""
    ref = np.asarray(ref, np.float64)
    return rel * (float(np.abs(ref).max()) if ref.size else 0.0) + abs_


# ----------------------------------------------------------------------------
# FP8 dispatch + FP8 GEMM-1   [TEP] §3.3 (activations cast to fp8 with a
# per-tensor dynamic scale before the transfer; tensor cores that support
# FP8 compute on it natively), §5.2 (cast before sending, per-tensor scale)
# ----------------------------------------------------------------------------
# E4M3: 1 sign, 4 exponent (bias 7), 3 mantissa bits; no infinities; the
# largest finite value is 448 (exponent 15, mantissa 6); 0x7F / 0xFF is NaN.
E4M3_MAX = 448.0


def e4m3_decode(codes) -> np.ndarray:
    """E4M3 codes (uint8) -> float64 values, from the format's definition."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c >> 7, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    val = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * 2.0 ** (e - 7.0))
    val = np.where((e == 15) & (m == 7), np.nan, val)
    return sign * val


_E4M3_POS = e4m3_decode(np.arange(0x7F, dtype=np.uint8))  # codes 0x00..0x7E, increasing


def e4m3_encode(x) -> np.ndarray:
    """Round finite values to E4M3: nearest representable value, ties to the
    even code (mantissa LSB 0), magnitudes past 448 saturate to 448."""
    a = np.asarray(x, dtype=np.float64)
    mag = np.abs(a)
    hi = np.searchsorted(_E4M3_POS, mag, side="left").clip(0, 0x7E)  # first value >= mag
    lo = (hi - 1).clip(0, 0x7E)
    d_hi = _E4M3_POS[hi] - mag
    d_lo = mag - _E4M3_POS[lo]
    pick_lo = (d_lo < d_hi) | ((d_lo == d_hi) & (lo % 2 == 0))
    code = np.where(pick_lo, lo, hi)
    code = np.where(mag >= E4M3_MAX, 0x7E, code)          # saturate
    code = code | np.where(np.signbit(a), 0x80, 0)
    code = np.where(np.isnan(a), 0x7F, code)
    return code.astype(np.uint8)


def fp8_quantize(x_f32, amax=None):
    """Per-tensor dynamic FP8 quantisation, every step in fp32 as the kernel does.

    amax = max |x| (the tensor's own unless given); inv = 448 / amax and
    x * inv are fp32 operations (round to nearest); codes = e4m3_encode of the
    product; the dequantisation scale is s = amax / 448 (fp32).  amax = 0
    gives inv = s = 1.  Returns (codes uint8, s float32).
    """
    x = np.asarray(x_f32, dtype=np.float32)
    if amax is None:
        amax = np.float32(np.abs(x).max()) if x.size else np.float32(0)
    amax = np.float32(amax)
    if amax > 0:
        inv = np.float32(E4M3_MAX) / amax
        s = amax / np.float32(E4M3_MAX)
    else:
        inv = np.float32(1.0)
        s = np.float32(1.0)
    y = (x * inv).astype(np.float32)
    return e4m3_encode(y), np.float32(s)


def fp8_quantize_experts(W_bits):
    """Per-expert quantisation of bf16 expert weights [E, rows, cols]:
    one scale per expert.  Returns (codes uint8 [E, rows, cols], s [E] float32)."""
    W = np.asarray(W_bits)
    E = W.shape[0]
    codes = np.empty(W.shape, dtype=np.uint8)
    s = np.empty(E, dtype=np.float32)
    for e in range(E):
        w = bf16_to_f64(W[e]).astype(np.float32)  # exact: bf16 widens to fp32
        codes[e], s[e] = fp8_quantize(w)
    return codes, s


def fp8_gemm1(Xq_rows, x_scale, W1q_e, w_scale_e) -> np.ndarray:
    """H = GELU((Xq * s_x) @ (W1q[e] * s_w[e])^T) on the dequantised FP8 operands."""
    x = e4m3_decode(Xq_rows) * float(x_scale)
    w = e4m3_decode(W1q_e) * float(w_scale_e)
    return gelu(x @ w.T)


def layer_forward_fp8(X_bits, W1q, w1_scale, W2_bits, k, score=SOFTMAX, renormalize=1,
                      logits=None, Wr_bits=None, temperature=1.0, min_prob=0.0):
    """The layer with FP8 dispatch and FP8 GEMM-1 (GEMM-2 and combine as in bf16).

    The dispatched activations are the tokens quantised with one per-tensor
    scale over all of X; GEMM-1 runs on the dequantised FP8 operands.
    """
    X = bf16_to_f64(X_bits)
    T, d = X.shape
    E = W1q.shape[0]
    if logits is None:
        L = router_logits(X, bf16_to_f64(Wr_bits)).astype(np.float32)
    else:
        L = np.asarray(logits, dtype=np.float32)
    idx, gates = route(L, k, score, renormalize, temperature, min_prob)
    counts, offsets, row_of, src_of = layout(idx, E)
    Xq, x_scale = fp8_quantize(X.astype(np.float32))
    Xe_q = np.zeros((src_of.size, d), dtype=np.uint8)
    ok = src_of >= 0
    Xe_q[ok] = Xq[src_of[ok] // k]
    R = src_of.size
    H = np.zeros((R, W1q.shape[1]))
    Ye = np.zeros((R, d))
    for e in range(E):
        a, b = int(offsets[e]), int(offsets[e + 1])
        if a == b:
            continue
        H[a:b] = fp8_gemm1(Xe_q[a:b], x_scale, W1q[e], w1_scale[e])
        Ye[a:b] = expert_gemm2(H[a:b], _as_f64(W2_bits[e]))
    Y = combine(Ye, row_of, gates, k)
    return dict(logits=L, topk_idx=idx, gates=gates, counts=counts, offsets=offsets,
                row_of=row_of, src_of=src_of, Xq=Xq, x_scale=x_scale, Xe_q=Xe_q, H=H, Ye=Ye, Y=Y)


def layer_forward_fp8_tokens(Xq, x_scale, W1q, w1_scale, W2_bits, topk_idx, gates, tokens):
    """The FP8 layer's Y for a subset of tokens, each computed on its own
    (the argument of layer_forward_tokens applies unchanged: a token's output
    depends on its own quantised row and its k experts only).

    Xq: the E4M3 codes of all of X (fp8_quantize over the whole tensor) or any
    array whose rows `tokens` index; W1q[e] / w1_scale[e]: expert e's codes and
    scale (only the routed experts are indexed).  Returns float64 [len(tokens), d].
    """
    tokens = np.asarray(tokens, dtype=np.int64)
    k = topk_idx.shape[1]
    xq = np.asarray(Xq)[tokens]
    idx = np.asarray(topk_idx)[tokens]
    g = np.asarray(gates, np.float64)[tokens]
    d = xq.shape[1]
    ye = np.zeros((len(tokens), k, d))
    by_e = {}
    for n in range(len(tokens)):
        for j in range(k):
            if idx[n, j] >= 0:
                by_e.setdefault(int(idx[n, j]), []).append((n, j))
    for e, pairs in sorted(by_e.items()):
        ns = np.array([p[0] for p in pairs])
        js = np.array([p[1] for p in pairs])
        h = fp8_gemm1(xq[ns], x_scale, W1q[e], w1_scale[e])
        ye[ns, js] = expert_gemm2(h, _as_f64(W2_bits[e]))
    Y = np.zeros((len(tokens), d))
    for j in range(k):
        Y += g[:, j:j + 1] * ye[:, j]
    return Y
