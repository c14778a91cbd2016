"""Seeded synthetic inputs for the MoE layer (shared by tests, bench and smoke).

This module draws random inputs and nothing else: it holds none of the
layer's arithmetic (no routing, layout, FFN or combine), so both the CUDA
path and the CPU oracle can consume its bytes without sharing method code.

Workloads mirror the shapes the source pages discuss (a Mixtral-class layer
with hidden size 4096 and 8 experts, top-1/top-2 routing; a DeepSeek-class
layer with 256 experts) -- the ThunderEP PCIe blog §1.2 for d=4096, the
DySHARP review §1 and the TensorRT-LLM large-EP article for 256 experts per
layer, the GPT-4 "2%" article §2.3 and the xDeepServe blog §5.3 for router
temperature and a minimum-probability threshold.
Nothing here is a dataset: every tensor is drawn from a seeded generator.

Draws
-----
* tokens ``X`` ~ N(0, 1), router logits ~ N(0, 1), router weights and expert
  weights ~ N(0, 0.02); all drawn in fp32 and rounded to bf16
  round-to-nearest-even (logits stay fp32).
* small tensors (tokens, logits, router weights) come from numpy's PCG64 on
  the host, so they are byte-identical on every machine;
* expert weights ``W1 [E, f, d]``, ``W2 [E, d, f]`` come from numpy on the
  host when ``device == 'cpu'`` and from torch's Philox generator on the
  device when ``device`` is a CUDA device (15 GB of host sampling would
  dominate a run).  Either way the same bytes then feed both sides.
* the skewed top-1 workload adds a per-expert bias ``scale * log(w_r)``
  with Zipf(s=1.2) rank weights ``w_r = r^-1.2 / sum_r' r'^-1.2``, expert e
  having rank e+1.  ``bias_scale`` defaults to 0.62, which gives the top
  expert ~40% of tokens; 2.0 (the literal factor, ~86%) is a stress variant.
"""
from __future__ import annotations

import hashlib
from dataclasses import dataclass, field, replace

import numpy as np
import torch

__all__ = ["LayerConfig", "WORKLOADS", "workload", "make_layer_inputs",
           "f32_to_bf16_bits", "bf16_bits_to_tensor", "subseed"]


@dataclass(frozen=True)
class LayerConfig:
    """Shape and routing recipe of one MoE layer workload."""
    name: str
    T: int            # tokens
    d: int            # model dim
    E: int            # experts
    k: int            # experts per token
    f: int            # FFN hidden dim
    router: str       # 'logits' (fp32 logits supplied) | 'weights' (bf16 router linear d->E)
    score: str        # 'softmax' | 'sigmoid'
    renormalize: int  # 1: gates renormalised over the chosen k
    bias_scale: float = 0.0   # > 0: Zipf(s=1.2) per-expert logit bias (skewed routing)
    zipf_s: float = 1.2
    x_std: float = 1.0
    w_std: float = 0.02
    logit_std: float = 1.0
    temperature: float = 1.0  # router temperature
    min_prob: float = 0.0     # > 0: drop chosen slots whose probability is not above it
    extra: dict = field(default_factory=dict)

    @property
    def R(self) -> int:
        return self.T * self.k


def _mk(name, T, d, E, k, f, router, score, renormalize, **kw):
    return LayerConfig(name=name, T=T, d=d, E=E, k=k, f=f, router=router,
                       score=score, renormalize=renormalize, **kw)


WORKLOADS: dict[str, LayerConfig] = {
    # Tiny layer the oracle finishes in well under a second.
    "tiny": _mk("tiny", 256, 128, 8, 2, 256, "logits", "softmax", 1),
    # Mixtral-shaped layer: bf16 router linear, softmax top-2 renormalised.
    "mixtral": _mk("mixtral", 4096, 4096, 8, 2, 14336, "weights", "softmax", 1),
    # Skewed top-1 routing (load-imbalance stress).
    "skewed_top1": _mk("skewed_top1", 4096, 4096, 8, 1, 14336, "logits", "softmax", 1,
                       bias_scale=0.62),
    "skewed_top1_harsh": _mk("skewed_top1_harsh", 4096, 4096, 8, 1, 14336, "logits",
                             "softmax", 1, bias_scale=2.0),
    # Fine-grained many-expert layer: 256 experts, sigmoid top-8 renormalised.
    "fine_grained": _mk("fine_grained", 8192, 7168, 256, 8, 2048, "logits", "sigmoid", 1),
}
# Routing variants on the Mixtral shape: temperature 1.3 and a 0.05 minimum
# probability (the values the pages discuss) -- some second choices are dropped.
WORKLOADS["mixtral_threshold"] = _mk("mixtral_threshold", 4096, 4096, 8, 2, 14336, "weights",
                                     "softmax", 1, temperature=1.3, min_prob=0.05)
WORKLOADS["tiny_threshold"] = _mk("tiny_threshold", 256, 128, 8, 2, 256, "logits", "softmax", 1,
                                  temperature=0.5, min_prob=0.2)
# The fine-grained layer's per-expert shape (d=7168, f=2048, top-8, ~256 rows
# per expert, sigmoid) over 32 experts: a case of a few GB for profiling the
# expert GEMMs (inputs still larger than L2: 1.9 GB of weights per step).
WORKLOADS["fine_grained_e32"] = _mk("fine_grained_e32", 1024, 7168, 32, 8, 2048, "logits",
                                    "sigmoid", 1)
for _T in (16, 64, 256, 1024):
    WORKLOADS[f"decode_{_T}"] = _mk(f"decode_{_T}", _T, 4096, 8, 2, 14336, "weights",
                                    "softmax", 1)


def workload(name: str, **overrides) -> LayerConfig:
    cfg = WORKLOADS[name]
    return replace(cfg, **overrides) if overrides else cfg


def subseed(seed: int, tag: str) -> int:
    """Stable 63-bit sub-seed per (seed, tensor name)."""
    h = hashlib.sha256(f"{seed}:{tag}".encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round finite fp32 values to bf16 (round-to-nearest-even); returns uint16 bits."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_tensor(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)


def _host_normal(seed: int, tag: str, shape, std: float) -> np.ndarray:
    rng = np.random.default_rng(subseed(seed, tag))
    out = rng.standard_normal(shape, dtype=np.float32)
    if std != 1.0:
        out *= np.float32(std)
    return out


def _host_bf16(seed, tag, shape, std) -> torch.Tensor:
    return bf16_bits_to_tensor(f32_to_bf16_bits(_host_normal(seed, tag, shape, std)))


def _expert_weights(seed, tag, shape, std, device) -> torch.Tensor:
    """[E, rows, cols] bf16 expert weights, generated where they will live."""
    dev = torch.device(device)
    if dev.type == "cpu":
        E = shape[0]
        out = torch.empty(shape, dtype=torch.bfloat16)
        for e in range(E):  # per expert keeps the fp32 temporary small
            out[e] = _host_bf16(seed, f"{tag}[{e}]", shape[1:], std)
        return out
    g = torch.Generator(device=dev)
    g.manual_seed(subseed(seed, tag))
    out = torch.empty(shape, dtype=torch.bfloat16, device=dev)
    per = max(1, (1 << 30) // (shape[1] * shape[2]))  # <= 4 GiB fp32 temporary
    for e0 in range(0, shape[0], per):
        e1 = min(shape[0], e0 + per)
        tmp = torch.randn((e1 - e0,) + tuple(shape[1:]), generator=g, device=dev,
                          dtype=torch.float32)
        tmp.mul_(std)
        out[e0:e1].copy_(tmp)  # fp32 -> bf16 conversion rounds to nearest even
        del tmp
    return out


def zipf_bias(cfg: LayerConfig) -> np.ndarray:
    r = np.arange(1, cfg.E + 1, dtype=np.float64)
    w = r ** (-cfg.zipf_s)
    w /= w.sum()
    return (cfg.bias_scale * np.log(w)).astype(np.float32)


def make_layer_inputs(cfg: LayerConfig, seed: int = 0, device="cpu",
                      with_weights: bool = True) -> dict:
    """Draw one layer's inputs.

    Returns a dict with host tensors ``X`` (bf16 [T,d]) and, by router kind,
    ``logits`` (fp32 [T,E]) or ``Wr`` (bf16 [E,d]); plus ``W1`` (bf16
    [E,f,d]) and ``W2`` (bf16 [E,d,f]) on ``device`` when ``with_weights``.
    """
    out = {"cfg": cfg, "seed": seed}
    out["X"] = _host_bf16(seed, "X", (cfg.T, cfg.d), cfg.x_std)
    if cfg.router == "weights":
        out["Wr"] = _host_bf16(seed, "Wr", (cfg.E, cfg.d), cfg.w_std)
        out["logits"] = None
    else:
        L = _host_normal(seed, "logits", (cfg.T, cfg.E), cfg.logit_std)
        if cfg.bias_scale > 0:
            L = L + zipf_bias(cfg)[None, :]
        out["logits"] = torch.from_numpy(np.ascontiguousarray(L, dtype=np.float32))
        out["Wr"] = None
    if with_weights:
        out["W1"] = _expert_weights(seed, "W1", (cfg.E, cfg.f, cfg.d), cfg.w_std, device)
        out["W2"] = _expert_weights(seed, "W2", (cfg.E, cfg.d, cfg.f), cfg.w_std, device)
    return out


def random_bf16(shape, seed: int, tag: str, std: float = 1.0) -> torch.Tensor:
    """A host bf16 tensor ~N(0, std^2) (used for stage-level parity inputs)."""
    return _host_bf16(seed, tag, tuple(shape), std)


def random_f32(shape, seed: int, tag: str, std: float = 1.0) -> torch.Tensor:
    return torch.from_numpy(_host_normal(seed, tag, tuple(shape), std))


def random_topk(T: int, E: int, k: int, seed: int, tag: str = "topk",
                skew: float = 0.0) -> torch.Tensor:
    """[T,k] int32 distinct expert ids per token (a valid routing, drawn directly)."""
    rng = np.random.default_rng(subseed(seed, tag))
    if skew > 0:
        p = np.arange(1, E + 1, dtype=np.float64) ** (-skew)
        p /= p.sum()
    else:
        p = None
    out = np.empty((T, k), dtype=np.int32)
    for t in range(T):
        out[t] = rng.choice(E, size=k, replace=False, p=p)
    return torch.from_numpy(out)
