"""Seeded synthetic workloads for the sparse FFN decode path.

This module only draws numbers: weights, predictor factors, biases, per-token
inputs and profiled neuron frequencies, in the shapes and distributions of the
five workloads below.  It computes no step of the method (no norm, predictor,
activation, gather or reduction); both the CUDA library and the fp64 oracle
consume what it returns.

Workload recipe (all draws from ``torch.Generator`` seeded per tensor):

* ``U`` (F x r) and ``V`` (r x d) ~ N(0, 0.05^2); ``W_gate = U V + 0.01 N(0, 1)``
  so that the low-rank pair (U, V) is an imperfect predictor of the gate.
  Non-gated layers use this matrix as ``W_1``.
* ``W_up`` (F x d) and ``W_down`` (d x F) ~ N(0, 0.02^2).
* Profiled firing probability: ``p_i = min(0.99, A * rank_i^-1.1)`` (Zipf 1.1,
  the power-law locality of PowerInfer (unite.ai), introduction, and
  PowerInfer (aibars.net), "Hot and cold neuron mechanism"), ranks a seeded
  random permutation so hot neurons are scattered in the original order, and
  ``A`` bisected so ``mean(p)`` is the target active fraction.
* Bias: ``c_i = ||W_gate[i]||_2 * Phi^-1(1 - p_i) + delta``.  For an input
  with ``||x||^2 = d`` and random direction, ``W_gate[i] . x`` is close to
  N(0, ||W_gate[i]||^2), so neuron i fires with probability close to p_i.
  ``delta`` is 0 except for sparsity sweeps, which move every bias by one
  common shift found by bisection on the same Gaussian model.
* INT4 (group 32, symmetric): per group of 32 consecutive elements of a
  neuron vector (a W_gate / W_up row or a W_down column), ``s = fp16(max|w| / 7)``,
  ``q = clamp(round_half_even(w / s), -8, 7)``, stored as the nibble ``q + 8``,
  low nibble first.  This is how the synthetic INT4 model file is written;
  the hot path only ever reads it.
* Router (MoE) ~ N(0, 0.02^2), fp16.  Token inputs ``r_t ~ N(0, 1)``, seed 99 + t.
* 8-bit predictor (``pdtype = "i8row"``): each row of U and of V gets
  ``s = fp32(max|w| / 127)`` and ``q = clamp(round_half_even(w / s), -127, 127)``
  as a signed byte (an all-zero row gets s = 0, q = 0).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import numpy as np
import torch

BASE_SEED = 1234

_TORCH_DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


@dataclass(frozen=True)
class FFNConfig:
    name: str
    n_layers: int
    d: int
    F: int
    rank: int
    act: str            # "relu" (non-gated), "reglu", "drelu"
    wdtype: str         # "f32" | "f16" | "bf16" | "int4g32"
    pdtype: str         # predictor format
    mean_active: float  # target mean firing probability (1 - sparsity)
    n_tokens: int
    n_experts: int = 1
    top_k: int = 1
    prefill_tokens: int = 0
    zipf_s: float = 1.1
    uv_std: float = 0.05
    noise_std: float = 0.01
    wud_std: float = 0.02
    router_std: float = 0.02
    sweep: tuple = ()   # alternative active fractions reached by a bias shift

    @property
    def gated(self) -> bool:
        return self.act != "relu"


CONFIGS = {
    # single ReLU-gated (ReGLU) FFN layer, fp32, L2-resident
    "relu1": FFNConfig("reglu-1x256x1024-f32", 1, 256, 1024, 32, "reglu", "f32", "f32",
                       0.10, 64),
    # Llama-2-7B-shaped ReGLU stack, fp16, ~90 % sparse
    "llama7b": FFNConfig("llama2-7b-reglu-32x4096x11008-f16", 32, 4096, 11008, 1024, "reglu",
                         "f16", "f16", 0.10, 256),
    # TurboSparse-Mistral-7B-shaped dReLU stack, bf16, sparsity swept by bias shift
    "mistral7b": FFNConfig("turbosparse-mistral-7b-drelu-32x4096x14336-bf16", 32, 4096, 14336,
                           1024, "drelu", "bf16", "bf16", 0.10, 256,
                           sweep=(0.50, 0.20, 0.10, 0.05)),
    # Falcon-40B-shaped non-gated ReLU stack, fp16, ~20 % active
    "falcon40b": FFNConfig("falcon-40b-relu-60x8192x32768-f16", 60, 8192, 32768, 1024, "relu",
                           "f16", "f16", 0.20, 128),
    # TurboSparse-Mixtral-47B-shaped MoE: 8 experts top-2, dReLU, INT4 g32, fp16 predictor
    "mixtral47b": FFNConfig("turbosparse-mixtral-47b-moe8top2-drelu-32x4096x14336-int4g32", 32,
                            4096, 14336, 1024, "drelu", "int4g32", "f16", 0.10, 256,
                            n_experts=8, top_k=2, prefill_tokens=512),
    # the same two shapes with the cheaper 8-bit per-row predictor
    "llama7b-i8pred": FFNConfig("llama2-7b-reglu-32x4096x11008-f16-i8pred", 32, 4096, 11008, 1024,
                                "reglu", "f16", "i8row", 0.10, 256),
    "mixtral47b-i8pred": FFNConfig("turbosparse-mixtral-47b-moe8top2-drelu-32x4096x14336-int4g32-i8pred",
                                   32, 4096, 14336, 1024, "drelu", "int4g32", "i8row", 0.10, 256,
                                   n_experts=8, top_k=2, prefill_tokens=512),
}


def small(cfg: FFNConfig, **kw) -> FFNConfig:
    """A reduced copy of a workload (same structure and distributions)."""
    return replace(cfg, **kw)


def _seed(layer: int, expert: int, tensor: int, base: int = BASE_SEED) -> int:
    return (base * 1_000_003 + layer * 10_007 + expert * 101 + tensor) % (2**62)


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _normal(shape, std, device, seed):
    return torch.randn(shape, generator=_gen(device, seed), device=device,
                       dtype=torch.float32) * std


# ---------------------------------------------------------------------------
# Workload-shaping helpers (Zipf profile, bias from the Gaussian model)
# ---------------------------------------------------------------------------
def zipf_profile(F: int, mean_active: float, s: float, seed: int) -> np.ndarray:
    """p_i = min(0.99, A rank_i^-s) with mean(p) = mean_active (A by bisection)."""
    rng = np.random.default_rng(seed)
    ranks = rng.permutation(F).astype(np.float64) + 1.0
    base = ranks ** (-s)
    lo, hi = 0.0, float(F)
    for _ in range(200):
        A = 0.5 * (lo + hi)
        if np.minimum(0.99, A * base).mean() < mean_active:
            lo = A
        else:
            hi = A
    return np.minimum(0.99, 0.5 * (lo + hi) * base)


def _ndtri(p: np.ndarray) -> np.ndarray:
    return torch.special.ndtri(torch.from_numpy(np.asarray(p, np.float64))).numpy()


def _ndtr(v: np.ndarray) -> np.ndarray:
    return torch.special.ndtr(torch.from_numpy(np.asarray(v, np.float64))).numpy()


def bias_for(norms: np.ndarray, p: np.ndarray, target: float | None = None) -> np.ndarray:
    """c_i = ||w_i|| Phi^-1(1 - p_i) + delta, delta moving the mean firing
    probability (Gaussian model) to `target` when given."""
    c = norms * _ndtri(1.0 - p)
    if target is None:
        return c
    lo, hi = -50.0 * norms.max(), 50.0 * norms.max()
    for _ in range(200):
        delta = 0.5 * (lo + hi)
        m = (1.0 - _ndtr((c + delta) / norms)).mean()
        if m > target:
            lo = delta
        else:
            hi = delta
    return c + 0.5 * (lo + hi)


# ---------------------------------------------------------------------------
# INT4 group-32 model format (writer side)
# ---------------------------------------------------------------------------
def quantize_int4_g32(w: torch.Tensor):
    """Rows of w (n x k, k % 32 == 0) -> (nibbles uint8 n x k/2, scales fp16 n x k/32)."""
    n, k = w.shape
    g = w.float().reshape(n, k // 32, 32)
    s16 = (g.abs().amax(dim=2) / 7.0).to(torch.float16)
    s = s16.float().unsqueeze(2)
    q = torch.where(s > 0, torch.round(g / torch.where(s > 0, s, torch.ones_like(s))),
                    torch.zeros_like(g))
    q = q.clamp_(-8, 7).to(torch.int32) + 8
    q = q.reshape(n, k)
    packed = (q[:, 0::2] | (q[:, 1::2] << 4)).to(torch.uint8)
    return packed.contiguous(), s16.contiguous()


def quantize_i8_rows(w: torch.Tensor):
    """Rows of w (n x k) -> (signed bytes int8 n x k, fp32 scales n)."""
    w = w.float()
    s = (w.abs().amax(dim=1) / 127.0).float()
    q = torch.where(s[:, None] > 0, torch.round(w / torch.where(s > 0, s, torch.ones_like(s))[:, None]),
                    torch.zeros_like(w))
    return q.clamp_(-127, 127).to(torch.int8).contiguous(), s.contiguous()


# ---------------------------------------------------------------------------
# Layers
# ---------------------------------------------------------------------------
@dataclass
class ExpertWeights:
    """One FFN / expert in stored format, original neuron order, on `device`.

    w_gate: F x d (W_1 when non-gated); w_up: F x d or None; w_down: d x F for
    float formats, neuron-major F x d (d/2 bytes per neuron) for INT4; s_*:
    INT4 scales (F x d/32 fp16); c: F fp32; U: F x r; V: r x d; freq: F
    profiled firing probabilities (float64 numpy)."""
    w_gate: torch.Tensor
    w_up: torch.Tensor | None
    w_down: torch.Tensor
    c: torch.Tensor
    U: torch.Tensor
    V: torch.Tensor
    freq: np.ndarray
    s_gate: torch.Tensor | None = None
    s_up: torch.Tensor | None = None
    s_down: torch.Tensor | None = None
    sU: torch.Tensor | None = None      # 8-bit predictor: fp32 scale per row of U
    sV: torch.Tensor | None = None      # and of V


@dataclass
class LayerWeights:
    experts: list
    router: torch.Tensor | None = None     # E x d fp16 (MoE)
    meta: dict = field(default_factory=dict)


def make_expert(cfg: FFNConfig, layer: int, expert: int, device="cpu",
                active: float | None = None) -> ExpertWeights:
    """Weights of one FFN (one expert).  `active` selects a sweep point: the
    biases are shifted so the mean firing probability moves to it."""
    d, F, r = cfg.d, cfg.F, cfg.rank
    U = _normal((F, r), cfg.uv_std, device, _seed(layer, expert, 1))
    V = _normal((r, d), cfg.uv_std, device, _seed(layer, expert, 2))
    wg = U @ V
    wg += _normal((F, d), cfg.noise_std, device, _seed(layer, expert, 3))
    wu = _normal((F, d), cfg.wud_std, device, _seed(layer, expert, 4)) if cfg.gated else None
    wd = _normal((d, F), cfg.wud_std, device, _seed(layer, expert, 5))
    p = zipf_profile(F, cfg.mean_active, cfg.zipf_s, _seed(layer, expert, 6))
    norms = torch.linalg.vector_norm(wg.double(), dim=1).cpu().numpy()
    shift_to = None if active is None or active == cfg.mean_active else active
    c = torch.from_numpy(bias_for(norms, p, shift_to).astype(np.float32)).to(device)
    # profiled frequency = firing probability under the (possibly shifted) bias
    freq = p if shift_to is None else 1.0 - _ndtr(c.cpu().double().numpy() / norms)
    if cfg.pdtype == "i8row":
        Up, sU = quantize_i8_rows(U)
        Vp, sV = quantize_i8_rows(V)
    else:
        pdt = _TORCH_DT[cfg.pdtype]
        Up, Vp, sU, sV = U.to(pdt).contiguous(), V.to(pdt).contiguous(), None, None
    if cfg.wdtype == "int4g32":
        qg, sg = quantize_int4_g32(wg)
        qu, su = quantize_int4_g32(wu) if wu is not None else (None, None)
        qd, sd = quantize_int4_g32(wd.t().contiguous())
        return ExpertWeights(qg, qu, qd, c, Up, Vp, freq, sg, su, sd, sU, sV)
    wdt = _TORCH_DT[cfg.wdtype]
    return ExpertWeights(wg.to(wdt).contiguous(),
                         None if wu is None else wu.to(wdt).contiguous(),
                         wd.to(wdt).contiguous(), c, Up, Vp, freq, sU=sU, sV=sV)


def make_layer(cfg: FFNConfig, layer: int, device="cpu", active: float | None = None) -> LayerWeights:
    experts = [make_expert(cfg, layer, e, device, active) for e in range(cfg.n_experts)]
    router = None
    if cfg.n_experts > 1:
        router = _normal((cfg.n_experts, cfg.d), cfg.router_std, device,
                         _seed(layer, 0, 7)).to(torch.float16).contiguous()
    return LayerWeights(experts, router, {"layer": layer, "active": active or cfg.mean_active})


def token_input(cfg: FFNConfig, t: int, device="cpu") -> torch.Tensor:
    """Residual-stream input of decode token t: r ~ N(0, 1) (d,), fp32."""
    return torch.randn((cfg.d,), generator=_gen(device, 99 + t), device=device,
                       dtype=torch.float32)


def token_inputs(cfg: FFNConfig, n: int, device="cpu", first: int = 0) -> torch.Tensor:
    return torch.stack([token_input(cfg, first + t, device) for t in range(n)])


def prefill_input(cfg: FFNConfig, T: int, device="cpu", seed: int = 4242) -> torch.Tensor:
    """Residual stream of a T-token prompt: T x d ~ N(0, 1), fp32."""
    return torch.randn((T, cfg.d), generator=_gen(device, seed), device=device,
                       dtype=torch.float32)


def to_numpy(t: torch.Tensor | None) -> np.ndarray | None:
    """Stored bytes of a tensor as numpy (bf16 as uint16 bit patterns)."""
    if t is None:
        return None
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()
