"""Seeded synthetic inputs for the DoRA hot path.

This module only draws random tensors with the shapes and distributions of the
workloads below; it contains none of the DoRA arithmetic (no norm, no scale,
no compose).  Both the CUDA path and the fp64 oracle are fed from here, and it
imports neither of them.

Reading of the distribution notation: the second argument of N(0, x) is the
standard deviation (as in ``torch.Tensor.normal_(mean, std)``), and
"kaiming-uniform" is ``kaiming_uniform_(a=sqrt(5))`` on [r, d_in], i.e.
U(-1/sqrt(d_in), 1/sqrt(d_in)), which is also what the ``DoRALinear`` listing
of the "DoRA" (aiwiki) page uses for A.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional, Sequence

import torch

# Tensor ids: each tensor gets its own generator stream, so drawing a subset
# (or a different token count) never shifts another tensor's values.
_W0, _A, _B, _M, _X, _BASE, _LORA, _DY, _EPS_M = range(9)


@dataclasses.dataclass(frozen=True)
class ModuleShape:
    name: str
    d_out: int
    d_in: int
    r: int
    alpha: float

    @property
    def s(self) -> float:
        return float(self.alpha) / float(self.r)


@dataclasses.dataclass(frozen=True)
class Workload:
    """One workload: a module shape (or a stack of them) plus token count."""
    key: str
    dtype: str                    # "f32" or "bf16": storage / arithmetic type of the inputs
    modules: Sequence[ModuleShape]
    tokens: int                   # 0 = norm only
    backward: bool
    seed: int
    description: str


def _layer_stack() -> List[ModuleShape]:
    mods = []
    per_layer = [("q", 4096, 4096), ("k", 1024, 4096), ("v", 1024, 4096),
                 ("o", 4096, 4096), ("gate", 14336, 4096), ("up", 14336, 4096),
                 ("down", 4096, 14336)]
    for layer in range(8):
        for nm, d_out, d_in in per_layer:
            mods.append(ModuleShape(f"L{layer}.{nm}", d_out, d_in, 384, 768.0))
    return mods


WORKLOADS: Dict[str, Workload] = {
    "tiny_fp32": Workload(
        "tiny_fp32", "f32", (ModuleShape("tiny", 64, 48, 8, 16.0),), 32, True, 1001,
        "tiny fp32 module d_out=64 d_in=48 r=8 alpha=16 (s=2), 32 tokens; norm + compose fwd + bwd"),
    "norm_4096_r64": Workload(
        "norm_4096_r64", "bf16", (ModuleShape("m4096", 4096, 4096, 64, 128.0),), 0, False, 1002,
        "single bf16 module d_out=d_in=4096 r=64 alpha=128, norm only"),
    "headline_8192_r384": Workload(
        "headline_8192_r384", "bf16", (ModuleShape("m8192", 8192, 8192, 384, 768.0),), 4096, True, 1003,
        "bf16 module d_out=d_in=8192 r=384 alpha=768; norm + compose on [4096, 8192] activations"),
    "mlp_up_25600x5120_r384": Workload(
        "mlp_up_25600x5120_r384", "bf16", (ModuleShape("up", 25600, 5120, 384, 768.0),), 8192, True, 1004,
        "bf16 MLP up-projection d_in=5120 d_out=25600 r=384 alpha=768; norm + compose fwd/bwd on [8192, 25600]"),
    "layer_stack_56": Workload(
        "layer_stack_56", "bf16", tuple(_layer_stack()), 0, False, 1005,
        "8 layers x 7 modules (q/o 4096x4096, k/v 1024x4096, gate/up 14336x4096, down 4096x14336), r=384 alpha=768; grouped norm"),
}

# Token counts of the compose sweep that goes with the layer stack.
STACK_SWEEP_TOKENS = (512, 2048, 8192, 32768)


def _gen(seed: int, tensor_id: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed * 64 + tensor_id)
    return g


def _tdtype(dtype: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[dtype]


def module_weights(w: Workload, index: int = 0, device="cpu"):
    """W0 [d_out, d_in], A [r, d_in], B [d_out, r] in the workload's dtype.

    tiny_fp32: W0 ~ N(0, 1/d_in), A ~ U(+-1/sqrt(d_in)), B ~ N(0, 0.01).
    Others:    W0 ~ N(0, 0.02),   A ~ U(+-1/sqrt(d_in)), B ~ N(0, 0.02).
    Values are drawn in fp32 and rounded (RNE) to bf16 where the dtype says so.
    """
    ms = w.modules[index]
    seed = w.seed * 131 + index
    if w.key == "tiny_fp32":
        w0_std, b_std = 1.0 / ms.d_in, 0.01
    else:
        w0_std, b_std = 0.02, 0.02
    dt = _tdtype(w.dtype)
    W0 = torch.empty(ms.d_out, ms.d_in, device=device).normal_(0.0, w0_std, generator=_gen(seed, _W0, device))
    bound = 1.0 / math.sqrt(ms.d_in)
    A = torch.empty(ms.r, ms.d_in, device=device).uniform_(-bound, bound, generator=_gen(seed, _A, device))
    B = torch.empty(ms.d_out, ms.r, device=device).normal_(0.0, b_std, generator=_gen(seed, _B, device))
    return W0.to(dt), A.to(dt), B.to(dt)


def magnitude_from_base_rows(w: Workload, W0: torch.Tensor, index: int = 0) -> torch.Tensor:
    """m_i = ||W0_i|| * (1 + noise), fp32, the magnitude-initialisation recipe
    m0 = ||w0|| of the pages perturbed as the workload states: U(-0.01, 0.01)
    for tiny_fp32, N(0, 0.005) otherwise."""
    seed = w.seed * 131 + index
    dev = W0.device
    rown = torch.linalg.vector_norm(W0.double(), dim=1)
    if w.key == "tiny_fp32":
        noise = torch.empty(W0.shape[0], device=dev).uniform_(-0.01, 0.01, generator=_gen(seed, _M, dev))
    else:
        noise = torch.empty(W0.shape[0], device=dev).normal_(0.0, 0.005, generator=_gen(seed, _M, dev))
    return (rown * (1.0 + noise.double())).float()


def magnitude_near_unity(w: Workload, n_ref: torch.Tensor, index: int = 0) -> torch.Tensor:
    """m_i = n_ref_i * (1 + e_i), e_i ~ N(0, 0.005) redrawn until |e_i| < 0.0099,
    so that |g - 1| < 1e-2 as the headline workload asks.  ``n_ref`` is a row
    norm supplied by the caller."""
    seed = w.seed * 131 + index
    dev = n_ref.device
    g = _gen(seed, _EPS_M, dev)
    e = torch.empty(n_ref.shape[0], device=dev).normal_(0.0, 0.005, generator=g)
    for _ in range(64):
        bad = e.abs() >= 0.0099
        if not bool(bad.any()):
            break
        redraw = torch.empty(n_ref.shape[0], device=dev).normal_(0.0, 0.005, generator=g)
        e = torch.where(bad, redraw, e)
    e = e.clamp(-0.0098, 0.0098)
    return (n_ref.double() * (1.0 + e.double())).float()


def activations(w: Workload, tokens: int, d_out: int, device="cpu", index: int = 0,
                which: Sequence[str] = ("base", "lora", "dy")):
    """base, lora, dy ~ N(0, 1) of shape [tokens, d_out] in the workload's dtype."""
    seed = w.seed * 131 + index + 7 * tokens
    dt = _tdtype(w.dtype)
    ids = {"base": _BASE, "lora": _LORA, "dy": _DY}
    out = []
    for nm in which:
        t = torch.empty(tokens, d_out, device=device).normal_(0.0, 1.0, generator=_gen(seed, ids[nm], device))
        out.append(t.to(dt))
    return tuple(out)


def tiny_activations(w: Workload, W0: torch.Tensor, A: torch.Tensor, B: torch.Tensor):
    """For tiny_fp32: x ~ N(0, 1) [tokens, d_in]; base = x W0^T and
    lora = (x A^T) B^T are the given activations (the frozen layer's output and
    the low-rank branch), evaluated in fp64 and rounded to fp32; dy ~ N(0, 1)."""
    seed = w.seed * 131
    T = w.tokens
    x = torch.empty(T, W0.shape[1]).normal_(0.0, 1.0, generator=_gen(seed, _X, "cpu")).double()
    base = (x @ W0.double().T).float()
    lora = ((x @ A.double().T) @ B.double().T).float()
    dy = torch.empty(T, W0.shape[0]).normal_(0.0, 1.0, generator=_gen(seed, _DY, "cpu"))
    return x.float(), base, lora, dy


def eps_for(dtype: str) -> float:
    """Default norm clamp: machine epsilon of the weight dtype (fp32 2^-23,
    bf16 2^-7).  The pages say only that eps is dtype-specific."""
    return {"f32": 2.0 ** -23, "bf16": 2.0 ** -7}[dtype]
