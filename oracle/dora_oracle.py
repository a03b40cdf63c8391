"""Plain fp64 CPU oracle for the DoRA linear-layer hot path.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute this module: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It
shares no code with the CUDA library (no kernels, headers, helpers or
constants) and imports nothing from the product package.

Everything is computed in float64 with numpy.  Inputs are upcast to float64
first (so bf16- or fp32-rounded inputs are taken at their exact values).
Matrix products use ``numpy.matmul`` as the one library primitive; there is no
blocking, fusion or reordering beyond the definitions cited below.

Sources (page title, then the section / listing used):

* [DoRA-aiwiki]  "DoRA" (aiwiki), the ``DoRALinear`` listing: the weight is
  ``W0 + scale * (B @ A)``, normalised by its per-output-row Euclidean norm
  (``norm(dim=1)``) which is detached, then multiplied by the magnitude.
* [LoRA&DoRA]  "LoRA & DoRA: The Math, Memory, and Trade-offs", section 1
  (W = W0 + sBA, s = alpha/r, y = W0 x + s B(Ax), parameter counts
  N_LoRA = r(d+k)) and section 2 (V' = W0 + sBA, w'_j = m_j v'_j/||v'_j||,
  m0 = ||w0||, B0 = 0 so the initial weight equals W0, N_DoRA = r(d+k)+k,
  the arrow and rotation examples), section 6 (merged weight).
* [ScalingDoRA]  "Scaling DoRA: High-Rank Adaptation via Factored Norms and
  Fused Kernels" (paperlayer summary of arXiv:2603.22276v1):
  section 2 "Factored Norm Computation" (squared row norm = base + cross +
  Gram terms, O(d_out r + r^2) intermediates); section 4 "Runtime Dispatch",
  precision bullet (g = m / max(wnorm, eps)); "Data Availability" (the
  composition contract dY = g*(s x A^T B^T) + (g-1)*Y_base, norm detached);
  section 3 "Fused Triton Kernels", numerical-stability and backward bullets
  (explicit (g-1) correction in fp32; dlora, dbase and a separate dmag
  reduction); appendix B (norm assembly clamps the sum at zero before the
  square root).

Conventions (the pages disagree on the norm axis; this oracle follows the
``DoRALinear`` listing and the "row-wise" wording of ScalingDoRA):
W0 is [d_out, d_in] (nn.Linear layout), A is [r, d_in], B is [d_out, r],
m, n, g are [d_out]; activations base, lora, dy, y are [T, d_out] with the
magnitude broadcast along the last axis.

Parity pins: every public function here is pinned by ``tests/test_oracle.py``
against values or identities that do not come from this module (worked
examples printed on the pages, closed forms, textbook routines, finite
differences).  No function is "parity unpinned".
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "lora_scale",
    "lora_param_count",
    "dora_param_count",
    "dense_row_norm",
    "factored_row_norm",
    "factored_row_norm_sq",
    "factored_intermediate_elems",
    "magnitude_scale",
    "compose_fwd",
    "compose_delta",
    "compose_bwd",
    "compose_inner",
    "compose_bwd_from_inner",
    "compose_bwd_frozen",
    "dora_linear_forward",
    "merged_weight",
    "merge_weight_given_norm",
    "rows_dense_row_norm",
]


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


# --------------------------------------------------------------------------
# LoRA bookkeeping  [LoRA&DoRA, section 1 and section 2]
# --------------------------------------------------------------------------

def lora_scale(alpha: float, r: int) -> float:
    """The adapter scaling factor s = alpha / r  [LoRA&DoRA, section 1]."""
    return float(alpha) / float(r)


def lora_param_count(d: int, k: int, r: int) -> int:
    """Trainable entries of a rank-r adapter on a d x k layer: r*(d + k).

    A is r x k and B is d x r  [LoRA&DoRA, section 1, N_LoRA]."""
    return r * (d + k)


def dora_param_count(d: int, k: int, r: int) -> int:
    """LoRA entries plus one magnitude per normalised vector.

    The page counts one magnitude per column of a d x k matrix, giving
    r(d + k) + k  [LoRA&DoRA, section 2, N_DoRA].  (This library normalises
    per output row of [d_out, d_in], so its magnitude has d_out entries; the
    page's count is kept as printed.)"""
    return r * (d + k) + k


def factored_intermediate_elems(d_out: int, r: int) -> int:
    """Elements of the rank-dependent intermediates of the factored norm.

    The cross term needs W0 A^T ([d_out, r]) and the Gram term needs
    G = A A^T ([r, r]): O(d_out r + r^2)  [ScalingDoRA, section 2,
    "Algebraic decomposition"]."""
    return d_out * r + r * r


# --------------------------------------------------------------------------
# The norm  [DoRA-aiwiki DoRALinear; LoRA&DoRA section 2; ScalingDoRA section 2]
# --------------------------------------------------------------------------

def dense_row_norm(W0, A, B, s: float) -> np.ndarray:
    """n_i = || (W0 + s B A)_i ||_2, materialising the dense [d_out, d_in] V.

    This is the definition the factored norm must reproduce: V' = W0 + sBA and
    the Euclidean norm of each output row  [DoRA-aiwiki, DoRALinear listing;
    LoRA&DoRA, section 2]."""
    W0, A, B = _f64(W0), _f64(A), _f64(B)
    V = W0 + s * (B @ A)
    return np.sqrt(np.sum(V * V, axis=1))


def rows_dense_row_norm(W0_rows, A, B_rows, s: float) -> np.ndarray:
    """``dense_row_norm`` restricted to a subset of rows (the rows of W0 and
    B that are passed).  Used to check sampled rows of very large layers."""
    return dense_row_norm(W0_rows, A, B_rows, s)


def factored_row_norm(W0, A, B, s: float) -> np.ndarray:
    """The factored form of the same norm, in fp64.

    ||W0_i + s B_i A||^2 = ||W0_i||^2 + 2 s B_i . (W0 A^T)_i + s^2 B_i G B_i^T
    with G = A A^T: a base, a cross and a Gram term built from [d_out, r] and
    [r, r] intermediates, never from the dense product BA  [ScalingDoRA,
    section 2].  The sum is clamped at zero before the square root, as the
    pages' norm assembly does  [ScalingDoRA, appendix B].
    """
    W0, A, B = _f64(W0), _f64(A), _f64(B)
    G = A @ A.T                       # [r, r]
    U = W0 @ A.T                      # [d_out, r]
    base = np.sum(W0 * W0, axis=1)
    cross = np.sum(B * U, axis=1)
    gram = np.sum((B @ G) * B, axis=1)
    sq = base + 2.0 * s * cross + (s * s) * gram
    return np.sqrt(np.maximum(sq, 0.0))


def factored_row_norm_sq(W0, A, B, s: float) -> np.ndarray:
    """The squared row norm in factored form, before the clamp and the square
    root: ||W0_i||^2 + 2 s B_i.(W0 A^T)_i + s^2 B_i (A A^T) B_i^T
    [ScalingDoRA, section 2].  Every term is a sum over the columns of W0 (and
    of A), so for a column split of W0 and A the values of the parts add up to
    the whole: the per-shard partial of a d_in-sharded norm [ScalingDoRA,
    section 6, chunk-wise partial sums followed by an all-reduce]."""
    W0, A, B = _f64(W0), _f64(A), _f64(B)
    base = np.sum(W0 * W0, axis=1)
    cross = np.sum(B * (W0 @ A.T), axis=1)
    gram = np.sum((B @ (A @ A.T)) * B, axis=1)
    return base + 2.0 * s * cross + (s * s) * gram


# --------------------------------------------------------------------------
# Magnitude scale  [ScalingDoRA, section 4 precision bullet]
# --------------------------------------------------------------------------

def magnitude_scale(m, n, eps: float):
    """Returns (g, g_minus_1, n_clamped).

    n_c = max(n, eps), g = m / n_c  [ScalingDoRA, section 4: "g = m/max(wnorm,
    eps)"].  The near-unity correction g - 1 is formed as (m - n_c)/n_c so it
    does not cancel when g is close to one  [ScalingDoRA, section 3,
    numerical stability]."""
    m, n = _f64(m), _f64(n)
    nc = np.maximum(n, eps)
    g = m / nc
    gm1 = (m - nc) / nc
    return g, gm1, nc


# --------------------------------------------------------------------------
# Compose forward and backward  [ScalingDoRA, Data Availability and section 3]
# --------------------------------------------------------------------------

def compose_fwd(base, lora, m, n, s: float, eps: float) -> np.ndarray:
    """y = base + dY with dY = (g - 1) * base + g * s * lora.

    ``base`` = x W0^T and ``lora`` = (x A^T) B^T are given activations
    [T, d_out]; g broadcasts along the last axis.  The composition contract is
    dY = g (s x A^T B^T) + (g - 1) Y_base, added to Y_base by the caller
    [ScalingDoRA, Data Availability]."""
    base, lora = _f64(base), _f64(lora)
    g, gm1, _ = magnitude_scale(m, n, eps)
    return base + (gm1 * base + g * s * lora)


def compose_delta(base, lora, m, n, s: float, eps: float) -> np.ndarray:
    """dY = g * s * lora + (g - 1) * base, the module output of the composition
    contract, which the caller adds to its Y_base  [ScalingDoRA, Data
    Availability]; g - 1 formed as in ``magnitude_scale``."""
    base, lora = _f64(base), _f64(lora)
    g, gm1, _ = magnitude_scale(m, n, eps)
    return g * s * lora + gm1 * base


def compose_bwd(dy, base, lora, m, n, s: float, eps: float):
    """Gradients of y = g (base + s lora) with n detached.

    d_base = g dy, d_lora = g s dy, and dm_j = sum_t dy_tj (base_tj +
    s lora_tj) / n_c,j.  The norm carries no gradient (it is detached in the
    ``DoRALinear`` listing and in ScalingDoRA's Data Availability bullet);
    d_lora and d_base come from one pass and dm from a column reduction over
    tokens  [ScalingDoRA, section 3, backward kernel]."""
    dy, base, lora = _f64(dy), _f64(base), _f64(lora)
    g, _, nc = magnitude_scale(m, n, eps)
    d_base = g * dy
    d_lora = (g * s) * dy
    dm = np.sum(dy * (base + s * lora), axis=0) / nc
    return d_base, d_lora, dm


# --------------------------------------------------------------------------
# Training-forward second output and the backward variants  [ScalingDoRA,
# section 4 "Tier 1: Fused Backward" and section 6]
# --------------------------------------------------------------------------

def compose_inner(base, lora, s: float) -> np.ndarray:
    """inner = base + s lora, the second output of the dual-output training
    forward: y = g * inner, so the backward's dm needs inner and dy only
    [ScalingDoRA, section 4, tier 1: output and inner computed together]."""
    return _f64(base) + s * _f64(lora)


def compose_bwd_from_inner(dy, inner, m, n, s: float, eps: float):
    """Gradients of y = g * inner (n detached) from dy and inner alone:
    d_base = g dy, d_lora = g s dy, dm_j = sum_t dy_tj inner_tj / n_c,j
    [ScalingDoRA, section 4, tier 1; section 3, backward kernel]."""
    dy, inner = _f64(dy), _f64(inner)
    g, _, nc = magnitude_scale(m, n, eps)
    return g * dy, (g * s) * dy, np.sum(dy * inner, axis=0) / nc


def compose_bwd_frozen(dy, m, n, s: float, eps: float):
    """d_base = g dy and d_lora = g s dy with the magnitude frozen: no dm and
    no inner [ScalingDoRA, section 4, tier 1 and section 6: with frozen
    magnitude the inner tensor is skipped]."""
    dy = _f64(dy)
    g, _, _ = magnitude_scale(m, n, eps)
    return g * dy, (g * s) * dy


# --------------------------------------------------------------------------
# Whole-layer definitions used as pins of the compose
# --------------------------------------------------------------------------

def merged_weight(W0, A, B, m, s: float) -> np.ndarray:
    """W' = m * (W0 + sBA) / ||W0 + sBA|| per output row  [LoRA&DoRA,
    section 6; DoRA-aiwiki, DoRALinear listing]."""
    W0, A, B, m = _f64(W0), _f64(A), _f64(B), _f64(m)
    V = W0 + s * (B @ A)
    n = np.sqrt(np.sum(V * V, axis=1))
    return (m / n)[:, None] * V


def dora_linear_forward(x, W0, A, B, m, s: float) -> np.ndarray:
    """y = x W'^T with the merged DoRA weight: the ``DoRALinear`` forward
    [DoRA-aiwiki]."""
    return _f64(x) @ merged_weight(W0, A, B, m, s).T


def merge_weight_given_norm(W0, A, B, m, n, s: float, eps: float) -> np.ndarray:
    """W' = g * (W0 + s B A) per output row with g = m / max(n, eps) for a
    given row norm n: the merged inference weight [LoRA&DoRA, section 6],
    with the magnitude scale of [ScalingDoRA, section 4 precision bullet]."""
    W0, A, B = _f64(W0), _f64(A), _f64(B)
    g, _, _ = magnitude_scale(m, n, eps)
    return g[:, None] * (W0 + s * (B @ A))
