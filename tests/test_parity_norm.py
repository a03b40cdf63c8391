"""Parity of the CUDA factored norm (and g = m / max(n, eps)) with the fp64
oracle's dense norm of W0 + sBA."""
import numpy as np
import pytest
import torch

import oracle
import dora_adapter_factored_b200 as dora
from dora_adapter_factored_b200 import synth
from tolerances import check_bf16, check_rel

pytestmark = pytest.mark.gpu


def _np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def _module(d_out, d_in, r, dtype, seed, b_std=0.02):
    g = torch.Generator().manual_seed(seed)
    W0 = (0.02 * torch.randn(d_out, d_in, generator=g)).to(dtype)
    bound = 1.0 / np.sqrt(d_in)
    A = torch.empty(r, d_in).uniform_(-bound, bound, generator=g).to(dtype)
    B = (b_std * torch.randn(d_out, r, generator=g)).to(dtype)
    m = (torch.linalg.vector_norm(W0.double(), dim=1) * (1 + 0.005 * torch.randn(d_out, generator=g).double())).float()
    return W0, A, B, m


def _check(W0, A, B, m, s, eps, n, g, rtol, what, rows=None):
    W, Aa, Bb = _np(W0), _np(A), _np(B)
    if rows is not None:
        W, Bb = W[rows], Bb[rows]
    ref = oracle.dense_row_norm(W, Aa, Bb, s)
    got_n = _np(n) if rows is None else _np(n)[rows]
    check_rel(got_n, ref, rtol, f"{what} n")
    if g is not None:
        mm = _np(m) if rows is None else _np(m)[rows]
        rg, _, _ = oracle.magnitude_scale(mm, ref, eps)
        got_g = _np(g) if rows is None else _np(g)[rows]
        check_rel(got_g, rg, rtol, f"{what} g")
    return ref


# (d_out, d_in, r): tensor-core path (d_in, r multiples of 8) with ragged
# tiles, ragged K, one or two accumulator chunks, and the maximum rank.
TC_SHAPES = [
    (128, 64, 16), (1, 64, 8), (7, 136, 72), (129, 200, 24), (300, 1000, 264),
    (256, 512, 384), (130, 256, 512), (64, 4096, 64), (1000, 72, 128), (513, 320, 320),
    (2048, 1024, 48),
]


@pytest.mark.parametrize("d_out,d_in,r", TC_SHAPES)
def test_norm_tensor_core_path(d_out, d_in, r):
    W0, A, B, m = _module(d_out, d_in, r, torch.bfloat16, d_out * 31 + d_in * 7 + r)
    s, eps = 2.0, 2.0 ** -7
    n, g = dora.dora_factored_norm(W0.cuda(), A.cuda(), B.cuda(), s, m.cuda(), eps)
    torch.cuda.synchronize()
    assert dora.dora_get_device_status() == 0
    _check(W0, A, B, m, s, eps, n, g, 1e-3, f"{d_out}x{d_in} r{r}")


@pytest.mark.parametrize("d_out,d_in,r", [(7, 37, 5), (33, 64, 12), (5, 100, 3), (64, 48, 8)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_norm_cuda_core_path(d_out, d_in, r, dtype):
    W0, A, B, m = _module(d_out, d_in, r, dtype, 7 + d_out + r, b_std=0.1)
    s, eps = 2.0, 2.0 ** -23
    n, g = dora.dora_factored_norm(W0.cuda(), A.cuda(), B.cuda(), s, m.cuda(), eps)
    torch.cuda.synchronize()
    _check(W0, A, B, m, s, eps, n, g, 1e-5 if dtype == torch.float32 else 1e-3,
           f"{dtype} {d_out}x{d_in} r{r}")


def test_norm_large_update_and_zero_rows():
    # A large s B A (n far from ||W0_i||), and rows where W0_i = 0 and B_i = 0
    # (n = 0, g = m / eps).
    d_out, d_in, r = 256, 256, 32
    W0, A, B, m = _module(d_out, d_in, r, torch.bfloat16, 77, b_std=0.5)
    W0[5] = 0
    B[5] = 0
    W0[200] = 0
    B[200] = 0
    eps = 2.0 ** -7
    n, g = dora.dora_factored_norm(W0.cuda(), A.cuda(), B.cuda(), 4.0, m.cuda(), eps)
    torch.cuda.synchronize()
    nn, gg = n.cpu(), g.cpu()
    assert nn[5] == 0 and nn[200] == 0
    assert gg[5] == torch.tensor(m[5].item() / eps, dtype=torch.float32)
    keep = [i for i in range(d_out) if i not in (5, 200)]
    _check(W0, A, B, m, 4.0, eps, n, g, 1e-3, "large update", rows=keep)


def test_norm_b_zero_equals_row_norm_of_w0():
    # B = 0: n_i = ||W0_i|| (the init state), against numpy's row norm.
    W0, A, _, _ = _module(384, 768, 64, torch.bfloat16, 3)
    B = torch.zeros(384, 64, dtype=torch.bfloat16)
    n, _ = dora.dora_factored_norm(W0.cuda(), A.cuda(), B.cuda(), 2.0)
    torch.cuda.synchronize()
    check_rel(_np(n), np.linalg.norm(_np(W0), axis=1), 1e-3, "B=0")


def test_norm_deterministic():
    W0, A, B, m = _module(1000, 2048, 384, torch.bfloat16, 11)
    args = (W0.cuda(), A.cuda(), B.cuda(), 2.0, m.cuda(), 2.0 ** -7)
    n1, g1 = dora.dora_factored_norm(*args)
    n2, g2 = dora.dora_factored_norm(*args)
    assert torch.equal(n1, n2) and torch.equal(g1, g2)


def test_tiny_fp32_workload_norm():
    w = synth.WORKLOADS["tiny_fp32"]
    W0, A, B = synth.module_weights(w)
    m = synth.magnitude_from_base_rows(w, W0)
    s, eps = w.modules[0].s, synth.eps_for("f32")
    n, g = dora.dora_factored_norm(W0.cuda(), A.cuda(), B.cuda(), s, m.cuda(), eps)
    torch.cuda.synchronize()
    _check(W0, A, B, m, s, eps, n, g, 1e-5, "tiny_fp32")


def test_norm_4096_r64_all_rows():
    w = synth.WORKLOADS["norm_4096_r64"]
    W0, A, B = synth.module_weights(w)
    m = synth.magnitude_from_base_rows(w, W0)
    s, eps = w.modules[0].s, synth.eps_for("bf16")
    n, g = dora.dora_factored_norm(W0.cuda(), A.cuda(), B.cuda(), s, m.cuda(), eps)
    torch.cuda.synchronize()
    _check(W0, A, B, m, s, eps, n, g, 1e-3, "norm_4096_r64")


def test_norm_mlp_up_25600x5120_all_rows():
    """Every row of the 25600 x 5120, r = 384 module (its norm spans many
    pair tiles and stream-K segment boundaries), against the oracle's dense
    norm taken over row blocks of 2048."""
    w = synth.WORKLOADS["mlp_up_25600x5120_r384"]
    W0, A, B = synth.module_weights(w, device="cuda")
    m = synth.magnitude_from_base_rows(w, W0)
    s, eps = w.modules[0].s, synth.eps_for("bf16")
    n, g = dora.dora_factored_norm(W0, A, B, s, m, eps)
    torch.cuda.synchronize()
    d_out = W0.shape[0]
    Aa = _np(A)
    ref = np.concatenate([oracle.rows_dense_row_norm(_np(W0[r0:r0 + 2048]), Aa,
                                                     _np(B[r0:r0 + 2048]), s)
                          for r0 in range(0, d_out, 2048)])
    check_rel(_np(n), ref, 1e-3, "mlp_up n")
    rg, _, _ = oracle.magnitude_scale(_np(m), ref, eps)
    check_rel(_np(g), rg, 1e-3, "mlp_up g")


def test_headline_norm_then_compose_full_path():
    """Norm -> g -> compose on the headline module, with m near unity built
    from the oracle's norm; y checked on sampled rows.  The compose bound adds
    the propagated norm error 2 * max_rel_err(n) * |g (base + s lora)|."""
    w = synth.WORKLOADS["headline_8192_r384"]
    W0, A, B = synth.module_weights(w)
    s, eps = w.modules[0].s, synth.eps_for("bf16")
    n_ref = oracle.dense_row_norm(_np(W0), _np(A), _np(B), s)
    m = synth.magnitude_near_unity(w, torch.from_numpy(n_ref))
    n, g = dora.dora_factored_norm(W0.cuda(), A.cuda(), B.cuda(), s, m.cuda(), eps)
    base, lora = synth.activations(w, w.tokens, W0.shape[0], which=("base", "lora"))
    y = dora.dora_compose_fwd(base.cuda(), lora.cuda(), m.cuda(), n, s, eps)
    torch.cuda.synchronize()
    check_rel(_np(n), n_ref, 1e-3, "n")
    rel = float(np.max(np.abs(_np(n) - n_ref) / n_ref))
    rows = torch.randperm(w.tokens, generator=torch.Generator().manual_seed(2))[:128]
    b, l = _np(base[rows]), _np(lora[rows])
    mm = _np(m)
    ref = oracle.compose_fwd(b, l, mm, n_ref, s, eps)
    gg, gm1, _ = oracle.magnitude_scale(mm, n_ref, eps)
    mag = np.abs(b) + np.abs(gm1 * b) + np.abs(gg * s * l)
    prop = 2 * rel * np.abs(gg * (b + s * l)) / (8 * 2.0 ** -24)
    check_bf16(_np(y[rows.cuda()]), ref, mag + prop, "y")
    gd = _np(g)
    assert np.all(np.abs(gd - 1) < 1e-2)
