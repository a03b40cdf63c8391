"""Parity of the CUDA compose forward/backward with the fp64 oracle.

Both sides get the same seeded inputs (bf16 or fp32 values, and the same fp32
m and n), so these checks isolate the compose from the norm."""
import numpy as np
import pytest
import torch

import oracle
import dora_adapter_factored_b200 as dora
from dora_adapter_factored_b200 import synth
from tolerances import check_bf16, check_dm, check_f32

pytestmark = pytest.mark.gpu

S = 2.0


def _np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def _inputs(T, d_out, dtype, seed, near_unity=True):
    g = torch.Generator().manual_seed(seed)
    base = torch.randn(T, d_out, generator=g).to(dtype)
    lora = torch.randn(T, d_out, generator=g).to(dtype)
    dy = torch.randn(T, d_out, generator=g).to(dtype)
    n = torch.empty(d_out).uniform_(0.5, 2.0, generator=g)
    if near_unity:
        m = n * (1 + 0.005 * torch.randn(d_out, generator=g))
    else:
        m = torch.empty(d_out).uniform_(0.25, 4.0, generator=g)
    return base, lora, dy, m.float(), n.float()


def _fwd_terms(base, lora, m, n, eps):
    g, gm1, _ = oracle.magnitude_scale(m, n, eps)
    return np.abs(base) + np.abs(gm1 * base) + np.abs(g * S * lora)


def _check_fwd(dtype, got, base, lora, m, n, eps, what):
    ref = oracle.compose_fwd(base, lora, m, n, S, eps)
    mag = _fwd_terms(base, lora, m, n, eps)
    if dtype == torch.bfloat16:
        check_bf16(got, ref, mag, what)
    else:
        check_f32(got, ref, mag, what)


SMALL = [(1, 1), (3, 7), (5, 129), (2, 8), (17, 1000), (64, 4096), (33, 24), (4, 4100)]


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("T,d_out", SMALL)
@pytest.mark.parametrize("near_unity", [True, False])
def test_compose_fwd_small(dtype, T, d_out, near_unity):
    base, lora, _, m, n = _inputs(T, d_out, dtype, 10 + T * 7 + d_out, near_unity)
    eps = synth.eps_for("bf16" if dtype == torch.bfloat16 else "f32")
    y = dora.dora_compose_fwd(base.cuda(), lora.cuda(), m.cuda(), n.cuda(), S, eps)
    torch.cuda.synchronize()
    _check_fwd(dtype, _np(y), _np(base), _np(lora), _np(m), _np(n), eps, f"y {T}x{d_out}")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("T,d_out", SMALL)
def test_compose_fwd_delta_small(dtype, T, d_out):
    base, lora, _, m, n = _inputs(T, d_out, dtype, 20 + T * 3 + d_out, True)
    eps = synth.eps_for("bf16" if dtype == torch.bfloat16 else "f32")
    d = dora.dora_compose_fwd_delta(base.cuda(), lora.cuda(), m.cuda(), n.cuda(), S, eps)
    torch.cuda.synchronize()
    b, l, mm, nn = map(_np, (base, lora, m, n))
    ref = oracle.compose_delta(b, l, mm, nn, S, eps)
    g, gm1, _ = oracle.magnitude_scale(mm, nn, eps)
    mag = np.abs(gm1 * b) + np.abs(g * S * l)
    chk = check_bf16 if dtype == torch.bfloat16 else check_f32
    chk(_np(d), ref, mag, f"dY {T}x{d_out}")


def test_compose_fwd_delta_in_place_empty_and_headline():
    eps = synth.eps_for("bf16")
    # in place over base, and T = 0
    base, lora, _, m, n = _inputs(9, 264, torch.bfloat16, 7)
    b = base.cuda()
    d = dora.dora_compose_fwd_delta(b, lora.cuda(), m.cuda(), n.cuda(), S, eps, dy_out=b)
    torch.cuda.synchronize()
    assert d.data_ptr() == b.data_ptr()
    bb, l, mm, nn = map(_np, (base, lora, m, n))
    g, gm1, _ = oracle.magnitude_scale(mm, nn, eps)
    check_bf16(_np(d), oracle.compose_delta(bb, l, mm, nn, S, eps),
               np.abs(gm1 * bb) + np.abs(g * S * l), "dY in place")
    e = torch.empty(0, 264, dtype=torch.bfloat16, device="cuda")
    dora.dora_compose_fwd_delta(e, e.clone(), m.cuda(), n.cuda(), S, eps)
    # headline activations [4096, 8192] near g = 1: every element
    T, d_out = 4096, 8192
    w = synth.WORKLOADS["headline_8192_r384"]
    s = w.modules[0].s
    base, lora = synth.activations(w, T, d_out, which=("base", "lora"))
    n = torch.empty(d_out).uniform_(1.2, 1.4, generator=torch.Generator().manual_seed(3))
    m = synth.magnitude_near_unity(w, n)
    d = dora.dora_compose_fwd_delta(base.cuda(), lora.cuda(), m.cuda(), n.cuda(), s, eps)
    torch.cuda.synchronize()
    bb, l, mm, nn = map(_np, (base, lora, m, n))
    g, gm1, _ = oracle.magnitude_scale(mm, nn, eps)
    check_bf16(_np(d), oracle.compose_delta(bb, l, mm, nn, s, eps),
               np.abs(gm1 * bb) + np.abs(g * s * l), "dY headline")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("T,d_out", SMALL)
def test_compose_bwd_small(dtype, T, d_out):
    base, lora, dy, m, n = _inputs(T, d_out, dtype, 99 + T * 5 + d_out)
    eps = synth.eps_for("bf16" if dtype == torch.bfloat16 else "f32")
    d_base, d_lora, dm = dora.dora_compose_bwd(dy.cuda(), base.cuda(), lora.cuda(), m.cuda(),
                                               n.cuda(), S, eps)
    torch.cuda.synchronize()
    b, l, d, mm, nn = map(_np, (base, lora, dy, m, n))
    rb, rl, rdm = oracle.compose_bwd(d, b, l, mm, nn, S, eps)
    g, _, nc = oracle.magnitude_scale(mm, nn, eps)
    chk = check_bf16 if dtype == torch.bfloat16 else check_f32
    chk(_np(d_base), rb, np.abs(rb), "d_base")
    chk(_np(d_lora), rl, np.abs(rl), "d_lora")
    check_dm(_np(dm), rdm, np.sum(np.abs(d * (b + S * l)), axis=0) / nc, "dm")


def test_compose_in_place_and_empty():
    base, lora, _, m, n = _inputs(9, 264, torch.bfloat16, 5)
    eps = synth.eps_for("bf16")
    b = base.cuda()
    y = dora.dora_compose_fwd(b, lora.cuda(), m.cuda(), n.cuda(), S, eps, y=b)
    torch.cuda.synchronize()
    assert y.data_ptr() == b.data_ptr()
    _check_fwd(torch.bfloat16, _np(y), _np(base), _np(lora), _np(m), _np(n), eps, "in place")
    # d_base may overwrite dy
    dy = torch.randn(9, 264, generator=torch.Generator().manual_seed(55)).bfloat16()
    d = dy.cuda()
    d_base, _, _ = dora.dora_compose_bwd(d, base.cuda(), lora.cuda(), m.cuda(), n.cuda(), S, eps,
                                         d_base=d)
    torch.cuda.synchronize()
    rb, _, _ = oracle.compose_bwd(_np(dy), _np(base), _np(lora), _np(m), _np(n), S, eps)
    check_bf16(_np(d_base), rb, np.abs(rb), "d_base in place")
    # T = 0 is a no-op
    e = torch.empty(0, 264, dtype=torch.bfloat16, device="cuda")
    dora.dora_compose_fwd(e, e.clone(), m.cuda(), n.cuda(), S, eps)
    _, _, dm = dora.dora_compose_bwd(e, e.clone(), e.clone(), m.cuda(), n.cuda(), S, eps)
    torch.cuda.synchronize()
    assert torch.all(dm == 0)


def test_compose_init_invariant_bitwise():
    # m == n and lora == 0: y must equal base exactly (g - 1 = 0, g s lora = 0).
    base, _, _, _, n = _inputs(16, 512, torch.bfloat16, 6)
    lora = torch.zeros_like(base)
    y = dora.dora_compose_fwd(base.cuda(), lora.cuda(), n.cuda(), n.cuda(), S, 2.0 ** -7)
    assert torch.equal(y.cpu(), base)


def test_compose_dm_deterministic():
    base, lora, dy, m, n = _inputs(1000, 4096, torch.bfloat16, 8)
    args = [t.cuda() for t in (dy, base, lora, m, n)]
    a = dora.dora_compose_bwd(*args, S, 2.0 ** -7)
    b = dora.dora_compose_bwd(*args, S, 2.0 ** -7)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_tiny_fp32_workload_compose():
    w = synth.WORKLOADS["tiny_fp32"]
    W0, A, B = synth.module_weights(w)
    m = synth.magnitude_from_base_rows(w, W0)
    _, base, lora, dy = synth.tiny_activations(w, W0, A, B)
    s = w.modules[0].s
    eps = synth.eps_for("f32")
    n = torch.from_numpy(oracle.dense_row_norm(W0.numpy(), A.numpy(), B.numpy(), s)).float()
    y = dora.dora_compose_fwd(base.cuda(), lora.cuda(), m.cuda(), n.cuda(), s, eps)
    d_base, d_lora, dm = dora.dora_compose_bwd(dy.cuda(), base.cuda(), lora.cuda(), m.cuda(),
                                               n.cuda(), s, eps)
    torch.cuda.synchronize()
    b, l, d, mm, nn = map(_np, (base, lora, dy, m, n))
    _check_fwd(torch.float32, _np(y), b, l, mm, nn, eps, "tiny y")
    rb, rl, rdm = oracle.compose_bwd(d, b, l, mm, nn, s, eps)
    check_f32(_np(d_base), rb, np.abs(rb), "tiny d_base")
    check_f32(_np(d_lora), rl, np.abs(rl), "tiny d_lora")
    _, _, nc = oracle.magnitude_scale(mm, nn, eps)
    check_dm(_np(dm), rdm, np.sum(np.abs(d * (b + s * l)), axis=0) / nc, "tiny dm")


def test_headline_compose_fwd_full_size():
    """[4096, 8192] bf16 activations, every element checked."""
    T, d_out = 4096, 8192
    w = synth.WORKLOADS["headline_8192_r384"]
    base, lora = synth.activations(w, T, d_out, which=("base", "lora"))
    n = torch.empty(d_out).uniform_(1.2, 1.4, generator=torch.Generator().manual_seed(3))
    m = synth.magnitude_near_unity(w, n)
    eps = synth.eps_for("bf16")
    y = dora.dora_compose_fwd(base.cuda(), lora.cuda(), m.cuda(), n.cuda(), w.modules[0].s, eps)
    torch.cuda.synchronize()
    _check_fwd(torch.bfloat16, _np(y), _np(base), _np(lora), _np(m), _np(n), eps, "headline y")


def test_mlp_up_compose_bwd_full_size_all_rows():
    """[8192, 25600] bf16: every element of y, d_base and d_lora, and dm on
    every column over all 8192 tokens, against the oracle taken over row
    chunks of 512 tokens (its dm is the sum of the chunks' sums)."""
    T, d_out = 8192, 25600
    w = synth.WORKLOADS["mlp_up_25600x5120_r384"]
    s = w.modules[0].s
    base, lora, dy = synth.activations(w, T, d_out, device="cuda")
    gen = torch.Generator().manual_seed(4)
    n = torch.empty(d_out).uniform_(1.2, 1.4, generator=gen)
    m = synth.magnitude_near_unity(w, n)
    eps = synth.eps_for("bf16")
    y = dora.dora_compose_fwd(base, lora, m.cuda(), n.cuda(), s, eps)
    d_base, d_lora, dm = dora.dora_compose_bwd(dy, base, lora, m.cuda(), n.cuda(), s, eps)
    torch.cuda.synchronize()
    mm, nn = _np(m), _np(n)
    _, _, nc = oracle.magnitude_scale(mm, nn, eps)
    rdm = np.zeros(d_out)
    scale = np.zeros(d_out)
    for r0 in range(0, T, 512):
        sl = slice(r0, r0 + 512)
        br, lr, dr = _np(base[sl]), _np(lora[sl]), _np(dy[sl])
        rb, rl, rdm_c = oracle.compose_bwd(dr, br, lr, mm, nn, s, eps)
        rdm += rdm_c
        scale += np.sum(np.abs(dr * (br + s * lr)), axis=0) / nc
        check_bf16(_np(d_base[sl]), rb, np.abs(rb), f"d_base rows {r0}+")
        check_bf16(_np(d_lora[sl]), rl, np.abs(rl), f"d_lora rows {r0}+")
        _check_fwd(torch.bfloat16, _np(y[sl]), br, lr, mm, nn, eps, f"y rows {r0}+")
    check_dm(_np(dm), rdm, scale, "dm")
