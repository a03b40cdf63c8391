"""Parity of the training-forward (y and inner), backward-from-inner and
frozen-magnitude backward calls with the fp64 oracle ("Scaling DoRA ...",
section 4, tier 1, and section 6).

Each call gets seeded synthetic inputs that both sides see; the oracle never
takes a value the CUDA path produced, except in the chained test, which runs
the forward and the backward on the GPU and compares the end result with the
oracle's backward from base and lora."""
import numpy as np
import pytest
import torch

import oracle
import dora_adapter_factored_b200 as dora
from dora_adapter_factored_b200 import synth
from tolerances import check_bf16, check_dm, check_f32

pytestmark = pytest.mark.gpu

S = 2.0
SHAPES = [(1, 1), (3, 7), (5, 129), (2, 8), (17, 1000), (64, 4096), (33, 24), (4, 4100),
          (300, 264)]


def _np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def _inputs(T, d_out, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    base = torch.randn(T, d_out, generator=g).to(dtype)
    lora = torch.randn(T, d_out, generator=g).to(dtype)
    dy = torch.randn(T, d_out, generator=g).to(dtype)
    inner = torch.randn(T, d_out, generator=g).to(dtype)
    n = torch.empty(d_out).uniform_(0.5, 2.0, generator=g)
    m = n * (1 + 0.005 * torch.randn(d_out, generator=g))
    return base, lora, dy, inner, m.float(), n.float()


def _eps(dtype):
    return synth.eps_for("bf16" if dtype == torch.bfloat16 else "f32")


def _chk(dtype):
    return check_bf16 if dtype == torch.bfloat16 else check_f32


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("T,d_out", SHAPES)
def test_fwd_train(dtype, T, d_out):
    base, lora, _, _, m, n = _inputs(T, d_out, dtype, 7 * T + d_out)
    eps = _eps(dtype)
    y, inner = dora.dora_compose_fwd_train(base.cuda(), lora.cuda(), m.cuda(), n.cuda(), S, eps)
    torch.cuda.synchronize()
    b, l, mm, nn = map(_np, (base, lora, m, n))
    g, gm1, _ = oracle.magnitude_scale(mm, nn, eps)
    ry = oracle.compose_fwd(b, l, mm, nn, S, eps)
    _chk(dtype)(_np(y), ry, np.abs(b) + np.abs(gm1 * b) + np.abs(g * S * l), f"y {T}x{d_out}")
    ri = oracle.compose_inner(b, l, S)
    _chk(dtype)(_np(inner), ri, np.abs(b) + np.abs(S * l), f"inner {T}x{d_out}")


def test_fwd_train_y_matches_plain_forward_bitwise():
    # Same per-element arithmetic as dora_compose_fwd: y is bit-identical.
    base, lora, _, _, m, n = _inputs(257, 4096, torch.bfloat16, 3)
    args = [t.cuda() for t in (base, lora, m, n)]
    y0 = dora.dora_compose_fwd(*args, S, 2.0 ** -7)
    y1, _ = dora.dora_compose_fwd_train(*args, S, 2.0 ** -7)
    assert torch.equal(y0, y1)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("T,d_out", SHAPES)
def test_bwd_inner(dtype, T, d_out):
    _, _, dy, inner, m, n = _inputs(T, d_out, dtype, 11 * T + d_out)
    eps = _eps(dtype)
    d_base, d_lora, dm = dora.dora_compose_bwd_inner(dy.cuda(), inner.cuda(), m.cuda(), n.cuda(),
                                                     S, eps)
    torch.cuda.synchronize()
    d, i, mm, nn = map(_np, (dy, inner, m, n))
    rb, rl, rdm = oracle.compose_bwd_from_inner(d, i, mm, nn, S, eps)
    _, _, nc = oracle.magnitude_scale(mm, nn, eps)
    _chk(dtype)(_np(d_base), rb, np.abs(rb), "d_base")
    _chk(dtype)(_np(d_lora), rl, np.abs(rl), "d_lora")
    check_dm(_np(dm), rdm, np.sum(np.abs(d * i), axis=0) / nc, "dm")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("T,d_out", SHAPES)
def test_bwd_frozen(dtype, T, d_out):
    _, _, dy, _, m, n = _inputs(T, d_out, dtype, 13 * T + d_out)
    eps = _eps(dtype)
    d_base, d_lora = dora.dora_compose_bwd_frozen(dy.cuda(), m.cuda(), n.cuda(), S, eps)
    torch.cuda.synchronize()
    rb, rl = oracle.compose_bwd_frozen(_np(dy), _np(m), _np(n), S, eps)
    _chk(dtype)(_np(d_base), rb, np.abs(rb), "d_base")
    _chk(dtype)(_np(d_lora), rl, np.abs(rl), "d_lora")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_train_chain_matches_oracle_backward(dtype):
    """GPU forward (y, inner) then GPU backward from inner, against the
    oracle's backward from base and lora.  d_base and d_lora do not depend on
    inner; dm carries inner's rounding to the activation dtype (at most half
    an ulp, 2^-9 relative for bf16, per element), so its bound adds
    2^-9 sum_t |dy inner| / n_c for bf16."""
    T, d_out = 1000, 4096
    base, lora, dy, _, m, n = _inputs(T, d_out, dtype, 21)
    eps = _eps(dtype)
    mc, nc_ = m.cuda(), n.cuda()
    _, inner = dora.dora_compose_fwd_train(base.cuda(), lora.cuda(), mc, nc_, S, eps)
    d_base, d_lora, dm = dora.dora_compose_bwd_inner(dy.cuda(), inner, mc, nc_, S, eps)
    torch.cuda.synchronize()
    b, l, d, mm, nn = map(_np, (base, lora, dy, m, n))
    rb, rl, rdm = oracle.compose_bwd(d, b, l, mm, nn, S, eps)
    _, _, ncl = oracle.magnitude_scale(mm, nn, eps)
    _chk(dtype)(_np(d_base), rb, np.abs(rb), "d_base")
    _chk(dtype)(_np(d_lora), rl, np.abs(rl), "d_lora")
    abs_sum = np.sum(np.abs(d * (b + S * l)), axis=0) / ncl
    if dtype == torch.bfloat16:
        err = np.abs(_np(dm) - rdm)
        bound = 2.0 ** -9 * abs_sum + 1e-5 * abs_sum + 1e-6 * np.abs(rdm)
        assert (err <= bound).all(), float(np.max(err / bound))
    else:
        check_dm(_np(dm), rdm, abs_sum, "dm")


def test_in_place_and_empty():
    base, lora, dy, inner, m, n = _inputs(9, 264, torch.bfloat16, 5)
    eps = 2.0 ** -7
    b, l = base.cuda(), lora.cuda()
    y, i = dora.dora_compose_fwd_train(b, l, m.cuda(), n.cuda(), S, eps, y=b, inner=l)
    torch.cuda.synchronize()
    assert y.data_ptr() == b.data_ptr() and i.data_ptr() == l.data_ptr()
    bb, ll, mm, nn = map(_np, (base, lora, m, n))
    check_bf16(_np(y), oracle.compose_fwd(bb, ll, mm, nn, S, eps), np.abs(bb) + np.abs(S * ll),
               "y in place")
    check_bf16(_np(i), oracle.compose_inner(bb, ll, S), np.abs(bb) + np.abs(S * ll), "inner")
    d = dy.cuda()
    db, _, _ = dora.dora_compose_bwd_inner(d, inner.cuda(), m.cuda(), n.cuda(), S, eps, d_base=d)
    d2 = dy.cuda()
    db2, _ = dora.dora_compose_bwd_frozen(d2, m.cuda(), n.cuda(), S, eps, d_base=d2)
    torch.cuda.synchronize()
    rb, _ = oracle.compose_bwd_frozen(_np(dy), mm, nn, S, eps)
    check_bf16(_np(db), rb, np.abs(rb), "d_base in place (inner)")
    check_bf16(_np(db2), rb, np.abs(rb), "d_base in place (frozen)")
    e = torch.empty(0, 264, dtype=torch.bfloat16, device="cuda")
    dora.dora_compose_fwd_train(e, e.clone(), m.cuda(), n.cuda(), S, eps)
    _, _, dm = dora.dora_compose_bwd_inner(e, e.clone(), m.cuda(), n.cuda(), S, eps)
    dora.dora_compose_bwd_frozen(e, m.cuda(), n.cuda(), S, eps)
    torch.cuda.synchronize()
    assert torch.all(dm == 0)
    assert dora.dora_get_device_status() == 0


def test_bwd_inner_dm_deterministic():
    _, _, dy, inner, m, n = _inputs(3000, 4096, torch.bfloat16, 8)
    args = [t.cuda() for t in (dy, inner, m, n)]
    a = dora.dora_compose_bwd_inner(*args, S, 2.0 ** -7)
    b = dora.dora_compose_bwd_inner(*args, S, 2.0 ** -7)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_headline_train_chain_sampled():
    """[4096, 8192] bf16 at the headline sizes in the launch configuration the
    bench uses: y and inner on sampled rows, dm on sampled columns."""
    T, d_out = 4096, 8192
    w = synth.WORKLOADS["headline_8192_r384"]
    s = w.modules[0].s
    base, lora, dy = synth.activations(w, T, d_out, device="cuda")
    gen = torch.Generator().manual_seed(5)
    n = torch.empty(d_out).uniform_(1.2, 1.4, generator=gen)
    m = synth.magnitude_near_unity(w, n)
    eps = synth.eps_for("bf16")
    y, inner = dora.dora_compose_fwd_train(base, lora, m.cuda(), n.cuda(), s, eps)
    d_base, d_lora, dm = dora.dora_compose_bwd_inner(dy, inner, m.cuda(), n.cuda(), s, eps)
    db_f, dl_f = dora.dora_compose_bwd_frozen(dy, m.cuda(), n.cuda(), s, eps)
    torch.cuda.synchronize()
    assert torch.equal(db_f, d_base) and torch.equal(dl_f, d_lora)
    rows = torch.randperm(T, generator=gen)[:64].sort().values.cuda()
    cols = torch.randperm(d_out, generator=gen)[:256].sort().values.cuda()
    mm, nn = _np(m), _np(n)
    br, lr, dr = _np(base[rows]), _np(lora[rows]), _np(dy[rows])
    g, gm1, ncl = oracle.magnitude_scale(mm, nn, eps)
    check_bf16(_np(y[rows]), oracle.compose_fwd(br, lr, mm, nn, s, eps),
               np.abs(br) + np.abs(gm1 * br) + np.abs(g * s * lr), "y")
    check_bf16(_np(inner[rows]), oracle.compose_inner(br, lr, s), np.abs(br) + np.abs(s * lr),
               "inner")
    rb, rl = oracle.compose_bwd_frozen(dr, mm, nn, s, eps)
    check_bf16(_np(d_base[rows]), rb, np.abs(rb), "d_base")
    check_bf16(_np(d_lora[rows]), rl, np.abs(rl), "d_lora")
    ic, dc = _np(inner[:, cols]), _np(dy[:, cols])
    cn = cols.cpu().numpy()
    _, _, rdm = oracle.compose_bwd_from_inner(dc, ic, mm[cn], nn[cn], s, eps)
    check_dm(_np(dm)[cn], rdm, np.sum(np.abs(dc * ic), axis=0) / ncl[cn], "dm")
