"""Parity of dora_merge_weight (W' = g (W0 + s B A), "LoRA & DoRA ...",
section 6) with the fp64 oracle.

Both sides get the same bf16 W0, A, B and fp32 m, n.  The bar is the bf16
output tolerance (2 bf16 ulps or 1e-2 relative), plus the fp32 evaluation
floor of the expression: 8 * 2^-24 * g (|W0| + s sum_k |B_ik A_kj|)."""
import numpy as np
import pytest
import torch

import oracle
import dora_adapter_factored_b200 as dora
from dora_adapter_factored_b200 import synth
from tolerances import check_bf16, check_rel

pytestmark = pytest.mark.gpu


def _np(t):
    return t.detach().double().cpu().numpy()


def _module(d_out, d_in, r, seed):
    g = torch.Generator().manual_seed(seed)
    W0 = (0.02 * torch.randn(d_out, d_in, generator=g)).bfloat16()
    A = (torch.rand(r, d_in, generator=g) * 2 - 1).div(d_in ** 0.5).bfloat16()
    B = (0.02 * torch.randn(d_out, r, generator=g)).bfloat16()
    n = torch.empty(d_out).uniform_(0.5, 2.0, generator=g)
    m = n * (1 + 0.01 * torch.randn(d_out, generator=g))
    return W0, A, B, m.float(), n.float()


def _check(got, W0, A, B, m, n, s, eps, what, rows=None):
    W0n, An, Bn, mn, nn = map(_np, (W0, A, B, m, n))
    if rows is not None:
        W0n, Bn, mn, nn = W0n[rows], Bn[rows], mn[rows], nn[rows]
    ref = oracle.merge_weight_given_norm(W0n, An, Bn, mn, nn, s, eps)
    g, _, _ = oracle.magnitude_scale(mn, nn, eps)
    mag = np.abs(g)[:, None] * (np.abs(W0n) + abs(s) * (np.abs(Bn) @ np.abs(An)))
    check_bf16(got, ref, mag, what)


@pytest.mark.parametrize("d_out,d_in,r", [(128, 128, 64), (200, 136, 24), (1, 8, 8),
                                          (300, 1000, 384), (256, 512, 512), (129, 264, 8),
                                          (640, 384, 128)])
def test_merge_small(d_out, d_in, r):
    W0, A, B, m, n = _module(d_out, d_in, r, d_out * 31 + d_in + r)
    s, eps = 2.0, 2.0 ** -7
    W = dora.dora_merge_weight(W0.cuda(), A.cuda(), B.cuda(), m.cuda(), n.cuda(), s, eps)
    torch.cuda.synchronize()
    assert dora.dora_get_device_status() == 0
    _check(_np(W), W0, A, B, m, n, s, eps, f"W' {d_out}x{d_in} r={r}")


def test_merge_in_place_and_repeatable():
    W0, A, B, m, n = _module(384, 640, 96, 7)
    s, eps = 0.5, 2.0 ** -7
    ref = dora.dora_merge_weight(W0.cuda(), A.cuda(), B.cuda(), m.cuda(), n.cuda(), s, eps)
    w = W0.cuda()
    out = dora.dora_merge_weight(w, A.cuda(), B.cuda(), m.cuda(), n.cuda(), s, eps, W_out=w)
    torch.cuda.synchronize()
    assert out.data_ptr() == w.data_ptr()
    assert torch.equal(out, ref)
    _check(_np(out), W0, A, B, m, n, s, eps, "in place")


def test_merge_init_is_w0():
    # B = 0, m = n: g = 1 and W' = W0 bit for bit.
    W0, A, _, _, n = _module(256, 256, 64, 9)
    B = torch.zeros(256, 64, dtype=torch.bfloat16)
    W = dora.dora_merge_weight(W0.cuda(), A.cuda(), B.cuda(), n.cuda(), n.cuda(), 2.0, 2.0 ** -7)
    assert torch.equal(W.cpu(), W0)


def test_headline_norm_then_merge_sampled():
    """8192 x 8192, r = 384: the GPU norm, then the merge; 64 sampled rows
    checked element by element against the oracle (given the GPU's n, an
    input of the merge), and every row's norm equal to m within the bf16
    rounding of W' (2^-8 relative)."""
    w = synth.WORKLOADS["headline_8192_r384"]
    W0, A, B = synth.module_weights(w, device="cuda")
    s = w.modules[0].s
    eps = synth.eps_for("bf16")
    n, _ = dora.dora_factored_norm(W0, A, B, s)
    m = synth.magnitude_near_unity(w, n.cpu()).cuda()
    W = dora.dora_merge_weight(W0, A, B, m, n, s, eps)
    torch.cuda.synchronize()
    rows = torch.randperm(8192, generator=torch.Generator().manual_seed(2))[:64].sort().values
    _check(_np(W[rows.cuda()]), W0, A, B, m, n, s, eps, "headline W'", rows=rows.numpy())
    row_norm = W.float().norm(dim=1)
    check_rel(_np(row_norm), _np(m), 2.0 ** -8, "row norms of W'")
