"""Parity of the grouped factored norm (one launch per stage for many modules)
with the fp64 oracle, per module."""
import numpy as np
import pytest
import torch

import oracle
import dora_adapter_factored_b200 as dora
from dora_adapter_factored_b200 import synth
from tolerances import check_rel

pytestmark = pytest.mark.gpu


def _np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def test_grouped_small_heterogeneous():
    shapes = [(128, 64, 16), (7, 136, 72), (300, 1000, 264), (130, 256, 512), (1, 64, 8),
              (1000, 512, 384)]
    gen = torch.Generator().manual_seed(21)
    items = []
    for d_out, d_in, r in shapes:
        W0 = (0.02 * torch.randn(d_out, d_in, generator=gen)).bfloat16()
        A = torch.empty(r, d_in).uniform_(-d_in ** -0.5, d_in ** -0.5, generator=gen).bfloat16()
        B = (0.05 * torch.randn(d_out, r, generator=gen)).bfloat16()
        m = torch.empty(d_out).uniform_(0.5, 1.5, generator=gen)
        items.append(dict(W0=W0.cuda(), A=A.cuda(), B=B.cuda(), s=1.5, m=m.cuda(),
                          n_out=torch.empty(d_out, device="cuda"),
                          g_out=torch.empty(d_out, device="cuda"), cpu=(W0, A, B, m)))
    eps = 2.0 ** -7
    dora.dora_factored_norm_grouped(items, eps)
    torch.cuda.synchronize()
    assert dora.dora_get_device_status() == 0
    for i, it in enumerate(items):
        W0, A, B, m = it["cpu"]
        ref = oracle.dense_row_norm(_np(W0), _np(A), _np(B), 1.5)
        check_rel(_np(it["n_out"]), ref, 1e-3, f"module {i} n")
        rg, _, _ = oracle.magnitude_scale(_np(m), ref, eps)
        check_rel(_np(it["g_out"]), rg, 1e-3, f"module {i} g")


def test_grouped_without_magnitude():
    gen = torch.Generator().manual_seed(5)
    items = []
    for d_out in (256, 64):
        W0 = (0.02 * torch.randn(d_out, 128, generator=gen)).bfloat16()
        A = (0.05 * torch.randn(32, 128, generator=gen)).bfloat16()
        B = (0.05 * torch.randn(d_out, 32, generator=gen)).bfloat16()
        items.append(dict(W0=W0.cuda(), A=A.cuda(), B=B.cuda(), s=2.0,
                          n_out=torch.empty(d_out, device="cuda"), cpu=(W0, A, B)))
    dora.dora_factored_norm_grouped(items, 0.0)
    torch.cuda.synchronize()
    for it in items:
        W0, A, B = it["cpu"]
        check_rel(_np(it["n_out"]), oracle.dense_row_norm(_np(W0), _np(A), _np(B), 2.0), 1e-3, "n")


def test_layer_stack_56_modules_sampled_rows():
    """All 56 adapted projections of an 8-layer stack in one grouped call;
    64 rows of every module checked (first, last and random)."""
    w = synth.WORKLOADS["layer_stack_56"]
    eps = synth.eps_for("bf16")
    items = []
    for i, ms in enumerate(w.modules):
        W0, A, B = synth.module_weights(w, i, device="cuda")
        m = synth.magnitude_from_base_rows(w, W0, i)
        items.append(dict(W0=W0, A=A, B=B, s=ms.s, m=m, n_out=torch.empty(ms.d_out, device="cuda"),
                          g_out=torch.empty(ms.d_out, device="cuda")))
    dora.dora_factored_norm_grouped(items, eps)
    torch.cuda.synchronize()
    assert dora.dora_get_device_status() == 0
    gen = torch.Generator().manual_seed(56)
    for i, it in enumerate(items):
        d_out = it["W0"].shape[0]
        rows = torch.cat([torch.tensor([0, 127, 128, d_out - 1]),
                          torch.randperm(d_out, generator=gen)[:60]]).unique().sort().values.cuda()
        ref = oracle.rows_dense_row_norm(_np(it["W0"][rows]), _np(it["A"]), _np(it["B"][rows]),
                                         it["s"])
        check_rel(_np(it["n_out"][rows]), ref, 1e-3, f"{w.modules[i].name} n")
        rg, _, _ = oracle.magnitude_scale(_np(it["m"][rows]), ref, eps)
        check_rel(_np(it["g_out"][rows]), rg, 1e-3, f"{w.modules[i].name} g")
        del it["W0"]
