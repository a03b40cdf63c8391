"""Out-of-bounds writes: every output of every entry point is a view into a
larger buffer whose guard zones before and after it hold a canary pattern;
after the call the canaries must be untouched (the sanitizer substitute for
stores, with the debug build's index checks).  Small odd shapes, so that
ragged tiles, column tails and row tails are all reached."""
import pytest
import torch

import dora_adapter_factored_b200 as dora

pytestmark = pytest.mark.gpu

GUARD = 4096  # elements on each side


def _guarded(shape, dtype):
    """(view, whole): `view` of `shape` inside `whole`, canaries around it."""
    n = 1
    for x in shape:
        n *= x
    whole = torch.empty(n + 2 * GUARD, dtype=dtype, device="cuda")
    if dtype == torch.float32:
        whole.view(torch.int32).fill_(0x7f7f1234)
    else:
        whole.view(torch.int16).fill_(0x7f13)
    return whole[GUARD:GUARD + n].view(*shape), whole


def _intact(whole, what):
    torch.cuda.synchronize()
    if whole.dtype == torch.float32:
        pre, post, pat = whole[:GUARD].view(torch.int32), whole[-GUARD:].view(torch.int32), 0x7f7f1234
    else:
        pre, post, pat = whole[:GUARD].view(torch.int16), whole[-GUARD:].view(torch.int16), 0x7f13
    assert bool((pre == pat).all()) and bool((post == pat).all()), f"{what}: guard zone written"


@pytest.mark.parametrize("d_out,d_in,r", [(300, 520, 8), (777, 1096, 264), (513, 4160, 384)])
def test_norm_outputs_and_workspace_guarded(d_out, d_in, r):
    g = torch.Generator().manual_seed(d_out)
    W0 = (0.02 * torch.randn(d_out, d_in, generator=g)).bfloat16().cuda()
    A = ((torch.rand(r, d_in, generator=g) - 0.5) / d_in ** 0.5).bfloat16().cuda()
    B = (0.02 * torch.randn(d_out, r, generator=g)).bfloat16().cuda()
    m = torch.rand(d_out, generator=g).cuda() + 0.5
    n, nw = _guarded((d_out,), torch.float32)
    gg, gw = _guarded((d_out,), torch.float32)
    # workspace: 256-byte aligned, canary bytes on both sides of its extent
    wsz = dora.dora_factored_norm_workspace_size(d_out, d_in, r, torch.bfloat16)
    whole = torch.full((wsz + 2 * GUARD + 256,), 0x5A, dtype=torch.uint8, device="cuda")
    off = GUARD + (-(whole.data_ptr() + GUARD)) % 256
    ws = whole[off:off + wsz]
    dora.dora_factored_norm(W0, A, B, 2.0, m=m, eps=2 ** -7, n_out=n, g_out=gg, ws=ws)
    _intact(nw, "n"); _intact(gw, "g")
    assert bool((whole[:off] == 0x5A).all()) and bool((whole[off + wsz:] == 0x5A).all()), \
        "workspace: guard zone written"
    assert dora.dora_get_device_status() == 0


def test_compose_outputs_guarded():
    T, d = 17, 1000
    g = torch.Generator().manual_seed(3)
    base, lora, dy = (torch.randn(T, d, generator=g).bfloat16().cuda() for _ in range(3))
    nn = torch.rand(d, generator=g).cuda() + 0.5
    m = nn * 1.01
    y, yw = _guarded((T, d), torch.bfloat16)
    dora.dora_compose_fwd(base, lora, m, nn, 2.0, 2 ** -7, y=y)
    _intact(yw, "y")
    dd, dw = _guarded((T, d), torch.bfloat16)
    dora.dora_compose_fwd_delta(base, lora, m, nn, 2.0, 2 ** -7, dy_out=dd)
    _intact(dw, "dY")
    y2, y2w = _guarded((T, d), torch.bfloat16)
    inner, iw = _guarded((T, d), torch.bfloat16)
    dora.dora_compose_fwd_train(base, lora, m, nn, 2.0, 2 ** -7, y=y2, inner=inner)
    _intact(y2w, "y (train)"); _intact(iw, "inner")
    db, dbw = _guarded((T, d), torch.bfloat16)
    dl, dlw = _guarded((T, d), torch.bfloat16)
    dm, dmw = _guarded((d,), torch.float32)
    dora.dora_compose_bwd(dy, base, lora, m, nn, 2.0, 2 ** -7, d_base=db, d_lora=dl, dm=dm)
    _intact(dbw, "d_base"); _intact(dlw, "d_lora"); _intact(dmw, "dm")
    assert dora.dora_get_device_status() == 0


def test_merge_output_guarded():
    d_out, d_in, r = 300, 520, 8
    g = torch.Generator().manual_seed(9)
    W0 = (0.02 * torch.randn(d_out, d_in, generator=g)).bfloat16().cuda()
    A = ((torch.rand(r, d_in, generator=g) - 0.5) / d_in ** 0.5).bfloat16().cuda()
    B = (0.02 * torch.randn(d_out, r, generator=g)).bfloat16().cuda()
    n, _ = dora.dora_factored_norm(W0, A, B, 2.0)
    out, ow = _guarded((d_out, d_in), torch.bfloat16)
    dora.dora_merge_weight(W0, A, B, n * 1.01, n, 2.0, 2 ** -7, W_out=out)
    _intact(ow, "W'")
    assert dora.dora_get_device_status() == 0
