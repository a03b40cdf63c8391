"""The cancellation-safe compose against a naive evaluation, near g = 1.

"Scaling DoRA" (section 3, numerical-stability bullets) reports that the
stable form -- (g - 1) formed in fp32 as (m - n)/n, fp32 intermediates, one
rounding -- has about 3.0x lower peak error than the naive form near g = 1, in
bf16, at d_out = 8192 and d_in = 2048 against an fp64 reference, with g
concentrated around 1 (std about 0.0015).

Reading: the [2048, 8192] activations of such a layer, g = 1 + N(0, 0.0015).
The naive form rounds g to bf16 first and evaluates
base + ((g - 1) base + g s lora) in bf16 arithmetic (each op rounded to bf16),
written here with torch ops for the test only.  The ratio of the two peak
errors is printed (the pages' 3.0x is context, not a bar); the test asserts
only that the stable form is the more accurate one and stays within the
parity bar (2 bf16 ulps or 1e-2 relative).
"""
import numpy as np
import pytest
import torch

import oracle
import dora_adapter_factored_b200 as dora
from tolerances import check_bf16

pytestmark = pytest.mark.gpu


def _case(T, d_out, lora_std, seed):
    g = torch.Generator().manual_seed(seed)
    base = torch.randn(T, d_out, generator=g).bfloat16()
    lora = (lora_std * torch.randn(T, d_out, generator=g)).bfloat16()
    n = torch.empty(d_out).uniform_(0.5, 2.0, generator=g)
    gg = 1.0 + 0.0015 * torch.randn(d_out, generator=g).double()
    m = (n.double() * gg).float()
    return base, lora, m, n.float()


@pytest.mark.parametrize("lora_std", [1.0, 0.05])
def test_stable_compose_beats_naive_bf16_near_unity(lora_std):
    T, d_out, s, eps = 2048, 8192, 2.0, 2.0 ** -7
    base, lora, m, n = _case(T, d_out, lora_std, 2048 + int(lora_std * 100))
    y = dora.dora_compose_fwd(base.cuda(), lora.cuda(), m.cuda(), n.cuda(), s, eps)
    # naive: g rounded to bf16, every operation in bf16
    gb = (m.cuda() / n.cuda().clamp_min(eps)).bfloat16()
    b, l = base.cuda(), lora.cuda()
    y_naive = b + ((gb - 1) * b + (gb * s) * l)
    torch.cuda.synchronize()
    ref = oracle.compose_fwd(base.double().numpy(), lora.double().numpy(), m.double().numpy(),
                             n.double().numpy(), s, eps)
    got = y.double().cpu().numpy()
    naive = y_naive.double().cpu().numpy()
    err_stable = float(np.max(np.abs(got - ref)))
    err_naive = float(np.max(np.abs(naive - ref)))
    ratio = err_naive / err_stable
    print(f"\nlora std {lora_std}: peak |error| stable {err_stable:.3e}, naive bf16 {err_naive:.3e},"
          f" ratio {ratio:.2f} (pages: 3.0x)")
    b64, l64 = base.double().numpy(), lora.double().numpy()
    check_bf16(got, ref, np.abs(b64) + np.abs(s * l64) * 1.01, "stable compose")
    assert err_stable < err_naive
