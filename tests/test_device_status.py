"""The bounded-wait give-up path: a kernel that waits on a barrier nothing
signals returns, records DORA_ERR_TIMEOUT, and leaves the context usable.  No
fault, trap or hang is involved: every wait in the library has a limit."""
import numpy as np
import pytest
import torch

import oracle
import dora_adapter_factored_b200 as dora
from dora_adapter_factored_b200 import _abi
from tolerances import check_rel

pytestmark = pytest.mark.gpu


def test_unsignalled_wait_gives_up_and_reports():
    assert dora.dora_get_device_status() == _abi.DORA_OK
    dora.dora_debug_unsignalled_wait(2_000_000)  # 2 ms
    assert dora.dora_get_device_status() == _abi.DORA_ERR_TIMEOUT
    assert dora.dora_get_device_status() == _abi.DORA_OK  # cleared
    x = torch.ones(4, 8, device="cuda")
    assert float((x * 2).sum()) == 64.0  # context still usable


def _module(seed):
    g = torch.Generator().manual_seed(seed)
    W0 = (0.02 * torch.randn(256, 1024, generator=g)).bfloat16()
    A = (0.03 * torch.randn(384, 1024, generator=g)).bfloat16()
    B = (0.02 * torch.randn(256, 384, generator=g)).bfloat16()
    return W0, A, B


def test_norm_pipeline_with_tiny_wait_limit_stays_usable():
    """With a 1 ns wait limit the tensor-core pipeline may give up at its first
    wait that does not succeed at once.  Whatever happens, the call returns, a
    give-up is reported as DORA_ERR_TIMEOUT, and with the default limit restored
    the next call is correct."""
    W0, A, B = _module(1)
    ref = oracle.dense_row_norm(W0.float().numpy(), A.float().numpy(), B.float().numpy(), 2.0)
    Wc, Ac, Bc = W0.cuda(), A.cuda(), B.cuda()
    try:
        dora.dora_set_wait_timeout_ns(1)
        n, _ = dora.dora_factored_norm(Wc, Ac, Bc, 2.0)
        st = dora.dora_get_device_status()
    finally:
        dora.dora_set_wait_timeout_ns(0)
    assert st in (_abi.DORA_OK, _abi.DORA_ERR_TIMEOUT)
    if st == _abi.DORA_OK:
        check_rel(n.cpu().double().numpy(), ref, 1e-3, "n (no give-up)")
    n2, _ = dora.dora_factored_norm(Wc, Ac, Bc, 2.0)
    assert dora.dora_get_device_status() == _abi.DORA_OK
    check_rel(n2.cpu().double().numpy(), ref, 1e-3, "n after restore")


def test_launch_counter_counts_kernels():
    W0, A, B = _module(2)
    before = dora.dora_launch_count()
    dora.dora_factored_norm(W0.cuda(), A.cuda(), B.cuda(), 2.0)
    torch.cuda.synchronize()
    assert dora.dora_launch_count() - before == 2  # counter reset, fused norm kernel (Gram, GEMM, finalize)
