"""dora_compose_bwd_static: the compose backward for callers that cannot pass
a workspace (a C host program without a device allocator, or a loop where
cudaMalloc is not allowed because it can synchronise the device).  Its dm
column partials live in the library's fixed device array instead.

The test calls the entry point through the C ABI twice in a row, on
different shapes and dtypes so that the second call reuses the array the
first one wrote, and checks each result against dora_compose_bwd (the
workspace entry point) with the same tolerances as the other parity tests.
It also checks that a shape needing more scratch than the array holds is
rejected before anything runs.  Collected last (file name) so that a run
stopping at the first failure has run every other test first.
"""
import ctypes

import numpy as np
import pytest
import torch

import dora_adapter_factored_b200 as dora
from dora_adapter_factored_b200 import _abi
from tolerances import check_bf16, check_dm, check_f32

pytestmark = pytest.mark.gpu


def _np(t):
    return t.detach().double().cpu().numpy()


def _inputs(T, d_out, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    dy = torch.randn(T, d_out, generator=g).to(dtype).cuda()
    base = torch.randn(T, d_out, generator=g).to(dtype).cuda()
    lora = torch.randn(T, d_out, generator=g).to(dtype).cuda()
    n = torch.empty(d_out).uniform_(0.5, 2.0, generator=g)
    m = (n * (1 + 0.005 * torch.randn(d_out, generator=g))).float()
    return dy, base, lora, m.cuda(), n.float().cuda()


@pytest.mark.parametrize("calls", [[(300, 4096, torch.bfloat16, 1), (1000, 2048, torch.bfloat16, 2),
                                    (77, 264, torch.float32, 3)]])
def test_static_scratch_backward_matches_workspace_backward(calls):
    s, eps = 2.0, 2.0 ** -7
    for T, d_out, dtype, seed in calls:
        dy, base, lora, m, n = _inputs(T, d_out, dtype, seed)
        ref_db, ref_dl, ref_dm = dora.dora_compose_bwd(dy, base, lora, m, n, s, eps)
        got_db, got_dl, got_dm = dora.dora_compose_bwd_static(dy, base, lora, m, n, s, eps)
        torch.cuda.synchronize()
        assert dora.dora_get_device_status() == 0
        chk = check_bf16 if dtype == torch.bfloat16 else check_f32
        chk(_np(got_db), _np(ref_db), np.abs(_np(ref_db)), f"d_base {T}x{d_out}")
        chk(_np(got_dl), _np(ref_dl), np.abs(_np(ref_dl)), f"d_lora {T}x{d_out}")
        d, b, l = _np(dy), _np(base), _np(lora)
        nc = np.maximum(_np(n), eps)
        check_dm(_np(got_dm), _np(ref_dm), np.sum(np.abs(d * (b + s * l)), axis=0) / nc,
                 f"dm {T}x{d_out}")


def test_static_scratch_rejects_shapes_beyond_the_array():
    lib = dora.load_library()
    p = ctypes.c_void_p(0x10000)  # never dereferenced: the size check comes first
    d_out = 1 << 21               # one chunk of 2^21 fp32 partials = 8 MiB > 4 MiB
    st = lib.dora_compose_bwd_static(p, ctypes.c_void_p(0x20000), ctypes.c_void_p(0x30000), p, p,
                                     2.0, 0.0, _abi.DORA_BF16, 64, d_out,
                                     ctypes.c_void_p(0x40000), ctypes.c_void_p(0x50000),
                                     ctypes.c_void_p(0x60000), None)
    assert st == _abi.DORA_ERR_UNSUPPORTED
    assert b"needs" in lib.dora_last_error()
