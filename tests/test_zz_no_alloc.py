"""dora_compose_bwd_static: the compose backward for callers that cannot pass
a workspace (a C host program without a device allocator, or a loop where
cudaMalloc is not allowed because it can synchronise the device).  Its dm
column partials live in the library's fixed device array instead.

The tests call the entry point through the C ABI several times in a row, on
different shapes and dtypes so that each call reuses the array the one before
wrote, and check every result against the fp64 oracle (the bars of the other
parity tests) and against dora_compose_bwd (the workspace entry point).  The
sequence includes T = 0, and a shape whose partial table is exactly as large
as the array right after a call that used more row chunks (so a stale row
would show).  A shape needing more scratch than the array holds is rejected
before anything runs.  Collected last (file name) so that a run stopping at
the first failure has run every other test first.
"""
import ctypes
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import oracle
import dora_adapter_factored_b200 as dora
from dora_adapter_factored_b200 import _abi
from tolerances import check_bf16, check_dm, check_f32

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SCRATCH_BYTES = 4 << 20  # the array's size, as include/dora.h states it


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


def _check_against_oracle_and_workspace_call(T, d_out, dtype, seed, s=2.0, eps=2.0 ** -7):
    dy, base, lora, m, n = _inputs(T, d_out, dtype, seed)
    got_db, got_dl, got_dm = dora.dora_compose_bwd_static(dy, base, lora, m, n, s, eps)
    ws_db, ws_dl, ws_dm = dora.dora_compose_bwd(dy, base, lora, m, n, s, eps)
    torch.cuda.synchronize()
    assert dora.dora_get_device_status() == 0
    d, b, l = _np(dy), _np(base), _np(lora)
    mm, nn = _np(m), _np(n)
    r_db, r_dl, r_dm = oracle.compose_bwd(d, b, l, mm, nn, s, eps)
    nc = np.maximum(nn, eps)
    chk = check_bf16 if dtype == torch.bfloat16 else check_f32
    what = f"{T}x{d_out} {dtype}"
    chk(_np(got_db), r_db, np.abs(r_db), f"d_base {what}")
    chk(_np(got_dl), r_dl, np.abs(r_dl), f"d_lora {what}")
    scale = np.sum(np.abs(d * (b + s * l)), axis=0) / nc
    check_dm(_np(got_dm), r_dm, scale, f"dm {what}")
    # The same computation as the workspace call, on the same inputs.
    chk(_np(got_db), _np(ws_db), np.abs(_np(ws_db)), f"d_base vs workspace call {what}")
    chk(_np(got_dl), _np(ws_dl), np.abs(_np(ws_dl)), f"d_lora vs workspace call {what}")
    check_dm(_np(got_dm), _np(ws_dm), scale, f"dm vs workspace call {what}")
    if T == 0:
        assert torch.count_nonzero(got_dm) == 0


def test_static_scratch_backward_matches_oracle_on_consecutive_calls():
    # [4096, 1024] bf16 uses many row chunks; [8, 2^20] bf16 then needs
    # exactly the whole array (one chunk of 2^20 fp32 partials); T = 0 and a
    # ragged fp32 shape follow.
    limit = (8, 1 << 20, torch.bfloat16)
    assert dora.dora_compose_bwd_workspace_size(limit[0], limit[1], limit[2]) == SCRATCH_BYTES
    assert dora.dora_compose_bwd_workspace_size(4096, 1024, torch.bfloat16) < SCRATCH_BYTES
    calls = [(300, 4096, torch.bfloat16, 1), (4096, 1024, torch.bfloat16, 2),
             (*limit, 3), (0, 4096, torch.bfloat16, 4), (1000, 2048, torch.bfloat16, 5),
             (77, 264, torch.float32, 6)]
    for T, d_out, dtype, seed in calls:
        _check_against_oracle_and_workspace_call(T, d_out, dtype, seed)


def test_static_scratch_rejects_shapes_beyond_the_array():
    lib = dora.load_library()
    p = ctypes.c_void_p(0x10000)  # never dereferenced: the size check comes first
    for T, d_out in ((8, (1 << 20) + 8), (64, 1 << 21)):
        assert dora.dora_compose_bwd_workspace_size(T, d_out, torch.bfloat16) > SCRATCH_BYTES
        st = lib.dora_compose_bwd_static(p, ctypes.c_void_p(0x20000), ctypes.c_void_p(0x30000),
                                         p, p, 2.0, 0.0, _abi.DORA_BF16, T, d_out,
                                         ctypes.c_void_p(0x40000), ctypes.c_void_p(0x50000),
                                         ctypes.c_void_p(0x60000), None)
        assert st == _abi.DORA_ERR_UNSUPPORTED
        assert b"needs" in lib.dora_last_error()
