"""CPU-side checks of the C ABI: the library loads, exports every function
include/dora.h declares, and rejects bad arguments on the host before any
launch.  No compute call runs here (there is no GPU in this suite)."""
import ctypes
import os
import re

import pytest

import dora_adapter_factored_b200 as dora
from dora_adapter_factored_b200 import _abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dora.h")


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b(dora_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_boundary(built_library):
    names = _declared_functions()
    for required in ("dora_factored_norm", "dora_factored_norm_grouped", "dora_compose_fwd",
                     "dora_compose_bwd"):
        assert required in names
    assert sorted(_abi.EXPORTED) == names


def test_library_exports_every_declared_symbol(built_library):
    lib = ctypes.CDLL(built_library)
    for name in _declared_functions():
        assert hasattr(lib, name), name


def test_status_strings_and_version(built_library):
    lib = dora.load_library(built_library)
    for code in range(8):
        assert len(dora.status_string(code)) > 0
    assert dora.status_string(99) == "unknown status"
    assert dora.dora_version() == 100


def test_host_validation_rejects_before_launch(built_library):
    lib = dora.load_library(built_library)
    before = dora.dora_launch_count()
    p = ctypes.c_void_p(0x10000)   # never dereferenced: validation fails first
    # null pointers
    assert lib.dora_factored_norm(None, p, p, _abi.DORA_BF16, 8, 8, 8, 2.0, None, 0.0, p, None,
                                  p, 1 << 20, None) == _abi.DORA_ERR_INVALID_ARG
    # rank above the TMEM limit
    assert lib.dora_factored_norm(p, p, p, _abi.DORA_BF16, 8, 8, 513, 2.0, None, 0.0, p, None,
                                  p, 1 << 20, None) == _abi.DORA_ERR_UNSUPPORTED
    # non-positive sizes
    assert lib.dora_factored_norm(p, p, p, _abi.DORA_BF16, 0, 8, 8, 2.0, None, 0.0, p, None,
                                  p, 1 << 20, None) == _abi.DORA_ERR_INVALID_ARG
    # m without g_out
    assert lib.dora_factored_norm(p, p, p, _abi.DORA_BF16, 8, 8, 8, 2.0, p, 0.0, p, None,
                                  p, 1 << 20, None) == _abi.DORA_ERR_INVALID_ARG
    # bad dtype
    assert lib.dora_factored_norm(p, p, p, 7, 8, 8, 8, 2.0, None, 0.0, p, None,
                                  p, 1 << 20, None) == _abi.DORA_ERR_INVALID_ARG
    # compose: y overlapping lora
    assert lib.dora_compose_fwd(p, ctypes.c_void_p(0x10000), p, p, 2.0, 0.0, _abi.DORA_BF16, 4, 8,
                                ctypes.c_void_p(0x10008), None) == _abi.DORA_ERR_INVALID_ARG
    # compose: negative T
    assert lib.dora_compose_fwd(p, p, p, p, 2.0, 0.0, _abi.DORA_BF16, -1, 8, p,
                                None) == _abi.DORA_ERR_INVALID_ARG
    # backward: d_lora aliasing dy
    assert lib.dora_compose_bwd(p, ctypes.c_void_p(0x20000), ctypes.c_void_p(0x30000), p, p, 2.0,
                                0.0, _abi.DORA_BF16, 4, 8, ctypes.c_void_p(0x40000), p,
                                ctypes.c_void_p(0x50000), p, 1 << 20,
                                None) == _abi.DORA_ERR_INVALID_ARG
    # grouped: too many problems, bad dtype
    arr = (_abi.NormProblem * 1)()
    assert lib.dora_factored_norm_grouped(arr, 0, _abi.DORA_BF16, 0.0, p, 1 << 20,
                                          None) == _abi.DORA_ERR_INVALID_ARG
    assert lib.dora_factored_norm_grouped(arr, 1, _abi.DORA_F32, 0.0, p, 1 << 20,
                                          None) == _abi.DORA_ERR_UNSUPPORTED
    assert dora.dora_launch_count() == before


def test_training_and_grouped_validation(built_library):
    lib = dora.load_library(built_library)
    before = dora.dora_launch_count()
    p = ctypes.c_void_p(0x10000)
    vp = ctypes.c_void_p
    # training forward: inner must be given, and may not overlap y
    assert lib.dora_compose_fwd_train(p, vp(0x20000), p, p, 2.0, 0.0, _abi.DORA_BF16, 4, 8,
                                      vp(0x30000), None, None) == _abi.DORA_ERR_INVALID_ARG
    assert lib.dora_compose_fwd_train(p, vp(0x20000), p, p, 2.0, 0.0, _abi.DORA_BF16, 4, 8,
                                      vp(0x30000), vp(0x30010), None) == _abi.DORA_ERR_INVALID_ARG
    # backward from inner: d_lora aliasing inner; missing dm
    assert lib.dora_compose_bwd_inner(p, vp(0x20000), p, p, 2.0, 0.0, _abi.DORA_BF16, 4, 8,
                                      vp(0x40000), vp(0x20000), vp(0x50000), p, 1 << 20,
                                      None) == _abi.DORA_ERR_INVALID_ARG
    assert lib.dora_compose_bwd_inner(p, vp(0x20000), p, p, 2.0, 0.0, _abi.DORA_BF16, 4, 8,
                                      vp(0x40000), vp(0x60000), None, p, 1 << 20,
                                      None) == _abi.DORA_ERR_INVALID_ARG
    # frozen backward: d_lora aliasing dy
    assert lib.dora_compose_bwd_frozen(p, p, p, 2.0, 0.0, _abi.DORA_BF16, 4, 8, vp(0x40000), p,
                                       None) == _abi.DORA_ERR_INVALID_ARG
    # grouped: a record with dm next to one without (mixed variants)
    arr = (_abi.ComposeProblem * 2)()
    for i in range(2):
        arr[i].dy, arr[i].d_base, arr[i].d_lora = 0x100000 * (i + 1), 0x110000 * (i + 1), \
            0x120000 * (i + 1)
        arr[i].m = arr[i].n = 0x10000
        arr[i].T, arr[i].d_out, arr[i].s = 4, 8, 1.0
    arr[0].dm, arr[0].inner = 0x900000, 0x910000
    assert lib.dora_compose_bwd_grouped(arr, 2, _abi.DORA_BF16, 0.0, p, 1 << 20,
                                        None) == _abi.DORA_ERR_INVALID_ARG
    assert lib.dora_compose_bwd_grouped_workspace_size(arr, 2, _abi.DORA_BF16) == 0
    big = (_abi.ComposeProblem * 65)()
    assert lib.dora_compose_fwd_grouped(big, 65, _abi.DORA_BF16, 0.0,
                                        None) == _abi.DORA_ERR_UNSUPPORTED
    assert lib.dora_compose_fwd_grouped(arr, 0, _abi.DORA_BF16, 0.0,
                                        None) == _abi.DORA_ERR_INVALID_ARG
    assert dora.dora_launch_count() == before


def test_merge_validation(built_library):
    lib = dora.load_library(built_library)
    before = dora.dora_launch_count()
    vp = ctypes.c_void_p
    W0, A, B, m, n, ws = (vp(0x100000), vp(0x200000), vp(0x300000), vp(0x400000),
                          vp(0x500000), vp(0x600000))
    out = vp(0x700000)
    # r not a multiple of 8, d_in not a multiple of 8, rank above the limit
    for d_in, r in ((64, 12), (60, 8), (64, 520)):
        assert lib.dora_merge_weight(W0, A, B, m, n, 2.0, 0.0, 16, d_in, r, out, ws, 1 << 20,
                                     None) == _abi.DORA_ERR_UNSUPPORTED
    # W_out overlapping A; missing workspace; null m
    assert lib.dora_merge_weight(W0, A, B, m, n, 2.0, 0.0, 16, 64, 8, vp(0x200010), ws, 1 << 20,
                                 None) == _abi.DORA_ERR_INVALID_ARG
    assert lib.dora_merge_weight(W0, A, B, m, n, 2.0, 0.0, 16, 64, 8, out, None, 0,
                                 None) == _abi.DORA_ERR_WORKSPACE
    assert lib.dora_merge_weight(W0, A, B, None, n, 2.0, 0.0, 16, 64, 8, out, ws, 1 << 20,
                                 None) == _abi.DORA_ERR_INVALID_ARG
    assert lib.dora_merge_weight_workspace_size(8192, 8192, 384) == 8192 * 384 * 2
    assert lib.dora_merge_weight_workspace_size(8, 8, 600) == 0
    assert dora.dora_launch_count() == before


def torch_cuda_available():
    import torch
    return torch.cuda.is_available()


def test_sharded_norm_validation(built_library):
    lib = dora.load_library(built_library)
    before = dora.dora_launch_count()
    vp = ctypes.c_void_p
    p = vp(0x10000)
    # squared partial: null output, rank above the limit
    assert lib.dora_factored_norm_sq(p, p, p, _abi.DORA_BF16, 8, 8, 8, 2.0, None, p, 1 << 20,
                                     None) == _abi.DORA_ERR_INVALID_ARG
    assert lib.dora_factored_norm_sq(p, p, p, _abi.DORA_BF16, 8, 8, 513, 2.0, vp(0x20000), p,
                                     1 << 20, None) == _abi.DORA_ERR_UNSUPPORTED
    # finalize: m without g_out; g_out overlapping n_out
    assert lib.dora_norm_finalize(p, vp(0x20000), 0.0, 8, vp(0x30000), None,
                                  None) == _abi.DORA_ERR_INVALID_ARG
    assert lib.dora_norm_finalize(p, vp(0x20000), 0.0, 8, vp(0x30000), vp(0x30010),
                                  None) == _abi.DORA_ERR_INVALID_ARG
    assert dora.dora_launch_count() == before
    # neither m nor g_out: valid arguments (the call then needs a device)
    if not torch_cuda_available():
        assert lib.dora_norm_finalize(p, None, 0.0, 8, vp(0x30000), None,
                                      None) == _abi.DORA_ERR_CUDA


def test_grouped_workspace_sizes(built_library):
    lib = dora.load_library(built_library)
    arr = (_abi.ComposeProblem * 3)()
    for i, (T, d) in enumerate([(512, 4096), (512, 1024), (7, 1000)]):
        arr[i].dy = arr[i].base = arr[i].lora = arr[i].d_base = arr[i].d_lora = 0x10000
        arr[i].m = arr[i].n = arr[i].dm = 0x10000
        arr[i].T, arr[i].d_out, arr[i].s = T, d, 1.0
    w = lib.dora_compose_bwd_grouped_workspace_size(arr, 3, _abi.DORA_BF16)
    assert (4096 + 1024 + 1000) * 4 <= w < 64 << 20 and w % 256 == 0
    for i in range(3):
        arr[i].dm = None
    assert lib.dora_compose_bwd_grouped_workspace_size(arr, 3, _abi.DORA_BF16) == 0


def test_workspace_sizes_are_host_computable(built_library):
    lib = dora.load_library(built_library)
    # headline module: G' + Gram partials + norm partials, all modest
    ws = lib.dora_factored_norm_workspace_size(8192, 8192, 384, _abi.DORA_BF16)
    assert 384 * 384 * 2 < ws < 64 << 20
    # fp32 path: the fp32 Gram matrix
    assert lib.dora_factored_norm_workspace_size(64, 48, 8, _abi.DORA_F32) >= 8 * 8 * 4
    assert lib.dora_factored_norm_workspace_size(8, 8, 600, _abi.DORA_BF16) == 0
    # backward partials: chunks x d_out fp32
    wb = lib.dora_compose_bwd_workspace_size(8192, 25600, _abi.DORA_BF16)
    assert 25600 * 4 <= wb < 64 << 20
    assert lib.dora_compose_bwd_workspace_size(0, 16, _abi.DORA_BF16) >= 0
    # the backward's blocks are 32 vectors (256 bf16 columns) wide: at the
    # headline shape 32 column blocks x 9 row chunks fill the 296 block slots,
    # so the workspace holds 9 rows of d_out fp32 partials
    assert lib.dora_compose_bwd_workspace_size(4096, 8192, _abi.DORA_BF16) == 9 * 8192 * 4


def test_binding_rejects_cpu_tensors(built_library):
    import torch
    dora.load_library(built_library)
    x = torch.zeros(4, 8, dtype=torch.bfloat16)
    m = torch.ones(8)
    with pytest.raises(ValueError):
        dora.dora_compose_fwd(x, x, m, m, 2.0)


def test_calls_without_a_device_fail_cleanly(built_library):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    lib = dora.load_library(built_library)
    p = ctypes.c_void_p(0x10000)
    st = lib.dora_compose_fwd(p, ctypes.c_void_p(0x90000), p, p, 2.0, 0.0, _abi.DORA_BF16, 4, 8,
                              ctypes.c_void_p(0x20000), None)
    assert st == _abi.DORA_ERR_CUDA
