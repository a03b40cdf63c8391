"""The C ABI on a non-default stream and captured in a CUDA graph gives the
same bits as on the default stream (all reductions have a fixed order)."""
import os
import subprocess
import sys

import pytest
import torch

import dora_adapter_factored_b200 as dora

pytestmark = pytest.mark.gpu


def _inputs():
    g = torch.Generator().manual_seed(77)
    W0 = (0.02 * torch.randn(640, 1024, generator=g)).bfloat16().cuda()
    A = (0.03 * torch.randn(384, 1024, generator=g)).bfloat16().cuda()
    B = (0.02 * torch.randn(640, 384, generator=g)).bfloat16().cuda()
    m = (1 + 0.01 * torch.randn(640, generator=g)).cuda()
    base = torch.randn(300, 640, generator=g).bfloat16().cuda()
    lora = torch.randn(300, 640, generator=g).bfloat16().cuda()
    dy = torch.randn(300, 640, generator=g).bfloat16().cuda()
    return W0, A, B, m, base, lora, dy


def _path(W0, A, B, m, base, lora, dy, out):
    dora.dora_factored_norm(W0, A, B, 2.0, m, 2.0 ** -7, n_out=out["n"], g_out=out["g"],
                            ws=out["ws"])
    dora.dora_compose_fwd(base, lora, m, out["n"], 2.0, 2.0 ** -7, y=out["y"])
    dora.dora_compose_bwd(dy, base, lora, m, out["n"], 2.0, 2.0 ** -7, d_base=out["db"],
                          d_lora=out["dl"], dm=out["dm"], ws=out["wsb"])


def _outs(W0, base):
    d_out = W0.shape[0]
    return dict(n=torch.empty(d_out, device="cuda"), g=torch.empty(d_out, device="cuda"),
                y=torch.empty_like(base), db=torch.empty_like(base), dl=torch.empty_like(base),
                dm=torch.empty(d_out, device="cuda"),
                ws=torch.empty(dora.dora_factored_norm_workspace_size(d_out, 1024, 384,
                                                                      torch.bfloat16),
                               dtype=torch.uint8, device="cuda"),
                wsb=torch.empty(max(256, dora.dora_compose_bwd_workspace_size(
                    base.shape[0], d_out, torch.bfloat16)), dtype=torch.uint8, device="cuda"))


def test_side_stream_and_graph_match_default_stream():
    ins = _inputs()
    ref = _outs(ins[0], ins[4])
    _path(*ins, ref)
    torch.cuda.synchronize()

    side = _outs(ins[0], ins[4])
    st = torch.cuda.Stream()
    with torch.cuda.stream(st):
        _path(*ins, side)
    torch.cuda.synchronize()

    gr = _outs(ins[0], ins[4])
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        _path(*ins, gr)
    graph.replay()
    graph.replay()
    torch.cuda.synchronize()
    assert dora.dora_get_device_status() == 0
    for k in ("n", "g", "y", "db", "dl", "dm"):
        assert torch.equal(ref[k], side[k]), k
        assert torch.equal(ref[k], gr[k]), k


# A fresh process whose first compose launches happen inside a stream capture:
# the one-time per-kernel setup of the streaming kernels (their L1/shared
# split preference) then runs during the capture, which must neither break
# the capture nor change a bit of the results.
_FIRST_CALL_IN_CAPTURE = r"""
import sys
sys.path.insert(0, sys.argv[1])
import torch
import dora_adapter_factored_b200 as dora
g = torch.Generator().manual_seed(5)
T, d = 300, 640
base, lora, dy = (torch.randn(T, d, generator=g).bfloat16().cuda() for _ in range(3))
m = (1 + 0.01 * torch.randn(d, generator=g)).cuda()
n = (1 + 0.05 * torch.rand(d, generator=g)).cuda()
y, db, dl = (torch.empty_like(base) for _ in range(3))
dm = torch.empty(d, device="cuda")
wsb = torch.empty(max(256, dora.dora_compose_bwd_workspace_size(T, d, torch.bfloat16)),
                  dtype=torch.uint8, device="cuda")
assert dora.dora_launch_count() == 0
graph = torch.cuda.CUDAGraph()
with torch.cuda.graph(graph):
    dora.dora_compose_fwd(base, lora, m, n, 2.0, 2.0 ** -7, y=y)
    dora.dora_compose_bwd(dy, base, lora, m, n, 2.0, 2.0 ** -7, d_base=db, d_lora=dl, dm=dm,
                          ws=wsb)
graph.replay()
torch.cuda.synchronize()
y2 = dora.dora_compose_fwd(base, lora, m, n, 2.0, 2.0 ** -7)
db2, dl2, dm2 = dora.dora_compose_bwd(dy, base, lora, m, n, 2.0, 2.0 ** -7)
torch.cuda.synchronize()
assert dora.dora_get_device_status() == 0
for name, a, b in (("y", y, y2), ("d_base", db, db2), ("d_lora", dl, dl2), ("dm", dm, dm2)):
    assert torch.equal(a, b), name
print("OK")
"""


def test_first_compose_calls_inside_a_capture():
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    res = subprocess.run([sys.executable, "-c", _FIRST_CALL_IN_CAPTURE, root],
                         capture_output=True, text=True, timeout=600)
    assert res.returncode == 0 and "OK" in res.stdout, res.stdout + res.stderr
