"""The DORA_DEBUG build: its kernels check the computed index of their global
stores, skip an out-of-range one and record DORA_ERR_BOUNDS (never a trap).
On the CPU: it builds and exports the same boundary.  On the GPU (a child
process, since a process loads one library): every entry point runs on small
odd shapes, agrees with the oracle and leaves the device status clean."""
import ctypes
import os
import subprocess
import sys

import pytest

import dora_adapter_factored_b200 as dora
from dora_adapter_factored_b200 import _abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_debug_library_exports_the_boundary(built_debug_library):
    lib = ctypes.CDLL(built_debug_library)
    for name in _abi.EXPORTED:
        assert hasattr(lib, name), name
    assert lib.dora_status_string  # loads


_CHILD = r'''
import sys, numpy as np, torch
sys.path.insert(0, sys.argv[1])
import oracle
import dora_adapter_factored_b200 as dora
from dora_adapter_factored_b200 import build as _b
dora.load_library(_b.library_path(debug=True))
torch.manual_seed(0)
dev = torch.device("cuda")
bad = []
def close(got, ref, tol, what):
    got = np.asarray(got, dtype=np.float64); ref = np.asarray(ref, dtype=np.float64)
    err = np.max(np.abs(got - ref) / (np.abs(ref) + 1e-3))
    if not err < tol: bad.append(f"{what}: {err}")
for d_out, d_in, r in ((300, 520, 8), (513, 1096, 72), (777, 4160, 264), (260, 2048, 384)):
    W0 = (0.02 * torch.randn(d_out, d_in)).bfloat16(); A = (torch.rand(r, d_in) - 0.5).bfloat16() / d_in ** 0.5
    B = (0.02 * torch.randn(d_out, r)).bfloat16()
    n, _ = dora.dora_factored_norm(W0.to(dev), A.to(dev), B.to(dev), 2.0)
    torch.cuda.synchronize()
    ref = oracle.factored_row_norm(W0.double().numpy(), A.double().numpy(), B.double().numpy(), 2.0)
    close(n.cpu().numpy(), ref, 1e-3, f"norm {d_out}x{d_in} r{r}")
mods = []
for i, (d_out, d_in, r) in enumerate(((300, 520, 8), (777, 1096, 264))):
    W0 = (0.02 * torch.randn(d_out, d_in)).bfloat16().to(dev); A = ((torch.rand(r, d_in) - 0.5) / d_in ** 0.5).bfloat16().to(dev)
    B = (0.02 * torch.randn(d_out, r)).bfloat16().to(dev)
    mods.append(dict(W0=W0, A=A, B=B, s=1.5, n_out=torch.empty(d_out, device=dev)))
dora.dora_factored_norm_grouped(mods)
torch.cuda.synchronize()
for k, md in enumerate(mods):
    ref = oracle.factored_row_norm(md["W0"].double().cpu().numpy(), md["A"].double().cpu().numpy(), md["B"].double().cpu().numpy(), 1.5)
    close(md["n_out"].cpu().numpy(), ref, 1e-3, f"grouped {k}")
for T, d in ((5, 129), (33, 1000), (17, 4104)):
    base, lora, dy = (torch.randn(T, d).bfloat16() for _ in range(3))
    nn = torch.rand(d) + 0.5; m = nn * 1.01
    y = dora.dora_compose_fwd(base.to(dev), lora.to(dev), m.to(dev), nn.to(dev), 2.0, 2 ** -7)
    dd = dora.dora_compose_fwd_delta(base.to(dev), lora.to(dev), m.to(dev), nn.to(dev), 2.0, 2 ** -7)
    db, dl, dm = dora.dora_compose_bwd(dy.to(dev), base.to(dev), lora.to(dev), m.to(dev), nn.to(dev), 2.0, 2 ** -7)
    torch.cuda.synchronize()
    b, l, g_, mm, n_ = (x.double().numpy() for x in (base, lora, dy, m, nn))
    close(y.double().cpu().numpy(), oracle.compose_fwd(b, l, mm, n_, 2.0, 2 ** -7), 2e-2, f"fwd {T}x{d}")
    close(dd.double().cpu().numpy(), oracle.compose_delta(b, l, mm, n_, 2.0, 2 ** -7), 5e-2, f"delta {T}x{d}")
    rb, rl, rdm = oracle.compose_bwd(g_, b, l, mm, n_, 2.0, 2 ** -7)
    close(dm.cpu().numpy(), rdm, 1e-3 * T, f"dm {T}x{d}")
st = dora.dora_get_device_status()
if st != 0: bad.append(f"device status {st}")
print("BAD" if bad else "OK", bad)
sys.exit(1 if bad else 0)
'''


@pytest.mark.gpu
def test_debug_build_runs_clean_on_odd_shapes(built_debug_library):
    res = subprocess.run([sys.executable, "-c", _CHILD, ROOT], capture_output=True, text=True,
                         timeout=600)
    assert res.returncode == 0, res.stdout + res.stderr
