"""Parity of the d_in-sharded norm ("Scaling DoRA ...", section 6) on one GPU:
each column shard's squared partial (dora_factored_norm_sq) against the
oracle's, and the finalized sum of the shards against the oracle's dense row
norm.  On one GPU the sum over shards is a plain tensor sum; the same
function with a one-rank NCCL group runs in a child process to exercise the
all-reduce path end to end."""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import oracle
import dora_adapter_factored_b200 as dora
from dora_adapter_factored_b200 import synth
from tolerances import check_rel

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _np(t):
    return t.detach().double().cpu().numpy()


def _module(d_out, d_in, r, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    W0 = (0.02 * torch.randn(d_out, d_in, generator=g)).to(dtype)
    A = ((torch.rand(r, d_in, generator=g) * 2 - 1) / d_in ** 0.5).to(dtype)
    B = (0.02 * torch.randn(d_out, r, generator=g)).to(dtype)
    return W0, A, B


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("d_out,d_in,r,world", [(512, 1000, 64, 3), (300, 4096, 384, 2),
                                                (129, 512, 24, 4), (64, 200, 8, 8)])
def test_shard_partials_and_finalized_norm(dtype, d_out, d_in, r, world):
    W0, A, B = _module(d_out, d_in, r, dtype, d_out + d_in + r)
    s, eps = 2.0, 2.0 ** -7
    Wn, An, Bn = _np(W0), _np(A), _np(B)
    total = torch.zeros(d_out, device="cuda")
    full_sq = oracle.factored_row_norm_sq(Wn, An, Bn, s)
    for rank in range(world):
        a, b = dora.column_shard(d_in, rank, world)
        if a == b:
            continue
        sq = dora.dora_factored_norm_sq(W0[:, a:b].contiguous().cuda(), A[:, a:b].contiguous().cuda(),
                                        B.cuda(), s)
        ref = oracle.factored_row_norm_sq(Wn[:, a:b], An[:, a:b], Bn, s)
        # a shard's partial can be small next to the whole: hold it to the
        # norm's relative bar taken on the whole squared norm
        err = np.abs(_np(sq) - ref)
        tol = (2e-3 if dtype == torch.bfloat16 else 2e-5) * np.abs(full_sq)
        assert (err <= tol).all(), f"shard {rank}: worst {float(np.max(err / tol)):.3g} of bar"
        total += sq
    m = torch.from_numpy(oracle.dense_row_norm(Wn, An, Bn, s) * 1.01).float().cuda()
    n, g = dora.dora_norm_finalize(total, m, eps)
    torch.cuda.synchronize()
    dense = oracle.dense_row_norm(Wn, An, Bn, s)
    rtol = 1e-3 if dtype == torch.bfloat16 else 1e-5
    check_rel(_np(n), dense, rtol, "n from shards")
    gref, _, _ = oracle.magnitude_scale(_np(m), dense, eps)
    check_rel(_np(g), gref, rtol, "g from shards")


def test_headline_two_shards_sampled_rows():
    w = synth.WORKLOADS["headline_8192_r384"]
    W0, A, B = synth.module_weights(w, device="cuda")
    s = w.modules[0].s
    sq = torch.zeros(8192, device="cuda")
    for rank in range(2):
        a, b = dora.column_shard(8192, rank, 2)
        sq += dora.dora_factored_norm_sq(W0[:, a:b].contiguous(), A[:, a:b].contiguous(), B, s)
    n, _ = dora.dora_norm_finalize(sq)
    torch.cuda.synchronize()
    rows = torch.randperm(8192, generator=torch.Generator().manual_seed(6))[:64].sort().values
    ref = oracle.rows_dense_row_norm(_np(W0[rows.cuda()]), _np(A), _np(B[rows.cuda()]), s)
    check_rel(_np(n)[rows.numpy()], ref, 1e-3, "headline n from two shards")


_CHILD = r"""
import datetime, os, sys, torch, torch.distributed as dist
sys.path.insert(0, sys.argv[1])
import dora_adapter_factored_b200 as dora
torch.cuda.set_device(0)
dist.init_process_group("nccl", init_method="tcp://127.0.0.1:" + sys.argv[2], rank=0,
                        world_size=1, timeout=datetime.timedelta(seconds=60),
                        device_id=torch.device("cuda", 0))
g = torch.Generator(device="cuda").manual_seed(3)
W0 = (0.02 * torch.randn(256, 512, device="cuda", generator=g)).bfloat16()
A = (0.04 * torch.randn(64, 512, device="cuda", generator=g)).bfloat16()
B = (0.02 * torch.randn(256, 64, device="cuda", generator=g)).bfloat16()
m = torch.rand(256, device="cuda", generator=g) + 0.5
n_sh, g_sh = dora.sharded_factored_norm(W0, A, B, 2.0, m, 2.0 ** -7)
n_1, g_1 = dora.dora_factored_norm(W0, A, B, 2.0, m, 2.0 ** -7)
torch.cuda.synchronize()
dist.destroy_process_group()
ok = torch.equal(n_sh, n_1) and torch.equal(g_sh, g_1)
print("SAME" if ok else "DIFF", float((n_sh - n_1).abs().max()))
"""


def test_sharded_norm_through_a_one_rank_nccl_group():
    """One rank holding every column: the all-reduce is an identity, so the
    result equals the single-call norm bit for bit (same kernels, same
    summation order, the square root moved to the finalize)."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    env = dict(os.environ, NCCL_NVLS_ENABLE="0")
    r = subprocess.run([sys.executable, "-c", _CHILD, ROOT, str(port)], capture_output=True,
                       text=True, timeout=240, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    assert "SAME" in r.stdout, r.stdout


def test_row_shards_on_one_gpu():
    """Row sharding: each rank's block of rows is an independent norm call;
    the blocks put together equal the oracle's norm of the whole module."""
    W0, A, B = _module(1000, 512, 64, torch.bfloat16, 41)
    s, parts = 2.0, []
    for rank in range(3):
        a, b = dora.row_shard(1000, rank, 3)
        n, _ = dora.dora_factored_norm(W0[a:b].contiguous().cuda(), A.cuda(),
                                       B[a:b].contiguous().cuda(), s)
        parts.append(n)
    torch.cuda.synchronize()
    ref = oracle.dense_row_norm(_np(W0), _np(A), _np(B), s)
    check_rel(_np(torch.cat(parts)), ref, 1e-3, "n from row shards")
