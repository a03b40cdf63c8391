"""Parity of the grouped compose calls (one launch for the modules of a
layer; "Scaling DoRA ...", section 6) with the fp64 oracle, module by module.

The groups mix shapes (ragged d_out, T = 0, tiny and large modules) and
scales s; the elementwise outputs must also equal the single-module calls
bit for bit (same per-element arithmetic), while dm, whose chunking depends on
the group's grid, is held to the oracle's tolerance and to run-to-run
reproducibility."""
import numpy as np
import pytest
import torch

import oracle
import dora_adapter_factored_b200 as dora
from dora_adapter_factored_b200 import synth
from tolerances import check_bf16, check_dm, check_f32

pytestmark = pytest.mark.gpu


def _np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


# A decoder layer's modules at reduced token counts, plus ragged and empty ones.
LAYER = [(512, 4096, 2.0), (512, 1024, 2.0), (512, 1024, 2.0), (512, 4096, 2.0),
         (512, 14336, 0.5), (512, 14336, 0.5), (512, 4096, 0.5)]
RAGGED = [(7, 1000, 1.0), (0, 64, 2.0), (33, 24, 2.0), (1, 1, 3.0), (300, 264, 0.25),
          (4, 4100, 2.0)]


def _module(T, d_out, s, dtype, seed, dev="cuda"):
    g = torch.Generator().manual_seed(seed)
    t = {k: torch.randn(T, d_out, generator=g).to(dtype).to(dev)
         for k in ("base", "lora", "dy", "inner")}
    n = torch.empty(d_out).uniform_(0.5, 2.0, generator=g)
    m = n * (1 + 0.005 * torch.randn(d_out, generator=g))
    t["m"], t["n"], t["s"] = m.float().to(dev), n.float().to(dev), s
    return t


def _group(spec, dtype, seed):
    return [_module(T, d, s, dtype, seed + 17 * i) for i, (T, d, s) in enumerate(spec)]


def _eps(dtype):
    return synth.eps_for("bf16" if dtype == torch.bfloat16 else "f32")


def _chk(dtype):
    return check_bf16 if dtype == torch.bfloat16 else check_f32


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("spec", [LAYER, RAGGED], ids=["layer", "ragged"])
@pytest.mark.parametrize("with_inner", [False, True])
def test_fwd_grouped(dtype, spec, with_inner):
    mods = _group(spec, dtype, 100)
    eps = _eps(dtype)
    items = []
    for p in mods:
        p["y"] = torch.empty_like(p["base"])
        it = dict(base=p["base"], lora=p["lora"], m=p["m"], n=p["n"], s=p["s"], y=p["y"])
        if with_inner:
            p["inner_out"] = torch.empty_like(p["base"])
            it["inner"] = p["inner_out"]
        items.append(it)
    dora.dora_compose_fwd_grouped(items, eps)
    torch.cuda.synchronize()
    for i, p in enumerate(mods):
        b, l, mm, nn = map(_np, (p["base"], p["lora"], p["m"], p["n"]))
        s = p["s"]
        g, gm1, _ = oracle.magnitude_scale(mm, nn, eps)
        _chk(dtype)(_np(p["y"]), oracle.compose_fwd(b, l, mm, nn, s, eps),
                    np.abs(b) + np.abs(gm1 * b) + np.abs(g * s * l), f"y[{i}]")
        y1 = dora.dora_compose_fwd(p["base"], p["lora"], p["m"], p["n"], s, eps)
        assert torch.equal(y1, p["y"]), f"y[{i}] differs from the single-module call"
        if with_inner:
            _chk(dtype)(_np(p["inner_out"]), oracle.compose_inner(b, l, s),
                        np.abs(b) + np.abs(s * l), f"inner[{i}]")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("spec", [LAYER, RAGGED], ids=["layer", "ragged"])
@pytest.mark.parametrize("mode", ["base_lora", "inner", "frozen"])
def test_bwd_grouped(dtype, spec, mode):
    mods = _group(spec, dtype, 200)
    eps = _eps(dtype)
    items = []
    for p in mods:
        p["d_base"] = torch.empty_like(p["dy"])
        p["d_lora"] = torch.empty_like(p["dy"])
        it = dict(dy=p["dy"], m=p["m"], n=p["n"], s=p["s"], d_base=p["d_base"],
                  d_lora=p["d_lora"])
        if mode != "frozen":
            p["dm"] = torch.empty(p["dy"].shape[1], device="cuda")
            it["dm"] = p["dm"]
            if mode == "inner":
                it["inner"] = p["inner"]
            else:
                it["base"], it["lora"] = p["base"], p["lora"]
        items.append(it)
    dora.dora_compose_bwd_grouped(items, eps)
    torch.cuda.synchronize()
    for i, p in enumerate(mods):
        d, mm, nn = _np(p["dy"]), _np(p["m"]), _np(p["n"])
        s = p["s"]
        rb, rl = oracle.compose_bwd_frozen(d, mm, nn, s, eps)
        _chk(dtype)(_np(p["d_base"]), rb, np.abs(rb), f"d_base[{i}]")
        _chk(dtype)(_np(p["d_lora"]), rl, np.abs(rl), f"d_lora[{i}]")
        db1, dl1 = dora.dora_compose_bwd_frozen(p["dy"], p["m"], p["n"], s, eps)
        assert torch.equal(db1, p["d_base"]) and torch.equal(dl1, p["d_lora"]), i
        if mode == "frozen":
            continue
        _, _, nc = oracle.magnitude_scale(mm, nn, eps)
        if mode == "inner":
            x = _np(p["inner"])
            _, _, rdm = oracle.compose_bwd_from_inner(d, x, mm, nn, s, eps)
        else:
            b, l = _np(p["base"]), _np(p["lora"])
            x = b + s * l
            _, _, rdm = oracle.compose_bwd(d, b, l, mm, nn, s, eps)
        check_dm(_np(p["dm"]), rdm, np.sum(np.abs(d * x), axis=0) / nc, f"dm[{i}]")


def test_bwd_grouped_dm_deterministic():
    mods = _group(LAYER, torch.bfloat16, 300)
    runs = []
    for _ in range(2):
        items = [dict(dy=p["dy"], base=p["base"], lora=p["lora"], m=p["m"], n=p["n"], s=p["s"],
                      d_base=torch.empty_like(p["dy"]), d_lora=torch.empty_like(p["dy"]),
                      dm=torch.empty(p["dy"].shape[1], device="cuda")) for p in mods]
        dora.dora_compose_bwd_grouped(items, 2.0 ** -7)
        runs.append([it["dm"].clone() for it in items])
    torch.cuda.synchronize()
    for a, b in zip(*runs):
        assert torch.equal(a, b)


def test_grouped_rejects_mixed_backward_records():
    mods = _group([(4, 64, 1.0), (4, 64, 1.0)], torch.bfloat16, 400)
    a = dict(dy=mods[0]["dy"], m=mods[0]["m"], n=mods[0]["n"], s=1.0,
             d_base=torch.empty_like(mods[0]["dy"]), d_lora=torch.empty_like(mods[0]["dy"]),
             dm=torch.empty(64, device="cuda"), inner=mods[0]["inner"])
    b = dict(dy=mods[1]["dy"], m=mods[1]["m"], n=mods[1]["n"], s=1.0,
             d_base=torch.empty_like(mods[1]["dy"]), d_lora=torch.empty_like(mods[1]["dy"]))
    with pytest.raises(dora.DoraError):
        dora.dora_compose_bwd_grouped([a, b], 2.0 ** -7)
