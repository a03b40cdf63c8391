"""The fused norm's schedule, checked on the host (no GPU): for single modules
and grouped calls of many sizes and pair counts, every W0 and G unit of every
tile is covered once and every tile's partial slots are distinct, complete
and within the workspace (dora_norm_plan_check in include/dora.h walks the
segments the kernel's roles take).  The GPU parity tests run some of these
schedules; this covers the bookkeeping for shapes and SM counts they do not."""
import random

import pytest

import dora_adapter_factored_b200 as dora
from dora_adapter_factored_b200._abi import DORA_ERR_INVALID_ARG

SINGLE = [
    (8192, 8192, 384),    # headline module
    (8192, 4096, 384),    # its d_in shard
    (25600, 5120, 384),   # MLP up-projection
    (4096, 4096, 64),
    (14336, 4096, 384), (4096, 14336, 384), (1024, 4096, 384),
    (2048, 8192, 512), (8192, 1024, 384), (513, 1000, 96), (1000, 704, 40),
    (64, 48, 8), (300, 136, 16), (1, 8, 8), (257, 64, 8), (100000, 64, 8),
]

LAYER = [(4096, 4096, 384), (1024, 4096, 384), (1024, 4096, 384), (4096, 4096, 384),
         (14336, 4096, 384), (14336, 4096, 384), (4096, 14336, 384)]


@pytest.mark.parametrize("pairs", [74, 37, 16, 3, 1])
@pytest.mark.parametrize("shape", SINGLE)
def test_single_module_schedules(shape, pairs):
    dora.dora_norm_plan_check([shape], pairs=pairs)
    dora.dora_norm_plan_check([shape], grouped=True, pairs=pairs)


@pytest.mark.parametrize("pairs", [74, 20, 5])
def test_layer_stack_schedule(pairs):
    dora.dora_norm_plan_check(LAYER * 8, grouped=True, pairs=pairs)   # 56 modules, 8 waves
    dora.dora_norm_plan_check(LAYER, grouped=True, pairs=pairs)


def test_random_groups():
    rng = random.Random(2024)
    for _ in range(60):
        count = rng.randint(2, 24)
        shapes = [(rng.randint(1, 20000), 8 * rng.randint(1, 2048), 8 * rng.randint(1, 64))
                  for _ in range(count)]
        pairs = rng.choice([74, 74, 50, 9, 2])
        dora.dora_norm_plan_check(shapes, grouped=True, pairs=pairs)


def test_rejects_bad_arguments():
    with pytest.raises(dora.DoraError) as e:
        dora.dora_norm_plan_check([(0, 64, 8)])
    assert e.value.status == DORA_ERR_INVALID_ARG
    with pytest.raises(dora.DoraError):
        dora.dora_norm_plan_check([(64, 64, 8), (64, 64, 8)], grouped=False)
    with pytest.raises(dora.DoraError):
        dora.dora_norm_plan_check([(64, 64, 8)], pairs=0)
