"""DoRA linear-layer hot path for NVIDIA B200 (sm_100a).

The computation lives in libdora.so (C ABI in include/dora.h); this package is
its ctypes binding (``_abi``), the in-tree build script (``build``) and the
seeded synthetic-input generators (``synth``).  The library is loaded on first
use, and every entry point raises if it cannot be loaded.
"""
from ._abi import (  # noqa: F401
    DORA_BF16, DORA_F32, DORA_MAX_COMPOSE_GROUP, DORA_MAX_GROUP, DORA_MAX_RANK, ComposeProblem,
    DoraError, EXPORTED, NormProblem,
    dora_compose_bwd, dora_compose_bwd_frozen, dora_compose_bwd_grouped,
    dora_compose_bwd_grouped_workspace_size, dora_compose_bwd_inner, dora_compose_bwd_static,
    dora_compose_bwd_workspace_size, dora_compose_fwd, dora_compose_fwd_grouped,
    dora_compose_fwd_train, dora_compose_fwd_delta, dora_debug_unsignalled_wait, dora_factored_norm,
    dora_factored_norm_grouped, dora_factored_norm_grouped_workspace_size,
    dora_factored_norm_sq, dora_factored_norm_workspace_size, dora_norm_finalize, dora_norm_plan_check,
    dora_get_device_status, dora_launch_count,
    dora_merge_weight, dora_merge_weight_workspace_size, dora_set_timing_events, dora_set_trace_buffer, dora_set_wait_timeout_ns, dora_version,
    load_library, status_string,
)

from .sharded import (  # noqa: F401,E402
    all_gather_rows, column_shard, module_shard, row_shard, sharded_factored_norm,
)

__version__ = "0.1.0"
