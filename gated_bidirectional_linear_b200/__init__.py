"""Gated bidirectional ReLU linear attention on B200 (sm_100a).

The operator runs in libgla.so (CUDA kernels for sm_100a behind a C ABI,
include/gla.h); this package holds its ctypes binding (gla.py), the in-tree
build (build.py) and the seeded synthetic workloads (workloads.py)."""
from .gla import (  # noqa: F401
    GLA_DTYPE_BF16, GLA_DTYPE_F32, GLA_PATH_AUTO, GLA_PATH_SIMT, GLA_PATH_TENSOR, GlaError,
    gla_block_causal_step, gla_block_causal_workspace_size, gla_causal_forward, gla_causal_step,
    gla_causal_workspace_size, gla_forward, gla_forward_debug,
    gla_forward_host, gla_forward_host_arena_size, gla_forward_workspace_size,
    gla_get_device_status, gla_plan, gla_selftest_wait_timeout,
)
