"""B200-native HARP rotation library: libharp.so (include/harp.h) and its binding."""
from .harp import (  # noqa: F401
    Plan, HarpError, last_kernel, apply_two_sided, workspace_bytes, theta_count, splitmix64, lib,
    off_block_energy, l_diag, inject_wait_timeout, moment_check,
    HARP_OK, HARP_ERR_INVALID_ARG, HARP_ERR_SCHEDULE, HARP_ERR_UNSUPPORTED,
    HARP_ERR_NOT_MATERIALIZED, HARP_ERR_ALLOC, HARP_ERR_CUDA, HARP_ERR_TIMEOUT,
    HARP_ERR_WRONG_DEVICE, HARP_F32, HARP_BF16, HARP_FORWARD, HARP_INVERSE,
)
