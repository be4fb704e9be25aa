"""SATA (symmetry-aware Taylor approximation) causal attention for NVIDIA B200.

The compute path is libsata.so (CUDA kernels for sm_100a behind the C ABI in
include/sata.h); this package is its ctypes binding plus seeded synthetic
workloads.  Build the library with ``python -m symmetric_taylor_self_b200.build``.
"""
from .binding import (  # noqa: F401
    EXPORTED, LIB_PATH, SataError, State, decode_step, load, prefill, sata_build_basis,
    sata_decode_step, sata_get_option, sata_num_features, sata_prefill, sata_prefill_ex,
    sata_set_option, sata_set_stream, sata_shutdown, sata_state, sata_state_bytes,
    sata_state_init, sata_sync_status, sata_version, sata_workspace_bytes,
    SATA_OK, SATA_EINVAL, SATA_EUNSUPPORTED, SATA_ECUDA, SATA_ETIMEOUT, SATA_ENOMEM,
    SATA_ERANGE, SATA_EALIGN, SATA_OPT_PREFILL_PATH, SATA_OPT_WAIT_LIMIT, SATA_OPT_TEST_STALL,
    SATA_OPT_TIME_KERNELS, SATA_OPT_DETERMINISTIC, sata_kernel_stats, sata_reset_kernel_stats, sata_decode_step_static,
    sata_prefill_host, sata_backward_workspace_bytes, sata_prefill_backward, prefill_backward,
    attention, sata_state_accumulate, sata_prefill_f32, prefill_f32,
)
