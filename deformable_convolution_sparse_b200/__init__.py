"""B200-native DCNv4 spatial aggregation: forward and backward.

The computation lives in libdcnv4.so (hand-written sm_100a CUDA kernels behind
the C ABI of include/dcnv4.h); this package is its thin Python binding.
``workloads`` holds the seeded synthetic input generators.
"""
from .binding import (  # noqa: F401
    DCNV4_BF16, DCNV4_F16, DCNV4_F32, DCNV4_OK, EXPORTS, LIBRARY_PATH, PLAN_FIELDS, STATUS, STATUS_NAMES,
    DCNv4Error, abi_version, backward, device_status, forward, forward_host, forward_host_noalloc, forward_plan,
    forward_trace, load_library, output_shape, predictor, probe_red_global, probe_red_shared, probe_smem_gather,
    sampling_index, selftest_wait_timeout, strerror, validate,
)
