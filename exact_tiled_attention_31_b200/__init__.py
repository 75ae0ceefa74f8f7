"""Exact tiled attention for NVIDIA B200 (sm_100a).

The CUDA kernels live in ``libfa.so`` (built from ``csrc/`` by
``exact_tiled_attention_31_b200.build``); ``api`` is a thin ctypes binding
over its C ABI (``include/fa.h``).  ``inputs`` draws the seeded synthetic
tensors used by the tests and the benchmark.
"""
from .api import (  # noqa: F401
    EXPORTS, FAError, backward, backward_noalloc, backward_varlen, check_device_error, decode, fa_bwd,
    fa_bwd_dropout, fa_bwd_finish, fa_bwd_main, fa_bwd_noalloc, fa_bwd_preprocess, fa_bwd_varlen,
    fa_bwd_varlen_workspace_size, fa_bwd_workspace_size, fa_check_device_error, fa_decode, fa_decode_num_splits,
    fa_decode_workspace_size, fa_fwd, fa_fwd_dropout, fa_fwd_varlen, fa_fwd_varlen_dropout, fa_bwd_varlen_dropout, fa_launch_count, fa_selftest_timeout,
    fa_status_string, forward, forward_varlen, load_library,
)
