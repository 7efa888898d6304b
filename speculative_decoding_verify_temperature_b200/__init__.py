"""B200-native verify/accept step of speculative decoding.

``spec_verify`` is the Python binding of ``libspecverify.so`` (C ABI in
``include/spec_verify.h``); ``workloads`` makes the seeded synthetic inputs.
"""
from . import workloads  # noqa: F401
from .spec_verify import (  # noqa: F401
    SpecError,
    Workspace,
    lib,
    spec_debug_filter_path,
    spec_debug_wait_budget,
    spec_launch_count,
    spec_profile_events,
    spec_read_device_status,
    spec_verify_chain,
    spec_verify_chain_filtered,
    spec_verify_chain_filtered_lazy,
    spec_verify_chain_lazy,
    spec_verify_chain_vocab_parallel,
    spec_verify_tree_greedy,
    spec_verify_tree_greedy_lazy,
    spec_verify_tree_mss,
    spec_verify_tree_mss_lazy,
    spec_verify_tree_sample,
    spec_verify_tree_sample_filtered,
    spec_verify_tree_sample_filtered_lazy,
    spec_verify_tree_sample_lazy,
    spec_workspace_bytes,
    spec_workspace_init,
)
