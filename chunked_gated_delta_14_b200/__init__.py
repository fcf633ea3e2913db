"""B200-native chunkwise gated delta rule, forward and backward (sm_100a).

The compute path is libgdn.so (CUDA, C ABI in include/gdn.h); this package is
its Python binding plus the seeded synthetic workloads used by the tests and
the benchmark.  Build the library with
``python -m chunked_gated_delta_14_b200.build``.
"""
from .gdn import (GDNError, BwdArgs, FwdArgs, GatedDeltaRule, abi_version,  # noqa: F401
                  bwd_workspace_bytes, call, call_bwd, chunk_bwd, chunk_fwd, clear_workspace_cache,
                  debug_chunk_T, device_check,
                  gated_delta_rule, last_error, lib, make_args, make_bwd_args, select_kernel, select_segments,
                  status_string, workspace_bytes, workspace_for)

__all__ = ["chunk_fwd", "chunk_bwd", "gated_delta_rule", "GatedDeltaRule", "BwdArgs",
           "make_bwd_args", "call_bwd", "bwd_workspace_bytes", "device_check", "workspace_bytes", "workspace_for", "GDNError", "FwdArgs", "make_args", "call", "select_kernel", "select_segments",
           "abi_version", "last_error", "status_string", "lib", "debug_chunk_T", "clear_workspace_cache"]
