"""B200-native chunkwise gated delta-rule forward (sm_100a).

The compute path is libgdn.so (CUDA, C ABI in include/gdn.h); this package is
its Python binding plus the seeded synthetic workloads used by the tests and
the benchmark.  Build the library with
``python -m chunked_gated_delta_14_b200.build``.
"""
from .gdn import (GDNError, FwdArgs, abi_version, call, chunk_fwd, device_check,  # noqa: F401
                  last_error, lib, make_args, select_kernel, status_string, workspace_bytes,
                  workspace_for)

__all__ = ["chunk_fwd", "device_check", "workspace_bytes", "workspace_for", "GDNError", "FwdArgs", "make_args", "call", "select_kernel",
           "abi_version", "last_error", "status_string", "lib"]
