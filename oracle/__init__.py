"""fp64 CPU oracle for the chunked gated delta rule -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never does, and this
package imports nothing from it: the two share no code.

Contents
--------
``recurrent``   token-by-token recurrences in plain C (fp64), and the
                adjoint of the gated delta rule for its gradients, loaded
                with ctypes from ``libgdn_oracle.so`` (compiled from
                ``gdn_oracle.c`` with gcc on first use).
``chunk_forms`` the intra-chunk pieces the pages define (the triangular
                inverse, the truncated Neumann series, the structural mask,
                the parallel residual correction) and a plain fp64 chunked
                forward that takes the inverse as a parameter, written with
                numpy.
``chunk_grad``  the gradient of the chunked form with the masked truncated
                Neumann inverse, and with its residual correction: the chunk
                model written in plain fp64 PyTorch ops, differentiated by
                autograd.
"""
from . import chunk_forms, chunk_grad, recurrent  # noqa: F401
from .recurrent import gated_delta_bwd, gated_delta_fwd, precond_two_gate_fwd  # noqa: F401
