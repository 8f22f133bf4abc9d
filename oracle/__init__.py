"""fp64 CPU oracle for exact attention.

TEST INFRASTRUCTURE ONLY: imported by the test-suite, by the package's smoke check and by
the bench's CPU-baseline / reference leg, never by the library's product path.  It shares
no code with the CUDA kernels.  See ``oracle.attention`` for what it computes and which
passage of the source pages each step follows.
"""
from .attention import (  # noqa: F401
    forward, backward, forward_head, backward_head,
    forward_rows, dq_rows, kv_grad_tail, scalar_loop_head, forward_head_block_sparse,
    forward_rows_block_sparse,
)
from . import fp8  # noqa: F401,E402
