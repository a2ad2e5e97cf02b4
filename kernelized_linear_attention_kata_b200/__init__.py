"""KATA (Kernelized Linear Attention) causal forward and its gradient for B200 (sm_100a).

The computation lives in libkata.so (CUDA, C ABI in include/kata.h); this
package is its thin Python binding plus the seeded workload generators.
"""

from .api import (alloc_workspace, bwd_chunked, bwd_chunked_workspace_bytes,  # noqa: F401
                  chunked_workspace_bytes, decode_step, fwd_chunked, fwd_quadratic, kata_bwd_chunked,
                  kata_decode_step, kata_fwd_chunked, kata_fwd_chunked_sequential,
                  kata_fwd_quadratic, kata_workspace_status, state_dim)
from ._lib import KataError, lib  # noqa: F401
