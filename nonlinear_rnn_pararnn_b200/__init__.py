"""Newton-solved diag-mix sLSTM on NVIDIA B200 (sm_100a).

The compute lives in libslstm.so (CUDA, C ABI in include/slstm.h); this
package is its Python binding plus the seeded synthetic workloads.
"""
from .api import (newton_backward, newton_forward, new_stats, preact_gemm, read_stats, scan_block4,
                  sequential_step, workspace, workspace_size)

__all__ = ["newton_backward", "newton_forward", "new_stats", "preact_gemm", "read_stats", "scan_block4",
           "sequential_step", "workspace", "workspace_size"]
