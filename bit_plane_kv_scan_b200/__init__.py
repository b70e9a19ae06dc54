"""B200 (sm_100a) implementation of the Fathom query-adaptive bit-plane key scan.

The compute path is libfathom.so (hand-written CUDA kernels behind the C ABI
in include/fathom.h); this package is its thin ctypes binding.  Importing the
package loads nothing: the library is loaded on the first call and a missing
library raises.
"""

from .fathom import (  # noqa: F401
    BF16, F32, FLAG_FORCE_FALLBACK, FLAG_NO_SAMPLING, FLAG_CUDA_CORES, PLANES_DEVICE,
    PLANES_HOST_MAPPED, BatchedScan, FathomError, Workspace, allocate, allocate_uniform, lib,
    append_planes, pack_planes,
    plane_words, profile_scan_kernel, read_report, scan_topk, scan_topk_batched,
    sparse_attention,
)
