"""B200 (sm_100a) implementation of the Fathom query-adaptive bit-plane key scan.

The compute path is libfathom.so (hand-written CUDA kernels behind the C ABI
in include/fathom.h); this package is its thin ctypes binding.  Importing the
package loads nothing: the library is loaded on the first call and a missing
library raises.
"""

from .fathom import (  # noqa: F401
    BF16, ERR_CUDA, ERR_DEVICE_CHECK, ERR_INVALID_ARGUMENT, ERR_UNSUPPORTED,
    ERR_WORKSPACE_TOO_SMALL, F32, FLAG_CUDA_CORES, FLAG_FORCE_FALLBACK, FLAG_NO_SAMPLING,
    MAX_MERGE_PARTS, OK, PLANES_DEVICE, PLANES_HOST_MAPPED, TOKEN_GROUP_QUANTUM, BatchedScan,
    FathomError, ScanReport,
    Workspace, allocate, allocate_uniform, append_planes, check_device_status, gather_parts, lib,
    merge_topk,
    pack_planes, plane_words, profile_scan_kernel, read_report, scan_topk, scan_topk_batched,
    sharded_scan_topk, sparse_attention,
)
