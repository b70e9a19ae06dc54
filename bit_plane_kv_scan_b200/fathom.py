"""ctypes binding of libfathom.so (the C ABI in include/fathom.h).

Argument marshalling only: every step of the scan runs in the library's
CUDA kernels.  PyTorch supplies device memory and the current stream.  There
is no CPU path: if the library is missing or the device is not a CUDA GPU,
calls raise.
"""

from __future__ import annotations

import ctypes
import os
import threading
from typing import List, Optional, Sequence, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# FATHOM_LIB=checked loads the checked build (device bounds checks on every
# plane-row, sample and candidate index; a failed check is a device fault in
# the scan report)
LIB_PATH = os.path.join(_HERE, "libfathom_checked.so" if os.environ.get("FATHOM_LIB") == "checked"
                        else "libfathom.so")

OK = 0
ERR_INVALID_ARGUMENT = 1
ERR_UNSUPPORTED = 2
ERR_WORKSPACE_TOO_SMALL = 3
ERR_CUDA = 4
ERR_DEVICE_CHECK = 5

F32 = 0
BF16 = 1
PLANES_DEVICE = 0
PLANES_HOST_MAPPED = 1
FLAG_NO_SAMPLING = 1
FLAG_FORCE_FALLBACK = 2
FLAG_CUDA_CORES = 4

EXPORTED = [
    "fathom_last_error", "fathom_plane_words", "fathom_planes_bytes", "fathom_pack_planes",
    "fathom_append_planes",
    "fathom_allocate", "fathom_allocate_uniform", "fathom_scan_topk_workspace_size",
    "fathom_scan_topk",
    "fathom_scan_topk_batched_workspace_size", "fathom_scan_topk_batched",
    "fathom_scan_read_report", "fathom_profile_scan_kernel", "fathom_scan_topk_noalloc",
    "fathom_scan_read_report_noalloc", "fathom_check_device_status", "fathom_merge_topk",
    "fathom_sparse_attention",
]
NOALLOC_SCRATCH_BYTES = 16 << 20
TOKEN_GROUP_QUANTUM = 65536
MAX_MERGE_PARTS = 64


class FathomError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__("fathom status %d: %s" % (status, message))
        self.status = status


class ScanArgs(ctypes.Structure):
    _fields_ = [
        ("planes", ctypes.c_void_p), ("planes_location", ctypes.c_int),
        ("qmin", ctypes.c_void_p), ("qscale", ctypes.c_void_p),
        ("q", ctypes.c_void_p), ("q_dtype", ctypes.c_int),
        ("alloc", ctypes.c_void_p), ("n", ctypes.c_int64),
        ("d", ctypes.c_int), ("h_q", ctypes.c_int), ("h_kv", ctypes.c_int), ("k", ctypes.c_int),
        ("out_idx", ctypes.c_void_p), ("out_score", ctypes.c_void_p),
        ("debug_scores", ctypes.c_void_p), ("flags", ctypes.c_uint32),
        ("token_group", ctypes.c_int64),
    ]


class AttentionArgs(ctypes.Structure):
    _fields_ = [
        ("q", ctypes.c_void_p), ("q_dtype", ctypes.c_int),
        ("k_rows", ctypes.c_void_p), ("v_rows", ctypes.c_void_p), ("idx", ctypes.c_void_p),
        ("n", ctypes.c_int64),
        ("d", ctypes.c_int), ("h_q", ctypes.c_int), ("h_kv", ctypes.c_int), ("k", ctypes.c_int),
        ("softmax_scale", ctypes.c_float),
        ("out", ctypes.c_void_p), ("lse", ctypes.c_void_p),
        ("kv_location", ctypes.c_int), ("k_codes", ctypes.c_void_p),
        ("k_qmin", ctypes.c_void_p), ("k_qscale", ctypes.c_void_p),
    ]


class Session(ctypes.Structure):
    _fields_ = [
        ("planes", ctypes.c_void_p), ("qmin", ctypes.c_void_p), ("qscale", ctypes.c_void_p),
        ("q", ctypes.c_void_p), ("alloc", ctypes.c_void_p), ("n", ctypes.c_int64),
        ("out_idx", ctypes.c_void_p), ("out_score", ctypes.c_void_p),
    ]


class BatchedArgs(ctypes.Structure):
    _fields_ = [
        ("sessions", ctypes.c_void_p), ("num_sessions", ctypes.c_int), ("n_max", ctypes.c_int64),
        ("d", ctypes.c_int), ("h_q", ctypes.c_int), ("h_kv", ctypes.c_int), ("k", ctypes.c_int),
        ("q_dtype", ctypes.c_int), ("planes_location", ctypes.c_int), ("flags", ctypes.c_uint32),
    ]


class ScanReport(ctypes.Structure):
    _fields_ = [("fallback_heads", ctypes.c_uint32), ("device_faults", ctypes.c_uint32),
                ("max_candidates", ctypes.c_uint32), ("union_planes", ctypes.c_uint32)]


_lib = None
_lock = threading.Lock()


def lib() -> ctypes.CDLL:
    """Load libfathom.so; raise if it has not been built."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise ImportError("libfathom.so is not built (python -m bit_plane_kv_scan_b200.build)")
        L = ctypes.CDLL(LIB_PATH)
        vp, i64, ci, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
        L.fathom_last_error.restype = ctypes.c_char_p
        L.fathom_last_error.argtypes = []
        L.fathom_plane_words.restype = i64
        L.fathom_plane_words.argtypes = [i64]
        L.fathom_planes_bytes.restype = sz
        L.fathom_planes_bytes.argtypes = [i64, ci, ci]
        L.fathom_pack_planes.restype = ci
        L.fathom_pack_planes.argtypes = [vp, i64, ci, ci, vp, vp]
        L.fathom_allocate.restype = ci
        L.fathom_allocate.argtypes = [vp, ci, vp, ci, ci, ci, ci, vp, vp]
        L.fathom_append_planes.restype = ci
        L.fathom_append_planes.argtypes = [vp, ctypes.c_int64, ctypes.c_int64, ci, ci, vp, vp, vp]
        L.fathom_allocate_uniform.restype = ci
        L.fathom_allocate_uniform.argtypes = [ci, ci, ci, vp, vp]
        L.fathom_sparse_attention.restype = ci
        L.fathom_sparse_attention.argtypes = [ctypes.POINTER(AttentionArgs), vp]
        L.fathom_scan_topk_workspace_size.restype = sz
        L.fathom_scan_topk_workspace_size.argtypes = [ctypes.POINTER(ScanArgs)]
        L.fathom_scan_topk.restype = ci
        L.fathom_scan_topk.argtypes = [ctypes.POINTER(ScanArgs), vp, sz, vp]
        L.fathom_scan_topk_batched_workspace_size.restype = sz
        L.fathom_scan_topk_batched_workspace_size.argtypes = [ctypes.POINTER(BatchedArgs)]
        L.fathom_scan_topk_batched.restype = ci
        L.fathom_scan_topk_batched.argtypes = [ctypes.POINTER(BatchedArgs), vp, sz, vp]
        L.fathom_scan_read_report.restype = ci
        L.fathom_scan_read_report.argtypes = [vp, ctypes.POINTER(ScanReport), vp]
        L.fathom_check_device_status.restype = ci
        L.fathom_check_device_status.argtypes = [vp, vp]
        L.fathom_profile_scan_kernel.restype = None
        L.fathom_profile_scan_kernel.argtypes = [vp, vp]
        L.fathom_scan_topk_noalloc.restype = ci
        L.fathom_scan_topk_noalloc.argtypes = [ctypes.POINTER(ScanArgs), vp]
        L.fathom_merge_topk.restype = ci
        L.fathom_merge_topk.argtypes = [vp, vp, ci, ctypes.POINTER(ctypes.c_int64), ci, ci, ci, vp,
                                        vp, vp]
        L.fathom_scan_read_report_noalloc.restype = ci
        L.fathom_scan_read_report_noalloc.argtypes = [ctypes.POINTER(ScanReport), vp]
        _lib = L
        return L


def _check(status: int):
    if status != OK:
        raise FathomError(status, lib().fathom_last_error().decode())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dtype_code(q: torch.Tensor) -> int:
    if q.dtype == torch.bfloat16:
        return BF16
    if q.dtype == torch.float32:
        return F32
    raise TypeError("q must be bfloat16 or float32, got %s" % q.dtype)


def plane_words(n: int) -> int:
    return int(lib().fathom_plane_words(n))


def pack_planes(codes: torch.Tensor, stream=None) -> torch.Tensor:
    """[h_kv, n, d/2] uint8 codes (CUDA) -> [h_kv, d, 4, W] plane words (int32 storage)."""
    if codes.dtype != torch.uint8 or codes.dim() != 3 or not codes.is_contiguous():
        raise TypeError("codes must be a contiguous uint8 [h_kv, n, d/2] tensor")
    h_kv, n, half = codes.shape
    d = 2 * half
    planes = torch.empty((h_kv, d, 4, plane_words(n)), dtype=torch.int32, device=codes.device)
    _check(lib().fathom_pack_planes(_ptr(codes), n, d, h_kv, _ptr(planes), _stream(stream)))
    return planes


def append_planes(planes: torch.Tensor, n: int, codes_new: torch.Tensor, stream=None) -> torch.Tensor:
    """Add m tokens' codes [h_kv, m, d/2] (uint8, CUDA) to a store of n tokens.

    Returns the store of n + m tokens: `planes` itself, updated in place, when
    the row length does not change, else a new tensor."""
    if codes_new.dtype != torch.uint8 or codes_new.dim() != 3 or not codes_new.is_contiguous():
        raise TypeError("codes_new must be a contiguous uint8 [h_kv, m, d/2] tensor")
    h_kv, m, half = codes_new.shape
    d = 2 * half
    if tuple(planes.shape) != (h_kv, d, 4, plane_words(n)):
        raise ValueError("planes must be [h_kv, d, 4, plane_words(n)]")
    if plane_words(n + m) == plane_words(n):
        out = planes
    else:
        out = torch.empty((h_kv, d, 4, plane_words(n + m)), dtype=torch.int32, device=planes.device)
    _check(lib().fathom_append_planes(_ptr(codes_new) if m else None, int(n), int(m), d, h_kv,
                                      _ptr(planes) if planes.numel() else None, _ptr(out),
                                      _stream(stream)))
    return out


def allocate(q: torch.Tensor, sigma: torch.Tensor, budget: int, stream=None,
             out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """q [h_q, d] (bf16/f32), sigma [h_kv, d] f32 -> bits per channel uint8 [h_q, d]."""
    h_q, d = q.shape
    h_kv = sigma.shape[0]
    if out is None:
        out = torch.empty((h_q, d), dtype=torch.uint8, device=q.device)
    _check(lib().fathom_allocate(_ptr(q.contiguous()), _dtype_code(q), _ptr(sigma.contiguous()),
                                 h_q, h_kv, d, int(budget), _ptr(out), _stream(stream)))
    return out


def allocate_uniform(h_q: int, d: int, budget: int, device=None, stream=None,
                     out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """The query-independent allocation of `budget` bits: uint8 [h_q, d] on `device`."""
    if out is None:
        out = torch.empty((h_q, d), dtype=torch.uint8, device=torch.device(device or "cuda"))
    _check(lib().fathom_allocate_uniform(int(h_q), int(d), int(budget), _ptr(out),
                                         _stream(stream)))
    return out


def sparse_attention(q: torch.Tensor, k_rows: Optional[torch.Tensor], v_rows: torch.Tensor,
                     idx: torch.Tensor, softmax_scale: Optional[float] = None, stream=None,
                     out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None, *,
                     k_codes: Optional[torch.Tensor] = None, k_qmin: Optional[torch.Tensor] = None,
                     k_qscale: Optional[torch.Tensor] = None, host_mapped: bool = False):
    """Attention of each query head over its selected keys only.

    q [h_q, d] (bf16/f32); v_rows [h_kv, n, d] bf16; keys either k_rows
    [h_kv, n, d] bf16 or 4-bit k_codes [h_kv, n, d/2] uint8 with k_qmin,
    k_qscale [h_kv, d] f32 (k = qmin + qscale * code); idx [h_q, k] int32
    (entries outside [0, n) are skipped).  host_mapped: the K and V tensors
    are pinned host memory read across the host link.  Returns (out [h_q, d]
    f32, lse [h_q] f32)."""
    h_q, d = q.shape
    h_kv, n, dv = v_rows.shape
    if v_rows.dtype != torch.bfloat16:
        raise TypeError("v_rows must be bfloat16")
    if k_codes is None:
        if k_rows is None or k_rows.dtype != torch.bfloat16 or k_rows.shape != v_rows.shape:
            raise TypeError("k_rows must be bfloat16 [h_kv, n, d] like v_rows")
    else:
        if k_codes.dtype != torch.uint8 or tuple(k_codes.shape) != (h_kv, n, d // 2):
            raise TypeError("k_codes must be uint8 [h_kv, n, d/2]")
        if k_qmin is None or k_qscale is None:
            raise TypeError("k_codes needs k_qmin and k_qscale")
    if dv != d:
        raise ValueError("v_rows must be [h_kv, n, d] with the query's d")
    if idx.dtype != torch.int32 or idx.dim() != 2 or idx.shape[0] != h_q:
        raise TypeError("idx must be an int32 [h_q, k] tensor")
    if softmax_scale is None:
        softmax_scale = 1.0 / float(d) ** 0.5
    if out is None:
        out = torch.empty((h_q, d), dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty((h_q,), dtype=torch.float32, device=q.device)
    q, idx = q.contiguous(), idx.contiguous()
    a = AttentionArgs(q=_ptr(q), q_dtype=_dtype_code(q),
                      k_rows=None if k_codes is not None else _ptr(k_rows), v_rows=_ptr(v_rows),
                      idx=_ptr(idx), n=n, d=d, h_q=h_q, h_kv=h_kv, k=idx.shape[1],
                      softmax_scale=float(softmax_scale), out=_ptr(out), lse=_ptr(lse),
                      kv_location=PLANES_HOST_MAPPED if host_mapped else PLANES_DEVICE,
                      k_codes=_ptr(k_codes), k_qmin=_ptr(k_qmin), k_qscale=_ptr(k_qscale))
    _check(lib().fathom_sparse_attention(ctypes.byref(a), _stream(stream)))
    return out, lse


class Workspace:
    """A reusable device workspace that grows to the largest request."""

    def __init__(self, device=None):
        self.device = torch.device(device or "cuda")
        self.buf = torch.empty(0, dtype=torch.uint8, device=self.device)

    def get(self, nbytes: int) -> torch.Tensor:
        if self.buf.numel() < nbytes:
            self.buf = torch.empty(nbytes + 256, dtype=torch.uint8, device=self.device)
        off = (-self.buf.data_ptr()) % 256
        return self.buf[off:off + nbytes]


_default_ws = {}


def _workspace(ws: Optional[Workspace], device) -> Workspace:
    if ws is not None:
        return ws
    device = torch.device(device)
    key = device.index if device.index is not None else torch.cuda.current_device()
    if key not in _default_ws:
        _default_ws[key] = Workspace(device)
    return _default_ws[key]


def scan_args(planes, qmin, qscale, q, alloc, k: int, n: int, out_idx, out_score,
              debug_scores=None, flags: int = 0, host_mapped: bool = False,
              token_group: int = 0) -> ScanArgs:
    h_q, d = q.shape
    h_kv = qmin.shape[0]
    return ScanArgs(planes=planes.data_ptr(),
                    planes_location=PLANES_HOST_MAPPED if host_mapped else PLANES_DEVICE,
                    qmin=qmin.data_ptr(), qscale=qscale.data_ptr(), q=q.data_ptr(),
                    q_dtype=_dtype_code(q), alloc=alloc.data_ptr(), n=int(n), d=d, h_q=h_q,
                    h_kv=h_kv, k=int(k), out_idx=out_idx.data_ptr(),
                    out_score=out_score.data_ptr(),
                    debug_scores=None if debug_scores is None else debug_scores.data_ptr(),
                    flags=int(flags), token_group=int(token_group))


def scan_topk(planes: torch.Tensor, qmin: torch.Tensor, qscale: torch.Tensor, q: torch.Tensor,
              alloc: torch.Tensor, k: int, n: int, *, host_mapped: bool = False,
              debug_scores: bool = False, flags: int = 0, workspace: Optional[Workspace] = None,
              stream=None, out: Optional[Tuple[torch.Tensor, torch.Tensor]] = None,
              token_group: int = 0):
    """Top-k keys per query head.  Returns (idx int32 [h_q,k], score f32 [h_q,k]) and,
    with debug_scores=True, also every score f32 [h_q, n].  token_group > 0 (a
    multiple of TOKEN_GROUP_QUANTUM) takes qmin/qscale as [h_kv, groups, d]
    statistics per run of token_group keys."""
    dev = q.device
    h_q = q.shape[0]
    if out is None:
        out = (torch.empty((h_q, k), dtype=torch.int32, device=dev),
               torch.empty((h_q, k), dtype=torch.float32, device=dev))
    dbg = torch.empty((h_q, n), dtype=torch.float32, device=dev) if debug_scores else None
    args = scan_args(planes, qmin, qscale, q, alloc, k, n, out[0], out[1], dbg, flags, host_mapped,
                     token_group)
    L = lib()
    need = L.fathom_scan_topk_workspace_size(ctypes.byref(args))
    if need == 0:
        _check(L.fathom_scan_topk(ctypes.byref(args), None, 0, _stream(stream)))
    ws = _workspace(workspace, dev)
    buf = ws.get(need)
    _check(L.fathom_scan_topk(ctypes.byref(args), _ptr(buf), need, _stream(stream)))
    if debug_scores:
        return out[0], out[1], dbg
    return out


class BatchedScan:
    """A prepared batched scan: the session descriptors are uploaded once, so
    repeated launches over the same buffers (a decode loop whose q and alloc
    are rewritten in place) issue no host-to-device copy of their own.  Each
    session dict holds planes, qmin, qscale, q, alloc, n (and optionally
    out_idx/out_score)."""

    def __init__(self, sessions: Sequence[dict], k: int, d: int, h_q: int, h_kv: int,
                 q_dtype: torch.dtype = torch.bfloat16, *, host_mapped: bool = False,
                 flags: int = 0, device=None):
        device = torch.device(device or sessions[0]["q"].device)
        S = len(sessions)
        arr = (Session * S)()
        self.outs: List[Tuple[torch.Tensor, torch.Tensor]] = []
        n_max = 0
        for i, s in enumerate(sessions):
            oi = s.get("out_idx")
            osc = s.get("out_score")
            if oi is None:
                oi = torch.empty((h_q, k), dtype=torch.int32, device=device)
                osc = torch.empty((h_q, k), dtype=torch.float32, device=device)
            self.outs.append((oi, osc))
            arr[i] = Session(planes=s["planes"].data_ptr(), qmin=s["qmin"].data_ptr(),
                             qscale=s["qscale"].data_ptr(), q=s["q"].data_ptr(),
                             alloc=s["alloc"].data_ptr(), n=int(s["n"]), out_idx=oi.data_ptr(),
                             out_score=osc.data_ptr())
            n_max = max(n_max, int(s["n"]))
        raw = torch.frombuffer(bytearray(bytes(arr)), dtype=torch.uint8)
        self.device = device
        self.desc = raw.to(device, non_blocking=False)
        self.args = BatchedArgs(sessions=self.desc.data_ptr(), num_sessions=S, n_max=n_max, d=d,
                                h_q=h_q, h_kv=h_kv, k=int(k),
                                q_dtype=BF16 if q_dtype == torch.bfloat16 else F32,
                                planes_location=PLANES_HOST_MAPPED if host_mapped
                                else PLANES_DEVICE, flags=int(flags))
        self.need = lib().fathom_scan_topk_batched_workspace_size(ctypes.byref(self.args))
        if self.need == 0:
            _check(lib().fathom_scan_topk_batched(ctypes.byref(self.args), None, 0, None))

    def __call__(self, workspace: Optional[Workspace] = None, stream=None):
        ws = _workspace(workspace, self.device)
        buf = ws.get(self.need)
        _check(lib().fathom_scan_topk_batched(ctypes.byref(self.args), _ptr(buf), self.need,
                                              _stream(stream)))
        # The descriptor tensor lives as long as this object; the workspace
        # also holds it so a one-shot caller may drop the object at once
        # (torch's caching allocator hands its block only to later work
        # ordered after these launches on this stream).
        ws.keepalive = self.desc
        return self.outs


def scan_topk_batched(sessions: Sequence[dict], k: int, d: int, h_q: int, h_kv: int,
                      q_dtype: torch.dtype = torch.bfloat16, *, host_mapped: bool = False,
                      flags: int = 0, workspace: Optional[Workspace] = None, stream=None,
                      device=None):
    """Many sessions in one launch set.  Each session dict holds planes, qmin, qscale, q,
    alloc, n (and optionally out_idx/out_score).  Returns a list of (idx, score)."""
    return BatchedScan(sessions, k, d, h_q, h_kv, q_dtype, host_mapped=host_mapped, flags=flags,
                       device=device)(workspace, stream)


def merge_topk(idx_parts: torch.Tensor, score_parts: torch.Tensor, offsets: Sequence[int], k: int,
               stream=None, out: Optional[Tuple[torch.Tensor, torch.Tensor]] = None):
    """The top-k of token-range shards' top-k lists.

    idx_parts int32 [parts, h_q, k_in] (local indices, -1 padding) and
    score_parts f32 [parts, h_q, k_in], each part sorted as fathom_scan_topk
    returns it; offsets[p] is the first token of part p's range.  Returns
    (idx int32 [h_q, k], score f32 [h_q, k]) with global indices."""
    if idx_parts.dtype != torch.int32 or score_parts.dtype != torch.float32:
        raise TypeError("idx_parts must be int32 and score_parts float32")
    if idx_parts.dim() != 3 or idx_parts.shape != score_parts.shape:
        raise ValueError("idx_parts and score_parts must both be [parts, h_q, k_in]")
    parts, h_q, k_in = idx_parts.shape
    if len(offsets) != parts:
        raise ValueError("one offset per part")
    if out is None:
        out = (torch.empty((h_q, k), dtype=torch.int32, device=idx_parts.device),
               torch.empty((h_q, k), dtype=torch.float32, device=idx_parts.device))
    offs = (ctypes.c_int64 * parts)(*[int(o) for o in offsets])
    ip, sp = idx_parts.contiguous(), score_parts.contiguous()
    _check(lib().fathom_merge_topk(_ptr(ip), _ptr(sp), parts, offs, h_q, k_in, int(k),
                                   _ptr(out[0]), _ptr(out[1]), _stream(stream)))
    return out


def gather_parts(idx: torch.Tensor, score: torch.Tensor, n_local: int, group=None):
    """The collective step of token-range sharding: every rank's top-k lists
    (idx int32 [h_q, k] local indices, score f32 [h_q, k]) and key count go to
    every rank.  Returns (idx_parts [world, h_q, k], score_parts
    [world, h_q, k], offsets) in rank order, offsets[r] being the first token
    of rank r's range (ranks hold consecutive ranges in rank order)."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    n_t = torch.tensor([int(n_local)], dtype=torch.int64, device=idx.device)
    ns = [torch.empty_like(n_t) for _ in range(world)]
    dist.all_gather(ns, n_t, group=group)
    counts = [int(x.item()) for x in ns]
    offsets = [sum(counts[:r]) for r in range(world)]
    idx_l = [torch.empty_like(idx) for _ in range(world)]
    sc_l = [torch.empty_like(score) for _ in range(world)]
    dist.all_gather(idx_l, idx.contiguous(), group=group)
    dist.all_gather(sc_l, score.contiguous(), group=group)
    return torch.stack(idx_l), torch.stack(sc_l), offsets


def sharded_scan_topk(planes: torch.Tensor, qmin: torch.Tensor, qscale: torch.Tensor,
                      q: torch.Tensor, alloc: torch.Tensor, k: int, n_local: int, *,
                      group=None, workspace: Optional[Workspace] = None, stream=None):
    """Token-range sharding over the ranks of a torch.distributed group.

    Every rank holds the planes of its own contiguous range of the context
    (rank order = token order; n_local keys here) and the same q and alloc.
    Each rank scans its range (fathom_scan_topk), one all-gather brings every
    rank's k (index, score) pairs per head to every rank (gather_parts), and
    fathom_merge_topk returns the context's top-k with global indices
    (identical on every rank).  The quantiser statistics (qmin, qscale) are
    the context's, shared by every range."""
    idx, sc = scan_topk(planes, qmin, qscale, q, alloc, k, n_local, workspace=workspace,
                        stream=stream)
    idx_all, sc_all, offsets = gather_parts(idx, sc, n_local, group=group)
    return merge_topk(idx_all, sc_all, offsets, k, stream=stream)


def profile_scan_kernel(begin: Optional[torch.cuda.Event], end: Optional[torch.cuda.Event]):
    """Record begin/end around the filtering scan kernel of later scans (None clears)."""
    if begin is None or end is None:
        lib().fathom_profile_scan_kernel(None, None)
        return
    lib().fathom_profile_scan_kernel(ctypes.c_void_p(begin.cuda_event),
                                     ctypes.c_void_p(end.cuda_event))


def read_report(workspace: Optional[Workspace] = None, device=None, stream=None) -> ScanReport:
    ws = _workspace(workspace, device or "cuda")
    rep = ScanReport()
    _check(lib().fathom_scan_read_report(_ptr(ws.buf[(-ws.buf.data_ptr()) % 256:]),
                                         ctypes.byref(rep), _stream(stream)))
    return rep


def check_device_status(workspace: Optional[Workspace] = None, device=None, stream=None) -> None:
    """Raises FathomError (ERR_DEVICE_CHECK) when the last scan on the
    workspace recorded a device-side fault; synchronises the stream."""
    ws = _workspace(workspace, device or "cuda")
    _check(lib().fathom_check_device_status(_ptr(ws.buf[(-ws.buf.data_ptr()) % 256:]),
                                            _stream(stream)))
