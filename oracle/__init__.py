"""CPU oracle for the Fathom key scan -- TEST INFRASTRUCTURE, not the product.

A ctypes wrapper over ``fathom_oracle.c``: a plain, slow, single-threaded fp64
statement of the scan (bit-plane packing, reverse water-filling allocation,
plane-prefix scores, brute-force top-k), written from the Fathom pages
("Fathom Makes KV-Cache Scans Query-Adaptive for Long-Context Decoding",
method paragraphs 2-3; arXiv 2609.17652 abstract).  Only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline / reference leg
import it.  It imports nothing from the CUDA library and the library imports
nothing from it.

Every function is pinned in ``tests/test_oracle_pins.py``.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fathom_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

_u8p = np.ctypeslib.ndpointer(dtype=np.uint8, flags="C_CONTIGUOUS")
_u32p = np.ctypeslib.ndpointer(dtype=np.uint32, flags="C_CONTIGUOUS")
_i32p = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")
_i64p = np.ctypeslib.ndpointer(dtype=np.int64, flags="C_CONTIGUOUS")
_f32p = np.ctypeslib.ndpointer(dtype=np.float32, flags="C_CONTIGUOUS")
_f64p = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")
_i64 = ctypes.c_int64
_int = ctypes.c_int


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain -O2, no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB_PATH) or \
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-std=c99",
                               "-fno-fast-math", "-ffp-contract=off", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        lib.oracle_plane_words.restype = _i64
        lib.oracle_plane_words.argtypes = [_i64]
        lib.oracle_pack_planes.restype = None
        lib.oracle_pack_planes.argtypes = [_u8p, _i64, _int, _int, _u32p]
        lib.oracle_prefix_values.restype = None
        lib.oracle_prefix_values.argtypes = [_u32p, _i64, _int, _int, _int, _u8p]
        lib.oracle_importance.restype = ctypes.c_double
        lib.oracle_importance.argtypes = [ctypes.c_double, ctypes.c_double]
        lib.oracle_allocate.restype = None
        lib.oracle_allocate.argtypes = [_f64p, _f64p, _int, _int, _u8p]
        lib.oracle_dequant_prefix.restype = ctypes.c_double
        lib.oracle_dequant_prefix.argtypes = [ctypes.c_double, ctypes.c_double, _int, ctypes.c_uint]
        lib.oracle_scores_from_codes.restype = None
        lib.oracle_scores_from_codes.argtypes = [_u8p, _i64, _int, _f32p, _f32p, _f64p, _u8p, _f64p]
        lib.oracle_scores_at.restype = None
        lib.oracle_scores_at.argtypes = [_u8p, _i64, _int, _f32p, _f32p, _f64p, _u8p, _i64p,
                                         _i64, _f64p]
        lib.oracle_scores_from_planes.restype = None
        lib.oracle_scores_from_planes.argtypes = [_u32p, _i64, _int, _f32p, _f32p, _f64p, _u8p,
                                                  _f64p]
        lib.oracle_topk.restype = None
        lib.oracle_topk.argtypes = [_f64p, _i64, _int, _i32p, _f64p]
        _lib = lib
        return lib


def _c(a, dtype):
    return np.ascontiguousarray(np.asarray(a), dtype=dtype)


def plane_words(n: int) -> int:
    return int(_load().oracle_plane_words(n))


def pack_planes(codes) -> np.ndarray:
    """[h_kv, n, d/2] nibble codes -> [h_kv, d, 4, W] uint32 plane words."""
    codes = _c(codes, np.uint8)
    h_kv, n, half = codes.shape
    d = 2 * half
    out = np.zeros((h_kv, d, 4, plane_words(n)), dtype=np.uint32)
    _load().oracle_pack_planes(codes, n, d, h_kv, out)
    return out


def prefix_values(planes, n: int, t: int) -> np.ndarray:
    """Value of the first t planes of every (KV head, token, channel): [h_kv, n, d]."""
    planes = _c(planes, np.uint32)
    h_kv, d = planes.shape[0], planes.shape[1]
    out = np.zeros((h_kv, n, d), dtype=np.uint8)
    _load().oracle_prefix_values(planes, n, d, h_kv, t, out)
    return out


def importance(q: float, sigma: float) -> float:
    return float(_load().oracle_importance(float(q), float(sigma)))


def allocate(q, sigma, budget: int) -> np.ndarray:
    """One query head: bits per channel, uint8 [d]."""
    q = _c(q, np.float64)
    sigma = _c(sigma, np.float64)
    t = np.zeros(q.shape[0], dtype=np.uint8)
    _load().oracle_allocate(q, sigma, q.shape[0], int(budget), t)
    return t


def allocate_heads(q, sigma, budget: int) -> np.ndarray:
    """All query heads: q [h_q, d], sigma [h_kv, d] (head h reads KV head h // G)."""
    q = np.asarray(q, dtype=np.float64)
    sigma = np.asarray(sigma, dtype=np.float64)
    G = q.shape[0] // sigma.shape[0]
    return np.stack([allocate(q[h], sigma[h // G], budget) for h in range(q.shape[0])])


def allocate_uniform(h_q: int, d: int, budget: int) -> np.ndarray:
    """The query-independent read of `budget` bits per key (the fixed-depth
    read the pages compare the adaptive one with): every channel takes
    budget // d planes and the first budget % d channels one more; the same
    row for every head.  uint8 [h_q, d]."""
    base, extra = divmod(int(budget), int(d))
    row = np.full(int(d), base, dtype=np.uint8)
    row[:extra] += 1
    return np.tile(row, (int(h_q), 1))


def dequant_prefix(m: float, s: float, t: int, v: int) -> float:
    return float(_load().oracle_dequant_prefix(float(m), float(s), int(t), int(v)))


def scores_from_codes(codes_g, qmin_g, qscale_g, q_h, t_h) -> np.ndarray:
    codes_g = _c(codes_g, np.uint8)
    n, half = codes_g.shape
    out = np.zeros(n, dtype=np.float64)
    _load().oracle_scores_from_codes(codes_g, n, 2 * half, _c(qmin_g, np.float32),
                                     _c(qscale_g, np.float32), _c(q_h, np.float64),
                                     _c(t_h, np.uint8), out)
    return out


def scores_at(codes_g, qmin_g, qscale_g, q_h, t_h, idx) -> np.ndarray:
    codes_g = _c(codes_g, np.uint8)
    n, half = codes_g.shape
    idx = _c(idx, np.int64)
    out = np.zeros(idx.shape[0], dtype=np.float64)
    _load().oracle_scores_at(codes_g, n, 2 * half, _c(qmin_g, np.float32),
                             _c(qscale_g, np.float32), _c(q_h, np.float64), _c(t_h, np.uint8),
                             idx, idx.shape[0], out)
    return out


def _group_rows(qmin_g, qscale_g, n: int, token_group: int):
    qmin_g = np.asarray(qmin_g, dtype=np.float32)
    qscale_g = np.asarray(qscale_g, dtype=np.float32)
    groups = (n + token_group - 1) // token_group
    if token_group <= 0 or qmin_g.ndim != 2 or qmin_g.shape[0] < groups or \
            qscale_g.shape != qmin_g.shape:
        raise ValueError("per-group statistics must be [ceil(n / token_group), d]")
    return qmin_g, qscale_g, groups


def scores_from_codes_grouped(codes_g, qmin_g, qscale_g, q_h, t_h, token_group: int) -> np.ndarray:
    """Scores under per-token-group quantiser statistics (the quantiser variant
    with one (m, s) per channel and run of token_group tokens; the pages give
    no group size).  Key i dequantises with row i // token_group of qmin_g and
    qscale_g ([groups][d]); so each group is scored exactly as a context of its
    own by scores_from_codes."""
    codes_g = np.asarray(codes_g)
    n = codes_g.shape[0]
    qmin_g, qscale_g, groups = _group_rows(qmin_g, qscale_g, n, token_group)
    out = np.zeros(n, dtype=np.float64)
    for j in range(groups):
        t0, t1 = j * token_group, min(n, (j + 1) * token_group)
        out[t0:t1] = scores_from_codes(codes_g[t0:t1], qmin_g[j], qscale_g[j], q_h, t_h)
    return out


def scores_at_grouped(codes_g, qmin_g, qscale_g, q_h, t_h, idx, token_group: int) -> np.ndarray:
    """scores_from_codes_grouped at the listed keys only."""
    codes_g = np.asarray(codes_g)
    n = codes_g.shape[0]
    qmin_g, qscale_g, groups = _group_rows(qmin_g, qscale_g, n, token_group)
    idx = np.asarray(idx, dtype=np.int64)
    out = np.zeros(idx.shape[0], dtype=np.float64)
    for j in range(groups):
        sel = np.nonzero(idx // token_group == j)[0]
        if sel.size:
            t0, t1 = j * token_group, min(n, (j + 1) * token_group)
            out[sel] = scores_at(codes_g[t0:t1], qmin_g[j], qscale_g[j], q_h, t_h, idx[sel] - t0)
    return out


def scores_from_planes(planes_g, n: int, qmin_g, qscale_g, q_h, t_h) -> np.ndarray:
    planes_g = _c(planes_g, np.uint32)
    d = planes_g.shape[0]
    out = np.zeros(n, dtype=np.float64)
    _load().oracle_scores_from_planes(planes_g, n, d, _c(qmin_g, np.float32),
                                      _c(qscale_g, np.float32), _c(q_h, np.float64),
                                      _c(t_h, np.uint8), out)
    return out


def topk(scores, k: int):
    """(index int32 [k], score float64 [k]) by score desc, index asc; pads with -1/-inf."""
    scores = _c(scores, np.float64)
    idx = np.zeros(k, dtype=np.int32)
    val = np.zeros(k, dtype=np.float64)
    _load().oracle_topk(scores, scores.shape[0], int(k), idx, val)
    return idx, val


def scan_step(codes, qmin, qscale, q, sigma, budget: int, k: int, heads=None):
    """One decode step for the listed query heads (default: all).

    Returns dict(alloc=[h_q, d] uint8, idx={h: int32[k]}, score={h: float64[k]},
    scores={h: float64[n]}).
    """
    codes = np.asarray(codes)
    q = np.asarray(q, dtype=np.float64)
    h_q = q.shape[0]
    h_kv = codes.shape[0]
    G = h_q // h_kv
    alloc = allocate_heads(q, sigma, budget)
    heads = range(h_q) if heads is None else heads
    res = dict(alloc=alloc, idx={}, score={}, scores={})
    for h in heads:
        g = h // G
        s = scores_from_codes(codes[g], qmin[g], qscale[g], q[h], alloc[h])
        i, v = topk(s, k)
        res["idx"][h] = i
        res["score"][h] = v
        res["scores"][h] = s
    return res


def sparse_attention(q, k_rows, v_rows, idx, scale: float):
    """Attention of each query head over its selected keys only (the step
    after the scan: only the few KV rows that win are fetched, method
    paragraph 1), by its definition in fp64:
        s_r = scale * <q_h, K[g][idx_r]>,  w = softmax(s),  o_h = sum_r w_r V[g][idx_r],
        lse_h = log sum_r exp(s_r),
    over the entries of head h's row that name a key, 0 <= idx_r < n (head h
    reads KV head h // G); other entries (the scan's -1 padding, anything at
    or past n) select nothing.
    q [h_q, d]; k_rows, v_rows [h_kv, n, d]; idx [h_q, k] int.
    Returns (o float64 [h_q, d], lse float64 [h_q]); a head with no selected
    key gets o = 0 and lse = -inf."""
    q = np.asarray(q, dtype=np.float64)
    k_rows = np.asarray(k_rows, dtype=np.float64)
    v_rows = np.asarray(v_rows, dtype=np.float64)
    idx = np.asarray(idx)
    h_q, d = q.shape
    G = h_q // k_rows.shape[0]
    n = k_rows.shape[1]
    out = np.zeros((h_q, d))
    lse = np.full(h_q, -np.inf)
    for h in range(h_q):
        sel = idx[h][(idx[h] >= 0) & (idx[h] < n)].astype(np.int64)
        if sel.size == 0:
            continue
        g = h // G
        s = (k_rows[g][sel] @ q[h]) * float(scale)
        m = s.max()
        w = np.exp(s - m)
        out[h] = (w @ v_rows[g][sel]) / w.sum()
        lse[h] = m + np.log(w.sum())
    return out, lse
