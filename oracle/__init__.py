"""Oracle for exact scaled-dot-product attention: ctypes wrapper over oracle.c.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The library path
(``exact_io_aware_94_b200``) never imports it and has no CPU fallback.

Every routine works in double precision on the plain definition of attention
(see the header of ``oracle.c`` for the page sections each one follows).
Inputs may be torch CPU bfloat16 tensors (read as their exact bit patterns) or
float64 numpy arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

F64 = 0
BF16 = 1

_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (gcc, OpenMP, -O2)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + ".tmp%d" % os.getpid()
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall", _SRC, "-o", tmp, "-lm"]
        )
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        i64, vp, dp, c_int = ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int
        lib.oracle_permitted_keys.restype = i64
        lib.oracle_permitted_keys.argtypes = [i64, i64, i64, c_int]
        lib.oracle_score_elements.restype = i64
        lib.oracle_score_elements.argtypes = [i64, i64, i64, i64]
        lib.oracle_forward.restype = None
        lib.oracle_forward.argtypes = [vp, vp, vp, c_int, dp, dp, i64, i64, i64, i64, i64, ctypes.c_double, c_int]
        lib.oracle_forward_rows.restype = None
        lib.oracle_forward_rows.argtypes = [vp, vp, vp, c_int, vp, i64, dp, dp, i64, i64, i64, i64, i64,
                                            ctypes.c_double, c_int]
        lib.oracle_forward_blockwise.restype = None
        lib.oracle_forward_blockwise.argtypes = [vp, vp, vp, c_int, dp, dp, i64, i64, i64, i64, i64,
                                                 ctypes.c_double, c_int, i64]
        lib.oracle_backward.restype = None
        lib.oracle_backward.argtypes = [vp, vp, vp, vp, c_int, dp, dp, dp, dp, i64, i64, i64, i64, i64,
                                        ctypes.c_double, c_int]
        lib.oracle_decode.restype = None
        lib.oracle_decode.argtypes = [vp, vp, vp, c_int, vp, dp, dp, i64, i64, i64, i64, ctypes.c_double]
        lib.oracle_forward_varlen.restype = None
        lib.oracle_forward_varlen.argtypes = [vp, vp, vp, c_int, dp, dp, vp, vp, i64, i64, i64, i64, ctypes.c_double,
                                              c_int]
        lib.oracle_decode_paged.restype = c_int
        lib.oracle_decode_paged.argtypes = [vp, vp, vp, c_int, vp, vp, dp, dp, i64, i64, i64, i64, i64, i64, i64,
                                            ctypes.c_double]
        lib.oracle_merge.restype = None
        lib.oracle_forward_blocksparse.argtypes = [vp, vp, vp, c_int, dp, dp, vp, i64, i64, i64, i64, i64, i64,
                                                   i64, i64, i64, ctypes.c_double, c_int]
        lib.oracle_merge.argtypes = [dp, dp, i64, i64, dp, dp]
        lib.oracle_num_threads.restype = c_int
        lib.oracle_num_threads.argtypes = []
        lib.oracle_set_num_threads.restype = None
        lib.oracle_set_num_threads.argtypes = [c_int]
        _lib = lib
    return _lib


def _as_input(x):
    """Return (keepalive, pointer, dtype code) for a tensor/array input.

    torch bfloat16 CPU tensors are passed as their bit patterns; anything else
    is converted to a contiguous float64 numpy array.
    """
    try:
        import torch

        if isinstance(x, torch.Tensor):
            if x.dtype == torch.bfloat16:
                t = x.detach().cpu().contiguous()
                return t, t.data_ptr(), BF16
            a = np.ascontiguousarray(x.detach().cpu().double().numpy())
            return a, a.ctypes.data, F64
    except ImportError:  # pragma: no cover - torch is always present here
        pass
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    return a, a.ctypes.data, F64


def _same_kind(*codes):
    if len(set(codes)) != 1:
        raise TypeError("oracle inputs must all be bfloat16 tensors or all be float arrays")
    return codes[0]


def permitted_keys(i: int, Lq: int, Lk: int, causal: bool) -> int:
    return int(_load().oracle_permitted_keys(i, Lq, Lk, int(causal)))


def score_elements(B: int, H: int, Lq: int, Lk: int) -> int:
    return int(_load().oracle_score_elements(B, H, Lq, Lk))


def forward(q, k, v, scale: float, causal: bool):
    """O [B,H,Lq,d] and LSE [B,H,Lq] (float64 numpy) by the two-pass definition."""
    B, H, Lq, d = q.shape
    Lk = k.shape[2]
    kq, pq, cq = _as_input(q)
    kk, pk, ck = _as_input(k)
    kv, pv, cv = _as_input(v)
    dt = _same_kind(cq, ck, cv)
    o = np.empty((B, H, Lq, d), np.float64)
    lse = np.empty((B, H, Lq), np.float64)
    _load().oracle_forward(pq, pk, pv, dt, o.ctypes.data, lse.ctypes.data, B, H, Lq, Lk, d, float(scale),
                           int(causal))
    return o, lse


def forward_rows(q, k, v, rows, scale: float, causal: bool):
    """Forward on flat row indices ``rows`` ((b*H+h)*Lq + i); returns O [n,d], LSE [n]."""
    B, H, Lq, d = q.shape
    Lk = k.shape[2]
    kq, pq, cq = _as_input(q)
    kk, pk, ck = _as_input(k)
    kv, pv, cv = _as_input(v)
    dt = _same_kind(cq, ck, cv)
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    if r.size and (r.min() < 0 or r.max() >= B * H * Lq):
        raise IndexError("row index out of range")
    o = np.empty((r.size, d), np.float64)
    lse = np.empty((r.size,), np.float64)
    _load().oracle_forward_rows(pq, pk, pv, dt, r.ctypes.data, r.size, o.ctypes.data, lse.ctypes.data, B, H,
                                Lq, Lk, d, float(scale), int(causal))
    return o, lse


def forward_blockwise(q, k, v, scale: float, causal: bool, block: int):
    """The running-statistics recurrence over key blocks of size ``block``."""
    B, H, Lq, d = q.shape
    Lk = k.shape[2]
    if block < 1:
        raise ValueError("block must be >= 1")
    kq, pq, cq = _as_input(q)
    kk, pk, ck = _as_input(k)
    kv, pv, cv = _as_input(v)
    dt = _same_kind(cq, ck, cv)
    o = np.empty((B, H, Lq, d), np.float64)
    lse = np.empty((B, H, Lq), np.float64)
    _load().oracle_forward_blockwise(pq, pk, pv, dt, o.ctypes.data, lse.ctypes.data, B, H, Lq, Lk, d,
                                     float(scale), int(causal), int(block))
    return o, lse


def backward(q, k, v, dO, scale: float, causal: bool):
    """dQ, dK, dV (float64, shapes of q, k, v) and D [B,H,Lq] by the naive backward."""
    B, H, Lq, d = q.shape
    Lk = k.shape[2]
    kq, pq, cq = _as_input(q)
    kk, pk, ck = _as_input(k)
    kv, pv, cv = _as_input(v)
    kg, pg, cg = _as_input(dO)
    dt = _same_kind(cq, ck, cv, cg)
    dq = np.empty((B, H, Lq, d), np.float64)
    dk = np.empty((B, H, Lk, d), np.float64)
    dv = np.empty((B, H, Lk, d), np.float64)
    D = np.empty((B, H, Lq), np.float64)
    _load().oracle_backward(pq, pk, pv, pg, dt, dq.ctypes.data, dk.ctypes.data, dv.ctypes.data, D.ctypes.data,
                            B, H, Lq, Lk, d, float(scale), int(causal))
    return dq, dk, dv, D


def decode(q, kcache, vcache, kv_lens, scale: float):
    """Single-query attention over caches: q [B,H,d], caches [B,H,cap,d]."""
    B, H, d = q.shape
    cap = kcache.shape[2]
    kq, pq, cq = _as_input(q)
    kk, pk, ck = _as_input(kcache)
    kv, pv, cv = _as_input(vcache)
    dt = _same_kind(cq, ck, cv)
    lens = np.ascontiguousarray(np.asarray(kv_lens, dtype=np.int32))
    if lens.shape != (B,):
        raise ValueError("kv_lens must have shape [B]")
    o = np.empty((B, H, d), np.float64)
    lse = np.empty((B, H), np.float64)
    _load().oracle_decode(pq, pk, pv, dt, lens.ctypes.data, o.ctypes.data, lse.ctypes.data, B, H, cap, d,
                          float(scale))
    return o, lse


def forward_varlen(q, k, v, cu_q, cu_k, scale: float, causal: bool):
    """Packed variable-length forward: q [total_q,H,d], k/v [total_k,H,d], cu_q/cu_k int32 [B+1].
    Returns O [total_q,H,d] and LSE [H,total_q] in float64."""
    total_q, H, d = q.shape
    kq, pq, cq = _as_input(q)
    kk, pk, ck = _as_input(k)
    kv, pv, cv = _as_input(v)
    dt = _same_kind(cq, ck, cv)
    cq_ = np.ascontiguousarray(np.asarray(cu_q, dtype=np.int32))
    ck_ = np.ascontiguousarray(np.asarray(cu_k, dtype=np.int32))
    B = cq_.shape[0] - 1
    if ck_.shape != cq_.shape or cq_[0] != 0 or ck_[0] != 0 or cq_[-1] != total_q or ck_[-1] != k.shape[0] \
            or np.any(np.diff(cq_) < 0) or np.any(np.diff(ck_) < 0):
        raise ValueError("cu_seqlens must start at 0, be non-decreasing and end at the packed lengths")
    o = np.empty((total_q, H, d), np.float64)
    lse = np.empty((H, total_q), np.float64)
    _load().oracle_forward_varlen(pq, pk, pv, dt, o.ctypes.data, lse.ctypes.data, cq_.ctypes.data, ck_.ctypes.data,
                                  B, H, total_q, d, float(scale), int(bool(causal)))
    return o, lse


def forward_blocksparse(q, k, v, mask, scale: float, causal: bool, block_q: int = 128, block_k: int = 128):
    """Forward under a block mask: q [B,H,Lq,d], k/v [B,H,Lk,d]; mask is uint8/bool, shape
    [Tq, Tk], [H, Tq, Tk] or [B, H, Tq, Tk] with Tq = ceil(Lq/block_q), Tk = ceil(Lk/block_k)
    (missing leading dimensions are shared).  Returns O [B,H,Lq,d] and LSE [B,H,Lq] in float64."""
    B, H, Lq, d = q.shape
    Lk = k.shape[2]
    if block_q < 1 or block_k < 1:
        raise ValueError("block sizes must be >= 1")
    tq, tk = -(-Lq // block_q), -(-Lk // block_k)
    m = np.ascontiguousarray(np.asarray(mask).astype(np.uint8))
    if m.shape[-2:] != (tq, tk) or m.ndim < 2 or m.ndim > 4 or (m.ndim >= 3 and m.shape[-3] != H) \
            or (m.ndim == 4 and m.shape[0] != B):
        raise ValueError("mask must have shape [Tq, Tk], [H, Tq, Tk] or [B, H, Tq, Tk]")
    sb = tq * tk * H if m.ndim == 4 else 0
    sh = tq * tk if m.ndim >= 3 else 0
    kq, pq, cq = _as_input(q)
    kk, pk, ck = _as_input(k)
    kv, pv, cv = _as_input(v)
    dt = _same_kind(cq, ck, cv)
    o = np.empty((B, H, Lq, d), np.float64)
    lse = np.empty((B, H, Lq), np.float64)
    _load().oracle_forward_blocksparse(pq, pk, pv, dt, o.ctypes.data, lse.ctypes.data, m.ctypes.data, sb, sh,
                                       int(block_q), int(block_k), B, H, Lq, Lk, d, float(scale), int(bool(causal)))
    return o, lse


def decode_paged(q, kpages, vpages, block_table, kv_lens, scale: float):
    """Single-query attention over a paged cache: q [B,H,d], pages [num_pages,Hkv,page_size,d],
    block_table int32 [B, max_blocks], kv_lens int32 [B].  Query head h reads KV head h // (H // Hkv)."""
    B, H, d = q.shape
    num_pages, Hkv, page_size = kpages.shape[0], kpages.shape[1], kpages.shape[2]
    kq, pq, cq = _as_input(q)
    kk, pk, ck = _as_input(kpages)
    kv, pv, cv = _as_input(vpages)
    dt = _same_kind(cq, ck, cv)
    bt = np.ascontiguousarray(np.asarray(block_table, dtype=np.int32))
    if bt.ndim != 2 or bt.shape[0] != B:
        raise ValueError("block_table must have shape [B, max_blocks]")
    lens = np.ascontiguousarray(np.asarray(kv_lens, dtype=np.int32))
    if lens.shape != (B,):
        raise ValueError("kv_lens must have shape [B]")
    o = np.empty((B, H, d), np.float64)
    lse = np.empty((B, H), np.float64)
    rc = _load().oracle_decode_paged(pq, pk, pv, dt, bt.ctypes.data, lens.ctypes.data, o.ctypes.data,
                                     lse.ctypes.data, B, H, Hkv, num_pages, page_size, bt.shape[1], d,
                                     float(scale))
    if rc == 1:
        raise ValueError("a block-table entry used by a valid key is outside [0, num_pages)")
    if rc == 2:
        raise ValueError("H must be a multiple of Hkv")
    return o, lse


def merge(o_parts, lse_parts):
    """Merge normalised partial outputs [n,d] with their LSE [n] into (O [d], LSE)."""
    op = np.ascontiguousarray(np.asarray(o_parts, dtype=np.float64))
    lp = np.ascontiguousarray(np.asarray(lse_parts, dtype=np.float64))
    n, d = op.shape
    o = np.empty((d,), np.float64)
    lse = np.empty((1,), np.float64)
    _load().oracle_merge(op.ctypes.data, lp.ctypes.data, n, d, o.ctypes.data, lse.ctypes.data)
    return o, float(lse[0])


def num_threads() -> int:
    """OpenMP threads the oracle's parallel regions use."""
    return int(_load().oracle_num_threads())


def set_num_threads(n: int) -> None:
    """Threads for the oracle's later parallel regions (timing only: results do not depend on it)."""
    _load().oracle_set_num_threads(int(n))
