"""Exact IO-aware attention for B200 (sm_100a): thin Python binding over the C-ABI library.

The binding only marshals arguments; every step of the attention path runs in
the library's CUDA kernels (``libfa_sm100.so``, built from ``csrc/`` by
``python -m exact_io_aware_94_b200.build``).  There is no CPU fallback: if the
library is missing or the device is not sm_100, every call raises.

Two levels:
  * ``fa_forward``, ``fa_backward``, ``fa_decode``, ``fa_*_workspace_size``,
    ``fa_check_status``, ``fa_status_string``: the C entry points with the same
    names and arguments (tensors may be passed for pointers), returning the
    status code.
  * ``forward``, ``backward``, ``decode``: allocate outputs (and workspace) with
    torch on the inputs' device, call the entry point on the current stream and
    raise ``FAError`` on a non-zero status.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

from .inputs import AttentionInputs, DecodeInputs, attention_inputs, decode_inputs  # noqa: F401

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libfa_sm100.so")

FA_OK = 0
FA_ERR_INVALID_ARG = 1
FA_ERR_UNSUPPORTED = 2
FA_ERR_WORKSPACE = 3
FA_ERR_CUDA = 4
FA_ERR_TIMEOUT = 5
FA_ERR_DEVICE = 6
FA_ERR_KV_LEN = 7
FA_ERR_TOO_LARGE = 8
FA_ERR_PAGE = 9
FA_ERR_SEQLEN = 10
FA_NOALLOC_MAX_ROWS = 1 << 20
FA_DT_BF16 = 0
FA_DT_F32 = 1

_DT = {torch.bfloat16: FA_DT_BF16, torch.float32: FA_DT_F32}

_lib = None


class FAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__("%s failed: %s" % (where, fa_status_string(status)))


def load_library():
    """Load libfa_sm100.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError("CUDA library %s is not built (python -m exact_io_aware_94_b200.build); "
                           "there is no fallback path" % LIB_PATH)
    lib = ctypes.CDLL(LIB_PATH)
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.fa_forward.restype = i
    lib.fa_forward.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, vp]
    lib.fa_backward_workspace_size.restype = sz
    lib.fa_backward_workspace_size.argtypes = [i, i, i, i, i]
    lib.fa_backward.restype = i
    lib.fa_backward.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, vp, sz, vp]
    lib.fa_backward_noalloc.restype = i
    lib.fa_backward_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, vp]
    lib.fa_decode_workspace_size.restype = sz
    lib.fa_decode_workspace_size.argtypes = [i, i, i, i]
    lib.fa_decode.restype = i
    lib.fa_decode.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, vp, sz, vp]
    lib.fa_forward_varlen.restype = i
    lib.fa_forward_varlen.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, i, vp]
    lib.fa_forward_blocksparse_workspace_size.restype = sz
    lib.fa_forward_blocksparse_workspace_size.argtypes = [i, i, i, i]
    lib.fa_forward_blocksparse.restype = i
    lib.fa_forward_blocksparse.argtypes = [vp, vp, vp, vp, vp, vp, ctypes.c_longlong, ctypes.c_longlong, i, i, i, i, i,
                                           f, i, i, vp, sz, vp]
    lib.fa_decode_paged_workspace_size.restype = sz
    lib.fa_decode_paged_workspace_size.argtypes = [i, i, i, i, i]
    lib.fa_decode_paged.restype = i
    lib.fa_decode_paged.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, f, i, vp, sz, vp]
    lib.fa_check_status.restype = i
    lib.fa_check_status.argtypes = [vp]
    lib.fa_status_string.restype = ctypes.c_char_p
    lib.fa_status_string.argtypes = [i]
    _lib = lib
    return lib


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, torch.Tensor):
        return x.data_ptr()
    return int(x)


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


# ----------------------------------------------------------------- C entry points, same names

def fa_status_string(status: int) -> str:
    return load_library().fa_status_string(int(status)).decode()


def fa_forward(q, k, v, o, lse, B, H, Lq, Lk, d, scale, causal, o_dtype, stream=None) -> int:
    return load_library().fa_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, Lq, Lk, d,
                                     float(scale), int(causal), int(o_dtype), _stream(stream))


def fa_backward_workspace_size(B, H, Lq, Lk, d) -> int:
    return int(load_library().fa_backward_workspace_size(B, H, Lq, Lk, d))


def fa_backward(q, k, v, o, dO, lse, dq, dk, dv, B, H, Lq, Lk, d, scale, causal, o_dtype, workspace,
                workspace_bytes, stream=None) -> int:
    return load_library().fa_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dO), _ptr(lse), _ptr(dq),
                                      _ptr(dk), _ptr(dv), B, H, Lq, Lk, d, float(scale), int(causal),
                                      int(o_dtype), _ptr(workspace), int(workspace_bytes), _stream(stream))


def fa_backward_noalloc(q, k, v, o, dO, lse, dq, dk, dv, B, H, Lq, Lk, d, scale, causal, o_dtype,
                        stream=None) -> int:
    return load_library().fa_backward_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dO), _ptr(lse), _ptr(dq),
                                              _ptr(dk), _ptr(dv), B, H, Lq, Lk, d, float(scale), int(causal),
                                              int(o_dtype), _stream(stream))


def fa_decode_workspace_size(B, H, cap, d) -> int:
    return int(load_library().fa_decode_workspace_size(B, H, cap, d))


def fa_decode(q, kcache, vcache, kv_lens, o, lse, B, H, cap, d, scale, o_dtype, workspace, workspace_bytes,
              stream=None) -> int:
    return load_library().fa_decode(_ptr(q), _ptr(kcache), _ptr(vcache), _ptr(kv_lens), _ptr(o), _ptr(lse), B,
                                    H, cap, d, float(scale), int(o_dtype), _ptr(workspace), int(workspace_bytes),
                                    _stream(stream))


def fa_forward_varlen(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, B, H, total_q, total_k, max_seqlen_q, d, scale,
                      causal, o_dtype, stream=None) -> int:
    return load_library().fa_forward_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(cu_seqlens_q),
                                            _ptr(cu_seqlens_k), B, H, total_q, total_k, max_seqlen_q, d, float(scale),
                                            int(causal), int(o_dtype), _stream(stream))


def fa_forward_blocksparse_workspace_size(B, H, Lq, Lk) -> int:
    return int(load_library().fa_forward_blocksparse_workspace_size(B, H, Lq, Lk))


def fa_forward_blocksparse(q, k, v, o, lse, block_mask, mask_stride_b, mask_stride_h, B, H, Lq, Lk, d, scale, causal,
                           o_dtype, workspace, workspace_bytes, stream=None) -> int:
    return load_library().fa_forward_blocksparse(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(block_mask),
                                                 int(mask_stride_b), int(mask_stride_h), B, H, Lq, Lk, d,
                                                 float(scale), int(causal), int(o_dtype), _ptr(workspace),
                                                 int(workspace_bytes), _stream(stream))


def fa_decode_paged_workspace_size(B, H, max_blocks, page_size, d) -> int:
    return int(load_library().fa_decode_paged_workspace_size(B, H, max_blocks, page_size, d))


def fa_decode_paged(q, kpages, vpages, block_table, kv_lens, o, lse, B, H, Hkv, num_pages, page_size, max_blocks, d,
                    scale, o_dtype, workspace, workspace_bytes, stream=None) -> int:
    return load_library().fa_decode_paged(_ptr(q), _ptr(kpages), _ptr(vpages), _ptr(block_table), _ptr(kv_lens),
                                          _ptr(o), _ptr(lse), B, H, Hkv, num_pages, page_size, max_blocks, d,
                                          float(scale), int(o_dtype), _ptr(workspace), int(workspace_bytes),
                                          _stream(stream))


def fa_check_status(stream=None) -> int:
    return load_library().fa_check_status(_stream(stream))


# ----------------------------------------------------------------- allocating helpers

def _check(rc: int, where: str):
    if rc != FA_OK:
        raise FAError(rc, where)


def _need(t: torch.Tensor, name: str, dtype=torch.bfloat16):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if t.dtype != dtype:
        raise ValueError("%s must be %s" % (name, dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)


def workspace(nbytes: int, device) -> torch.Tensor:
    """A caller-owned device workspace of at least nbytes (256-byte aligned by the allocator)."""
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def forward(q, k, v, scale=None, causal=False, out_dtype=torch.float32, out=None, lse=None, stream=None):
    """O [B,H,Lq,d] (out_dtype) and LSE [B,H,Lq] (fp32) for bf16 q [B,H,Lq,d], k/v [B,H,Lk,d]."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n)
    B, H, Lq, d = q.shape
    Lk = k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((B, H, Lq, d), dtype=out_dtype, device=q.device)
    if lse is None:
        lse = torch.empty((B, H, Lq), dtype=torch.float32, device=q.device)
    rc = fa_forward(q, k, v, out, lse, B, H, Lq, Lk, d, scale, causal, _DT[out.dtype], stream)
    _check(rc, "fa_forward")
    return out, lse


def backward(q, k, v, o, dO, lse, scale=None, causal=False, ws=None, stream=None):
    """dQ, dK, dV (bf16) with P recomputed from lse."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (dO, "dO")):
        _need(t, n)
    B, H, Lq, d = q.shape
    Lk = k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    nbytes = fa_backward_workspace_size(B, H, Lq, Lk, d)
    if ws is None:
        ws = workspace(nbytes, q.device)
    dq = torch.empty_like(q)
    dk = torch.empty_like(k)
    dv = torch.empty_like(v)
    rc = fa_backward(q, k, v, o, dO, lse, dq, dk, dv, B, H, Lq, Lk, d, scale, causal, _DT[o.dtype], ws,
                     ws.numel() * ws.element_size(), stream)
    _check(rc, "fa_backward")
    return dq, dk, dv


def decode(q, kcache, vcache, kv_lens, scale=None, out_dtype=torch.float32, ws=None, stream=None):
    """o [B,H,d] and lse [B,H] for q [B,H,d], caches [B,H,cap,d], kv_lens int32 [B] (device)."""
    for t, n in ((q, "q"), (kcache, "kcache"), (vcache, "vcache")):
        _need(t, n)
    _need(kv_lens, "kv_lens", torch.int32)
    B, H, cap, d = kcache.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    nbytes = fa_decode_workspace_size(B, H, cap, d)
    if ws is None:
        ws = workspace(nbytes, q.device)
    o = torch.empty((B, H, d), dtype=out_dtype, device=q.device)
    lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    rc = fa_decode(q, kcache, vcache, kv_lens, o, lse, B, H, cap, d, scale, _DT[out_dtype], ws,
                   ws.numel() * ws.element_size(), stream)
    _check(rc, "fa_decode")
    return o, lse


def decode_paged(q, kpages, vpages, block_table, kv_lens, scale=None, out_dtype=torch.float32, ws=None, stream=None):
    """o [B,H,d] and lse [B,H] for q [B,H,d], pages [num_pages,Hkv,page_size,d] (bf16),
    block_table int32 [B,max_blocks] and kv_lens int32 [B] (device)."""
    for t, n in ((q, "q"), (kpages, "kpages"), (vpages, "vpages")):
        _need(t, n)
    _need(block_table, "block_table", torch.int32)
    _need(kv_lens, "kv_lens", torch.int32)
    B, H, d = q.shape
    num_pages, Hkv, page_size = kpages.shape[0], kpages.shape[1], kpages.shape[2]
    max_blocks = block_table.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    nbytes = fa_decode_paged_workspace_size(B, H, max_blocks, page_size, d)
    if ws is None:
        ws = workspace(nbytes, q.device)
    o = torch.empty((B, H, d), dtype=out_dtype, device=q.device)
    lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    rc = fa_decode_paged(q, kpages, vpages, block_table, kv_lens, o, lse, B, H, Hkv, num_pages, page_size, max_blocks,
                         d, scale, _DT[out_dtype], ws, ws.numel() * ws.element_size(), stream)
    _check(rc, "fa_decode_paged")
    return o, lse


def forward_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, scale=None, causal=False,
                   out_dtype=torch.float32, stream=None):
    """Packed batch: q [total_q,H,d], k/v [total_k,H,d] (bf16), cu_seqlens int32 [B+1] (device).
    Returns o [total_q,H,d] (out_dtype) and lse [H,total_q] (fp32)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n)
    _need(cu_seqlens_q, "cu_seqlens_q", torch.int32)
    _need(cu_seqlens_k, "cu_seqlens_k", torch.int32)
    total_q, H, d = q.shape
    total_k = k.shape[0]
    B = cu_seqlens_q.shape[0] - 1
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    o = torch.empty((total_q, H, d), dtype=out_dtype, device=q.device)
    lse = torch.empty((H, total_q), dtype=torch.float32, device=q.device)
    rc = fa_forward_varlen(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, B, H, total_q, total_k, int(max_seqlen_q), d,
                           scale, causal, _DT[out_dtype], stream)
    _check(rc, "fa_forward_varlen")
    return o, lse


BLOCKSPARSE_BLOCK = 128


def forward_blocksparse(q, k, v, block_mask, scale=None, causal=False, out_dtype=torch.float32, ws=None,
                        stream=None):
    """Forward under a block mask: bf16 q [B,H,Lq,d], k/v [B,H,Lk,d]; block_mask uint8 or bool on the device
    with shape [Tq,Tk], [H,Tq,Tk] or [B,H,Tq,Tk] (Tq = ceil(Lq/128), Tk = ceil(Lk/128)); size-1 or
    expanded leading dimensions are shared.  Returns O [B,H,Lq,d] (out_dtype) and LSE [B,H,Lq] (fp32)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n)
    B, H, Lq, d = q.shape
    Lk = k.shape[2]
    tq, tk = -(-Lq // BLOCKSPARSE_BLOCK), -(-Lk // BLOCKSPARSE_BLOCK)
    m = block_mask
    if not isinstance(m, torch.Tensor) or not m.is_cuda or m.dtype not in (torch.uint8, torch.bool):
        raise ValueError("block_mask must be a CUDA uint8 or bool tensor")
    if m.dtype == torch.bool:
        m = m.view(torch.uint8)
    while m.dim() < 4:
        m = m.unsqueeze(0)
    if m.dim() != 4 or tuple(m.shape[2:]) != (tq, tk) or m.shape[0] not in (1, B) or m.shape[1] not in (1, H) \
            or m.stride(3) != 1 or (tq > 1 and m.stride(2) != tk):
        raise ValueError("block_mask must have shape [Tq,Tk], [H,Tq,Tk] or [B,H,Tq,Tk] = [.., %d, %d] with "
                         "contiguous rows" % (tq, tk))
    sb = 0 if m.shape[0] == 1 else m.stride(0)
    sh = 0 if m.shape[1] == 1 else m.stride(1)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    nbytes = fa_forward_blocksparse_workspace_size(B, H, Lq, Lk)
    if ws is None:
        ws = workspace(nbytes, q.device)
    o = torch.empty((B, H, Lq, d), dtype=out_dtype, device=q.device)
    lse = torch.empty((B, H, Lq), dtype=torch.float32, device=q.device)
    rc = fa_forward_blocksparse(q, k, v, o, lse, m, sb, sh, B, H, Lq, Lk, d, scale, causal, _DT[out_dtype], ws,
                                ws.numel() * ws.element_size(), stream)
    _check(rc, "fa_forward_blocksparse")
    return o, lse
