"""The C-ABI library: it builds, loads, exports every entry point its header
declares, and rejects bad arguments before touching the GPU."""
import ctypes
import os
import re

import pytest
import torch

import exact_io_aware_94_b200 as fa
from exact_io_aware_94_b200 import build as fa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if not h.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", h)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*(fa_[a-z_0-9]+)\s*\(", text, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    fa_build.build()
    return fa.load_library()


def test_header_declares_the_entry_points():
    names = header_functions()
    for n in ("fa_forward", "fa_backward", "fa_backward_workspace_size", "fa_decode", "fa_decode_workspace_size",
              "fa_decode_paged", "fa_decode_paged_workspace_size", "fa_forward_varlen", "fa_check_status",
              "fa_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    raw = ctypes.CDLL(fa.LIB_PATH)
    for n in header_functions():
        assert hasattr(raw, n), "missing export %s" % n


def test_status_strings(lib):
    for code in range(0, 11):
        assert fa.fa_status_string(code)
    assert "unknown" in fa.fa_status_string(99)


# Fake, 16-byte aligned addresses: every call below must be rejected by the
# argument checks, which run before any CUDA call, so nothing is dereferenced.
P = 1 << 20


@pytest.mark.parametrize("args,code", [
    (dict(q=0), fa.FA_ERR_INVALID_ARG),
    (dict(d=96), fa.FA_ERR_UNSUPPORTED),
    (dict(d=32), fa.FA_ERR_UNSUPPORTED),
    (dict(B=0), fa.FA_ERR_INVALID_ARG),
    (dict(Lq=0), fa.FA_ERR_INVALID_ARG),
    (dict(Lk=-3), fa.FA_ERR_INVALID_ARG),
    (dict(causal=1, Lq=300, Lk=200), fa.FA_ERR_INVALID_ARG),
    (dict(q=P + 8), fa.FA_ERR_INVALID_ARG),
    (dict(o_dtype=7), fa.FA_ERR_UNSUPPORTED),
    (dict(scale=float("nan")), fa.FA_ERR_INVALID_ARG),
    (dict(scale=float("inf")), fa.FA_ERR_INVALID_ARG),
    (dict(scale=0.0), fa.FA_ERR_INVALID_ARG),    # -inf masks times a zero scale would give NaN
    (dict(scale=-0.125), fa.FA_ERR_INVALID_ARG),  # the running max is taken over raw scores
])
def test_forward_argument_checks(lib, args, code):
    a = dict(q=P, k=P, v=P, o=P, lse=P, B=1, H=1, Lq=64, Lk=64, d=64, scale=0.125, causal=0, o_dtype=0)
    a.update(args)
    rc = fa.fa_forward(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["H"], a["Lq"], a["Lk"], a["d"],
                       a["scale"], a["causal"], a["o_dtype"], 0)
    assert rc == code


@pytest.mark.parametrize("args,code", [
    (dict(kv=0), fa.FA_ERR_INVALID_ARG),
    (dict(d=80), fa.FA_ERR_UNSUPPORTED),
    (dict(cap=0), fa.FA_ERR_INVALID_ARG),
    (dict(ws=0), fa.FA_ERR_WORKSPACE),
    (dict(ws_bytes=16), fa.FA_ERR_WORKSPACE),
    (dict(ws=P + 16), fa.FA_ERR_WORKSPACE),
    (dict(scale=0.0), fa.FA_ERR_INVALID_ARG),
    (dict(scale=-1.0), fa.FA_ERR_INVALID_ARG),
])
def test_decode_argument_checks(lib, args, code):
    a = dict(q=P, k=P, v=P, kv=P, o=P, lse=P, B=2, H=2, cap=4096, d=128, ws=P, ws_bytes=1 << 30, scale=0.1)
    a.update(args)
    rc = fa.fa_decode(a["q"], a["k"], a["v"], a["kv"], a["o"], a["lse"], a["B"], a["H"], a["cap"], a["d"], a["scale"], 0,
                      a["ws"], a["ws_bytes"], 0)
    assert rc == code


@pytest.mark.parametrize("args,code", [
    (dict(bt=0), fa.FA_ERR_INVALID_ARG),
    (dict(kv=0), fa.FA_ERR_INVALID_ARG),
    (dict(d=96), fa.FA_ERR_UNSUPPORTED),
    (dict(Hkv=3), fa.FA_ERR_INVALID_ARG),       # H = 8 is not a multiple of 3
    (dict(Hkv=0), fa.FA_ERR_INVALID_ARG),
    (dict(ps=48), fa.FA_ERR_INVALID_ARG),       # not a power of two
    (dict(ps=1 << 17), fa.FA_ERR_INVALID_ARG),
    (dict(pages=0), fa.FA_ERR_INVALID_ARG),
    (dict(blocks=0), fa.FA_ERR_INVALID_ARG),
    (dict(kp=P + 8), fa.FA_ERR_INVALID_ARG),
    (dict(o_dtype=5), fa.FA_ERR_UNSUPPORTED),
    (dict(ws=0), fa.FA_ERR_WORKSPACE),
    (dict(ws_bytes=16), fa.FA_ERR_WORKSPACE),
    (dict(ws=P + 16), fa.FA_ERR_WORKSPACE),
    (dict(scale=0.0), fa.FA_ERR_INVALID_ARG),
])
def test_decode_paged_argument_checks(lib, args, code):
    a = dict(q=P, kp=P, vp=P, bt=P, kv=P, o=P, lse=P, B=2, H=8, Hkv=2, pages=64, ps=16, blocks=32, d=128,
             o_dtype=0, ws=P, ws_bytes=1 << 30, scale=0.1)
    a.update(args)
    rc = fa.fa_decode_paged(a["q"], a["kp"], a["vp"], a["bt"], a["kv"], a["o"], a["lse"], a["B"], a["H"], a["Hkv"],
                            a["pages"], a["ps"], a["blocks"], a["d"], a["scale"], a["o_dtype"], a["ws"], a["ws_bytes"], 0)
    assert rc == code


def test_decode_paged_workspace_size(lib):
    # the same partials as a contiguous decode over max_blocks * page_size keys
    assert fa.fa_decode_paged_workspace_size(3, 8, 32, 64, 128) == fa.fa_decode_workspace_size(3, 8, 2048, 128)
    assert fa.fa_decode_paged_workspace_size(3, 8, 0, 64, 128) == 0


@pytest.mark.parametrize("args,code", [
    (dict(cq=0), fa.FA_ERR_INVALID_ARG),
    (dict(q=0), fa.FA_ERR_INVALID_ARG),
    (dict(d=96), fa.FA_ERR_UNSUPPORTED),
    (dict(B=0), fa.FA_ERR_INVALID_ARG),
    (dict(tq=-1), fa.FA_ERR_INVALID_ARG),
    (dict(tk=0), fa.FA_ERR_INVALID_ARG),
    (dict(k=P + 4), fa.FA_ERR_INVALID_ARG),
    (dict(o_dtype=3), fa.FA_ERR_UNSUPPORTED),
    (dict(tq=0), fa.FA_OK),            # nothing to do: no launch
    (dict(maxq=0), fa.FA_OK),
    (dict(scale=-0.5), fa.FA_ERR_INVALID_ARG),
])
def test_forward_varlen_argument_checks(lib, args, code):
    a = dict(q=P, k=P, v=P, o=P, lse=P, cq=P, ck=P, B=3, H=4, tq=100, tk=120, maxq=64, d=128, o_dtype=0, scale=0.1)
    a.update(args)
    rc = fa.fa_forward_varlen(a["q"], a["k"], a["v"], a["o"], a["lse"], a["cq"], a["ck"], a["B"], a["H"], a["tq"],
                              a["tk"], a["maxq"], a["d"], a["scale"], 1, a["o_dtype"], 0)
    assert rc == code


@pytest.mark.parametrize("scale,code", [(0.125, fa.FA_ERR_WORKSPACE), (0.0, fa.FA_ERR_INVALID_ARG),
                                        (-0.125, fa.FA_ERR_INVALID_ARG), (float("nan"), fa.FA_ERR_INVALID_ARG)])
def test_backward_scale_checks(lib, scale, code):
    """The backward masks scores to -inf before the exponent as the forward does: the
    scale must be positive.  (A valid scale reaches the workspace check, which fails.)"""
    rc = fa.fa_backward(P, P, P, P, P, P, P, P, P, 1, 1, 64, 64, 64, scale, 1, 0, 0, 0, 0)
    assert rc == code
    rc = fa.fa_backward_noalloc(P, P, P, P, P, P, P, P, P, 1, 1, 64, 64, 64, scale, 1, 0, 0)
    assert rc == (fa.FA_ERR_INVALID_ARG if code == fa.FA_ERR_INVALID_ARG else rc)


@pytest.mark.parametrize("args,code", [
    (dict(mask=0), fa.FA_ERR_INVALID_ARG),
    (dict(q=0), fa.FA_ERR_INVALID_ARG),
    (dict(d=96), fa.FA_ERR_UNSUPPORTED),
    (dict(o_dtype=4), fa.FA_ERR_UNSUPPORTED),
    (dict(sb=-1), fa.FA_ERR_INVALID_ARG),
    (dict(sh=-8), fa.FA_ERR_INVALID_ARG),
    (dict(Lq=0), fa.FA_ERR_INVALID_ARG),
    (dict(causal=1, Lq=600, Lk=520), fa.FA_ERR_INVALID_ARG),
    (dict(Lk=128 * 16384 + 1), fa.FA_ERR_INVALID_ARG),  # key-block index must fit 14 bits
    (dict(scale=0.0), fa.FA_ERR_INVALID_ARG),
    (dict(o=P + 8), fa.FA_ERR_INVALID_ARG),
    (dict(ws=0), fa.FA_ERR_WORKSPACE),
    (dict(ws=P + 16), fa.FA_ERR_WORKSPACE),
    (dict(ws_bytes=256), fa.FA_ERR_WORKSPACE),
])
def test_forward_blocksparse_argument_checks(lib, args, code):
    a = dict(q=P, k=P, v=P, o=P, lse=P, mask=P + 3, sb=0, sh=40, B=2, H=3, Lq=300, Lk=520, d=128, scale=0.1,
             causal=0, o_dtype=0, ws=P, ws_bytes=1 << 30)
    a.update(args)
    rc = fa.fa_forward_blocksparse(a["q"], a["k"], a["v"], a["o"], a["lse"], a["mask"], a["sb"], a["sh"], a["B"],
                                   a["H"], a["Lq"], a["Lk"], a["d"], a["scale"], a["causal"], a["o_dtype"], a["ws"],
                                   a["ws_bytes"], 0)
    assert rc == code


def test_forward_blocksparse_workspace_size(lib):
    # per 256-row unit: 16 bytes of metadata, a union list and two own lists of up to Tk key
    # blocks (uint16 each); each of the three parts 256-byte aligned
    n_units, tk = 2 * 3 * 2, 5
    up = lambda x: -(-x // 256) * 256  # noqa: E731
    want = up(n_units * 16) + up(n_units * tk * 2) + up(2 * n_units * tk * 2)
    assert fa.fa_forward_blocksparse_workspace_size(2, 3, 300, 520) == want
    assert fa.fa_forward_blocksparse_workspace_size(0, 3, 300, 520) == 0
    assert fa.fa_forward_blocksparse_workspace_size(1, 1, 128, 128 * 16384 + 1) == 0


def test_decode_workspace_size(lib):
    # 2 heads x 4 chunks of 1024 keys x 128 fp32 + LSE + lengths + prefix sums
    n = fa.fa_decode_workspace_size(1, 2, 4096, 128)
    assert n >= 2 * 4 * 128 * 4 + 2 * 4 * 4
    assert fa.fa_decode_workspace_size(0, 2, 4096, 128) == 0


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks behaviour without a CUDA device")
def test_valid_call_without_gpu_fails_loudly(lib):
    """No device: a well-formed call must return an error, never run a CPU path."""
    rc = fa.fa_forward(P, P, P, P, P, 1, 1, 64, 64, 64, 0.125, 0, 0, 0)
    assert rc in (fa.FA_ERR_CUDA, fa.FA_ERR_DEVICE)
    with pytest.raises(ValueError):
        fa.forward(torch.zeros(1, 1, 4, 64, dtype=torch.bfloat16), torch.zeros(1, 1, 4, 64, dtype=torch.bfloat16),
                   torch.zeros(1, 1, 4, 64, dtype=torch.bfloat16))
