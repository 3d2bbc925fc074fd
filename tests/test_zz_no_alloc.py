"""fa_backward_noalloc: the backward pass for callers that cannot allocate
device memory (a host framework that owns every allocation and offers no
workspace hook, or a loop that cannot afford cudaMalloc's implicit
synchronisation).  Its scratch is a fixed static device array, so its results
must match fa_backward, which takes a caller-provided workspace, call after
call.  This file is collected last on purpose."""
import math

import pytest
import torch

import exact_io_aware_94_b200 as fa
from exact_io_aware_94_b200.inputs import attention_inputs

from .parity import rel_fro, to_np


def _noalloc(q, k, v, o, g, lse, B, H, Lq, Lk, d, scale, causal, o_dtype):
    outs = [torch.full_like(q, float("nan")), torch.full_like(k, float("nan")), torch.full_like(v, float("nan"))]
    rc = fa.fa_backward_noalloc(q, k, v, o, g, lse, outs[0], outs[1], outs[2], B, H, Lq, Lk, d, scale, int(causal),
                                o_dtype, None)
    assert rc == fa.FA_OK, fa.fa_status_string(rc)
    assert fa.fa_check_status() == fa.FA_OK
    return outs


@pytest.mark.gpu
@pytest.mark.parametrize("d,Lq,Lk,causal,out_dtype", [
    (128, 700, 700, True, torch.float32),
    (64, 700, 700, True, torch.bfloat16),
    (128, 300, 650, True, torch.bfloat16),   # fewer queries than keys: bottom-right causal
    (64, 257, 513, False, torch.float32),
    (256, 300, 300, True, torch.float32),
])
def test_noalloc_backward_matches_workspace_backward_twice(cuda_device, d, Lq, Lk, causal, out_dtype):
    dev = cuda_device
    B, H = 2, 3
    scale = 1.0 / math.sqrt(d)
    inp = attention_inputs(B, H, Lq, Lk, d, seed=77 + d + Lk, with_dO=True)
    q, k, v, g = (t.to(dev) for t in (inp.q, inp.k, inp.v, inp.dO))
    o, lse = fa.forward(q, k, v, scale=scale, causal=causal, out_dtype=out_dtype)
    ref = fa.backward(q, k, v, o, g, lse, scale=scale, causal=causal)
    o_dtype = fa.FA_DT_F32 if out_dtype == torch.float32 else fa.FA_DT_BF16
    for call in range(2):
        outs = _noalloc(q, k, v, o, g, lse, B, H, Lq, Lk, d, scale, causal, o_dtype)
        for name, x, r in zip(("dQ", "dK", "dV"), outs, ref):
            assert torch.isfinite(x).all(), (call, name)
            assert rel_fro(to_np(x), to_np(r)) <= 1e-2, (call, name)


@pytest.mark.gpu
def test_noalloc_backward_at_its_largest_size_then_smaller(cuda_device):
    """B*H*Lq equal to FA_NOALLOC_MAX_ROWS uses the scratch up to its last row; a
    smaller call made next reads a scratch still holding the large call's values
    and must not be affected by them."""
    dev = cuda_device
    d = 64
    B, H, Lk = 1, 8, 128
    Lq = fa.FA_NOALLOC_MAX_ROWS // (B * H)
    scale = 1.0 / math.sqrt(d)
    gen = torch.Generator(device=dev).manual_seed(5)
    q = torch.randn(B, H, Lq, d, generator=gen, device=dev).to(torch.bfloat16)
    g = torch.randn(B, H, Lq, d, generator=gen, device=dev).to(torch.bfloat16)
    k = torch.randn(B, H, Lk, d, generator=gen, device=dev).to(torch.bfloat16)
    v = torch.randn(B, H, Lk, d, generator=gen, device=dev).to(torch.bfloat16)
    o, lse = fa.forward(q, k, v, scale=scale, causal=False)
    outs = _noalloc(q, k, v, o, g, lse, B, H, Lq, Lk, d, scale, False, fa.FA_DT_F32)
    for name, x in zip(("dQ", "dK", "dV"), outs):
        assert torch.isfinite(x).all(), name
    tail = [t[:, :, -256:].contiguous() for t in (q, o, g, lse)]
    ref_last = fa.backward(tail[0], k, v, tail[1], tail[2], tail[3], scale=scale, causal=False)
    # the last query rows' dQ only depend on those rows: check them against fa_backward
    assert rel_fro(to_np(outs[0][:, :, -256:]), to_np(ref_last[0])) <= 1e-2
    del q, g, o, lse, outs
    B, H, L = 2, 2, 333
    inp = attention_inputs(B, H, L, L, d, seed=78, with_dO=True)
    q, k, v, g = (t.to(dev) for t in (inp.q, inp.k, inp.v, inp.dO))
    o, lse = fa.forward(q, k, v, scale=scale, causal=True)
    ref = fa.backward(q, k, v, o, g, lse, scale=scale, causal=True)
    outs = _noalloc(q, k, v, o, g, lse, B, H, L, L, d, scale, True, fa.FA_DT_F32)
    for name, x, r in zip(("dQ", "dK", "dV"), outs, ref):
        assert rel_fro(to_np(x), to_np(r)) <= 1e-2, name


@pytest.mark.gpu
def test_noalloc_backward_rejects_sizes_beyond_its_scratch(cuda_device):
    dev = cuda_device
    d = 64
    t = torch.zeros(16, dtype=torch.bfloat16, device=dev)
    lse = torch.zeros(4, dtype=torch.float32, device=dev)
    # B*H*Lq one past the fixed scratch: refused before anything is launched
    rows = fa.FA_NOALLOC_MAX_ROWS + 1
    rc = fa.fa_backward_noalloc(t, t, t, t, t, lse, t, t, t, 1, 1, rows, rows, d, 0.125, 1, fa.FA_DT_F32, None)
    assert rc == fa.FA_ERR_TOO_LARGE
    assert "FA_NOALLOC_MAX_ROWS" in fa.fa_status_string(rc)
