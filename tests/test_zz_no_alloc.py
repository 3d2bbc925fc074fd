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


@pytest.mark.gpu
def test_noalloc_backward_matches_workspace_backward_twice(cuda_device):
    dev = cuda_device
    B, H, L, d = 2, 3, 700, 128
    scale = 1.0 / math.sqrt(d)
    inp = attention_inputs(B, H, L, L, d, seed=77, with_dO=True)
    q, k, v, g = (t.to(dev) for t in (inp.q, inp.k, inp.v, inp.dO))
    o, lse = fa.forward(q, k, v, scale=scale, causal=True)
    ref = fa.backward(q, k, v, o, g, lse, scale=scale, causal=True)
    for call in range(2):
        outs = [torch.full_like(q, float("nan")), torch.full_like(k, float("nan")), torch.full_like(v, float("nan"))]
        rc = fa.fa_backward_noalloc(q, k, v, o, g, lse, outs[0], outs[1], outs[2], B, H, L, L, d, scale, 1,
                                    fa.FA_DT_F32, None)
        assert rc == fa.FA_OK, fa.fa_status_string(rc)
        assert fa.fa_check_status() == fa.FA_OK
        for name, x, r in zip(("dQ", "dK", "dV"), outs, ref):
            assert torch.isfinite(x).all(), (call, name)
            assert rel_fro(to_np(x), to_np(r)) <= 1e-2, (call, name)


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
