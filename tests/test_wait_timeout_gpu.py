"""Bounded waits: a wait that runs out ends the kernel with FA_ERR_TIMEOUT, and the
device stays usable.

These tests load the fault-injection build of the library
(libfa_sm100_testhooks.so: the same sources compiled with FA_TEST_HOOKS, so
every wait gives up after 20 ms and fa_test_inject_fault is exported), never the
product library.  The fault is an omission on the issuing side: a producer warp
does not issue one copy (neither its expected byte count nor the copy itself),
so the consumer's wait for it runs out.  Nothing faults, traps or hangs; the
kernel drains what it did issue, frees its tensor memory and exits.
"""
import ctypes
import math

import pytest
import torch

import exact_io_aware_94_b200 as fa
import oracle
from exact_io_aware_94_b200 import build as fa_build
from exact_io_aware_94_b200.inputs import attention_inputs, decode_inputs

from .parity import check_lse, check_o, rel_fro, to_np

pytestmark = pytest.mark.gpu

FWD_SKIP_K, BWD_SKIP_KV, PAGED_SKIP_STAGE = 1, 2, 3


@pytest.fixture(scope="module")
def hooks(cuda_device):
    lib = ctypes.CDLL(fa_build.build(test_hooks=True))
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.fa_test_inject_fault.restype = i
    lib.fa_test_inject_fault.argtypes = [i]
    lib.fa_forward.restype = i
    lib.fa_forward.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, vp]
    lib.fa_backward.restype = i
    lib.fa_backward.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, vp, sz, vp]
    lib.fa_decode_paged.restype = i
    lib.fa_decode_paged.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, f, i, vp, sz, vp]
    lib.fa_check_status.restype = i
    lib.fa_check_status.argtypes = [vp]
    assert lib.fa_check_status(None) == fa.FA_OK
    return lib


def _stream():
    return torch.cuda.current_stream().cuda_stream


def _forward(lib, q, k, v, causal):
    B, H, L, d = q.shape
    o = torch.full((B, H, L, d), float("nan"), dtype=torch.float32, device=q.device)
    lse = torch.full((B, H, L), float("nan"), dtype=torch.float32, device=q.device)
    rc = lib.fa_forward(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, H, L, L, d,
                        1.0 / math.sqrt(d), int(causal), fa.FA_DT_F32, _stream())
    assert rc == fa.FA_OK
    torch.cuda.synchronize()
    return o, lse


def test_forward_wait_runs_out_and_status_is_sticky(hooks, cuda_device):
    B, H, L, d = 1, 1, 256, 128
    inp = attention_inputs(B, H, L, L, d, seed=91)
    q, k, v = (t.to(cuda_device) for t in (inp.q, inp.k, inp.v))
    assert hooks.fa_test_inject_fault(FWD_SKIP_K) == fa.FA_OK
    o1, _ = _forward(hooks, q, k, v, False)   # its K tile 0 never arrives: the MMA warp's wait runs out
    assert torch.isnan(o1).all()              # one CTA, aborted before its epilogue
    o2, lse2 = _forward(hooks, q, k, v, False)  # before clearing: exits at once, writes nothing
    assert torch.isnan(o2).all() and torch.isnan(lse2).all()
    assert hooks.fa_check_status(None) == fa.FA_ERR_TIMEOUT
    assert hooks.fa_check_status(None) == fa.FA_OK
    o3, lse3 = _forward(hooks, q, k, v, True)  # after clearing: computes again
    assert hooks.fa_check_status(None) == fa.FA_OK
    o_ref, lse_ref = oracle.forward(inp.q, inp.k, inp.v, 1.0 / math.sqrt(d), True)
    check_o(o3, o_ref, "forward after a timeout")
    check_lse(lse3, lse_ref, "forward after a timeout")


def test_backward_wait_runs_out(hooks, cuda_device):
    B, H, L, d = 1, 2, 384, 64
    scale = 1.0 / math.sqrt(d)
    inp = attention_inputs(B, H, L, L, d, seed=92, with_dO=True)
    q, k, v, g = (t.to(cuda_device) for t in (inp.q, inp.k, inp.v, inp.dO))
    o, lse = fa.forward(q, k, v, scale=scale, causal=True)  # product library
    ref = fa.backward(q, k, v, o, g, lse, scale=scale, causal=True)
    ws = fa.workspace(fa.fa_backward_workspace_size(B, H, L, L, d), cuda_device)

    def bwd():
        outs = [torch.full_like(t, float("nan")) for t in (q, k, v)]
        rc = hooks.fa_backward(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), g.data_ptr(), lse.data_ptr(),
                               outs[0].data_ptr(), outs[1].data_ptr(), outs[2].data_ptr(), B, H, L, L, d, scale, 1,
                               fa.FA_DT_F32, ws.data_ptr(), ws.numel(), _stream())
        assert rc == fa.FA_OK
        torch.cuda.synchronize()
        return outs

    assert hooks.fa_test_inject_fault(BWD_SKIP_KV) == fa.FA_OK
    outs = bwd()
    assert hooks.fa_check_status(None) == fa.FA_ERR_TIMEOUT
    # the dQ pass started after the timeout was recorded, so it wrote nothing
    assert torch.isnan(outs[0]).all()
    outs = bwd()
    assert hooks.fa_check_status(None) == fa.FA_OK
    for name, x, r in zip(("dQ", "dK", "dV"), outs, ref):
        assert rel_fro(to_np(x), to_np(r)) <= 1e-6, name  # same kernels, same inputs: same result


def test_paged_decode_wait_runs_out(hooks, cuda_device):
    B, H, Hkv, d, ps, nblk = 2, 8, 2, 128, 64, 8
    cap = ps * nblk
    inp = decode_inputs(B, H, cap, d, seed=93, len_lo=200, len_hi=cap)
    kv_lens = inp.kv_lens.to(cuda_device)
    # one page per block, pages in order: sequence b's block j is page b * nblk + j
    kpages = inp.kcache[:, :Hkv].reshape(B, Hkv, nblk, ps, d).permute(0, 2, 1, 3, 4).reshape(B * nblk, Hkv, ps, d)
    vpages = inp.vcache[:, :Hkv].reshape(B, Hkv, nblk, ps, d).permute(0, 2, 1, 3, 4).reshape(B * nblk, Hkv, ps, d)
    table = torch.arange(B * nblk, dtype=torch.int32).reshape(B, nblk)
    kp, vp, tb, q = (t.contiguous().to(cuda_device) for t in (kpages, vpages, table, inp.q))
    ws = fa.workspace(fa.fa_decode_paged_workspace_size(B, H, nblk, ps, d), cuda_device)

    def dec():
        o = torch.full((B, H, d), float("nan"), dtype=torch.float32, device=cuda_device)
        lse = torch.full((B, H), float("nan"), dtype=torch.float32, device=cuda_device)
        rc = hooks.fa_decode_paged(q.data_ptr(), kp.data_ptr(), vp.data_ptr(), tb.data_ptr(), kv_lens.data_ptr(),
                                   o.data_ptr(), lse.data_ptr(), B, H, Hkv, B * nblk, ps, nblk, d, 1.0 / math.sqrt(d),
                                   fa.FA_DT_F32, ws.data_ptr(), ws.numel(), _stream())
        assert rc == fa.FA_OK
        torch.cuda.synchronize()
        return o, lse

    assert hooks.fa_test_inject_fault(PAGED_SKIP_STAGE) == fa.FA_OK
    dec()
    assert hooks.fa_check_status(None) == fa.FA_ERR_TIMEOUT
    o, lse = dec()
    assert hooks.fa_check_status(None) == fa.FA_OK
    o_ref, lse_ref = oracle.decode_paged(inp.q, kpages.contiguous(), vpages.contiguous(), table, inp.kv_lens,
                                         1.0 / math.sqrt(d))
    check_o(o, o_ref, "paged decode after a timeout")
    check_lse(lse, lse_ref, "paged decode after a timeout")
