"""Backward kernels (recomputation from the saved LSE) vs the oracle (GPU)."""
import math

import numpy as np
import pytest
import torch

import exact_io_aware_94_b200 as fa
import oracle
from exact_io_aware_94_b200.inputs import WORKLOADS, attention_inputs

from .parity import check_grad, rel_fro, to_np

pytestmark = pytest.mark.gpu


def gpu_fwd_bwd(inp, scale, causal, dev, o_dtype=torch.float32):
    q, k, v, g = (t.to(dev) for t in (inp.q, inp.k, inp.v, inp.dO))
    o, lse = fa.forward(q, k, v, scale=scale, causal=causal, out_dtype=o_dtype)
    dq, dk, dv = fa.backward(q, k, v, o, g, lse, scale=scale, causal=causal)
    assert fa.fa_check_status() == fa.FA_OK
    return dq, dk, dv


SMALL = [
    # B, H, Lq, Lk, d, causal
    (1, 1, 1, 1, 64, False),
    (1, 2, 17, 17, 64, True),
    (2, 2, 130, 130, 128, True),
    (1, 1, 256, 256, 128, False),
    (1, 2, 384, 384, 128, True),
    (1, 1, 100, 300, 128, True),   # bottom-right causal
    (1, 1, 300, 100, 64, False),
    (1, 1, 200, 333, 64, True),
    (2, 1, 520, 520, 128, True),
    # head dimension 256 (dK/dV by halves of d, 64-query and 64-key tiles)
    (1, 1, 3, 3, 256, True),       # (a single key gives dQ = 0 exactly: no relative error to grade)
    (1, 2, 70, 70, 256, True),
    (2, 1, 200, 200, 256, False),
    (1, 1, 100, 300, 256, True),   # bottom-right causal
    (1, 1, 300, 130, 256, False),
    (1, 2, 384, 384, 256, True),
]


@pytest.mark.parametrize("B,H,Lq,Lk,d,causal", SMALL)
def test_backward_small_shapes(cuda_device, B, H, Lq, Lk, d, causal):
    inp = attention_inputs(B, H, Lq, Lk, d, seed=300 + Lq + Lk + d, with_dO=True)
    scale = 1.0 / math.sqrt(d)
    dq_r, dk_r, dv_r, _ = oracle.backward(inp.q, inp.k, inp.v, inp.dO, scale, causal)
    for o_dtype in (torch.float32, torch.bfloat16):
        dq, dk, dv = gpu_fwd_bwd(inp, scale, causal, cuda_device, o_dtype)
        check_grad(dq, dq_r, "dQ")
        check_grad(dk, dk_r, "dK")
        check_grad(dv, dv_r, "dV")


def test_backward_invariants_and_determinism(cuda_device):
    """sum_j dK_j = 0 and sum_j dV_j = sum_i dO_i hold for the GPU outputs; two
    runs give bitwise identical gradients (no atomics anywhere)."""
    inp = attention_inputs(1, 2, 640, 640, 128, seed=9, with_dO=True)
    scale = 1.0 / math.sqrt(128)
    dq, dk, dv = gpu_fwd_bwd(inp, scale, True, cuda_device)
    dq2, dk2, dv2 = gpu_fwd_bwd(inp, scale, True, cuda_device)
    assert torch.equal(dq, dq2) and torch.equal(dk, dk2) and torch.equal(dv, dv2)
    dk_sum = to_np(dk).sum(axis=2)
    assert np.abs(dk_sum).max() <= 2e-2 * np.abs(to_np(dk)).sum(axis=2).max()
    dv_sum = to_np(dv).sum(axis=2)
    g_sum = inp.dO.double().numpy().sum(axis=2)
    assert rel_fro(dv_sum, g_sum) < 1e-2


@pytest.mark.slow
def test_backward_full_size_sampled_heads(cuda_device):
    """The training workload (B=2, H=16, L=8192, d=128, causal) as the benchmark
    times it; the oracle runs the full backward of two heads (heads are
    independent), and properties that hold at any size are checked on all."""
    w = WORKLOADS["train_L8192"]
    B, H, L, d = w["B"], w["H"], w["L"], w["d"]
    inp = attention_inputs(B, H, L, L, d, seed=w["seed"], q_scale=w["q_scale"], with_dO=True)
    scale = 1.0 / math.sqrt(d)
    dev = cuda_device
    q, k, v, g = (t.to(dev) for t in (inp.q, inp.k, inp.v, inp.dO))
    o, lse = fa.forward(q, k, v, scale=scale, causal=True)
    ws = fa.workspace(fa.fa_backward_workspace_size(B, H, L, L, d), dev)
    torch.cuda.synchronize()
    torch.cuda.reset_peak_memory_stats()
    base = torch.cuda.memory_allocated()
    dq, dk, dv = fa.backward(q, k, v, o, g, lse, scale=scale, causal=True, ws=ws)
    torch.cuda.synchronize()
    grown = torch.cuda.max_memory_allocated() - base
    assert fa.fa_check_status() == fa.FA_OK
    assert grown <= 3 * q.numel() * 2 + (1 << 20)  # the three gradients only
    for t in (dq, dk, dv):
        assert torch.isfinite(t).all()
    for (b, h) in ((0, 0), (1, H - 1)):
        sl = (slice(b, b + 1), slice(h, h + 1))
        dq_r, dk_r, dv_r, _ = oracle.backward(inp.q[sl], inp.k[sl], inp.v[sl], inp.dO[sl], scale, True)
        check_grad(dq[sl], dq_r, "dQ b=%d h=%d" % (b, h))
        check_grad(dk[sl], dk_r, "dK b=%d h=%d" % (b, h))
        check_grad(dv[sl], dv_r, "dV b=%d h=%d" % (b, h))
    dv_sum = dv.double().sum(dim=2).cpu().numpy()
    g_sum = inp.dO.double().sum(dim=2).numpy()
    assert rel_fro(dv_sum, g_sum) < 1e-2


def test_backward_d256_full_size_sampled_heads(cuda_device):
    """The d = 256 workload (B=4, H=16, L=4096, causal) as the benchmark times it;
    the oracle runs the full backward of two heads, and properties that hold at
    any size are checked on all."""
    w = WORKLOADS["fwd_d256_L4096"]
    B, H, L, d = w["B"], w["H"], w["L"], w["d"]
    inp = attention_inputs(B, H, L, L, d, seed=w["seed"], q_scale=w["q_scale"], with_dO=True)
    scale = 1.0 / math.sqrt(d)
    dev = cuda_device
    q, k, v, g = (t.to(dev) for t in (inp.q, inp.k, inp.v, inp.dO))
    o, lse = fa.forward(q, k, v, scale=scale, causal=True)
    ws = fa.workspace(fa.fa_backward_workspace_size(B, H, L, L, d), dev)
    torch.cuda.synchronize()
    torch.cuda.reset_peak_memory_stats()
    base = torch.cuda.memory_allocated()
    dq, dk, dv = fa.backward(q, k, v, o, g, lse, scale=scale, causal=True, ws=ws)
    torch.cuda.synchronize()
    grown = torch.cuda.max_memory_allocated() - base
    assert fa.fa_check_status() == fa.FA_OK
    assert grown <= 3 * q.numel() * 2 + (1 << 20)  # the three gradients only
    for t in (dq, dk, dv):
        assert torch.isfinite(t).all()
    for (b, h) in ((0, 1), (B - 1, H - 2)):
        sl = (slice(b, b + 1), slice(h, h + 1))
        dq_r, dk_r, dv_r, _ = oracle.backward(inp.q[sl], inp.k[sl], inp.v[sl], inp.dO[sl], scale, True)
        check_grad(dq[sl], dq_r, "dQ b=%d h=%d" % (b, h))
        check_grad(dk[sl], dk_r, "dK b=%d h=%d" % (b, h))
        check_grad(dv[sl], dv_r, "dV b=%d h=%d" % (b, h))
    # the sum over keys of dV equals the sum over queries of dO (the rows of P sum to 1)
    dv_sum = dv.double().sum(dim=2).cpu().numpy()
    g_sum = inp.dO.double().sum(dim=2).numpy()
    assert rel_fro(dv_sum, g_sum) < 1e-2


def test_backward_d256_determinism(cuda_device):
    """d = 256: two runs give bitwise identical gradients (no atomics)."""
    inp = attention_inputs(1, 2, 333, 333, 256, seed=19, with_dO=True)
    scale = 1.0 / 16.0
    a = gpu_fwd_bwd(inp, scale, True, cuda_device)
    b = gpu_fwd_bwd(inp, scale, True, cuda_device)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
