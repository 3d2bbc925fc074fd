"""Forward kernel vs the oracle on the same bf16 inputs (GPU)."""
import math

import numpy as np
import pytest
import torch

import exact_io_aware_94_b200 as fa
import oracle
from exact_io_aware_94_b200.inputs import WORKLOADS, attention_inputs

from .parity import check_lse, check_o, check_o_bf16, padded_like, sample_rows

pytestmark = pytest.mark.gpu


def run_forward(inp, scale, causal, dev, out_dtype=torch.float32, poison=True):
    q, k, v = (t.to(dev) for t in (inp.q, inp.k, inp.v))
    if poison:
        # inputs padded with NaN past their end, outputs pre-filled with NaN
        qp, _ = padded_like(q.shape, torch.bfloat16, dev)
        kp, _ = padded_like(k.shape, torch.bfloat16, dev)
        vp, _ = padded_like(v.shape, torch.bfloat16, dev)
        qp.copy_(q), kp.copy_(k), vp.copy_(v)
        q, k, v = qp, kp, vp
    B, H, Lq, d = q.shape
    o = torch.full((B, H, Lq, d), float("nan"), dtype=out_dtype, device=dev)
    lse = torch.full((B, H, Lq), float("nan"), dtype=torch.float32, device=dev)
    fa.forward(q, k, v, scale=scale, causal=causal, out=o, lse=lse)
    assert fa.fa_check_status() == fa.FA_OK
    return o, lse


SMALL = [
    # B, H, Lq, Lk, d, causal, q_scale
    (1, 1, 1, 1, 64, False, 1.0),
    (1, 1, 1, 1, 128, True, 1.0),
    (1, 2, 17, 17, 64, True, 1.0),
    (2, 3, 130, 130, 128, True, 1.0),
    (1, 2, 256, 256, 64, False, 1.0),
    (1, 1, 384, 384, 128, True, 4.0),
    (1, 2, 1000, 1000, 128, False, 1.0),
    (1, 1, 100, 300, 128, True, 1.0),     # Lq < Lk: bottom-right causal alignment
    (1, 1, 300, 100, 64, False, 1.0),     # Lq > Lk, non-causal
    (1, 1, 257, 513, 64, True, 4.0),
    (2, 1, 600, 600, 128, True, 8.0),     # very peaky rows
    # head dimension 256 (one 128-row Q tile per unit, 64-key tiles)
    (1, 1, 1, 1, 256, True, 1.0),
    (1, 2, 63, 63, 256, False, 1.0),
    (2, 2, 200, 200, 256, True, 1.0),
    (1, 1, 384, 384, 256, True, 4.0),
    (1, 2, 700, 700, 256, False, 1.0),
    (1, 1, 100, 321, 256, True, 1.0),     # Lq < Lk: bottom-right causal alignment
    (1, 1, 300, 65, 256, False, 1.0),     # Lq > Lk, non-causal
    (1, 1, 520, 520, 256, True, 8.0),     # very peaky rows: rescaling in the split rows
]


@pytest.mark.parametrize("B,H,Lq,Lk,d,causal,qs", SMALL)
def test_forward_small_shapes(cuda_device, B, H, Lq, Lk, d, causal, qs):
    inp = attention_inputs(B, H, Lq, Lk, d, seed=100 + Lq + Lk + d, q_scale=qs)
    scale = 1.0 / math.sqrt(d)
    o_ref, lse_ref = oracle.forward(inp.q, inp.k, inp.v, scale, causal)
    o, lse = run_forward(inp, scale, causal, cuda_device)
    check_o(o, o_ref, "fp32 O")
    check_lse(lse, lse_ref, "LSE")
    o16, lse16 = run_forward(inp, scale, causal, cuda_device, out_dtype=torch.bfloat16)
    check_o_bf16(o16, o_ref, "bf16 O")
    check_lse(lse16, lse_ref, "LSE (bf16 O call)")


def test_forward_tiny_workload_full(cuda_device):
    """B=1, H=2, L=256, d=64, non-causal: every output element against the oracle."""
    w = WORKLOADS["tiny_fwd"]
    inp = attention_inputs(w["B"], w["H"], w["L"], w["L"], w["d"], seed=w["seed"], q_scale=w["q_scale"])
    scale = 1.0 / math.sqrt(w["d"])
    o_ref, lse_ref = oracle.forward(inp.q, inp.k, inp.v, scale, w["causal"])
    o, lse = run_forward(inp, scale, w["causal"], cuda_device)
    check_o(o, o_ref)
    check_lse(lse, lse_ref)


def test_forward_scale_and_value_linearity(cuda_device):
    """Scaling V by 2 (exact in bf16) scales O by 2 and leaves LSE unchanged."""
    inp = attention_inputs(1, 2, 200, 200, 128, seed=7)
    o1, l1 = fa.forward(inp.q.to(cuda_device), inp.k.to(cuda_device), inp.v.to(cuda_device), causal=True)
    o2, l2 = fa.forward(inp.q.to(cuda_device), inp.k.to(cuda_device), (2 * inp.v).to(cuda_device), causal=True)
    torch.testing.assert_close(o2, 2 * o1, rtol=0, atol=1e-5)
    torch.testing.assert_close(l2, l1, rtol=0, atol=0)


@pytest.mark.slow
@pytest.mark.parametrize("name", ["fwd_L4096_peaky", "train_L8192", "long_L65536", "fwd_d256_L4096"])
def test_forward_full_size_sampled_rows(cuda_device, name):
    """Full-size workloads, in the configuration the benchmark times; rows sampled
    (row sampling is exact: each output row depends only on its own query row)."""
    w = WORKLOADS[name]
    B, H, L, d = w["B"], w["H"], w["L"], w["d"]
    inp = attention_inputs(B, H, L, L, d, seed=w["seed"], q_scale=w["q_scale"])
    scale = 1.0 / math.sqrt(d)
    dev = cuda_device
    q, k, v = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev)
    torch.cuda.synchronize()
    before = torch.cuda.max_memory_allocated()
    torch.cuda.reset_peak_memory_stats()
    base = torch.cuda.memory_allocated()
    o, lse = fa.forward(q, k, v, scale=scale, causal=w["causal"])
    torch.cuda.synchronize()
    grown = torch.cuda.max_memory_allocated() - base
    assert fa.fa_check_status() == fa.FA_OK
    # only O (fp32) and LSE are allocated; an L x L score matrix would be B*H*L*L*2 bytes
    assert grown <= o.numel() * 4 + lse.numel() * 4 + (1 << 20), grown
    # far below one bf16 score matrix: the outputs are 2d/L of one (1/8 at d = 256, L = 4,096)
    assert grown * 4 < B * H * L * L * 2
    del before
    rows = sample_rows(B, H, L, n_random=256, seed=w["seed"])
    o_ref, lse_ref = oracle.forward_rows(inp.q, inp.k, inp.v, rows, scale, w["causal"])
    o_s = o.reshape(-1, d)[torch.as_tensor(rows, device=dev)]
    lse_s = lse.reshape(-1)[torch.as_tensor(rows, device=dev)]
    check_o(o_s, o_ref, name)
    check_lse(lse_s, lse_ref, name)
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()
