"""Split-KV decode kernels vs the oracle on the same bf16 inputs (GPU)."""
import math

import numpy as np
import pytest
import torch

import exact_io_aware_94_b200 as fa
import oracle
from exact_io_aware_94_b200.inputs import WORKLOADS, decode_inputs

from .parity import check_lse, check_o, check_o_bf16

pytestmark = pytest.mark.gpu


def poison_past_lengths(kc, vc, lens):
    """Fill every cache slot at or past kv_lens[b] with NaN: any read of one leaks NaN."""
    for b, n in enumerate(lens.tolist()):
        kc[b, :, n:] = float("nan")
        vc[b, :, n:] = float("nan")


@pytest.mark.parametrize("d", [64, 128, 256])
def test_decode_small_with_edge_lengths(cuda_device, d):
    B, H, cap = 6, 3, 5000
    inp = decode_inputs(B, H, cap, d, seed=11 + d, len_lo=1, len_hi=cap)
    lens = torch.tensor([1, 1023, 1024, 1025, cap, 0], dtype=torch.int32)  # chunk edges, full, empty
    scale = 1.0 / math.sqrt(d)
    o_ref, lse_ref = oracle.decode(inp.q, inp.kcache, inp.vcache, lens.numpy(), scale)
    dev = cuda_device
    kc, vc = inp.kcache.to(dev), inp.vcache.to(dev)
    poison_past_lengths(kc, vc, lens)
    for out_dtype in (torch.float32, torch.bfloat16):
        o, lse = fa.decode(inp.q.to(dev), kc, vc, lens.to(dev), scale=scale, out_dtype=out_dtype)
        assert fa.fa_check_status() == fa.FA_OK
        if out_dtype == torch.float32:
            check_o(o, o_ref, "decode O")
        else:
            check_o_bf16(o, o_ref, "decode bf16 O")
        check_lse(lse, lse_ref, "decode LSE")
    assert (o[5] == 0).all() and torch.isneginf(lse[5]).all()


def test_decode_bad_length_is_clamped_and_flagged(cuda_device):
    B, H, cap, d = 2, 2, 2048, 128
    inp = decode_inputs(B, H, cap, d, seed=3, len_lo=1, len_hi=cap)
    lens = torch.tensor([cap + 100, 700], dtype=torch.int32)
    dev = cuda_device
    o, lse = fa.decode(inp.q.to(dev), inp.kcache.to(dev), inp.vcache.to(dev), lens.to(dev))
    assert fa.fa_check_status() == fa.FA_ERR_KV_LEN
    assert fa.fa_check_status() == fa.FA_OK  # reading clears the word
    o_ref, lse_ref = oracle.decode(inp.q, inp.kcache, inp.vcache, np.array([cap, 700], np.int32),
                                   1.0 / math.sqrt(d))
    check_o(o, o_ref)
    check_lse(lse, lse_ref)


@pytest.mark.slow
def test_decode_full_size_sampled_heads(cuda_device):
    """The full decode workload (B=64, H=32, cap=32768, lengths U[1024, 32768]),
    in the configuration the benchmark times, with slots past each length
    poisoned; every head's LSE and output compared on a seeded sample of heads
    (each (b, h) is independent)."""
    w = WORKLOADS["decode_cap32768"]
    B, H, cap, d = w["B"], w["H"], w["cap"], w["d"]
    dev = cuda_device
    gen = torch.Generator("cpu").manual_seed(w["seed"])
    lens = torch.randint(w["len_lo"], w["len_hi"] + 1, (B,), generator=gen).to(torch.int32)
    q = torch.randn(B, H, d, generator=gen).to(torch.bfloat16)
    kc = torch.empty(B, H, cap, d, dtype=torch.bfloat16, device=dev)
    vc = torch.empty(B, H, cap, d, dtype=torch.bfloat16, device=dev)
    # Seeded per sequence, on the host, only up to that sequence's length
    # (slots past it are never read and are poisoned below).
    sel = np.random.default_rng(0).choice(B * H, size=48, replace=False)
    sel_b = sorted(set(int(x) // H for x in sel))
    k_sel, v_sel = {}, {}
    for b in range(B):
        n = int(lens[b])
        kb = torch.randn(H, n, d, generator=gen).to(torch.bfloat16)
        vb = torch.randn(H, n, d, generator=gen).to(torch.bfloat16)
        kc[b, :, :n] = kb.to(dev)
        vc[b, :, :n] = vb.to(dev)
        if b in sel_b:
            k_sel[b], v_sel[b] = kb, vb
    poison_past_lengths(kc, vc, lens)
    scale = 1.0 / math.sqrt(d)
    o, lse = fa.decode(q.to(dev), kc, vc, lens.to(dev), scale=scale)
    assert fa.fa_check_status() == fa.FA_OK
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()
    o_c, lse_c = o.cpu(), lse.cpu()
    for x in sel:
        b, h = int(x) // H, int(x) % H
        n = int(lens[b])
        kk = k_sel[b][h][None, None]
        vv = v_sel[b][h][None, None]
        o_ref, lse_ref = oracle.forward(q[b, h][None, None, None], kk, vv, scale, False)
        check_o(o_c[b, h][None], o_ref[0, 0], "decode b=%d h=%d" % (b, h))
        check_lse(lse_c[b, h][None], lse_ref[0, 0], "decode b=%d h=%d" % (b, h))
