"""Paged, grouped-head decode vs the oracle on the same bf16 inputs (GPU)."""
import math

import numpy as np
import pytest
import torch

import exact_io_aware_94_b200 as fa
import oracle
from exact_io_aware_94_b200.inputs import WORKLOADS, paged_decode_inputs

from .parity import check_lse, check_o, check_o_bf16

pytestmark = pytest.mark.gpu


def poison_unused_rows(kp, vp, table, lens):
    """NaN in every page row that no valid key uses (whole unused pages, and the
    rows past a sequence's length in its last page): any read of one leaks NaN."""
    ps = kp.shape[2]
    keep = torch.zeros(kp.shape[0], ps, dtype=torch.bool)
    for b, n in enumerate(lens.tolist()):
        for blk in range((n + ps - 1) // ps):
            keep[int(table[b, blk]), : min(ps, n - blk * ps)] = True
    mask = (~keep)[:, None, :, None].expand(-1, kp.shape[1], -1, kp.shape[3]).to(kp.device)
    kp.masked_fill_(mask, float("nan"))
    vp.masked_fill_(mask, float("nan"))


def make_inputs(B, H, Hkv, ps, max_blocks, d, seed, lens):
    """Seeded paged inputs whose table covers the given lengths."""
    cap = ps * max_blocks
    inp = paged_decode_inputs(B, H, Hkv, ps, max_blocks, d, seed=seed, len_lo=cap, len_hi=cap, spare_pages=3)
    return inp.q, inp.kpages, inp.vpages, inp.block_table, torch.tensor(lens, dtype=torch.int32)


@pytest.mark.parametrize("d,H,Hkv,ps,max_blocks", [
    (128, 8, 8, 16, 160),   # one query head per KV head
    (128, 8, 4, 64, 40),    # groups of 2
    (128, 8, 2, 64, 40),    # groups of 4
    (128, 16, 2, 32, 80),   # groups of 8: two head groups per KV head
    (64, 6, 2, 1, 2600),    # groups of 3, one key per page
    (64, 8, 2, 128, 20),    # groups of 4 at d = 64
    (256, 8, 2, 64, 40),    # groups of 4 at d = 256 (two-stage ring)
    (256, 6, 3, 16, 160),   # groups of 2 at d = 256
])
def test_decode_paged_parity_edge_lengths(cuda_device, d, H, Hkv, ps, max_blocks):
    cap = ps * max_blocks
    lens = [1, max(1, ps - 1), ps, ps + 1, 1025, cap, 0]  # page edges, a chunk edge, full, empty
    B = len(lens)
    q, kp, vp, table, lens_t = make_inputs(B, H, Hkv, ps, max_blocks, d, seed=40 + d + H + ps, lens=lens)
    scale = 1.0 / math.sqrt(d)
    o_ref, lse_ref = oracle.decode_paged(q, kp, vp, table.numpy(), lens_t.numpy(), scale)
    dev = cuda_device
    kpd, vpd = kp.to(dev), vp.to(dev)
    poison_unused_rows(kpd, vpd, table, lens_t)
    for out_dtype in (torch.float32, torch.bfloat16):
        o, lse = fa.decode_paged(q.to(dev), kpd, vpd, table.to(dev), lens_t.to(dev), scale=scale,
                                 out_dtype=out_dtype)
        assert fa.fa_check_status() == fa.FA_OK
        if out_dtype == torch.float32:
            check_o(o, o_ref, "paged decode O")
        else:
            check_o_bf16(o, o_ref, "paged decode bf16 O")
        check_lse(lse, lse_ref, "paged decode LSE")
    assert (o[B - 1] == 0).all() and torch.isneginf(lse[B - 1]).all()


def test_decode_paged_bad_page_is_flagged(cuda_device):
    """A table entry outside the pool is flagged and read as page 0; nothing faults."""
    B, H, Hkv, ps, max_blocks, d = 2, 4, 2, 16, 8, 128
    q, kp, vp, table, lens = make_inputs(B, H, Hkv, ps, max_blocks, d, seed=9, lens=[40, 20])
    bad = table.clone()
    bad[0, 1] = kp.shape[0] + 1000
    dev = cuda_device
    o, lse = fa.decode_paged(q.to(dev), kp.to(dev), vp.to(dev), bad.to(dev), lens.to(dev))
    assert fa.fa_check_status() == fa.FA_ERR_PAGE
    assert fa.fa_check_status() == fa.FA_OK
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()
    # the sequence whose table is intact is unaffected
    o_ref, lse_ref = oracle.decode_paged(q[1:], kp, vp, table[1:].numpy(), lens[1:].numpy(), 1.0 / math.sqrt(d))
    check_o(o[1:], o_ref)
    check_lse(lse[1:], lse_ref)


@pytest.mark.slow
def test_decode_paged_full_size_sampled_sequences(cuda_device):
    """The paged, grouped-head workload the benchmark times (B=64, H=32, Hkv=8,
    64-token pages in shuffled order, lengths U[1024, 32768]); unused page rows
    poisoned; a seeded sample of sequences compared with the oracle in full."""
    w = WORKLOADS["decode_paged_gqa"]
    inp = paged_decode_inputs(w["B"], w["H"], w["Hkv"], w["page_size"], w["max_blocks"], w["d"], seed=w["seed"],
                              len_lo=w["len_lo"], len_hi=w["len_hi"])
    dev = cuda_device
    kp, vp = inp.kpages.to(dev), inp.vpages.to(dev)
    poison_unused_rows(kp, vp, inp.block_table, inp.kv_lens)
    scale = 1.0 / math.sqrt(w["d"])
    o, lse = fa.decode_paged(inp.q.to(dev), kp, vp, inp.block_table.to(dev), inp.kv_lens.to(dev), scale=scale)
    assert fa.fa_check_status() == fa.FA_OK
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()
    sel = np.sort(np.random.default_rng(1).choice(w["B"], size=6, replace=False))
    o_ref, lse_ref = oracle.decode_paged(inp.q[sel], inp.kpages, inp.vpages, inp.block_table[sel].numpy(),
                                         inp.kv_lens[sel].numpy(), scale)
    check_o(o.cpu()[sel], o_ref, "paged decode (sampled sequences)")
    check_lse(lse.cpu()[sel], lse_ref, "paged decode (sampled sequences)")
