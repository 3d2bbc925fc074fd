"""Block-sparse forward vs the oracle on the same bf16 inputs (GPU)."""
import math

import numpy as np
import pytest
import torch

import exact_io_aware_94_b200 as fa
import oracle
from exact_io_aware_94_b200.inputs import WORKLOADS, attention_inputs, blocksparse_mask

from .parity import check_lse, check_o, check_o_bf16

pytestmark = pytest.mark.gpu

BLK = fa.BLOCKSPARSE_BLOCK


def tiles(L):
    return -(-L // BLK)


def run_both(inp, mask_dev, mask_np, causal, dev, what):
    """GPU in fp32 and bf16 output against the oracle on the same mask."""
    d = inp.q.shape[-1]
    scale = 1.0 / math.sqrt(d)
    o_ref, lse_ref = oracle.forward_blocksparse(inp.q, inp.k, inp.v, mask_np, scale, causal, BLK, BLK)
    q, k, v = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev)
    for out_dtype in (torch.float32, torch.bfloat16):
        o, lse = fa.forward_blocksparse(q, k, v, mask_dev, scale=scale, causal=causal, out_dtype=out_dtype)
        assert fa.fa_check_status() == fa.FA_OK
        if out_dtype == torch.float32:
            check_o(o, o_ref, what)
        else:
            check_o_bf16(o, o_ref, what + " (bf16 O)")
        check_lse(lse, lse_ref, what)
    return o_ref, lse_ref


@pytest.mark.parametrize("d", [128, 256])
@pytest.mark.parametrize("causal", [True, False])
def test_all_ones_mask_equals_dense_forward_bitwise(cuda_device, causal, d):
    """With every block permitted each query block walks the same key tiles as in the dense
    forward, in the same order, with the same arithmetic: bit-identical output."""
    B, H, L = 1, 2, 700
    inp = attention_inputs(B, H, L, L, d, seed=50)
    q, k, v = inp.q.to(cuda_device), inp.k.to(cuda_device), inp.v.to(cuda_device)
    ones = torch.ones(tiles(L), tiles(L), dtype=torch.uint8, device=cuda_device)
    o, lse = fa.forward_blocksparse(q, k, v, ones, causal=causal)
    od, ld = fa.forward(q, k, v, causal=causal)
    assert fa.fa_check_status() == fa.FA_OK
    assert torch.equal(o, od) and torch.equal(lse, ld)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("Lq,Lk", [(300, 520), (513, 129), (1000, 1000)])
def test_random_per_head_masks_noncausal(cuda_device, d, Lq, Lk):
    """A different random mask per (b, h) (density 1/2), ragged lengths on both sides."""
    B, H = 2, 3
    inp = attention_inputs(B, H, Lq, Lk, d, seed=51 + d + Lq)
    rng = np.random.default_rng(Lq + Lk)
    mask = (rng.random((B, H, tiles(Lq), tiles(Lk))) < 0.5).astype(np.uint8)
    run_both(inp, torch.from_numpy(mask).to(cuda_device), mask, False, cuda_device, "random masks")


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("Lq,Lk", [(1000, 1000), (384, 900)])
def test_sink_window_random_causal(cuda_device, d, Lq, Lk):
    """The benchmark's pattern (sink, local window, random blocks below the diagonal), one mask
    per head shared by the batch, causal with a cached prefix when Lq < Lk."""
    B, H = 2, 3
    inp = attention_inputs(B, H, Lq, Lk, d, seed=52 + d + Lq)
    mask = blocksparse_mask(H, Lq, Lk, seed=9, sink=1, window=2, p_random=0.3, causal=True)
    run_both(inp, mask.to(cuda_device), mask.numpy(), True, cuda_device, "sink/window/random")


@pytest.mark.parametrize("d", [128, 256])
def test_rows_with_no_key_are_zero_with_lse_minus_inf(cuda_device, d):
    """Query blocks whose mask row is empty -- one block of a pair, and a whole 256-row unit --
    get O = 0 and LSE = -inf; so does a causal row block permitted only above its diagonal."""
    B, H, L = 1, 2, 900
    inp = attention_inputs(B, H, L, L, d, seed=53)
    t = tiles(L)
    mask = np.ones((H, t, t), np.uint8)
    mask[0, 1, :] = 0          # head 0: the second block of unit 0 sees nothing
    mask[1, 2:4, :] = 0        # head 1: both blocks of unit 1 see nothing
    mask[1, 5, :] = 0
    mask[1, 5, 6] = 1          # head 1, block 5: only a block above its diagonal (causal removes it)
    o_ref, lse_ref = run_both(inp, torch.from_numpy(mask).to(cuda_device), mask, True, cuda_device, "empty rows")
    assert np.isneginf(lse_ref[0, 0, 128:256]).all() and np.isneginf(lse_ref[0, 1, 256:512]).all()
    o, lse = fa.forward_blocksparse(inp.q.to(cuda_device), inp.k.to(cuda_device), inp.v.to(cuda_device),
                                    torch.from_numpy(mask).to(cuda_device), causal=True)
    assert (o[0, 1, 256:512] == 0).all() and torch.isneginf(lse[0, 1, 640:768]).all()


@pytest.mark.parametrize("d", [128, 256])
def test_blocks_nobody_sees_hold_nan(cuda_device, d):
    """K/V rows of key blocks that no query block may see are NaN.  A unit whose two query
    blocks see nothing still runs one fully masked tile, which may be such a block: its rows
    must still be exactly 0 with LSE = -inf, and every other row must match the oracle."""
    B, H, L = 1, 2, 640
    inp = attention_inputs(B, H, L, L, d, seed=56)
    t = tiles(L)
    mask = np.zeros((H, t, t), np.uint8)
    mask[:, 0:2, 4] = 1  # query blocks 0-1 see key block 4
    mask[:, 4, 3] = 1    # query block 4 sees key block 3; blocks 2-3 (one unit) see nothing
    k, v = inp.k.clone(), inp.v.clone()
    k[:, :, : 3 * BLK] = float("nan")  # key blocks 0-2: seen by nobody
    v[:, :, : 3 * BLK] = float("nan")
    scale = 1.0 / math.sqrt(d)
    o_ref, lse_ref = oracle.forward_blocksparse(inp.q, k, v, mask, scale, False, BLK, BLK)
    o, lse = fa.forward_blocksparse(inp.q.to(cuda_device), k.to(cuda_device), v.to(cuda_device),
                                    torch.from_numpy(mask).to(cuda_device), scale=scale)
    assert fa.fa_check_status() == fa.FA_OK
    assert (o[:, :, 2 * BLK:4 * BLK] == 0).all() and torch.isneginf(lse[:, :, 2 * BLK:4 * BLK]).all()
    check_o(o, o_ref, "NaN in unseen blocks")
    check_lse(lse, lse_ref, "NaN in unseen blocks")


@pytest.mark.parametrize("d", [64, 256])
@pytest.mark.parametrize("causal", [True, False])
def test_all_zero_mask(cuda_device, causal, d):
    """No block permitted anywhere: every unit runs only its one fully masked entry, and every
    row gets O = 0 and LSE = -inf, in both output types."""
    B, H, L = 2, 2, 333
    inp = attention_inputs(B, H, L, L, d, seed=57)
    zeros = torch.zeros(tiles(L), tiles(L), dtype=torch.uint8, device=cuda_device)
    for out_dtype in (torch.float32, torch.bfloat16):
        o, lse = fa.forward_blocksparse(inp.q.to(cuda_device), inp.k.to(cuda_device), inp.v.to(cuda_device), zeros,
                                        causal=causal, out_dtype=out_dtype)
        assert fa.fa_check_status() == fa.FA_OK
        assert (o == 0).all() and torch.isneginf(lse).all()


def test_shared_and_expanded_masks(cuda_device):
    """One [Tq, Tk] mask for every (b, h), and a mask expanded over the batch (stride 0)."""
    B, H, L, d = 2, 2, 640, 64
    inp = attention_inputs(B, H, L, L, d, seed=54)
    rng = np.random.default_rng(7)
    m2 = (rng.random((tiles(L), tiles(L))) < 0.6).astype(np.uint8)
    run_both(inp, torch.from_numpy(m2).to(cuda_device), m2, False, cuda_device, "shared mask")
    m3 = (rng.random((H, tiles(L), tiles(L))) < 0.6).astype(np.uint8)
    dev3 = torch.from_numpy(m3).to(cuda_device)[None].expand(B, -1, -1, -1)
    run_both(inp, dev3, m3, True, cuda_device, "mask expanded over the batch")
    boolmask = torch.from_numpy(m3).to(cuda_device).bool()
    o1, _ = fa.forward_blocksparse(inp.q.to(cuda_device), inp.k.to(cuda_device), inp.v.to(cuda_device), boolmask)
    o2, _ = fa.forward_blocksparse(inp.q.to(cuda_device), inp.k.to(cuda_device), inp.v.to(cuda_device), dev3)
    assert torch.equal(o1, o2)


@pytest.mark.slow
def test_full_size_workload_sampled_query_blocks(cuda_device):
    """The benchmark's block-sparse workload (B=2, H=16, L=16384, causal): seeded query blocks
    of a few heads compared in full with the oracle run on that block alone (its rows, the keys
    up to its diagonal, its mask row: the same permitted keys, bottom-right aligned)."""
    w = WORKLOADS["prefill_blocksparse"]
    B, H, L, d = w["B"], w["H"], w["L"], w["d"]
    inp = attention_inputs(B, H, L, L, d, seed=w["seed"])
    mask = blocksparse_mask(H, L, L, seed=w["seed"], sink=w["sink"], window=w["window"], p_random=w["p_random"])
    dev = cuda_device
    o, lse = fa.forward_blocksparse(inp.q.to(dev), inp.k.to(dev), inp.v.to(dev), mask.to(dev), causal=True)
    assert fa.fa_check_status() == fa.FA_OK
    o, lse = o.cpu(), lse.cpu()
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()
    rng = np.random.default_rng(2)
    picks = [(0, 0, 0), (1, 15, tiles(L) - 1)] + [(int(rng.integers(B)), int(rng.integers(H)),
                                                   int(rng.integers(tiles(L)))) for _ in range(4)]
    scale = 1.0 / math.sqrt(d)
    for b, h, r in picks:
        rows = slice(r * BLK, (r + 1) * BLK)
        keys = slice(0, (r + 1) * BLK)
        qs = inp.q[b:b + 1, h:h + 1, rows].contiguous()
        ks = inp.k[b:b + 1, h:h + 1, keys].contiguous()
        vs = inp.v[b:b + 1, h:h + 1, keys].contiguous()
        m_row = mask[h, r:r + 1, :r + 1].numpy()
        o_ref, lse_ref = oracle.forward_blocksparse(qs, ks, vs, m_row, scale, True, BLK, BLK)
        check_o(o[b:b + 1, h:h + 1, rows], o_ref, "block-sparse (b=%d, h=%d, block %d)" % (b, h, r))
        check_lse(lse[b:b + 1, h:h + 1, rows], lse_ref, "block-sparse (b=%d, h=%d, block %d)" % (b, h, r))
