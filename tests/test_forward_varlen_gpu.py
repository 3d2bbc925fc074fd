"""Packed variable-length forward vs the oracle on the same bf16 inputs (GPU)."""
import math

import numpy as np
import pytest
import torch

import exact_io_aware_94_b200 as fa
import oracle
from exact_io_aware_94_b200.inputs import WORKLOADS, varlen_inputs

from .parity import check_lse, check_o, check_o_bf16

pytestmark = pytest.mark.gpu


def run(inp, H, d, causal, out_dtype, dev):
    """Call the library with NaN-prefilled outputs, so any row it fails to write shows."""
    tq, tk = inp.q.shape[0], inp.k.shape[0]
    lens_q = (inp.cu_q[1:] - inp.cu_q[:-1]).tolist()
    o = torch.full((tq, H, d), float("nan"), dtype=out_dtype, device=dev)
    lse = torch.full((H, tq), float("nan"), dtype=torch.float32, device=dev)
    rc = fa.fa_forward_varlen(inp.q.to(dev), inp.k.to(dev), inp.v.to(dev), o, lse, inp.cu_q.to(dev),
                              inp.cu_k.to(dev), len(lens_q), H, tq, tk, max(lens_q), d, 1.0 / math.sqrt(d), causal,
                              fa.FA_DT_F32 if out_dtype == torch.float32 else fa.FA_DT_BF16)
    assert rc == fa.FA_OK
    torch.cuda.synchronize()
    return o, lse


CASES = [
    # lengths of queries, lengths of keys (causal: keys = queries + a cached prefix)
    ([1, 127, 128, 129, 256, 300, 700, 0, 1000], [1, 127, 133, 229, 256, 556, 700, 3, 1024]),
    ([513, 2, 255, 257], [513, 64, 255, 400]),
]


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("case", range(len(CASES)))
def test_varlen_forward_parity(cuda_device, d, causal, case):
    lens_q, lens_k = CASES[case]
    if not causal:
        lens_k = [max(1, n) for n in lens_k[::-1]]  # key lengths independent of the query lengths
    H = 3
    inp = varlen_inputs(lens_q, lens_k, H, d, seed=60 + d + case + 7 * causal)
    o_ref, lse_ref = oracle.forward_varlen(inp.q, inp.k, inp.v, inp.cu_q.numpy(), inp.cu_k.numpy(),
                                           1.0 / math.sqrt(d), causal)
    for out_dtype in (torch.float32, torch.bfloat16):
        o, lse = run(inp, H, d, causal, out_dtype, cuda_device)
        assert fa.fa_check_status() == fa.FA_OK
        if out_dtype == torch.float32:
            check_o(o, o_ref, "varlen O")
        else:
            check_o_bf16(o, o_ref, "varlen bf16 O")
        check_lse(lse, lse_ref, "varlen LSE")


def test_varlen_many_sequences(cuda_device):
    """Forty sequences of random lengths (including empty ones), causal, d = 128:
    many units per CTA, and sequence boundaries inside tiles everywhere."""
    rng = np.random.default_rng(5)
    lens_q = [int(x) for x in rng.integers(0, 400, size=40)]
    lens_k = [n + int(rng.integers(0, 64)) for n in lens_q]
    H, d = 4, 128
    inp = varlen_inputs(lens_q, lens_k, H, d, seed=77)
    o_ref, lse_ref = oracle.forward_varlen(inp.q, inp.k, inp.v, inp.cu_q.numpy(), inp.cu_k.numpy(),
                                           1.0 / math.sqrt(d), True)
    o, lse = run(inp, H, d, True, torch.float32, cuda_device)
    assert fa.fa_check_status() == fa.FA_OK
    check_o(o, o_ref, "varlen O (40 sequences)")
    check_lse(lse, lse_ref, "varlen LSE (40 sequences)")


@pytest.mark.parametrize("d", [64, 256])
def test_varlen_invalid_sequence_is_skipped_and_flagged(cuda_device, d):
    """A causal sequence with more queries than keys is flagged and left unwritten;
    the other sequences are computed as usual."""
    lens_q, lens_k = [100, 50, 200], [100, 20, 200]  # sequence 1: 50 queries, 20 keys
    H = 2
    inp = varlen_inputs(lens_q, lens_k, H, d, seed=8)
    o, lse = run(inp, H, d, True, torch.float32, cuda_device)
    assert fa.fa_check_status() == fa.FA_ERR_SEQLEN
    assert fa.fa_check_status() == fa.FA_OK
    assert torch.isnan(o[100:150]).all()  # the skipped sequence's rows are untouched
    keep = np.r_[0:100, 150:350]
    q_k = torch.cat([inp.q[0:100], inp.q[150:350]])
    k_k = torch.cat([inp.k[0:100], inp.k[120:320]])
    v_k = torch.cat([inp.v[0:100], inp.v[120:320]])
    cu = np.array([0, 100, 300], np.int32)
    o_ref, lse_ref = oracle.forward_varlen(q_k, k_k, v_k, cu, cu, 1.0 / math.sqrt(d), True)
    check_o(o[keep], o_ref, "varlen O (kept sequences)")
    check_lse(lse[:, keep], lse_ref, "varlen LSE (kept sequences)")


@pytest.mark.slow
def test_varlen_benchmark_workload_sampled_rows(cuda_device):
    """The packed prefill batch the benchmark times (16 causal sequences with
    lengths U[512, 8192] from the workload's seed, H16, d128; up to 32 pairs of
    query tiles and 64 key tiles per unit), with O prefilled with NaN: every row
    must be written, and sampled rows of every (sequence, head) must match the
    oracle.  The sample holds each sequence's first and last rows, the rows on
    both sides of the 128- and 256-row tile boundaries of several units, every
    row of the last partial 32-row box (written row by row), and random rows."""
    w = WORKLOADS["prefill_varlen"]
    B, H, d = w["B"], w["H"], w["d"]
    cg = torch.Generator("cpu").manual_seed(w["seed"])
    lens = [int(x) for x in torch.randint(w["len_lo"], w["len_hi"] + 1, (B,), generator=cg)]
    inp = varlen_inputs(lens, lens, H, d, seed=w["seed"])
    o, lse = run(inp, H, d, True, torch.float32, cuda_device)
    assert fa.fa_check_status() == fa.FA_OK
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()
    scale = 1.0 / math.sqrt(d)
    rng = np.random.default_rng(w["seed"])
    cu = inp.cu_q.tolist()
    n_checked = 0
    for b, L in enumerate(lens):
        fixed = {0, 1, L - 1}
        for u in (0, 1, L // 512, (L - 1) // 256):
            for r in (u * 256 - 1, u * 256, u * 256 + 127, u * 256 + 128):
                fixed.add(r)
        fixed.update(range(L - L % 32, L))  # the last partial 32-row box (empty when L % 32 == 0)
        fixed = sorted(r for r in fixed if 0 <= r < L)
        # one sequence as a batched [1, H, L, d] problem for the oracle
        qb, kb, vb = (t[cu[b]:cu[b + 1]].permute(1, 0, 2).unsqueeze(0).contiguous() for t in (inp.q, inp.k, inp.v))
        rows = []
        for h in range(H):
            pick = set(fixed) | set(rng.integers(0, L, size=16).tolist())
            rows += [h * L + r for r in sorted(pick)]
        rows = np.array(rows, dtype=np.int64)
        o_ref, lse_ref = oracle.forward_rows(qb, kb, vb, rows, scale, True)
        h_idx, r_idx = rows // L, rows % L
        tok = torch.as_tensor(cu[b] + r_idx, device=cuda_device)
        hh = torch.as_tensor(h_idx, device=cuda_device)
        check_o(o[tok, hh], o_ref, "varlen benchmark workload O (sequence %d)" % b)
        check_lse(lse[hh, tok], lse_ref, "varlen benchmark workload LSE (sequence %d)" % b)
        n_checked += rows.size
    assert n_checked >= 256 * H
