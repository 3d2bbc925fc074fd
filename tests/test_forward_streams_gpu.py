"""Forward calls running at the same time on different streams, and forward calls
captured into a CUDA graph and replayed on several streams at once.

The forward kernels hand out their work units from a per-stream counter that the
last block of each call returns to zero; under graph capture they deal the units
statically instead.  These tests run the cases in which a shared counter would
skip or repeat units: many short calls overlapping a long one, and concurrent
replays of one graph.  Outputs are prefilled with NaN, so a unit that no CTA
computed shows."""
import math

import numpy as np
import pytest
import torch

import exact_io_aware_94_b200 as fa
import oracle
from exact_io_aware_94_b200.inputs import attention_inputs

from .parity import check_lse, check_o, sample_rows

pytestmark = pytest.mark.gpu


def _call(q, k, v, o, lse, causal, stream):
    B, H, L, d = q.shape
    rc = fa.fa_forward(q, k, v, o, lse, B, H, L, k.shape[2], d, 1.0 / math.sqrt(d), int(causal), fa.FA_DT_F32,
                       stream)
    assert rc == fa.FA_OK


def test_short_forwards_overlapping_a_long_one(cuda_device):
    dev = cuda_device
    gen = torch.Generator(device=dev).manual_seed(12)
    Bl, Hl, Ll, d = 1, 16, 65536, 128
    ql, kl, vl = (torch.randn(Bl, Hl, Ll, d, generator=gen, device=dev).to(torch.bfloat16) for _ in range(3))
    ol = torch.full((Bl, Hl, Ll, d), float("nan"), dtype=torch.float32, device=dev)
    lsel = torch.full((Bl, Hl, Ll), float("nan"), dtype=torch.float32, device=dev)
    inp = attention_inputs(1, 2, 256, 256, d, seed=13)
    qs, ks, vs = (t.to(dev) for t in (inp.q, inp.k, inp.v))
    n_short = 300  # more than the 256 per-device counters
    outs = [(torch.full((1, 2, 256, d), float("nan"), dtype=torch.float32, device=dev),
             torch.full((1, 2, 256), float("nan"), dtype=torch.float32, device=dev)) for _ in range(n_short)]
    s_long, s_short = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    torch.cuda.synchronize()
    with torch.cuda.stream(s_long):
        _call(ql, kl, vl, ol, lsel, True, s_long.cuda_stream)  # about 15 ms on a B200
        done = torch.cuda.Event()
        done.record(s_long)
    with torch.cuda.stream(s_short):
        for o, lse in outs:
            _call(qs, ks, vs, o, lse, False, s_short.cuda_stream)
    overlapped = not done.query()  # the long call was still running after the last short one was issued
    torch.cuda.synchronize()
    assert fa.fa_check_status() == fa.FA_OK
    o_ref, lse_ref = oracle.forward(inp.q, inp.k, inp.v, 1.0 / math.sqrt(d), False)
    o0, l0 = outs[0]
    check_o(o0, o_ref, "short forward")
    check_lse(l0, lse_ref, "short forward")
    for o, lse in outs[1:]:
        assert torch.equal(o, o0) and torch.equal(lse, l0)
    assert torch.isfinite(ol).all() and torch.isfinite(lsel).all()
    rows = sample_rows(Bl, Hl, Ll, n_random=64, seed=14)
    qc, kc, vc = (t.cpu() for t in (ql, kl, vl))
    o_ref, lse_ref = oracle.forward_rows(qc, kc, vc, rows, 1.0 / math.sqrt(d), True)
    idx = torch.as_tensor(rows, device=dev)
    check_o(ol.reshape(-1, d)[idx], o_ref, "long forward")
    check_lse(lsel.reshape(-1)[idx], lse_ref, "long forward")
    if not overlapped:
        pytest.skip("the long forward finished before the short ones were issued: nothing overlapped")


def test_graph_replayed_on_two_streams_at_once(cuda_device):
    dev = cuda_device
    B, H, L, d = 2, 4, 1024, 128
    inp = attention_inputs(B, H, L, L, d, seed=15)
    q, k, v = (t.to(dev) for t in (inp.q, inp.k, inp.v))
    o = torch.empty(B, H, L, d, dtype=torch.float32, device=dev)
    lse = torch.empty(B, H, L, dtype=torch.float32, device=dev)
    _call(q, k, v, o, lse, True, torch.cuda.current_stream().cuda_stream)  # first call outside any capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        _call(q, k, v, o, lse, True, torch.cuda.current_stream().cuda_stream)
    streams = [torch.cuda.Stream(dev), torch.cuda.Stream(dev)]
    o_ref, lse_ref = oracle.forward(inp.q, inp.k, inp.v, 1.0 / math.sqrt(d), True)
    for _ in range(3):
        o.fill_(float("nan"))
        lse.fill_(float("nan"))
        torch.cuda.synchronize()
        for _ in range(8):
            for s in streams:  # replays on the two streams run at the same time
                with torch.cuda.stream(s):
                    g.replay()
        torch.cuda.synchronize()
        assert fa.fa_check_status() == fa.FA_OK
        check_o(o, o_ref, "graph replays")
        check_lse(lse, lse_ref, "graph replays")
    # eager calls on a stream still compute everything after the replays
    o.fill_(float("nan"))
    _call(q, k, v, o, lse, True, streams[0].cuda_stream)
    torch.cuda.synchronize()
    check_o(o, o_ref, "eager call after graph replays")
    del g
    assert np.isfinite(lse.cpu().numpy()).all()
