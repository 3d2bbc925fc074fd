"""Pins for the oracle: checks against facts the pages and the mathematics fix.

None of these retype the oracle's formula.  Each case is a closed form, a
limit, a textbook/library routine on a special case, a brute-force finite
difference, an invariant of the definition, or a figure printed on a page.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
from scipy.special import softmax as scipy_softmax

import oracle
from exact_io_aware_94_b200.inputs import attention_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rnd(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


# --- figures printed on the pages -------------------------------------------------------

def test_score_matrix_counts_match_pages():
    """Glossary "Worked example": 4,096^2 = 16,777,216 elements = 32 MiB at 2 B;
    8,192 gives 128 MiB.  "What Is FlashAttention?": 100,000 tokens, 10^10 entries."""
    with open(os.path.join(GOLDEN, "score_matrix_counts.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        n = oracle.score_elements(c["B"], c["H"], c["L"], c["L"])
        assert n == c["elements"]
        if "bytes_at_2_bytes_each" in c:
            assert 2 * n == c["bytes_at_2_bytes_each"]
            assert 2 * n == c["mib"] * 2**20
    assert oracle.score_elements(1, 1, 8192, 8192) == 4 * oracle.score_elements(1, 1, 4096, 4096)


def test_hand_worked_example():
    with open(os.path.join(GOLDEN, "hand_example.json")) as f:
        g = json.load(f)
    o, lse = oracle.forward(np.array(g["q"]), np.array(g["k"]), np.array(g["v"]), g["scale"], g["causal"])
    np.testing.assert_allclose(o, np.array(g["o"]), rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse, np.array(g["lse"]), rtol=0, atol=1e-14)


# --- the definition on special inputs --------------------------------------------------

@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Lq,Lk", [(5, 5), (3, 7), (6, 6)])
def test_identity_values_give_probability_rows(causal, Lq, Lk):
    """With V = I the output rows are the probability rows P_i: they must equal a
    library softmax of the masked scaled scores, sum to 1, be >= 0, and be zero on
    masked keys."""
    d = Lk
    q = rnd((1, 1, Lq, d), 1)
    k = rnd((1, 1, Lk, d), 2)
    v = np.eye(Lk).reshape(1, 1, Lk, d)
    scale = 0.37
    o, lse = oracle.forward(q, k, v, scale, causal)
    P = o[0, 0]
    scores = scale * q[0, 0] @ k[0, 0].T
    for i in range(Lq):
        allowed = np.arange(Lk) <= i + (Lk - Lq) if causal else np.ones(Lk, bool)
        ref = np.zeros(Lk)
        ref[allowed] = scipy_softmax(scores[i, allowed])
        np.testing.assert_allclose(P[i], ref, rtol=0, atol=1e-13)
        assert abs(P[i].sum() - 1.0) < 1e-12
        assert (P[i] >= 0).all()
        assert (P[i][~allowed] == 0).all()
        np.testing.assert_allclose(lse[0, 0, i], np.log(np.exp(scores[i, allowed]).sum()), rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_uniform_scores_give_mean_of_values(causal):
    """Q = 0 makes every permitted score 0, so P is uniform: O_i is the mean of the
    permitted V rows and LSE_i = ln(#permitted)."""
    B, H, L, d = 2, 3, 9, 4
    q = np.zeros((B, H, L, d))
    k = rnd((B, H, L, d), 3)
    v = rnd((B, H, L, d), 4)
    o, lse = oracle.forward(q, k, v, 0.5, causal)
    for i in range(L):
        n = i + 1 if causal else L
        np.testing.assert_allclose(o[:, :, i], v[:, :, :n].mean(axis=2), rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse[:, :, i], math.log(n), rtol=0, atol=1e-13)


def test_dominant_key_returns_its_value_row():
    """q_i = alpha * k_j* with keys nearly orthogonal: as alpha grows, O_i -> v_j*
    and LSE_i -> the dominant scaled score."""
    L, d = 6, 8
    k = np.eye(d)[:L].reshape(1, 1, L, d)  # orthonormal keys
    v = rnd((1, 1, L, d), 5)
    jstar = 3
    errs = []
    for alpha in (5.0, 20.0, 60.0):
        q = np.zeros((1, 1, 1, d))
        q[0, 0, 0] = alpha * k[0, 0, jstar]
        o, lse = oracle.forward(q, k, v, 1.0, False)
        errs.append(np.abs(o[0, 0, 0] - v[0, 0, jstar]).max())
        # closed form: other scores are 0, so LSE = ln(e^alpha + (L-1))
        assert abs(lse[0, 0, 0] - math.log(math.exp(alpha) + (L - 1))) < 1e-12
    assert errs[0] > errs[1] > errs[2]
    assert errs[2] < 1e-20  # other weights are e^-60 of the dominant one


def test_causal_row_zero_and_single_key():
    """Causal row 0 sees only key 0: O_0 = v_0 exactly, LSE_0 = scale * q_0.k_0.
    With Lk = 1 every row (causal or not) returns v_0."""
    B, H, L, d = 1, 2, 7, 5
    q, k, v = rnd((B, H, L, d), 6), rnd((B, H, L, d), 7), rnd((B, H, L, d), 8)
    o, lse = oracle.forward(q, k, v, 0.3, True)
    np.testing.assert_array_equal(o[:, :, 0], v[:, :, 0])
    np.testing.assert_allclose(lse[:, :, 0], 0.3 * np.einsum("bhd,bhd->bh", q[:, :, 0], k[:, :, 0]), atol=1e-14)
    o1, _ = oracle.forward(q, k[:, :, :1], v[:, :, :1], 0.3, False)
    np.testing.assert_array_equal(o1, np.broadcast_to(v[:, :, :1], o1.shape))


def test_bottom_right_causal_alignment():
    """Lq < Lk under the causal mask: the last query row sees every key, the first
    sees Lk - Lq + 1 keys (query i sits at absolute position i + Lk - Lq)."""
    assert oracle.permitted_keys(0, 3, 10, True) == 8
    assert oracle.permitted_keys(2, 3, 10, True) == 10
    assert oracle.permitted_keys(0, 10, 10, True) == 1
    assert oracle.permitted_keys(4, 10, 10, False) == 10
    q, k, v = rnd((1, 1, 3, 4), 9), rnd((1, 1, 10, 4), 10), rnd((1, 1, 10, 4), 11)
    o_c, _ = oracle.forward(q, k, v, 0.5, True)
    o_full, _ = oracle.forward(q[:, :, 2:], k, v, 0.5, False)
    np.testing.assert_allclose(o_c[:, :, 2], o_full[:, :, 0], atol=1e-14)
    o_pref, _ = oracle.forward(q[:, :, :1], k[:, :, :8], v[:, :, :8], 0.5, False)
    np.testing.assert_allclose(o_c[:, :, 0], o_pref[:, :, 0], atol=1e-14)


def test_symmetries():
    """Non-causal: permuting keys together with their values leaves O unchanged;
    scaling V by alpha scales O by alpha; LSE is unchanged by either."""
    q, k, v = rnd((1, 2, 5, 6), 12), rnd((1, 2, 9, 6), 13), rnd((1, 2, 9, 6), 14)
    o, lse = oracle.forward(q, k, v, 0.4, False)
    perm = np.random.default_rng(0).permutation(9)
    o2, lse2 = oracle.forward(q, k[:, :, perm], v[:, :, perm], 0.4, False)
    np.testing.assert_allclose(o2, o, atol=1e-13)
    np.testing.assert_allclose(lse2, lse, atol=1e-13)
    o3, lse3 = oracle.forward(q, k, 2.5 * v, 0.4, False)
    np.testing.assert_allclose(o3, 2.5 * o, atol=1e-13)
    np.testing.assert_allclose(lse3, lse, atol=0)


def test_bf16_inputs_read_exactly():
    """bf16 tensors are read as their exact values: same result as the float64 copy."""
    inp = attention_inputs(1, 2, 33, 33, 8, seed=0)
    o_b, l_b = oracle.forward(inp.q, inp.k, inp.v, 0.35, True)
    o_d, l_d = oracle.forward(inp.q.double().numpy(), inp.k.double().numpy(), inp.v.double().numpy(), 0.35, True)
    np.testing.assert_array_equal(o_b, o_d)
    np.testing.assert_array_equal(l_b, l_d)


def test_forward_rows_matches_full():
    q, k, v = rnd((2, 2, 11, 4), 15), rnd((2, 2, 11, 4), 16), rnd((2, 2, 11, 4), 17)
    o, lse = oracle.forward(q, k, v, 0.5, True)
    rows = [0, 5, 10, 11, 30, 43]
    o_r, lse_r = oracle.forward_rows(q, k, v, rows, 0.5, True)
    np.testing.assert_array_equal(o_r, o.reshape(-1, 4)[rows])
    np.testing.assert_array_equal(lse_r, lse.reshape(-1)[rows])


# --- the running-statistics recurrence -------------------------------------------------

@pytest.mark.parametrize("block", [1, 3, 7, 64])
@pytest.mark.parametrize("causal", [False, True])
def test_blockwise_recurrence_equals_two_pass(block, causal):
    """The m / l / O~ recurrence over key blocks (any block size, including ones
    that do not divide L) reproduces the two-pass softmax to rounding."""
    L, d = 37, 8
    q, k, v = rnd((1, 2, L, d), 18, 2.0), rnd((1, 2, L, d), 19), rnd((1, 2, L, d), 20)
    o, lse = oracle.forward(q, k, v, 0.7, causal)
    ob, lseb = oracle.forward_blockwise(q, k, v, 0.7, causal, block)
    np.testing.assert_allclose(ob, o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lseb, lse, rtol=0, atol=1e-12)


# --- merge of partial results (split-KV) -----------------------------------------------

def test_merge_of_key_splits_equals_unsplit():
    Lk, d = 23, 5
    q, k, v = rnd((1, 1, 1, d), 21), rnd((1, 1, Lk, d), 22), rnd((1, 1, Lk, d), 23)
    o, lse = oracle.forward(q, k, v, 0.6, False)
    cuts = [0, 4, 5, 17, 23]
    parts = [oracle.forward(q, k[:, :, a:b], v[:, :, a:b], 0.6, False) for a, b in zip(cuts[:-1], cuts[1:])]
    op = np.stack([p[0][0, 0, 0] for p in parts])
    lp = np.array([p[1][0, 0, 0] for p in parts])
    om, lm = oracle.merge(op, lp)
    np.testing.assert_allclose(om, o[0, 0, 0], atol=1e-13)
    assert abs(lm - lse[0, 0, 0]) < 1e-13
    # associativity: merging merged halves gives the same answer
    a = oracle.merge(op[:2], lp[:2])
    b = oracle.merge(op[2:], lp[2:])
    o2, l2 = oracle.merge(np.stack([a[0], b[0]]), np.array([a[1], b[1]]))
    np.testing.assert_allclose(o2, om, atol=1e-13)
    assert abs(l2 - lm) < 1e-13
    # an empty part (LSE = -inf) contributes nothing
    o3, l3 = oracle.merge(np.vstack([op, np.zeros((1, d))]), np.append(lp, -np.inf))
    np.testing.assert_allclose(o3, om, atol=1e-15)


def test_decode_equals_forward_over_prefix_and_edge_lengths():
    B, H, cap, d = 3, 2, 16, 4
    q, kc, vc = rnd((B, H, d), 24), rnd((B, H, cap, d), 25), rnd((B, H, cap, d), 26)
    lens = np.array([16, 1, 0], np.int32)
    o, lse = oracle.decode(q, kc, vc, lens, 0.5)
    o_f, lse_f = oracle.forward(q[0][None, :, None], kc[0][None], vc[0][None], 0.5, False)
    np.testing.assert_allclose(o[0], o_f[0, :, 0], atol=1e-14)
    np.testing.assert_allclose(lse[0], lse_f[0, :, 0], atol=1e-14)
    np.testing.assert_array_equal(o[1], vc[1, :, 0])  # one key: its value row
    np.testing.assert_allclose(lse[1], 0.5 * np.einsum("hd,hd->h", q[1], kc[1, :, 0]), atol=1e-14)
    assert (o[2] == 0).all() and np.isneginf(lse[2]).all()  # empty cache


# --- backward --------------------------------------------------------------------------

@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Lq,Lk", [(6, 6), (4, 7)])
def test_backward_matches_finite_differences(causal, Lq, Lk):
    """Central differences (eps = 1e-6, double) of f = sum(G * O) with respect to
    every entry of Q, K and V match dQ, dK, dV to 1e-6 relative; also with fewer
    queries than keys (bottom-right causal alignment)."""
    B, H, d = 1, 2, 3
    q, k, v = rnd((B, H, Lq, d), 27), rnd((B, H, Lk, d), 28), rnd((B, H, Lk, d), 29)
    G = rnd((B, H, Lq, d), 30)
    scale = 0.8
    dq, dk, dv, _ = oracle.backward(q, k, v, G, scale, causal)

    def f(args):
        return float((G * oracle.forward(args["q"], args["k"], args["v"], scale, causal)[0]).sum())

    eps = 1e-6
    base = {"q": q, "k": k, "v": v}
    for name, grad in (("q", dq), ("k", dk), ("v", dv)):
        x = base[name]
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            num[idx] = (f({**base, name: xp}) - f({**base, name: xm})) / (2 * eps)
        rel = np.linalg.norm(num - grad) / np.linalg.norm(grad)
        assert rel < 1e-6, (name, rel)


@pytest.mark.parametrize("causal", [False, True])
def test_backward_invariants(causal):
    """sum_j dS_ij = 0 gives sum_j dK_j = 0; sum_j P_ij = 1 gives
    sum_j dV_j = sum_i dO_i; D_i = dO_i . O_i."""
    B, H, L, d = 2, 2, 13, 4
    q, k, v, g = (rnd((B, H, L, d), s) for s in (31, 32, 33, 34))
    dq, dk, dv, D = oracle.backward(q, k, v, g, 0.45, causal)
    o, _ = oracle.forward(q, k, v, 0.45, causal)
    np.testing.assert_allclose(dk.sum(axis=2), 0.0, atol=1e-12)
    np.testing.assert_allclose(dv.sum(axis=2), g.sum(axis=2), atol=1e-12)
    np.testing.assert_allclose(D, (g * o).sum(axis=3), atol=1e-12)


def test_backward_single_key_closed_form():
    """Lk = 1: O_i = v_0 whatever Q and K are, so dQ = dK = 0 and dV_0 = sum_i dO_i."""
    q, k, v, g = rnd((1, 1, 4, 3), 35), rnd((1, 1, 1, 3), 36), rnd((1, 1, 1, 3), 37), rnd((1, 1, 4, 3), 38)
    dq, dk, dv, _ = oracle.backward(q, k, v, g, 0.9, False)
    np.testing.assert_allclose(dq, 0.0, atol=1e-15)
    np.testing.assert_allclose(dk, 0.0, atol=1e-15)
    np.testing.assert_allclose(dv[0, 0, 0], g[0, 0].sum(axis=0), atol=1e-14)


# ----------------------------------------------------------------------------- paged, grouped-head decode
def _paged_from_cache(kc, vc, page_size, order):
    """Cut contiguous caches [B, Hkv, cap, d] into pages [B*nblk, Hkv, page_size, d]; page
    order[b*nblk + blk] holds block blk of sequence b.  Returns (kpages, vpages, table)."""
    B, Hkv, cap, d = kc.shape
    nblk = cap // page_size
    kp = torch.empty((B * nblk, Hkv, page_size, d), dtype=kc.dtype)
    vp = torch.empty_like(kp)
    table = np.zeros((B, nblk), np.int32)
    for b in range(B):
        for blk in range(nblk):
            pg = int(order[b * nblk + blk])
            kp[pg] = kc[b, :, blk * page_size:(blk + 1) * page_size]
            vp[pg] = vc[b, :, blk * page_size:(blk + 1) * page_size]
            table[b, blk] = pg
    return kp, vp, table


@pytest.mark.parametrize("permute", [False, True])
def test_paged_decode_equals_contiguous_decode(permute):
    """With one KV head per query head, gathering through the block table must give
    exactly the contiguous-cache decode, whatever order the pages are stored in."""
    g = torch.Generator("cpu").manual_seed(11)
    B, H, cap, d, ps = 3, 2, 48, 8, 16
    kc = torch.randn(B, H, cap, d, generator=g).to(torch.bfloat16)
    vc = torch.randn(B, H, cap, d, generator=g).to(torch.bfloat16)
    q = torch.randn(B, H, d, generator=g).to(torch.bfloat16)
    lens = np.array([1, 31, 48], np.int32)  # single key, mid-page end, full capacity
    order = np.random.default_rng(3).permutation(B * cap // ps) if permute else np.arange(B * cap // ps)
    kp, vp, table = _paged_from_cache(kc, vc, ps, order)
    o_p, l_p = oracle.decode_paged(q, kp, vp, table, lens, 0.3)
    o_c, l_c = oracle.decode(q, kc, vc, lens, 0.3)
    assert np.max(np.abs(o_p - o_c)) <= 1e-12
    assert np.max(np.abs(l_p - l_c)) <= 1e-12


def test_paged_decode_grouped_heads_equal_replicated_cache():
    """Query head h reads KV head h // (H // Hkv): equal to a contiguous decode whose
    cache repeats each KV head for its group of query heads."""
    g = torch.Generator("cpu").manual_seed(12)
    B, H, Hkv, cap, d, ps = 2, 8, 2, 32, 8, 8
    kc = torch.randn(B, Hkv, cap, d, generator=g).to(torch.bfloat16)
    vc = torch.randn(B, Hkv, cap, d, generator=g).to(torch.bfloat16)
    q = torch.randn(B, H, d, generator=g).to(torch.bfloat16)
    lens = np.array([29, 17], np.int32)
    kp, vp, table = _paged_from_cache(kc, vc, ps, np.random.default_rng(5).permutation(B * cap // ps))
    o_p, l_p = oracle.decode_paged(q, kp, vp, table, lens, 0.25)
    group = H // Hkv
    kr = kc.repeat_interleave(group, dim=1)  # [B, H, cap, d]: head h holds KV head h // group
    vr = vc.repeat_interleave(group, dim=1)
    o_c, l_c = oracle.decode(q, kr, vr, lens, 0.25)
    assert np.max(np.abs(o_p - o_c)) <= 1e-12
    assert np.max(np.abs(l_p - l_c)) <= 1e-12
    # heads of one group see the same keys but different queries: results differ across the group
    assert np.max(np.abs(o_p[:, 0] - o_p[:, 1])) > 1e-3


def test_paged_decode_unused_slots_and_errors():
    g = torch.Generator("cpu").manual_seed(13)
    B, H, Hkv, d, ps, nblk = 2, 4, 2, 4, 4, 3
    kp = torch.randn(5, Hkv, ps, d, generator=g).to(torch.bfloat16)
    vp = torch.randn(5, Hkv, ps, d, generator=g).to(torch.bfloat16)
    q = torch.randn(B, H, d, generator=g).to(torch.bfloat16)
    table = np.array([[2, 0, 4], [1, 3, 0]], np.int32)
    lens = np.array([6, 0], np.int32)  # sequence 0 uses blocks 0-1; sequence 1 is empty
    o, l = oracle.decode_paged(q, kp, vp, table, lens, 0.5)
    # entries past the last used block are never read
    t2 = table.copy()
    t2[0, 2] = 10 ** 6
    t2[1, :] = -7
    o2, l2 = oracle.decode_paged(q, kp, vp, t2, lens, 0.5)
    assert np.array_equal(o, o2) and np.array_equal(l, l2)
    # an empty sequence gives O = 0 and LSE = -inf
    assert np.all(o[1] == 0.0) and np.all(np.isneginf(l[1]))
    # a used entry outside [0, num_pages) is an error, and so is H not a multiple of Hkv
    t3 = table.copy()
    t3[0, 1] = 5
    with pytest.raises(ValueError):
        oracle.decode_paged(q, kp, vp, t3, lens, 0.5)
    with pytest.raises(ValueError):
        oracle.decode_paged(torch.randn(B, 3, d).to(torch.bfloat16), kp, vp, table, lens, 0.5)


# ----------------------------------------------------------------------------- packed variable-length forward
def _pack(seqs):
    """[L_b, H, d] tensors -> packed [sum L_b, H, d] and cu_seqlens [B+1]."""
    cu = np.zeros(len(seqs) + 1, np.int32)
    cu[1:] = np.cumsum([s.shape[0] for s in seqs])
    return torch.cat(seqs, 0), cu


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_forward_equals_per_sequence_forward(causal):
    """Each packed sequence is attended to on its own: equal to the batched oracle
    run on that sequence alone (chunked prefill: Lq < Lk, bottom-right causal)."""
    g = torch.Generator("cpu").manual_seed(21)
    H, d = 3, 8
    lq = [5, 1, 0, 17, 9]
    lk = [5, 4, 3, 25, 9] if causal else [7, 1, 2, 11, 9]
    qs = [torch.randn(n, H, d, generator=g).to(torch.bfloat16) for n in lq]
    ks = [torch.randn(n, H, d, generator=g).to(torch.bfloat16) for n in lk]
    vs = [torch.randn(n, H, d, generator=g).to(torch.bfloat16) for n in lk]
    q, cq = _pack(qs)
    k, ck = _pack(ks)
    v, _ = _pack(vs)
    o, lse = oracle.forward_varlen(q, k, v, cq, ck, 0.35, causal)
    for b in range(len(lq)):
        if lq[b] == 0:
            continue
        ob, lb = oracle.forward(qs[b].permute(1, 0, 2)[None].contiguous(), ks[b].permute(1, 0, 2)[None].contiguous(),
                                vs[b].permute(1, 0, 2)[None].contiguous(), 0.35, causal)
        assert np.max(np.abs(o[cq[b]:cq[b + 1]] - ob[0].transpose(1, 0, 2))) <= 1e-12
        assert np.max(np.abs(lse[:, cq[b]:cq[b + 1]] - lb[0])) <= 1e-12


def test_varlen_forward_repacking_permutes_outputs():
    g = torch.Generator("cpu").manual_seed(22)
    H, d = 2, 4
    lens = [3, 6, 2]
    qs = [torch.randn(n, H, d, generator=g).to(torch.bfloat16) for n in lens]
    ks = [torch.randn(n, H, d, generator=g).to(torch.bfloat16) for n in lens]
    vs = [torch.randn(n, H, d, generator=g).to(torch.bfloat16) for n in lens]
    q, cu = _pack(qs)
    o, lse = oracle.forward_varlen(q, _pack(ks)[0], _pack(vs)[0], cu, cu, 0.5, True)
    order = [2, 0, 1]
    q2, cu2 = _pack([qs[i] for i in order])
    o2, lse2 = oracle.forward_varlen(q2, _pack([ks[i] for i in order])[0], _pack([vs[i] for i in order])[0],
                                     cu2, cu2, 0.5, True)
    for new_b, b in enumerate(order):
        assert np.array_equal(o2[cu2[new_b]:cu2[new_b + 1]], o[cu[b]:cu[b + 1]])
        assert np.array_equal(lse2[:, cu2[new_b]:cu2[new_b + 1]], lse[:, cu[b]:cu[b + 1]])
    with pytest.raises(ValueError):
        oracle.forward_varlen(q, _pack(ks)[0], _pack(vs)[0], np.array([0, 5, 4, 11], np.int32), cu, 0.5, True)


# ---- block-sparse forward: the dense rules AND a per-block mask over the score matrix.

def _bs_inputs(seed, B, H, Lq, Lk, d):
    g = torch.Generator("cpu").manual_seed(seed)
    q = torch.randn(B, H, Lq, d, generator=g).to(torch.bfloat16)
    k = torch.randn(B, H, Lk, d, generator=g).to(torch.bfloat16)
    v = torch.randn(B, H, Lk, d, generator=g).to(torch.bfloat16)
    return q, k, v


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("bq,bk", [(3, 5), (4, 4), (11, 1)])
def test_blocksparse_all_ones_equals_dense(causal, bq, bk):
    q, k, v = _bs_inputs(31, 2, 2, 11, 13, 6)
    tq, tk = -(-11 // bq), -(-13 // bk)
    o, lse = oracle.forward_blocksparse(q, k, v, np.ones((tq, tk), np.uint8), 0.4, causal, bq, bk)
    od, ld = oracle.forward(q, k, v, 0.4, causal)
    assert np.array_equal(o, od) and np.array_equal(lse, ld)


def test_blocksparse_one_key_block_per_query_block():
    """Query block r may see key block c(r) = (3r + 1) mod Tk only: its rows equal the dense
    attention of those rows over that key block alone.  An asymmetric pattern, so reading
    the mask transposed, or a block index off by one, fails."""
    bq, bk, Lq, Lk = 4, 3, 14, 17
    tq, tk = -(-Lq // bq), -(-Lk // bk)
    q, k, v = _bs_inputs(32, 1, 2, Lq, Lk, 5)
    mask = np.zeros((tq, tk), np.uint8)
    cols = [(3 * r + 1) % tk for r in range(tq)]
    for r, c in enumerate(cols):
        mask[r, c] = 1
    o, lse = oracle.forward_blocksparse(q, k, v, mask, 0.6, False, bq, bk)
    for r, c in enumerate(cols):
        rows = slice(r * bq, min(Lq, (r + 1) * bq))
        keys = slice(c * bk, min(Lk, (c + 1) * bk))
        od, ld = oracle.forward(q[:, :, rows].contiguous(), k[:, :, keys].contiguous(), v[:, :, keys].contiguous(),
                                0.6, False)
        assert np.max(np.abs(o[:, :, rows] - od)) <= 1e-12
        assert np.max(np.abs(lse[:, :, rows] - ld)) <= 1e-12


def test_blocksparse_complementary_masks_merge_to_dense():
    """Splitting the key set of every row into two disjoint parts (a random block mask and its
    complement) and merging the two results by their log-sum-exps gives the dense result:
    the merge rule of the running statistics ([L] "The Three Running Statistics")."""
    rng = np.random.default_rng(3)
    bq, bk, Lq, Lk = 2, 3, 9, 10
    tq, tk = -(-Lq // bq), -(-Lk // bk)
    q, k, v = _bs_inputs(33, 2, 3, Lq, Lk, 4)
    a = (rng.random((2, 3, tq, tk)) < 0.5).astype(np.uint8)
    oa, la = oracle.forward_blocksparse(q, k, v, a, 0.5, False, bq, bk)
    ob, lb = oracle.forward_blocksparse(q, k, v, 1 - a, 0.5, False, bq, bk)
    od, ld = oracle.forward(q, k, v, 0.5, False)
    lm = np.logaddexp(la, lb)
    wa = np.where(np.isneginf(la), 0.0, np.exp(la - lm))[..., None]
    wb = np.where(np.isneginf(lb), 0.0, np.exp(lb - lm))[..., None]
    assert np.max(np.abs(lm - ld)) <= 1e-12
    assert np.max(np.abs(wa * oa + wb * ob - od)) <= 1e-12


def test_blocksparse_brute_force_per_head_masks_and_causal():
    """Tiny case against an explicit element mask and a full softmax (brute force), with a
    different mask per (b, h), a causal cut with Lq < Lk, and rows left with no key."""
    rng = np.random.default_rng(4)
    B, H, Lq, Lk, d, bq, bk, scale = 2, 2, 7, 10, 3, 2, 4, 0.7
    tq, tk = -(-Lq // bq), -(-Lk // bk)
    q, k, v = _bs_inputs(34, B, H, Lq, Lk, d)
    mask = (rng.random((B, H, tq, tk)) < 0.5).astype(np.uint8)
    mask[0, 1, 0, :] = 0  # rows 0-1 of (b=0, h=1) see nothing
    o, lse = oracle.forward_blocksparse(q, k, v, mask, scale, True, bq, bk)
    qd, kd, vd = (x.double().numpy() for x in (q, k, v))
    for b in range(B):
        for h in range(H):
            for i in range(Lq):
                allowed = [j for j in range(Lk) if j <= i + (Lk - Lq) and mask[b, h, i // bq, j // bk]]
                if not allowed:
                    assert np.all(o[b, h, i] == 0.0) and np.isneginf(lse[b, h, i])
                    continue
                t = np.array([scale * float(qd[b, h, i] @ kd[b, h, j]) for j in allowed])
                w = np.exp(t - t.max())
                ref = (w[:, None] * vd[b, h, allowed]).sum(0) / w.sum()
                assert np.max(np.abs(o[b, h, i] - ref)) <= 1e-12
                assert abs(lse[b, h, i] - (t.max() + np.log(w.sum()))) <= 1e-12
    assert np.isneginf(lse[0, 1, :2]).all()


def test_blocksparse_shared_mask_equals_replicated_and_checks_shape():
    q, k, v = _bs_inputs(35, 2, 3, 8, 8, 4)
    m = (np.random.default_rng(5).random((2, 2)) < 0.6).astype(np.uint8)
    m[:, 0] = 1
    o1, l1 = oracle.forward_blocksparse(q, k, v, m, 0.5, False, 4, 4)
    o2, l2 = oracle.forward_blocksparse(q, k, v, np.broadcast_to(m, (3, 2, 2)), 0.5, False, 4, 4)
    o3, l3 = oracle.forward_blocksparse(q, k, v, np.broadcast_to(m, (2, 3, 2, 2)), 0.5, False, 4, 4)
    assert np.array_equal(o1, o2) and np.array_equal(o1, o3) and np.array_equal(l1, l3)
    with pytest.raises(ValueError):
        oracle.forward_blocksparse(q, k, v, np.ones((2, 3), np.uint8), 0.5, False, 4, 4)
