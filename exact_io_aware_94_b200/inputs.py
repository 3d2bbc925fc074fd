"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module draws random numbers and nothing else: it holds none of the
attention arithmetic, so the GPU library and the oracle can both be fed from it
without sharing any computation.

Recipe (one ``torch.Generator('cpu')`` per workload, seeded with the workload's
seed): draw, in this order, the per-sequence cache lengths (decode only), then
Q, K, V and, for the backward, dO, each as float32 N(0, 1) of the full tensor
shape; multiply Q by ``q_scale`` (4 for the peaky-row workload); round every
tensor to bfloat16 with round-to-nearest-even (``Tensor.to``).  Layout is
contiguous [B, H, L, d]; caches are [B, H, cap, d].
"""
from __future__ import annotations

from dataclasses import dataclass

import torch


@dataclass
class AttentionInputs:
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    dO: torch.Tensor | None = None


@dataclass
class DecodeInputs:
    q: torch.Tensor
    kcache: torch.Tensor
    vcache: torch.Tensor
    kv_lens: torch.Tensor


def _normal(gen: torch.Generator, shape) -> torch.Tensor:
    return torch.randn(*shape, generator=gen, dtype=torch.float32)


def attention_inputs(B: int, H: int, Lq: int, Lk: int, d: int, seed: int, q_scale: float = 1.0,
                     with_dO: bool = False) -> AttentionInputs:
    """bf16 CPU tensors Q [B,H,Lq,d], K/V [B,H,Lk,d] (and dO [B,H,Lq,d])."""
    gen = torch.Generator("cpu").manual_seed(seed)
    q = (_normal(gen, (B, H, Lq, d)) * q_scale).to(torch.bfloat16)
    k = _normal(gen, (B, H, Lk, d)).to(torch.bfloat16)
    v = _normal(gen, (B, H, Lk, d)).to(torch.bfloat16)
    dO = _normal(gen, (B, H, Lq, d)).to(torch.bfloat16) if with_dO else None
    return AttentionInputs(q, k, v, dO)


def decode_inputs(B: int, H: int, cap: int, d: int, seed: int, len_lo: int, len_hi: int) -> DecodeInputs:
    """Decode workload: kv_lens ~ U{len_lo..len_hi} (int32 [B]), q [B,H,d], caches [B,H,cap,d].

    Every cache slot holds N(0,1) data, including slots past a sequence's
    length (a poison test overwrites those separately).
    """
    gen = torch.Generator("cpu").manual_seed(seed)
    kv_lens = torch.randint(len_lo, len_hi + 1, (B,), generator=gen, dtype=torch.int64).to(torch.int32)
    q = _normal(gen, (B, H, d)).to(torch.bfloat16)
    kc = torch.empty((B, H, cap, d), dtype=torch.bfloat16)
    vc = torch.empty((B, H, cap, d), dtype=torch.bfloat16)
    # Drawn one sequence at a time to bound the float32 temporaries.
    for b in range(B):
        kc[b] = _normal(gen, (H, cap, d)).to(torch.bfloat16)
    for b in range(B):
        vc[b] = _normal(gen, (H, cap, d)).to(torch.bfloat16)
    return DecodeInputs(q, kc, vc, kv_lens)


@dataclass
class VarlenInputs:
    q: torch.Tensor       # [total_q, H, d] bf16
    k: torch.Tensor       # [total_k, H, d] bf16
    v: torch.Tensor       # [total_k, H, d] bf16
    cu_q: torch.Tensor    # int32 [B+1]
    cu_k: torch.Tensor    # int32 [B+1]


def varlen_inputs(lens_q, lens_k, H: int, d: int, seed: int) -> VarlenInputs:
    """Packed batch: sequence b has lens_q[b] queries and lens_k[b] keys.  Draw order:
    Q, K, V of the packed tensors, N(0,1), bf16."""
    gen = torch.Generator("cpu").manual_seed(seed)
    cu_q = torch.zeros(len(lens_q) + 1, dtype=torch.int32)
    cu_k = torch.zeros(len(lens_k) + 1, dtype=torch.int32)
    cu_q[1:] = torch.cumsum(torch.tensor(lens_q, dtype=torch.int64), 0).to(torch.int32)
    cu_k[1:] = torch.cumsum(torch.tensor(lens_k, dtype=torch.int64), 0).to(torch.int32)
    tq, tk = int(cu_q[-1]), int(cu_k[-1])
    q = _normal(gen, (tq, H, d)).to(torch.bfloat16)
    k = _normal(gen, (tk, H, d)).to(torch.bfloat16)
    v = _normal(gen, (tk, H, d)).to(torch.bfloat16)
    return VarlenInputs(q, k, v, cu_q, cu_k)


@dataclass
class PagedDecodeInputs:
    q: torch.Tensor            # [B, H, d] bf16
    kpages: torch.Tensor       # [num_pages, Hkv, page_size, d] bf16
    vpages: torch.Tensor       # [num_pages, Hkv, page_size, d] bf16
    block_table: torch.Tensor  # int32 [B, max_blocks]
    kv_lens: torch.Tensor      # int32 [B]


def paged_decode_inputs(B: int, H: int, Hkv: int, page_size: int, max_blocks: int, d: int, seed: int,
                        len_lo: int, len_hi: int, spare_pages: int = 0) -> PagedDecodeInputs:
    """Paged decode workload.  Draw order: kv_lens ~ U{len_lo..len_hi}, then a random
    permutation that assigns each used (sequence, block) a distinct page of the pool,
    then q, then K pages and V pages (N(0,1), bf16).  Pages are [num_pages, Hkv,
    page_size, d]; table slots past a sequence's last used block point at page 0, and
    the pool has `spare_pages` pages that no sequence uses."""
    gen = torch.Generator("cpu").manual_seed(seed)
    kv_lens = torch.randint(len_lo, len_hi + 1, (B,), generator=gen, dtype=torch.int64).to(torch.int32)
    used = [(int(n) + page_size - 1) // page_size for n in kv_lens]
    num_pages = max(1, sum(used) + spare_pages)
    perm = torch.randperm(num_pages, generator=gen)
    table = torch.zeros((B, max_blocks), dtype=torch.int32)
    at = 0
    for b in range(B):
        table[b, : used[b]] = perm[at:at + used[b]].to(torch.int32)
        at += used[b]
    q = _normal(gen, (B, H, d)).to(torch.bfloat16)
    kp = torch.empty((num_pages, Hkv, page_size, d), dtype=torch.bfloat16)
    vp = torch.empty((num_pages, Hkv, page_size, d), dtype=torch.bfloat16)
    chunk = max(1, (1 << 24) // (Hkv * page_size * d))  # bounds the float32 temporaries
    for p0 in range(0, num_pages, chunk):
        p1 = min(num_pages, p0 + chunk)
        kp[p0:p1] = _normal(gen, (p1 - p0, Hkv, page_size, d)).to(torch.bfloat16)
    for p0 in range(0, num_pages, chunk):
        p1 = min(num_pages, p0 + chunk)
        vp[p0:p1] = _normal(gen, (p1 - p0, Hkv, page_size, d)).to(torch.bfloat16)
    return PagedDecodeInputs(q, kp, vp, table, kv_lens)


def blocksparse_mask(H: int, Lq: int, Lk: int, seed: int, sink: int = 1, window: int = 8, p_random: float = 0.1,
                     causal: bool = True, block: int = 128) -> torch.Tensor:
    """uint8 [H, Tq, Tk] block mask (Tq = ceil(Lq/block), Tk = ceil(Lk/block)) for query blocks of
    ``block`` rows and key blocks of ``block`` keys: per head, the first ``sink`` key blocks, the
    ``window`` key blocks ending at the block holding the query block's last permitted key
    (bottom-right causal position; the last key block when not causal), and each other block up to
    there with probability ``p_random`` (one ``torch.rand`` draw per block, generator seeded with
    ``seed``)."""
    tq, tk = -(-Lq // block), -(-Lk // block)
    gen = torch.Generator("cpu").manual_seed(seed)
    draw = torch.rand(H, tq, tk, generator=gen) < p_random
    r = torch.arange(tq)[:, None]
    c = torch.arange(tk)[None, :]
    if causal:
        last = (torch.clamp((r + 1) * block - 1, max=Lq - 1) + (Lk - Lq)) // block
    else:
        last = torch.full_like(r, tk - 1)
    reach = c <= last
    keep = (c < sink) | ((c > last - window) & reach) | (draw & reach)
    return keep.to(torch.uint8)


# The workloads the library is measured and checked on.  Shapes and value
# distributions follow the pages' sizes: the 4,096-token example, a training
# shape at 8,192, a 65,536-token context and a decode batch over a long cache.
WORKLOADS = {
    "tiny_fwd": dict(kind="fwd", B=1, H=2, L=256, d=64, causal=False, q_scale=1.0, seed=1),
    "fwd_L4096_peaky": dict(kind="fwd", B=4, H=16, L=4096, d=128, causal=True, q_scale=4.0, seed=2),
    "train_L8192": dict(kind="fwdbwd", B=2, H=16, L=8192, d=128, causal=True, q_scale=1.0, seed=3),
    "long_L65536": dict(kind="fwd", B=1, H=8, L=65536, d=128, causal=True, q_scale=1.0, seed=4),
    # Head dimension 256 at the 4,096-token shape.
    "fwd_d256_L4096": dict(kind="fwd", B=4, H=16, L=4096, d=256, causal=True, q_scale=1.0, seed=9),
    "decode_cap32768": dict(kind="decode", B=64, H=32, cap=32768, d=128, len_lo=1024, len_hi=32768, seed=5),
    # Packed prefill batch of 16 causal sequences of 512 to 8,192 tokens.
    "prefill_varlen": dict(kind="varlen", B=16, H=16, d=128, len_lo=512, len_hi=8192, causal=True, seed=7),
    # Causal prefill under a block-sparse mask (one mask per head, shared by the batch): an
    # attention-sink block, a local window of 8 key blocks ending at the diagonal, and 10% of
    # the other blocks below the diagonal at random.
    "prefill_blocksparse": dict(kind="blocksparse", B=2, H=16, L=16384, d=128, causal=True, sink=1, window=8,
                                p_random=0.1, seed=8),
    # Paged cache with grouped heads: the same batch and lengths as the decode workload,
    # 8 KV heads shared by groups of 4 query heads, 64-token pages in shuffled order.
    "decode_paged_gqa": dict(kind="decode_paged", B=64, H=32, Hkv=8, page_size=64, max_blocks=512, d=128,
                             len_lo=1024, len_hi=32768, seed=6),
}
