"""Host-side logic of the benchmark and the input generators (CPU only)."""


def test_blocksparse_pair_count_matches_brute_force():
    """The benchmark's work count for the block-sparse forward against counting every permitted
    (query, key) pair one by one, on ragged lengths, causal (Lq < Lk) and not."""
    import numpy as np

    import bench

    rng = np.random.default_rng(3)
    for Lq, Lk, causal, blk in ((37, 50, True, 8), (37, 50, False, 8), (64, 64, True, 16), (5, 9, True, 4)):
        tq, tk = -(-Lq // blk), -(-Lk // blk)
        mask = (rng.random((2, tq, tk)) < 0.6).astype(np.uint8)
        want = 0
        for h in range(2):
            for i in range(Lq):
                for j in range(Lk):
                    if mask[h, i // blk, j // blk] and (not causal or j <= i + Lk - Lq):
                        want += 1
        assert bench.blocksparse_pairs(mask, Lq, Lk, causal, blk) == want
    # the benchmark's shape: a full causal mask at L = 16384 counts L (L + 1) / 2 pairs
    t = 16384 // 128
    assert bench.blocksparse_pairs(np.tril(np.ones((t, t))), 16384, 16384, True) == 16384 * 16385 / 2


def test_blocksparse_mask_recipe():
    """The seeded block mask of the block-sparse workload: the sink block and the window ending
    at each query block's last reachable key block are always kept, nothing past that reach is
    ever kept, the random share of the rest is near p_random, and the same seed gives the same
    mask."""
    import torch

    from exact_io_aware_94_b200.inputs import blocksparse_mask

    H, L, w, p = 4, 128 * 64, 8, 0.1
    m = blocksparse_mask(H, L, L, seed=8, sink=1, window=w, p_random=p)
    t = L // 128
    assert m.shape == (H, t, t) and m.dtype == torch.uint8
    r = torch.arange(t)[:, None]
    c = torch.arange(t)[None, :]
    assert (m[:, :, 0] == 1).all()                                # sink
    window = ((c <= r) & (c > r - w)).expand(H, t, t)
    assert (m[window] == 1).all()                                 # local window up to the diagonal
    assert (m[(c > r).expand(H, t, t)] == 0).all()                # causal reach
    rest = ((c < r - w + 1) & (c >= 1)).expand(H, t, t)
    assert abs(m[rest].float().mean().item() - p) < 0.02          # random share
    assert torch.equal(m, blocksparse_mask(H, L, L, seed=8, sink=1, window=w, p_random=p))
    # bottom-right reach when Lq < Lk: query block r reaches key block r + (Lk - Lq) / 128
    m2 = blocksparse_mask(1, 256, 1024, seed=1, sink=0, window=1, p_random=0.0)
    assert m2[0].tolist() == [[0, 0, 0, 0, 0, 0, 1, 0], [0, 0, 0, 0, 0, 0, 0, 1]]


def test_traffic_records_match_their_capture_summaries():
    """Every DRAM-traffic record the benchmark can report names a committed ncu summary that
    states the same kernel-source hash, and its kernel family is one the benchmark hashes."""
    import json
    import os
    import re

    import bench

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    with open(os.path.join(root, "profiles", "traffic.json")) as fh:
        rec = json.load(fh)
    assert rec
    for kernel, workloads in rec.items():
        assert kernel in bench.KERNEL_SOURCES, kernel
        for workload, e in workloads.items():
            assert ("bytes_per_launch" in e) != ("traffic_over_algorithmic" in e), (kernel, workload)
            with open(os.path.join(root, e["capture"])) as fh:
                text = fh.read()
            m = re.search(r"Kernel source state: hash `([0-9a-f]{16})`", text)
            assert m and m.group(1) == e["source_hash"], (kernel, workload, e["capture"])
