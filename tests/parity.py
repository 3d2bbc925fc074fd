"""Comparison helpers for the GPU-vs-oracle parity tests.

Tolerances (the bar the library is held to):
  O        max |O - O_ref| <= 1e-2 and mean |O - O_ref| <= 1e-3, graded on fp32 O
  LSE      max |LSE - LSE_ref| <= 1e-3
  dQ/dK/dV ||X - X_ref||_F / ||X_ref||_F <= 1e-2
bf16 O is checked against the oracle rounded the same way, within one bf16
rounding step of the fp32 bound (half an ulp of |O| plus the fp32 error).
"""
import numpy as np
import torch

O_MAX_ABS = 1e-2
O_MEAN_ABS = 1e-3
LSE_MAX_ABS = 1e-3
GRAD_REL_FRO = 1e-2


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def check_o(o_gpu, o_ref, what=""):
    o = to_np(o_gpu) if isinstance(o_gpu, torch.Tensor) else o_gpu
    assert np.isfinite(o).all(), "%s: non-finite output" % what
    err = np.abs(o - o_ref)
    assert err.max() <= O_MAX_ABS, "%s: O max-abs %.3g" % (what, err.max())
    assert err.mean() <= O_MEAN_ABS, "%s: O mean-abs %.3g" % (what, err.mean())
    return float(err.max()), float(err.mean())


def check_o_bf16(o_gpu, o_ref, what=""):
    o = to_np(o_gpu)
    assert np.isfinite(o).all(), "%s: non-finite output" % what
    # bf16 storage adds at most half an ulp: 2^-8 relative to the leading bit.
    bound = O_MAX_ABS + np.abs(o_ref) * 2.0 ** -8
    err = np.abs(o - o_ref)
    assert (err <= bound).all(), "%s: bf16 O beyond storage bound (max err %.3g)" % (what, err.max())


def check_lse(lse_gpu, lse_ref, what=""):
    lse = to_np(lse_gpu) if isinstance(lse_gpu, torch.Tensor) else lse_gpu
    fin = np.isfinite(lse_ref)
    assert (np.isfinite(lse) == fin).all(), "%s: LSE finiteness differs" % what
    assert (lse[~fin] == lse_ref[~fin]).all()
    err = np.abs(lse[fin] - lse_ref[fin]) if fin.any() else np.zeros(1)
    assert err.max() <= LSE_MAX_ABS, "%s: LSE max-abs %.3g" % (what, err.max())
    return float(err.max())


def rel_fro(x, ref):
    x = to_np(x) if isinstance(x, torch.Tensor) else x
    return float(np.linalg.norm((x - ref).ravel()) / max(np.linalg.norm(ref.ravel()), 1e-300))


def check_grad(x_gpu, x_ref, what=""):
    x = to_np(x_gpu)
    assert np.isfinite(x).all(), "%s: non-finite gradient" % what
    r = rel_fro(x, x_ref)
    assert r <= GRAD_REL_FRO, "%s: relative Frobenius error %.3g" % (what, r)
    return r


def sample_rows(B, H, L, n_random, seed, must=(0, 1, 127, 128, 255, 256)):
    """Flat row indices: fixed rows (and L-1) of every head plus seeded random ones."""
    rng = np.random.default_rng(seed)
    rows = set()
    for bh in range(B * H):
        for i in tuple(must) + (L - 1,):
            if 0 <= i < L:
                rows.add(bh * L + i)
    rows.update(rng.integers(0, B * H * L, size=n_random).tolist())
    return np.array(sorted(rows), dtype=np.int64)


def padded_like(shape, dtype, device, pad_elems=4096, fill=float("nan")):
    """A contiguous tensor of `shape` carved from a larger buffer whose tail is
    filled with `fill`; a read past the end of the tensor would pick it up."""
    n = int(np.prod(shape))
    buf = torch.full((n + pad_elems,), fill, dtype=dtype, device=device)
    return buf[:n].view(shape), buf
