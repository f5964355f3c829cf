"""Helpers shared by the GPU parity tests: oracle views of a workload and the
comparison rule.

The bar is the stated one, flat: max-abs <= 1e-2 on O, dQ, dK, dV and
<= 1e-3 on LSE, element by element (-inf LSE and zero O exactly where a row has
no allowed key).  One excuse only: outputs are bf16, and a correctly rounded
bf16 value of an exact result of magnitude >= 4 already carries up to half a
bf16 ulp (0.0156 in [4, 8)) of pure output rounding, so an element whose oracle
value has |x| >= 4 passes if its error is within 1e-2 + half a bf16 ulp of that
value.  Every excused element is recorded with its raw error.

Every comparison records the raw max-abs error per output under the running
test's id; ``tests/conftest.py`` prints the table at the end of the run (and
writes it as JSON where ``BSA_PARITY_LOG`` names a file)."""

import os

import numpy as np
import torch

import oracle

O_TOL = 1e-2
LSE_TOL = 1e-3
EXCUSE_ABS = 4.0  # |oracle| at or above which half a bf16 ulp of output rounding is excused

# {test id: {output name: {"raw": max-abs, "n": elements, "excused": [(index, oracle, error), ...]}}}
REPORT: dict = {}


def _test_id() -> str:
    return os.environ.get("PYTEST_CURRENT_TEST", "?").rsplit(" (", 1)[0]


def np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def mask_desc(wl) -> oracle.MaskDesc:
    return oracle.MaskDesc(**wl.mask_numpy())


def half_ulp_bf16(x):
    """Half the spacing of bf16 numbers at |x| (8 significant bits): the error a
    correctly rounded bf16 output of the exact value may carry by itself."""
    ax = np.maximum(np.abs(x), np.float64(2.0 ** -126))
    return np.ldexp(1.0, np.floor(np.log2(ax)).astype(np.int64) - 8)


def _record(name: str, raw: float, n: int, excused=()):
    ent = REPORT.setdefault(_test_id(), {})
    key, i = name, 2
    while key in ent:  # the same output checked twice in one test
        key, i = f"{name}#{i}", i + 1
    ent[key] = {"raw": raw, "n": int(n), "excused": list(excused)}


def check(name: str, x_gpu, ref, tol: float = O_TOL) -> float:
    """Raw max |x_gpu - ref| over all elements; asserts the flat bar.

    An element fails when its error exceeds ``tol``, unless |ref| >= 4 and the
    error is within tol + half a bf16 ulp of ref (output rounding; listed in the
    report).  NaN anywhere fails."""
    a = np64(x_gpu) if isinstance(x_gpu, torch.Tensor) else np.asarray(x_gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert a.shape == ref.shape, (name, a.shape, ref.shape)
    err = np.abs(a - ref)
    assert not np.isnan(err).any(), f"{name}: NaN in the comparison"
    raw = float(err.max()) if err.size else 0.0
    over = err > tol
    excusable = over & (np.abs(ref) >= EXCUSE_ABS) & (err <= tol + half_ulp_bf16(ref))
    bad = over & ~excusable
    idx = np.argwhere(excusable)
    excused = [(tuple(int(v) for v in ix), float(ref[tuple(ix)]), float(err[tuple(ix)])) for ix in idx[:50]]
    _record(name, raw, err.size, excused)
    if bad.any():
        first = tuple(int(v) for v in np.argwhere(bad)[0])
        raise AssertionError(
            f"{name}: max-abs {raw:.5f} > {tol} on {int(bad.sum())} element(s) not excused by output "
            f"rounding; first at {first}: gpu {a[first]:.6f} oracle {ref[first]:.6f}")
    return raw


def compare_out(o_gpu, o_ref, rows=None, tol=O_TOL, name="O"):
    """Raw max |O_gpu - O_ref| over the given rows (all rows if None), checked
    against the flat bar by :func:`check`."""
    a = np64(o_gpu)
    if rows is not None:
        a = a[:, rows]
        o_ref = o_ref[:, rows]
    return check(name, a, o_ref, tol)


def compare_lse(l_gpu, l_ref, rows=None, name="LSE"):
    """(max |LSE_gpu - LSE_ref| over finite entries, -inf pattern equal); the
    error is recorded, the caller asserts it against LSE_TOL."""
    a = l_gpu.detach().cpu().numpy().astype(np.float64)
    if rows is not None:
        a = a[..., rows]
        l_ref = l_ref[..., rows]
    fin = np.isfinite(l_ref)
    same = bool(np.array_equal(fin, np.isfinite(a)) and np.all(np.isneginf(a[~fin])))
    err = float(np.max(np.abs(a[fin] - l_ref[fin]))) if fin.any() else 0.0
    _record(name, err, int(fin.sum()))
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
