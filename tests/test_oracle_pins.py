"""The fp64 oracle pinned to things other than itself (CPU only).

Pins: scalar brute force, the library SDPA routine, autograd, central finite
differences, closed forms and the invariants the pages state.
"""

import math

import numpy as np
import pytest

import oracle
from oracle import MaskDesc
from tests import oracle_pins as P

SCALE = 0.37


@pytest.mark.parametrize("case", list(P.tiny_masks(2, 9, 11).keys()))
def test_forward_matches_brute_force(case):
    q, k, v, _ = P.tiny_inputs(1, B=2)
    mask = P.tiny_masks(2, 9, 11)[case]
    O, L = oracle.attention_forward(q, k, v, mask, SCALE)
    allowed = P.dense_allowed(mask, 2, 9, 11)
    Ob, Lb = P.brute_force_forward(q, k, v, allowed, SCALE)
    assert np.max(np.abs(O - Ob)) < 1e-12
    fin = np.isfinite(Lb)
    assert np.array_equal(fin, np.isfinite(L))
    assert np.max(np.abs(L[fin] - Lb[fin])) < 1e-12


@pytest.mark.parametrize("case", ["none", "causal", "window3", "padding", "segments", "seg+window",
                                  "prefix_lm", "dilated", "doc_causal"])
def test_forward_matches_library_sdpa(case):
    q, k, v, _ = P.tiny_inputs(2, B=2, Sq=12, Skv=12, D=6)
    mask = P.tiny_masks(2, 12, 12, seed=3)[case]
    allowed = P.dense_allowed(mask, 2, 12, 12)
    if not all(a.any(axis=1).all() for a in allowed):
        pytest.skip("SDPA is undefined on rows without keys")
    O, _ = oracle.attention_forward(q, k, v, mask, SCALE)
    Os = P.sdpa_forward(q, k, v, allowed, SCALE)
    assert np.max(np.abs(O - Os)) < 1e-12


@pytest.mark.parametrize("case", ["none", "causal", "window3", "padding", "segments", "prefix_lm",
                                  "dilated"])
def test_backward_matches_autograd(case):
    q, k, v, dO = P.tiny_inputs(4, B=2, Sq=10, Skv=10, D=4)
    v = v[..., :4].copy()
    dO = dO[..., :4].copy()
    mask = P.tiny_masks(2, 10, 10, seed=5)[case]
    allowed = P.dense_allowed(mask, 2, 10, 10)
    if not all(a.any(axis=1).all() for a in allowed):
        pytest.skip("SDPA is undefined on rows without keys")
    dq, dk, dv = oracle.attention_backward(q, k, v, dO, mask, SCALE)
    aq, ak, av = P.autograd_backward(q, k, v, dO, allowed, SCALE)
    for x, y in ((dq, aq), (dk, ak), (dv, av)):
        assert np.max(np.abs(x - y)) < 1e-11


def test_backward_matches_finite_differences_with_empty_rows():
    # A window on Sq > Skv leaves the first rows without keys: gradients through
    # them are zero and the rest must still match central differences.
    q, k, v, dO = P.tiny_inputs(6, B=1, Sq=8, Skv=6, D=3)
    mask = MaskDesc(window=2)
    fwd = lambda a, b_, c: oracle.attention_forward(a, b_, c, mask, SCALE)[0]
    dq, dk, dv = oracle.attention_backward(q, k, v, dO, mask, SCALE)
    rng = np.random.default_rng(0)
    for which, grad, shp in ((0, dq, q.shape), (1, dk, k.shape), (2, dv, v.shape)):
        idx = [tuple(int(rng.integers(0, s)) for s in shp) for _ in range(12)]
        fd = P.finite_difference_grad(fwd, q, k, v, dO, which, idx)
        an = np.array([grad[i] for i in idx])
        assert np.max(np.abs(fd - an)) < 1e-7
    O, L = oracle.attention_forward(q, k, v, mask, SCALE)
    assert np.all(O[0, :2] == 0) and np.all(np.isneginf(L[0, :, :2]))
    assert np.all(dq[0, :2] == 0)


# ---------------------------------------------------------------- closed forms

def test_closed_form_equal_keys_give_mean_of_values():
    rng = np.random.default_rng(7)
    q = rng.standard_normal((1, 5, 1, 4))
    k = np.repeat(rng.standard_normal((1, 1, 1, 4)), 9, axis=1)
    v = rng.standard_normal((1, 9, 1, 3))
    mask = MaskDesc(kv_valid_len=np.array([6]))
    O, L = oracle.attention_forward(q, k, v, mask, SCALE)
    assert np.allclose(O[0, :, 0], v[0, :6, 0].mean(axis=0), atol=1e-13)
    s = SCALE * (q[0, :, 0] @ k[0, 0, 0])
    assert np.allclose(L[0, 0], s + math.log(6), atol=1e-13)


def test_closed_form_single_key():
    rng = np.random.default_rng(8)
    q, k, v = (rng.standard_normal((1, 6, 1, 4)) for _ in range(3))
    # window=1: each row sees exactly its own (diagonal) key
    O, L = oracle.attention_forward(q, k, v, MaskDesc(window=1), SCALE)
    assert np.allclose(O[0, :, 0], v[0, :, 0], atol=1e-14)
    assert np.allclose(L[0, 0], SCALE * (q[0, :, 0] * k[0, :, 0]).sum(1), atol=1e-14)


def test_closed_form_zero_query_is_uniform():
    rng = np.random.default_rng(9)
    q = np.zeros((1, 4, 1, 4))
    k, v = (rng.standard_normal((1, 7, 1, 4)) for _ in range(2))
    O, L = oracle.attention_forward(q, k, v, MaskDesc(), SCALE)
    assert np.allclose(O[0, :, 0], v[0, :, 0].mean(axis=0), atol=1e-14)
    assert np.allclose(L, math.log(7), atol=1e-14)


def test_wide_window_is_plain_causal():
    q, k, v, _ = P.tiny_inputs(10, Sq=7, Skv=9, D=3)
    a, la = oracle.attention_forward(q, k, v, MaskDesc(window=50), SCALE)
    b, lb = oracle.attention_forward(q, k, v, MaskDesc(window=0), SCALE)
    assert np.array_equal(a, b) and np.array_equal(la, lb)


def test_mask_predicates_count_keys():
    Sq, Skv, W = 40, 56, 7
    o = Skv - Sq
    a = oracle.allowed_rows(MaskDesc(window=W), 0, np.arange(Sq), Sq, Skv)
    for i in range(Sq):
        lo, hi = max(0, i + o - W + 1), min(Skv - 1, i + o)
        assert a[i].sum() == max(0, hi - lo + 1)
        assert a[i, hi] and (lo == 0 or not a[i, lo - 1])
    assert a[Sq - 1, Skv - 1]  # bottom-right alignment
    cu = np.array([0, 10, 25, 31, 40])
    a = oracle.allowed_rows(MaskDesc(cu_seqlens=cu, n_align_tail=1), 0, np.arange(40), 40, 40)
    for s in range(3):
        for i in range(cu[s], cu[s + 1]):
            assert a[i].sum() == cu[s + 1] - cu[s] and a[i, cu[s]:cu[s + 1]].all()
    assert not a[31:].any() and not a[:, 31:].any()
    a = oracle.allowed_rows(MaskDesc(kv_valid_len=np.array([5, 9])), 1, np.arange(4), 4, 12)
    assert (a.sum(axis=1) == 9).all()


def test_prefix_lm_predicate_counts_keys():
    # causal with a bidirectional prefix of P keys: row i sees keys 0 .. max(P, i+1) - 1
    Sq = Skv = 40
    for P_ in (0, 7, 40, 60):
        a = oracle.allowed_rows(MaskDesc(window=0, prefix_len=np.array([P_])), 0, np.arange(Sq), Sq, Skv)
        for i in range(Sq):
            n = min(Skv, max(P_, i + 1))
            assert a[i].sum() == n and a[i, :n].all()
    # with a window of 5: the prefix 0..6 and the band i-4 .. i, overlapping or not
    a = oracle.allowed_rows(MaskDesc(window=5, prefix_len=np.array([7])), 0, np.arange(Sq), Sq, Skv)
    for i in range(Sq):
        band_lo = max(0, i - 4)
        assert a[i].sum() == (max(7, i + 1) if band_lo <= 7 else 7 + 5)
        assert a[i, :7].all() and a[i, band_lo:i + 1].all()


def test_dilated_window_predicate_counts_keys():
    # span W = 10, dilation 3: keys i, i-3, i-6, i-9 (those >= 0)
    Sq = Skv = 20
    a = oracle.allowed_rows(MaskDesc(window=10, dilation=3), 0, np.arange(Sq), Sq, Skv)
    for i in range(Sq):
        assert a[i].sum() == min(4, i // 3 + 1)
        assert a[i, i] and (i < 3 or a[i, i - 3]) and (i < 1 or not a[i, i - 1])
        assert i < 12 or not a[i, i - 12]
    # bottom-right alignment with Sq < Skv: the last row's diagonal is the last key
    a = oracle.allowed_rows(MaskDesc(window=8, dilation=2), 0, np.arange(6), 6, 13)
    assert a[5].nonzero()[0].tolist() == [6, 8, 10, 12]
    with pytest.raises(ValueError):
        oracle.allowed_rows(MaskDesc(dilation=2), 0, np.arange(4), 4, 4)


def test_prefix_covering_every_key_is_no_mask():
    q, k, v, _ = P.tiny_inputs(12, B=1, Sq=9, Skv=11, D=4)
    O, _ = oracle.attention_forward(q, k, v, MaskDesc(window=2, prefix_len=np.array([11])), SCALE)
    allowed = [np.ones((9, 11), dtype=bool)]
    assert np.max(np.abs(O - P.sdpa_forward(q, k, v, allowed, SCALE))) < 1e-12


def test_dilated_rows_equal_attention_over_gathered_keys():
    # each row's output is plain attention over its own keys i+o, i+o-d, ...
    q, k, v, _ = P.tiny_inputs(13, B=1, Sq=10, Skv=14, D=5)
    O, L = oracle.attention_forward(q, k, v, MaskDesc(window=9, dilation=4), SCALE)
    o = 14 - 10
    for i in range(10):
        keys = [i + o - 4 * t for t in range(3) if i + o - 4 * t >= 0]
        s = SCALE * (k[0, keys, 0, :] @ q[0, i, 0, :])
        w = np.exp(s - s.max())
        assert np.allclose(O[0, i, 0], (w / w.sum()) @ v[0, keys, 0, :], atol=1e-13)
        assert abs(L[0, 0, i] - (s.max() + math.log(w.sum()))) < 1e-13


# ---------------------------------------------------------------- invariants

def test_constant_segment_ids_equal_no_mask():
    q, k, v, dO = P.tiny_inputs(11, B=2, Sq=12, Skv=12, D=4)
    v, dO = v[..., :4].copy(), dO[..., :4].copy()
    seg = np.full((2, 12), 3)
    m = MaskDesc(seg_q=seg, seg_kv=seg)
    a = oracle.attention_forward(q, k, v, m, SCALE)
    b = oracle.attention_forward(q, k, v, MaskDesc(), SCALE)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    ga = oracle.attention_backward(q, k, v, dO, m, SCALE)
    gb = oracle.attention_backward(q, k, v, dO, MaskDesc(), SCALE)
    for x, y in zip(ga, gb):
        assert np.array_equal(x, y)


def test_alignment_rows_never_reach_real_rows():
    rng = np.random.default_rng(12)
    cu = np.array([0, 13, 21, 24])
    m = MaskDesc(cu_seqlens=cu, n_align_tail=1)
    q, k, v = (rng.standard_normal((1, 24, 2, 4)) for _ in range(3))
    O, L = oracle.attention_forward(q, k, v, m, SCALE)
    q2, k2, v2 = q.copy(), k.copy(), v.copy()
    for t in (q2, k2, v2):
        t[:, 21:] = rng.standard_normal(t[:, 21:].shape) * 50
    O2, L2 = oracle.attention_forward(q2, k2, v2, m, SCALE)
    assert np.array_equal(O[:, :21], O2[:, :21]) and np.array_equal(L[..., :21], L2[..., :21])
    assert np.all(O[:, 21:] == 0) and np.all(np.isneginf(L[..., 21:]))


def test_padding_contents_do_not_matter():
    rng = np.random.default_rng(13)
    m = MaskDesc(kv_valid_len=np.array([10]))
    q = rng.standard_normal((1, 8, 1, 4))
    k, v = (rng.standard_normal((1, 16, 1, 4)) for _ in range(2))
    O, L = oracle.attention_forward(q, k, v, m, SCALE)
    k2, v2 = k.copy(), v.copy()
    k2[:, 10:] *= 100
    v2[:, 10:] = 1e6  # finite: 0 * NaN would be NaN in any product
    O2, L2 = oracle.attention_forward(q, k2, v2, m, SCALE)
    assert np.array_equal(O, O2) and np.array_equal(L, L2)


def test_fixed_m_equals_online():
    q, k, v, _ = P.tiny_inputs(14, B=2, Sq=20, Skv=24, D=6)
    for name, m in P.tiny_masks(2, 20, 24, seed=2).items():
        a = oracle.attention_forward(q, k, v, m, SCALE)
        b = oracle.attention_forward_fixed_m(q, k, v, m, SCALE)
        assert np.max(np.abs(a[0] - b[0])) < 1e-12, name
        fin = np.isfinite(a[1])
        assert np.array_equal(fin, np.isfinite(b[1]))
        assert np.max(np.abs(a[1][fin] - b[1][fin])) < 1e-12, name


def test_fixed_m_bound_dominates_every_score_and_gate_separates_sink():
    rng = np.random.default_rng(15)
    D, S = 16, 64
    q = rng.standard_normal((1, S, 2, D)) * math.sqrt(0.5)
    k = rng.standard_normal((1, S + 8, 2, D)) * math.sqrt(0.5)
    k[0, :4, 0] *= 20  # sink keys on head 0
    k[0, S:] *= 100  # padding keys
    m = MaskDesc(kv_valid_len=np.array([S]))
    scale = 1 / math.sqrt(D)
    kmax, qmax, bound, gate = oracle.fixed_m_bound(q, k, m, scale, gate_limit=64.0)
    for h in range(2):
        s = scale * q[0, :, h] @ k[0, :S, h].T
        assert np.abs(s).max() <= bound[0, h] + 1e-12
        assert kmax[0, h] == np.linalg.norm(k[0, :S, h], axis=1).max()
    assert not gate[0, 0] and gate[0, 1]


def test_smoothed_bound_closed_form_two_keys():
    # keys u + e and u - e: center u, radius ||e||; with q along e the first
    # key's score reaches the bound exactly
    u = np.array([3.0, -1.0, 2.0, 0.5])
    e = np.array([0.0, 2.0, 0.0, 0.0])
    k = np.stack([u + e, u - e])[None, :, None, :]
    q = np.array([[0.0, 1.5, 0.0, 0.0]])[None, :, None, :]
    kbar, radius, qmax, bound, gate = oracle.fixed_m_bound_smoothed(q, k, MaskDesc(), 0.5)
    assert np.allclose(kbar[0, 0], u, atol=1e-15) and abs(radius[0, 0] - 2.0) < 1e-15
    assert abs(bound[0, 0] - 0.5 * 1.5 * 2.0) < 1e-15
    s = 0.5 * (k[0, :, 0] @ q[0, 0, 0])
    assert abs(s.max() - 0.5 * (q[0, 0, 0] @ u + 1.5 * 2.0)) < 1e-14


def test_smoothed_bound_is_translation_invariant_and_dominates():
    rng = np.random.default_rng(21)
    D, S = 16, 50
    q = rng.standard_normal((1, S, 2, D))
    k = rng.standard_normal((1, S + 6, 2, D))
    k[0, S:] *= 100  # padding keys never enter the center or the radius
    m = MaskDesc(kv_valid_len=np.array([S]))
    scale = 0.3
    kbar, radius, qmax, bound, gate = oracle.fixed_m_bound_smoothed(q, k, m, scale)
    shift = rng.standard_normal(D) * 7
    k2 = k + shift
    kbar2, radius2, _, _, _ = oracle.fixed_m_bound_smoothed(q, k2, m, scale)
    assert np.allclose(kbar2, kbar + shift, atol=1e-12)
    assert np.allclose(radius2, radius, atol=1e-12)
    kmax2 = oracle.fixed_m_bound(q, k2, m, scale)[0]
    assert (kmax2 > radius2 + 5).all()  # the plain bound grows with the offset
    for h in range(2):
        s = scale * q[0, :, h] @ k2[0, :S, h].T
        mi = scale * (q[0, :, h] @ kbar2[0, h] + np.linalg.norm(q[0, :, h], axis=1) * radius2[0, h])
        assert (s.max(axis=1) <= mi + 1e-12).all()
        assert (mi - s.max(axis=1) <= 2 * scale * np.linalg.norm(q[0, :, h], axis=1) * radius2[0, h] + 1e-12).all()


def test_smoothing_widens_gate_and_stays_exact():
    # a common key offset of norm 12: the plain gate fails, the smoothed one holds
    rng = np.random.default_rng(22)
    D, S = 16, 40
    q = rng.standard_normal((1, S, 1, D)) * math.sqrt(0.5)
    k = rng.standard_normal((1, S, 1, D)) * math.sqrt(0.5)
    k[0, :, 0, 0] += 12.0
    v = rng.standard_normal((1, S, 1, D))
    scale = 1 / math.sqrt(D)
    plain = oracle.fixed_m_bound(q, k, MaskDesc(window=0), scale, gate_limit=16.0)
    smooth = oracle.fixed_m_bound_smoothed(q, k, MaskDesc(window=0), scale, gate_limit=16.0)
    assert not plain[3][0, 0] and smooth[4][0, 0]
    O, L = oracle.attention_forward(q, k, v, MaskDesc(window=0), scale)
    Os, Ls = oracle.attention_forward_fixed_m(q, k, v, MaskDesc(window=0), scale, kmax=smooth[1],
                                              kbar=smooth[0])
    assert np.max(np.abs(O - Os)) < 1e-12 and np.max(np.abs(L - Ls)) < 1e-12


@pytest.mark.parametrize("H_kv", [1, 2])
def test_gqa_matches_library_sdpa_and_autograd(H_kv):
    # torch's SDPA with enable_gqa (a library routine) and autograd through it
    import torch
    q, k, v, dO = P.tiny_inputs(23, B=2, Sq=10, Skv=12, D=4, H=4)
    k, v = k[:, :, :H_kv].copy(), v[:, :, :H_kv].copy()
    v, dO = v[..., :4].copy(), dO[..., :4].copy()
    mask = P.tiny_masks(2, 10, 12, seed=4)["window3"]
    allowed = P.dense_allowed(mask, 2, 10, 12)
    O, _ = oracle.attention_forward(q, k, v, mask, SCALE)
    dq, dk, dv = oracle.attention_backward(q, k, v, dO, mask, SCALE)
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x)).permute(0, 2, 1, 3).clone().requires_grad_(True)
    qt, kt, vt = t(q), t(k), t(v)
    m = torch.from_numpy(np.stack(allowed))[:, None, :, :]
    ot = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=m, scale=SCALE,
                                                          enable_gqa=True)
    (ot * torch.from_numpy(dO).permute(0, 2, 1, 3)).sum().backward()
    back = lambda x: x.detach().permute(0, 2, 1, 3).numpy()
    assert np.max(np.abs(O - back(ot))) < 1e-12
    for x, y in ((dq, qt.grad), (dk, kt.grad), (dv, vt.grad)):
        assert np.max(np.abs(x - back(y))) < 1e-11


def test_gqa_equals_mha_with_repeated_kv_heads():
    q, k, v, dO = P.tiny_inputs(24, B=1, Sq=9, Skv=9, D=4, H=6)
    k, v = k[:, :, :2].copy(), v[:, :, :2].copy()
    mask = MaskDesc(window=0)
    kr, vr = np.repeat(k, 3, axis=2), np.repeat(v, 3, axis=2)
    assert oracle.kv_head_of(6, 2)(4) == 1
    a = oracle.attention_forward(q, k, v, mask, SCALE)
    b = oracle.attention_forward(q, kr, vr, mask, SCALE)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    gq, gk, gv = oracle.attention_backward(q, k, v, dO, mask, SCALE)
    rq, rk, rv = oracle.attention_backward(q, kr, vr, dO, mask, SCALE)
    assert np.array_equal(gq, rq)
    assert np.max(np.abs(gk - rk.reshape(1, 9, 2, 3, -1).sum(axis=3))) < 1e-13
    assert np.max(np.abs(gv - rv.reshape(1, 9, 2, 3, -1).sum(axis=3))) < 1e-13
    with pytest.raises(ValueError):
        oracle.kv_head_of(6, 4)


def test_gradient_identities():
    q, k, v, dO = P.tiny_inputs(16, B=1, Sq=9, Skv=9, D=4)
    v, dO = v[..., :4].copy(), dO[..., :4].copy()
    m = MaskDesc(window=3)
    dq, dk, dv = oracle.attention_backward(q, k, v, dO, m, SCALE)
    # sum over keys of dV equals the sum of dO over rows that see any key
    assert np.allclose(dv.sum(axis=1), dO.sum(axis=1), atol=1e-12)
    # rows of dS sum to zero: with every key equal, dQ vanishes
    k_eq = np.repeat(k[:, :1], 9, axis=1)
    dq0, _, _ = oracle.attention_backward(q, k_eq, v, dO, m, SCALE)
    assert np.max(np.abs(dq0)) < 1e-12


def test_key_permutation_with_mask_leaves_output():
    rng = np.random.default_rng(17)
    q = rng.standard_normal((1, 6, 1, 4))
    k, v = (rng.standard_normal((1, 10, 1, 4)) for _ in range(2))
    seg_q = np.array([[0, 0, 1, 1, 2, 2]])
    seg_kv = np.array([[0, 1, 2, 0, 1, 2, 0, 1, 2, 2]])
    perm = rng.permutation(10)
    a = oracle.attention_forward(q, k, v, MaskDesc(seg_q=seg_q, seg_kv=seg_kv), SCALE)
    b = oracle.attention_forward(q, k[:, perm], v[:, perm],
                                 MaskDesc(seg_q=seg_q, seg_kv=seg_kv[:, perm]), SCALE)
    assert np.allclose(a[0], b[0], atol=1e-14) and np.allclose(a[1], b[1], atol=1e-14)


def test_useful_flops_per_tile():
    assert oracle.useful_flops(1, 128) == 4 * 128 * 128 * 128
    assert oracle.useful_flops(2, 64, backward=True) == 2.5 * 2 * 4 * 128 * 128 * 64


def test_valid_keys_of_varlen_exclude_the_alignment_tail():
    """The fixed-m bound's kmax runs over the keys a real row can see: with
    cu_seqlens the keys of the trailing alignment segments never enter it.
    Alignment keys scaled x100 dominate every norm; kmax must still be the
    largest norm among the real segments' keys, a closed form taken straight
    from the cu_seqlens boundaries; with no alignment tail it is the largest
    norm over all keys.  Padding (kv_valid_len) and varlen together: the
    smaller of the two boundaries."""
    rng = np.random.default_rng(41)
    T, H, D = 90, 2, 8
    cu = np.array([0, 30, 70, 78, 90])
    q = rng.standard_normal((1, T, H, D))
    k = rng.standard_normal((1, T, H, D))
    k[0, 70:] *= 100.0  # the two alignment segments [70, 78) and [78, 90)
    for tail, real_end in ((2, 70), (1, 78), (0, 90)):
        m = MaskDesc(cu_seqlens=cu, n_align_tail=tail)
        kmax, _, _, _ = oracle.fixed_m_bound(q, k, m, SCALE)
        for h in range(H):
            assert kmax[0, h] == np.linalg.norm(k[0, :real_end, h], axis=1).max()
        vk = oracle.valid_keys(m, 0, T)
        assert vk[:real_end].all() and not vk[real_end:].any()
    m = MaskDesc(cu_seqlens=cu, n_align_tail=1, kv_valid_len=np.array([50]))
    kmax, _, _, _ = oracle.fixed_m_bound(q, k, m, SCALE)
    assert kmax[0, 0] == np.linalg.norm(k[0, :50, 0], axis=1).max()
    kbar, radius, _, _, _ = oracle.fixed_m_bound_smoothed(q, k, MaskDesc(cu_seqlens=cu, n_align_tail=2), SCALE)
    assert np.allclose(kbar[0, 1], k[0, :70, 1].mean(axis=0), atol=1e-13)
