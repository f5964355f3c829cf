"""Planted mistakes: each test swaps one plausible error into the oracle (on the
CPU, through monkeypatch, for that test only) and checks that one of the pins
in tests/test_oracle_pins.py then fails.  A pin set that stayed green under one
of these would not be pinning that part of the oracle."""

import numpy as np
import pytest

import oracle
import oracle.attention as A
from tests import test_oracle_pins as pins


def _must_fail(pin, *args):
    with pytest.raises(AssertionError):
        pin(*args)


def test_alignment_keys_in_the_bound_are_caught(monkeypatch):
    # valid_keys forgetting the varlen alignment tail
    orig = A.valid_keys

    def broken(mask, b, Skv):
        m = oracle.MaskDesc(**{**mask.__dict__, "cu_seqlens": None, "n_align_tail": 0})
        return orig(m, b, Skv)

    monkeypatch.setattr(A, "valid_keys", broken)
    monkeypatch.setattr(oracle, "valid_keys", broken)
    _must_fail(pins.test_valid_keys_of_varlen_exclude_the_alignment_tail)


def test_a_dropped_delta_term_is_caught(monkeypatch):
    # dS = P o dP (the -Delta term dropped): re-run the backward with O := 0,
    # which zeroes Delta and nothing else
    orig = A.attention_backward

    def broken(q, k, v, dO, mask, scale, **kw):
        gq, gk, gv = orig(q, k, v, dO, mask, scale, **kw)
        # dQ and dK carry scale * sum_j P_ij Delta_i k_j (dK: q_i); add it back
        qq, kk, dd = A._as64(q), A._as64(k), A._as64(dO)
        B, Sq, H, D = qq.shape
        for b in range(B):
            a = A.allowed_rows(mask, b, np.arange(Sq), Sq, kk.shape[1])
            for h in range(H):
                s = np.where(a, scale * qq[b, :, h] @ kk[b, :, h].T, -np.inf)
                has = a.any(axis=1)
                mx = np.where(has, s.max(axis=1), 0.0)
                e = np.where(a, np.exp(s - mx[:, None]), 0.0)
                P_ = e / np.where(has, e.sum(axis=1), 1.0)[:, None]
                O = P_ @ A._as64(v)[b, :, h]
                delta = (dd[b, :, h] * O).sum(axis=1)
                gq[b, :, h] += scale * (P_ * delta[:, None]) @ kk[b, :, h]
                gk[b, :, h] += scale * (P_ * delta[:, None]).T @ qq[b, :, h]
        return gq, gk, gv

    monkeypatch.setattr(oracle, "attention_backward", broken)
    _must_fail(pins.test_backward_matches_autograd, "causal")


def test_a_missing_scale_on_dk_is_caught(monkeypatch):
    orig = A.attention_backward

    def broken(q, k, v, dO, mask, scale, **kw):
        gq, gk, gv = orig(q, k, v, dO, mask, scale, **kw)
        return gq, gk / scale, gv

    monkeypatch.setattr(oracle, "attention_backward", broken)
    _must_fail(pins.test_backward_matches_autograd, "window3")


def test_a_window_off_by_one_is_caught(monkeypatch):
    # the band t <= W instead of t < W: one key too many per row
    orig = A.allowed_rows

    def broken(mask, b, rows, Sq, Skv):
        if mask.window:
            mask = oracle.MaskDesc(**{**mask.__dict__, "window": mask.window + 1})
        return orig(mask, b, rows, Sq, Skv)

    monkeypatch.setattr(oracle, "allowed_rows", broken)
    _must_fail(pins.test_mask_predicates_count_keys)


def test_an_lse_without_its_max_is_caught(monkeypatch):
    # LSE = ln sum exp(s - M), the row max M dropped
    orig = A.attention_forward

    def broken(q, k, v, mask, scale, **kw):
        O, L = orig(q, k, v, mask, scale, **kw)
        s_max = np.zeros_like(L)
        qq, kk = A._as64(q), A._as64(k)
        for b in range(qq.shape[0]):
            a = A.allowed_rows(mask, b, np.arange(qq.shape[1]), qq.shape[1], kk.shape[1])
            for h in range(qq.shape[2]):
                s = np.where(a, scale * qq[b, :, h] @ kk[b, :, h].T, -np.inf)
                s_max[b, h] = np.where(a.any(axis=1), s.max(axis=1), 0.0)
        return O, L - s_max

    monkeypatch.setattr(oracle, "attention_forward", broken)
    _must_fail(pins.test_forward_matches_brute_force, "window3")


def test_a_wrong_key_index_in_the_segment_mask_is_caught(monkeypatch):
    # key j compared with the id of key Skv - 1 - j (a reversed index); the
    # oracle's forward uses the broken predicate, the brute force its own copy
    orig = A.allowed_rows

    def broken(mask, b, rows, Sq, Skv):
        if mask.seg_kv is not None:
            mask = oracle.MaskDesc(**{**mask.__dict__, "seg_kv": np.ascontiguousarray(mask.seg_kv[:, ::-1])})
        return orig(mask, b, rows, Sq, Skv)

    monkeypatch.setattr(A, "allowed_rows", broken)
    _must_fail(pins.test_forward_matches_brute_force, "segments")


def test_a_block_bound_over_the_diagonal_block_only_is_caught(monkeypatch):
    # kmax of q-block m taken over kv block m alone instead of every block its
    # rows reach: a window row whose allowed keys lie in earlier blocks is no
    # longer bounded
    import oracle.bound as Bd

    def broken(q, k, mask, scale, gate_limit=64.0, tile=128):
        q, k = A._as64(q), A._as64(k)
        B, Sq, H, D = q.shape
        nM = -(-Sq // tile)
        kmax = np.zeros((B, H, nM))
        qmax = np.zeros((B, H, nM))
        for b in range(B):
            for h in range(H):
                kn = np.sqrt((k[b, :, h] ** 2).sum(axis=1))
                qn = np.sqrt((q[b, :, h] ** 2).sum(axis=1))
                for m in range(nM):
                    kmax[b, h, m] = kn[m * tile:(m + 1) * tile].max() if m * tile < kn.size else 0.0
                    qmax[b, h, m] = qn[m * tile:(m + 1) * tile].max()
        bound = scale * qmax * kmax
        return kmax, qmax, bound, 2 * bound <= gate_limit

    from tests import test_oracle_bound_blocks as tb
    monkeypatch.setattr(Bd, "fixed_m_bound_blocks", broken)
    monkeypatch.setattr(oracle, "fixed_m_bound_blocks", broken)
    _must_fail(tb.test_block_bound_dominates_allowed_scores_and_the_head_bound, "window3")
