"""Pins of the per q-block fixed-m bound (oracle/bound.py), CPU only: Cauchy-
Schwarz dominance of every allowed score, never looser than the per-head bound
and equal to it without a mask, a closed form on packed segments with one hot
segment, and the fixed-m form with these references equal to online softmax."""

import math

import numpy as np
import pytest

import oracle
from oracle import MaskDesc
from tests import oracle_pins as P

SCALE = 0.37
TILE = 4  # small tiles, so that tiny inputs span several q- and kv-blocks


@pytest.mark.parametrize("case", list(P.tiny_masks(2, 18, 22).keys()))
def test_block_bound_dominates_allowed_scores_and_the_head_bound(case):
    q, k, v, _ = P.tiny_inputs(51, B=2, Sq=18, Skv=22, D=5)
    mask = P.tiny_masks(2, 18, 22, seed=3)[case]
    kmax, qmax, bound, gate = oracle.fixed_m_bound_blocks(q, k, mask, SCALE, tile=TILE)
    kh = oracle.fixed_m_bound(q, k, mask, SCALE)[0]
    m_rows = oracle.row_references_blocks(q, kmax, SCALE, tile=TILE)
    for b in range(2):
        a = oracle.allowed_rows(mask, b, np.arange(18), 18, 22)
        for h in range(2):
            s = SCALE * q[b, :, h] @ k[b, :, h].T
            assert (np.where(a, s, -np.inf) <= m_rows[b, h][:, None] + 1e-12).all(), case
            # a q-block's reachable keys are a subset of the valid keys
            assert (kmax[b, h] <= kh[b, h] + 1e-15).all()
            for mb in range(kmax.shape[2]):
                rows = slice(mb * TILE, (mb + 1) * TILE)
                assert qmax[b, h, mb] == np.linalg.norm(q[b, rows, h], axis=1).max()
    assert np.array_equal(gate, 2 * SCALE * qmax * kmax <= 64.0)


def test_block_bound_without_a_mask_is_the_head_bound():
    q, k, _, _ = P.tiny_inputs(52, B=1, Sq=16, Skv=20, D=6)
    kmax, _, _, _ = oracle.fixed_m_bound_blocks(q, k, MaskDesc(), SCALE, tile=TILE)
    kh = oracle.fixed_m_bound(q, k, MaskDesc(), SCALE)[0]
    for h in range(2):
        assert (kmax[0, h] == kh[0, h]).all()


def test_block_bound_closed_form_with_one_hot_segment():
    """Packed segments of 16 keys (two 8-key blocks each); the keys of segment 1
    are scaled x20.  Each q-block reaches exactly its own segment's two kv
    blocks, so its kmax is the largest key norm of its segment, taken straight
    from the key slice; with a gate limit between the cold and the hot
    segments' bounds, every q-block but the hot segment's passes, while the
    per-head gate (whose kmax includes the hot keys) fails everywhere."""
    rng = np.random.default_rng(53)
    S, H, D, tile = 64, 2, 8, 8
    q = rng.standard_normal((1, S, H, D))
    k = rng.standard_normal((1, S, H, D))
    k[0, 16:32] *= 20.0
    seg = (np.arange(S) // 16)[None, :]
    mask = MaskDesc(seg_q=seg, seg_kv=seg)
    scale = 1 / math.sqrt(D)
    kmax, qmax, bound, _ = oracle.fixed_m_bound_blocks(q, k, mask, scale, tile=tile)
    for h in range(H):
        for mb in range(S // tile):
            s = mb // 2
            assert kmax[0, h, mb] == np.linalg.norm(k[0, 16 * s:16 * s + 16, h], axis=1).max()
    cold = 2 * bound[0][:, [0, 1, 4, 5, 6, 7]].max()
    hot = 2 * bound[0][:, [2, 3]].min()
    assert cold < hot
    G = 0.5 * (cold + hot)
    gate = oracle.fixed_m_bound_blocks(q, k, mask, scale, gate_limit=G, tile=tile)[3]
    assert gate[0][:, [0, 1, 4, 5, 6, 7]].all() and not gate[0][:, [2, 3]].any()
    assert not oracle.fixed_m_bound(q, k, mask, scale, gate_limit=G)[3].any()
    # per row: a q-block that passes passes every one of its rows (qmax bounds
    # each row's norm); in a failing block at least the row of largest norm fails
    rows = oracle.gate_rows_blocks(q, kmax, scale, gate_limit=G, tile=tile)
    for h in range(H):
        for mb in range(S // tile):
            r = rows[0, h, mb * tile:(mb + 1) * tile]
            if gate[0, h, mb]:
                assert r.all()
            else:
                assert not r[np.argmax(np.linalg.norm(q[0, mb * tile:(mb + 1) * tile, h], axis=1))]


def test_fixed_m_with_block_references_equals_online():
    q, k, v, _ = P.tiny_inputs(54, B=2, Sq=20, Skv=24, D=6)
    for name, m in P.tiny_masks(2, 20, 24, seed=4).items():
        kmax = oracle.fixed_m_bound_blocks(q, k, m, SCALE, tile=TILE)[0]
        m_rows = oracle.row_references_blocks(q, kmax, SCALE, tile=TILE)
        a = oracle.attention_forward(q, k, v, m, SCALE)
        b = oracle.attention_forward_fixed_m(q, k, v, m, SCALE, m_rows=m_rows)
        assert np.max(np.abs(a[0] - b[0])) < 1e-12, name
        fin = np.isfinite(a[1])
        assert np.array_equal(fin, np.isfinite(b[1]))
        assert np.max(np.abs(a[1][fin] - b[1][fin])) < 1e-12, name
