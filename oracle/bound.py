"""fp64 oracle: the fixed-m bound per q-block (TEST INFRASTRUCTURE ONLY, see the
package docstring).

Source: "Fixed-m softmax for 2D-ring x Ulysses attention (WAN 2.2)",
introduction and "Notes".  The page pins each query's reference to the
Cauchy-Schwarz bound scale * ||q_i|| * max_j ||k_j|| and gates per head; its
"Notes" list a per-segment kmax beside k-smoothing as the ways to tighten the
bound.  Any set of keys that contains every key row i may see gives a valid
bound for that row.  Reading taken for "per-segment kmax": the keys of the kv
blocks that the block map lets q-block m reach (its non-empty tiles), so that

  kmax[b, h, m]  = max over valid keys j in the kv blocks n with tile (m, n)
                   non-empty of ||k_j||           (0 when the row block sees none)
  qmax[b, h, m]  = max over rows i of q-block m of ||q_i||
  bound[b, h, m] = scale * qmax * kmax
  gate[b, h, m]  = 2 * bound <= gate_limit        (the per-head gate's two-sided
                                                  reading, per q-block)
  m_i            = scale * ||q_i|| * kmax[b, h, m(i)]

For segment-id masks whose segments are whole kv blocks this is exactly the
per-segment maximum; windows and documents restrict it further.  It is never
looser than the per-head bound (a subset of the valid keys).
"""

from __future__ import annotations

import numpy as np

from .attention import MaskDesc, _as64, kv_head_of, valid_keys
from .blockmap import EMPTY, tile_classes


def fixed_m_bound_blocks(q, k, mask: MaskDesc, scale: float, gate_limit: float = 64.0,
                         tile: int = 128):
    """(kmax, qmax, bound, gate), each [B, H, nM] (gate bool), per q-block as in
    the module docstring."""
    q, k = _as64(q), _as64(k)
    B, Sq, H, D = q.shape
    Skv = k.shape[1]
    kvh = kv_head_of(H, k.shape[2])
    cls = tile_classes(mask, B, Sq, Skv, tile)
    nM, nN = cls.shape[1], cls.shape[2]
    kmax = np.zeros((B, H, nM))
    qmax = np.zeros((B, H, nM))
    for b in range(B):
        vk = valid_keys(mask, b, Skv)
        for h in range(H):
            kn = np.sqrt((k[b, :, kvh(h), :] ** 2).sum(axis=1))
            kn = np.where(vk, kn, 0.0)
            qn = np.sqrt((q[b, :, h, :] ** 2).sum(axis=1))
            for m in range(nM):
                qmax[b, h, m] = qn[m * tile:(m + 1) * tile].max()
                for n in np.nonzero(cls[b, m] != EMPTY)[0]:
                    seg = kn[n * tile:(n + 1) * tile]
                    kmax[b, h, m] = max(kmax[b, h, m], seg.max())
    bound = scale * qmax * kmax
    gate = 2.0 * bound <= gate_limit
    return kmax, qmax, bound, gate


def row_references_blocks(q, kmax_blocks, scale: float, tile: int = 128):
    """m_i = scale * ||q_i|| * kmax[b, h, i // tile], [B, H, Sq]."""
    q = _as64(q)
    B, Sq, H, D = q.shape
    qn = np.sqrt((q ** 2).sum(axis=3)).transpose(0, 2, 1)  # [B, H, Sq]
    blk = np.arange(Sq) // tile
    return scale * qn * np.asarray(kmax_blocks)[:, :, blk]


def gate_rows_blocks(q, kmax_blocks, scale: float, gate_limit: float = 64.0, tile: int = 128):
    """The per-row gate of the per q-block bound, [B, H, Sq] bool: row i runs
    fixed-m iff 2 * scale * ||q_i|| * kmax[b, h, m(i)] <= gate_limit (every
    score of the row lies within +-scale ||q_i|| kmax, so the pinned reference
    sits at most that far above the row's true maximum)."""
    return 2.0 * row_references_blocks(q, kmax_blocks, scale, tile) <= gate_limit
