"""fp64 oracle: dense masked softmax attention, analytic backward, fixed-m form.

TEST INFRASTRUCTURE ONLY (see the package docstring).  Every quantity is the
plain dense definition, evaluated in float64 on the CPU one (batch, head, row
chunk) at a time.  Row chunking is a memory measure only: each row's softmax is
independent, so no reordering beyond the definition takes place.

Sources (the pages of the subject):

* "Fixed-m softmax for 2D-ring x Ulysses attention (WAN 2.2)" (maxdiffusion
  PR #452), introduction and "Notes": exact softmax attention whose per-query max
  may be pinned to the Cauchy-Schwarz bound scale*||q_i||*max_j ||k_j||; the
  output is exact either way; the per-row LSE is the quantity partial results
  merge in.
* "Let splash attention exceed 524,288 tokens when packing is off" (maxtext
  PR #4929), summary: the segment-id mask (query i sees key j iff their segment
  ids are equal); constant ids give the same result as no ids.
* maxdiffusion PR #404 review, comment on the padding mask: KV padding exists
  only at the end of the global sequence and is masked by global position.
* sglang PR #47566, "Modifications": varlen ``cu_seqlens`` whose trailing
  alignment segment is never attended by real rows; alignment rows are zeroed.
* "Add more optimal dk order optional arg" (flash-attention PR #2512): sliding
  window masks (causal band of W keys) and the backward dQ/dK/dV.  Its
  benchmark ("The numbers") also names prefix_lm, dilated_sliding_window and
  document masks without defining them; the readings taken are stated in
  :class:`MaskDesc` and :func:`allowed_rows`.
"""

from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import numpy as np

NEG_INF = -np.inf


@dataclass
class MaskDesc:
    """The enabled mask predicates.  ``None`` / absent means the predicate is off.

    seg_q, seg_kv : int arrays [B, Sq] / [B, Skv]   (segment ids)
    kv_valid_len  : int array [B]                    (global KV padding)
    cu_seqlens    : int array [n_seqs + 1]           (varlen, requires B == 1)
    n_align_tail  : number of trailing cu_seqlens segments that are alignment rows
    window        : None = no window; 0 = plain causal; W > 0 = causal band of W
                    keys including the diagonal, bottom-right aligned.
    dilation      : (with a window) keep only the keys whose distance back from
                    the diagonal is a multiple of ``dilation`` (<= 1: all keys);
                    the reading taken for "dilated_sliding_window".
    prefix_len    : int array [B] (with a window): keys j < prefix_len[b] are
                    seen by every row as well; the reading taken for
                    "prefix_lm" (a bidirectional prefix, causal after it).
    "document" masks are segment ids (one id per document), optionally with
    a window (document-causal).
    """

    seg_q: Optional[np.ndarray] = None
    seg_kv: Optional[np.ndarray] = None
    kv_valid_len: Optional[np.ndarray] = None
    cu_seqlens: Optional[np.ndarray] = None
    n_align_tail: int = 0
    window: Optional[int] = None
    dilation: int = 1
    prefix_len: Optional[np.ndarray] = None


def _segment_of(cu_seqlens: np.ndarray, pos: np.ndarray) -> np.ndarray:
    """Index of the cu_seqlens segment that holds each position."""
    return np.searchsorted(np.asarray(cu_seqlens), pos, side="right") - 1


def allowed_rows(mask: MaskDesc, b: int, rows: np.ndarray, Sq: int, Skv: int) -> np.ndarray:
    """bool [len(rows), Skv]: allowed(i, j), the AND of every enabled predicate.

    * segment ids (maxtext PR #4929): seg_q[b, i] == seg_kv[b, j]
    * global KV padding (maxdiffusion PR #404 review): j < kv_valid_len[b]
    * varlen (sglang PR #47566, "Modifications"): i and j lie in the same
      cu_seqlens segment and neither lies in one of the trailing ``n_align_tail``
      alignment segments
    * causal window (flash-attention PR #2512 sliding_window masks; causal and
      bottom-right aligned when Sq != Skv): with o = Skv - Sq and the distance
      t = i + o - j of key j back from the diagonal,
      0 <= t < W   (W = 0: only 0 <= t),
      with a dilation d > 1 also t mod d == 0 (dilated_sliding_window), and with
      a prefix OR j < prefix_len[b] (prefix_lm).
    """
    rows = np.asarray(rows, dtype=np.int64)
    i = rows[:, None]
    j = np.arange(Skv, dtype=np.int64)[None, :]
    ok = np.ones((rows.size, Skv), dtype=bool)
    if mask.seg_q is not None:
        sq = np.asarray(mask.seg_q)[b, rows]
        sk = np.asarray(mask.seg_kv)[b]
        ok &= sq[:, None] == sk[None, :]
    if mask.kv_valid_len is not None:
        ok &= j < int(np.asarray(mask.kv_valid_len)[b])
    if mask.cu_seqlens is not None:
        cu = np.asarray(mask.cu_seqlens, dtype=np.int64)
        n_real = (cu.size - 1) - int(mask.n_align_tail)
        si = _segment_of(cu, rows)
        sj = _segment_of(cu, np.arange(Skv))
        ok &= (si[:, None] == sj[None, :]) & (si[:, None] < n_real) & (sj[None, :] < n_real)
    if mask.window is not None:
        t = (i + (Skv - Sq)) - j
        band = t >= 0
        if mask.window > 0:
            band &= t < int(mask.window)
        if mask.dilation > 1:
            band &= np.mod(t, int(mask.dilation)) == 0
        if mask.prefix_len is not None:
            band |= j < int(np.asarray(mask.prefix_len)[b])
        ok &= band
    elif mask.prefix_len is not None or mask.dilation > 1:
        raise ValueError("a prefix or a dilation modifies the causal window; set window")
    return ok


def valid_keys(mask: MaskDesc, b: int, Skv: int) -> np.ndarray:
    """bool [Skv]: keys that some real row may see at all.

    The fixed-m bound takes its max ||k_j|| over these keys only: padding keys
    (maxdiffusion PR #404 review) and alignment keys (sglang PR #47566) are
    never attended, so they must not loosen the bound.  Segment ids and the
    window restrict keys per row, not globally, so they do not enter.
    """
    ok = np.ones(Skv, dtype=bool)
    j = np.arange(Skv)
    if mask.kv_valid_len is not None:
        ok &= j < int(np.asarray(mask.kv_valid_len)[b])
    if mask.cu_seqlens is not None:
        cu = np.asarray(mask.cu_seqlens, dtype=np.int64)
        n_real = (cu.size - 1) - int(mask.n_align_tail)
        ok &= _segment_of(cu, j) < n_real
    return ok


def _as64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def kv_head_of(H: int, H_kv: int):
    """Grouped-query attention (GQA / MQA): query head h reads key/value head
    h // (H / H_kv), so consecutive query heads share one kv head (H_kv == H is
    plain multi-head attention, H_kv == 1 multi-query).  The pages only name the
    "kv_mode" column of the dk-order benchmark (all of whose rows are MHA); this
    contiguous grouping is the reading taken."""
    if H_kv < 1 or H % H_kv != 0:
        raise ValueError("H must be a multiple of the kv head count")
    g = H // H_kv
    return lambda h: h // g


def _row_chunks(rows: np.ndarray, chunk: int):
    for s in range(0, rows.size, chunk):
        yield rows[s:s + chunk]


def attention_forward(q, k, v, mask: MaskDesc, scale: float, rows=None, heads=None,
                      batches=None, chunk: int = 1024):
    """O = softmax(scale * Q K^T + mask) V and LSE, dense, per row.

    q: [B, Sq, H, D], k, v: [B, Skv, H_kv, D] (any float type; computed in fp64),
    H a multiple of H_kv (:func:`kv_head_of`).
    Returns (O [B, Sq, H, D] fp64, LSE [B, H, Sq] fp64).  Rows outside ``rows``
    (and heads/batches outside the given subsets) are left as NaN.

    A row with no allowed key has O = 0 and LSE = -inf (the log of an empty sum);
    the pages never state this case, this is the reading the build takes.
    """
    q, k, v = _as64(q), _as64(k), _as64(v)
    B, Sq, H, D = q.shape
    Skv = k.shape[1]
    rows = np.arange(Sq) if rows is None else np.asarray(rows)
    heads = range(H) if heads is None else heads
    batches = range(B) if batches is None else batches
    kvh = kv_head_of(H, k.shape[2])
    O = np.full((B, Sq, H, v.shape[3]), np.nan)
    LSE = np.full((B, H, Sq), np.nan)
    for b in batches:
        for r in _row_chunks(rows, chunk):
            a = allowed_rows(mask, b, r, Sq, Skv)
            has = a.any(axis=1)
            for h in heads:
                hk = kvh(h)
                s = scale * (q[b, r, h, :] @ k[b, :, hk, :].T)
                s = np.where(a, s, NEG_INF)
                M = np.where(has, s.max(axis=1), 0.0)
                e = np.where(a, np.exp(s - M[:, None]), 0.0)
                l = e.sum(axis=1)
                safe_l = np.where(has, l, 1.0)
                P = e / safe_l[:, None]
                O[b, r, h, :] = P @ v[b, :, hk, :]
                LSE[b, h, r] = np.where(has, M + np.log(safe_l), NEG_INF)
    return O, LSE


def attention_backward(q, k, v, dO, mask: MaskDesc, scale: float, chunk: int = 1024,
                       heads=None, batches=None, ds_out=None):
    """Analytic gradient of sum(O * dO) for the dense definition above.

    With P the softmax weights (0 on masked entries and on empty rows):
      Delta_i = sum_d dO_id O_id   (O from this oracle's own forward)
      dP = dO V^T,  dS = P o (dP - Delta),
      dQ = scale * dS K,  dK = scale * dS^T Q,  dV = P^T dO,
    with dK and dV of a shared kv head summed over the query heads of its group.
    Returns (dQ, dK, dV) fp64 with the input layouts.  A dict passed as
    ``ds_out`` also receives dS as ds_out[(b, h)] = [Sq, Skv] (small inputs).
    """
    q, k, v, dO = _as64(q), _as64(k), _as64(v), _as64(dO)
    B, Sq, H, D = q.shape
    Skv = k.shape[1]
    heads = range(H) if heads is None else heads
    batches = range(B) if batches is None else batches
    kvh = kv_head_of(H, k.shape[2])
    dQ = np.zeros_like(q)
    dK = np.zeros_like(k)
    dV = np.zeros_like(v)
    rows = np.arange(Sq)
    for b in batches:
        for r in _row_chunks(rows, chunk):
            a = allowed_rows(mask, b, r, Sq, Skv)
            has = a.any(axis=1)
            for h in heads:
                hk = kvh(h)
                s = scale * (q[b, r, h, :] @ k[b, :, hk, :].T)
                s = np.where(a, s, NEG_INF)
                M = np.where(has, s.max(axis=1), 0.0)
                e = np.where(a, np.exp(s - M[:, None]), 0.0)
                l = np.where(has, e.sum(axis=1), 1.0)
                P = e / l[:, None]
                O = P @ v[b, :, hk, :]
                do = dO[b, r, h, :]
                delta = (do * O).sum(axis=1)
                dP = do @ v[b, :, hk, :].T
                dS = P * (dP - delta[:, None])
                if ds_out is not None:
                    ds_out.setdefault((b, h), np.zeros((Sq, Skv)))[r, :] = dS
                dQ[b, r, h, :] = scale * (dS @ k[b, :, hk, :])
                dK[b, :, hk, :] += scale * (dS.T @ q[b, r, h, :])
                dV[b, :, hk, :] += P.T @ do
    return dQ, dK, dV


def attention_forward_fixed_m(q, k, v, mask: MaskDesc, scale: float, kmax=None,
                              rows=None, heads=None, batches=None, chunk: int = 1024,
                              kbar=None, m_rows=None):
    """The fixed-m form ("Fixed-m softmax ...", introduction).

    Instead of the row max, each query's reference is pinned before streaming to
      m_i = scale * ||q_i|| * kmax[b, h],   kmax = max over valid keys of ||k_j||
    (Cauchy-Schwarz: s_ij <= m_i for every key).  Then
      l_i = sum_{j allowed} exp(s_ij - m_i),  LSE_i = m_i + ln l_i,
      O_i = sum_j exp(s_ij - m_i) v_j / l_i.
    In exact arithmetic this equals :func:`attention_forward`; ``kmax`` may be a
    caller-supplied bound [B, H] (any upper bound keeps the result exact).

    With a key center ``kbar`` [B, H, D] (k-smoothing, see
    :func:`fixed_m_bound_smoothed`) ``kmax`` is the radius max_j ||k_j - kbar||
    and the pinned reference is m_i = scale * (q_i . kbar + ||q_i|| * kmax),
    again an upper bound of every s_ij by Cauchy-Schwarz on k_j - kbar.

    ``m_rows`` [B, H, Sq], when given, is each row's pinned reference itself
    (e.g. the per q-block bound of :mod:`oracle.bound`); ``kmax`` and ``kbar``
    are then unused.
    """
    q, k, v = _as64(q), _as64(k), _as64(v)
    B, Sq, H, D = q.shape
    Skv = k.shape[1]
    if kmax is None and m_rows is None:
        kmax = fixed_m_bound(q, k, mask, scale)[0]
    kmax = _as64(kmax) if m_rows is None else None
    kvh = kv_head_of(H, k.shape[2])
    rows = np.arange(Sq) if rows is None else np.asarray(rows)
    heads = range(H) if heads is None else heads
    batches = range(B) if batches is None else batches
    O = np.full((B, Sq, H, v.shape[3]), np.nan)
    LSE = np.full((B, H, Sq), np.nan)
    for b in batches:
        for r in _row_chunks(rows, chunk):
            a = allowed_rows(mask, b, r, Sq, Skv)
            has = a.any(axis=1)
            for h in heads:
                qr = q[b, r, h, :]
                if m_rows is not None:
                    m = _as64(m_rows)[b, h, r]
                else:
                    m = scale * np.sqrt((qr * qr).sum(axis=1)) * kmax[b, h]
                    if kbar is not None:
                        m = m + scale * (qr @ _as64(kbar)[b, h])
                s = scale * (qr @ k[b, :, kvh(h), :].T)
                e = np.where(a, np.exp(s - m[:, None]), 0.0)
                l = e.sum(axis=1)
                safe_l = np.where(has, l, 1.0)
                O[b, r, h, :] = (e / safe_l[:, None]) @ v[b, :, kvh(h), :]
                LSE[b, h, r] = np.where(has, m + np.log(safe_l), NEG_INF)
    return O, LSE


def fixed_m_bound(q, k, mask: MaskDesc, scale: float, gate_limit: float = 64.0):
    """kmax, qmax, per-head bound and gate ("Fixed-m softmax ...", "Notes").

      kmax[b, h] = max over valid keys j of ||k_j||_2
      qmax[b, h] = max over all rows i < Sq of ||q_i||_2
      bound[b, h] = scale * qmax * kmax
      gate[b, h]  = 2 * bound <= gate_limit

    Every score satisfies |s_ij| <= bound, so the gap between the pinned m_i and
    the true row max is at most 2 * bound (the two-sided reading of the page's
    "halved bound").  A head passes the gate when that worst gap is at most
    ``gate_limit`` natural-log units; heads that fail keep online softmax.
    Returns (kmax, qmax, bound, gate) as fp64 / bool arrays [B, H].
    """
    q, k = _as64(q), _as64(k)
    B, Sq, H, D = q.shape
    Skv = k.shape[1]
    kvh = kv_head_of(H, k.shape[2])
    kmax = np.zeros((B, H))
    qmax = np.zeros((B, H))
    for b in range(B):
        vk = valid_keys(mask, b, Skv)
        for h in range(H):
            kn = np.sqrt((k[b, :, kvh(h), :] ** 2).sum(axis=1))
            kmax[b, h] = kn[vk].max() if vk.any() else 0.0
            qmax[b, h] = np.sqrt((q[b, :, h, :] ** 2).sum(axis=1)).max()
    bound = scale * qmax * kmax
    gate = 2.0 * bound <= gate_limit
    return kmax, qmax, bound, gate


def fixed_m_bound_smoothed(q, k, mask: MaskDesc, scale: float, gate_limit: float = 64.0):
    """The k-smoothed bound ("Fixed-m softmax ...", "Notes": k-smoothing, impossible
    on a ring because no rank holds the full K, is possible when one device holds
    all of K).

    Softmax is invariant to a per-row shift, and s_ij = scale * q_i . kbar +
    scale * q_i . (k_j - kbar) for any vector kbar.  Reading taken: kbar is the
    mean of the valid keys of the head, R its radius, and

      kbar[b, h]   = mean over valid keys j of k_j
      radius[b, h] = max over valid keys j of ||k_j - kbar||
      m_i          = scale * (q_i . kbar + ||q_i|| * radius)     (>= every s_ij)
      bound[b, h]  = scale * qmax * radius
      gate[b, h]   = 2 * bound <= gate_limit

    since every s_ij - scale * q_i . kbar lies in [-scale ||q_i|| radius,
    scale ||q_i|| radius], the pinned m_i sits at most 2 * bound above the row
    max.  Returns (kbar [B, H, D], radius, qmax, bound, gate), indexed by query
    head (with GQA the query heads of a group share their kv head's values).
    """
    q, k = _as64(q), _as64(k)
    B, Sq, H, D = q.shape
    Skv = k.shape[1]
    kvh = kv_head_of(H, k.shape[2])
    kbar = np.zeros((B, H, D))
    radius = np.zeros((B, H))
    qmax = np.zeros((B, H))
    for b in range(B):
        vk = valid_keys(mask, b, Skv)
        for h in range(H):
            if vk.any():
                kv = k[b, vk, kvh(h), :]
                kbar[b, h] = kv.mean(axis=0)
                radius[b, h] = np.sqrt(((kv - kbar[b, h]) ** 2).sum(axis=1)).max()
            qmax[b, h] = np.sqrt((q[b, :, h, :] ** 2).sum(axis=1)).max()
    bound = scale * qmax * radius
    gate = 2.0 * bound <= gate_limit
    return kbar, radius, qmax, bound, gate


def useful_flops(n_tiles: int, D: int, tile: int = 128, backward: bool = False) -> float:
    """Flops credited to the non-empty tiles of a block map.

    Forward: two tile GEMMs (S = Q K^T and O += P V), 2 * 2 * tile * tile * D.
    Backward: five tile GEMMs (S, dP, dV, dK, dQ), 2.5x the forward.
    """
    f = 4.0 * tile * tile * D * n_tiles
    return 2.5 * f if backward else f
