"""fp64-free integer oracle: block map, kv-column orders, ranks, dQ semaphores.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Sources:

* "Let splash attention exceed 524,288 tokens when packing is off" (maxtext
  PR #4929), "Effect": a block mask over (q-block, kv-block) tiles; the build
  keeps it as per-tile classes instead of a dense SMEM-resident mask.
* "Add more optimal dk order optional arg" (flash-attention PR #2512),
  "Sliding window perf issue" and "A simplish fix": per-m_block dQ semaphores,
  rank(m, n) = the value the semaphore must reach before column n may add its
  contribution to dQ[m], kv-column iteration orders (ascending, descending, an
  arbitrary permutation), and one unified list per column walked in rank order
  instead of "partial blocks first, then full blocks".
"""

from __future__ import annotations

import numpy as np

from .attention import MaskDesc, allowed_rows

EMPTY, PARTIAL, FULL = 0, 1, 2


def tile_classes(mask: MaskDesc, B: int, Sq: int, Skv: int, tile: int = 128) -> np.ndarray:
    """uint8 [B, nM, nN]: EMPTY / PARTIAL / FULL for every (q-block, kv-block) tile.

    Classified from the dense mask by brute force: rows i < Sq of block m and
    columns j < nN * tile of block n, where columns j >= Skv are never allowed.
    EMPTY: no allowed pair.  FULL: every pair allowed.  PARTIAL otherwise.
    """
    nM = -(-Sq // tile)
    nN = -(-Skv // tile)
    cls = np.zeros((B, nM, nN), dtype=np.uint8)
    for b in range(B):
        for m in range(nM):
            rows = np.arange(m * tile, min((m + 1) * tile, Sq))
            a = np.zeros((rows.size, nN * tile), dtype=bool)
            a[:, :Skv] = allowed_rows(mask, b, rows, Sq, Skv)
            blk = a.reshape(rows.size, nN, tile)
            anyv = blk.any(axis=(0, 2))
            allv = blk.all(axis=(0, 2))
            cls[b, m] = np.where(allv, FULL, np.where(anyv, PARTIAL, EMPTY))
    return cls


def column_order(nN: int, order: str = "asc", perm=None, cls=None) -> np.ndarray:
    """pi: the kv-column iteration order (flash-attention PR #2512, "What does this
    do" and "The numbers").

    "asc" walks columns left to right, "desc" right to left, "perm" takes an
    arbitrary permutation of range(nN).  The page's table also names
    "outside_in" and "greedy" without defining them; the readings taken here:

    * outside_in: the two ends first, then inwards: 0, nN-1, 1, nN-2, ...
    * greedy: see :func:`greedy_order` (needs the tile classes ``cls``).
    """
    if order == "asc":
        return np.arange(nN)
    if order == "desc":
        return np.arange(nN)[::-1].copy()
    if order == "outside_in":
        out = []
        lo, hi = 0, nN - 1
        while lo <= hi:
            out.append(lo)
            if hi != lo:
                out.append(hi)
            lo, hi = lo + 1, hi - 1
        return np.asarray(out, dtype=np.int64)
    if order == "greedy":
        return greedy_order(cls)
    if order == "perm":
        p = np.asarray(perm, dtype=np.int64)
        if sorted(p.tolist()) != list(range(nN)):
            raise ValueError("perm is not a permutation of the kv blocks")
        return p
    raise ValueError(order)


def greedy_order(cls: np.ndarray) -> np.ndarray:
    """A greedy order on presumed semaphore wait (flash-attention PR #2512, "What
    does this do": a scheduling heuristic for presumed semaphore wait time).

    Reading taken: the columns are placed one at a time.  Placing column n gives
    each of its non-empty tiles (b, m, n) the rank cnt[b, m] = number of columns
    already placed that also reach row block m, and that column must wait for
    all of them.  At every step the unplaced column with the smallest total
    presumed wait sum_{b, m non-empty} cnt[b, m] is placed (ties: smaller n),
    then cnt[b, m] += 1 for its rows.
    """
    B, nM, nN = cls.shape
    ne = cls != EMPTY
    cnt = np.zeros((B, nM), dtype=np.int64)
    placed = np.zeros(nN, dtype=bool)
    out = []
    for _ in range(nN):
        best, best_w = -1, None
        for n in range(nN):
            if placed[n]:
                continue
            w = int((cnt * ne[:, :, n]).sum())
            if best_w is None or w < best_w:
                best, best_w = n, w
        out.append(best)
        placed[best] = True
        cnt += ne[:, :, best]
    return np.asarray(out, dtype=np.int64)


def kv_ranks(cls: np.ndarray, pi: np.ndarray) -> np.ndarray:
    """int32 [B, nM, nN]: rank(m, n), -1 where the tile is EMPTY.

    rank(m, n) = number of non-empty columns n' of row m that come before n in
    the order pi (flash-attention PR #2512, "Sliding window perf issue": the
    semaphore value of dQ m_block that column n waits for).
    """
    B, nM, nN = cls.shape
    pos = np.empty(nN, dtype=np.int64)
    pos[np.asarray(pi)] = np.arange(nN)
    rank = np.full((B, nM, nN), -1, dtype=np.int32)
    for b in range(B):
        for m in range(nM):
            cols = [n for n in range(nN) if cls[b, m, n] != EMPTY]
            cols.sort(key=lambda n: pos[n])
            for r, n in enumerate(cols):
                rank[b, m, n] = r
    return rank


def column_lists(cls: np.ndarray, rank: np.ndarray):
    """Per (b, n): the unified partial+full list of (m, rank, is_full), sorted by
    (rank, m) ("A simplish fix": one list per column, walked in rank-dependency
    order so that a column never blocks on an entry while an earlier-ranked one
    of its own is still pending).
    """
    B, nM, nN = cls.shape
    out = {}
    for b in range(B):
        for n in range(nN):
            ent = [(int(rank[b, m, n]), m, bool(cls[b, m, n] == FULL))
                   for m in range(nM) if cls[b, m, n] != EMPTY]
            ent.sort()
            out[(b, n)] = [(m, r, f) for (r, m, f) in ent]
    return out


def partial_then_full_lists(cls: np.ndarray, rank: np.ndarray):
    """The pre-fix walk ("Sliding window perf issue"): partial entries of a column
    first, then its full entries, each in ascending m.  Kept for the stall
    comparison only; the build's kernels walk :func:`column_lists`.
    """
    B, nM, nN = cls.shape
    out = {}
    for b in range(B):
        for n in range(nN):
            part = [(m, int(rank[b, m, n]), False) for m in range(nM) if cls[b, m, n] == PARTIAL]
            full = [(m, int(rank[b, m, n]), True) for m in range(nM) if cls[b, m, n] == FULL]
            out[(b, n)] = part + full
    return out


def simulate_dq_semaphores(lists, pi, B: int, nM: int, n_workers: int,
                           max_steps: int = 10_000_000):
    """Discrete replay of the deterministic dQ protocol.

    Columns are handed out as tickets in the order (b, pi[0]), (b, pi[1]), ...
    for b = 0..B-1 to ``n_workers`` workers.  A worker walks its column's list;
    for entry (m, rank) it may proceed only when sem[b, m] == rank, then it adds
    its dQ[m] contribution and increments sem[b, m].  One entry per worker per
    step.  Returns (finished, steps, order) where ``order[(b, m)]`` is the
    sequence of columns whose contributions reached dQ[m], and ``finished`` is
    False if no worker could make progress (a deadlock).
    """
    tickets = [(b, int(n)) for b in range(B) for n in pi]
    sem = np.zeros((B, nM), dtype=np.int64)
    order = {(b, m): [] for b in range(B) for m in range(nM)}
    workers = [None] * n_workers  # (b, n, position in list)
    nxt = 0
    steps = 0
    while True:
        for w in range(n_workers):
            if workers[w] is None and nxt < len(tickets):
                b, n = tickets[nxt]
                nxt += 1
                workers[w] = [b, n, 0]
        active = [w for w in range(n_workers) if workers[w] is not None]
        if not active and nxt >= len(tickets):
            return True, steps, order
        progressed = False
        grants = []
        for w in active:
            b, n, p = workers[w]
            lst = lists[(b, n)]
            if p >= len(lst):
                workers[w] = None
                progressed = True
                continue
            m, r, _ = lst[p]
            if sem[b, m] == r:
                grants.append((w, b, m, n))
        for (w, b, m, n) in grants:
            order[(b, m)].append(n)
            sem[b, m] += 1
            workers[w][2] += 1
            progressed = True
        steps += 1
        if not progressed or steps > max_steps:
            return False, steps, order
