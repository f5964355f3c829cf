"""The block-map / rank / semaphore oracle pinned to closed forms, the page's
worked rank example and a discrete simulation (CPU only)."""

import json
import os

import numpy as np
import pytest

import oracle
from oracle import EMPTY, FULL, PARTIAL, MaskDesc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _counts(cls):
    return int((cls != EMPTY).sum()), int((cls == FULL).sum()), int((cls == PARTIAL).sum())


def test_window_8192_tile_counts_closed_form():
    # Row block m >= 4 reaches kv blocks m-4 (partial: left window edge),
    # m-3..m-1 (full) and m (partial: the diagonal); rows 0..3 are clipped.
    cls = oracle.tile_classes(MaskDesc(window=512), 1, 8192, 8192)
    assert _counts(cls) == (310, 186, 124)
    for m in range(4, 64):
        row = cls[0, m]
        assert row[m - 4] == PARTIAL and row[m] == PARTIAL
        assert (row[m - 3:m] == FULL).all() and (row != EMPTY).sum() == 5


def test_window_rect_tile_counts_closed_form():
    # Sq=4096, Skv=8192 bottom-right: row block m reaches kv blocks m+28..m+32.
    cls = oracle.tile_classes(MaskDesc(window=512), 1, 4096, 8192)
    assert _counts(cls) == (160, 96, 64)
    for m in range(32):
        assert cls[0, m, m + 28] == PARTIAL and cls[0, m, m + 32] == PARTIAL
        assert (cls[0, m, m + 29:m + 32] == FULL).all()


def test_varlen_alignment_tiles_closed_form():
    # cu_seqlens = [0, 33002, 33024]: 258 blocks; the last q block holds 106 real
    # rows and the 22 alignment rows, the last kv block likewise.
    cls = oracle.tile_classes(MaskDesc(cu_seqlens=np.array([0, 33002, 33024]), n_align_tail=1),
                              1, 33024, 33024)
    assert cls.shape == (1, 258, 258)
    assert (cls[0, :257, :257] == FULL).all()
    assert (cls[0, 257, :] == PARTIAL).all() and (cls[0, :, 257] == PARTIAL).all()


def test_padding_tiles_closed_form_video_shape():
    # Skv = 75776 = 592 blocks, valid keys < 75600: block 590 straddles the end
    # of the valid keys, block 591 is pure padding.
    Sq, Skv = 75600, 75776
    cls = oracle.tile_classes(MaskDesc(kv_valid_len=np.array([Sq])), 1, 256, Skv)
    assert (cls[0, :, :590] == FULL).all()
    assert (cls[0, :, 590] == PARTIAL).all() and (cls[0, :, 591] == EMPTY).all()


def test_segment_tiles_closed_form_aligned_runs():
    ids = np.repeat(np.arange(4), [128, 256, 128, 512])[None, :]
    cls = oracle.tile_classes(MaskDesc(seg_q=ids, seg_kv=ids), 1, 1024, 1024)
    blk_seg = ids[0, ::128]
    expect = np.where(blk_seg[:, None] == blk_seg[None, :], FULL, EMPTY)
    assert np.array_equal(cls[0], expect)
    const = np.zeros((1, 1000), dtype=np.int32)
    cls = oracle.tile_classes(MaskDesc(seg_q=const, seg_kv=const), 1, 1000, 1000)
    # out-of-range columns of the ragged last kv block make it partial
    assert (cls[0, :, :7] == FULL).all() and (cls[0, :, 7] == PARTIAL).all()


def test_rank_example_of_the_page():
    g = json.load(open(os.path.join(GOLDEN, "rank_example_sliding_window.json")))
    w, n = g["band_width_blocks"], g["column"]
    nb = 12
    cls = np.zeros((1, nb, nb), dtype=np.uint8)
    for m in range(nb):
        for c in range(m, min(nb, m + w)):
            cls[0, m, c] = PARTIAL if c in (m, m + w - 1) else FULL
    pi = oracle.column_order(nb, g["order"])
    rank = oracle.kv_ranks(cls, pi)
    assert [int(rank[0, m, n]) for m in g["partial_m"]] == g["partial_rank"]
    first = oracle.partial_then_full_lists(cls, rank)[(0, n)][0]
    assert (first[0], first[1]) == (g["partial_then_full_walk_first_item"]["m"],
                                    g["partial_then_full_walk_first_item"]["rank"])
    unified = oracle.column_lists(cls, rank)[(0, n)]
    assert [r for (_, r, _) in unified] == sorted(r for (_, r, _) in unified)
    assert unified[0][0] == 4 and unified[0][1] == 0


def test_ranks_closed_form_for_causal_window():
    cls = oracle.tile_classes(MaskDesc(window=512), 1, 4096, 4096)
    asc = oracle.kv_ranks(cls, oracle.column_order(32, "asc"))
    desc = oracle.kv_ranks(cls, oracle.column_order(32, "desc"))
    for m in range(4, 32):
        for n in range(m - 4, m + 1):
            assert asc[0, m, n] == n - (m - 4)
            assert desc[0, m, n] == m - n
    assert (asc[cls == EMPTY] == -1).all()


@pytest.mark.parametrize("order", ["asc", "desc", "perm"])
@pytest.mark.parametrize("workers", [1, 3, 40])
def test_semaphore_protocol_deadlock_free_and_ordered(order, workers):
    rng = np.random.default_rng(0)
    cls = oracle.tile_classes(MaskDesc(window=512), 2, 2048, 3072)
    nN = cls.shape[2]
    pi = oracle.column_order(nN, order, rng.permutation(nN) if order == "perm" else None)
    rank = oracle.kv_ranks(cls, pi)
    lists = oracle.column_lists(cls, rank)
    done, _, acc = oracle.simulate_dq_semaphores(lists, pi, 2, cls.shape[1], workers)
    assert done
    for (b, m), seq in acc.items():
        expect = [int(n) for n in pi if cls[b, m, n] != EMPTY]
        assert seq == expect
        # the final count is the row's number of non-empty tiles: the dQ
        # convert takes a q-block as complete exactly when its semaphore
        # reaches the row list's length
        assert len(seq) == int((cls[b, m] != EMPTY).sum())


def test_unified_list_never_slower_than_partial_then_full():
    cls = oracle.tile_classes(MaskDesc(window=512), 1, 8192, 8192)
    pi = oracle.column_order(64, "asc")
    rank = oracle.kv_ranks(cls, pi)
    _, t_unified, _ = oracle.simulate_dq_semaphores(oracle.column_lists(cls, rank), pi, 1, 64, 64)
    done, t_old, _ = oracle.simulate_dq_semaphores(oracle.partial_then_full_lists(cls, rank),
                                                   pi, 1, 64, 64)
    assert done and t_unified < t_old


def test_random_segment_ids_classes_are_consistent_with_dense_mask():
    rng = np.random.default_rng(3)
    ids = rng.integers(0, 3, size=(1, 700)).astype(np.int32)
    cls = oracle.tile_classes(MaskDesc(seg_q=ids, seg_kv=ids), 1, 700, 700)
    a = oracle.allowed_rows(MaskDesc(seg_q=ids, seg_kv=ids), 0, np.arange(700), 700, 700)
    for m in range(cls.shape[1]):
        for n in range(cls.shape[2]):
            blk = a[m * 128:(m + 1) * 128, n * 128:(n + 1) * 128]
            full = blk.all() and blk.shape[1] == 128
            assert cls[0, m, n] == (FULL if full else PARTIAL if blk.any() else EMPTY)


def test_outside_in_order_closed_form():
    assert oracle.column_order(6, "outside_in").tolist() == [0, 5, 1, 4, 2, 3]
    assert oracle.column_order(5, "outside_in").tolist() == [0, 4, 1, 3, 2]
    assert oracle.column_order(1, "outside_in").tolist() == [0]


def test_greedy_order_hand_worked_causal_example():
    # Causal 3 x 3 block map: column 0 reaches rows {0,1,2}, column 1 {1,2},
    # column 2 {2}.  Step 1: every wait is 0 -> column 0.  Step 2: column 1
    # would wait 1 + 1 = 2, column 2 only 1 -> column 2.  Then column 1.
    cls = np.array([[[PARTIAL, EMPTY, EMPTY],
                     [FULL, PARTIAL, EMPTY],
                     [FULL, FULL, PARTIAL]]], dtype=np.uint8)
    assert oracle.greedy_order(cls).tolist() == [0, 2, 1]


def test_greedy_order_is_a_permutation_with_minimal_step_waits():
    cls = oracle.tile_classes(MaskDesc(window=512), 2, 2048, 3072)
    pi = oracle.column_order(cls.shape[2], "greedy", cls=cls)
    assert sorted(pi.tolist()) == list(range(cls.shape[2]))
    ne = cls != EMPTY
    cnt = np.zeros(cls.shape[:2], dtype=np.int64)
    placed = set()
    for n in pi:
        waits = {c: int((cnt * ne[:, :, c]).sum()) for c in range(cls.shape[2]) if c not in placed}
        assert waits[int(n)] == min(waits.values())
        assert int(n) == min(c for c, w in waits.items() if w == waits[int(n)])
        placed.add(int(n))
        cnt += ne[:, :, n]


@pytest.mark.parametrize("order", ["outside_in", "greedy"])
def test_new_orders_deadlock_free_and_ordered(order):
    cls = oracle.tile_classes(MaskDesc(window=512), 1, 4096, 4096)
    nN = cls.shape[2]
    pi = oracle.column_order(nN, order, cls=cls)
    rank = oracle.kv_ranks(cls, pi)
    done, _, acc = oracle.simulate_dq_semaphores(oracle.column_lists(cls, rank), pi, 1, cls.shape[1], 24)
    assert done
    for (b, m), seq in acc.items():
        assert seq == [int(n) for n in pi if cls[b, m, n] != EMPTY]


def test_prefix_lm_tile_counts_closed_form():
    # causal, prefix of 2048 keys = kv blocks 0..15: rows m < 16 reach exactly
    # those 16 blocks (all full); row m >= 16 adds blocks 16..m-1 (full) and the
    # diagonal block m (partial): 16*16 + sum_{m=16}^{63} (m + 1) tiles.
    cls = oracle.tile_classes(MaskDesc(window=0, prefix_len=np.array([2048])), 1, 8192, 8192)
    assert _counts(cls) == (2200, 2152, 48)


def test_dilated_window_tile_counts_closed_form():
    # span 1024, dilation 2: row block m reaches blocks max(0, m-8) .. m; no
    # 128-key block can be full when only every other key is kept.
    cls = oracle.tile_classes(MaskDesc(window=1024, dilation=2), 1, 8192, 8192)
    assert _counts(cls) == (36 + 56 * 9, 0, 540)


def test_document_causal_tile_counts_closed_form():
    # documents of 128, 256, 128, 512 tokens, causal inside each: the diagonal
    # blocks are partial, the same-document blocks below them full.
    ids = np.repeat(np.arange(4), [128, 256, 128, 512])[None, :]
    cls = oracle.tile_classes(MaskDesc(seg_q=ids, seg_kv=ids, window=0), 1, 1024, 1024)
    assert _counts(cls) == (15, 7, 8)
