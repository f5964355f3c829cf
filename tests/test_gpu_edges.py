"""Edge cases of the GPU path: empty problems, the longest sequence the library
accepts (checked on slices the oracle computes exactly), and rows or whole
batches with no allowed key."""

import numpy as np
import pytest
import torch

import block_sparse_attention_map_b200 as bsa
import oracle
from tests.gpu_common import LSE_TOL, check, compare_lse, compare_out, np64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,Sq", [(0, 256), (2, 0)])
def test_empty_problem_gives_empty_results(B, Sq):
    """No batch entry or no query row: nothing is launched and the outputs are
    empty, except that with key rows and no query row the backward writes
    dK = dV = 0 (one kernel)."""
    g = torch.Generator(device="cuda")
    g.manual_seed(9)
    Skv, H, D = 300, 2, 64
    q = torch.randn(B, Sq, H, D, device="cuda", generator=g).bfloat16()
    k = torch.randn(B, Skv, H, D, device="cuda", generator=g).bfloat16()
    v = torch.randn(B, Skv, H, D, device="cuda", generator=g).bfloat16()
    seg = {"seg_q": torch.zeros(B, Sq, dtype=torch.int32), "seg_kv": torch.zeros(B, Skv, dtype=torch.int32)}
    for mask in ({}, {"window": 0}, seg):
        n0 = bsa.launch_count()
        o, lse, ws = bsa.attn_fwd(q, k, v, mask)
        assert bsa.launch_count() == n0 and ws.nbytes == 0
        assert o.shape == q.shape and lse.shape == (B, H, Sq)
        dk0 = torch.full_like(k, float("nan"))
        dv0 = torch.full_like(v, float("nan"))
        dq, dk, dv, _ = bsa.attn_bwd(q, k, v, o, torch.zeros_like(q), lse, mask, dk=dk0, dv=dv0)
        torch.cuda.synchronize()
        assert bsa.launch_count() == n0 + (1 if B > 0 else 0)
        assert dq.shape == q.shape and dk.shape == k.shape
        assert (dk == 0).all() and (dv == 0).all()


@pytest.mark.parametrize("mode", ["online", "fixed_m"])
@pytest.mark.parametrize("D", [64, 128])
def test_rows_and_batches_without_keys(mode, D):
    """Batch 0 has no valid key (kv_valid_len 0) and 100 rows of batch 1 carry
    a segment id no key has: those rows give O = 0, LSE = -inf and dQ = 0, and
    keys no row sees get dK = dV = 0; the rest matches the oracle."""
    B, H, Sq, Skv = 2, 2, 300, 260
    g = torch.Generator(device="cuda")
    g.manual_seed(13)
    q, do = (torch.randn(B, Sq, H, D, device="cuda", generator=g).bfloat16() for _ in range(2))
    k, v = (torch.randn(B, Skv, H, D, device="cuda", generator=g).bfloat16() for _ in range(2))
    seg_q = np.zeros((B, Sq), np.int32)
    seg_q[1, :100] = 5
    seg_kv = np.zeros((B, Skv), np.int32)
    kvl = np.array([0, 200], np.int32)
    mask = {"seg_q": seg_q, "seg_kv": seg_kv, "kv_valid_len": kvl}
    o, lse, ws = bsa.attn_fwd(q, k, v, mask, softmax_mode=mode)
    dq, dk, dv, wsb = bsa.attn_bwd(q, k, v, o, do, lse, mask, workspace=ws)
    torch.cuda.synchronize()
    assert ws.status() == 0 and wsb.status() == 0
    md = oracle.MaskDesc(seg_q=seg_q, seg_kv=seg_kv, kv_valid_len=kvl)
    O_ref, L_ref = oracle.attention_forward(np64(q), np64(k), np64(v), md, D ** -0.5)
    compare_out(o, O_ref)
    el, same = compare_lse(lse, L_ref)
    assert el <= LSE_TOL and same
    assert (o[0] == 0).all() and (o[1, :100] == 0).all()
    assert torch.isneginf(lse[0]).all() and torch.isneginf(lse[1, :, :100]).all()
    gq, gk, gv = oracle.attention_backward(np64(q), np64(k), np64(v), np64(do), md, D ** -0.5)
    for name, x, ref in (("dQ", dq, gq), ("dK", dk, gk), ("dV", dv, gv)):
        check(name, x, ref)
    assert (dq[0] == 0).all() and (dq[1, :100] == 0).all()
    assert (dk[0] == 0).all() and (dv[0] == 0).all() and (dk[1, 200:] == 0).all() and (dv[1, 200:] == 0).all()


def test_longest_sequence_window_slices_match_oracle():
    """Sq = Skv = 2^21, the longest sequence the library accepts, one head,
    D = 128, the causal window of 512 keys (16384 x 16384 tiles in the map).
    Under the window, rows [s0, s0 + n) see only keys [s0 - 640, s0 + n), and a
    key j >= s0 gets gradient only from rows [j, j + 512), so the oracle on
    that slice is the exact reference for those rows (O, LSE, dQ) and for the
    keys whose rows all lie in it (dK, dV).  Slices at the start, at an offset
    off the 128-row tiles in the middle, and at the end."""
    S, H, D, W, n, halo = 1 << 21, 1, 128, 512, 4096, 640
    g = torch.Generator(device="cuda")
    g.manual_seed(2)
    q, k, v, do = (torch.randn(1, S, H, D, device="cuda", generator=g).bfloat16() for _ in range(4))
    mask = {"window": W}
    o, lse, ws = bsa.attn_fwd(q, k, v, mask)
    dq, dk, dv, wsb = bsa.attn_bwd(q, k, v, o, do, lse, mask, order="desc", workspace=ws)
    torch.cuda.synchronize()
    assert ws.status() == 0 and wsb.status() == 0
    md = oracle.MaskDesc(window=W)
    for s0 in (0, S // 2 + 64, S - n):
        k0 = max(s0 - halo, 0)
        rq, rk = slice(s0, s0 + n), slice(k0, s0 + n)
        qs, ks, vs, dos = np64(q[:, rq]), np64(k[:, rk]), np64(v[:, rk]), np64(do[:, rq])
        O_ref, L_ref = oracle.attention_forward(qs, ks, vs, md, D ** -0.5)
        compare_out(o[:, rq], O_ref)
        el, same = compare_lse(lse[..., rq], L_ref)
        assert el <= LSE_TOL and same
        gq, gk, gv = oracle.attention_backward(qs, ks, vs, dos, md, D ** -0.5)
        check("dQ", dq[:, rq], gq)
        # keys [s0, s0 + n - halo), or to the end of the sequence for the last slice
        end = s0 + n if s0 + n == S else s0 + n - halo
        kk = slice(s0 - k0, end - k0)
        check("dK", dk[:, s0:end], gk[:, kk])
        check("dV", dv[:, s0:end], gv[:, kk])
