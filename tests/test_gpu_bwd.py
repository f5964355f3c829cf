"""GPU parity of the backward (Delta, deterministic semaphore-ordered dQ, dK/dV)
against the oracle's analytic gradient on the flat bar (max-abs 1e-2), with the
library's defaults unless a test says otherwise; run-to-run bit identity, the
non-deterministic variant, the configuration the bench times, and the bounded
semaphore wait."""

import numpy as np
import pytest
import torch

import block_sparse_attention_map_b200 as bsa
import oracle
from block_sparse_attention_map_b200.workloads import make_workload
from tests.gpu_common import check, compare_lse, compare_out, LSE_TOL, mask_desc, np64, sample_rows

pytestmark = pytest.mark.gpu


def _grads(wl, fwd_kw=None, **kw):
    """Forward then backward on the forward's workspace, library defaults
    otherwise (the O residual is kept and used: Delta exact to the fp32 O)."""
    o, lse, ws = bsa.attn_fwd(wl.q, wl.k, wl.v, wl.mask, **(fwd_kw or {}))
    dq, dk, dv, wsb = bsa.attn_bwd(wl.q, wl.k, wl.v, o, wl.dO, lse, wl.mask, workspace=ws, **kw)
    torch.cuda.synchronize()
    return o, lse, dq, dk, dv, wsb


def _oracle_grads(wl, heads=None, batches=None):
    """Oracle gradients; ``heads`` (query heads) must cover whole kv-head groups."""
    q, k, v, do = np64(wl.q), np64(wl.k), np64(wl.v), np64(wl.dO)
    if heads is not None:
        g = wl.H // wl.k.shape[2]
        kvh = sorted({h // g for h in heads})
        q, do = q[:, :, heads], do[:, :, heads]
        k, v = k[:, :, kvh], v[:, :, kvh]
    return oracle.attention_backward(q, k, v, do, mask_desc(wl), wl.scale, batches=batches)


def _check_grads(dq, dk, dv, ref, q_idx=(slice(None),), kv_idx=(slice(None),)):
    gq, gk, gv = ref
    return (check("dQ", np64(dq)[q_idx], gq[q_idx]), check("dK", np64(dk)[kv_idx], gk[kv_idx]),
            check("dV", np64(dv)[kv_idx], gv[kv_idx]))


SMALL = ["tiny", "packed", "window", "window_rect", "varlen", "video", "prefix_lm", "dilated", "document",
         "gqa"]


def _with_dO(wl):
    if wl.dO is None:
        g = torch.Generator(device="cuda")
        g.manual_seed(99)
        wl.dO = torch.randn(wl.q.shape, device="cuda", generator=g).bfloat16()
    return wl


@pytest.mark.parametrize("name", SMALL)
def test_bwd_matches_oracle(name):
    wl = _with_dO(make_workload(name, device="cuda", small=True))
    _, _, dq, dk, dv, ws = _grads(wl)
    assert ws.status() == 0
    ref = _oracle_grads(wl)
    if name == "video":
        # Head 0 of the video shape carries the 8 "sink" keys scaled x20: its
        # scores reach ~110 nats and every row puts weight ~1/8 on each sink
        # key, so dV of a sink key sums ~|rows| / 8 bf16-rounded weights and dQ
        # multiplies dS by |k| ~ 40.  The video workload is forward-only; its
        # forward parity covers the sink head, the backward the normal heads.
        _check_grads(dq, dk, dv, ref, (slice(None), slice(None), slice(1, None)),
                     (slice(None), slice(None), slice(1, None)))
    else:
        _check_grads(dq, dk, dv, ref)


@pytest.mark.parametrize("name", ["window", "packed", "gqa"])
def test_bwd_without_o_residual_matches_oracle(name):
    """The opt-out o_residual="drop" (Delta from the bf16 O): on the flat bar
    where rows see many keys; on masks whose rows can see only a handful of
    keys (document starts, dilated bands near the start) the output's rounding
    in Delta can move dQ / dK past it, which is why it is not the default."""
    wl = make_workload(name, device="cuda", small=True)
    _, _, dq, dk, dv, ws = _grads(wl, fwd_kw={"o_residual": "drop"}, o_residual="drop")
    assert ws.status() == 0
    _check_grads(dq, dk, dv, _oracle_grads(wl))


@pytest.mark.parametrize("order", ["asc", "desc", "perm", "outside_in", "greedy"])
def test_bwd_orders_match_oracle_and_repeat_bitwise(order):
    wl = make_workload("window", device="cuda", small=True)
    nN = -(-wl.Skv // 128)
    perm = np.random.default_rng(3).permutation(nN) if order == "perm" else None
    o, lse, dq, dk, dv, ws = _grads(wl, order=order, perm=perm)
    assert ws.status() == 0
    _check_grads(dq, dk, dv, _oracle_grads(wl))
    for _ in range(9):
        dq2, dk2, dv2, ws2 = bsa.attn_bwd(wl.q, wl.k, wl.v, o, wl.dO, lse, wl.mask, order=order, perm=perm,
                                          workspace=ws)
        torch.cuda.synchronize()
        assert ws2.status() == 0
        assert torch.equal(dq, dq2) and torch.equal(dk, dk2) and torch.equal(dv, dv2)


def test_gqa_bwd_dq_equals_mha_with_repeated_kv_and_dkv_sum_the_group():
    # dQ: the same per-head contributions added in the same order pi -> equal
    # bits.  dK/dV of a kv head: the group's sum, accumulated in fp32 before
    # one rounding, against the bf16 sum of the per-head MHA gradients.
    wl = make_workload("gqa", device="cuda", small=True)
    g = wl.H // wl.k.shape[2]
    o, lse, dq, dk, dv, ws = _grads(wl)
    assert ws.status() == 0
    kr = wl.k.repeat_interleave(g, dim=2).contiguous()
    vr = wl.v.repeat_interleave(g, dim=2).contiguous()
    dq2, dk2, dv2, ws2 = bsa.attn_bwd(wl.q, kr, vr, o, wl.dO, lse, wl.mask, workspace=ws)
    torch.cuda.synchronize()
    assert ws2.status() == 0
    assert torch.equal(dq, dq2)
    B, S, Hk, D = wl.k.shape
    sk = dk2.float().view(B, S, Hk, g, D).sum(3)
    sv = dv2.float().view(B, S, Hk, g, D).sum(3)
    # the bf16 roundings of g per-head gradients against one rounding of their sum
    assert (dk.float() - sk).abs().max().item() <= g * 1e-2
    assert (dv.float() - sv).abs().max().item() <= g * 1e-2
    _check_grads(dq, dk, dv, _oracle_grads(wl))


def test_bwd_nondeterministic_matches_oracle():
    wl = make_workload("packed", device="cuda", small=True)
    _, _, dq, dk, dv, ws = _grads(wl, deterministic=False)
    assert ws.status() == 0
    _check_grads(dq, dk, dv, _oracle_grads(wl))


@pytest.mark.parametrize("small", [True, False])
def test_bwd_constant_segment_ids_bitwise_equal_no_mask(small):
    """Constant segment ids are the same mask as no ids ("Let splash attention
    exceed 524,288 tokens ...", summary): the backward gives the same bits, at
    the small shape and at the packed workload's full size (B=2, H=8, S=4096)."""
    wl = make_workload("packed_const", device="cuda", small=small)
    o, lse, ws = bsa.attn_fwd(wl.q, wl.k, wl.v, wl.mask)
    a = bsa.attn_bwd(wl.q, wl.k, wl.v, o, wl.dO, lse, wl.mask, workspace=ws)
    o2, lse2, ws2 = bsa.attn_fwd(wl.q, wl.k, wl.v, None)
    b = bsa.attn_bwd(wl.q, wl.k, wl.v, o2, wl.dO, lse2, None, workspace=ws2)
    torch.cuda.synchronize()
    assert a[3].status() == 0 and b[3].status() == 0
    assert torch.equal(o, o2) and torch.equal(lse, lse2)
    for x, y in zip(a[:3], b[:3]):
        assert torch.equal(x, y)


def test_bwd_ragged_and_d64():
    g = torch.Generator(device="cuda")
    g.manual_seed(21)
    for (Sq, Skv, D, W) in [(77, 300, 64, 0), (300, 77, 128, 40), (129, 257, 128, None), (1, 1, 64, None)]:
        q = torch.randn(2, Sq, 3, D, device="cuda", generator=g).bfloat16()
        k = torch.randn(2, Skv, 3, D, device="cuda", generator=g).bfloat16()
        v = torch.randn(2, Skv, 3, D, device="cuda", generator=g).bfloat16()
        do = torch.randn(2, Sq, 3, D, device="cuda", generator=g).bfloat16()
        mask = {"window": W} if W is not None else {}
        o, lse, wsf = bsa.attn_fwd(q, k, v, mask)
        dq, dk, dv, ws = bsa.attn_bwd(q, k, v, o, do, lse, mask, workspace=wsf)
        torch.cuda.synchronize()
        assert ws.status() == 0
        ref = oracle.attention_backward(np64(q), np64(k), np64(v), np64(do), oracle.MaskDesc(**mask), 1 / D ** 0.5)
        _check_grads(dq, dk, dv, ref)


# Every family at full size, in the kv-column order that is fastest for it
# (the window in both): library defaults otherwise, ten runs bit-identical,
# each run's status checked, one kv head's gradients against the oracle.
@pytest.mark.parametrize("name,order", [
    ("window", "desc"), ("window", "asc"), ("window_rect", "desc"), ("prefix_lm", "asc"),
    ("dilated", "desc"), ("document", "desc"), ("gqa", "desc"), ("packed", "desc")])
def test_bwd_full_size_one_head_and_ten_run_identity(name, order):
    wl = make_workload(name, device="cuda")
    o, lse, ws = bsa.attn_fwd(wl.q, wl.k, wl.v, wl.mask)
    ref = None
    for it in range(10):
        dq, dk, dv, wsb = bsa.attn_bwd(wl.q, wl.k, wl.v, o, wl.dO, lse, wl.mask, order=order, workspace=ws)
        torch.cuda.synchronize()
        assert wsb.status() == 0, it
        if ref is None:
            ref = (dq.clone(), dk.clone(), dv.clone())
        else:
            assert all(torch.equal(x, y) for x, y in zip(ref, (dq, dk, dv))), it
    g = wl.H // wl.k.shape[2]
    gq, gk, gv = _oracle_grads(wl, heads=list(range(g)))  # kv head 0 and its query heads, every batch
    check("dQ", np64(ref[0][:, :, :g]), gq)
    check("dK", np64(ref[1][:, :, [0]]), gk)
    check("dV", np64(ref[2][:, :, [0]]), gv)


def test_bench_step_full_size_matches_oracle_and_repeats_bitwise():
    """The step bench.py times, on its workload (causal window 512, B=1, H=16,
    8192 x 8192, D=128): plan and bound in one call, fixed-m gated forward,
    Delta, the deterministic backward in the descending kv-column order and the
    dQ convert, through the per-stage C-ABI calls on one workspace.  O and LSE
    of heads 0 and 15 on sampled rows and the gradients of heads 0 and 15
    against the oracle; ten steps bit-identical."""
    wl = make_workload("window", device="cuda")
    st = bsa.Stages(wl.q, wl.k, wl.v, wl.mask, softmax_mode="fixed_m", order="desc")
    outs = None
    for it in range(10):
        st.plan_and_bound()
        st.forward()
        st.preprocess(wl.dO)
        st.backward_main(wl.dO)
        st.convert()
        torch.cuda.synchronize()
        assert st.ws.status() == 0, it
        cur = tuple(t.clone() for t in (st.out, st.lse, st.dq, st.dk, st.dv))
        if outs is None:
            outs = cur
        else:
            assert all(torch.equal(x, y) for x, y in zip(outs, cur)), it
    assert st.ws.gate().cpu().numpy().all()  # every head of this workload runs fixed-m
    o, lse, dq, dk, dv = outs
    rows = sample_rows(wl.Sq, seed=7)
    heads = [0, wl.H - 1]
    q, k, v = np64(wl.q[:, :, heads]), np64(wl.k[:, :, heads]), np64(wl.v[:, :, heads])
    O_ref, L_ref = oracle.attention_forward(q, k, v, mask_desc(wl), wl.scale, rows=rows)
    compare_out(o[:, :, heads], O_ref, rows)
    el, same = compare_lse(lse[:, heads], L_ref, rows)
    assert el <= LSE_TOL and same
    # the first and the last head: the forward hands units out and the dQ
    # convert takes q-blocks with the heads interleaved
    for h in (0, wl.H - 1):
        gq, gk, gv = _oracle_grads(wl, heads=[h])
        check("dQ", np64(dq[:, :, [h]]), gq)
        check("dK", np64(dk[:, :, [h]]), gk)
        check("dV", np64(dv[:, :, [h]]), gv)


def test_packed_full_size_forward_and_backward_per_batch():
    """The packed-segments workload at full size (B=2, H=8, S=4096, segment runs
    of 256..2048): forward and backward of one head in each batch row against
    the oracle (the gradients over all rows and keys of that head)."""
    wl = make_workload("packed", device="cuda")
    o, lse, dq, dk, dv, ws = _grads(wl)
    assert ws.status() == 0
    for h in (0, wl.H - 1):
        q, k, v = np64(wl.q[:, :, [h]]), np64(wl.k[:, :, [h]]), np64(wl.v[:, :, [h]])
        O_ref, L_ref = oracle.attention_forward(q, k, v, mask_desc(wl), wl.scale)
        compare_out(o[:, :, [h]], O_ref)
        el, same = compare_lse(lse[:, [h]], L_ref)
        assert el <= LSE_TOL and same
        gq, gk, gv = _oracle_grads(wl, heads=[h])
        check("dQ", np64(dq[:, :, [h]]), gq)
        check("dK", np64(dk[:, :, [h]]), gk)
        check("dV", np64(dv[:, :, [h]]), gv)


def test_semaphore_wait_is_bounded_and_reported():
    # Corrupt one rank in the caller-owned plan so that its dQ wait can never be
    # satisfied: the wait gives up after the bound, the status word says so and
    # the context stays usable.
    wl = make_workload("window", device="cuda", small=True)
    o, lse, _ = bsa.attn_fwd(wl.q, wl.k, wl.v, wl.mask)
    ws = bsa.plan_build(wl.q, wl.k, wl.v, wl.mask, backward=True)
    torch.cuda.synchronize()
    off = ws.view.off_col_rank
    ranks = ws.buf[off:off + 4 * 8].view(torch.int32)
    ranks[3] = 1000
    dq, dk, dv, _ = bsa.attn_bwd(wl.q, wl.k, wl.v, o, wl.dO, lse, wl.mask, workspace=ws,
                                 plan_ready=True, sem_timeout_ns=50_000_000)
    torch.cuda.synchronize()
    assert ws.status(clear=True) == 5  # BSA_ERR_SEM_TIMEOUT
    # the device is still healthy: a clean run afterwards succeeds
    _, _, dq2, dk2, dv2, ws2 = _grads(wl)
    assert ws2.status() == 0
    _check_grads(dq2, dk2, dv2, _oracle_grads(wl))


def test_plan_mismatch_is_reported():
    wl = make_workload("window", device="cuda", small=True)
    ws = bsa.plan_build(wl.q, wl.k, wl.v, {"window": 7})
    o, lse, _ = bsa.attn_fwd(wl.q, wl.k, wl.v, wl.mask, workspace=ws, plan_ready=True)
    torch.cuda.synchronize()
    assert ws.status(clear=True) == 6  # BSA_ERR_PLAN_MISMATCH


def test_residual_is_used_only_for_the_output_it_was_kept_for():
    """o_residual="auto": the backward uses the residual only when the
    workspace's record names the same `out` the forward wrote.  With the
    forward's workspace the result equals an explicit "keep"; with another
    output buffer holding the same values it equals "drop" (bf16-O Delta).  A
    plan rebuild keeps the record (the composite backward rebuilds the plan); a
    forward that keeps no residual clears it."""
    wl = make_workload("document", device="cuda", small=True)
    o, lse, ws = bsa.attn_fwd(wl.q, wl.k, wl.v, wl.mask)
    auto = bsa.attn_bwd(wl.q, wl.k, wl.v, o, wl.dO, lse, wl.mask, workspace=ws)
    keep = bsa.attn_bwd(wl.q, wl.k, wl.v, o, wl.dO, lse, wl.mask, workspace=ws, o_residual="keep")
    drop = bsa.attn_bwd(wl.q, wl.k, wl.v, o, wl.dO, lse, wl.mask, workspace=ws, o_residual="drop")
    other = bsa.attn_bwd(wl.q, wl.k, wl.v, o.clone(), wl.dO, lse, wl.mask, workspace=ws)
    torch.cuda.synchronize()
    assert all(torch.equal(x, y) for x, y in zip(auto[:3], keep[:3]))
    assert all(torch.equal(x, y) for x, y in zip(other[:3], drop[:3]))
    assert not all(torch.equal(x, y) for x, y in zip(auto[:3], drop[:3]))
    bsa.plan_build(wl.q, wl.k, wl.v, wl.mask, workspace=ws)
    rebuilt = bsa.attn_bwd(wl.q, wl.k, wl.v, o, wl.dO, lse, wl.mask, workspace=ws)
    bsa.attn_fwd(wl.q, wl.k, wl.v, wl.mask, workspace=ws, out=o, lse=lse, o_residual="drop")
    cleared = bsa.attn_bwd(wl.q, wl.k, wl.v, o, wl.dO, lse, wl.mask, workspace=ws)
    torch.cuda.synchronize()
    assert ws.status() == 0
    assert all(torch.equal(x, y) for x, y in zip(rebuilt[:3], auto[:3]))
    assert all(torch.equal(x, y) for x, y in zip(cleared[:3], drop[:3]))


def test_fp16_q_from_the_forward_equals_the_delta_pass_conversion():
    """With the O residual kept, the forward also writes the fp16 copy of Q the
    backward's products read, and the Delta pass skips Q when the workspace's
    record names this very q.  A backward given a copy of q (another pointer,
    the same values) converts Q itself: the gradients are the same bits."""
    wl = make_workload("window", device="cuda", small=True)
    o, lse, ws = bsa.attn_fwd(wl.q, wl.k, wl.v, wl.mask)
    a = bsa.attn_bwd(wl.q, wl.k, wl.v, o, wl.dO, lse, wl.mask, workspace=ws)
    b = bsa.attn_bwd(wl.q.clone(), wl.k, wl.v, o, wl.dO, lse, wl.mask, workspace=ws)
    torch.cuda.synchronize()
    assert ws.status() == 0
    assert all(torch.equal(x, y) for x, y in zip(a[:3], b[:3]))


@pytest.mark.parametrize("deterministic", [True, False])
def test_stage_calls_equal_the_composite_calls(deterministic):
    """The per-stage C-ABI calls (plan, bound, forward, Delta, backward main,
    dQ convert) give the composite calls' results: bit for bit with the
    deterministic backward, and within the bar of the oracle with the atomic
    one, whose dQ comes out of the convert stage."""
    wl = make_workload("window", device="cuda", small=True)
    st = bsa.Stages(wl.q, wl.k, wl.v, wl.mask, softmax_mode="fixed_m", order="desc",
                    deterministic=deterministic)
    st.plan()
    st.bound()
    st.forward()
    st.preprocess(wl.dO)
    st.backward_main(wl.dO)
    st.convert()
    o, lse, wsf = bsa.attn_fwd(wl.q, wl.k, wl.v, wl.mask, softmax_mode="fixed_m", order="desc")
    dq, dk, dv, ws = bsa.attn_bwd(wl.q, wl.k, wl.v, o, wl.dO, lse, wl.mask, order="desc",
                                  deterministic=deterministic, workspace=wsf)
    torch.cuda.synchronize()
    assert st.ws.status() == 0 and ws.status() == 0
    assert torch.equal(st.out, o) and torch.equal(st.lse, lse)
    if deterministic:
        assert torch.equal(st.dq, dq) and torch.equal(st.dk, dk) and torch.equal(st.dv, dv)
    else:
        _check_grads(st.dq, st.dk, st.dv, _oracle_grads(wl))


def test_dq_convert_polls_then_falls_back_and_repeats_bitwise():
    """After a semaphore-ordered Delta pass the dQ convert polls each quarter's
    semaphore rather than waiting for the backward grid.  With no backward main
    kernel in between the counts never complete: each poll gives up after its
    bound, the call still finishes (no error is recorded: it falls back to the
    grid wait), and a backward run afterwards gives the composite call's dQ.  A
    second convert on complete semaphores gives the same dQ bit for bit."""
    import time
    wl = make_workload("window", device="cuda", small=True)
    st = bsa.Stages(wl.q, wl.k, wl.v, wl.mask, softmax_mode="fixed_m", order="desc")
    st.plan_and_bound()
    st.forward()
    st.preprocess(wl.dO)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    st.convert()
    torch.cuda.synchronize()
    assert time.perf_counter() - t0 < 5.0
    assert st.ws.status() == 0
    st.preprocess(wl.dO)
    st.backward_main(wl.dO)
    st.convert()
    torch.cuda.synchronize()
    first = st.dq.clone()
    st.convert()
    torch.cuda.synchronize()
    assert st.ws.status() == 0
    assert torch.equal(st.dq, first)
    o, lse, wsf = bsa.attn_fwd(wl.q, wl.k, wl.v, wl.mask, softmax_mode="fixed_m", order="desc")
    dq, _, _, ws = bsa.attn_bwd(wl.q, wl.k, wl.v, o, wl.dO, lse, wl.mask, order="desc", workspace=wsf)
    torch.cuda.synchronize()
    assert ws.status() == 0 and torch.equal(st.dq, dq)


def test_unsorted_segment_ids_plan_forward_backward():
    """Segment ids in no order (each position's id drawn from three values, so
    most tiles mix segments and the block bounds settle few of them): the
    planner's prep launch summarises both id arrays, the element check settles
    the rest, and the tile classes equal the oracle's exactly; the forward and
    the backward meet the bar.  B = 2, a ragged 700-token sequence."""
    from block_sparse_attention_map_b200.workloads import Workload
    g = torch.Generator(device="cuda")
    g.manual_seed(11)
    B, H, S, D = 2, 2, 700, 128
    q, k, v, do = (torch.randn(B, S, H, D, generator=g, device="cuda").to(torch.bfloat16) for _ in range(4))
    ids = torch.randint(0, 3, (B, S), generator=g, device="cuda", dtype=torch.int32)
    wl = Workload(name="unsorted_ids", B=B, H=H, Sq=S, Skv=S, D=D, q=q, k=k, v=v, dO=do,
                  mask={"seg_q": ids, "seg_kv": ids.clone()}, scale=D ** -0.5)
    ws = bsa.plan_build(wl.q, wl.k, wl.v, wl.mask, backward=True)
    torch.cuda.synchronize()
    assert ws.status() == 0
    ref_cls = oracle.tile_classes(mask_desc(wl), B, S, S)
    assert np.array_equal(ws.tile_classes().cpu().numpy(), ref_cls)
    o, lse, dq, dk, dv, wsb = _grads(wl)
    assert wsb.status() == 0
    O_ref, L_ref = oracle.attention_forward(np64(q), np64(k), np64(v), mask_desc(wl), wl.scale)
    check("O", np64(o), O_ref)
    el, same = compare_lse(lse, L_ref)
    assert el <= LSE_TOL and same
    _check_grads(dq, dk, dv, _oracle_grads(wl))
