"""GPU parity: the block-map planner and the forward kernel against the oracle."""

import numpy as np
import pytest
import torch

import block_sparse_attention_map_b200 as bsa
import oracle
from block_sparse_attention_map_b200.workloads import make_workload
from tests.gpu_common import LSE_TOL, O_TOL, compare_lse, compare_out, mask_desc, np64, sample_rows

pytestmark = pytest.mark.gpu

SMALL = ["tiny", "packed", "packed_const", "window", "window_rect", "varlen", "video", "prefix_lm",
         "dilated", "document", "gqa"]


@pytest.mark.parametrize("name", SMALL)
def test_plan_tile_classes_match_oracle(name):
    wl = make_workload(name, device="cuda", small=True)
    ws = bsa.plan_build(wl.q, wl.k, wl.v, wl.mask)
    cls = ws.tile_classes().cpu().numpy()
    ref = oracle.tile_classes(mask_desc(wl), wl.B, wl.Sq, wl.Skv)
    assert np.array_equal(cls, ref)
    assert ws.status() == 0


@pytest.mark.parametrize("name,B,Sq,Skv", [("window", 1, 8192, 8192), ("window_rect", 1, 4096, 8192),
                                            ("prefix_lm", 1, 8192, 8192), ("dilated", 1, 8192, 8192),
                                            ("document", 1, 8192, 8192)])
def test_plan_full_size_window_counts(name, B, Sq, Skv):
    wl = make_workload(name, device="cuda")
    ws = bsa.plan_build(wl.q, wl.k, wl.v, wl.mask)
    cls = ws.tile_classes().cpu().numpy()
    ref = oracle.tile_classes(mask_desc(wl), B, Sq, Skv)
    assert np.array_equal(cls, ref)


@pytest.mark.parametrize("order", ["asc", "desc", "perm", "outside_in", "greedy"])
@pytest.mark.parametrize("name", ["window", "packed", "window_rect", "varlen", "prefix_lm", "dilated",
                                  "document"])
def test_plan_ranks_and_column_lists(name, order):
    wl = make_workload(name, device="cuda", small=True)
    nN = -(-wl.Skv // 128)
    perm = np.random.default_rng(5).permutation(nN) if order == "perm" else None
    ws = bsa.plan_build(wl.q, wl.k, wl.v, wl.mask, order=order, perm=perm)
    cls = oracle.tile_classes(mask_desc(wl), wl.B, wl.Sq, wl.Skv)
    pi = oracle.column_order(nN, order, perm, cls=cls)
    assert np.array_equal(ws.perm().cpu().numpy(), pi)
    rank = oracle.kv_ranks(cls, pi)
    assert np.array_equal(ws.ranks().cpu().numpy(), rank)
    lists = oracle.column_lists(cls, rank)
    ptr, ent, rk = ws.col_lists()
    for b in range(wl.B):
        for n in range(nN):
            s, e = ptr[b * nN + n], ptr[b * nN + n + 1]
            got = [(int(x & (bsa._binding.FULL_BIT - 1)), int(r), bool(x & bsa._binding.FULL_BIT))
                   for x, r in zip(ent[s:e], rk[s:e])]
            assert got == lists[(b, n)]
    rptr, rent = ws.row_lists()
    for b in range(wl.B):
        for m in range(cls.shape[1]):
            s, e = rptr[b * cls.shape[1] + m], rptr[b * cls.shape[1] + m + 1]
            got = [(int(x & (bsa._binding.FULL_BIT - 1)), bool(x & bsa._binding.FULL_BIT)) for x in rent[s:e]]
            exp = [(n, cls[b, m, n] == oracle.FULL) for n in range(nN) if cls[b, m, n] != oracle.EMPTY]
            assert got == exp


@pytest.mark.parametrize("name", ["window", "video"])
def test_plan_greedy_order_full_size(name):
    # the greedy kernel over every column of the full-size block maps
    wl = make_workload(name, device="cuda")
    ws = bsa.plan_build(wl.q, wl.k, wl.v, wl.mask, order="greedy")
    cls = ws.tile_classes().cpu().numpy()
    if name == "window":
        assert np.array_equal(cls, oracle.tile_classes(mask_desc(wl), wl.B, wl.Sq, wl.Skv))
    assert np.array_equal(ws.perm().cpu().numpy(), oracle.greedy_order(cls))
    assert ws.status() == 0


def _fwd_vs_oracle(wl, mode="online", rows=None, **kw):
    o, lse, ws = bsa.attn_fwd(wl.q, wl.k, wl.v, wl.mask, softmax_mode=mode, **kw)
    torch.cuda.synchronize()
    assert ws.status() == 0
    q, k, v = np64(wl.q), np64(wl.k), np64(wl.v)
    O_ref, L_ref = oracle.attention_forward(q, k, v, mask_desc(wl), wl.scale, rows=rows)
    eo = compare_out(o, O_ref, rows)
    el, same = compare_lse(lse, L_ref, rows)
    return eo, el, same, o, lse, ws


@pytest.mark.parametrize("name", SMALL)
def test_fwd_online_matches_oracle(name):
    wl = make_workload(name, device="cuda", small=True)
    eo, el, same, *_ = _fwd_vs_oracle(wl)
    assert el <= LSE_TOL and same, (eo, el, same)


@pytest.mark.parametrize("name", ["video", "tiny", "window", "varlen"])
def test_fwd_fixed_m_matches_oracle(name):
    wl = make_workload(name, device="cuda", small=True)
    eo, el, same, o, lse, ws = _fwd_vs_oracle(wl, "fixed_m")
    assert el <= LSE_TOL and same, (eo, el, same)


def test_fixed_m_bound_and_gate_match_oracle():
    wl = make_workload("video", device="cuda", small=True)
    _, _, ws = bsa.attn_fwd(wl.q, wl.k, wl.v, wl.mask, softmax_mode="fixed_m")
    torch.cuda.synchronize()
    kmax, qmax, bound, gate = oracle.fixed_m_bound(np64(wl.q), np64(wl.k), mask_desc(wl), wl.scale)
    assert np.allclose(ws.kmax().cpu().numpy(), kmax, rtol=1e-5)
    assert np.allclose(ws.qmax().cpu().numpy(), qmax, rtol=1e-5)
    g = ws.gate().cpu().numpy().astype(bool)
    # the gate decision is taken in fp32 on the device: equal unless the bound
    # sits within 1e-4 of the limit
    close = np.abs(2 * bound - 64.0) < 1e-4 * 64
    assert np.array_equal(g[~close], gate[~close])
    assert not g[0, 0] and g[0, 1:].all()  # the sink head falls back


def _with_key_offset(wl, norm=40.0):
    """The same workload with a common offset of the given norm added to every
    key (along the first head dim): the case k-smoothing is for."""
    k = wl.k.float()
    k[..., 0] += norm
    wl.k = k.to(torch.bfloat16)
    return wl


@pytest.mark.parametrize("name", ["window", "video", "packed", "varlen"])
def test_smoothed_bound_matches_oracle(name):
    wl = make_workload(name, device="cuda", small=True)
    if name == "window":
        wl = _with_key_offset(wl)
    eo, el, same, o, lse, ws = _fwd_vs_oracle(wl, "fixed_m", bound_mode="smoothed")
    assert el <= LSE_TOL and same, (eo, el, same)
    kbar, radius, qmax, bound, gate = oracle.fixed_m_bound_smoothed(np64(wl.q), np64(wl.k), mask_desc(wl),
                                                                    wl.scale)
    # the center is summed in 2^-20 fixed point, then divided in fp64 and rounded to fp32
    assert np.abs(ws.kbar().cpu().numpy() - kbar).max() <= 1e-5 * max(1.0, np.abs(kbar).max())
    assert np.allclose(ws.kmax().cpu().numpy(), radius, rtol=1e-4, atol=1e-4)
    assert np.allclose(ws.qmax().cpu().numpy(), qmax, rtol=1e-5)
    g = ws.gate().cpu().numpy().astype(bool)
    close = np.abs(2 * bound - 64.0) < 1e-3 * 64
    assert np.array_equal(g[~close], gate[~close])


def test_smoothing_widens_the_gate_and_stays_exact_and_deterministic():
    wl = _with_key_offset(make_workload("window", device="cuda", small=True))
    _, _, ws_plain = bsa.attn_fwd(wl.q, wl.k, wl.v, wl.mask, softmax_mode="fixed_m")
    o, lse, ws = bsa.attn_fwd(wl.q, wl.k, wl.v, wl.mask, softmax_mode="fixed_m", bound_mode="smoothed")
    torch.cuda.synchronize()
    plain = oracle.fixed_m_bound(np64(wl.q), np64(wl.k), mask_desc(wl), wl.scale)[3]
    assert not plain.any() and not ws_plain.gate().cpu().numpy().any()  # the offset breaks the plain gate
    assert ws.gate().cpu().numpy().all()                               # the centred keys pass it
    for _ in range(3):
        o2, l2, _ = bsa.attn_fwd(wl.q, wl.k, wl.v, wl.mask, softmax_mode="fixed_m", bound_mode="smoothed")
        assert torch.equal(o, o2) and torch.equal(lse, l2)
    o3, l3, _ = bsa.attn_fwd(wl.q, wl.k, wl.v, wl.mask, softmax_mode="online")
    torch.cuda.synchronize()
    assert (o - o3).abs().max().item() <= O_TOL
    fin = torch.isfinite(l3)
    assert (lse[fin] - l3[fin]).abs().max().item() <= LSE_TOL


@pytest.mark.parametrize("mode", ["online", "fixed_m"])
def test_gqa_forward_equals_mha_with_repeated_kv_bitwise(mode):
    wl = make_workload("gqa", device="cuda", small=True)
    g = wl.H // wl.k.shape[2]
    o1, l1, _ = bsa.attn_fwd(wl.q, wl.k, wl.v, wl.mask, softmax_mode=mode)
    kr = wl.k.repeat_interleave(g, dim=2).contiguous()
    vr = wl.v.repeat_interleave(g, dim=2).contiguous()
    o2, l2, _ = bsa.attn_fwd(wl.q, kr, vr, wl.mask, softmax_mode=mode)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_gqa_full_size_sampled_rows():
    wl = make_workload("gqa", device="cuda")
    g = wl.H // wl.k.shape[2]
    rows = sample_rows(wl.Sq, seed=3)
    heads = [0, wl.H - 1]
    o, lse, ws = bsa.attn_fwd(wl.q, wl.k, wl.v, wl.mask, softmax_mode="fixed_m")
    torch.cuda.synchronize()
    assert ws.status() == 0
    kvh = [h // g for h in heads]
    q, k, v = np64(wl.q[:, :, heads]), np64(wl.k[:, :, kvh]), np64(wl.v[:, :, kvh])
    O_ref, L_ref = oracle.attention_forward(q, k, v, mask_desc(wl), wl.scale, rows=rows)
    compare_out(o[:, :, heads], O_ref, rows)
    el, same = compare_lse(lse[:, heads], L_ref, rows)
    assert el <= LSE_TOL and same


def test_fixed_m_and_online_agree_bitwise_on_fallback_head():
    wl = make_workload("video", device="cuda", small=True)
    o1, l1, _ = bsa.attn_fwd(wl.q, wl.k, wl.v, wl.mask, softmax_mode="online")
    o2, l2, ws = bsa.attn_fwd(wl.q, wl.k, wl.v, wl.mask, softmax_mode="fixed_m")
    torch.cuda.synchronize()
    # head 0 fails the gate and runs the online body: identical bits
    assert torch.equal(o1[:, :, 0], o2[:, :, 0]) and torch.equal(l1[:, 0], l2[:, 0])
    assert (o1 - o2).abs().max().item() <= O_TOL


def test_constant_segment_ids_bitwise_equal_no_mask():
    wl = make_workload("packed_const", device="cuda", small=True)
    o1, l1, _ = bsa.attn_fwd(wl.q, wl.k, wl.v, wl.mask)
    o2, l2, _ = bsa.attn_fwd(wl.q, wl.k, wl.v, None)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_alignment_rows_zero_and_isolated():
    wl = make_workload("varlen", device="cuda", small=True)
    T_real = wl.mask["cu_seqlens"][-1 - wl.mask["n_align_tail"]]
    o1, l1, _ = bsa.attn_fwd(wl.q, wl.k, wl.v, wl.mask)
    q2, k2, v2 = wl.q.clone(), wl.k.clone(), wl.v.clone()
    for t in (q2, k2, v2):
        t[:, T_real:] = (torch.randn_like(t[:, T_real:].float()) * 30).to(t.dtype)
    o2, l2, _ = bsa.attn_fwd(q2, k2, v2, wl.mask)
    torch.cuda.synchronize()
    assert torch.equal(o1[:, :T_real], o2[:, :T_real]) and torch.equal(l1[..., :T_real], l2[..., :T_real])
    assert (o1[:, T_real:] == 0).all() and torch.isneginf(l1[..., T_real:]).all()


def test_padding_contents_do_not_matter():
    wl = make_workload("video", device="cuda", small=True)
    L = int(wl.mask["kv_valid_len"][0])
    o1, l1, _ = bsa.attn_fwd(wl.q, wl.k, wl.v, wl.mask)
    k2, v2 = wl.k.clone(), wl.v.clone()
    k2[:, L:] = 0
    v2[:, L:] = 1000
    o2, l2, _ = bsa.attn_fwd(wl.q, k2, v2, wl.mask)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_fwd_deterministic_run_to_run():
    wl = make_workload("packed", device="cuda", small=True)
    o1, l1, _ = bsa.attn_fwd(wl.q, wl.k, wl.v, wl.mask)
    for _ in range(3):
        o2, l2, _ = bsa.attn_fwd(wl.q, wl.k, wl.v, wl.mask)
        assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_ragged_shapes_and_d64():
    g = torch.Generator(device="cuda")
    g.manual_seed(11)
    for (Sq, Skv, D, W) in [(1, 1, 64, None), (77, 300, 64, 0), (300, 77, 128, 40), (129, 129, 128, None)]:
        q = torch.randn(2, Sq, 3, D, device="cuda", generator=g).bfloat16()
        k = torch.randn(2, Skv, 3, D, device="cuda", generator=g).bfloat16()
        v = torch.randn(2, Skv, 3, D, device="cuda", generator=g).bfloat16()
        mask = {"window": W} if W is not None else {}
        o, lse, ws = bsa.attn_fwd(q, k, v, mask)
        torch.cuda.synchronize()
        assert ws.status() == 0
        O_ref, L_ref = oracle.attention_forward(np64(q), np64(k), np64(v), oracle.MaskDesc(**mask), 1 / D ** 0.5)
        compare_out(o, O_ref)
        el, same = compare_lse(lse, L_ref)
        assert el <= LSE_TOL and same


def test_strided_inputs():
    g = torch.Generator(device="cuda")
    g.manual_seed(12)
    base = torch.randn(1, 300, 4, 3 * 128, device="cuda", generator=g).bfloat16()
    q, k, v = base[..., :128], base[..., 128:256], base[..., 256:]
    out = torch.empty(1, 300, 4, 256, device="cuda", dtype=torch.bfloat16)[..., 64:192]
    o, lse, _ = bsa.attn_fwd(q, k, v, {"window": 100}, out=out)
    torch.cuda.synchronize()
    O_ref, L_ref = oracle.attention_forward(np64(q), np64(k), np64(v), oracle.MaskDesc(window=100), 128 ** -0.5)
    compare_out(o, O_ref)


@pytest.mark.parametrize("name,extra", [("window", ()), ("window_rect", ()), ("varlen", (33002,)),
                                        ("packed", ()), ("prefix_lm", (2047, 2048)), ("dilated", ()),
                                        ("document", ())])
def test_fwd_full_size_sampled_rows(name, extra):
    wl = make_workload(name, device="cuda")
    rows = sample_rows(wl.Sq, seed=1, extra=extra)
    heads = [0, wl.H - 1]
    o, lse, ws = bsa.attn_fwd(wl.q, wl.k, wl.v, wl.mask)
    torch.cuda.synchronize()
    assert ws.status() == 0
    q, k, v = np64(wl.q[:, :, heads]), np64(wl.k[:, :, heads]), np64(wl.v[:, :, heads])
    O_ref, L_ref = oracle.attention_forward(q, k, v, mask_desc(wl), wl.scale, rows=rows)
    compare_out(o[:, :, heads], O_ref, rows)
    el, same = compare_lse(lse[:, heads], L_ref, rows)
    assert el <= LSE_TOL and same


@pytest.mark.parametrize("mode", ["online", "fixed_m"])
def test_fwd_video_full_size_sampled_rows(mode):
    wl = make_workload("video", device="cuda")
    rows = sample_rows(wl.Sq, seed=2, extra=(75600,))[::3]
    heads = [0, 1, 39]
    o, lse, ws = bsa.attn_fwd(wl.q, wl.k, wl.v, wl.mask, softmax_mode=mode)
    torch.cuda.synchronize()
    assert ws.status() == 0
    if mode == "fixed_m":
        g = ws.gate().cpu().numpy()
        assert g[0, 0] == 0 and g[0, 1:].all()
    q, k, v = np64(wl.q[:, :, heads]), np64(wl.k[:, :, heads]), np64(wl.v[:, :, heads])
    O_ref, L_ref = oracle.attention_forward(q, k, v, mask_desc(wl), wl.scale, rows=rows)
    compare_out(o[:, :, heads], O_ref, rows)
    el, same = compare_lse(lse[:, heads], L_ref, rows)
    assert el <= LSE_TOL and same


@pytest.mark.parametrize("name", ["window", "varlen", "document"])
def test_plan_beside_bound_equals_plan_then_bound(name):
    # bsa_plan_and_bound runs the planner on the library's side stream next to
    # the bound (sequentially for varlen masks): the forward that follows must
    # see exactly the state plan-then-bound leaves, on the caller's stream with
    # no synchronisation in between
    wl = make_workload(name, device="cuda", small=True)
    outs = []
    for together in (False, True):
        st = bsa.Stages(wl.q, wl.k, wl.v, wl.mask, softmax_mode="fixed_m", order="desc")
        for _ in range(3):  # repeated: each call forks and joins again
            if together:
                st.plan_and_bound()
            else:
                st.plan()
                st.bound()
            st.forward()
        torch.cuda.synchronize()
        assert st.ws.status() == 0
        outs.append((st.out.clone(), st.lse.clone()))
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])
    rows = sample_rows(wl.Sq, seed=4)
    f = lambda t: t.float().cpu().numpy().astype(np.float64)
    O_ref, L_ref = oracle.attention_forward(f(wl.q), f(wl.k), f(wl.v), mask_desc(wl), wl.scale, rows=rows)
    compare_out(outs[1][0], O_ref, rows)


def _gate_edge_inputs():
    """Every query along one direction u and every key along -u: s_ij =
    -scale a_i c_j, so the pinned m_i = scale a_i kmax sits scale a_i (kmax +
    c_j) above each score.  With query norms up to 16 and key norms in
    [15, 15.8] at D = 64, 2 B_h = 63.2, just under the gate limit 64, and the
    worst row's reference is 61.6 nats above its true maximum."""
    B, H, S, D, W = 1, 2, 1000, 64, 256
    rng = np.random.default_rng(31)
    u = rng.standard_normal(D)
    u /= np.linalg.norm(u)
    a = rng.uniform(2.0, 16.0, size=(B, S, H))
    a[0, 700] = 16.0
    c = rng.uniform(15.0, 15.8, size=(B, S, H))
    q = torch.from_numpy(a[..., None] * u).to(torch.bfloat16).cuda()
    k = torch.from_numpy(-c[..., None] * u).to(torch.bfloat16).cuda()
    v = torch.from_numpy(rng.standard_normal((B, S, H, D))).to(torch.bfloat16).cuda()
    return q, k, v, {"window": W}, D ** -0.5


def test_fixed_m_at_the_gate_edge_stays_exact():
    """A head whose pinned reference sits as far above the true row maximum as
    the gate allows still passes the gate, runs fixed-m without a gate warning,
    and matches the oracle and the online forward."""
    q, k, v, mask, scale = _gate_edge_inputs()
    md = oracle.MaskDesc(window=mask["window"])
    _, _, bound, gate = oracle.fixed_m_bound(np64(q), np64(k), md, scale)
    assert gate.all() and (2 * bound > 63.0).all()
    o, lse, ws = bsa.attn_fwd(q, k, v, mask, softmax_mode="fixed_m")
    o_on, lse_on, _ = bsa.attn_fwd(q, k, v, mask)
    torch.cuda.synchronize()
    assert ws.status() == 0  # no row summed below 2^-100
    assert ws.gate().cpu().numpy().all()
    O_ref, L_ref = oracle.attention_forward(np64(q), np64(k), np64(v), md, scale)
    compare_out(o, O_ref)
    el, same = compare_lse(lse, L_ref)
    assert el <= LSE_TOL and same
    assert float((o.float() - o_on.float()).abs().max()) <= O_TOL
    assert float((lse - lse_on).abs().max()) <= LSE_TOL


def _gate_rows_count(wl, kmax, G=64.0):
    """(rows the oracle's per-row gate pins, rows within 1e-3 of the limit) over
    the q-blocks the forward visits (those with a non-empty tile)."""
    cls = oracle.tile_classes(mask_desc(wl), wl.B, wl.Sq, wl.Skv)
    vis = (cls != oracle.EMPTY).any(axis=2)  # [B, nM]
    ref2 = 2.0 * oracle.row_references_blocks(np64(wl.q), kmax, wl.scale)  # [B, H, Sq]
    blk = np.arange(wl.Sq) // 128
    live = vis[:, None, blk]  # [B, 1, Sq]
    live = np.broadcast_to(live, ref2.shape)
    sure = live & (ref2 <= G * (1 - 1e-3))
    near = live & (np.abs(ref2 - G) < G * 1e-3)
    return int(sure.sum()), int(near.sum())


@pytest.mark.parametrize("name", ["window", "packed", "document", "varlen", "video", "dilated", "gqa"])
def test_block_bound_matches_oracle(name):
    """The per q-block bound (BSA_BOUND_BLOCK): each q-block's kmax equals the
    oracle's (the largest valid key norm over the kv blocks its row list
    reaches), the rows the device ran fixed-m are the rows the oracle's per-row
    gate passes, and O / LSE match the oracle."""
    wl = make_workload(name, device="cuda", small=True)
    eo, el, same, o, lse, ws = _fwd_vs_oracle(wl, "fixed_m", bound_mode="block")
    assert el <= LSE_TOL and same, (eo, el, same)
    kmax, qmax, bound, gate = oracle.fixed_m_bound_blocks(np64(wl.q), np64(wl.k), mask_desc(wl), wl.scale)
    cls = oracle.tile_classes(mask_desc(wl), wl.B, wl.Sq, wl.Skv)
    vis = np.broadcast_to((cls != oracle.EMPTY).any(axis=2)[:, None, :], kmax.shape)
    got = ws.kmax_q().cpu().numpy()
    assert np.allclose(got[vis], kmax[vis], rtol=1e-5, atol=0)
    sure, near = _gate_rows_count(wl, kmax)
    assert sure <= ws.fixed_rows() <= sure + near


def test_block_bound_gates_rows_the_head_gate_sends_online():
    """Packed segments with one hot segment (batch 0, its last segment, keys
    x20): the per-head gate sends both heads of batch 0 to online softmax, the
    per q-block bound pins every row of batch 0 whose q-block does not reach
    the hot keys; the results match the oracle either way."""
    wl = make_workload("packed", device="cuda", small=True)
    seg0 = wl.mask["seg_kv"][0].cpu().numpy()
    hot_np = seg0 == seg0[-1]
    assert np.argmax(hot_np) >= 256  # the first two q-blocks see only cold keys
    hot = torch.from_numpy(hot_np).to(wl.k.device)
    k = wl.k.float()
    k[0, hot] *= 20.0
    wl.k = k.to(torch.bfloat16)
    _, _, _, _, _, ws_head = _fwd_vs_oracle(wl, "fixed_m")
    g = ws_head.gate().cpu().numpy()
    assert not g[0].any() and g[1].all()
    assert ws_head.fixed_rows() == wl.H * wl.Sq  # batch 1 only
    _, _, _, _, _, ws_blk = _fwd_vs_oracle(wl, "fixed_m", bound_mode="block")
    kmax = oracle.fixed_m_bound_blocks(np64(wl.q), np64(wl.k), mask_desc(wl), wl.scale)[0]
    sure, near = _gate_rows_count(wl, kmax)
    assert sure <= ws_blk.fixed_rows() <= sure + near
    assert ws_blk.fixed_rows() > wl.H * wl.Sq + wl.H * 128  # pinned rows in batch 0 too
