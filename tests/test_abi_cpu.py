"""The C ABI without a GPU: the library loads, exports every function the header
declares, the ctypes structs match the C layout, and argument errors come back
as status codes before anything touches CUDA."""

import ctypes
import os
import subprocess
import tempfile

import pytest

from block_sparse_attention_map_b200 import _binding as bd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    if not os.path.exists(bd.LIB_PATH):
        from block_sparse_attention_map_b200 import build
        build.build()
    return bd.lib()


def test_exports_every_declared_function(L):
    names = bd.header_functions()
    assert {"bsa_attn_fwd", "bsa_attn_bwd", "bsa_plan_build", "bsa_workspace_size",
            "bsa_get_device_status", "bsa_status_string"} <= set(names)
    for n in names:
        assert hasattr(L, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", bd.LIB_PATH], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert set(names) <= exported
    # nothing but the C ABI is exported
    assert {e for e in exported if e.startswith("bsa_")} == set(names)


def _c_layout():
    src = r"""
#include <stdio.h>
#include <stddef.h>
#include "bsa.h"
#define P(T, f) printf(#T "." #f " %zu\n", offsetof(T, f));
int main(void) {
  printf("bsa_problem %zu\nbsa_mask_spec %zu\nbsa_options %zu\nbsa_workspace_view %zu\n",
         sizeof(bsa_problem), sizeof(bsa_mask_spec), sizeof(bsa_options), sizeof(bsa_workspace_view));
  P(bsa_problem, q_stride) P(bsa_problem, o_stride) P(bsa_problem, scale)
  P(bsa_mask_spec, seg_q) P(bsa_mask_spec, cu_seqlens) P(bsa_mask_spec, n_align_tail)
  P(bsa_mask_spec, prefix_len) P(bsa_mask_spec, dilation)
  P(bsa_options, kmax_override) P(bsa_options, perm) P(bsa_options, sem_timeout_ns) P(bsa_options, plan_ready)
  P(bsa_options, bound_mode) P(bsa_options, o_residual) P(bsa_workspace_view, off_qdot)
  P(bsa_workspace_view, off_o_resid) P(bsa_problem, H_kv) P(bsa_workspace_view, off_kmax_q)
  P(bsa_workspace_view, off_sem) P(bsa_workspace_view, nN)
  return 0;
}
"""
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "l.c")
        exe = os.path.join(d, "l")
        open(c, "w").write(src)
        subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), c, "-o", exe], check=True)
        out = subprocess.run([exe], capture_output=True, text=True, check=True).stdout
    return dict((k, int(v)) for k, v in (line.split() for line in out.splitlines()))


def test_ctypes_structs_match_c_layout():
    c = _c_layout()
    assert c["bsa_problem"] == ctypes.sizeof(bd.Problem)
    assert c["bsa_mask_spec"] == ctypes.sizeof(bd.MaskSpec)
    assert c["bsa_options"] == ctypes.sizeof(bd.Options)
    assert c["bsa_workspace_view"] == ctypes.sizeof(bd.WorkspaceView)
    assert c["bsa_problem.q_stride"] == bd.Problem.q_stride.offset
    assert c["bsa_problem.o_stride"] == bd.Problem.o_stride.offset
    assert c["bsa_problem.scale"] == bd.Problem.scale.offset
    assert c["bsa_mask_spec.seg_q"] == bd.MaskSpec.seg_q.offset
    assert c["bsa_mask_spec.cu_seqlens"] == bd.MaskSpec.cu_seqlens.offset
    assert c["bsa_mask_spec.n_align_tail"] == bd.MaskSpec.n_align_tail.offset
    assert c["bsa_mask_spec.prefix_len"] == bd.MaskSpec.prefix_len.offset
    assert c["bsa_mask_spec.dilation"] == bd.MaskSpec.dilation.offset
    assert c["bsa_options.bound_mode"] == bd.Options.bound_mode.offset
    assert c["bsa_workspace_view.off_qdot"] == bd.WorkspaceView.off_qdot.offset
    assert c["bsa_options.o_residual"] == bd.Options.o_residual.offset
    assert c["bsa_workspace_view.off_o_resid"] == bd.WorkspaceView.off_o_resid.offset
    assert c["bsa_workspace_view.off_kmax_q"] == bd.WorkspaceView.off_kmax_q.offset
    assert c["bsa_problem.H_kv"] == bd.Problem.H_kv.offset
    assert c["bsa_options.kmax_override"] == bd.Options.kmax_override.offset
    assert c["bsa_options.perm"] == bd.Options.perm.offset
    assert c["bsa_options.sem_timeout_ns"] == bd.Options.sem_timeout_ns.offset
    assert c["bsa_options.plan_ready"] == bd.Options.plan_ready.offset
    assert c["bsa_workspace_view.off_sem"] == bd.WorkspaceView.off_sem.offset
    assert c["bsa_workspace_view.nN"] == bd.WorkspaceView.nN.offset


def _prob(B=1, H=2, Sq=256, Skv=256, D=64):
    p = bd.Problem()
    p.B, p.H, p.Sq, p.Skv, p.D = B, H, Sq, Skv, D
    return p


def _size(L, p, m=None, bwd=1):
    n = ctypes.c_size_t(0)
    rc = L.bsa_workspace_size(ctypes.byref(p), ctypes.byref(m) if m is not None else None, bwd,
                              ctypes.byref(n))
    return rc, n.value


def test_workspace_size_and_validation(L):
    rc, fwd = _size(L, _prob(), bwd=0)
    assert rc == 0 and fwd > 0
    rc, tot = _size(L, _prob(), bwd=1)
    # the backward adds Delta, the fp32 dQ accumulator [B,H,nM*128,D] and semaphores
    assert rc == 0 and tot >= fwd + 4 * 2 * 256 * 64 + 4 * 2 * 256
    assert _size(L, _prob(D=96))[0] == 2          # unsupported head dim
    assert _size(L, _prob(H=0))[0] == 1           # invalid
    assert _size(L, _prob(Skv=0))[0] == 1         # no key at all: invalid
    assert _size(L, _prob(Sq=1 << 21, Skv=1 << 21))[0] == 0  # the longest sequence accepted
    assert _size(L, _prob(Sq=(1 << 21) + 1))[0] == 2
    assert _size(L, _prob(Skv=(1 << 21) + 1))[0] == 2
    p = _prob()
    p.q_stride[:] = (256 * 2 * 64, 2 * 64 + 4, 64)  # row stride not a multiple of 16 bytes
    assert _size(L, p)[0] == 2
    m = bd.MaskSpec()
    m.flags = bd.MASK_SEGMENT_IDS                   # ids missing
    assert _size(L, _prob(), m)[0] == 1
    m = bd.MaskSpec()
    m.flags = bd.MASK_VARLEN
    m.cu_seqlens = 16
    m.n_seqs = 2
    assert _size(L, _prob(B=2), m)[0] == 1          # varlen needs B == 1
    assert _size(L, _prob(Sq=100, Skv=120), m)[0] == 1  # and Sq == Skv
    m.flags = 1 << 7                                # unknown flag
    assert _size(L, _prob(), m)[0] == 1
    m = bd.MaskSpec()
    m.flags = bd.MASK_PREFIX_LM | bd.MASK_CAUSAL_WINDOW  # prefix lengths missing
    assert _size(L, _prob(), m)[0] == 1
    m.prefix_len = 16
    assert _size(L, _prob(), m)[0] == 0
    m.flags = bd.MASK_PREFIX_LM                     # a prefix needs the window
    assert _size(L, _prob(), m)[0] == 1
    m = bd.MaskSpec()
    m.dilation = 2                                  # a dilation needs the window
    assert _size(L, _prob(), m)[0] == 1
    m.flags = bd.MASK_CAUSAL_WINDOW
    assert _size(L, _prob(), m)[0] == 0
    m.dilation = -1
    assert _size(L, _prob(), m)[0] == 1


def test_every_mask_and_shape_check_rejects_its_case(L):
    """The remaining rejection branches of the problem and mask checks, each
    against an otherwise valid problem."""
    def varlen(**kw):
        m = bd.MaskSpec()
        m.flags = bd.MASK_VARLEN
        m.cu_seqlens, m.n_seqs, m.n_align_tail = 16, 2, 0
        for k_, v_ in kw.items():
            setattr(m, k_, v_)
        return m
    sq = dict(Sq=256, Skv=256)
    assert _size(L, _prob(**sq), varlen())[0] == 0                   # the valid case
    assert _size(L, _prob(**sq), varlen(n_seqs=0))[0] == 1          # no sequence
    assert _size(L, _prob(**sq), varlen(n_align_tail=3))[0] == 1    # more alignment segments than segments
    assert _size(L, _prob(**sq), varlen(n_align_tail=-1))[0] == 1
    assert _size(L, _prob(**sq), varlen(cu_seqlens=None))[0] == 1
    both = varlen(flags=bd.MASK_VARLEN | bd.MASK_SEGMENT_IDS, seg_q=16, seg_kv=16)
    assert _size(L, _prob(**sq), both)[0] == 1                        # varlen and segment ids exclude each other
    m = bd.MaskSpec()
    m.flags = bd.MASK_CAUSAL_WINDOW
    m.window = -1                                                     # a negative window
    assert _size(L, _prob(), m)[0] == 1
    m = bd.MaskSpec()
    m.flags = bd.MASK_KV_VALID_LEN                                    # lengths missing
    assert _size(L, _prob(), m)[0] == 1
    m.kv_valid_len = 16
    assert _size(L, _prob(), m)[0] == 0
    p = _prob(H=6)
    p.H_kv = 4                                                        # H not a multiple of H_kv
    assert _size(L, p)[0] == 1
    p.H_kv = -1
    assert _size(L, p)[0] == 1
    p.H_kv = 3
    assert _size(L, p)[0] == 0
    p = _prob()
    p.k_stride[:] = (0, -128, 64)                                     # a non-positive stride
    assert _size(L, p)[0] == 1


def test_calls_reject_bad_arguments_before_cuda(L):
    p = _prob()
    o = bd.Options()
    # null tensor pointers
    assert L.bsa_attn_fwd(ctypes.byref(p), None, ctypes.byref(o), None, None, None, None, None,
                          None, 0, None) == 1
    # misaligned pointers
    assert L.bsa_attn_fwd(ctypes.byref(p), None, ctypes.byref(o), 8, 256, 512, 1024, 4096,
                          4096, 1 << 20, None) == 2
    # the plan beside the bound: null and misaligned inputs
    assert L.bsa_plan_and_bound(ctypes.byref(p), None, ctypes.byref(o), None, 256, 4096, 1 << 20,
                                None) == 1
    assert L.bsa_plan_and_bound(ctypes.byref(p), None, ctypes.byref(o), 8, 256, 4096, 1 << 20,
                                None) == 2
    # bad order and a non-permutation
    o.bwd_order = 7
    assert L.bsa_plan_build(ctypes.byref(p), None, ctypes.byref(o), 4096, 1 << 30, None) == 1
    o.bwd_order = 2
    bad = (ctypes.c_int32 * 2)(0, 0)
    o.perm = ctypes.cast(bad, ctypes.c_void_p)
    assert L.bsa_plan_build(ctypes.byref(p), None, ctypes.byref(o), 4096, 1 << 30, None) == 1
    # an order past the last one
    o = bd.Options()
    o.bwd_order = 5
    assert L.bsa_plan_build(ctypes.byref(p), None, ctypes.byref(o), 4096, 16, None) == 1
    # unknown bound mode; the smoothed and per q-block bounds with a caller-supplied kmax
    o = bd.Options()
    o.bound_mode = 3
    assert L.bsa_plan_build(ctypes.byref(p), None, ctypes.byref(o), 4096, 1 << 30, None) == 1
    for mode in (1, 2):
        o.bound_mode = mode
        o.kmax_override = 4096
        assert L.bsa_plan_build(ctypes.byref(p), None, ctypes.byref(o), 4096, 1 << 30, None) == 1
    o.bound_mode = 1
    o.kmax_override = None
    wide = _prob(H=200, D=128)                      # centers of 200 heads exceed shared memory
    assert L.bsa_plan_build(ctypes.byref(wide), None, ctypes.byref(o), 4096, 1 << 40, None) == 2
    # an unknown O-residual mode; KEEP needs the backward-sized workspace, AUTO
    # and DROP do not
    o = bd.Options()
    o.o_residual = 3
    assert L.bsa_plan_build(ctypes.byref(p), None, ctypes.byref(o), 4096, 1 << 30, None) == 1
    o.o_residual = -1
    assert L.bsa_plan_build(ctypes.byref(p), None, ctypes.byref(o), 4096, 1 << 30, None) == 1
    o.o_residual = bd.O_RESIDUAL["keep"]
    fwd_only = _size(L, p, bwd=0)[1]
    assert L.bsa_plan_build(ctypes.byref(p), None, ctypes.byref(o), 4096, fwd_only, None) == 3
    # workspace too small
    o = bd.Options()
    assert L.bsa_plan_build(ctypes.byref(p), None, ctypes.byref(o), 4096, 16, None) == 3
    assert L.bsa_status_string(0).decode() == "ok"
    assert L.bsa_status_string(5).decode().startswith("a bounded device wait")


def test_empty_problem_is_a_checked_no_op(L):
    """B == 0 or Sq == 0: arguments are still checked, then every call returns
    ok with null tensors and workspace, no device and no launch; the one
    exception is the backward with key rows but no query row, which zeroes dK
    and dV."""
    for p in (_prob(B=0), _prob(Sq=0), _prob(B=0, Sq=0, D=128)):
        assert _size(L, p, bwd=0) == (0, 0) and _size(L, p, bwd=1) == (0, 0)
        v = bd.WorkspaceView()
        assert L.bsa_workspace_layout(ctypes.byref(p), None, ctypes.byref(v)) == 0
        assert v.total_bytes == v.fwd_bytes == v.off_delta == v.off_sem == 0
        assert (v.nM, v.nN) == ((p.Sq + 127) // 128, 2)
    for bad in (_prob(B=-1), _prob(Sq=-1), _prob(B=0, Skv=0), _prob(Sq=0, H=0)):
        assert _size(L, bad)[0] == 1
    assert _size(L, _prob(B=0, D=96))[0] == 2       # still an unsupported head dim
    seg = bd.MaskSpec()
    seg.flags = bd.MASK_SEGMENT_IDS                 # arrays of no element may be null
    assert _size(L, _prob(B=0), seg) == (0, 0)
    assert _size(L, _prob(), seg)[0] == 1
    before = L.bsa_launch_count()
    for p in (_prob(B=0), _prob(Sq=0)):
        P, o = ctypes.byref(p), ctypes.byref(bd.Options())
        n = None
        assert L.bsa_workspace_size(P, ctypes.byref(seg), 1, ctypes.byref(ctypes.c_size_t())) == 0
        assert L.bsa_plan_build(P, None, o, n, 0, n) == 0
        assert L.bsa_attn_fwd(P, None, o, n, n, n, n, n, n, 0, n) == 0
        assert L.bsa_attn_fwd(P, ctypes.byref(seg), o, n, n, n, n, n, n, 0, n) == 0
        if p.B == 0:
            assert L.bsa_attn_bwd(P, None, o, n, n, n, n, n, n, n, n, n, n, 0, n) == 0
            assert L.bsa_bwd_main(P, None, o, n, n, n, n, n, n, n, n, 0, n) == 0
        else:
            # keys but no query row: dK = dV = 0 must be written, so dk and dv
            # are checked and a device is needed (none here)
            assert L.bsa_attn_bwd(P, None, o, n, n, n, n, n, n, n, n, n, n, 0, n) == 1
            assert L.bsa_attn_bwd(P, None, o, n, n, n, n, n, n, n, 8, 4096, n, 0, n) == 2
            assert L.bsa_attn_bwd(P, None, o, n, n, n, n, n, n, n, 4096, 8192, n, 0, n) == 9
            assert L.bsa_bwd_main(P, None, o, n, n, n, n, n, n, 4096, n, 0, n) == 1
            assert L.bsa_bwd_main(P, None, o, n, n, n, n, n, 4096, 8192, n, 0, n) == 9
        assert L.bsa_fixed_m_bound(P, None, o, n, n, n, 0, n) == 0
        assert L.bsa_plan_and_bound(P, None, o, n, n, n, 0, n) == 0
        assert L.bsa_bwd_preprocess(P, None, o, n, n, n, n, 0, n) == 0
        assert L.bsa_bwd_convert(P, None, n, n, 0, n) == 0
        f = L.bsa_attn_fwd_static_scratch
        f.restype = ctypes.c_int32
        f.argtypes = [ctypes.POINTER(bd.Problem), ctypes.POINTER(bd.MaskSpec), ctypes.POINTER(bd.Options)] + \
            [ctypes.c_void_p] * 6
        assert f(P, None, o, n, n, n, n, n, n) == 0
        # the options are still checked
        bad = bd.Options()
        bad.softmax_mode = 7
        assert L.bsa_attn_fwd(P, None, ctypes.byref(bad), n, n, n, n, n, n, 0, n) == 1
        assert f(P, None, ctypes.byref(bad), n, n, n, n, n, n) == 1
    assert L.bsa_launch_count() == before


def test_layout_offsets_are_aligned(L):
    v = bd.WorkspaceView()
    assert L.bsa_workspace_layout(ctypes.byref(_prob(B=2, H=3, Sq=1000, Skv=777, D=128)), None,
                                  ctypes.byref(v)) == 0
    assert v.nM == 8 and v.nN == 7
    offs = [getattr(v, f) for f, _ in bd.WorkspaceView._fields_ if f.startswith("off_")]
    assert all(o % 4 == 0 for o in offs)
    assert v.off_status == 0 and v.fwd_bytes <= v.off_delta < v.total_bytes
