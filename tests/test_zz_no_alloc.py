"""The allocation-free forward (bsa_attn_fwd_static_scratch) against the
regular bsa_attn_fwd, called through the C ABI.  This file is collected last on
purpose: if it fails, a run stopping at the first failure has already run every
other test.  It passes alone in a fresh process and after the other tests."""

import ctypes

import pytest
import torch

import block_sparse_attention_map_b200 as bsa
from block_sparse_attention_map_b200 import _binding as bd
from block_sparse_attention_map_b200.workloads import make_workload

pytestmark = pytest.mark.gpu

O_TOL, LSE_TOL = 1e-2, 1e-3


def _fn():
    f = bd.lib().bsa_attn_fwd_static_scratch
    P = ctypes.POINTER
    f.restype = ctypes.c_int32
    f.argtypes = [P(bd.Problem), P(bd.MaskSpec), P(bd.Options)] + [ctypes.c_void_p] * 6
    return f


def _static_fwd(wl, softmax_mode):
    out = torch.empty_like(wl.q)
    lse = torch.empty(wl.B, wl.H, wl.Sq, dtype=torch.float32, device=wl.q.device)
    prob = bd.make_problem(wl.q, wl.k, wl.v, out)
    mask = bd.Mask(wl.mask, wl.q.device)
    opt = bd.make_options(softmax_mode)
    rc = _fn()(ctypes.byref(prob), ctypes.byref(mask.spec), ctypes.byref(opt), wl.q.data_ptr(),
               wl.k.data_ptr(), wl.v.data_ptr(), out.data_ptr(), lse.data_ptr(),
               torch.cuda.current_stream().cuda_stream)
    assert rc == 0, bd.STATUS.get(rc, rc)
    return out, lse


@pytest.mark.parametrize("name,mode", [("tiny", "online"), ("window", "fixed_m"), ("varlen", "online")])
def test_static_scratch_forward_matches_regular_forward_twice(name, mode):
    wl = make_workload(name, device="cuda", small=True)
    o_ref, l_ref, ws = bsa.attn_fwd(wl.q, wl.k, wl.v, wl.mask, softmax_mode=mode)
    torch.cuda.synchronize()
    assert ws.status() == 0
    for _ in range(2):
        o, l = _static_fwd(wl, mode)
        torch.cuda.synchronize()
        assert (o.float() - o_ref.float()).abs().max().item() <= O_TOL
        fin = torch.isfinite(l_ref)
        assert torch.equal(fin, torch.isfinite(l))
        assert (l[fin] - l_ref[fin]).abs().max().item() <= LSE_TOL


def test_static_scratch_rejects_oversized_problems():
    wl = make_workload("tiny", device="cuda")
    out = torch.empty_like(wl.q)
    lse = torch.empty(wl.B, wl.H, wl.Sq, dtype=torch.float32, device="cuda")
    prob = bd.Problem()
    prob.B, prob.H, prob.Sq, prob.Skv, prob.D = 64, 64, 32768, 32768, 128  # far beyond 32 MiB
    opt = bd.make_options("online")
    rc = _fn()(ctypes.byref(prob), None, ctypes.byref(opt), wl.q.data_ptr(), wl.k.data_ptr(),
               wl.v.data_ptr(), out.data_ptr(), lse.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == 3  # BSA_ERR_WORKSPACE_TOO_SMALL, before any launch
