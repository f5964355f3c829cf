"""The allocation-free forward (bsa_attn_fwd_static_scratch) against the
regular bsa_attn_fwd, called through the C ABI.

Some callers cannot allocate device memory: plugin code run by a framework
that owns every device allocation and forbids cudaMalloc in its callbacks, or
code that must not risk the implicit synchronisation of cudaMalloc / cudaFree.
This entry point serves them with a fixed device array inside the library.

This file is collected last on purpose: if it fails, a run stopping at the
first failure has already run every other test.  It passes alone in a fresh
process and after the other tests."""

import ctypes

import numpy as np
import pytest
import torch

import block_sparse_attention_map_b200 as bsa
from block_sparse_attention_map_b200 import _binding as bd
from block_sparse_attention_map_b200.workloads import make_workload

pytestmark = pytest.mark.gpu


def _stream():
    return torch.cuda.current_stream().cuda_stream


def _static_fwd(q, k, v, mask_desc, softmax_mode):
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[0], q.shape[2], q.shape[1], dtype=torch.float32, device=q.device)
    prob = bd.make_problem(q, k, v, out)
    mask = bd.Mask(mask_desc, q.device)
    opt = bd.make_options(softmax_mode)
    rc = bd.lib().bsa_attn_fwd_static_scratch(ctypes.byref(prob), ctypes.byref(mask.spec), ctypes.byref(opt),
                                              q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                              lse.data_ptr(), _stream())
    assert rc == 0, bd.STATUS.get(rc, rc)
    return out, lse, mask


def _static_status(clear=False):
    return int(bd.lib().bsa_static_scratch_status(_stream(), 1 if clear else 0))


@pytest.mark.parametrize("name,mode", [("tiny", "online"), ("window", "fixed_m"), ("varlen", "online"),
                                       ("document", "fixed_m"), ("video", "fixed_m")])
def test_static_scratch_forward_equals_regular_forward_twice(name, mode):
    """Two calls in a row give exactly the regular forward's bits (the same plan,
    bound and kernels), report a clean status, and the second call allocates no
    device memory (free device memory unchanged across it)."""
    assert bd.lib().bsa_static_scratch_init() == 0
    wl = make_workload(name, device="cuda", small=True)
    o_ref, l_ref, ws = bsa.attn_fwd(wl.q, wl.k, wl.v, wl.mask, softmax_mode=mode, o_residual="drop")
    torch.cuda.synchronize()
    assert ws.status() == 0
    out = torch.empty_like(wl.q)
    lse = torch.empty_like(l_ref)
    prob = bd.make_problem(wl.q, wl.k, wl.v, out)
    mask = bd.Mask(wl.mask, wl.q.device)
    opt = bd.make_options(mode)
    free = []
    for _ in range(2):
        out.fill_(7.0)
        lse.fill_(7.0)
        torch.cuda.synchronize()
        free.append(torch.cuda.mem_get_info()[0])
        rc = bd.lib().bsa_attn_fwd_static_scratch(ctypes.byref(prob), ctypes.byref(mask.spec), ctypes.byref(opt),
                                                  wl.q.data_ptr(), wl.k.data_ptr(), wl.v.data_ptr(),
                                                  out.data_ptr(), lse.data_ptr(), _stream())
        assert rc == 0, bd.STATUS.get(rc, rc)
        assert _static_status() == 0
        assert torch.equal(out, o_ref) and torch.equal(lse, l_ref)
    free.append(torch.cuda.mem_get_info()[0])
    assert free[1] == free[2]  # the second call took no device memory


def test_static_scratch_reports_a_bad_cu_seqlens():
    """A non-monotone cu_seqlens is a host-supplied bad input that the planner
    checks on the device (its reads stay inside the array): both the regular
    and the allocation-free forward record BSA_ERR_BAD_MASK_DATA, each where its
    caller can read it, and a clean call afterwards reports ok again."""
    wl = make_workload("varlen", device="cuda", small=True)
    bad = dict(wl.mask)
    bad["cu_seqlens"] = np.asarray([0, 400, 300, 650, 704], dtype=np.int32)
    assert bad["cu_seqlens"][-1] == wl.Sq
    _, _, ws = bsa.attn_fwd(wl.q, wl.k, wl.v, bad)
    torch.cuda.synchronize()
    assert ws.status(clear=True) == 7  # BSA_ERR_BAD_MASK_DATA
    _static_fwd(wl.q, wl.k, wl.v, bad, "online")
    assert _static_status() == 7
    assert _static_status(clear=True) == 7
    assert _static_status() == 0
    _static_fwd(wl.q, wl.k, wl.v, wl.mask, "online")
    assert _static_status() == 0


def test_static_scratch_rejects_oversized_problems():
    wl = make_workload("tiny", device="cuda")
    out = torch.empty_like(wl.q)
    lse = torch.empty(wl.B, wl.H, wl.Sq, dtype=torch.float32, device="cuda")
    prob = bd.Problem()
    prob.B, prob.H, prob.Sq, prob.Skv, prob.D = 64, 64, 32768, 32768, 128  # far beyond 32 MiB
    opt = bd.make_options("online")
    rc = bd.lib().bsa_attn_fwd_static_scratch(ctypes.byref(prob), None, ctypes.byref(opt), wl.q.data_ptr(),
                                              wl.k.data_ptr(), wl.v.data_ptr(), out.data_ptr(),
                                              lse.data_ptr(), _stream())
    assert rc == 3  # BSA_ERR_WORKSPACE_TOO_SMALL, before any launch
