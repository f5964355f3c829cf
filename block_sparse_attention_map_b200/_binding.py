"""ctypes binding of libbsa (include/bsa.h).  Argument marshalling only: every
step of the computation runs in the library's CUDA kernels.  PyTorch supplies
device memory and the current stream.  There is no fallback: if the library is
missing or a call fails, an exception is raised."""

from __future__ import annotations

import ctypes
import math
import os
import re
from typing import Optional

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libbsa.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "bsa.h")

c_i32, c_u32, c_i64, c_f32, c_vp = ctypes.c_int32, ctypes.c_uint32, ctypes.c_int64, ctypes.c_float, ctypes.c_void_p

# --- constants mirrored from include/bsa.h
TILE = 128
TILE_EMPTY, TILE_PARTIAL, TILE_FULL = 0, 1, 2
MASK_SEGMENT_IDS, MASK_KV_VALID_LEN, MASK_VARLEN, MASK_CAUSAL_WINDOW, MASK_PREFIX_LM = 1, 2, 4, 8, 16
SOFTMAX_ONLINE, SOFTMAX_FIXED_M_GATED = 0, 1
BOUND = {"norm": 0, "smoothed": 1, "block": 2}
ORDER = {"asc": 0, "desc": 1, "perm": 2, "outside_in": 3, "greedy": 4}
O_RESIDUAL = {"auto": 0, "keep": 1, "drop": 2}
FULL_BIT = 1 << 30
STATUS = {
    0: "BSA_OK", 1: "BSA_ERR_INVALID_ARG", 2: "BSA_ERR_UNSUPPORTED",
    3: "BSA_ERR_WORKSPACE_TOO_SMALL", 4: "BSA_ERR_CUDA", 5: "BSA_ERR_SEM_TIMEOUT",
    6: "BSA_ERR_PLAN_MISMATCH", 7: "BSA_ERR_BAD_MASK_DATA", 8: "BSA_WARN_GATE_VIOLATION",
    9: "BSA_ERR_NO_DEVICE", 10: "BSA_ERR_INPUT_RANGE",
}


class Problem(ctypes.Structure):
    _fields_ = [("B", c_i32), ("H", c_i32), ("Sq", c_i32), ("Skv", c_i32), ("D", c_i32),
                ("H_kv", c_i32), ("q_stride", c_i64 * 3), ("k_stride", c_i64 * 3),
                ("v_stride", c_i64 * 3), ("o_stride", c_i64 * 3), ("scale", c_f32),
                ("reserved1", c_i32)]


class MaskSpec(ctypes.Structure):
    _fields_ = [("flags", c_u32), ("window", c_i32), ("seg_q", c_vp), ("seg_kv", c_vp),
                ("kv_valid_len", c_vp), ("cu_seqlens", c_vp), ("n_seqs", c_i32),
                ("n_align_tail", c_i32), ("prefix_len", c_vp), ("dilation", c_i32),
                ("reserved", c_i32)]


class Options(ctypes.Structure):
    _fields_ = [("softmax_mode", c_i32), ("gate_limit", c_f32), ("kmax_override", c_vp),
                ("bwd_order", c_i32), ("deterministic", c_i32), ("perm", c_vp),
                ("sem_timeout_ns", c_i64), ("plan_ready", c_i32), ("bound_ready", c_i32),
                ("bound_mode", c_i32), ("o_residual", c_i32)]


class WorkspaceView(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in (
        "total_bytes", "fwd_bytes", "off_status", "off_tile_class", "off_rank", "off_row_ptr",
        "off_row_ent", "off_col_ptr", "off_col_ent", "off_col_rank", "off_perm", "off_kmax",
        "off_qmax", "off_gate", "off_delta", "off_dq_accum", "off_sem", "off_kbar", "off_qdot",
        "off_o_resid", "off_kblk", "off_kmax_q")] + \
        [("nM", c_i32), ("nN", c_i32)]


class BsaError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {STATUS.get(code, code)} ({_lib_status_string(code)})")


_LIB = None


def header_functions() -> list[str]:
    """Names of every function include/bsa.h declares."""
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*BSA_API\s+(?:const\s+)?[a-z_0-9]+\s*\*?\s*(bsa_[a-z_0-9]+)\s*\(", text, re.M)))


def lib() -> ctypes.CDLL:
    """The loaded libbsa.  Raises if it has not been built: there is no fallback."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing; build it with `python -m block_sparse_attention_map_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.POINTER
        sig = {
            "bsa_workspace_size": (c_i32, [P(Problem), P(MaskSpec), c_i32, P(ctypes.c_size_t)]),
            "bsa_workspace_layout": (c_i32, [P(Problem), P(MaskSpec), P(WorkspaceView)]),
            "bsa_plan_build": (c_i32, [P(Problem), P(MaskSpec), P(Options), c_vp, ctypes.c_size_t, c_vp]),
            "bsa_attn_fwd": (c_i32, [P(Problem), P(MaskSpec), P(Options), c_vp, c_vp, c_vp, c_vp, c_vp,
                                     c_vp, ctypes.c_size_t, c_vp]),
            "bsa_attn_bwd": (c_i32, [P(Problem), P(MaskSpec), P(Options), c_vp, c_vp, c_vp, c_vp, c_vp,
                                     c_vp, c_vp, c_vp, c_vp, c_vp, ctypes.c_size_t, c_vp]),
            "bsa_fixed_m_bound": (c_i32, [P(Problem), P(MaskSpec), P(Options), c_vp, c_vp, c_vp,
                                          ctypes.c_size_t, c_vp]),
            "bsa_plan_and_bound": (c_i32, [P(Problem), P(MaskSpec), P(Options), c_vp, c_vp, c_vp,
                                           ctypes.c_size_t, c_vp]),
            "bsa_bwd_preprocess": (c_i32, [P(Problem), P(MaskSpec), P(Options), c_vp, c_vp, c_vp, c_vp,
                                           ctypes.c_size_t, c_vp]),
            "bsa_bwd_main": (c_i32, [P(Problem), P(MaskSpec), P(Options), c_vp, c_vp, c_vp, c_vp, c_vp,
                                     c_vp, c_vp, c_vp, ctypes.c_size_t, c_vp]),
            "bsa_bwd_convert": (c_i32, [P(Problem), P(MaskSpec), c_vp, c_vp, ctypes.c_size_t, c_vp]),
            "bsa_get_device_status": (c_i32, [c_vp, ctypes.c_size_t, c_vp, c_i32]),
            "bsa_status_string": (ctypes.c_char_p, [c_i32]),
            "bsa_attn_fwd_static_scratch": (c_i32, [P(Problem), P(MaskSpec), P(Options), c_vp, c_vp, c_vp, c_vp,
                                                    c_vp, c_vp]),
            "bsa_static_scratch_init": (c_i32, []),
            "bsa_static_scratch_status": (c_i32, [c_vp, c_i32]),
            "bsa_launch_count": (ctypes.c_uint64, []),
            "bsa_fixed_rows": (c_i32, [c_vp, ctypes.c_size_t, c_vp, P(ctypes.c_uint64)]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = L
    return _LIB


def _lib_status_string(code: int) -> str:
    try:
        return lib().bsa_status_string(code).decode()
    except Exception:
        return "?"


def _check(code: int, what: str):
    if code != 0:
        raise BsaError(code, what)


def launch_count() -> int:
    return int(lib().bsa_launch_count())


# ------------------------------------------------------------------ marshalling

def _strides(t: torch.Tensor):
    if t.dim() != 4:
        raise ValueError("expected a [B, S, H, D] tensor")
    if t.stride(3) != 1:
        raise ValueError("the head dimension must be contiguous")
    return (t.stride(0), t.stride(1), t.stride(2))


def make_problem(q, k, v, o=None, scale: Optional[float] = None) -> Problem:
    for t in (q, k, v):
        if t.dtype != torch.bfloat16 or not t.is_cuda:
            raise ValueError("q, k, v must be bf16 CUDA tensors")
    B, Sq, H, D = q.shape
    H_kv = k.shape[2]
    if k.shape[0] != B or H_kv < 1 or H % H_kv != 0 or k.shape[3] != D or v.shape != k.shape:
        raise ValueError("k and v must be [B, Skv, H_kv, D] with q's B and D and H a multiple of H_kv")
    p = Problem()
    p.B, p.H, p.Sq, p.Skv, p.D, p.H_kv = B, H, Sq, k.shape[1], D, H_kv
    p.q_stride[:] = _strides(q)
    p.k_stride[:] = _strides(k)
    p.v_stride[:] = _strides(v)
    p.o_stride[:] = _strides(o) if o is not None else (max(Sq, 1) * H * D, H * D, D)
    p.scale = float(scale) if scale else 1.0 / math.sqrt(D)
    return p


class Mask:
    """Mask predicates for the library, as device int32 tensors kept alive here.

    Keys of ``desc`` (all optional): ``seg_q``, ``seg_kv`` ([B, S] ints),
    ``kv_valid_len`` ([B]), ``cu_seqlens`` ([n_seqs + 1]) with ``n_align_tail``,
    ``window`` (None: off, 0: causal, W: causal band of W keys) with
    ``dilation`` (keep every d-th key back from the diagonal) and ``prefix_len``
    ([B]: keys below it are seen by every row)."""

    def __init__(self, desc: Optional[dict], device):
        desc = desc or {}
        self.spec = MaskSpec()
        self._keep = []

        def dev(x):
            t = torch.as_tensor(np.asarray(x.cpu() if isinstance(x, torch.Tensor) else x),
                                dtype=torch.int32).to(device).contiguous()
            self._keep.append(t)
            return t

        if desc.get("seg_q") is not None:
            self.spec.flags |= MASK_SEGMENT_IDS
            self.spec.seg_q = dev(desc["seg_q"]).data_ptr()
            self.spec.seg_kv = dev(desc["seg_kv"]).data_ptr()
        if desc.get("kv_valid_len") is not None:
            self.spec.flags |= MASK_KV_VALID_LEN
            self.spec.kv_valid_len = dev(desc["kv_valid_len"]).data_ptr()
        if desc.get("cu_seqlens") is not None:
            cu = dev(desc["cu_seqlens"])
            self.spec.flags |= MASK_VARLEN
            self.spec.cu_seqlens = cu.data_ptr()
            self.spec.n_seqs = cu.numel() - 1
            self.spec.n_align_tail = int(desc.get("n_align_tail", 0))
        if desc.get("window") is not None:
            self.spec.flags |= MASK_CAUSAL_WINDOW
            self.spec.window = int(desc["window"])
        if desc.get("dilation") is not None:
            self.spec.dilation = int(desc["dilation"])
        if desc.get("prefix_len") is not None:
            self.spec.flags |= MASK_PREFIX_LM
            self.spec.prefix_len = dev(desc["prefix_len"]).data_ptr()


def make_options(softmax_mode="online", gate_limit=0.0, kmax_override=None, order="asc",
                 perm=None, deterministic=True, sem_timeout_ns=0, plan_ready=False,
                 bound_ready=False, bound_mode="norm", o_residual="auto"):
    o = Options()
    o.softmax_mode = SOFTMAX_FIXED_M_GATED if softmax_mode in ("fixed_m", SOFTMAX_FIXED_M_GATED) else SOFTMAX_ONLINE
    o.gate_limit = float(gate_limit)
    o.kmax_override = kmax_override.data_ptr() if kmax_override is not None else None
    o.bwd_order = ORDER[order] if isinstance(order, str) else int(order)
    o.deterministic = 1 if deterministic else 0
    o.sem_timeout_ns = int(sem_timeout_ns)
    o.plan_ready = 1 if plan_ready else 0
    o.bound_ready = 1 if bound_ready else 0
    o.bound_mode = BOUND[bound_mode] if isinstance(bound_mode, str) else int(bound_mode)
    o.o_residual = O_RESIDUAL[o_residual] if isinstance(o_residual, str) else int(o_residual)
    o._perm_buf = None
    if perm is not None:
        buf = (c_i32 * len(perm))(*[int(x) for x in perm])
        o._perm_buf = buf
        o.perm = ctypes.cast(buf, c_vp)
    return o


class Workspace:
    """A caller-owned workspace (torch uint8 buffer) and its layout."""

    def __init__(self, prob: Problem, mask: Mask, backward: bool, device):
        view = WorkspaceView()
        _check(lib().bsa_workspace_layout(ctypes.byref(prob), ctypes.byref(mask.spec), ctypes.byref(view)),
               "bsa_workspace_layout")
        self.view = view
        self.nbytes = view.total_bytes if backward else view.fwd_bytes
        self.buf = torch.empty(self.nbytes, dtype=torch.uint8, device=device)
        self.B, self.H, self.D, self.nM, self.nN = prob.B, prob.H, prob.D, view.nM, view.nN
        self.H_kv = prob.H_kv or prob.H

    def ptr(self):
        return self.buf.data_ptr()

    def _arr(self, off, count, dtype):
        n = count * torch.tensor([], dtype=dtype).element_size()
        return self.buf[off:off + n].view(dtype)

    # inspection helpers (tests)
    def header(self):
        """The workspace header's 64 uint32 words (status, tickets, plan signature, records)."""
        return self._arr(self.view.off_status, 64, torch.int32)

    def tile_classes(self):
        return self._arr(self.view.off_tile_class, self.B * self.nM * self.nN, torch.uint8).view(
            self.B, self.nM, self.nN)

    def ranks(self):
        return self._arr(self.view.off_rank, self.B * self.nM * self.nN, torch.int32).view(
            self.B, self.nM, self.nN)

    def row_lists(self):
        ptr = self._arr(self.view.off_row_ptr, self.B * self.nM + 1, torch.int32).cpu().numpy()
        ent = self._arr(self.view.off_row_ent, int(ptr[-1]), torch.int32).cpu().numpy().astype(np.int64)
        return ptr, ent

    def col_lists(self):
        ptr = self._arr(self.view.off_col_ptr, self.B * self.nN + 1, torch.int32).cpu().numpy()
        nnz = int(ptr[-1])
        ent = self._arr(self.view.off_col_ent, nnz, torch.int32).cpu().numpy().astype(np.int64)
        rk = self._arr(self.view.off_col_rank, nnz, torch.int32).cpu().numpy()
        return ptr, ent, rk

    def perm(self):
        return self._arr(self.view.off_perm, self.nN, torch.int32)

    def kmax(self):
        return self._arr(self.view.off_kmax, self.B * self.H, torch.float32).view(self.B, self.H)

    def qmax(self):
        return self._arr(self.view.off_qmax, self.B * self.H, torch.float32).view(self.B, self.H)

    def gate(self):
        return self._arr(self.view.off_gate, self.B * self.H, torch.int32).view(self.B, self.H)

    def kmax_q(self):
        """Each q-block's kmax [B, H, nM] (the per q-block bound, as the forward used it)."""
        return self._arr(self.view.off_kmax_q, self.B * self.H * self.nM, torch.float32).view(
            self.B, self.H, self.nM)

    def kblk(self):
        """Per kv block and key head, the largest valid ||k_j|| [B, H_kv, nN] (block bound)."""
        return self._arr(self.view.off_kblk, self.B * self.H_kv * self.nN, torch.float32).view(
            self.B, self.H_kv, self.nN)

    def kbar(self):
        """The k-smoothing centers [B, H_kv, D] (after a smoothed bound)."""
        return self._arr(self.view.off_kbar, self.B * self.H_kv * self.D, torch.float32).view(
            self.B, self.H_kv, self.D)

    def fixed_rows(self):
        """Query rows the forwards since the last plan build ran fixed-m."""
        n = ctypes.c_uint64(0)
        _check(lib().bsa_fixed_rows(self.ptr(), self.nbytes, _stream(), ctypes.byref(n)), "bsa_fixed_rows")
        return int(n.value)

    def status(self, clear=False):
        s = torch.cuda.current_stream().cuda_stream
        return int(lib().bsa_get_device_status(self.ptr(), self.nbytes, s, 1 if clear else 0))


def _stream():
    return torch.cuda.current_stream().cuda_stream


def workspace_size(q, k, v, mask=None, backward=True) -> int:
    prob = make_problem(q, k, v)
    m = Mask(mask, q.device)
    n = ctypes.c_size_t(0)
    _check(lib().bsa_workspace_size(ctypes.byref(prob), ctypes.byref(m.spec), 1 if backward else 0,
                                    ctypes.byref(n)), "bsa_workspace_size")
    return n.value


def plan_build(q, k, v, mask=None, workspace: Optional[Workspace] = None, backward=True, **opt):
    prob = make_problem(q, k, v)
    m = Mask(mask, q.device)
    o = make_options(**opt)
    ws = workspace or Workspace(prob, m, backward, q.device)
    _check(lib().bsa_plan_build(ctypes.byref(prob), ctypes.byref(m.spec), ctypes.byref(o), ws.ptr(),
                                ws.nbytes, _stream()), "bsa_plan_build")
    ws._mask = m
    return ws


def attn_fwd(q, k, v, mask=None, softmax_mode="online", gate_limit=0.0, kmax_override=None,
             workspace: Optional[Workspace] = None, out=None, lse=None, plan_ready=False,
             scale=None, order="asc", perm=None, bound_mode="norm", o_residual="auto",
             for_backward=True):
    """O = softmax(scale Q K^T + mask) V and LSE [B, H, Sq] through bsa_attn_fwd.

    The workspace it allocates (unless one is given) is sized for a backward
    (``for_backward``), so that with the default ``o_residual="auto"`` it keeps
    O's bf16 rounding residual: an ``attn_bwd(..., workspace=ws)`` on the
    returned workspace then takes Delta exact to the fp32 O.  Returns
    (out, lse, workspace)."""
    B, Sq, H, D = q.shape
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty(B, H, Sq, dtype=torch.float32, device=q.device) if lse is None else lse
    prob = make_problem(q, k, v, out, scale)
    m = Mask(mask, q.device)
    o = make_options(softmax_mode, gate_limit, kmax_override, order, perm, True, 0, plan_ready,
                     bound_mode=bound_mode, o_residual=o_residual)
    ws = workspace or Workspace(prob, m, for_backward or o_residual == "keep", q.device)
    _check(lib().bsa_attn_fwd(ctypes.byref(prob), ctypes.byref(m.spec), ctypes.byref(o), q.data_ptr(),
                              k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), ws.ptr(),
                              ws.nbytes, _stream()), "bsa_attn_fwd")
    ws._mask = m
    return out, lse, ws


def attn_bwd(q, k, v, out, dout, lse, mask=None, order="asc", perm=None, deterministic=True,
             workspace: Optional[Workspace] = None, plan_ready=False, scale=None,
             dq=None, dk=None, dv=None, sem_timeout_ns=0, o_residual="auto"):
    """dQ, dK, dV of sum(O * dO) through bsa_attn_bwd.  Pass the forward's
    workspace: with ``o_residual="auto"`` (or "keep") Delta then uses the O
    residual that attn_fwd kept there for this ``out`` (checked on the device);
    without it, or with "drop", Delta comes from the bf16 O."""
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    prob = make_problem(q, k, v, out, scale)
    m = Mask(mask, q.device)
    o = make_options("online", 0.0, None, order, perm, deterministic, sem_timeout_ns, plan_ready,
                     o_residual=o_residual)
    ws = workspace or Workspace(prob, m, True, q.device)
    _check(lib().bsa_attn_bwd(ctypes.byref(prob), ctypes.byref(m.spec), ctypes.byref(o), q.data_ptr(),
                              k.data_ptr(), v.data_ptr(), out.data_ptr(), dout.data_ptr(), lse.data_ptr(),
                              dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), ws.ptr(), ws.nbytes,
                              _stream()), "bsa_attn_bwd")
    ws._mask = m
    return dq, dk, dv, ws


class Stages:
    """The hot path one C-ABI call per stage (a1+a6 plan, a2 bound, a3 forward,
    a4 preprocess, a5 backward main, a7 dQ convert), on one preallocated
    workspace, for callers that time or schedule stages separately."""

    def __init__(self, q, k, v, mask=None, softmax_mode="online", order="asc", perm=None,
                 deterministic=True, gate_limit=0.0, bound_mode="norm", o_residual="auto"):
        self.q, self.k, self.v = q, k, v
        B, Sq, H, D = q.shape
        self.out = torch.empty_like(q)
        self.lse = torch.empty(B, H, Sq, dtype=torch.float32, device=q.device)
        self.dq, self.dk, self.dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        self.prob = make_problem(q, k, v, self.out)
        self.mask = Mask(mask, q.device)
        self.fixed = softmax_mode in ("fixed_m", SOFTMAX_FIXED_M_GATED)
        self.opt = make_options(softmax_mode, gate_limit, None, order, perm, deterministic, 0,
                                plan_ready=True, bound_ready=True, bound_mode=bound_mode,
                                o_residual=o_residual)
        self.ws = Workspace(self.prob, self.mask, True, q.device)
        self._args = (ctypes.byref(self.prob), ctypes.byref(self.mask.spec), ctypes.byref(self.opt))

    def plan(self):
        _check(lib().bsa_plan_build(*self._args, self.ws.ptr(), self.ws.nbytes, _stream()), "bsa_plan_build")

    def bound(self):
        if self.fixed:
            _check(lib().bsa_fixed_m_bound(*self._args, self.q.data_ptr(), self.k.data_ptr(), self.ws.ptr(),
                                           self.ws.nbytes, _stream()), "bsa_fixed_m_bound")

    def plan_and_bound(self):
        """The plan and, in fixed-m mode, the bound in one call (the planner beside
        the bound's row-norm pass, on the library's side stream)."""
        if self.fixed:
            _check(lib().bsa_plan_and_bound(*self._args, self.q.data_ptr(), self.k.data_ptr(), self.ws.ptr(),
                                            self.ws.nbytes, _stream()), "bsa_plan_and_bound")
        else:
            self.plan()

    def forward(self):
        _check(lib().bsa_attn_fwd(*self._args, self.q.data_ptr(), self.k.data_ptr(), self.v.data_ptr(),
                                  self.out.data_ptr(), self.lse.data_ptr(), self.ws.ptr(), self.ws.nbytes,
                                  _stream()), "bsa_attn_fwd")

    def preprocess(self, dout):
        _check(lib().bsa_bwd_preprocess(*self._args, self.q.data_ptr(), self.out.data_ptr(), dout.data_ptr(),
                                        self.ws.ptr(), self.ws.nbytes, _stream()), "bsa_bwd_preprocess")

    def backward_main(self, dout):
        _check(lib().bsa_bwd_main(*self._args, self.q.data_ptr(), self.k.data_ptr(), self.v.data_ptr(),
                                  dout.data_ptr(), self.lse.data_ptr(), self.dk.data_ptr(),
                                  self.dv.data_ptr(), self.ws.ptr(), self.ws.nbytes, _stream()),
               "bsa_bwd_main")

    def convert(self):
        _check(lib().bsa_bwd_convert(ctypes.byref(self.prob), ctypes.byref(self.mask.spec),
                                     self.dq.data_ptr(), self.ws.ptr(), self.ws.nbytes, _stream()),
               "bsa_bwd_convert")
