"""Seeded synthetic inputs for the five workloads (shapes, distributions, masks).

This module only draws inputs; it holds none of the attention arithmetic, so the
tests, the bench and the oracle can share it without sharing the method.

Workloads (names used by the tests and ``bench.py``):

``tiny``       B=1, H=2, Sq=Skv=256, D=64, N(0,1), no mask.
``packed``     B=2, H=8, S=4096, D=128, N(0,1); segment ids from contiguous runs
               of length uniform{256..2048} (last run truncated), block-diagonal.
``packed_const`` the same tensors with one constant segment id per batch row.
``window``     B=1, H=16, Sq=Skv=8192, D=128, causal sliding window of 512 keys.
``window_rect`` B=1, H=16, Sq=4096, Skv=8192, same window, bottom-right aligned.
``varlen``     B=1 (packed), H=24, T=33024, D=128, cu_seqlens=[0, 33002, 33024],
               the last segment (22 rows) being alignment padding; non-causal.
``video``      B=1, H=40, Sq=75600 (21x45x80 latent grid), Skv=75776 (padded to a
               multiple of 2048, padding masked), D=128; q, k ~ N(0, 0.5) with a
               3-axis rotary embedding, v ~ N(0, 1); head 0 has 8 "sink" keys
               scaled x20.

The three mask families the dk-order benchmark names besides sliding windows,
at its 8192x8192 shape and the sliding-window workload's B, H, D and seed
(the benchmark table states neither their head counts nor their parameters):

``prefix_lm``  causal with a bidirectional prefix of 2048 keys.
``dilated``    causal band spanning 1024 keys, every second key kept (512 per
               row, as many as the 512-key sliding window).
``document``   document-causal: segment ids from runs of uniform{256..2048}
               tokens, causal inside each document.

And one grouped-query shape (the benchmark's "kv_mode" column is MHA in every
row; the grouping is this build's reading):

``gqa``        B=1, H=16 query heads over H_kv=4 key/value heads, Sq=Skv=8192,
               D=128, causal sliding window of 512 keys, N(0,1), seed 5.

``small=True`` shrinks the sequence lengths (same structure, same recipe) so the
fp64 oracle finishes in seconds; the parity tests use it for the full-oracle
comparison and sample rows at full size.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import numpy as np
import torch


@dataclass
class Workload:
    name: str
    B: int
    H: int
    Sq: int
    Skv: int
    D: int
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    dO: Optional[torch.Tensor]
    mask: dict = field(default_factory=dict)
    scale: float = 0.0
    backward: bool = True

    def mask_text(self) -> str:
        """The mask parameters in words (arrays by their length)."""
        parts = []
        for key, val in self.mask.items():
            if isinstance(val, (torch.Tensor, np.ndarray)):
                arr = val.cpu().numpy() if isinstance(val, torch.Tensor) else val
                parts.append(f"{key}={arr.tolist()}" if arr.size <= 4 else f"{key}[{arr.shape}]")
            else:
                parts.append(f"{key}={val}")
        return ", ".join(parts) or "none"

    def mask_numpy(self) -> dict:
        """The mask description with every array on the host (numpy)."""
        out = {}
        for key, val in self.mask.items():
            out[key] = val.cpu().numpy() if isinstance(val, torch.Tensor) else val
        return out


WORKLOADS = ("tiny", "packed", "packed_const", "window", "window_rect", "varlen", "video",
             "prefix_lm", "dilated", "document", "gqa")


def _normal(shape, gen, device, std=1.0):
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    return x * std if std != 1.0 else x


def _segment_runs(rng: np.random.Generator, S: int, lo: int = 256, hi: int = 2048) -> np.ndarray:
    """Segment ids 0, 1, 2, ... in contiguous runs of length uniform{lo..hi};
    the last run is truncated at S."""
    ids = np.empty(S, dtype=np.int32)
    pos, sid = 0, 0
    while pos < S:
        run = int(rng.integers(lo, hi + 1))
        ids[pos:pos + run] = sid
        pos += run
        sid += 1
    return ids


def _rope_3axis(x: torch.Tensor, grid=(21, 45, 80), pairs=(22, 21, 21), theta=10000.0):
    """Rotary embedding over (t, h, w) latent positions, t-major token order.

    x: [B, S, H, D] fp32 with S == prod(grid) and D == 2 * sum(pairs).  Pair p of
    axis a rotates by pos_a * theta^(-2 k / d_a) with k the pair's index within
    the axis and d_a = 2 * pairs[a].  Rotation keeps every vector's norm."""
    T, Hh, W = grid
    S = T * Hh * W
    dev = x.device
    s = torch.arange(S, device=dev)
    pos = (s // (Hh * W), (s // W) % Hh, s % W)
    angles = []
    for a, n_pairs in enumerate(pairs):
        d_a = 2 * n_pairs
        inv = theta ** (-2.0 * torch.arange(n_pairs, device=dev, dtype=torch.float64) / d_a)
        angles.append(pos[a].to(torch.float64)[:, None] * inv[None, :])
    ang = torch.cat(angles, dim=1).to(torch.float32)  # [S, D/2]
    c = torch.cos(ang)[None, :, None, :]
    sn = torch.sin(ang)[None, :, None, :]
    x0 = x[..., 0::2]
    x1 = x[..., 1::2]
    out = torch.empty_like(x)
    out[..., 0::2] = x0 * c - x1 * sn
    out[..., 1::2] = x0 * sn + x1 * c
    return out


def make_workload(name: str, device="cpu", small: bool = False, seed: Optional[int] = None) -> Workload:
    """Draw one workload's bf16 inputs on ``device`` from its fixed seed."""
    dev = torch.device(device)
    bf16 = torch.bfloat16

    def gen_for(s):
        g = torch.Generator(device=dev)
        g.manual_seed(s)
        return g

    if name == "tiny":
        sd = 0 if seed is None else seed
        B, H, S, D = 1, 2, 256, 64
        g = gen_for(sd)
        q, k, v, dO = (_normal((B, S, H, D), g, dev).to(bf16) for _ in range(4))
        return Workload(name, B, H, S, S, D, q, k, v, dO, {}, 1.0 / math.sqrt(D))

    if name in ("packed", "packed_const"):
        sd = 1 if seed is None else seed
        B, H, S, D = 2, 8, 4096, 128
        lo, hi = 256, 2048
        if small:
            H, S, lo, hi = 2, 1024, 64, 512
        g = gen_for(sd)
        q, k, v, dO = (_normal((B, S, H, D), g, dev).to(bf16) for _ in range(4))
        if name == "packed":
            rng = np.random.default_rng(sd)
            ids = np.stack([_segment_runs(rng, S, lo, hi) for _ in range(B)])
        else:
            ids = np.zeros((B, S), dtype=np.int32) + 7
        seg = torch.from_numpy(ids).to(dev)
        mask = {"seg_q": seg, "seg_kv": seg.clone()}
        return Workload(name, B, H, S, S, D, q, k, v, dO, mask, 1.0 / math.sqrt(D))

    if name in ("window", "window_rect"):
        sd = 2 if seed is None else seed
        B, H, D, W = 1, 16, 128, 512
        Sq, Skv = (8192, 8192) if name == "window" else (4096, 8192)
        if small:
            H, W = 2, 256
            Sq, Skv = (1000, 1000) if name == "window" else (600, 1000)
        g = gen_for(sd)
        q = _normal((B, Sq, H, D), g, dev).to(bf16)
        k = _normal((B, Skv, H, D), g, dev).to(bf16)
        v = _normal((B, Skv, H, D), g, dev).to(bf16)
        dO = _normal((B, Sq, H, D), g, dev).to(bf16)
        return Workload(name, B, H, Sq, Skv, D, q, k, v, dO, {"window": W}, 1.0 / math.sqrt(D))

    if name in ("prefix_lm", "dilated", "document"):
        sd = 2 if seed is None else seed
        B, H, D, S = 1, 16, 128, 8192
        prefix, span, dil, lo, hi = 2048, 1024, 2, 256, 2048
        if small:
            H, S = 2, 1000
            prefix, span, dil, lo, hi = 300, 384, 3, 64, 400
        g = gen_for(sd)
        q, k, v, dO = (_normal((B, S, H, D), g, dev).to(bf16) for _ in range(4))
        if name == "prefix_lm":
            mask = {"window": 0, "prefix_len": np.full(B, prefix, dtype=np.int32)}
        elif name == "dilated":
            mask = {"window": span, "dilation": dil}
        else:
            rng = np.random.default_rng(sd)
            seg = torch.from_numpy(np.stack([_segment_runs(rng, S, lo, hi) for _ in range(B)])).to(dev)
            mask = {"seg_q": seg, "seg_kv": seg.clone(), "window": 0}
        return Workload(name, B, H, S, S, D, q, k, v, dO, mask, 1.0 / math.sqrt(D))

    if name == "gqa":
        sd = 5 if seed is None else seed
        B, H, H_kv, D, S, W = 1, 16, 4, 128, 8192, 512
        if small:
            H, H_kv, S, W = 4, 2, 1000, 256
        g = gen_for(sd)
        q = _normal((B, S, H, D), g, dev).to(bf16)
        k = _normal((B, S, H_kv, D), g, dev).to(bf16)
        v = _normal((B, S, H_kv, D), g, dev).to(bf16)
        dO = _normal((B, S, H, D), g, dev).to(bf16)
        return Workload(name, B, H, S, S, D, q, k, v, dO, {"window": W}, 1.0 / math.sqrt(D))

    if name == "varlen":
        sd = 3 if seed is None else seed
        H, D = 24, 128
        cu = [0, 33002, 33024]
        if small:
            H, cu = 2, [0, 300, 620, 650, 704]
        T = cu[-1]
        g = gen_for(sd)
        q, k, v = (_normal((1, T, H, D), g, dev).to(bf16) for _ in range(3))
        mask = {"cu_seqlens": np.asarray(cu, dtype=np.int32), "n_align_tail": 1}
        return Workload(name, 1, H, T, T, D, q, k, v, None, mask, 1.0 / math.sqrt(D),
                        backward=False)

    if name == "video":
        sd = 4 if seed is None else seed
        H, D = 40, 128
        grid = (21, 45, 80)
        if small:
            H, grid = 3, (3, 9, 20)
        Sq = grid[0] * grid[1] * grid[2]
        Skv = -(-Sq // 2048) * 2048
        g = gen_for(sd)
        std = math.sqrt(0.5)
        q = _rope_3axis(_normal((1, Sq, H, D), g, dev, std), grid)
        k_real = _rope_3axis(_normal((1, Sq, H, D), g, dev, std), grid)
        k_real[:, 0:8, 0, :] *= 20.0  # the sink keys of head 0
        k_pad = _normal((1, Skv - Sq, H, D), g, dev, 100.0)
        k = torch.cat([k_real, k_pad], dim=1)
        v = _normal((1, Skv, H, D), g, dev)
        mask = {"kv_valid_len": np.asarray([Sq], dtype=np.int32)}
        return Workload(name, 1, H, Sq, Skv, D, q.to(bf16), k.to(bf16), v.to(bf16), None,
                        mask, 1.0 / math.sqrt(D), backward=False)

    raise ValueError(f"unknown workload {name!r}")
