"""Helpers of the pins for the fp64 oracle (tests/test_oracle_pins.py; the
planted-mistake tests in tests/test_oracle_planted.py run those pins against a
deliberately broken oracle).  Nothing here re-types the oracle's formulas: every pin
compares it with something else fixed by the pages or by mathematics (a scalar
brute force, a library routine, autograd, finite differences, closed forms)."""

from __future__ import annotations

import math

import numpy as np
import torch

from oracle import MaskDesc, allowed_rows


def brute_force_forward(q, k, v, allowed, scale):
    """Scalar triple loop (tiny inputs only): O and LSE straight from the
    definition of a softmax over the allowed keys."""
    B, Sq, H, D = q.shape
    Skv = k.shape[1]
    O = np.zeros((B, Sq, H, v.shape[3]))
    L = np.zeros((B, H, Sq))
    for b in range(B):
        for h in range(H):
            for i in range(Sq):
                keys = [j for j in range(Skv) if allowed[b][i, j]]
                if not keys:
                    L[b, h, i] = -math.inf
                    continue
                s = {}
                for j in keys:
                    acc = 0.0
                    for d in range(D):
                        acc += float(q[b, i, h, d]) * float(k[b, j, h, d])
                    s[j] = scale * acc
                top = max(s.values())
                z = sum(math.exp(s[j] - top) for j in keys)
                L[b, h, i] = top + math.log(z)
                for d in range(v.shape[3]):
                    O[b, i, h, d] = sum(math.exp(s[j] - top) / z * float(v[b, j, h, d]) for j in keys)
    return O, L


def dense_allowed(mask: MaskDesc, B, Sq, Skv):
    return [allowed_rows(mask, b, np.arange(Sq), Sq, Skv) for b in range(B)]


def sdpa_forward(q, k, v, allowed, scale):
    """torch scaled_dot_product_attention in float64 (a library routine)."""
    B, Sq, H, D = q.shape
    qt = torch.from_numpy(np.ascontiguousarray(q)).permute(0, 2, 1, 3)
    kt = torch.from_numpy(np.ascontiguousarray(k)).permute(0, 2, 1, 3)
    vt = torch.from_numpy(np.ascontiguousarray(v)).permute(0, 2, 1, 3)
    m = torch.from_numpy(np.stack(allowed))[:, None, :, :]
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=m, scale=scale)
    return o.permute(0, 2, 1, 3).numpy()


def autograd_backward(q, k, v, dO, allowed, scale):
    """dQ, dK, dV by torch.autograd through the library SDPA (float64)."""
    qt = torch.from_numpy(np.ascontiguousarray(q)).permute(0, 2, 1, 3).clone().requires_grad_(True)
    kt = torch.from_numpy(np.ascontiguousarray(k)).permute(0, 2, 1, 3).clone().requires_grad_(True)
    vt = torch.from_numpy(np.ascontiguousarray(v)).permute(0, 2, 1, 3).clone().requires_grad_(True)
    m = torch.from_numpy(np.stack(allowed))[:, None, :, :]
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=m, scale=scale)
    g = torch.from_numpy(np.ascontiguousarray(dO)).permute(0, 2, 1, 3)
    (o * g).sum().backward()
    return tuple(t.grad.permute(0, 2, 1, 3).numpy() for t in (qt, kt, vt))


def finite_difference_grad(fwd, q, k, v, dO, which, idx_list, h=1e-6):
    """Central differences of sum(O * dO) w.r.t. single entries of q/k/v."""
    out = []
    for idx in idx_list:
        args = [q.copy(), k.copy(), v.copy()]
        args[which][idx] += h
        op = (fwd(*args) * dO).sum()
        args[which][idx] -= 2 * h
        om = (fwd(*args) * dO).sum()
        out.append((op - om) / (2 * h))
    return np.array(out)


def tiny_inputs(seed, B=1, Sq=9, Skv=11, H=2, D=5):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, Sq, H, D))
    k = rng.standard_normal((B, Skv, H, D))
    v = rng.standard_normal((B, Skv, H, D + 1))
    dO = rng.standard_normal((B, Sq, H, D + 1))
    return q, k, v, dO


def tiny_masks(B, Sq, Skv, seed=0):
    """A spread of mask combinations on tiny shapes (every row keeps >= 1 key
    except where a case says otherwise)."""
    rng = np.random.default_rng(seed)
    seg_q = np.sort(rng.integers(0, 3, size=(B, Sq)), axis=1)
    seg_kv = np.sort(rng.integers(0, 3, size=(B, Skv)), axis=1)
    return {
        "none": MaskDesc(),
        "causal": MaskDesc(window=0),
        "window3": MaskDesc(window=3),
        "padding": MaskDesc(kv_valid_len=np.array([Skv - 3] * B)),
        "segments": MaskDesc(seg_q=seg_q, seg_kv=seg_kv),
        "seg+window": MaskDesc(seg_q=seg_q, seg_kv=seg_kv, window=4),
        "pad+causal": MaskDesc(kv_valid_len=np.array([Skv - 2] * B), window=0),
        "prefix_lm": MaskDesc(window=0, prefix_len=np.array([3, 1] * B)[:B]),
        "dilated": MaskDesc(window=6, dilation=2),
        "doc_causal": MaskDesc(seg_q=seg_q, seg_kv=seg_kv, window=0),
    }
