"""Pure-Python per-element attention, for tiny inputs only.

TEST INFRASTRUCTURE ONLY.  A second, independently written statement of the
attention definition (nested lists, ``math.exp``, no numpy arithmetic), used to
pin the C oracle on small shapes.  It follows the same sources:

* "Core 注意力", section "选择最窄的入口": PyTorch SDPA contract, GQA expansion.
* same page, example section (closing paragraph): bool mask = keep, float mask added.
* "MLA Prefill", parameter table: qkScale multiplies Q*K^T; q*k + qRope*kRope;
  per-sequence qSeqLen / kvSeqLen in the packed layout.

Every score is computed from scratch; the softmax is evaluated as
exp(s - max) / sum exp(s - max) over the kept keys, and a row with no kept key
is all zeros.
"""
from __future__ import annotations

import math


def _tolist(x):
    if x is None:
        return None
    if hasattr(x, "detach"):
        import torch
        x = x.detach().cpu()
        if x.dtype in (torch.bfloat16, torch.float16):
            x = x.float()
        return x.double().tolist()
    if hasattr(x, "tolist"):
        return x.tolist()
    return x


def _row_attention(qi, qri, keys, krs, vals, scale, extra, keep):
    """qi: [D]; keys: list of [D]; vals: list of [Dv]; extra/keep: per key."""
    scores = []
    for j, kj in enumerate(keys):
        dot = 0.0
        for a, b in zip(qi, kj):
            dot += a * b
        if qri is not None:
            for a, b in zip(qri, krs[j]):
                dot += a * b
        scores.append(dot * scale + extra[j])
    kept = [j for j in range(len(keys)) if keep[j]]
    dv = len(vals[0]) if vals else 0
    if not kept:
        return [0.0] * dv
    m = max(scores[j] for j in kept)
    weights = {j: math.exp(scores[j] - m) for j in kept}
    total = sum(weights.values())
    return [sum(weights[j] * vals[j][e] for j in kept) / total for e in range(dv)]


def sdpa_dense(q, k, v, *, scale, mask=None, mask_kind="none", qrope=None, krope=None):
    """q [B,Hq,Lq,D], k [B,Hkv,Lk,D], v [B,Hkv,Lk,Dv] -> nested list [B,Hq,Lq,Dv].
    ``mask`` must already have the full [B,Hq,Lq,Lk] shape."""
    q, k, v = _tolist(q), _tolist(k), _tolist(v)
    qrope, krope, mask = _tolist(qrope), _tolist(krope), _tolist(mask)
    B, Hq, Lq = len(q), len(q[0]), len(q[0][0])
    Hkv, Lk = len(k[0]), len(k[0][0])
    per_group = Hq // Hkv
    out = []
    for b in range(B):
        ob = []
        for h in range(Hq):
            g = h // per_group
            oh = []
            for i in range(Lq):
                extra = [0.0] * Lk
                keep = [True] * Lk
                for j in range(Lk):
                    if mask_kind == "causal":
                        keep[j] = j <= i + (Lk - Lq)
                    elif mask_kind == "keep":
                        keep[j] = bool(mask[b][h][i][j])
                    elif mask_kind == "add":
                        extra[j] = float(mask[b][h][i][j])
                oh.append(_row_attention(
                    q[b][h][i], None if qrope is None else qrope[b][h][i],
                    k[b][g], None if krope is None else krope[b][g],
                    v[b][g], scale, extra, keep))
            ob.append(oh)
        out.append(ob)
    return out


def sdpa_packed(q, k, v, q_seqlen, kv_seqlen, *, scale, causal=False, qrope=None, krope=None):
    """q [T,Hq,D], k [Tk,Hkv,D], v [Tk,Hkv,Dv] packed by sequence -> nested [T,Hq,Dv]."""
    q, k, v = _tolist(q), _tolist(k), _tolist(v)
    qrope, krope = _tolist(qrope), _tolist(krope)
    qs, ks = [int(x) for x in _tolist(q_seqlen)], [int(x) for x in _tolist(kv_seqlen)]
    Hq, Hkv = len(q[0]), len(k[0])
    per_group = Hq // Hkv
    out = [None] * len(q)
    q_start = k_start = 0
    for lq, lk in zip(qs, ks):
        for i in range(lq):
            row = []
            for h in range(Hq):
                g = h // per_group
                keys = [k[k_start + j][g] for j in range(lk)]
                krs = None if krope is None else [krope[k_start + j][g] for j in range(lk)]
                vals = [v[k_start + j][g] for j in range(lk)]
                keep = [(not causal) or (j <= i + (lk - lq)) for j in range(lk)]
                row.append(_row_attention(
                    q[q_start + i][h], None if qrope is None else qrope[q_start + i][h],
                    keys, krs, vals, scale, [0.0] * lk, keep))
            out[q_start + i] = row
        q_start += lq
        k_start += lk
    return out
