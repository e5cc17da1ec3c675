"""Dual chunk attention (the skeleton's reading) -- fp64, row by row.

TEST INFRASTRUCTURE ONLY (see the package docstring).

The "Dual Chunk Attention" article gives no formulas; it describes splitting
a long sequence into chunks and attending within a chunk, to the neighbouring
chunk and across chunks with remapped relative positions.  The reading taken
here keeps the structure and leaves the position remapping to the caller:
the sequence is cut into chunks of `chunk` positions, and every query comes in
three forms, already rotated for the three position maps.  Query i (chunk
c_i = i // chunk) attends causally to keys j <= i, scoring key j with

    q_intra[i] . k[j]   if c_j == c_i        (same chunk)
    q_succ[i]  . k[j]   if c_j == c_i - 1    (successive chunk)
    q_inter[i] . k[j]   if c_j <  c_i - 1    (earlier chunks)

times qk_scale, and one softmax over all of them.  GQA as in the forward
(kv head = h / (H / Hkv)).
"""
from __future__ import annotations

import numpy as np


def _f64(x):
    if hasattr(x, "detach"):
        x = x.detach().cpu().double().numpy()       # exact widening of bf16 / fp16 / fp32
    return np.asarray(x, dtype=np.float64)


# Planted mistakes for the pin tests (0 = faithful).
DCA_PLANTS = {
    1: "successive-chunk and inter-chunk query forms swapped",
    2: "whole own chunk visible (no causal cut inside the chunk)",
}


def dca(q_intra, q_succ, q_inter, k, v, chunk: int, qk_scale: float, with_lse: bool = False,
        plant: int = 0):
    """q_*: [B, H, L, D], k: [B, Hkv, L, D], v: [B, Hkv, L, Dv] -> out [B, H, L, Dv]."""
    qi, qs, qe = _f64(q_intra), _f64(q_succ), _f64(q_inter)
    kk, vv = _f64(k), _f64(v)
    B, H, L, _ = qi.shape
    Hk = kk.shape[1]
    G = H // Hk
    out = np.zeros((B, H, L, vv.shape[-1]))
    lse = np.full((B, H, L), -np.inf)
    cj = np.arange(L) // chunk
    for b in range(B):
        for h in range(H):
            kh, vh = kk[b, h // G], vv[b, h // G]
            s_intra = qi[b, h] @ kh.T                  # [L, L]
            s_succ = qs[b, h] @ kh.T
            s_inter = qe[b, h] @ kh.T
            for i in range(L):
                ci = i // chunk
                js = np.arange(min(L, (ci + 1) * chunk) if plant == 2 else i + 1)
                rel = ci - cj[js]
                near, far = (s_inter, s_succ) if plant == 1 else (s_succ, s_inter)
                s = np.where(rel == 0, s_intra[i, js], np.where(rel == 1, near[i, js], far[i, js]))
                s = s * qk_scale
                m = s.max()
                p = np.exp(s - m)
                out[b, h, i] = p @ vh[js] / p.sum()
                lse[b, h, i] = m + np.log(p.sum())
    return (out, lse) if with_lse else out
