"""Pins for the fp64 oracle: checks against facts that do not come from the
oracle itself.  Each pin takes ``plant`` (0 = the faithful oracle build, n > 0 =
a build with planted mistake n) and returns True when the oracle passes.

Kinds of pin used here:
  * the page's own example facts (tests/golden/*.json, each with its source);
  * a library special case: torch's CPU ``scaled_dot_product_attention`` in
    fp64, which "Core 注意力" (section "选择最窄的入口") says the entry follows;
  * an independent pure-Python per-element loop (oracle/brute.py);
  * closed forms: with q = 0 every score is equal, so the output is the mean of
    the visible V rows (a running mean under a causal mask, restarting at each
    packed sequence, taken per kv group);
  * invariants: -inf additive == false keep, all-true keep == no mask, a per-row
    constant added to the scores changes nothing, key order does not matter.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch
import torch.nn.functional as F

import oracle
from oracle import brute

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _close(a, b, tol=1e-10):
    a, b = np.asarray(a, dtype=np.float64), np.asarray(b, dtype=np.float64)
    return a.shape == b.shape and bool(np.all(np.abs(a - b) <= tol * (1 + np.abs(b))))


def _rng(seed):
    g = torch.Generator().manual_seed(seed)
    return g


def _randn(g, *shape):
    return torch.randn(*shape, generator=g, dtype=torch.float64)


def _torch_ref(q, k, v, scale, mask=None):
    """torch fp64 SDPA with GQA expansion by repeat_interleave."""
    group = q.shape[1] // k.shape[1]
    k = k.repeat_interleave(group, dim=1)
    v = v.repeat_interleave(group, dim=1)
    return F.scaled_dot_product_attention(q, k, v, attn_mask=mask, dropout_p=0.0, scale=scale)


# --------------------------------------------------------------------------- pins

def pin_page_example_shape(plant=0):
    """'Core 注意力' example: seed 7, q/k/v randn in order, output (2,8,32,96)."""
    gd = golden("page_example.json")
    torch.manual_seed(gd["seed"])
    q = torch.randn(*gd["q_shape"])
    k = torch.randn(*gd["k_shape"])
    v = torch.randn(*gd["v_shape"])
    out = oracle.sdpa(q, k, v, qk_scale=1 / math.sqrt(gd["q_shape"][-1]), plant=plant)
    return list(out.shape) == gd["out_shape"]


def pin_torch_no_mask(plant=0):
    g = _rng(11)
    q, k, v = _randn(g, 2, 4, 13, 16), _randn(g, 2, 4, 21, 16), _randn(g, 2, 4, 21, 24)
    ref = _torch_ref(q, k, v, 0.3)
    return _close(oracle.sdpa(q, k, v, qk_scale=0.3, plant=plant), ref.numpy())


def pin_torch_gqa(plant=0):
    g = _rng(12)
    q, k, v = _randn(g, 2, 6, 9, 8), _randn(g, 2, 2, 11, 8), _randn(g, 2, 2, 11, 5)
    ref = _torch_ref(q, k, v, 0.5)
    return _close(oracle.sdpa(q, k, v, qk_scale=0.5, plant=plant), ref.numpy())


def pin_torch_keep_mask(plant=0):
    g = _rng(13)
    q, k, v = _randn(g, 2, 4, 10, 8), _randn(g, 2, 2, 12, 8), _randn(g, 2, 2, 12, 8)
    keep = torch.rand(2, 4, 10, 12, generator=g) < 0.6
    keep[..., 3] = True          # every row keeps a key: torch gives NaN otherwise
    ref = _torch_ref(q, k, v, 0.7, keep)
    return _close(oracle.sdpa(q, k, v, mask=keep, mask_kind="keep", qk_scale=0.7, plant=plant),
                  ref.numpy())


def pin_torch_additive_mask(plant=0):
    g = _rng(14)
    q, k, v = _randn(g, 1, 4, 7, 8), _randn(g, 1, 4, 9, 8), _randn(g, 1, 4, 9, 6)
    add = _randn(g, 1, 1, 7, 9) * 2.0      # broadcast over heads
    ref = _torch_ref(q, k, v, 0.4, add)
    return _close(oracle.sdpa(q, k, v, mask=add, mask_kind="add", qk_scale=0.4, plant=plant),
                  ref.numpy())


def pin_torch_causal_square(plant=0):
    g = _rng(15)
    q, k, v = _randn(g, 2, 2, 17, 8), _randn(g, 2, 2, 17, 8), _randn(g, 2, 2, 17, 8)
    ref = F.scaled_dot_product_attention(q, k, v, is_causal=True, scale=0.35)
    return _close(oracle.sdpa(q, k, v, mask_kind="causal", qk_scale=0.35, plant=plant), ref.numpy())


def pin_torch_causal_bottom_right(plant=0):
    """Lq < Lk: query i sees keys j <= i + (Lk - Lq) (bottom-right reading)."""
    g = _rng(16)
    lq, lk = 6, 15
    q, k, v = _randn(g, 1, 2, lq, 8), _randn(g, 1, 2, lk, 8), _randn(g, 1, 2, lk, 8)
    keep = torch.ones(lq, lk, dtype=torch.bool).tril(diagonal=lk - lq)
    ref = _torch_ref(q, k, v, 0.5, keep)
    return _close(oracle.sdpa(q, k, v, mask_kind="causal", qk_scale=0.5, plant=plant), ref.numpy())


def pin_torch_mla_concat(plant=0):
    """MLA split contraction == one contraction over the concatenated [q, qRope]."""
    g = _rng(17)
    T, H, D, R = 12, 3, 16, 8
    q, qr = _randn(g, T, H, D), _randn(g, T, H, R)
    k, kr, v = _randn(g, T, H, D), _randn(g, T, H, R), _randn(g, T, H, D)
    lens = torch.tensor([5, 7], dtype=torch.int32)
    scale = 1 / math.sqrt(D + R)
    out = oracle.sdpa(q, k, v, qrope=qr, krope=kr, q_seqlen=lens, kv_seqlen=lens,
                      mask_kind="causal", qk_scale=scale, plant=plant)
    ok = True
    start = 0
    for L in lens.tolist():
        sl = slice(start, start + L)
        qq = torch.cat([q[sl], qr[sl]], -1).transpose(0, 1)[None]
        kk = torch.cat([k[sl], kr[sl]], -1).transpose(0, 1)[None]
        vv = v[sl].transpose(0, 1)[None]
        ref = F.scaled_dot_product_attention(qq, kk, vv, is_causal=True, scale=scale)
        ok &= _close(out[sl], ref[0].transpose(0, 1).numpy())
        start += L
    return ok


def pin_brute_dense(plant=0):
    g = _rng(18)
    q, k, v = _randn(g, 1, 4, 5, 4), _randn(g, 1, 2, 7, 4), _randn(g, 1, 2, 7, 3)
    qr, kr = _randn(g, 1, 4, 5, 2), _randn(g, 1, 2, 7, 2)
    keep = torch.rand(1, 4, 5, 7, generator=g) < 0.5
    add = _randn(g, 1, 4, 5, 7)
    ok = True
    for kind, m in (("none", None), ("causal", None), ("keep", keep), ("add", add)):
        ref = brute.sdpa_dense(q, k, v, scale=0.6, mask=m, mask_kind=kind, qrope=qr, krope=kr)
        got = oracle.sdpa(q, k, v, qrope=qr, krope=kr, mask=m, mask_kind=kind, qk_scale=0.6,
                          plant=plant)
        ok &= _close(got, ref)
    return ok


def pin_brute_packed(plant=0):
    g = _rng(19)
    ql = torch.tensor([3, 1, 4], dtype=torch.int32)
    kl = torch.tensor([5, 2, 4], dtype=torch.int32)
    q, qr = _randn(g, 8, 4, 4), _randn(g, 8, 4, 2)
    k, kr, v = _randn(g, 11, 2, 4), _randn(g, 11, 2, 2), _randn(g, 11, 2, 3)
    ok = True
    for causal in (False, True):
        ref = brute.sdpa_packed(q, k, v, ql, kl, scale=0.8, causal=causal, qrope=qr, krope=kr)
        got = oracle.sdpa(q, k, v, qrope=qr, krope=kr, q_seqlen=ql, kv_seqlen=kl,
                          mask_kind="causal" if causal else "none", qk_scale=0.8, plant=plant)
        ok &= _close(got, ref)
    return ok


def pin_uniform_closed_form(plant=0):
    """q = 0: every score equal, out = mean of the visible V rows of the head's
    kv group; causal -> running mean; packed -> restarts per sequence."""
    g = _rng(20)
    ok = True
    # dense, GQA 6 -> 3 with a distinct V per kv head, causal and not
    lk = 9
    v = _randn(g, 1, 3, lk, 4)
    k = _randn(g, 1, 3, lk, 4)
    q = torch.zeros(1, 6, lk, 4, dtype=torch.float64)
    out = oracle.sdpa(q, k, v, qk_scale=1.0, plant=plant)
    for h in range(6):
        ok &= _close(out[0, h], np.broadcast_to(v[0, h // 2].mean(0).numpy(), (lk, 4)))
    out = oracle.sdpa(q, k, v, mask_kind="causal", qk_scale=1.0, plant=plant)
    run = np.cumsum(v.numpy(), axis=2) / np.arange(1, lk + 1)[None, None, :, None]
    for h in range(6):
        ok &= _close(out[0, h], run[0, h // 2])
    # causal with Lq < Lk: row i averages keys 0 .. i + Lk - Lq
    qs = torch.zeros(1, 6, 4, 4, dtype=torch.float64)
    out = oracle.sdpa(qs, k, v, mask_kind="causal", qk_scale=1.0, plant=plant)
    for h in range(6):
        ok &= _close(out[0, h], run[0, h // 2, lk - 4:])
    # packed sequences: running means restart at each sequence boundary
    lens = torch.tensor([3, 5, 1], dtype=torch.int32)
    vp = _randn(g, 9, 2, 3)
    kp = _randn(g, 9, 2, 3)
    qp = torch.zeros(9, 2, 3, dtype=torch.float64)
    out = oracle.sdpa(qp, kp, vp, q_seqlen=lens, kv_seqlen=lens, mask_kind="causal",
                      qk_scale=1.0, plant=plant)
    start = 0
    for L in lens.tolist():
        seg = vp[start:start + L].numpy()
        ok &= _close(out[start:start + L], np.cumsum(seg, 0) / np.arange(1, L + 1)[:, None, None])
        start += L
    return ok


def pin_mask_invariants(plant=0):
    g = _rng(21)
    q, k, v = _randn(g, 1, 2, 6, 8), _randn(g, 1, 2, 10, 8), _randn(g, 1, 2, 10, 8)
    keep = torch.rand(1, 2, 6, 10, generator=g) < 0.5
    keep[..., 0] = True
    ok = True
    # -inf additive == false keep
    add = torch.where(keep, torch.zeros(()), torch.full((), -math.inf)).double()
    a = oracle.sdpa(q, k, v, mask=add, mask_kind="add", qk_scale=0.5, plant=plant)
    b = oracle.sdpa(q, k, v, mask=keep, mask_kind="keep", qk_scale=0.5, plant=plant)
    ok &= _close(a, b)
    # all-true keep == no mask
    a = oracle.sdpa(q, k, v, mask=torch.ones(1, 1, 6, 10, dtype=torch.bool), mask_kind="keep",
                    qk_scale=0.5, plant=plant)
    b = oracle.sdpa(q, k, v, qk_scale=0.5, plant=plant)
    ok &= _close(a, b)
    # a per-row constant in the additive mask changes nothing
    base = _randn(g, 1, 2, 6, 10)
    shift = _randn(g, 1, 2, 6, 1) * 5
    a = oracle.sdpa(q, k, v, mask=base, mask_kind="add", qk_scale=0.5, plant=plant)
    b = oracle.sdpa(q, k, v, mask=base + shift, mask_kind="add", qk_scale=0.5, plant=plant)
    ok &= _close(a, b, 1e-9)
    # key order does not matter without a causal mask
    perm = torch.randperm(10, generator=g)
    a = oracle.sdpa(q, k, v, qk_scale=0.5, plant=plant)
    b = oracle.sdpa(q, k[:, :, perm], v[:, :, perm], qk_scale=0.5, plant=plant)
    ok &= _close(a, b, 1e-9)
    # and with the mask permuted along with the keys
    a = oracle.sdpa(q, k, v, mask=keep, mask_kind="keep", qk_scale=0.5, plant=plant)
    b = oracle.sdpa(q, k[:, :, perm], v[:, :, perm], mask=keep[..., perm], mask_kind="keep",
                    qk_scale=0.5, plant=plant)
    ok &= _close(a, b, 1e-9)
    return ok


def pin_fully_masked_rows(plant=0):
    """A row with no kept key is zero and its LSE is -inf (reading of a silent case)."""
    g = _rng(22)
    q, k, v = _randn(g, 1, 1, 4, 8), _randn(g, 1, 1, 5, 8), _randn(g, 1, 1, 5, 8)
    keep = torch.ones(1, 1, 4, 5, dtype=torch.bool)
    keep[0, 0, 2] = False
    out, lse = oracle.sdpa(q, k, v, mask=keep, mask_kind="keep", qk_scale=1.0, with_lse=True,
                           plant=plant)
    ok = bool(np.all(out[0, 0, 2] == 0.0)) and lse[0, 0, 2] == -np.inf
    # causal with Lq > Lk: the first Lq - Lk rows see nothing
    qc = _randn(g, 1, 1, 7, 8)
    out = oracle.sdpa(qc, k, v, mask_kind="causal", qk_scale=1.0, plant=plant)
    ok &= bool(np.all(out[0, 0, :2] == 0.0)) and bool(np.all(out[0, 0, 2:] != 0.0))
    return ok


def pin_lse(plant=0):
    g = _rng(23)
    q, k, v = _randn(g, 1, 2, 5, 8), _randn(g, 1, 2, 9, 8), _randn(g, 1, 2, 9, 8)
    _, lse = oracle.sdpa(q, k, v, qk_scale=0.25, with_lse=True, plant=plant)
    ref = torch.logsumexp(q @ k.transpose(-1, -2) * 0.25, dim=-1).numpy()
    return _close(lse, ref)


PINS = [pin_page_example_shape, pin_torch_no_mask, pin_torch_gqa, pin_torch_keep_mask,
        pin_torch_additive_mask, pin_torch_causal_square, pin_torch_causal_bottom_right,
        pin_torch_mla_concat, pin_brute_dense, pin_brute_packed, pin_uniform_closed_form,
        pin_mask_invariants, pin_fully_masked_rows, pin_lse]

# ------------------------------------------------------------- merge pins
# Each takes ``plant`` = a key of oracle.MERGE_PLANTS (0 = faithful merge).

def _torch_lse(q, k, scale, mask=None):
    group = q.shape[1] // k.shape[1]
    s = q @ k.repeat_interleave(group, dim=1).transpose(-1, -2) * scale
    if mask is not None:
        s = s.masked_fill(~mask, -math.inf)
    return torch.logsumexp(s, dim=-1)


def pin_merge_random_key_sets(plant=0):
    """Keys dealt at random into three disjoint sets (keep-masks); merging the
    three partial results gives torch's attention and logsumexp over all keys."""
    g = _rng(40)
    q, k, v = _randn(g, 2, 4, 9, 8), _randn(g, 2, 2, 13, 8), _randn(g, 2, 2, 13, 5)
    owner = torch.randint(0, 3, (13,), generator=g)
    outs, lses = [], []
    for s_ in range(3):
        keep = (owner == s_).view(1, 1, 1, 13).expand(2, 4, 9, 13).to(torch.uint8)
        o, l = oracle.sdpa(q, k, v, mask=keep, mask_kind="keep", qk_scale=0.3, with_lse=True)
        outs.append(o)
        lses.append(l)
    out, lse = oracle.merge(np.stack(outs), np.stack(lses), plant=plant)
    return _close(out, _torch_ref(q, k, v, 0.3).numpy()) and _close(lse, _torch_lse(q, k, 0.3).numpy())


def pin_merge_causal_halves(plant=0):
    """Causal rows split at key 5: rows 0..4 have nothing in the second half
    (lse -inf, weight 0); the merge equals torch's causal attention."""
    g = _rng(41)
    q, k, v = _randn(g, 1, 2, 10, 8), _randn(g, 1, 2, 10, 8), _randn(g, 1, 2, 10, 6)
    tril = torch.ones(10, 10, dtype=torch.bool).tril()
    j = torch.arange(10)
    outs, lses = [], []
    for half in (j < 5, j >= 5):
        keep = (tril & half.view(1, 10)).view(1, 1, 10, 10).expand(1, 2, 10, 10).to(torch.uint8)
        o, l = oracle.sdpa(q, k, v, mask=keep, mask_kind="keep", qk_scale=0.5, with_lse=True)
        outs.append(o)
        lses.append(l)
    ok = bool(np.all(lses[1][0, :, :5] == -np.inf))
    out, lse = oracle.merge(np.stack(outs), np.stack(lses), plant=plant)
    ref = _torch_ref(q, k, v, 0.5, mask=tril).numpy()
    return ok and _close(out, ref) and _close(lse, _torch_lse(q, k, 0.5, tril).numpy())


def pin_merge_closed_forms(plant=0):
    """Equal lse: the mean of the parts and lse + ln 2.  One part at -inf: the
    other part unchanged.  All parts at -inf: zero and -inf."""
    a = np.array([[1.0, -2.0, 4.0]])
    b = np.array([[3.0, 0.0, -4.0]])
    out, lse = oracle.merge(np.stack([a, b]), np.array([[0.7], [0.7]]), plant=plant)
    ok = _close(out, (a + b) / 2) and _close(lse, [0.7 + math.log(2.0)])
    out, lse = oracle.merge(np.stack([a, b]), np.array([[-np.inf], [1.5]]), plant=plant)
    ok &= _close(out, b) and _close(lse, [1.5])
    out, lse = oracle.merge(np.stack([a, b]), np.array([[-np.inf], [-np.inf]]), plant=plant)
    ok &= bool(np.all(out == 0.0)) and lse[0] == -np.inf
    return ok


MERGE_PINS = [pin_merge_random_key_sets, pin_merge_causal_halves, pin_merge_closed_forms]


# --------------------------------------------------------------- DCA pins

def pin_dca_equal_queries_is_causal_attention(plant=0):
    """All three query forms equal: plain causal attention (torch, GQA)."""
    g = _rng(60)
    q, k, v = _randn(g, 1, 4, 21, 8), _randn(g, 1, 2, 21, 8), _randn(g, 1, 2, 21, 5)
    out = oracle.dca(q, q, q, k, v, chunk=4, qk_scale=0.4, plant=plant)
    tril = torch.ones(21, 21, dtype=torch.bool).tril()
    return _close(out, _torch_ref(q, k, v, 0.4, mask=tril).numpy())


def pin_dca_one_chunk_is_intra_only(plant=0):
    """A chunk at least the sequence long: only the intra-chunk form is used."""
    g = _rng(61)
    qi, qs, qe = _randn(g, 1, 2, 9, 8), _randn(g, 1, 2, 9, 8), _randn(g, 1, 2, 9, 8)
    k, v = _randn(g, 1, 2, 9, 8), _randn(g, 1, 2, 9, 6)
    out = oracle.dca(qi, qs, qe, k, v, chunk=9, qk_scale=0.3, plant=plant)
    tril = torch.ones(9, 9, dtype=torch.bool).tril()
    return _close(out, _torch_ref(qi, k, v, 0.3, mask=tril).numpy())


def pin_dca_brute_force(plant=0):
    """Independent per-element loop: the query form picked key by key."""
    g = _rng(62)
    qi, qs, qe = _randn(g, 1, 2, 11, 3), _randn(g, 1, 2, 11, 3), _randn(g, 1, 2, 11, 3)
    k, v = _randn(g, 1, 1, 11, 3), _randn(g, 1, 1, 11, 2)
    out = oracle.dca(qi, qs, qe, k, v, chunk=3, qk_scale=0.7, plant=plant)
    ref = np.zeros_like(out)
    for h in range(2):
        for i in range(11):
            w = []
            for j in range(i + 1):
                d = i // 3 - j // 3
                qq = qi if d == 0 else (qs if d == 1 else qe)
                w.append(math.exp(0.7 * sum(float(qq[0, h, i, t]) * float(k[0, 0, j, t]) for t in range(3))))
            tot = sum(w)
            for c in range(2):
                ref[0, h, i, c] = sum(w[j] * float(v[0, 0, j, c]) for j in range(i + 1)) / tot
    return _close(out, ref)


DCA_PINS = [pin_dca_equal_queries_is_causal_attention, pin_dca_one_chunk_is_intra_only,
            pin_dca_brute_force]

# Planted mistakes compiled into copies of the oracle (ORACLE_PLANT=n).
PLANTS = {
    1: "GQA group index h % kvHeadNum instead of h / (headNum / kvHeadNum)",
    2: "causal aligned top-left instead of bottom-right",
    3: "rope term dropped from the MLA contraction",
    4: "keep-mask polarity flipped",
    5: "additive mask applied before the qkScale multiplication",
    6: "sign flipped in the softmax exponent",
    7: "masked keys counted in the softmax normaliser",
}
