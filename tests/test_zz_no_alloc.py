"""The allocation-free packed-sequence entry point.

wf_attn_fwd_varlen_noalloc is for callers that cannot allocate device memory
while they run (graph-captured work that must leave the allocator alone,
runtimes that own the whole device through a pool, fixed budgets): it keeps
the packed-sequence schedule in a fixed array inside the library instead of
a cudaMalloc'd workspace.  Checked against the regular entry point (two calls
in a row) and against the fp64 oracle element by element (ragged lengths,
both causal alignments and no mask, the MLA rope part); that a call on a
fresh stream leaves the device's free memory unchanged while the regular
entry point's first call on a fresh stream does not; and its rejections.
This file is named so that pytest collects it last."""
import ctypes
import math

import pytest
import torch

import oracle
from attention_forward_tmem_b200 import _lib as L
from attention_forward_tmem_b200 import api
from attention_forward_tmem_b200 import workloads as W
from tests.gpu_helpers import MAX_ABS, compare

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _noalloc(q, k, v, ql, kl, *, qrope=None, krope=None, causal=True, scale, out,
             mask_type=None, stream=None):
    d = [api.describe(x) for x in (q, qrope, k, krope, v, ql, kl)]
    r = lambda x: ctypes.byref(x) if x is not None else None  # noqa: E731
    od = api.describe(out)
    mt = mask_type if mask_type is not None else (L.WF_MASK_CAUSAL if causal else L.WF_MASK_NONE)
    stream = stream or torch.cuda.current_stream()
    st = L.load().wf_attn_fwd_varlen_noalloc(*[r(x) for x in d], q.shape[1], k.shape[1],
                                             float(scale), int(mt), ctypes.byref(od),
                                             stream.cuda_stream)
    return st


def _case(lens_q, lens_k, hq, hk, drope, seed):
    ql = torch.tensor(lens_q, dtype=torch.int32)
    kl = torch.tensor(lens_k, dtype=torch.int32)
    d = W.packed_inputs(ql, kl, hq, hk, 128, 128, drope, torch.bfloat16, seed)
    g = {n: t.to(DEV) for n, t in d.items()}
    return g, ql.to(DEV), kl.to(DEV), 1 / math.sqrt(128 + drope)


def test_noalloc_matches_wf_attn_fwd_twice():
    cases = [_case([1, 127, 128, 129, 300, 5], [1, 127, 128, 129, 300, 5], 4, 2, 0, 3),
             _case([200, 7, 385], [260, 90, 385], 4, 4, 64, 4)]
    for g, ql, kl, s in cases:               # two calls in a row, different shapes
        ref = api.attn_fwd(g["q"], g["k"], g["v"], qrope=g.get("qrope"), krope=g.get("krope"),
                           q_seqlen=ql, kv_seqlen=kl, mask_type=api.MaskType.CAUSAL, qk_scale=s)
        out = torch.full_like(ref, float("nan"))
        st = _noalloc(g["q"], g["k"], g["v"], ql, kl, qrope=g.get("qrope"), krope=g.get("krope"),
                      scale=s, out=out)
        assert st == L.WF_OK, L.load().wf_last_error_message()
        api.device_status()
        assert torch.isfinite(out).all()
        err = (out.float() - ref.float()).abs().max().item()
        assert err <= MAX_ABS[torch.bfloat16], err


def test_noalloc_rejects_oversize_schedule():
    g, ql, kl, s = _case([4] * 30000, [4] * 30000, 1, 1, 0, 5)
    out = torch.empty_like(g["q"])
    st = _noalloc(g["q"], g["k"], g["v"], ql, kl, scale=s, out=out)
    assert st == L.WF_ERR_INVALID_ARG
    assert b"at most" in L.load().wf_last_error_message()


ORACLE_CASES = [
    # qlens, klens, Hq, Hk, drope, mask type, oracle mask kind
    ([1, 127, 128, 129, 300, 5], [1, 127, 128, 129, 300, 5], 4, 2, 0, L.WF_MASK_NONE, "none"),
    ([200, 0, 385, 7], [260, 90, 385, 7], 4, 4, 64, L.WF_MASK_CAUSAL, "causal"),
    ([300, 129, 1], [130, 400, 3], 4, 1, 0, L.WF_MASK_CAUSAL_TOP_LEFT, "top_left"),
]


def _oracle_packed(d, ql, kl, hq, s, kind):
    if kind != "top_left":
        return oracle.sdpa(d["q"], d["k"], d["v"], qrope=d.get("qrope"), krope=d.get("krope"),
                           q_seqlen=ql, kv_seqlen=kl, mask_kind=kind, qk_scale=s)
    # top-left causal: per sequence, the dense oracle with the keep-mask j <= i
    import numpy as np
    qls, kls = ql.tolist(), kl.tolist()
    cq = np.concatenate([[0], np.cumsum(qls)])
    ck = np.concatenate([[0], np.cumsum(kls)])
    ref = np.zeros((cq[-1], hq, d["v"].shape[-1]))
    for b, (lq, lk) in enumerate(zip(qls, kls)):
        if lq == 0:
            continue
        f = lambda t, lo, hi: t[lo:hi].permute(1, 0, 2).unsqueeze(0)  # noqa: E731
        keep = torch.ones(lq, lk, dtype=torch.bool).tril().expand(1, hq, lq, lk)
        r = oracle.sdpa(f(d["q"], cq[b], cq[b + 1]), f(d["k"], ck[b], ck[b + 1]),
                        f(d["v"], ck[b], ck[b + 1]), mask=keep, mask_kind="keep", qk_scale=s)
        ref[cq[b]:cq[b + 1]] = r[0].transpose(1, 0, 2)
    return ref


def test_noalloc_matches_oracle():
    """Element by element against the fp64 oracle, three calls in a row."""
    for i, (qls, kls, hq, hk, drope, mt, kind) in enumerate(ORACLE_CASES):
        ql = torch.tensor(qls, dtype=torch.int32)
        kl = torch.tensor(kls, dtype=torch.int32)
        d = W.packed_inputs(ql, kl, hq, hk, 128, 128, drope, torch.bfloat16, 20 + i)
        g = {n: t.to(DEV) for n, t in d.items()}
        s = 1 / math.sqrt(128 + drope)
        out = torch.full((g["q"].shape[0], hq, 128), float("nan"), dtype=torch.bfloat16, device=DEV)
        st = _noalloc(g["q"], g["k"], g["v"], ql.to(DEV), kl.to(DEV), qrope=g.get("qrope"),
                      krope=g.get("krope"), scale=s, out=out, mask_type=mt)
        assert st == L.WF_OK, L.load().wf_last_error_message()
        api.device_status()
        compare(out, _oracle_packed(d, ql, kl, hq, s, kind), torch.bfloat16, f"noalloc {kind}")


def test_noalloc_allocates_nothing():
    """After a first call (which loads the kernels), a call on a stream the
    library has never seen leaves the device's free memory unchanged; the
    regular entry point's first call on a fresh stream does not (it creates
    that stream's workspace), which shows the check can see an allocation."""
    g, ql, kl, s = _case([100, 300], [100, 300], 2, 1, 0, 6)
    out = torch.empty(g["q"].shape[0], 2, 128, dtype=torch.bfloat16, device=DEV)
    assert _noalloc(g["q"], g["k"], g["v"], ql, kl, scale=s, out=out) == L.WF_OK
    torch.cuda.synchronize()
    fresh, control = torch.cuda.Stream(), torch.cuda.Stream()
    torch.cuda.synchronize()
    before = torch.cuda.mem_get_info()[0]
    assert _noalloc(g["q"], g["k"], g["v"], ql, kl, scale=s, out=out, stream=fresh) == L.WF_OK
    torch.cuda.synchronize()
    after = torch.cuda.mem_get_info()[0]
    api.device_status()
    assert after == before, (before, after)
    with torch.cuda.stream(control):
        api.attn_fwd(g["q"], g["k"], g["v"], q_seqlen=ql, kv_seqlen=kl,
                     mask_type=api.MaskType.CAUSAL, qk_scale=s, out=out)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] < after


def test_noalloc_rejects_other_dtypes_and_layouts():
    g, ql, kl, s = _case([64, 64], [64, 64], 2, 2, 0, 7)
    h = {n: t.half() for n, t in g.items()}
    out16 = torch.empty_like(h["q"])
    assert _noalloc(h["q"], h["k"], h["v"], ql, kl, scale=s, out=out16) == L.WF_ERR_UNSUPPORTED
    qd, kd, vd = (t.to(DEV) for t in W.dense_inputs(1, 2, 2, 64, 64, 128, 128, torch.bfloat16, 8))
    outd = torch.empty_like(qd)
    assert _noalloc(qd, kd, vd, ql, kl, scale=s, out=outd) == L.WF_ERR_INVALID_ARG
    out = torch.empty_like(g["q"])
    assert _noalloc(g["q"], g["k"], g["v"], ql, kl, scale=s, out=out,
                    mask_type=L.WF_MASK_BOOL_KEEP) == L.WF_ERR_UNSUPPORTED
