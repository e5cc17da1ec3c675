"""The allocation-free packed-sequence entry point against wf_attn_fwd.

wf_attn_fwd_varlen_noalloc is for callers that cannot allocate device memory
while they run (graph-captured work that must leave the allocator alone,
runtimes that own the whole device through a pool, fixed budgets): it keeps
the packed-sequence schedule in a fixed array inside the library instead of
a cudaMalloc'd workspace.  Two calls in a row, each checked against the
regular entry point within the bf16 tolerance of the parity tests.  This file
is named so that pytest collects it last."""
import ctypes
import math

import pytest
import torch

from attention_forward_tmem_b200 import _lib as L
from attention_forward_tmem_b200 import api
from attention_forward_tmem_b200 import workloads as W
from tests.gpu_helpers import MAX_ABS

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _noalloc(q, k, v, ql, kl, *, qrope=None, krope=None, causal=True, scale, out):
    d = [api.describe(x) for x in (q, qrope, k, krope, v, ql, kl)]
    r = lambda x: ctypes.byref(x) if x is not None else None
    od = api.describe(out)
    st = L.load().wf_attn_fwd_varlen_noalloc(*[r(x) for x in d], q.shape[1], k.shape[1],
                                             float(scale), 1 if causal else 0, ctypes.byref(od),
                                             torch.cuda.current_stream().cuda_stream)
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
