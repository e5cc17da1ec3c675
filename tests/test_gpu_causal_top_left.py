"""The top-left causal kind (WF_MASK_CAUSAL_TOP_LEFT: key j visible to query i
iff j <= i, the alignment of PyTorch SDPA's is_causal, "Core 注意力" section
"选择最窄的入口"), generated in the kernel, against the fp64 oracle given the
same predicate as an explicit keep-mask.  Lengths differ (Lq < Lk and Lq > Lk),
where the two causal alignments disagree; dense and packed layouts, GQA, the
MLA rope part, fp32 and the split-KV path."""
import math

import numpy as np
import pytest
import torch

import oracle
from attention_forward_tmem_b200 import api
from attention_forward_tmem_b200 import workloads as W
from tests.gpu_helpers import compare

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _tril(lq, lk):
    return torch.ones(lq, lk, dtype=torch.bool).tril()


@pytest.mark.parametrize("cfg", [
    # B, Hq, Hk, Lq, Lk, D, dtype
    (1, 4, 2, 200, 333, 128, torch.bfloat16),
    (2, 4, 1, 333, 200, 128, torch.bfloat16),
    (1, 2, 2, 129, 700, 64, torch.bfloat16),
    (1, 2, 1, 100, 150, 128, torch.float32),
    (1, 2, 2, 150, 60, 96, torch.float32),
], ids=lambda c: "x".join(str(x) for x in c[:6]) + ("-f32" if c[6] == torch.float32 else "-bf16"))
def test_dense_top_left(cfg):
    B, Hq, Hk, Lq, Lk, D, dtype = cfg
    q, k, v = W.dense_inputs(B, Hq, Hk, Lq, Lk, D, D, dtype, 61)
    s = 1.0 / math.sqrt(D)
    out = api.attn_fwd(q.to(DEV), k.to(DEV), v.to(DEV), mask_type=api.MaskType.CAUSAL_TOP_LEFT,
                       qk_scale=s)
    api.device_status()
    ref = oracle.sdpa(q, k, v, mask=_tril(Lq, Lk).expand(B, Hq, Lq, Lk), mask_kind="keep", qk_scale=s)
    compare(out, ref, dtype, f"top-left {cfg}")


def test_dense_top_left_split_kv_and_lse():
    """Few query rows over many keys: the automatic split-KV path and the LSE."""
    B, H, Lq, Lk, D = 1, 2, 200, 3000, 128
    q, k, v = W.dense_inputs(B, H, H, Lq, Lk, D, D, torch.bfloat16, 62)
    s = 1.0 / math.sqrt(D)
    out, lse = api.attn_fwd(q.to(DEV), k.to(DEV), v.to(DEV), mask_type=api.MaskType.CAUSAL_TOP_LEFT,
                            qk_scale=s, return_lse=True)
    api.device_status()
    keep = _tril(Lq, Lk).expand(B, H, Lq, Lk)
    ref = oracle.sdpa(q, k, v, mask=keep, mask_kind="keep", qk_scale=s)
    compare(out, ref, torch.bfloat16, "top-left split")
    # LSE of row i: logsumexp of its visible scaled scores (keys 0..i)
    qf, kf = q.double(), k.double()
    sc = torch.einsum("bhid,bhjd->bhij", qf, kf) * s
    sc = sc.masked_fill(~keep, float("-inf"))
    want = torch.logsumexp(sc, dim=-1).numpy()
    got = lse.cpu().double().numpy()
    assert np.abs(got - want).max() <= 1e-3


@pytest.mark.parametrize("drope", [0, 64])
def test_packed_top_left(drope):
    qlens = [1, 127, 300, 129, 40]
    klens = [5, 300, 130, 129, 0]
    Hq, Hk, D = 4, 2 if drope == 0 else 4, 128
    ql = torch.tensor(qlens, dtype=torch.int32)
    kl = torch.tensor(klens, dtype=torch.int32)
    d = W.packed_inputs(ql, kl, Hq, Hk, D, D, drope, torch.bfloat16, 63)
    s = 1.0 / math.sqrt(D + drope)
    g = {kk: vv.to(DEV) for kk, vv in d.items()}
    out = api.attn_fwd(g["q"], g["k"], g["v"], qrope=g.get("qrope"), krope=g.get("krope"),
                       q_seqlen=ql.to(DEV), kv_seqlen=kl.to(DEV),
                       mask_type=api.MaskType.CAUSAL_TOP_LEFT, qk_scale=s)
    api.device_status()
    # per sequence: the dense oracle with the top-left keep-mask
    cq = np.concatenate([[0], np.cumsum(qlens)])
    ck = np.concatenate([[0], np.cumsum(klens)])
    ref = np.zeros((cq[-1], Hq, D))
    for b, (lq, lk) in enumerate(zip(qlens, klens)):
        if lq == 0:
            continue
        sl_q, sl_k = slice(cq[b], cq[b + 1]), slice(ck[b], ck[b + 1])
        dq = lambda t, sl: t[sl].permute(1, 0, 2).unsqueeze(0)  # noqa: E731  [T,H,D] -> [1,H,T,D]
        qr = dq(d["qrope"], sl_q) if drope else None
        kr = dq(d["krope"], sl_k) if drope else None
        r = oracle.sdpa(dq(d["q"], sl_q), dq(d["k"], sl_k), dq(d["v"], sl_k), qrope=qr, krope=kr,
                        mask=_tril(lq, lk).expand(1, Hq, lq, lk), mask_kind="keep", qk_scale=s)
        ref[sl_q] = r[0].transpose(1, 0, 2)
    compare(out, ref, torch.bfloat16, f"packed top-left rope={drope}")


def test_square_top_left_equals_causal():
    """Lq == Lk: both alignments are the same mask, and the same kernel path."""
    q, k, v = W.dense_inputs(1, 4, 2, 300, 300, 128, 128, torch.bfloat16, 64)
    a = api.attn_fwd(q.to(DEV), k.to(DEV), v.to(DEV), mask_type=api.MaskType.CAUSAL_TOP_LEFT)
    b = api.attn_fwd(q.to(DEV), k.to(DEV), v.to(DEV), mask_type=api.MaskType.CAUSAL)
    api.device_status()
    assert torch.equal(a, b)
