"""GPU parity of the fp16 inputs and of the padded K/V layout ("MLA Prefill"
parameter table: Q/QRope/K/kRope/V are float16 or bf16; K/kRope/V may be
[batch, max_seq, kv_head * D] with packed queries) against the fp64 oracle.
The oracle is layout-free: the padded tensors are compared against the same
keys packed, gathered here on the host."""
import math

import numpy as np
import pytest
import torch

import oracle
from attention_forward_tmem_b200 import api
from attention_forward_tmem_b200 import workloads as W
from tests.gpu_helpers import compare
from tests.test_gpu_lse_split import compare_lse

pytestmark = pytest.mark.gpu
DEV = "cuda"
F16 = torch.float16


DENSE_F16 = [
    # B, Hq, Hk, Lq, Lk, D, Dv, mask
    (2, 8, 2, 300, 300, 128, 128, "causal"),
    (1, 4, 4, 200, 333, 128, 128, "causal"),
    (1, 4, 2, 129, 257, 64, 64, "none"),
    (1, 2, 2, 130, 140, 96, 96, "causal"),
    (1, 2, 1, 100, 150, 64, 128, "none"),
]


@pytest.mark.parametrize("cfg", DENSE_F16, ids=lambda c: "x".join(map(str, c)))
def test_dense_fp16(cfg):
    B, Hq, Hk, Lq, Lk, D, Dv, kind = cfg
    q, k, v = W.dense_inputs(B, Hq, Hk, Lq, Lk, D, Dv, F16, 7, 1.0)
    s = 1 / math.sqrt(D)
    mt = api.MaskType.CAUSAL if kind == "causal" else api.MaskType.NONE
    out, lse = api.attn_fwd(q.to(DEV), k.to(DEV), v.to(DEV), mask_type=mt, qk_scale=s,
                            return_lse=True)
    api.device_status()
    assert out.dtype == F16
    ref, ref_lse = oracle.sdpa(q, k, v, mask_kind=kind, qk_scale=s, with_lse=True)
    compare(out, ref, F16, str(cfg))
    compare_lse(lse, ref_lse, torch.bfloat16, str(cfg))     # products exact as for bf16


@pytest.mark.parametrize("kind,mdtype", [("keep", torch.bool), ("add", F16), ("add", torch.float32)])
def test_masks_fp16(kind, mdtype):
    q, k, v = W.dense_inputs(2, 4, 2, 150, 270, 128, 128, F16, 9, 1.0)
    g = torch.Generator().manual_seed(10)
    if kind == "keep":
        m = torch.rand(2, 4, 150, 270, generator=g) < 0.7
        m[:, :, 3] = False
    else:
        m = torch.randn(2, 4, 150, 270, generator=g).to(mdtype)
    s = 1 / math.sqrt(128)
    out = api.attn_fwd(q.to(DEV), k.to(DEV), v.to(DEV), mask=m.to(DEV), qk_scale=s)
    api.device_status()
    ref = oracle.sdpa(q, k, v, mask=m.float() if kind == "add" else m, mask_kind=kind, qk_scale=s)
    compare(out, ref, F16, f"{kind} {mdtype}")


def test_packed_mla_fp16_split():
    ql = torch.tensor([200, 7, 385], dtype=torch.int32)
    kl = torch.tensor([260, 90, 385], dtype=torch.int32)
    d = W.packed_inputs(ql, kl, 4, 4, 128, 128, 64, F16, 7)
    s = 1 / math.sqrt(192)
    g = {k: v.to(DEV) for k, v in d.items()}
    for splits in (1, 3):
        out = api.attn_fwd(g["q"], g["k"], g["v"], qrope=g["qrope"], krope=g["krope"],
                           q_seqlen=ql.to(DEV), kv_seqlen=kl.to(DEV), mask_type=api.MaskType.CAUSAL,
                           qk_scale=s, num_splits=splits)
        api.device_status()
        ref = oracle.sdpa(d["q"], d["k"], d["v"], qrope=d["qrope"], krope=d["krope"], q_seqlen=ql,
                          kv_seqlen=kl, mask_kind="causal", qk_scale=s)
        compare(out, ref, F16, f"mla fp16 s{splits}")


# ---------------------------------------------------------------- padded K/V
def _padded(kv_packed, klens, max_seq, fill, gen):
    """[Tk, H, D] packed rows -> [B, max_seq, H, D], pad rows = finite garbage."""
    B = len(klens)
    H, D = kv_packed.shape[1], kv_packed.shape[2]
    out = (torch.rand(B, max_seq, H, D, generator=gen) * 2 - 1) * fill
    out = out.to(kv_packed.dtype)
    start = 0
    for b, L in enumerate(klens):
        out[b, :L] = kv_packed[start:start + L]
        start += L
    return out


PADDED = [
    # qlens, klens, max_seq, Hq, Hk, drope, causal, dtype, splits
    ([1, 127, 128, 129, 300, 5], [1, 127, 128, 129, 300, 5], 320, 4, 2, 0, True, torch.bfloat16, 1),
    ([200, 7, 385], [260, 90, 385], 400, 4, 4, 64, True, torch.bfloat16, 1),   # MLA
    ([200, 7, 385], [260, 90, 385], 400, 4, 4, 64, True, F16, 2),
    ([0, 50, 0, 130], [10, 60, 0, 130], 256, 2, 1, 0, True, torch.bfloat16, 1),
    ([70, 257], [300, 31], 300, 2, 2, 0, False, torch.bfloat16, 3),
]


@pytest.mark.parametrize("cfg", PADDED, ids=lambda c: f"{len(c[0])}seq-pad{c[2]}-r{c[5]}-{c[7]}-s{c[8]}")
def test_padded_kv(cfg):
    qlens, klens, max_seq, Hq, Hk, drope, causal, dtype, splits = cfg
    ql = torch.tensor(qlens, dtype=torch.int32)
    kl = torch.tensor(klens, dtype=torch.int32)
    d = W.packed_inputs(ql, kl, Hq, Hk, 128, 128, drope, dtype, 7)
    gen = torch.Generator().manual_seed(99)
    # pad rows hold large finite values: they must get weight exactly zero
    pk = _padded(d["k"], klens, max_seq, 300.0, gen)
    pv = _padded(d["v"], klens, max_seq, 300.0, gen)
    pkr = _padded(d["krope"], klens, max_seq, 300.0, gen) if drope else None
    s = 1 / math.sqrt(128 + drope)
    mt = api.MaskType.CAUSAL if causal else api.MaskType.NONE
    out = api.attn_fwd(d["q"].to(DEV), pk.to(DEV), pv.to(DEV),
                       qrope=d["qrope"].to(DEV) if drope else None,
                       krope=pkr.to(DEV) if drope else None, q_seqlen=ql.to(DEV),
                       kv_seqlen=kl.to(DEV), mask_type=mt, qk_scale=s, num_splits=splits)
    api.device_status()
    ref = oracle.sdpa(d["q"], d["k"], d["v"], qrope=d.get("qrope"), krope=d.get("krope"),
                      q_seqlen=ql, kv_seqlen=kl, mask_kind="causal" if causal else "none", qk_scale=s)
    compare(out, ref, dtype, str(cfg))


def test_padded_flattened_views():
    """The table's flattened forms: q [T, Hq*D], k/v [B, max_seq, Hkv*D]."""
    ql = torch.tensor([100, 29], dtype=torch.int32)
    d = W.packed_inputs(ql, ql, 4, 2, 128, 128, 0, torch.bfloat16, 3)
    gen = torch.Generator().manual_seed(5)
    pk = _padded(d["k"], [100, 29], 128, 1.0, gen).reshape(2, 128, 2 * 128)
    pv = _padded(d["v"], [100, 29], 128, 1.0, gen).reshape(2, 128, 2 * 128)
    q2 = d["q"].reshape(129, 4 * 128)
    out = api.attn_fwd(q2.to(DEV), pk.to(DEV), pv.to(DEV), q_seqlen=ql.to(DEV), kv_seqlen=ql.to(DEV),
                       head_num=4, kv_head_num=2, kv_layout="padded", mask_type=api.MaskType.CAUSAL)
    api.device_status()
    ref = oracle.sdpa(d["q"], d["k"], d["v"], q_seqlen=ql, kv_seqlen=ql, mask_kind="causal",
                      qk_scale=1 / math.sqrt(128))
    compare(out, ref, torch.bfloat16, "flattened")


def test_padded_kv_length_over_max_seq_is_rejected_on_device():
    ql = torch.tensor([10, 20], dtype=torch.int32)
    kl = torch.tensor([10, 200], dtype=torch.int32)          # 200 > max_seq 128
    q = torch.randn(30, 2, 128).to(torch.bfloat16)
    k = torch.randn(2, 128, 2, 128).to(torch.bfloat16)
    out = torch.full((30, 2, 128), 4.0, dtype=torch.bfloat16, device=DEV)
    api.attn_fwd(q.to(DEV), k.to(DEV), k.to(DEV), q_seqlen=ql.to(DEV), kv_seqlen=kl.to(DEV), out=out)
    with pytest.raises(api.WfError) as e:
        api.device_status()
    assert e.value.status == 1
    assert torch.all(out == 4.0)
