"""api.scaled_dot_product_attention on the GPU against the fp64 oracle: the
PyTorch SDPA signature of "Core 注意力" (section "选择最窄的入口") with GQA,
both mask kinds and is_causal, including the top-left causal alignment torch
uses when L != S."""
import math

import pytest
import torch

import oracle
from attention_forward_tmem_b200 import api
from attention_forward_tmem_b200 import workloads as W
from tests.gpu_helpers import compare

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("L,S", [(200, 200), (130, 300), (300, 130)])
def test_is_causal_top_left(L, S):
    B, Hq, Hk, E = 1, 4, 2, 128
    q, k, v = W.dense_inputs(B, Hq, Hk, L, S, E, E, torch.bfloat16, 41)
    out = api.scaled_dot_product_attention(q.to(DEV), k.to(DEV), v.to(DEV), is_causal=True,
                                           enable_gqa=True)
    api.device_status()
    keep = torch.ones(L, S, dtype=torch.bool).tril().expand(B, Hq, L, S)
    ref = oracle.sdpa(q, k, v, mask=keep, mask_kind="keep", qk_scale=1 / math.sqrt(E))
    compare(out, ref, torch.bfloat16, f"is_causal L={L} S={S}")


@pytest.mark.parametrize("kind", ["keep", "add"])
def test_attn_mask_and_scale(kind):
    B, H, L, S, E = 2, 2, 150, 170, 64
    q, k, v = W.dense_inputs(B, H, H, L, S, E, E, torch.bfloat16, 42)
    g = torch.Generator().manual_seed(43)
    if kind == "keep":
        m = torch.rand(L, S, generator=g) < 0.6
        m[:, 0] = True
    else:
        m = torch.randn(H, L, S, generator=g)
    out = api.scaled_dot_product_attention(q.to(DEV), k.to(DEV), v.to(DEV), attn_mask=m.to(DEV),
                                           scale=0.1)
    api.device_status()
    ref = oracle.sdpa(q, k, v, mask=m.expand(B, H, L, S), mask_kind=kind, qk_scale=0.1)
    compare(out, ref, torch.bfloat16, f"attn_mask {kind}")
