"""GPU parity of dual chunk attention (wf_attn_dca) against the fp64 oracle
(oracle.dca, the reading documented there: three query forms chosen by the
chunk distance of each key, one causal softmax)."""
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


def _inputs(B, H, Hk, L, D, Dv, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    qs = [torch.randn(B, H, L, D, generator=g).to(dtype) for _ in range(3)]
    k = torch.randn(B, Hk, L, D, generator=g).to(dtype)
    v = torch.randn(B, Hk, L, Dv, generator=g).to(dtype)
    return qs, k, v


@pytest.mark.parametrize("B,H,Hk,L,chunk,dtype", [
    (1, 4, 2, 700, 128, torch.bfloat16),     # 6 chunks, ragged last, GQA
    (2, 2, 2, 515, 256, torch.float16),      # 3 chunks, two sequences
    (1, 2, 1, 300, 1000, torch.bfloat16),    # one chunk: causal attention with q_intra
    (1, 2, 2, 512, 256, torch.bfloat16),     # two chunks: no inter part
])
def test_dca_matches_oracle(B, H, Hk, L, chunk, dtype):
    (qi, qs, qe), k, v = _inputs(B, H, Hk, L, 128, 128, dtype, 70 + L)
    s = 1 / math.sqrt(128)
    out, lse = api.dca(qi.to(DEV), qs.to(DEV), qe.to(DEV), k.to(DEV), v.to(DEV), chunk, qk_scale=s,
                       return_lse=True)
    api.device_status()
    ref, ref_lse = oracle.dca(qi, qs, qe, k, v, chunk, s, with_lse=True)
    compare(out, ref, dtype, f"dca L{L} C{chunk}")
    compare_lse(lse, ref_lse, torch.bfloat16, f"dca L{L} C{chunk}")


def test_dca_with_equal_queries_is_causal_attention():
    (qi, _, _), k, v = _inputs(1, 4, 2, 640, 128, 128, torch.bfloat16, 5)
    qd, kd, vd = qi.to(DEV), k.to(DEV), v.to(DEV)
    out = api.dca(qd, qd, qd, kd, vd, 128)
    ref = api.attn_fwd(qd, kd, vd, mask_type=api.MaskType.CAUSAL)
    api.device_status()
    assert (out.float() - ref.float()).abs().max().item() <= 2e-2
