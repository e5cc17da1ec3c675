"""Output rows are written with 32-byte stores when a row starts on a 32-byte
boundary and with 16-byte stores otherwise.  Both forms against the fp64
oracle, through output views into wider buffers (row stride a multiple of 32
bytes, view offset 0 or 16 bytes), with the bytes outside the view checked to
be untouched; dense and packed, 16-bit and fp32."""
import math

import pytest
import torch

import oracle
from attention_forward_tmem_b200 import api
from attention_forward_tmem_b200 import workloads as W
from tests.gpu_helpers import compare

pytestmark = pytest.mark.gpu
DEV = "cuda"
FILL = 7.0


def _view(shape, dtype, offset_bytes):
    """A view of `shape` into a buffer 32 bytes wider per row, starting
    `offset_bytes` into each row; the buffer is pre-filled with FILL."""
    es = torch.tensor([], dtype=dtype).element_size()
    pad, off = 32 // es, offset_bytes // es
    big = torch.full((*shape[:-1], shape[-1] + pad), FILL, dtype=dtype, device=DEV)
    return big, big[..., off:off + shape[-1]], off


def _untouched(big, off, n):
    rest = torch.cat([big[..., :off], big[..., off + n:]], dim=-1)
    return bool(torch.all(rest == FILL))


@pytest.mark.parametrize("offset", [0, 16])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16, torch.float32])
def test_dense_output_views(dtype, offset):
    B, Hq, Hk, L, D = 1, 4, 2, 200, 128
    q, k, v = W.dense_inputs(B, Hq, Hk, L, L, D, D, dtype, 21, 1.0)
    s = 1 / math.sqrt(D)
    big, out, off = _view((B, Hq, L, D), dtype, offset)
    api.attn_fwd(q.to(DEV), k.to(DEV), v.to(DEV), mask_type=api.MaskType.CAUSAL, qk_scale=s, out=out)
    api.device_status()
    ref = oracle.sdpa(q, k, v, mask_kind="causal", qk_scale=s)
    compare(out, ref, dtype, f"dense {dtype} offset {offset}")
    assert _untouched(big, off, D)


@pytest.mark.parametrize("offset", [0, 16])
def test_packed_output_views(offset):
    lens = torch.tensor([130, 1, 257], dtype=torch.int32)
    H, D = 4, 128
    d = W.packed_inputs(lens, lens, H, H, D, D, 0, torch.bfloat16, 22)
    s = 1 / math.sqrt(D)
    T = int(lens.sum())
    big, out, off = _view((T, H, D), torch.bfloat16, offset)
    g = {a: b.to(DEV) for a, b in d.items()}
    api.attn_fwd(g["q"], g["k"], g["v"], q_seqlen=lens.to(DEV), kv_seqlen=lens.to(DEV),
                 mask_type=api.MaskType.CAUSAL, qk_scale=s, out=out)
    api.device_status()
    ref = oracle.sdpa(d["q"], d["k"], d["v"], q_seqlen=lens, kv_seqlen=lens, mask_kind="causal",
                      qk_scale=s)
    compare(out, ref, torch.bfloat16, f"packed offset {offset}")
    assert _untouched(big, off, D)
