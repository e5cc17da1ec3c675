"""The fused chunk call (wf_kvcache_update_attend) against the unfused calls
(update -> cached views -> wf_attn_fwd) of "Core 注意力", section "Block KV
cache 的调用顺序": identical outputs and identical cache contents, chunk by
chunk through a rolling window, in both cache layouts; the fp64 oracle on the
logical cache contents; the fallback for caches the kernel cannot fuse; and
the order / argument errors."""
import math

import numpy as np
import pytest
import torch

import oracle
from attention_forward_tmem_b200 import api
from tests.gpu_helpers import compare

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _chunk(i, B, Hq, Hk, C, D, dtype, seq_dim):
    g = torch.Generator().manual_seed(500 + i)
    q = torch.randn(B, Hq, C, D, generator=g).to(dtype)
    k = torch.randn(B, Hk, C, D, generator=g).to(dtype)
    v = torch.randn(B, Hk, C, D, generator=g).to(dtype)
    if seq_dim == 1:
        k, v = k.transpose(1, 2).contiguous(), v.transpose(1, 2).contiguous()
    return q.to(DEV), k.to(DEV), v.to(DEV)


def _pair(B, Hk, L, D, dtype, seq_dim, chunk, sink, window):
    shape = (B, Hk, L, D) if seq_dim == 2 else (B, L, Hk, D)
    mk = lambda: api.BlockKVCache.allocate(shape, shape, seq_dim=seq_dim, chunk_size=chunk,
                                           window_size=window, sink_size=sink, device=DEV, dtype=dtype)
    return mk(), mk()


@pytest.mark.parametrize("seq_dim", [2, 1])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_fused_equals_unfused_through_a_rolling_window(seq_dim, dtype):
    B, Hq, Hk, D = 1, 8, 4, 128
    chunk, sink, window = 256, 256, 768             # 4 slots: 1 sink + 3 rolling
    L = sink + window
    unf, fus = _pair(B, Hk, L, D, dtype, seq_dim, chunk, sink, window)
    s = 1 / math.sqrt(D)
    for i in range(9):
        q, k, v = _chunk(i, B, Hq, Hk, chunk, D, dtype, seq_dim)
        unf.before_update(i)
        unf.update(k, v)
        out_u = api.attn_fwd(q, unf.cached_k(), unf.cached_v(), mask_type=api.MaskType.NONE, qk_scale=s)
        unf.after_update(i)
        fus.before_update(i)
        out_f = fus.update_attend(k, v, q, qk_scale=s)
        assert fus.state()[4] == 3                    # as after cached_k / cached_v
        vis = fus.state()[3]
        if i in (0, 4, 8):
            ko, vo = fus.gather_logical()
            if seq_dim == 1:                          # logical copies come in the buffer's layout
                ko, vo = ko.transpose(1, 2), vo.transpose(1, 2)
            ref = oracle.sdpa(q.cpu(), ko[:, :, :vis].cpu(), vo[:, :, :vis].cpu(), qk_scale=s)
            compare(out_f, ref, dtype, f"chunk {i}")
        fus.after_update(i)
        api.device_status()
        assert torch.equal(out_u, out_f), f"chunk {i}: outputs differ"
        assert torch.equal(unf.k_buf, fus.k_buf) and torch.equal(unf.v_buf, fus.v_buf), f"chunk {i}: caches differ"


def test_fused_repeat_of_a_chunk_index_overwrites_the_same_slot():
    B, Hq, Hk, D = 1, 4, 4, 128
    unf, fus = _pair(B, Hk, 512, D, torch.bfloat16, 2, 128, 128, 384)
    for i, idx in enumerate([0, 1, 1, 2, 3, 4, 4, 5]):
        q, k, v = _chunk(i, B, Hq, Hk, 128, D, torch.bfloat16, 2)
        unf.before_update(idx)
        unf.update(k, v)
        out_u = api.attn_fwd(q, unf.cached_k(), unf.cached_v(), qk_scale=0.1)
        unf.after_update(idx)
        fus.before_update(idx)
        out_f = fus.update_attend(k, v, q, qk_scale=0.1)
        fus.after_update(idx)
        api.device_status()
        assert torch.equal(out_u, out_f) and torch.equal(unf.k_buf, fus.k_buf) and torch.equal(unf.v_buf, fus.v_buf)


@pytest.mark.parametrize("dtype,chunk", [(torch.float32, 128), (torch.bfloat16, 64)])
def test_unfusable_caches_fall_back_to_the_unfused_calls(dtype, chunk):
    """fp32 buffers, or a chunk that is not a multiple of 128 keys: the call
    runs the copy and the attention separately, with the same results."""
    B, Hq, Hk, D = 1, 2, 2, 64
    unf, fus = _pair(B, Hk, 4 * chunk, D, dtype, 2, chunk, chunk, 3 * chunk)
    for i in range(6):
        q, k, v = _chunk(i, B, Hq, Hk, chunk, D, dtype, 2)
        unf.before_update(i)
        unf.update(k, v)
        out_u = api.attn_fwd(q, unf.cached_k(), unf.cached_v(), qk_scale=0.125)
        unf.after_update(i)
        fus.before_update(i)
        out_f = fus.update_attend(k, v, q, qk_scale=0.125)
        fus.after_update(i)
        api.device_status()
        assert torch.equal(out_u, out_f) and torch.equal(unf.k_buf, fus.k_buf)


def test_fused_call_errors_leave_the_cache_unchanged():
    B, Hk, D = 1, 2, 128
    fus, _ = _pair(B, Hk, 512, D, torch.bfloat16, 2, 128, 128, 384)
    q, k, v = _chunk(0, B, 2, Hk, 128, D, torch.bfloat16, 2)
    with pytest.raises(api.WfError) as e:
        fus.update_attend(k, v, q)                     # no before_update
    assert e.value.status == 3
    fus.before_update(0)
    before = fus.k_buf.clone()
    with pytest.raises(api.WfError) as e:
        fus.update_attend(k, v, q[:, :, :, :64])       # q head size differs from the cache's
    assert e.value.status == 1
    torch.cuda.synchronize()
    assert torch.equal(before, fus.k_buf) and fus.state()[4] == 1
    out = fus.update_attend(k, v, q)                   # the same chunk, now valid
    fus.after_update(0)
    api.device_status()
    assert out.shape == (1, 2, 128, 128)
