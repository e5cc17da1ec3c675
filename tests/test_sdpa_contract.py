"""api.scaled_dot_product_attention: the PyTorch SDPA signature of "Core 注意力"
(section "选择最窄的入口") mapped onto attn_fwd.  Host-side checks of the
mapping (the call into the library is captured), and of the predicate of
the top-left causal kind that is_causal maps to when L != S, against torch's
own is_causal on the CPU."""
import math

import pytest
import torch
import torch.nn.functional as F

from attention_forward_tmem_b200 import api


@pytest.fixture
def captured(monkeypatch):
    calls = []

    def fake_attn_fwd(q, k, v, **kw):
        calls.append((q, k, v, kw))
        return torch.zeros(q.shape[:3] + (v.shape[-1],), dtype=q.dtype)

    monkeypatch.setattr(api, "attn_fwd", fake_attn_fwd)
    return calls


def _qkv(B=2, Hq=4, Hk=4, L=16, S=16, E=8, Ev=8, dtype=torch.float64):
    g = torch.Generator().manual_seed(3)
    q = torch.randn(B, Hq, L, E, generator=g, dtype=dtype)
    k = torch.randn(B, Hk, S, E, generator=g, dtype=dtype)
    v = torch.randn(B, Hk, S, Ev, generator=g, dtype=dtype)
    return q, k, v


def test_rejections(captured):
    q, k, v = _qkv()
    with pytest.raises(ValueError, match="dropout"):
        api.scaled_dot_product_attention(q, k, v, dropout_p=0.1)
    with pytest.raises(ValueError, match="is_causal"):
        api.scaled_dot_product_attention(q, k, v, attn_mask=torch.ones(16, 16, dtype=torch.bool),
                                         is_causal=True)
    qg, kg, vg = _qkv(Hq=4, Hk=2)
    with pytest.raises(ValueError, match="enable_gqa"):
        api.scaled_dot_product_attention(qg, kg, vg)
    with pytest.raises(ValueError):
        api.scaled_dot_product_attention(q, k, v, attn_mask=torch.ones(1, 1, 1, 16, 16, dtype=torch.bool))
    assert not captured


def test_plain_gqa_scale_and_causal_square(captured):
    q, k, v = _qkv(Hq=4, Hk=2)
    api.scaled_dot_product_attention(q, k, v, enable_gqa=True, scale=0.3)
    api.scaled_dot_product_attention(q, k, v, enable_gqa=True, is_causal=True)
    (_, _, _, kw0), (_, _, _, kw1) = captured
    assert kw0["mask"] is None and kw0["mask_type"] == api.MaskType.NONE and kw0["qk_scale"] == 0.3
    assert kw1["mask"] is None and kw1["mask_type"] == api.MaskType.CAUSAL and kw1["qk_scale"] is None


@pytest.mark.parametrize("L,S", [(5, 12), (12, 5)])
def test_causal_with_unequal_lengths_is_top_left(captured, L, S):
    """is_causal with L != S maps to the kernel's top-left causal kind (no
    mask tensor); its documented predicate, key j visible to query i iff
    j <= i, reproduces torch's own is_causal."""
    q, k, v = _qkv(L=L, S=S)
    api.scaled_dot_product_attention(q, k, v, is_causal=True)
    (_, _, _, kw), = captured
    assert kw["mask_type"] == api.MaskType.CAUSAL_TOP_LEFT and kw["mask"] is None
    i = torch.arange(L)[:, None]
    j = torch.arange(S)[None, :]
    keep = j <= i
    want = F.scaled_dot_product_attention(q, k, v, is_causal=True)
    got = F.scaled_dot_product_attention(q, k, v, attn_mask=keep)
    finite = torch.isfinite(want).all(-1)             # torch gives NaN rows where no key is visible
    assert torch.allclose(got[finite], want[finite], atol=1e-12)


def test_masks_keep_their_meaning(captured):
    q, k, v = _qkv(dtype=torch.bfloat16)
    keep = torch.rand(16, 16) < 0.5
    add64 = torch.randn(2, 1, 16, 16, dtype=torch.float64)
    add_bf16 = torch.randn(4, 16, 16).to(torch.bfloat16)
    api.scaled_dot_product_attention(q, k, v, attn_mask=keep)
    api.scaled_dot_product_attention(q, k, v, attn_mask=add64)
    api.scaled_dot_product_attention(q, k, v, attn_mask=add_bf16)
    (_, _, _, a), (_, _, _, b), (_, _, _, c) = captured
    assert a["mask_type"] == api.MaskType.BOOL_KEEP and a["mask"].shape == (1, 1, 16, 16)
    assert torch.equal(a["mask"][0, 0], keep)
    assert b["mask_type"] == api.MaskType.ADDITIVE and b["mask"].dtype == torch.float32
    assert torch.equal(b["mask"], add64.float())
    assert c["mask_type"] == api.MaskType.ADDITIVE and c["mask"].dtype == torch.bfloat16
    assert c["mask"].shape == (1, 4, 16, 16)             # trailing-aligned broadcast: dim 0 is H


def test_three_dim_inputs(captured):
    q, k, v = _qkv(B=1, Ev=6)
    out = api.scaled_dot_product_attention(q[0], k[0], v[0], scale=1 / math.sqrt(8))
    (qq, kk, vv, kw), = captured
    assert qq.shape == (1, 4, 16, 8) and vv.shape == (1, 4, 16, 6)
    assert out.shape == (4, 16, 6)


def test_backend_keyword_is_accepted(captured):
    q, k, v = _qkv()
    api.scaled_dot_product_attention(q, k, v, dropout_p=0.0, backend="math")
    (_, _, _, kw), = captured
    assert kw["mask_type"] == api.MaskType.NONE


def test_cache_constructor_forms():
    """The page's keyword form (shapes, device, dtype) and the buffer form;
    anything mixed is refused, and a host device is refused loudly."""
    shape = (1, 1, 4, 2)
    with pytest.raises(ValueError, match="either"):
        api.BlockKVCache(chunk_size=2, window_size=4)
    with pytest.raises(ValueError, match="either"):
        api.BlockKVCache(torch.zeros(shape), k_shape=shape, v_shape=shape, chunk_size=2, window_size=4)
    with pytest.raises(ValueError, match="either"):
        api.BlockKVCache(k_shape=shape, chunk_size=2, window_size=4)
    with pytest.raises(api.WfError, match="no CPU path"):
        api.BlockKVCache(k_shape=shape, v_shape=(1, 1, 4, 3), seq_dim=2, chunk_size=2, window_size=4,
                         device="cpu", dtype=torch.float32)
    with pytest.raises(api.WfError, match="no CPU path"):
        api.BlockKVCache(torch.zeros(shape), torch.zeros(1, 1, 4, 3), chunk_size=2, window_size=4)
