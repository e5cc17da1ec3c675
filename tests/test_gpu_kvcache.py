"""BlockKVCache on the GPU against the plain Python model (exact contents and
state) and the fp64 oracle (attention over the visible cache).

Sources: "Core 注意力" (WorldFoundry docs), section "Block KV cache 的调用顺序"
(call order, repeat / +1 / skip rules, sink + window sizes, the example with
2, 4, then 4 rolled visible tokens)."""
import math

import numpy as np
import pytest
import torch

import oracle
from attention_forward_tmem_b200 import api
from attention_forward_tmem_b200 import workloads as W
from oracle.kvcache_model import BlockKVCacheModel, OrderError
from tests.gpu_helpers import compare
from tests.oracle_pins import golden

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_page_example_exact():
    gd = golden("blockkv_page_example.json")
    cache = api.BlockKVCache.allocate(gd["k_shape"], gd["v_shape"], seq_dim=gd["seq_dim"],
                                      chunk_size=gd["chunk_size"], window_size=gd["window_size"],
                                      device=DEV, dtype=torch.float32)
    for c in range(gd["n_chunks"]):
        k = torch.full((1, 1, 2, 2), float(c), device=DEV)
        v = torch.full((1, 1, 2, 3), float(c), device=DEV)
        cache.before_update(c)
        cache.update(k, v)
        vis_k = cache.cached_k()
        assert vis_k.shape[2] == gd["visible_tokens"][c]
        ko, vo = cache.gather_logical()
        torch.cuda.synchronize()
        assert ko[0, 0, :, 0].tolist() == [float(x) for x in gd["logical_token_values"][c]]
        assert vo[0, 0, :, 0].tolist() == [float(x) for x in gd["logical_token_values"][c]]
        phys = [None if x is None else float(x) for x in gd["physical_token_values"][c]]
        got = cache.k_buf[0, 0, :, 0].tolist()
        assert [g for g, p in zip(got, phys) if p is not None] == [p for p in phys if p is not None]
        cache.after_update(c)


def test_order_errors_through_the_library():
    cache = api.BlockKVCache.allocate((1, 2, 8, 64), (1, 2, 8, 64), chunk_size=2, window_size=6,
                                      sink_size=2, device=DEV, dtype=torch.bfloat16)
    kv = torch.zeros(1, 2, 2, 64, dtype=torch.bfloat16, device=DEV)

    def expect_order(fn, *a):
        before = cache.state()
        with pytest.raises(api.WfError) as e:
            fn(*a)
        assert e.value.status == 3
        assert cache.state() == before

    expect_order(cache.before_update, 1)          # the first chunk index is 0
    cache.before_update(0)
    expect_order(cache.cached_k)                  # cached before update
    cache.update(kv, kv)
    expect_order(cache.after_update, 0.0 + 1)     # another index
    cache.cached_k()
    cache.after_update(0)
    expect_order(cache.before_update, 2)          # skipped index
    cache.before_update(1)
    cache.update(kv, kv)
    cache.cached_v()
    cache.after_update(1)
    cache.before_update(1)                        # repeat overwrites chunk 1
    expect_order(cache.before_update, 1)          # before_update twice
    with pytest.raises(api.WfError) as e:         # not exactly chunk_size positions
        cache.update(torch.zeros(1, 2, 3, 64, dtype=torch.bfloat16, device=DEV), kv)
    assert e.value.status == 1


def test_rolling_workload_exact_cache_and_attention():
    """The 16-chunk rolling workload: exact buffer contents and state against
    the model after every chunk; attention of each chunk's queries over the
    visible cache against the oracle on sampled rows."""
    cfg = W.BLOCKKV
    C, S, Wn = cfg["chunk_size"], cfg["sink_size"], cfg["window_size"]
    H, D = 12, 128
    L = S + Wn
    cache = api.BlockKVCache.allocate((1, H, L, D), (1, H, L, D), chunk_size=C, window_size=Wn,
                                      sink_size=S, device=DEV, dtype=torch.bfloat16)
    model = BlockKVCacheModel(L, C, Wn, S)
    scale = 1 / math.sqrt(D)
    gd = golden("blockkv_rolling_sequence.json")
    rng = np.random.default_rng(7)
    for i in range(cfg["n_chunks"]):
        q, k, v = W.blockkv_chunk(i, H, C, D)
        cache.before_update(i)
        model.before_update(i)
        cache.update(k.to(DEV), v.to(DEV))
        slot = model.update((k, v), C)
        kview, vview = cache.cached_k(), cache.cached_v()
        vis, phys = model.cached()
        out = api.attn_fwd(q.to(DEV), kview, vview, qk_scale=scale)
        api.device_status()
        cur, com, wslot, gvis, phase = cache.state()
        assert (cur, wslot, gvis) == (i, gd["slots"][i], gd["visible"][i]) == (i, slot, vis)
        # exact buffer contents: slot s holds the chunk the model put there
        kb, vb = cache.k_buf.cpu(), cache.v_buf.cpu()
        for s, (kk, vv) in enumerate(phys):
            assert torch.equal(kb[:, :, s * C:(s + 1) * C], kk)
            assert torch.equal(vb[:, :, s * C:(s + 1) * C], vv)
        # attention over the visible keys (logical order: no causal mask, so
        # the physical ring order gives the same result)
        ks = torch.cat([p[0] for p in model.cached_logical()], dim=2)
        vs = torch.cat([p[1] for p in model.cached_logical()], dim=2)
        if i in (0, 1, 7, 8, 15):
            heads = [0, 5, 11]
            rows = np.array([(0, h, r) for h in heads
                             for r in sorted({0, 1, 127, 128, C - 1, *rng.integers(0, C, 8)})])
            ref = oracle.sdpa_rows(q, ks, vs, rows, qk_scale=scale)
            got = out.cpu()[0, rows[:, 1], rows[:, 2]]
            compare(got, ref, torch.bfloat16, f"chunk {i}")
        cache.after_update(i)
        model.after_update(i)
    assert model.logical_chunks(cfg["n_chunks"] - 1) == gd["logical_chunks_after_15"]


def test_seq_dim_1_layout():
    """[B, L, H, D] buffers (seq_dim 1): same rolling rule, views usable as k / v."""
    B, H, D, C = 1, 2, 64, 128
    cache = api.BlockKVCache.allocate((B, 4 * C, H, D), (B, 4 * C, H, D), seq_dim=1, chunk_size=C,
                                      window_size=3 * C, sink_size=C, device=DEV,
                                      dtype=torch.bfloat16)
    model = BlockKVCacheModel(4 * C, C, 3 * C, C)
    for i in range(6):
        q, k, v = W.dense_inputs(B, H, H, C, C, D, D, torch.bfloat16, 50 + i)
        kl, vl = k.transpose(1, 2).contiguous(), v.transpose(1, 2).contiguous()   # [B, C, H, D]
        cache.before_update(i)
        model.before_update(i)
        cache.update(kl.to(DEV), vl.to(DEV))
        model.update((k, v), C)
        model.cached()
        out = api.attn_fwd(q.to(DEV), cache.cached_k(), cache.cached_v(), qk_scale=1 / 8)
        api.device_status()
        ks = torch.cat([p[0] for p in model.cached_logical()], dim=2)
        vs = torch.cat([p[1] for p in model.cached_logical()], dim=2)
        compare(out, oracle.sdpa(q, ks, vs, qk_scale=1 / 8), torch.bfloat16, f"seq_dim 1 chunk {i}")
        cache.after_update(i)
        model.after_update(i)
