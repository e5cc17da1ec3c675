"""Full-size parity: the benchmark's workloads, in the launch configuration
bench.py times, checked against the fp64 oracle on sampled rows (each over
its complete key range) and on properties that hold at any size.

Sampled rows: the tile edges {0, 1, 127, 128, 129, 255, 256, L-2, L-1} plus
random rows (seed 7) of a few heads.  Any-size property: under a causal mask
query row 0 sees only key 0, so its output is exactly V[0] of its kv head
(p = 1 is exact in bf16 and l = 1), for every head."""
import math

import numpy as np
import pytest
import torch

import oracle
from attention_forward_tmem_b200 import api
from attention_forward_tmem_b200 import workloads as W
from tests.gpu_helpers import compare, sample_rows

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _dense_full(name, heads_checked, per):
    w = W.WORKLOADS[name]
    q, k, v = W.dense_inputs(w.batch, w.head_num, w.kv_head_num, w.seq, w.seq, w.dqk, w.dv,
                             w.dtype, W.SEED, w.input_scale)
    out = api.attn_fwd(q.to(DEV), k.to(DEV), v.to(DEV), mask_type=api.MaskType.CAUSAL,
                       qk_scale=w.qk_scale)
    api.device_status()
    out_c = out.cpu()
    assert torch.isfinite(out_c.float()).all()
    g = w.head_num // w.kv_head_num
    # any size: causal row 0 == V[0] of the head's kv group, bit for bit
    v0 = v[:, :, 0].repeat_interleave(g, dim=1)
    assert torch.equal(out_c[:, :, 0], v0)
    # sampled rows against the oracle, one GQA group at a time
    for b in range(w.batch):
        for h in heads_checked:
            grp = h // g
            hs = slice(grp * g, grp * g + g)
            rows = sample_rows(1, [h - grp * g], [w.seq], per, seed=7 + b * 131 + h)
            ref = oracle.sdpa_rows(q[b:b + 1, hs], k[b:b + 1, grp:grp + 1], v[b:b + 1, grp:grp + 1],
                                   rows, mask_kind="causal", qk_scale=w.qk_scale, head_num=g,
                                   kv_head_num=1)
            got = out_c[b, h, rows[:, 2]]
            compare(got, ref, torch.bfloat16, f"{name} b{b} h{h}")


def test_gqa_causal_prefill_full_size():
    """B 4, 32/8 heads, L 4096, D 128, bf16, causal."""
    _dense_full("gqa_causal_prefill", heads_checked=[0, 5, 18, 31], per=24)


def test_long_gqa_causal_full_size():
    """B 1, 64/8 heads, L 65536, D 128, bf16 x 0.5, causal (near-uniform rows)."""
    _dense_full("long_gqa_causal", heads_checked=[0, 27, 63], per=16)


def test_mla_varlen_prefill_full_size():
    """8 packed sequences (lengths seeded in [512, 4096]), 128 heads, q/k/v 128 +
    qRope/kRope 64, causal."""
    w = W.WORKLOADS["mla_varlen_prefill"]
    d = W.mla_varlen_prefill()
    g = {n: t.to(DEV) for n, t in d.items()}
    out = api.attn_fwd(g["q"], g["k"], g["v"], qrope=g["qrope"], krope=g["krope"],
                       q_seqlen=g["q_seqlen"], kv_seqlen=g["kv_seqlen"],
                       mask_type=api.MaskType.CAUSAL, qk_scale=w.qk_scale)
    api.device_status()
    out_c = out.cpu()
    assert torch.isfinite(out_c.float()).all()
    lens = d["q_seqlen"].tolist()
    starts = np.concatenate([[0], np.cumsum(lens)[:-1]]).astype(np.int64)
    # any size: first row of every sequence == its first V row, every head
    for s0 in starts:
        assert torch.equal(out_c[s0], d["v"][s0])
    for h in (0, 37, 127):
        hs = slice(h, h + 1)
        rows = sample_rows(len(lens), [0], lens, 12, seed=h)
        ref = oracle.sdpa_rows(d["q"][:, hs], d["k"][:, hs], d["v"][:, hs], rows,
                               qrope=d["qrope"][:, hs], krope=d["krope"][:, hs],
                               q_seqlen=d["q_seqlen"], kv_seqlen=d["kv_seqlen"],
                               mask_kind="causal", qk_scale=w.qk_scale, head_num=1, kv_head_num=1)
        got = out_c[starts[rows[:, 0]] + rows[:, 2], h]
        compare(got, ref, torch.bfloat16, f"mla h{h}")


def test_blockkv_rolling_fused_full_size():
    """The rolling-cache workload as bench.py times it (fused chunk call, 12
    heads, chunk 1024, sink 1024, window 7168, 16 chunks): outputs and cache
    contents bit-identical to the separate calls after every chunk, and the
    last chunk's sampled rows against the oracle over the logical cache."""
    w = W.WORKLOADS["blockkv_rolling"]
    c = W.BLOCKKV
    L = c["sink_size"] + c["window_size"]
    shape = (1, w.head_num, L, w.dqk)
    mk = lambda: api.BlockKVCache.allocate(shape, shape, chunk_size=c["chunk_size"],
                                           window_size=c["window_size"], sink_size=c["sink_size"],
                                           device=DEV, dtype=w.dtype)
    unf, fus = mk(), mk()
    for i in range(c["n_chunks"]):
        q, k, v = (t.to(DEV) for t in W.blockkv_chunk(i, w.head_num, c["chunk_size"], w.dqk, w.dtype))
        unf.before_update(i)
        unf.update(k, v)
        out_u = api.attn_fwd(q, unf.cached_k(), unf.cached_v(), qk_scale=w.qk_scale)
        unf.after_update(i)
        fus.before_update(i)
        out_f = fus.update_attend(k, v, q, qk_scale=w.qk_scale)
        if i == c["n_chunks"] - 1:
            ko, vo = fus.gather_logical()
            rng = np.random.default_rng(7)
            rows = np.array([(0, h, r) for h in (0, 5, 11)
                             for r in sorted({0, 1, 127, 128, 1022, 1023} | set(rng.integers(0, 1024, 12).tolist()))])
            ref = oracle.sdpa_rows(q.cpu(), ko.cpu(), vo.cpu(), rows, qk_scale=w.qk_scale)
            compare(out_f[0, rows[:, 1], rows[:, 2]], ref, w.dtype, "rolling fused, last chunk")
        fus.after_update(i)
        api.device_status()
        assert torch.equal(out_u, out_f), f"chunk {i}: outputs differ"
        assert torch.equal(unf.k_buf, fus.k_buf) and torch.equal(unf.v_buf, fus.v_buf), f"chunk {i}: caches differ"
