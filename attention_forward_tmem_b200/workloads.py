"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle checks.

This module holds no arithmetic of the attention method: it only draws random
tensors (CPU ``torch.Generator``, fp32 draws, then a cast) in the shapes of the
five workloads below, so that the device path and the fp64 oracle see the same
values.  Importing it does not load the CUDA library.

Workloads (all seeded with 7 unless stated):

* ``tiny_sdpa_fp32`` -- the example of "Core 注意力", section
  "一个可以在 CPU 或 GPU 上运行的例子": ``torch.manual_seed(7)``, q
  ``randn(2,8,32,64)``, k ``randn(2,8,48,64)``, v ``randn(2,8,48,96)``, fp32,
  output ``(2,8,32,96)``; then a keep-mask (``rand < 0.8``, key 0 forced on in any
  empty row) and an additive mask ``randn`` of shape ``(2,8,32,48)``.
* ``gqa_causal_prefill`` -- B 4, 32 query heads, 8 kv heads, L 4096, D 128,
  bf16 N(0,1), causal.
* ``mla_varlen_prefill`` -- 8 sequences, lengths ``randint(512, 4097)``, 128
  heads, q/k/v 128 + qRope/kRope 64, bf16 N(0,1), causal, packed layout of
  "MLA Prefill" (parameter table).
* ``blockkv_rolling`` -- 1 x 12 heads x D 128, chunk 1024, sink 1024,
  window 7168, 16 chunks of fresh N(0,1) q/k/v.
* ``long_gqa_causal`` -- B 1, 64 query heads, 8 kv heads, L 65536, D 128,
  bf16 N(0,1) * 0.5, causal.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch

SEED = 7


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    head_num: int
    kv_head_num: int
    seq: int
    dqk: int
    dv: int
    drope: int
    dtype: torch.dtype
    mask: str
    qk_scale: float
    input_scale: float = 1.0


WORKLOADS = {
    "tiny_sdpa_fp32": Workload("tiny_sdpa_fp32", 2, 8, 8, 32, 64, 96, 0, torch.float32, "none",
                               1.0 / math.sqrt(64)),
    "gqa_causal_prefill": Workload("gqa_causal_prefill", 4, 32, 8, 4096, 128, 128, 0,
                                   torch.bfloat16, "causal", 1.0 / math.sqrt(128)),
    "mla_varlen_prefill": Workload("mla_varlen_prefill", 8, 128, 128, 4096, 128, 128, 64,
                                   torch.bfloat16, "causal", 1.0 / math.sqrt(192)),
    "blockkv_rolling": Workload("blockkv_rolling", 1, 12, 12, 1024, 128, 128, 0, torch.bfloat16,
                                "none", 1.0 / math.sqrt(128)),
    "long_gqa_causal": Workload("long_gqa_causal", 1, 64, 8, 65536, 128, 128, 0, torch.bfloat16,
                                "causal", 1.0 / math.sqrt(128), 0.5),
}

BLOCKKV = dict(chunk_size=1024, sink_size=1024, window_size=7168, n_chunks=16)


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def _randn(g, shape, dtype, scale=1.0):
    x = torch.randn(*shape, generator=g, dtype=torch.float32)
    if scale != 1.0:
        x = x * scale
    return x.to(dtype)


def page_example():
    """q, k, v of the page's example, drawn exactly as printed there (global seed)."""
    torch.manual_seed(SEED)
    q = torch.randn(2, 8, 32, 64)
    k = torch.randn(2, 8, 48, 64)
    v = torch.randn(2, 8, 48, 96)
    return q, k, v


def page_example_masks():
    """The example's q, k, v followed by a keep-mask and an additive mask."""
    q, k, v = page_example()
    keep = torch.rand(2, 8, 32, 48) < 0.8
    empty = ~keep.any(dim=-1)
    keep[..., 0] |= empty
    add = torch.randn(2, 8, 32, 48)
    return q, k, v, keep, add


def dense_inputs(batch, head_num, kv_head_num, lq, lk, dqk, dv, dtype=torch.bfloat16,
                 seed=SEED, scale=1.0):
    """q [B,Hq,Lq,Dqk], k [B,Hkv,Lk,Dqk], v [B,Hkv,Lk,Dv] on the CPU."""
    g = _gen(seed)
    q = _randn(g, (batch, head_num, lq, dqk), dtype, scale)
    k = _randn(g, (batch, kv_head_num, lk, dqk), dtype, scale)
    v = _randn(g, (batch, kv_head_num, lk, dv), dtype, scale)
    return q, k, v


def growing_score_inputs(batch, head_num, kv_head_num, lq, lk, dqk, dv, dtype=torch.bfloat16,
                         seed=SEED, growth=0.02, q_bias=4.0, noise=0.5, drope=0):
    """Dense q, k, v whose scores grow along the key index, so that an online
    softmax raises its running row maximum on every key tile: every query
    carries q_bias * u and key j carries growth * j * u, for one shared unit
    vector u, over N(0, noise^2) entries; q_i . k_j is then ~q_bias * growth * j
    plus noise (with the defaults and qk_scale 1, ~15 log2 units more per
    128 keys).  drope > 0 appends N(0, noise^2) rope parts qRope [B,Hq,Lq,drope]
    and kRope [B,Hkv,Lk,drope] to the returned tuple."""
    g = _gen(seed)
    u = torch.randn(dqk, generator=g, dtype=torch.float32)
    u = u / u.norm()
    q = _randn(g, (batch, head_num, lq, dqk), torch.float32, noise) + q_bias * u
    j = torch.arange(lk, dtype=torch.float32).view(1, 1, lk, 1)
    k = _randn(g, (batch, kv_head_num, lk, dqk), torch.float32, noise) + growth * j * u
    v = _randn(g, (batch, kv_head_num, lk, dv), dtype)
    if drope:
        qr = _randn(g, (batch, head_num, lq, drope), dtype, noise)
        kr = _randn(g, (batch, kv_head_num, lk, drope), dtype, noise)
        return q.to(dtype), k.to(dtype), v, qr, kr
    return q.to(dtype), k.to(dtype), v


def seqlens(batch, lo, hi, seed=SEED):
    """Per-sequence lengths uniform in [lo, hi] (inclusive)."""
    g = _gen(seed)
    return torch.randint(lo, hi + 1, (batch,), generator=g, dtype=torch.int64).to(torch.int32)


def packed_inputs(q_lens, kv_lens, head_num, kv_head_num, dqk, dv, drope=0,
                  dtype=torch.bfloat16, seed=SEED, scale=1.0):
    """Packed q [T,Hq,Dqk], k [Tk,Hkv,Dqk], v [Tk,Hkv,Dv] (+ qRope/kRope) on the CPU."""
    g = _gen(seed + 1)
    t = int(torch.as_tensor(q_lens).sum())
    tk = int(torch.as_tensor(kv_lens).sum())
    out = {
        "q": _randn(g, (t, head_num, dqk), dtype, scale),
        "k": _randn(g, (tk, kv_head_num, dqk), dtype, scale),
        "v": _randn(g, (tk, kv_head_num, dv), dtype, scale),
    }
    if drope:
        out["qrope"] = _randn(g, (t, head_num, drope), dtype, scale)
        out["krope"] = _randn(g, (tk, kv_head_num, drope), dtype, scale)
    return out


def mla_varlen_prefill(seed=SEED):
    """The full packed MLA workload: lengths, then q, qRope, k, kRope, v."""
    w = WORKLOADS["mla_varlen_prefill"]
    lens = seqlens(w.batch, 512, 4096, seed)
    d = packed_inputs(lens, lens, w.head_num, w.kv_head_num, w.dqk, w.dv, w.drope, w.dtype, seed)
    d["q_seqlen"] = lens
    d["kv_seqlen"] = lens.clone()
    return d


def blockkv_chunk(i, heads=12, chunk=1024, d=128, dtype=torch.bfloat16, seed=SEED):
    """q, k, v of chunk i of the rolling-cache workload (fresh draws per chunk)."""
    g = _gen(seed * 1000 + i)
    q = _randn(g, (1, heads, chunk, d), dtype)
    k = _randn(g, (1, heads, chunk, d), dtype)
    v = _randn(g, (1, heads, chunk, d), dtype)
    return q, k, v
