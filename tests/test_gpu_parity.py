"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle,
element by element, on shapes the oracle finishes in seconds.  Shapes span
several 128-row tiles with ragged tails, GQA groups, both layouts, every mask
kind, the MLA rope part and the degenerate cases (rows that see no key,
empty sequences)."""
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


def _run_dense(B, Hq, Hk, Lq, Lk, D, Dv, mask_kind, dtype, seed=7, scale=1.0):
    q, k, v = W.dense_inputs(B, Hq, Hk, Lq, Lk, D, Dv, dtype, seed, scale)
    s = 1.0 / math.sqrt(D)
    mt = api.MaskType.CAUSAL if mask_kind == "causal" else api.MaskType.NONE
    out = api.attn_fwd(q.to(DEV), k.to(DEV), v.to(DEV), mask_type=mt, qk_scale=s)
    api.device_status()
    ref = oracle.sdpa(q, k, v, mask_kind=mask_kind, qk_scale=s)
    return out, ref


def test_page_example_fp32():
    """'Core 注意力' example: seed 7, randn q/k/v, output (2, 8, 32, 96)."""
    q, k, v = W.page_example()
    out = api.attn_fwd(q.to(DEV), k.to(DEV), v.to(DEV), qk_scale=1 / 8)
    api.device_status()
    assert tuple(out.shape) == (2, 8, 32, 96)
    compare(out, oracle.sdpa(q, k, v, qk_scale=1 / 8), torch.float32, "page example")


@pytest.mark.parametrize("kind", ["keep", "add"])
def test_page_example_masks_fp32(kind):
    q, k, v, keep, add = W.page_example_masks()
    m = keep if kind == "keep" else add
    out = api.attn_fwd(q.to(DEV), k.to(DEV), v.to(DEV), mask=m.to(DEV), qk_scale=1 / 8)
    api.device_status()
    compare(out, oracle.sdpa(q, k, v, mask=m, mask_kind=kind, qk_scale=1 / 8), torch.float32,
            f"page example {kind}")


DENSE_BF16 = [
    # B, Hq, Hk, Lq, Lk, D, Dv, mask
    (2, 8, 2, 300, 300, 128, 128, "causal"),
    (2, 8, 2, 300, 300, 128, 128, "none"),
    (1, 4, 4, 200, 333, 128, 128, "causal"),     # Lq < Lk: bottom-right diagonal
    (1, 4, 1, 333, 200, 128, 128, "causal"),     # Lq > Lk: first rows see no key
    (1, 4, 2, 129, 257, 64, 64, "none"),
    (1, 2, 2, 130, 140, 96, 96, "causal"),
    (1, 2, 1, 100, 150, 64, 128, "none"),
    (1, 2, 1, 100, 150, 128, 64, "causal"),
    (1, 3, 3, 1, 1, 128, 128, "none"),
    (1, 2, 2, 1, 700, 128, 128, "causal"),
    (3, 6, 3, 512, 512, 128, 128, "causal"),
]


@pytest.mark.parametrize("cfg", DENSE_BF16, ids=lambda c: "x".join(map(str, c)))
def test_dense_bf16(cfg):
    out, ref = _run_dense(*cfg, dtype=torch.bfloat16)
    compare(out, ref, torch.bfloat16, str(cfg))


GROWING = [
    # B, Hq, Hk, Lq, Lk, D, Dv, mask, num_splits
    (1, 4, 2, 640, 640, 128, 128, "causal", None),
    (1, 4, 2, 300, 700, 128, 128, "none", None),
    (1, 2, 2, 256, 1024, 128, 128, "none", 3),       # split-KV partials and the merge
    (1, 2, 1, 200, 333, 64, 64, "causal", None),
    (1, 2, 2, 333, 200, 96, 128, "none", None),
]


@pytest.mark.parametrize("cfg", GROWING, ids=lambda c: "x".join(map(str, c)))
def test_running_max_grows_every_tile(cfg):
    """Scores that grow along the key index: the running row maximum rises by
    more than the lazy-rescale threshold (2^8) on every 128-key tile, so O is
    rescaled in tensor memory on every step, before that step's P (or the part
    of it handed over first) reaches the PV product."""
    B, Hq, Hk, Lq, Lk, D, Dv, mk, ns = cfg
    q, k, v = W.growing_score_inputs(B, Hq, Hk, Lq, Lk, D, Dv)
    mt = api.MaskType.CAUSAL if mk == "causal" else api.MaskType.NONE
    out = api.attn_fwd(q.to(DEV), k.to(DEV), v.to(DEV), mask_type=mt, qk_scale=1.0, num_splits=ns)
    api.device_status()
    ref = oracle.sdpa(q, k, v, mask_kind=mk, qk_scale=1.0)
    compare(out, ref, torch.bfloat16, str(cfg))


@pytest.mark.parametrize("kind", ["keep", "add"])
def test_running_max_grows_every_tile_masked(kind):
    """Growing scores through the explicit-mask instance, whose softmax step
    scales the scores (and adds the mask) before taking the row maximum."""
    B, Hq, Hk, Lq, Lk = 1, 4, 2, 300, 640
    q, k, v = W.growing_score_inputs(B, Hq, Hk, Lq, Lk, 128, 128)
    g = torch.Generator().manual_seed(13)
    if kind == "keep":
        m = torch.rand(1, 1, Lq, Lk, generator=g) < 0.8
    else:
        m = torch.randn(1, 1, Lq, Lk, generator=g).to(torch.bfloat16)
    out = api.attn_fwd(q.to(DEV), k.to(DEV), v.to(DEV), mask=m.to(DEV), qk_scale=1.0)
    api.device_status()
    ref = oracle.sdpa(q, k, v, mask=m.float() if kind == "add" else m, mask_kind=kind, qk_scale=1.0)
    compare(out, ref, torch.bfloat16, f"growing scores, {kind} mask")


@pytest.mark.parametrize("mk", ["causal", "none"])
def test_running_max_grows_every_tile_negative_scale(mk):
    """A negative qk_scale: the plain instance then scales the scores before
    the row maximum (max and a negative factor do not commute).  q carries
    -4u, so qk_scale * q.k still grows along the key index."""
    q, k, v = W.growing_score_inputs(1, 4, 2, 400, 640, 128, 128, q_bias=-4.0)
    mt = api.MaskType.CAUSAL if mk == "causal" else api.MaskType.NONE
    out = api.attn_fwd(q.to(DEV), k.to(DEV), v.to(DEV), mask_type=mt, qk_scale=-1.0)
    api.device_status()
    ref = oracle.sdpa(q, k, v, mask_kind=mk, qk_scale=-1.0)
    compare(out, ref, torch.bfloat16, f"growing scores, qk_scale -1, {mk}")


def test_zero_scale_gives_the_mean_of_visible_values():
    """qk_scale 0: every visible key has the same weight, so each output row is
    the mean of the V rows its causal range covers (checked against the
    oracle and against that mean directly)."""
    q, k, v = W.dense_inputs(1, 2, 1, 300, 300, 128, 128, torch.bfloat16, 21)
    out = api.attn_fwd(q.to(DEV), k.to(DEV), v.to(DEV), mask_type=api.MaskType.CAUSAL, qk_scale=0.0)
    api.device_status()
    ref = oracle.sdpa(q, k, v, mask_kind="causal", qk_scale=0.0)
    compare(out, ref, torch.bfloat16, "qk_scale 0")
    vf = v[0, 0].double().numpy()
    mean = np.cumsum(vf, axis=0) / np.arange(1, 301)[:, None]
    assert np.abs(ref[0, 0] - mean).max() < 1e-9 and np.abs(ref[0, 1] - mean).max() < 1e-9


def test_running_max_grows_every_tile_mla_packed():
    """The same growth through the rope instance (packed, one sequence):
    that instance hands P to the PV product whole."""
    H, L = 4, 520
    q, k, v, qr, kr = W.growing_score_inputs(1, H, H, L, L, 128, 128, drope=64)
    pk = lambda t: t[0].transpose(0, 1).contiguous()  # noqa: E731  [1,H,L,D] -> [L,H,D]
    lens = torch.tensor([L], dtype=torch.int32)
    out = api.attn_fwd(pk(q).to(DEV), pk(k).to(DEV), pk(v).to(DEV), qrope=pk(qr).to(DEV),
                       krope=pk(kr).to(DEV), q_seqlen=lens.to(DEV), kv_seqlen=lens.to(DEV),
                       mask_type=api.MaskType.CAUSAL, qk_scale=1.0)
    api.device_status()
    ref = oracle.sdpa(pk(q), pk(k), pk(v), qrope=pk(qr), krope=pk(kr), q_seqlen=lens, kv_seqlen=lens,
                      mask_kind="causal", qk_scale=1.0)
    compare(out, ref, torch.bfloat16, "growing scores, MLA packed")


DENSE_F32 = [
    (1, 4, 2, 300, 270, 128, 128, "causal"),     # one pipeline stage (large fp32 tiles)
    (2, 2, 2, 50, 77, 96, 96, "none"),
    (1, 2, 1, 200, 200, 64, 96, "causal"),
    (1, 2, 2, 140, 260, 128, 64, "none"),
]


@pytest.mark.parametrize("cfg", DENSE_F32, ids=lambda c: "x".join(map(str, c)))
def test_dense_fp32(cfg):
    out, ref = _run_dense(*cfg, dtype=torch.float32)
    compare(out, ref, torch.float32, str(cfg))


def test_dense_lq_gt_lk_rows_are_zero():
    out, _ = _run_dense(1, 2, 2, 300, 100, 128, 128, "causal", torch.bfloat16)
    assert torch.all(out[:, :, :200] == 0)
    assert torch.all(out[:, :, 200:].abs().sum(-1) > 0)


def _run_packed(qlens, klens, Hq, Hk, D, Dv, drope, causal, dtype=torch.bfloat16, seed=7):
    ql = torch.tensor(qlens, dtype=torch.int32)
    kl = torch.tensor(klens, dtype=torch.int32)
    d = W.packed_inputs(ql, kl, Hq, Hk, D, Dv, drope, dtype, seed)
    s = 1.0 / math.sqrt(D + drope)
    mt = api.MaskType.CAUSAL if causal else api.MaskType.NONE
    g = {k: v.to(DEV) for k, v in d.items()}
    out = api.attn_fwd(g["q"], g["k"], g["v"], qrope=g.get("qrope"), krope=g.get("krope"),
                       q_seqlen=ql.to(DEV), kv_seqlen=kl.to(DEV), mask_type=mt, qk_scale=s)
    api.device_status()
    ref = oracle.sdpa(d["q"], d["k"], d["v"], qrope=d.get("qrope"), krope=d.get("krope"),
                      q_seqlen=ql, kv_seqlen=kl, mask_kind="causal" if causal else "none",
                      qk_scale=s)
    return out, ref


PACKED = [
    # qlens, klens, Hq, Hk, D, Dv, drope, causal
    ([1, 127, 128, 129, 300, 5], [1, 127, 128, 129, 300, 5], 4, 2, 128, 128, 0, True),
    ([1, 127, 128, 129, 300, 5], [1, 127, 128, 129, 300, 5], 4, 2, 128, 128, 0, False),
    ([200, 7, 385], [200, 7, 385], 4, 4, 128, 128, 64, True),    # MLA split contraction
    ([200, 7, 385], [260, 90, 385], 4, 4, 128, 128, 64, True),   # Lq <= Lk per sequence
    ([0, 50, 0, 130], [10, 60, 0, 130], 2, 1, 128, 128, 0, True),  # empty sequences
    ([70, 257], [300, 31], 2, 2, 64, 64, 0, False),
]


@pytest.mark.parametrize("cfg", PACKED, ids=lambda c: f"{len(c[0])}seq-h{c[2]}-{c[3]}-r{c[6]}-{'c' if c[7] else 'n'}")
def test_packed(cfg):
    out, ref = _run_packed(*cfg)
    compare(out, ref, torch.bfloat16, str(cfg))


@pytest.mark.parametrize("causal", [True, False])
def test_packed_many_sequences(causal):
    """64 sequences of seeded random lengths in [0, 300] (kv lengths at least
    the query lengths): many more work items than CTAs, so every CTA takes
    several items through the scheduling ring, with empty sequences and
    items whose second tile is empty among them."""
    rng = np.random.default_rng(31)
    ql = rng.integers(0, 301, 64)
    ql[[3, 17, 40]] = 0
    kl = ql + rng.integers(0, 60, 64)
    out, ref = _run_packed(ql.tolist(), kl.tolist(), 8, 2, 128, 128, 0, causal, seed=32)
    compare(out, ref, torch.bfloat16, f"64 sequences causal={causal}")


@pytest.mark.parametrize("kind,mdtype,bshape", [
    ("keep", torch.bool, "full"), ("keep", torch.bool, "bcast"),
    ("add", torch.float32, "full"), ("add", torch.bfloat16, "full"), ("add", torch.float32, "bcast"),
])
def test_masks_bf16(kind, mdtype, bshape):
    B, Hq, Hk, Lq, Lk = 2, 4, 2, 150, 270
    q, k, v = W.dense_inputs(B, Hq, Hk, Lq, Lk, 128, 128, torch.bfloat16, 11)
    g = torch.Generator().manual_seed(12)
    shp = (B, Hq, Lq, Lk) if bshape == "full" else (1, 1, Lq, Lk)
    if kind == "keep":
        m = torch.rand(*shp, generator=g) < 0.7
        m[..., 5, :] = False                         # a row that sees nothing
    else:
        m = (torch.randn(*shp, generator=g) * 2).to(mdtype)
        m[..., 3, 100:] = -math.inf
    out = api.attn_fwd(q.to(DEV), k.to(DEV), v.to(DEV), mask=m.to(DEV), qk_scale=1 / math.sqrt(128))
    api.device_status()
    ref = oracle.sdpa(q, k, v, mask=m.float() if kind == "add" else m, mask_kind=kind,
                      qk_scale=1 / math.sqrt(128))
    compare(out, ref, torch.bfloat16, f"{kind} {mdtype} {bshape}")
    if kind == "keep":
        assert torch.all(out[:, :, 5] == 0)


@pytest.mark.parametrize("kind,mdtype,bshape", [
    ("keep", torch.bool, "full"), ("keep", torch.bool, "keys_strided"),
    ("add", torch.float32, "bcast"), ("add", torch.bfloat16, "full"),
])
def test_masks_full_aligned_tiles(kind, mdtype, bshape):
    """Lk = 384 (three full key tiles, every mask row 16-byte aligned): the
    16-byte vector loads of the mask; a mask whose key dim is strided takes the
    element loads."""
    B, Hq, Hk, Lq, Lk = 1, 4, 2, 200, 384
    q, k, v = W.dense_inputs(B, Hq, Hk, Lq, Lk, 128, 128, torch.bfloat16, 14)
    g = torch.Generator().manual_seed(15)
    if kind == "keep":
        if bshape == "keys_strided":
            m = (torch.rand(1, 1, Lk, Lq, generator=g) < 0.7).transpose(2, 3)
        else:
            m = torch.rand(B, Hq, Lq, Lk, generator=g) < 0.7
        m[..., 7, :] = False
    else:
        shp = (B, Hq, Lq, Lk) if bshape == "full" else (1, 1, Lq, Lk)
        m = (torch.randn(*shp, generator=g) * 2).to(mdtype)
        m[..., 3, 200:] = -math.inf
    out = api.attn_fwd(q.to(DEV), k.to(DEV), v.to(DEV), mask=m.to(DEV), qk_scale=1 / math.sqrt(128))
    api.device_status()
    ref = oracle.sdpa(q, k, v, mask=m.float() if kind == "add" else m, mask_kind=kind,
                      qk_scale=1 / math.sqrt(128))
    compare(out, ref, torch.bfloat16, f"{kind} {mdtype} {bshape}")
    if kind == "keep":
        assert torch.all(out[:, :, 7] == 0)


def test_output_guard_bands():
    """Writes stay inside `out`: canary rows before and after it are untouched."""
    B, Hq, Hk, L, D = 1, 2, 1, 200, 128
    q, k, v = W.dense_inputs(B, Hq, Hk, L, L, D, D, torch.bfloat16, 3)
    pad = 64
    buf = torch.full((B, Hq, L + 2 * pad, D), 7.0, dtype=torch.bfloat16, device=DEV)
    out = buf[:, :, pad:pad + L]
    api.attn_fwd(q.to(DEV), k.to(DEV), v.to(DEV), mask_type=api.MaskType.CAUSAL, out=out)
    api.device_status()
    assert torch.all(buf[:, :, :pad] == 7.0) and torch.all(buf[:, :, pad + L:] == 7.0)
    compare(out, oracle.sdpa(q, k, v, mask_kind="causal", qk_scale=1 / math.sqrt(D)),
            torch.bfloat16, "guard")


def test_packed_guard_bands():
    ql = torch.tensor([100, 29], dtype=torch.int32)
    d = W.packed_inputs(ql, ql, 2, 2, 128, 128, 0, torch.bfloat16, 5)
    T = int(ql.sum())
    buf = torch.full((T + 256, 2, 128), -3.0, dtype=torch.bfloat16, device=DEV)
    out = buf[128:128 + T]
    api.attn_fwd(d["q"].to(DEV), d["k"].to(DEV), d["v"].to(DEV), q_seqlen=ql.to(DEV),
                 kv_seqlen=ql.to(DEV), mask_type=api.MaskType.CAUSAL, out=out)
    api.device_status()
    assert torch.all(buf[:128] == -3.0) and torch.all(buf[128 + T:] == -3.0)


def test_bad_lengths_reported_on_device():
    """Lengths that sum past the packed tensors: nothing is computed and the
    device status reports WF_ERR_INVALID_ARG."""
    ql = torch.tensor([100, 100], dtype=torch.int32)
    d = W.packed_inputs(torch.tensor([100, 50]), torch.tensor([100, 50]), 2, 2, 128, 128)
    out = torch.full((150, 2, 128), 5.0, dtype=torch.bfloat16, device=DEV)
    api.attn_fwd(d["q"].to(DEV), d["k"].to(DEV), d["v"].to(DEV), q_seqlen=ql.to(DEV),
                 kv_seqlen=ql.to(DEV), out=out)
    with pytest.raises(api.WfError) as e:
        api.device_status()
    assert e.value.status == 1
    assert torch.all(out == 5.0)
    api.device_status()      # cleared


def test_bounded_wait_times_out_and_device_stays_usable():
    """The debug switch starves the first K tile: the MMA stage's bounded wait
    runs out, the kernel records WF_ERR_TIMEOUT and returns; the next normal
    call is correct."""
    q, k, v = W.dense_inputs(1, 2, 2, 128, 256, 128, 128, torch.bfloat16, 9)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    api.attn_fwd(qd[:, :1], kd[:, :1], vd[:, :1], debug_flags=1, timeout_cycles=20_000_000)
    with pytest.raises(api.WfError) as e:
        api.device_status()
    assert e.value.status == 6
    out = api.attn_fwd(qd, kd, vd, qk_scale=1 / math.sqrt(128))
    api.device_status()
    compare(out, oracle.sdpa(q, k, v, qk_scale=1 / math.sqrt(128)), torch.bfloat16, "after timeout")


def test_non_contiguous_inputs():
    """Strided q/k/v/out views ([B, L, H, D] storage viewed as [B, H, L, D])."""
    B, Hq, Hk, L, D = 2, 4, 2, 190, 128
    q, k, v = W.dense_inputs(B, Hq, Hk, L, L, D, D, torch.bfloat16, 21)
    qs = q.transpose(1, 2).contiguous().to(DEV).transpose(1, 2)
    ks = k.transpose(1, 2).contiguous().to(DEV).transpose(1, 2)
    vs = v.transpose(1, 2).contiguous().to(DEV).transpose(1, 2)
    ob = torch.empty(B, L, Hq, D, dtype=torch.bfloat16, device=DEV)
    out = ob.transpose(1, 2)
    api.attn_fwd(qs, ks, vs, mask_type=api.MaskType.CAUSAL, out=out)
    api.device_status()
    compare(out, oracle.sdpa(q, k, v, mask_kind="causal", qk_scale=1 / math.sqrt(D)),
            torch.bfloat16, "strided")


def test_repeated_calls_are_deterministic():
    q, k, v = W.dense_inputs(2, 8, 2, 640, 640, 128, 128, torch.bfloat16, 4)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    a = api.attn_fwd(qd, kd, vd, mask_type=api.MaskType.CAUSAL)
    b = api.attn_fwd(qd, kd, vd, mask_type=api.MaskType.CAUSAL)
    api.device_status()
    assert torch.equal(a, b)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("kind", ["none", "causal"])
def test_dense_without_keys_gives_zero_rows(dtype, kind):
    """Lk = 0: every row sees no key, so it is 0 with LSE -inf (the silent case's reading)."""
    q = torch.randn(1, 4, 200, 128).to(dtype).to(DEV)
    k = torch.empty(1, 2, 0, 128, dtype=dtype, device=DEV)
    v = torch.empty(1, 2, 0, 128, dtype=dtype, device=DEV)
    mt = api.MaskType.CAUSAL if kind == "causal" else api.MaskType.NONE
    out, lse = api.attn_fwd(q, k, v, mask_type=mt, return_lse=True)
    api.device_status()
    assert torch.all(out == 0) and torch.all(torch.isneginf(lse))


def test_packed_without_keys_gives_zero_rows():
    ql = torch.tensor([30, 0, 70], dtype=torch.int32)
    kl = torch.tensor([0, 0, 0], dtype=torch.int32)
    q = torch.randn(100, 2, 128).to(torch.bfloat16).to(DEV)
    k = torch.empty(0, 2, 128, dtype=torch.bfloat16, device=DEV)
    out = torch.full((100, 2, 128), 3.0, dtype=torch.bfloat16, device=DEV)
    out, lse = api.attn_fwd(q, k, k, q_seqlen=ql.to(DEV), kv_seqlen=kl.to(DEV), out=out, return_lse=True)
    api.device_status()
    assert torch.all(out == 0) and torch.all(torch.isneginf(lse))
