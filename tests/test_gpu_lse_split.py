"""GPU parity of the LSE output, split-KV and the merge entry point against the
fp64 oracle (oracle.sdpa with its LSE, oracle.merge).

LSE tolerance, from the arithmetic: with bf16 inputs every score product is
exact in fp32 and the fp32 sums over <= 192 terms err by well under 1e-3
here; exp2 / log2 approximations add ~1e-6.  With fp32 inputs the TF32
products round each operand to 11 bits (relative 2^-11), which moves a score
by at most ~5e-3 on the page example's sizes; the LSE, a softmax-weighted
mean of the scores plus a log, moves by no more.  Rows without a visible key
must be -inf on both sides."""
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
LSE_TOL = {torch.bfloat16: 1e-3, torch.float32: 5e-3}


def compare_lse(got, ref, dtype, what=""):
    g = got.detach().cpu().numpy().astype(np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert g.shape == ref.shape, f"{what}: lse shape {g.shape} vs {ref.shape}"
    inf_ref = np.isneginf(ref)
    assert np.array_equal(np.isneginf(g), inf_ref), f"{what}: -inf rows differ"
    fin = ~inf_ref
    assert np.all(np.isfinite(g[fin])), f"{what}: non-finite lse"
    err = float(np.abs(g[fin] - ref[fin]).max()) if fin.any() else 0.0
    assert err <= LSE_TOL[dtype], f"{what}: lse max-abs {err:.3e} > {LSE_TOL[dtype]}"


def _dense(B, Hq, Hk, Lq, Lk, D, Dv, kind, dtype, splits, seed=7):
    q, k, v = W.dense_inputs(B, Hq, Hk, Lq, Lk, D, Dv, dtype, seed, 1.0)
    s = 1.0 / math.sqrt(D)
    mt = api.MaskType.CAUSAL if kind == "causal" else api.MaskType.NONE
    out, lse = api.attn_fwd(q.to(DEV), k.to(DEV), v.to(DEV), mask_type=mt, qk_scale=s,
                            return_lse=True, num_splits=splits)
    api.device_status()
    ref, ref_lse = oracle.sdpa(q, k, v, mask_kind=kind, qk_scale=s, with_lse=True)
    return out, lse, ref, ref_lse


DENSE = [
    # B, Hq, Hk, Lq, Lk, D, Dv, mask, splits
    (2, 8, 2, 300, 300, 128, 128, "causal", 1),
    (2, 8, 2, 300, 300, 128, 128, "causal", 2),
    (2, 8, 2, 300, 300, 128, 128, "none", 3),
    (1, 4, 4, 200, 700, 128, 128, "causal", 3),     # Lq < Lk, bottom-right diagonal
    (1, 4, 1, 333, 200, 128, 128, "causal", 2),     # Lq > Lk: rows with no key in any split
    (1, 4, 2, 129, 257, 64, 64, "none", 5),         # more splits than some units have tiles
    (1, 2, 2, 130, 140, 96, 96, "causal", 64),      # most splits empty
    (1, 2, 1, 100, 650, 128, 64, "none", 4),
    (1, 2, 2, 1, 700, 128, 128, "causal", 6),
]


@pytest.mark.parametrize("cfg", DENSE, ids=lambda c: "x".join(map(str, c)))
def test_dense_bf16_lse_and_splits(cfg):
    *shape, splits = cfg
    out, lse, ref, ref_lse = _dense(*shape, torch.bfloat16, splits)
    compare(out, ref, torch.bfloat16, str(cfg))
    compare_lse(lse, ref_lse, torch.bfloat16, str(cfg))


@pytest.mark.parametrize("splits", [1, 2, 3])
def test_dense_fp32_lse_and_splits(splits):
    out, lse, ref, ref_lse = _dense(1, 4, 2, 300, 270, 128, 128, "causal", torch.float32, splits)
    compare(out, ref, torch.float32, f"fp32 s{splits}")
    compare_lse(lse, ref_lse, torch.float32, f"fp32 s{splits}")


@pytest.mark.parametrize("kind", ["keep", "add"])
@pytest.mark.parametrize("splits", [1, 2])
def test_page_example_masks_lse(kind, splits):
    """'Core 注意力' example with masks (fp32): one 48-key tile, so with two
    splits the second one sees no key for any row."""
    q, k, v, keep, add = W.page_example_masks()
    m = keep if kind == "keep" else add
    out, lse = api.attn_fwd(q.to(DEV), k.to(DEV), v.to(DEV), mask=m.to(DEV), qk_scale=1 / 8,
                            return_lse=True, num_splits=splits)
    api.device_status()
    ref, ref_lse = oracle.sdpa(q, k, v, mask=m, mask_kind=kind, qk_scale=1 / 8, with_lse=True)
    compare(out, ref, torch.float32, kind)
    compare_lse(lse, ref_lse, torch.float32, kind)


def test_bool_mask_empty_row_lse_is_neg_inf():
    """An all-false keep row: out 0 and lse -inf, with and without splits."""
    q, k, v = W.dense_inputs(1, 2, 2, 150, 300, 128, 128, torch.bfloat16, 11, 1.0)
    g = torch.Generator().manual_seed(12)
    keep = torch.rand(1, 2, 150, 300, generator=g) < 0.5
    keep[:, :, 7] = False
    for splits in (1, 3):
        out, lse = api.attn_fwd(q.to(DEV), k.to(DEV), v.to(DEV), mask=keep.to(DEV),
                                qk_scale=1 / math.sqrt(128), return_lse=True, num_splits=splits)
        api.device_status()
        assert torch.all(out[:, :, 7] == 0) and torch.all(torch.isneginf(lse[:, :, 7]))
        ref, ref_lse = oracle.sdpa(q, k, v, mask=keep, mask_kind="keep", qk_scale=1 / math.sqrt(128),
                                   with_lse=True)
        compare(out, ref, torch.bfloat16, f"keep s{splits}")
        compare_lse(lse, ref_lse, torch.bfloat16, f"keep s{splits}")


PACKED = [
    # qlens, klens, Hq, Hk, D, Dv, drope, causal, splits
    ([1, 127, 128, 129, 300, 5], [1, 127, 128, 129, 300, 5], 4, 2, 128, 128, 0, True, 1),
    ([1, 127, 128, 129, 300, 5], [1, 127, 128, 129, 300, 5], 4, 2, 128, 128, 0, True, 3),
    ([200, 7, 385], [260, 90, 385], 4, 4, 128, 128, 64, True, 2),     # MLA, Lq <= Lk
    ([0, 50, 0, 130], [10, 60, 0, 130], 2, 1, 128, 128, 0, True, 4),  # empty sequences
    ([70, 257], [300, 31], 2, 2, 64, 64, 0, False, 7),
]


@pytest.mark.parametrize("cfg", PACKED, ids=lambda c: f"{len(c[0])}seq-r{c[6]}-s{c[8]}")
def test_packed_lse_and_splits(cfg):
    qlens, klens, Hq, Hk, D, Dv, drope, causal, splits = cfg
    ql = torch.tensor(qlens, dtype=torch.int32)
    kl = torch.tensor(klens, dtype=torch.int32)
    d = W.packed_inputs(ql, kl, Hq, Hk, D, Dv, drope, torch.bfloat16, 7)
    s = 1.0 / math.sqrt(D + drope)
    mt = api.MaskType.CAUSAL if causal else api.MaskType.NONE
    g = {k: v.to(DEV) for k, v in d.items()}
    T = int(ql.sum())
    # head-major LSE buffer [Hq, T], passed transposed as [T, Hq]
    lse_hm = torch.full((Hq, T), 123.0, dtype=torch.float32, device=DEV)
    out, lse = api.attn_fwd(g["q"], g["k"], g["v"], qrope=g.get("qrope"), krope=g.get("krope"),
                            q_seqlen=ql.to(DEV), kv_seqlen=kl.to(DEV), mask_type=mt, qk_scale=s,
                            lse=lse_hm.t(), num_splits=splits)
    api.device_status()
    ref, ref_lse = oracle.sdpa(d["q"], d["k"], d["v"], qrope=d.get("qrope"), krope=d.get("krope"),
                               q_seqlen=ql, kv_seqlen=kl, mask_kind="causal" if causal else "none",
                               qk_scale=s, with_lse=True)
    compare(out, ref, torch.bfloat16, str(cfg))
    compare_lse(lse_hm, ref_lse, torch.bfloat16, str(cfg))      # oracle packed LSE is [H, T]


def test_packed_split_leaves_other_tokens_alone():
    """Tokens past the sequences' total are neither attended nor merged."""
    ql = torch.tensor([100, 29], dtype=torch.int32)
    T = int(ql.sum())
    d = W.packed_inputs(torch.tensor([T + 60]), torch.tensor([T + 60]), 2, 2, 128, 128, 0,
                        torch.bfloat16, 5)
    out = torch.full((T + 60, 2, 128), -3.0, dtype=torch.bfloat16, device=DEV)
    lse = torch.full((T + 60, 2), 9.0, dtype=torch.float32, device=DEV)
    api.attn_fwd(d["q"].to(DEV), d["k"].to(DEV), d["v"].to(DEV), q_seqlen=ql.to(DEV),
                 kv_seqlen=ql.to(DEV), mask_type=api.MaskType.CAUSAL, out=out, lse=lse, num_splits=3)
    api.device_status()
    assert torch.all(out[T:] == -3.0) and torch.all(lse[T:] == 9.0)
    ref, ref_lse = oracle.sdpa(d["q"][:T], d["k"][:T], d["v"][:T], q_seqlen=ql, kv_seqlen=ql,
                               mask_kind="causal", qk_scale=1 / math.sqrt(128), with_lse=True)
    compare(out[:T], ref, torch.bfloat16, "packed split")
    compare_lse(lse[:T].t(), ref_lse, torch.bfloat16, "packed split")


def test_split_bad_lengths_merge_nothing():
    """A rejected length set: the merge pass writes nothing either."""
    ql = torch.tensor([100, 100], dtype=torch.int32)
    d = W.packed_inputs(torch.tensor([100, 50]), torch.tensor([100, 50]), 2, 2, 128, 128)
    out = torch.full((150, 2, 128), 5.0, dtype=torch.bfloat16, device=DEV)
    api.attn_fwd(d["q"].to(DEV), d["k"].to(DEV), d["v"].to(DEV), q_seqlen=ql.to(DEV),
                 kv_seqlen=ql.to(DEV), out=out, num_splits=2)
    with pytest.raises(api.WfError) as e:
        api.device_status()
    assert e.value.status == 1
    assert torch.all(out == 5.0)


def test_automatic_split_on_an_underfilled_grid():
    """One rolling-cache chunk against a full cache (q [1,12,1024,128], 8192
    keys): 48 work units on 148 SMs, so the automatic choice splits.  Same
    result as the forced split of the same count, and within tolerance of the
    unsplit run and of the oracle on sampled rows."""
    q, k, v = W.dense_inputs(1, 12, 12, 1024, 8192, 128, 128, torch.bfloat16, 21, 1.0)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    s = 1 / math.sqrt(128)
    auto, auto_lse = api.attn_fwd(qd, kd, vd, qk_scale=s, return_lse=True)
    n_sm = torch.cuda.get_device_properties(0).multi_processor_count
    n = max(1, min(n_sm // 48, 64 // 4))
    forced, forced_lse = api.attn_fwd(qd, kd, vd, qk_scale=s, return_lse=True, num_splits=n)
    one, one_lse = api.attn_fwd(qd, kd, vd, qk_scale=s, return_lse=True, num_splits=1)
    api.device_status()
    assert n > 1
    assert torch.equal(auto, forced) and torch.equal(auto_lse, forced_lse)
    assert (auto.float() - one.float()).abs().max().item() <= 2e-2
    assert (auto_lse - one_lse).abs().max().item() <= 1e-3
    rng = np.random.default_rng(3)
    rows = np.array([(0, h, r) for h in range(12) for r in
                     sorted({0, 1, 127, 128, 1022, 1023} | set(rng.integers(0, 1024, 20).tolist()))])
    ref, ref_lse = oracle.sdpa_rows(q, k, v, rows, qk_scale=s, with_lse=True)
    got = auto[0, rows[:, 1], rows[:, 2]]
    compare(got, ref, torch.bfloat16, "auto split rows")
    compare_lse(auto_lse[0, rows[:, 1], rows[:, 2]], ref_lse, torch.bfloat16, "auto split rows")


# ------------------------------------------------------------------- merge
def test_merge_of_gpu_halves_equals_full_attention():
    """Attention over two halves of the keys on the GPU (with LSE), merged by
    wf_attn_merge, against the oracle over all keys."""
    q, k, v = W.dense_inputs(2, 4, 2, 200, 600, 128, 128, torch.bfloat16, 31, 1.0)
    s = 1 / math.sqrt(128)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    parts, lses = [], []
    for sl in (slice(0, 256), slice(256, 600)):
        o, l = api.attn_fwd(qd, kd[:, :, sl].contiguous(), vd[:, :, sl].contiguous(), qk_scale=s,
                            return_lse=True, num_splits=1)
        parts.append(o)
        lses.append(l)
    out, lse = api.merge(torch.stack(parts), torch.stack(lses))
    api.device_status()
    ref, ref_lse = oracle.sdpa(q, k, v, qk_scale=s, with_lse=True)
    compare(out, ref, torch.bfloat16, "merged halves")
    compare_lse(lse, ref_lse, torch.bfloat16, "merged halves")


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("n_sets", [3, 6])
def test_merge_against_oracle_merge(out_dtype, n_sets):
    """Parts from the oracle over random disjoint key sets (fp32; three sets
    take the single-batch merge for few parts, six the general one), some
    rows with an empty set, one row empty everywhere; NaN planted in rows whose
    LSE is -inf must not leak."""
    g = torch.Generator().manual_seed(44)
    q = torch.randn(1, 3, 40, 64, generator=g)
    k = torch.randn(1, 3, 90, 64, generator=g)
    v = torch.randn(1, 3, 90, 96, generator=g)
    owner = torch.randint(0, n_sets, (90,), generator=g)
    outs, lses = [], []
    for s_ in range(n_sets):
        keep = (owner == s_).view(1, 1, 1, 90).expand(1, 3, 40, 90).clone()
        keep[:, :, 5] = False                    # row 5 empty everywhere
        if s_ == 1:
            keep[:, :, 9] = False                # row 9 empty in set 1
        o, l = oracle.sdpa(q, k, v, mask=keep.to(torch.uint8), mask_kind="keep", qk_scale=0.2,
                           with_lse=True)
        outs.append(o)
        lses.append(l)
    ref, ref_lse = oracle.merge(np.stack(outs), np.stack(lses))
    parts = torch.tensor(np.stack(outs), dtype=torch.float32)
    parts[1, :, :, 9] = float("nan")
    out, lse = api.merge(parts.to(DEV), torch.tensor(np.stack(lses), dtype=torch.float32).to(DEV),
                         out=torch.empty(1, 3, 40, 96, dtype=out_dtype, device=DEV))
    api.device_status()
    tol = 1e-5 if out_dtype == torch.float32 else 1e-2
    got = out.float().cpu().numpy()
    assert np.all(np.isfinite(got))
    assert np.abs(got - ref).max() <= tol
    assert np.all(got[:, :, 5] == 0) and np.all(np.isneginf(lse.cpu().numpy()[:, :, 5]))
    fin = ~np.isneginf(ref_lse)
    assert np.abs(lse.cpu().numpy()[fin] - ref_lse[fin]).max() <= 1e-5


def test_timeout_during_split_launch_then_clean_split_call():
    """An automatic-split launch (2 units, 16 KV tiles -> 4 splits) that times
    out; after the status call the next split launches are correct."""
    q, k, v = W.dense_inputs(1, 2, 2, 256, 2048, 128, 128, torch.bfloat16, 13, 1.0)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    s = 1 / math.sqrt(128)
    api.attn_fwd(qd, kd, vd, qk_scale=s, debug_flags=1, timeout_cycles=20_000_000)
    with pytest.raises(api.WfError) as e:
        api.device_status()
    assert e.value.status == 6
    for _ in range(2):
        out, lse = api.attn_fwd(qd, kd, vd, qk_scale=s, return_lse=True, num_splits=4)
        api.device_status()
        ref, ref_lse = oracle.sdpa(q, k, v, qk_scale=s, with_lse=True)
        compare(out, ref, torch.bfloat16, "split after timeout")
        compare_lse(lse, ref_lse, torch.bfloat16, "split after timeout")
