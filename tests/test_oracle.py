"""The oracle against its pins (CPU only), and the pins against planted mistakes."""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import brute
from tests import oracle_pins as P


@pytest.mark.parametrize("pin", P.PINS, ids=lambda f: f.__name__)
def test_pin_holds(pin):
    assert pin(0)


@pytest.mark.parametrize("plant", sorted(P.PLANTS), ids=lambda n: P.PLANTS[n])
def test_planted_mistake_is_caught(plant):
    oracle.build_oracle(plant)
    failed = [p.__name__ for p in P.PINS if not p(plant)]
    assert failed, f"no pin catches planted mistake {plant}: {P.PLANTS[plant]}"


@pytest.mark.parametrize("pin", P.MERGE_PINS, ids=lambda f: f.__name__)
def test_merge_pin_holds(pin):
    assert pin(0)


@pytest.mark.parametrize("plant", sorted(oracle.MERGE_PLANTS), ids=lambda n: oracle.MERGE_PLANTS[n])
def test_merge_planted_mistake_is_caught(plant):
    failed = [p.__name__ for p in P.MERGE_PINS if not p(plant)]
    assert failed, f"no pin catches planted merge mistake {plant}: {oracle.MERGE_PLANTS[plant]}"


@pytest.mark.parametrize("pin", P.DCA_PINS, ids=lambda f: f.__name__)
def test_dca_pin_holds(pin):
    assert pin()


@pytest.mark.parametrize("plant", sorted(oracle.DCA_PLANTS), ids=lambda n: oracle.DCA_PLANTS[n])
def test_dca_planted_mistake_is_caught(plant):
    failed = [p.__name__ for p in P.DCA_PINS if not p(plant)]
    assert failed, f"no pin catches planted DCA mistake {plant}: {oracle.DCA_PLANTS[plant]}"


def test_rows_mode_matches_full():
    g = torch.Generator().manual_seed(30)
    lens = torch.tensor([7, 3, 9], dtype=torch.int32)
    q = torch.randn(19, 4, 8, generator=g, dtype=torch.float64)
    k = torch.randn(19, 2, 8, generator=g, dtype=torch.float64)
    v = torch.randn(19, 2, 5, generator=g, dtype=torch.float64)
    full, lse = oracle.sdpa(q, k, v, q_seqlen=lens, kv_seqlen=lens, mask_kind="causal",
                            qk_scale=0.5, with_lse=True)
    rows = np.array([[0, 0, 0], [0, 3, 6], [1, 2, 2], [2, 1, 8], [2, 0, 4]])
    got, got_lse = oracle.sdpa_rows(q, k, v, rows, q_seqlen=lens, kv_seqlen=lens,
                                    mask_kind="causal", qk_scale=0.5, with_lse=True)
    starts = np.array([0, 7, 10])
    for t, (b, h, i) in enumerate(rows):
        assert np.array_equal(got[t], full[starts[b] + i, h])
        assert got_lse[t] == lse[h, starts[b] + i]
    # dense rows
    qd, kd, vd = q[None, :, :2].transpose(1, 2), k[None, :, :1].transpose(1, 2), v[None, :, :1].transpose(1, 2)
    full = oracle.sdpa(qd, kd, vd, qk_scale=0.3, head_num=2, kv_head_num=1)
    rows = np.array([[0, 1, 18], [0, 0, 0]])
    got = oracle.sdpa_rows(qd, kd, vd, rows, qk_scale=0.3, head_num=2, kv_head_num=1)
    assert np.array_equal(got[0], full[0, 1, 18]) and np.array_equal(got[1], full[0, 0, 0])


def test_oracle_rejects_bad_args():
    q = torch.zeros(1, 3, 4, 8, dtype=torch.float64)
    k = torch.zeros(1, 2, 4, 8, dtype=torch.float64)
    with pytest.raises(ValueError):
        oracle.sdpa(q, k, k, qk_scale=1.0)      # 3 % 2 != 0
    lens = torch.tensor([4], dtype=torch.int32)
    with pytest.raises(ValueError):
        oracle.sdpa(q[0].transpose(0, 1), k[0].transpose(0, 1), k[0].transpose(0, 1),
                    q_seqlen=lens, kv_seqlen=lens, mask=torch.ones(4, 4), mask_kind="keep",
                    qk_scale=1.0, head_num=3, kv_head_num=3)


def test_empty_and_zero_length_sequences():
    """Empty batch entries and Lk = 0 give zeros, nothing else."""
    lens_q = torch.tensor([2, 0, 3], dtype=torch.int32)
    lens_k = torch.tensor([0, 4, 3], dtype=torch.int32)
    g = torch.Generator().manual_seed(31)
    q = torch.randn(5, 2, 4, generator=g, dtype=torch.float64)
    k = torch.randn(7, 2, 4, generator=g, dtype=torch.float64)
    v = torch.randn(7, 2, 4, generator=g, dtype=torch.float64)
    out = oracle.sdpa(q, k, v, q_seqlen=lens_q, kv_seqlen=lens_k, qk_scale=1.0)
    assert np.all(out[:2] == 0.0)
    ref = brute.sdpa_packed(q[2:], k[4:], v[4:], [3], [3], scale=1.0)
    assert np.allclose(out[2:], ref, rtol=1e-12, atol=1e-12)


def test_extreme_scores_stay_finite():
    """Scores in the thousands: the max subtraction keeps exp finite."""
    q = torch.full((1, 1, 3, 4), 30.0, dtype=torch.float64)
    k = torch.full((1, 1, 5, 4), 30.0, dtype=torch.float64)
    k[0, 0, 2] = 31.0
    v = torch.arange(5, dtype=torch.float64).reshape(1, 1, 5, 1)
    out = oracle.sdpa(q, k, v, qk_scale=1.0)
    assert np.all(np.isfinite(out))
    # 30*31*4 - 30*30*4 = 120 nats apart: key 2 takes all the weight
    assert np.allclose(out, 2.0, atol=1e-30)


def test_threads_reported():
    assert oracle.oracle_threads() >= 1
    assert math.isfinite(float(oracle.oracle_threads()))
