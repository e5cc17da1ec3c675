"""Host checks of the synthetic input recipes that GPU tests rely on."""
import numpy as np
import torch

from attention_forward_tmem_b200 import workloads as W

LOG2E = 1.4426950408889634


def _tile_max_steps(q, k, causal):
    """Per (head, row): increases of the running maximum (log2 units, qk_scale
    1) from each 128-key tile of the row's visible keys to the next (tiles of
    which fewer than 64 keys are visible left out)."""
    lq, lk = q.shape[2], k.shape[2]
    grp = q.shape[1] // k.shape[1]
    steps = []
    for h in range(q.shape[1]):
        s = (q[0, h].double() @ k[0, h // grp].double().T).numpy() * LOG2E
        for i in range(lq):
            last = min(lk - 1, i + lk - lq) if causal else lk - 1
            if last < 128:
                continue
            run = -np.inf
            for t0 in range(0, last + 1, 128):
                m = s[i, t0:min(t0 + 128, last + 1)].max()
                if t0 > 0 and last + 1 - t0 >= 64:     # tiles with at least half their keys visible
                    steps.append(max(m, run) - run)
                run = max(run, m)
    return np.array(steps)


def test_growing_scores_raise_the_running_max_on_every_tile():
    """The premise of the GPU rescale tests: with qk_scale 1 the running row
    maximum rises by more than 8 log2 units (the lazy-rescale threshold) from
    one 128-key tile to the next for most rows and tiles (by ~13-15 units at
    the median)."""
    for cfg in [(4, 2, 640, 640, 128, True), (2, 2, 256, 1024, 128, False), (2, 1, 200, 333, 64, True)]:
        hq, hk, lq, lk, d, causal = cfg
        q, k, _ = W.growing_score_inputs(1, hq, hk, lq, lk, d, d)
        st = _tile_max_steps(q, k, causal)
        assert st.size > 0
        assert (st > 8).mean() > 0.8, (cfg, float((st > 8).mean()))
        assert np.median(st) > 12, (cfg, float(np.median(st)))


def test_growing_scores_with_rope_parts():
    q, k, v, qr, kr = W.growing_score_inputs(1, 2, 2, 130, 130, 128, 128, drope=64)
    assert qr.shape == (1, 2, 130, 64) and kr.shape == (1, 2, 130, 64)
    assert q.dtype == k.dtype == v.dtype == qr.dtype == torch.bfloat16
