"""The plain Python BlockKVCache model against the page's facts (CPU only)."""
import numpy as np
import pytest

import oracle
from oracle.kvcache_model import BlockKVCacheModel, OrderError
from tests.oracle_pins import golden


def _run_page_example():
    gd = golden("blockkv_page_example.json")
    L = gd["k_shape"][gd["seq_dim"]]
    m = BlockKVCacheModel(L, gd["chunk_size"], gd["window_size"], gd["sink_size"])
    seen = []
    for c in range(gd["n_chunks"]):
        m.before_update(c)
        m.update([float(c)] * gd["chunk_size"], gd["chunk_size"])
        vis, phys = m.cached()
        logical = [x for chunk in m.cached_logical() for x in chunk]
        physical = [None] * L
        for s, slot in enumerate(m.slots):
            if slot is not None:
                for t in range(gd["chunk_size"]):
                    physical[s * gd["chunk_size"] + t] = slot[1][t]
        seen.append((vis, logical, physical))
        m.after_update(c)
    return gd, seen


def test_page_example_visibility():
    gd, seen = _run_page_example()
    assert [s[0] for s in seen] == gd["visible_tokens"]


def test_page_example_contents():
    gd, seen = _run_page_example()
    assert [s[1] for s in seen] == [[float(x) for x in r] for r in gd["logical_token_values"]]
    assert [s[2] for s in seen] == [[None if x is None else float(x) for x in r]
                                   for r in gd["physical_token_values"]]


def test_page_example_uniform_attention():
    """q = 0 over the visible cache (physical order) = mean of the visible V values."""
    gd, seen = _run_page_example()
    for (vis, logical, physical), expect in zip(seen, gd["uniform_attention_out"]):
        vals = np.array(physical[:vis], dtype=np.float64)
        v = np.repeat(vals[None, None, :, None], 3, axis=-1)
        k = np.zeros((1, 1, vis, 2))
        q = np.zeros((1, 1, 1, 2))
        out = oracle.sdpa(q, k, v, qk_scale=1.0)
        assert np.allclose(out, expect, rtol=0, atol=1e-15)


def test_rolling_workload_sequence():
    gd = golden("blockkv_rolling_sequence.json")
    L = gd["sink_size"] + gd["window_size"]
    m = BlockKVCacheModel(L, gd["chunk_size"], gd["window_size"], gd["sink_size"])
    slots, vis = [], []
    for c in range(gd["n_chunks"]):
        m.before_update(c)
        slots.append(m.update(c, gd["chunk_size"]))
        vis.append(m.cached()[0])
        m.after_update(c)
    assert slots == gd["slots"]
    assert vis == gd["visible"]
    assert sum(vis) == gd["visible_total"]
    assert m.logical_chunks(gd["n_chunks"] - 1) == gd["logical_chunks_after_15"]
    # the sink chunk is never evicted
    assert m.slots[0][0] == 0


def test_repeat_overwrites_same_slot():
    m = BlockKVCacheModel(8, 2, 6, 2)
    for c, payload in ((0, "a"), (1, "b"), (1, "b2"), (2, "c")):
        m.before_update(c)
        m.update(payload, 2)
        m.cached()
        m.after_update(c)
    assert [None if s is None else s[1] for s in m.slots] == ["a", "b2", "c", None]


@pytest.mark.parametrize("seq", [
    [("before", 1)],                                   # first index must be 0
    [("cycle", 0), ("before", 2)],                     # skip
    [("cycle", 0), ("cycle", 1), ("before", 0)],       # going back
    [("update",)],                                     # update without before_update
    [("before", 0), ("cached",)],                      # cached before update
    [("before", 0), ("update",), ("after", 0)],        # after_update before cached
    [("before", 0), ("update",), ("cached",), ("after", 1)],  # mismatched index
    [("before", 0), ("before", 0)],                    # before_update twice
])
def test_order_errors_leave_state(seq):
    m = BlockKVCacheModel(8, 2, 6, 2)
    *prefix, last = seq

    def do(step):
        op = step[0]
        if op == "cycle":
            m.before_update(step[1]); m.update(0, 2); m.cached(); m.after_update(step[1])
        elif op == "before":
            m.before_update(step[1])
        elif op == "update":
            m.update(0, 2)
        elif op == "cached":
            m.cached()
        elif op == "after":
            m.after_update(step[1])

    for s in prefix:
        do(s)
    before = m.state()
    with pytest.raises(OrderError):
        do(last)
    assert m.state() == before


@pytest.mark.parametrize("L,chunk,window,sink", [
    (8, 3, 8, 0),     # not divisible
    (8, 2, 4, 2),     # sum != L
    (8, 4, 6, 2),     # sink not a multiple of chunk
    (8, 2, 0, 8),     # no window
])
def test_bad_sizes(L, chunk, window, sink):
    with pytest.raises(ValueError):
        BlockKVCacheModel(L, chunk, window, sink)


def test_update_size_checked():
    m = BlockKVCacheModel(4, 2, 4)
    m.before_update(0)
    with pytest.raises(ValueError):
        m.update(0, 3)
